"""Device buffers of one synthetic decode step (inputs only; see torch_gen for the recipe).

``shared_inputs`` builds what does not depend on the draft depth (the verify layers' paged KV,
the draft ring and the native draft cache, sized for the deepest step asked for);
``step_inputs`` adds the per-depth tensors (queries, new draft rows, logits, tokens, lengths).
"""
from typing import Dict, Optional, Sequence

import numpy as np
import torch

from . import torch_gen as tg


def shared_inputs(w, device, seed: Optional[int] = None, max_nq_verify: int = 8,
                  max_gamma: int = 7, window: Optional[int] = None, n_layers: Optional[int] = None,
                  arms: Sequence[str] = ("windowed", "native"), slack: int = 0,
                  kv8: bool = False) -> Dict:
    """``slack`` extra positions in the verify layers' caches and the native draft cache, for a
    decode loop that advances the committed context.  ``kv8``: every K/V cache holds E4M3 codes
    (uint8) of N(0, 2^2) values instead of bf16."""
    seed = w.seed if seed is None else seed
    g = tg.generator(seed, device)
    lens = tg.contexts(w, seed)
    P, D = w.page_size, w.D
    n_layers = w.verify_layers if n_layers is None else n_layers
    window = w.windows[0] if window is None else window
    lens_v = [L + max_nq_verify + slack for L in lens]
    table_v, npg_v = tg.page_table(lens_v, P, seed + 1)
    k_pools, v_pools = [], []
    for _ in range(n_layers):
        if kv8:
            k, v = tg.kv_rows_fp8((npg_v, w.Hkv, P, D), g, device)
        else:
            k, v = tg.paged_kv(lens_v, w.Hkv, D, P, g, device, table_v, npg_v, w.k_scale, w.outlier_p)
        k_pools.append(k)
        v_pools.append(v)
    out = dict(lens=lens, lens_v_alloc=lens_v, table_v=torch.from_numpy(table_v).to(device),
               k_pools=k_pools, v_pools=v_pools, g=g, window=window, n_sink=w.n_sink, kv8=kv8)
    if "windowed" in arms:
        C = w.n_sink + window
        if kv8:
            ring_k, ring_v = tg.kv_rows_fp8((w.B, w.Hkv, C, D), g, device)
        else:
            ring_k, ring_v = tg.kv_rows_bf16((w.B, w.Hkv, C, D), g, device, w.k_scale, w.outlier_p)
        out.update(ring_k=ring_k, ring_v=ring_v,
                   ring_len0=torch.tensor(lens, dtype=torch.int64, device=device))
    if "native" in arms:
        lens_d = [L + 2 * max_gamma + 1 + slack for L in lens]
        table_d, npg_d = tg.page_table(lens_d, P, seed + 2)
        if kv8:
            kd, vd = tg.kv_rows_fp8((npg_d, w.Hkv, P, D), g, device)
        else:
            kd, vd = tg.paged_kv(lens_d, w.Hkv, D, P, g, device, table_d, npg_d, w.k_scale, w.outlier_p)
        out.update(k_draft=kd, v_draft=vd, table_d=torch.from_numpy(table_d).to(device))
    return out


def step_inputs(w, shared: Dict, gamma: int, device, seed: Optional[int] = None,
                lens: Optional[Sequence[int]] = None) -> Dict:
    """Keyword arguments for StepBuffers at draft depth gamma.  ``lens`` runs the step at shorter
    committed contexts than the buffers were built for (the context sweep): the caches and page
    tables are reused, only the lengths change."""
    seed = (w.seed if seed is None else seed) * 1000 + gamma
    g = tg.generator(seed, device)
    if lens is None:
        lens = shared["lens"]
    else:
        lens = [int(x) for x in lens]
        if any(a > b for a, b in zip(lens, shared["lens"])) or len(lens) != len(shared["lens"]):
            raise ValueError("step_inputs: lens must not exceed the built contexts")
    B, Hq, Hkv, D = w.B, w.Hq, w.Hkv, w.D
    n_q = w.tree_nodes if w.tree_nodes else gamma + 1
    n_layers = len(shared["k_pools"])
    tree = None
    if w.tree_nodes:
        tree = torch.from_numpy(tg.tree_parents(w.seed, B, w.tree_nodes)).to(device)

    def rn(*shape):
        return tg.fill_normal_bf16(torch.empty(shape, dtype=torch.bfloat16, device=device), g)

    kv8 = shared.get("kv8", False)

    def rkv(*shape):
        if kv8:
            return tg.kv_rows_fp8(shape, g, device)[0]
        return rn(*shape)

    logits = torch.rand((B, n_q, w.vocab), generator=g, device=device) * 2 - 1
    tokens = torch.randint(0, w.vocab, (B, n_q), generator=g, device=device, dtype=torch.int32)
    kw = dict(
        k_pools=shared["k_pools"], v_pools=shared["v_pools"], table_v=shared["table_v"],
        kv_len_v=torch.tensor([L + n_q for L in lens], dtype=torch.int32, device=device),
        q_verify=rn(n_layers, B, n_q, Hq, D), tree_parent=tree, logits=logits, tokens=tokens,
        q_ctx=rn(B, gamma + 1, Hq, D), q_fwd=rn(gamma, B, 1, Hq, D),
        k_ctx=rkv(B, gamma + 1, Hkv, D), v_ctx=rkv(B, gamma + 1, Hkv, D),
        k_fwd=rkv(gamma, B, 1, Hkv, D), v_fwd=rkv(gamma, B, 1, Hkv, D),
        n_sink=shared["n_sink"], window=shared["window"], sm_scale=w.sm_scale,
    )
    if kv8:
        kw.update(kv8=True, k_scale=0.5, v_scale=0.5)
    if "ring_k" in shared:
        kw.update(ring_k=shared["ring_k"], ring_v=shared["ring_v"],
                  ring_len=torch.tensor(lens, dtype=torch.int64, device=device))
    if "k_draft" in shared:
        kw.update(k_draft=shared["k_draft"], v_draft=shared["v_draft"], table_d=shared["table_d"],
                  kv_len_ctx=torch.tensor([L + gamma + 1 for L in lens], dtype=torch.int32, device=device),
                  kv_len_fwd=[torch.tensor([L + gamma + 2 + j for L in lens], dtype=torch.int32,
                                           device=device) for j in range(gamma)])
    return kw
