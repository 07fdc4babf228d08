"""GPU parity at the workloads' full sizes, in the launch configuration the benchmark times,
on sampled outputs the fp64 oracle computes row by row (1M-key rows take the oracle ~0.5 s).

Workloads: 128K context (GQA 16/2), 1M context (GQA 32/4), a ragged batch of 8 with per-request
rings and an 8-node draft tree, and 1M NoPE context (GQA 64/8) with 1% outlier rows across the
window sweep 4 + {1020, 2044, 4092, 8188, 16380}.  The draft KV is appended to the rings by the
library's own bulk append (only survivors are written) and paged into the pool for the full
draft; the verify layer has its own paged KV holding the step's nodes.  The 1M workload also
runs with every cache in fp8 (E4M3) codes.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_speculative_kv_b200 import api
from synthetic import configs
from synthetic import torch_gen as tg
from tests.gpu_util import assert_attn_close, assert_lse_close, to_f64

pytestmark = pytest.mark.gpu


def _draft_and_target(w, lens, n_q, seed, device="cuda"):
    g = tg.generator(seed, device)
    Lmax = max(lens)
    k_d, v_d = tg.kv_rows_bf16((w.B, Lmax, w.Hkv, w.D), g, device, w.k_scale, w.outlier_p)
    lens_v = [L + n_q for L in lens]
    k_t, v_t = tg.kv_rows_bf16((w.B, max(lens_v), w.Hkv, w.D), g, device, w.k_scale, w.outlier_p)
    return g, k_d, v_d, k_t, v_t, lens_v


def _sample_check(out, lse, q_bits, k_tok, v_tok, L_tot, b, h, G, rows, mode, sm_scale, **kw):
    kb = tg.host_head_sequence(k_tok, b, h, L_tot)
    vb = tg.host_head_sequence(v_tok, b, h, L_tot)
    qb = np.ascontiguousarray(q_bits[b:b + 1, :, h * G:(h + 1) * G])
    ref, ref_lse = oracle.attention(qb, kb, vb, [L_tot], mode, sm_scale,
                                    rows=[(0, i, g) for i, g in rows], **kw)
    got = to_f64(out)
    gl = lse.cpu().numpy()
    r_idx = [(i, g) for i, g in rows]
    a = np.stack([got[b, i, h * G + g] for i, g in r_idx])
    r = np.stack([ref[0, i, g] for i, g in r_idx])
    assert_attn_close(a, r, f"b{b} h{h}")
    assert_lse_close(np.array([gl[b, i, h * G + g] for i, g in r_idx]),
                     np.array([ref_lse[0, i, g] for i, g in r_idx]))


def _nan_outputs(q):
    B, n_q, Hq, _ = q.shape
    return (torch.full_like(q, float("nan")),
            torch.full((B, n_q, Hq), float("nan"), dtype=torch.float32, device=q.device))


def _q(g, B, n_q, Hq, D, device="cuda"):
    q = tg.fill_normal_bf16(torch.empty((B, n_q, Hq, D), dtype=torch.bfloat16, device=device), g)
    return q, q.cpu().view(torch.int16).numpy().view(np.uint16)


def _run_workload(w, gamma, window, samples, seed_offset=0, tree=False):
    device = "cuda"
    lens = tg.contexts(w, w.seed)
    n_q = w.tree_nodes if tree else gamma + 1
    g, k_d, v_d, k_t, v_t, lens_v = _draft_and_target(w, lens, n_q, w.seed + seed_offset)
    G, P = w.G, w.page_size
    # ---- verify (one target layer) ------------------------------------------------------
    table_v, npg_v = tg.page_table(lens_v, P, w.seed + 1)
    kp = tg.paginate_tokens(k_t, lens_v, table_v, npg_v, P)
    vp = tg.paginate_tokens(v_t, lens_v, table_v, npg_v, P)
    qv, qv_bits = _q(g, w.B, n_q, w.Hq, w.D)
    parent = tg.tree_parents(w.seed, w.B, n_q) if tree else None
    ws = api.alloc_workspace(w.B, max(n_q, gamma + 1), w.Hq, w.Hkv)
    tdev = torch.from_numpy(table_v).cuda()
    kvl = torch.tensor(lens_v, dtype=torch.int32, device=device)
    # NaN-filled outputs: a row the library never writes shows up in every run
    out, lse = _nan_outputs(qv)
    out, lse = api.verify_attn(qv, kp, vp, tdev, kvl, w.sm_scale, ws,
                               tree_parent=None if parent is None else torch.from_numpy(parent).cuda(),
                               out=out, lse=lse)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    for b, h, rows in samples(n_q):
        _sample_check(out, lse, qv_bits, k_t, v_t, lens_v[b], b, h, G, rows,
                      oracle.MODE_TREE if tree else oracle.MODE_CAUSAL, w.sm_scale,
                      tree_parent=None if parent is None else parent[b:b + 1])
    del kp, vp, k_t, v_t
    # ---- draft: full (paged) and windowed (ring filled by one bulk append) ---------------
    table_d, npg_d = tg.page_table(lens, P, w.seed + 2)
    kpd = tg.paginate_tokens(k_d, lens, table_d, npg_d, P)
    vpd = tg.paginate_tokens(v_d, lens, table_d, npg_d, P)
    tdd = torch.from_numpy(table_d).cuda()
    kvd = torch.tensor(lens, dtype=torch.int32, device=device)
    for nq_d in (1, gamma + 1):
        qd, qd_bits = _q(g, w.B, nq_d, w.Hq, w.D)
        out, lse = api.draft_attn_full(qd, kpd, vpd, tdd, kvd, w.sm_scale, ws, *_nan_outputs(qd))
        torch.cuda.synchronize()
        assert api.device_status() == 0
        for b, h, rows in samples(nq_d):
            _sample_check(out, lse, qd_bits, k_d, v_d, lens[b], b, h, G, rows, oracle.MODE_CAUSAL,
                          w.sm_scale)
    del kpd, vpd
    windows = window if isinstance(window, (list, tuple)) else [window]
    for W in windows:
        C = w.n_sink + W
        ring_k = torch.full((w.B, w.Hkv, C, w.D), float("nan"), dtype=torch.bfloat16, device=device)
        ring_v = ring_k.clone()
        rlen = torch.zeros(w.B, dtype=torch.int64, device=device)
        for b in range(w.B):
            api.ring_kv_append(ring_k[b:b + 1], ring_v[b:b + 1], rlen[b:b + 1],
                               k_d[b:b + 1, :lens[b]], v_d[b:b + 1, :lens[b]], w.n_sink)
        for nq_d in (1, gamma + 1):
            qd, qd_bits = _q(g, w.B, nq_d, w.Hq, w.D)
            out, lse = api.draft_attn_window(qd, ring_k, ring_v, rlen, w.n_sink, W, w.sm_scale, ws,
                                             *_nan_outputs(qd))
            torch.cuda.synchronize()
            assert api.device_status() == 0
            assert torch.equal(rlen.cpu(), torch.tensor(lens))
            for b, h, rows in samples(nq_d):
                _sample_check(out, lse, qd_bits, k_d, v_d, lens[b], b, h, G, rows,
                              oracle.MODE_WINDOW, w.sm_scale, n_sink=w.n_sink, window=W)


def _samples_factory(heads, G, n_rows=6, B=1, seed=0):
    rng = np.random.default_rng(seed)

    def samples(n_q):
        out = []
        for b in range(B):
            for h in heads:
                rows = sorted({(int(rng.integers(n_q)), int(rng.integers(G))) for _ in range(n_rows)}
                              | {(n_q - 1, G - 1), (0, 0)})
                out.append((b, h, rows))
        return out
    return samples


def test_ctx128k():
    w = configs.CTX128K
    _run_workload(w, 3, 4092, _samples_factory([0, 1], w.G))


@pytest.mark.parametrize("gamma", [3, 7])
def test_ctx1m(gamma):
    """gamma = 3 is the benchmark's headline step (32-row verify units, 4-query context pass);
    gamma = 7 runs the 64-row verify units on the tcgen05 kernel."""
    w = configs.CTX1M
    _run_workload(w, gamma, 4092, _samples_factory([0, 3], w.G, n_rows=4, seed=gamma))


def test_batch8_ragged_tree():
    w = configs.BATCH8_TREE
    rng = np.random.default_rng(1)

    def samples(n_q):
        return [(b, int(rng.integers(w.Hkv)),
                 sorted({(int(rng.integers(n_q)), int(rng.integers(w.G))) for _ in range(3)} | {(n_q - 1, 0)}))
                for b in (0, 3, 7)]
    _run_workload(w, 3, 4092, samples, tree=True)


def test_nope1m_outliers_window_sweep():
    w = configs.NOPE1M
    _run_workload(w, 5, list(w.windows), _samples_factory([0, 7], w.G, n_rows=3))


# ----------------------------------------------------------------------------- fp8 (E4M3) KV
def _paginate8(tok, lens, table, num_pages, P):
    """Token-major [B, Lmax, Hkv, D] codes -> pool [num_pages, Hkv, P, D]; rows past each
    request's end hold the NaN code."""
    B, Lmax, Hkv, D = tok.shape
    pool = torch.full((num_pages, Hkv, P, D), 0x7F, dtype=torch.uint8, device=tok.device)
    for b in range(B):
        L = int(lens[b])
        n_full = L // P
        if n_full:
            pages = torch.from_numpy(table[b, :n_full].astype(np.int64)).to(tok.device)
            pool.index_copy_(0, pages, tok[b, :n_full * P].view(n_full, P, Hkv, D).permute(0, 2, 1, 3).contiguous())
        r = L - n_full * P
        if r:
            pool[int(table[b, n_full]), :, :r] = tok[b, n_full * P:L].permute(1, 0, 2)
    return pool


def _sample_check8(out, lse, q_bits, k_tok, v_tok, L_tot, b, h, G, rows, mode, sm_scale, ks, vs, **kw):
    kb = k_tok[b, :L_tot, h].contiguous().cpu().numpy().reshape(1, 1, L_tot, -1)
    vb = v_tok[b, :L_tot, h].contiguous().cpu().numpy().reshape(1, 1, L_tot, -1)
    qb = np.ascontiguousarray(q_bits[b:b + 1, :, h * G:(h + 1) * G])
    ref, ref_lse = oracle.attention_kv8(qb, kb, vb, [L_tot], mode, sm_scale, ks, vs,
                                        rows=[(0, i, g) for i, g in rows], **kw)
    got = to_f64(out)
    gl = lse.cpu().numpy()
    a = np.stack([got[b, i, h * G + g] for i, g in rows])
    r = np.stack([ref[0, i, g] for i, g in rows])
    assert_attn_close(a, r, f"fp8 b{b} h{h}")
    assert_lse_close(np.array([gl[b, i, h * G + g] for i, g in rows]),
                     np.array([ref_lse[0, i, g] for i, g in rows]))


def test_ctx1m_fp8_kv():
    """The 1M workload with every cache in E4M3 codes: verify at 32 rows (register widening)
    and 64 rows (tcgen05 with converter warps), the full draft, and the windowed draft over a
    ring filled by the fp8 bulk append."""
    w = configs.CTX1M
    dev = "cuda"
    KS, VS = 0.5, 0.5
    L = w.L
    G, P = w.G, w.page_size
    g = tg.generator(w.seed + 77, dev)
    samples = _samples_factory([0, 3], G, n_rows=3)
    ws = api.alloc_workspace(1, 8, w.Hq, w.Hkv)
    for gamma in (3, 7):
        n_q = gamma + 1
        Lv = L + n_q
        k_t, v_t = tg.kv_rows_fp8((1, Lv, w.Hkv, w.D), g, dev)
        table, npg = tg.page_table([Lv], P, w.seed + 1)
        kp, vp = _paginate8(k_t, [Lv], table, npg, P), _paginate8(v_t, [Lv], table, npg, P)
        q, q_bits = _q(g, 1, n_q, w.Hq, w.D)
        out, lse = api.verify_attn_fp8(q, kp, vp, torch.from_numpy(table).cuda(),
                                       torch.tensor([Lv], dtype=torch.int32, device=dev), w.sm_scale,
                                       KS, VS, ws)
        torch.cuda.synchronize()
        assert api.device_status() == 0
        for b, h, rows in samples(n_q):
            _sample_check8(out, lse, q_bits, k_t, v_t, Lv, b, h, G, rows, oracle.MODE_CAUSAL, w.sm_scale, KS, VS)
        del kp, vp
    # draft: full over the paged cache, windowed over the ring (bulk fp8 append)
    table, npg = tg.page_table([L], P, w.seed + 2)
    kp, vp = _paginate8(k_t[:, :L], [L], table, npg, P), _paginate8(v_t[:, :L], [L], table, npg, P)
    q, q_bits = _q(g, 1, 1, w.Hq, w.D)
    out, lse = api.draft_attn_full_fp8(q, kp, vp, torch.from_numpy(table).cuda(),
                                       torch.tensor([L], dtype=torch.int32, device=dev), w.sm_scale, KS, VS, ws)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    for b, h, rows in samples(1):
        _sample_check8(out, lse, q_bits, k_t, v_t, L, b, h, G, rows, oracle.MODE_CAUSAL, w.sm_scale, KS, VS)
    del kp, vp
    W = w.windows[0]
    C = w.n_sink + W
    ring_k = torch.full((1, w.Hkv, C, w.D), 0x7F, dtype=torch.uint8, device=dev)
    ring_v = ring_k.clone()
    rlen = torch.zeros(1, dtype=torch.int64, device=dev)
    api.ring_kv_append_fp8(ring_k, ring_v, rlen, k_t[:, :L].contiguous(), v_t[:, :L].contiguous(), w.n_sink)
    for nq in (1, 4):
        q, q_bits = _q(g, 1, nq, w.Hq, w.D)
        out, lse = api.draft_attn_window_fp8(q, ring_k, ring_v, rlen, w.n_sink, W, w.sm_scale, KS, VS, ws)
        torch.cuda.synchronize()
        assert api.device_status() == 0
        for b, h, rows in samples(nq):
            _sample_check8(out, lse, q_bits, k_t, v_t, L, b, h, G, rows, oracle.MODE_WINDOW, w.sm_scale,
                           KS, VS, n_sink=w.n_sink, window=W)
