"""Device-resident synthetic workloads for the large sizes (seeded torch generators on the GPU).

Same recipe as ``gen`` (N(0, 1) float32 -> K scaling and outlier rows -> round-to-nearest-even
bf16; random page-table permutation; NaN in the tail rows of each request's last page), drawn
with ``torch.Generator(device)`` because the million-token tensors are too large to draw on the
host.  Tests that check these sizes copy the tensors (or the parts they sample) to the host
for the oracle.  No arithmetic of the method lives here.
"""
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

from . import gen

CHUNK = 1 << 26    # elements per generation chunk (256 MiB of float32)


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def fill_normal_bf16(t: torch.Tensor, g: torch.Generator, scale: float = 1.0) -> torch.Tensor:
    """Fills a bf16 tensor with N(0, 1) * scale, drawn in float32 chunks, rounded once."""
    flat = t.view(-1)
    for s in range(0, flat.numel(), CHUNK):
        n = min(CHUNK, flat.numel() - s)
        x = torch.randn(n, generator=g, device=t.device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        flat[s:s + n].copy_(x)
    return t


def kv_rows_bf16(shape, g: torch.Generator, device, k_scale: float = 1.0, outlier_p: float = 0.0,
                 outlier_factor: float = 8.0):
    """K and V of ``shape`` (rows = last axis); outlier rows scale both K and V before rounding."""
    k = torch.empty(shape, dtype=torch.bfloat16, device=device)
    v = torch.empty(shape, dtype=torch.bfloat16, device=device)
    rows = int(np.prod(shape[:-1]))
    D = shape[-1]
    kf, vf = k.view(rows, D), v.view(rows, D)
    step = max(1, CHUNK // D)
    for s in range(0, rows, step):
        n = min(step, rows - s)
        xk = torch.randn((n, D), generator=g, device=device, dtype=torch.float32)
        if k_scale != 1.0:
            xk.mul_(k_scale)
        xv = torch.randn((n, D), generator=g, device=device, dtype=torch.float32)
        if outlier_p > 0.0:
            m = torch.rand((n, 1), generator=g, device=device) < outlier_p
            f = torch.where(m, torch.full_like(xk[:, :1], outlier_factor), torch.ones_like(xk[:, :1]))
            xk.mul_(f)
            xv.mul_(f)
        kf[s:s + n].copy_(xk)
        vf[s:s + n].copy_(xv)
    return k, v


def page_table(lens: Sequence[int], page_size: int, seed: int, max_pages: Optional[int] = None):
    """(table int32 [B, max_pages] on the host, number of pages): a seeded permutation."""
    rng = np.random.default_rng(seed)
    table = gen.page_table(rng, [int(x) for x in lens], page_size, max_pages)
    return table, gen.n_pages(lens, page_size)


def poison_tails(pool: torch.Tensor, table: np.ndarray, lens: Sequence[int], page_size: int):
    """NaN into the rows past each request's end in its last page."""
    for b, L in enumerate(lens):
        L = int(L)
        r = L % page_size
        if r:
            pool[int(table[b, (L - 1) // page_size]), :, r:, :] = float("nan")


def paged_kv(lens: Sequence[int], Hkv: int, D: int, page_size: int, g: torch.Generator, device,
             table: np.ndarray, num_pages: int, k_scale: float = 1.0, outlier_p: float = 0.0):
    """A K/V pool pair [num_pages, Hkv, P, D] filled with random rows, tails poisoned."""
    k, v = kv_rows_bf16((num_pages, Hkv, page_size, D), g, device, k_scale, outlier_p)
    poison_tails(k, table, lens, page_size)
    poison_tails(v, table, lens, page_size)
    return k, v


def logical_from_pool(pool: torch.Tensor, table_row: np.ndarray, L: int, head: int,
                      page_size: int) -> np.ndarray:
    """Host copy (bf16 bits) of one request's logical [L, D] sequence for one kv head."""
    n = (L + page_size - 1) // page_size
    idx = torch.from_numpy(np.ascontiguousarray(table_row[:n]).astype(np.int64)).to(pool.device)
    seq = pool.index_select(0, idx)[:, head].reshape(n * page_size, pool.shape[-1])[:L]
    return seq.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def tree_parents(seed: int, B: int, n: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.stack([gen.draft_tree(rng, n) for _ in range(B)]).astype(np.int32)


def contexts(w, seed: int) -> List[int]:
    """Committed context per request: fixed L, or U[lo, hi] per request when ragged."""
    if w.ragged[1] > 0:
        rng = np.random.default_rng(seed)
        return [int(x) for x in gen.ragged_contexts(rng, w.B, w.ragged[0], w.ragged[1])]
    return [w.L] * w.B


def paginate_tokens(tok: torch.Tensor, lens: Sequence[int], table: np.ndarray, num_pages: int,
                    page_size: int) -> torch.Tensor:
    """Token-major [B, Lmax, Hkv, D] -> pool [num_pages, Hkv, P, D]; rows past each request's end
    are NaN."""
    B, Lmax, Hkv, D = tok.shape
    pool = torch.full((num_pages, Hkv, page_size, D), float("nan"), dtype=tok.dtype, device=tok.device)
    for b in range(B):
        L = int(lens[b])
        n_full = L // page_size
        if n_full:
            pages = torch.from_numpy(table[b, :n_full].astype(np.int64)).to(tok.device)
            blk = tok[b, :n_full * page_size].view(n_full, page_size, Hkv, D).permute(0, 2, 1, 3)
            pool.index_copy_(0, pages, blk.contiguous())
        r = L - n_full * page_size
        if r:
            pool[int(table[b, n_full]), :, :r] = tok[b, n_full * page_size:L].permute(1, 0, 2)
    return pool


def host_head_sequence(tok: torch.Tensor, b: int, h: int, L: int) -> np.ndarray:
    """bf16 bits [1, 1, L, D] of request b, kv head h, from a token-major device tensor."""
    seq = tok[b, :L, h].contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    return seq.reshape(1, 1, L, -1)


def kv_rows_fp8(shape, g: torch.Generator, device, scale: float = 2.0):
    """K and V of ``shape`` as E4M3 codes (uint8): N(0, scale^2) rounded to the nearest code."""
    k = torch.empty(shape, dtype=torch.uint8, device=device)
    v = torch.empty(shape, dtype=torch.uint8, device=device)
    for t in (k, v):
        flat = t.view(-1)
        for s in range(0, flat.numel(), CHUNK):
            n = min(CHUNK, flat.numel() - s)
            x = torch.randn(n, generator=g, device=device, dtype=torch.float32).mul_(scale)
            flat[s:s + n].copy_(x.to(torch.float8_e4m3fn).view(torch.uint8))
    return k, v
