"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle's tests.

This module holds no arithmetic of the method itself: it draws random tensors, rounds them to
bf16 once (both sides then read the same bits), lays them out (paged pool, page table), and
builds draft trees, lengths and synthetic target logits.

Recipe (seeded numpy PCG64 unless a torch device generator is asked for):
  * Q, K, V ~ N(0, 1) drawn in float32, K multiplied by ``k_scale``, outlier rows (each
    (token, kv-head) row chosen with probability p, the same choice for K and V) multiplied by
    ``outlier_factor``, then rounded to nearest-even bf16.
  * Page table: a random permutation of exactly sum_b ceil(L_b / P) physical pages; the tail
    rows of each sequence's last page are NaN, so any read of them shows up in the output.
  * Draft tree of n nodes: nodes 0..3 form a chain; each later node picks a uniformly random
    parent among the nodes that have fewer than 2 children and depth <= 2.
  * Synthetic target logits for the lossless-decoding harness: a counter-based generator,
    splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number generators", 2014)
    over (seed, last four tokens, prefix length, vocabulary index) -> 24-bit uniform -> U(-1, 1).
"""
from typing import List, Optional, Sequence, Tuple

import numpy as np

_MASK64 = np.uint64(0xFFFFFFFFFFFFFFFF)


# ----------------------------------------------------------------------------- bf16 bits
def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even; NaN -> quiet NaN."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


BF16_NAN = np.uint16(0x7FC0)


def normal_bf16(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    return bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(scale))


def kv_pair_bf16(rng: np.random.Generator, shape, k_scale: float = 1.0, outlier_p: float = 0.0,
                 outlier_factor: float = 8.0, row_axes: int = 3) -> Tuple[np.ndarray, np.ndarray]:
    """K and V bits of ``shape``; a row is the last axis.  Outlier rows (probability outlier_p
    over the leading ``row_axes`` axes) scale both K and V by outlier_factor before rounding."""
    k = rng.standard_normal(shape, dtype=np.float32) * np.float32(k_scale)
    v = rng.standard_normal(shape, dtype=np.float32)
    if outlier_p > 0.0:
        rows = rng.random(shape[:row_axes]) < outlier_p
        k[rows] *= np.float32(outlier_factor)
        v[rows] *= np.float32(outlier_factor)
    return bf16_bits(k), bf16_bits(v)


# ----------------------------------------------------------------------------- paged layout
def n_pages(lens: Sequence[int], page_size: int) -> int:
    return int(sum((int(L) + page_size - 1) // page_size for L in lens))


def page_table(rng: np.random.Generator, lens: Sequence[int], page_size: int,
               max_pages: Optional[int] = None) -> np.ndarray:
    """int32 [B, max_pages]: a random permutation of exactly sum ceil(L_b/P) pages; unused
    entries are -1."""
    need = [(int(L) + page_size - 1) // page_size for L in lens]
    if max_pages is None:
        max_pages = max(need) if need else 0
    perm = rng.permutation(sum(need)).astype(np.int32)
    table = np.full((len(lens), max_pages), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[off:off + n]
        off += n
    return table


def paginate(linear: np.ndarray, lens: Sequence[int], table: np.ndarray, page_size: int,
             poison: bool = True) -> np.ndarray:
    """Scatter a logical [B, Hkv, Lmax, D] sequence into a pool [num_pages, Hkv, P, D]; rows past
    each sequence's end are NaN when ``poison``."""
    B, Hkv, Lmax, D = linear.shape
    num = n_pages(lens, page_size)
    pool = np.full((num, Hkv, page_size, D), BF16_NAN if poison else 0, dtype=np.uint16)
    for b in range(B):
        L = int(lens[b])
        for t in range((L + page_size - 1) // page_size):
            r0 = t * page_size
            r1 = min(L, r0 + page_size)
            pool[table[b, t], :, : r1 - r0, :] = linear[b, :, r0:r1, :]
    return pool


def gather_logical(pool: np.ndarray, table_row: np.ndarray, L: int, page_size: int,
                   heads: Optional[Sequence[int]] = None) -> np.ndarray:
    """Inverse view: the logical [Hsel, L, D] sequence of one request from a pool."""
    n = (L + page_size - 1) // page_size
    pages = pool[table_row[:n]]                     # [n, Hkv, P, D]
    if heads is not None:
        pages = pages[:, list(heads)]
    seq = np.transpose(pages, (1, 0, 2, 3)).reshape(pages.shape[1], n * page_size, pages.shape[3])
    return np.ascontiguousarray(seq[:, :L])


# ----------------------------------------------------------------------------- trees, lengths
def draft_tree(rng: np.random.Generator, n: int = 8, chain: int = 4, max_children: int = 2,
               max_parent_depth: int = 2) -> np.ndarray:
    """int32 parent array: parent[0] = -1, nodes 1..chain-1 extend a chain, later nodes attach to
    a uniformly drawn node with < max_children children and depth <= max_parent_depth."""
    parent = np.full(n, -1, dtype=np.int32)
    depth = np.zeros(n, dtype=np.int64)
    children = np.zeros(n, dtype=np.int64)
    for i in range(1, min(chain, n)):
        parent[i] = i - 1
        depth[i] = depth[i - 1] + 1
        children[i - 1] += 1
    for i in range(min(chain, n), n):
        cand = [j for j in range(i) if children[j] < max_children and depth[j] <= max_parent_depth]
        p = int(cand[int(rng.integers(len(cand)))])
        parent[i] = p
        depth[i] = depth[p] + 1
        children[p] += 1
    return parent


def chain_parents(n: int) -> np.ndarray:
    return np.arange(-1, n - 1, dtype=np.int32)


def ragged_contexts(rng: np.random.Generator, B: int, lo: int, hi: int) -> np.ndarray:
    return rng.integers(lo, hi + 1, size=B).astype(np.int64)


def uniform_logits(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.uniform(-1.0, 1.0, size=shape).astype(np.float32)


# ----------------------------------------------------------------------------- splitmix64
def splitmix64(x: np.ndarray) -> np.ndarray:
    """The splitmix64 output function applied to (x + golden gamma), vectorised over uint64."""
    with np.errstate(over="ignore"):
        z = (np.asarray(x, dtype=np.uint64) + np.uint64(0x9E3779B97F4A7C15)) & _MASK64
        z = ((z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)) & _MASK64
        z = ((z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)) & _MASK64
        return z ^ (z >> np.uint64(31))


def target_logits(seed: int, prefix: Sequence[int], vocab: int) -> np.ndarray:
    """Synthetic target: f32 logits for the next token after ``prefix`` (a deterministic function
    of the seed, the last four tokens and the prefix length)."""
    h = splitmix64(np.uint64(seed & 0xFFFFFFFFFFFFFFFF))
    last = list(prefix[-4:])
    last = [-1] * (4 - len(last)) + last
    for t in last:
        h = splitmix64(h ^ np.uint64((int(t) + 1) & 0xFFFFFFFF))
    h = splitmix64(h ^ np.uint64(len(prefix)))
    z = splitmix64(h ^ np.arange(vocab, dtype=np.uint64))
    u = (z >> np.uint64(40)).astype(np.float64) / float(1 << 24)
    return (2.0 * u - 1.0).astype(np.float32)


def draft_proposals(policy: str, rng: np.random.Generator, target_next, gamma: int, vocab: int,
                    n_correct: int = 0) -> List[int]:
    """gamma proposed tokens.  ``target_next(tokens_so_far)`` gives the target's greedy next
    token after the committed prefix extended by the given proposals (used by the 'correct',
    'adversarial' and 'correct-then-wrong' policies).  'random' ignores it."""
    out: List[int] = []
    for j in range(gamma):
        if policy == "random":
            out.append(int(rng.integers(vocab)))
            continue
        t = int(target_next(out))
        if policy == "correct" or (policy == "correct-then-wrong" and j < n_correct):
            out.append(t)
        else:
            out.append((t + 1 + int(rng.integers(vocab - 1))) % vocab)
    return out


def hash_draft_tokens(target_seed: int, draft_seed: int, prefix: Sequence[int], gamma: int,
                      vocab: int, agree24: int) -> List[int]:
    """gamma chained proposals of the counter-based synthetic draft: proposal j extends the
    prefix (and proposals 0..j-1) by the synthetic target's greedy token when
    (z >> 40) < agree24, z = mix(mix(draft_seed ^ length) ^ (uint32)(last + 1)), and by
    (greedy + 1 + mix(z) mod (vocab - 1)) mod vocab otherwise (mix = splitmix64)."""
    out: List[int] = []
    for _ in range(gamma):
        path = list(prefix) + out
        greedy = int(np.argmax(target_logits(target_seed, path, vocab)))
        z = splitmix64(splitmix64(np.uint64(draft_seed & 0xFFFFFFFFFFFFFFFF) ^ np.uint64(len(path)))
                       ^ np.uint64((int(path[-1]) + 1) & 0xFFFFFFFF))
        agree = int(z >> np.uint64(40)) < agree24
        r = int(splitmix64(z)) % (vocab - 1)
        out.append(greedy if agree else (greedy + 1 + r) % vocab)
    return out


# ----------------------------------------------------------------------------- fp8 (E4M3) codes
def _e4m3_grid() -> np.ndarray:
    """Values of the positive E4M3 codes 0 .. 126 (OCP OFP8: bias 7, subnormals (m/8) 2^-6,
    S.1111.111 reserved for NaN)."""
    vals = [m / 8.0 * 2.0 ** -6 for m in range(8)]
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                break
            vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.asarray(vals, dtype=np.float64)


_E4M3_GRID = _e4m3_grid()


def e4m3_codes(x) -> np.ndarray:
    """uint8 E4M3 codes of x: round to nearest, ties to the even code, saturating at +-448
    (how an fp8 KV cache writer quantises); NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 448.0)
    idx = np.clip(np.searchsorted(_E4M3_GRID, a), 1, len(_E4M3_GRID) - 1)
    lo, hi = _E4M3_GRID[idx - 1], _E4M3_GRID[idx]
    dlo, dhi = a - lo, hi - a
    take_hi = (dhi < dlo) | ((dhi == dlo) & (idx % 2 == 0))
    code = np.where(take_hi, idx, idx - 1).astype(np.uint8)
    code = np.where(x < 0, code | np.uint8(0x80), code).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)
