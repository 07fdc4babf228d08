"""Seeded random shapes against the fp64 oracle, across every kernel-selection boundary: rows per
unit (n_q x query heads per kv head) from 1 to 128 (the mma.sync layouts of <= 16 and 17-32 rows,
the tcgen05 kernel of 33-64, two row blocks above 64), ragged request lengths from 1 key to a few
thousand (tiles split over CTAs or finished inside one), chain and tree verify, full and windowed
draft, bf16 and fp8 (E4M3) caches.

Sources: Pith verdict on arXiv 2607.21535, pith_extraction.key_machinery (draft attention over the
sink plus the recent window; verification with full attention over the gamma + 1 positions or the
tree) and forward_implications[4] (fp8 KV).
"""
import numpy as np
import pytest

import oracle
from tests.gpu_util import assert_attn_close, assert_lse_close
from tests.test_gpu_attention import paged_case, ring_case, run_paged, run_window
from tests.test_gpu_fp8 import KS, VS, paged8_case, run_paged8

pytestmark = pytest.mark.gpu

D = 128
SC = 128 ** -0.5


def _shape(rng):
    Hkv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([1, 2, 4, 8, 16]))
    n_q = int(rng.integers(1, 9))
    B = int(rng.integers(1, 5))
    lens = [int(x) for x in rng.integers(1, 3000, size=B)]
    return B, Hkv, G, n_q, lens


def _tree(rng, B, n_q):
    """Parent of node i < i (node 0 the root), drawn per request."""
    par = np.zeros((B, n_q), np.int32)
    for b in range(B):
        par[b, 0] = -1
        for i in range(1, n_q):
            par[b, i] = int(rng.integers(0, i))
    return par


@pytest.mark.parametrize("seed", range(12))
def test_random_verify_and_full_draft(seed):
    rng = np.random.default_rng(1000 + seed)
    B, Hkv, G, n_q, lens = _shape(rng)
    tree = seed % 3 == 2
    lens_v = [L + n_q for L in lens]
    c = paged_case(2000 + seed, lens_v, Hkv * G, Hkv, n_q)
    par = _tree(rng, B, n_q) if tree else None
    out, lse = run_paged(c, "verify", SC, tree=par)
    if tree:
        ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_TREE, SC,
                                        tree_parent=par)
    else:
        ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_CAUSAL, SC)
    where = f"verify seed {seed}: B {B}, Hkv {Hkv}, G {G}, n_q {n_q}, tree {tree}, lens {lens_v}"
    assert_attn_close(out, ref, where)
    assert_lse_close(lse, ref_lse, where)
    c = paged_case(3000 + seed, lens, Hkv * G, Hkv, n_q)
    out, lse = run_paged(c, "full", SC)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_CAUSAL, SC)
    assert_attn_close(out, ref, f"full draft seed {seed}")
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("seed", range(8))
def test_random_windowed_draft(seed):
    rng = np.random.default_rng(4000 + seed)
    B, Hkv, G, n_q, lens = _shape(rng)
    n_q = min(n_q, 4)
    s = int(rng.choice([0, 4]))
    W = int(rng.choice([60, 252, 1020]))
    C = s + W + int(rng.integers(0, 5))
    c = ring_case(5000 + seed, lens, Hkv * G, Hkv, n_q, s, W, C)
    out, lse = run_window(c, SC)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_WINDOW, SC,
                                    n_sink=s, window=W)
    where = f"window seed {seed}: B {B}, Hkv {Hkv}, G {G}, n_q {n_q}, s {s}, W {W}, C {C}, lens {lens}"
    assert_attn_close(out, ref, where)
    assert_lse_close(lse, ref_lse, where)


@pytest.mark.parametrize("seed", range(6))
def test_random_fp8_verify_and_full_draft(seed):
    rng = np.random.default_rng(6000 + seed)
    B, Hkv, G, n_q, lens = _shape(rng)
    lens_v = [L + n_q for L in lens]
    c = paged8_case(7000 + seed, lens_v, Hkv * G, Hkv, n_q)
    out, lse = run_paged8(c, "verify", SC)
    ref, ref_lse = oracle.attention_kv8(c["q"], c["k8"], c["v8"], c["lens"], oracle.MODE_CAUSAL, SC, KS, VS)
    where = f"fp8 verify seed {seed}: B {B}, Hkv {Hkv}, G {G}, n_q {n_q}, lens {lens_v}"
    assert_attn_close(out, ref, where)
    assert_lse_close(lse, ref_lse, where)
    c = paged8_case(8000 + seed, lens, Hkv * G, Hkv, 1)
    out, lse = run_paged8(c, "full", SC)
    ref, ref_lse = oracle.attention_kv8(c["q"], c["k8"], c["v8"], c["lens"], oracle.MODE_CAUSAL, SC, KS, VS)
    assert_attn_close(out, ref, f"fp8 full draft seed {seed}")
    assert_lse_close(lse, ref_lse)
