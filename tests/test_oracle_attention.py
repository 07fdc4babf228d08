"""Pins for the oracle's fp64 attention (CPU only): closed forms, textbook special cases and
invariants, chosen so that a dropped term, a sign or index slip or a swapped operand fails.

Source: Pith verdict on arXiv 2607.21535, pith_extraction.key_machinery (windowing changes only
the draft's key set; the attention itself is ordinary softmax attention over cached keys).
"""
import math

import numpy as np
import pytest
from scipy.special import logsumexp

import oracle
from synthetic import gen
from tests.conftest import read_golden


def _bits(x):
    return gen.bf16_bits(np.asarray(x, dtype=np.float32))


def _f(bits):
    return gen.bf16_to_f32(bits).astype(np.float64)


def test_two_keys_hand_worked():
    g = {r[0]: float(r[1]) for r in read_golden("two_key_attention.txt")}
    D = 8
    q = np.zeros((1, 1, 1, D), np.float32); q[..., 0] = 1
    k = np.zeros((1, 1, 2, D), np.float32); k[0, 0, 1, 0] = 2
    v = np.zeros((1, 1, 2, D), np.float32); v[0, 0, 0, 0] = 1; v[0, 0, 1, 1] = 1
    o, lse = oracle.attention(_bits(q), _bits(k), _bits(v), np.array([2]), oracle.MODE_CAUSAL, 0.5)
    assert o[0, 0, 0, 0] == pytest.approx(g["o0"], abs=1e-15)
    assert o[0, 0, 0, 1] == pytest.approx(g["o1"], abs=1e-15)
    assert np.all(o[0, 0, 0, 2:] == 0)
    assert lse[0, 0, 0] == pytest.approx(g["lse"], abs=1e-15)


def test_single_key_returns_its_value_exactly():
    rng = np.random.default_rng(5)
    D = 128
    q = gen.normal_bf16(rng, (1, 1, 4, D))
    k, v = gen.kv_pair_bf16(rng, (1, 2, 1, D))
    o, lse = oracle.attention(q, k, v, np.array([1]), oracle.MODE_CAUSAL, 0.125)
    for h in range(4):
        assert np.array_equal(o[0, 0, h], _f(v[0, h // 2, 0]))          # GQA: kv head = h // G
        assert lse[0, 0, h] == pytest.approx(0.125 * float(_f(q[0, 0, h]) @ _f(k[0, h // 2, 0])),
                                             rel=1e-14)


def test_identical_keys_average_values():
    rng = np.random.default_rng(6)
    D, L = 32, 9
    q = gen.normal_bf16(rng, (1, 1, 1, D))
    krow = gen.normal_bf16(rng, (D,))
    k = np.broadcast_to(krow, (1, 1, L, D)).copy()
    v = gen.normal_bf16(rng, (1, 1, L, D))
    o, lse = oracle.attention(q, k, v, np.array([L]), oracle.MODE_CAUSAL, 0.7)
    np.testing.assert_allclose(o[0, 0, 0], _f(v[0, 0]).mean(axis=0), rtol=0, atol=1e-14)
    s = 0.7 * float(_f(q[0, 0, 0]) @ _f(krow))
    assert lse[0, 0, 0] == pytest.approx(s + math.log(L), rel=1e-13)


def test_matches_dense_textbook_softmax_attention():
    """n_q = 1 with every key visible is dense softmax(s QK^T) V: numpy, per head."""
    rng = np.random.default_rng(7)
    B, Hq, Hkv, L, D = 2, 6, 3, 23, 16
    q = gen.normal_bf16(rng, (B, 1, Hq, D))
    k, v = gen.kv_pair_bf16(rng, (B, Hkv, L, D))
    sc = 0.3
    o, lse = oracle.attention(q, k, v, np.array([L, L]), oracle.MODE_CAUSAL, sc)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            logits = sc * (_f(k[b, h // G]) @ _f(q[b, 0, h]))
            p = np.exp(logits - logits.max()); p /= p.sum()
            np.testing.assert_allclose(o[b, 0, h], p @ _f(v[b, h // G]), rtol=0, atol=1e-13)
            assert lse[b, 0, h] == pytest.approx(logsumexp(logits), rel=1e-13)


def test_causal_query_equals_prefix_attention():
    """Query i of an n_q-query causal call equals a one-query call over the prefix ending at it."""
    rng = np.random.default_rng(8)
    B, Hq, Hkv, L, D, n_q = 1, 4, 2, 31, 16, 5
    q = gen.normal_bf16(rng, (B, n_q, Hq, D))
    k, v = gen.kv_pair_bf16(rng, (B, Hkv, L, D))
    o, lse = oracle.attention(q, k, v, np.array([L]), oracle.MODE_CAUSAL, 0.2)
    for i in range(n_q):
        p_i = L - n_q + i
        oi, li = oracle.attention(q[:, i:i + 1], k[:, :, :p_i + 1], v[:, :, :p_i + 1],
                                  np.array([p_i + 1]), oracle.MODE_CAUSAL, 0.2)
        np.testing.assert_allclose(o[:, i], oi[:, 0], rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[:, i], li[:, 0], rtol=0, atol=1e-14)
    assert np.abs(o[:, 0] - o[:, -1]).max() > 1e-3    # the cut really differs per query


def test_key_permutation_invariance():
    rng = np.random.default_rng(9)
    L, D = 40, 16
    q = gen.normal_bf16(rng, (1, 1, 2, D))
    k, v = gen.kv_pair_bf16(rng, (1, 1, L, D))
    perm = rng.permutation(L)
    o1, l1 = oracle.attention(q, k, v, np.array([L]), oracle.MODE_CAUSAL, 0.4)
    o2, l2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], np.array([L]), oracle.MODE_CAUSAL, 0.4)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-13)


def test_empty_key_set_gives_zero_and_minus_inf():
    rng = np.random.default_rng(10)
    q = gen.normal_bf16(rng, (1, 2, 2, 8))
    k, v = gen.kv_pair_bf16(rng, (1, 1, 4, 8))
    # kv_len 1 with 2 queries: query 0 sits at position -1 and sees nothing.
    o, lse = oracle.attention(q, k, v, np.array([1]), oracle.MODE_CAUSAL, 1.0)
    assert np.all(o[0, 0] == 0) and np.all(lse[0, 0] == -np.inf)
    assert np.array_equal(o[0, 1, 0], _f(v[0, 0, 0]))


def test_rows_subset_matches_full_computation():
    rng = np.random.default_rng(12)
    q = gen.normal_bf16(rng, (2, 3, 4, 16))
    k, v = gen.kv_pair_bf16(rng, (2, 2, 20, 16))
    lens = np.array([20, 13])
    o, lse = oracle.attention(q, k, v, lens, oracle.MODE_WINDOW, 0.3, n_sink=2, window=5)
    rows = [(1, 2, 3), (0, 0, 1)]
    os_, ls = oracle.attention(q, k, v, lens, oracle.MODE_WINDOW, 0.3, n_sink=2, window=5, rows=rows)
    for b, i, h in rows:
        assert np.array_equal(os_[b, i, h], o[b, i, h]) and ls[b, i, h] == lse[b, i, h]
    assert np.isnan(os_[0, 1, 0]).all()


def test_thread_count_does_not_change_results():
    rng = np.random.default_rng(13)
    q = gen.normal_bf16(rng, (1, 4, 8, 32))
    k, v = gen.kv_pair_bf16(rng, (1, 2, 300, 32))
    a = oracle.attention(q, k, v, np.array([300]), oracle.MODE_CAUSAL, 0.2, n_threads=1)
    b = oracle.attention(q, k, v, np.array([300]), oracle.MODE_CAUSAL, 0.2, n_threads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
