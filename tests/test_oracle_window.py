"""Pins for the oracle's draft-window key set and windowed attention (CPU only).

Source: Pith verdict on arXiv 2607.21535, pith_extraction.key_machinery: the draft's
per-request KV index is truncated to the first n_sink tokens plus the last W tokens; the keys
already carry their rotary phase, so dropping the middle does not disturb the remaining scores.
"""
import itertools

import numpy as np
import pytest

import oracle
from synthetic import gen


@pytest.mark.parametrize("L", list(range(0, 65, 3)) + [64])
def test_window_set_brute_force(L):
    """The kept set is literally positions[:s] + positions[-W:], for every s <= 4, W <= 16."""
    positions = list(range(L))
    for s, W in itertools.product(range(5), range(17)):
        expect = set(positions[:s]) | (set(positions[-W:]) if W > 0 else set())
        got = {j for j in range(-2, L + 3) if oracle.window_member(L, j, s, W)}
        assert got == expect, (L, s, W)


def test_window_key_visible_is_causal_per_query():
    """Multi-query draft call: the window is anchored on the request's length, then causal."""
    L, n_q, s, W = 30, 4, 2, 6
    for i in range(n_q):
        p_i = L - n_q + i
        vis = {j for j in range(L) if oracle.key_visible(oracle.MODE_WINDOW, L, n_q, i, j, s, W)}
        assert vis == {j for j in range(L) if (j < s or j >= L - W) and j <= p_i}


def _rand_case(seed, B, Hq, Hkv, Lmax, n_q, D=16):
    rng = np.random.default_rng(seed)
    q = gen.normal_bf16(rng, (B, n_q, Hq, D))
    k, v = gen.kv_pair_bf16(rng, (B, Hkv, Lmax, D))
    return q, k, v


@pytest.mark.parametrize("L,s,W,n_q", [(10, 4, 6, 1), (10, 4, 8, 3), (33, 1, 40, 2), (5, 4, 1, 1)])
def test_window_covering_context_equals_full(L, s, W, n_q):
    """s + W >= L: windowing drops nothing, so the result is identical to full attention."""
    q, k, v = _rand_case(1, 2, 4, 2, L, n_q)
    lens = np.array([L, L], dtype=np.int64)
    ow, lw = oracle.attention(q, k, v, lens, oracle.MODE_WINDOW, 0.3, n_sink=s, window=W)
    of, lf = oracle.attention(q, k, v, lens, oracle.MODE_CAUSAL, 0.3)
    assert np.array_equal(ow, of) and np.array_equal(lw, lf)


@pytest.mark.parametrize("L,s,W", [(40, 4, 8), (64, 2, 16), (17, 0, 5), (9, 3, 1)])
def test_window_equals_full_attention_on_kept_subsequence(L, s, W):
    """Windowed attention over L keys equals plain attention over the gathered kept keys."""
    q, k, v = _rand_case(2, 1, 8, 2, L, 1)
    kept = [j for j in range(L) if j < s or j >= L - W]
    ow, lw = oracle.attention(q, k, v, np.array([L]), oracle.MODE_WINDOW, 0.25, n_sink=s, window=W)
    ks, vs = k[:, :, kept], v[:, :, kept]
    of, lf = oracle.attention(q, ks, vs, np.array([len(kept)]), oracle.MODE_CAUSAL, 0.25)
    np.testing.assert_allclose(ow, of, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lw, lf, rtol=0, atol=1e-13)


def test_window_differs_from_full_when_keys_dropped():
    """Sanity: with a short window the result must change (the mask is really applied)."""
    q, k, v = _rand_case(3, 1, 4, 1, 50, 1)
    ow, _ = oracle.attention(q, k, v, np.array([50]), oracle.MODE_WINDOW, 0.3, n_sink=1, window=4)
    of, _ = oracle.attention(q, k, v, np.array([50]), oracle.MODE_CAUSAL, 0.3)
    assert np.abs(ow - of).max() > 1e-3
