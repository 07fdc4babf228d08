"""Pins of the oracle's fp8 (E4M3) KV path (CPU only).

Pith verdict on arXiv 2607.21535, pith_extraction.forward_implications[4]: windowing composes
with KV quantisation (fp8).  The format's values come from the OCP 8-bit floating point
specification (golden table with its citation); attention over an fp8 cache is the fp64
definition on the dequantised keys and values, pinned against the bf16 oracle where both hold
the same numbers, and against closed forms for the scales.
"""
import math

import numpy as np
import pytest

import oracle
from synthetic import gen
from tests.conftest import read_golden
D = 16


def test_published_e4m3_values():
    for code, val in read_golden("e4m3_values.txt"):
        got = oracle.e4m3_value(int(code, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val), code


def test_e4m3_codes_are_ordered_and_finite_except_nan():
    vals = [oracle.e4m3_value(c) for c in range(256)]
    nans = [c for c in range(256) if math.isnan(vals[c])]
    assert nans == [0x7F, 0xFF]                     # no infinities, two NaNs
    pos = vals[:0x7F]
    assert all(a < b for a, b in zip(pos, pos[1:]))  # codes 0..126 strictly increasing
    assert all(vals[c | 0x80] == -vals[c] for c in range(0x7F))
    assert max(pos) == 448.0 and len(set(pos)) == 127


def test_generator_rounds_to_the_nearest_code():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(4000) * 3, [500.0, -1e6, 0.0, 2.0 ** -12, 0.0068359375]])
    codes = gen.e4m3_codes(x)
    vals = oracle.e4m3_decode(codes)
    grid = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    for xi, vi in zip(np.clip(x, -448, 448), vals):
        best = np.min(np.abs(grid - abs(xi)))
        assert abs(abs(vi) - abs(xi)) == pytest.approx(best, abs=1e-12)


def _fp8_case(seed, lens, Hq, Hkv, n_q):
    rng = np.random.default_rng(seed)
    B, L = len(lens), max(lens)
    q = gen.normal_bf16(rng, (B, n_q, Hq, D))
    k8 = gen.e4m3_codes(rng.standard_normal((B, Hkv, L, D)) * 2)
    v8 = gen.e4m3_codes(rng.standard_normal((B, Hkv, L, D)) * 2)
    return q, k8, v8, np.asarray(lens, np.int64)


def _as_bf16(codes):
    return oracle.oracle._f64_to_bf16_bits_exact(oracle.e4m3_decode(codes))


def test_unit_scales_equal_the_bf16_oracle_on_the_same_values():
    q, k8, v8, lens = _fp8_case(1, [77, 200], 8, 2, 3)
    got, lse = oracle.attention_kv8(q, k8, v8, lens, oracle.MODE_CAUSAL, 0.1, 1.0, 1.0)
    ref, ref_lse = oracle.attention(q, _as_bf16(k8), _as_bf16(v8), lens, oracle.MODE_CAUSAL, 0.1)
    assert np.array_equal(got, ref) and np.array_equal(lse, ref_lse)


def test_scales_act_as_scaled_keys_and_values():
    # a power-of-two scale is exact in bf16: k_scale = 2 equals doubled keys, v_scale = 0.5 halves
    q, k8, v8, lens = _fp8_case(2, [150], 8, 2, 2)
    got, lse = oracle.attention_kv8(q, k8, v8, lens, oracle.MODE_WINDOW, 0.05, 2.0, 0.5,
                                    n_sink=4, window=40)
    kd = oracle.e4m3_decode(k8) * 2.0
    vd = oracle.e4m3_decode(v8) * 0.5
    ref, ref_lse = oracle.attention(q, oracle.oracle._f64_to_bf16_bits_exact(kd),
                                    oracle.oracle._f64_to_bf16_bits_exact(vd), lens,
                                    oracle.MODE_WINDOW, 0.05, n_sink=4, window=40)
    assert np.allclose(got, ref, rtol=0, atol=1e-12) and np.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_single_key_returns_its_scaled_value():
    q, k8, v8, _ = _fp8_case(3, [1], 4, 1, 1)
    out, lse = oracle.attention_kv8(q, k8, v8, np.array([1]), oracle.MODE_CAUSAL, 0.3, 1.7, 0.37)
    want = oracle.e4m3_decode(v8[0, 0, 0]) * 0.37
    for h in range(4):
        assert np.allclose(out[0, 0, h], want, rtol=0, atol=1e-15)
