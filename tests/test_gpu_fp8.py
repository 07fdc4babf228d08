"""GPU parity of the fp8 (E4M3) KV calls against the fp64 oracle on the dequantised cache.

Source: Pith verdict on arXiv 2607.21535, pith_extraction.forward_implications[4] (windowing
composes with fp8 KV quantisation).  Codes come from N(0, 2^2) values rounded to E4M3; key and
value scales are not powers of two; page tails hold NaN codes and unwritten ring slots hold
garbage, so a stray read shows.  Row counts 8, 24, 25, 32, 48 and 64 per unit exercise every
fp8 layout.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_speculative_kv_b200 import api
from synthetic import gen
from tests.gpu_util import assert_attn_close, assert_lse_close, to_dev_bf16, to_f64

pytestmark = pytest.mark.gpu

D = 128
P = 64
KS, VS = 0.37, 1.9


def codes(rng, shape):
    return gen.e4m3_codes(rng.standard_normal(shape) * 2.0)


def paginate8(lin8, lens, table):
    """[B, Hkv, L, 128] codes -> pool [pages, Hkv, 64, 128]; tail rows of last pages are NaN-ish."""
    pool16 = gen.paginate(np.ascontiguousarray(lin8).view(np.uint16), lens, table, P)
    return np.ascontiguousarray(pool16).view(np.uint8)


def dev8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def paged8_case(seed, lens, Hq, Hkv, n_q):
    rng = np.random.default_rng(seed)
    B, L = len(lens), max(lens)
    q = gen.normal_bf16(rng, (B, n_q, Hq, D))
    k8, v8 = codes(rng, (B, Hkv, L, D)), codes(rng, (B, Hkv, L, D))
    table = gen.page_table(rng, lens, P)
    return dict(q=q, k8=k8, v8=v8, kp=paginate8(k8, lens, table), vp=paginate8(v8, lens, table),
                table=table, lens=np.asarray(lens, np.int64))


def run_paged8(c, fn, sm_scale, tree=None):
    B, n_q, Hq, _ = c["q"].shape
    Hkv = c["k8"].shape[1]
    ws = api.alloc_workspace(B, n_q, Hq, Hkv)
    args = (to_dev_bf16(c["q"]), dev8(c["kp"]), dev8(c["vp"]), torch.from_numpy(c["table"]).cuda(),
            torch.from_numpy(c["lens"].astype(np.int32)).cuda())
    if fn == "verify":
        t = None if tree is None else torch.from_numpy(np.ascontiguousarray(tree, np.int32)).cuda()
        out, lse = api.verify_attn_fp8(*args, sm_scale, KS, VS, ws, tree_parent=t)
    else:
        out, lse = api.draft_attn_full_fp8(*args, sm_scale, KS, VS, ws)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return to_f64(out), lse.cpu().numpy()


@pytest.mark.parametrize("lens,Hq,Hkv,n_q", [
    ([2048], 8, 2, 1),                       # 8 rows per unit
    ([130, 1000, 4097, 7], 16, 2, 1),        # ragged, several splits
    ([3000, 65], 8, 1, 4),                   # 32 rows
    ([1500], 32, 4, 1),
    ([64] * 30, 8, 2, 1),                    # units finished inside one CTA
])
def test_draft_full_fp8_matches_oracle(lens, Hq, Hkv, n_q):
    sc = 128 ** -0.5
    c = paged8_case(11, lens, Hq, Hkv, n_q)
    out, lse = run_paged8(c, "full", sc)
    ref, ref_lse = oracle.attention_kv8(c["q"], c["k8"], c["v8"], c["lens"], oracle.MODE_CAUSAL, sc, KS, VS)
    assert_attn_close(out, ref, "draft_attn_full_fp8")
    assert_lse_close(lse, ref_lse, "draft_attn_full_fp8 lse")


@pytest.mark.parametrize("lens,Hq,Hkv,n_q", [
    ([5000], 32, 4, 4),                      # gamma 3: 32 rows
    ([64, 2047, 9000], 16, 2, 3),            # 24 rows: a ragged second m-tile
    ([5, 300], 20, 4, 5),                    # 25 rows; the first request holds only the step
    ([777, 2500], 16, 2, 6),                 # 48 rows
    ([4100], 16, 2, 8),                      # 64 rows
])
def test_verify_chain_fp8_matches_oracle(lens, Hq, Hkv, n_q):
    sc = 128 ** -0.5
    c = paged8_case(12, lens, Hq, Hkv, n_q)
    out, lse = run_paged8(c, "verify", sc)
    ref, ref_lse = oracle.attention_kv8(c["q"], c["k8"], c["v8"], c["lens"], oracle.MODE_CAUSAL, sc, KS, VS)
    assert_attn_close(out, ref, "verify_attn_fp8 chain")
    assert_lse_close(lse, ref_lse, "verify_attn_fp8 chain lse")


@pytest.mark.parametrize("Hq,Hkv,n_q", [
    (32, 4, 8),                              # 64 rows
    (32, 4, 4),                              # 32 rows
])
def test_verify_tree_fp8_matches_oracle(Hq, Hkv, n_q):
    sc = 128 ** -0.5
    lens = [900, 3000, 70]
    c = paged8_case(13, lens, Hq, Hkv, n_q)
    rng = np.random.default_rng(13)
    tree = np.stack([gen.draft_tree(rng, n_q) for _ in lens])
    out, lse = run_paged8(c, "verify", sc, tree=tree)
    ref, ref_lse = oracle.attention_kv8(c["q"], c["k8"], c["v8"], c["lens"], oracle.MODE_TREE, sc, KS, VS,
                                        tree_parent=tree)
    assert_attn_close(out, ref, "verify_attn_fp8 tree")
    assert_lse_close(lse, ref_lse, "verify_attn_fp8 tree lse")


@pytest.mark.parametrize("L,n_q,s,W,C", [
    (5000, 1, 4, 252, 256),      # wrapped ring, one query
    (5000, 4, 4, 252, 259),      # context pass, slack 3
    (180, 1, 4, 252, 256),       # context shorter than the window
])
def test_ring_fp8_append_and_window_attention(L, n_q, s, W, C):
    rng = np.random.default_rng(L + n_q)
    B, Hq, Hkv = 2, 16, 2
    k_tok, v_tok = codes(rng, (B, L, Hkv, D)), codes(rng, (B, L, Hkv, D))
    ring_k = dev8(np.full((B, Hkv, C, D), 0x7F, np.uint8))
    ring_v = dev8(np.full((B, Hkv, C, D), 0x7F, np.uint8))
    rlen = torch.zeros(B, dtype=torch.int64, device="cuda")
    cut = L - 3
    api.ring_kv_append_fp8(ring_k, ring_v, rlen, dev8(k_tok[:, :cut]), dev8(v_tok[:, :cut]), s)
    for t in range(cut, L):
        api.ring_kv_append_fp8(ring_k, ring_v, rlen, dev8(k_tok[:, t:t + 1]), dev8(v_tok[:, t:t + 1]), s)
    # ring bytes equal the oracle's ring (the slot rule does not depend on the element type)
    rk16 = np.full((B, Hkv, C, D // 2), 0x7F7F, np.uint16)
    rv16 = rk16.copy()
    rl = np.zeros(B, np.int64)
    oracle.ring_kv_append(rk16, rv16, rl, np.ascontiguousarray(k_tok).view(np.uint16),
                          np.ascontiguousarray(v_tok).view(np.uint16), s)
    assert np.array_equal(ring_k.cpu().numpy(), rk16.view(np.uint8))
    assert np.array_equal(ring_v.cpu().numpy(), rv16.view(np.uint8))
    assert rlen.cpu().tolist() == [L, L]
    q = gen.normal_bf16(rng, (B, n_q, Hq, D))
    ws = api.alloc_workspace(B, n_q, Hq, Hkv)
    sc = 128 ** -0.5
    out, lse = api.draft_attn_window_fp8(to_dev_bf16(q), ring_k, ring_v, rlen, s, W, sc, KS, VS, ws)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    k_lin = np.ascontiguousarray(k_tok.transpose(0, 2, 1, 3))
    v_lin = np.ascontiguousarray(v_tok.transpose(0, 2, 1, 3))
    ref, ref_lse = oracle.attention_kv8(q, k_lin, v_lin, np.array([L, L]), oracle.MODE_WINDOW, sc, KS, VS,
                                        n_sink=s, window=W)
    assert_attn_close(to_f64(out), ref, "draft_attn_window_fp8")
    assert_lse_close(lse.cpu().numpy(), ref_lse, "draft_attn_window_fp8 lse")


@pytest.mark.parametrize("W", [124, 316, 636, 1276, 2556])
@pytest.mark.parametrize("n_q", [1, 4, 8])
def test_fp8_window_every_cluster_size(W, n_q):
    """fp8 rings whose windows span 2, 5, 10, 20 and 40 tiles: the cluster window kernel with
    1, 2, 4, 8 and 16 CTAs per unit, against the oracle on the dequantised cache."""
    rng = np.random.default_rng(W + n_q)
    B, Hq, Hkv, s = 2, 32, 4, 4
    C = s + W
    lens = [3 * C + 37, 2 * C + 5]
    L = max(lens)
    k_tok, v_tok = codes(rng, (B, L, Hkv, D)), codes(rng, (B, L, Hkv, D))
    ring_k = dev8(np.full((B, Hkv, C, D), 0x7F, np.uint8))
    ring_v = dev8(np.full((B, Hkv, C, D), 0x7F, np.uint8))
    rlen = torch.zeros(B, dtype=torch.int64, device="cuda")
    for b in range(B):
        api.ring_kv_append_fp8(ring_k[b:b + 1], ring_v[b:b + 1], rlen[b:b + 1],
                               dev8(k_tok[b:b + 1, :lens[b]]), dev8(v_tok[b:b + 1, :lens[b]]), s)
    q = gen.normal_bf16(rng, (B, n_q, Hq, D))
    ws = api.alloc_workspace(B, n_q, Hq, Hkv)
    sc = 128 ** -0.5
    out, lse = api.draft_attn_window_fp8(to_dev_bf16(q), ring_k, ring_v, rlen, s, W, sc, KS, VS, ws)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    k_lin = np.ascontiguousarray(k_tok.transpose(0, 2, 1, 3))
    v_lin = np.ascontiguousarray(v_tok.transpose(0, 2, 1, 3))
    ref, ref_lse = oracle.attention_kv8(q, k_lin, v_lin, np.array(lens), oracle.MODE_WINDOW, sc, KS, VS,
                                        n_sink=s, window=W)
    assert_attn_close(to_f64(out), ref, "draft_attn_window_fp8")
    assert_lse_close(lse.cpu().numpy(), ref_lse, "draft_attn_window_fp8 lse")


def test_fp8_equals_bf16_path_on_identical_values():
    """With unit scales, the fp8 call and the bf16 call on the same (exactly representable)
    numbers agree to within the two paths' rounding of the weights (fp16 vs bf16)."""
    sc = 128 ** -0.5
    c = paged8_case(14, [3000], 16, 2, 1)
    B, n_q, Hq, _ = c["q"].shape
    ws = api.alloc_workspace(B, n_q, Hq, 2)
    qd, tb = to_dev_bf16(c["q"]), torch.from_numpy(c["table"]).cuda()
    kl = torch.from_numpy(c["lens"].astype(np.int32)).cuda()
    o8, _ = api.draft_attn_full_fp8(qd, dev8(c["kp"]), dev8(c["vp"]), tb, kl, sc, 1.0, 1.0, ws)
    as16 = lambda p: oracle.oracle._f64_to_bf16_bits_exact(oracle.e4m3_decode(p))
    o16, _ = api.draft_attn_full(qd, to_dev_bf16(as16(c["kp"])), to_dev_bf16(as16(c["vp"])), tb, kl, sc, ws)
    torch.cuda.synchronize()
    ref, _ = oracle.attention_kv8(c["q"], c["k8"], c["v8"], c["lens"], oracle.MODE_CAUSAL, sc, 1.0, 1.0)
    assert_attn_close(to_f64(o8), ref, "fp8 path")
    assert_attn_close(to_f64(o16), ref, "bf16 path")


@pytest.mark.parametrize("Hq,Hkv,n_q", [
    (8, 2, 1),                               # 4 rows: shared-memory Q layout
    (8, 2, 4),                               # 16 rows: shared-memory Q layout, 4 queries
    (32, 4, 4),                              # 32 rows: register layout
])
def test_fp8_empty_and_short_sequences(Hq, Hkv, n_q):
    """kv_len 0 gives out 0 / lse -inf; kv_len < n_q leaves the early queries with no keys."""
    sc = 0.1
    c = paged8_case(15, [0, 2, 70], Hq, Hkv, n_q)
    out, lse = run_paged8(c, "full", sc)
    ref, ref_lse = oracle.attention_kv8(c["q"], c["k8"], c["v8"], c["lens"], oracle.MODE_CAUSAL, sc, KS, VS)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert_attn_close(out, ref, "draft_attn_full_fp8 short")
    assert_lse_close(lse, ref_lse, "draft_attn_full_fp8 short lse")


def test_fp8_bad_page_id_sets_status_and_skips_tile():
    sc = 128 ** -0.5
    c = paged8_case(16, [640, 640], 8, 2, 1)
    bad = c["table"].copy()
    bad[1, 3] = 10 ** 6                                  # out of range for request 1 only
    B, n_q, Hq, _ = c["q"].shape
    ws = api.alloc_workspace(B, n_q, Hq, 2)
    out, _ = api.draft_attn_full_fp8(to_dev_bf16(c["q"]), dev8(c["kp"]), dev8(c["vp"]),
                                     torch.from_numpy(bad).cuda(),
                                     torch.from_numpy(c["lens"].astype(np.int32)).cuda(), sc, KS, VS, ws)
    assert api.device_status() == -6
    assert api.device_status() == 0                      # read-and-clear
    ref, _ = oracle.attention_kv8(c["q"], c["k8"], c["v8"], c["lens"], oracle.MODE_CAUSAL, sc, KS, VS)
    assert_attn_close(to_f64(out)[:1], ref[:1], "request 0 unaffected")
    assert not np.isnan(to_f64(out)).any()
