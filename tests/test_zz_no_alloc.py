"""draft_attn_window_noalloc, the entry point for callers that cannot allocate device memory on
their decode path (engines with a fixed memory plan, loops that cannot take cudaMalloc's implicit
synchronisation): it must give the same result as draft_attn_window with a caller workspace.

Called through the C ABI twice in a row with different shapes and inputs, so that the second
call runs on scratch the first one left behind; each result is also checked against the fp64
oracle.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from long_context_speculative_kv_b200 import _lib
from synthetic import gen
from tests.gpu_util import assert_attn_close, assert_lse_close, to_dev_bf16, to_f64

pytestmark = pytest.mark.gpu

D = 128


def _case(seed, B, L, Hq, Hkv, n_q, s, W):
    rng = np.random.default_rng(seed)
    C = s + W
    k_tok, v_tok = gen.kv_pair_bf16(rng, (B, L, Hkv, D))
    q_bits = gen.normal_bf16(rng, (B, n_q, Hq, D))
    q = to_dev_bf16(q_bits)
    ring_k = torch.full((B, Hkv, C, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ring_v = ring_k.clone()
    rlen = torch.zeros(B, dtype=torch.int64, device="cuda")
    lib = _lib.lib()
    kd, vd = to_dev_bf16(k_tok), to_dev_bf16(v_tok)
    rc = lib.ring_kv_append(ring_k.data_ptr(), ring_v.data_ptr(), rlen.data_ptr(), kd.data_ptr(),
                            vd.data_ptr(), B, L, Hkv, D, s, C, None)
    assert rc == 0
    # oracle on the linear token layout [B, Hkv, L, D]
    ref, ref_lse = oracle.attention(q_bits, np.ascontiguousarray(k_tok.transpose(0, 2, 1, 3)),
                                    np.ascontiguousarray(v_tok.transpose(0, 2, 1, 3)),
                                    np.full(B, L, np.int64), oracle.MODE_WINDOW, 128 ** -0.5,
                                    n_sink=s, window=W)
    return q, ring_k, ring_v, rlen, C, ref, ref_lse


def _both(q, ring_k, ring_v, rlen, Hkv, s, W, C, sc):
    lib = _lib.lib()
    B, n_q, Hq, _ = q.shape
    outs = []
    for noalloc in (True, False):
        out = torch.empty_like(q)
        lse = torch.empty((B, n_q, Hq), dtype=torch.float32, device="cuda")
        if noalloc:
            rc = lib.draft_attn_window_noalloc(q.data_ptr(), ring_k.data_ptr(), ring_v.data_ptr(),
                                               rlen.data_ptr(), B, n_q, Hq, Hkv, D, s, W, C, sc,
                                               out.data_ptr(), lse.data_ptr(), None)
        else:
            n = lib.wmtp_workspace_bytes(B, n_q, Hq, Hkv, D)
            ws = torch.zeros(n, dtype=torch.uint8, device="cuda")   # control block zero
            rc = lib.draft_attn_window(q.data_ptr(), ring_k.data_ptr(), ring_v.data_ptr(),
                                       rlen.data_ptr(), B, n_q, Hq, Hkv, D, s, W, C, sc,
                                       out.data_ptr(), lse.data_ptr(), ws.data_ptr(), n, None)
        assert rc == 0, _lib.status_string(rc)
        torch.cuda.synchronize()
        outs.append((to_f64(out), lse.cpu().numpy()))
    return outs


def test_noalloc_matches_workspace_call_twice_in_a_row():
    sc = 128 ** -0.5
    # call 1: the 1M workload's draft forward shape (B 1, GQA 32/4, one query, 4 + 4092 window)
    q, rk, rv, rl, C, ref, ref_lse = _case(11, 1, 20000, 32, 4, 1, 4, 4092)
    (a, la), (b, lb) = _both(q, rk, rv, rl, 4, 4, 4092, C, sc)
    assert_attn_close(a, b, "noalloc call 1")
    assert_lse_close(la, lb)
    assert_attn_close(a, ref, "noalloc call 1 vs oracle")
    assert_lse_close(la, ref_lse)
    # call 2: a different shape on the scratch call 1 left behind (ragged batch, 4 queries)
    q, rk, rv, rl, C, ref, ref_lse = _case(12, 3, 5000, 16, 2, 4, 4, 1020)
    (a, la), (b, lb) = _both(q, rk, rv, rl, 2, 4, 1020, C, sc)
    assert_attn_close(a, b, "noalloc call 2")
    assert_lse_close(la, lb)
    assert_attn_close(a, ref, "noalloc call 2 vs oracle")
    assert_lse_close(la, ref_lse)


def test_noalloc_rejects_shapes_beyond_the_scratch():
    lib = _lib.lib()
    # 64-row units (8 queries x 8 heads per kv head), 16 x 8 of them: with one or two CTAs per SM
    # that is more than the 254 slots of 64 rows the 8 MiB scratch holds
    B, n_q, Hq, Hkv, C = 16, 8, 64, 8, 64
    q = torch.zeros((B, n_q, Hq, D), dtype=torch.bfloat16, device="cuda")
    ring = torch.zeros((B, Hkv, C, D), dtype=torch.bfloat16, device="cuda")
    rl = torch.full((B,), C, dtype=torch.int64, device="cuda")
    out = torch.empty_like(q)
    n0 = lib.wmtp_launch_count()
    rc = lib.draft_attn_window_noalloc(q.data_ptr(), ring.data_ptr(), ring.data_ptr(), rl.data_ptr(),
                                       B, n_q, Hq, Hkv, D, 4, C - 4, C, 0.1, out.data_ptr(), None, None)
    assert rc == -9 and "scratch" in _lib.status_string(rc)
    assert lib.wmtp_launch_count() == n0
