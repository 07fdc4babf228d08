"""GPU parity of draft_attn_window_append: a draft forward's ring append fused into the windowed
attention kernel (one launch).  The ring and its lengths must come out bit-identical to
ring_kv_append's, and the attention must match the fp64 oracle's windowed attention over the
linear token sequence, step after step through the ring's wraparound.

Sources: Pith verdict on arXiv 2607.21535, pith_extraction.key_machinery (each draft forward
writes its token's draft KV and attends over the first n_sink plus the last W tokens) and
referee_report.minor_comments (App. A pseudocode: the compact ring addressed by logical
position).  Unwritten ring slots hold NaN, so a stale or skipped row shows up.
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


def _nan_ring(B, Hkv, C, kv8):
    if kv8:
        return torch.full((B, Hkv, C, D), 0x7F, dtype=torch.uint8, device="cuda")
    return torch.from_numpy(np.full((B, Hkv, C, D), gen.BF16_NAN, np.uint16).view(np.int16)).view(
        torch.bfloat16).cuda()


def _tokens(rng, B, L, Hkv, kv8):
    """Token-major draft K/V rows [B, L, Hkv, D]: bf16 bits, or E4M3 codes of N(0, 2^2)."""
    if kv8:
        k = gen.e4m3_codes(rng.standard_normal((B, L, Hkv, D)) * 2.0)
        v = gen.e4m3_codes(rng.standard_normal((B, L, Hkv, D)) * 2.0)
        return k, v
    return gen.kv_pair_bf16(rng, (B, L, Hkv, D))


def _dev(x, kv8):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda() if kv8 else to_dev_bf16(x)


def _append(kv8, *args):
    (api.ring_kv_append_fp8 if kv8 else api.ring_kv_append)(*args)


@pytest.mark.parametrize("lens,Hq,Hkv,s,W,C,steps,n_new,kv8", [
    ([20000], 32, 4, 4, 4092, 4096, 5, 1, False),      # the 1M workload's draft forward shape, wrapped
    ([2049, 2100, 2303], 16, 2, 4, 252, 256, 8, 1, False),   # ragged, wrap points at different slots
    ([900, 2500], 32, 4, 4, 252, 260, 4, 4, False),    # context pass: 4 new rows and 4 queries, slack 4
    ([600], 64, 8, 4, 1020, 1024, 3, 6, False),        # 6 queries x 8 heads = 48 rows
    ([10], 8, 2, 0, 1000, 1024, 20, 1, False),         # no sink, growing from a short context
    ([1, 2], 8, 2, 4, 252, 256, 6, 1, False),          # first rows land in the sink slots
    ([3000], 16, 2, 4, 1020, 1024, 4, 1, True),        # fp8 (E4M3) ring
    ([700, 1500], 32, 4, 4, 252, 260, 3, 4, True),     # fp8 context pass
    # one unit with a window of 1041 tiles: the call takes the stream-K path (append kernel, then
    # attention and LSE merge over every SM) instead of the cluster kernel
    ([70000], 8, 1, 4, 66556, 66560, 3, 1, False),
    ([70000], 8, 1, 4, 66556, 66560, 2, 1, True),
])
def test_fused_forward_sequence(lens, Hq, Hkv, s, W, C, steps, n_new, kv8):
    sc = 128 ** -0.5
    KS, VS = 0.37, 1.9
    rng = np.random.default_rng(sum(lens) + steps)
    B = len(lens)
    n_q = n_new
    L_end = max(lens) + steps * n_new
    k_tok, v_tok = _tokens(rng, B, L_end, Hkv, kv8)
    # two rings: A takes the fused calls, B the separate append (the reference ring)
    ring = {x: (_nan_ring(B, Hkv, C, kv8), _nan_ring(B, Hkv, C, kv8)) for x in "AB"}
    rlen = {x: torch.zeros(B, dtype=torch.int64, device="cuda") for x in "AB"}
    for x in "AB":
        for b in range(B):
            _append(kv8, ring[x][0][b:b + 1], ring[x][1][b:b + 1], rlen[x][b:b + 1],
                    _dev(k_tok[b:b + 1, :lens[b]], kv8), _dev(v_tok[b:b + 1, :lens[b]], kv8), s)
    ws = api.alloc_workspace(B, n_q, Hq, Hkv)
    cur = list(lens)
    for step in range(steps):
        # new rows of request b: positions cur[b] .. cur[b] + n_new
        kn = np.stack([k_tok[b, cur[b]:cur[b] + n_new] for b in range(B)])
        vn = np.stack([v_tok[b, cur[b]:cur[b] + n_new] for b in range(B)])
        q_bits = gen.normal_bf16(rng, (B, n_q, Hq, D))
        q = to_dev_bf16(q_bits)
        if kv8:
            out, lse = api.draft_attn_window_append_fp8(q, ring["A"][0], ring["A"][1], rlen["A"],
                                                        _dev(kn, kv8), _dev(vn, kv8), s, W, sc, KS, VS, ws)
        else:
            out, lse = api.draft_attn_window_append(q, ring["A"][0], ring["A"][1], rlen["A"],
                                                    _dev(kn, kv8), _dev(vn, kv8), s, W, sc, ws)
        _append(kv8, ring["B"][0], ring["B"][1], rlen["B"], _dev(kn, kv8), _dev(vn, kv8), s)
        torch.cuda.synchronize()
        assert api.device_status() == 0
        cur = [L + n_new for L in cur]
        assert rlen["A"].cpu().tolist() == cur == rlen["B"].cpu().tolist()
        for t in range(2):
            assert torch.equal(ring["A"][t].view(torch.uint8), ring["B"][t].view(torch.uint8)), \
                f"step {step}: ring {'KV'[t]} differs from ring_kv_append's"
        assert int(ws[:256].count_nonzero()) == 0          # the control block is left zero
        k_lin = np.zeros((B, Hkv, max(cur), D), k_tok.dtype)
        v_lin = np.zeros_like(k_lin)
        for b in range(B):
            k_lin[b, :, :cur[b]] = np.transpose(k_tok[b, :cur[b]], (1, 0, 2))
            v_lin[b, :, :cur[b]] = np.transpose(v_tok[b, :cur[b]], (1, 0, 2))
        if kv8:
            ref, ref_lse = oracle.attention_kv8(q_bits, k_lin, v_lin, np.array(cur, np.int64),
                                                oracle.MODE_WINDOW, sc, KS, VS, n_sink=s, window=W)
        else:
            ref, ref_lse = oracle.attention(q_bits, k_lin, v_lin, np.array(cur, np.int64),
                                            oracle.MODE_WINDOW, sc, n_sink=s, window=W)
        assert_attn_close(to_f64(out), ref, f"fused forward, step {step}")
        assert_lse_close(lse.cpu().numpy(), ref_lse)


def test_more_new_rows_than_the_window():
    """n_new > W: the rows outside the key set still land in the ring (the call appends as its
    own kernel first), and the attention is that of the oracle."""
    sc = 128 ** -0.5
    rng = np.random.default_rng(41)
    B, Hq, Hkv, s, W, C, L0, n_new = 1, 8, 2, 4, 60, 72, 100, 90
    k_tok, v_tok = gen.kv_pair_bf16(rng, (B, L0 + n_new, Hkv, D))
    rings = [(_nan_ring(B, Hkv, C, False), _nan_ring(B, Hkv, C, False)) for _ in range(2)]
    rl = [torch.zeros(B, dtype=torch.int64, device="cuda") for _ in range(2)]
    for i in range(2):
        api.ring_kv_append(rings[i][0], rings[i][1], rl[i], to_dev_bf16(k_tok[:, :L0]), to_dev_bf16(v_tok[:, :L0]), s)
    n_q = 2                                            # queries at the last two positions
    q_bits = gen.normal_bf16(rng, (B, n_q, Hq, D))
    ws = api.alloc_workspace(B, n_q, Hq, Hkv)
    kn, vn = to_dev_bf16(k_tok[:, L0:]), to_dev_bf16(v_tok[:, L0:])
    out, lse = api.draft_attn_window_append(to_dev_bf16(q_bits), rings[0][0], rings[0][1], rl[0], kn, vn, s, W,
                                            sc, ws)
    api.ring_kv_append(rings[1][0], rings[1][1], rl[1], kn, vn, s)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    assert torch.equal(rl[0], rl[1]) and int(rl[0][0]) == L0 + n_new
    for t in range(2):
        assert torch.equal(rings[0][t].view(torch.uint8), rings[1][t].view(torch.uint8))
    k_lin = np.ascontiguousarray(np.transpose(k_tok, (0, 2, 1, 3)))
    v_lin = np.ascontiguousarray(np.transpose(v_tok, (0, 2, 1, 3)))
    ref, ref_lse = oracle.attention(q_bits, k_lin, v_lin, np.array([L0 + n_new]), oracle.MODE_WINDOW, sc,
                                    n_sink=s, window=W)
    assert_attn_close(to_f64(out), ref, "n_new > W")
    assert_lse_close(lse.cpu().numpy(), ref_lse)


def test_fused_forwards_in_a_cuda_graph():
    """Three fused forwards captured once and replayed: each replay appends three more rows (the
    lengths live on the device) and matches eager calls on a twin ring."""
    sc = 128 ** -0.5
    rng = np.random.default_rng(43)
    B, Hq, Hkv, s, W, C, L0 = 2, 32, 4, 4, 252, 256, 1000
    k_tok, v_tok = gen.kv_pair_bf16(rng, (B, L0 + 64, Hkv, D))
    rings = [(_nan_ring(B, Hkv, C, False), _nan_ring(B, Hkv, C, False)) for _ in range(2)]
    rl = [torch.zeros(B, dtype=torch.int64, device="cuda") for _ in range(2)]
    for i in range(2):
        api.ring_kv_append(rings[i][0], rings[i][1], rl[i], to_dev_bf16(k_tok[:, :L0]), to_dev_bf16(v_tok[:, :L0]), s)
    ws = [api.alloc_workspace(B, 1, Hq, Hkv) for _ in range(2)]
    kn = torch.empty((3, B, 1, Hkv, D), dtype=torch.bfloat16, device="cuda")
    vn = torch.empty_like(kn)
    q = torch.empty((3, B, 1, Hq, D), dtype=torch.bfloat16, device="cuda")
    outs = [torch.empty((B, 1, Hq, D), dtype=torch.bfloat16, device="cuda") for _ in range(2)]

    def fwd(i, j):
        api.draft_attn_window_append(q[j], rings[i][0], rings[i][1], rl[i], kn[j], vn[j], s, W, sc, ws[i],
                                     out=outs[i], want_lse=False)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for j in range(3):
                fwd(0, j)
    torch.cuda.current_stream().wait_stream(side)
    pos = L0
    for rep in range(4):
        for j in range(3):
            kn[j].copy_(to_dev_bf16(k_tok[:, pos + j:pos + j + 1]))
            vn[j].copy_(to_dev_bf16(v_tok[:, pos + j:pos + j + 1]))
            q[j].copy_(to_dev_bf16(gen.normal_bf16(rng, (B, 1, Hq, D))))
        g.replay()
        for j in range(3):
            fwd(1, j)
        torch.cuda.synchronize()
        pos += 3
        assert rl[0].cpu().tolist() == [pos, pos] == rl[1].cpu().tolist()
        for t in range(2):
            assert torch.equal(rings[0][t].view(torch.uint8), rings[1][t].view(torch.uint8))
        assert torch.equal(outs[0], outs[1])
    assert api.device_status() == 0
