"""GPU parity of the three attention calls through the C ABI against the fp64 oracle.

Sources: Pith verdict on arXiv 2607.21535, pith_extraction.key_machinery (draft window = first
n_sink plus last W tokens of the per-request KV index; the verifier keeps full attention) and
forward_implications (tree-shaped speculation); AI field-notes abstract (native draft = full
attention over the whole KV cache).  Sizes span several tiles, ragged tails, several splits and
units finished inside one CTA; pool page tails and unwritten ring slots hold NaN, so any stray
read shows up.
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


def paged_case(seed, lens, Hq, Hkv, n_q, k_scale=1.0, outlier_p=0.0):
    rng = np.random.default_rng(seed)
    B, Lmax = len(lens), max(max(lens), 1)
    q = gen.normal_bf16(rng, (B, n_q, Hq, D))
    k_lin, v_lin = gen.kv_pair_bf16(rng, (B, Hkv, Lmax, D), k_scale=k_scale, outlier_p=outlier_p)
    table = gen.page_table(rng, lens, 64, max_pages=max(1, (Lmax + 63) // 64))
    if gen.n_pages(lens, 64) == 0:
        table[:] = 0
    kp = gen.paginate(k_lin, lens, table, 64)
    vp = gen.paginate(v_lin, lens, table, 64)
    if kp.shape[0] == 0:
        kp = np.full((1, Hkv, 64, D), gen.BF16_NAN, np.uint16)
        vp = kp.copy()
    return dict(q=q, k=k_lin, v=v_lin, kp=kp, vp=vp, table=table, lens=np.asarray(lens, np.int64))


def run_paged(c, fn, sm_scale, tree=None):
    B, n_q, Hq, _ = c["q"].shape
    Hkv = c["k"].shape[1]
    ws = api.alloc_workspace(B, n_q, Hq, Hkv)
    args = (to_dev_bf16(c["q"]), to_dev_bf16(c["kp"]), to_dev_bf16(c["vp"]),
            torch.from_numpy(c["table"]).cuda(), torch.from_numpy(c["lens"].astype(np.int32)).cuda())
    if fn == "verify":
        t = None if tree is None else torch.from_numpy(np.ascontiguousarray(tree, np.int32)).cuda()
        out, lse = api.verify_attn(*args, sm_scale, ws, tree_parent=t)
    else:
        out, lse = api.draft_attn_full(*args, sm_scale, ws)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return to_f64(out), lse.cpu().numpy()


@pytest.mark.parametrize("lens,Hq,Hkv,n_q", [
    ([2048], 8, 2, 1), ([2048], 8, 2, 4),                   # the tiny workload's shapes
    ([1, 63, 64, 65], 16, 2, 1), ([130, 1000, 4097, 7], 16, 2, 3),
    ([777, 3000], 8, 8, 2),                                 # G = 1
    ([1500], 32, 2, 1),                                     # G = 16
    ([64] * 40, 8, 2, 1),                                   # many units finished inside a CTA
])
def test_draft_full_matches_oracle(lens, Hq, Hkv, n_q):
    sc = 128 ** -0.5
    c = paged_case(1, lens, Hq, Hkv, n_q)
    out, lse = run_paged(c, "full", sc)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_CAUSAL, sc)
    assert_attn_close(out, ref, "draft_attn_full")
    assert_lse_close(lse, ref_lse, "draft_attn_full lse")


def test_tiny_workload_scaled_keys():
    """K scaled by 1/sqrt(128) before rounding and sm_scale = 1 (the tiny workload's recipe)."""
    c = paged_case(0, [2048], 8, 2, 4, k_scale=128 ** -0.5)
    out, lse = run_paged(c, "full", 1.0)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_CAUSAL, 1.0)
    assert_attn_close(out, ref)
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("L,n_q,Hq,Hkv", [
    (2048, 4, 8, 2), (5000, 4, 32, 4), (3000, 8, 32, 4), (2500, 6, 64, 8), (1000, 16, 32, 4),
    (300, 2, 8, 1),
])
def test_verify_chain_matches_oracle(L, n_q, Hq, Hkv):
    sc = 128 ** -0.5
    c = paged_case(2, [L + n_q], Hq, Hkv, n_q)
    out, lse = run_paged(c, "verify", sc)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_CAUSAL, sc)
    assert_attn_close(out, ref, "verify chain")
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("n_q", [4, 8])
def test_verify_many_ragged_requests(n_q):
    """Twenty requests of ragged lengths (more than the kernels' early L2 prefetch plans for):
    32-row units on the mma.sync kernel, 64-row units on the tcgen05 kernel, units split over
    several CTAs and units finished inside one."""
    sc = 128 ** -0.5
    rng = np.random.default_rng(11)
    lens = [int(x) + n_q for x in rng.integers(1, 3000, size=20)]
    c = paged_case(3, lens, 32, 4, n_q)
    out, lse = run_paged(c, "verify", sc)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_CAUSAL, sc)
    assert_attn_close(out, ref, "verify, 20 ragged requests")
    assert_lse_close(lse, ref_lse)


def test_verify_tree_matches_oracle():
    sc = 128 ** -0.5
    lens_committed = [3000, 1234, 777]
    n_q = 8
    c = paged_case(3, [L + n_q for L in lens_committed], 32, 4, n_q, outlier_p=0.01)
    rng = np.random.default_rng(3)
    tree = np.stack([gen.draft_tree(rng, n_q) for _ in lens_committed])
    out, lse = run_paged(c, "verify", sc, tree=tree)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_TREE, sc,
                                    tree_parent=tree)
    assert_attn_close(out, ref, "verify tree")
    assert_lse_close(lse, ref_lse)
    # a chain passed as a tree equals the chain call
    chain = np.tile(gen.chain_parents(n_q), (3, 1))
    o1, _ = run_paged(c, "verify", sc, tree=chain)
    o2, _ = run_paged(c, "verify", sc, tree=None)
    assert np.array_equal(o1, o2)


def test_page_table_permutation_invariance_bit_exact():
    sc = 128 ** -0.5
    c1 = paged_case(4, [9000, 4321], 32, 4, 4)
    rng = np.random.default_rng(99)
    table2 = gen.page_table(rng, list(c1["lens"]), 64, max_pages=c1["table"].shape[1])
    c2 = dict(c1, table=table2, kp=gen.paginate(c1["k"], c1["lens"], table2, 64),
              vp=gen.paginate(c1["v"], c1["lens"], table2, 64))
    o1, l1 = run_paged(c1, "verify", sc)
    o2, l2 = run_paged(c2, "verify", sc)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_empty_and_short_sequences():
    """kv_len 0 gives out 0 / lse -inf; kv_len < n_q leaves the early queries with no keys."""
    sc = 0.1
    c = paged_case(5, [0, 2, 70], 8, 2, 4)
    out, lse = run_paged(c, "full", sc)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_CAUSAL, sc)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert_attn_close(out, ref)
    assert_lse_close(lse, ref_lse)


def test_bad_page_id_sets_status_and_skips_tile():
    sc = 128 ** -0.5
    c = paged_case(6, [640, 640], 8, 2, 1)
    bad = c["table"].copy()
    bad[1, 3] = 10 ** 6                                  # out of range for request 1 only
    B, n_q, Hq, _ = c["q"].shape
    ws = api.alloc_workspace(B, n_q, Hq, 2)
    out, _ = api.draft_attn_full(to_dev_bf16(c["q"]), to_dev_bf16(c["kp"]), to_dev_bf16(c["vp"]),
                                 torch.from_numpy(bad).cuda(),
                                 torch.from_numpy(c["lens"].astype(np.int32)).cuda(), sc, ws)
    assert api.device_status() == -6
    assert api.device_status() == 0                      # read-and-clear
    ref, _ = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_CAUSAL, sc)
    assert_attn_close(to_f64(out)[:1], ref[:1])          # request 0 unaffected
    assert not np.isnan(to_f64(out)).any()


# ------------------------------------------------------------------------------ windowed draft
def ring_case(seed, lens, Hq, Hkv, n_q, s, W, C, chunked=False):
    """Draft KV of every request appended into NaN-initialised rings by the library itself."""
    rng = np.random.default_rng(seed)
    B, Lmax = len(lens), max(lens)
    q = gen.normal_bf16(rng, (B, n_q, Hq, D))
    k_tok, v_tok = gen.kv_pair_bf16(rng, (B, Lmax, Hkv, D))         # token-major, as appended
    ring_k = torch.from_numpy(np.full((B, Hkv, C, D), gen.BF16_NAN, np.uint16).view(np.int16)).view(
        torch.bfloat16).cuda()
    ring_v = ring_k.clone()
    rlen = torch.zeros(B, dtype=torch.int64, device="cuda")
    # equal-length requests share appends; ragged ones are appended one request at a time
    for b in range(B):
        kb, vb = to_dev_bf16(k_tok[b:b + 1, :lens[b]]), to_dev_bf16(v_tok[b:b + 1, :lens[b]])
        rk, rv, rl = ring_k[b:b + 1], ring_v[b:b + 1], rlen[b:b + 1]
        if chunked:
            off = 0
            for n in ([lens[b] - 7, 1, 1, 5] if lens[b] > 7 else [lens[b]]):
                api.ring_kv_append(rk, rv, rl, kb[:, off:off + n].contiguous(), vb[:, off:off + n].contiguous(), s)
                off += n
        else:
            api.ring_kv_append(rk, rv, rl, kb, vb, s)
    k_lin = np.ascontiguousarray(np.transpose(k_tok, (0, 2, 1, 3)))
    v_lin = np.ascontiguousarray(np.transpose(v_tok, (0, 2, 1, 3)))
    return dict(q=q, k=k_lin, v=v_lin, ring_k=ring_k, ring_v=ring_v, rlen=rlen,
                lens=np.asarray(lens, np.int64), s=s, W=W)


def run_window(c, sm_scale):
    B, n_q, Hq, _ = c["q"].shape
    Hkv = c["k"].shape[1]
    ws = api.alloc_workspace(B, n_q, Hq, Hkv)
    out, lse = api.draft_attn_window(to_dev_bf16(c["q"]), c["ring_k"], c["ring_v"], c["rlen"],
                                     c["s"], c["W"], sm_scale, ws)
    torch.cuda.synchronize()
    assert api.device_status() == 0
    return to_f64(out), lse.cpu().numpy()


@pytest.mark.parametrize("lens,Hq,Hkv,n_q,s,W,C", [
    ([2048], 8, 2, 1, 4, 252, 256),            # the tiny workload's windowed draft
    ([2048], 8, 2, 4, 4, 252, 256),
    ([2049, 2100, 2303], 16, 2, 1, 4, 252, 256),   # wrap point at different slots
    ([20000], 32, 4, 1, 4, 4092, 4096),
    ([9000], 32, 4, 4, 4, 4092, 4100),         # slack d = 4: the ring holds more than the window
    ([5000, 300], 16, 2, 3, 0, 1000, 1024),    # no sink
    ([100, 3, 257], 8, 2, 1, 4, 252, 256),     # shorter than the window
    ([600], 64, 8, 6, 4, 1020, 1024),
])
def test_draft_window_matches_oracle(lens, Hq, Hkv, n_q, s, W, C):
    sc = 128 ** -0.5
    c = ring_case(7, lens, Hq, Hkv, n_q, s, W, C, chunked=(n_q == 1))
    out, lse = run_window(c, sc)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_WINDOW, sc,
                                    n_sink=s, window=W)
    assert_attn_close(out, ref, "draft_attn_window")
    assert_lse_close(lse, ref_lse)


@pytest.mark.parametrize("W", [124, 316, 636, 1276, 2556])
@pytest.mark.parametrize("n_q", [1, 4, 8])
def test_window_every_cluster_size(W, n_q):
    """Windows of 2, 5, 10, 20 and 40 tiles: the cluster window kernel runs with clusters of 1, 2,
    4, 8 and 16 CTAs per unit (the largest size that leaves each CTA at least two tiles), each
    merging its partials through distributed shared memory; 8, 32 and 64 rows per unit (its
    three layouts); wrapped rings, ragged last tiles."""
    sc = 128 ** -0.5
    s = 4
    lens = [3 * (s + W) + 37, 2 * (s + W) + 5]
    c = ring_case(11 + W, lens, 32, 4, n_q, s, W, s + W)
    out, lse = run_window(c, sc)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_WINDOW, sc,
                                    n_sink=s, window=W)
    assert_attn_close(out, ref, "draft_attn_window")
    assert_lse_close(lse, ref_lse)


def test_window_covering_context_equals_full():
    """s + W >= L: the windowed call equals the full call (both vs the oracle, and each other)."""
    sc = 128 ** -0.5
    lens, n_q = [900, 1700], 2
    cw = ring_case(8, lens, 16, 2, n_q, 4, 2044, 2048)
    rng = np.random.default_rng(8)
    table = gen.page_table(rng, lens, 64)
    cp = dict(q=cw["q"], k=cw["k"], v=cw["v"], table=table, lens=cw["lens"],
              kp=gen.paginate(cw["k"], lens, table, 64), vp=gen.paginate(cw["v"], lens, table, 64))
    ow, lw = run_window(cw, sc)
    of, lf = run_paged(cp, "full", sc)
    ref, _ = oracle.attention(cw["q"], cw["k"], cw["v"], cw["lens"], oracle.MODE_CAUSAL, sc)
    assert_attn_close(ow, ref)
    assert_attn_close(of, ref)
    assert np.abs(ow - of).max() <= 1e-2


def test_graph_replays_match_eager_calls():
    """The attention calls captured once in a CUDA graph and replayed (each replay finds the
    previous replay's partials in the workspace) give the eager results every time."""
    sc = 128 ** -0.5
    c = paged_case(9, [7000, 3000], 32, 4, 4)
    cw = ring_case(10, [9000, 5000], 32, 4, 1, 4, 4092, 4096)
    B, n_q, Hq, _ = c["q"].shape
    ws = api.alloc_workspace(B, n_q, Hq, 4)
    args = (to_dev_bf16(c["q"]), to_dev_bf16(c["kp"]), to_dev_bf16(c["vp"]),
            torch.from_numpy(c["table"]).cuda(), torch.from_numpy(c["lens"].astype(np.int32)).cuda())
    qw = to_dev_bf16(cw["q"])
    ov, lv = torch.empty_like(args[0]), torch.empty(args[0].shape[:3], dtype=torch.float32, device="cuda")
    ow, lw = torch.empty_like(qw), torch.empty(qw.shape[:3], dtype=torch.float32, device="cuda")

    def calls():
        api.verify_attn(*args, sc, ws, out=ov, lse=lv)
        api.draft_attn_window(qw, cw["ring_k"], cw["ring_v"], cw["rlen"], 4, 4092, sc, ws, out=ow, lse=lw)

    calls()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (ov, lv, ow, lw)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        calls()                                   # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        calls()
    for _ in range(3):
        for t in (ov, lv, ow, lw):
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        for t, r in zip((ov, lv, ow, lw), ref):
            assert torch.equal(t, r)
    assert api.device_status() == 0


@pytest.mark.parametrize("n_q,Hq,Hkv,tree", [(8, 32, 4, False), (8, 32, 4, True), (6, 64, 8, False),
                                             (4, 32, 4, False), (1, 32, 4, False)])
def test_rising_scores_move_the_running_maximum(n_q, Hq, Hkv, tree):
    """Scores that grow along the context move every row's running maximum many times (the
    kernels' rescale paths, which random N(0, 1) inputs rarely reach)."""
    sc = 128 ** -0.5
    rng = np.random.default_rng(21)
    L = 5000 + n_q
    rise = np.linspace(0.0, 20.0, L, dtype=np.float32)[None, None, :, None]
    q = gen.bf16_bits(0.2 + 0.05 * rng.standard_normal((1, n_q, Hq, D), dtype=np.float32))
    k = gen.bf16_bits(rise + 0.3 * rng.standard_normal((1, Hkv, L, D), dtype=np.float32))
    v = gen.normal_bf16(rng, (1, Hkv, L, D))
    table = gen.page_table(rng, [L], 64)
    c = dict(q=q, k=k, v=v, table=table, lens=np.array([L], np.int64),
             kp=gen.paginate(k, [L], table, 64), vp=gen.paginate(v, [L], table, 64))
    parent = gen.draft_tree(np.random.default_rng(5), n_q)[None] if tree else None
    out, lse = run_paged(c, "verify", sc, tree=parent)
    mode = oracle.MODE_TREE if tree else oracle.MODE_CAUSAL
    ref, ref_lse = oracle.attention(q, k, v, c["lens"], mode, sc, tree_parent=parent)
    assert_attn_close(out, ref, "rising scores")
    assert_lse_close(lse, ref_lse)


def test_bounded_wait_times_out_and_context_stays_usable():
    """The failure path every kernel wait shares, on purpose: a wait that nothing satisfies gives
    up after its limit, the status word reports WMTP_ERR_TIMEOUT (read and cleared), and the next
    call on the same context still matches the oracle."""
    assert api.device_status() == 0
    api.selftest_wait_timeout(20_000_000)                # 20 ms
    assert api.device_status() == -8                     # WMTP_ERR_TIMEOUT
    assert api.device_status() == 0
    sc = 128 ** -0.5
    c = paged_case(7, [300, 1000], 8, 2, 1)
    out, lse = run_paged(c, "full", sc)
    ref, ref_lse = oracle.attention(c["q"], c["k"], c["v"], c["lens"], oracle.MODE_CAUSAL, sc)
    assert_attn_close(out, ref)
    assert_lse_close(lse, ref_lse)
