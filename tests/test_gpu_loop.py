"""GPU parity of the device decode loop (ring rollback, commit, synthetic heads) through the C ABI.

Sources: Pith verdict on arXiv 2607.21535, pith_extraction.key_machinery (Eq. 1's step: draft
context pass, gamma draft forwards, verify) and referee_report.minor_comments (App. A: ring slots
with "+d slack"); AI field-notes abstract (the target decides every accepted token).

Checks, per arm: the committed tokens equal the synthetic target's own greedy sequence and the
per-step accepted counts equal the CPU loop's (oracle acceptance); the ring equals the oracle's
ring after the same appends and rollbacks, byte for byte, and its window slots hold the latest
row of every window position (the slack keeps rolled-back slots out of the window); the last
step's draft and verify attention outputs match the fp64 oracle on the logical sequences.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_speculative_kv_b200 import api
from long_context_speculative_kv_b200.loop import DecodeLoop, LoopState
from long_context_speculative_kv_b200.step import StepBuffers
from synthetic import gen
from tests.gpu_util import assert_attn_close, assert_lse_close, to_bits, to_dev_bf16, to_f64
from tests.lossless_harness import hash_draft_loop, target_greedy

pytestmark = pytest.mark.gpu

D = 128
P = 64


def _accept(logits, tokens, parent):
    return oracle.accept_greedy(logits, tokens, parent)


class Case:
    def __init__(self, seed=5, prompt_lens=(700, 1500), Hq=8, Hkv=2, gamma=3, n_sink=4, window=124,
                 steps=24, n_layers=2, vocab=1024, agree=0.7, slack=None):
        rng = np.random.default_rng(seed)
        self.B, self.Hq, self.Hkv, self.gamma = len(prompt_lens), Hq, Hkv, gamma
        self.n_sink, self.window, self.steps, self.vocab = n_sink, window, steps, vocab
        self.C = n_sink + window + (gamma if slack is None else slack)
        self.tseed, self.dseed = 1000 + seed, 2000 + seed
        self.agree24 = int(round(agree * (1 << 24)))
        self.sm_scale = 128 ** -0.5
        n_q = gamma + 1
        self.prompts = [[int(t) for t in rng.integers(0, vocab, size=T)] for T in prompt_lens]
        self.max_tokens = max(prompt_lens) + n_q * steps + 8
        # target layers: fixed rows per position, paged
        self.lens_v = [T + n_q * (steps + 1) for T in prompt_lens]
        self.table_v = gen.page_table(rng, self.lens_v, P)
        self.kv_lin = [gen.kv_pair_bf16(rng, (self.B, Hkv, max(self.lens_v), D)) for _ in range(n_layers)]
        self.pools = [(gen.paginate(k, self.lens_v, self.table_v, P), gen.paginate(v, self.lens_v, self.table_v, P))
                      for k, v in self.kv_lin]
        # native draft cache: fixed rows per position, paged
        self.lens_d = [T + n_q * (steps + 1) + gamma for T in prompt_lens]
        self.table_d = gen.page_table(rng, self.lens_d, P)
        self.kd_lin, self.vd_lin = gen.kv_pair_bf16(rng, (self.B, Hkv, max(self.lens_d), D))
        self.kd_pool = gen.paginate(self.kd_lin, self.lens_d, self.table_d, P)
        self.vd_pool = gen.paginate(self.vd_lin, self.lens_d, self.table_d, P)
        # windowed draft: prompt rows (positions [0, T0 - 1)), then per-step rows
        self.pre_n = [T - 1 for T in prompt_lens]
        self.k_pre, self.v_pre = gen.kv_pair_bf16(rng, (self.B, max(max(self.pre_n), 1), Hkv, D))
        self.k_ctx, self.v_ctx = gen.kv_pair_bf16(rng, (self.B, n_q, Hkv, D))
        self.k_fwd, self.v_fwd = gen.kv_pair_bf16(rng, (gamma, self.B, 1, Hkv, D))
        self.q_verify = gen.normal_bf16(rng, (n_layers, self.B, n_q, Hq, D))
        self.q_ctx = gen.normal_bf16(rng, (self.B, n_q, Hq, D))
        self.q_fwd = gen.normal_bf16(rng, (gamma, self.B, 1, Hq, D))

    def device_loop(self):
        dev = torch.device("cuda")
        t = lambda a: to_dev_bf16(a)
        ring_k = torch.full((self.B, self.Hkv, self.C, D), float("nan"), dtype=torch.bfloat16, device=dev)
        ring_v = torch.full_like(ring_k, float("nan"))
        ring_len = torch.zeros(self.B, dtype=torch.int64, device=dev)
        api.ring_kv_append_at(ring_k, ring_v, ring_len, t(self.k_pre), t(self.v_pre),
                              torch.zeros(self.B, dtype=torch.int64, device=dev),
                              torch.tensor(self.pre_n, dtype=torch.int32, device=dev), self.n_sink)
        hist = torch.zeros((self.B, self.max_tokens), dtype=torch.int32)
        for b, pr in enumerate(self.prompts):
            hist[b, :len(pr)] = torch.tensor(pr, dtype=torch.int32)
        state = LoopState.start(hist.to(dev), [len(pr) for pr in self.prompts], self.gamma)
        bufs = StepBuffers(
            k_pools=[t(k) for k, _ in self.pools], v_pools=[t(v) for _, v in self.pools],
            table_v=torch.from_numpy(self.table_v).to(dev), kv_len_v=state.verify_len,
            q_verify=t(self.q_verify), tree_parent=None,
            logits=torch.empty(0, device=dev), tokens=torch.empty(0, dtype=torch.int32, device=dev),
            q_ctx=t(self.q_ctx), q_fwd=t(self.q_fwd), k_ctx=t(self.k_ctx), v_ctx=t(self.v_ctx),
            k_fwd=t(self.k_fwd), v_fwd=t(self.v_fwd), ring_k=ring_k, ring_v=ring_v, ring_len=ring_len,
            n_sink=self.n_sink, window=self.window, k_draft=t(self.kd_pool), v_draft=t(self.vd_pool),
            table_d=torch.from_numpy(self.table_d).to(dev), sm_scale=self.sm_scale)
        return DecodeLoop(bufs, self.gamma, state, self.vocab, self.tseed, self.dseed, self.agree24)


def run_steps(case, loop, arm):
    """Runs the steps one by one; returns per-step records for the CPU replay."""
    recs = []
    for _ in range(case.steps):
        s = loop.s
        rec = dict(pos=s.append_pos.cpu().numpy().copy(), n_app=s.n_append.cpu().numpy().copy(),
                   T=s.n_tokens.cpu().numpy().copy())
        loop.step(arm)
        torch.cuda.synchronize()
        rec["n_acc"] = loop.n_accepted.cpu().numpy().copy()
        recs.append(rec)
    assert api.device_status() == 0
    return recs


def check_tokens(case, loop, recs):
    hist = loop.s.history.cpu().numpy()
    T_end = loop.s.n_tokens.cpu().numpy()
    for b, prompt in enumerate(case.prompts):
        seq, counts = hash_draft_loop(case.tseed, case.dseed, prompt, case.steps, case.vocab, case.gamma,
                                      case.agree24, _accept)
        assert [int(r["n_acc"][b]) for r in recs] == counts
        assert T_end[b] == len(prompt) + len(seq)
        got = [int(x) for x in hist[b, len(prompt):T_end[b]]]
        assert got == seq
        assert got == target_greedy(case.tseed, prompt, len(got), case.vocab)
    return T_end


def replay_ring(case, recs):
    """The oracle's ring after the same appends (prefill, then per step: context rows at the
    committed position, gamma forward rows), plus each position's latest row."""
    B, Hkv, C = case.B, case.Hkv, case.C
    rk = np.full((B, Hkv, C, D), gen.BF16_NAN, np.uint16)
    rv = rk.copy()
    latest = [dict() for _ in range(B)]
    for b in range(B):
        def app(pos, k_rows, v_rows):        # k_rows [n, Hkv, D]
            n = k_rows.shape[0]
            if n == 0:
                return
            kb, vb = rk[b:b + 1].copy(), rv[b:b + 1].copy()
            rl = np.array([pos], np.int64)
            oracle.ring_kv_append(kb, vb, rl, k_rows[None], v_rows[None], case.n_sink)
            rk[b:b + 1], rv[b:b + 1] = kb, vb
            for t in range(n):
                latest[b][pos + t] = (k_rows[t], v_rows[t])
        app(0, case.k_pre[b, :case.pre_n[b]], case.v_pre[b, :case.pre_n[b]])
        for r in recs:
            app(int(r["pos"][b]), case.k_ctx[b, :int(r["n_app"][b])], case.v_ctx[b, :int(r["n_app"][b])])
            for j in range(case.gamma):
                app(int(r["T"][b]) + j, case.k_fwd[j, b], case.v_fwd[j, b])
    return rk, rv, latest


def logical(case, latest_b, L):
    k = np.stack([latest_b[p][0] for p in range(L)], axis=1)      # [Hkv, L, D]
    v = np.stack([latest_b[p][1] for p in range(L)], axis=1)
    return k, v


@pytest.mark.parametrize("agree", [0.7, 0.0, 1.0])
def test_windowed_loop_tokens_ring_and_attention(agree):
    case = Case(agree=agree)
    loop = case.device_loop()
    recs = run_steps(case, loop, "windowed")
    check_tokens(case, loop, recs)
    rk, rv, latest = replay_ring(case, recs)
    b_ = loop.b
    assert np.array_equal(to_bits(b_.ring_k), rk)
    assert np.array_equal(to_bits(b_.ring_v), rv)
    # window slots hold the latest row of each window position after the last step's forwards
    ring_len = b_.ring_len.cpu().numpy()
    last = recs[-1]
    for b in range(case.B):
        L = int(ring_len[b])
        assert L == int(last["T"][b]) + case.gamma
        for p in list(range(min(case.n_sink, L))) + list(range(max(case.n_sink, L - case.window), L)):
            slot = oracle.ring_slot(p, case.n_sink, case.C)
            assert np.array_equal(rk[b, :, slot], latest[b][p][0])
    # last step's attention: context pass (L_tot = T) and the last forward (L_tot = T + gamma - 1 + 1)
    Ls_ctx = [int(x) for x in last["T"]]
    Ls_fwd = [L + case.gamma for L in Ls_ctx]
    Lmax = max(Ls_fwd)
    k_log = np.full((case.B, case.Hkv, Lmax, D), gen.BF16_NAN, np.uint16)
    v_log = k_log.copy()
    for b in range(case.B):
        k_log[b, :, :Ls_fwd[b]], v_log[b, :, :Ls_fwd[b]] = logical(case, latest[b], Ls_fwd[b])
    ref, ref_lse = oracle.attention(case.q_ctx, k_log, v_log, np.array(Ls_ctx), oracle.MODE_WINDOW,
                                    case.sm_scale, n_sink=case.n_sink, window=case.window)
    assert_attn_close(to_f64(b_.out["ctx"]), ref, "loop window ctx")
    assert_lse_close(b_.out["ctx_lse"].cpu().numpy(), ref_lse, "loop window ctx lse")
    ref, ref_lse = oracle.attention(case.q_fwd[-1], k_log, v_log, np.array(Ls_fwd), oracle.MODE_WINDOW,
                                    case.sm_scale, n_sink=case.n_sink, window=case.window)
    assert_attn_close(to_f64(b_.out["fwd"]), ref, "loop window fwd")
    # last verify layer: kv_len = T - 1 + n_q over the fixed target rows
    n_q = case.gamma + 1
    Lv = np.array([L - 1 + n_q for L in Ls_ctx])
    kl, vl = case.kv_lin[-1]
    ref, ref_lse = oracle.attention(case.q_verify[-1], kl, vl, Lv, oracle.MODE_CAUSAL, case.sm_scale)
    assert_attn_close(to_f64(b_.out["verify"]), ref, "loop verify")
    assert_lse_close(b_.out["verify_lse"].cpu().numpy(), ref_lse, "loop verify lse")


def test_native_loop_commits_the_same_tokens():
    case = Case(agree=0.7)
    loop = case.device_loop()
    recs = run_steps(case, loop, "native")
    check_tokens(case, loop, recs)
    last = recs[-1]
    Ls_ctx = np.array([int(x) for x in last["T"]])
    ref, _ = oracle.attention(case.q_ctx, case.kd_lin, case.vd_lin, Ls_ctx, oracle.MODE_CAUSAL, case.sm_scale)
    assert_attn_close(to_f64(loop.b.out["ctx"]), ref, "loop full ctx")
    ref, _ = oracle.attention(case.q_fwd[-1], case.kd_lin, case.vd_lin, Ls_ctx + case.gamma,
                              oracle.MODE_CAUSAL, case.sm_scale)
    assert_attn_close(to_f64(loop.b.out["fwd"]), ref, "loop full fwd")


def test_loop_refuses_a_ring_without_rollback_slack():
    """capacity = n_sink + window leaves no room for the gamma rolled-back rows: refused."""
    case = Case(agree=0.0, slack=0, steps=2)
    with pytest.raises(ValueError):
        case.device_loop()


def test_graph_replayed_loop_matches_eager():
    case = Case(agree=0.7, steps=12)
    eager = case.device_loop()
    run_steps(case, eager, "windowed")
    g_loop = case.device_loop()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        g_loop.step("windowed")            # warm-up step (also the first real step)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        g_loop.step("windowed")
    for _ in range(case.steps - 1):
        graph.replay()
    torch.cuda.synchronize()
    assert api.device_status() == 0
    assert torch.equal(g_loop.s.n_tokens, eager.s.n_tokens)
    assert torch.equal(g_loop.s.history, eager.s.history)
    assert np.array_equal(to_bits(g_loop.b.ring_k), to_bits(eager.b.ring_k))
    assert np.array_equal(to_bits(g_loop.b.ring_v), to_bits(eager.b.ring_v))


def test_synthetic_heads_match_the_generators():
    rng = np.random.default_rng(9)
    B, T_max, V, gamma = 5, 300, 1024, 4
    Ts = [1, 2, 3, 150, 300]
    hist = np.zeros((B, T_max), np.int32)
    for b, T in enumerate(Ts):
        hist[b, :T] = rng.integers(0, V, size=T)
    h = torch.from_numpy(hist).cuda()
    nt = torch.tensor(Ts, dtype=torch.int64).cuda()
    toks = api.synth_draft_tokens(h, nt, gamma, V, 77, 78, int(0.5 * (1 << 24)))
    parents = np.stack([gen.draft_tree(rng, gamma + 1) for _ in range(B)]).astype(np.int32)
    lg_chain = api.synth_target_logits(h, nt, toks, V, 77)
    lg_tree = api.synth_target_logits(h, nt, toks, V, 77, tree_parent=torch.from_numpy(parents).cuda())
    torch.cuda.synchronize()
    assert api.device_status() == 0
    toks, lg_chain, lg_tree = toks.cpu().numpy(), lg_chain.cpu().numpy(), lg_tree.cpu().numpy()
    for b, T in enumerate(Ts):
        prefix = [int(x) for x in hist[b, :T]]
        props = gen.hash_draft_tokens(77, 78, prefix, gamma, V, int(0.5 * (1 << 24)))
        assert [int(x) for x in toks[b]] == [prefix[-1]] + props
        for i in range(gamma + 1):
            path = prefix + [int(x) for x in toks[b, 1:i + 1]]
            assert np.array_equal(lg_chain[b, i], gen.target_logits(77, path, V))
            anc, cur = [], i
            while cur > 0:
                anc.append(int(toks[b, cur]))
                cur = int(parents[b, cur])
            assert np.array_equal(lg_tree[b, i], gen.target_logits(77, prefix + anc[::-1], V))
