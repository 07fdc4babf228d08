"""GPU parity of accept_stochastic (rejection-sampling acceptance) against the oracle, bit for bit.

Sources: AI field-notes abstract for arXiv 2607.21535 (the target's verified output distribution
is preserved); Pith verdict, referee_report.significance (standard speculative-decoding theorem);
the rule itself: Leviathan, Kalman and Matias, ICML 2023; Chen et al., 2023.  Both sides take
every decision in exact arithmetic from the same integer uniforms, so accepted tokens and counts
must be identical.  Inputs: softmax rows of random logits at several temperatures (fp32), drafts
drawn from q on the host, uniforms from a seeded generator; edge cases: no drafts, q = p (all
kept), disjoint supports (first draft always rejected), a large vocabulary, an out-of-range
draft.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_speculative_kv_b200 import api

pytestmark = pytest.mark.gpu


def softmax_rows(rng, shape, temp):
    x = rng.standard_normal(shape) / temp
    x = np.exp(x - x.max(axis=-1, keepdims=True))
    return (x / x.sum(axis=-1, keepdims=True)).astype(np.float32)


def make_case(seed, B, n_q, V, temp_p=1.0, temp_q=1.5, q_equals_p=False, disjoint=False):
    rng = np.random.default_rng(seed)
    p = softmax_rows(rng, (B, n_q, V), temp_p)
    q = p[:, :n_q - 1].copy() if q_equals_p else softmax_rows(rng, (B, n_q - 1, V), temp_q)
    if disjoint:
        half = V // 2
        p[:, :, :half] = 0
        p /= p.sum(axis=-1, keepdims=True)
        q[:, :, half:] = 0
        q /= q.sum(axis=-1, keepdims=True)
        p, q = p.astype(np.float32), q.astype(np.float32)
    tokens = np.zeros((B, n_q), np.int32)
    tokens[:, 0] = rng.integers(0, V, size=B)
    for b in range(B):
        for i in range(1, n_q):
            w = q[b, i - 1].astype(np.float64)
            tokens[b, i] = rng.choice(V, p=w / w.sum())
    u_acc = rng.integers(0, 1 << 24, size=(B, max(n_q - 1, 0)), dtype=np.uint32)
    u_s = rng.integers(0, 1 << 32, size=B, dtype=np.uint64).astype(np.uint32)
    return p, q, tokens, u_acc, u_s


def run_gpu(p, q, tokens, u_acc, u_s):
    dev = torch.device("cuda")
    B, n_q, V = p.shape
    to_i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(dev)
    acc, n = api.accept_stochastic(torch.from_numpy(p).to(dev),
                                   torch.from_numpy(q).to(dev) if n_q > 1 else None,
                                   torch.from_numpy(tokens).to(dev),
                                   to_i32(u_acc) if n_q > 1 else None, to_i32(u_s))
    torch.cuda.synchronize()
    return acc.cpu().numpy(), n.cpu().numpy()


@pytest.mark.parametrize("B,n_q,V,tp,tq", [
    (64, 4, 1024, 1.0, 1.5),       # the workloads' vocabulary, gamma = 3
    (32, 8, 1024, 0.5, 0.7),       # sharper distributions, gamma = 7
    (16, 6, 32000, 1.0, 1.0),      # a large vocabulary (1024-thread draw)
    (7, 64, 13, 2.0, 2.0),         # the longest chain, tiny vocabulary
    (9, 1, 50, 1.0, 1.0),          # no drafts: the bonus draw alone
])
def test_matches_oracle_bit_for_bit(B, n_q, V, tp, tq):
    case = make_case(B * 131 + n_q, B, n_q, V, tp, tq)
    got_acc, got_n = run_gpu(*case)
    assert api.device_status() == 0
    ref_acc, ref_n = oracle.accept_stochastic(*case)
    assert np.array_equal(got_n, ref_n)
    assert np.array_equal(got_acc, ref_acc)
    assert (got_n >= 1).all() and (got_n <= n_q).all()


def test_identical_distributions_keep_every_draft():
    case = make_case(5, 32, 5, 1024, q_equals_p=True)
    got_acc, got_n = run_gpu(*case)
    assert (got_n == 5).all()
    assert np.array_equal(got_acc[:, :4], case[2][:, 1:])
    ref_acc, ref_n = oracle.accept_stochastic(*case)
    assert np.array_equal(got_acc, ref_acc)


def test_disjoint_supports_reject_the_first_draft():
    case = make_case(6, 32, 4, 1024, disjoint=True)
    got_acc, got_n = run_gpu(*case)
    assert (got_n == 1).all()
    assert (got_acc[:, 0] >= 512).all()        # drawn from the target's half
    ref_acc, _ = oracle.accept_stochastic(*case)
    assert np.array_equal(got_acc, ref_acc)


def test_out_of_range_draft_is_rejected_and_flagged():
    p, q, tokens, u_acc, u_s = make_case(8, 4, 4, 256)
    tokens[2, 1] = 999
    got_acc, got_n = run_gpu(p, q, tokens, u_acc, u_s)
    assert api.device_status() == -6            # WMTP_ERR_DEVICE_INDEX
    ref_acc, ref_n = oracle.accept_stochastic(p, q, tokens, u_acc, u_s)
    assert got_n[2] == 1
    assert np.array_equal(got_acc, ref_acc) and np.array_equal(got_n, ref_n)
