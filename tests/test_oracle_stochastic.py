"""Pins of the oracle's stochastic (rejection-sampling) acceptance (CPU only).

The rule is the standard speculative-sampling one (Leviathan, Kalman and Matias, ICML 2023;
Chen et al., 2023), which the Windowed-MTP pages invoke for distributional losslessness (AI
field-notes abstract: the target's verified output distribution is preserved; Pith verdict,
referee_report.significance).  Its defining property is that the emitted token is distributed
exactly as the target's distribution p whatever the draft's q.  The oracle takes its
randomness as integers and decides in exact arithmetic, so that property can be checked
EXACTLY: the acceptance is a threshold in u_accept and the resampled token a monotone step
function of u_sample, so binary searches over the oracle as a black box give every region's
measure, and the resulting distribution must equal p up to the rule's 2^-24 / 2^-32 / 2^-40
quantisation.
"""
import numpy as np
import pytest

import oracle

U24 = 1 << 24
U32 = 1 << 32


def _call(p_rows, q_rows, tokens, u_acc, u_s):
    p = np.asarray(p_rows, np.float32)[None]
    q = np.asarray(q_rows, np.float32)[None]
    acc, n = oracle.accept_stochastic(p, q, np.asarray(tokens, np.int32)[None],
                                      np.asarray(u_acc, np.uint32)[None], np.asarray([u_s], np.uint32))
    return [int(x) for x in acc[0, :int(n[0])]]


def _dist(V, rng, sparsity=0.0):
    w = rng.gamma(0.7, size=V)
    if sparsity:
        w[rng.random(V) < sparsity] = 0.0
        if w.sum() == 0:
            w[0] = 1.0
    return (w / w.sum()).astype(np.float32)


def _first_reject_u(f):
    """Smallest u in [0, 2^24] with f(u) False (f is True on a prefix)."""
    lo, hi = 0, U24
    while lo < hi:
        mid = (lo + hi) // 2
        if f(mid):
            lo = mid + 1
        else:
            hi = mid
    return lo


def _sample_measure(f, V):
    """Measure (over u in [0, 2^32)) of each output of a nondecreasing step function f."""
    bounds = []
    for k in range(V + 1):
        lo, hi = 0, U32                       # smallest u with f(u) >= k
        while lo < hi:
            mid = (lo + hi) // 2
            if f(mid) >= k:
                hi = mid
            else:
                lo = mid + 1
        bounds.append(lo)
    bounds.append(U32)
    meas = np.zeros(V)
    for k in range(V):
        meas[k] = (bounds[k + 1] - bounds[k]) / U32
    return meas


def _position_distribution(p_rows, q_rows, prefix_tokens, pos, V, u_prefix):
    """Exact distribution of the token emitted at chain position `pos` (0-based among drafts),
    given that the drafts before it (prefix_tokens) were accepted with u_prefix, summing over
    the draft x ~ q_rows[pos]."""
    n_q = len(q_rows) + 1
    out = np.zeros(V)
    q = np.asarray(q_rows[pos], np.float64)
    for x in range(V):
        if q[x] == 0:
            continue
        toks = [0] + list(prefix_tokens) + [x] + [0] * (n_q - 2 - pos)

        def emitted(u_acc_x, u_s):
            u = list(u_prefix) + [u_acc_x] + [U24 - 1] * (n_q - 2 - pos)
            return _call(p_rows, q_rows, toks, u, u_s)

        # region of acceptance of x: u_acc_x < A
        A = _first_reject_u(lambda u: len(emitted(u, 0)) > pos + 1 and emitted(u, 0)[pos] == x)
        out[x] += q[x] * A / U24
        if A < U24:
            meas = _sample_measure(lambda us: emitted(U24 - 1, us)[pos], V)
            out += q[x] * (1 - A / U24) * meas
    return out


@pytest.mark.parametrize("seed", range(4))
def test_emitted_token_is_distributed_as_the_target(seed):
    rng = np.random.default_rng(seed)
    V = 5
    p = [_dist(V, rng, 0.2 * (seed % 2)), _dist(V, rng)]
    q = [_dist(V, rng, 0.3 * (seed >= 2))]
    got = _position_distribution(p, q, [], 0, V, [])
    assert np.abs(got - p[0]).max() < 2e-6, (got, p[0])


def test_second_position_uses_the_second_rows():
    # gamma = 2: given draft 1 accepted, the token emitted at position 2 follows p[1], and after
    # both drafts are accepted the bonus follows p[2].
    rng = np.random.default_rng(7)
    V = 4
    p = [_dist(V, rng), _dist(V, rng), _dist(V, rng)]
    q = [_dist(V, rng), _dist(V, rng)]
    x1 = int(np.argmax(np.minimum(p[0], q[0])))
    got = _position_distribution(p, q, [x1], 1, V, [0])
    assert np.abs(got - p[1]).max() < 2e-6, (got, p[1])
    x2 = int(np.argmax(np.minimum(p[1], q[1])))
    bonus = _sample_measure(lambda us: _call(p, q, [0, x1, x2], [0, 0], us)[2], V)
    assert np.abs(bonus - p[2]).max() < 1e-6       # p[2] sums to 1 only to float32 rounding


def test_identical_distributions_accept_everything():
    rng = np.random.default_rng(3)
    V, gamma = 16, 4
    for _ in range(50):
        d = [_dist(V, rng) for _ in range(gamma)]
        toks = [0] + [int(rng.choice(V, p=r.astype(np.float64) / r.astype(np.float64).sum())) for r in d]
        u = rng.integers(0, U24, size=gamma)
        out = _call(d + [_dist(V, rng)], d, toks, u, int(rng.integers(0, U32)))
        assert len(out) == gamma + 1 and out[:gamma] == toks[1:]


def test_disjoint_supports_reject_and_resample_from_the_target():
    p = [[0.0, 0.0, 0.25, 0.75], [0.25, 0.25, 0.25, 0.25]]
    q = [[0.5, 0.5, 0.0, 0.0]]
    for u_s, want in ((0, 2), (U32 // 4 - 1, 2), (U32 // 4, 3), (U32 - 1, 3)):
        assert _call(p, q, [9, 1], [0], u_s) == [want]


def test_greedy_limit_one_hot_distributions():
    V = 8
    one = lambda k: [1.0 if i == k else 0.0 for i in range(V)]
    # draft agrees with the target's certain token: accepted, then the bonus
    assert _call([one(3), one(5)], [one(3)], [0, 3], [U24 - 1], 12345) == [3, 5]
    # draft disagrees: rejected, the target's token emitted
    assert _call([one(3), one(5)], [one(6)], [0, 6], [0], 12345) == [3]


def test_acceptance_threshold_is_p_over_q():
    # p(x) / q(x) = 0.3 / 0.6: exactly half of the 24-bit accept values accept
    p = [[0.3, 0.7], [0.5, 0.5]]
    q = [[0.6, 0.4]]
    A = _first_reject_u(lambda u: len(_call(p, q, [1, 0], [u], 0)) == 2)
    assert A == pytest.approx(U24 * (np.float32(0.3) / np.float32(0.6)), abs=1)


def test_zero_residual_falls_back_to_the_target():
    # p = q / 2 (an unnormalised target): a rejection finds no residual mass and draws from p
    q = [[0.25, 0.25, 0.5]]
    p = [[0.125, 0.125, 0.25], [1.0, 0.0, 0.0]]
    meas = _sample_measure(lambda us: _call(p, q, [0, 2], [U24 - 1], us)[0], 3)
    assert np.abs(meas - np.array([0.25, 0.25, 0.5])).max() < 1e-9
