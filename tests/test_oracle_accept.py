"""Pins for the oracle's greedy acceptance (CPU only).

Source: AI field-notes entry for arXiv 2607.21535 (English abstract; lossless by construction:
the target decides every accepted token) and the Pith verdict, pith_extraction.
forward_implications (greedy-exact in exact arithmetic; composes with tree speculation).
"""
import itertools

import numpy as np
import pytest

import oracle
from synthetic import gen
from tests.conftest import read_golden
from tests.lossless_harness import speculative_greedy, target_greedy


def test_hand_worked_chain_examples():
    V = 4
    argmaxes = [2, 0, 3, 1]
    logits = np.zeros((1, 4, V), np.float32)
    for i, a in enumerate(argmaxes):
        logits[0, i, a] = 1.0
    cases = read_golden("accept_examples.txt")
    assert len(cases) == 4
    for row in cases:
        toks = [int(x) for x in row[3:7]]
        n_exp = int(row[8])
        acc_exp = [int(x) for x in row[9:13]]
        acc, n = oracle.accept_greedy(logits, np.array([toks], np.int32))
        assert int(n[0]) == n_exp and list(acc[0]) == acc_exp, row[1]


def test_ties_take_lowest_index():
    rng = np.random.default_rng(0)
    logits = (rng.integers(0, 4, size=(3, 5, 64)) / 4.0).astype(np.float32)   # 4 levels
    tokens = rng.integers(0, 64, size=(3, 5)).astype(np.int32)
    tokens[:, 1:] = np.argmax(logits[:, :-1], axis=-1)      # all drafts equal np.argmax (first max)
    acc, n = oracle.accept_greedy(logits, tokens)
    assert (n == 5).all()
    assert np.array_equal(acc[:, 4], np.argmax(logits[:, 4], axis=-1))


@pytest.mark.parametrize("gamma", [1, 2, 3])
def test_chain_brute_force_all_drafts(gamma):
    """Every draft sequence over V = 8: the committed tokens are the target's greedy
    continuation, of length 1 + (number of leading drafts that match it)."""
    V, seed, prompt = 8, 42, [1, 5]
    for drafts in itertools.product(range(V), repeat=gamma):
        paths = [prompt + list(drafts[:i]) for i in range(gamma + 1)]
        logits = np.stack([gen.target_logits(seed, p, V) for p in paths])[None]
        toks = np.array([[prompt[-1]] + list(drafts)], np.int32)
        acc, n = oracle.accept_greedy(logits, toks)
        truth = target_greedy(seed, prompt, gamma + 1, V)
        lead = 0
        while lead < gamma and drafts[lead] == truth[lead]:
            lead += 1
        assert int(n[0]) == lead + 1
        assert list(acc[0, :lead + 1]) == truth[:lead + 1]
        assert all(x == -1 for x in acc[0, lead + 1:])


@pytest.mark.parametrize("gamma", [1, 3, 5, 7])
def test_all_wrong_accepts_one_all_right_accepts_gamma_plus_one(gamma):
    V, seed = 32, 5
    _, counts = speculative_greedy(seed, [3], 40, V, gamma, "adversarial", _oracle_accept)
    assert set(counts) == {1}
    _, counts = speculative_greedy(seed, [3], 40, V, gamma, "correct", _oracle_accept)
    assert all(c == gamma + 1 for c in counts[:-1])


def _oracle_accept(logits, tokens, parent):
    return oracle.accept_greedy(logits, tokens, parent)


@pytest.mark.parametrize("policy", ["random", "correct", "adversarial", "correct-then-wrong"])
@pytest.mark.parametrize("gamma", [1, 3, 7])
def test_lossless_chain(policy, gamma):
    V, seed, prompt, n = 16, 11, [2, 7, 1], 60
    spec, _ = speculative_greedy(seed, prompt, n, V, gamma, policy, _oracle_accept, n_correct=2)
    assert spec == target_greedy(seed, prompt, n, V)


@pytest.mark.parametrize("policy", ["random", "correct", "adversarial", "correct-then-wrong"])
@pytest.mark.parametrize("tree_seed", [3, 4])
def test_lossless_tree(policy, tree_seed):
    V, seed, prompt, n = 16, 13, [4], 60
    parent = gen.draft_tree(np.random.default_rng(tree_seed), 8)
    spec, counts = speculative_greedy(seed, prompt, n, V, 0, policy, _oracle_accept,
                                      tree_parent=parent, n_correct=3)
    assert spec == target_greedy(seed, prompt, n, V)
    if policy == "correct":
        assert max(counts) == 4                      # the chain nodes 0..3 give depth 3 + bonus


def test_tree_brute_force_small_vocab():
    """All 3^7 token assignments of a fixed 8-node tree, V = 3: the emitted tokens are the greedy
    continuation, and the walk length equals 1 + the depth of the deepest node whose root path
    matches that continuation, taking the lowest-index child at every step."""
    V, seed, prompt = 3, 9, [0, 2]
    parent = gen.draft_tree(np.random.default_rng(3), 8)
    truth = target_greedy(seed, prompt, 5, V)
    for assign in itertools.product(range(V), repeat=7):
        toks = [prompt[-1]] + list(assign)
        paths = [list(prompt)]
        for i in range(1, 8):
            paths.append(paths[parent[i]] + [toks[i]])
        logits = np.stack([gen.target_logits(seed, p, V) for p in paths])[None]
        acc, n = oracle.accept_greedy(logits, np.array([toks], np.int32), parent[None])
        k = int(n[0])
        assert list(acc[0, :k]) == truth[:k]
        # brute force walk: at each depth the lowest-index matching child
        cur, depth = 0, 0
        while True:
            kids = [c for c in range(1, 8) if parent[c] == cur and toks[c] == truth[depth]]
            if not kids:
                break
            cur, depth = min(kids), depth + 1
        assert k == depth + 1
