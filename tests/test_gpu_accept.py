"""GPU parity: accept_greedy through the C ABI against the oracle, bit-exact, and the lossless
property with the library deciding acceptance.

Source: AI field-notes abstract for arXiv 2607.21535 (the target decides every accepted token;
windowing changes only which tokens are proposed); Pith verdict, pith_extraction.
forward_implications (greedy-exact; composes with tree speculation).
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_speculative_kv_b200 import api
from synthetic import gen
from tests.lossless_harness import speculative_greedy, target_greedy

pytestmark = pytest.mark.gpu


def gpu_accept(logits, tokens, parent):
    acc, n = api.accept_greedy(torch.from_numpy(np.ascontiguousarray(logits)).cuda(),
                               torch.from_numpy(np.ascontiguousarray(tokens, np.int32)).cuda(),
                               None if parent is None else
                               torch.from_numpy(np.ascontiguousarray(parent, np.int32)).cuda())
    return acc.cpu().numpy(), n.cpu().numpy()


@pytest.mark.parametrize("B,n_q,V,levels", [(1, 4, 1024, 0), (8, 8, 1024, 4), (3, 2, 7, 2),
                                            (5, 64, 50, 3), (2, 6, 1024, 0)])
def test_accept_chain_matches_oracle(B, n_q, V, levels):
    rng = np.random.default_rng(B * 100 + n_q)
    logits = gen.uniform_logits(rng, (B, n_q, V))
    if levels:
        logits = (np.floor((logits + 1) * levels / 2) / levels).astype(np.float32)   # ties
    tokens = rng.integers(0, V, size=(B, n_q)).astype(np.int32)
    # make some drafts right so that acceptance runs deep
    am = np.argmax(logits, axis=-1)
    for b in range(B):
        k = int(rng.integers(0, n_q))
        tokens[b, 1:k + 1] = am[b, :k]
    ea, en = oracle.accept_greedy(logits, tokens)
    ga, gn = gpu_accept(logits, tokens, None)
    assert np.array_equal(ga, ea) and np.array_equal(gn, en)


def test_accept_tree_matches_oracle():
    rng = np.random.default_rng(3)
    B, n_q, V = 8, 8, 1024
    parent = np.stack([gen.draft_tree(rng, n_q) for _ in range(B)])
    logits = gen.uniform_logits(rng, (B, n_q, V))
    am = np.argmax(logits, axis=-1)
    tokens = rng.integers(0, V, size=(B, n_q)).astype(np.int32)
    for b in range(B):                 # child token = parent's argmax with probability 1/2
        for i in range(1, n_q):
            if rng.random() < 0.5:
                tokens[b, i] = am[b, parent[b, i]]
    ea, en = oracle.accept_greedy(logits, tokens, parent)
    ga, gn = gpu_accept(logits, tokens, parent)
    assert np.array_equal(ga, ea) and np.array_equal(gn, en)


@pytest.mark.parametrize("policy", ["random", "correct", "adversarial", "correct-then-wrong"])
def test_lossless_with_library_acceptance(policy):
    V, seed, prompt, n = 64, 21, [5, 9], 50
    spec, _ = speculative_greedy(seed, prompt, n, V, 3, policy, gpu_accept, n_correct=2)
    assert spec == target_greedy(seed, prompt, n, V)
    parent = gen.draft_tree(np.random.default_rng(4), 8)
    spec, _ = speculative_greedy(seed, prompt, n, V, 0, policy, gpu_accept, tree_parent=parent,
                                 n_correct=3)
    assert spec == target_greedy(seed, prompt, n, V)
