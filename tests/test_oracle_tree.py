"""Pins for the oracle's verify key sets, chain and tree (CPU only).

Source: Pith verdict on arXiv 2607.21535, pith_extraction.key_machinery (the target verifies
with full attention, untouched by windowing) and forward_implications (windowing composes with
tree-shaped speculation).  Node i of a verify step sits at cache position L + i; it sees the
committed prefix [0, L) and the nodes on its own root path.
"""
import numpy as np
import pytest

import oracle
from synthetic import gen


def _ancestors_by_dfs(parent):
    """Independent brute force: root paths via a DFS from the root over child lists."""
    n = len(parent)
    children = {i: [c for c in range(n) if parent[c] == i] for i in range(n)}
    paths = {}
    stack = [(0, [0])]
    while stack:
        node, path = stack.pop()
        paths[node] = set(path)
        for c in children[node]:
            stack.append((c, path + [c]))
    return paths


@pytest.mark.parametrize("seed", range(6))
def test_tree_visibility_brute_force(seed):
    parent = gen.draft_tree(np.random.default_rng(seed), 8)
    paths = _ancestors_by_dfs(parent)
    assert len(paths) == 8
    for i in range(8):
        for j in range(8):
            assert oracle.tree_visible(parent, i, j) == (j in paths[i])


@pytest.mark.parametrize("seed", range(20))
def test_tree_generator_shape(seed):
    parent = gen.draft_tree(np.random.default_rng(seed), 8)
    assert parent[0] == -1 and list(parent[1:4]) == [0, 1, 2]
    assert all(parent[i] < i for i in range(1, 8))
    counts = np.bincount(parent[1:], minlength=8)
    assert counts.max() <= 2
    depth = [0] * 8
    for i in range(1, 8):
        depth[i] = depth[parent[i]] + 1
    assert max(depth) == 3                       # four levels ("depth 4")


def _case(seed, n_q, L, Hq=4, Hkv=2, D=16, B=1):
    rng = np.random.default_rng(seed)
    q = gen.normal_bf16(rng, (B, n_q, Hq, D))
    k, v = gen.kv_pair_bf16(rng, (B, Hkv, L + n_q, D))
    return q, k, v


def test_chain_tree_equals_causal():
    n_q, L = 6, 25
    q, k, v = _case(1, n_q, L)
    chain = gen.chain_parents(n_q)[None]
    ot, lt = oracle.attention(q, k, v, np.array([L + n_q]), oracle.MODE_TREE, 0.3, tree_parent=chain)
    oc, lc = oracle.attention(q, k, v, np.array([L + n_q]), oracle.MODE_CAUSAL, 0.3)
    assert np.array_equal(ot, oc) and np.array_equal(lt, lc)


@pytest.mark.parametrize("seed", [0, 3, 7])
def test_tree_node_equals_chain_along_root_path(seed):
    """Closed-form decomposition: node i's output equals the last query of a chain verify whose
    in-step keys are exactly the nodes on i's root path."""
    n_q, L = 8, 19
    q, k, v = _case(seed, n_q, L)
    parent = gen.draft_tree(np.random.default_rng(seed), n_q)
    ot, lt = oracle.attention(q, k, v, np.array([L + n_q]), oracle.MODE_TREE, 0.25,
                              tree_parent=parent[None])
    for i in range(n_q):
        path = []
        c = i
        while c >= 0:
            path.append(c)
            c = parent[c]
        path = path[::-1]
        keep = list(range(L)) + [L + j for j in path]
        qc = q[:, path]
        oc, lc = oracle.attention(qc, k[:, :, keep], v[:, :, keep], np.array([len(keep)]),
                                  oracle.MODE_CAUSAL, 0.25)
        np.testing.assert_allclose(ot[:, i], oc[:, -1], rtol=0, atol=1e-14)
        np.testing.assert_allclose(lt[:, i], lc[:, -1], rtol=0, atol=1e-14)
