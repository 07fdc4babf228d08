"""Greedy speculative-decoding loop over a synthetic target, for the lossless property.

Source: AI field-notes entry for arXiv 2607.21535 (English abstract): the full-attention target
decides every accepted token, so windowing the draft changes only which tokens are proposed,
never which are accepted; Pith verdict, pith_extraction.forward_implications (greedy-exact in
exact arithmetic).  The harness runs the same loop for any draft policy and any acceptance
routine (the oracle's on the CPU, the CUDA library's on the GPU) and returns the committed
sequence, to be compared token for token with the target's own greedy sequence.
"""
from typing import Callable, List, Optional

import numpy as np

from synthetic import gen


def target_greedy(seed: int, prompt: List[int], n_tokens: int, vocab: int) -> List[int]:
    seq = list(prompt)
    while len(seq) < len(prompt) + n_tokens:
        seq.append(int(np.argmax(gen.target_logits(seed, seq, vocab))))
    return seq[len(prompt):]


def speculative_greedy(seed: int, prompt: List[int], n_tokens: int, vocab: int, gamma: int,
                       policy: str, accept: Callable, tree_parent: Optional[np.ndarray] = None,
                       policy_seed: int = 0, n_correct: int = 1):
    """Returns (generated tokens, list of accepted counts per step).

    accept(logits[1, n_q, V] f32, tokens[1, n_q] i32, parent[1, n_q] i32 or None)
        -> (accepted[1, n_q] i32, n_accepted[1] i32)
    Chain when tree_parent is None (n_q = gamma + 1); otherwise node i > 0 drafts a token for
    the position after its parent's.
    """
    rng = np.random.default_rng(policy_seed)
    seq = list(prompt)
    counts = []
    greedy_next = lambda ctx: int(np.argmax(gen.target_logits(seed, ctx, vocab)))
    while len(seq) < len(prompt) + n_tokens:
        if tree_parent is None:
            props = gen.draft_proposals(policy, rng, lambda p: greedy_next(seq + p), gamma, vocab,
                                        n_correct=n_correct)
            nodes = [seq[-1]] + props
            paths = [seq + props[:i] for i in range(len(nodes))]
            parent = None
        else:
            n_q = len(tree_parent)
            nodes = [seq[-1]]
            paths = [list(seq)]
            for i in range(1, n_q):
                ctx = paths[tree_parent[i]]
                if policy == "random":
                    tok = int(rng.integers(vocab))
                elif policy == "correct" or (policy == "correct-then-wrong" and i <= n_correct):
                    tok = greedy_next(ctx)
                else:
                    tok = (greedy_next(ctx) + 1 + int(rng.integers(vocab - 1))) % vocab
                nodes.append(tok)
                paths.append(ctx + [tok])
            parent = np.asarray(tree_parent, dtype=np.int32)[None]
        logits = np.stack([gen.target_logits(seed, p, vocab) for p in paths])[None]
        toks = np.asarray(nodes, dtype=np.int32)[None]
        acc, n_acc = accept(logits, toks, parent)
        n = int(n_acc[0])
        counts.append(n)
        seq.extend(int(t) for t in acc[0, :n])
    return seq[len(prompt):len(prompt) + n_tokens], counts


def hash_draft_loop(target_seed: int, draft_seed: int, prompt: List[int], steps: int, vocab: int,
                    gamma: int, agree24: int, accept: Callable):
    """The decode loop of the device library on the CPU: per step the counter-based synthetic
    draft proposes gamma chained tokens, the synthetic target scores the gamma + 1 nodes, and
    ``accept`` (chain) decides.  Returns (committed sequence after the prompt, accepted counts)."""
    seq = list(prompt)
    counts = []
    for _ in range(steps):
        props = gen.hash_draft_tokens(target_seed, draft_seed, seq, gamma, vocab, agree24)
        nodes = [seq[-1]] + props
        paths = [seq + props[:i] for i in range(gamma + 1)]
        logits = np.stack([gen.target_logits(target_seed, p, vocab) for p in paths])[None]
        acc, n_acc = accept(logits, np.asarray(nodes, dtype=np.int32)[None], None)
        n = int(n_acc[0])
        counts.append(n)
        seq.extend(int(t) for t in acc[0, :n])
    return seq[len(prompt):], counts
