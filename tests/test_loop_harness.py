"""The device decode loop's CPU counterpart (CPU only): with the counter-based synthetic draft
and the oracle's greedy acceptance, the committed sequence is the synthetic target's own greedy
sequence whatever the draft's agreement rate (AI field-notes abstract for arXiv 2607.21535: the
target decides every accepted token, so the draft changes only what is proposed), and the
accepted counts hit the rule's two closed-form extremes."""
import numpy as np
import pytest

import oracle
from synthetic import gen
from tests.lossless_harness import hash_draft_loop, target_greedy

VOCAB = 64


def _accept(logits, tokens, parent):
    return oracle.accept_greedy(logits, tokens, parent)


@pytest.mark.parametrize("agree", [0.0, 0.3, 0.8, 1.0])
@pytest.mark.parametrize("gamma", [1, 3, 5])
def test_hash_draft_loop_is_lossless(agree, gamma):
    prompt = [5, 17, 3, 60, 22]
    agree24 = int(round(agree * (1 << 24)))
    seq, counts = hash_draft_loop(11, 12, prompt, 20, VOCAB, gamma, agree24, _accept)
    assert seq == target_greedy(11, prompt, len(seq), VOCAB)
    assert all(1 <= n <= gamma + 1 for n in counts)
    if agree24 == 0:
        assert counts == [1] * 20                    # every proposal differs from the target's token
    if agree24 == 1 << 24:
        assert counts == [gamma + 1] * 20            # every proposal is the target's token


def test_hash_draft_agreement_rate():
    # proposals equal the target's greedy token at about the requested rate (a 24-bit threshold)
    hits, total = 0, 0
    rng = np.random.default_rng(3)
    for t in range(400):
        prefix = list(rng.integers(0, VOCAB, size=6))
        p = gen.hash_draft_tokens(7, 8, prefix, 1, VOCAB, int(0.6 * (1 << 24)))[0]
        hits += p == int(np.argmax(gen.target_logits(7, prefix, VOCAB)))
        total += 1
    assert abs(hits / total - 0.6) < 0.08
