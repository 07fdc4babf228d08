"""Pins for the oracle's ring slot mapping and ring append (CPU only).

Source: Pith verdict on arXiv 2607.21535, referee_report.minor_comments (App. A pseudocode:
"slot = ring_base(r) + logical_pos", with "+d slack"); AI field-notes abstract (the unread draft
KV is reclaimed via a compact ring buffer).
"""
import numpy as np
import pytest

import oracle
from synthetic import gen
from tests.conftest import read_golden


def test_slot_mapping_hand_worked():
    rows = read_golden("ring_slots_s2_c6.txt")
    assert len(rows) == 14
    for p, slot in rows:
        assert oracle.ring_slot(int(p), 2, 6) == int(slot)


def test_slot_mapping_rejects_bad_args():
    assert oracle.ring_slot(-1, 2, 6) == -1
    assert oracle.ring_slot(3, 6, 6) == -1     # no room past the sink


def _fill(B, Hkv, C, D, s, lens_chunks, seed):
    """Appends chunks through the oracle; returns (ring_k, ring_v, ring_len, logical k, v)."""
    rng = np.random.default_rng(seed)
    total = sum(lens_chunks)
    k_lin, v_lin = gen.kv_pair_bf16(rng, (B, total, Hkv, D))
    ring_k = np.full((B, Hkv, C, D), gen.BF16_NAN, dtype=np.uint16)
    ring_v = np.full((B, Hkv, C, D), gen.BF16_NAN, dtype=np.uint16)
    ring_len = np.zeros(B, dtype=np.int64)
    off = 0
    for n in lens_chunks:
        oracle.ring_kv_append(ring_k, ring_v, ring_len, k_lin[:, off:off + n], v_lin[:, off:off + n], s)
        off += n
    return ring_k, ring_v, ring_len, k_lin, v_lin


@pytest.mark.parametrize("s,C,chunks", [
    (2, 6, [14]), (2, 6, [1] * 14), (4, 20, [3, 7, 1, 30, 2]), (0, 8, [5, 5, 5]),
    (4, 256, [2048]), (3, 16, [16]), (3, 16, [15]),
])
def test_ring_matches_linear_layout_through_wraparound(s, C, chunks):
    """Every slot holds the LAST position that maps to it (brute force over all positions), and
    never-written slots stay untouched."""
    B, Hkv, D = 2, 3, 8
    rk, rv, rl, k_lin, v_lin = _fill(B, Hkv, C, D, s, chunks, seed=11)
    L = sum(chunks)
    assert (rl == L).all()
    owner = {}
    for p in range(L):                       # brute force: later positions overwrite
        owner[p if p < s else s + (p - s) % (C - s)] = p
    for slot in range(C):
        for b in range(B):
            for h in range(Hkv):
                if slot in owner:
                    p = owner[slot]
                    assert (rk[b, h, slot] == k_lin[b, p, h]).all()
                    assert (rv[b, h, slot] == v_lin[b, p, h]).all()
                else:
                    assert (rk[b, h, slot] == gen.BF16_NAN).all()


def test_bulk_append_equals_single_appends_tiny_config():
    """A bulk append of 2048 tokens into a 256-slot ring equals 2048 single appends."""
    a = _fill(1, 2, 256, 128, 4, [2048], seed=0)
    b = _fill(1, 2, 256, 128, 4, [1] * 2048, seed=0)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("s,W,L", [(4, 12, 40), (2, 4, 6), (4, 252, 2048), (1, 7, 8), (3, 5, 3)])
def test_ring_holds_exactly_the_window(s, W, L):
    """With capacity s + W, the positions present in the ring after L appends are exactly the
    draft window's key set (first s plus last W positions) -- ring and window agree."""
    C = s + W
    held = set()
    for slot in range(C):
        ps = [p for p in range(L) if oracle.ring_slot(p, s, C) == slot]
        if ps:
            held.add(max(ps))
    window = {j for j in range(L) if oracle.window_member(L, j, s, W)}
    assert held == window
