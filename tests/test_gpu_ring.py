"""GPU parity: ring_kv_append through the C ABI against the oracle's ring, bit-exact.

Source: Pith verdict on arXiv 2607.21535, referee_report.minor_comments (App. A pseudocode:
"slot = ring_base(r) + logical_pos"); AI field-notes abstract (compact ring buffer).
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_speculative_kv_b200 import api
from synthetic import gen
from tests.gpu_util import to_bits, to_dev_bf16

pytestmark = pytest.mark.gpu


def _run(B, Hkv, s, C, chunks, seed):
    rng = np.random.default_rng(seed)
    D = 128
    total = sum(chunks)
    k_lin, v_lin = gen.kv_pair_bf16(rng, (B, total, Hkv, D))
    ring_k = np.full((B, Hkv, C, D), gen.BF16_NAN, dtype=np.uint16)
    ring_v = ring_k.copy()
    ring_len = rng.integers(0, 3, size=B).astype(np.int64) * 0      # start empty
    gk, gv = to_dev_bf16(ring_k), to_dev_bf16(ring_v)
    glen = torch.from_numpy(ring_len.copy()).cuda()
    off = 0
    for n in chunks:
        kn, vn = k_lin[:, off:off + n], v_lin[:, off:off + n]
        oracle.ring_kv_append(ring_k, ring_v, ring_len, kn, vn, s)
        api.ring_kv_append(gk, gv, glen, to_dev_bf16(kn), to_dev_bf16(vn), s)
        off += n
        torch.cuda.synchronize()
        assert np.array_equal(glen.cpu().numpy(), ring_len)
        assert np.array_equal(to_bits(gk), ring_k), f"K after {off} tokens"
        assert np.array_equal(to_bits(gv), ring_v), f"V after {off} tokens"


@pytest.mark.parametrize("B,Hkv,s,C,chunks", [
    (1, 2, 4, 256, [1] * 300),                          # single appends through wraparound
    (1, 2, 4, 256, [2048]),                             # one bulk append, 8 wraps
    (2, 2, 4, 256, [3, 1, 300, 1, 17, 600, 5, 1]),      # mixed; multi-CTA bulk path
    (3, 4, 4, 4096, [5000, 1, 1, 4095, 7]),
    (2, 8, 4, 1024, [3, 1200, 2]),
    (2, 2, 0, 64, [70, 1, 63]),                         # no sink
    (1, 2, 64, 128, [10, 100, 1, 200]),                 # a sink as long as a tile
])
def test_ring_append_matches_oracle(B, Hkv, s, C, chunks):
    _run(B, Hkv, s, C, chunks, seed=hash((B, Hkv, s, C, len(chunks))) % 2 ** 32)


def test_bulk_equals_single_appends_tiny_workload():
    """The tiny workload's ring: 2048 single appends == one bulk append of 2048 tokens."""
    rng = np.random.default_rng(0)
    k_lin, v_lin = gen.kv_pair_bf16(rng, (1, 2048, 2, 128))
    outs = []
    for chunks in ([2048], [1] * 2048):
        gk = torch.zeros((1, 2, 256, 128), dtype=torch.bfloat16, device="cuda")
        gv = torch.zeros_like(gk)
        glen = torch.zeros(1, dtype=torch.int64, device="cuda")
        kd, vd = to_dev_bf16(k_lin), to_dev_bf16(v_lin)
        off = 0
        for n in chunks:
            api.ring_kv_append(gk, gv, glen, kd[:, off:off + n].contiguous(), vd[:, off:off + n].contiguous(), 4)
            off += n
        torch.cuda.synchronize()
        outs.append((to_bits(gk), to_bits(gv), glen.item()))
    assert outs[0][2] == outs[1][2] == 2048
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])
