"""Helpers shared by the GPU parity tests: bits <-> torch tensors and the attention tolerance.

Tolerance (attention outputs, fp64 oracle vs the library's bf16 output), absolute:
|gpu - ref| <= 2e-2 per element and mean |gpu - ref| <= 2e-3 over the checked elements.  The one
relaxation is where a bf16 output cannot meet the absolute bound at all: from |ref| = 8 up, half
a bf16 ulp is already >= 3.1e-2, and there an element may differ from the reference by one bf16
ulp of |ref| (the rounding of an fp32 result that itself sits within a fraction of an ulp).
LSE (fp32): |gpu - ref| <= 1e-3 * max(1, |ref|), equal infinities allowed.
"""
import numpy as np
import torch

MAX_ERR = 2e-2
MEAN_ERR = 2e-3


def to_dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (normal range): 2^(floor(log2 |x|) - 7)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float64).tiny)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def attn_bound(ref: np.ndarray) -> np.ndarray:
    """Per-element bound: 2e-2, or one bf16 ulp of |ref| where |ref| >= 8."""
    return np.where(np.abs(ref) >= 8.0, np.maximum(MAX_ERR, bf16_ulp(ref)), MAX_ERR)


def attn_errors(got: np.ndarray, ref: np.ndarray):
    """(max of err / bound, mean absolute error): the first must be <= 1, the second <= 2e-3."""
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert not np.isnan(got).any(), "NaN in the library output"
    e = np.abs(got - ref)
    return float((e / attn_bound(ref)).max()), float(e.mean())


def assert_attn_close(got, ref, what=""):
    ratio, mean = attn_errors(got, ref)
    e = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    assert ratio <= 1.0 and mean <= MEAN_ERR, \
        f"{what}: max abs {e.max():.3e} ({ratio:.2f} of its bound) mean abs {mean:.3e}"
    return float(e.max()), mean


def assert_lse_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    inf = np.isinf(ref)
    assert np.array_equal(np.isinf(got), inf) and np.array_equal(got[inf], ref[inf]), what
    fin = ~inf
    if fin.any():
        err = np.abs(got[fin] - ref[fin]) / np.maximum(1.0, np.abs(ref[fin]))
        assert err.max() <= 1e-3, f"{what}: lse err {err.max():.3e}"
