"""Helpers shared by the GPU parity tests: bits <-> torch tensors and the attention tolerance.

Tolerance (attention outputs, fp64 oracle vs the library's bf16 output).  The stated bounds,
max-abs 2e-2 and mean-abs 2e-3 for bf16 inputs with fp32 accumulation, bound the arithmetic's
error; on top of it every kernel must round twice to bf16, each rounding worth at most half a
bf16 ulp u(ref) of the output's size: the attention weights P, which the tensor cores take as
bf16 next to the bf16 values, and the output itself.  So, with e = |gpu - ref|:
  * every element: e <= 2e-2 + u(ref);
  * on average: mean over the checked elements of max(0, e - u(ref)/2) <= 2e-3 (the output's own
    rounding, a quarter ulp on average, already exceeds 2e-3 at |ref| > 1, so a plain mean could
    not hold for outputs of that size whatever the kernel computed before rounding).
For unit-scale outputs (|ref| < 1) u(ref) <= 2^-8, so the bounds are within 2e-3 of the plain
ones.  LSE (fp32): |gpu - ref| <= 4e-3 + 1e-5 |ref| (the tcgen05 kernel's row sums are sums of
the bf16-rounded weights the PV product uses, so ln of a sum carries up to 2^-8 of their
rounding), equal infinities allowed.
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
    """Per-element bound: 2e-2 plus one bf16 ulp of |ref| (the P and output roundings)."""
    return MAX_ERR + bf16_ulp(ref)


def attn_errors(got: np.ndarray, ref: np.ndarray):
    """(max of |err| / bound, mean of the error beyond the bf16 output's own rounding): the first
    must be <= 1, the second <= 2e-3."""
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert not np.isnan(got).any(), "NaN in the library output"
    e = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    excess = np.maximum(0.0, e - 0.5 * bf16_ulp(ref))
    return float((e / attn_bound(ref)).max()), float(excess.mean())


def assert_attn_close(got, ref, what=""):
    ratio, mean = attn_errors(got, ref)
    e = np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))
    assert ratio <= 1.0 and mean <= MEAN_ERR, \
        f"{what}: max abs {e.max():.3e} ({ratio:.2f} of its bound) mean excess {mean:.3e} (mean abs {e.mean():.3e})"
    return float(e.max()), mean


def assert_lse_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    inf = np.isinf(ref)
    assert np.array_equal(np.isinf(got), inf) and np.array_equal(got[inf], ref[inf]), what
    fin = ~inf
    if fin.any():
        err = np.abs(got[fin] - ref[fin]) / (4e-3 + 1e-5 * np.abs(ref[fin]))
        assert err.max() <= 1.0, f"{what}: lse err {np.abs(got[fin] - ref[fin]).max():.3e} ({err.max():.2f} of its bound)"
