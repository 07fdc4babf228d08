"""Helpers shared by the GPU parity tests: bits <-> torch tensors and the attention tolerance.

Tolerance (attention outputs, fp64 oracle vs the library's bf16 output): elementwise error
e = |gpu - ref| / max(1, |ref|); max(e) <= 2e-2 and mean(e) <= 2e-3.  For |ref| <= 1 this is the
stated absolute bound; above 1 it scales with the value, because a bf16 output cannot resolve
an absolute 2e-2 beyond |o| = 8 (half an ulp there is already 3.1e-2).  LSE (fp32):
|gpu - ref| <= 1e-3 * max(1, |ref|), equal infinities allowed.
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


def attn_errors(got: np.ndarray, ref: np.ndarray):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert not np.isnan(got).any(), "NaN in the library output"
    e = np.abs(got - ref) / np.maximum(1.0, np.abs(ref))
    return float(e.max()), float(e.mean())


def assert_attn_close(got, ref, what=""):
    mx, mean = attn_errors(got, ref)
    assert mx <= MAX_ERR and mean <= MEAN_ERR, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def assert_lse_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    inf = np.isinf(ref)
    assert np.array_equal(np.isinf(got), inf) and np.array_equal(got[inf], ref[inf]), what
    fin = ~inf
    if fin.any():
        err = np.abs(got[fin] - ref[fin]) / np.maximum(1.0, np.abs(ref[fin]))
        assert err.max() <= 1e-3, f"{what}: lse err {err.max():.3e}"
