"""KV accounting against the numbers the pages print (CPU only)."""
import pytest

from long_context_speculative_kv_b200 import accounting as acc
from tests.conftest import read_golden


def _golden():
    return {r[0]: (float(r[1]), float(r[2])) for r in read_golden("kv_accounting.txt")}


def test_dropped_fraction_at_1m():
    v, tol = _golden()["dropped_fraction_1M_window4096"]
    got = acc.dropped_fraction(1 << 20, 4096)
    assert got == pytest.approx(1 - 4096 / 2 ** 20, abs=1e-15)     # 0.99609375
    assert abs(got - v) <= tol


def test_reclaimed_share_of_total_kv_range():
    g = _golden()
    lo, tol_lo = g["reclaimed_total_low"]
    hi, tol_hi = g["reclaimed_total_high"]
    # 12 target attention layers (hybrid target) -> low end; 8 layers -> high end
    r12 = acc.reclaimed_share_of_total(1 << 20, 4096, 12)
    r8 = acc.reclaimed_share_of_total(1 << 20, 4096, 8)
    assert abs(r12 - lo) <= tol_lo
    assert abs(r8 - hi) <= tol_hi
    assert r12 == pytest.approx(0.99609375 / 13, rel=1e-12)


def test_step_bytes_shapes():
    L, g = 1 << 20, 3
    w = acc.step_bytes(L, g, g + 1, 4, 128, 12, 4, 4092, windowed=True)
    f = acc.step_bytes(L, g, g + 1, 4, 128, 12, 4, 4092, windowed=False)
    assert w.fwd_draft == 4096 * 4 * 128 * 4          # 8 MiB
    assert f.fwd_draft == (L + 2 * g + 1) * 4 * 128 * 4
    assert w.verify == f.verify == 12 * (L + g + 1) * 4 * 128 * 4
    assert acc.window_keys(100, 4, 4092) == 100


def test_linear_fit_recovers_an_exact_line():
    xs = [65536, 131072, 262144, 524288, 1048576]
    ys = [3.5 + 2.25e-4 * x for x in xs]
    m, c, r2 = acc.linear_fit(xs, ys)
    assert m == pytest.approx(2.25e-4, rel=1e-12)
    assert c == pytest.approx(3.5, rel=1e-9)
    assert r2 == pytest.approx(1.0, abs=1e-12)


def test_linear_fit_anscombe_first_set():
    # Anscombe (1973), data set I: fitted line y = 3.00 + 0.500 x with r^2 = 0.67 (the published
    # summary statistics all four sets share).
    x = [10, 8, 13, 9, 11, 14, 6, 4, 12, 7, 5]
    y = [8.04, 6.95, 7.58, 8.81, 8.33, 9.96, 7.24, 4.26, 10.84, 4.82, 5.68]
    m, c, r2 = acc.linear_fit(x, y)
    assert m == pytest.approx(0.500, abs=5e-4)
    assert c == pytest.approx(3.00, abs=5e-3)
    assert r2 == pytest.approx(0.67, abs=5e-3)


def test_linear_fit_flat_series_has_zero_slope():
    m, c, r2 = acc.linear_fit([1, 2, 3, 4], [7.0, 7.0, 7.0, 7.0])
    assert m == 0 and c == 7.0 and r2 == 1.0
    with pytest.raises(ValueError):
        acc.linear_fit([1, 1], [2.0, 3.0])
