"""Draft-KV accounting for one decode step: bytes the attention calls must move, and the KV
memory the ring buffer reclaims.

Sources: AI field-notes entry for arXiv 2607.21535 (English abstract: the window bounds the
draft's KV working set to a constant, dropping about 99% of KV entries at 1M; the unread draft
KV, 7.7-11% of total KV at 1M, is reclaimed by a compact ring buffer); Pith verdict,
pith_extraction.key_machinery (t_step = t_verify + t_ctx_draft + gamma * t_fwd_draft, Eq. 1).

Reading adopted for the reclaimed share of TOTAL KV: the draft layer's KV has the shape of one
target attention layer's KV, so with n target attention layers the draft pool is 1/(n+1) of all
KV, and the ring keeps C of its L positions.
"""
from dataclasses import dataclass

BF16 = 2


def kv_row_bytes(Hkv: int, D: int) -> int:
    """K plus V bytes of one token position, all kv heads."""
    return Hkv * D * BF16 * 2


def window_keys(L_tot: int, n_sink: int, window: int) -> int:
    """Keys a windowed draft call reads: the union of the sink and the recent window."""
    return min(L_tot, n_sink + window)


def draft_full_bytes(L_tot: int, Hkv: int, D: int) -> int:
    return L_tot * kv_row_bytes(Hkv, D)


def draft_window_bytes(L_tot: int, n_sink: int, window: int, Hkv: int, D: int) -> int:
    return window_keys(L_tot, n_sink, window) * kv_row_bytes(Hkv, D)


def verify_layer_bytes(L: int, n_q: int, Hkv: int, D: int) -> int:
    return (L + n_q) * kv_row_bytes(Hkv, D)


def append_bytes(n_new: int, Hkv: int, D: int) -> int:
    return n_new * kv_row_bytes(Hkv, D)


def dropped_fraction(L: int, capacity: int) -> float:
    """Share of the draft's KV entries the windowed draft never reads or keeps."""
    return 1.0 - min(capacity, L) / L


def reclaimed_share_of_total(L: int, capacity: int, n_attn_layers: int) -> float:
    """Share of ALL KV (target layers + draft layer) the ring reclaims."""
    return (L - min(capacity, L)) / (L * (n_attn_layers + 1))


@dataclass
class StepBytes:
    """Algorithmic KV bytes of one decode step (Eq. 1's terms), per arm."""
    ctx_draft: int
    fwd_draft: int          # one draft forward (gamma of them per step)
    verify: int             # all verify layers
    gamma: int

    @property
    def draft(self) -> int:
        return self.ctx_draft + self.gamma * self.fwd_draft

    @property
    def total(self) -> int:
        return self.draft + self.verify


def step_bytes(L: int, gamma: int, n_q_verify: int, Hkv: int, D: int, n_layers: int,
               n_sink: int, window: int, windowed: bool) -> StepBytes:
    """Bytes of one step with L committed tokens: the context pass sees L + gamma + 1 draft
    positions, draft forward j sees L + gamma + 1 + j, and verify reads L + n_q per layer."""
    base = L + gamma + 1
    if windowed:
        ctx = draft_window_bytes(base, n_sink, window, Hkv, D)
        fwd = draft_window_bytes(base + gamma, n_sink, window, Hkv, D)
    else:
        ctx = draft_full_bytes(base, Hkv, D)
        fwd = draft_full_bytes(base + gamma, Hkv, D)
    return StepBytes(ctx, fwd, n_layers * verify_layer_bytes(L, n_q_verify, Hkv, D), gamma)


def linear_fit(x, y):
    """Ordinary least squares y = intercept + slope * x, with the coefficient of determination.

    The cost identity's draft terms are fitted against context length this way (Pith verdict on
    arXiv 2607.21535, referee_report.minor_comments on App. B, Table 6: fitted slopes and
    intercepts with R^2): a full-context draft forward grows with L, a windowed one should not.
    Returns (slope, intercept, r2); r2 is 1.0 when y is constant and exactly fitted.
    """
    n = len(x)
    if n != len(y) or n < 2:
        raise ValueError("linear_fit needs two or more (x, y) pairs")
    mx = sum(x) / n
    my = sum(y) / n
    sxx = sum((a - mx) ** 2 for a in x)
    if sxx == 0:
        raise ValueError("linear_fit needs two distinct x values")
    sxy = sum((a - mx) * (b - my) for a, b in zip(x, y))
    slope = sxy / sxx
    intercept = my - slope * mx
    ss_res = sum((b - (intercept + slope * a)) ** 2 for a, b in zip(x, y))
    ss_tot = sum((b - my) ** 2 for b in y)
    r2 = 1.0 - ss_res / ss_tot if ss_tot > 0 else 1.0
    return slope, intercept, r2
