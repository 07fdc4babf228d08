"""Python binding of libwmtp.so with the C ABI's names: argument marshalling only.

Tensors are torch CUDA tensors (bf16 for Q/K/V/out, fp32 for logits and LSE, int32/int64 for
lengths, tables and tokens).  Every call launches the library's kernels on the current torch
stream (or ``stream``) and returns without synchronizing; errors raise WmtpError.  Shapes:

    q, out        [B, n_q, Hq, 128]        bf16
    ring_k/v      [B, Hkv, C, 128]         bf16,  ring_len [B] int64
    k/v pool      [pages, Hkv, 64, 128]    bf16,  page_table [B, max_pages] int32, kv_len [B] int32
    logits        [B, n_q, V] fp32, tokens / tree_parent / accepted [B, n_q] int32
"""
from typing import Optional, Tuple

import torch

from ._lib import check, lib


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _want(t: torch.Tensor, dtype, name: str, ndim: int) -> None:
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or t.dim() != ndim:
        raise TypeError(f"{name}: expected a {ndim}-d {dtype} tensor")
    if not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name}: expected a contiguous CUDA tensor")


def workspace_bytes(B: int, n_q: int, Hq: int, Hkv: int, D: int = 128) -> int:
    return int(lib().wmtp_workspace_bytes(B, n_q, Hq, Hkv, D))


def alloc_workspace(B: int, n_q: int, Hq: int, Hkv: int, device=None) -> torch.Tensor:
    """A zeroed workspace (its control block must start at zero; calls leave it zero)."""
    n = workspace_bytes(B, n_q, Hq, Hkv)
    if n == 0:
        raise ValueError("invalid shape for the workspace")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def ring_kv_append(ring_k, ring_v, ring_len, k_new, v_new, n_sink: int, stream=None) -> None:
    _want(ring_k, torch.bfloat16, "ring_k", 4)
    _want(ring_v, torch.bfloat16, "ring_v", 4)
    _want(ring_len, torch.int64, "ring_len", 1)
    _want(k_new, torch.bfloat16, "k_new", 4)
    _want(v_new, torch.bfloat16, "v_new", 4)
    B, Hkv, C, D = ring_k.shape
    n_new = k_new.shape[1]
    if k_new.shape != (B, n_new, Hkv, D) or v_new.shape != k_new.shape or ring_v.shape != ring_k.shape:
        raise ValueError("ring_kv_append: inconsistent shapes")
    check("ring_kv_append", lib().ring_kv_append(
        _ptr(ring_k), _ptr(ring_v), _ptr(ring_len), _ptr(k_new), _ptr(v_new),
        B, n_new, Hkv, D, int(n_sink), C, _stream(stream)))


def _outs(q, out, lse, want_lse):
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    return out, lse


def draft_attn_window(q, ring_k, ring_v, ring_len, n_sink: int, window: int, sm_scale: float,
                      ws: torch.Tensor, out=None, lse=None, want_lse: bool = True,
                      stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    _want(q, torch.bfloat16, "q", 4)
    _want(ring_k, torch.bfloat16, "ring_k", 4)
    _want(ring_v, torch.bfloat16, "ring_v", 4)
    _want(ring_len, torch.int64, "ring_len", 1)
    B, n_q, Hq, D = q.shape
    _, Hkv, C, _ = ring_k.shape
    out, lse = _outs(q, out, lse, want_lse)
    check("draft_attn_window", lib().draft_attn_window(
        _ptr(q), _ptr(ring_k), _ptr(ring_v), _ptr(ring_len), B, n_q, Hq, Hkv, D, int(n_sink),
        int(window), C, float(sm_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def draft_attn_window_append(q, ring_k, ring_v, ring_len, k_new, v_new, n_sink: int, window: int,
                             sm_scale: float, ws: torch.Tensor, out=None, lse=None,
                             want_lse: bool = True, stream=None):
    """ring_kv_append(k_new, v_new) then draft_attn_window, in one launch when the new rows fit
    the window.  k_new, v_new [B, n_new, Hkv, 128]; ws must come from alloc_workspace (zeroed)."""
    _want(q, torch.bfloat16, "q", 4)
    _want(ring_k, torch.bfloat16, "ring_k", 4)
    _want(ring_v, torch.bfloat16, "ring_v", 4)
    _want(ring_len, torch.int64, "ring_len", 1)
    _want(k_new, torch.bfloat16, "k_new", 4)
    _want(v_new, torch.bfloat16, "v_new", 4)
    B, n_q, Hq, D = q.shape
    _, Hkv, C, _ = ring_k.shape
    n_new = k_new.shape[1]
    if k_new.shape != (B, n_new, Hkv, D) or v_new.shape != k_new.shape or ring_v.shape != ring_k.shape:
        raise ValueError("draft_attn_window_append: inconsistent shapes")
    out, lse = _outs(q, out, lse, want_lse)
    check("draft_attn_window_append", lib().draft_attn_window_append(
        _ptr(q), _ptr(ring_k), _ptr(ring_v), _ptr(ring_len), _ptr(k_new), _ptr(v_new), n_new,
        B, n_q, Hq, Hkv, D, int(n_sink), int(window), C, float(sm_scale), _ptr(out), _ptr(lse),
        _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def draft_attn_window_noalloc(q, ring_k, ring_v, ring_len, n_sink: int, window: int,
                              sm_scale: float, out=None, lse=None, want_lse: bool = True,
                              stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """draft_attn_window for callers that cannot allocate a workspace: the library's built-in
    scratch array holds the split partials (one array per GPU, shared by all calls, so calls
    must not overlap on the GPU)."""
    _want(q, torch.bfloat16, "q", 4)
    _want(ring_k, torch.bfloat16, "ring_k", 4)
    _want(ring_v, torch.bfloat16, "ring_v", 4)
    _want(ring_len, torch.int64, "ring_len", 1)
    B, n_q, Hq, D = q.shape
    _, Hkv, C, _ = ring_k.shape
    out, lse = _outs(q, out, lse, want_lse)
    check("draft_attn_window_noalloc", lib().draft_attn_window_noalloc(
        _ptr(q), _ptr(ring_k), _ptr(ring_v), _ptr(ring_len), B, n_q, Hq, Hkv, D, int(n_sink),
        int(window), C, float(sm_scale), _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def _paged_checks(q, k_pool, v_pool, page_table, kv_len):
    _want(q, torch.bfloat16, "q", 4)
    _want(k_pool, torch.bfloat16, "k_pool", 4)
    _want(v_pool, torch.bfloat16, "v_pool", 4)
    _want(page_table, torch.int32, "page_table", 2)
    _want(kv_len, torch.int32, "kv_len", 1)
    if v_pool.shape != k_pool.shape:
        raise ValueError("k_pool and v_pool differ in shape")


def draft_attn_full(q, k_pool, v_pool, page_table, kv_len, sm_scale: float, ws: torch.Tensor,
                    out=None, lse=None, want_lse: bool = True, stream=None):
    _paged_checks(q, k_pool, v_pool, page_table, kv_len)
    B, n_q, Hq, D = q.shape
    num_pages, Hkv, P, _ = k_pool.shape
    out, lse = _outs(q, out, lse, want_lse)
    check("draft_attn_full", lib().draft_attn_full(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(kv_len), B, n_q, Hq, Hkv, D, P,
        page_table.shape[1], num_pages, float(sm_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
        _stream(stream)))
    return out, lse


def verify_attn(q, k_pool, v_pool, page_table, kv_len, sm_scale: float, ws: torch.Tensor,
                tree_parent=None, out=None, lse=None, want_lse: bool = True, stream=None):
    _paged_checks(q, k_pool, v_pool, page_table, kv_len)
    if tree_parent is not None:
        _want(tree_parent, torch.int32, "tree_parent", 2)
    B, n_q, Hq, D = q.shape
    num_pages, Hkv, P, _ = k_pool.shape
    out, lse = _outs(q, out, lse, want_lse)
    check("verify_attn", lib().verify_attn(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(kv_len), _ptr(tree_parent),
        B, n_q, Hq, Hkv, D, P, page_table.shape[1], num_pages, float(sm_scale), _ptr(out),
        _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def accept_greedy(logits, tokens, tree_parent=None, accepted=None, n_accepted=None, stream=None):
    _want(logits, torch.float32, "logits", 3)
    _want(tokens, torch.int32, "tokens", 2)
    if tree_parent is not None:
        _want(tree_parent, torch.int32, "tree_parent", 2)
    B, n_q, V = logits.shape
    if accepted is None:
        accepted = torch.empty((B, n_q), dtype=torch.int32, device=logits.device)
    if n_accepted is None:
        n_accepted = torch.empty((B,), dtype=torch.int32, device=logits.device)
    check("accept_greedy", lib().accept_greedy(
        _ptr(logits), _ptr(tokens), _ptr(tree_parent), B, n_q, V, _ptr(accepted), _ptr(n_accepted),
        _stream(stream)))
    return accepted, n_accepted


def device_status(stream=None) -> int:
    """Reads and clears the device status word (synchronizes the stream); 0 when clean."""
    return int(lib().wmtp_device_status(_stream(stream)))


def selftest_wait_timeout(limit_ns: int = 50_000_000, stream=None) -> None:
    """Runs the library's bounded-wait failure path on purpose (a wait nothing satisfies); the
    next device_status() returns WMTP_ERR_TIMEOUT."""
    check("wmtp_selftest_wait_timeout", lib().wmtp_selftest_wait_timeout(int(limit_ns), _stream(stream)))


def launch_count() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib().wmtp_launch_count())


# ----------------------------------------------------------------------------- decode loop
def ring_kv_append_at(ring_k, ring_v, ring_len, k_new, v_new, pos, n_new, n_sink: int,
                      stream=None) -> None:
    """Request b writes rows [0, n_new[b]) of k_new/v_new [B, n_max, Hkv, 128] at draft positions
    pos[b] ..; ring_len[b] becomes pos[b] + n_new[b] (rolling back anything past it)."""
    _want(ring_k, torch.bfloat16, "ring_k", 4)
    _want(ring_v, torch.bfloat16, "ring_v", 4)
    _want(ring_len, torch.int64, "ring_len", 1)
    _want(k_new, torch.bfloat16, "k_new", 4)
    _want(v_new, torch.bfloat16, "v_new", 4)
    _want(pos, torch.int64, "pos", 1)
    _want(n_new, torch.int32, "n_new", 1)
    B, Hkv, C, D = ring_k.shape
    n_max = k_new.shape[1]
    if k_new.shape != (B, n_max, Hkv, D) or v_new.shape != k_new.shape or ring_v.shape != ring_k.shape:
        raise ValueError("ring_kv_append_at: inconsistent shapes")
    check("ring_kv_append_at", lib().ring_kv_append_at(
        _ptr(ring_k), _ptr(ring_v), _ptr(ring_len), _ptr(k_new), _ptr(v_new), _ptr(pos), _ptr(n_new),
        B, n_max, Hkv, D, int(n_sink), C, _stream(stream)))


def spec_commit(accepted, n_accepted, history, n_tokens, append_pos, n_append, verify_len=None,
                n_q_verify: int = 0, draft_len=None, stream=None) -> None:
    """Commits accept_greedy's output into the loop state (see wmtp_loop.h)."""
    _want(accepted, torch.int32, "accepted", 2)
    _want(n_accepted, torch.int32, "n_accepted", 1)
    _want(history, torch.int32, "history", 2)
    _want(n_tokens, torch.int64, "n_tokens", 1)
    _want(append_pos, torch.int64, "append_pos", 1)
    _want(n_append, torch.int32, "n_append", 1)
    if verify_len is not None:
        _want(verify_len, torch.int32, "verify_len", 1)
    n_draft = 0
    if draft_len is not None:
        _want(draft_len, torch.int32, "draft_len", 2)
        n_draft = draft_len.shape[0]
    B, n_q = accepted.shape
    check("spec_commit", lib().spec_commit(
        _ptr(accepted), _ptr(n_accepted), B, n_q, _ptr(history), history.shape[1], _ptr(n_tokens),
        _ptr(append_pos), _ptr(n_append), _ptr(verify_len), int(n_q_verify), _ptr(draft_len), n_draft,
        _stream(stream)))


def synth_draft_tokens(history, n_tokens, gamma: int, vocab: int, target_seed: int, draft_seed: int,
                       agree24: int, tokens=None, stream=None):
    """Synthetic draft head: tokens [B, gamma + 1] (last committed token, then gamma proposals)."""
    _want(history, torch.int32, "history", 2)
    _want(n_tokens, torch.int64, "n_tokens", 1)
    B = history.shape[0]
    if tokens is None:
        tokens = torch.empty((B, gamma + 1), dtype=torch.int32, device=history.device)
    _want(tokens, torch.int32, "tokens", 2)
    check("wmtp_synth_draft_tokens", lib().wmtp_synth_draft_tokens(
        _ptr(history), _ptr(n_tokens), B, history.shape[1], int(gamma), int(vocab),
        int(target_seed) & 0xFFFFFFFFFFFFFFFF, int(draft_seed) & 0xFFFFFFFFFFFFFFFF, int(agree24),
        _ptr(tokens), _stream(stream)))
    return tokens


def synth_target_logits(history, n_tokens, tokens, vocab: int, target_seed: int, tree_parent=None,
                        logits=None, stream=None):
    """Synthetic target head: logits [B, n_q, vocab] of the verify nodes ``tokens`` [B, n_q]."""
    _want(history, torch.int32, "history", 2)
    _want(n_tokens, torch.int64, "n_tokens", 1)
    _want(tokens, torch.int32, "tokens", 2)
    if tree_parent is not None:
        _want(tree_parent, torch.int32, "tree_parent", 2)
    B, n_q = tokens.shape
    if logits is None:
        logits = torch.empty((B, n_q, vocab), dtype=torch.float32, device=tokens.device)
    _want(logits, torch.float32, "logits", 3)
    check("wmtp_synth_target_logits", lib().wmtp_synth_target_logits(
        _ptr(history), _ptr(n_tokens), B, history.shape[1], _ptr(tokens), _ptr(tree_parent), n_q,
        int(vocab), int(target_seed) & 0xFFFFFFFFFFFFFFFF, _ptr(logits), _stream(stream)))
    return logits


def accept_stochastic(p, q, tokens, u_accept, u_sample, accepted=None, n_accepted=None, stream=None):
    """Rejection-sampling acceptance of drafted chains (see wmtp.h).  p [B, n_q, V] and
    q [B, n_q - 1, V] float32 probabilities; tokens [B, n_q] int32; u_accept [B, n_q - 1] and
    u_sample [B] 32-bit integers (int32 or uint32 tensors holding the bit patterns)."""
    _want(p, torch.float32, "p", 3)
    _want(tokens, torch.int32, "tokens", 2)
    B, n_q, V = p.shape
    if n_q > 1:
        _want(q, torch.float32, "q", 3)
        if q.shape != (B, n_q - 1, V):
            raise ValueError("accept_stochastic: q must be [B, n_q - 1, V]")
        if u_accept.dtype not in (torch.int32, torch.uint32) or u_accept.shape != (B, n_q - 1) \
                or not u_accept.is_contiguous() or not u_accept.is_cuda:
            raise TypeError("u_accept: expected a contiguous [B, n_q - 1] 32-bit CUDA tensor")
    if u_sample.dtype not in (torch.int32, torch.uint32) or u_sample.shape != (B,) or not u_sample.is_cuda:
        raise TypeError("u_sample: expected a [B] 32-bit CUDA tensor")
    if accepted is None:
        accepted = torch.empty((B, n_q), dtype=torch.int32, device=p.device)
    if n_accepted is None:
        n_accepted = torch.empty((B,), dtype=torch.int32, device=p.device)
    check("accept_stochastic", lib().accept_stochastic(
        _ptr(p), _ptr(q) if n_q > 1 else None, _ptr(tokens), _ptr(u_accept) if n_q > 1 else None,
        _ptr(u_sample), B, n_q, V, _ptr(accepted), _ptr(n_accepted), _stream(stream)))
    return accepted, n_accepted


# ----------------------------------------------------------------------------- fp8 (E4M3) KV
_FP8_DTYPES = (torch.uint8, torch.float8_e4m3fn)


def _want8(t, name: str, ndim: int) -> None:
    if not isinstance(t, torch.Tensor) or t.dtype not in _FP8_DTYPES or t.dim() != ndim:
        raise TypeError(f"{name}: expected a {ndim}-d uint8 / float8_e4m3fn tensor of E4M3 codes")
    if not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name}: expected a contiguous CUDA tensor")


def ring_kv_append_fp8(ring_k, ring_v, ring_len, k_new, v_new, n_sink: int, stream=None) -> None:
    """ring_kv_append on E4M3 rows: ring [B, Hkv, C, 128], new rows [B, n_new, Hkv, 128]."""
    _want8(ring_k, "ring_k", 4)
    _want8(ring_v, "ring_v", 4)
    _want(ring_len, torch.int64, "ring_len", 1)
    _want8(k_new, "k_new", 4)
    _want8(v_new, "v_new", 4)
    B, Hkv, C, D = ring_k.shape
    n_new = k_new.shape[1]
    if k_new.shape != (B, n_new, Hkv, D) or v_new.shape != k_new.shape or ring_v.shape != ring_k.shape:
        raise ValueError("ring_kv_append_fp8: inconsistent shapes")
    check("ring_kv_append_fp8", lib().ring_kv_append_fp8(
        _ptr(ring_k), _ptr(ring_v), _ptr(ring_len), _ptr(k_new), _ptr(v_new),
        B, n_new, Hkv, D, int(n_sink), C, _stream(stream)))


def draft_attn_window_fp8(q, ring_k, ring_v, ring_len, n_sink: int, window: int, sm_scale: float,
                          k_scale: float, v_scale: float, ws: torch.Tensor, out=None, lse=None,
                          want_lse: bool = True, stream=None):
    _want(q, torch.bfloat16, "q", 4)
    _want8(ring_k, "ring_k", 4)
    _want8(ring_v, "ring_v", 4)
    _want(ring_len, torch.int64, "ring_len", 1)
    B, n_q, Hq, D = q.shape
    _, Hkv, C, _ = ring_k.shape
    out, lse = _outs(q, out, lse, want_lse)
    check("draft_attn_window_fp8", lib().draft_attn_window_fp8(
        _ptr(q), _ptr(ring_k), _ptr(ring_v), _ptr(ring_len), B, n_q, Hq, Hkv, D, int(n_sink),
        int(window), C, float(sm_scale), float(k_scale), float(v_scale), _ptr(out), _ptr(lse),
        _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def draft_attn_window_append_fp8(q, ring_k, ring_v, ring_len, k_new, v_new, n_sink: int, window: int,
                                 sm_scale: float, k_scale: float, v_scale: float, ws: torch.Tensor,
                                 out=None, lse=None, want_lse: bool = True, stream=None):
    """draft_attn_window_append on E4M3 rings and new rows."""
    _want(q, torch.bfloat16, "q", 4)
    _want8(ring_k, "ring_k", 4)
    _want8(ring_v, "ring_v", 4)
    _want(ring_len, torch.int64, "ring_len", 1)
    _want8(k_new, "k_new", 4)
    _want8(v_new, "v_new", 4)
    B, n_q, Hq, D = q.shape
    _, Hkv, C, _ = ring_k.shape
    n_new = k_new.shape[1]
    if k_new.shape != (B, n_new, Hkv, D) or v_new.shape != k_new.shape or ring_v.shape != ring_k.shape:
        raise ValueError("draft_attn_window_append_fp8: inconsistent shapes")
    out, lse = _outs(q, out, lse, want_lse)
    check("draft_attn_window_append_fp8", lib().draft_attn_window_append_fp8(
        _ptr(q), _ptr(ring_k), _ptr(ring_v), _ptr(ring_len), _ptr(k_new), _ptr(v_new), n_new,
        B, n_q, Hq, Hkv, D, int(n_sink), int(window), C, float(sm_scale), float(k_scale),
        float(v_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def _paged8_checks(q, k_pool, v_pool, page_table, kv_len):
    _want(q, torch.bfloat16, "q", 4)
    _want8(k_pool, "k_pool", 4)
    _want8(v_pool, "v_pool", 4)
    _want(page_table, torch.int32, "page_table", 2)
    _want(kv_len, torch.int32, "kv_len", 1)
    if v_pool.shape != k_pool.shape:
        raise ValueError("k_pool and v_pool differ in shape")


def draft_attn_full_fp8(q, k_pool, v_pool, page_table, kv_len, sm_scale: float, k_scale: float,
                        v_scale: float, ws: torch.Tensor, out=None, lse=None, want_lse: bool = True,
                        stream=None):
    _paged8_checks(q, k_pool, v_pool, page_table, kv_len)
    B, n_q, Hq, D = q.shape
    num_pages, Hkv, P, _ = k_pool.shape
    out, lse = _outs(q, out, lse, want_lse)
    check("draft_attn_full_fp8", lib().draft_attn_full_fp8(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(kv_len), B, n_q, Hq, Hkv, D, P,
        page_table.shape[1], num_pages, float(sm_scale), float(k_scale), float(v_scale), _ptr(out),
        _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse


def verify_attn_fp8(q, k_pool, v_pool, page_table, kv_len, sm_scale: float, k_scale: float,
                    v_scale: float, ws: torch.Tensor, tree_parent=None, out=None, lse=None,
                    want_lse: bool = True, stream=None):
    _paged8_checks(q, k_pool, v_pool, page_table, kv_len)
    if tree_parent is not None:
        _want(tree_parent, torch.int32, "tree_parent", 2)
    B, n_q, Hq, D = q.shape
    num_pages, Hkv, P, _ = k_pool.shape
    out, lse = _outs(q, out, lse, want_lse)
    check("verify_attn_fp8", lib().verify_attn_fp8(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(page_table), _ptr(kv_len), _ptr(tree_parent),
        B, n_q, Hq, Hkv, D, P, page_table.shape[1], num_pages, float(sm_scale), float(k_scale),
        float(v_scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return out, lse
