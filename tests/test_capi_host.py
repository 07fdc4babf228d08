"""The C-ABI library loads, exports every entry point include/wmtp.h declares, and rejects bad
arguments on the host (these checks return before any CUDA call, so they run without a GPU)."""
import ctypes
import re
import subprocess

import pytest

from long_context_speculative_kv_b200 import _lib
from long_context_speculative_kv_b200.build import build


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.lib()


def _headers_src():
    parts = []
    for h in _lib.HEADERS:
        with open(h) as f:
            parts.append(f.read())
    return "\n".join(parts)


def _declared():
    return set(re.findall(r"^WMTP_API\s+[\w\s\*]*?\b(\w+)\s*\(", _headers_src(), re.M))


def test_header_declares_the_five_calls_and_helpers():
    names = _declared()
    assert {"ring_kv_append", "draft_attn_window", "draft_attn_full", "verify_attn",
            "accept_greedy", "wmtp_workspace_bytes", "wmtp_status_string",
            "wmtp_device_status", "wmtp_launch_count", "draft_attn_window_noalloc",
            "accept_stochastic", "ring_kv_append_at", "spec_commit", "ring_kv_append_fp8",
            "draft_attn_window_fp8", "draft_attn_full_fp8", "verify_attn_fp8", "wmtp_synth_draft_tokens",
            "wmtp_synth_target_logits", "wmtp_selftest_wait_timeout", "draft_attn_window_append",
            "draft_attn_window_append_fp8"} == names
    assert set(_lib._SIGNATURES) == names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert _declared() <= exported
    for name in _declared():
        assert hasattr(lib, name)


def test_status_strings(lib):
    for code, name in _lib.STATUS.items():
        s = _lib.status_string(code)
        assert isinstance(s, str) and s and s != "unknown status", name
    assert _lib.status_string(12345) == "unknown status"


def test_binding_signatures_match_header_arity():
    src = _headers_src()
    for name, (args, _) in _lib._SIGNATURES.items():
        m = re.search(r"^WMTP_API\s+[\w\s\*]*?\b" + name + r"\s*\(([^)]*)\)", src, re.S | re.M)
        assert m, name
        params = [p for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        assert len(params) == len(args), name


BAD = ctypes.c_void_p(0x1001)      # misaligned fake pointer: never dereferenced on the host
GOOD = ctypes.c_void_p(0x10000)    # aligned fake pointer: never dereferenced on the host


def test_ring_append_host_checks(lib):
    f = lib.ring_kv_append
    assert f(None, GOOD, GOOD, GOOD, GOOD, 1, 1, 2, 128, 4, 256, None) == -1      # null ring
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, 1, 1, 2, 64, 4, 256, None) == -2       # D != 128
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, 1, 1, 2, 128, 4, 4, None) == -1        # C <= n_sink
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, 1, -1, 2, 128, 4, 256, None) == -1     # n_new < 0
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, 1, 0, 2, 128, 4, 256, None) == 0       # no-op
    assert f(BAD, GOOD, GOOD, GOOD, GOOD, 1, 1, 2, 128, 4, 256, None) == -3       # misaligned


def test_attention_host_checks(lib):
    w = lib.draft_attn_window
    # (q, rk, rv, rlen, B, n_q, Hq, Hkv, D, s, W, C, scale, out, lse, ws, ws_bytes, stream)
    assert w(GOOD, GOOD, GOOD, GOOD, 1, 1, 8, 3, 128, 4, 252, 256, 1.0, GOOD, None, GOOD, 1 << 30, None) == -2
    assert w(GOOD, GOOD, GOOD, GOOD, 1, 1, 8, 2, 96, 4, 252, 256, 1.0, GOOD, None, GOOD, 1 << 30, None) == -2
    assert w(GOOD, GOOD, GOOD, GOOD, 1, 65, 8, 2, 128, 4, 252, 256, 1.0, GOOD, None, GOOD, 1 << 30, None) == -2
    assert w(GOOD, GOOD, GOOD, GOOD, 1, 1, 8, 2, 128, 4, 253, 256, 1.0, GOOD, None, GOOD, 1 << 30, None) == -1
    assert w(GOOD, GOOD, GOOD, GOOD, 1, 1, 8, 2, 128, 4, 252, 256, -1.0, GOOD, None, GOOD, 1 << 30, None) == -1
    assert w(GOOD, None, GOOD, GOOD, 1, 1, 8, 2, 128, 4, 252, 256, 1.0, GOOD, None, GOOD, 1 << 30, None) == -1
    assert w(BAD, GOOD, GOOD, GOOD, 1, 1, 8, 2, 128, 4, 252, 256, 1.0, GOOD, None, GOOD, 1 << 30, None) == -3
    f = lib.draft_attn_full
    # (q, kp, vp, pt, kvlen, B, n_q, Hq, Hkv, D, P, max_pages, num_pages, scale, out, lse, ws, n, s)
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, 1, 1, 8, 2, 128, 32, 4, 4, 1.0, GOOD, None, GOOD, 1 << 30, None) == -2
    assert f(GOOD, GOOD, GOOD, None, GOOD, 1, 1, 8, 2, 128, 64, 4, 4, 1.0, GOOD, None, GOOD, 1 << 30, None) == -1
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, 1, 1, 8, 2, 128, 64, 0, 4, 1.0, GOOD, None, GOOD, 1 << 30, None) == -1
    v = lib.verify_attn
    assert v(GOOD, GOOD, GOOD, GOOD, GOOD, BAD, 1, 4, 8, 2, 128, 64, 4, 4, 1.0, GOOD, None, GOOD, 1 << 30, None) == -3
    assert v(GOOD, GOOD, GOOD, GOOD, GOOD, None, 0, 4, 8, 2, 128, 64, 4, 4, 1.0, GOOD, None, GOOD, 1 << 30, None) == -1


def test_window_append_host_checks(lib):
    f = lib.draft_attn_window_append
    # (q, rk, rv, rlen, k_new, v_new, n_new, B, n_q, Hq, Hkv, D, s, W, C, scale, out, lse, ws, n, stream)
    ok = (GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 1, 1, 1, 8, 2, 128, 4, 252, 256, 1.0, GOOD, None, GOOD, 1 << 30, None)

    def call(**kw):
        a = list(ok)
        for k, v in kw.items():
            a[int(k[1:])] = v
        return f(*a)
    assert call(a6=-1) == -1                          # n_new < 0
    assert call(a4=None) == -1                        # k_new missing with n_new > 0
    assert call(a5=BAD) == -3                         # v_new misaligned
    assert call(a3=ctypes.c_void_p(0x10004)) == -3    # ring_len not 8-byte aligned
    assert call(a10=3) == -2                          # Hq % Hkv != 0
    assert call(a13=253) == -1                        # window > capacity - n_sink
    g = lib.draft_attn_window_append_fp8
    assert g(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, 1, 1, 1, 8, 2, 128, 4, 252, 256, 1.0, -1.0, 1.0,
             GOOD, None, GOOD, 1 << 30, None) == -1   # k_scale <= 0


def test_selftest_wait_limit_checked_on_host(lib):
    f = lib.wmtp_selftest_wait_timeout
    assert f(999_999, None) == -1                 # below 1 ms
    assert f(2_000_000_001, None) == -1           # above the kernels' own 2 s limit
    assert f(0, None) == -1


def test_accept_host_checks(lib):
    a = lib.accept_greedy
    assert a(None, GOOD, None, 1, 4, 1024, GOOD, GOOD, None) == -1
    assert a(GOOD, GOOD, None, 1, 65, 1024, GOOD, GOOD, None) == -1
    assert a(GOOD, GOOD, None, 1, 4, 0, GOOD, GOOD, None) == -1
    assert a(ctypes.c_void_p(0x10002), GOOD, None, 1, 4, 1024, GOOD, GOOD, None) == -3


def test_fp8_host_checks(lib):
    w = lib.draft_attn_window_fp8
    # (q, rk, rv, rlen, B, n_q, Hq, Hkv, D, s, W, C, scale, k_scale, v_scale, out, lse, ws, n, stream)
    assert w(GOOD, GOOD, GOOD, GOOD, 1, 1, 8, 2, 128, 4, 252, 256, 1.0, 0.0, 1.0, GOOD, None, GOOD, 1 << 30, None) == -1
    assert w(GOOD, GOOD, GOOD, GOOD, 1, 1, 8, 2, 128, 4, 252, 256, 1.0, 1.0, float("inf"), GOOD, None, GOOD, 1 << 30, None) == -1
    assert w(GOOD, GOOD, GOOD, GOOD, 1, 1, 8, 3, 128, 4, 252, 256, 1.0, 1.0, 1.0, GOOD, None, GOOD, 1 << 30, None) == -2
    f = lib.draft_attn_full_fp8
    assert f(GOOD, GOOD, GOOD, GOOD, GOOD, 1, 1, 8, 2, 128, 32, 4, 4, 1.0, 1.0, 1.0, GOOD, None, GOOD, 1 << 30, None) == -2
    v = lib.verify_attn_fp8
    assert v(GOOD, GOOD, GOOD, GOOD, GOOD, BAD, 1, 4, 8, 2, 128, 64, 4, 4, 1.0, 1.0, 1.0, GOOD, None, GOOD, 1 << 30, None) == -3
    r = lib.ring_kv_append_fp8
    assert r(GOOD, GOOD, GOOD, GOOD, GOOD, 1, 1, 2, 64, 4, 256, None) == -2
    assert r(GOOD, GOOD, GOOD, GOOD, GOOD, 1, 0, 2, 128, 4, 256, None) == 0


def test_stochastic_accept_host_checks(lib):
    a = lib.accept_stochastic
    # (p, q, tokens, u_acc, u_samp, B, n_q, V, accepted, n_accepted, stream)
    assert a(GOOD, None, GOOD, None, GOOD, 1, 4, 1024, GOOD, GOOD, None) == -1       # q missing
    assert a(GOOD, GOOD, GOOD, GOOD, GOOD, 1, 65, 1024, GOOD, GOOD, None) == -1      # n_q > 64
    assert a(GOOD, GOOD, GOOD, GOOD, GOOD, 1, 4, 1 << 24, GOOD, GOOD, None) == -1    # V >= 2^24
    assert a(GOOD, GOOD, GOOD, GOOD, None, 1, 4, 1024, GOOD, GOOD, None) == -1       # u_sample
    assert a(GOOD, GOOD, ctypes.c_void_p(0x10002), GOOD, GOOD, 1, 4, 1024, GOOD, GOOD, None) == -3


def test_loop_host_checks(lib):
    r = lib.ring_kv_append_at
    # (rk, rv, rlen, k_new, v_new, pos, n_new, B, n_max, Hkv, D, s, C, stream)
    G2 = ctypes.c_void_p(0x20000)
    assert r(GOOD, GOOD, GOOD, GOOD, GOOD, G2, None, 1, 4, 2, 128, 4, 256, None) == -1   # null n_new
    assert r(GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, G2, 1, 4, 2, 128, 4, 256, None) == -1   # pos aliases ring_len
    assert r(GOOD, GOOD, GOOD, GOOD, GOOD, G2, G2, 1, 0, 2, 128, 4, 256, None) == -1     # n_max < 1
    assert r(GOOD, GOOD, GOOD, GOOD, GOOD, G2, G2, 1, 4, 2, 64, 4, 256, None) == -2      # D != 128
    assert r(GOOD, GOOD, GOOD, GOOD, GOOD, ctypes.c_void_p(0x20004), G2, 1, 4, 2, 128, 4, 256, None) == -3
    c = lib.spec_commit
    # (acc, n_acc, B, n_q, hist, max_tokens, n_tokens, append_pos, n_append, vlen, nqv, dlen, nd, s)
    assert c(GOOD, GOOD, 1, 4, None, 100, GOOD, GOOD, GOOD, None, 4, None, 0, None) == -1
    assert c(GOOD, GOOD, 1, 65, GOOD, 100, GOOD, GOOD, GOOD, None, 4, None, 0, None) == -1
    assert c(GOOD, GOOD, 1, 4, GOOD, (1 << 31) - 2, GOOD, GOOD, GOOD, None, 4, None, 0, None) == -1
    assert c(GOOD, GOOD, 1, 4, GOOD, 100, ctypes.c_void_p(0x10004), GOOD, GOOD, None, 4, None, 0, None) == -3
    d = lib.wmtp_synth_draft_tokens
    # (hist, n_tokens, B, max_tokens, gamma, V, tseed, dseed, agree24, tokens, s)
    assert d(GOOD, GOOD, 1, 100, 3, 1, 1, 2, 1 << 23, GOOD, None) == -1                  # V < 2
    assert d(GOOD, GOOD, 1, 100, 64, 1024, 1, 2, 1 << 23, GOOD, None) == -1              # gamma + 1 > 64
    assert d(GOOD, GOOD, 1, 100, 3, 1024, 1, 2, (1 << 24) + 1, GOOD, None) == -1         # agree24 > 2^24
    t = lib.wmtp_synth_target_logits
    # (hist, n_tokens, B, max_tokens, tokens, parent, n_q, V, tseed, logits, s)
    assert t(GOOD, GOOD, 1, 100, GOOD, None, 0, 1024, 1, GOOD, None) == -1
    assert t(GOOD, GOOD, 1, 100, GOOD, None, 4, 1024, 1, None, None) == -1
    assert t(GOOD, GOOD, 1, 100, GOOD, ctypes.c_void_p(0x10002), 4, 1024, 1, GOOD, None) == -3


def test_workspace_query_without_gpu_is_zero_or_positive(lib):
    # With no GPU the device query fails and the size is reported as 0 (invalid); with one, > 0.
    n = lib.wmtp_workspace_bytes(1, 1, 8, 2, 128)
    assert n >= 0
    assert lib.wmtp_workspace_bytes(1, 1, 8, 3, 128) == 0


def test_binding_fails_loudly_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libwmtp.so"))
    with pytest.raises(FileNotFoundError):
        _lib.lib()


def test_launch_counter_starts_without_launches(lib):
    assert lib.wmtp_launch_count() == 0      # host-only checks above launched nothing
