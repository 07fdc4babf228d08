"""ctypes loader for the in-tree libwmtp.so (the C ABI declared in include/wmtp.h).

The library must exist: there is no fallback.  Loading raises when it is missing.
"""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libwmtp.so")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")
HEADER = os.path.join(INCLUDE, "wmtp.h")
HEADERS = sorted(os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h"))

STATUS = {
    0: "WMTP_OK", -1: "WMTP_ERR_ARG", -2: "WMTP_ERR_SHAPE", -3: "WMTP_ERR_ALIGN",
    -4: "WMTP_ERR_WORKSPACE", -5: "WMTP_ERR_CUDA", -6: "WMTP_ERR_DEVICE_INDEX",
    -7: "WMTP_ERR_UNSUPPORTED", -8: "WMTP_ERR_TIMEOUT", -9: "WMTP_ERR_SCRATCH_LIMIT",
}


class WmtpError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status_string(status)})")


_lib = None

P = ctypes.c_void_p
I = ctypes.c_int
F = ctypes.c_float
SZ = ctypes.c_size_t
I64 = ctypes.c_int64
U64 = ctypes.c_uint64
U32 = ctypes.c_uint32

_SIGNATURES = {
    "wmtp_status_string": ([I], ctypes.c_char_p),
    "wmtp_workspace_bytes": ([I, I, I, I, I], SZ),
    "ring_kv_append": ([P, P, P, P, P, I, I, I, I, I, I, P], I),
    "draft_attn_window": ([P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, SZ, P], I),
    "draft_attn_full": ([P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, SZ, P], I),
    "verify_attn": ([P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, SZ, P], I),
    "accept_greedy": ([P, P, P, I, I, I, P, P, P], I),
    "wmtp_device_status": ([P], I),
    "wmtp_launch_count": ([], ctypes.c_uint64),
    "wmtp_selftest_wait_timeout": ([ctypes.c_uint64, P], I),
    "draft_attn_window_append": ([P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, F, P, P, P, SZ, P], I),
    "draft_attn_window_append_fp8": ([P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, F, F, F, P, P, P, SZ, P], I),
    "draft_attn_window_noalloc": ([P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P], I),
    "accept_stochastic": ([P, P, P, P, P, I, I, I, P, P, P], I),
    "ring_kv_append_fp8": ([P, P, P, P, P, I, I, I, I, I, I, P], I),
    "draft_attn_window_fp8": ([P, P, P, P, I, I, I, I, I, I, I, I, F, F, F, P, P, P, SZ, P], I),
    "draft_attn_full_fp8": ([P, P, P, P, P, I, I, I, I, I, I, I, I, F, F, F, P, P, P, SZ, P], I),
    "verify_attn_fp8": ([P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, F, F, P, P, P, SZ, P], I),
    "ring_kv_append_at": ([P, P, P, P, P, P, P, I, I, I, I, I, I, P], I),
    "spec_commit": ([P, P, I, I, P, I64, P, P, P, P, I, P, I, P], I),
    "wmtp_synth_draft_tokens": ([P, P, I, I64, I, I, U64, U64, U32, P, P], I),
    "wmtp_synth_target_logits": ([P, P, I, I64, P, P, I, I, U64, P, P], I),
}


def lib() -> ctypes.CDLL:
    """The loaded library (raises FileNotFoundError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise FileNotFoundError(
                f"{LIB_PATH} is missing: build it with `python -m long_context_speculative_kv_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            f = getattr(l, name)
            f.argtypes = args
            f.restype = res
        _lib = l
    return _lib


def status_string(status: int) -> str:
    return lib().wmtp_status_string(int(status)).decode()


def check(fn: str, status: int) -> None:
    if status != 0:
        raise WmtpError(fn, status)
