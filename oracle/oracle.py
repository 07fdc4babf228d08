"""ctypes wrapper around the fp64 CPU oracle (``liboracle.so``, built from ``oracle.c``).

TEST INFRASTRUCTURE ONLY (see the package docstring).  Arrays are numpy; bf16 tensors are
passed as their uint16 bit patterns.  Every function cites, through ``oracle.c``, the passage of
the Windowed-MTP pages it follows.
"""
import ctypes
import os

import numpy as np

from .build_oracle import LIB, build

MODE_CAUSAL = 0
MODE_WINDOW = 1
MODE_TREE = 2

_lib = None


_lib_path = LIB


def use_library(path=None):
    """Points the wrapper at another build of oracle.c (the mutation tests use this); None
    restores the default library."""
    global _lib, _lib_path
    _lib = None
    _lib_path = LIB if path is None else path


def _load():
    global _lib
    if _lib is None:
        if _lib_path == LIB and not os.path.exists(LIB):
            build()
        lib = ctypes.CDLL(_lib_path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        LL = ctypes.c_longlong
        lib.orc_ring_slot.argtypes = [LL, I, I]
        lib.orc_ring_slot.restype = LL
        lib.orc_ring_kv_append.argtypes = [P, P, P, P, P, I, I, I, I, I, I]
        lib.orc_ring_kv_append.restype = I
        lib.orc_window_member.argtypes = [LL, LL, I, I]
        lib.orc_window_member.restype = I
        lib.orc_tree_visible.argtypes = [P, I, I, I]
        lib.orc_tree_visible.restype = I
        lib.orc_key_visible.argtypes = [I, LL, I, I, LL, I, I, P]
        lib.orc_key_visible.restype = I
        lib.orc_attention.argtypes = [P, P, P, P, LL, I, I, I, I, I, I, I, I, P, ctypes.c_double,
                                      P, I, P, P, I]
        lib.orc_attention.restype = I
        lib.orc_accept_greedy.argtypes = [P, P, P, I, I, I, P, P]
        lib.orc_accept_greedy.restype = I
        lib.orc_accept_stochastic.argtypes = [P, P, P, P, P, I, I, I, P, P]
        lib.orc_accept_stochastic.restype = I
        lib.orc_e4m3_value.argtypes = [ctypes.c_uint]
        lib.orc_e4m3_value.restype = ctypes.c_double
        lib.orc_e4m3_decode.argtypes = [P, ctypes.c_size_t, P]
        lib.orc_e4m3_decode.restype = None
        lib.orc_max_threads.argtypes = []
        lib.orc_max_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def max_threads() -> int:
    return _load().orc_max_threads()


def ring_slot(p: int, n_sink: int, capacity: int) -> int:
    return _load().orc_ring_slot(int(p), int(n_sink), int(capacity))


def window_member(L_tot: int, j: int, n_sink: int, window: int) -> bool:
    return bool(_load().orc_window_member(int(L_tot), int(j), int(n_sink), int(window)))


def tree_visible(parent, i: int, j: int) -> bool:
    parent = _c(parent, np.int32)
    return bool(_load().orc_tree_visible(_ptr(parent), parent.size, int(i), int(j)))


def key_visible(mode: int, L_tot: int, n_q: int, i: int, j: int, n_sink: int = 0,
                window: int = 0, parent=None) -> bool:
    parent = None if parent is None else _c(parent, np.int32)
    return bool(_load().orc_key_visible(int(mode), int(L_tot), int(n_q), int(i), int(j),
                                        int(n_sink), int(window), _ptr(parent)))


def ring_kv_append(ring_k, ring_v, ring_len, k_new, v_new, n_sink: int):
    """In-place append.  ring_k/ring_v: uint16 [B, Hkv, C, D]; ring_len: int64 [B];
    k_new/v_new: uint16 [B, n_new, Hkv, D]."""
    for a in (ring_k, ring_v):
        assert a.dtype == np.uint16 and a.flags.c_contiguous
    assert ring_len.dtype == np.int64 and ring_len.flags.c_contiguous
    B, Hkv, C, D = ring_k.shape
    k_new = _c(k_new, np.uint16)
    v_new = _c(v_new, np.uint16)
    n_new = k_new.shape[1]
    assert k_new.shape == (B, n_new, Hkv, D) and v_new.shape == k_new.shape
    rc = _load().orc_ring_kv_append(_ptr(ring_k), _ptr(ring_v), _ptr(ring_len), _ptr(k_new),
                                    _ptr(v_new), B, n_new, Hkv, D, int(n_sink), C)
    if rc != 0:
        raise ValueError("orc_ring_kv_append: bad arguments")


def attention(q, k, v, kv_len, mode: int, sm_scale: float, n_sink: int = 0, window: int = 0,
              tree_parent=None, rows=None, n_threads: int = 0):
    """fp64 attention.  q: uint16 [B, n_q, Hq, D]; k, v: uint16 [B, Hkv, Lmax, D] (logical
    order); kv_len: [B] lengths including this call's n_q positions.  ``rows`` optionally lists
    (b, i, h) triples to compute.  Returns (out [B, n_q, Hq, D] f64, lse [B, n_q, Hq] f64);
    rows not computed are NaN."""
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    B, n_q, Hq, D = q.shape
    Bk, Hkv, Lmax, Dk = k.shape
    assert Bk == B and Dk == D and v.shape == k.shape
    kv_len = _c(kv_len, np.int64)
    parent = None if tree_parent is None else _c(tree_parent, np.int32)
    if parent is not None:
        assert parent.shape == (B, n_q)
    out = np.full((B, n_q, Hq, D), np.nan, dtype=np.float64)
    lse = np.full((B, n_q, Hq), np.nan, dtype=np.float64)
    if rows is not None:
        rows = _c(rows, np.int32).reshape(-1, 3)
        n_rows = rows.shape[0]
    else:
        n_rows = 0
    rc = _load().orc_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_len), Lmax, B, n_q, Hq, Hkv, D,
                               int(mode), int(n_sink), int(window), _ptr(parent), float(sm_scale),
                               _ptr(rows), n_rows, _ptr(out), _ptr(lse), int(n_threads))
    if rc != 0:
        raise ValueError("orc_attention: bad arguments")
    return out, lse


def accept_greedy(logits, tokens, tree_parent=None):
    """logits: f32 [B, n_q, V]; tokens: int32 [B, n_q]; tree_parent: int32 [B, n_q] or None.
    Returns (accepted int32 [B, n_q] padded with -1, n_accepted int32 [B])."""
    logits = _c(logits, np.float32)
    tokens = _c(tokens, np.int32)
    B, n_q, V = logits.shape
    parent = None if tree_parent is None else _c(tree_parent, np.int32)
    accepted = np.empty((B, n_q), dtype=np.int32)
    n_acc = np.empty((B,), dtype=np.int32)
    rc = _load().orc_accept_greedy(_ptr(logits), _ptr(tokens), _ptr(parent), B, n_q, V,
                                   _ptr(accepted), _ptr(n_acc))
    if rc != 0:
        raise ValueError("orc_accept_greedy: bad arguments")
    return accepted, n_acc


def accept_stochastic(p, q, tokens, u_accept, u_sample):
    """Rejection-sampling acceptance of drafted chains.  p: f32 [B, n_q, V] target
    probabilities; q: f32 [B, n_q - 1, V] draft probabilities; tokens: int32 [B, n_q];
    u_accept: uint32 [B, n_q - 1] (< 2^24); u_sample: uint32 [B].  Returns (accepted int32
    [B, n_q] padded with -1, n_accepted int32 [B])."""
    p = _c(p, np.float32)
    tokens = _c(tokens, np.int32)
    B, n_q, V = p.shape
    q = _c(q, np.float32).reshape(B, n_q - 1, V)
    u_accept = _c(u_accept, np.uint32).reshape(B, n_q - 1)
    u_sample = _c(u_sample, np.uint32).reshape(B)
    assert tokens.shape == (B, n_q)
    accepted = np.empty((B, n_q), dtype=np.int32)
    n_acc = np.empty((B,), dtype=np.int32)
    rc = _load().orc_accept_stochastic(_ptr(p), _ptr(q), _ptr(tokens), _ptr(u_accept), _ptr(u_sample),
                                       B, n_q, V, _ptr(accepted), _ptr(n_acc))
    if rc != 0:
        raise ValueError("orc_accept_stochastic: bad arguments")
    return accepted, n_acc


def e4m3_value(code: int) -> float:
    """The value of one OCP E4M3 code (NaN for S.1111.111)."""
    return float(_load().orc_e4m3_value(int(code) & 0xFF))


def e4m3_decode(codes) -> np.ndarray:
    """float64 values of an array of E4M3 codes (uint8), same shape."""
    codes = _c(codes, np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    _load().orc_e4m3_decode(_ptr(codes), codes.size, _ptr(out))
    return out


def _f64_to_bf16_bits_exact(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of float64 values that bf16 represents exactly (every finite E4M3
    value does: 3 mantissa bits, exponents -9 .. 8); NaN stays NaN."""
    f = x.astype(np.float32)
    bits = f.view(np.uint32)
    assert not np.any((bits & 0xFFFF)[np.isfinite(f)]), "value not exactly representable in bf16"
    return (bits >> 16).astype(np.uint16)


def attention_kv8(q, k8, v8, kv_len, mode: int, sm_scale: float, k_scale: float, v_scale: float,
                  n_sink: int = 0, window: int = 0, tree_parent=None, rows=None, n_threads: int = 0):
    """attention() over fp8 (E4M3) keys and values: key = k_scale * e4m3(k8), value =
    v_scale * e4m3(v8).  k8, v8: uint8 [B, Hkv, Lmax, D] in logical order.  The decoded codes are
    exact bf16 values, the key scale multiplies every score (folded into sm_scale) and the value
    scale every output, so this is the fp64 definition on the dequantised cache."""
    kb = _f64_to_bf16_bits_exact(e4m3_decode(k8))
    vb = _f64_to_bf16_bits_exact(e4m3_decode(v8))
    out, lse = attention(q, kb, vb, kv_len, mode, float(sm_scale) * float(k_scale), n_sink=n_sink,
                         window=window, tree_parent=tree_parent, rows=rows, n_threads=n_threads)
    return out * float(v_scale), lse
