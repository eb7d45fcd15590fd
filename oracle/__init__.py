"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's cpu_baseline and
reference legs use this package.  The CUDA library never imports, links or
calls it, and it shares no code with the CUDA library: the arithmetic lives in
``attn_oracle.c`` (plain C, fp64, OpenMP over output rows), and this module is
ctypes marshalling only.

Every entry here states what it computes and which page passage it follows;
see the header of ``attn_oracle.c`` for the full list of readings (scale,
bottom-right causal alignment, grouped-head mapping, empty rows, LSE).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_dp = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_fp = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_u8 = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_i64 = np.ctypeslib.ndpointer(dtype=np.int64, flags="C_CONTIGUOUS")
_I = ctypes.c_int
_LL = ctypes.c_longlong


def build(force: bool = False) -> str:
    """Compile attn_oracle.c with gcc into liboracle.so (fp64, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.oracle_attn_fwd.argtypes = [_dp, _dp, _dp, _dp, _dp] + [_I] * 7 + [ctypes.c_double]
        L.oracle_attn_fwd.restype = _I
        L.oracle_attn_fwd_rows.argtypes = ([_dp, _dp, _dp, _dp, _dp] + [_I] * 7 +
                                           [ctypes.c_double, _i64, _LL])
        L.oracle_attn_fwd_rows.restype = _I
        L.oracle_attn_online.argtypes = ([_dp, _dp, _dp, _dp, _dp] + [_I] * 7 +
                                         [ctypes.c_double, _I, ctypes.c_double,
                                          ctypes.POINTER(_LL)])
        L.oracle_attn_online.restype = _I
        L.oracle_attn_fwd_window.argtypes = ([_dp, _dp, _dp, _dp, _dp] + [_I] * 7 +
                                             [ctypes.c_double, _LL, _LL])
        L.oracle_attn_fwd_window.restype = _I
        L.oracle_combine.argtypes = [_dp, _dp, _I, _LL, _I, _dp, _dp]
        L.oracle_combine.restype = _I
        L.oracle_gemm_add.argtypes = [_dp, _dp, ctypes.c_void_p, _dp, _LL, _LL, _LL]
        L.oracle_gemm_add.restype = _I
        L.oracle_attn_bruteforce.argtypes = [_dp, _dp, _dp, _dp, _dp] + [_I] * 7 + [ctypes.c_double]
        L.oracle_attn_bruteforce.restype = _I
        L.oracle_mask.argtypes = [_I, _I, _I, _u8]
        L.oracle_mask.restype = None
        L.oracle_hadamard.argtypes = [_I, _dp, _dp]
        L.oracle_hadamard.restype = _I
        L.oracle_rotate_rows.argtypes = [_dp, _LL, _I, _dp, _dp]
        L.oracle_rotate_rows.restype = _I
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.oracle_e4m3_encode.restype = ctypes.c_uint
        L.oracle_e4m3_encode_array.argtypes = [_dp, _LL, _u8]
        L.oracle_e4m3_encode_array.restype = None
        L.oracle_e4m3_decode_array.argtypes = [_u8, _LL, _dp]
        L.oracle_e4m3_decode_array.restype = None
        L.oracle_quant_e4m3_f32.argtypes = [_fp, _LL, ctypes.c_float, _u8]
        L.oracle_quant_e4m3_f32.restype = None
        _lib = L
    return _lib


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _shape(q, k, Hkv):
    B, Nq, Hq, d = q.shape
    Bk, Nk, Hk, dk = k.shape
    assert (B, d) == (Bk, dk) and Hk == Hkv
    return B, Nq, Hq, d, Nk


def attn_fwd(q, k, v, causal: bool, scale: float):
    """Two-pass exact attention (the definition).  q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d] fp64.
    Returns O [B,Nq,Hq,d] and LSE [B,Hq,Nq] (natural log of the scaled scores)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d, Nk = _shape(q, k, k.shape[2])
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Nq))
    rc = lib().oracle_attn_fwd(q, k, v, o, lse, B, Hq, k.shape[2], Nq, Nk, d, int(causal), scale)
    if rc:
        raise ValueError(f"oracle_attn_fwd failed ({rc})")
    return o, lse


def attn_fwd_window(q, k, v, causal: bool, scale: float, k0: int, k1: int):
    """The definition over the keys [k0, k1) only (causal rule in absolute key
    indices): one window's partial result.  Returns O [B,Nq,Hq,d], LSE [B,Hq,Nq];
    rows with no allowed key in the window get O = 0, LSE = -inf."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d, Nk = _shape(q, k, k.shape[2])
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Nq))
    rc = lib().oracle_attn_fwd_window(q, k, v, o, lse, B, Hq, k.shape[2], Nq, Nk, d, int(causal), scale,
                                      int(k0), int(k1))
    if rc:
        raise ValueError(f"oracle_attn_fwd_window failed ({rc})")
    return o, lse


def gemm_add(a, b, c=None):
    """D = A B + C in fp64: a [M, K], b [K, N], c [M, N] or None."""
    a, b = _f64(a), _f64(b)
    M, K = a.shape
    K2, N = b.shape
    if K2 != K:
        raise ValueError("inner sizes differ")
    cc = None if c is None else _f64(c)
    d = np.zeros((M, N))
    cptr = None if cc is None else cc.ctypes.data_as(ctypes.c_void_p)
    if lib().oracle_gemm_add(a, b, cptr, d, M, N, K):
        raise ValueError("oracle_gemm_add failed")
    return d


def combine(o_parts, lse_parts):
    """Merge S partial results: o_parts [S, ..., d] and lse_parts [S, ...] with
    matching row order.  Returns O [..., d] and LSE [...]."""
    o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
    S, d = o_parts.shape[0], o_parts.shape[-1]
    R = int(np.prod(o_parts.shape[1:-1]))
    if lse_parts.shape[0] != S or int(np.prod(lse_parts.shape[1:])) != R:
        raise ValueError("o_parts / lse_parts shapes do not match")
    o = np.zeros(o_parts.shape[1:])
    lse = np.zeros(lse_parts.shape[1:])
    if lib().oracle_combine(o_parts, lse_parts, S, R, d, o, lse):
        raise ValueError("oracle_combine failed")
    return o, lse


def combine_bnhd(o_parts, lse_parts):
    """combine() for the library's partial layouts: o_parts [S,B,Nq,Hq,d],
    lse_parts [S,B,Hq,Nq].  Returns O [B,Nq,Hq,d] and LSE [B,Hq,Nq]."""
    lse_rows = np.ascontiguousarray(np.transpose(_f64(lse_parts), (0, 1, 3, 2)))  # [S,B,Nq,Hq]
    o, lse = combine(o_parts, lse_rows)
    return o, np.ascontiguousarray(np.transpose(lse, (0, 2, 1)))


def attn_fwd_rows(q, k, v, causal: bool, scale: float, rows):
    """The definition for selected rows only; rows are flat (b*Hq + h)*Nq + i.
    Returns O [n, d] and LSE [n]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d, Nk = _shape(q, k, k.shape[2])
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    o = np.zeros((rows.size, d))
    lse = np.zeros(rows.size)
    rc = lib().oracle_attn_fwd_rows(q, k, v, o, lse, B, Hq, k.shape[2], Nq, Nk, d, int(causal),
                                    scale, rows, rows.size)
    if rc:
        raise ValueError(f"oracle_attn_fwd_rows failed ({rc})")
    return o, lse


def attn_online(q, k, v, causal: bool, scale: float, block: int, tau: float = 0.0):
    """Blockwise online-softmax recurrence; tau (natural-log units) is the lazy
    threshold on moving the reference max.  Returns O, LSE, number of rescales."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d, Nk = _shape(q, k, k.shape[2])
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Nq))
    n = _LL(0)
    rc = lib().oracle_attn_online(q, k, v, o, lse, B, Hq, k.shape[2], Nq, Nk, d, int(causal),
                                  scale, block, tau, ctypes.byref(n))
    if rc:
        raise ValueError(f"oracle_attn_online failed ({rc})")
    return o, lse, n.value


def attn_bruteforce(q, k, v, causal: bool, scale: float):
    """Long-double brute force for Nk <= 64 (materialised S, no max subtraction)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d, Nk = _shape(q, k, k.shape[2])
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Nq))
    rc = lib().oracle_attn_bruteforce(q, k, v, o, lse, B, Hq, k.shape[2], Nq, Nk, d,
                                      int(causal), scale)
    if rc:
        raise ValueError(f"oracle_attn_bruteforce failed ({rc})")
    return o, lse


def mask(Nq: int, Nk: int, causal: bool) -> np.ndarray:
    """Elementwise allowed(i, j) as a bool [Nq, Nk] array."""
    m = np.zeros((Nq, Nk), dtype=np.uint8)
    lib().oracle_mask(Nq, Nk, int(causal), m)
    return m.astype(bool)


def hadamard(d: int, signs) -> np.ndarray:
    """M = diag(signs) H_d / sqrt(d), d x d fp64."""
    M = np.zeros((d, d))
    if lib().oracle_hadamard(d, _f64(signs), M):
        raise ValueError("d must be a power of two")
    return M


def rotate_rows(x, M) -> np.ndarray:
    """Y = X M for X [..., d] (last axis rotated)."""
    x = _f64(x)
    d = x.shape[-1]
    y = np.zeros_like(x)
    lib().oracle_rotate_rows(x, x.size // d, d, _f64(M), y)
    return y


def e4m3_decode(codes) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.zeros(c.shape)
    lib().oracle_e4m3_decode_array(c.reshape(-1), c.size, out.reshape(-1))
    return out


def e4m3_encode(x) -> np.ndarray:
    x = _f64(x)
    out = np.zeros(x.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(x.reshape(-1), x.size, out.reshape(-1))
    return out


def quant_e4m3_f32(x_f32, amax: float) -> np.ndarray:
    """Per-tensor quantisation in fp32: code = E4M3(x * (448/amax))."""
    x = np.ascontiguousarray(x_f32, dtype=np.float32)
    out = np.zeros(x.shape, dtype=np.uint8)
    lib().oracle_quant_e4m3_f32(x.reshape(-1), x.size, np.float32(amax), out.reshape(-1))
    return out


def fp8_prepare(x_f64, signs=None):
    """The FP8 input preparation of page "FlashAttention-3 — 闪电注意力-3" section 3,
    in fp64: optional rotation x M, per-tensor amax, descale = amax/448, codes =
    E4M3(x / descale).  Returns (codes uint8, descale float)."""
    x = _f64(x_f64)
    if signs is not None:
        x = rotate_rows(x, hadamard(x.shape[-1], signs))
    amax = float(np.max(np.abs(x)))
    descale = amax / 448.0
    return e4m3_encode(x / descale), descale
