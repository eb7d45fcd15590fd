"""Python binding of libattn, the sm_100a fused exact-attention forward.

Each function here has the name of a C entry point in ``include/attn.h`` and
only marshals arguments (tensor -> device pointer, stream -> handle) before
calling into ``libattn.so``; every step of the computation runs in the CUDA
kernels.  There is no fallback: if the shared library is missing or cannot be
loaded, importing this package raises.

``attention()`` is a convenience wrapper that allocates the outputs with
PyTorch and calls ``attn_fwd``.
"""
from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "ATTN_BF16", "ATTN_FP8_E4M3", "AttnError", "attn_fwd", "attn_fwd_fp8", "attn_hadamard_quant_fp8",
    "attn_hadamard_quant_fp8_workspace_bytes", "attn_get_last_device_error", "attn_status_string",
    "attn_kv_tile_count", "attn_tile_kind", "attn_debug_unsatisfied_wait", "attn_debug_exp2", "attention",
    "attn_fwd_schedule", "attn_hadamard_quant_fp8_noalloc", "attn_fwd_splitkv", "attn_splitkv_workspace_bytes",
    "attn_combine", "attn_kv_tile_count_window", "attn_tile_kind_window", "attn_gemm_add", "lib_path", "EXPORTS",
    "attn_debug_map_cache_stats", "attn_fwd_part", "attn_shard_units", "attention_shard", "attn_fwd_host",
]

ATTN_BF16 = 0
ATTN_FP8_E4M3 = 1
STATUS = {0: "ATTN_OK", 1: "ATTN_ERR_INVALID_ARG", 2: "ATTN_ERR_UNSUPPORTED", 3: "ATTN_ERR_MISALIGNED",
          4: "ATTN_ERR_CUDA", 5: "ATTN_ERR_DEVICE_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libattn.so")

# every symbol include/attn.h declares
EXPORTS = (
    "attn_fwd", "attn_fwd_fp8", "attn_hadamard_quant_fp8", "attn_hadamard_quant_fp8_workspace_bytes",
    "attn_get_last_device_error", "attn_status_string", "attn_kv_tile_count", "attn_tile_kind",
    "attn_debug_unsatisfied_wait", "attn_debug_exp2", "attn_hadamard_quant_fp8_noalloc", "attn_fwd_schedule",
    "attn_fwd_splitkv", "attn_splitkv_workspace_bytes", "attn_combine", "attn_kv_tile_count_window",
    "attn_tile_kind_window", "attn_gemm_add", "attn_debug_map_cache_stats", "attn_fwd_part", "attn_shard_units",
    "attn_fwd_host",
)

if not os.path.exists(lib_path):
    raise ImportError(f"libattn.so is not built ({lib_path}); run `python exact_attention_140_b200/build.py` "
                      "or __graft_entry__.build()")
_lib = ctypes.CDLL(lib_path)

_vp, _I, _LL, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
_lib.attn_fwd.argtypes = [_vp] * 5 + [_I] * 7 + [_F, _I, _vp]
_lib.attn_fwd.restype = _I
_lib.attn_fwd_part.argtypes = [_vp] * 5 + [_I] * 7 + [_F, _I] + [_I] * 4 + [_vp]
_lib.attn_fwd_part.restype = _I
_lib.attn_shard_units.argtypes = [_I] * 4 + [ctypes.POINTER(_I)]
_lib.attn_fwd_host.argtypes = [_vp] * 10 + [_I] * 7 + [_F, _I, _vp]
_lib.attn_fwd_host.restype = _I
_lib.attn_shard_units.restype = _I
_lib.attn_fwd_fp8.argtypes = [_vp] * 5 + [_I] * 7 + [_F, _vp, _vp, _vp, _vp]
_lib.attn_fwd_fp8.restype = _I
_lib.attn_hadamard_quant_fp8.argtypes = [_vp, _vp, _vp, _vp, _LL, _I, _vp, _vp]
_lib.attn_hadamard_quant_fp8.restype = _I
_lib.attn_hadamard_quant_fp8_noalloc.argtypes = [_vp, _vp, _vp, _LL, _I, _vp, _vp]
_lib.attn_hadamard_quant_fp8_noalloc.restype = _I
_lib.attn_hadamard_quant_fp8_workspace_bytes.argtypes = []
_lib.attn_hadamard_quant_fp8_workspace_bytes.restype = _LL
_lib.attn_get_last_device_error.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint)]
_lib.attn_get_last_device_error.restype = _I
_lib.attn_status_string.argtypes = [_I]
_lib.attn_status_string.restype = ctypes.c_char_p
_lib.attn_kv_tile_count.argtypes = [_I] * 6
_lib.attn_kv_tile_count.restype = _I
_lib.attn_tile_kind.argtypes = [_I] * 7
_lib.attn_tile_kind.restype = _I
_lib.attn_fwd_schedule.argtypes = [_I] * 3
_lib.attn_fwd_schedule.restype = _I
_lib.attn_debug_unsatisfied_wait.argtypes = [_LL, _vp]
_lib.attn_debug_unsatisfied_wait.restype = _I
_lib.attn_debug_exp2.argtypes = [_vp, _vp, _LL, _I, _vp]
_lib.attn_debug_exp2.restype = _I
_lib.attn_splitkv_workspace_bytes.argtypes = [_I] * 7
_lib.attn_splitkv_workspace_bytes.restype = _LL
_lib.attn_fwd_splitkv.argtypes = [_vp] * 5 + [_I] * 7 + [_F, _I, _vp, _LL, _vp]
_lib.attn_fwd_splitkv.restype = _I
_lib.attn_combine.argtypes = [_vp, _vp] + [_I] * 5 + [_vp, _vp, _vp]
_lib.attn_combine.restype = _I
_lib.attn_kv_tile_count_window.argtypes = [_I] * 7
_lib.attn_kv_tile_count_window.restype = _I
_lib.attn_tile_kind_window.argtypes = [_I] * 8
_lib.attn_tile_kind_window.restype = _I
_lib.attn_gemm_add.argtypes = [_vp] * 4 + [_I] * 3 + [_vp]
_lib.attn_gemm_add.restype = _I
_lib.attn_debug_map_cache_stats.argtypes = [ctypes.POINTER(ctypes.c_ulonglong)] * 2
_lib.attn_debug_map_cache_stats.restype = _I


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({attn_status_string(status)})")


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int, where: str, raise_on_error: bool):
    if rc != 0 and raise_on_error:
        raise AttnError(rc, where)
    return rc


def attn_status_string(status: int) -> str:
    return _lib.attn_status_string(int(status)).decode()


def attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, dtype=ATTN_BF16, stream=None,
             raise_on_error=True):
    rc = _lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d, int(causal),
                       float(scale), int(dtype), _stream(stream))
    return _check(rc, "attn_fwd", raise_on_error)


def attn_fwd_part(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, dtype, b_begin, b_end, kvh_begin,
                  kvh_end, stream=None, raise_on_error=True):
    rc = _lib.attn_fwd_part(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d, int(causal),
                            float(scale), int(dtype), int(b_begin), int(b_end), int(kvh_begin), int(kvh_end),
                            _stream(stream))
    return _check(rc, "attn_fwd_part", raise_on_error)


def attn_fwd_host(q_h, k_h, v_h, o_h, lse_h, q_d, k_d, v_d, o_d, lse_d, B, Hq, Hkv, Nq, Nk, d, causal, scale,
                  n_chunks=0, stream=None, raise_on_error=True):
    """attn_fwd with host inputs/outputs (pinned for overlap) and caller-owned
    device buffers; the copies in, kernels and copies out are pipelined over
    n_chunks runs of (batch, key/value head) units (0: the library's default)."""
    rc = _lib.attn_fwd_host(_ptr(q_h), _ptr(k_h), _ptr(v_h), _ptr(o_h), _ptr(lse_h), _ptr(q_d), _ptr(k_d),
                            _ptr(v_d), _ptr(o_d), _ptr(lse_d), B, Hq, Hkv, Nq, Nk, d, int(causal), float(scale),
                            int(n_chunks), _stream(stream))
    return _check(rc, "attn_fwd_host", raise_on_error)


def attn_shard_units(B, Hkv, world, rank):
    """Rank `rank`'s share of the B x Hkv (batch, key/value head) units as a list
    of (b_begin, b_end, kvh_begin, kvh_end) rectangles."""
    buf = (_I * 12)()
    n = _lib.attn_shard_units(int(B), int(Hkv), int(world), int(rank), buf)
    if n < 0:
        raise AttnError(1, "attn_shard_units")
    return [tuple(buf[4 * i:4 * i + 4]) for i in range(n)]


def attention_shard(q, k, v, o, lse, rank, world, causal=False, scale=None, stream=None):
    """This rank's share of attention over full bf16 tensors q [B,Nq,Hq,d],
    k/v [B,Nk,Hkv,d] into o/lse (the other ranks' rows are not written);
    returns the rectangles computed."""
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rects = attn_shard_units(B, Hkv, world, rank)
    for (b0, b1, g0, g1) in rects:
        attn_fwd_part(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, ATTN_BF16, b0, b1, g0, g1, stream)
    return rects


def attn_splitkv_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, n_splits=0) -> int:
    return int(_lib.attn_splitkv_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, n_splits))


def attn_fwd_splitkv(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, n_splits, workspace, workspace_bytes,
                     stream=None, raise_on_error=True):
    rc = _lib.attn_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d, int(causal),
                               float(scale), int(n_splits), _ptr(workspace), int(workspace_bytes), _stream(stream))
    return _check(rc, "attn_fwd_splitkv", raise_on_error)


def attn_combine(o_parts, lse_parts, n_splits, B, Hq, Nq, d, o, lse, stream=None, raise_on_error=True):
    rc = _lib.attn_combine(_ptr(o_parts), _ptr(lse_parts), n_splits, B, Hq, Nq, d, _ptr(o), _ptr(lse),
                           _stream(stream))
    return _check(rc, "attn_combine", raise_on_error)


def attn_gemm_add(a, b, c, d, M, N, K, stream=None, raise_on_error=True):
    rc = _lib.attn_gemm_add(_ptr(a), _ptr(b), _ptr(c), _ptr(d), M, N, K, _stream(stream))
    return _check(rc, "attn_gemm_add", raise_on_error)


def attn_fwd_fp8(q8, k8, v8, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, descale_q, descale_k, descale_v,
                 stream=None, raise_on_error=True):
    rc = _lib.attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d, int(causal),
                           float(scale), _ptr(descale_q), _ptr(descale_k), _ptr(descale_v), _stream(stream))
    return _check(rc, "attn_fwd_fp8", raise_on_error)


def attn_hadamard_quant_fp8_workspace_bytes() -> int:
    return int(_lib.attn_hadamard_quant_fp8_workspace_bytes())


def attn_hadamard_quant_fp8(x, x8, descale, workspace, rows, d, signs=None, stream=None, raise_on_error=True):
    rc = _lib.attn_hadamard_quant_fp8(_ptr(x), _ptr(x8), _ptr(descale), _ptr(workspace), int(rows), int(d),
                                      _ptr(signs), _stream(stream))
    return _check(rc, "attn_hadamard_quant_fp8", raise_on_error)


def attn_hadamard_quant_fp8_noalloc(x, x8, descale, rows, d, signs=None, stream=None, raise_on_error=True):
    """attn_hadamard_quant_fp8 with the library's own static scratch (no workspace)."""
    rc = _lib.attn_hadamard_quant_fp8_noalloc(_ptr(x), _ptr(x8), _ptr(descale), int(rows), int(d), _ptr(signs),
                                              _stream(stream))
    return _check(rc, "attn_hadamard_quant_fp8_noalloc", raise_on_error)


def attn_get_last_device_error(stream=None):
    """Returns (status, raw error word); synchronises the stream."""
    w = ctypes.c_uint(0)
    rc = _lib.attn_get_last_device_error(_stream(stream), ctypes.byref(w))
    return rc, w.value


def attn_kv_tile_count(row0, row1, Nq, Nk, bn, causal) -> int:
    return int(_lib.attn_kv_tile_count(row0, row1, Nq, Nk, bn, int(causal)))


def attn_tile_kind(row0, row1, kt, Nq, Nk, bn, causal) -> int:
    return int(_lib.attn_tile_kind(row0, row1, kt, Nq, Nk, bn, int(causal)))


def attn_kv_tile_count_window(row0, row1, Nq, Nk, shift, bn, causal) -> int:
    return int(_lib.attn_kv_tile_count_window(row0, row1, Nq, Nk, shift, bn, int(causal)))


def attn_tile_kind_window(row0, row1, kt, Nq, Nk, shift, bn, causal) -> int:
    return int(_lib.attn_tile_kind_window(row0, row1, kt, Nq, Nk, shift, bn, int(causal)))


def attn_fwd_schedule(Nk, d, causal) -> int:
    """1 if attn_fwd runs the persistent kernel for Nk keys at head size d, 0 for one block per item."""
    return int(_lib.attn_fwd_schedule(Nk, d, int(causal)))


def attn_debug_unsatisfied_wait(limit_ns: int, stream=None, raise_on_error=True):
    rc = _lib.attn_debug_unsatisfied_wait(int(limit_ns), _stream(stream))
    return _check(rc, "attn_debug_unsatisfied_wait", raise_on_error)


def attn_debug_map_cache_stats():
    """(hits, encodes) of the library's tensor-map cache."""
    h, e = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    _check(_lib.attn_debug_map_cache_stats(ctypes.byref(h), ctypes.byref(e)), "attn_debug_map_cache_stats", True)
    return h.value, e.value


def attn_debug_exp2(x, y, n, mode, stream=None, raise_on_error=True):
    rc = _lib.attn_debug_exp2(_ptr(x), _ptr(y), int(n), int(mode), _stream(stream))
    return _check(rc, "attn_debug_exp2", raise_on_error)


def attention(q, k, v, causal: bool = False, scale: float | None = None, return_lse: bool = True, stream=None):
    """O, LSE for torch tensors q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d] (bf16, CUDA, contiguous)."""
    import torch
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("attention() takes bf16 tensors; use attn_fwd_fp8 for e4m3")
    for t in (q, k, v):
        if not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous")
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if return_lse else None
    attn_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, causal, scale, ATTN_BF16, stream)
    return (o, lse) if return_lse else o
