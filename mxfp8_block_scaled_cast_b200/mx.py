"""Thin ctypes binding of libmx (include/mx.h).

Argument marshalling only: every function named ``mx_*`` here passes device
pointers of caller-owned torch tensors, sizes and the current CUDA stream to
the C entry point of the same name and raises ``MXError`` on a non-zero
status. The convenience wrappers (``cast_dim0`` ...) only allocate the output
tensors with torch and call those. No computation happens in Python and there
is no fallback: if libmx.so is missing or no GPU is present, calls raise.
"""
from __future__ import annotations

import ctypes
import itertools
import os
import weakref

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmx.so")

_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t

# name -> (restype, argtypes); the table mirrors include/mx.h
_SIGNATURES = {
    "mx_last_error": (ctypes.c_char_p, []),
    "mx_scale_bytes": (_sz, [_i64, _i64]),
    "mx_padded_rows_capacity": (_i64, [_i64, _i32]),
    "mx_device_error": (ctypes.c_int, [_vp]),
    "mx_cast_dim0": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "mx_cast_dim1": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "mx_cast_2d": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "mx_cast_w32x32": (ctypes.c_int, [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "mx_cast_dim0_grouped": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i32, _i64, _vp, _vp, _vp]),
    "mx_cast_dim1_grouped": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i32, _i64, _vp, _vp, _vp]),
    "mx_cast_2d_grouped": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i32, _i64, _vp, _vp, _vp, _vp, _vp]),
    "mx_cast_dim0_grouped_scatter": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i32, _i64, ctypes.POINTER(_vp),
                                                    ctypes.POINTER(_vp), _vp]),
    "mx_cast_2d_grouped_scatter": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i32, _i64, ctypes.POINTER(_vp),
                                                  ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                                  ctypes.POINTER(_i64), _vp]),
    "mx_grouped_mm": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i64, _i64, _i64, _i64, _vp]),
    "mx_grouped_mm_experts": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _i64, _i64, _i64,
                                             _i64, _vp]),
    "mx_grouped_mm_experts_to_rows": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                                     ctypes.POINTER(_vp), _i64, _i64, _i64, _i64, _vp]),
    "mx_wcache_create": (_vp, []),
    "mx_wcache_evict": (None, [_vp, _vp]),
    "mx_wcache_clear": (None, [_vp]),
    "mx_wcache_destroy": (None, [_vp]),
    "mx_wcache_stats": (ctypes.c_int, [_vp, ctypes.POINTER(_i64), ctypes.POINTER(_i64), ctypes.POINTER(_i64)]),
    "mx_linear_ws_bytes": (_sz, [_i64, _i64, _i64]),
    "mx_linear_fwd": (ctypes.c_int, [_vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_uint64, _vp, _vp, _sz, _vp]),
    "mx_linear_bwd": (ctypes.c_int, [_vp, _vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_uint64, _vp, _vp, _vp, _sz,
                                     _vp]),
    "mx_linear_fwd_noalloc": (ctypes.c_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp]),
    "mx_linear_train_ws_bytes": (_sz, [_i64, _i64, _i64]),
    "mx_linear_fwd_train": (ctypes.c_int, [_vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_uint64, _vp, _vp, _sz, _vp]),
    "mx_linear_bwd_after_fwd": (ctypes.c_int, [_vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_uint64, _vp, _vp, _vp,
                                               _sz, _vp]),
    "mx_cast_ex": (ctypes.c_int, [_vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "mx_grouped_mm_bf16": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i32, _vp, _i64, _i64, _i64, _vp]),
    "mx_dequant_dim0": (ctypes.c_int, [_vp, _vp, _i64, _i64, _i64, _vp, _vp]),
    "mx_dequant_dim0_grouped": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i64, _i64, _i64, _vp, _vp]),
    "mx_scales_unswizzle": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp]),
    "mx_selftest_wait_timeout": (ctypes.c_int, [_vp]),
}

MX_RCEIL = 0
MX_FLOOR = 1

# size of the library's fixed scratch array used by mx_linear_fwd_noalloc
MX_LINEAR_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024

MX_GROUPS_M = 0
MX_GROUPS_K = 1
MX_GROUPS_M_KN = 2

_lib = None


class MXError(RuntimeError):
    def __init__(self, name, status, detail):
        super().__init__(f"{name} failed with status {status}: {detail}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libmx (loaded once; raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m mxfp8_block_scaled_cast_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def exported_names():
    return list(_SIGNATURES)


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_raw_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream(stream=None):
    """cudaStream_t of `stream`, or of the current stream (read without building a Stream object)."""
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    if _raw_stream is not None and _raw_device is not None:
        return ctypes.c_void_p(_raw_stream(_raw_device()))
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmx takes device tensors only")
    if not t.is_contiguous():
        raise ValueError("libmx takes contiguous tensors only (call .contiguous() first)")
    return ctypes.c_void_p(t.data_ptr())


def _call(name, *args):
    status = getattr(lib(), name)(*args)
    if status != 0:
        raise MXError(name, status, lib().mx_last_error().decode())


# ------------------------------------------------------------ raw entries --
def mx_scale_bytes(rows, cols) -> int:
    return int(lib().mx_scale_bytes(rows, cols))


def mx_padded_rows_capacity(m_total, groups) -> int:
    return int(lib().mx_padded_rows_capacity(m_total, groups))


def mx_device_error(stream=None):
    _call("mx_device_error", _stream(stream))


def mx_cast_dim0(x, q, s, stream=None):
    R, C = x.shape
    _call("mx_cast_dim0", _p(x), R, C, _p(q), _p(s), _stream(stream))


def mx_cast_dim1(x, qt, st, stream=None):
    R, C = x.shape
    _call("mx_cast_dim1", _p(x), R, C, _p(qt), _p(st), _stream(stream))


def mx_cast_2d(x, q, s, qt, st, stream=None):
    R, C = x.shape
    _call("mx_cast_2d", _p(x), R, C, _p(q), _p(s), _p(qt), _p(st), _stream(stream))


def mx_cast_w32x32(w, q, s_fwd, qt=None, s_dgrad=None, stream=None):
    G, N, K = w.shape if w.dim() == 3 else (1, *w.shape)
    _call("mx_cast_w32x32", _p(w), G, N, K, _p(q), _p(s_fwd), _p(qt), _p(s_dgrad), _stream(stream))


def mx_cast_ex(x, dims, rule, q=None, s=None, qt=None, st=None, stream=None):
    R, C = x.shape
    _call("mx_cast_ex", _p(x), R, C, dims, rule, _p(q), _p(s), _p(qt), _p(st), _stream(stream))


def mx_cast_dim0_grouped(x, offs, m_cap, q, s, stream=None):
    M, K = x.shape
    _call("mx_cast_dim0_grouped", _p(x), M, K, _p(offs), offs.numel(), m_cap, _p(q), _p(s),
          _stream(stream))


def mx_cast_dim1_grouped(x, offs, m_cap, qt, st, stream=None):
    M, K = x.shape
    _call("mx_cast_dim1_grouped", _p(x), M, K, _p(offs), offs.numel(), m_cap, _p(qt), _p(st),
          _stream(stream))


def mx_cast_2d_grouped(x, offs, m_cap, q, s, qt, st, stream=None):
    M, K = x.shape
    _call("mx_cast_2d_grouped", _p(x), M, K, _p(offs), offs.numel(), m_cap, _p(q), _p(s), _p(qt),
          _p(st), _stream(stream))


def mx_cast_dim0_grouped_scatter(x, offs, m_cap, dst_q, dst_s, stream=None):
    """Grouped rowwise cast with group g's padded rows written at device address
    dst_q[g] and its scale bands at dst_s[g] (lists of G integers, which may be
    peer-mapped addresses)."""
    M, K = x.shape
    G = offs.numel()
    if len(dst_q) != G or len(dst_s) != G:
        raise ValueError("one code and one scale destination per group")
    arr_q = (_vp * G)(*[int(v) for v in dst_q])
    arr_s = (_vp * G)(*[int(v) for v in dst_s])
    _call("mx_cast_dim0_grouped_scatter", _p(x), M, K, _p(offs), G, m_cap, arr_q, arr_s, _stream(stream))


def mx_cast_2d_grouped_scatter(x, offs, m_cap, dst_q, dst_s, dst_qt, dst_st, dst_cap, stream=None):
    """Fused grouped cast with group g's rowwise outputs at dst_q[g] / dst_s[g]
    and its columnwise outputs at dst_qt[g] / dst_st[g] in a destination of
    padded capacity dst_cap[g] (lists of G integers; addresses may be
    peer-mapped)."""
    M, K = x.shape
    G = offs.numel()
    if not (len(dst_q) == len(dst_s) == len(dst_qt) == len(dst_st) == len(dst_cap) == G):
        raise ValueError("one destination of each kind per group")
    arrs = [(_vp * G)(*[int(v) for v in lst]) for lst in (dst_q, dst_s, dst_qt, dst_st)]
    caps = (_i64 * G)(*[int(v) for v in dst_cap])
    _call("mx_cast_2d_grouped_scatter", _p(x), M, K, _p(offs), G, m_cap, *arrs, caps, _stream(stream))


def mx_grouped_mm(a_q, a_s, b_q, b_s, offs, G, mode, out, M, N, K, m_cap, stream=None):
    _call("mx_grouped_mm", _p(a_q), _p(a_s), _p(b_q), _p(b_s), _p(offs), G, mode, _p(out), M, N, K,
          m_cap, _stream(stream))


def mx_grouped_mm_experts(a_q, a_s, b_q, b_s, offs, G, E, mode, out, M, N, K, m_cap, stream=None):
    _call("mx_grouped_mm_experts", _p(a_q), _p(a_s), _p(b_q), _p(b_s), _p(offs), G, E, mode, _p(out), M, N, K,
          m_cap, _stream(stream))


def mx_grouped_mm_experts_to_rows(a_q, a_s, b_q, b_s, offs, G, E, mode, out_rows, M, N, K, m_cap, stream=None):
    """M-group GEMM with group g's output rows at device address out_rows[g] (a
    list of G integers, which may be peer-mapped addresses)."""
    if len(out_rows) != G:
        raise ValueError("one output destination per group")
    arr = (_vp * G)(*[int(v) for v in out_rows])
    _call("mx_grouped_mm_experts_to_rows", _p(a_q), _p(a_s), _p(b_q), _p(b_s), _p(offs), G, E, mode, arr, M, N, K,
          m_cap, _stream(stream))


def mx_linear_ws_bytes(M, N, K) -> int:
    return int(lib().mx_linear_ws_bytes(M, N, K))


def mx_linear_fwd(x, w, cache, w_version, y, ws, stream=None):
    M, K = x.shape
    N = w.shape[0]
    _call("mx_linear_fwd", _p(x), _p(w), M, N, K, cache.handle if cache is not None else None,
          int(w_version), _p(y), _p(ws), ws.numel(), _stream(stream))


def mx_linear_bwd(dy, x, w, cache, w_version, dx, dw, ws, stream=None):
    M, K = x.shape
    N = w.shape[0]
    _call("mx_linear_bwd", _p(dy), _p(x), _p(w), M, N, K, cache.handle if cache is not None else None,
          int(w_version), _p(dx), _p(dw), _p(ws), ws.numel(), _stream(stream))


def mx_linear_train_ws_bytes(M, N, K) -> int:
    return int(lib().mx_linear_train_ws_bytes(M, N, K))


def mx_linear_fwd_train(x, w, cache, w_version, y, ws, stream=None):
    """Forward of a training step: as mx_linear_fwd, and keeps x's columnwise
    cast (and, without a cache, w's quantization) in `ws` for mx_linear_bwd_after_fwd."""
    M, K = x.shape
    N = w.shape[0]
    _call("mx_linear_fwd_train", _p(x), _p(w), M, N, K, cache.handle if cache is not None else None,
          int(w_version), _p(y), _p(ws), ws.numel(), _stream(stream))


def mx_linear_bwd_after_fwd(dy, w, cache, w_version, dx, dw, ws, stream=None):
    """Backward of the step whose forward was mx_linear_fwd_train on `ws`: casts dY only."""
    M, N = dy.shape
    K = w.shape[1]
    _call("mx_linear_bwd_after_fwd", _p(dy), _p(w), M, N, K, cache.handle if cache is not None else None,
          int(w_version), _p(dx), _p(dw), _p(ws), ws.numel(), _stream(stream))


def mx_linear_fwd_noalloc(x, w, y, stream=None):
    """Linear forward whose scratch is the library's fixed device array (no allocation)."""
    M, K = x.shape
    N = w.shape[0]
    for name, t in (("x", x), ("w", w), ("y", y)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"mx_linear_fwd_noalloc takes bf16 tensors ({name} is {t.dtype})")
    if w.dim() != 2 or w.shape[1] != K or tuple(y.shape) != (M, N):
        raise ValueError(f"shapes must be x [M, K], w [N, K], y [M, N] (got {tuple(x.shape)}, "
                         f"{tuple(w.shape)}, {tuple(y.shape)})")
    _call("mx_linear_fwd_noalloc", _p(x), _p(w), M, N, K, _p(y), _stream(stream))


def mx_grouped_mm_bf16(a, b, offs, G, mode, out, M, N, K, stream=None):
    _call("mx_grouped_mm_bf16", _p(a), _p(b), _p(offs), G, mode, _p(out), M, N, K, _stream(stream))


def mx_dequant_dim0(q, s, G, R, C, out, stream=None):
    _call("mx_dequant_dim0", _p(q), _p(s), G, R, C, _p(out), _stream(stream))


def mx_dequant_dim0_grouped(q, s, offs, M, K, m_cap, out, stream=None):
    _call("mx_dequant_dim0_grouped", _p(q), _p(s), _p(offs), offs.numel(), M, K, m_cap, _p(out),
          _stream(stream))


def mx_scales_unswizzle(s, R, C32, out, stream=None):
    _call("mx_scales_unswizzle", _p(s), R, C32, _p(out), _stream(stream))


def _evict_on_free(cache_ref, key, addrs):
    """Finalizer of a tracked weight: unbind every address it was cached under."""
    cache = cache_ref()
    if cache is None:
        return
    cache._tracked.pop(key, None)
    if cache.handle:
        for a in addrs:
            lib().mx_wcache_evict(cache.handle, ctypes.c_void_p(a))


class WeightCache:
    """Owner of an mx_wcache: quantized weights reused while their version is unchanged.

    The library keys an entry by the weight's device address, and torch's
    caching allocator readily hands a freed weight's block to the next tensor
    of the same size, whose ``_version`` starts at 0 again. Two guards keep
    such a tensor from receiving the freed weight's codes ("incorrect cache
    invalidation could cause silent wrong numerics", prime-rl PR #3388,
    Note): ``key_version`` folds a serial number that is never reused, one per
    tensor object, into the version the library compares; and a finalizer on
    every cached tensor unbinds its entries when it is garbage-collected.

    ``clear_after_backward`` (default on): the MXFP8 linear's backward drops
    the weight's entry when it has finished, as the page's cache is cleared
    after backward (same page, Overview); a recompute forward inside the
    backward (activation checkpointing) still hits. That holds for
    non-reentrant checkpointing; the reentrant form recomputes on detached
    aliases of the weights, new tensor objects to this cache, so there the
    recompute re-quantizes (correct, not faster).
    """

    _serials = itertools.count(1)

    def __init__(self, clear_after_backward=True):
        self.handle = ctypes.c_void_p(lib().mx_wcache_create())
        if not self.handle:
            raise MemoryError("mx_wcache_create failed")
        self.clear_after_backward = clear_after_backward
        self._tracked = {}           # id(tensor) -> [weakref, serial, addresses, finalizer]

    def key_version(self, w):
        """The w_version to pass for ``w``: (serial of this tensor object << 32) | w._version."""
        ent = self._tracked.get(id(w))
        if ent is None or ent[0]() is not w:
            addrs = set()
            fin = weakref.finalize(w, _evict_on_free, weakref.ref(self), id(w), addrs)
            ent = [weakref.ref(w), next(WeightCache._serials), addrs, fin]
            self._tracked[id(w)] = ent
        ent[2].add(w.data_ptr())
        return (ent[1] << 32) | (w._version & 0xFFFFFFFF)

    def evict(self, w):
        """Unbind the entry of ``w`` (its buffer is kept for a later miss of the same shape)."""
        lib().mx_wcache_evict(self.handle, ctypes.c_void_p(w.data_ptr()))

    def clear(self):
        lib().mx_wcache_clear(self.handle)

    def stats(self):
        h, m, e = _i64(), _i64(), _i64()
        _call("mx_wcache_stats", self.handle, ctypes.byref(h), ctypes.byref(m), ctypes.byref(e))
        return {"hits": h.value, "misses": m.value, "entries": e.value}

    def close(self):
        if self.handle:
            for ent in list(self._tracked.values()):
                ent[3].detach()
            self._tracked.clear()
            lib().mx_wcache_destroy(self.handle)
            self.handle = ctypes.c_void_p(None)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# --------------------------------------------------- allocating wrappers --
def _u8(*shape, device):
    return torch.empty(*shape, dtype=torch.uint8, device=device)


def _check_bf16(x):
    if x.dtype != torch.bfloat16:
        raise TypeError("libmx casts take bf16 input")
    return x.contiguous()


def cast_dim0(x):
    x = _check_bf16(x)
    R, C = x.shape
    q, s = _u8(R, C, device=x.device), _u8(mx_scale_bytes(R, C // 32), device=x.device)
    mx_cast_dim0(x, q, s)
    return q, s


def cast_dim1(x):
    x = _check_bf16(x)
    R, C = x.shape
    qt, st = _u8(C, R, device=x.device), _u8(mx_scale_bytes(C, R // 32), device=x.device)
    mx_cast_dim1(x, qt, st)
    return qt, st


def cast_2d(x):
    x = _check_bf16(x)
    R, C = x.shape
    q, s = _u8(R, C, device=x.device), _u8(mx_scale_bytes(R, C // 32), device=x.device)
    qt, st = _u8(C, R, device=x.device), _u8(mx_scale_bytes(C, R // 32), device=x.device)
    mx_cast_2d(x, q, s, qt, st)
    return q, s, qt, st


def cast_w32x32(w, transposed=True, dgrad_scales=None):
    """32x32 cast: (q, s_fwd, qt or None, s_dgrad or None).

    The dgrad scale view is written when ``dgrad_scales`` is true (default: with
    the transposed codes); the MN-major dgrad needs it without ``qt``."""
    w = _check_bf16(w)
    dgrad_scales = transposed if dgrad_scales is None else dgrad_scales
    G, N, K = w.shape if w.dim() == 3 else (1, *w.shape)
    dev = w.device
    q = _u8(*w.shape, device=dev)
    s_fwd = _u8(G * mx_scale_bytes(N, K // 32), device=dev)
    qt = _u8(*((G, K, N) if w.dim() == 3 else (K, N)), device=dev) if transposed else None
    s_dgrad = _u8(G * mx_scale_bytes(K, N // 32), device=dev) if dgrad_scales else None
    mx_cast_w32x32(w, q, s_fwd, qt, s_dgrad)
    return q, s_fwd, qt, s_dgrad


def cast_dim0_grouped(x, offs, m_cap=None):
    x = _check_bf16(x)
    M, K = x.shape
    m_cap = mx_padded_rows_capacity(M, offs.numel()) if m_cap is None else m_cap
    q, s = _u8(m_cap, K, device=x.device), _u8(mx_scale_bytes(m_cap, K // 32), device=x.device)
    mx_cast_dim0_grouped(x, offs, m_cap, q, s)
    return q, s


def cast_dim1_grouped(x, offs, m_cap=None):
    x = _check_bf16(x)
    M, K = x.shape
    m_cap = mx_padded_rows_capacity(M, offs.numel()) if m_cap is None else m_cap
    qt, st = _u8(K, m_cap, device=x.device), _u8(mx_scale_bytes(K, m_cap // 32), device=x.device)
    mx_cast_dim1_grouped(x, offs, m_cap, qt, st)
    return qt, st


def cast_2d_grouped(x, offs, m_cap=None):
    x = _check_bf16(x)
    M, K = x.shape
    m_cap = mx_padded_rows_capacity(M, offs.numel()) if m_cap is None else m_cap
    dev = x.device
    q, s = _u8(m_cap, K, device=dev), _u8(mx_scale_bytes(m_cap, K // 32), device=dev)
    qt, st = _u8(K, m_cap, device=dev), _u8(mx_scale_bytes(K, m_cap // 32), device=dev)
    mx_cast_2d_grouped(x, offs, m_cap, q, s, qt, st)
    return q, s, qt, st


def grouped_mm(a_q, a_s, b_q, b_s, offs, M, m_cap=None):
    """M-groups GEMM: out[M, N] bf16 from padded A [rows, K] and experts B [G, N, K]."""
    G = b_q.shape[0] if b_q.dim() == 3 else 1
    N, K = b_q.shape[-2], b_q.shape[-1]
    if offs is not None and m_cap is None:
        m_cap = a_q.shape[0]
    out = torch.empty(M, N, dtype=torch.bfloat16, device=a_q.device)
    mx_grouped_mm(a_q, a_s, b_q, b_s, offs, G, MX_GROUPS_M, out, M, N, K, m_cap or 0)
    return out


def grouped_mm_wgrad(a_q, a_s, b_q, b_s, offs, M, G=None):
    """K-groups GEMM: out[G, N, K] bf16 from A [N, L] and B [K, L] over token groups."""
    N, L = a_q.shape
    K = b_q.shape[0]
    G = (offs.numel() if offs is not None else 1) if G is None else G
    out = torch.empty(G, N, K, dtype=torch.bfloat16, device=a_q.device)
    mx_grouped_mm(a_q, a_s, b_q, b_s, offs, G, MX_GROUPS_K, out, M, N, K, L if offs is not None else 0)
    return out


def linear_workspace(M, N, K, device="cuda", train=False):
    """Workspace of mx_linear_fwd / mx_linear_bwd, or (train=True) of the
    training pair mx_linear_fwd_train / mx_linear_bwd_after_fwd."""
    n = mx_linear_train_ws_bytes(M, N, K) if train else mx_linear_ws_bytes(M, N, K)
    return torch.empty(n, dtype=torch.uint8, device=device)


def _version_of(w, cache):
    return cache.key_version(w) if cache is not None else w._version


def linear_fwd(x, w, cache=None, version=None, ws=None):
    """y = x w^T through the MXFP8 path; version defaults to the cache's key for w."""
    x, w = _check_bf16(x), _check_bf16(w)
    M, K = x.shape
    N = w.shape[0]
    ws = linear_workspace(M, N, K, x.device) if ws is None else ws
    y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    mx_linear_fwd(x, w, cache, _version_of(w, cache) if version is None else version, y, ws)
    return y


def linear_bwd(dy, x, w, cache=None, version=None, ws=None):
    """(dx, dw) of y = x w^T; a strided or stride-0 dy is materialised first."""
    dy, x, w = _check_bf16(dy), _check_bf16(x), _check_bf16(w)
    M, K = x.shape
    N = w.shape[0]
    ws = linear_workspace(M, N, K, x.device) if ws is None else ws
    dx = torch.empty(M, K, dtype=torch.bfloat16, device=x.device)
    dw = torch.empty(N, K, dtype=torch.bfloat16, device=x.device)
    mx_linear_bwd(dy, x, w, cache, _version_of(w, cache) if version is None else version, dx, dw, ws)
    return dx, dw


def cast_floor(x, dims=3):
    """FLOOR-rule cast: returns (q, s, qt, st) with None for the unused direction."""
    x = _check_bf16(x)
    R, C = x.shape
    q = s = qt = st = None
    if dims & 1:
        q, s = _u8(R, C, device=x.device), _u8(mx_scale_bytes(R, C // 32), device=x.device)
    if dims & 2:
        qt, st = _u8(C, R, device=x.device), _u8(mx_scale_bytes(C, R // 32), device=x.device)
    mx_cast_ex(x, dims, MX_FLOOR, q, s, qt, st)
    return q, s, qt, st


# ------------------------------------------------- backward-override arms --
def grouped_mm_bf16(a, b, offs):
    """Row groups (dgrad form): out[rows of g] = a[rows of g] @ b[g]; a [M, K], b [G, K, N]."""
    a, b = _check_bf16(a), _check_bf16(b)
    M, K = a.shape
    G, _, N = b.shape
    out = torch.empty(M, N, dtype=torch.bfloat16, device=a.device)
    mx_grouped_mm_bf16(a, b, offs, G if offs is not None else 1, MX_GROUPS_M, out, M, N, K)
    return out


def grouped_mm_bf16_wgrad(a, b, offs):
    """Token groups (wgrad form): out[g] = a[rows of g]^T @ b[rows of g]; a [M, N], b [M, K]."""
    a, b = _check_bf16(a), _check_bf16(b)
    M, N = a.shape
    K = b.shape[1]
    G = offs.numel() if offs is not None else 1
    out = torch.empty(G, N, K, dtype=torch.bfloat16, device=a.device)
    mx_grouped_mm_bf16(a, b, offs, G, MX_GROUPS_K, out, M, N, K)
    return out


def dequant_dim0(q, s):
    """bf16 values of rowwise-scaled codes q [R, C] or a stack [G, R, C] (s blocked per matrix)."""
    G, R, C = q.shape if q.dim() == 3 else (1, *q.shape)
    out = torch.empty(*q.shape, dtype=torch.bfloat16, device=q.device)
    mx_dequant_dim0(q, s, G, R, C, out)
    return out


def dequant_dim0_grouped(q, s, offs, M):
    """bf16 rows of a padded grouped dim0 cast, back in the unpadded order [M, K]."""
    m_cap, K = q.shape
    out = torch.empty(M, K, dtype=torch.bfloat16, device=q.device)
    mx_dequant_dim0_grouped(q, s, offs, M, K, m_cap, out)
    return out


def scales_unswizzle(s, R, C32):
    """Logical scales [R, C32] (uint8) from a blocked scale buffer."""
    out = torch.empty(R, C32, dtype=torch.uint8, device=s.device)
    mx_scales_unswizzle(s, R, C32, out)
    return out


BACKWARD_OVERRIDES = (None, "quantized", "high_precision", "dequantized")


class MXFP8GroupedMM:
    """MXFP8 grouped GEMM of an MoE layer, y[rows of g] = x[rows of g] @ w[g]^T.

    forward(x [M, K], w [G, N, K], offs) casts x into the padded group layout
    and w in 32x32 tiles, and runs the scaled grouped GEMM; backward(dy)
    returns (dx, dw). In the MXFP8 backward x is cast rowwise and columnwise
    from one read in the forward (the fused grouped cast), and its columnwise
    codes -- one byte per element -- are kept for the wgrad instead of x
    itself, so the backward casts dy alone. ``backward_override`` selects
    where the gradients come from (ao "[moe training] Add backward_override to
    the MXFP8 grouped GEMM", Design notes): None or "quantized" (alias) is the
    MXFP8 backward;
    "high_precision" uses bf16 grouped GEMMs on the saved bf16 x and w;
    "dequantized" uses the same bf16 GEMMs on the forward's codes turned back
    into bf16 (the gradient of the function the quantized forward computes).
    ``wgrad_with_hp`` (same page, Known follow-ups: the existing knob that
    "high_precision" extends to both gradients) keeps the MXFP8 dgrad and
    takes dw from a bf16 grouped GEMM on the saved bf16 x; under
    "high_precision" it changes nothing, and with "dequantized" it is
    rejected (the two would take dw from different operands).
    Only bf16 operands are accepted; a strided dy is made contiguous first.
    """

    def __init__(self, backward_override=None, wgrad_with_hp=False):
        if backward_override not in BACKWARD_OVERRIDES:
            raise ValueError(f"backward_override must be one of {BACKWARD_OVERRIDES}, "
                             f"got {backward_override!r}")
        self.backward_override = None if backward_override == "quantized" else backward_override
        if wgrad_with_hp and self.backward_override == "dequantized":
            raise ValueError("wgrad_with_hp takes dw from the bf16 activations, the dequantized arm from the "
                             "forward's codes: set one of them")
        self.wgrad_with_hp = bool(wgrad_with_hp) and self.backward_override is None
        self._saved = None

    def forward(self, x, w, offs):
        for name, t in (("x", x), ("w", w)):
            if t.dtype != torch.bfloat16:
                raise TypeError(f"MXFP8GroupedMM takes bf16 operands ({name} is {t.dtype})")
        x, w = x.contiguous(), w.contiguous()
        M, K = x.shape
        G, N, _ = w.shape
        if offs.numel() != G:
            raise ValueError("offs must hold one end offset per expert")
        m_cap = mx_padded_rows_capacity(M, G)
        keep_codes = self.backward_override is None and not self.wgrad_with_hp
        if keep_codes:          # the wgrad's columnwise codes of x, from the forward's one read of x
            xq, xs, xqt, xst = cast_2d_grouped(x, offs, m_cap)
        else:
            xq, xs = cast_dim0_grouped(x, offs, m_cap)
        wq, wsf, _, wsd = cast_w32x32(w, transposed=False, dgrad_scales=self.backward_override is None)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
        mx_grouped_mm(xq, xs, wq, wsf, offs, G, MX_GROUPS_M, y, M, N, K, m_cap)
        if self.backward_override == "high_precision":
            self._saved = (x, w, offs)
        elif self.backward_override == "dequantized":
            self._saved = (xq, xs, wq, wsf, offs, M, m_cap)
        elif keep_codes:
            self._saved = ((xqt, xst, M, K), wq, wsd, offs, m_cap)
        else:
            self._saved = (x, wq, wsd, offs, m_cap)
        return y

    def backward(self, dy):
        if self._saved is None:
            raise RuntimeError("backward before forward")
        if dy.dtype != torch.bfloat16:
            raise TypeError("MXFP8GroupedMM takes a bf16 gradient")
        dy = dy.contiguous()
        saved, self._saved = self._saved, None
        if self.backward_override == "high_precision":
            x, w, offs = saved
            return grouped_mm_bf16(dy, w, offs), grouped_mm_bf16_wgrad(dy, x, offs)
        if self.backward_override == "dequantized":
            xq, xs, wq, wsf, offs, M, m_cap = saved
            xd = dequant_dim0_grouped(xq, xs, offs, M)
            wd = dequant_dim0(wq, wsf)
            return grouped_mm_bf16(dy, wd, offs), grouped_mm_bf16_wgrad(dy, xd, offs)
        acts, wq, wsd, offs, m_cap = saved       # x (wgrad_with_hp) or (x's columnwise codes, scales, M, K)
        G, N, _ = wq.shape
        if self.wgrad_with_hp:
            x = acts
            M, K = x.shape
            dq, ds = cast_dim0_grouped(dy, offs, m_cap)
            dx = torch.empty(M, K, dtype=torch.bfloat16, device=x.device)
            mx_grouped_mm(dq, ds, wq, wsd, offs, G, MX_GROUPS_M_KN, dx, M, K, N, m_cap)
            return dx, grouped_mm_bf16_wgrad(dy, x, offs)
        xqt, xst, M, K = acts
        dq, ds, dqt, dst = cast_2d_grouped(dy, offs, m_cap)
        dx = torch.empty(M, K, dtype=torch.bfloat16, device=dy.device)
        mx_grouped_mm(dq, ds, wq, wsd, offs, G, MX_GROUPS_M_KN, dx, M, K, N, m_cap)
        dw = torch.empty(G, N, K, dtype=torch.bfloat16, device=dy.device)
        mx_grouped_mm(dqt, dst, xqt, xst, offs, G, MX_GROUPS_K, dw, M, N, K, m_cap)
        return dx, dw


# ------------------------------------------------------------- autograd --
def _flatten_saved(obj, tensors):
    """The layout of a nested tuple; its tensors are appended to `tensors` in order."""
    if isinstance(obj, torch.Tensor):
        tensors.append(obj)
        return ("t", len(tensors) - 1)
    if isinstance(obj, tuple):
        return ("tuple", tuple(_flatten_saved(o, tensors) for o in obj))
    return ("v", obj)


def _unflatten_saved(layout, tensors):
    kind, val = layout
    if kind == "t":
        return tensors[val]
    if kind == "tuple":
        return tuple(_unflatten_saved(v, tensors) for v in val)
    return val


class _GroupedMMFn(torch.autograd.Function):
    """Autograd wrapper of MXFP8GroupedMM: forward and backward are its calls.
    What the backward needs (x's columnwise codes, or the bf16 operands for the
    high-precision arms, the weight's codes and the offsets) is saved with
    save_for_backward, so that activation checkpointing drops it after the
    forward and re-creates it by recompute."""

    @staticmethod
    def forward(ctx, x, w, offs, backward_override, wgrad_with_hp):
        op = MXFP8GroupedMM(backward_override=backward_override, wgrad_with_hp=wgrad_with_hp)
        y = op.forward(x, w, offs)
        tensors = []
        ctx.layout = _flatten_saved(op._saved, tensors)
        op._saved = None
        ctx.save_for_backward(*tensors)
        ctx.op = op
        return y

    @staticmethod
    def backward(ctx, dy):
        op, ctx.op = ctx.op, None
        op._saved = _unflatten_saved(ctx.layout, ctx.saved_tensors)
        dx, dw = op.backward(dy)
        return dx, dw, None, None, None


def mxfp8_grouped_mm(x, w, offs, backward_override=None, wgrad_with_hp=False):
    """y[rows of g] = x[rows of g] @ w[g]^T through the MXFP8 path, differentiable.

    x bf16 [M, K], w bf16 [G, N, K], offs int32 [G] on the device (cumulative
    group ends). ``backward_override`` and ``wgrad_with_hp`` as in
    MXFP8GroupedMM (ao "[moe training] Add backward_override to the MXFP8
    grouped GEMM", Design notes and Known follow-ups).
    """
    return _GroupedMMFn.apply(x, w, offs, backward_override, wgrad_with_hp)


class _LinearFn(torch.autograd.Function):
    """Autograd wrapper of the MXFP8 linear. When a gradient is wanted the
    forward is mx_linear_fwd_train and the backward mx_linear_bwd_after_fwd:
    the forward's casts of x and w serve the backward, so x itself is not
    saved (its columnwise codes are, in the workspace, one byte per element)
    and the backward casts dY only. Otherwise the forward is mx_linear_fwd."""

    @staticmethod
    def forward(ctx, x, w, cache):
        x, w = _check_bf16(x), _check_bf16(w)
        version = _version_of(w, cache)
        M, K = x.shape
        N = w.shape[0]
        y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
        if not any(ctx.needs_input_grad[:2]):
            mx_linear_fwd(x, w, cache, version, y, linear_workspace(M, N, K, x.device))
            return y
        ws = linear_workspace(M, N, K, x.device, train=True)
        mx_linear_fwd_train(x, w, cache, version, y, ws)
        # w: autograd refuses the backward if it is updated in place meanwhile; the
        # workspace (x's codes) is saved the same way, so that activation
        # checkpointing drops it after the forward and re-creates it by recompute
        ctx.save_for_backward(w, ws)
        ctx.cache, ctx.version, ctx.M = cache, version, M
        return y

    @staticmethod
    def backward(ctx, dy):
        w, ws = ctx.saved_tensors
        dy = _check_bf16(dy)
        N, K = w.shape
        dx = torch.empty(ctx.M, K, dtype=torch.bfloat16, device=w.device)
        dw = torch.empty(N, K, dtype=torch.bfloat16, device=w.device)
        mx_linear_bwd_after_fwd(dy, w, ctx.cache, ctx.version, dx, dw, ws)
        if ctx.cache is not None and ctx.cache.clear_after_backward:
            ctx.cache.evict(w)
        return dx, dw, None


def mxfp8_linear(x, w, cache=None):
    """y = x @ w^T through the MXFP8 linear, differentiable (ao PR #4705,
    "MXFP8Linear training paths"). With a WeightCache, the 32x32 quantization
    of w is reused while w is the same tensor with an unchanged version
    counter, and (by default) dropped once w's backward has run."""
    return _LinearFn.apply(x, w, cache)
