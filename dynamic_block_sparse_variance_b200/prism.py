"""Python binding of the C ABI in include/prism.h (ctypes; argument marshalling only).

Every function here forwards device pointers and the caller's current CUDA
stream to the shared library; every step of the path runs in its kernels.
There is no fallback: if the library is missing, loading it raises.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libprism_b200.so")

PRISM_OK, PRISM_EINVAL, PRISM_ECAPACITY, PRISM_ECUDA, PRISM_ETIMEOUT, PRISM_EBOUNDS = 0, -1, -2, -3, -4, -5
PRISM_BF16, PRISM_F32 = 0, 1
PRISM_WS_INDICATOR, PRISM_WS_SELECT, PRISM_WS_FWD, PRISM_WS_BWD = 0, 1, 2, 3
PRISM_OPT_ATTN_BACKEND, PRISM_OPT_WAIT_LIMIT, PRISM_OPT_DEBUG_STALL = 0, 1, 2

# Entry points declared in include/prism.h, in declaration order.
ENTRY_POINTS = (
    "prism_workspace_size", "prism_audio_norms", "prism_zone_records", "prism_zone_finalize", "prism_zone_indicator", "prism_zone_indicator_noalloc", "prism_assign_blocks",
    "prism_permute",
    "prism_unpermute", "prism_block_select", "prism_bsa_fwd", "prism_bsa_bwd",
    "prism_set_option", "prism_set_trace", "prism_device_status", "prism_last_error",
)

TRACE_FN = ctypes.CFUNCTYPE(None, ctypes.c_void_p, ctypes.c_char_p, ctypes.c_int, ctypes.c_void_p)


class PrismError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"prism error {code}: {msg}")
        self.code = code


class prism_params(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("tau128", ctypes.c_float), ("tau256", ctypes.c_float), ("eps", ctypes.c_float),
                ("top_k", ctypes.c_int32), ("top_p", ctypes.c_float), ("scale", ctypes.c_float),
                ("fixed_shape", ctypes.c_int32), ("sparsity", ctypes.c_float)]


class prism_block(ctypes.Structure):
    _fields_ = [("start", ctypes.c_int32), ("size", ctypes.c_int32), ("zone", ctypes.c_int32),
                ("shape", ctypes.c_int32)]


PRISM_DYNAMIC_SHAPES = 0
PRISM_FIXED_444 = 3 + 1      # PRISM_FIXED_SHAPE(3): the 4x4x4 box


def make_params(T, H, W, heads, head_dim, top_k, top_p, tau128=0.5, tau256=0.25, eps=1e-4, scale=0.0,
                fixed_shape=PRISM_DYNAMIC_SHAPES, sparsity=0.0):
    """fixed_shape: 0 = dynamic shapes, s + 1 = canonical shape s everywhere;
    sparsity: 0 = absolute top_k, else k = max(1, ceil((1 - sparsity) * nblk))."""
    return prism_params(T, H, W, heads, head_dim, tau128, tau256, eps, top_k, top_p, scale, fixed_shape, sparsity)


_lib = None
_P = ctypes.c_void_p


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it first (python -m "
                               "dynamic_block_sparse_variance_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        i64, sz, pp = ctypes.c_int64, ctypes.c_size_t, ctypes.POINTER(prism_params)
        sig = {
            "prism_workspace_size": [pp, ctypes.c_int, i64, ctypes.POINTER(sz), ctypes.POINTER(sz)],
            "prism_audio_norms": [_P, ctypes.c_int, i64, ctypes.c_int, _P, _P],
            "prism_zone_records": [pp, _P, ctypes.c_int, _P, _P, _P, sz, _P],
            "prism_zone_finalize": [pp, _P, ctypes.c_int, _P, _P, _P, _P],
            "prism_zone_indicator": [pp, _P, ctypes.c_int, _P, _P, _P, _P, _P, sz, _P],
            "prism_zone_indicator_noalloc": [pp, _P, ctypes.c_int, _P, _P, _P, _P, _P],
            "prism_assign_blocks": [pp, _P, _P, _P, _P, _P, _P, _P],
            "prism_permute": [pp, _P, _P, _P, ctypes.c_int, _P, _P, _P],
            "prism_unpermute": [pp, _P, _P, ctypes.c_int, _P, ctypes.c_int, _P],
            "prism_block_select": [pp, _P, _P, _P, _P, _P, i64, _P, _P, sz, _P],
            "prism_bsa_fwd": [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, sz, _P],
            "prism_bsa_bwd": [pp, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, i64, _P, _P, _P,
                              _P, sz, _P],
            "prism_set_option": [ctypes.c_int, i64],
            "prism_set_trace": [TRACE_FN, _P],
            "prism_device_status": [_P],
            "prism_last_error": [],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_char_p if name == "prism_last_error" else ctypes.c_int
        _lib = L
    return _lib


def _check(rc):
    if rc != PRISM_OK:
        raise PrismError(rc, lib().prism_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype(t):
    if t.dtype == torch.bfloat16:
        return PRISM_BF16
    if t.dtype == torch.float32:
        return PRISM_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


# ---- one wrapper per entry point -------------------------------------------

def prism_workspace_size(p, kind, col_capacity=0):
    a, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib().prism_workspace_size(ctypes.byref(p), kind, col_capacity, ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def prism_audio_norms(h, a):
    """a[n] = ||h[n, :]||_2 for a row-major [N, C] tensor h (bf16 or f32)."""
    _check(lib().prism_audio_norms(_ptr(h), _dtype(h), h.shape[0], h.shape[1] if h.dim() > 1 else 0, _ptr(a),
                                   _stream()))


PRISM_ZONE_RECORD = 9


def prism_zone_records(p, V, audio, records, workspace):
    """Per-zone indicator records [Z, 9] float64 of the grid p describes (a T-slab or the whole grid)."""
    _check(lib().prism_zone_records(ctypes.byref(p), _ptr(V), _dtype(V), _ptr(audio), _ptr(records),
                                    _ptr(workspace), workspace.numel(), _stream()))


def prism_zone_finalize(p, records, has_audio, g, rho, debug=None):
    """g, rho (and debug) of the whole grid p from the records of all its zones."""
    _check(lib().prism_zone_finalize(ctypes.byref(p), _ptr(records), int(bool(has_audio)), _ptr(g), _ptr(rho),
                                     _ptr(debug), _stream()))


def prism_zone_indicator(p, V, audio, g, rho, debug, workspace):
    _check(lib().prism_zone_indicator(ctypes.byref(p), _ptr(V), _dtype(V), _ptr(audio), _ptr(g), _ptr(rho),
                                      _ptr(debug), _ptr(workspace), workspace.numel(), _stream()))


def prism_zone_indicator_noalloc(p, V, audio, g, rho, debug=None):
    """The indicator with no workspace argument (fixed scratch inside the library)."""
    _check(lib().prism_zone_indicator_noalloc(ctypes.byref(p), _ptr(V), _dtype(V), _ptr(audio), _ptr(g), _ptr(rho),
                                              _ptr(debug), _stream()))


def prism_assign_blocks(p, g, rho, shape_id, zone_blk_base, blocks, nblk):
    _check(lib().prism_assign_blocks(ctypes.byref(p), _ptr(g), _ptr(rho), _ptr(shape_id), _ptr(zone_blk_base),
                                     _ptr(blocks), _ptr(nblk), _stream()))


def prism_permute(p, shape_id, zone_blk_base, x, x_perm, pooled=None):
    _check(lib().prism_permute(ctypes.byref(p), _ptr(shape_id), _ptr(zone_blk_base), _ptr(x), _dtype(x),
                               _ptr(x_perm), _ptr(pooled), _stream()))


def prism_unpermute(p, shape_id, x_perm, x):
    _check(lib().prism_unpermute(ctypes.byref(p), _ptr(shape_id), _ptr(x_perm), _dtype(x_perm), _ptr(x),
                                 _dtype(x), _stream()))


def prism_block_select(p, nblk, q_pooled, k_pooled, row_ptr, col, nnz, workspace):
    _check(lib().prism_block_select(ctypes.byref(p), _ptr(nblk), _ptr(q_pooled), _ptr(k_pooled), _ptr(row_ptr),
                                    _ptr(col), col.numel(), _ptr(nnz), _ptr(workspace), workspace.numel(),
                                    _stream()))


def prism_bsa_fwd(p, blocks, zone_blk_base, nblk, q, k, v, row_ptr, col, o, lse, o_res=None, workspace=None):
    _check(lib().prism_bsa_fwd(ctypes.byref(p), _ptr(blocks), _ptr(zone_blk_base), _ptr(nblk), _ptr(q), _ptr(k),
                               _ptr(v), _ptr(row_ptr), _ptr(col), _ptr(o), _ptr(o_res), _ptr(lse),
                               _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream()))


def prism_bsa_bwd(p, blocks, zone_blk_base, nblk, q, k, v, o, o_res, dout, lse, row_ptr, col, nnz, dq, dk, dv,
                  workspace):
    _check(lib().prism_bsa_bwd(ctypes.byref(p), _ptr(blocks), _ptr(zone_blk_base), _ptr(nblk), _ptr(q),
                               _ptr(k), _ptr(v), _ptr(o), _ptr(o_res), _ptr(dout), _ptr(lse), _ptr(row_ptr),
                               _ptr(col), _ptr(nnz), col.numel(), _ptr(dq), _ptr(dk), _ptr(dv),
                               _ptr(workspace), workspace.numel(), _stream()))


def prism_set_option(option, value):
    _check(lib().prism_set_option(option, value))


def prism_device_status():
    """Synchronise the current stream and raise if a kernel latched an error."""
    _check(lib().prism_device_status(_stream()))


class KernelTrace:
    """Records a CUDA event pair around every kernel the library launches.

    Use as a context manager; ``summary()`` (after a synchronize) gives, per
    kernel name, the number of launches and their total device time in ms.
    """

    def __init__(self):
        self.events = []          # (name, start_event, end_event)
        self._open = {}
        self._cb = TRACE_FN(self._hook)

    def _hook(self, user, name, end, stream):
        s = torch.cuda.ExternalStream(stream) if stream else torch.cuda.default_stream()
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(s)
        key = name.decode()
        if not end:
            self._open[key] = ev
        else:
            self.events.append((key, self._open.pop(key), ev))

    def __enter__(self):
        _check(lib().prism_set_trace(self._cb, None))
        return self

    def __exit__(self, *exc):
        lib().prism_set_trace(TRACE_FN(), None)
        return False

    def summary(self):
        out = {}
        for name, a, b in self.events:
            n, t = out.get(name, (0, 0.0))
            out[name] = (n + 1, t + a.elapsed_time(b))
        return out
