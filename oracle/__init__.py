"""Plain fp64 CPU oracle for the fused all-reduce + residual-add + RMSNorm
(+FP8-e4m3) epilogue.

TEST INFRASTRUCTURE ONLY.  The product (``reduce_residual_add_b200``) never
imports this package; only the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference legs do.  The arithmetic lives in
``far_oracle.c`` (plain C, fp64, one row at a time); this module only marshals
numpy arrays of raw 16-bit / 8-bit patterns in and out of it.

What it computes, per row t (see the header of ``far_oracle.c`` for the
sources and for the readings taken where the pages are silent):

    y    = sum_r partials[r][t] + residual[t]      (new residual; exact, or in
                                                    fp32 with acc32=True)
    rinv = 1 / sqrt(mean(y^2) + eps)
    o    = y * rinv * (gamma + weight_bias)        (normed output)
    static FP8:  q = e4m3(fp32(fp32(o) / scale))
    per-token:   scale_t = fp32(max|fp32(o)| / 448); q = e4m3(fp32(fp32(o) / scale_t))
    per-tensor:  one scale = fp32(max over the rows of |fp32(o)| / 448), in scale_out[0]
    per-group:   one scale per (row, group of `group` elements), amax / 448
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

BF16, FP16 = 0, 1
AR_RESIDUAL_RMSNORM, FP8_STATIC, FP8_TOKEN, FP8_TENSOR, FP8_GROUP = 0, 1, 2, 3, 4

_lib = None


def load(path: str) -> ctypes.CDLL:
    """Open an oracle shared library at ``path`` and declare its signatures."""
    L = ctypes.CDLL(path)
    L.far_oracle_decode16.restype = ctypes.c_double
    L.far_oracle_decode16.argtypes = [ctypes.c_uint16, ctypes.c_int]
    L.far_oracle_round16.restype = ctypes.c_uint16
    L.far_oracle_round16.argtypes = [ctypes.c_double, ctypes.c_int]
    L.far_oracle_e4m3_decode.restype = ctypes.c_double
    L.far_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.far_oracle_e4m3_encode.restype = ctypes.c_uint8
    L.far_oracle_e4m3_encode.argtypes = [ctypes.c_double]
    vp = ctypes.c_void_p
    for fn in (L.far_oracle_fused, L.far_oracle_fused_acc32):
        fn.restype = ctypes.c_int
        fn.argtypes = [
            ctypes.POINTER(vp), ctypes.c_int, vp, vp,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
            ctypes.c_float, ctypes.c_float, ctypes.c_int, ctypes.c_int64,
            ctypes.c_int64, ctypes.c_int64,
            vp, vp, vp, vp, vp, vp, vp, vp]
    return L


def lib() -> ctypes.CDLL:
    """The oracle's shared library (built first if it is missing or stale)."""
    global _lib
    if _lib is None:
        _lib = load(_build.build())
    return _lib


def dtype_code(dtype) -> int:
    """Map 'bf16' / 'fp16' (or the integer codes) to the oracle's code."""
    if dtype in (BF16, "bf16", "bfloat16"):
        return BF16
    if dtype in (FP16, "fp16", "float16", "half"):
        return FP16
    raise ValueError("unsupported dtype %r" % (dtype,))


def decode16(bits: int, dtype) -> float:
    return lib().far_oracle_decode16(int(bits), dtype_code(dtype))


def round16(x: float, dtype) -> int:
    return int(lib().far_oracle_round16(float(x), dtype_code(dtype)))


def e4m3_decode(code: int) -> float:
    return lib().far_oracle_e4m3_decode(int(code))


def e4m3_encode(x: float) -> int:
    return int(lib().far_oracle_e4m3_encode(float(x)))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _u16_2d(a: np.ndarray, H: int) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("expected raw 16-bit patterns (uint16), got %s" % a.dtype)
    return a.reshape(-1, H)


def fused(partials: Sequence[np.ndarray], residual: Optional[np.ndarray],
          gamma: np.ndarray, dtype, eps: float, weight_bias: float = 0.0,
          pattern: int = AR_RESIDUAL_RMSNORM, scale_in: Optional[float] = None,
          rows: Optional[tuple] = None, want_norm: bool = True,
          want_residual_out: bool = True, debug: bool = False,
          out: Optional[dict] = None, group: int = 0, acc32: bool = False) -> dict:
    """Run the oracle on raw bit patterns.

    ``acc32``: accumulate the partials and the residual in fp32 (partial 0,
    1, ..., W-1, then the residual, each addition rounded to fp32) instead
    of exactly -- the pages' fp32_acc=True taken literally.  The two agree
    except where a rounded running sum meets cancellation.

    ``partials`` are W arrays of uint16 patterns of shape (..., H) (any
    leading shape is flattened to (T, H), as the PR #45307 report does for
    3-D inputs); ``residual`` has the same shape or is None; ``gamma`` is (H,).
    ``rows=(b, e)`` restricts the work to rows [b, e); outputs for other rows
    are left as they are in ``out`` (zeros when ``out`` is not given).

    Returns a dict with ``residual_out`` (uint16, T x H), ``norm_out``
    (uint16 or None), ``quant_out`` (uint8 or None), ``scale_out`` (float32
    (T,) per token, (1,) per tensor, or None) and, with ``debug``, fp64 ``y``, ``o`` (T x H) and ``rinv`` (T,).
    """
    dt = dtype_code(dtype)
    gamma = np.ascontiguousarray(gamma, dtype=np.uint16).reshape(-1)
    H = gamma.shape[0]
    ps = [_u16_2d(p, H) for p in partials]
    W = len(ps)
    T = ps[0].shape[0]
    for p in ps:
        if p.shape != (T, H):
            raise ValueError("partials disagree in shape")
    res = None if residual is None else _u16_2d(residual, H)
    if res is not None and res.shape != (T, H):
        raise ValueError("residual shape mismatch")
    b, e = (0, T) if rows is None else (int(rows[0]), int(rows[1]))

    o = {} if out is None else out
    if want_residual_out:
        o.setdefault("residual_out", np.zeros((T, H), np.uint16))
    else:
        o["residual_out"] = None
    if want_norm:
        o.setdefault("norm_out", np.zeros((T, H), np.uint16))
    else:
        o["norm_out"] = None
    if pattern in (FP8_STATIC, FP8_TOKEN, FP8_TENSOR, FP8_GROUP):
        o.setdefault("quant_out", np.zeros((T, H), np.uint8))
    else:
        o["quant_out"] = None
    if pattern == FP8_TOKEN:
        o.setdefault("scale_out", np.zeros((T,), np.float32))
    elif pattern == FP8_TENSOR:
        o.setdefault("scale_out", np.zeros((1,), np.float32))
    elif pattern == FP8_GROUP:
        if group < 1 or H % group:
            raise ValueError("group must divide H")
        o.setdefault("scale_out", np.zeros((T, H // group), np.float32))
    else:
        o["scale_out"] = None
    sin = None
    if pattern == FP8_STATIC:
        if scale_in is None:
            raise ValueError("static FP8 needs scale_in")
        sin = np.array([scale_in], dtype=np.float32)
    if debug:
        o.setdefault("y", np.zeros((T, H), np.float64))
        o.setdefault("o", np.zeros((T, H), np.float64))
        o.setdefault("rinv", np.zeros((T,), np.float64))

    arr = (ctypes.c_void_p * W)(*[p.ctypes.data for p in ps])
    fn = lib().far_oracle_fused_acc32 if acc32 else lib().far_oracle_fused
    rc = fn(
        arr, W, _ptr(res), _ptr(gamma), T, H, dt,
        float(eps), float(weight_bias), int(pattern), int(group), b, e,
        _ptr(o["residual_out"]), _ptr(o["norm_out"]), _ptr(o["quant_out"]),
        _ptr(sin), _ptr(o["scale_out"]),
        _ptr(o.get("y")), _ptr(o.get("o")), _ptr(o.get("rinv")))
    if rc != 0:
        raise ValueError("oracle rejected its arguments (rc=%d)" % rc)
    return o


__all__ = ["BF16", "FP16", "AR_RESIDUAL_RMSNORM", "FP8_STATIC", "FP8_TOKEN", "FP8_TENSOR",
           "FP8_GROUP",
           "load", "lib", "dtype_code", "decode16", "round16", "e4m3_decode",
           "e4m3_encode", "fused"]
