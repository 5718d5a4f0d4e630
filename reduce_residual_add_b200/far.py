"""ctypes binding of libfar.so (include/far.h), same entry-point names.

Argument marshalling only: every step of the epilogue runs in the library's
CUDA kernels.  torch supplies device memory and streams.  If the library is
missing, every call raises -- there is no other code path.

Tensor-level entry points (``far_fused`` / ``far_fused_rows``) take CUDA
tensors: W partials of shape (..., H), a residual of the same shape (or
None), gamma (H,), and optional outputs.  Leading dimensions are flattened to
(T, H) as views, as the PR #45307 report's fix does for 3-D
[batch, tokens, hidden] inputs.  ``lib()`` exposes the raw C functions.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

from . import build as _build

FAR_OK = 0
FAR_ERR_INVALID_ARG = 1
FAR_ERR_UNSUPPORTED = 2
FAR_ERR_ALIGNMENT = 3
FAR_ERR_CUDA = 4
FAR_ERR_TIMEOUT = 5
FAR_ERR_INTERNAL = 6

FAR_BF16 = 0
FAR_FP16 = 1

FAR_AR_RESIDUAL_RMSNORM = 0
FAR_AR_RESIDUAL_RMSNORM_FP8_STATIC = 1
FAR_AR_RESIDUAL_RMSNORM_FP8_TOKEN = 2
FAR_AR_RESIDUAL_RMSNORM_FP8_TENSOR = 3
FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP = 4

FAR_REGIME_AUTO = 0
FAR_REGIME_DECODE = 1
FAR_REGIME_PREFILL = 2

FAR_MAX_W = 16
FAR_MAX_H = 16384
FAR_FP8_TENSOR_NOALLOC_MAX_ROWS = 65536

# Every symbol include/far.h declares.
EXPORTS = ("far_create", "far_destroy", "far_fused", "far_fused_rows",
           "far_fp8_tensor_workspace_bytes", "far_fused_fp8_tensor",
           "far_fused_fp8_tensor_noalloc", "far_fused_fp8_group",
           "far_host_staging_bytes", "far_fused_host", "far_validate",
           "far_set_regime", "far_describe_launch", "far_describe_launch_pattern",
           "far_check", "far_test_stall", "far_status_string", "far_last_error",
           "far_version")

_DTYPES = {torch.bfloat16: FAR_BF16, torch.float16: FAR_FP16}


class far_launch_info(ctypes.Structure):
    _fields_ = [("regime", ctypes.c_int), ("ctas_per_row", ctypes.c_int),
                ("rows_per_cta", ctypes.c_int), ("threads_per_cta", ctypes.c_int),
                ("packs_per_thread", ctypes.c_int), ("grid_ctas", ctypes.c_int64),
                ("kernel", ctypes.c_int), ("ring_slots", ctypes.c_int),
                ("ring_gamma_smem", ctypes.c_int)]


class FarError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        msg = "%s%s" % (far_status_string(status), (" in " + where) if where else "")
        if status == FAR_ERR_CUDA or status == FAR_ERR_UNSUPPORTED:
            detail = far_last_error()
            if detail:
                msg += ": " + detail
        super().__init__(msg)


_lib = None


def lib_path() -> str:
    return _build.LIB


def lib() -> ctypes.CDLL:
    """The loaded library with its C signatures declared."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise RuntimeError(
            "libfar.so is not built (%s); run `python -m reduce_residual_add_b200.build` "
            "-- there is no fallback path" % path)
    L = ctypes.CDLL(path)
    vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    pp = ctypes.POINTER(vp)
    L.far_create.argtypes = [ctypes.POINTER(vp), i32]
    L.far_create.restype = i32
    L.far_destroy.argtypes = [vp]
    L.far_destroy.restype = i32
    common = [pp, i32, vp, vp, vp, i64, i64, i32, f32, f32, i32, vp, vp, vp, vp]
    L.far_fused.argtypes = [vp] + common + [vp]
    L.far_fused.restype = i32
    L.far_fused_rows.argtypes = [vp, i64, i64] + common + [vp]
    L.far_fused_rows.restype = i32
    L.far_validate.argtypes = [i64, i64] + common
    L.far_validate.restype = i32
    L.far_fp8_tensor_workspace_bytes.argtypes = [i64]
    L.far_fp8_tensor_workspace_bytes.restype = ctypes.c_size_t
    L.far_fused_fp8_tensor.argtypes = [vp, i64, i64, pp, i32, vp, vp, vp, i64, i64, i32, f32, f32,
                                       vp, vp, vp, vp, ctypes.c_size_t, vp]
    L.far_fused_fp8_tensor.restype = i32
    L.far_fused_fp8_tensor_noalloc.argtypes = [vp, i64, i64, pp, i32, vp, vp, vp, i64, i64, i32,
                                               f32, f32, vp, vp, vp, vp]
    L.far_fused_fp8_tensor_noalloc.restype = i32
    L.far_fused_fp8_group.argtypes = [vp, i64, i64, pp, i32, vp, vp, vp, i64, i64, i32, f32, f32,
                                      i32, vp, vp, vp, vp]
    L.far_fused_fp8_group.restype = i32
    L.far_host_staging_bytes.argtypes = [i32, i64, i64]
    L.far_host_staging_bytes.restype = ctypes.c_size_t
    L.far_fused_host.argtypes = [vp, pp, i32, vp, vp, vp, i64, i64, i32, f32, f32, i32, i32,
                                 vp, vp, vp, vp, i64, vp, ctypes.c_size_t, vp]
    L.far_fused_host.restype = i32
    L.far_set_regime.argtypes = [vp, i32, i32]
    L.far_set_regime.restype = i32
    L.far_describe_launch.argtypes = [vp, i64, i64, i32, i32, i32, i32,
                                      ctypes.POINTER(far_launch_info)]
    L.far_describe_launch.restype = i32
    L.far_describe_launch_pattern.argtypes = [vp, i64, i64, i32, i32, i32, i32, i32,
                                              ctypes.POINTER(far_launch_info)]
    L.far_describe_launch_pattern.restype = i32
    L.far_test_stall.argtypes = [vp, i64, ctypes.c_uint32]
    L.far_test_stall.restype = i32
    L.far_check.argtypes = [vp, vp]
    L.far_check.restype = i32
    L.far_status_string.argtypes = [i32]
    L.far_status_string.restype = ctypes.c_char_p
    L.far_last_error.argtypes = []
    L.far_last_error.restype = ctypes.c_char_p
    L.far_version.argtypes = []
    L.far_version.restype = i32
    _lib = L
    return L


def far_status_string(status: int) -> str:
    return lib().far_status_string(int(status)).decode()


def far_last_error() -> str:
    return lib().far_last_error().decode()


def far_version() -> int:
    return int(lib().far_version())


class FarContext:
    """Owns a far_ctx* for one CUDA device."""

    def __init__(self, device: int = 0):
        self.device = int(device)
        self._ptr = ctypes.c_void_p()
        st = lib().far_create(ctypes.byref(self._ptr), self.device)
        if st != FAR_OK:
            raise FarError(st, "far_create")

    @property
    def handle(self) -> ctypes.c_void_p:
        if not self._ptr:
            raise RuntimeError("context destroyed")
        return self._ptr

    def close(self) -> None:
        if self._ptr:
            lib().far_destroy(self._ptr)
            self._ptr = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


def far_create(device: int = 0) -> FarContext:
    return FarContext(device)


def far_destroy(ctx: FarContext) -> None:
    ctx.close()


def far_set_regime(ctx: FarContext, regime: int, decode_max_rows: int = -1) -> None:
    st = lib().far_set_regime(ctx.handle, int(regime), int(decode_max_rows))
    if st != FAR_OK:
        raise FarError(st, "far_set_regime")


def far_describe_launch(ctx: FarContext, rows: int, H: int, dtype=torch.bfloat16, W: int = 8,
                        has_residual: bool = True, has_norm_out: bool = False,
                        pattern: Optional[int] = None) -> dict:
    """The launch geometry of a call; `pattern` None: far_fused / far_fused_rows
    (far_describe_launch), else that pattern's own plan (far_describe_launch_pattern)."""
    info = far_launch_info()
    dt = _DTYPES.get(dtype, dtype)
    if pattern is None:
        st = lib().far_describe_launch(ctx.handle, int(rows), int(H), dt, int(W),
                                       int(bool(has_residual)), int(bool(has_norm_out)),
                                       ctypes.byref(info))
    else:
        st = lib().far_describe_launch_pattern(ctx.handle, int(rows), int(H), dt, int(W),
                                               int(bool(has_residual)), int(bool(has_norm_out)),
                                               int(pattern), ctypes.byref(info))
    if st != FAR_OK:
        raise FarError(st, "far_describe_launch")
    return {name: getattr(info, name) for name, _ in far_launch_info._fields_}


def far_test_stall(ctx: FarContext, segment: int, wait_limit_us: int = 0) -> None:
    """Test hook: make the ring kernel's wait for one segment run out
    (see include/far.h); segment < 0 switches it off."""
    st = lib().far_test_stall(ctx.handle, int(segment), int(wait_limit_us))
    if st != FAR_OK:
        raise FarError(st, "far_test_stall")


def far_check(ctx: FarContext, stream=None) -> None:
    """Synchronise `stream` and raise FarError(FAR_ERR_TIMEOUT) if a kernel's
    bounded wait gave up since the last check (see include/far.h)."""
    st = lib().far_check(ctx.handle, _stream(stream))
    if st != FAR_OK:
        raise FarError(st, "far_check")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _flat(t: Optional[torch.Tensor], H: int, name: str, host: bool = False) -> Optional[torch.Tensor]:
    if t is None:
        return None
    if t.is_cuda == host:
        raise ValueError("%s must be a %s tensor" % (name, "host (CPU)" if host else "CUDA"))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.view(-1, H) if t.dim() != 2 else t


def _args(partials, residual, gamma, residual_out, norm_out, quant_out, scale_in, scale_out,
          scale_out_elems=None, host=False):
    where = "host (CPU)" if host else "CUDA"
    if isinstance(partials, torch.Tensor):
        partials = [partials]
    if len(partials) == 0:
        raise ValueError("need at least one partial")
    if not gamma.is_contiguous() or gamma.is_cuda == host:
        raise ValueError("gamma must be a contiguous %s tensor" % where)
    H = gamma.numel()
    ps = [_flat(p, H, "partials[%d]" % i, host) for i, p in enumerate(partials)]
    T = ps[0].shape[0]
    dt = _DTYPES.get(ps[0].dtype)
    if dt is None:
        raise ValueError("dtype %s not supported (bf16 / fp16)" % ps[0].dtype)
    for p in ps:
        if p.shape != (T, H) or p.dtype != ps[0].dtype:
            raise ValueError("partials must share shape and dtype")
    arr = (ctypes.c_void_p * len(ps))(*[p.data_ptr() for p in ps])
    # the C side sees plain pointers: make sure each buffer covers (T, H)
    res = _flat(residual, H, "residual", host)
    rout = _flat(residual_out, H, "residual_out", host)
    nout = _flat(norm_out, H, "norm_out", host)
    qout = _flat(quant_out, H, "quant_out", host)
    for name, t in (("residual", res), ("residual_out", rout), ("norm_out", nout)):
        if t is not None and (t.shape != (T, H) or t.dtype != ps[0].dtype):
            raise ValueError("%s must be (%d, %d) %s" % (name, T, H, ps[0].dtype))
    if qout is not None and (qout.shape != (T, H) or qout.element_size() != 1):
        raise ValueError("quant_out must be (%d, %d) of 1-byte elements" % (T, H))
    if gamma.dtype != ps[0].dtype:
        raise ValueError("gamma must be %s" % ps[0].dtype)
    for name, t, n in (("scale_in", scale_in, 1),
                       ("scale_out", scale_out, T if scale_out_elems is None else scale_out_elems)):
        if t is not None and (t.is_cuda == host or t.dtype != torch.float32 or t.numel() < n
                              or not t.is_contiguous()):
            raise ValueError("%s must be a contiguous %s float32 tensor of >= %d elements"
                             % (name, where, n))
    return (arr, len(ps), _ptr(res), _ptr(rout), _ptr(gamma), T, H, dt,
            _ptr(nout), _ptr(qout), _ptr(scale_in), _ptr(scale_out))


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def far_fused_rows(ctx: FarContext, row_begin: int, row_end: int,
                   partials: Sequence[torch.Tensor], residual: Optional[torch.Tensor],
                   gamma: torch.Tensor, eps: float, weight_bias: float = 0.0,
                   pattern: int = FAR_AR_RESIDUAL_RMSNORM, *,
                   residual_out: Optional[torch.Tensor] = None,
                   norm_out: Optional[torch.Tensor] = None,
                   quant_out: Optional[torch.Tensor] = None,
                   scale_in: Optional[torch.Tensor] = None,
                   scale_out: Optional[torch.Tensor] = None, stream=None) -> None:
    """Rows [row_begin, row_end) of the fused epilogue (see include/far.h)."""
    (arr, W, res, rout, gam, T, H, dt, nout, qout, sin, sout) = _args(
        partials, residual, gamma, residual_out, norm_out, quant_out, scale_in, scale_out)
    st = lib().far_fused_rows(ctx.handle, int(row_begin), int(row_end), arr, W, res, rout, gam,
                              T, H, dt, float(eps), float(weight_bias), int(pattern),
                              nout, qout, sin, sout, _stream(stream))
    if st != FAR_OK:
        raise FarError(st, "far_fused_rows")


def far_fused_addrs(ctx: FarContext, partial_addrs: Sequence[int], T: int,
                    residual: Optional[torch.Tensor], gamma: torch.Tensor, eps: float,
                    weight_bias: float = 0.0, pattern: int = FAR_AR_RESIDUAL_RMSNORM, *,
                    residual_out: Optional[torch.Tensor] = None,
                    norm_out: Optional[torch.Tensor] = None,
                    quant_out: Optional[torch.Tensor] = None,
                    scale_in: Optional[torch.Tensor] = None,
                    scale_out: Optional[torch.Tensor] = None, stream=None) -> None:
    """far_fused with the W partials given as raw device addresses, each of a
    contiguous (T, H) tensor of gamma's dtype -- for partials that are not
    tensors of this process, such as another GPU's buffers mapped into this
    one's address space.  The library checks alignment and overlap as for
    far_fused; the caller vouches that each address holds T x H elements."""
    if len(partial_addrs) == 0:
        raise ValueError("need at least one partial")
    H = gamma.numel()
    dt = _DTYPES.get(gamma.dtype)
    if dt is None or not gamma.is_cuda or not gamma.is_contiguous():
        raise ValueError("gamma must be a contiguous CUDA bf16 / fp16 tensor")
    arr = (ctypes.c_void_p * len(partial_addrs))(*[int(a) for a in partial_addrs])
    res = _flat(residual, H, "residual")
    rout = _flat(residual_out, H, "residual_out")
    nout = _flat(norm_out, H, "norm_out")
    qout = _flat(quant_out, H, "quant_out")
    for name, t in (("residual", res), ("residual_out", rout), ("norm_out", nout)):
        if t is not None and (t.shape != (T, H) or t.dtype != gamma.dtype):
            raise ValueError("%s must be (%d, %d) %s" % (name, T, H, gamma.dtype))
    if qout is not None and (qout.shape != (T, H) or qout.element_size() != 1):
        raise ValueError("quant_out must be (%d, %d) of 1-byte elements" % (T, H))
    for name, t, n in (("scale_in", scale_in, 1), ("scale_out", scale_out, T)):
        if t is not None and (not t.is_cuda or t.dtype != torch.float32 or t.numel() < n
                              or not t.is_contiguous()):
            raise ValueError("%s must be a contiguous CUDA float32 tensor of >= %d elements"
                             % (name, n))
    st = lib().far_fused(ctx.handle, arr, len(partial_addrs), _ptr(res), _ptr(rout), _ptr(gamma),
                         int(T), H, dt, float(eps), float(weight_bias), int(pattern), _ptr(nout),
                         _ptr(qout), _ptr(scale_in), _ptr(scale_out), _stream(stream))
    if st != FAR_OK:
        raise FarError(st, "far_fused")


def far_fused(ctx: FarContext, partials: Sequence[torch.Tensor],
              residual: Optional[torch.Tensor], gamma: torch.Tensor, eps: float,
              weight_bias: float = 0.0, pattern: int = FAR_AR_RESIDUAL_RMSNORM, *,
              residual_out: Optional[torch.Tensor] = None,
              norm_out: Optional[torch.Tensor] = None,
              quant_out: Optional[torch.Tensor] = None,
              scale_in: Optional[torch.Tensor] = None,
              scale_out: Optional[torch.Tensor] = None, stream=None) -> None:
    """All rows of the fused epilogue (see include/far.h)."""
    (arr, W, res, rout, gam, T, H, dt, nout, qout, sin, sout) = _args(
        partials, residual, gamma, residual_out, norm_out, quant_out, scale_in, scale_out)
    st = lib().far_fused(ctx.handle, arr, W, res, rout, gam, T, H, dt, float(eps),
                         float(weight_bias), int(pattern), nout, qout, sin, sout, _stream(stream))
    if st != FAR_OK:
        raise FarError(st, "far_fused")


def far_validate(row_begin: int, row_end: int, partial_ptrs: Sequence[int], residual: int,
                 residual_out: int, gamma: int, T: int, H: int, dtype: int, eps: float,
                 weight_bias: float, pattern: int, norm_out: int, quant_out: int,
                 scale_in: int, scale_out: int, W: Optional[int] = None) -> int:
    """Host-only argument check on raw addresses (integers; 0 = NULL).
    ``W`` defaults to the number of partial pointers."""
    arr = None
    if partial_ptrs is not None:
        arr = (ctypes.c_void_p * max(1, len(partial_ptrs)))(*[p or None for p in partial_ptrs])
    if W is None:
        W = len(partial_ptrs) if partial_ptrs is not None else 0
    vp = lambda a: ctypes.c_void_p(a) if a else None  # noqa: E731
    return int(lib().far_validate(int(row_begin), int(row_end), arr, int(W),
                                  vp(residual), vp(residual_out), vp(gamma), int(T), int(H),
                                  int(dtype), float(eps), float(weight_bias), int(pattern),
                                  vp(norm_out), vp(quant_out), vp(scale_in), vp(scale_out)))


def far_fp8_tensor_workspace_bytes(rows: int) -> int:
    return int(lib().far_fp8_tensor_workspace_bytes(int(rows)))


def far_fused_fp8_tensor(ctx: FarContext, partials: Sequence[torch.Tensor],
                         residual: Optional[torch.Tensor], gamma: torch.Tensor, eps: float,
                         weight_bias: float = 0.0, *, quant_out: torch.Tensor,
                         scale_out: torch.Tensor, workspace: torch.Tensor,
                         residual_out: Optional[torch.Tensor] = None,
                         norm_out: Optional[torch.Tensor] = None, rows=None, stream=None) -> None:
    """Dynamic per-tensor FP8 over rows [b, e) (all rows by default): one
    scale in scale_out[0].  ``workspace`` is a CUDA tensor of at least
    far_fp8_tensor_workspace_bytes(e - b) bytes (see include/far.h)."""
    (arr, W, res, rout, gam, T, H, dt, nout, qout, sin, sout) = _args(
        partials, residual, gamma, residual_out, norm_out, quant_out, None, scale_out,
        scale_out_elems=1)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    b, e = (0, T) if rows is None else (int(rows[0]), int(rows[1]))
    st = lib().far_fused_fp8_tensor(ctx.handle, b, e, arr, W, res, rout, gam, T, H, dt,
                                    float(eps), float(weight_bias), nout, qout, sout,
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream))
    if st != FAR_OK:
        raise FarError(st, "far_fused_fp8_tensor")


def far_fused_fp8_tensor_noalloc(ctx: FarContext, partials: Sequence[torch.Tensor],
                                 residual: Optional[torch.Tensor], gamma: torch.Tensor,
                                 eps: float, weight_bias: float = 0.0, *,
                                 quant_out: torch.Tensor, scale_out: torch.Tensor,
                                 residual_out: Optional[torch.Tensor] = None,
                                 norm_out: Optional[torch.Tensor] = None, rows=None,
                                 stream=None) -> None:
    """far_fused_fp8_tensor without a workspace: the library's own scratch,
    at most FAR_FP8_TENSOR_NOALLOC_MAX_ROWS rows per call; calls that overlap
    on the GPU race (see include/far.h)."""
    (arr, W, res, rout, gam, T, H, dt, nout, qout, sin, sout) = _args(
        partials, residual, gamma, residual_out, norm_out, quant_out, None, scale_out,
        scale_out_elems=1)
    b, e = (0, T) if rows is None else (int(rows[0]), int(rows[1]))
    st = lib().far_fused_fp8_tensor_noalloc(ctx.handle, b, e, arr, W, res, rout, gam, T, H, dt,
                                            float(eps), float(weight_bias), nout, qout, sout,
                                            _stream(stream))
    if st != FAR_OK:
        raise FarError(st, "far_fused_fp8_tensor_noalloc")


class FarCall:
    """One far_fused_rows call with its arguments marshalled once.

    Calling the object enqueues the kernel again on the same buffers (whose
    contents may change between calls) with no per-call argument checks in
    Python; the library still checks every argument on its side.  Meant for
    loops of small calls (decode) where the binding's own marshalling would
    dominate the launch.  Keyword arguments as far_fused; ``rows=(b, e)``
    restricts the call to a row range.
    """

    def __init__(self, ctx: FarContext, partials: Sequence[torch.Tensor],
                 residual: Optional[torch.Tensor], gamma: torch.Tensor, eps: float,
                 weight_bias: float = 0.0, pattern: int = FAR_AR_RESIDUAL_RMSNORM, *,
                 residual_out: Optional[torch.Tensor] = None,
                 norm_out: Optional[torch.Tensor] = None,
                 quant_out: Optional[torch.Tensor] = None,
                 scale_in: Optional[torch.Tensor] = None,
                 scale_out: Optional[torch.Tensor] = None, rows=None, stream=None):
        (arr, W, res, rout, gam, T, H, dt, nout, qout, sin, sout) = _args(
            partials, residual, gamma, residual_out, norm_out, quant_out, scale_in, scale_out)
        b, e = (0, T) if rows is None else (int(rows[0]), int(rows[1]))
        # keep every tensor alive for as long as the call may be replayed
        self._keep = (list(partials) if not isinstance(partials, torch.Tensor) else [partials],
                      residual, gamma, residual_out, norm_out, quant_out, scale_in, scale_out)
        self._ctx = ctx
        self._fn = lib().far_fused_rows
        self._args = (ctx.handle, ctypes.c_int64(b), ctypes.c_int64(e), arr, ctypes.c_int(W), res,
                      rout, gam, ctypes.c_int64(T), ctypes.c_int64(H), ctypes.c_int(dt),
                      ctypes.c_float(eps), ctypes.c_float(weight_bias), ctypes.c_int(pattern),
                      nout, qout, sin, sout, _stream(stream))

    def __call__(self) -> None:
        st = self._fn(*self._args)
        if st != FAR_OK:
            raise FarError(st, "far_fused_rows")


def far_fused_fp8_group(ctx: FarContext, partials: Sequence[torch.Tensor],
                        residual: Optional[torch.Tensor], gamma: torch.Tensor, eps: float,
                        weight_bias: float = 0.0, *, group_size: int, quant_out: torch.Tensor,
                        scale_out: torch.Tensor, residual_out: Optional[torch.Tensor] = None,
                        norm_out: Optional[torch.Tensor] = None, rows=None, stream=None) -> None:
    """Per-group FP8: one scale per row and group of ``group_size``
    consecutive elements, scale_out of T x (H / group_size) floats."""
    H = gamma.numel()
    T = partials[0].numel() // H if len(partials) else 0
    if group_size < 1 or H % group_size:
        raise ValueError("group_size must divide H")
    (arr, W, res, rout, gam, T, H, dt, nout, qout, sin, sout) = _args(
        partials, residual, gamma, residual_out, norm_out, quant_out, None, scale_out,
        scale_out_elems=T * (H // group_size))
    b, e = (0, T) if rows is None else (int(rows[0]), int(rows[1]))
    st = lib().far_fused_fp8_group(ctx.handle, b, e, arr, W, res, rout, gam, T, H, dt, float(eps),
                                   float(weight_bias), int(group_size), nout, qout, sout,
                                   _stream(stream))
    if st != FAR_OK:
        raise FarError(st, "far_fused_fp8_group")


def far_host_staging_bytes(W: int, H: int, chunk_rows: int = 0) -> int:
    """Device staging bytes far_fused_host needs (0 for W or H out of range)."""
    return int(lib().far_host_staging_bytes(int(W), int(H), int(chunk_rows)))


def far_fused_host(ctx: FarContext, partials: Sequence[torch.Tensor],
                   residual: Optional[torch.Tensor], gamma: torch.Tensor, eps: float,
                   weight_bias: float = 0.0, pattern: int = FAR_AR_RESIDUAL_RMSNORM, *,
                   staging: torch.Tensor, chunk_rows: int = 0, group_size: int = 0,
                   residual_out: Optional[torch.Tensor] = None,
                   norm_out: Optional[torch.Tensor] = None,
                   quant_out: Optional[torch.Tensor] = None,
                   scale_in: Optional[torch.Tensor] = None,
                   scale_out: Optional[torch.Tensor] = None, stream=None) -> None:
    """The fused epilogue on host (CPU) tensors, through the device buffer
    ``staging`` (uint8, at least far_host_staging_bytes(W, H, chunk_rows)
    bytes) in chunks of rows; pin the host tensors for the copies to overlap
    the kernels.  Every host tensor, scale_in included, is a CPU tensor; the
    results are there once ``stream`` reaches the end of the call."""
    H = gamma.numel()
    T = partials[0].numel() // H if len(partials) else 0
    n_sc = T * (H // group_size) if pattern == FAR_AR_RESIDUAL_RMSNORM_FP8_GROUP and group_size > 0 else None
    (arr, W, res, rout, gam, T, H, dt, nout, qout, sin, sout) = _args(
        partials, residual, gamma, residual_out, norm_out, quant_out, scale_in, scale_out,
        scale_out_elems=n_sc, host=True)
    if not staging.is_cuda or not staging.is_contiguous():
        raise ValueError("staging must be a contiguous CUDA tensor")
    nbytes = staging.numel() * staging.element_size()
    st = lib().far_fused_host(ctx.handle, arr, W, res, rout, gam, T, H, dt, float(eps),
                              float(weight_bias), int(pattern), int(group_size), nout, qout, sin,
                              sout, int(chunk_rows), ctypes.c_void_p(staging.data_ptr()), nbytes,
                              _stream(stream))
    if st != FAR_OK:
        raise FarError(st, "far_fused_host")
