"""Helpers of the GPU parity tests: run the CUDA path through the binding and
compare it with the oracle under the stated tolerances.

Tolerances:
* bf16 / fp16 outputs: at most 1 ulp from the oracle's correctly rounded
  value (distance on the format's ordered grid, subnormals included; the sign
  of a zero is not compared);
* e4m3 codes: at most 1 step on the ordered code grid; a code the oracle
  saturates (+-448) must be saturated on the GPU too (except where no code
  can be clamped, see ``compare``); NaN codes must agree;
* per-token scales: relative error at most 1e-6 (exact when 0);
* all of these against the oracle with exact accumulation, except at the
  rare elements where the pages' fp32 accumulation is not exact (a rounded
  running sum followed by cancellation): there against the oracle with fp32
  accumulation (see ``compare``).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from reduce_residual_add_b200 import far
from reduce_residual_add_b200.inputs import as_u16

SCALE_RTOL = 1e-6


def _ordered(bits: np.ndarray, width: int) -> np.ndarray:
    b = bits.astype(np.int64)
    sign = 1 << (width - 1)
    mag = b & (sign - 1)
    return np.where(b & sign, -mag, mag)


def _is_nan16(bits: np.ndarray, dtype: str) -> np.ndarray:
    b = bits.astype(np.int64) & 0x7FFF
    if dtype == "bf16":
        return b > 0x7F80
    return b > 0x7C00


def ulp16(a: np.ndarray, b: np.ndarray, dtype: str) -> np.ndarray:
    d = np.abs(_ordered(a, 16) - _ordered(b, 16))
    na, nb = _is_nan16(a, dtype), _is_nan16(b, dtype)
    d = np.where(na & nb, 0, d)
    return np.where(na ^ nb, 1 << 20, d)


def code_steps(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    d = np.abs(_ordered(a, 8) - _ordered(b, 8))
    na, nb = (a & 0x7F) == 0x7F, (b & 0x7F) == 0x7F
    d = np.where(na & nb, 0, d)
    return np.where(na ^ nb, 1 << 20, d)


def to_gpu(inp: dict, device="cuda") -> dict:
    g = {"partials": [p.to(device) for p in inp["partials"]],
         "residual": None if inp["residual"] is None else inp["residual"].to(device),
         "gamma": inp["gamma"].to(device)}
    return g


def run_gpu(ctx, g: dict, eps: float, wb: float, pattern: int, scale_in=None, rows=None,
            want_norm: bool = True, want_residual_out: bool = True, in_place: bool = False,
            stream=None, guard: int = 0, group: int = 0) -> dict:
    """One call of the CUDA path; returns numpy arrays of the outputs (full T).

    ``guard`` > 0 surrounds every output with that many canary bytes (0xA5)
    and checks afterwards that none of them changed."""
    ps = g["partials"]
    T, H = ps[0].reshape(-1, g["gamma"].numel()).shape
    dt = ps[0].dtype
    dev = ps[0].device
    canaries = []

    def alloc(n_elems, dtype_):
        es = torch.empty((), dtype=dtype_).element_size()
        gb = (guard + 15) // 16 * 16
        raw = torch.full((gb * 2 + n_elems * es,), 0xA5, dtype=torch.uint8, device=dev)
        view = raw[gb:gb + n_elems * es].view(dtype_)
        if guard:
            canaries.append((raw, gb, n_elems * es))
        else:
            view.zero_()
        return view

    res = g["residual"]
    rout = None
    if res is not None and in_place:
        res = res.clone()
    elif want_residual_out:
        rout = alloc(T * H, dt).view(T, H)
    nout = alloc(T * H, dt).view(T, H) if want_norm else None
    qout = alloc(T * H, torch.uint8).view(T, H) if pattern != 0 else None
    sout = (alloc({2: T, 3: 1, 4: T * (H // group if group else 1)}[pattern], torch.float32)
            if pattern in (2, 3, 4) else None)
    sin = torch.tensor([scale_in], dtype=torch.float32, device=dev) if pattern == 1 else None
    if pattern == 4:
        far.far_fused_fp8_group(ctx, ps, res, g["gamma"], eps, wb, group_size=group, quant_out=qout,
                                scale_out=sout, residual_out=rout, norm_out=nout, rows=rows,
                                stream=stream)
    elif pattern == 3:
        nrows = T if rows is None else rows[1] - rows[0]
        ws = torch.empty(far.far_fp8_tensor_workspace_bytes(nrows), dtype=torch.uint8, device=dev)
        assert ws.data_ptr() % 256 == 0
        far.far_fused_fp8_tensor(ctx, ps, res, g["gamma"], eps, wb, quant_out=qout, scale_out=sout,
                                 workspace=ws, residual_out=rout, norm_out=nout, rows=rows,
                                 stream=stream)
    else:
        kw = dict(residual_out=rout, norm_out=nout, quant_out=qout, scale_in=sin, scale_out=sout,
                  stream=stream)
        if rows is None:
            far.far_fused(ctx, ps, res, g["gamma"], eps, wb, pattern, **kw)
        else:
            far.far_fused_rows(ctx, rows[0], rows[1], ps, res, g["gamma"], eps, wb, pattern, **kw)
    torch.cuda.synchronize()
    far.far_check(ctx, stream)          # no bounded wait inside the kernel gave up
    for raw, gb, n in canaries:
        head, tail = raw[:gb], raw[gb + n:]
        assert bool((head == 0xA5).all()) and bool((tail == 0xA5).all()), "write outside an output"
    out = {}
    if in_place and res is not None:
        out["residual_out"] = as_u16(res.cpu().reshape(T, H))
    elif rout is not None:
        out["residual_out"] = as_u16(rout.cpu())
    else:
        out["residual_out"] = None
    out["norm_out"] = None if nout is None else as_u16(nout.cpu())
    out["quant_out"] = None if qout is None else qout.cpu().numpy()
    out["scale_out"] = None if sout is None else sout.cpu().numpy()
    if pattern == 4:
        out["scale_out"] = out["scale_out"].reshape(T, H // group)
    return out


def run_oracle(inp: dict, dtype: str, eps, wb, pattern, scale_in=None, rows=None, want_norm=True,
               want_residual_out=True, row_list=None, group=0, acc32=False) -> dict:
    """The oracle's outputs for the call (exact accumulation of the partials),
    with ``_redo32``: a function that recomputes them with fp32
    accumulation (oracle.fused acc32), used by ``compare`` only for elements
    that miss the tolerances."""
    ps = [as_u16(p) for p in inp["partials"]]
    res = None if inp["residual"] is None else as_u16(inp["residual"])
    gam = as_u16(inp["gamma"])
    if row_list is not None and pattern == 3:
        raise ValueError("the per-tensor scale needs every row of the call")
    if row_list is None:
        out = oracle.fused(ps, res, gam, dtype, eps, wb, pattern, scale_in=scale_in, rows=rows,
                           want_norm=want_norm, want_residual_out=want_residual_out, group=group,
                           acc32=acc32)
    else:
        out = None
        for t in row_list:
            out = oracle.fused(ps, res, gam, dtype, eps, wb, pattern, scale_in=scale_in,
                               rows=(int(t), int(t) + 1), want_norm=want_norm,
                               want_residual_out=want_residual_out, out=out, group=group,
                               acc32=acc32)
    if not acc32:
        out["_redo32"] = lambda: run_oracle(inp, dtype, eps, wb, pattern, scale_in=scale_in,
                                            rows=rows, want_norm=want_norm,
                                            want_residual_out=want_residual_out,
                                            row_list=row_list, group=group, acc32=True)
    return out


def _ref32(ref: dict):
    """The fp32-accumulation reference of ``ref`` (computed once), or None."""
    if "_ref32" not in ref:
        redo = ref.get("_redo32")
        ref["_ref32"] = redo() if redo is not None else None
    return ref["_ref32"]


def _cancellation_mask(ref: dict, r32: dict, sel) -> np.ndarray:
    """Elements (of the selected rows) where fp32 accumulation changes any
    output: there the pages' fp32 sum is not exact."""
    m = None
    for key in ("residual_out", "norm_out", "quant_out"):
        if ref.get(key) is not None and r32.get(key) is not None:
            k = ref[key][sel] != r32[key][sel]
            m = k if m is None else (m | k)
    return m


def _scale_rel(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    a, b = a.astype(np.float64), b.astype(np.float64)
    return np.where(b == 0, np.abs(a), np.abs(a - b) / np.where(b == 0, 1, np.abs(b)))


def compare(gpu: dict, ref: dict, dtype: str, rows=None, exact_saturation: bool = True) -> dict:
    """Assert the tolerances on the selected rows; return match statistics.

    The reference is the oracle with exact accumulation of the partials.
    The pages prescribe fp32 accumulation (fp32_acc=True), which is exact
    unless a rounded running sum meets cancellation; an element that misses
    a tolerance passes only if it is such an element -- the oracle with fp32
    accumulation (``run_oracle``'s ``_redo32``) gives a different output
    there -- and the GPU meets the same tolerance against that reference.
    ``stats[key][2]`` counts the elements that took this path.

    ``exact_saturation``: where the oracle's code is +-448 the GPU's must be
    too.  Per-tensor FP8 whose codes come from the stored new residual or
    norm_out passes False: its quotient never exceeds 448 (the scale is
    amax / 448), so no code is clamped, and a code that rounds up to 448
    follows the one-step rule like every other code."""
    sel = slice(None) if rows is None else rows
    stats = {}

    def check(key, dist, tol):
        d = dist(gpu[key][sel], ref[key][sel])
        n32 = 0
        bad = d > tol
        if bad.any():
            r32 = _ref32(ref)
            assert r32 is not None, (key, int(d.max()), np.argwhere(bad)[:5].tolist())
            cancel = _cancellation_mask(ref, r32, sel)
            d32 = dist(gpu[key][sel], r32[key][sel])
            ok = cancel & (d32 <= tol)
            assert np.all(ok[bad]), (key, int(d.max()), np.argwhere(bad & ~ok)[:5].tolist())
            n32 = int(bad.sum())
            d = np.where(bad, d32, d)
        stats[key] = (int(d.max()) if d.size else 0, float((d == 0).mean()) if d.size else 1.0, n32)
        return d

    for key in ("residual_out", "norm_out"):
        if ref.get(key) is None:
            continue
        assert gpu[key] is not None, key
        check(key, lambda a, b: ulp16(a, b, dtype), 1)
    if ref.get("quant_out") is not None:
        check("quant_out", code_steps, 1)
        if exact_saturation:
            a, b = gpu["quant_out"][sel], ref["quant_out"][sel]
            sat = (b & 0x7F) == 0x7E
            if not np.array_equal(a[sat], b[sat]):
                r32 = _ref32(ref)
                b32 = r32["quant_out"][sel]
                sat32 = (b32 & 0x7F) == 0x7E
                assert np.array_equal(a[sat & sat32], b[sat & sat32]) and np.all(
                    (a == b) | (a == b32) | ~sat), "saturated codes differ"
    if ref.get("scale_out") is not None:
        a, b = gpu["scale_out"][sel], ref["scale_out"][sel]
        rel = _scale_rel(a, b)
        n32 = 0
        if rel.size and rel.max() > SCALE_RTOL:
            # a scale whose amax element is a cancellation element
            b32 = _ref32(ref)["scale_out"][sel]
            rel32 = _scale_rel(a, b32)
            bad = rel > SCALE_RTOL
            assert np.all((rel32 <= SCALE_RTOL)[bad] & (b32 != b)[bad]), ("scale_out", float(rel.max()))
            n32 = int(bad.sum())
            rel = np.where(bad, rel32, rel)
        stats["scale_out"] = (float(rel.max()) if rel.size else 0.0,
                              float((a == b).mean()) if a.size else 1.0, n32)
    return stats
