"""far_fused_fp8_tensor_noalloc: per-tensor FP8 for callers that cannot
allocate device memory.

Some callers cannot call cudaMalloc: servers that give all free device
memory to a fixed pool at start-up, plain-C callers without a device
allocator, loops that cannot take the synchronisation of cudaMalloc /
cudaFree.  This entry point runs the same two-pass per-tensor FP8 epilogue
as far_fused_fp8_tensor, with the library's own fixed scratch in place of a
caller workspace.  The test calls it through the C ABI twice in a row -- the
second call on smaller inputs, so a scratch that still held the first call's
amax would give the wrong scale -- and checks each result bit for bit against
far_fused_fp8_tensor (the entry point with a workspace) and against the
oracle within the parity tolerances used everywhere else, on whole calls and
on row ranges that start past row 0.  It runs alone or after the other tests.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from gpu_util import compare, run_oracle, to_gpu
from reduce_residual_add_b200 import far
from reduce_residual_add_b200.inputs import as_u16, random_inputs

pytestmark = pytest.mark.gpu


def _outputs(T, H, dtype, with_norm=True):
    return {"residual_out": torch.zeros(T, H, dtype=dtype, device="cuda"),
            "norm_out": torch.zeros(T, H, dtype=dtype, device="cuda") if with_norm else None,
            "quant_out": torch.zeros(T, H, dtype=torch.uint8, device="cuda"),
            "scale_out": torch.zeros(1, dtype=torch.float32, device="cuda")}


def _numpy(o):
    return {"residual_out": as_u16(o["residual_out"].cpu()),
            "norm_out": None if o["norm_out"] is None else as_u16(o["norm_out"].cpu()),
            "quant_out": o["quant_out"].cpu().numpy(), "scale_out": o["scale_out"].cpu().numpy()}


def _c_abi_noalloc(ctx, g, out, eps, wb, rows):
    """One far_fused_fp8_tensor_noalloc call through the raw C function."""
    ps = g["partials"]
    T, H = ps[0].shape
    arr = (ctypes.c_void_p * len(ps))(*[p.data_ptr() for p in ps])
    vp = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    dt = far.FAR_BF16 if ps[0].dtype == torch.bfloat16 else far.FAR_FP16
    return far.lib().far_fused_fp8_tensor_noalloc(
        ctx.handle, rows[0], rows[1], arr, len(ps), vp(g["residual"]), vp(out["residual_out"]),
        vp(g["gamma"]), T, H, dt, eps, wb, vp(out["norm_out"]), vp(out["quant_out"]),
        vp(out["scale_out"]), stream)


def _check_call(ctx, inp, dt, dtype, rows, with_norm):
    """One no-alloc call: against the workspace entry point on the same
    inputs (bit for bit: the same kernels and plan) and against the oracle
    (the stated tolerances)."""
    g = to_gpu(inp)
    T, H = g["partials"][0].shape
    mine = _outputs(T, H, dtype, with_norm)
    st = _c_abi_noalloc(ctx, g, mine, 1e-6, 0.5, rows)
    assert st == far.FAR_OK, far.far_status_string(st) + " " + far.far_last_error()
    ref = _outputs(T, H, dtype, with_norm)
    ws = torch.empty(far.far_fp8_tensor_workspace_bytes(rows[1] - rows[0]), dtype=torch.uint8,
                     device="cuda")
    far.far_fused_fp8_tensor(ctx, g["partials"], g["residual"], g["gamma"], 1e-6, 0.5,
                             quant_out=ref["quant_out"], scale_out=ref["scale_out"],
                             workspace=ws, residual_out=ref["residual_out"],
                             norm_out=ref["norm_out"], rows=rows)
    torch.cuda.synchronize()
    far.far_check(ctx)
    a, b = _numpy(mine), _numpy(ref)
    for k in a:
        if a[k] is not None:
            assert np.array_equal(a[k], b[k]), k
    orc = run_oracle(inp, dt, 1e-6, 0.5, 3, rows=rows, want_norm=with_norm)
    compare(a, orc, dt, rows=slice(rows[0], rows[1]), exact_saturation=False)


@pytest.mark.parametrize("W,T,H,dtype,rows,with_norm", [
    (4, 3000, 8192, torch.bfloat16, None, True),
    (8, 40, 7168, torch.float16, None, True),
    (4, 3000, 8192, torch.bfloat16, (1000, 3000), False),   # a row offset into the scratch
    (3, 700, 2048, torch.float16, (5, 650), True),
])
def test_noalloc_matches_workspace_entry_point_and_oracle_on_two_calls(W, T, H, dtype, rows, with_norm):
    ctx = far.FarContext(0)
    try:
        dt = "bf16" if dtype == torch.bfloat16 else "fp16"
        rr = (0, T) if rows is None else rows
        for call, sigma in enumerate((1.0, 0.25)):     # the second call has the smaller amax
            inp = random_inputs(W, T, H, dtype=dt, seed=900 + call, partial_sigma=sigma,
                                residual_sigma=sigma)
            _check_call(ctx, inp, dt, dtype, rr, with_norm)
    finally:
        ctx.close()


def test_noalloc_rejects_more_rows_than_its_scratch():
    ctx = far.FarContext(0)
    try:
        T, H = far.FAR_FP8_TENSOR_NOALLOC_MAX_ROWS + 1, 8
        p = torch.zeros(T, H, dtype=torch.bfloat16, device="cuda")
        out = _outputs(T, H, torch.bfloat16)
        g = {"partials": [p], "residual": None, "gamma": torch.ones(H, dtype=torch.bfloat16, device="cuda")}
        st = _c_abi_noalloc(ctx, g, out, 1e-6, 0.0, (0, T))
        assert st == far.FAR_ERR_UNSUPPORTED
        assert "at most %d rows" % far.FAR_FP8_TENSOR_NOALLOC_MAX_ROWS in far.far_last_error()
        # the largest call it accepts
        st = _c_abi_noalloc(ctx, g, out, 1e-6, 0.0, (1, T))
        assert st == far.FAR_OK
        torch.cuda.synchronize()
        far.far_check(ctx)
    finally:
        ctx.close()
