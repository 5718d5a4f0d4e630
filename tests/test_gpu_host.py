"""far_fused_host: the fused epilogue on host buffers, copied through a
device staging area in chunks of rows (copy in, kernel and copy out of
neighbouring chunks overlap on three streams).

Every case is checked against the oracle within the parity tolerances, and
one is checked bit for bit against far_fused run on each chunk's rows on
the device (the host call launches, per chunk, the kernel far_fused would).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import compare, run_oracle
from reduce_residual_add_b200 import far
from reduce_residual_add_b200.inputs import as_u16, random_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ctx():
    c = far.FarContext(0)
    yield c
    c.close()


def _host_outputs(T, H, tdt, pattern, group, want_norm, pin):
    def e(shape, dt):
        t = torch.empty(shape, dtype=dt)
        return t.pin_memory() if pin else t
    o = {"residual_out": e((T, H), tdt),
         "norm_out": e((T, H), tdt) if want_norm else None,
         "quant_out": e((T, H), torch.uint8) if pattern else None,
         "scale_out": None}
    if pattern == 2:
        o["scale_out"] = e((T,), torch.float32)
    elif pattern == 4:
        o["scale_out"] = e((T * (H // group),), torch.float32)
    return o


def run_host(ctx, inp, eps, wb, pattern, *, chunk_rows=0, group=0, scale=0.05, want_norm=True,
             in_place=False, pin=True, stream=None, staging=None):
    ps = [p.pin_memory() if pin else p.clone() for p in inp["partials"]]
    res = None if inp["residual"] is None else (inp["residual"].pin_memory() if pin
                                                else inp["residual"].clone())
    gam = inp["gamma"].clone()
    T, H = ps[0].shape
    o = _host_outputs(T, H, ps[0].dtype, pattern, group, want_norm, pin)
    rout = None if in_place else o["residual_out"]
    W = len(ps)
    if staging is None:
        staging = torch.empty(far.far_host_staging_bytes(W, H, chunk_rows), dtype=torch.uint8,
                              device="cuda")
    sin = torch.tensor([scale], dtype=torch.float32) if pattern == 1 else None
    far.far_fused_host(ctx, ps, res, gam, eps, wb, pattern, staging=staging,
                       chunk_rows=chunk_rows, group_size=group, residual_out=rout,
                       norm_out=o["norm_out"], quant_out=o["quant_out"], scale_in=sin,
                       scale_out=o["scale_out"], stream=stream)
    torch.cuda.synchronize()
    far.far_check(ctx, stream)
    src = res if in_place else rout   # where the new residual went
    out = {"residual_out": as_u16(src.reshape(T, H)),
           "norm_out": None if o["norm_out"] is None else as_u16(o["norm_out"]),
           "quant_out": None if o["quant_out"] is None else o["quant_out"].numpy(),
           "scale_out": None if o["scale_out"] is None else o["scale_out"].numpy()}
    if pattern == 4:
        out["scale_out"] = out["scale_out"].reshape(T, H // group)
    return out


@pytest.mark.parametrize("case", [
    # W, T, H, dtype, pattern, group, chunk_rows, has_res, in_place, wb
    (2, 50, 1024, "bf16", 0, 0, 7, True, False, 0.0),      # ragged last chunk
    (4, 300, 8192, "bf16", 1, 0, 64, True, True, 0.0),     # in place into the host residual
    (8, 90, 7168, "fp16", 2, 0, 0, True, False, 1.0),      # default chunk: one chunk
    (3, 41, 2048, "bf16", 4, 128, 10, True, False, 0.0),   # per-group
    (4, 33, 4096, "bf16", 2, 0, 5, False, False, 0.0),     # no residual ("First" pattern)
    (2, 5000, 4096, "bf16", 2, 0, 2500, True, False, 0.0),  # chunks on the ring kernel
    (8, 3, 4096, "bf16", 0, 0, 1, True, False, 0.0),       # decode-sized chunks of one row
], ids=lambda c: "W%d_T%d_H%d_%s_p%d_g%d_chunk%d_res%d_inpl%d_wb%g" % c)
def test_host_matches_oracle(ctx, case):
    W, T, H, dt, pattern, group, chunk, has_res, in_place, wb = case
    inp = random_inputs(W, T, H, dtype=dt, seed=4000 + T + H, has_residual=has_res)
    got = run_host(ctx, inp, 1e-6, wb, pattern, chunk_rows=chunk, group=group, in_place=in_place,
                   want_norm=(pattern == 0 or W % 2 == 0))
    ref = run_oracle(inp, dt, 1e-6, wb, pattern, scale_in=0.05, group=group,
                     want_norm=(pattern == 0 or W % 2 == 0))
    compare(got, ref, dt)


def test_host_chunks_equal_device_calls_bitwise(ctx):
    """Each chunk's outputs are those of far_fused on that chunk's rows."""
    W, T, H, R = 4, 700, 4096, 256
    inp = random_inputs(W, T, H, seed=4321)
    got = run_host(ctx, inp, 1e-6, 0.0, 2, chunk_rows=R)
    for r0 in range(0, T, R):
        n = min(R, T - r0)
        ps = [p[r0:r0 + n].cuda() for p in inp["partials"]]
        res = inp["residual"][r0:r0 + n].cuda()
        rout = torch.empty_like(res)
        q = torch.empty(n, H, dtype=torch.uint8, device="cuda")
        sc = torch.empty(n, dtype=torch.float32, device="cuda")
        nout = torch.empty_like(res)
        far.far_fused(ctx, ps, res, inp["gamma"].cuda(), 1e-6, 0.0, 2, residual_out=rout,
                      norm_out=nout, quant_out=q, scale_out=sc)
        torch.cuda.synchronize()
        assert np.array_equal(got["residual_out"][r0:r0 + n], as_u16(rout.cpu()))
        assert np.array_equal(got["norm_out"][r0:r0 + n], as_u16(nout.cpu()))
        assert np.array_equal(got["quant_out"][r0:r0 + n], q.cpu().numpy())
        assert np.array_equal(got["scale_out"][r0:r0 + n], sc.cpu().numpy())


def test_host_calls_back_to_back_share_staging(ctx):
    """Two calls on different streams with one staging area and context:
    the second waits, through the context's events, for the first one's
    copies out of each staging buffer."""
    W, H, R = 2, 2048, 16
    a = random_inputs(W, 100, H, seed=11)
    b = random_inputs(W, 37, H, seed=12)
    staging = torch.empty(far.far_host_staging_bytes(W, H, R), dtype=torch.uint8, device="cuda")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    got_a = run_host(ctx, a, 1e-6, 0.0, 1, chunk_rows=R, stream=s1, staging=staging)
    got_b = run_host(ctx, b, 1e-6, 0.0, 1, chunk_rows=R, stream=s2, staging=staging)
    compare(got_a, run_oracle(a, "bf16", 1e-6, 0.0, 1, scale_in=0.05), "bf16")
    compare(got_b, run_oracle(b, "bf16", 1e-6, 0.0, 1, scale_in=0.05), "bf16")


def test_host_calls_overlap_on_two_streams(ctx):
    """Two calls with one staging area and context, on two streams, enqueued
    back to back with no wait between them: the second rewrites gamma and
    the static scale only after the first call's kernels are done, and each
    staging buffer only after the first call copied it out."""
    W, H, R = 2, 2048, 16
    a = random_inputs(W, 100, H, seed=21)
    b = random_inputs(W, 37, H, seed=22)
    b["gamma"] = b["gamma"] * 2          # a late overwrite of gamma would show
    staging = torch.empty(far.far_host_staging_bytes(W, H, R), dtype=torch.uint8, device="cuda")
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    calls = []
    for inp, s, scale in ((a, s1, 0.05), (b, s2, 0.1)):
        T = inp["partials"][0].shape[0]
        keep = {"ps": [p.pin_memory() for p in inp["partials"]],
                "res": inp["residual"].pin_memory(),
                "rout": torch.empty(T, H, dtype=torch.bfloat16).pin_memory(),
                "nout": torch.empty(T, H, dtype=torch.bfloat16).pin_memory(),
                "q": torch.empty(T, H, dtype=torch.uint8).pin_memory(),
                "sin": torch.tensor([scale], dtype=torch.float32)}
        far.far_fused_host(ctx, keep["ps"], keep["res"], inp["gamma"], 1e-6, 0.0, 1,
                           staging=staging, chunk_rows=R, residual_out=keep["rout"],
                           norm_out=keep["nout"], quant_out=keep["q"], scale_in=keep["sin"],
                           stream=s)
        calls.append((inp, scale, keep))    # the host tensors live until the end
    torch.cuda.synchronize()
    far.far_check(ctx)
    for inp, scale, keep in calls:
        got = {"residual_out": as_u16(keep["rout"]), "norm_out": as_u16(keep["nout"]),
               "quant_out": keep["q"].numpy(), "scale_out": None}
        compare(got, run_oracle(inp, "bf16", 1e-6, 0.0, 1, scale_in=scale), "bf16")


def test_host_pageable_memory(ctx):
    inp = random_inputs(2, 60, 1024, seed=13)
    got = run_host(ctx, inp, 1e-6, 0.0, 2, chunk_rows=16, pin=False)
    compare(got, run_oracle(inp, "bf16", 1e-6, 0.0, 2), "bf16")


def test_host_empty_and_errors(ctx):
    inp = random_inputs(2, 8, 256, seed=14)
    ps = [p.pin_memory() for p in inp["partials"]]
    res, gam = inp["residual"].pin_memory(), inp["gamma"]
    staging = torch.empty(far.far_host_staging_bytes(2, 256, 4), dtype=torch.uint8, device="cuda")
    q = torch.empty(8, 256, dtype=torch.uint8)
    sc = torch.empty(8, dtype=torch.float32)
    rout = torch.empty(8, 256, dtype=torch.bfloat16)
    kw = dict(staging=staging, chunk_rows=4, residual_out=rout, quant_out=q, scale_out=sc)
    # T = 0 is a no-op
    e0 = [p[:0] for p in ps]
    far.far_fused_host(ctx, e0, res[:0], gam, 1e-6, 0.0, 2, staging=staging, chunk_rows=4,
                       residual_out=rout[:0], quant_out=q[:0], scale_out=sc[:0])
    with pytest.raises(far.FarError) as e:   # per-tensor FP8: refused
        far.far_fused_host(ctx, ps, res, gam, 1e-6, 0.0, 3, **kw)
    assert e.value.status == far.FAR_ERR_UNSUPPORTED
    with pytest.raises(far.FarError) as e:   # staging sized for smaller chunks
        far.far_fused_host(ctx, ps, res, gam, 1e-6, 0.0, 2, **dict(kw, chunk_rows=8))
    assert e.value.status == far.FAR_ERR_INVALID_ARG
    with pytest.raises(far.FarError) as e:
        far.far_fused_host(ctx, ps, res, gam, 1e-6, 0.0, 2, **dict(kw, chunk_rows=-1))
    assert e.value.status == far.FAR_ERR_INVALID_ARG
    big = torch.empty(staging.numel() + 512, dtype=torch.uint8, device="cuda")
    with pytest.raises(far.FarError) as e:   # staging not 256-byte aligned
        far.far_fused_host(ctx, ps, res, gam, 1e-6, 0.0, 2, **dict(kw, staging=big[16:]))
    assert e.value.status == far.FAR_ERR_ALIGNMENT
    with pytest.raises(ValueError):          # device tensors are refused by the binding
        far.far_fused_host(ctx, [p.cuda() for p in ps], res, gam, 1e-6, 0.0, 2, **kw)
    # nothing was written by the refused calls
    torch.cuda.synchronize()
