"""Multi-rank host logic on CPU (gloo, world sizes 2 and 4).

* The sequence-parallel path (sp.SequenceParallelEpilogue): every rank holds
  its own partial and its rows of the residual; the row exchange, the local
  epilogue and the all-gather give the full-batch result bit for bit (the
  oracle stands in for the kernel as the local step; the GPU tests check
  the kernel on row slices and on W = G partials).
* bench.py's timing rule: the reported time is the max over ranks and the
  bytes are summed over ranks.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from reduce_residual_add_b200 import sp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_step(ctx, partials, residual, gamma, eps, wb, pattern, *, residual_out=None,
                 norm_out=None, quant_out=None, scale_in=None, scale_out=None, stream=None):
    """The local step of the sequence-parallel path with the oracle in place
    of the kernel: same signature as far.far_fused, CPU tensors."""
    import oracle
    from reduce_residual_add_b200.inputs import as_u16
    dt = "bf16" if gamma.dtype == torch.bfloat16 else "fp16"
    ps = [as_u16(p_) for p_ in partials]
    res = None if residual is None else as_u16(residual)
    r = oracle.fused(ps, res, as_u16(gamma), dt, eps, wb, pattern,
                     scale_in=None if scale_in is None else float(scale_in[0]),
                     want_norm=norm_out is not None)
    rout = residual_out if residual_out is not None else residual
    if rout is not None:
        rout.copy_(torch.from_numpy(r["residual_out"].view(np.int16)).view(gamma.dtype))
    if norm_out is not None:
        norm_out.copy_(torch.from_numpy(r["norm_out"].view(np.int16)).view(gamma.dtype))
    if quant_out is not None:
        quant_out.copy_(torch.from_numpy(r["quant_out"]))
    if scale_out is not None:
        scale_out.copy_(torch.from_numpy(r["scale_out"]))


def _worker(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import oracle
        from reduce_residual_add_b200.inputs import as_u16, random_inputs
        import bench

        T, H = 64, 256
        results = []
        for pattern, dt, in_place, gather_res in ((0, "bf16", False, True), (1, "fp16", True, False),
                                                  (2, "bf16", False, True), (2, "fp16", True, True)):
            # the whole problem: W = world partials, one per rank
            inp = random_inputs(world, T, H, dtype=dt, seed=123 + pattern)
            ps = [as_u16(p_) for p_ in inp["partials"]]
            res, gam = as_u16(inp["residual"]), as_u16(inp["gamma"])
            scale = 0.05 if pattern == 1 else None
            full = oracle.fused(ps, res, gam, dt, 1e-6, 0.5, pattern, scale_in=scale,
                                want_norm=pattern == 0)
            b, e = sp.rows_for_rank(T, world, rank)
            step = sp.SequenceParallelEpilogue(None, T, H, inp["gamma"].dtype, pattern, "cpu",
                                               gather_residual=gather_res, local_step=_oracle_step)
            my_res = inp["residual"][b:e].clone()
            rout = None if in_place else torch.empty_like(my_res)
            sin = torch.tensor([scale], dtype=torch.float32) if pattern == 1 else None
            out = step(inp["partials"][rank], my_res, inp["gamma"], 1e-6, 0.5, residual_out=rout,
                       scale_in=sin)
            ok = np.array_equal(as_u16(out["residual_out"]), full["residual_out"][b:e])
            if in_place:
                ok = ok and out["residual_out"].data_ptr() == my_res.data_ptr()
            if pattern == 0:
                ok = ok and np.array_equal(as_u16(out["norm_out"]), full["norm_out"])
            else:
                ok = ok and np.array_equal(out["quant_out"].numpy(), full["quant_out"])
            if pattern == 2:
                ok = ok and np.array_equal(out["scale_out"].numpy(), full["scale_out"])
            if gather_res:
                ok = ok and np.array_equal(as_u16(out["residual_all"]), full["residual_out"])
            results.append(bool(ok))
        # bench's reductions: max of times, sum of bytes
        t = bench.max_over_ranks(1.0 + rank, world, device="cpu")
        nbytes = bench.sum_over_ranks(100.0 * (rank + 1), world, device="cpu")
        q.put((rank, results, t, nbytes))
        dist.destroy_process_group()
    except Exception as ex:  # report instead of hanging the parent
        import traceback
        q.put((rank, "error: %r %s" % (ex, traceback.format_exc()), None, None))


@pytest.mark.parametrize("world", [2, 4])
def test_sequence_parallel_epilogue_equals_one_gpu_result(world):
    """ReduceScatter (as a row exchange) -> local epilogue -> AllGather over
    gloo ranks gives the full-batch result bit for bit, for the norm, static
    and per-token FP8 patterns, in place and into residual_out."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    for rank, ok, t, nbytes in out:
        assert isinstance(ok, list) and all(ok), ok
        assert t == float(world)
        assert nbytes == 100.0 * world * (world + 1) / 2


def test_row_partition_rules():
    assert sp.rows_for_rank(8192, 4, 0) == (0, 2048)
    assert sp.rows_for_rank(8192, 4, 3) == (6144, 8192)
    assert sp.is_applicable(1024, 2) and not sp.is_applicable(1023, 2)
    assert sp.padded_tokens(1023, 2) == 1024
    with pytest.raises(ValueError):
        sp.rows_for_rank(10, 4, 0)
    with pytest.raises(ValueError):
        sp.rows_for_rank(8, 2, 2)
