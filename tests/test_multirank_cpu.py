"""World-size-2 checks of the multi-rank host logic on CPU (gloo).

* The sequence-parallel decomposition: each rank owns a contiguous block of
  rows (sp.rows_for_rank), runs the epilogue on it, and an all-gather of the
  blocks equals the full-row result bit for bit (the oracle stands in for
  the kernel here; the GPU tests check the kernel's row slices).
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


def _worker(rank, world, port, q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        import oracle
        from reduce_residual_add_b200.inputs import as_u16, random_inputs
        import bench

        inp = random_inputs(4, 64, 256, seed=123)     # every rank sees all partials
        ps = [as_u16(p) for p in inp["partials"]]
        res, gam = as_u16(inp["residual"]), as_u16(inp["gamma"])
        b, e = sp.rows_for_rank(64, world, rank)
        local = oracle.fused(ps, res, gam, "bf16", 1e-6, 0.0, 2, rows=(b, e))
        # all-gather the local blocks (int32 carriers for the 16-bit patterns)
        mine_n = torch.from_numpy(local["norm_out"][b:e].astype(np.int32))
        mine_q = torch.from_numpy(local["quant_out"][b:e].astype(np.int32))
        mine_s = torch.from_numpy(local["scale_out"][b:e].copy())
        gn = [torch.empty_like(mine_n) for _ in range(world)]
        gq = [torch.empty_like(mine_q) for _ in range(world)]
        gs = [torch.empty_like(mine_s) for _ in range(world)]
        dist.all_gather(gn, mine_n)
        dist.all_gather(gq, mine_q)
        dist.all_gather(gs, mine_s)
        full = oracle.fused(ps, res, gam, "bf16", 1e-6, 0.0, 2)
        ok = (np.array_equal(torch.cat(gn).numpy().astype(np.uint16), full["norm_out"]) and
              np.array_equal(torch.cat(gq).numpy().astype(np.uint8), full["quant_out"]) and
              np.array_equal(torch.cat(gs).numpy(), full["scale_out"]))
        # bench's reductions: max of times, sum of bytes
        t = bench.max_over_ranks(1.0 + rank, world, device="cpu")
        nbytes = bench.sum_over_ranks(100.0 * (rank + 1), world, device="cpu")
        q.put((rank, ok, t, nbytes))
        dist.destroy_process_group()
    except Exception as ex:  # report instead of hanging the parent
        q.put((rank, "error: %r" % (ex,), None, None))


def test_two_rank_row_decomposition_and_bench_reductions():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    for rank, ok, t, nbytes in out:
        assert ok is True, ok
        assert t == 2.0
        assert nbytes == 300.0


def test_row_partition_rules():
    assert sp.rows_for_rank(8192, 4, 0) == (0, 2048)
    assert sp.rows_for_rank(8192, 4, 3) == (6144, 8192)
    assert sp.is_applicable(1024, 2) and not sp.is_applicable(1023, 2)
    assert sp.padded_tokens(1023, 2) == 1024
    with pytest.raises(ValueError):
        sp.rows_for_rank(10, 4, 0)
    with pytest.raises(ValueError):
        sp.rows_for_rank(8, 2, 2)
