"""The sequence-parallel path on a B200 through NCCL, at one rank.

Each variant of reduce_residual_add_b200.sp -- the row exchange
(SequenceParallelEpilogue) and the one-shot form whose kernel reads the
partials from symmetric memory (PeerSequenceParallelEpilogue) -- runs in a
child process with a one-rank NCCL group and must give far_fused's outputs
bit for bit.  (More ranks need more GPUs; the multi-rank host logic is
covered over gloo in test_multirank_cpu.py.)
"""
from __future__ import annotations

import datetime
import socket

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _child(port, q):
    try:
        import torch.distributed as dist
        from reduce_residual_add_b200 import far, sp
        from reduce_residual_add_b200.inputs import random_inputs
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        dist.init_process_group("nccl", rank=0, world_size=1,
                                init_method="tcp://127.0.0.1:%d" % port,
                                timeout=datetime.timedelta(seconds=60), device_id=dev)
        ctx = far.FarContext(0)
        T, H = 512, 4096
        inp = random_inputs(1, T, H, seed=5)
        p = inp["partials"][0].to(dev)
        res = inp["residual"].to(dev)
        gam = inp["gamma"].to(dev)
        results = []
        for pattern in (0, 1, 2):
            sin = torch.tensor([0.05], device=dev) if pattern == 1 else None
            ref = {"norm_out": torch.empty_like(res) if pattern == 0 else None,
                   "quant_out": torch.empty(T, H, dtype=torch.uint8, device=dev) if pattern else None,
                   "scale_out": torch.empty(T, device=dev) if pattern == 2 else None}
            rref = torch.empty_like(res)
            far.far_fused(ctx, [p], res, gam, 1e-6, 0.0, pattern, residual_out=rref, scale_in=sin,
                          **ref)
            a = sp.SequenceParallelEpilogue(dist.group.WORLD, T, H, torch.bfloat16, pattern, dev,
                                            ctx=ctx)
            ra = torch.empty_like(res)
            oa = a(p, res, gam, 1e-6, 0.0, residual_out=ra, scale_in=sin)
            b = sp.PeerSequenceParallelEpilogue(dist.group.WORLD, T, H, torch.bfloat16, pattern,
                                                dev, ctx=ctx)
            b.partial.copy_(p)
            rb = torch.empty_like(res)
            ob = b(res, gam, 1e-6, 0.0, residual_out=rb, scale_in=sin)
            torch.cuda.synchronize()
            ok = torch.equal(ra, rref) and torch.equal(rb, rref)
            for key, want in ref.items():
                if want is not None:
                    ok = ok and torch.equal(oa[key], want) and torch.equal(ob[key], want)
            results.append(bool(ok))
            del a, b
        far.far_check(ctx)
        ctx.close()
        dist.destroy_process_group()
        q.put(results)
    except Exception as ex:  # report instead of hanging the parent
        import traceback
        q.put("error: %r %s" % (ex, traceback.format_exc()))


def test_sequence_parallel_variants_at_one_rank_equal_far_fused():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    proc = ctx.Process(target=_child, args=(_free_port(), q))
    proc.start()
    out = q.get(timeout=240)
    proc.join(timeout=60)
    assert isinstance(out, list) and all(out), out
