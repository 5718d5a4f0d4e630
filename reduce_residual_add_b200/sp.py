"""Sequence-parallel decomposition of the fused epilogue across ranks.

vllm.compilation.sequence_parallelism (SequenceParallelismPass docstring)
rewrites AllReduce -> RMSNorm as ReduceScatter -> local RMSNorm -> AllGather
over the token (row) dimension; its is_applicable() asks that the number of
tokens be divisible by the tensor-parallel size (or be padded to it).

``SequenceParallelEpilogue`` runs that decomposition over a process group of
G ranks (one per GPU).  Every rank holds its own partial -- the (T, H)
output of its row-parallel linear before the reduction -- and the n = T / G
rows of the residual it owns (rows [r n, (r + 1) n) on rank r).  One call:

1. exchange: rank r sends rows [j n, (j + 1) n) of its partial to rank j
   (``all_to_all_single`` over rows), so every rank receives the G partial
   blocks of its own rows as G separate buffers.  This is the reduce-scatter
   with its reduction moved into the kernel: the G blocks are summed in fp32
   by the epilogue kernel (W = G partials), not in the 2-byte format by the
   collective, so the result is the one-GPU result -- bit for bit when the
   local call runs with the one-GPU call's packs per thread and threads per
   row (far_describe_launch), else within the parity tolerances;
2. local step: the fused epilogue on those n rows (``far_fused``), writing
   the rows' new residual (in place, or into ``residual_out``) and the
   normed outputs;
3. all-gather of the normed outputs -- norm_out, and the FP8 codes and
   scales -- into (T, ...) tensors on every rank (the input of the next
   column-parallel layer); the new residual stays with its rows, as in the
   pages' rewrite, unless ``gather_residual`` asks for it too.

Collectives move bytes only: every buffer is exchanged through a 32-bit
view of its storage, so the same code runs over NCCL on GPUs and over gloo
(which has no 16-bit types) on CPU.  The local step is the CUDA path
(``far.far_fused``); a caller may pass another callable with its signature.
Per-tensor FP8 is not offered here: its one scale would need a reduction
across ranks between the two passes.

``PeerSequenceParallelEpilogue`` is the one-shot form of the same step: the
partials live in symmetric memory that every peer maps, and rank r's kernel
reads rows [r n, (r + 1) n) of every peer's partial itself over NVLink
(plain loads and bulk copies without cluster multicast), so step 1's copy
disappears into the kernel.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch


def is_applicable(num_tokens: int, world_size: int) -> bool:
    """True when the rows split evenly across ranks."""
    return world_size >= 1 and num_tokens % world_size == 0


def padded_tokens(num_tokens: int, world_size: int) -> int:
    """Rows after padding up to a multiple of the world size."""
    return -(-num_tokens // world_size) * world_size


def rows_for_rank(num_tokens: int, world_size: int, rank: int) -> tuple:
    """[begin, end) of the rows rank `rank` owns; requires an even split."""
    if not 0 <= rank < world_size:
        raise ValueError("rank %d outside world of %d" % (rank, world_size))
    if not is_applicable(num_tokens, world_size):
        raise ValueError("%d rows do not split over %d ranks; pad to %d"
                         % (num_tokens, world_size, padded_tokens(num_tokens, world_size)))
    n = num_tokens // world_size
    return rank * n, (rank + 1) * n


def _words(t: torch.Tensor) -> torch.Tensor:
    """The tensor's bytes as a flat int32 view (its size must be a multiple of 4)."""
    flat = t.reshape(-1)
    if (flat.numel() * flat.element_size()) % 4:
        raise ValueError("buffer of %d bytes is not a whole number of 32-bit words"
                         % (flat.numel() * flat.element_size()))
    return flat.view(torch.uint8).view(torch.int32) if flat.element_size() != 4 else flat.view(torch.int32)


class SequenceParallelEpilogue:
    """ReduceScatter -> local fused epilogue -> AllGather over ``group``.

    T: rows of the whole batch (T % G == 0); H: hidden size; dtype: bf16 or
    fp16; pattern: 0 (norm), 1 (static FP8) or 2 (per-token FP8).  Buffers
    are allocated once on ``device`` (the exchange's receive blocks and the
    gathered outputs) and reused by every call.
    """

    def __init__(self, group, T: int, H: int, dtype: torch.dtype, pattern: int,
                 device, *, with_norm: bool = False, gather_residual: bool = False,
                 local_step: Optional[Callable] = None, ctx=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if pattern not in (0, 1, 2):
            raise ValueError("pattern %d: the sequence-parallel path takes the norm, static "
                             "FP8 and per-token FP8 patterns" % pattern)
        self.T, self.H, self.dtype, self.pattern = T, H, dtype, pattern
        self.b, self.e = rows_for_rank(T, self.G, self.rank)
        n = self.n = self.e - self.b
        self.with_norm = with_norm or pattern == 0
        self.gather_residual = gather_residual
        self.ctx = ctx
        if local_step is None:
            from . import far
            local_step = far.far_fused
        self.local_step = local_step
        dev = torch.device(device)
        # the G partial blocks of this rank's rows, block j from rank j
        self.recv = torch.empty(self.G, n, H, dtype=dtype, device=dev)
        # this rank's outputs and their gathered (T, ...) forms
        self.norm_local = torch.empty(n, H, dtype=dtype, device=dev) if self.with_norm else None
        self.quant_local = torch.empty(n, H, dtype=torch.uint8, device=dev) if pattern else None
        self.scale_local = torch.empty(n, dtype=torch.float32, device=dev) if pattern == 2 else None
        self.norm_all = torch.empty(T, H, dtype=dtype, device=dev) if self.with_norm else None
        self.quant_all = torch.empty(T, H, dtype=torch.uint8, device=dev) if pattern else None
        self.scale_all = torch.empty(T, dtype=torch.float32, device=dev) if pattern == 2 else None
        self.residual_all = torch.empty(T, H, dtype=dtype, device=dev) if gather_residual else None

    def __call__(self, partial: torch.Tensor, residual: Optional[torch.Tensor], gamma: torch.Tensor,
                 eps: float, weight_bias: float = 0.0, *, residual_out: Optional[torch.Tensor] = None,
                 scale_in: Optional[torch.Tensor] = None, stream=None) -> dict:
        """One sequence-parallel step.

        partial: this rank's (T, H) partial; residual: this rank's (n, H)
        rows of the residual (None for the "First" pattern); residual_out:
        where the rows' new residual goes (None: in place into residual).
        Returns the gathered outputs (``norm_out``, ``quant_out``,
        ``scale_out`` as (T, ...) tensors, absent ones None) and the local
        new residual (``residual_out``, (n, H)), plus ``residual_all`` when
        gather_residual is set."""
        dist = self.dist
        T, H, n = self.T, self.H, self.n
        if partial.shape != (T, H) or partial.dtype != self.dtype:
            raise ValueError("partial must be (%d, %d) %s" % (T, H, self.dtype))
        if residual is not None and residual.shape != (n, H):
            raise ValueError("residual must hold this rank's %d rows" % n)
        # 1. rows of every rank's partial to their owner
        dist.all_to_all_single(_words(self.recv), _words(partial.contiguous()), group=self.group)
        # 2. the fused epilogue on this rank's rows, the G blocks as W = G partials
        rout = residual_out
        self.local_step(self.ctx, [self.recv[j] for j in range(self.G)], residual, gamma, eps,
                        weight_bias, self.pattern, residual_out=rout, norm_out=self.norm_local,
                        quant_out=self.quant_local, scale_in=scale_in, scale_out=self.scale_local,
                        stream=stream)
        new_res = rout if rout is not None else residual
        # 3. the normed outputs (and optionally the new residual) to every rank
        out = {"norm_out": None, "quant_out": None, "scale_out": None, "residual_out": new_res}
        for key, local, full in (("norm_out", self.norm_local, self.norm_all),
                                 ("quant_out", self.quant_local, self.quant_all),
                                 ("scale_out", self.scale_local, self.scale_all),
                                 ("residual_all", new_res if self.gather_residual else None,
                                  self.residual_all)):
            if local is None or full is None:
                continue
            dist.all_gather_into_tensor(_words(full), _words(local), group=self.group)
            out[key] = full
        return out


class PeerSequenceParallelEpilogue:
    """One-shot variant: the kernel pulls its rows straight from the peers.

    Every rank's partial lives in a buffer of symmetric memory
    (``self.partial``, (T, H)) that every peer has mapped into its address
    space (torch.distributed._symmetric_memory, its CUDA backend: peer
    mappings over NVLink).  Rank r's epilogue kernel gets, as its W = G
    partials, the addresses of rows [r n, (r + 1) n) in each peer's buffer
    and reads them over NVLink with the same loads it uses on local memory
    (plain 16-byte loads, or bulk copies without cluster multicast), so the
    row exchange of SequenceParallelEpilogue -- a staging copy of (G-1)/G of
    each partial -- disappears into the kernel.  One call, in stream order:

    1. a one-element all-reduce over the group: it completes on a rank only
       after every rank has reached it, i.e. after every rank's partial (the
       work before it in that rank's stream) is complete;
    2. far_fused on this rank's n rows, partials read from the G peers;
    3. all-gather of the normed outputs (as SequenceParallelEpilogue).  It
       completes on a rank only after every rank's step 2 has finished, so
       no peer is still reading this rank's partial once the next write into
       ``self.partial`` (after the call, in stream order) begins.

    The caller writes its partial into ``self.partial`` before each call.
    Results equal SequenceParallelEpilogue's bit for bit (the same kernel
    and launch geometry on the same values).
    """

    def __init__(self, group, T: int, H: int, dtype: torch.dtype, pattern: int, device, *,
                 with_norm: bool = False, ctx=None):
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        self.dist = dist
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if pattern not in (0, 1, 2):
            raise ValueError("pattern %d: the sequence-parallel path takes the norm, static "
                             "FP8 and per-token FP8 patterns" % pattern)
        self.T, self.H, self.dtype, self.pattern = T, H, dtype, pattern
        self.b, self.e = rows_for_rank(T, self.G, self.rank)
        n = self.n = self.e - self.b
        self.with_norm = with_norm or pattern == 0
        self.ctx = ctx
        dev = torch.device(device)
        self.partial = symm_mem.empty((T, H), dtype=dtype, device=dev)
        self.handle = symm_mem.rendezvous(self.partial, group)
        row_bytes = H * self.partial.element_size()
        # this rank's rows in every peer's partial, peer j's first
        self.addrs = [int(base) + self.b * row_bytes for base in self.handle.buffer_ptrs]
        self.ready = torch.zeros(1, dtype=torch.int32, device=dev)
        self.norm_local = torch.empty(n, H, dtype=dtype, device=dev) if self.with_norm else None
        self.quant_local = torch.empty(n, H, dtype=torch.uint8, device=dev) if pattern else None
        self.scale_local = torch.empty(n, dtype=torch.float32, device=dev) if pattern == 2 else None
        self.norm_all = torch.empty(T, H, dtype=dtype, device=dev) if self.with_norm else None
        self.quant_all = torch.empty(T, H, dtype=torch.uint8, device=dev) if pattern else None
        self.scale_all = torch.empty(T, dtype=torch.float32, device=dev) if pattern == 2 else None

    def __call__(self, residual: Optional[torch.Tensor], gamma: torch.Tensor, eps: float,
                 weight_bias: float = 0.0, *, residual_out: Optional[torch.Tensor] = None,
                 scale_in: Optional[torch.Tensor] = None) -> dict:
        """One step on the partial the caller wrote into ``self.partial``;
        arguments and result as SequenceParallelEpilogue.__call__ (on the
        current stream)."""
        from . import far
        dist = self.dist
        n, H = self.n, self.H
        if residual is not None and residual.shape != (n, H):
            raise ValueError("residual must hold this rank's %d rows" % n)
        dist.all_reduce(self.ready, group=self.group)
        far.far_fused_addrs(self.ctx, self.addrs, n, residual, gamma, eps, weight_bias,
                            self.pattern, residual_out=residual_out, norm_out=self.norm_local,
                            quant_out=self.quant_local, scale_in=scale_in,
                            scale_out=self.scale_local)
        out = {"norm_out": None, "quant_out": None, "scale_out": None,
               "residual_out": residual_out if residual_out is not None else residual}
        for key, local, full in (("norm_out", self.norm_local, self.norm_all),
                                 ("quant_out", self.quant_local, self.quant_all),
                                 ("scale_out", self.scale_local, self.scale_all)):
            if local is None:
                continue
            dist.all_gather_into_tensor(_words(full), _words(local), group=self.group)
            out[key] = full
        return out
