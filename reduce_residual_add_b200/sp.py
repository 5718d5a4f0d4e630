"""Row partition of the sequence-parallel decomposition.

vllm.compilation.sequence_parallelism (SequenceParallelismPass docstring)
rewrites AllReduce -> RMSNorm as ReduceScatter -> local RMSNorm -> AllGather
over the token (row) dimension; its is_applicable() asks that the number of
tokens be divisible by the tensor-parallel size (or be padded to it).  Each
rank then runs far_fused_rows() on its own contiguous block of rows, and the
gather is the row layout itself.
"""
from __future__ import annotations


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
