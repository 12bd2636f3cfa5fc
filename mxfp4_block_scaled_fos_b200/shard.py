"""Data-parallel sharding of the quantizer, one process per GPU.

Blocks are independent of each other.  The only value that crosses a shard
boundary is the per-tensor amax behind S_t (the FP32 per-tensor scale of
NVFP4, "Como funciona FP4" in the Ultralytics FP4 glossary).  There are two
ways to split the work:

* **By batch entry** (the experts of an MoE layer): every entry has its own
  S_t, so each rank quantizes its own entries and no collective runs.
* **By rows of one tensor**: each rank reduces the max of its rows, one
  all-reduce(MAX) of ``batch`` floats gives the global amax, and each rank
  quantizes its rows with it.  Shards start on multiples of 16 rows, so a
  16x16 tile or a colwise 16-block never straddles two ranks.  Stochastic
  rounding draws are keyed on the global element index, which is passed as
  ``elem_offset``, so the result is bit-identical to one unsharded call.

``ops`` is the pair of per-shard calls (amax, quantize).  It defaults to the
CUDA library through :mod:`fos`.  Any object with the same two methods
works, which lets the host logic here run on CPU process groups.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import fos as F

ROW_ALIGN = 16


def split_range(n: int, world: int, rank: int, align: int = 1) -> Tuple[int, int]:
    """[lo, hi) of rank's share of n items, cut on multiples of align.

    The n // align whole units are split as evenly as possible (the first
    ranks take one more); a ragged tail of n % align items goes to the last
    rank.  Ranks with nothing to do get an empty range.
    """
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d outside world of %d" % (rank, world))
    units = n // align
    base, extra = divmod(units, world)
    lo = (rank * base + min(rank, extra)) * align
    hi = lo + (base + (1 if rank < extra else 0)) * align
    if rank == world - 1:
        hi = n
    return lo, hi


def row_range(rows: int, world: int, rank: int) -> Tuple[int, int]:
    """Rows [lo, hi) of a row shard; lo is a multiple of 16."""
    return split_range(rows, world, rank, ROW_ALIGN)


def batch_range(batch: int, world: int, rank: int) -> Tuple[int, int]:
    """Batch entries [lo, hi) of an entry shard."""
    return split_range(batch, world, rank, 1)


class CudaOps:
    """The per-shard calls on the CUDA library."""

    @staticmethod
    def amax(x: torch.Tensor, rht: bool = False, seed: int = 0) -> torch.Tensor:
        return F.amax(x, rht=rht, seed=seed)

    @staticmethod
    def quantize(x: torch.Tensor, amax: Optional[torch.Tensor], elem_offset: int, **kw):
        return F.quantize(x, amax=amax, elem_offset=elem_offset, **kw)


def _world(group) -> int:
    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


def global_amax(local: torch.Tensor, group=None) -> torch.Tensor:
    """Max over ranks of each batch entry's amax (in place, returned)."""
    if _world(group) > 1:
        dist.all_reduce(local, op=dist.ReduceOp.MAX, group=group)
    return local


def quantize_row_shard(x_local: torch.Tensor, row0: int, cols: int, group=None, ops=None,
                       rht: bool = False, seed: int = 0, **kw):
    """Quantize rows [row0, row0 + x_local.shape[-2]) of a [rows, cols] tensor.

    Every rank of ``group`` calls this with its own rows (from
    :func:`row_range`).  The ranks first agree on the global amax, with one
    collective, then quantize their rows locally.  Returns what
    ``ops.quantize`` returns for the local rows.
    """
    ops = ops or CudaOps
    if x_local.dim() == 3 and x_local.shape[0] != 1:
        raise ValueError("row sharding takes one tensor; shard a batch by entry instead")
    if row0 % ROW_ALIGN:
        raise ValueError("row shards start on a multiple of 16 rows")
    a = ops.amax(x_local, rht=rht, seed=seed)
    a = global_amax(a, group)
    return ops.quantize(x_local, amax=a, elem_offset=row0 * cols, rht=rht, seed=seed, **kw)


def quantize_entry_shard(x_local: torch.Tensor, entry0: int, rows: int, cols: int, ops=None,
                         **kw):
    """Quantize batch entries [entry0, entry0 + x_local.shape[0]) of a
    [batch, rows, cols] tensor.  Each entry keeps its own S_t, so no
    collective runs; SR draws still follow the global element index."""
    ops = ops or CudaOps
    return ops.quantize(x_local, amax=kw.pop("amax", None), elem_offset=entry0 * rows * cols, **kw)
