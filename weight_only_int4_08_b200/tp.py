"""Tensor-parallel (TP) sharding of one W4A16 linear layer over the ranks of a process group.

The tensor-parallel decode of the kerneldigest.dev page on LLM inference with TP
(section "Arquitectura del Sistema") splits every linear layer over the GPUs of a node
and ends a parallel layer with an all-reduce on the decode critical path. A weight-only
int4 layer splits two ways:

* Column-parallel (along N). Rank r owns output columns [c0, c1): the packed words
  b_packed[:, c0/8:c1/8], scales[:, c0:c1] and qzeros[:, c0/8:c1/8]. Each rank computes
  its columns with the full activations and no exchange; an all-gather along N rebuilds
  the full output where the next step needs it (gather_columns). Columns are split in
  whole packed words (8 columns); 128-column units keep every shard on the tensor-core
  GEMM's tile grid.
* Row-parallel (along K). Rank r owns rows [k0, k1) with k0, k1 multiples of the group
  size G, so every quantisation group lies on one rank: b_packed[k0:k1], scales and
  qzeros rows [k0/G, k1/G), and activation columns a[:, k0:k1] (the layout a
  column-parallel layer before it leaves on each rank). Each rank computes the fp32 sums
  of its slice of K (w4a16_gemm with out_f32=True); the output is the sum over ranks,
  rounded once to fp16. collect_partials brings the partials together, by an all-gather
  (every rank then adds them in rank order with w4a16_reduce_partials: bit-identical
  outputs on every rank) or by an all-reduce (half the traffic; the collective's own
  summation order), and round_partials does the sum and the rounding on the GPU.

Host logic only: the shard bounds, the tensor slicing and the torch.distributed calls.
All arithmetic runs in the library's kernels; the collectives run on whatever backend the
process group has (NCCL over NVLink on a GPU node).
"""
from __future__ import annotations

from typing import NamedTuple

import torch
import torch.distributed as dist


class Shard(NamedTuple):
    """One rank's part of a layer: kernel-layout tensors and the [lo, hi) range it covers
    (output columns for a column shard, rows of K for a row shard)."""
    b_packed: torch.Tensor
    scales: torch.Tensor
    qzeros: torch.Tensor | None
    lo: int
    hi: int


def split_bounds(extent: int, world: int, rank: int, unit: int) -> tuple[int, int]:
    """[lo, hi) of rank's share of `extent`, in whole `unit`s, as even as possible: rank r
    takes units [floor(U r / P), floor(U (r+1) / P)) of the U = extent / unit units."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if unit < 1 or extent % unit:
        raise ValueError(f"extent {extent} is not a multiple of the unit {unit}")
    units = extent // unit
    if units < world:
        raise ValueError(f"{units} units of {unit} cannot be shared by {world} ranks")
    return units * rank // world * unit, units * (rank + 1) // world * unit


def column_shard(b_packed: torch.Tensor, scales: torch.Tensor, qzeros: torch.Tensor | None, rank: int, world: int,
                 unit: int = 8) -> Shard:
    """Rank's output columns of a kernel-layout layer (b_packed [K, N/8], scales [K/G, N],
    qzeros [K/G, N/8] or None), as contiguous tensors. `unit` (a multiple of 8) is the
    column granularity of the split."""
    if unit % 8:
        raise ValueError("the column unit must be a multiple of 8 (one packed word)")
    N = scales.shape[1]
    if b_packed.shape[1] * 8 != N:
        raise ValueError("b_packed and scales disagree on N")
    c0, c1 = split_bounds(N, world, rank, unit)
    w0, w1 = c0 // 8, c1 // 8
    z = None if qzeros is None else qzeros[:, w0:w1].contiguous()
    return Shard(b_packed[:, w0:w1].contiguous(), scales[:, c0:c1].contiguous(), z, c0, c1)


def row_shard(b_packed: torch.Tensor, scales: torch.Tensor, qzeros: torch.Tensor | None, group_size: int, rank: int,
              world: int, unit: int | None = None) -> Shard:
    """Rank's rows of K of a kernel-layout layer: whole quantisation groups (`unit`, a
    multiple of group_size, defaults to group_size)."""
    G = group_size
    unit = G if unit is None else unit
    if unit % G:
        raise ValueError("the row unit must be a multiple of the group size")
    K = b_packed.shape[0]
    if scales.shape[0] * G != K:
        raise ValueError("b_packed and scales disagree on K / group_size")
    k0, k1 = split_bounds(K, world, rank, unit)
    z = None if qzeros is None else qzeros[k0 // G:k1 // G].contiguous()
    return Shard(b_packed[k0:k1].contiguous(), scales[k0 // G:k1 // G].contiguous(), z, k0, k1)


def row_shard_activations(a: torch.Tensor, shard: Shard) -> torch.Tensor:
    """The activation columns a row shard multiplies, as a contiguous [M, hi - lo] array."""
    return a[:, shard.lo:shard.hi].contiguous()


def _world(group):
    return dist.get_world_size(group) if dist.is_initialized() else 1


def gather_columns(out_shard: torch.Tensor, N: int, unit: int = 8, group=None) -> torch.Tensor:
    """All-gather column shards [M, c1 - c0] (split by split_bounds(N, world, r, unit)) into
    the full [M, N] output. Uneven shards are padded to the widest for the collective."""
    world = _world(group)
    if world == 1:
        return out_shard
    bounds = [split_bounds(N, world, r, unit) for r in range(world)]
    width = max(hi - lo for lo, hi in bounds)
    M = out_shard.shape[0]
    rank = dist.get_rank(group)
    if out_shard.shape[1] != bounds[rank][1] - bounds[rank][0]:
        raise ValueError("out_shard's width is not this rank's share of N")
    send = out_shard
    if out_shard.shape[1] != width:
        send = out_shard.new_zeros((M, width))
        send[:, :out_shard.shape[1]] = out_shard
    recv = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(recv, send.contiguous(), group=group)
    return torch.cat([recv[r][:, :hi - lo] for r, (lo, hi) in enumerate(bounds)], dim=1)


def collect_partials(partial: torch.Tensor, mode: str = "gather", group=None) -> list[torch.Tensor]:
    """Bring the ranks' fp32 partials [M, N] together.

    mode="gather": all-gather; returns the P partials in rank order (each rank then sums
    them in that order, so every rank holds the same bits). mode="sum": all-reduce with
    SUM in place; returns [partial], already summed in the collective's order."""
    world = _world(group)
    if world == 1:
        return [partial]
    if mode == "sum":
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
        return [partial]
    if mode != "gather":
        raise ValueError(f"unknown mode {mode!r}")
    stacked = partial.new_empty((world,) + tuple(partial.shape))
    parts = list(stacked.unbind(0))
    dist.all_gather(parts, partial.contiguous(), group=group)
    return parts


def round_partials(parts: list[torch.Tensor], out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """fp16(parts[0] + parts[1] + ...) on the GPU (w4a16_reduce_partials)."""
    from . import w4a16_reduce_partials
    return w4a16_reduce_partials(parts, out=out, stream=stream)


def column_parallel_linear(a: torch.Tensor, shard: Shard, group_size: int, zp_bias: int = 8, N: int | None = None,
                           unit: int = 8, gather: bool = False, group=None, **gemm_kw) -> torch.Tensor:
    """This rank's output columns [M, hi - lo] (or, with gather, the full [M, N])."""
    from . import w4a16_gemm
    out = w4a16_gemm(a, shard.b_packed, shard.scales, shard.qzeros, group_size, zp_bias, **gemm_kw)
    if not gather:
        return out
    if N is None:
        raise ValueError("gather needs the layer's N")
    return gather_columns(out, N, unit, group)


def row_parallel_linear(a_shard: torch.Tensor, shard: Shard, group_size: int, zp_bias: int = 8, mode: str = "gather",
                        group=None, **gemm_kw) -> torch.Tensor:
    """The layer's fp16 output [M, N] from this rank's activation columns and row shard:
    fp32 partial of the shard, collected over the group, summed and rounded once."""
    from . import w4a16_gemm
    partial = w4a16_gemm(a_shard, shard.b_packed, shard.scales, shard.qzeros, group_size, zp_bias, out_f32=True,
                         **gemm_kw)
    return round_partials(collect_partials(partial, mode, group))
