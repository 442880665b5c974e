"""Tensor-parallel SpMM over torch.distributed (the Flash-LLM review, section 5
item 5: the integration supports distributed inference by model parallelism).

Two shardings of one weight A (M x K) over R ranks:

* rows (column-parallel layers: QKV, MLP1): rank r owns a run of whole 64-row
  strips and computes those rows of C.  No exchange: C stays sharded by rows.
  ``TCSL.slice_rows`` gives the shard as a view of a full encoding.
* K (row-parallel layers: out-proj, MLP2): rank r owns a run of 64-wide K
  tiles, multiplies them with its K-slice of B in fp32, the ranks' partials are
  summed by an all-reduce, and the sum is rounded to fp16 once.
  ``TCSL.slice_cols`` gives the shard as a view.

``spmm_lscd_ksplit`` is the collective baseline for the K split: the library's
SpMM (fp32 output), one ``all_reduce`` of the fp32 partials through the
process group (NCCL over NVLink on GPUs), and the library's rounding kernel.
The shard boundaries below are the ones both shardings use.
"""
from __future__ import annotations

import ctypes

import torch
import torch.distributed as dist

from . import binding


def shard_range(extent: int, tile: int, rank: int, world: int) -> tuple:
    """[begin, end) of rank's share of `extent` rows or columns, cut on `tile`
    boundaries into near-equal runs of whole tiles (the last may be ragged)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    tiles = -(-extent // tile)
    t0, t1 = rank * tiles // world, (rank + 1) * tiles // world
    return min(extent, t0 * tile), min(extent, t1 * tile)


def round_f16(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """fp32 -> fp16, round to nearest even, in the library's kernel."""
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise TypeError("x must be a contiguous float32 CUDA tensor")
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float16, device=x.device)
    binding._check(binding.load_library().flashspmm_round_f16(
        ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(out.data_ptr()), x.numel(), binding._stream_handle(stream)),
        "round_f16")
    return out


def spmm_lscd_ksplit(shard: binding.TCSL, B_shard: torch.Tensor, group=None, stream=None) -> torch.Tensor:
    """C = sum over ranks of shard_r x B_shard_r, as fp16 ``[N, M]`` on every rank.

    shard    this rank's K range of A (a view from ``TCSL.slice_cols`` or its own encoding).
    B_shard  the matching contiguous ``[N, K_shard]`` fp16 slice of B.
    Every rank of `group` must call this with the same M and N."""
    N, M = B_shard.shape[0], shard.M
    partial = torch.empty((N, M), dtype=torch.float32, device=B_shard.device)
    binding.spmm_lscd(shard, B_shard, partial, stream=stream)
    dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return round_f16(partial, stream=stream)
