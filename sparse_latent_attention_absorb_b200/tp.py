"""Tensor-parallel decode across ranks, one process per GPU.

The MLA constructor excerpt on the atlas page "Queries" (model.py 523-539)
builds wkv_b as a ColumnParallelLinear, so each of the world_size ranks holds
n_local_heads = 128 / world_size heads and the decode views its rows of wkv_b
as [n_local_heads, 256, 512]; wo is a RowParallelLinear (16384 -> dim), whose
per-rank partial outputs are summed across the ranks after the projection.
The latent cache, the rotary key cache and the index rows are shared by all
heads, so every rank holds them whole.

One decode step of a rank:
    out_r   = mla_sparse_decode_heads(q_nope[:, heads_r], q_pe[:, heads_r], caches, indices,
                                      wkv_b rows of heads_r)          [B, n_local_heads, 128]
    delta_r = mla_output_projection_shard(out_r flattened, wo[:, columns of heads_r])   [B, dim]
    delta   = all_reduce(delta_r, SUM)                                 (torch.distributed, NCCL)

The partials are bf16 and summed by the all-reduce in bf16, as the row-parallel
layer's output is.  Everything here is slicing and marshalling; the arithmetic
runs in the library's kernels and the collective.  ``decode`` and ``project``
may be replaced by other callables with the same signatures (the multi-rank
CPU tests do this).
"""
from __future__ import annotations

import torch

from . import binding

H = binding.H
D_V = binding.D_V
ROWS_PER_HEAD = binding.D_NOPE + binding.D_V  # rows of one head in wkv_b


def head_range(world_size: int, rank: int, n_heads: int = H) -> tuple[int, int]:
    """Heads [h0, h1) of `rank`: n_heads / world_size consecutive heads (the
    column-parallel split of wkv_b's output rows, head by head)."""
    if world_size < 1 or n_heads % world_size:
        raise ValueError(f"{n_heads} heads do not split evenly over {world_size} ranks")
    if not 0 <= rank < world_size:
        raise ValueError(f"rank {rank} outside [0, {world_size})")
    n = n_heads // world_size
    return rank * n, (rank + 1) * n


def shard(world_size: int, rank: int, q_nope, q_pe, wkv_b, wo=None) -> dict:
    """The rank's slices: its heads' queries (contiguous copies), its rows of
    wkv_b ([n_local*256, 512], a contiguous view) and, if given, its columns
    of wo ([dim, n_local*128], a strided view of the full matrix)."""
    h0, h1 = head_range(world_size, rank, q_nope.shape[1])
    s = {
        "heads": (h0, h1),
        "q_nope": q_nope[:, h0:h1].contiguous(),
        "q_pe": q_pe[:, h0:h1].contiguous(),
        "wkv_b": wkv_b.reshape(-1, ROWS_PER_HEAD, wkv_b.shape[-1])[h0:h1].reshape(-1, wkv_b.shape[-1]),
    }
    if wo is not None:
        s["wo"] = wo[:, h0 * D_V:h1 * D_V]
    return s


def decode_project(sh: dict, kv_cache, pe_cache, end_pos, topk_idx, scale: float, group=None, decode=None,
                   project=None, all_reduce: bool = True):
    """One tensor-parallel decode step followed by the row-parallel output
    projection on this rank; returns (delta, out_r).  With all_reduce the
    partial projection is summed over the ranks of `group` in place, so
    every rank returns the projection of all heads."""
    decode = decode or binding.mla_sparse_decode_heads
    project = project or binding.mla_output_projection_shard
    out_r = decode(sh["q_nope"], sh["q_pe"], kv_cache, pe_cache, end_pos, topk_idx, sh["wkv_b"], scale)
    B = out_r.shape[0]
    delta = project(out_r.reshape(B, -1), sh["wo"])
    if all_reduce and torch.distributed.is_initialized():
        torch.distributed.all_reduce(delta, op=torch.distributed.ReduceOp.SUM, group=group)
    return delta, out_r
