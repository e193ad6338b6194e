"""A batch split by context across ranks (one process per GPU).

Rank r of W holds chunks [floor(n_b r / W), floor(n_b (r + 1) / W)) of every
sequence b (n_b = ceil(T_b / L) chunks of L tokens).  Shards are whole chunks,
so routing, regrouping, packing and decoding a shard give exactly what the
whole sequence gives on those chunks; routing freezing (chunk 0 of a sequence
kept at FP16) applies on the rank that holds chunk 0, which is rank 0.  Each
rank computes one record per (sequence, query head) with
mq_decode_attn_partial; the records of all ranks are all-gathered (NCCL over
NVLink on GPUs; any torch.distributed backend works) and merged with
mq_combine_partials.

This module only plans shards and moves records; every step of the method
runs in the CUDA library.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np


def shard_ranges(lens, chunk_len: int, rank: int, world: int) -> Tuple[np.ndarray, np.ndarray]:
    """Token range [lo, hi) of every sequence held by `rank` (int64 arrays)."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world {world}")
    lens = np.asarray(lens, np.int64)
    n = (lens + chunk_len - 1) // chunk_len
    c0 = (n * rank) // world
    c1 = (n * (rank + 1)) // world
    return np.minimum(c0 * chunk_len, lens), np.minimum(c1 * chunk_len, lens)


def shard_lengths(lens, chunk_len: int, rank: int, world: int) -> np.ndarray:
    """Tokens of every sequence held by `rank` (int32, for the C ABI)."""
    lo, hi = shard_ranges(lens, chunk_len, rank, world)
    return (hi - lo).astype(np.int32)


def routing_freeze(rank: int) -> bool:
    """Whether this rank's shards start at chunk 0 of their sequences."""
    return rank == 0


def shard_rows(x, lens, lo, hi):
    """Rows of a varlen tensor / array [T, ...] (sequences back to back) that
    fall in the ranges [lo_b, hi_b) of each sequence, concatenated."""
    lens = np.asarray(lens, np.int64)
    starts = np.concatenate([[0], np.cumsum(lens)])
    idx = np.concatenate([np.arange(starts[b] + lo[b], starts[b] + hi[b], dtype=np.int64)
                          for b in range(len(lens))] or [np.zeros(0, np.int64)])
    if hasattr(x, "index_select"):
        import torch
        return x.index_select(0, torch.as_tensor(idx, device=x.device))
    return x[idx]


def shard_chunk_map(chunk_expert, lens, chunk_len: int, rank: int, world: int) -> np.ndarray:
    """The entries of a whole-batch chunk map that belong to `rank`'s shards."""
    lens = np.asarray(lens, np.int64)
    n = (lens + chunk_len - 1) // chunk_len
    starts = np.concatenate([[0], np.cumsum(n)])
    c0 = (n * rank) // world
    c1 = (n * (rank + 1)) // world
    m = np.asarray(chunk_expert)
    parts = [m[starts[b] + c0[b]:starts[b] + c1[b]] for b in range(len(lens))]
    return np.concatenate(parts) if parts else np.zeros(0, m.dtype)


def gather_records(partial, group=None):
    """All-gather of this rank's records [B, Hq, d + 4] into [W, B, Hq, d + 4]
    (rank order).  Every rank must call it, in the same order."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return partial.unsqueeze(0)
    world = dist.get_world_size(group)
    if world == 1:
        return partial.unsqueeze(0)
    part = partial.contiguous()
    out = torch.empty((world,) + tuple(part.shape), dtype=part.dtype, device=part.device)
    if part.is_cuda:
        dist.all_gather_into_tensor(out, part, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), part, group=group)
    return out
