"""Split-KV decode attention across devices, for contexts too long to keep on
one GPU or to scan quickly from one: one process per GPU, each holding one
token range of every sequence's latent cache.

Per decode step every rank
  1. attends its own range with mla_decode_attn_range and merges its split
     partials into one float32 result per (sequence, head) with
     mla_combine_splits_f32;
  2. exchanges those results in one all-gather (NCCL over NVLink on GPUs):
     n_h * (d_c + 1) float32 per sequence per rank;
  3. merges the ranges with mla_merge_ranges (log-sum-exp algebra, in rank
     order, so every rank obtains the same ctx_lat bit for bit).

The arithmetic runs in the library's kernels; this module only cuts the token
ranges and moves the per-range results between ranks.  The "DeepSeek-V3"
reading note's inference deployment runs decode attention data-parallel with
sequence parallelism; the exchange is the one extra step this path has over
the single-GPU step.
"""

from __future__ import annotations

import numpy as np

from . import (mla_combine_splits_f32, mla_decode_attn_range, mla_merge_ranges)

TILE = 64   # tokens per tile of the split plan; a range starts on a tile


def token_ranges(ctx_len, world: int, tile: int = TILE):
    """Token range of each rank for each sequence: (begin, end), int64 arrays
    [world, B].  Sequence b's ceil(ctx_b / tile) tiles are cut into `world`
    consecutive runs whose sizes differ by at most one tile; rank r holds
    tokens begin[r, b] .. end[r, b] - 1 (an empty range when begin == end).
    Every begin is a multiple of the tile, as mla_decode_attn_range requires."""
    if world < 1:
        raise ValueError("world must be >= 1")
    ctx = np.asarray(ctx_len, dtype=np.int64)
    if np.any(ctx < 0):
        raise ValueError("context lengths must be >= 0")
    tiles = (ctx + tile - 1) // tile
    r = np.arange(world + 1, dtype=np.int64)[:, None]
    cut = (tiles[None, :] * r) // world * tile              # [world + 1, B], multiples of the tile
    end = np.minimum(cut[1:], ctx[None, :])
    begin = np.minimum(cut[:-1], end)
    return begin, end


def gather_ranges(ctx_part, lse_part, group=None):
    """All-gather of every rank's float32 range result: ctx_part [B, n_h, d_c]
    and lse_part [B, n_h] -> ([world, B, n_h, d_c], [world, B, n_h]) in rank
    order.  One collective per tensor over the process group."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    ctx_all = [torch.empty_like(ctx_part) for _ in range(world)]
    lse_all = [torch.empty_like(lse_part) for _ in range(world)]
    dist.all_gather(ctx_all, ctx_part.contiguous(), group=group)
    dist.all_gather(lse_all, lse_part.contiguous(), group=group)
    return torch.stack(ctx_all), torch.stack(lse_all)


def decode_attn_split_kv(handle, q_abs, cache, cache_len, block_table, max_blocks_per_seq, ctx_begin,
                         ctx_len, B, num_parts, workspace, ws_bytes, ctx_part, lse_part, ctx_lat, lse=None,
                         group=None, stream=None):
    """One rank's share of split-KV attention, then the exchange and the merge.

    ctx_begin / ctx_len (device int32 [B]) give this rank's token range;
    ctx_part [B, n_h, d_c] and lse_part [B, n_h] are float32 device buffers for
    this rank's range result; ctx_lat [B, n_h, d_c] (the configuration's
    dtype) and lse [B, n_h] float32 (or None) receive the merged result, the
    same on every rank.  `stream` must be torch's current stream (or None):
    the all-gather is enqueued there, between the library's calls."""
    import torch.distributed as dist
    mla_decode_attn_range(handle, q_abs, cache, cache_len, block_table, max_blocks_per_seq, ctx_begin, ctx_len,
                          B, num_parts, workspace, ws_bytes, stream)
    mla_combine_splits_f32(handle, workspace, ws_bytes, B, num_parts, ctx_part, lse_part, stream)
    parts, lses = gather_ranges(ctx_part, lse_part, group)
    mla_merge_ranges(handle, parts, lses, dist.get_world_size(group), B, ctx_lat, lse, stream)
