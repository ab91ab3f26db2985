"""Split-KV across devices, host side on CPU: the token-range partition and
the all-gather of per-range results, as two gloo ranks on 127.0.0.1.  Each
rank computes its range's partial with the oracle (the attention restricted to
its tokens), the ranks exchange them through the module's gather, and the
oracle's log-sum-exp merge of the gathered ranges must equal the oracle's
attention over the whole context."""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp
from hypothesis import given, settings
from hypothesis import strategies as st

from head_latent_attention_09_b200.splitkv import TILE, token_ranges


@pytest.mark.parametrize("world", [1, 2, 3, 5, 8])
def test_token_ranges_partition_each_sequence(world):
    ctx = np.array([0, 1, 63, 64, 65, 130, 1000, 131072, 4097])
    begin, end = token_ranges(ctx, world)
    assert begin.shape == end.shape == (world, len(ctx))
    assert np.all(begin % TILE == 0) and np.all(begin <= end)
    assert np.all(begin[0] == 0) and np.array_equal(end[-1], ctx)
    for b, c in enumerate(ctx):
        toks = np.concatenate([np.arange(begin[r, b], end[r, b]) for r in range(world)])
        assert np.array_equal(toks, np.arange(c)), (world, c)
        tiles = np.ceil((end[:, b] - begin[:, b]) / TILE)
        assert tiles.max() - tiles.min() <= 1


@settings(max_examples=60, deadline=None, derandomize=True)
@given(ctx=st.lists(st.integers(0, 300_000), min_size=1, max_size=12), world=st.integers(1, 16),
       tile=st.sampled_from([64, 128, 256]))
def test_token_ranges_partition_any_lengths(ctx, world, tile):
    """The same properties for drawn lengths, world sizes and tiles: the
    ranges cover each sequence exactly, in rank order, every begin on a tile,
    and the tile counts of the ranks differ by at most one."""
    ctx = np.array(ctx)
    begin, end = token_ranges(ctx, world, tile)
    assert np.all(begin % tile == 0) and np.all(begin <= end)
    assert np.all(begin[0] == 0) and np.array_equal(end[-1], ctx)
    assert np.array_equal(begin[1:], end[:-1])
    tiles = (end - begin + tile - 1) // tile
    assert np.all(tiles.max(axis=0) - tiles.min(axis=0) <= 1)


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    rng = np.random.default_rng(2024)
    ctx = np.array([300, 64, 1, 777])
    n_h, d_c, d_r = 4, 32, 8
    rows = [rng.standard_normal((c, d_c + d_r)) for c in ctx]
    q = rng.standard_normal((len(ctx), n_h, d_c + d_r)) * 0.5
    return ctx, rows, q, d_c


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    from oracle import mla_oracle as O
    from head_latent_attention_09_b200.splitkv import gather_ranges
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ctx, rows, q, d_c = _inputs()
        begin, end = token_ranges(ctx, world)
        scale = 0.3
        part_ctx, part_lse = [], []
        for b in range(len(ctx)):
            c, l = O.latent_attention(q[b], rows[b][begin[rank, b]:end[rank, b]], d_c=d_c, scale=scale)
            part_ctx.append(c)
            part_lse.append(l)
        ctx_all, lse_all = gather_ranges(torch.from_numpy(np.stack(part_ctx)), torch.from_numpy(np.stack(part_lse)))
        merged = []
        for b in range(len(ctx)):
            parts = [(ctx_all[r, b].numpy(), lse_all[r, b].numpy()) for r in range(world)]
            merged.append(O.combine_partials(parts))
        dist.barrier()
        out.put((rank, [m[0] for m in merged], [m[1] for m in merged]))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_gather_and_merge_match_the_whole_context(world):
    from oracle import mla_oracle as O
    ctxq = mp.get_context("spawn")
    q_out = ctxq.Queue()
    port = _free_port()
    procs = [ctxq.Process(target=_worker, args=(r, world, port, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            rank, c, l = q_out.get(timeout=150)
            got[rank] = (c, l)
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    assert sorted(got) == list(range(world))
    ctx, rows, q, d_c = _inputs()
    for b in range(len(ctx)):
        want_c, want_l = O.latent_attention(q[b], rows[b], d_c=d_c, scale=0.3)
        for r in range(world):      # every rank holds the same merged result
            c, l = got[r][0][b], got[r][1][b]
            assert np.allclose(c, want_c, rtol=1e-12, atol=1e-12)
            assert np.allclose(l, want_l, rtol=1e-12, atol=1e-12)
