"""GPU parity of split-KV across devices, its device side on one GPU: the
token ranges of R ranks are attended one after another with
mla_decode_attn_range, each merged into its float32 range result with
mla_combine_splits_f32, and the R results merged with mla_merge_ranges,
against the oracle's attention over the whole context.  (The all-gather
between ranks is covered by the gloo test of the host side; this run has one
GPU.)  Both cache layouts a rank may hold: the whole contiguous cache, and a
paged pool that holds only the rank's own blocks (the others -1 in its block
table)."""

import numpy as np
import pytest
import torch

import head_latent_attention_09_b200 as M
from head_latent_attention_09_b200.splitkv import token_ranges
from oracle import mla_oracle as O
from tests.gpu_harness import compare, config_of, strict_on, to_dev, to_host, torch_dtype
from workloads import WORKLOADS, bf16_round, random_cache

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from head_latent_attention_09_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _queries(wl, B, seed):
    q = np.random.default_rng(seed).standard_normal((B, wl.n_h, wl.D)).astype(np.float32) * 0.5
    return bf16_round(q) if wl.dtype == "bf16" else q


def _oracle(wl, q, rows, ctx):
    scale = O.softmax_scale(wl.d_h, wl.d_r)
    out_c, out_l = {}, {}
    for b in range(len(ctx)):
        out_c[b], out_l[b] = O.latent_attention(q[b], rows[b, :ctx[b]], d_c=wl.d_c, scale=scale)
    return out_c, out_l


def _merge_on_gpu(handle, wl, parts_c, parts_l, B):
    R = len(parts_c)
    pc = torch.stack(parts_c).contiguous()
    pl = torch.stack(parts_l).contiguous()
    out = torch.empty((B, wl.n_h, wl.d_c), dtype=torch_dtype(wl), device="cuda")
    lse = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
    M.mla_merge_ranges(handle, pc, pl, R, B, out, lse)
    return to_host(out), to_host(lse)


@pytest.mark.parametrize("name", ["v2_b64_ctx8k", "v2lite_b32_ctx4k", "tiny_fp32"])
@pytest.mark.parametrize("world", [2, 3])
def test_ranges_of_a_contiguous_cache(name, world):
    wl = WORKLOADS[name]
    ctx = np.array([1000, 64, 1, 0, 2049])
    B, T = len(ctx), int(ctx.max())
    rows = random_cache(wl.with_(B=B), T, 1.0)
    q = _queries(wl, B, 5)
    handle = M.mla_create(config_of(wl))
    try:
        strict_on(handle, wl)
        cache, q_d = to_dev(rows, wl), to_dev(q, wl)
        begin, end = token_ranges(ctx, world)
        P = M.mla_default_num_parts(handle)
        ws_bytes = M.mla_decode_workspace_size(handle, B, P)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        parts_c, parts_l = [], []
        for r in range(world):
            b_d = torch.from_numpy(begin[r].astype(np.int32)).cuda()
            e_d = torch.from_numpy(end[r].astype(np.int32)).cuda()
            pc = torch.empty((B, wl.n_h, wl.d_c), dtype=torch.float32, device="cuda")
            pl = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
            M.mla_decode_attn_range(handle, q_d, cache, T, None, 0, b_d, e_d, B, P, ws, ws_bytes)
            M.mla_combine_splits_f32(handle, ws, ws_bytes, B, P, pc, pl)
            parts_c.append(pc)
            parts_l.append(pl)
        got_c, got_l = _merge_on_gpu(handle, wl, parts_c, parts_l, B)
        assert M.mla_get_device_status(handle) == M.MLA_OK
    finally:
        M.mla_destroy(handle)
    want_c, want_l = _oracle(wl, q, rows, ctx)
    seqs = [b for b in range(B) if ctx[b] > 0]
    compare(got_c, want_c, wl, f"ctx_lat over {world} ranges", seqs)
    compare(got_l, want_l, wl, f"lse over {world} ranges", seqs)
    assert np.all(got_c[3] == 0) and np.all(np.isneginf(got_l[3]))


@pytest.mark.parametrize("world", [2, 4])
def test_each_rank_holds_only_its_pages(world):
    wl = WORKLOADS["v2lite_paged_ragged_b128"]
    ps = wl.page_size
    ctx = np.array([3000, 700, 65, 1])
    B, T = len(ctx), int(ctx.max())
    rows = random_cache(wl.with_(B=B), T, 1.0)
    q = _queries(wl, B, 6)
    begin, end = token_ranges(ctx, world)
    max_blk = (T + ps - 1) // ps
    handle = M.mla_create(config_of(wl))
    try:
        strict_on(handle, wl)
        q_d = to_dev(q, wl)
        e_all = torch.from_numpy(ctx.astype(np.int32)).cuda()
        P = M.mla_default_num_parts(handle)
        ws_bytes = M.mla_decode_workspace_size(handle, B, P)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        rng = np.random.default_rng(11)
        parts_c, parts_l = [], []
        for r in range(world):
            # this rank's pool: only the blocks of its ranges, in a random order
            blocks = [(b, j) for b in range(B) for j in range(begin[r, b] // ps, (end[r, b] + ps - 1) // ps)]
            order = rng.permutation(len(blocks)) if blocks else np.zeros(0, np.int64)
            table = np.full((B, max_blk), -1, dtype=np.int32)
            pool = np.zeros((max(len(blocks), 1), ps, wl.D), dtype=np.float32)
            for slot, k in enumerate(order):
                b, j = blocks[k]
                table[b, j] = slot
                seg = rows[b, j * ps:(j + 1) * ps]
                pool[slot, :len(seg)] = seg
            pc = torch.empty((B, wl.n_h, wl.d_c), dtype=torch.float32, device="cuda")
            pl = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
            pool_d, table_d = to_dev(pool, wl), torch.from_numpy(table).cuda()
            b_d = torch.from_numpy(begin[r].astype(np.int32)).cuda()
            M.mla_decode_attn_range(handle, q_d, pool_d, pool.shape[0], table_d, max_blk, b_d,
                                    torch.from_numpy(end[r].astype(np.int32)).cuda(), B, P, ws, ws_bytes)
            M.mla_combine_splits_f32(handle, ws, ws_bytes, B, P, pc, pl)
            parts_c.append(pc)
            parts_l.append(pl)
            assert M.mla_get_device_status(handle) == M.MLA_OK
        del e_all
        got_c, got_l = _merge_on_gpu(handle, wl, parts_c, parts_l, B)
    finally:
        M.mla_destroy(handle)
    want_c, want_l = _oracle(wl, q, rows, ctx)
    compare(got_c, want_c, wl, "ctx_lat (paged, own pages)", list(range(B)))
    compare(got_l, want_l, wl, "lse (paged, own pages)", list(range(B)))


def test_range_start_off_the_tile_grid_is_flagged():
    wl = WORKLOADS["v2lite_b32_ctx4k"]
    B, T = 2, 256
    rows = random_cache(wl.with_(B=B), T, 1.0)
    q = _queries(wl, B, 7)
    handle = M.mla_create(config_of(wl))
    try:
        cache, q_d = to_dev(rows, wl), to_dev(q, wl)
        P = 4
        ws_bytes = M.mla_decode_workspace_size(handle, B, P)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        b_d = torch.tensor([100, 0], dtype=torch.int32, device="cuda")     # 100: not a multiple of 64
        e_d = torch.tensor([T, T], dtype=torch.int32, device="cuda")
        pc = torch.empty((B, wl.n_h, wl.d_c), dtype=torch.float32, device="cuda")
        pl = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
        M.mla_decode_attn_range(handle, q_d, cache, T, None, 0, b_d, e_d, B, P, ws, ws_bytes)
        M.mla_combine_splits_f32(handle, ws, ws_bytes, B, P, pc, pl)
        assert M.mla_get_device_status(handle) == M.MLA_ERR_DEVICE_BOUNDS
        got_c, got_l = to_host(pc), to_host(pl)
    finally:
        M.mla_destroy(handle)
    scale = O.softmax_scale(wl.d_h, wl.d_r)
    # the start is rounded down to token 64
    want = {0: O.latent_attention(q[0], rows[0, 64:T], d_c=wl.d_c, scale=scale),
            1: O.latent_attention(q[1], rows[1, :T], d_c=wl.d_c, scale=scale)}
    compare(got_c, {b: w[0] for b, w in want.items()}, wl, "ctx_lat", [0, 1])
    compare(got_l, {b: w[1] for b, w in want.items()}, wl, "lse", [0, 1])
