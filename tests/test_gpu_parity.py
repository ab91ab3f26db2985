"""GPU parity: the CUDA library, called through its C ABI, against the CPU
oracle on the same seeded inputs.

* Full decode steps of every workload at its full size, in the launch
  configuration the benchmark times (default number of work partitions),
  checked on sampled sequences the oracle computes one by one.
* The attention step alone on directly drawn caches, at sizes that span many
  tiles and ragged tails, with every split count from 1 to more shares than
  tiles.
* Edge cases: empty and one-token contexts, contexts that end inside a tile,
  NaN garbage beyond each context, paged caches, the output projection W^O.
"""

import numpy as np
import pytest
import torch

import head_latent_attention_09_b200 as M
from oracle import mla_oracle as O
from tests.gpu_harness import (compare, config_of, oracle_step, run_decode_step, strict_on, to_dev,
                               to_host, torch_dtype)
from workloads import WORKLOADS, ctx_lengths, random_cache

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from head_latent_attention_09_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _check_step(wl, got, seqs, with_wo=False, explicit_heads=None):
    want = oracle_step(wl, seqs, with_wo=with_wo, explicit_heads=explicit_heads)
    compare(got["cache_new_rows"], want["cache_new_rows"], wl, "cache row", seqs)
    compare(got["q_abs"], want["q_abs"], wl, "q_abs", seqs)
    compare(got["ctx_lat"], want["ctx_lat"], wl, "ctx_lat", seqs)
    compare(got["lse"], want["lse"], wl, "lse", seqs)
    compare(got["o"], want["o"], wl, "o", seqs)
    if with_wo:
        compare(got["u"], want["u"], wl, "u", seqs)
    if explicit_heads is not None:
        g = {b: got["o"][b][list(explicit_heads)] for b in seqs}
        compare(g, want["o_explicit"], wl, "o (explicit per-head keys)", seqs)


# ---------------------------------------------------------------------------
# full decode steps of the five workloads
# ---------------------------------------------------------------------------

def test_tiny_fp32_full_step():
    wl = WORKLOADS["tiny_fp32"]
    got = run_decode_step(wl, with_wo=True)
    _check_step(wl, got, [0, 1], with_wo=True, explicit_heads=range(wl.n_h))


@pytest.mark.parametrize("parts", [1, 2, 5])
def test_tiny_fp32_split_counts(parts):
    wl = WORKLOADS["tiny_fp32"]
    got = run_decode_step(wl, num_parts=parts)
    _check_step(wl, got, [0, 1])


def test_v2lite_b32_ctx4k_full():
    wl = WORKLOADS["v2lite_b32_ctx4k"]
    got = run_decode_step(wl)
    _check_step(wl, got, [0, 13, 31], explicit_heads=range(0, 16, 5))


def test_v2_b64_ctx8k_full():
    wl = WORKLOADS["v2_b64_ctx8k"]
    got = run_decode_step(wl)
    _check_step(wl, got, [0, 37, 63], explicit_heads=[0, 64, 127])


def test_ragged_paged_full():
    wl = WORKLOADS["v2lite_paged_ragged_b128"]
    ctx = ctx_lengths(wl)
    got = run_decode_step(wl)
    seqs = sorted({int(np.argmin(ctx)), int(np.argmax(ctx)), 5, 77})
    _check_step(wl, got, seqs, explicit_heads=[3, 11])


def test_128k_full():
    wl = WORKLOADS["v2lite_b4_ctx128k"]
    got = run_decode_step(wl)
    rng = np.random.default_rng(wl.seed)
    heads = sorted(rng.choice(wl.n_h, 8, replace=False).tolist())
    _check_step(wl, got, [2], explicit_heads=heads)     # 8 heads explicit, all 16 absorbed


# ---------------------------------------------------------------------------
# small shapes of the fast paths: ragged, empty, one-token contexts, W^O
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name,ctx", [
    ("v2_b64_ctx8k", (1, 63, 64, 65, 200, 0, 129)),
    ("v2lite_b32_ctx4k", (1, 2, 64, 100, 0, 1000, 4097)),
])
def test_small_ragged_steps(name, ctx):
    wl = WORKLOADS[name].with_(B=len(ctx), ctx=ctx)
    got = run_decode_step(wl, with_wo=True)
    seqs = [b for b in range(wl.B) if ctx[b] > 0]
    _check_step(wl, got, seqs, with_wo=True)
    for b in range(wl.B):
        if ctx[b] == 0:
            assert np.all(got["ctx_lat"][b] == 0) and np.all(np.isneginf(got["lse"][b]))


def test_paged_128_heads():
    """The 128-head pair kernel over a paged pool (64-token pages, each 128-token
    half of a tile staged as two page boxes), ragged contexts, W^O."""
    wl = WORKLOADS["v2_b64_ctx8k"].with_(B=5, ctx=(1, 64, 65, 300, 1000), page_size=64)
    got = run_decode_step(wl, with_wo=True)
    _check_step(wl, got, list(range(5)), with_wo=True, explicit_heads=[0, 127])


def test_paged_small():
    wl = WORKLOADS["v2lite_paged_ragged_b128"].with_(B=6, ctx=(1, 64, 65, 300, 1, 130))
    got = run_decode_step(wl)
    _check_step(wl, got, list(range(6)))


# ---------------------------------------------------------------------------
# the attention step alone on drawn caches
# ---------------------------------------------------------------------------

def _attention_only(wl, ctx, parts, q_scale=0.5, cache_std=1.0, plant=None):
    cfg = config_of(wl)
    handle = M.mla_create(cfg)
    try:
        strict_on(handle, wl)
        ctx = np.asarray(ctx)
        B, T = len(ctx), int(max(1, ctx.max()))
        w2 = wl.with_(B=B)
        rows = random_cache(w2, T, cache_std)                       # [B, T, D]
        rng = np.random.default_rng(1234)
        q = rng.standard_normal((B, wl.n_h, wl.D)).astype(np.float32) * q_scale
        if plant is not None:
            plant(rows, q)
        from workloads import bf16_round
        if wl.dtype == "bf16":
            q = bf16_round(q)
        for b in range(B):                                         # garbage past each context
            rows[b, ctx[b]:] = np.nan
        cache = to_dev(rows, wl)
        q_d = to_dev(q, wl)
        ctx_d = torch.from_numpy(ctx.astype(np.int32)).cuda()
        ws_bytes = M.mla_decode_workspace_size(handle, B, parts)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        out = torch.empty((B, wl.n_h, wl.d_c), dtype=torch_dtype(wl), device="cuda")
        lse = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
        M.mla_decode_attn(handle, q_d, cache, T, None, 0, ctx_d, B, parts, ws, ws_bytes)
        M.mla_combine_splits(handle, ws, ws_bytes, B, parts, out, lse)
        assert M.mla_get_device_status(handle) == M.MLA_OK
        got_ctx, got_lse = to_host(out), to_host(lse)
    finally:
        M.mla_destroy(handle)
    scale = O.softmax_scale(wl.d_h, wl.d_r)
    want_ctx, want_lse = {}, {}
    for b in range(B):
        want_ctx[b], want_lse[b] = O.latent_attention(q[b], rows[b, :ctx[b]], d_c=wl.d_c,
                                                      scale=scale)
    return got_ctx, got_lse, want_ctx, want_lse


@pytest.mark.parametrize("name", ["v2_b64_ctx8k", "v2lite_b32_ctx4k", "tiny_fp32"])
@pytest.mark.parametrize("parts", [1, 3, 16, 74, 148, 5000])
def test_attention_split_counts(name, parts):
    wl = WORKLOADS[name]
    ctx = [700, 1, 64, 0, 129, 2000, 63]
    gc, gl, wc, wlse = _attention_only(wl, ctx, parts)
    seqs = [b for b in range(len(ctx)) if ctx[b] > 0]
    compare(gc, wc, wl, f"ctx_lat parts={parts}", seqs)
    compare(gl, wlse, wl, f"lse parts={parts}", seqs)
    assert np.all(gc[3] == 0) and np.all(np.isneginf(gl[3]))


@pytest.mark.parametrize("name", ["v2_b64_ctx8k", "v2lite_b32_ctx4k"])
def test_attention_long_ragged_contexts(name):
    """Long contexts of unequal length at the default split count: shares cut
    in the kernel's own tile (256 or 128 tokens) cross sequence ends that are
    not on a tile boundary."""
    wl = WORKLOADS[name]
    ctx = [40000, 1, 70001, 257, 0, 12345]
    gc, gl, wc, wlse = _attention_only(wl, ctx, 0)
    seqs = [b for b in range(len(ctx)) if ctx[b] > 0]
    compare(gc, wc, wl, "ctx_lat long ragged", seqs)
    compare(gl, wlse, wl, "lse long ragged", seqs)


@pytest.mark.parametrize("name", ["v2_b64_ctx8k", "v2lite_b32_ctx4k"])
def test_attention_many_short_sequences(name):
    """300 short ragged sequences at the default split count: many pieces per
    share, sequences of one token and empty ones."""
    wl = WORKLOADS[name]
    rng = np.random.default_rng(77)
    ctx = rng.integers(0, 700, size=300)
    ctx[::37] = 0
    ctx[5::41] = 1
    gc, gl, wc, wlse = _attention_only(wl, ctx.tolist(), 0)
    seqs = [b for b in range(len(ctx)) if ctx[b] > 0][::7]
    compare(gc, wc, wl, "ctx_lat many short", seqs)
    compare(gl, wlse, wl, "lse many short", seqs)
    for b in np.nonzero(ctx == 0)[0]:
        assert np.all(gc[b] == 0) and np.all(np.isneginf(gl[b]))


@pytest.mark.parametrize("name", ["v2_b64_ctx8k", "v2lite_b32_ctx4k"])
def test_attention_more_sequences_than_plan_threads(name):
    """1500 short sequences, more than the split plan's 1024 threads: each
    thread scans two sequences (and the last threads none) in both prefix
    scans; default split count, so every share spans many sequences."""
    wl = WORKLOADS[name]
    rng = np.random.default_rng(1500)
    ctx = rng.integers(0, 48, size=1500)
    ctx[::97] = 0
    ctx[3::89] = 1
    gc, gl, wc, wlse = _attention_only(wl, ctx.tolist(), 0)
    seqs = [b for b in range(len(ctx)) if ctx[b] > 0]
    compare(gc, wc, wl, "ctx_lat 1500 sequences", seqs)
    compare(gl, wlse, wl, "lse 1500 sequences", seqs)
    for b in np.nonzero(ctx == 0)[0]:
        assert np.all(gc[b] == 0) and np.all(np.isneginf(gl[b]))


@pytest.mark.parametrize("name", ["v2_b64_ctx8k", "v2lite_b32_ctx4k"])
def test_attention_late_dominant_key(name):
    """A key far above the others late in the sequence forces the running
    maximum to jump (the rescale path)."""
    wl = WORKLOADS[name]

    d_c = wl.d_c

    def plant(rows, q):
        # the dominance sits in the rotary part (keys only), so the output stays O(1)
        rows[:, 1500, d_c] = 30.0
        q[:, :, :] *= 0.1
        q[:, :, d_c] = 4.0

    ctx = [1800, 1600]
    gc, gl, wc, wlse = _attention_only(wl, ctx, 7, plant=plant)
    compare(gc, wc, wl, "ctx_lat dominant", [0, 1])
    compare(gl, wlse, wl, "lse dominant", [0, 1])


# ---------------------------------------------------------------------------
# lengths the cache cannot hold, and strict tensor-core mode
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["v2_b64_ctx8k", "v2lite_b32_ctx4k", "tiny_fp32"])
def test_length_past_the_cache_is_flagged_and_clamped(name):
    """ctx_len = cache_len + 1 (contiguous cache): the call flags
    MLA_ERR_DEVICE_BOUNDS and attends the cache_len tokens that exist, in the
    split plan and in the attention kernel alike (each kernel kind)."""
    wl = WORKLOADS[name]
    T = 300
    ctx = np.array([T + 1, 5, T, 0])
    B = len(ctx)
    handle = M.mla_create(config_of(wl))
    try:
        strict_on(handle, wl)
        rows = random_cache(wl.with_(B=B), T, 1.0)
        rng = np.random.default_rng(77)
        q = rng.standard_normal((B, wl.n_h, wl.D)).astype(np.float32) * 0.5
        from workloads import bf16_round
        if wl.dtype == "bf16":
            q = bf16_round(q)
        cache, q_d = to_dev(rows, wl), to_dev(q, wl)
        ctx_d = torch.from_numpy(ctx.astype(np.int32)).cuda()
        for parts in (0, 3):
            P = parts or M.mla_default_num_parts(handle)
            ws_bytes = M.mla_decode_workspace_size(handle, B, P)
            ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
            out = torch.empty((B, wl.n_h, wl.d_c), dtype=torch_dtype(wl), device="cuda")
            lse = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
            M.mla_decode_attn(handle, q_d, cache, T, None, 0, ctx_d, B, P, ws, ws_bytes)
            M.mla_combine_splits(handle, ws, ws_bytes, B, P, out, lse)
            assert M.mla_get_device_status(handle) == M.MLA_ERR_DEVICE_BOUNDS
            assert M.mla_get_device_status(handle) == M.MLA_OK       # read and cleared
            got_c, got_l = to_host(out), to_host(lse)
            scale = O.softmax_scale(wl.d_h, wl.d_r)
            want_c, want_l = {}, {}
            for b in range(3):
                n = min(int(ctx[b]), T)
                want_c[b], want_l[b] = O.latent_attention(q[b], rows[b, :n], d_c=wl.d_c, scale=scale)
            compare(got_c, want_c, wl, f"ctx_lat clamped, parts={P}", [0, 1, 2])
            compare(got_l, want_l, wl, f"lse clamped, parts={P}", [0, 1, 2])
            assert np.all(got_c[3] == 0) and np.all(np.isneginf(got_l[3]))
    finally:
        M.mla_destroy(handle)


def test_paged_length_past_the_block_table_is_flagged_and_clamped():
    wl = WORKLOADS["v2lite_paged_ragged_b128"]
    ps = wl.page_size
    max_blk = 3
    ctx = np.array([max_blk * ps + 10, 70])
    B = len(ctx)
    handle = M.mla_create(config_of(wl))
    try:
        strict_on(handle, wl)
        n_pool = B * max_blk
        pool_rows = random_cache(wl.with_(B=1), n_pool * ps, 1.0)[0]
        perm = np.random.default_rng(5).permutation(n_pool).astype(np.int32)
        table = perm.reshape(B, max_blk)
        rng = np.random.default_rng(78)
        from workloads import bf16_round
        q = bf16_round(rng.standard_normal((B, wl.n_h, wl.D)).astype(np.float32) * 0.5)
        pool = to_dev(pool_rows.reshape(n_pool, ps, wl.D), wl)
        q_d = to_dev(q, wl)
        tbl = torch.from_numpy(table).cuda()
        ctx_d = torch.from_numpy(ctx.astype(np.int32)).cuda()
        P = M.mla_default_num_parts(handle)
        ws_bytes = M.mla_decode_workspace_size(handle, B, P)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        out = torch.empty((B, wl.n_h, wl.d_c), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
        M.mla_decode_attn(handle, q_d, pool, n_pool, tbl, max_blk, ctx_d, B, P, ws, ws_bytes)
        M.mla_combine_splits(handle, ws, ws_bytes, B, P, out, lse)
        assert M.mla_get_device_status(handle) == M.MLA_ERR_DEVICE_BOUNDS
        got_c, got_l = to_host(out), to_host(lse)
    finally:
        M.mla_destroy(handle)
    scale = O.softmax_scale(wl.d_h, wl.d_r)
    flat = pool_rows.reshape(n_pool, ps, wl.D)
    want_c, want_l = {}, {}
    for b in range(B):
        n = min(int(ctx[b]), max_blk * ps)
        seq = np.concatenate([flat[table[b, j]] for j in range(max_blk)])[:n]
        want_c[b], want_l[b] = O.latent_attention(q[b], seq, d_c=wl.d_c, scale=scale)
    compare(got_c, want_c, wl, "ctx_lat clamped (paged)", [0, 1])
    compare(got_l, want_l, wl, "lse clamped (paged)", [0, 1])


def test_strict_mode_refuses_instead_of_substituting():
    """With strict mode on, arguments the tensor-core kernels cannot take (a
    pointer that is not 16-byte aligned) make the call fail before any launch
    instead of running the CUDA-core kernel."""
    wl = WORKLOADS["v2_b64_ctx8k"]
    B = 2
    handle = M.mla_create(config_of(wl))
    try:
        M.mla_set_strict(handle, 1)
        bf = torch.bfloat16
        buf = torch.zeros(B * wl.n_h * wl.D + 64, dtype=bf, device="cuda")
        odd = buf.data_ptr() + 2                       # 2-byte aligned only
        cache = torch.zeros((B, 64, wl.D), dtype=bf, device="cuda")
        ctx_d = torch.full((B,), 64, dtype=torch.int32, device="cuda")
        ws_bytes = M.mla_decode_workspace_size(handle, B, 0)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        with pytest.raises(M.MlaError) as err:
            M.mla_decode_attn(handle, odd, cache, 64, None, 0, ctx_d, B, 0, ws, ws_bytes)
        assert err.value.status == M.MLA_ERR_UNSUPPORTED
        q_nope = torch.zeros((B, wl.n_h, wl.d_h), dtype=bf, device="cuda")
        q_rope = torch.zeros((B, wl.n_h, wl.d_r), dtype=bf, device="cuda")
        w_uk = torch.zeros((wl.n_h * wl.d_h, wl.d_c), dtype=bf, device="cuda")
        pos = torch.zeros(B, dtype=torch.int32, device="cuda")
        q_abs = torch.empty((B, wl.n_h, wl.D), dtype=bf, device="cuda")
        with pytest.raises(M.MlaError) as err:
            M.mla_absorb_q(handle, odd, q_rope, pos, w_uk, q_abs, B)
        assert err.value.status == M.MLA_ERR_UNSUPPORTED
        o = torch.empty((B, wl.n_h, wl.d_h), dtype=bf, device="cuda")
        with pytest.raises(M.MlaError) as err:
            M.mla_out_proj(handle, odd, w_uk, None, o, None, B)
        assert err.value.status == M.MLA_ERR_UNSUPPORTED
        torch.cuda.synchronize()
        assert M.mla_get_device_status(handle) == M.MLA_OK
    finally:
        M.mla_destroy(handle)


def test_plan_tile_follows_the_attention_kernel():
    # the split plan counts tiles of the attention kernel's own MMA tile
    for n_h, tile, tile_fp8 in ((128, 256, 64), (16, 128, 128), (32, 128, 128), (8, 64, 64)):
        wl = WORKLOADS["v2lite_b32_ctx4k"].with_(n_h=n_h)
        h = M.mla_create(config_of(wl))
        try:
            assert M.mla_plan_tile(h) == tile and M.mla_plan_tile(h, fp8=True) == tile_fp8
        finally:
            M.mla_destroy(h)
