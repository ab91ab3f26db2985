"""The allocation-free attention entry point, for callers that cannot allocate
device memory where attention runs (allocator callbacks, runtimes that forbid
cudaMalloc after start-up, embeddings that only lend existing buffers).  Its
partials live in the library's fixed scratch array instead of a workspace.

Checked through the C ABI against the workspace-based entry points
(mla_decode_attn + mla_combine_splits) on two calls in a row with different
inputs, so that a call reading the previous call's leftovers would show.
This file is collected last so that a run stopping at its first failure has
already run every other test."""

import numpy as np
import pytest
import torch

import head_latent_attention_09_b200 as M
from tests.gpu_harness import compare, config_of, to_dev, to_host, torch_dtype
from workloads import WORKLOADS, bf16_round

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from head_latent_attention_09_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _inputs(wl, ctx, seed):
    rng = np.random.default_rng(seed)
    B, T = len(ctx), int(max(ctx))
    rows = rng.standard_normal((B, T, wl.D)).astype(np.float32)
    q = (rng.standard_normal((B, wl.n_h, wl.D)) * 0.5).astype(np.float32)
    if wl.dtype == "bf16":
        rows, q = bf16_round(rows), bf16_round(q)
    return (to_dev(rows, wl), to_dev(q, wl),
            torch.from_numpy(np.asarray(ctx, np.int32)).cuda(), T)


def _with_workspace(handle, wl, cache, q, ctx_d, T, B):
    P = M.mla_default_num_parts(handle)
    nbytes = M.mla_decode_workspace_size(handle, B, P)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.empty((B, wl.n_h, wl.d_c), dtype=torch_dtype(wl), device="cuda")
    lse = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
    M.mla_decode_attn(handle, q, cache, T, None, 0, ctx_d, B, P, ws, nbytes)
    M.mla_combine_splits(handle, ws, nbytes, B, P, out, lse)
    return to_host(out), to_host(lse)


def _without_allocation(handle, wl, cache, q, ctx_d, T, B):
    out = torch.empty((B, wl.n_h, wl.d_c), dtype=torch_dtype(wl), device="cuda")
    lse = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
    M.mla_decode_attn_combine_noalloc(handle, q, cache, T, None, 0, ctx_d, B, 0, out, lse)
    assert M.mla_get_device_status(handle) == M.MLA_OK
    return to_host(out), to_host(lse)


@pytest.mark.parametrize("name", ["v2_b64_ctx8k", "v2lite_b32_ctx4k", "tiny_fp32"])
def test_noalloc_matches_workspace_entry_points(name):
    wl = WORKLOADS[name]
    handle = M.mla_create(config_of(wl))
    try:
        for call, ctx in enumerate([[700, 1, 129, 0, 2048], [300, 64, 65]]):
            cache, q, ctx_d, T = _inputs(wl, ctx, seed=10 + call)
            B = len(ctx)
            want_o, want_l = _with_workspace(handle, wl, cache, q, ctx_d, T, B)
            got_o, got_l = _without_allocation(handle, wl, cache, q, ctx_d, T, B)
            seqs = [b for b in range(B) if ctx[b] > 0]
            compare(got_o, {b: want_o[b] for b in seqs}, wl, f"ctx_lat call {call}", seqs)
            compare(got_l, {b: want_l[b] for b in seqs}, wl, f"lse call {call}", seqs)
            for b in range(B):
                if ctx[b] == 0:
                    assert np.all(got_o[b] == 0) and np.all(np.isneginf(got_l[b]))
    finally:
        M.mla_destroy(handle)


def test_noalloc_first_call_on_a_fresh_handle_allocates_nothing():
    """The scratch array is made resident when the handle is created; the first
    call of the entry point on a fresh handle leaves the device's free memory
    unchanged (its kernels are loaded first by the workspace path)."""
    wl = WORKLOADS["v2_b64_ctx8k"]
    ctx = [700, 129]
    cache, q, ctx_d, T = _inputs(wl, ctx, seed=21)
    B = len(ctx)
    warm = M.mla_create(config_of(wl))
    try:
        want_o, want_l = _with_workspace(warm, wl, cache, q, ctx_d, T, B)
    finally:
        M.mla_destroy(warm)
    out = torch.empty((B, wl.n_h, wl.d_c), dtype=torch_dtype(wl), device="cuda")
    lse = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
    handle = M.mla_create(config_of(wl))
    try:
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        M.mla_decode_attn_combine_noalloc(handle, q, cache, T, None, 0, ctx_d, B, 0, out, lse)
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert M.mla_get_device_status(handle) == M.MLA_OK
        assert free1 == free0, f"free device memory changed by {free0 - free1} bytes"
        compare(to_host(out), {b: want_o[b] for b in range(B)}, wl, "ctx_lat", list(range(B)))
        compare(to_host(lse), {b: want_l[b] for b in range(B)}, wl, "lse", list(range(B)))
    finally:
        M.mla_destroy(handle)


def test_noalloc_lowers_the_default_split_count_to_fit():
    """At 128 heads the default split count's partials for a batch of 64 do
    not fit the array; the entry point uses the largest split count that does
    and matches the workspace entry points run at that count."""
    wl = WORKLOADS["v2_b64_ctx8k"]
    B = 64
    ctx = [256 + 37 * b for b in range(B)]
    cache, q, ctx_d, T = _inputs(wl, ctx, seed=31)
    handle = M.mla_create(config_of(wl))
    try:
        limit = M.mla_noalloc_scratch_bytes()
        P = M.mla_default_num_parts(handle)
        assert M.mla_decode_workspace_size(handle, B, P) > limit     # the case this test is for
        while P > 1 and M.mla_decode_workspace_size(handle, B, P) > limit:
            P -= 1
        assert P > 1
        nbytes = M.mla_decode_workspace_size(handle, B, P)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        want_o = torch.empty((B, wl.n_h, wl.d_c), dtype=torch_dtype(wl), device="cuda")
        want_l = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
        M.mla_decode_attn(handle, q, cache, T, None, 0, ctx_d, B, P, ws, nbytes)
        M.mla_combine_splits(handle, ws, nbytes, B, P, want_o, want_l)
        for call in range(2):
            got_o, got_l = _without_allocation(handle, wl, cache, q, ctx_d, T, B)
            wo, wl_ = to_host(want_o), to_host(want_l)
            # the same split count: the same summation order, bit for bit
            assert np.array_equal(got_o, wo), f"call {call}: ctx_lat differs"
            assert np.array_equal(got_l, wl_), f"call {call}: lse differs"
    finally:
        M.mla_destroy(handle)


def test_noalloc_rejects_what_does_not_fit():
    wl = WORKLOADS["v2_b64_ctx8k"]
    handle = M.mla_create(config_of(wl))
    try:
        limit = M.mla_noalloc_scratch_bytes()
        per_piece = wl.n_h * (wl.d_c + 1) * 4
        B = limit // per_piece + 1            # even one split per sequence is too much
        out = torch.empty(1, device="cuda")
        dummy = torch.empty(1, dtype=torch.int32, device="cuda")
        with pytest.raises(M.MlaError) as err:
            M.mla_decode_attn_combine_noalloc(handle, out, out, 1, None, 0, dummy, B, 0, out, None)
        assert err.value.status == M.MLA_ERR_WORKSPACE
        with pytest.raises(M.MlaError) as err:   # an explicit split count that does not fit
            M.mla_decode_attn_combine_noalloc(handle, out, out, 1, None, 0, dummy, 4, 100000, out, None)
        assert err.value.status == M.MLA_ERR_WORKSPACE
    finally:
        M.mla_destroy(handle)
