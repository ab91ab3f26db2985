"""Guard bands around every buffer the library writes (a stand-in for a
memory sanitizer, which this pool does not offer): each output tensor sits in
the middle of a larger allocation whose first and last 4 KB hold a sentinel
byte pattern.  One step of every entry point that writes device memory runs
on small ragged shapes (DeepSeek-V2 and V2-Lite, contiguous and paged caches,
bf16, FP8 and fp32, with W^O and the query path), and afterwards every
sentinel byte must be unchanged and the device status clean.  Values are not
checked here (the parity tests do that); only that nothing is written outside
its buffer.
"""

import numpy as np
import pytest
import torch

import head_latent_attention_09_b200 as M
from tests.gpu_harness import config_of
from workloads import WORKLOADS, block_table

pytestmark = pytest.mark.gpu

GUARD = 4096
SENTINEL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _built():
    from head_latent_attention_09_b200 import build
    build.build()
    assert torch.cuda.is_available()


class Guarded:
    """Device tensors with sentinel bands on both sides."""

    def __init__(self):
        self.bufs = []

    def empty(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((GUARD + n + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.bufs.append((raw, n))
        return raw[GUARD:GUARD + n].view(dtype).view(shape)

    def raw_bytes(self, n):
        raw = torch.full((GUARD + n + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.bufs.append((raw, n))
        return raw[GUARD:GUARD + n]

    def check(self):
        torch.cuda.synchronize()
        for k, (raw, n) in enumerate(self.bufs):
            head = raw[:GUARD].cpu().numpy()
            tail = raw[GUARD + n:].cpu().numpy()
            assert np.all(head == SENTINEL), f"buffer {k}: {int((head != SENTINEL).sum())} bytes written before it"
            assert np.all(tail == SENTINEL), f"buffer {k}: {int((tail != SENTINEL).sum())} bytes written after it"


def _rand(shape, dt, std=1.0, seed=[0]):
    seed[0] += 1
    g = torch.Generator(device="cuda")
    g.manual_seed(1234 + seed[0])
    return (torch.randn(*shape, generator=g, device="cuda") * std).to(dt)


def _step(wl, ctx, fp8=False, with_wo=True, query=True):
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    B, H, D, d = len(ctx), wl.n_h, wl.D, wl.d_model
    wl = wl.with_(B=B, ctx=tuple(ctx))
    ctx = np.asarray(ctx, np.int64)
    G = Guarded()
    handle = M.mla_create(config_of(wl))
    try:
        w_dkv = _rand((wl.d_c, d), dt, d ** -0.5)
        w_kr = _rand((wl.d_r, d), dt, d ** -0.5)
        w_uk = _rand((H * wl.d_h, wl.d_c), dt, wl.d_c ** -0.5)
        w_uv = _rand((H * wl.d_h, wl.d_c), dt, wl.d_c ** -0.5)
        w_o = _rand((d, H * wl.d_h), dt, (H * wl.d_h) ** -0.5) if with_wo else None
        if wl.page_size:
            tbl_np, nblk = block_table(wl, ctx)
            tbl = torch.from_numpy(tbl_np).cuda()
            max_blk, cache_len, rows = tbl_np.shape[1], nblk, nblk * wl.page_size
        else:
            tbl, max_blk = None, 0
            cache_len = int(ctx.max())
            rows = B * cache_len
        pos = torch.from_numpy(np.maximum(ctx - 1, 0).astype(np.int32)).cuda()
        ctx_d = torch.from_numpy(ctx.astype(np.int32)).cuda()
        h_all = _rand((B, int(ctx.max()), d), dt)
        groups = M.mla_fp8_scale_groups(handle)
        if fp8:
            cache = G.empty((rows, D), torch.uint8)
            scales = G.empty((rows, groups), torch.float32)
            cache.fill_(0)
            scales.fill_(0)
            aws = M.mla_cache_append_fp8_workspace_size(handle, 1, int(ctx.max()))
            aw = G.raw_bytes(aws)
        else:
            cache = G.empty((rows, D), dt)
            cache.fill_(0)
        # fill every sequence's rows one sequence at a time (a batch of one)
        for b in range(B):
            n = int(ctx[b])
            if n == 0:
                continue
            start = torch.zeros(1, dtype=torch.int32, device="cuda")
            if wl.page_size:
                cp, tp = cache.data_ptr(), tbl.data_ptr() + 4 * b * max_blk
            else:
                cp, tp = cache.data_ptr() + cache.element_size() * b * cache_len * D, None
            if fp8:
                sp = scales.data_ptr() + (0 if wl.page_size else 4 * b * cache_len * groups)
                M.mla_cache_append_fp8(handle, h_all[b, :n].contiguous(), 1, n, start, w_dkv, w_kr, cp, sp,
                                       cache_len, tp, max_blk, aw, aws)
            else:
                M.mla_cache_append(handle, h_all[b, :n].contiguous(), 1, n, start, w_dkv, w_kr, cp, cache_len,
                                   tp, max_blk)
        q_nope = G.empty((B, H, wl.d_h), dt)
        q_rope = G.empty((B, H, wl.d_r), dt)
        if query:
            x = _rand((B, d), dt)
            if wl.d_cq:
                w_dq = _rand((wl.d_cq, d), dt, d ** -0.5)
                w_uq = _rand((H * wl.d_h, wl.d_cq), dt, wl.d_cq ** -0.5)
                w_qr = _rand((H * wl.d_r, wl.d_cq), dt, wl.d_cq ** -0.5)
                c_q = G.empty((B, wl.d_cq), dt)
            else:
                w_dq, c_q = None, None
                w_uq = _rand((H * wl.d_h, d), dt, d ** -0.5)
                w_qr = _rand((H * wl.d_r, d), dt, d ** -0.5)
            M.mla_query_proj(handle, x, B, w_dq, wl.d_cq or 0, w_uq, w_qr, c_q, q_nope, q_rope)
        else:
            q_nope.copy_(_rand((B, H, wl.d_h), dt))
            q_rope.copy_(_rand((B, H, wl.d_r), dt))
        q_abs = G.empty((B, H, D), dt)
        M.mla_absorb_q(handle, q_nope, q_rope, pos, w_uk, q_abs, B)
        P = M.mla_default_num_parts(handle)
        ws_bytes = M.mla_decode_workspace_size(handle, B, P)
        ws = G.raw_bytes(ws_bytes)
        if fp8:
            M.mla_decode_attn_fp8(handle, q_abs, cache, scales, cache_len, tbl, max_blk, ctx_d, B, P, ws, ws_bytes)
        else:
            M.mla_decode_attn(handle, q_abs, cache, cache_len, tbl, max_blk, ctx_d, B, P, ws, ws_bytes)
        ctx_lat = G.empty((B, H, wl.d_c), dt)
        lse = G.empty((B, H), torch.float32)
        M.mla_combine_splits(handle, ws, ws_bytes, B, P, ctx_lat, lse)
        o = G.empty((B, H, wl.d_h), dt)
        u = G.empty((B, d), dt) if with_wo else None
        M.mla_out_proj(handle, ctx_lat, w_uv, w_o, o, u, B)
        o2 = G.empty((B, H, wl.d_h), dt)
        u2 = G.empty((B, d), dt) if with_wo else None
        ctx2 = G.empty((B, H, wl.d_c), dt)
        lse2 = G.empty((B, H), torch.float32)
        M.mla_combine_out_proj(handle, ws, ws_bytes, B, P, w_uv, w_o, o2, u2, ctx2, lse2)
        ctx3 = G.empty((B, H, wl.d_c), torch.float32)
        lse3 = G.empty((B, H), torch.float32)
        M.mla_combine_splits_f32(handle, ws, ws_bytes, B, P, ctx3, lse3)
        ctx4 = G.empty((B, H, wl.d_c), dt)
        lse4 = G.empty((B, H), torch.float32)
        M.mla_merge_ranges(handle, ctx3, lse3, 1, B, ctx4, lse4)
        assert M.mla_get_device_status(handle) == M.MLA_OK
        G.check()
    finally:
        M.mla_destroy(handle)


@pytest.mark.parametrize("name,ctx,fp8", [
    ("v2_b64_ctx8k", (1, 130, 0, 300, 64), False),            # 128 heads, tensor-core GEMMs, d'_c = 1536
    ("v2lite_b32_ctx4k", (5, 700, 64, 1, 129, 0, 300), False),  # 16 heads, uncompressed query
    ("v2lite_paged_ragged_b128", (1, 64, 65, 300, 130), False),  # paged pool
    ("v2lite_b32_ctx4k", (5, 700, 64, 129), True),              # FP8 cache, contiguous
    ("v2lite_paged_ragged_b128", (65, 1, 300), True),            # FP8 cache, paged
    ("tiny_fp32", (17, 64), False),                              # fp32, CUDA-core kernels
])
def test_no_write_outside_the_buffers(name, ctx, fp8):
    _step(WORKLOADS[name], ctx, fp8=fp8)
