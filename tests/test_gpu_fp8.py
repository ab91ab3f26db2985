"""GPU parity of the FP8 (E4M3) latent cache against the oracle.

Format (oracle `quantize_rows_fp8`): per token and 128-channel group (over
c^KV, then over k^R), sigma = amax / 448 and codes E4M3(x / sigma), the
decisions taken in float32 on both sides.

* `mla_quantize_rows_fp8` on rows given to both sides exactly (bf16 or fp32
  values): codes and scales bit-exact.
* `mla_cache_append_fp8`: the GPU forms the rows with fp32 accumulation, the
  oracle in float64, so a value within a rounding error of a decision
  boundary may round to the neighbouring code.  Checked: scales within 1e-5
  relative; every code equal to the oracle's, or the neighbouring one where
  the oracle's x / sigma lies within 2e-5 (448 + |x / sigma|) of the midpoint
  between the two; the stored value within half a step of the oracle's row
  (2^-4 |x| + 2^-10 sigma) plus 8e-3 sigma for the accumulation difference.
* `mla_decode_attn_fp8` + `mla_combine_splits`: against the oracle's softmax
  over the dequantised rows of the same codes, with the bf16 tolerances of
  the step (max abs 2e-2, rel L2 5e-3; fp32 1e-5).  The tensor-core kernel
  rounds code * sigma to bf16, which these tolerances cover.
"""

import numpy as np
import pytest
import torch

import head_latent_attention_09_b200 as M
from oracle import mla_oracle as O
from tests.gpu_harness import (compare, config_of, create_handle, rope_arg, to_dev, to_host,
                               torch_dtype)
from workloads import (WORKLOADS, bf16_round, block_table, ctx_lengths, draw_weights,
                       hidden_states, queries, random_cache)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from head_latent_attention_09_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _codes_close(got_codes, got_sc, rows, d_c, d_r, what):
    """Append-path check (see the module docstring).  rows: oracle float64."""
    rows = np.asarray(rows, np.float64)
    want_codes, want_sc = O.quantize_rows_fp8(rows, d_c, d_r)
    got_sc = np.asarray(got_sc, np.float64)
    ref_sc = np.zeros_like(got_sc)
    for gi, (a, b) in enumerate(O.fp8_groups(d_c, d_r)):
        ref_sc[:, gi] = np.abs(rows[:, a:b]).max(axis=1) / 448.0
    assert np.all(np.abs(got_sc - ref_sc) <= 1e-5 * ref_sc + 1e-30), f"{what}: scales"
    deq = O.dequantize_rows_fp8(got_codes, got_sc, d_c, d_r)
    sig = np.zeros_like(rows)
    v = np.zeros_like(rows)
    for gi, (a, b) in enumerate(O.fp8_groups(d_c, d_r)):
        sig[:, a:b] = ref_sc[:, gi:gi + 1]
        v[:, a:b] = rows[:, a:b] / np.where(ref_sc[:, gi:gi + 1] > 0, ref_sc[:, gi:gi + 1], 1.0)
    bound = 2.0 ** -4 * np.abs(rows) + 2.0 ** -10 * sig + 8e-3 * sig
    assert np.all(np.abs(deq - rows) <= bound), f"{what}: stored values"
    diff = got_codes != want_codes
    if diff.any():
        a_val = O.e4m3_decode(got_codes[diff])
        b_val = O.e4m3_decode(want_codes[diff])
        mid = (a_val + b_val) / 2
        vv = v[diff]
        near = np.abs(vv - mid) <= 2e-5 * (448.0 + np.abs(vv))
        # neighbours: no representable value strictly between the two
        assert np.all(near), f"{what}: {int((~near).sum())} codes differ away from a rounding boundary"
    assert diff.mean() < 1e-3, f"{what}: {diff.mean():.2e} of the codes differ"


# ---------------------------------------------------------------------------
# quantisation of given rows: bit-exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["v2lite_b32_ctx4k", "tiny_fp32"])
def test_quantize_rows_bit_exact(name):
    wl = WORKLOADS[name]
    n = 777
    rows = random_cache(wl.with_(B=1), n, 1.0)[0].astype(np.float32)
    rng = np.random.default_rng(9)
    rows[1, :128] = 0.0                                   # an all-zero group
    rows[2, 5] = 1e4                                      # an outlier: its group's other values go subnormal
    rows[3] *= np.float32(2.0 ** -30)                     # tiny but normal float32 values
    rows[4, wl.d_c:] = rng.choice([-1.0, 1.0], wl.d_r)    # a flat rotary group: every value is +-amax
    if wl.dtype == "bf16":
        rows = bf16_round(rows)
    handle = M.mla_create(config_of(wl))
    try:
        G = M.mla_fp8_scale_groups(handle)
        assert G == len(O.fp8_groups(wl.d_c, wl.d_r))
        src = to_dev(rows, wl)
        codes = torch.full((n, wl.D), 0xFF, dtype=torch.uint8, device="cuda")
        sc = torch.full((n, G), float("nan"), dtype=torch.float32, device="cuda")
        M.mla_quantize_rows_fp8(handle, src, n, codes, sc)
        assert M.mla_get_device_status(handle) == M.MLA_OK
        got_c, got_s = codes.cpu().numpy(), sc.cpu().numpy()
    finally:
        M.mla_destroy(handle)
    want_c, want_s = O.quantize_rows_fp8(rows, wl.d_c, wl.d_r)
    assert np.array_equal(got_s.view(np.uint32), want_s.view(np.uint32))
    bad = np.argwhere(got_c != want_c)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[:3].tolist()}"


# ---------------------------------------------------------------------------
# a decode step on an FP8 cache
# ---------------------------------------------------------------------------

class Fp8Cache:
    """FP8 codes and scales of a workload's cache on the device (contiguous or
    paged), positions 0 .. ctx_b - 2 filled through mla_cache_append_fp8.
    Unwritten rows hold NaN codes and NaN scales."""

    def __init__(self, wl, handle, w, ctx):
        self.wl, self.ctx = wl, ctx
        D, G = wl.D, M.mla_fp8_scale_groups(handle)
        self.G = G
        if wl.page_size:
            self.table_np, nblk = block_table(wl, ctx)
            self.max_blk = self.table_np.shape[1]
            self.table = torch.from_numpy(self.table_np).cuda()
            self.codes = torch.full((nblk, wl.page_size, D), 0x7F, dtype=torch.uint8, device="cuda")
            self.scales = torch.full((nblk, wl.page_size, G), float("nan"), dtype=torch.float32,
                                     device="cuda")
            self.cache_len = nblk
        else:
            self.table_np, self.table, self.max_blk = None, None, 0
            self.cap = int(max(1, ctx.max()))
            self.codes = torch.full((wl.B, self.cap, D), 0x7F, dtype=torch.uint8, device="cuda")
            self.scales = torch.full((wl.B, self.cap, G), float("nan"), dtype=torch.float32,
                                     device="cuda")
            self.cache_len = self.cap
        chunk = 4096
        ws_bytes = M.mla_cache_append_fp8_workspace_size(handle, 1, chunk)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        for b in range(wl.B):
            n = int(ctx[b]) - 1
            if n <= 0:
                continue
            hb = hidden_states(wl, b, n)
            for t0 in range(0, n, chunk):
                t1 = min(n, t0 + chunk)
                sp = torch.full((1,), t0, dtype=torch.int32, device="cuda")
                cp, sp_ptr, tp = self.seq_view(b)
                M.mla_cache_append_fp8(handle, to_dev(hb[t0:t1], wl), 1, t1 - t0, sp, w["w_dkv"],
                                       w["w_kr"], cp, sp_ptr, self.cache_len, tp, self.max_blk, ws,
                                       ws_bytes)

    def seq_view(self, b):
        if self.wl.page_size:
            return (self.codes.data_ptr(), self.scales.data_ptr(),
                    self.table.data_ptr() + 4 * b * self.max_blk)
        return (self.codes.data_ptr() + b * self.cap * self.wl.D,
                self.scales.data_ptr() + 4 * b * self.cap * self.G, None)

    def rows_of(self, b, n):
        """(codes [n, D], scales [n, G]) of positions 0 .. n-1 of sequence b."""
        if self.wl.page_size:
            ps = self.wl.page_size
            pos = np.arange(n)
            idx = torch.from_numpy(self.table_np[b, pos // ps].astype(np.int64) * ps + pos % ps).cuda()
            return (self.codes.view(-1, self.wl.D)[idx].cpu().numpy(),
                    self.scales.view(-1, self.G)[idx].cpu().numpy())
        return self.codes[b, :n].cpu().numpy(), self.scales[b, :n].cpu().numpy()


def run_fp8_step(wl, num_parts=0):
    handle = create_handle(wl)
    try:
        w = {k: to_dev(v, wl) for k, v in draw_weights(wl).items()}
        ctx = ctx_lengths(wl)
        B, dt = wl.B, torch_dtype(wl)
        cache = Fp8Cache(wl, handle, w, ctx)
        h_new = np.stack([hidden_states(wl, b, int(ctx[b]))[-1] if ctx[b] > 0
                          else np.zeros(wl.d_model, np.float32) for b in range(B)])
        qn, qr = queries(wl)
        pos = torch.from_numpy(np.maximum(ctx - 1, 0).astype(np.int32)).cuda()
        ctx_d = torch.from_numpy(ctx.astype(np.int32)).cuda()
        ws_a = M.mla_cache_append_fp8_workspace_size(handle, B, 1)
        ws_app = torch.empty(ws_a, dtype=torch.uint8, device="cuda")
        h_d = to_dev(h_new, wl).view(B, 1, wl.d_model)
        for b in range(B):
            if ctx[b] > 0:
                cp, sp_ptr, tp = cache.seq_view(b)
                M.mla_cache_append_fp8(handle, h_d[b:b + 1], 1, 1, pos[b:b + 1], w["w_dkv"],
                                       w["w_kr"], cp, sp_ptr, cache.cache_len, tp, cache.max_blk,
                                       ws_app, ws_a)
        q_abs = torch.empty((B, wl.n_h, wl.D), dtype=dt, device="cuda")
        ctx_lat = torch.empty((B, wl.n_h, wl.d_c), dtype=dt, device="cuda")
        lse = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
        o = torch.empty((B, wl.n_h, wl.d_h), dtype=dt, device="cuda")
        P = num_parts or M.mla_default_num_parts(handle)
        ws_bytes = M.mla_decode_workspace_size(handle, B, P)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        M.mla_absorb_q(handle, to_dev(qn, wl), to_dev(qr, wl), pos, w["w_uk"], q_abs, B)
        M.mla_decode_attn_fp8(handle, q_abs, cache.codes, cache.scales, cache.cache_len,
                              cache.table, cache.max_blk, ctx_d, B, P, ws, ws_bytes)
        M.mla_combine_splits(handle, ws, ws_bytes, B, P, ctx_lat, lse)
        M.mla_out_proj(handle, ctx_lat, w["w_uv"], None, o, None, B)
        st = M.mla_get_device_status(handle)
        assert st == M.MLA_OK, M.mla_status_string(st)
        return {"q_abs": to_host(q_abs), "ctx_lat": to_host(ctx_lat), "lse": to_host(lse),
                "o": to_host(o), "ctx": ctx, "cache": cache}
    finally:
        M.mla_destroy(handle)


def check_fp8_step(wl, got, seqs, code_row_stride=1):
    w = draw_weights(wl)
    qn, qr = queries(wl)
    base = rope_arg(wl)
    kw = dict(n_h=wl.n_h, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, base=base)
    want = {k: {} for k in ("q_abs", "ctx_lat", "lse", "o")}
    for b in seqs:
        n = int(got["ctx"][b])
        rows = O.cache_rows(hidden_states(wl, b, n), w["w_dkv"], w["w_kr"], np.arange(n), base)
        codes, sc = got["cache"].rows_of(b, n)
        k = code_row_stride
        _codes_close(codes[::k], sc[::k], rows[::k], wl.d_c, wl.d_r, f"cache of sequence {b}")
        stored = O.dequantize_rows_fp8(codes, sc, wl.d_c, wl.d_r)
        r = O.mla_decode_absorbed(qn[b], qr[b], n - 1, stored, w["w_uk"], w["w_uv"], **kw)
        for k in want:
            want[k][b] = r[k]
    for k in want:
        compare(got[k], want[k], wl, f"fp8 {k}", seqs)


@pytest.mark.parametrize("name,over", [
    ("v2lite_b32_ctx4k", {"ctx": (1, 63, 64, 65, 700, 0, 129)}),          # 16 heads: tensor cores
    ("v2lite_b32_ctx4k", {"ctx": (300, 2000, 1), "n_h": 32}),             # 32 heads: tensor cores
    ("v2lite_paged_ragged_b128", {"ctx": (1, 64, 65, 300, 1, 130)}),      # paged, 64-token pages
    ("tiny_fp32", {}),                                                    # fp32: CUDA cores
    ("v2_b64_ctx8k", {"ctx": (70, 5, 0)}),                                # 128 heads: CUDA cores
])
def test_fp8_decode_step(name, over):
    over = dict(over)
    if "ctx" in over:
        over["B"] = len(over["ctx"])
    wl = WORKLOADS[name].with_(**over)
    got = run_fp8_step(wl)
    seqs = [b for b in range(wl.B) if got["ctx"][b] > 0]
    check_fp8_step(wl, got, seqs)
    for b in range(wl.B):
        if got["ctx"][b] == 0:
            assert np.all(got["ctx_lat"][b] == 0) and np.all(np.isneginf(got["lse"][b]))


@pytest.mark.parametrize("parts", [1, 5, 300])
def test_fp8_split_counts(parts):
    wl = WORKLOADS["v2lite_b32_ctx4k"].with_(B=3, ctx=(1000, 64, 333))
    got = run_fp8_step(wl, num_parts=parts)
    check_fp8_step(wl, got, [0, 1, 2])


def test_fp8_128k_full():
    """The FP8 benchmark workload at full size (B = 4 x 131072 tokens), in the
    launch configuration the benchmark times; sequence 1 checked whole."""
    wl = WORKLOADS["v2lite_b4_ctx128k"]
    got = run_fp8_step(wl)
    check_fp8_step(wl, got, [1], code_row_stride=16)


def test_fp8_attention_rejects_missing_scales():
    wl = WORKLOADS["v2lite_b32_ctx4k"].with_(B=1, ctx=(64,))
    handle = M.mla_create(config_of(wl))
    try:
        q = torch.zeros((1, wl.n_h, wl.D), dtype=torch.bfloat16, device="cuda")
        codes = torch.zeros((1, 64, wl.D), dtype=torch.uint8, device="cuda")
        ctx_d = torch.full((1,), 64, dtype=torch.int32, device="cuda")
        ws_bytes = M.mla_decode_workspace_size(handle, 1, 4)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        with pytest.raises(M.MlaError):
            M.mla_decode_attn_fp8(handle, q, codes, None, 64, None, 0, ctx_d, 1, 4, ws, ws_bytes)
        small = torch.empty(64, dtype=torch.uint8, device="cuda")
        with pytest.raises(M.MlaError):
            M.mla_cache_append_fp8(handle, q, 1, 1, ctx_d, q, q, codes,
                                   torch.empty(5, device="cuda"), 64, None, 0, small, 64)
    finally:
        M.mla_destroy(handle)


@pytest.mark.parametrize("n_h", [16, 32])
def test_fp8_attention_every_code(n_h):
    """Attention over codes drawn directly (not by the quantiser): each row and
    scale group holds either all 254 non-NaN E4M3 codes at random, or only the
    subnormal codes (exponent field 0, both signs), with the group's scale
    chosen so that both kinds carry values of the same size.  Against the
    oracle's softmax over the dequantised rows (value = code * sigma), this
    pins the kernel's widening of every code, subnormals included, which the
    quantiser's output reaches only by chance."""
    wl = WORKLOADS["v2lite_b32_ctx4k"].with_(B=3, ctx=(700, 129, 1), n_h=n_h)
    D, G, cache_len = wl.D, 5, 704
    rng = np.random.default_rng(8675309 + n_h)
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    subnormal = np.array([c for c in range(256) if (c & 0x78) == 0], dtype=np.uint8)
    codes = rng.choice(finite, size=(wl.B, cache_len, D)).astype(np.uint8)
    sub_group = rng.random((wl.B, cache_len, G)) < 0.4
    groups = O.fp8_groups(wl.d_c, wl.d_r)
    scales = np.empty((wl.B, cache_len, G), np.float32)
    for g, (a, b) in enumerate(groups):
        sub_codes = rng.choice(subnormal, size=(wl.B, cache_len, b - a)).astype(np.uint8)
        codes[:, :, a:b] = np.where(sub_group[:, :, g:g + 1], sub_codes, codes[:, :, a:b])
        # largest magnitude of the group: 448 for all codes, 7 * 2^-9 for subnormals
        top = np.where(sub_group[:, :, g], 7.0 * 2.0 ** -9, 448.0)
        scales[:, :, g] = (0.5 * np.exp2(rng.uniform(-2.0, 2.0, (wl.B, cache_len))) / top).astype(np.float32)
    q_abs = bf16_round(rng.standard_normal((wl.B, n_h, D)).astype(np.float32))
    ctx = np.asarray(wl.ctx, np.int32)

    handle = create_handle(wl)
    try:
        P = M.mla_default_num_parts(handle)
        ws_bytes = M.mla_decode_workspace_size(handle, wl.B, P)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        ctx_lat = torch.empty((wl.B, n_h, wl.d_c), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((wl.B, n_h), dtype=torch.float32, device="cuda")
        M.mla_decode_attn_fp8(handle, torch.from_numpy(q_abs).to(torch.bfloat16).cuda(),
                              torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                              cache_len, None, 0, torch.from_numpy(ctx).cuda(), wl.B, P, ws, ws_bytes)
        M.mla_combine_splits(handle, ws, ws_bytes, wl.B, P, ctx_lat, lse)
        assert M.mla_get_device_status(handle) == M.MLA_OK
        got = {"ctx_lat": to_host(ctx_lat), "lse": to_host(lse)}
    finally:
        M.mla_destroy(handle)
    scale = O.attention_scale(wl.d_h, wl.d_r, rope_arg(wl))
    want = {"ctx_lat": {}, "lse": {}}
    for b in range(wl.B):
        rows = O.dequantize_rows_fp8(codes[b, :ctx[b]], scales[b, :ctx[b]], wl.d_c, wl.d_r)
        want["ctx_lat"][b], want["lse"][b] = O.latent_attention(q_abs[b], rows, d_c=wl.d_c, scale=scale)
    for k in want:
        compare(got[k], want[k], wl, f"fp8 every code {k}")
    # each 128-column group on its own, so that an error confined to one
    # group's widening is not diluted by the other groups' norm
    for b in range(wl.B):
        for g, (a, e) in enumerate(groups[:4]):
            err = got["ctx_lat"][b][:, a:e] - want["ctx_lat"][b][:, a:e]
            ref = np.linalg.norm(want["ctx_lat"][b][:, a:e])
            assert np.linalg.norm(err) <= 5e-3 * max(ref, 1e-30), (b, g, np.linalg.norm(err) / ref)
