"""Drive one decode step of the CUDA library through its C ABI on a workload,
and compute the same step with the CPU oracle, on the same seeded inputs.

The GPU side only marshals buffers: every step runs in libmla.so.  The oracle
side never sees a GPU result: it rebuilds the cache from the same hidden
states in float64.
"""

from __future__ import annotations

import numpy as np
import torch

import head_latent_attention_09_b200 as M
from oracle import mla_oracle as O
from workloads import (bf16_bits, block_table, ctx_lengths, draw_weights, hidden_states, queries)

# Tolerances stated by the spec: bf16 inputs with fp32 accumulation must match
# within max |err| <= 2e-2 and relative L2 <= 5e-3; the fp32 tiny workload
# within 1e-5 relative.
BF16_MAX_ABS = 2e-2
BF16_REL_L2 = 5e-3
FP32_REL = 1e-5


def to_dev(x: np.ndarray, wl, dev="cuda"):
    if wl.dtype == "bf16":
        return torch.from_numpy(bf16_bits(x).view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(dev)


def to_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def config_of(wl) -> M.mla_config:
    return M.mla_config(n_h=wl.n_h, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, d_model=wl.d_model,
                        page_size=wl.page_size, rope_base=wl.rope_base,
                        dtype=M.MLA_BF16 if wl.dtype == "bf16" else M.MLA_FP32)


def rope_arg(wl):
    """The oracle's `base` argument for a workload: a plain base, or a RopeSpec
    carrying its YaRN scaling."""
    if wl.rope_scaling is None:
        return wl.rope_base
    s, orig, alpha, beta, coef = wl.rope_scaling
    return O.RopeSpec(base=wl.rope_base, factor=s, original_ctx=orig, alpha=alpha, beta=beta,
                      mscale_coef=coef)


def strict_on(handle, wl, strict=None):
    """Strict tensor-core mode for bf16 workloads (strict=None): a call whose
    tensor-core kernel cannot take its arguments then fails instead of
    silently running the CUDA-core kernel, so a passing bf16 parity test shows
    that the tensor-core path ran."""
    if strict is None:
        strict = wl.dtype == "bf16"
    M.mla_set_strict(handle, 1 if strict else 0)
    return handle


def create_handle(wl, strict=None) -> int:
    """mla_create for the workload, with its RoPE scaling applied and strict
    tensor-core mode on for bf16 (see strict_on)."""
    handle = M.mla_create(config_of(wl))
    try:
        if wl.rope_scaling is not None:
            M.mla_set_rope_scaling(handle, *wl.rope_scaling)
        strict_on(handle, wl, strict)
    except Exception:
        M.mla_destroy(handle)
        raise
    return handle


def torch_dtype(wl):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


class DeviceCache:
    """The latent cache of a workload on the device (contiguous or paged), with
    positions 0 .. ctx_b - 2 of every sequence filled through mla_cache_append
    from the generator's hidden states."""

    def __init__(self, wl, handle, w, ctx, dev="cuda", fill_rows=None):
        self.wl, self.ctx = wl, ctx
        D = wl.D
        dt = torch_dtype(wl)
        if wl.page_size:
            self.table_np, self.num_blocks = block_table(wl, ctx)
            self.max_blk = self.table_np.shape[1]
            self.table = torch.from_numpy(self.table_np).to(dev)
            self.data = torch.empty((self.num_blocks, wl.page_size, D), dtype=dt, device=dev)
            self.cache_len = self.num_blocks
        else:
            self.table_np, self.table, self.max_blk = None, None, 0
            self.cap = int(max(1, ctx.max()))
            self.data = torch.empty((wl.B, self.cap, D), dtype=dt, device=dev)
            self.cache_len = self.cap
        # Fill with NaN so that any read of an unwritten row shows up.
        self.data.fill_(float("nan"))
        zero = torch.zeros(1, dtype=torch.int32, device=dev)
        chunk = 4096
        for b in range(wl.B):
            n = int(ctx[b]) - 1                      # the last position is appended by the step
            if n <= 0:
                continue
            hb = hidden_states(wl, b, n) if fill_rows is None else fill_rows(b, n)
            for t0 in range(0, n, chunk):
                t1 = min(n, t0 + chunk)
                hd = to_dev(hb[t0:t1], wl, dev)
                sp = torch.full((1,), t0, dtype=torch.int32, device=dev)
                cache_ptr, tbl_ptr = self.seq_view(b)
                M.mla_cache_append(handle, hd, 1, t1 - t0, sp, w["w_dkv"], w["w_kr"], cache_ptr,
                                   self.cache_len, tbl_ptr, self.max_blk)
        del zero

    def seq_view(self, b):
        """(cache pointer, block-table pointer) that make sequence b look like
        sequence 0 of a batch of one."""
        esz = self.data.element_size()
        if self.wl.page_size:
            return self.data.data_ptr(), self.table.data_ptr() + 4 * b * self.max_blk
        return self.data.data_ptr() + esz * b * self.cap * self.wl.D, None

    def rows_of(self, b, positions):
        pos = np.asarray(positions)
        if self.wl.page_size:
            ps = self.wl.page_size
            blk = self.table_np[b, pos // ps]
            idx = torch.from_numpy((blk.astype(np.int64) * ps + pos % ps)).to(self.data.device)
            return to_host(self.data.view(-1, self.wl.D)[idx])
        return to_host(self.data[b, torch.from_numpy(pos).to(self.data.device)])


def run_decode_step(wl, num_parts=0, with_wo=False, dev="cuda", keep=False, fill_rows=None, fused=False):
    """One decode step for every sequence of the workload.  Returns host arrays.

    With fused=True the same workspace is then also finished by
    mla_combine_out_proj, twice: with ctx_lat and lse written ("fused_*") and
    with both left out ("fused_o_bare")."""
    handle = create_handle(wl)
    try:
        wnp = draw_weights(wl, with_wo=with_wo)
        w = {k: to_dev(v, wl, dev) for k, v in wnp.items()}
        ctx = ctx_lengths(wl)
        cache = DeviceCache(wl, handle, w, ctx, dev, fill_rows=fill_rows)
        B = wl.B
        dt = torch_dtype(wl)
        # inputs of the step
        h_new = np.stack([(hidden_states(wl, b, int(ctx[b])) if fill_rows is None
                           else fill_rows(b, int(ctx[b])))[-1] if ctx[b] > 0
                          else np.zeros(wl.d_model, np.float32) for b in range(B)])
        qn, qr = queries(wl)
        h_d = to_dev(h_new, wl, dev)
        qn_d, qr_d = to_dev(qn, wl, dev), to_dev(qr, wl, dev)
        pos = torch.from_numpy(np.maximum(ctx - 1, 0).astype(np.int32)).to(dev)
        ctx_d = torch.from_numpy(ctx.astype(np.int32)).to(dev)
        q_abs = torch.empty((B, wl.n_h, wl.D), dtype=dt, device=dev)
        ctx_lat = torch.empty((B, wl.n_h, wl.d_c), dtype=dt, device=dev)
        lse = torch.empty((B, wl.n_h), dtype=torch.float32, device=dev)
        o = torch.empty((B, wl.n_h, wl.d_h), dtype=dt, device=dev)
        u = torch.empty((B, wl.d_model), dtype=dt, device=dev) if with_wo else None
        P = num_parts or M.mla_default_num_parts(handle)
        ws_bytes = M.mla_decode_workspace_size(handle, B, P)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

        has_new = ctx > 0
        # append the step's own token (sequences with ctx = 0 append nothing: give them
        # a position past the cache so nothing is written -- done by excluding them)
        if has_new.all():
            M.mla_cache_append(handle, h_d.view(B, 1, wl.d_model), B, 1, pos, w["w_dkv"], w["w_kr"],
                               cache.data, cache.cache_len, cache.table, cache.max_blk)
        else:
            for b in np.nonzero(has_new)[0]:
                cp, tp = cache.seq_view(int(b))
                M.mla_cache_append(handle, h_d[int(b)].view(1, 1, wl.d_model), 1, 1,
                                   pos[int(b):int(b) + 1], w["w_dkv"], w["w_kr"], cp,
                                   cache.cache_len, tp, cache.max_blk)
        M.mla_absorb_q(handle, qn_d, qr_d, pos, w["w_uk"], q_abs, B)
        M.mla_decode_attn(handle, q_abs, cache.data, cache.cache_len, cache.table, cache.max_blk,
                          ctx_d, B, P, ws, ws_bytes)
        M.mla_combine_splits(handle, ws, ws_bytes, B, P, ctx_lat, lse)
        M.mla_out_proj(handle, ctx_lat, w["w_uv"], w.get("w_o"), o, u, B)
        fused_out = {}
        if fused:
            ctx_f = torch.full_like(ctx_lat, float("nan"))
            lse_f = torch.full_like(lse, float("nan"))
            o_f = torch.full_like(o, float("nan"))
            u_f = torch.full_like(u, float("nan")) if with_wo else None
            M.mla_combine_out_proj(handle, ws, ws_bytes, B, P, w["w_uv"], w.get("w_o"), o_f, u_f, ctx_f, lse_f)
            o_bare = torch.full_like(o, float("nan"))
            u_bare = torch.full_like(u, float("nan")) if with_wo else None
            M.mla_combine_out_proj(handle, ws, ws_bytes, B, P, w["w_uv"], w.get("w_o"), o_bare, u_bare)
            fused_out = {"fused_ctx_lat": to_host(ctx_f), "fused_lse": to_host(lse_f), "fused_o": to_host(o_f),
                         "fused_u": to_host(u_f) if with_wo else None, "fused_o_bare": to_host(o_bare)}
        st = M.mla_get_device_status(handle)
        if st != M.MLA_OK:
            raise M.MlaError(st, "device status")
        out = {
            "q_abs": to_host(q_abs), "ctx_lat": to_host(ctx_lat), "lse": to_host(lse),
            "o": to_host(o), "u": to_host(u) if with_wo else None,
            "cache_new_rows": np.stack([cache.rows_of(b, [max(int(ctx[b]) - 1, 0)])[0]
                                        for b in range(B)]),
            "ctx": ctx,
            **fused_out,
        }
        if keep:
            out["_cache"] = cache
            out["_handle"] = handle
        return out
    finally:
        if not keep:
            M.mla_destroy(handle)


def oracle_step(wl, seqs, with_wo=False, explicit_heads=None, fill_rows=None):
    """The oracle's decode step for the listed sequences (float64)."""
    w = draw_weights(wl, with_wo=with_wo)
    ctx = ctx_lengths(wl)
    qn, qr = queries(wl)
    res = {k: {} for k in ("q_abs", "ctx_lat", "lse", "o", "u", "cache_new_rows", "o_explicit")}
    base = rope_arg(wl)
    kw = dict(n_h=wl.n_h, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, base=base)
    for b in seqs:
        n = int(ctx[b])
        hb = hidden_states(wl, b, n) if fill_rows is None else fill_rows(b, n)
        rows = O.cache_rows(hb, w["w_dkv"], w["w_kr"], np.arange(n), base)
        r = O.mla_decode_absorbed(qn[b], qr[b], max(n - 1, 0), rows, w["w_uk"], w["w_uv"],
                                  w_o=w.get("w_o"), **kw)
        for k in ("q_abs", "ctx_lat", "lse", "o", "u"):
            res[k][b] = r[k]
        res["cache_new_rows"][b] = rows[-1] if n > 0 else None
        if explicit_heads is not None:
            res["o_explicit"][b] = O.mla_decode_explicit(qn[b], qr[b], n - 1, rows, w["w_uk"],
                                                         w["w_uv"], heads=explicit_heads, **kw)[0]
    return res


def compare(got, want: dict, wl, what: str, seqs=None):
    """Check the GPU arrays (indexed by sequence) against the oracle's dict
    {b: array}; raises AssertionError with the error figures."""
    seqs = list(want.keys()) if seqs is None else seqs
    g = np.stack([np.asarray(got[b], np.float64) for b in seqs if want[b] is not None])
    r = np.stack([np.asarray(want[b], np.float64) for b in seqs if want[b] is not None])
    err = g - r
    fin = np.isfinite(r)
    assert np.array_equal(np.isfinite(g), fin), f"{what}: non-finite mismatch"
    err = np.where(fin, err, 0.0)
    rel = float(np.linalg.norm(err) / max(np.linalg.norm(np.where(fin, r, 0.0)), 1e-30))
    mx = float(np.abs(err).max()) if err.size else 0.0
    if wl.dtype == "bf16":
        assert mx <= BF16_MAX_ABS and rel <= BF16_REL_L2, \
            f"{what}: max abs {mx:.3e} (<= {BF16_MAX_ABS}), rel L2 {rel:.3e} (<= {BF16_REL_L2})"
    else:
        scale = max(float(np.abs(np.where(fin, r, 0.0)).max()), 1e-30)
        assert rel <= FP32_REL and mx <= FP32_REL * scale, \
            f"{what}: rel L2 {rel:.3e}, max abs/scale {mx / scale:.3e} (<= {FP32_REL})"
    return mx, rel
