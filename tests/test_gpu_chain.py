"""GPU parity of one whole decode step started from the hidden state, as the
workloads with query compression define it (the tiny fp32 workload and the
DeepSeek-V2 shapes):

    h_t --mla_query_proj (W^DQ, W^UQ, W^QR)--> q^C, q^R
        --mla_cache_append (W^DKV, W^KR)-----> the step's own cache row
        --mla_absorb_q --> mla_decode_attn --> mla_combine_splits
        --mla_out_proj (W^UV [, W^O])--------> o [, u]

All on the device through the C ABI, each call feeding the next, against the
oracle's whole chain in float64: c^Q = W^DQ h, q^C = W^UQ c^Q, q^R = W^QR c^Q
("DeepSeek-V2" §2.1.2 query compression, §2.1.3 decoupled query; the
"DeepSeek-V3" note's MLA equations), the cached rows from the same hidden
states, and textbook softmax attention on explicit per-head keys and values
(the same note's o_{t,i}), plus the absorbed form for every head.

bf16 workloads run with strict tensor-core mode on, so every step of the chain
is shown to have run on its tcgen05 kernel.  Tolerances are the spec's: bf16
max |err| <= 2e-2 and relative L2 <= 5e-3; fp32 1e-5 relative.
"""

import numpy as np
import pytest
import torch

import head_latent_attention_09_b200 as M
from oracle import mla_oracle as O
from tests.gpu_harness import DeviceCache, compare, create_handle, rope_arg, to_dev, to_host, torch_dtype
from workloads import WORKLOADS, ctx_lengths, draw_query_weights, draw_weights, hidden_states

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from head_latent_attention_09_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _chain_on_gpu(wl, with_wo):
    handle = create_handle(wl)
    try:
        wnp = draw_weights(wl, with_wo=with_wo)
        w = {k: to_dev(v, wl) for k, v in wnp.items()}
        qw = {k: to_dev(v, wl) for k, v in draw_query_weights(wl).items()}
        ctx = ctx_lengths(wl)
        cache = DeviceCache(wl, handle, w, ctx)          # positions 0 .. ctx-2
        B, dt = wl.B, torch_dtype(wl)
        h_new = np.stack([hidden_states(wl, b, int(ctx[b]))[-1] for b in range(B)])
        h_d = to_dev(h_new, wl)
        pos = torch.from_numpy((ctx - 1).astype(np.int32)).cuda()
        ctx_d = torch.from_numpy(ctx.astype(np.int32)).cuda()
        c_q = torch.empty((B, wl.d_cq), dtype=dt, device="cuda")
        q_nope = torch.empty((B, wl.n_h, wl.d_h), dtype=dt, device="cuda")
        q_rope = torch.empty((B, wl.n_h, wl.d_r), dtype=dt, device="cuda")
        q_abs = torch.empty((B, wl.n_h, wl.D), dtype=dt, device="cuda")
        ctx_lat = torch.empty((B, wl.n_h, wl.d_c), dtype=dt, device="cuda")
        lse = torch.empty((B, wl.n_h), dtype=torch.float32, device="cuda")
        o = torch.empty((B, wl.n_h, wl.d_h), dtype=dt, device="cuda")
        u = torch.empty((B, wl.d_model), dtype=dt, device="cuda") if with_wo else None
        P = M.mla_default_num_parts(handle)
        ws_bytes = M.mla_decode_workspace_size(handle, B, P)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        M.mla_query_proj(handle, h_d, B, qw["w_dq"], wl.d_cq, qw["w_uq"], qw["w_qr"], c_q, q_nope, q_rope)
        M.mla_cache_append(handle, h_d.view(B, 1, wl.d_model), B, 1, pos, w["w_dkv"], w["w_kr"],
                           cache.data, cache.cache_len, cache.table, cache.max_blk)
        M.mla_absorb_q(handle, q_nope, q_rope, pos, w["w_uk"], q_abs, B)
        M.mla_decode_attn(handle, q_abs, cache.data, cache.cache_len, cache.table, cache.max_blk,
                          ctx_d, B, P, ws, ws_bytes)
        M.mla_combine_splits(handle, ws, ws_bytes, B, P, ctx_lat, lse)
        M.mla_out_proj(handle, ctx_lat, w["w_uv"], w.get("w_o"), o, u, B)
        assert M.mla_get_device_status(handle) == M.MLA_OK
        return {"o": to_host(o), "lse": to_host(lse), "u": to_host(u) if with_wo else None}
    finally:
        M.mla_destroy(handle)


def _chain_in_oracle(wl, seqs, heads, with_wo):
    w = draw_weights(wl, with_wo=with_wo)
    qw = draw_query_weights(wl)
    ctx = ctx_lengths(wl)
    base = rope_arg(wl)
    kw = dict(n_h=wl.n_h, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, base=base)
    out = {"o": {}, "o_explicit": {}, "lse": {}, "u": {}}
    for b in seqs:
        n = int(ctx[b])
        hb = hidden_states(wl, b, n)
        rows = O.cache_rows(hb, w["w_dkv"], w["w_kr"], np.arange(n), base)
        qc, qr = O.query_from_hidden(hb[-1], qw, wl.n_h, wl.d_h, wl.d_r)
        res = O.mla_decode_absorbed(qc, qr, n - 1, rows, w["w_uk"], w["w_uv"], w_o=w.get("w_o"), **kw)
        out["o"][b], out["lse"][b], out["u"][b] = res["o"], res["lse"], res["u"]
        out["o_explicit"][b] = O.mla_decode_explicit(qc, qr, n - 1, rows, w["w_uk"], w["w_uv"],
                                                     heads=heads, **kw)[0]
    return out


@pytest.mark.parametrize("name,B,seqs,heads,with_wo", [
    ("tiny_fp32", 2, [0, 1], [0, 1, 2, 3], True),           # the whole workload, W^O too
    ("v2_b64_ctx8k", 4, [0, 3], [0, 77, 127], False),        # DeepSeek-V2 shapes, ctx 8192
])
def test_decode_step_from_hidden_state(name, B, seqs, heads, with_wo):
    wl = WORKLOADS[name]
    if B != wl.B:
        wl = wl.with_(B=B, ctx=wl.ctx[:B])
    got = _chain_on_gpu(wl, with_wo)
    want = _chain_in_oracle(wl, seqs, heads, with_wo)
    compare(got["o"], want["o"], wl, "o (absorbed oracle, every head)", seqs)
    compare({b: got["o"][b][heads] for b in seqs}, want["o_explicit"], wl,
            "o (explicit per-head keys and values)", seqs)
    compare(got["lse"], want["lse"], wl, "lse", seqs)
    if with_wo:
        compare(got["u"], want["u"], wl, "u", seqs)
