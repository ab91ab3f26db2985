"""GPU parity of mla_query_proj, the query projection from the hidden state.

It is checked against the oracle's query_from_hidden ("DeepSeek-V2" §2.1.2
query compression and §2.1.3 decoupled query; Appendix B for the form without
W^DQ), on the workloads' own query weights:

  - c_q against the fp64 c^Q = W^DQ h;
  - q_nope / q_rope against the oracle's up-projections of the c_q the GPU
    stored (this isolates the up-projection kernels from c_q's rounding);
  - q_nope / q_rope against the whole fp64 chain from h.

Tolerances (bf16 storage, fp32 accumulation):
  - one step: |got - want| <= 2^-8 |want| + 1e-5.  Rounding the output to bf16
    costs at most 2^-9 |want|; fp32 accumulation over K <= 5120 products of
    unit-scale terms stays below 1e-5.
  - whole chain: |got - want| <= 2^-8 |want| + 8e-3 and rel L2 <= 5e-3.
    c_q is rounded to bf16 (2^-9 relative, uniform), and the up-projection
    carries that into q as an absolute error of std ~ 2^-9 / sqrt(3) ~ 1.1e-3
    for unit-variance q.  8e-3 is seven standard deviations.
  - fp32 storage: the harness's fp32 bound (rel L2 and max abs / max |want|
    both <= 1e-5).
"""

import numpy as np
import pytest
import torch

import head_latent_attention_09_b200 as M
from oracle import mla_oracle as O
from tests.gpu_harness import create_handle, to_dev, to_host, torch_dtype, compare
from workloads import WORKLOADS
from workloads.synth import draw_query_weights, hidden_states

pytestmark = pytest.mark.gpu

STEP_RTOL, STEP_ATOL = 2.0 ** -8, 1e-5
CHAIN_RTOL, CHAIN_ATOL, CHAIN_REL_L2 = 2.0 ** -8, 8e-3, 5e-3


def _hidden(wl):
    """One new token per sequence: the last of b+1 drawn hidden states."""
    return np.stack([hidden_states(wl, b, b + 1)[-1] for b in range(wl.B)])


def _run(wl, x, qw, strict):
    handle = create_handle(wl, strict=strict)
    try:
        dt = torch_dtype(wl)
        w = {k: to_dev(v, wl) for k, v in qw.items()}
        x_d = to_dev(x, wl)
        q_nope = torch.empty((wl.B, wl.n_h, wl.d_h), dtype=dt, device="cuda")
        q_rope = torch.empty((wl.B, wl.n_h, wl.d_r), dtype=dt, device="cuda")
        if "w_dq" in w:
            c_q = torch.empty((wl.B, wl.d_cq), dtype=dt, device="cuda")
            M.mla_query_proj(handle, x_d, wl.B, w["w_dq"], wl.d_cq, w["w_uq"], w["w_qr"],
                             c_q, q_nope, q_rope)
        else:
            c_q = None
            M.mla_query_proj(handle, x_d, wl.B, None, 0, w["w_q"], w["w_qr"], None,
                             q_nope, q_rope)
        assert M.mla_get_device_status(handle) == M.MLA_OK
        return (to_host(c_q) if c_q is not None else None), to_host(q_nope), to_host(q_rope)
    finally:
        M.mla_destroy(handle)


def _close(got, want, rtol, atol, what):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    bound = rtol * np.abs(want) + atol
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), \
        f"{what}: |err| {err.flat[worst]:.3e} > {bound.flat[worst]:.3e} at flat index {worst}"
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))


def _check(wl, strict=None):
    qw = draw_query_weights(wl)
    x = _hidden(wl)
    c_q, q_nope, q_rope = _run(wl, x, qw, strict)
    H, dh, dr = wl.n_h, wl.d_h, wl.d_r
    chain = [O.query_from_hidden(x[b], qw, H, dh, dr) for b in range(wl.B)]
    if wl.dtype == "fp32":
        compare({b: q_nope[b] for b in range(wl.B)}, {b: c[0] for b, c in enumerate(chain)},
                wl, "q_nope")
        compare({b: q_rope[b] for b in range(wl.B)}, {b: c[1] for b, c in enumerate(chain)},
                wl, "q_rope")
        if c_q is not None:
            want = {b: np.asarray(qw["w_dq"], np.float64) @ x[b] for b in range(wl.B)}
            compare({b: c_q[b] for b in range(wl.B)}, want, wl, "c_q")
        return
    if c_q is not None:
        want_cq = np.stack([np.asarray(qw["w_dq"], np.float64) @ np.asarray(x[b], np.float64)
                            for b in range(wl.B)])
        _close(c_q, want_cq, STEP_RTOL, STEP_ATOL, "c_q")
        # the up-projections alone, from the c_q the GPU stored: the form without
        # W^DQ with W^Q := W^UQ applied to that c_q
        up = {"w_q": qw["w_uq"], "w_qr": qw["w_qr"]}
        step = [O.query_from_hidden(c_q[b], up, H, dh, dr) for b in range(wl.B)]
        _close(q_nope, np.stack([s[0] for s in step]), STEP_RTOL, STEP_ATOL, "q_nope (step)")
        _close(q_rope, np.stack([s[1] for s in step]), STEP_RTOL, STEP_ATOL, "q_rope (step)")
        rtol, atol = CHAIN_RTOL, CHAIN_ATOL
    else:
        rtol, atol = STEP_RTOL, STEP_ATOL
    for i, (name, got) in enumerate((("q_nope", q_nope), ("q_rope", q_rope))):
        rel = _close(got, np.stack([c[i] for c in chain]), rtol, atol, name)
        assert rel <= CHAIN_REL_L2, f"{name}: rel L2 {rel:.3e}"


@pytest.mark.parametrize("name,B,over", [
    ("tiny_fp32", 2, {}),                               # fp32: CUDA-core kernel, d'_c = 96
    ("tiny_fp32", 3, {"dtype": "bf16"}),                # bf16, W^DQ on tensor cores, K = 96 on CUDA cores
    ("v2_b64_ctx8k", 64, {}),                           # V2 shapes, full batch, tensor cores
    ("v2_b64_ctx8k", 5, {}),                            # ragged batch: 5 of a 16-wide tile
    ("v2lite_b32_ctx4k", 32, {}),                       # V2-Lite: W^Q, no query compression
    ("v2lite_b32_ctx4k", 7, {"d_model": 2000}),         # K % 64 != 0: CUDA-core fallback in bf16
])
def test_query_proj_matches_oracle(name, B, over):
    wl = WORKLOADS[name].with_(B=B, ctx=(1,) * B, **over)
    # the overridden shapes run (part of) the projection on CUDA cores by design
    _check(wl, strict=False if over else None)


def test_query_proj_empty_batch_and_bad_arguments():
    wl = WORKLOADS["v2_b64_ctx8k"].with_(B=2, ctx=(1, 1))
    handle = create_handle(wl)
    try:
        dt = torch_dtype(wl)
        x = torch.zeros((2, wl.d_model), dtype=dt, device="cuda")
        w_dq = torch.zeros((wl.d_cq, wl.d_model), dtype=dt, device="cuda")
        w_uq = torch.zeros((wl.n_h * wl.d_h, wl.d_cq), dtype=dt, device="cuda")
        w_qr = torch.zeros((wl.n_h * wl.d_r, wl.d_cq), dtype=dt, device="cuda")
        qn = torch.full((2, wl.n_h, wl.d_h), 7.0, dtype=dt, device="cuda")
        qr = torch.full((2, wl.n_h, wl.d_r), 7.0, dtype=dt, device="cuda")
        # B = 0 launches nothing and leaves the outputs alone
        M.mla_query_proj(handle, x, 0, w_dq, wl.d_cq, w_uq, w_qr, None, qn, qr)
        torch.cuda.synchronize()
        assert bool((qn == 7).all()) and bool((qr == 7).all())
        # W^DQ without a c_q buffer, or without a width
        with pytest.raises(M.MlaError):
            M.mla_query_proj(handle, x, 2, w_dq, wl.d_cq, w_uq, w_qr, None, qn, qr)
        cq = torch.empty((2, wl.d_cq), dtype=dt, device="cuda")
        with pytest.raises(M.MlaError):
            M.mla_query_proj(handle, x, 2, w_dq, 0, w_uq, w_qr, cq, qn, qr)
        with pytest.raises(M.MlaError):
            M.mla_query_proj(handle, x, 2, w_dq, wl.d_cq, w_uq, None, cq, qn, qr)
        assert M.mla_get_device_status(handle) == M.MLA_OK
    finally:
        M.mla_destroy(handle)
