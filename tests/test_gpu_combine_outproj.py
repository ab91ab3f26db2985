"""GPU parity of mla_combine_out_proj: the split combine fused with the output
projection ("DeepSeek-V2" Appendix C, W^UV applied after the softmax-weighted
sum of latents), run on the same workspace as the two-call path
(mla_combine_splits, then mla_out_proj).

* ctx_lat and lse, when asked for, equal mla_combine_splits' bit for bit (the
  merge is the same arithmetic in the same order).
* o equals the oracle's within the spec's tolerances, and mla_out_proj's
  within one bf16 rounding (the fused kernel sums the 512-long products in one
  accumulator, the two-call path in two K halves).
* Leaving ctx_lat and lse out changes nothing in o.
* Shapes: tiles of 16, 32 and 64 sequences, a batch past one tile with a
  ragged last tile, empty and one-token contexts, a paged cache, W^O, and the
  fp32 workload (CUDA-core kernel).  bf16 runs in strict tensor-core mode.
"""

import numpy as np
import pytest
import torch

from tests.gpu_harness import compare, oracle_step, run_decode_step
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from head_latent_attention_09_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _bf16_ulp(x):
    """One unit in the last place of bfloat16 at |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def _check_fused(wl, got, seqs, with_wo=False):
    # merged latents and log-sum-exps: identical to the combine's
    assert np.array_equal(got["fused_ctx_lat"], got["ctx_lat"]), "ctx_lat differs from mla_combine_splits"
    same_lse = (got["fused_lse"] == got["lse"]) | (np.isneginf(got["fused_lse"]) & np.isneginf(got["lse"]))
    assert same_lse.all(), "lse differs from mla_combine_splits"
    # leaving ctx_lat / lse out does not change o
    assert np.array_equal(got["fused_o_bare"], got["fused_o"]), "o depends on whether ctx_lat is written"
    # o against the two-call path
    if wl.dtype == "bf16":
        d = np.abs(got["fused_o"] - got["o"])
        lim = 2 * _bf16_ulp(got["o"]) + 1e-6
        assert np.all(d <= lim), f"o: {int((d > lim).sum())} elements differ by more than two bf16 ulps"
    else:
        scale = max(float(np.abs(got["o"]).max()), 1e-30)
        assert float(np.abs(got["fused_o"] - got["o"]).max()) <= 1e-6 * scale
    # o (and u) against the oracle
    want = oracle_step(wl, seqs, with_wo=with_wo)
    compare(got["fused_o"], want["o"], wl, "o (fused)", seqs)
    compare(got["fused_ctx_lat"], want["ctx_lat"], wl, "ctx_lat (fused)", seqs)
    if with_wo:
        compare(got["fused_u"], want["u"], wl, "u (fused)", seqs)


def test_fused_tiny_fp32():
    wl = WORKLOADS["tiny_fp32"]
    got = run_decode_step(wl, with_wo=True, fused=True)
    _check_fused(wl, got, [0, 1], with_wo=True)


def test_fused_v2_b64_ctx8k():
    wl = WORKLOADS["v2_b64_ctx8k"]
    got = run_decode_step(wl, fused=True)
    _check_fused(wl, got, [0, 37, 63])


def test_fused_v2lite_b32_ctx4k():
    wl = WORKLOADS["v2lite_b32_ctx4k"]
    got = run_decode_step(wl, fused=True)
    _check_fused(wl, got, [0, 13, 31])


@pytest.mark.parametrize("name,ctx", [
    ("v2_b64_ctx8k", (1, 63, 64, 65, 200, 0, 129)),                  # 16-sequence tile, empty row
    ("v2lite_b32_ctx4k", (1, 2, 64, 100, 0, 1000, 4097)),
    ("v2_b64_ctx8k", tuple(int(x) for x in (np.arange(70) * 37 % 700))),  # 64 + ragged 6, ctx 0 too
    ("v2_b64_ctx8k", tuple(range(1, 25))),                           # 32-sequence tile
])
def test_fused_small_ragged(name, ctx):
    wl = WORKLOADS[name].with_(B=len(ctx), ctx=ctx)
    got = run_decode_step(wl, with_wo=True, fused=True)
    seqs = [b for b in range(wl.B) if ctx[b] > 0][:6]
    _check_fused(wl, got, seqs, with_wo=True)
    for b in range(wl.B):
        if ctx[b] == 0:
            assert np.all(got["fused_o"][b] == 0) and np.all(np.isneginf(got["fused_lse"][b]))


def test_fused_paged():
    wl = WORKLOADS["v2lite_paged_ragged_b128"].with_(B=6, ctx=(1, 64, 65, 300, 1, 130))
    got = run_decode_step(wl, fused=True)
    _check_fused(wl, got, list(range(6)))


@pytest.mark.parametrize("parts", [1, 3, 300])
def test_fused_split_counts(parts):
    wl = WORKLOADS["v2lite_b32_ctx4k"].with_(B=5, ctx=(4096, 1, 700, 2048, 3000))
    got = run_decode_step(wl, num_parts=parts, fused=True)
    _check_fused(wl, got, [0, 2, 4])
