"""GPU parity with YaRN long-context scaling of the rotary part ("DeepSeek-V2"
§3.2.4; the "DeepSeek-V3" note's context extension: s = 40, alpha = 1,
beta = 32, sqrt(t) = c ln s + 1), set through mla_set_rope_scaling, against
the oracle's RopeSpec on the same seeded inputs: full decode steps (cache
append, absorption, attention, combine, output projection)."""

import numpy as np
import pytest
import torch

from tests.gpu_harness import oracle_step, run_decode_step, compare
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu

V2_YARN = (40.0, 4096, 1.0, 32.0, 0.0707)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from head_latent_attention_09_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _check(wl, seqs, explicit_heads=None):
    got = run_decode_step(wl)
    want = oracle_step(wl, seqs, explicit_heads=explicit_heads)
    for key in ("cache_new_rows", "q_abs", "ctx_lat", "lse", "o"):
        compare(got[key], want[key], wl, key, seqs)
    if explicit_heads is not None:
        g = {b: got["o"][b][list(explicit_heads)] for b in seqs}
        compare(g, want["o_explicit"], wl, "o (explicit per-head keys)", seqs)


@pytest.mark.parametrize("coef", [0.0707, 0.1])
def test_tiny_fp32_with_yarn(coef):
    # a 16-token "original window" puts the tiny rotary pairs on both sides of the ramp
    wl = WORKLOADS["tiny_fp32"].with_(rope_scaling=(40.0, 16, 1.0, 32.0, coef))
    _check(wl, [0, 1], explicit_heads=range(wl.n_h))


def test_v2lite_long_context_with_v2_yarn():
    wl = WORKLOADS["v2lite_b32_ctx4k"].with_(B=2, ctx=(16384, 9001), rope_scaling=V2_YARN)
    _check(wl, [0, 1], explicit_heads=[0, 7])


def test_v2_pair_kernel_with_v2_yarn():
    wl = WORKLOADS["v2_b64_ctx8k"].with_(B=2, ctx=(8192, 3001), rope_scaling=V2_YARN)
    _check(wl, [0, 1], explicit_heads=[0, 77])


def test_scaling_factor_one_restores_plain_rope():
    import head_latent_attention_09_b200 as M
    from tests.gpu_harness import config_of
    wl = WORKLOADS["tiny_fp32"]
    h = M.mla_create(config_of(wl))
    try:
        M.mla_set_rope_scaling(h, 40.0, 16, 1.0, 32.0, 0.1)
        M.mla_set_rope_scaling(h, 1.0, 16, 1.0, 32.0, 0.1)
        with pytest.raises(M.MlaError):
            M.mla_set_rope_scaling(h, 0.5, 16, 1.0, 32.0, 0.1)
    finally:
        M.mla_destroy(h)
    got = run_decode_step(wl.with_(rope_scaling=(1.0, 16, 1.0, 32.0, 0.1)))
    want = oracle_step(wl, [0, 1])
    compare(got["ctx_lat"], want["ctx_lat"], wl, "ctx_lat", [0, 1])
    compare(got["q_abs"], want["q_abs"], wl, "q_abs", [0, 1])
