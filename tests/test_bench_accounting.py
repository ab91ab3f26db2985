"""The byte counts behind bench.py's roofline and throughput figures, against
hand counts from the shapes (DeepSeek-V2 and V2-Lite, bf16)."""

import bench
from workloads import WORKLOADS


def test_step_bytes_v2_b64_ctx8k():
    wl = WORKLOADS["v2_b64_ctx8k"]
    ctx_sum = 64 * 8192
    cache = ctx_sum * 576 * 2                               # 604.0 MB of latent rows
    weights = (576 * 5120 + 2 * 128 * 128 * 512) * 2        # W_DKV | W_KR, W_UK, W_UV
    assert cache == 603_979_776
    assert bench.algorithmic_bytes(wl, ctx_sum) == cache + weights
    assert bench.algorithmic_bytes(wl, ctx_sum, with_wo=True) == cache + weights + 5120 * 16384 * 2


def test_query_projection_bytes():
    v2 = WORKLOADS["v2_b64_ctx8k"]
    # W^DQ [1536, 5120], W^UQ [16384, 1536], W^QR [8192, 1536]; h read, c^Q written
    # and read by both up-projections, q^C and q^R written
    w = 1536 * 5120 + (16384 + 8192) * 1536
    act = 64 * 5120 + 3 * 64 * 1536 + 64 * (16384 + 8192)
    assert bench.query_proj_bytes(v2, 64) == 2 * (w + act) == 95_617_024
    lite = WORKLOADS["v2lite_b32_ctx4k"]                    # no query compression
    assert bench.query_proj_bytes(lite, 32) == 2 * ((2048 + 1024) * 2048 + 32 * 2048 + 32 * 3072)


def test_fp8_cache_bytes_per_token():
    # 576 E4M3 codes and five float32 group scales per token (596 B), against 1152 B in bf16
    tokens = 4 * 131072
    assert bench.fp8_cache_bytes(tokens, 576, 5) == tokens * 596 == 312_475_648
    assert bench.fp8_cache_bytes(1, 144, 2) == 152                  # the tiny shapes: d_c 128, d_r 16
