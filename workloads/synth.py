"""Workload shapes and seeded generators.

Shapes follow the pages: DeepSeek-V2 attention (n_h = 128, d_h = 128,
d_c = 512, d'_c = 1536, d_h^R = 64, d = 5120; "DeepSeek-V2: Strong,
Economical, Efficient", §3.2.1 model hyper-parameters) and DeepSeek-V2-Lite
(16 heads, d = 2048, no query compression; same paper, Appendix B).  Every
weight is drawn from N(0, 1/fan_in), hidden states from N(0, 1).

Random streams are independent children of one ``SeedSequence(seed)`` so a
caller can draw one group (for example the hidden states of a single
sequence) without drawing the others:

    child 0   key/value weights  W_DKV, W_KR, W_UK, W_UV, [W_O]
    child 1   query weights      W_DQ, W_UQ, W_QR  or  W_Q, W_QR
    child 2   context lengths, then the block permutation of the paged pool
    child 3   query inputs       q^C (q_nope) and q^R before RoPE (q_rope)
    child 4   directly drawn latent caches (attention-only tests)
    child 5+b hidden states of sequence b, positions 0 .. ctx_b - 1

Nothing here computes any part of attention.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np

_N_FIXED_CHILDREN = 5


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    n_h: int
    d_h: int
    d_c: int
    d_r: int
    d_model: int
    dtype: str                      # "fp32" or "bf16": storage and input precision
    seed: int
    ctx: tuple = ()                 # fixed per-sequence context lengths, or () for drawn ones
    ctx_loguniform: tuple = ()      # (lo, hi) for log-uniform lengths
    d_cq: int | None = None         # query compression width d'_c, None = no query compression
    page_size: int = 0              # 0 = contiguous cache, else tokens per block
    rope_base: float = 10000.0
    # YaRN long-context scaling of the rotary part, passed through unchanged to
    # the library and the oracle: (factor s, original window, alpha, beta,
    # coefficient c of sqrt(t) = c ln s + 1); None = plain RoPE.
    rope_scaling: tuple | None = None
    note: str = field(default="", compare=False)

    @property
    def D(self) -> int:
        """Cached elements per token per layer: d_c + d_h^R."""
        return self.d_c + self.d_r

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload(
        name="tiny_fp32", B=2, n_h=4, d_h=32, d_c=128, d_r=16, d_model=256, dtype="fp32",
        seed=0, ctx=(17, 64), d_cq=96,
        note="tiny fp32 MLA decode, one layer, ragged contexts 17 and 64"),
    "v2lite_b32_ctx4k": Workload(
        name="v2lite_b32_ctx4k", B=32, n_h=16, d_h=128, d_c=512, d_r=64, d_model=2048,
        dtype="bf16", seed=1, ctx=(4096,) * 32,
        note="DeepSeek-V2-Lite shapes, contiguous cache [32, 4096, 576]"),
    "v2_b64_ctx8k": Workload(
        name="v2_b64_ctx8k", B=64, n_h=128, d_h=128, d_c=512, d_r=64, d_model=5120,
        dtype="bf16", seed=2, ctx=(8192,) * 64, d_cq=1536,
        note="DeepSeek-V2 shapes, contiguous cache [64, 8192, 576]"),
    "v2lite_paged_ragged_b128": Workload(
        name="v2lite_paged_ragged_b128", B=128, n_h=16, d_h=128, d_c=512, d_r=64,
        d_model=2048, dtype="bf16", seed=3, ctx_loguniform=(256, 32768), page_size=64,
        note="V2-Lite shapes, 128 log-uniform contexts in [256, 32768], 64-token pages"),
    "v2lite_b4_ctx128k": Workload(
        name="v2lite_b4_ctx128k", B=4, n_h=16, d_h=128, d_c=512, d_r=64, d_model=2048,
        dtype="bf16", seed=4, ctx=(131072,) * 4,
        note="V2-Lite shapes, 128K contexts, contiguous cache [4, 131072, 576]"),
}


# ----------------------------------------------------------------------------
# precision helpers (input quantisation only)
# ----------------------------------------------------------------------------

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even) and
    return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 array whose values are exactly the bfloat16 roundings of ``x``."""
    return (bf16_bits(x).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _store(wl: Workload, x: np.ndarray) -> np.ndarray:
    x = x.astype(np.float32, copy=False)
    return bf16_round(x) if wl.dtype == "bf16" else x


def _child_rng(wl: Workload, idx: int) -> np.random.Generator:
    # SeedSequence.spawn is deterministic in the index, so spawning up to idx is enough.
    return np.random.default_rng(np.random.SeedSequence(wl.seed).spawn(idx + 1)[idx])


def _normal(rng, shape, std) -> np.ndarray:
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(std))


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------

def draw_weights(wl: Workload, with_wo: bool = False) -> dict:
    """Key/value-side weights, row-major [out, in], N(0, 1/fan_in).

    W_DKV [d_c, d], W_KR [d_h^R, d], W_UK [n_h d_h, d_c], W_UV [n_h d_h, d_c],
    optionally W_O [d, n_h d_h].
    """
    rng = _child_rng(wl, 0)
    d, dc, dr, H, dh = wl.d_model, wl.d_c, wl.d_r, wl.n_h, wl.d_h
    w = {
        "w_dkv": _store(wl, _normal(rng, (dc, d), 1.0 / math.sqrt(d))),
        "w_kr": _store(wl, _normal(rng, (dr, d), 1.0 / math.sqrt(d))),
        "w_uk": _store(wl, _normal(rng, (H * dh, dc), 1.0 / math.sqrt(dc))),
        "w_uv": _store(wl, _normal(rng, (H * dh, dc), 1.0 / math.sqrt(dc))),
    }
    if with_wo:
        w["w_o"] = _store(wl, _normal(rng, (d, H * dh), 1.0 / math.sqrt(H * dh)))
    return w


def draw_query_weights(wl: Workload) -> dict:
    """Query-side weights.  With query compression (d'_c given): W_DQ [d'_c, d],
    W_UQ [n_h d_h, d'_c], W_QR [n_h d_h^R, d'_c].  Without (V2-Lite):
    W_Q [n_h d_h, d], W_QR [n_h d_h^R, d]."""
    rng = _child_rng(wl, 1)
    d, H, dh, dr = wl.d_model, wl.n_h, wl.d_h, wl.d_r
    if wl.d_cq:
        cq = wl.d_cq
        return {
            "w_dq": _store(wl, _normal(rng, (cq, d), 1.0 / math.sqrt(d))),
            "w_uq": _store(wl, _normal(rng, (H * dh, cq), 1.0 / math.sqrt(cq))),
            "w_qr": _store(wl, _normal(rng, (H * dr, cq), 1.0 / math.sqrt(cq))),
        }
    return {
        "w_q": _store(wl, _normal(rng, (H * dh, d), 1.0 / math.sqrt(d))),
        "w_qr": _store(wl, _normal(rng, (H * dr, d), 1.0 / math.sqrt(d))),
    }


def ctx_lengths(wl: Workload) -> np.ndarray:
    """Per-sequence context lengths (int64 [B]); the query sits at ctx-1."""
    if wl.ctx:
        assert len(wl.ctx) == wl.B, "fixed ctx tuple must have B entries"
        return np.asarray(wl.ctx, dtype=np.int64)
    lo, hi = wl.ctx_loguniform
    rng = _child_rng(wl, 2)
    u = rng.uniform(math.log(lo), math.log(hi), size=wl.B)
    return np.clip(np.floor(np.exp(u)), lo, hi).astype(np.int64)


def block_table(wl: Workload, ctx: np.ndarray):
    """Random-permutation placement of each sequence's 64-token blocks in a pool
    of sum(ceil(ctx/page)) blocks.  Returns (table int32 [B, max_blocks],
    num_blocks); unused entries are -1."""
    ps = wl.page_size
    assert ps > 0
    nblk = (ctx + ps - 1) // ps
    pool = int(nblk.sum())
    rng = _child_rng(wl, 2)
    rng.uniform(size=wl.B)          # skip the context-length draws of the same stream
    perm = rng.permutation(pool).astype(np.int32)
    max_blk = int(nblk.max()) if wl.B else 0
    table = np.full((wl.B, max(max_blk, 1)), -1, dtype=np.int32)
    off = 0
    for b in range(wl.B):
        n = int(nblk[b])
        table[b, :n] = perm[off:off + n]
        off += n
    return table, pool


def hidden_states(wl: Workload, b: int, n_tokens: int) -> np.ndarray:
    """Attention inputs h_t of sequence b for positions 0 .. n_tokens-1
    (float32 [n_tokens, d], rounded to the storage precision)."""
    rng = _child_rng(wl, _N_FIXED_CHILDREN + b)
    return _store(wl, rng.standard_normal((n_tokens, wl.d_model), dtype=np.float32))


def queries(wl: Workload):
    """Query inputs at the boundary: q_nope = q^C [B, n_h, d_h] and q_rope =
    q^R before rotation [B, n_h, d_h^R].  Under N(0, 1/fan_in) projection
    weights both have unit variance, so they are drawn from N(0, 1)."""
    rng = _child_rng(wl, 3)
    q_nope = _store(wl, rng.standard_normal((wl.B, wl.n_h, wl.d_h), dtype=np.float32))
    q_rope = _store(wl, rng.standard_normal((wl.B, wl.n_h, wl.d_r), dtype=np.float32))
    return q_nope, q_rope


def random_cache(wl: Workload, n_tokens: int, std: float = 1.0) -> np.ndarray:
    """A latent cache drawn directly, [B, n_tokens, d_c + d_h^R], for tests of
    the attention step in isolation."""
    rng = _child_rng(wl, 4)
    return _store(wl, _normal(rng, (wl.B, n_tokens, wl.D), std))
