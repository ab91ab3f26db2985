"""CPU oracle for decode-time Multi-head Latent Attention (MLA).

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  The CUDA library never
calls it, and it shares no code with the CUDA library.

Everything is plain NumPy in float64.  Each function follows the equations of
the pages, written out directly:

* "DeepSeek-V3 Technical Report" reading note (dogely.com), section on MLA:
  c^KV_t = W^DKV h_t;  k^C_t = W^UK c^KV_t;  k^R_t = RoPE(W^KR h_t);
  k_{t,i} = [k^C_{t,i}; k^R_t];  v^C_t = W^UV c^KV_t;
  c^Q_t = W^DQ h_t;  q^C_t = W^UQ c^Q_t;  q^R_t = RoPE(W^QR c^Q_t);
  q_{t,i} = [q^C_{t,i}; q^R_{t,i}];
  o_{t,i} = sum_{j=1..t} Softmax_j(q_{t,i}^T k_{j,i} / sqrt(d_h + d_h^R)) v^C_{j,i};
  u_t = W^O [o_{t,1}; ...; o_{t,n_h}].
* "DeepSeek-V2: Strong, Economical, Efficient" (Chinese translation,
  wiki.maxwellmou.com), §2.1.2 (only c^KV is cached), §2.1.3 (decoupled RoPE:
  a shared k^R_t of width d_h^R is cached too, so a token costs
  (d_c + d_h^R) elements per layer), Appendix B (V2-Lite computes the query
  directly from h_t), Appendix C (W^UK can be absorbed into the query side and
  W^UV into the output side by associativity).

Readings of points the pages leave open:

* RoPE follows the RoFormer form the pages cite (Su et al.): consecutive pairs
  (x_{2k}, x_{2k+1}) rotated by angle p * theta_k, theta_k = base^(-2k/d_h^R),
  base 10000, rotation [[cos, -sin], [sin, cos]].
* The query of a decode step sits at position ctx-1 and its own key is in the
  cache, so the softmax runs over positions 0 .. ctx-1 (the sum over j = 1..t).
* ctx = 0 yields a zero output and log-sum-exp = -inf.
* The log-sum-exp reported with an output is over the scaled scores
  s_j = q^T k_j / sqrt(d_h + d_h^R), in natural-log units.
* Long-context RoPE scaling ("DeepSeek-V2", §3.2.4; the "DeepSeek-V3" note's
  context-extension section) names YaRN (Peng et al.) with s = 40, alpha = 1,
  beta = 32 over a 4K original window, applied to the decoupled rotary part,
  and a length-scaling factor sqrt(t) = c ln s + 1 with c = 0.0707 in the V2
  paper and c = 0.1 in the V3 note.  Reading: YaRN's per-frequency ramp (a
  pair that turns more than beta times over the original window keeps its
  frequency, one that turns fewer than alpha times is slowed by s, linear in
  between), and sqrt(t) scaling both the query and the key, i.e. every score
  (content and rotary part) multiplied by t = (c ln s + 1)^2; c is a
  parameter, 0.0707 by default.  s = 1 is plain RoPE.  (YaRN itself writes
  its logit temperature the same way: the square root of the factor on the
  logits is 0.1 ln s + 1, applied as a scale on both q and k, so the logits
  carry its square.)
* FP8 latent cache ("DeepSeek-V2" §3.2.3 quantises the deployed KV cache to
  about 6 bits per element without giving the format; the "DeepSeek-V3" note's
  FP8 section quantises activations tile-wise, per token and per 128 channels,
  with the group's absolute maximum setting the scale).  Reading: each cached
  row is cut into 128-channel groups, over c^KV and separately over k^R; a
  group's scale is sigma = amax / 448 and its elements are stored as OCP FP8
  E4M3 codes of x / sigma (round to nearest even, saturating at 448), both
  divisions in float32, which is also where the GPU takes these decisions.  A
  group of zeros has sigma = 0 and zero codes.  The stored value is
  code * sigma.

Parity pins: every function below is pinned by tests/test_oracle_pins.py
(closed forms, invariants, brute force, the pages' printed cache sizes).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

F64 = np.float64


# ----------------------------------------------------------------------------
# RoPE (decoupled part only)
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class RopeSpec:
    """RoPE frequencies with optional YaRN scaling.  Every function that takes
    ``base`` accepts either a plain base (float) or a RopeSpec."""
    base: float = 10000.0
    factor: float = 1.0          # s: context-extension ratio (1 = plain RoPE)
    original_ctx: int = 4096     # the window the frequencies were trained on
    alpha: float = 1.0           # below alpha turns over the window: fully slowed by s
    beta: float = 32.0           # above beta turns: unchanged
    mscale_coef: float = 0.0707  # c in sqrt(t) = c ln s + 1


def _spec(base) -> RopeSpec:
    return base if isinstance(base, RopeSpec) else RopeSpec(base=float(base))


def rope_theta(d_r: int, base) -> np.ndarray:
    """Rotation frequency of each pair k = 0 .. d_r/2 - 1.

    Plain RoPE (RoFormer): theta_k = base^(-2k/d_r).  With YaRN (s > 1): the
    pair turns r_k = L / (2 pi / theta_k) times over the original window L;
    gamma_k = clip((r_k - alpha) / (beta - alpha), 0, 1) blends the slowed
    frequency theta_k / s (gamma = 0) with the original one (gamma = 1)."""
    spec = _spec(base)
    k = np.arange(d_r // 2, dtype=F64)
    theta = np.power(F64(spec.base), -2.0 * k / F64(d_r))
    if spec.factor <= 1.0:
        return theta
    turns = F64(spec.original_ctx) * theta / (2.0 * math.pi)
    gamma = np.clip((turns - spec.alpha) / (spec.beta - spec.alpha), 0.0, 1.0)
    return (1.0 - gamma) * theta / F64(spec.factor) + gamma * theta


def attention_temperature(base) -> float:
    """Multiplier t of every score: (c ln s + 1)^2 with YaRN (sqrt(t) scales
    both the query and the key), 1 for plain RoPE."""
    spec = _spec(base)
    if spec.factor <= 1.0:
        return 1.0
    m = spec.mscale_coef * math.log(spec.factor) + 1.0
    return m * m


def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate consecutive pairs of the last axis of ``x`` by pos * theta_k.

    ``pos`` is a scalar or an array broadcastable to x.shape[:-1]; ``base``
    is a plain base or a RopeSpec.
    """
    x = np.asarray(x, dtype=F64)
    d_r = x.shape[-1]
    assert d_r % 2 == 0
    theta = rope_theta(d_r, base)
    ang = np.asarray(pos, dtype=F64)[..., None] * theta          # [..., d_r/2]
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (d_r,)), dtype=F64)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# ----------------------------------------------------------------------------
# cache (what a token leaves behind)
# ----------------------------------------------------------------------------

def cache_rows(h: np.ndarray, w_dkv: np.ndarray, w_kr: np.ndarray, positions,
               base: float) -> np.ndarray:
    """Cached row of each token: [c^KV_t ; k^R_t] with c^KV_t = W^DKV h_t and
    k^R_t = RoPE(W^KR h_t) at the token's position.  h: [T, d] -> [T, d_c + d_r]."""
    h = np.asarray(h, dtype=F64)
    c = h @ np.asarray(w_dkv, dtype=F64).T
    kr = rope(h @ np.asarray(w_kr, dtype=F64).T, np.asarray(positions), base)
    return np.concatenate([c, kr], axis=-1)


def kv_cache_elements_per_token(kind: str, *, n_h: int, d_h: int, layers: int = 1,
                                n_g: int = 0, d_c: int = 0, d_r: int = 0) -> int:
    """Per-token KV-cache size in elements for the mechanisms the pages compare
    (V2 paper §2.1.4, Table 1): MHA 2 n_h d_h l, GQA 2 n_g d_h l, MQA 2 d_h l,
    MLA (d_c + d_h^R) l."""
    if kind == "MHA":
        return 2 * n_h * d_h * layers
    if kind == "GQA":
        return 2 * n_g * d_h * layers
    if kind == "MQA":
        return 2 * d_h * layers
    if kind == "MLA":
        return (d_c + d_r) * layers
    raise ValueError(kind)


# ----------------------------------------------------------------------------
# FP8 (E4M3) latent cache: per-token, per-128-channel-group scales
# ----------------------------------------------------------------------------

E4M3_MAX = 448.0
FP8_GROUP = 128


def e4m3_decode(codes) -> np.ndarray:
    """Value of each OCP FP8 E4M3 code (float64): sign bit, four exponent bits
    with bias 7, three mantissa bits; exponent field 0 holds the subnormals
    m * 2^-9; S.1111.111 is NaN and there are no infinities."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(F64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2((e - 7).astype(F64)))
    mag = np.where((e == 15) & (c & 7 == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(v) -> np.ndarray:
    """E4M3 code of each value (uint8): round to nearest, ties to even, finite
    values beyond 448 saturate to +-448.  ``v`` is taken as float32."""
    x = np.asarray(v, dtype=np.float32).astype(F64)
    sign = np.signbit(x)
    a = np.abs(x)
    # spacing of representable magnitudes around a: 2^(e-3) in the binade
    # [2^e, 2^(e+1)) for e >= -6, and 2^-9 below 2^-6 (subnormals)
    e = np.frexp(np.where(a > 0, a, 1.0))[1] - 1
    e = np.maximum(e, -6)
    quantum = np.exp2((e - 3).astype(F64))
    mag = np.rint(a / quantum) * quantum            # exact scaling; rint is half-to-even
    mag = np.minimum(mag, E4M3_MAX)
    sub = mag < 2.0 ** -6
    ef = np.frexp(np.where(sub, 1.0, mag))[1] - 1   # binade of a normal result
    mant = np.where(sub, mag / 2.0 ** -9, mag / np.exp2(ef.astype(F64)) * 8.0 - 8.0)
    efield = np.where(sub, 0, ef + 7)
    code = (sign.astype(np.int64) << 7) | (efield.astype(np.int64) << 3) | np.rint(mant).astype(np.int64)
    return code.astype(np.uint8)


def fp8_groups(d_c: int, d_r: int):
    """Channel ranges [a, b) of a cached row's scale groups: 128-wide groups
    over c^KV, then over k^R (the last group of each part may be narrower)."""
    g = [(a, min(a + FP8_GROUP, d_c)) for a in range(0, d_c, FP8_GROUP)]
    g += [(d_c + a, d_c + min(a + FP8_GROUP, d_r)) for a in range(0, d_r, FP8_GROUP)]
    return g


def quantize_rows_fp8(rows, d_c: int, d_r: int):
    """Quantise cached rows [n, d_c + d_r]: per row and group, sigma = amax / 448
    and codes E4M3(x / sigma), with x, the maximum and both divisions in float32.
    Returns (codes uint8 [n, d_c + d_r], scales float32 [n, groups])."""
    x = np.asarray(rows, dtype=np.float32)
    x = x.reshape(-1, d_c + d_r)
    groups = fp8_groups(d_c, d_r)
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.zeros((x.shape[0], len(groups)), dtype=np.float32)
    for gi, (a, b) in enumerate(groups):
        blk = x[:, a:b]
        amax = np.max(np.abs(blk), axis=1)
        sigma = (amax / np.float32(E4M3_MAX)).astype(np.float32)
        nz = sigma > 0
        q = blk[nz] / sigma[nz][:, None]
        codes[nz, a:b] = e4m3_encode(q.astype(np.float32))
        scales[:, gi] = sigma
    return codes, scales


def dequantize_rows_fp8(codes, scales, d_c: int, d_r: int) -> np.ndarray:
    """Stored values of FP8 rows: code * sigma of the element's group (float64)."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, d_c + d_r)
    sc = np.asarray(scales, dtype=np.float32).reshape(c.shape[0], -1).astype(F64)
    out = e4m3_decode(c)
    for gi, (a, b) in enumerate(fp8_groups(d_c, d_r)):
        out[:, a:b] *= sc[:, gi:gi + 1]
    return out


# ----------------------------------------------------------------------------
# query (upstream of the decode boundary; used by oracle-only cross-checks)
# ----------------------------------------------------------------------------

def query_from_hidden(h_q: np.ndarray, qw: dict, n_h: int, d_h: int, d_r: int):
    """q^C and q^R before rotation for one token, shapes [n_h, d_h], [n_h, d_r].

    With query compression: c^Q = W^DQ h, q^C = W^UQ c^Q, q^R_raw = W^QR c^Q.
    Without (V2-Lite, Appendix B): q^C = W^Q h, q^R_raw = W^QR h."""
    h_q = np.asarray(h_q, dtype=F64)
    if "w_dq" in qw:
        cq = np.asarray(qw["w_dq"], F64) @ h_q
        qc = np.asarray(qw["w_uq"], F64) @ cq
        qr = np.asarray(qw["w_qr"], F64) @ cq
    else:
        qc = np.asarray(qw["w_q"], F64) @ h_q
        qr = np.asarray(qw["w_qr"], F64) @ h_q
    return qc.reshape(n_h, d_h), qr.reshape(n_h, d_r)


# ----------------------------------------------------------------------------
# explicit (textbook) attention: per-head keys and values are materialised
# ----------------------------------------------------------------------------

def explicit_keys_values(rows: np.ndarray, w_uk: np.ndarray, w_uv: np.ndarray,
                         n_h: int, d_h: int, d_c: int, heads=None):
    """k_{j,i} = [W^UK_i c_j ; k^R_j] and v_{j,i} = W^UV_i c_j, where W^UK_i is
    rows i*d_h .. (i+1)*d_h of W^UK.  rows: [S, d_c + d_r].
    Returns k [h, S, d_h + d_r], v [h, S, d_h] for the selected heads."""
    rows = np.asarray(rows, dtype=F64)
    c, kr = rows[:, :d_c], rows[:, d_c:]
    heads = range(n_h) if heads is None else heads
    ks, vs = [], []
    for i in heads:
        wk = np.asarray(w_uk[i * d_h:(i + 1) * d_h], dtype=F64)     # [d_h, d_c]
        wv = np.asarray(w_uv[i * d_h:(i + 1) * d_h], dtype=F64)
        ks.append(np.concatenate([c @ wk.T, kr], axis=1))
        vs.append(c @ wv.T)
    return np.stack(ks), np.stack(vs)


def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Textbook attention for one query per head.  q [h, e], k [h, S, e],
    v [h, S, f] -> (o [h, f], lse [h]); lse is log sum_j exp(scale q.k_j)."""
    q, k, v = (np.asarray(a, dtype=F64) for a in (q, k, v))
    S = k.shape[1]
    if S == 0:
        return np.zeros((q.shape[0], v.shape[2])), np.full(q.shape[0], -np.inf)
    s = np.einsum("he,hse->hs", q, k) * F64(scale)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    o = np.einsum("hs,hsf->hf", p / l, v)
    return o, (m + np.log(l))[:, 0]


def softmax_scale(d_h: int, d_r: int) -> float:
    """1 / sqrt(d_h + d_h^R): the scores divide by the root of the full
    (content + rotary) query/key width."""
    return 1.0 / math.sqrt(d_h + d_r)


def attention_scale(d_h: int, d_r: int, base) -> float:
    """The factor every score q . k is multiplied by: the softmax scale times
    the YaRN temperature (1 for plain RoPE)."""
    return softmax_scale(d_h, d_r) * attention_temperature(base)


def mla_decode_explicit(q_nope, q_rope_raw, pos: int, rows, w_uk, w_uv, *, n_h, d_h, d_c,
                        d_r, base, heads=None):
    """One decode step for one sequence in the explicit form.
    q_nope [n_h, d_h], q_rope_raw [n_h, d_r] (before RoPE), rows [S, d_c+d_r].
    Returns (o [h, d_h], lse [h]) for the selected heads."""
    heads = list(range(n_h)) if heads is None else list(heads)
    qr = rope(np.asarray(q_rope_raw, F64)[heads], pos, base)
    q = np.concatenate([np.asarray(q_nope, F64)[heads], qr], axis=1)
    k, v = explicit_keys_values(rows, w_uk, w_uv, n_h, d_h, d_c, heads)
    return softmax_attention(q, k, v, attention_scale(d_h, d_r, base))


# ----------------------------------------------------------------------------
# absorbed form (Appendix C): attention runs on the cached rows directly
# ----------------------------------------------------------------------------

def absorb_query(q_nope, q_rope_raw, pos: int, w_uk, *, n_h, d_h, d_r, base) -> np.ndarray:
    """q_abs_i = [W^UK_i^T q^C_i ; RoPE(q^R_i, pos)]  -> [n_h, d_c + d_r].
    Then q_abs_i . [c_j ; k^R_j] = q^C_i . (W^UK_i c_j) + q^R_i . k^R_j."""
    q_nope = np.asarray(q_nope, F64)
    out = []
    for i in range(n_h):
        wk = np.asarray(w_uk[i * d_h:(i + 1) * d_h], F64)           # [d_h, d_c]
        out.append(wk.T @ q_nope[i])
    lat = np.stack(out)
    return np.concatenate([lat, rope(np.asarray(q_rope_raw, F64), pos, base)], axis=1)


def latent_attention(q_abs, rows, *, d_c: int, scale: float):
    """Softmax over the latent rows: ctx_lat_i = sum_j p_ij c_j with
    p_ij = softmax_j(scale q_abs_i . row_j).  Returns (ctx_lat [h, d_c], lse [h])."""
    q_abs, rows = np.asarray(q_abs, F64), np.asarray(rows, F64)
    if rows.shape[0] == 0:
        return np.zeros((q_abs.shape[0], d_c)), np.full(q_abs.shape[0], -np.inf)
    s = (q_abs @ rows.T) * F64(scale)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    return (p / l) @ rows[:, :d_c], (m + np.log(l))[:, 0]


def out_project(ctx_lat, w_uv, *, n_h, d_h, w_o=None):
    """o_i = W^UV_i ctx_lat_i (W^UV absorbed to the output side), and optionally
    u = W^O [o_1; ...; o_{n_h}]."""
    ctx_lat = np.asarray(ctx_lat, F64)
    o = np.stack([np.asarray(w_uv[i * d_h:(i + 1) * d_h], F64) @ ctx_lat[i]
                  for i in range(n_h)])
    if w_o is None:
        return o, None
    return o, np.asarray(w_o, F64) @ o.reshape(-1)


def mla_decode_absorbed(q_nope, q_rope_raw, pos, rows, w_uk, w_uv, *, n_h, d_h, d_c, d_r,
                        base, w_o=None):
    """Full absorbed decode step for one sequence: returns dict with q_abs,
    ctx_lat, lse, o (and u when W^O is given)."""
    q_abs = absorb_query(q_nope, q_rope_raw, pos, w_uk, n_h=n_h, d_h=d_h, d_r=d_r, base=base)
    ctx_lat, lse = latent_attention(q_abs, rows, d_c=d_c, scale=attention_scale(d_h, d_r, base))
    o, u = out_project(ctx_lat, w_uv, n_h=n_h, d_h=d_h, w_o=w_o)
    return {"q_abs": q_abs, "ctx_lat": ctx_lat, "lse": lse, "o": o, "u": u}


# ----------------------------------------------------------------------------
# split-KV partials and their log-sum-exp merge
# ----------------------------------------------------------------------------

def split_partials(q_abs, rows, bounds, *, d_c: int, scale: float):
    """Attention over each token range [a, b) of ``bounds`` separately:
    list of (ctx_lat_part [h, d_c], lse_part [h])."""
    return [latent_attention(q_abs, np.asarray(rows)[a:b], d_c=d_c, scale=scale)
            for a, b in bounds]


def combine_partials(parts):
    """Merge per-range results: with m = max_s lse_s and w_s = exp(lse_s - m),
    ctx = sum_s w_s ctx_s / sum_s w_s and lse = m + log sum_s w_s.  Ranges with
    lse = -inf carry no weight; if all are -inf the result is 0 and -inf."""
    lses = np.stack([p[1] for p in parts])                      # [S, h]
    outs = np.stack([p[0] for p in parts])                      # [S, h, d]
    m = lses.max(axis=0)
    finite = np.isfinite(m)
    msafe = np.where(finite, m, 0.0)
    w = np.where(np.isfinite(lses), np.exp(lses - msafe), 0.0)
    tot = w.sum(axis=0)
    ctx = np.einsum("sh,shd->hd", w, outs) / np.where(tot > 0, tot, 1.0)[:, None]
    lse = np.where(finite, msafe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return np.where(finite[:, None], ctx, 0.0), lse


# ----------------------------------------------------------------------------
# brute force (pure Python loops) for tiny inputs
# ----------------------------------------------------------------------------

def brute_force_decode(h_seq, q_nope, q_rope_raw, w: dict, *, n_h, d_h, d_c, d_r, base):
    """Scalar-loop decode step for one sequence from its hidden states:
    builds every cached row, every per-head key/value, and the softmax, one
    multiply-add at a time.  Returns (o as nested lists [n_h][d_h], lse list [n_h])."""
    S = len(h_seq)
    d = len(h_seq[0])
    # Frequencies and score scale again, one pair at a time (a second reading
    # of the same definitions as rope_theta / attention_scale): a pair that
    # turns at least beta times over the original window keeps theta, at most
    # alpha times gets theta / s, and in between the linear blend.
    spec = _spec(base)
    theta = []
    for p in range(d_r // 2):
        th = spec.base ** (-2.0 * p / d_r)
        if spec.factor > 1.0:
            turns = spec.original_ctx * th / (2.0 * math.pi)
            if turns >= spec.beta:
                frac = 1.0
            elif turns <= spec.alpha:
                frac = 0.0
            else:
                frac = (turns - spec.alpha) / (spec.beta - spec.alpha)
            th = frac * th + (1.0 - frac) * th / spec.factor
        theta.append(th)
    scale = 1.0 / math.sqrt(d_h + d_r)
    if spec.factor > 1.0:
        scale *= (spec.mscale_coef * math.log(spec.factor) + 1.0) ** 2
    rows = []
    for t in range(S):
        c = [sum(float(w["w_dkv"][r][k]) * float(h_seq[t][k]) for k in range(d))
             for r in range(d_c)]
        kr_raw = [sum(float(w["w_kr"][r][k]) * float(h_seq[t][k]) for k in range(d))
                  for r in range(d_r)]
        kr = [0.0] * d_r
        for p in range(d_r // 2):
            a = t * theta[p]
            kr[2 * p] = kr_raw[2 * p] * math.cos(a) - kr_raw[2 * p + 1] * math.sin(a)
            kr[2 * p + 1] = kr_raw[2 * p] * math.sin(a) + kr_raw[2 * p + 1] * math.cos(a)
        rows.append((c, kr))
    pos = S - 1
    out, lses = [], []
    for i in range(n_h):
        qr = [0.0] * d_r
        for p in range(d_r // 2):
            a = pos * theta[p]
            x0, x1 = float(q_rope_raw[i][2 * p]), float(q_rope_raw[i][2 * p + 1])
            qr[2 * p] = x0 * math.cos(a) - x1 * math.sin(a)
            qr[2 * p + 1] = x0 * math.sin(a) + x1 * math.cos(a)
        scores, vals = [], []
        for t in range(S):
            c, kr = rows[t]
            kc = [sum(float(w["w_uk"][i * d_h + r][k]) * c[k] for k in range(d_c))
                  for r in range(d_h)]
            vc = [sum(float(w["w_uv"][i * d_h + r][k]) * c[k] for k in range(d_c))
                  for r in range(d_h)]
            dot = sum(float(q_nope[i][r]) * kc[r] for r in range(d_h))
            dot += sum(qr[r] * kr[r] for r in range(d_r))
            scores.append(dot * scale)
            vals.append(vc)
        mx = max(scores)
        e = [math.exp(s - mx) for s in scores]
        z = sum(e)
        out.append([sum(e[t] * vals[t][r] for t in range(S)) / z for r in range(d_h)])
        lses.append(mx + math.log(z))
    return out, lses
