"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- values the pages print, closed forms, invariants of the
mathematics, brute force on tiny inputs -- so that a dropped term, a wrong sign
or index, or a transposed operand fails at least one of them."""

import math
import os

import numpy as np
import pytest

from oracle import mla_oracle as O
from workloads import WORKLOADS, draw_query_weights, draw_weights, hidden_states, queries

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TINY = WORKLOADS["tiny_fp32"]


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, val = line.split()[:2]
                out[key] = float(val)
    return out


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# --------------------------------------------------------------------------
# cache size: the pages print it
# --------------------------------------------------------------------------

def test_cache_size_matches_pages():
    g = _golden("kv_cache_per_token.txt")
    n_h, d_h, d_c, d_r = (int(g[k]) for k in ("v2_n_h", "v2_d_h", "v2_d_c", "v2_d_r"))
    assert d_c == g["d_c_per_d_h"] * d_h
    assert d_r == g["d_r_per_d_h"] * d_h
    mla = O.kv_cache_elements_per_token("MLA", n_h=n_h, d_h=d_h, d_c=d_c, d_r=d_r)
    assert mla == g["mla_per_d_h"] * d_h == 576
    gqa = O.kv_cache_elements_per_token("GQA", n_h=n_h, d_h=d_h, n_g=1)
    assert mla / gqa == g["mla_gqa_groups"]
    mha = O.kv_cache_elements_per_token("MHA", n_h=n_h, d_h=d_h, layers=int(g["v2_layers"]))
    assert O.kv_cache_elements_per_token("MLA", n_h=n_h, d_h=d_h, d_c=d_c, d_r=d_r,
                                         layers=int(g["v2_layers"])) / mha == 576 / 32768
    assert O.kv_cache_elements_per_token("MQA", n_h=n_h, d_h=d_h) == 2 * d_h
    # the oracle's cached row has exactly d_c + d_h^R entries
    rng = np.random.default_rng(0)
    d = 64
    rows = O.cache_rows(rng.standard_normal((3, d)), rng.standard_normal((d_c, d)),
                        rng.standard_normal((d_r, d)), np.arange(3), 10000.0)
    assert rows.shape == (3, mla)
    # V2-Lite shares the per-token row width
    assert int(g["lite_d_c"]) + int(g["lite_d_r"]) == mla


# --------------------------------------------------------------------------
# RoPE: hand values of the RoFormer rotation, and its invariants
# --------------------------------------------------------------------------

def test_rope_hand_values():
    # d = 2: one pair, theta_0 = 1.  Position 1 rotates by one radian.
    assert np.allclose(O.rope([1.0, 0.0], 1, 10000.0), [math.cos(1), math.sin(1)], atol=1e-15)
    assert np.allclose(O.rope([0.0, 1.0], 1, 10000.0), [-math.sin(1), math.cos(1)], atol=1e-15)
    # d = 4, base 10000: theta_1 = 10000^(-1/2) = 0.01, so position 100 turns pair 1 by 1 rad
    # and pair 0 by 100 rad.
    x = O.rope([1.0, 0.0, 1.0, 0.0], 100, 10000.0)
    assert np.allclose(x, [math.cos(100), math.sin(100), math.cos(1), math.sin(1)], atol=1e-13)
    # position 0 is the identity
    v = np.arange(16.0)
    assert np.array_equal(O.rope(v, 0, 10000.0), v)


def test_rope_preserves_norm():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((50, 64))
    pos = rng.integers(0, 131072, size=50)
    y = O.rope(x, pos, 10000.0)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in [(0, 5), (17, 3), (131071, 130000)]:
        ref = O.rope(q, m, 10000.0) @ O.rope(k, n, 10000.0)
        for delta in (1, 977, 4096):
            got = O.rope(q, m + delta, 10000.0) @ O.rope(k, n + delta, 10000.0)
            assert abs(got - ref) <= 1e-9 * max(1.0, abs(ref))


# --------------------------------------------------------------------------
# absorbed form == explicit form (associativity), and why RoPE is decoupled
# --------------------------------------------------------------------------

def _tiny_inputs(seed=0, S=23):
    wl = TINY
    rng = np.random.default_rng(seed)
    w = draw_weights(wl)
    rows = rng.standard_normal((S, wl.D))
    qn = rng.standard_normal((wl.n_h, wl.d_h))
    qr = rng.standard_normal((wl.n_h, wl.d_r))
    return wl, w, rows, qn, qr


def test_absorbed_equals_explicit():
    wl, w, rows, qn, qr = _tiny_inputs()
    kw = dict(n_h=wl.n_h, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, base=wl.rope_base)
    o_e, lse_e = O.mla_decode_explicit(qn, qr, 22, rows, w["w_uk"], w["w_uv"], **kw)
    res = O.mla_decode_absorbed(qn, qr, 22, rows, w["w_uk"], w["w_uv"], **kw)
    assert _rel(res["o"], o_e) <= 1e-12
    assert np.allclose(res["lse"], lse_e, rtol=1e-13, atol=1e-13)


def test_absorption_fails_if_rope_touches_content_keys():
    """Rotating k^C (coupled RoPE) puts a position-dependent matrix between
    W^Q and W^UK, so the absorbed form no longer matches: the oracle's
    absorbed form must notice the difference."""
    wl, w, rows, qn, qr = _tiny_inputs(seed=3)
    d_h, d_c = wl.d_h, wl.d_c
    S = rows.shape[0]
    k_exp, v_exp = O.explicit_keys_values(rows, w["w_uk"], w["w_uv"], wl.n_h, d_h, d_c)
    k_coupled = k_exp.copy()
    k_coupled[:, :, :d_h] = O.rope(k_exp[:, :, :d_h], np.arange(S)[None, :], wl.rope_base)
    q = np.concatenate([qn, O.rope(qr, S - 1, wl.rope_base)], axis=1)
    o_coupled, _ = O.softmax_attention(q, k_coupled, v_exp, O.softmax_scale(d_h, wl.d_r))
    res = O.mla_decode_absorbed(qn, qr, S - 1, rows, w["w_uk"], w["w_uv"], n_h=wl.n_h, d_h=d_h,
                                d_c=d_c, d_r=wl.d_r, base=wl.rope_base)
    assert _rel(res["o"], o_coupled) > 1e-3


# --------------------------------------------------------------------------
# closed forms of the softmax and its scale
# --------------------------------------------------------------------------

def _one_head_setup(d_h=32, d_c=128, d_r=16):
    """W^UK_0 = W^UV_0 = [I_{d_h} 0] so that the per-head key/value of a row
    are its first d_h latent entries."""
    w_uk = np.zeros((d_h, d_c))
    w_uk[:, :d_h] = np.eye(d_h)
    return w_uk, w_uk.copy()


def test_two_token_softmax_closed_form():
    """Scores that differ by ln(3) give weights 3/4 and 1/4 -- the scale must be
    1/sqrt(d_h + d_h^R)."""
    d_h, d_c, d_r = 32, 128, 16
    w_uk, w_uv = _one_head_setup(d_h, d_c, d_r)
    gap = math.log(3.0) * math.sqrt(d_h + d_r)      # raw dot-product difference
    rows = np.zeros((2, d_c + d_r))
    rows[0, 0] = gap            # key 0 content: e_0 * gap
    rows[0, 1] = 5.0            # value 0: 5 in coordinate 1
    rows[1, 2] = -7.0           # value 1: -7 in coordinate 2, score 0
    qn = np.zeros((1, d_h))
    qn[0, 0] = 1.0
    qr = np.zeros((1, d_r))
    o, lse = O.mla_decode_explicit(qn, qr, 1, rows, w_uk, w_uv, n_h=1, d_h=d_h, d_c=d_c,
                                   d_r=d_r, base=10000.0)
    assert np.isclose(o[0, 0], 0.75 * gap, rtol=1e-14)
    assert np.isclose(o[0, 1], 0.75 * 5.0, rtol=1e-14)
    assert np.isclose(o[0, 2], 0.25 * -7.0, rtol=1e-14)
    # lse = log(e^{ln 3} + e^0) = log 4
    assert np.isclose(lse[0], math.log(4.0), rtol=1e-14)


def test_rope_part_enters_scores():
    """Only the decoupled parts differ: q^R = k^R_0 rotated to the same place
    gives score |k^R|^2 / sqrt(d_h + d_r) for key 0 and 0 for key 1."""
    d_h, d_c, d_r = 32, 128, 16
    w_uk, w_uv = _one_head_setup(d_h, d_c, d_r)
    rows = np.zeros((2, d_c + d_r))
    kr = np.zeros(d_r)
    kr[0] = math.sqrt(math.log(3.0) * math.sqrt(d_h + d_r))   # |k^R|^2 = ln3 sqrt(48)
    rows[0, d_c:] = O.rope(kr, 0, 10000.0)
    rows[0, 1], rows[1, 1] = 1.0, 0.0
    # query at position 1 whose rotated q^R equals kr rotated by 0: pre-rotate by -1
    qr = O.rope(kr, -1, 10000.0)[None, :]
    qn = np.zeros((1, d_h))
    o, _ = O.mla_decode_explicit(qn, qr, 1, rows, w_uk, w_uv, n_h=1, d_h=d_h, d_c=d_c, d_r=d_r,
                                 base=10000.0)
    assert np.isclose(o[0, 1], 0.75, rtol=1e-12)


def test_ctx1_constant_and_zero_query():
    wl, w, rows, qn, qr = _tiny_inputs(seed=5, S=9)
    kw = dict(n_h=wl.n_h, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, base=wl.rope_base)
    wuv = w["w_uv"].astype(np.float64)
    per_head = lambda c: np.stack([wuv[i * wl.d_h:(i + 1) * wl.d_h] @ c for i in range(wl.n_h)])
    # ctx = 1: the only value is returned
    o, lse = O.mla_decode_explicit(qn, qr, 0, rows[:1], w["w_uk"], w["w_uv"], **kw)
    assert _rel(o, per_head(rows[0, :wl.d_c])) <= 1e-13
    # all rows equal: softmax weights are uniform, output is that value; lse = s + log S
    same = np.repeat(rows[:1], 9, axis=0)
    o, lse = O.mla_decode_explicit(qn, qr, 8, same, w["w_uk"], w["w_uv"], **kw)
    assert _rel(o, per_head(rows[0, :wl.d_c])) <= 1e-13
    # q = 0: uniform weights -> mean of the values, lse = log S
    o, lse = O.mla_decode_explicit(np.zeros_like(qn), np.zeros_like(qr), 8, rows, w["w_uk"],
                                   w["w_uv"], **kw)
    assert _rel(o, per_head(rows[:, :wl.d_c].mean(axis=0))) <= 1e-13
    assert np.allclose(lse, math.log(9), rtol=1e-14)


def test_dominant_key_wins():
    d_h, d_c, d_r = 32, 128, 16
    w_uk, w_uv = _one_head_setup(d_h, d_c, d_r)
    rng = np.random.default_rng(9)
    rows = rng.standard_normal((40, d_c + d_r)) * 0.1
    rows[13, 0] = 400.0
    qn = np.zeros((1, d_h))
    qn[0, 0] = 1.0
    o, _ = O.mla_decode_explicit(qn, np.zeros((1, d_r)), 39, rows, w_uk, w_uv, n_h=1, d_h=d_h,
                                 d_c=d_c, d_r=d_r, base=10000.0)
    assert np.allclose(o[0], rows[13, :d_h], atol=1e-12)


def test_empty_context():
    wl, w, rows, qn, qr = _tiny_inputs()
    q_abs = O.absorb_query(qn, qr, 0, w["w_uk"], n_h=wl.n_h, d_h=wl.d_h, d_r=wl.d_r,
                           base=wl.rope_base)
    ctx, lse = O.latent_attention(q_abs, rows[:0], d_c=wl.d_c, scale=0.1)
    assert np.all(ctx == 0) and np.all(np.isneginf(lse))


# --------------------------------------------------------------------------
# split-KV: any partition merged by log-sum-exp equals one pass
# --------------------------------------------------------------------------

@pytest.mark.parametrize("cuts", [(0, 64), (0, 1, 64), (0, 10, 11, 40, 64), (0, 0, 30, 30, 64)])
def test_split_combine_is_exact(cuts):
    rng = np.random.default_rng(11)
    H, d_c, d_r = 4, 128, 16
    rows = rng.standard_normal((64, d_c + d_r))
    q_abs = rng.standard_normal((H, d_c + d_r))
    scale = O.softmax_scale(32, d_r)
    full_ctx, full_lse = O.latent_attention(q_abs, rows, d_c=d_c, scale=scale)
    parts = O.split_partials(q_abs, rows, list(zip(cuts[:-1], cuts[1:])), d_c=d_c, scale=scale)
    ctx, lse = O.combine_partials(parts)
    assert _rel(ctx, full_ctx) <= 1e-13
    assert np.allclose(lse, full_lse, rtol=1e-14)


def test_combine_all_empty():
    parts = [(np.zeros((2, 8)), np.full(2, -np.inf))] * 3
    ctx, lse = O.combine_partials(parts)
    assert np.all(ctx == 0) and np.all(np.isneginf(lse))


# --------------------------------------------------------------------------
# brute force on the tiny workload, from hidden states to outputs
# --------------------------------------------------------------------------

@pytest.mark.parametrize("b", [0, 1])
def test_brute_force_tiny_workload(b):
    wl = TINY
    w = draw_weights(wl)
    ctx = wl.ctx[b]
    h = hidden_states(wl, b, ctx)
    qn, qr = queries(wl)
    kw = dict(n_h=wl.n_h, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, base=wl.rope_base)
    rows = O.cache_rows(h, w["w_dkv"], w["w_kr"], np.arange(ctx), wl.rope_base)
    res = O.mla_decode_absorbed(qn[b], qr[b], ctx - 1, rows, w["w_uk"], w["w_uv"], **kw)
    o_ex, lse_ex = O.mla_decode_explicit(qn[b], qr[b], ctx - 1, rows, w["w_uk"], w["w_uv"], **kw)
    bf_o, bf_lse = O.brute_force_decode(h.tolist(), qn[b].tolist(), qr[b].tolist(),
                                        {k: v.tolist() for k, v in w.items()}, **kw)
    assert _rel(res["o"], bf_o) <= 1e-12
    assert _rel(o_ex, bf_o) <= 1e-12
    assert np.allclose(res["lse"], bf_lse, rtol=1e-12)


def test_full_equations_with_query_compression():
    """From h through c^Q, q^C, q^R (V3 note equations) to o: explicit and
    absorbed agree, and u = W^O [o_1; ...; o_n] is the per-element sum."""
    wl = TINY
    w = draw_weights(wl, with_wo=True)
    qw = draw_query_weights(wl)
    ctx = wl.ctx[1]
    h = hidden_states(wl, 1, ctx)
    qc, qr = O.query_from_hidden(h[-1], qw, wl.n_h, wl.d_h, wl.d_r)
    # c^Q path by hand for one element
    cq = np.asarray(qw["w_dq"], np.float64) @ h[-1].astype(np.float64)
    assert np.isclose(qc[2, 5], np.asarray(qw["w_uq"], np.float64)[2 * wl.d_h + 5] @ cq)
    rows = O.cache_rows(h, w["w_dkv"], w["w_kr"], np.arange(ctx), wl.rope_base)
    kw = dict(n_h=wl.n_h, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, base=wl.rope_base)
    res = O.mla_decode_absorbed(qc, qr, ctx - 1, rows, w["w_uk"], w["w_uv"], w_o=w["w_o"], **kw)
    o_ex, _ = O.mla_decode_explicit(qc, qr, ctx - 1, rows, w["w_uk"], w["w_uv"], **kw)
    assert _rel(res["o"], o_ex) <= 1e-12
    wo = np.asarray(w["w_o"], np.float64)
    flat = res["o"].reshape(-1)
    for j in (0, 77, wl.d_model - 1):
        assert np.isclose(res["u"][j], sum(wo[j, k] * flat[k] for k in range(flat.size)),
                          rtol=1e-12)


def test_cache_rows_by_hand():
    """One cached row element by element: c = W^DKV h, k^R = RoPE(W^KR h, p)."""
    rng = np.random.default_rng(4)
    d, d_c, d_r, p = 12, 6, 4, 7
    h = rng.standard_normal((1, d))
    wd, wk = rng.standard_normal((d_c, d)), rng.standard_normal((d_r, d))
    row = O.cache_rows(h, wd, wk, [p], 10000.0)[0]
    assert np.allclose(row[:d_c], [sum(wd[r, k] * h[0, k] for k in range(d)) for r in range(d_c)])
    raw = [sum(wk[r, k] * h[0, k] for k in range(d)) for r in range(d_r)]
    a0, a1 = p * 1.0, p * 10000.0 ** (-0.5)
    want = [raw[0] * math.cos(a0) - raw[1] * math.sin(a0), raw[0] * math.sin(a0) + raw[1] * math.cos(a0),
            raw[2] * math.cos(a1) - raw[3] * math.sin(a1), raw[2] * math.sin(a1) + raw[3] * math.cos(a1)]
    assert np.allclose(row[d_c:], want, atol=1e-13)


# --------------------------------------------------------------------------
# YaRN long-context scaling of the rotary part ("DeepSeek-V2" §3.2.4; the
# "DeepSeek-V3" note's context extension): s = 40, alpha = 1, beta = 32 over a
# 4K window, sqrt(t) = c ln s + 1
# --------------------------------------------------------------------------

V2_YARN = O.RopeSpec(base=10000.0, factor=40.0, original_ctx=4096, alpha=1.0, beta=32.0,
                     mscale_coef=0.0707)


def test_yarn_with_factor_one_is_plain_rope():
    spec = O.RopeSpec(base=10000.0, factor=1.0)
    assert np.array_equal(O.rope_theta(64, spec), O.rope_theta(64, 10000.0))
    assert O.attention_temperature(spec) == 1.0
    x = np.random.default_rng(3).standard_normal((5, 64))
    assert np.array_equal(O.rope(x, 777, spec), O.rope(x, 777, 10000.0))


def test_yarn_keeps_fast_pairs_and_slows_slow_pairs_by_s():
    d_r = 64
    plain = O.rope_theta(d_r, 10000.0)
    ratio = O.rope_theta(d_r, V2_YARN) / plain
    # turns of each pair over the original 4096-token window
    turns = 4096 * plain / (2 * math.pi)
    assert turns[0] > 32 and turns[-1] < 1                      # both regimes occur at d_r = 64
    assert np.all(ratio[turns >= 32] == 1.0)                    # fast pairs unchanged
    assert np.allclose(ratio[turns <= 1], 1 / 40.0, rtol=1e-15) # slow pairs slowed by s
    mid = (turns > 1) & (turns < 32)
    assert mid.any() and np.all((ratio[mid] > 1 / 40.0) & (ratio[mid] < 1.0))
    assert np.all(np.diff(ratio) <= 1e-15)                      # never faster for slower pairs


def test_yarn_rope_keeps_norm_and_relative_position():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((20, 64))
    pos = rng.integers(0, 163840, size=20)
    y = O.rope(x, pos, V2_YARN)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    ref = O.rope(q, 131071, V2_YARN) @ O.rope(k, 5, V2_YARN)
    got = O.rope(q, 131071 - 5, V2_YARN) @ O.rope(k, 0, V2_YARN)
    assert abs(got - ref) <= 1e-9 * max(1.0, abs(ref))


def test_yarn_temperature_acts_as_a_query_scale():
    # Every score is multiplied by t, so the step equals a plain-temperature
    # step (same frequencies) on the query scaled by t.
    wl, w, rows, qn, qr = _tiny_inputs(seed=5)
    kw = dict(n_h=wl.n_h, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r)
    spec = O.RopeSpec(base=wl.rope_base, factor=40.0, original_ctx=16, alpha=1.0, beta=32.0,
                      mscale_coef=0.0707)
    t = O.attention_temperature(spec)
    assert t > 1.0
    assert O.attention_temperature(O.RopeSpec(factor=40.0, mscale_coef=0.1)) > t
    res = O.mla_decode_absorbed(qn, qr, 22, rows, w["w_uk"], w["w_uv"], base=spec, **kw)
    q_abs = O.absorb_query(qn, qr, 22, w["w_uk"], n_h=wl.n_h, d_h=wl.d_h, d_r=wl.d_r, base=spec)
    ctx, lse = O.latent_attention(q_abs * t, rows, d_c=wl.d_c, scale=O.softmax_scale(wl.d_h, wl.d_r))
    assert _rel(res["ctx_lat"], ctx) <= 1e-13
    assert np.allclose(res["lse"], lse, rtol=1e-13)


def test_yarn_temperature_matches_page_values():
    # sqrt(t) = c ln s + 1 with the pages' s and c, squared by hand
    # (tests/golden/yarn_scaling.txt): t multiplies every score.
    g = _golden("yarn_scaling.txt")
    for coef, want in ((g["v2_coef"], g["v2_t"]), (g["v3_coef"], g["v3_t"])):
        spec = O.RopeSpec(base=10000.0, factor=g["yarn_s"], original_ctx=int(g["yarn_window"]),
                          alpha=g["yarn_alpha"], beta=g["yarn_beta"], mscale_coef=coef)
        assert abs(O.attention_temperature(spec) - want) <= 1e-14 * want
    assert abs(g["v2_sqrt_t"] ** 2 - g["v2_t"]) <= 1e-14 and abs(g["v3_sqrt_t"] ** 2 - g["v3_t"]) <= 1e-14


@pytest.mark.parametrize("which", ["v2", "v3"])
def test_yarn_two_token_softmax_closed_form(which):
    # Two cached tokens whose content keys give raw scores differing by delta,
    # no rotary signal: the decode step must weight them p0 / p1 =
    # exp(t delta / sqrt(d_h + d_h^R)) with the hand-computed t of the pages'
    # sqrt(t) = c ln s + 1.
    g = _golden("yarn_scaling.txt")
    spec = O.RopeSpec(base=10000.0, factor=g["yarn_s"], original_ctx=int(g["yarn_window"]),
                      alpha=g["yarn_alpha"], beta=g["yarn_beta"], mscale_coef=g[which + "_coef"])
    t = g[which + "_t"]
    n_h, d_h, d_c, d_r = 1, 2, 2, 2
    w_uk = np.eye(2)                       # k^C = c
    w_uv = np.eye(2)                       # o = ctx_lat
    rows = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 1.0, 0.0, 0.0]])
    qn = np.array([[1.3, -0.4]])           # raw scores 1.3 and -0.4
    qr = np.zeros((1, 2))
    res = O.mla_decode_absorbed(qn, qr, 1, rows, w_uk, w_uv, n_h=n_h, d_h=d_h, d_c=d_c, d_r=d_r,
                                base=spec)
    delta = 1.3 - (-0.4)
    k = t * delta / math.sqrt(d_h + d_r)
    p0 = 1.0 / (1.0 + math.exp(-k))
    assert np.allclose(res["o"][0], [p0, 1.0 - p0], rtol=0, atol=1e-14)
    lse = t * 1.3 / math.sqrt(d_h + d_r) + math.log(1.0 + math.exp(-k))
    assert abs(res["lse"][0] - lse) <= 1e-13


def test_yarn_interior_ramp_hand_values():
    # Frequencies of pairs that turn between alpha and beta times over the
    # trained window: YaRN's ramp is linear in the number of turns, values
    # worked out by hand in tests/golden/yarn_scaling.txt.
    g = _golden("yarn_scaling.txt")
    spec = O.RopeSpec(base=10000.0, factor=g["yarn_s"], original_ctx=int(g["yarn_window"]),
                      alpha=g["yarn_alpha"], beta=g["yarn_beta"], mscale_coef=g["v2_coef"])
    theta = O.rope_theta(64, spec)
    for k in (12, 16, 20):
        want = g[f"yarn_theta_k{k}"]
        assert abs(theta[k] - want) <= 1e-13 * want, (k, theta[k], want)


@pytest.mark.parametrize("coef", [0.0707, 0.1])
def test_yarn_absorbed_explicit_and_brute_force_agree(coef):
    wl = TINY
    w = draw_weights(wl)
    b, ctx = 1, wl.ctx[1]
    h = hidden_states(wl, b, ctx)
    qn, qr = queries(wl)
    spec = O.RopeSpec(base=wl.rope_base, factor=40.0, original_ctx=16, alpha=1.0, beta=32.0,
                      mscale_coef=coef)
    assert not np.array_equal(O.rope_theta(wl.d_r, spec), O.rope_theta(wl.d_r, wl.rope_base))
    kw = dict(n_h=wl.n_h, d_h=wl.d_h, d_c=wl.d_c, d_r=wl.d_r, base=spec)
    rows = O.cache_rows(h, w["w_dkv"], w["w_kr"], np.arange(ctx), spec)
    res = O.mla_decode_absorbed(qn[b], qr[b], ctx - 1, rows, w["w_uk"], w["w_uv"], **kw)
    o_ex, lse_ex = O.mla_decode_explicit(qn[b], qr[b], ctx - 1, rows, w["w_uk"], w["w_uv"], **kw)
    bf_o, bf_lse = O.brute_force_decode(h.tolist(), qn[b].tolist(), qr[b].tolist(),
                                        {k: v.tolist() for k, v in w.items()}, **kw)
    assert _rel(res["o"], bf_o) <= 1e-12
    assert _rel(o_ex, bf_o) <= 1e-12
    assert np.allclose(res["lse"], bf_lse, rtol=1e-12)


# --------------------------------------------------------------------------
# FP8 (E4M3) latent cache
# --------------------------------------------------------------------------

def _torch_e4m3():
    torch = pytest.importorskip("torch")
    return torch, torch.float8_e4m3fn


def test_e4m3_decode_matches_library_for_every_code():
    torch, f8 = _torch_e4m3()
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(f8).float().numpy().astype(np.float64)
    mine = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    assert np.isnan(mine).sum() == 2                      # S.1111.111 only; no infinities
    fin = ~np.isnan(ref)
    assert np.array_equal(mine[fin], ref[fin])


def test_e4m3_format_values():
    # the format's defining values: largest finite 448 = 0.1111.110, 1 = 0.0111.000,
    # smallest normal 2^-6 = 0.0001.000, smallest subnormal 2^-9 = 0.0000.001
    enc = lambda x: int(O.e4m3_encode(np.float32(x)))
    assert enc(448.0) == 0x7E and enc(-448.0) == 0xFE
    assert enc(1.0) == 0x38 and enc(-2.0) == 0xC0
    assert enc(2.0 ** -6) == 0x08 and enc(2.0 ** -9) == 0x01
    assert enc(0.0) == 0x00 and enc(2.0 ** -11) == 0x00   # below half the smallest subnormal
    # finite values past the largest code saturate
    assert all(enc(x) == 0x7E for x in (449.0, 463.9, 464.0, 1e4, 3e38))


def test_e4m3_encode_matches_library_rounding():
    torch, f8 = _torch_e4m3()
    rng = np.random.default_rng(7)
    finite = O.e4m3_decode(np.arange(256, dtype=np.uint8))
    finite = finite[~np.isnan(finite)]
    pos = np.unique(finite[finite > 0])
    mids = (pos[:-1] + pos[1:]) / 2                        # ties: must go to the even code
    near = np.concatenate([np.nextafter(mids.astype(np.float32), np.float32(0)),
                           np.nextafter(mids.astype(np.float32), np.float32(1e9))])
    v = np.concatenate([finite, mids, -mids, near, rng.uniform(-448, 448, 20000),
                        rng.uniform(-0.03, 0.03, 20000), rng.standard_normal(20000)]).astype(np.float32)
    ref = torch.from_numpy(v.copy()).to(f8).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(v), ref)


def test_e4m3_encode_brute_force_nearest():
    # exhaustive nearest-code search over the finite codes, ties to the even mantissa
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    rng = np.random.default_rng(3)
    xs = np.concatenate([rng.uniform(-460, 460, 300), rng.uniform(-0.02, 0.02, 300)]).astype(np.float32)
    for x in xs:
        xv = float(x)
        if abs(xv) >= 448.0:
            want = 0x7E | (0x80 if xv < 0 else 0)
        else:
            d = [abs(xv - float(v)) for v in vals]
            best = min(d)
            cand = [int(codes[i]) for i in range(len(codes)) if d[i] == best]
            if len(cand) > 1:
                cand = [c for c in cand if c & 1 == 0] or cand
                # +0 and -0 tie at zero: the sign of x decides
                cand = [c for c in cand if (c & 0x80) == (0x80 if np.signbit(x) else 0)] or cand
            want = cand[0]
        assert int(O.e4m3_encode(x)) == want, (xv, hex(int(O.e4m3_encode(x))), hex(want))


def test_fp8_groups_of_the_cached_row():
    # V2 shapes: four 128-channel groups over c^KV and one over the 64-wide k^R
    assert O.fp8_groups(512, 64) == [(0, 128), (128, 256), (256, 384), (384, 512), (512, 576)]
    assert O.fp8_groups(128, 16) == [(0, 128), (128, 144)]
    assert O.fp8_groups(200, 16) == [(0, 128), (128, 200), (200, 216)]


def test_fp8_quantize_rows_invariants():
    rng = np.random.default_rng(11)
    d_c, d_r = 512, 64
    rows = rng.standard_normal((40, d_c + d_r)).astype(np.float32)
    rows[3, :128] = 0.0                                      # an all-zero group
    rows[5, 200] = 300.0                                     # an outlier confined to its group
    rows[7, 512:] *= 1e-3                                    # a small rotary group
    codes, sc = O.quantize_rows_fp8(rows, d_c, d_r)
    assert codes.dtype == np.uint8 and codes.shape == rows.shape and sc.shape == (40, 5)
    deq = O.dequantize_rows_fp8(codes, sc, d_c, d_r)
    for gi, (a, b) in enumerate(O.fp8_groups(d_c, d_r)):
        blk = rows[:, a:b].astype(np.float64)
        amax = np.abs(blk).max(axis=1)
        # scale = amax / 448 in float32
        assert np.array_equal(sc[:, gi], (np.abs(rows[:, a:b]).max(axis=1) / np.float32(448)).astype(np.float32))
        # the group's largest element is stored as +-448 sigma, i.e. amax itself
        k = np.abs(blk).argmax(axis=1)
        got = np.abs(deq[np.arange(40), a + k])
        assert np.allclose(got, amax, rtol=2 ** -22, atol=0)
        # error bound from the format's spacing: half a step, 2^-4 relative for
        # normals, 2^-10 sigma for subnormals
        err = np.abs(deq[:, a:b] - blk)
        bound = 2.0 ** -4 * np.abs(blk) + 2.0 ** -10 * sc[:, gi:gi + 1].astype(np.float64)
        assert np.all(err <= bound * (1 + 1e-6))
    assert np.all(codes[3, :128] == 0) and sc[3, 0] == 0.0
    # the outlier's group alone carries a large scale
    assert sc[5, 1] > 100 * np.median(sc[:, 1]) and sc[5, 0] < 2 * np.median(sc[:, 0])


def test_fp8_quantize_is_scale_invariant_under_powers_of_two():
    # multiplying a row by 2^k is exact in float32: same codes, scales times 2^k
    rng = np.random.default_rng(5)
    rows = rng.standard_normal((16, 144)).astype(np.float32)
    c0, s0 = O.quantize_rows_fp8(rows, 128, 16)
    for k in (-20, -3, 5, 30):
        ck, sk = O.quantize_rows_fp8(rows * np.float32(2.0 ** k), 128, 16)
        assert np.array_equal(ck, c0)
        assert np.array_equal(sk, (s0 * np.float32(2.0 ** k)).astype(np.float32))
