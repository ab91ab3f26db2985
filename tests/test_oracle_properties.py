"""Randomised forms of three of the oracle's pins, over drawn shapes,
positions and partitions (hypothesis, derandomised so that every run draws the
same cases): the log-sum-exp merge of any split equals one pass, RoPE scores
depend on relative position only, and the absorbed form equals the explicit
one ("DeepSeek-V2", Appendix C) whatever the head count and widths."""

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import mla_oracle as O

SETTINGS = settings(max_examples=40, deadline=None, derandomize=True)
SEEDS = st.integers(0, 2**31 - 1)


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@SETTINGS
@given(seed=SEEDS, S=st.integers(1, 60), ncut=st.integers(0, 6))
def test_split_combine_is_exact_for_any_partition(seed, S, ncut):
    """Any cut of the context into consecutive parts (empty parts included),
    merged by the log-sum-exp algebra, gives the one-pass softmax."""
    rng = np.random.default_rng(seed)
    H, d_c, d_r = 3, 64, 16
    rows = rng.standard_normal((S, d_c + d_r)) * rng.uniform(0.1, 3.0)
    q_abs = rng.standard_normal((H, d_c + d_r))
    scale = O.softmax_scale(32, d_r)
    cuts = sorted(int(c) for c in rng.integers(0, S + 1, size=ncut))
    bounds = list(zip([0, *cuts], [*cuts, S]))
    full_ctx, full_lse = O.latent_attention(q_abs, rows, d_c=d_c, scale=scale)
    ctx, lse = O.combine_partials(O.split_partials(q_abs, rows, bounds, d_c=d_c, scale=scale))
    assert _rel(ctx, full_ctx) <= 1e-12
    assert np.allclose(lse, full_lse, rtol=1e-13, atol=1e-13)


@SETTINGS
@given(seed=SEEDS, half=st.sampled_from([1, 4, 8, 32]), m=st.integers(0, 200_000),
       n=st.integers(0, 200_000), delta=st.integers(0, 100_000))
def test_rope_scores_depend_on_relative_position_for_any_positions(seed, half, m, n, delta):
    """RoPE(q, m) . RoPE(k, n) is unchanged when both positions move by the
    same amount, for any pair count and positions past 128K."""
    rng = np.random.default_rng(seed)
    q, k = rng.standard_normal(2 * half), rng.standard_normal(2 * half)
    ref = O.rope(q, m, 10000.0) @ O.rope(k, n, 10000.0)
    got = O.rope(q, m + delta, 10000.0) @ O.rope(k, n + delta, 10000.0)
    assert abs(got - ref) <= 1e-8 * max(1.0, float(np.linalg.norm(q) * np.linalg.norm(k)))


@SETTINGS
@given(seed=SEEDS, n_h=st.integers(1, 4), d_h=st.sampled_from([8, 16, 32]),
       d_c=st.sampled_from([16, 32, 64]), d_r=st.sampled_from([2, 8, 16]), S=st.integers(1, 40))
def test_absorbed_equals_explicit_for_any_shape(seed, n_h, d_h, d_c, d_r, S):
    """W^UK absorbed into the query and W^UV applied after the weighted sum of
    latents give the explicit per-head keys' and values' attention."""
    rng = np.random.default_rng(seed)
    w_uk = rng.standard_normal((n_h * d_h, d_c)) / np.sqrt(d_c)
    w_uv = rng.standard_normal((n_h * d_h, d_c)) / np.sqrt(d_c)
    rows = rng.standard_normal((S, d_c + d_r))
    qn = rng.standard_normal((n_h, d_h))
    qr = rng.standard_normal((n_h, d_r))
    kw = dict(n_h=n_h, d_h=d_h, d_c=d_c, d_r=d_r, base=10000.0)
    o_e, lse_e = O.mla_decode_explicit(qn, qr, S - 1, rows, w_uk, w_uv, **kw)
    res = O.mla_decode_absorbed(qn, qr, S - 1, rows, w_uk, w_uv, **kw)
    assert _rel(res["o"], o_e) <= 1e-11
    assert np.allclose(res["lse"], lse_e, rtol=1e-12, atol=1e-12)
