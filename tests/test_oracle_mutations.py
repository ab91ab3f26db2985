"""Plant plausible mistakes in the oracle (on the CPU, one at a time) and check
that at least one pin fails for each.  This is what makes the pins worth
trusting: each guards against a concrete error."""

import math

import numpy as np
import pytest

from oracle import mla_oracle as O
import tests.test_oracle_pins as P


def _rope_sign_flipped(x, pos, base):
    x = np.asarray(x, np.float64)
    th = O.rope_theta(x.shape[-1], base)
    a = np.asarray(pos, np.float64)[..., None] * th
    out = np.empty(np.broadcast_shapes(x.shape, a.shape[:-1] + (x.shape[-1],)))
    out[..., 0::2] = x[..., 0::2] * np.cos(a) + x[..., 1::2] * np.sin(a)
    out[..., 1::2] = -x[..., 0::2] * np.sin(a) + x[..., 1::2] * np.cos(a)
    return out


def _rope_half_split(x, pos, base):
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    th = O.rope_theta(d, base)
    a = np.asarray(pos, np.float64)[..., None] * th
    x0, x1 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x0 * np.cos(a) - x1 * np.sin(a), x0 * np.sin(a) + x1 * np.cos(a)], -1)


def _absorb_without_rope(q_nope, q_rope_raw, pos, w_uk, *, n_h, d_h, d_r, base):
    lat = np.stack([np.asarray(w_uk[i * d_h:(i + 1) * d_h], np.float64).T @ q_nope[i]
                    for i in range(n_h)])
    return np.concatenate([lat, np.asarray(q_rope_raw, np.float64)], axis=1)


def _kv_wrong_head_block(rows, w_uk, w_uv, n_h, d_h, d_c, heads=None):
    # uses columns of W^UK instead of its row block for head i
    rows = np.asarray(rows, np.float64)
    c, kr = rows[:, :d_c], rows[:, d_c:]
    heads = range(n_h) if heads is None else heads
    ks, vs = [], []
    for i in heads:
        wk = np.asarray(w_uk, np.float64).reshape(d_c, n_h, d_h)[:, i, :].T
        wv = np.asarray(w_uv[i * d_h:(i + 1) * d_h], np.float64)
        ks.append(np.concatenate([c @ wk.T, kr], axis=1))
        vs.append(c @ wv.T)
    return np.stack(ks), np.stack(vs)


_ORIG_COMBINE = O.combine_partials


def _combine_bad_lse(parts):
    ctx, lse = _ORIG_COMBINE(parts)
    return ctx, lse + 1e-6

_ORIG_THETA = O.rope_theta


def _yarn_ramp_inverted(d_r, base):
    # slows the fast pairs and keeps the slow ones (the ramp read backwards)
    spec = O._spec(base)
    plain = _ORIG_THETA(d_r, spec.base)
    if spec.factor <= 1.0:
        return plain
    scaled = _ORIG_THETA(d_r, spec)
    return plain * plain / np.where(scaled == 0, 1.0, scaled) / spec.factor


def _yarn_ramp_linear_in_pair_index(d_r, base):
    # blends linearly in the pair index between the (fractional) indices where
    # a pair turns beta and alpha times, instead of linearly in the turns
    spec = O._spec(base)
    plain = _ORIG_THETA(d_r, spec.base)
    if spec.factor <= 1.0:
        return plain
    k = np.arange(d_r // 2, dtype=np.float64)

    def index_at(turns):
        return -(d_r / 2.0) * math.log(2 * math.pi * turns / spec.original_ctx) / math.log(spec.base)

    k_fast, k_slow = index_at(spec.beta), index_at(spec.alpha)
    gamma = np.clip((k_slow - k) / (k_slow - k_fast), 0.0, 1.0)
    return (1.0 - gamma) * plain / spec.factor + gamma * plain


def _temperature_not_squared(base):
    spec = O._spec(base)
    return 1.0 if spec.factor <= 1.0 else spec.mscale_coef * math.log(spec.factor) + 1.0


_ORIG_ENCODE = O.e4m3_encode


def _e4m3_truncating(v):
    # rounds magnitudes toward zero instead of to nearest even
    x = np.asarray(v, np.float32).astype(np.float64)
    a = np.abs(x)
    e = np.maximum(np.frexp(np.where(a > 0, a, 1.0))[1] - 1, -6)
    q = np.exp2((e - 3).astype(np.float64))
    return _ORIG_ENCODE((np.sign(x) * np.floor(a / q) * q).astype(np.float32))


def _groups_across_parts(d_c, d_r):
    # 128-channel groups over the whole row, mixing c^KV and k^R
    D = d_c + d_r
    return [(a, min(a + 128, D)) for a in range(0, D, 128)]


def _quantize_with_e5m2_max(rows, d_c, d_r):
    # scale from the other FP8 format's largest value
    x = np.asarray(rows, np.float32).reshape(-1, d_c + d_r)
    codes, sc = np.zeros(x.shape, np.uint8), np.zeros((x.shape[0], len(O.fp8_groups(d_c, d_r))), np.float32)
    for gi, (a, b) in enumerate(O.fp8_groups(d_c, d_r)):
        sig = (np.abs(x[:, a:b]).max(axis=1) / np.float32(57344.0)).astype(np.float32)
        nz = sig > 0
        codes[nz, a:b] = O.e4m3_encode(x[nz, a:b] / sig[nz][:, None])
        sc[:, gi] = sig
    return codes, sc


MUTATIONS = [
    ("scale_without_rope_width", "softmax_scale", lambda d_h, d_r: 1.0 / math.sqrt(d_h),
     [P.test_two_token_softmax_closed_form]),
    ("rope_rotates_backwards", "rope", _rope_sign_flipped, [P.test_rope_hand_values]),
    ("rope_half_split_pairs", "rope", _rope_half_split, [P.test_rope_hand_values]),
    ("query_rope_dropped", "absorb_query", _absorb_without_rope,
     [lambda: P.test_brute_force_tiny_workload(1)]),
    ("wrong_uk_block", "explicit_keys_values", _kv_wrong_head_block,
     [lambda: P.test_brute_force_tiny_workload(0)]),
    ("combine_lse_off", "combine_partials", _combine_bad_lse,
     [lambda: P.test_split_combine_is_exact((0, 10, 11, 40, 64))]),
    ("yarn_ramp_inverted", "rope_theta", _yarn_ramp_inverted,
     [P.test_yarn_keeps_fast_pairs_and_slows_slow_pairs_by_s,
      lambda: P.test_yarn_absorbed_explicit_and_brute_force_agree(0.0707)]),
    ("yarn_temperature_not_squared", "attention_temperature", _temperature_not_squared,
     [P.test_yarn_temperature_matches_page_values,
      lambda: P.test_yarn_two_token_softmax_closed_form("v2"),
      lambda: P.test_yarn_two_token_softmax_closed_form("v3")]),
    ("yarn_ramp_linear_in_pair_index", "rope_theta", _yarn_ramp_linear_in_pair_index,
     [P.test_yarn_interior_ramp_hand_values]),
    ("e4m3_truncates", "e4m3_encode", _e4m3_truncating,
     [P.test_e4m3_encode_matches_library_rounding, P.test_e4m3_encode_brute_force_nearest]),
    ("fp8_groups_mix_parts", "fp8_groups", _groups_across_parts,
     [P.test_fp8_groups_of_the_cached_row]),
    ("fp8_scale_from_e5m2_max", "quantize_rows_fp8", _quantize_with_e5m2_max,
     [P.test_fp8_quantize_rows_invariants]),
]


@pytest.mark.parametrize("name,attr,bad,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pin_catches_mutation(monkeypatch, name, attr, bad, pins):
    monkeypatch.setattr(O, attr, bad)
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught == len(pins), f"mutation {name} slipped through"
