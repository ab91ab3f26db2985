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


def _temperature_not_squared(base):
    spec = O._spec(base)
    return 1.0 if spec.factor <= 1.0 else spec.mscale_coef * math.log(spec.factor) + 1.0


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
     [lambda: P.test_yarn_absorbed_explicit_and_brute_force_agree(0.1)]),
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
