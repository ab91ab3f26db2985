"""The seeded input generators: determinism, shapes, distributions, and the
validity of the paged block table."""

import numpy as np

from workloads import (WORKLOADS, bf16_bits, bf16_round, block_table, ctx_lengths,
                       draw_weights, hidden_states, queries)


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 3.0e38, 1e-40], np.float32)
    r = bf16_round(x)
    assert r[0] == 1.0
    assert r[1] == 1.0                      # tie -> even mantissa
    assert r[2] == np.float32(1.0 + 2 ** -7)  # above the tie -> up
    assert r[3] == -2.5
    assert np.all(bf16_round(r) == r)       # idempotent
    assert bf16_bits(np.array([1.0], np.float32))[0] == 0x3F80


def test_generators_are_deterministic_and_shaped():
    wl = WORKLOADS["v2lite_b32_ctx4k"]
    w1, w2 = draw_weights(wl), draw_weights(wl)
    for k in w1:
        assert np.array_equal(w1[k], w2[k])
    assert w1["w_dkv"].shape == (512, 2048) and w1["w_kr"].shape == (64, 2048)
    assert w1["w_uk"].shape == (16 * 128, 512)
    assert np.isclose(w1["w_dkv"].std(), 1 / np.sqrt(2048), rtol=0.02)
    assert np.array_equal(hidden_states(wl, 3, 5), hidden_states(wl, 3, 7)[:5])
    assert not np.array_equal(hidden_states(wl, 3, 5), hidden_states(wl, 4, 5))
    qn, qr = queries(wl)
    assert qn.shape == (32, 16, 128) and qr.shape == (32, 16, 64)
    assert np.all(bf16_round(qn) == qn)


def test_ragged_lengths_and_block_table():
    wl = WORKLOADS["v2lite_paged_ragged_b128"]
    ctx = ctx_lengths(wl)
    assert ctx.shape == (128,) and ctx.min() >= 256 and ctx.max() <= 32768
    # log-uniform: the median sits near the geometric mean of the range
    assert 1024 < np.median(ctx) < 8192
    table, pool = block_table(wl, ctx)
    nblk = (ctx + 63) // 64
    assert pool == nblk.sum()
    used = np.concatenate([table[b, :nblk[b]] for b in range(wl.B)])
    assert np.array_equal(np.sort(used), np.arange(pool))      # a permutation of the pool
    assert all(np.all(table[b, nblk[b]:] == -1) for b in range(wl.B))
    t2, _ = block_table(wl, ctx)
    assert np.array_equal(table, t2)
