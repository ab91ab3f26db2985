"""The C ABI without a GPU: the library builds for sm_100a, loads, exports every
symbol include/mla.h declares, and its host-only logic (configuration checks,
status strings, the split plan) behaves as documented."""

import ctypes
import os
import re

import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import head_latent_attention_09_b200 as M
from head_latent_attention_09_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "mla.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"{n} declared in mla.h but not exported"
    assert set(names) == set(M.EXPORTED)


def test_status_strings(lib):
    for code, name in [(0, "MLA_OK"), (1, "MLA_ERR_INVALID_ARG"), (5, "MLA_ERR_TIMEOUT"),
                       (6, "MLA_ERR_DEVICE_BOUNDS")]:
        assert M.mla_status_string(code) == name
    assert M.mla_status_string(99) == "MLA_ERR_UNKNOWN"


def _cfg(**kw):
    base = dict(n_h=128, d_h=128, d_c=512, d_r=64, d_model=5120, page_size=0, rope_base=10000.0,
                dtype=M.MLA_BF16)
    base.update(kw)
    return M.mla_config(**base)


def test_config_validation(lib):
    assert M.mla_config_validate(_cfg()) == M.MLA_OK
    assert M.mla_config_validate(_cfg(dtype=M.MLA_FP32, n_h=4, d_h=32, d_c=128, d_r=16,
                                      d_model=256)) == M.MLA_OK
    assert M.mla_config_validate(_cfg(d_r=63)) == M.MLA_ERR_INVALID_ARG
    assert M.mla_config_validate(_cfg(n_h=0)) == M.MLA_ERR_INVALID_ARG
    assert M.mla_config_validate(_cfg(rope_base=0.0)) == M.MLA_ERR_INVALID_ARG
    assert M.mla_config_validate(_cfg(dtype=7)) == M.MLA_ERR_INVALID_ARG
    assert M.mla_config_validate(_cfg(page_size=-1)) == M.MLA_ERR_INVALID_ARG
    assert M.mla_config_validate(_cfg(d_c=1024)) == M.MLA_ERR_UNSUPPORTED
    assert lib.mla_config_validate(None) == M.MLA_ERR_INVALID_ARG


def test_create_without_device_fails_cleanly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    h = ctypes.c_void_p(123)
    st = lib.mla_create(ctypes.byref(_cfg()), ctypes.byref(h))
    assert st == M.MLA_ERR_CUDA and h.value is None
    lib.mla_destroy(None)
    # NULL handles are rejected before any CUDA call
    assert lib.mla_decode_workspace_size(None, 4, 0) == 0
    assert lib.mla_get_device_status(None, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_absorb_q(None, None, None, None, None, None, 1, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_set_rope_scaling(None, 40.0, 4096, 1.0, 32.0, 0.0707) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_query_proj(None, None, 1, None, 0, None, None, None, None, None,
                              None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_selftest_wait_timeout(None, 5000000, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_fp8_scale_groups(None) == 0
    assert lib.mla_cache_append_fp8_workspace_size(None, 4, 1) == 0
    assert lib.mla_cache_append_fp8(None, None, 1, 1, None, None, None, None, None, 0, None, 0,
                                    None, 0, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_quantize_rows_fp8(None, None, 1, None, None, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_attn_fp8(None, None, None, None, 0, None, 0, None, 1, 0, None, 0,
                                   None) == M.MLA_ERR_INVALID_ARG


# Entry points that take the handle first and answer a query instead of a
# status: their documented value for a NULL handle.
NULL_HANDLE_QUERIES = {
    "mla_decode_workspace_size": 0,
    "mla_cache_append_fp8_workspace_size": 0,
    "mla_default_num_parts": 0,
    "mla_fp8_scale_groups": 0,
    "mla_plan_tile": -1,
}
NOT_HANDLE_FIRST = {"mla_status_string", "mla_config_validate", "mla_create", "mla_destroy",
                    "mla_plan_pieces", "mla_plan_pieces_tiled", "mla_noalloc_scratch_bytes"}


def null_handle_args(fn):
    """Arguments for a call with a NULL handle: NULL pointers, batch and
    counts of 1, sizes of 0, the scalars 1."""
    out = []
    for t in fn.argtypes:
        if t is ctypes.c_void_p or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
            out.append(None)
        elif t is ctypes.c_size_t:
            out.append(0)
        elif t is ctypes.c_double:
            out.append(1.0)
        else:
            out.append(1)
    return out


def test_every_entry_point_rejects_a_null_handle(lib):
    """The header's convention: a NULL handle is rejected on the host before
    any CUDA call (here, with no device, a CUDA call would fail differently):
    MLA_ERR_INVALID_ARG from every status-returning entry point, the
    documented value from the queries."""
    names = [n for n in declared_functions() if n not in NOT_HANDLE_FIRST]
    assert len(names) >= 20
    for name in names:
        fn = getattr(lib, name)
        assert fn.argtypes and fn.argtypes[0] is ctypes.c_void_p, name
        got = fn(*null_handle_args(fn))
        want = NULL_HANDLE_QUERIES.get(name, M.MLA_ERR_INVALID_ARG)
        assert got == want, (name, got, want)


def python_plan(ctx, P, tile=64):
    """Independent restatement of the split plan for checking the library's."""
    tiles = [(c + tile - 1) // tile for c in ctx]
    starts = np.concatenate([[0], np.cumsum(tiles)]).astype(int)
    total = int(starts[-1])
    P = min(P, total)
    if total == 0:
        return 0, [0] * (len(ctx) + 1), []
    share = [(w * total // P, (w + 1) * total // P) for w in range(P)]
    pieces = []
    for w, (a, b) in enumerate(share):
        for s in range(len(ctx)):
            lo, hi = max(a, starts[s]), min(b, starts[s + 1])
            if lo < hi:
                pieces.append((s, w, lo, hi))
    pieces.sort()
    base, k = [], 0
    for s in range(len(ctx)):
        base.append(k)
        k += sum(1 for p in pieces if p[0] == s)
    base.append(k)
    return len(pieces), base, share


@pytest.mark.parametrize("seed", range(6))
def test_plan_matches_independent_restatement(lib, seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 40))
    ctx = rng.integers(0, 3000, size=B)
    ctx[rng.random(B) < 0.2] = 0
    for P in (1, 3, 74, 148, 1000):
        n, base = M.mla_plan_pieces(ctx.tolist(), P)
        n2, base2, share = python_plan(ctx.tolist(), P)
        assert n == n2 and base == base2
        assert n <= P + B
        # equal shares: sizes differ by at most one tile
        if share:
            sizes = [b - a for a, b in share]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


@pytest.mark.parametrize("tile", [64, 128, 256])
@pytest.mark.parametrize("seed", range(3))
def test_tiled_plan_matches_independent_restatement(lib, seed, tile):
    rng = np.random.default_rng(100 + seed)
    B = int(rng.integers(1, 40))
    ctx = rng.integers(0, 5000, size=B)
    ctx[rng.random(B) < 0.2] = 0
    for P in (1, 3, 74, 148, 1000):
        n, base = M.mla_plan_pieces_tiled(ctx.tolist(), P, tile)
        n2, base2, _ = python_plan(ctx.tolist(), P, tile)
        assert n == n2 and base == base2 and n <= P + B
    assert M.mla_plan_pieces_tiled(ctx.tolist(), 4, 96)[0] == -1     # not a multiple of 64
    assert M.mla_plan_pieces_tiled(ctx.tolist(), 4, 64) == M.mla_plan_pieces(ctx.tolist(), 4)


def test_plan_v2_workload(lib):
    n, base = M.mla_plan_pieces([8192] * 64, 74)
    assert n <= 74 + 64 and base[-1] == n
    # every sequence is split: 74 shares of 110.7 tiles over 128-tile sequences
    assert all(base[b + 1] - base[b] >= 1 for b in range(64))
    assert M.mla_plan_pieces([], 5)[0] == 0
    assert lib.mla_plan_pieces(None, 0, 1, None) == -1


@settings(max_examples=50, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.function_scoped_fixture])
@given(ctx=st.lists(st.integers(0, 20_000), min_size=1, max_size=120), P=st.integers(1, 600),
       tile=st.sampled_from([64, 128, 256]))
def test_tiled_plan_matches_restatement_for_any_batch(lib, ctx, P, tile):
    """The library's split plan against the restatement over drawn batches,
    split counts (more or fewer than the tiles) and tiles."""
    n, base = M.mla_plan_pieces_tiled(ctx, P, tile)
    n2, base2, _ = python_plan(ctx, P, tile)
    assert n == n2 and base == base2
    assert n <= P + len(ctx)
