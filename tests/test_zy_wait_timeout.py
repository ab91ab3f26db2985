"""The device-side time-out path, run on the GPU in the one form this pool
allows: a kernel whose wait has a short limit, on a barrier that nothing
completes, gives up and sets the time-out bit that the host then reads.  The
context must stay usable: a full decode step afterwards still matches the
oracle.  (Every wait in the decode kernels takes the same path past its 2 s
limit.)  Collected last: nothing else runs after a failure here under -x."""

import time

import pytest
import torch

import head_latent_attention_09_b200 as M
from tests.gpu_harness import compare, config_of, oracle_step, run_decode_step
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from head_latent_attention_09_b200 import build
    build.build()
    assert torch.cuda.is_available()


def test_wait_gives_up_with_timeout_status_and_context_survives():
    wl = WORKLOADS["tiny_fp32"]
    handle = M.mla_create(config_of(wl))
    try:
        assert M.mla_get_device_status(handle) == M.MLA_OK
        t0 = time.perf_counter()
        M.mla_selftest_wait_timeout(handle, 5_000_000)          # 5 ms
        st = M.mla_get_device_status(handle)                    # synchronises
        elapsed = time.perf_counter() - t0
        assert st == M.MLA_ERR_TIMEOUT, M.mla_status_string(st)
        assert elapsed < 1.0, f"the wait took {elapsed:.3f} s for a 5 ms limit"
        assert M.mla_get_device_status(handle) == M.MLA_OK     # read and cleared
        with pytest.raises(M.MlaError):
            M.mla_selftest_wait_timeout(handle, 10)             # limit out of range
    finally:
        M.mla_destroy(handle)
    got = run_decode_step(wl)
    want = oracle_step(wl, range(wl.B))
    for key in ("cache_new_rows", "q_abs", "ctx_lat", "lse", "o"):
        compare(got[key], want[key], wl, key)
