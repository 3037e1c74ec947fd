"""Failure detection on the GPU without a GPU fault.

Every wait in libtv is bounded: when it runs out, the kernel ORs
TV_DEVERR_TIMEOUT into the caller's error word and returns.  The self-test
entry point makes one such wait run out for real (an mbarrier that nothing
completes, a 1 ms limit); the host reads the status, and the context must
still run the hot path correctly afterwards.
"""
import pytest
import torch

import oracle
from gpu_util import (assert_parity, err_word, gpu_append, gpu_decode,
                      oracle_after_append, require_gpu, upload)
from paged_kv_cache_376_b200 import _lib
from paged_kv_cache_376_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def test_a_wait_that_runs_out_sets_the_timeout_bit_and_returns():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    _lib.tv_selftest_wait_timeout(err, 1_000_000, waited)   # 1 ms
    torch.cuda.synchronize()
    assert int(err.item()) & _lib.DEVERR_TIMEOUT
    w = int(waited.item())
    assert 1_000_000 <= w < 200_000_000, w


def test_the_context_is_usable_after_a_time_out():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.tv_selftest_wait_timeout(err, 100_000)
    torch.cuda.synchronize()
    wl = W.decode_workload([40, 300, 17], seed=501)
    db = upload(wl)
    gpu_append(db)
    out = gpu_decode(db, wl.scale)
    torch.cuda.synchronize()
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert_parity(out, ref, "decode after a time-out")
    assert err_word(db) == 0


def test_limits_are_checked_on_the_host():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(_lib.TVError, match="INVALID_ARG"):
        _lib.tv_selftest_wait_timeout(err, -1)
