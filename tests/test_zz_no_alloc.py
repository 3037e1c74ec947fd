"""tv_paged_decode_split_static: the allocation-free split-KV decode.

It serves callers that cannot allocate on the decode path (engines that give
nearly all device memory to the KV page pool, step loops that cannot afford
cudaMalloc's blocking, C hosts without a device allocator).  Its output must
match the existing two-call path (tv_paged_decode_split into caller buffers,
then tv_split_merge) within the parity bound of the other tests, on two calls
in a row, since every call reuses the same library-owned scratch array; and,
because both paths run the same kernels, it must also match the fp64 CPU
oracle's decode directly, so that a fault the two share cannot hide.

This file is collected last so that, if it fails, a run stopping at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

import oracle
from gpu_util import (REL, ABS, assert_parity, err_word, gpu_append,
                      gpu_merge, gpu_split, oracle_after_append, require_gpu,
                      to_f64, upload)
from paged_kv_cache_376_b200 import _lib
from paged_kv_cache_376_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _existing_path(db, scale, pt, maxp):
    po, pl = gpu_split(db, scale, pt, maxp)
    return gpu_merge(db, po, pl, pt)


def _static_path(db, scale, pt, maxp):
    out = torch.empty_like(db.q)
    _lib.tv_paged_decode_split_static(out, db.q, db.k_pool, db.v_pool,
                                      db.block_tables, db.context_lens, scale,
                                      pt, maxp, err=db.err)
    return out


def test_static_scratch_matches_the_two_call_path_on_consecutive_calls():
    pt = 512
    # call 1: a larger problem; call 2: a smaller one that reuses (and must
    # not be disturbed by) what call 1 left in the shared array
    cases = [W.decode_workload([1, 700, 5000, 12345, 3000], seed=41),
             W.decode_workload([17, 513, 64], seed=42)]
    for wl in cases:
        maxp = -(-int(wl.context_lens.max()) // pt)
        db = upload(wl)
        gpu_append(db)
        want = _existing_path(db, wl.scale, pt, maxp)
        got = _static_path(db, wl.scale, pt, maxp)
        torch.cuda.synchronize()
        assert_parity(got, to_f64(want), f"static scratch, batch {wl.num_seqs}",
                      rel=REL, abs_=ABS)
        kp, vp = oracle_after_append(wl)
        ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables,
                                  wl.context_lens, wl.scale)
        assert_parity(got, ref, f"static scratch vs oracle, batch "
                      f"{wl.num_seqs}", rel=REL, abs_=ABS)
        assert err_word(db) == 0


def test_same_inputs_twice_give_identical_results():
    wl = W.decode_workload([900, 2048, 33], seed=43)
    db = upload(wl)
    gpu_append(db)
    a = _static_path(db, wl.scale, 256, 8)
    b = _static_path(db, wl.scale, 256, 8)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_oversized_call_is_rejected_before_launch():
    lib = _lib.load()
    p = ctypes.c_void_p(0x10000)
    # 64 seqs x 32 heads x 4096 partitions x 65 floats > 2^23 floats
    st = lib.tv_paged_decode_split_static(p, p, p, p, p, 8192, p, 64, 32, 8,
                                          64, 16, 1 << 20, 0.125, 512, 4096,
                                          None, None)
    assert st == _lib.TV_ERR_SCRATCH_LIMIT
    assert lib.tv_status_string(st) == b"TV_ERR_SCRATCH_LIMIT"
    # the long-context configuration (8 x 131072 tokens, 512-token
    # partitions) fits; the call above does not
    assert 64 * 32 * 4096 * 65 > _lib.STATIC_SCRATCH_FLOATS >= 8 * 32 * 256 * 65
