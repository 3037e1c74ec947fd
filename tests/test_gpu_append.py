"""KV append on the GPU: bit-exact against the oracle over the whole pool."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (bf16_bits, err_word, gpu_append, require_gpu, upload)
from paged_kv_cache_376_b200 import _lib
from paged_kv_cache_376_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("make", [W.tiny_decode,
                                  lambda: W.continuous_mix(256),
                                  W.chunked_prefill],
                         ids=["tiny", "mix", "prefill-chunk"])
def test_append_is_bit_exact_over_the_whole_pool(make):
    wl = make()
    db = upload(wl)
    gpu_append(db)
    torch.cuda.synchronize()
    kp, vp, bad = oracle.kv_append(wl.k_new, wl.v_new, wl.slot_mapping,
                                   wl.k_pool, wl.v_pool)
    assert bad == 0
    np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
    np.testing.assert_array_equal(bf16_bits(db.v_pool), vp)
    assert err_word(db) == 0


def test_negative_slots_are_skipped_and_bad_slots_flagged():
    wl = W.decode_workload([5, 9, 40, 3], num_pages=8, seed=7)
    slots = wl.slot_mapping.copy()
    slots[1] = -1
    slots[2] = wl.num_pages * wl.page_size + 3     # past the pool
    wl.slot_mapping = slots
    db = upload(wl)
    gpu_append(db)
    torch.cuda.synchronize()
    kp, vp, bad = oracle.kv_append(wl.k_new, wl.v_new, slots, wl.k_pool,
                                   wl.v_pool)
    assert bad == 1
    np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
    np.testing.assert_array_equal(bf16_bits(db.v_pool), vp)
    assert err_word(db) == _lib.DEVERR_BAD_SLOT


def test_zero_tokens_is_a_no_op():
    wl = W.tiny_decode()
    db = upload(wl)
    empty = db.k_new[:0]
    _lib.tv_kv_append(empty, empty, db.slot_mapping[:0], db.k_pool, db.v_pool)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bf16_bits(db.k_pool), wl.k_pool)
