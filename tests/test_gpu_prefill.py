"""Chunked prefill on the tcgen05 tensor cores against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_parity, bf16_bits, err_word, gpu_append,
                      gpu_decode, gpu_prefill, oracle_after_append,
                      require_gpu, upload)
from paged_kv_cache_376_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _run(wl):
    db = upload(wl)
    gpu_append(db)
    maxq = int(np.diff(wl.query_start_loc).max())
    out = gpu_prefill(db, wl.scale, maxq)
    torch.cuda.synchronize()
    kp, vp = oracle_after_append(wl)
    return db, out, kp, vp


@pytest.mark.parametrize("prefixes,chunks", [
    ([0], [1]),
    ([0], [200]),
    ([0, 5, 16, 100], [1, 31, 33, 64]),
    ([7, 129, 1000], [95, 130, 257]),
    ([4096, 0, 333], [32, 512, 17]),
], ids=["one-row", "no-prefix", "ragged", "mixed", "long-prefix"])
def test_prefill_matches_oracle_on_every_row(prefixes, chunks):
    wl = W.prefill_workload(prefixes, chunks, seed=31)
    db, out, kp, vp = _run(wl)
    ref = oracle.paged_prefill(wl.q, wl.query_start_loc, kp, vp,
                               wl.block_tables, wl.context_lens, wl.scale)
    assert_parity(out, ref, f"prefill {prefixes} {chunks}")
    assert err_word(db) == 0


def test_chunked_prefill_config_every_row():
    """The 16 x 512-row chunked prefill over prefixes U{0..4096} at full
    size, in the launch the benchmark times (with the costliest-first
    ordering workspace): every (row, head) output against the oracle."""
    from paged_kv_cache_376_b200 import _lib
    wl = W.chunked_prefill()
    db = upload(wl)
    gpu_append(db)
    maxq = int(np.diff(wl.query_start_loc).max())
    out = torch.empty_like(db.q)
    ws = _lib.prefill_workspace(wl.num_seqs, maxq)
    _lib.tv_paged_prefill(out, db.q, db.query_start_loc, db.k_pool, db.v_pool,
                          db.block_tables, db.context_lens, wl.scale, maxq,
                          workspace=ws, err=db.err)
    torch.cuda.synchronize()
    assert err_word(db) == 0
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_prefill(wl.q, wl.query_start_loc, kp, vp,
                               wl.block_tables, wl.context_lens, wl.scale)
    assert_parity(out, ref, "chunked prefill, every row")


def test_bad_page_ids_are_flagged_and_left_out():
    """Block-table entries outside the pool: one in a cached prefix, one
    under the first keys of a sequence with a prefix, and one covering every
    key that the first 16 rows of a prefix-free sequence see (those rows
    attend to nothing and come out zero).  The kernel flags the call and
    leaves those keys out, as the oracle does with ``allow_bad``."""
    from paged_kv_cache_376_b200 import _lib
    wl = W.prefill_workload([100, 40, 0], [70, 30, 20], seed=37)
    db = upload(wl)
    gpu_append(db)                       # appended through the slot mapping
    kp, vp = oracle_after_append(wl)
    bt = wl.block_tables.copy()
    bt[0, 2] = wl.num_pages + 5          # keys 32..47 of sequence 0
    bt[1, 0] = -3                        # keys 0..15 of sequence 1
    bt[2, 0] = wl.num_pages              # keys 0..15 of sequence 2
    db.block_tables.copy_(torch.from_numpy(bt))
    maxq = int(np.diff(wl.query_start_loc).max())
    out = gpu_prefill(db, wl.scale, maxq)
    torch.cuda.synchronize()
    assert err_word(db) & _lib.DEVERR_BAD_PAGE
    ref = oracle.paged_prefill(wl.q, wl.query_start_loc, kp, vp, bt,
                               wl.context_lens, wl.scale, allow_bad=True)
    first = int(wl.query_start_loc[2])
    assert not np.any(ref[first:first + 16])
    assert_parity(out, ref, "prefill with bad page ids")


def test_one_row_chunk_equals_decode():
    lens = [1, 40, 777]
    wl = W.prefill_workload([n - 1 for n in lens], [1] * len(lens), seed=32)
    db = upload(wl)
    gpu_append(db)
    a = gpu_prefill(db, wl.scale, 1)
    b = gpu_decode(db, wl.scale)
    torch.cuda.synchronize()
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert_parity(a, ref, "prefill T=1")
    assert_parity(b, ref, "decode")


def test_rows_do_not_see_later_keys():
    wl = W.prefill_workload([50], [100], seed=33)
    db, out, kp, vp = _run(wl)
    # change keys/values from position 50 + 60 on: rows 0..59 must not move
    cut = 50 + 60
    for j in range(cut, 150):
        page, off = wl.block_tables[0, j // 16], j % 16
        kp[page, off] = 0x3F80
        vp[page, off] = 0x4000
    wl.k_pool, wl.v_pool = kp, vp
    db2 = upload(wl)
    out2 = gpu_prefill(db2, wl.scale, 100)
    torch.cuda.synchronize()
    a, b = bf16_bits(out), bf16_bits(out2)
    np.testing.assert_array_equal(a[:60], b[:60])
    assert not np.array_equal(a[60:], b[60:])


def test_physical_page_permutation_is_bit_identical():
    wl = W.prefill_workload([300, 20], [70, 33], num_pages=80, seed=34)
    kp, vp = oracle_after_append(wl)
    perm = np.random.default_rng(6).permutation(wl.num_pages)
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    bt2 = np.where(wl.block_tables >= 0,
                   perm[np.maximum(wl.block_tables, 0)], -1).astype(np.int32)
    outs = []
    for k, v, bt in ((kp, vp, wl.block_tables), (kp2, vp2, bt2)):
        wl.k_pool, wl.v_pool, wl.block_tables = k, v, bt
        db = upload(wl)
        outs.append(bf16_bits(gpu_prefill(db, wl.scale, 70)))
    np.testing.assert_array_equal(outs[0], outs[1])


def test_cost_ordered_dispatch_is_bit_identical_to_grid_order():
    """The dispatch order changes only which CTA runs when: both orders give
    the same bits, and both match the oracle.  Prefixes of very different
    lengths make the cost order differ from the grid order; one sequence has
    fewer rows than max_query_len (blocks with no work sort last), and the
    workspace is filled with garbage first (it needs no initial contents)."""
    from paged_kv_cache_376_b200 import _lib
    wl = W.prefill_workload([3000, 0, 17, 1500, 64, 4000],
                            [100, 257, 64, 31, 190, 65], seed=77)
    db = upload(wl)
    gpu_append(db)
    maxq = int(np.diff(wl.query_start_loc).max())
    outs = []
    for ordered in (False, True):
        out = torch.full_like(db.q, float("nan"))
        ws = _lib.prefill_workspace(wl.num_seqs, maxq)
        ws.fill_(0xA5)
        _lib.tv_paged_prefill(out, db.q, db.query_start_loc, db.k_pool,
                              db.v_pool, db.block_tables, db.context_lens,
                              wl.scale, maxq, err=db.err, workspace=ws,
                              ordered=ordered)
        torch.cuda.synchronize()
        outs.append(out)
    np.testing.assert_array_equal(bf16_bits(outs[0]), bf16_bits(outs[1]))
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_prefill(wl.q, wl.query_start_loc, kp, vp,
                               wl.block_tables, wl.context_lens, wl.scale)
    assert_parity(outs[1], ref, "cost-ordered prefill")
    assert err_word(db) == 0


@pytest.mark.parametrize("hq,hkv", [(32, 32), (32, 16), (32, 4), (64, 8)],
                         ids=["gqa1", "gqa2", "gqa8", "gqa8-hq64"])
def test_group_sizes_match_oracle_in_both_orders(hq, hkv):
    """Group sizes 1, 2 and 8: an MMA tile is 128 / G query rows x G heads,
    so a CTA covers 256 / G rows and the blocks, the ordering list and the
    q boxes all change with G.  Ragged chunks over prefixes that are not
    multiples of a tile; grid order and cost order give the same bits, and
    both match the oracle on every (row, head)."""
    from paged_kv_cache_376_b200 import _lib
    wl = W.prefill_workload([0, 77, 300, 1000], [130, 45, 257, 9], seed=41,
                            num_q_heads=hq, num_kv_heads=hkv)
    db = upload(wl)
    gpu_append(db)
    maxq = int(np.diff(wl.query_start_loc).max())
    outs = []
    for ordered in (False, True):
        out = torch.full_like(db.q, float("nan"))
        ws = _lib.prefill_workspace(wl.num_seqs, maxq)
        ws.fill_(0x5A)
        _lib.tv_paged_prefill(out, db.q, db.query_start_loc, db.k_pool,
                              db.v_pool, db.block_tables, db.context_lens,
                              wl.scale, maxq, err=db.err, workspace=ws,
                              ordered=ordered)
        torch.cuda.synchronize()
        outs.append(out)
    np.testing.assert_array_equal(bf16_bits(outs[0]), bf16_bits(outs[1]))
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_prefill(wl.q, wl.query_start_loc, kp, vp,
                               wl.block_tables, wl.context_lens, wl.scale)
    assert_parity(outs[0], ref, f"prefill hq={hq} hkv={hkv}")
    assert err_word(db) == 0


def test_growing_keys_move_the_running_maximum():
    """Keys scaled by 2^(position // 128) (up to 2^6): every row's maximum
    keeps growing by far more than 2^8 over later key tiles, so the softmax
    redoes tiles against the new maximum and rescales O in tensor memory,
    repeatedly; every row against the oracle."""
    from gpu_util import grow_keys
    wl = grow_keys(W.prefill_workload([1000, 300, 0, 2000], [64, 200, 130, 48],
                                      seed=35))
    db, out, kp, vp = _run(wl)
    ref = oracle.paged_prefill(wl.q, wl.query_start_loc, kp, vp,
                               wl.block_tables, wl.context_lens, wl.scale)
    assert_parity(out, ref, "prefill, growing keys")
    assert err_word(db) == 0
