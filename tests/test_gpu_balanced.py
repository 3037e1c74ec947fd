"""Work-balanced decode (tv_paged_decode_balanced) against the oracle.

The balanced grid cuts the flattened pages of all (sequence, KV head) pairs
into equal per-warp ranges, so these cases aim at its bookkeeping: pairs
inside one range, pairs cut over hundreds of ranges (the last-arriver merge),
many tiny pairs per range, empty contexts, the fused append, workspace reuse
and the fallback above 512 sequences.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_parity, bf16_bits, err_word, gpu_append,
                      gpu_decode, oracle_after_append, require_gpu, upload)
from paged_kv_cache_376_b200 import _lib
from paged_kv_cache_376_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _ws(db):
    b, hq, _ = db.q.shape
    return _lib.decode_workspace(b, hq, db.k_pool.shape[2])


def _balanced(db, wl, ws, fused):
    out = torch.empty_like(db.q)
    kw = dict(k_new=db.k_new, v_new=db.v_new) if fused else {}
    _lib.tv_paged_decode_balanced(out, db.q, db.k_pool, db.v_pool,
                                  db.block_tables, db.context_lens, wl.scale,
                                  ws, err=db.err, **kw)
    torch.cuda.synchronize()
    return out


def _check(wl, fused, what):
    """Balanced decode (after a separate append, or fused with it) against
    the oracle's append + decode; the fused call must leave the pools equal
    to the oracle's."""
    db = upload(wl)
    if not fused:
        gpu_append(db)
    ws = _ws(db)
    out = _balanced(db, wl, ws, fused)
    kp, vp = oracle_after_append(wl)
    if fused:
        np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
        np.testing.assert_array_equal(bf16_bits(db.v_pool), vp)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert_parity(out, ref, what)
    assert err_word(db) == 0
    # every counter is back at zero for the next call
    nc = wl.num_seqs * wl.k_pool.shape[2]
    assert int(ws[:4 * nc].count_nonzero()) == 0
    return db, out


@pytest.mark.parametrize("fused", [False, True], ids=["decode", "fused"])
@pytest.mark.parametrize("make", [W.tiny_decode, W.llama_decode,
                                  W.continuous_mix],
                         ids=["tiny", "llama", "mix"])
def test_configs(make, fused):
    wl = make()
    _check(wl, fused, f"balanced {wl.name} fused={fused}")


@pytest.mark.parametrize("fused", [False, True], ids=["decode", "fused"])
@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (16, 8), (32, 4),
                                    (8, 1)],
                         ids=["gqa4", "mha", "gqa2", "gqa8", "hkv1"])
def test_ragged_contexts_and_group_sizes(hq, hkv, fused):
    lens = [1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129, 1000,
            4099]
    wl = W.decode_workload(lens, num_pages=sum(-(-n // 16) for n in lens) + 7,
                           seed=301, num_q_heads=hq, num_kv_heads=hkv)
    _check(wl, fused, f"hq={hq} hkv={hkv} fused={fused}")


def test_one_long_sequence_cut_over_hundreds_of_warps():
    # 8 pairs of 6250 pages each: every pair is merged from ~300 partials
    wl = W.decode_workload([100_000], seed=302)
    _check(wl, True, "one sequence, 100k tokens")


def test_many_tiny_sequences_per_warp():
    rng = np.random.default_rng(303)
    lens = rng.integers(1, 40, size=500).tolist()
    wl = W.decode_workload(lens, seed=304)
    _check(wl, True, "500 short sequences")


def test_long_and_short_mixed():
    lens = [131072, 3, 1, 70000, 17, 16, 5000] + [33] * 40
    wl = W.decode_workload(lens, seed=305)
    _check(wl, False, "long + short")


def test_empty_contexts_give_zero_rows():
    wl = W.decode_workload([3, 40, 7, 300], num_pages=40, seed=306)
    db = upload(wl)
    gpu_append(db)
    db.context_lens[0] = 0
    db.context_lens[2] = 0
    out = _balanced(db, wl, _ws(db), False)
    assert (out[0].float() == 0).all() and (out[2].float() == 0).all()
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables,
                              np.array([0, 40, 0, 300], np.int32), wl.scale)
    assert_parity(out, ref, "ctx 0")
    assert err_word(db) == 0


def test_consecutive_calls_reuse_the_workspace():
    # one workspace, sized for the largest batch, serves calls of different
    # shapes in a row; repeated inputs give bit-identical outputs
    big = W.decode_workload([5000, 12, 900, 2048, 1], seed=307)
    small = W.decode_workload([100, 3000], seed=308)
    dbb, dbs = upload(big), upload(small)
    gpu_append(dbb)
    gpu_append(dbs)
    ws = _lib.decode_workspace(5, 32, 8)
    outs = [bf16_bits(_balanced(dbb, big, ws, False)),
            bf16_bits(_balanced(dbs, small, ws, False)),
            bf16_bits(_balanced(dbb, big, ws, False))]
    np.testing.assert_array_equal(outs[0], outs[2])
    for wl, db, o in ((big, dbb, outs[2]), (small, dbs, outs[1])):
        kp, vp = oracle_after_append(wl)
        ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables,
                                  wl.context_lens, wl.scale)
        assert_parity(W.bf16_to_f64(o), ref, wl.name)
    # the per-pair counters (the first bytes) are back at zero; the partial
    # slots after them keep whatever the last call wrote
    assert int(ws[:4 * 5 * 8].count_nonzero()) == 0


def test_physical_page_permutation_is_bit_identical():
    wl = W.decode_workload([70, 513, 16, 200, 4000], num_pages=400, seed=309)
    kp, vp = oracle_after_append(wl)
    perm = np.random.default_rng(4).permutation(wl.num_pages)
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    bt2 = np.where(wl.block_tables >= 0,
                   perm[np.maximum(wl.block_tables, 0)], -1).astype(np.int32)
    outs = []
    for k, v, bt in ((kp, vp, wl.block_tables), (kp2, vp2, bt2)):
        wl.k_pool, wl.v_pool, wl.block_tables = k, v, bt
        db = upload(wl)
        outs.append(bf16_bits(_balanced(db, wl, _ws(db), False)))
    np.testing.assert_array_equal(outs[0], outs[1])


def test_bad_page_id_is_flagged_and_left_out():
    wl = W.decode_workload([50, 900], num_pages=70, seed=310)
    kp, vp = oracle_after_append(wl)
    wl.k_pool, wl.v_pool = kp, vp
    bt = wl.block_tables.copy()
    bt[1, 20] = wl.num_pages + 5
    wl.block_tables = bt
    db = upload(wl)
    out = _balanced(db, wl, _ws(db), False)
    assert err_word(db) & _lib.DEVERR_BAD_PAGE
    ref = oracle.paged_decode(wl.q, kp, vp, bt, wl.context_lens, wl.scale,
                              allow_bad=True)
    assert_parity(out, ref, "bad page")


def test_above_512_sequences_uses_the_per_pair_kernel():
    rng = np.random.default_rng(311)
    lens = rng.integers(1, 300, size=600).tolist()
    wl = W.decode_workload(lens, seed=312)
    db = upload(wl)
    gpu_append(db)
    ws = _ws(db)
    out = _balanced(db, wl, ws, False)
    np.testing.assert_array_equal(bf16_bits(out),
                                  bf16_bits(gpu_decode(db, wl.scale)))
    assert int(ws.count_nonzero()) == 0


def test_workspace_too_small_is_rejected():
    wl = W.decode_workload([100, 200], seed=313)
    db = upload(wl)
    ws = _ws(db)
    with pytest.raises(_lib.TVError, match="INVALID_ARG"):
        _balanced(db, wl, ws[:1024], False)


@pytest.mark.parametrize("scale", [-0.125, 0.0, 1.0])
def test_scales_of_either_sign(scale):
    """The balanced kernel scales each fp32 score before the maximum as
    well: any finite scale, cut and uncut pairs, fused append."""
    lens = [1, 16, 17, 300, 2049, 5000]
    wl = W.decode_workload(lens, seed=302)
    wl.scale = scale
    _check(wl, True, f"balanced scale={scale}")


@pytest.mark.parametrize("fused", [False, True], ids=["decode", "fused"])
def test_growing_keys_move_the_running_maximum(fused):
    """Keys scaled by 2^(position // 128): repeated rescales across pages,
    in pairs cut over several ranges and merged by the last arriver."""
    from gpu_util import grow_keys
    wl = grow_keys(W.decode_workload([1, 130, 300, 1000, 4099, 6000], seed=303))
    _check(wl, fused, f"balanced growing keys fused={fused}")
