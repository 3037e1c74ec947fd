"""RoPE on K during the append (tv_kv_append_rope) and inside the fused
decode step (tv_paged_decode_append_rope) against the oracle's rotation.

The rotation's arithmetic is fixed to the rounding (binary32 products and
sums, bf16 round to nearest even), so the pools must equal the oracle's bit
for bit; the attention outputs are held to the usual parity bound."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, bf16_bits, err_word, require_gpu, upload
from paged_kv_cache_376_b200 import _lib
from paged_kv_cache_376_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _table(max_pos, d=64, base=500000.0):
    """cos/sin [max_pos][2][d/2] of the angle pos * base^(-2i/d)."""
    inv = base ** (-np.arange(0, d, 2, dtype=np.float64) / d)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv[None, :]
    return np.stack([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)


def _positions(wl):
    """Position in its sequence of every appended token."""
    pos = np.empty(wl.slot_mapping.shape[0], np.int32)
    qsl, ctx = wl.query_start_loc, wl.context_lens
    for s in range(wl.num_seqs):
        t0, t1 = int(qsl[s]), int(qsl[s + 1])
        pos[t0:t1] = np.arange(int(ctx[s]) - (t1 - t0), int(ctx[s]))
    return pos


@pytest.mark.parametrize("page_size", [16, 32])
@pytest.mark.parametrize("kind", ["decode", "prefill"])
def test_append_rope_pools_are_bit_exact(kind, page_size):
    if kind == "decode":
        wl = W.decode_workload([1, 17, 33, 100, 2049], seed=81,
                               page_size=page_size)
    else:
        wl = W.prefill_workload([0, 37, 500], [40, 9, 200], seed=82,
                                page_size=page_size)
    pos = _positions(wl)
    cs = _table(4096)
    db = upload(wl)
    g_cs = torch.from_numpy(cs).cuda()
    _lib.tv_kv_append_rope(db.k_new, db.v_new, db.slot_mapping,
                           torch.from_numpy(pos).cuda(), db.k_pool, db.v_pool,
                           g_cs, err=db.err)
    kp, vp, bad, bad_pos = oracle.kv_append_rope(
        wl.k_new, wl.v_new, wl.slot_mapping, pos, cs, wl.k_pool, wl.v_pool)
    assert bad == 0 and bad_pos == 0
    np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
    np.testing.assert_array_equal(bf16_bits(db.v_pool), vp)
    assert err_word(db) == 0


def test_positions_outside_the_table_are_flagged_and_written_unrotated():
    wl = W.decode_workload([3, 20, 70], seed=83)
    pos = _positions(wl)
    cs = _table(32)              # position 69 is outside the table
    db = upload(wl)
    _lib.tv_kv_append_rope(db.k_new, db.v_new, db.slot_mapping,
                           torch.from_numpy(pos).cuda(), db.k_pool, db.v_pool,
                           torch.from_numpy(cs).cuda(), err=db.err)
    kp, vp, _, bad_pos = oracle.kv_append_rope(
        wl.k_new, wl.v_new, wl.slot_mapping, pos, cs, wl.k_pool, wl.v_pool)
    assert bad_pos == 1
    np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
    np.testing.assert_array_equal(bf16_bits(db.v_pool), vp)
    assert err_word(db) & _lib.DEVERR_BAD_POSITION


@pytest.mark.parametrize("page_size", [16, 32])
def test_fused_decode_append_rope_matches_the_oracle(page_size):
    lens = [1, 2, 16, 17, 31, 32, 33, 100, 1000, 2049]
    wl = W.decode_workload(lens, seed=84, page_size=page_size)
    pos = (wl.context_lens - 1).astype(np.int32)
    cs = _table(4096)
    db = upload(wl)
    out = torch.empty_like(db.q)
    _lib.tv_paged_decode_append_rope(out, db.q, db.k_new, db.v_new, db.k_pool,
                                     db.v_pool, db.block_tables,
                                     db.context_lens, wl.scale,
                                     torch.from_numpy(cs).cuda(), err=db.err)
    torch.cuda.synchronize()
    kp, vp, bad, bad_pos = oracle.kv_append_rope(
        wl.k_new, wl.v_new, wl.slot_mapping, pos, cs, wl.k_pool, wl.v_pool)
    assert bad == 0 and bad_pos == 0
    np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
    np.testing.assert_array_equal(bf16_bits(db.v_pool), vp)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert_parity(out, ref, "fused decode with RoPE")
    assert err_word(db) == 0
    # the same as the rotated append followed by the plain decode, bit for bit
    db2 = upload(wl)
    _lib.tv_kv_append_rope(db2.k_new, db2.v_new, db2.slot_mapping,
                           torch.from_numpy(pos).cuda(), db2.k_pool,
                           db2.v_pool, torch.from_numpy(cs).cuda())
    out2 = torch.empty_like(db2.q)
    _lib.tv_paged_decode(out2, db2.q, db2.k_pool, db2.v_pool,
                         db2.block_tables, db2.context_lens, wl.scale)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bf16_bits(out), bf16_bits(out2))
