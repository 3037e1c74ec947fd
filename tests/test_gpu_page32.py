"""32-token pages (the other page size [P3] 内存池管理 recommends) through every
entry point, against the oracle.

The kernels stream 16-token blocks; a 32-token page is two of them, so these
cases aim at the block -> (page, half) mapping: contexts that end in either
half of a page, appends into either half, split partitions of 16- and
32-token multiples, prefill key tiles of two pages, and the device pool's
slot arithmetic.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_parity, bf16_bits, err_word, gpu_append,
                      gpu_decode, gpu_merge, gpu_prefill, gpu_split,
                      oracle_after_append, require_gpu, upload)
from oracle.pool import PagePool
from paged_kv_cache_376_b200 import _lib
from paged_kv_cache_376_b200 import workloads as W

pytestmark = pytest.mark.gpu

PS = 32
LENS = [1, 2, 15, 16, 17, 31, 32, 33, 48, 63, 64, 65, 100, 1000, 4099]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _decode_wl(seed, **kw):
    return W.decode_workload(LENS, seed=seed, page_size=PS, **kw)


def test_append_is_bit_exact():
    wl = _decode_wl(401)
    db = upload(wl)
    gpu_append(db)
    kp, vp = oracle_after_append(wl)
    np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
    np.testing.assert_array_equal(bf16_bits(db.v_pool), vp)
    assert err_word(db) == 0


@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (32, 4)],
                         ids=["gqa4", "mha", "gqa8"])
def test_decode_and_fused_decode(hq, hkv):
    wl = _decode_wl(402, num_q_heads=hq, num_kv_heads=hkv)
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    db = upload(wl)
    gpu_append(db)
    assert_parity(gpu_decode(db, wl.scale), ref, f"decode PS32 {hq}/{hkv}")
    db = upload(wl)
    out = torch.empty_like(db.q)
    _lib.tv_paged_decode_append(out, db.q, db.k_new, db.v_new, db.k_pool,
                                db.v_pool, db.block_tables, db.context_lens,
                                wl.scale, err=db.err)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
    assert_parity(out, ref, f"fused PS32 {hq}/{hkv}")
    assert err_word(db) == 0


@pytest.mark.parametrize("pt", [32, 64, 512])
def test_split_and_merge(pt):
    wl = _decode_wl(403)
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    db = upload(wl)
    gpu_append(db)
    maxp = -(-int(wl.context_lens.max()) // pt)
    po, pl = gpu_split(db, wl.scale, pt, maxp)
    assert_parity(gpu_merge(db, po, pl, pt), ref, f"split PS32 pt={pt}")


@pytest.mark.parametrize("fused", [False, True], ids=["decode", "fused"])
def test_balanced(fused):
    wl = _decode_wl(404)
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    db = upload(wl)
    if not fused:
        gpu_append(db)
    ws = _lib.decode_workspace(wl.num_seqs, wl.num_q_heads, wl.num_kv_heads)
    out = torch.empty_like(db.q)
    kw = dict(k_new=db.k_new, v_new=db.v_new) if fused else {}
    _lib.tv_paged_decode_balanced(out, db.q, db.k_pool, db.v_pool,
                                  db.block_tables, db.context_lens, wl.scale,
                                  ws, err=db.err, **kw)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
    assert_parity(out, ref, f"balanced PS32 fused={fused}")
    assert err_word(db) == 0


@pytest.mark.parametrize("hq,hkv", [(32, 8), (32, 4), (16, 16)],
                         ids=["gqa4", "gqa8", "mha"])
def test_prefill(hq, hkv):
    wl = W.prefill_workload([0, 5, 16, 40, 1000, 333], [1, 31, 33, 64, 130, 17],
                            seed=405, page_size=PS, num_q_heads=hq,
                            num_kv_heads=hkv)
    db = upload(wl)
    gpu_append(db)
    maxq = int(np.diff(wl.query_start_loc).max())
    out = gpu_prefill(db, wl.scale, maxq)
    torch.cuda.synchronize()
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_prefill(wl.q, wl.query_start_loc, kp, vp,
                               wl.block_tables, wl.context_lens, wl.scale)
    assert_parity(out, ref, f"prefill PS32 hq={hq} hkv={hkv}")
    assert err_word(db) == 0


def test_pool_and_decode_step():
    """The device pool with 32-token pages: a prefill-sized reservation, a
    fork, then decode steps, tables and pools checked against the model."""
    rng = np.random.default_rng(406)
    batch, mb, num_pages, hkv, d = 6, 12, 64, 8, 64
    bt = np.full((batch, mb), -1, np.int64)
    ctx = np.zeros(batch, np.int64)
    kp = W.bf16_bits(rng.standard_normal((num_pages, PS, hkv, d))
                     .astype(np.float32))
    vp = W.bf16_bits(rng.standard_normal((num_pages, PS, hkv, d))
                     .astype(np.float32))
    pool = PagePool(num_pages, page_size=PS)

    def t(a, dt=torch.int32):
        return torch.tensor(np.asarray(a), device="cuda").to(dt)

    def bits(a):
        return torch.tensor(a.view(np.int16), device="cuda").view(
            torch.bfloat16)

    g_bt, g_ctx, g_kp, g_vp = t(bt), t(ctx), bits(kp), bits(vp)
    st = _lib.pool_state(num_pages)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.tv_pool_init(st, page_size=PS, err=err)
    n = [40, 31, 32, 1, 0, 65]
    slots, _ = pool.append_slots(bt, ctx, n, kp, vp)
    g_slots = torch.zeros(int(sum(n)), dtype=torch.int32, device="cuda")
    _lib.tv_pool_append_slots(st, g_bt, g_ctx, g_kp, g_vp,
                              num_new_tokens=t(n), slot_mapping=g_slots,
                              err=err)
    np.testing.assert_array_equal(g_slots.cpu().numpy(), slots)
    kn = W.bf16_bits(rng.standard_normal((len(slots), hkv, d))
                     .astype(np.float32))
    kp, vp, _ = oracle.kv_append(kn, kn, slots, kp, vp)
    _lib.tv_kv_append(bits(kn), bits(kn), g_slots, g_kp, g_vp, err=err)
    pool.fork(bt, ctx, [(0, 4)])
    _lib.tv_pool_fork(st, g_bt, g_ctx, t([0]), t([4]), err=err)
    for step in range(4):
        q = W.bf16_bits(rng.standard_normal((batch, 32, d)).astype(np.float32))
        k1 = W.bf16_bits(rng.standard_normal((batch, hkv, d)).astype(np.float32))
        v1 = W.bf16_bits(rng.standard_normal((batch, hkv, d)).astype(np.float32))
        out = torch.empty((batch, 32, d), dtype=torch.bfloat16, device="cuda")
        _lib.tv_decode_step(st, out, bits(q), bits(k1), bits(v1), g_kp, g_vp,
                            g_bt, g_ctx, 0.125, err=err)
        live = (ctx > 0).astype(np.int64)
        pool.append_slots(bt, ctx, live, kp, vp)
        sl = np.full(batch, -1, np.int32)
        for s in range(batch):
            if live[s]:
                p = ctx[s] - 1
                sl[s] = bt[s][p // PS] * PS + p % PS
        kp, vp, _ = oracle.kv_append(k1, v1, sl, kp, vp)
        ref = oracle.paged_decode(q, kp, vp, bt.astype(np.int32),
                                  ctx.astype(np.int32), 0.125)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(g_bt.cpu().numpy(), bt)
        np.testing.assert_array_equal(g_ctx.cpu().numpy(), ctx)
        np.testing.assert_array_equal(bf16_bits(g_kp), kp)
        assert_parity(out, ref, f"PS32 decode step {step}")
    assert int(err.item()) == 0
