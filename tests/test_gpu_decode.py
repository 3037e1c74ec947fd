"""Paged decode on the GPU against the oracle (elementwise parity bound)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_parity, bf16_bits, err_word, gpu_append,
                      gpu_decode, oracle_after_append, require_gpu, upload)
from paged_kv_cache_376_b200 import _lib
from paged_kv_cache_376_b200 import workloads as W
from paged_kv_cache_376_b200.workloads import bf16_bits as f32_to_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _run(wl):
    """Append then decode on the GPU; oracle append then decode on the CPU."""
    db = upload(wl)
    gpu_append(db)
    out = gpu_decode(db, wl.scale)
    torch.cuda.synchronize()
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    return db, out, ref


def test_tiny_decode_config():
    wl = W.tiny_decode()
    db, out, ref = _run(wl)
    assert_parity(out, ref, "tiny")
    # context 1: the output is the appended V row, bit for bit
    v0 = np.repeat(wl.v_new[0], 4, axis=0)
    np.testing.assert_array_equal(bf16_bits(out[0]), v0)
    assert err_word(db) == 0


@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (16, 8), (32, 4)],
                         ids=["gqa4", "mha", "gqa2", "gqa8"])
def test_ragged_contexts_and_group_sizes(hq, hkv):
    lens = [1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129, 1000,
            4099]
    wl = W.decode_workload(lens, num_pages=sum(-(-n // 16) for n in lens) + 7,
                           seed=101, num_q_heads=hq, num_kv_heads=hkv)
    db, out, ref = _run(wl)
    assert_parity(out, ref, f"hq={hq} hkv={hkv}")
    assert err_word(db) == 0


def test_llama_decode_config_full():
    wl = W.llama_decode()
    db, out, ref = _run(wl)
    assert_parity(out, ref, "llama b64 ctx2048")
    assert err_word(db) == 0


def test_continuous_mix_config_full():
    wl = W.continuous_mix()
    db, out, ref = _run(wl)
    assert_parity(out, ref, "mix b256")
    assert err_word(db) == 0


def test_empty_context_gives_zero_rows():
    wl = W.decode_workload([3, 40], num_pages=8, seed=5)
    db = upload(wl)
    gpu_append(db)
    db.context_lens[0] = 0
    out = gpu_decode(db, wl.scale)
    torch.cuda.synchronize()
    assert (out[0].float() == 0).all()
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables,
                              np.array([0, 40], np.int32), wl.scale)
    assert_parity(out, ref, "ctx 0")


def test_physical_page_permutation_is_bit_identical():
    wl = W.decode_workload([70, 513, 16, 200], num_pages=60, seed=9)
    kp, vp = oracle_after_append(wl)
    rng = np.random.default_rng(3)
    perm = rng.permutation(wl.num_pages)
    kp2, vp2 = np.empty_like(kp), np.empty_like(vp)
    kp2[perm], vp2[perm] = kp, vp
    bt2 = np.where(wl.block_tables >= 0,
                   perm[np.maximum(wl.block_tables, 0)], -1).astype(np.int32)
    outs = []
    for k, v, bt in ((kp, vp, wl.block_tables), (kp2, vp2, bt2)):
        wl.k_pool, wl.v_pool, wl.block_tables = k, v, bt
        db = upload(wl)
        outs.append(bf16_bits(gpu_decode(db, wl.scale)))
    np.testing.assert_array_equal(outs[0], outs[1])


def test_needle_dominates_at_long_context():
    n = 20000
    wl = W.decode_workload([n, 333], seed=11)
    kp, vp = oracle_after_append(wl)
    g = 3
    q = wl.q.copy()
    q[0, 4 * g:4 * g + 4] = q[0, 4 * g]          # same query for the group
    needle = 12345
    page, off = wl.block_tables[0, needle // 16], needle % 16
    qf = W.bf16_to_f64(q[0, 4 * g]).astype(np.float32)
    kp[page, off, g] = f32_to_bf16(qf * 8.0)     # logit ~ |q|^2 ~ 64
    wl.q, wl.k_pool, wl.v_pool = q, kp, vp
    db = upload(wl)
    out = gpu_decode(db, wl.scale)
    torch.cuda.synchronize()
    got = bf16_bits(out[0, 4 * g:4 * g + 4])
    want = np.repeat(vp[page, off, g][None], 4, axis=0)
    np.testing.assert_array_equal(got, want)


def test_bad_page_id_is_flagged_and_left_out():
    wl = W.decode_workload([50, 90], num_pages=12, seed=13)
    kp, vp = oracle_after_append(wl)
    wl.k_pool, wl.v_pool = kp, vp
    bt = wl.block_tables.copy()
    bt[1, 2] = wl.num_pages + 5
    wl.block_tables = bt
    db = upload(wl)
    out = gpu_decode(db, wl.scale)
    assert err_word(db) & _lib.DEVERR_BAD_PAGE
    ref = oracle.paged_decode(wl.q, kp, vp, bt, wl.context_lens, wl.scale,
                              allow_bad=True)
    assert_parity(out, ref, "bad page")


def test_context_beyond_block_table_is_clamped_and_flagged():
    wl = W.decode_workload([40], num_pages=4, seed=17)
    kp, vp = oracle_after_append(wl)
    wl.k_pool, wl.v_pool = kp, vp
    db = upload(wl)
    db.context_lens[0] = 10_000
    gpu_decode(db, wl.scale)
    assert err_word(db) & _lib.DEVERR_BAD_CONTEXT


# ---- fused append + decode (one launch per decode step) ---------------------

def _fused(wl):
    db = upload(wl)
    out = torch.empty_like(db.q)
    _lib.tv_paged_decode_append(out, db.q, db.k_new, db.v_new, db.k_pool,
                                db.v_pool, db.block_tables, db.context_lens,
                                wl.scale, err=db.err)
    torch.cuda.synchronize()
    return db, out


@pytest.mark.parametrize("make", [W.tiny_decode, W.llama_decode,
                                  W.continuous_mix],
                         ids=["tiny", "llama", "mix"])
def test_fused_append_decode_matches_oracle_and_appends(make):
    wl = make()
    db, out = _fused(wl)
    kp, vp = oracle_after_append(wl)
    # the pools hold exactly what a separate append would have written
    np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
    np.testing.assert_array_equal(bf16_bits(db.v_pool), vp)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert_parity(out, ref, f"fused {wl.name}")
    assert err_word(db) == 0


def test_fused_equals_append_then_decode_bitwise():
    lens = [1, 2, 16, 17, 31, 32, 33, 100, 1000, 2049]
    wl = W.decode_workload(lens, seed=55)
    _, fused = _fused(wl)
    db = upload(wl)
    gpu_append(db)
    sep = gpu_decode(db, wl.scale)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bf16_bits(fused), bf16_bits(sep))


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 4)],
                         ids=["mha", "gqa2", "gqa8"])
def test_fused_group_sizes(hq, hkv):
    lens = [1, 15, 16, 17, 300]
    wl = W.decode_workload(lens, seed=56, num_q_heads=hq, num_kv_heads=hkv)
    db, out = _fused(wl)
    kp, vp = oracle_after_append(wl)
    np.testing.assert_array_equal(bf16_bits(db.k_pool), kp)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert_parity(out, ref, f"fused hq={hq} hkv={hkv}")


@pytest.mark.parametrize("scale", [-0.125, 0.0, 0.37, 1.0])
def test_scales_of_either_sign(scale):
    """Any finite scale (the decode scales each fp32 score before taking the
    maximum): a negative one reverses the weights, 0 weighs every visible
    key equally (the output is the mean of V), 1.0 makes the softmax peaked.
    Plain and fused decode against the oracle at the same scale."""
    lens = [1, 16, 17, 300, 2049]
    wl = W.decode_workload(lens, seed=57)
    wl.scale = scale
    db, out, ref = _run(wl)
    assert_parity(out, ref, f"scale={scale}")
    assert err_word(db) == 0
    if scale == 0.0:
        kp, vp = oracle_after_append(wl)
        for s, n in enumerate(lens):
            rows = [vp[wl.block_tables[s, t // 16], t % 16]
                    for t in range(n)]
            mean = np.mean(W.bf16_to_f64(np.stack(rows)), axis=0)  # [Hkv][D]
            np.testing.assert_allclose(
                W.bf16_to_f64(bf16_bits(out[s])),
                np.repeat(mean, 4, axis=0), rtol=2**-7, atol=1e-3)
    db2, fused = _fused(wl)
    assert_parity(fused, ref, f"fused scale={scale}")
    assert err_word(db2) == 0


def test_growing_keys_move_the_running_maximum():
    """Keys scaled by 2^(position // 128) (up to 2^6): the page maxima keep
    growing past the 2^8 lag the online softmax allows, so the accumulators
    are rescaled again and again; plain and fused decode against the
    oracle."""
    from gpu_util import grow_keys
    wl = grow_keys(W.decode_workload([1, 130, 300, 1000, 4099], seed=58))
    db, out, ref = _run(wl)
    assert_parity(out, ref, "growing keys")
    assert err_word(db) == 0
    db2, fused = _fused(wl)
    assert_parity(fused, ref, "fused, growing keys")
    assert err_word(db2) == 0
