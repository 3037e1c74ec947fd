"""Split-KV decode partials and their log-sum-exp merge on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_parity, bf16_bits, err_word, gpu_append,
                      gpu_decode, gpu_merge, gpu_split, oracle_after_append,
                      require_gpu, to_f64, upload)
from paged_kv_cache_376_b200 import workloads as W
from paged_kv_cache_376_b200.workloads import bf16_bits as f32_to_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _lse_close(gpu, ref, what):
    g = to_f64(gpu)
    fin = np.isfinite(ref)
    assert (np.isneginf(g) == ~fin).all(), f"{what}: empty partitions differ"
    np.testing.assert_allclose(g[fin], ref[fin], rtol=1e-5, atol=1e-4,
                               err_msg=what)


@pytest.mark.parametrize("pt", [16, 512])
def test_partials_match_oracle(pt):
    lens = [1, 17, 511, 512, 513, 1500, 3000]
    wl = W.decode_workload(lens, seed=21)
    maxp = -(-max(lens) // pt) + 1          # one always-empty partition
    db = upload(wl)
    gpu_append(db)
    po, pl = gpu_split(db, wl.scale, pt, maxp)
    torch.cuda.synchronize()
    kp, vp = oracle_after_append(wl)
    ro, rl = oracle.paged_decode_partials(wl.q, kp, vp, wl.block_tables,
                                          wl.context_lens, wl.scale, pt, maxp)
    assert_parity(po, ro, f"o_p pt={pt}")
    _lse_close(pl, rl, f"lse_p pt={pt}")
    assert err_word(db) == 0


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 4)],
                         ids=["mha", "gqa2", "gqa8"])
def test_partials_group_sizes(hq, hkv):
    """Split partials and the merge at every supported group size (the page
    step pads the G heads of a KV head to the 8 columns of its products)."""
    lens = [1, 17, 512, 513, 3000]
    wl = W.decode_workload(lens, seed=25, num_q_heads=hq, num_kv_heads=hkv)
    pt = 512
    maxp = -(-max(lens) // pt) + 1
    db = upload(wl)
    gpu_append(db)
    po, pl = gpu_split(db, wl.scale, pt, maxp)
    out = gpu_merge(db, po, pl, pt)
    torch.cuda.synchronize()
    kp, vp = oracle_after_append(wl)
    ro, rl = oracle.paged_decode_partials(wl.q, kp, vp, wl.block_tables,
                                          wl.context_lens, wl.scale, pt, maxp)
    assert_parity(po, ro, f"o_p hq={hq} hkv={hkv}")
    _lse_close(pl, rl, f"lse_p hq={hq} hkv={hkv}")
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert_parity(out, ref, f"merged hq={hq} hkv={hkv}")
    assert err_word(db) == 0


def test_merge_kernel_matches_oracle_merge_on_the_same_partials():
    wl = W.decode_workload([100, 2000, 4097], seed=22)
    kp, vp = oracle_after_append(wl)
    pt = 512
    maxp = 10
    ro, rl = oracle.paged_decode_partials(wl.q, kp, vp, wl.block_tables,
                                          wl.context_lens, wl.scale, pt, maxp)
    ro32, rl32 = ro.astype(np.float32), rl.astype(np.float32)
    db = upload(wl)
    out = gpu_merge(db, torch.from_numpy(ro32).cuda(),
                    torch.from_numpy(rl32).cuda(), pt)
    ref = oracle.split_merge(ro32.astype(np.float64), rl32.astype(np.float64),
                             wl.context_lens, pt)
    assert_parity(out, ref, "merge")


def test_split_then_merge_matches_decode_oracle():
    lens = [1, 600, 5000, 9999]
    wl = W.decode_workload(lens, seed=23)
    pt = 512
    maxp = -(-max(lens) // pt)
    db = upload(wl)
    gpu_append(db)
    po, pl = gpu_split(db, wl.scale, pt, maxp)
    out = gpu_merge(db, po, pl, pt)
    torch.cuda.synchronize()
    kp, vp = oracle_after_append(wl)
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert_parity(out, ref, "split+merge")


def test_one_partition_equals_unsplit_decode_bitwise():
    lens = [3, 77, 480, 512]
    wl = W.decode_workload(lens, seed=24)
    db = upload(wl)
    gpu_append(db)
    po, pl = gpu_split(db, wl.scale, 512, 1)
    merged = gpu_merge(db, po, pl, 512)
    direct = gpu_decode(db, wl.scale)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bf16_bits(merged), bf16_bits(direct))


def test_long_split_config_every_row_partials_and_needles():
    """The 8 x 131072-token configuration at full size, in the launch shape
    the benchmark times (512-token partitions): every (sequence, head) output
    row and every partial (o_p, lse_p) against the oracle, plus planted
    needles whose output must equal their V row bit for bit."""
    wl = W.long_split()
    pt = wl.partition_tokens
    maxp = wl.max_partitions()
    kp, vp = oracle_after_append(wl)
    # needles: sequence s, head group 2, at the first, a middle and the last
    # partition, and at a page's last slot; each needle query group shares q
    q = wl.q.copy()
    needles = {1: 5, 3: 131072 // 2 + 77, 5: 131071 - 3, 6: 16 * 4000 + 15}
    for s, pos in needles.items():
        g = 2
        q[s, 4 * g:4 * g + 4] = q[s, 4 * g]
        page, off = wl.block_tables[s, pos // 16], pos % 16
        qf = W.bf16_to_f64(q[s, 4 * g]).astype(np.float32)
        kp[page, off, g] = f32_to_bf16(qf * 8.0)
    wl.q, wl.k_pool, wl.v_pool = q, kp, vp
    db = upload(wl)
    po, pl = gpu_split(db, wl.scale, pt, maxp)
    out = gpu_merge(db, po, pl, pt)
    torch.cuda.synchronize()
    assert err_word(db) == 0
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert_parity(out, ref, "long, every row")
    ro, rl = oracle.paged_decode_partials(wl.q, kp, vp, wl.block_tables,
                                          wl.context_lens, wl.scale, pt, maxp)
    assert_parity(po, ro, "long, every o_p")
    _lse_close(pl, rl, "long, every lse_p")
    for s, pos in needles.items():
        page, off = wl.block_tables[s, pos // 16], pos % 16
        got = bf16_bits(out[s, 8:12])
        np.testing.assert_array_equal(got, np.repeat(vp[page, off, 2][None],
                                                     4, axis=0))


def test_growing_keys_partials_and_merge():
    """Keys scaled by 2^(position // 128) (up to 2^6): partitions whose lse
    differ by hundreds, and rescales inside each partition; partials and
    the merged output against the oracle."""
    from gpu_util import grow_keys
    lens = [1, 300, 1000, 4099]
    wl = grow_keys(W.decode_workload(lens, seed=26))
    pt = 512
    maxp = -(-max(lens) // pt)
    db = upload(wl)
    gpu_append(db)
    po, pl = gpu_split(db, wl.scale, pt, maxp)
    out = gpu_merge(db, po, pl, pt)
    torch.cuda.synchronize()
    kp, vp = oracle_after_append(wl)
    ro, rl = oracle.paged_decode_partials(wl.q, kp, vp, wl.block_tables,
                                          wl.context_lens, wl.scale, pt, maxp)
    assert_parity(po, ro, "growing keys o_p")
    _lse_close(pl, rl, "growing keys lse_p")
    ref = oracle.paged_decode(wl.q, kp, vp, wl.block_tables, wl.context_lens,
                              wl.scale)
    assert_parity(out, ref, "growing keys merged")
    assert err_word(db) == 0
