"""Pins for the CPU oracle (no GPU needed).

Each test checks the oracle against something other than itself: an
independent contiguous brute force (tests/brute.py), torch's own
scaled_dot_product_attention, closed forms, invariances, and the two worked
facts the source pages print (tests/golden/).
"""
import math
import os

import numpy as np
import pytest
import torch

import brute
import oracle
from paged_kv_cache_376_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _paged_case(rng, lens, hq=32, hkv=8, d=64, ps=16, extra_pages=5):
    k_seqs = [brute.random_bf16(rng, (n, hkv, d)) for n in lens]
    v_seqs = [brute.random_bf16(rng, (n, hkv, d)) for n in lens]
    npages = sum(-(-n // ps) for n in lens) + extra_pages
    kp, vp, bt = brute.paginate_pair(k_seqs, v_seqs, ps, npages, rng)
    return k_seqs, v_seqs, kp, vp, bt


# ---------------------------------------------------------------- golden --

def test_golden_bf16_values_decode_exactly():
    """A 1-token context returns V exactly, so V's decoded values must equal
    the hand-derived values of each bf16 pattern (page 1, BF16 section)."""
    rows = _read_golden("bf16_format.txt")
    bits = np.array([int(r[0], 16) for r in rows], dtype=np.uint16)
    want = np.array([float(r[1]) for r in rows])
    d = len(bits)
    q = np.full((1, 1, d), 0x3F80, dtype=np.uint16)
    k = np.zeros((1, 1, 1, d), dtype=np.uint16)
    v = bits.reshape(1, 1, 1, d)
    out = oracle.paged_decode(q, k, v, np.zeros((1, 1), np.int32),
                              np.array([1], np.int32), 1.0)
    np.testing.assert_array_equal(out.reshape(-1), want)


def test_golden_page_bytes_match_pool_layout():
    """Page 3's 16 KB page: the workloads' pool layout must give exactly that
    many bytes per page per tensor."""
    (ps, hkv, d, esz, nbytes), = [[int(x) for x in r]
                                  for r in _read_golden("page_bytes.txt")]
    wl = W.tiny_decode()
    assert (wl.page_size, wl.num_kv_heads, wl.head_dim) == (ps, hkv, d)
    assert wl.k_pool.itemsize == esz
    assert wl.k_pool[0].nbytes == nbytes
    assert wl.v_pool[0].nbytes == nbytes


# --------------------------------------------------------------- decode --

@pytest.mark.parametrize("hq,hkv,d,ps", [(32, 8, 64, 16), (4, 4, 64, 16),
                                         (8, 2, 8, 4), (6, 3, 16, 32)])
def test_decode_matches_contiguous_brute_force(hq, hkv, d, ps):
    rng = np.random.default_rng(11)
    lens = [1, ps - 1, ps, ps + 1, 3 * ps + 5, 100]
    k_seqs, v_seqs, kp, vp, bt = _paged_case(rng, lens, hq, hkv, d, ps)
    q = brute.random_bf16(rng, (len(lens), hq, d))
    scale = 1.0 / math.sqrt(d)
    got = oracle.paged_decode(q, kp, vp, bt, np.array(lens, np.int32), scale)
    for s, n in enumerate(lens):
        want = brute.attention(brute.bits_to_f64(q[s:s + 1]),
                               brute.bits_to_f64(k_seqs[s]),
                               brute.bits_to_f64(v_seqs[s]),
                               np.ones((1, n), bool), scale)[0]
        np.testing.assert_allclose(got[s], want, rtol=1e-12, atol=1e-13)


def test_decode_matches_torch_sdpa():
    """Library routine: torch's scaled_dot_product_attention in float64 on
    the contiguous K/V (GQA expanded by repeat_interleave)."""
    rng = np.random.default_rng(12)
    lens = [7, 64, 129]
    k_seqs, v_seqs, kp, vp, bt = _paged_case(rng, lens)
    q = brute.random_bf16(rng, (len(lens), 32, 64))
    got = oracle.paged_decode(q, kp, vp, bt, np.array(lens, np.int32), 0.125)
    for s, n in enumerate(lens):
        qt = torch.from_numpy(brute.bits_to_f64(q[s])).unsqueeze(1)  # [H,1,D]
        kt = torch.from_numpy(brute.bits_to_f64(k_seqs[s])).permute(1, 0, 2)
        vt = torch.from_numpy(brute.bits_to_f64(v_seqs[s])).permute(1, 0, 2)
        kt = kt.repeat_interleave(4, dim=0)
        vt = vt.repeat_interleave(4, dim=0)
        want = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, scale=0.125)[:, 0, :].numpy()
        np.testing.assert_allclose(got[s], want, rtol=1e-11, atol=1e-12)


def test_single_token_returns_v_exactly():
    wl = W.tiny_decode()
    kp, vp, _ = oracle.kv_append(wl.k_new, wl.v_new, wl.slot_mapping,
                                 wl.k_pool, wl.v_pool)
    out = oracle.paged_decode(wl.q, kp, vp, wl.block_tables,
                              wl.context_lens, wl.scale)
    assert wl.context_lens[0] == 1
    v0 = W.bf16_to_f64(wl.v_new[0])           # [Hkv][D]
    want = np.repeat(v0, 4, axis=0)
    np.testing.assert_array_equal(out[0], want)


def test_equal_keys_give_mean_of_v():
    rng = np.random.default_rng(13)
    n = 37
    key = brute.random_bf16(rng, (1, 2, 16))
    k_seq = np.repeat(key, n, axis=0)
    v_seq = brute.random_bf16(rng, (n, 2, 16))
    kp, vp, bt = brute.paginate_pair([k_seq], [v_seq], 16, 8, rng)
    q = brute.random_bf16(rng, (1, 4, 16))
    out = oracle.paged_decode(q, kp, vp, bt, np.array([n], np.int32), 0.25)
    mean_v = brute.bits_to_f64(v_seq).mean(axis=0)          # [Hkv][D]
    np.testing.assert_allclose(out[0], np.repeat(mean_v, 2, axis=0),
                               rtol=1e-13, atol=1e-15)


def test_needle_key_dominates():
    rng = np.random.default_rng(14)
    n, pos = 300, 161
    k_seq = brute.random_bf16(rng, (n, 1, 64), sigma=0.05)
    v_seq = brute.random_bf16(rng, (n, 1, 64))
    q = brute.random_bf16(rng, (1, 1, 64))
    k_seq[pos, 0] = q[0, 0]        # logit = |q|^2 * 2 = ~128 above the rest
    kp, vp, bt = brute.paginate_pair([k_seq], [v_seq], 16, 30, rng)
    out = oracle.paged_decode(q, kp, vp, bt, np.array([n], np.int32), 2.0)
    np.testing.assert_allclose(out[0, 0], brute.bits_to_f64(v_seq[pos, 0]),
                               rtol=1e-9, atol=1e-12)


def test_physical_page_permutation_is_invisible():
    rng = np.random.default_rng(15)
    lens = [33, 90, 1, 16]
    _, _, kp, vp, bt = _paged_case(rng, lens)
    q = brute.random_bf16(rng, (len(lens), 32, 64))
    ctx = np.array(lens, np.int32)
    a = oracle.paged_decode(q, kp, vp, bt, ctx, 0.125)
    perm = rng.permutation(kp.shape[0])          # new id of old page i
    kp2 = np.empty_like(kp)
    vp2 = np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    b = oracle.paged_decode(q, kp2, vp2, bt2, ctx, 0.125)
    np.testing.assert_array_equal(a, b)


def test_gqa_group_with_identical_queries_is_identical():
    rng = np.random.default_rng(16)
    _, _, kp, vp, bt = _paged_case(rng, [50])
    q = brute.random_bf16(rng, (1, 32, 64))
    q[0, 4:8] = q[0, 4]
    out = oracle.paged_decode(q, kp, vp, bt, np.array([50], np.int32), 0.125)
    for h in range(5, 8):
        np.testing.assert_array_equal(out[0, h], out[0, 4])
    assert not np.array_equal(out[0, 3], out[0, 4])


def test_lse_matches_scipy_logsumexp():
    from scipy.special import logsumexp
    rng = np.random.default_rng(17)
    lens = [5, 77]
    k_seqs, _, kp, vp, bt = _paged_case(rng, lens)
    q = brute.random_bf16(rng, (2, 32, 64))
    _, lse = oracle.paged_decode(q, kp, vp, bt, np.array(lens, np.int32),
                                 0.125, with_lse=True)
    for s, n in enumerate(lens):
        qd = brute.bits_to_f64(q[s])
        kd = np.repeat(brute.bits_to_f64(k_seqs[s]), 4, axis=1)
        scores = np.einsum("hd,nhd->hn", qd, kd) * 0.125
        np.testing.assert_allclose(lse[s], logsumexp(scores, axis=1),
                                   rtol=1e-13)


def test_empty_context_gives_zero():
    rng = np.random.default_rng(18)
    _, _, kp, vp, bt = _paged_case(rng, [20, 3])
    q = brute.random_bf16(rng, (2, 32, 64))
    out, lse = oracle.paged_decode(q, kp, vp, bt, np.array([0, 3], np.int32),
                                   0.125, with_lse=True)
    assert (out[0] == 0).all() and np.isneginf(lse[0]).all()


def test_stale_nan_slots_are_never_read():
    """Slots past the context in the last page and unused pages are NaN in
    every workload; a finite output proves the oracle never touches them."""
    wl = W.decode_workload([5, 18, 40], num_pages=12, seed=3)
    kp, vp, _ = oracle.kv_append(wl.k_new, wl.v_new, wl.slot_mapping,
                                 wl.k_pool, wl.v_pool)
    out = oracle.paged_decode(wl.q, kp, vp, wl.block_tables,
                              wl.context_lens, wl.scale)
    assert np.isfinite(out).all()


# ---------------------------------------------------------- split/merge --

@pytest.mark.parametrize("pt", [16, 48, 512])
def test_merge_of_partials_equals_decode(pt):
    rng = np.random.default_rng(19)
    lens = [1, 47, 48, 49, 300]
    _, _, kp, vp, bt = _paged_case(rng, lens)
    q = brute.random_bf16(rng, (len(lens), 32, 64))
    ctx = np.array(lens, np.int32)
    maxp = -(-max(lens) // pt)
    o_p, lse_p = oracle.paged_decode_partials(q, kp, vp, bt, ctx, 0.125, pt,
                                              maxp)
    merged = oracle.split_merge(o_p, lse_p, ctx, pt)
    direct = oracle.paged_decode(q, kp, vp, bt, ctx, 0.125)
    np.testing.assert_allclose(merged, direct, rtol=1e-12, atol=1e-14)
    # partitions past a sequence's end are empty
    for s, n in enumerate(lens):
        used = -(-n // pt)
        assert np.isneginf(lse_p[s, :, used:]).all()
        assert np.isfinite(lse_p[s, :, :used]).all()


def test_partial_equals_brute_force_on_its_range():
    rng = np.random.default_rng(20)
    n, pt = 130, 32
    k_seqs, v_seqs, kp, vp, bt = _paged_case(rng, [n])
    q = brute.random_bf16(rng, (1, 32, 64))
    o_p, _ = oracle.paged_decode_partials(q, kp, vp, bt,
                                          np.array([n], np.int32), 0.125, pt,
                                          5)
    for p in range(5):
        j0, j1 = p * pt, min(n, (p + 1) * pt)
        want = brute.attention(brute.bits_to_f64(q),
                               brute.bits_to_f64(k_seqs[0][j0:j1]),
                               brute.bits_to_f64(v_seqs[0][j0:j1]),
                               np.ones((1, j1 - j0), bool), 0.125)[0]
        np.testing.assert_allclose(o_p[0, :, p], want, rtol=1e-12,
                                   atol=1e-13)


def test_merge_with_a_single_partition_is_identity():
    o = np.random.default_rng(21).standard_normal((2, 3, 1, 8))
    lse = np.array([[[0.3], [-2.0], [5.0]], [[1.0], [1.0], [1.0]]])
    out = oracle.split_merge(o, lse, np.array([10, 4], np.int32), 16)
    np.testing.assert_array_equal(out, o[:, :, 0, :])


# -------------------------------------------------------------- prefill --

def _prefill_case(rng, prefixes, chunks, hq=32, hkv=8, d=64, ps=16):
    lens = [p + c for p, c in zip(prefixes, chunks)]
    k_seqs, v_seqs, kp, vp, bt = _paged_case(rng, lens, hq, hkv, d, ps)
    q = brute.random_bf16(rng, (sum(chunks), hq, d))
    qsl = np.zeros(len(chunks) + 1, np.int32)
    qsl[1:] = np.cumsum(chunks)
    return k_seqs, v_seqs, kp, vp, bt, q, qsl, np.array(lens, np.int32)


def test_prefill_without_prefix_is_causal_self_attention():
    rng = np.random.default_rng(22)
    k_seqs, v_seqs, kp, vp, bt, q, qsl, ctx = _prefill_case(
        rng, [0, 0], [40, 17])
    got = oracle.paged_prefill(q, qsl, kp, vp, bt, ctx, 0.125)
    for s in range(2):
        rows = slice(qsl[s], qsl[s + 1])
        qt = torch.from_numpy(brute.bits_to_f64(q[rows])).permute(1, 0, 2)
        kt = torch.from_numpy(brute.bits_to_f64(k_seqs[s])).permute(1, 0, 2)
        vt = torch.from_numpy(brute.bits_to_f64(v_seqs[s])).permute(1, 0, 2)
        want = torch.nn.functional.scaled_dot_product_attention(
            qt, kt.repeat_interleave(4, 0), vt.repeat_interleave(4, 0),
            is_causal=True, scale=0.125).permute(1, 0, 2).numpy()
        np.testing.assert_allclose(got[rows], want, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("hq,hkv,d,ps", [(32, 8, 64, 16), (32, 8, 64, 32),
                                         (8, 2, 8, 4), (8, 8, 8, 4),
                                         (8, 4, 8, 4), (16, 2, 8, 4)],
                         ids=["gqa4", "gqa4-p32", "gqa4-small", "mha",
                              "gqa2", "gqa8"])
def test_prefill_with_prefix_matches_brute_force(hq, hkv, d, ps):
    rng = np.random.default_rng(23)
    prefixes, chunks = [0, 5, 33, 100], [3, 20, 16, 9]
    k_seqs, v_seqs, kp, vp, bt, q, qsl, ctx = _prefill_case(
        rng, prefixes, chunks, hq, hkv, d, ps)
    got = oracle.paged_prefill(q, qsl, kp, vp, bt, ctx, 0.125)
    for s, (p, c) in enumerate(zip(prefixes, chunks)):
        vis = np.arange(p + c)[None, :] <= (p + np.arange(c))[:, None]
        want = brute.attention(brute.bits_to_f64(q[qsl[s]:qsl[s + 1]]),
                               brute.bits_to_f64(k_seqs[s]),
                               brute.bits_to_f64(v_seqs[s]), vis, 0.125)
        np.testing.assert_allclose(got[qsl[s]:qsl[s + 1]], want, rtol=1e-12,
                                   atol=1e-13)


def test_prefill_of_one_token_equals_decode():
    rng = np.random.default_rng(24)
    _, _, kp, vp, bt, q, qsl, ctx = _prefill_case(rng, [0, 31, 64],
                                                  [1, 1, 1])
    a = oracle.paged_prefill(q, qsl, kp, vp, bt, ctx, 0.125)
    b = oracle.paged_decode(q, kp, vp, bt, ctx, 0.125)
    np.testing.assert_array_equal(a, b)


def test_prefill_rows_do_not_see_later_keys():
    rng = np.random.default_rng(25)
    prefixes, chunks = [20], [30]
    k_seqs, v_seqs, kp, vp, bt, q, qsl, ctx = _prefill_case(
        rng, prefixes, chunks)
    a = oracle.paged_prefill(q, qsl, kp, vp, bt, ctx, 0.125)
    # change every key/value from position 35 on (row 15 of the chunk)
    k2 = [k_seqs[0].copy()]
    v2 = [v_seqs[0].copy()]
    k2[0][35:] = brute.random_bf16(rng, k2[0][35:].shape)
    v2[0][35:] = brute.random_bf16(rng, v2[0][35:].shape)
    kp2 = kp.copy()
    vp2 = vp.copy()
    for j in range(35, 50):
        kp2[bt[0, j // 16], j % 16] = k2[0][j]
        vp2[bt[0, j // 16], j % 16] = v2[0][j]
    b = oracle.paged_prefill(q, qsl, kp2, vp2, bt, ctx, 0.125)
    np.testing.assert_array_equal(a[:15], b[:15])
    assert not np.array_equal(a[15:], b[15:])


# --------------------------------------------------------------- append --

def test_append_writes_exactly_the_mapped_slots():
    rng = np.random.default_rng(26)
    np_, ps, hkv, d = 6, 4, 2, 8
    kp = brute.random_bf16(rng, (np_, ps, hkv, d))
    vp = brute.random_bf16(rng, (np_, ps, hkv, d))
    kn = brute.random_bf16(rng, (5, hkv, d))
    vn = brute.random_bf16(rng, (5, hkv, d))
    slots = np.array([0, 23, -1, 9, 10], np.int32)
    k2, v2, bad = oracle.kv_append(kn, vn, slots, kp, vp)
    assert bad == 0
    kf, vf = kp.reshape(-1, hkv, d).copy(), vp.reshape(-1, hkv, d).copy()
    for t, sl in enumerate(slots):
        if sl >= 0:
            kf[sl], vf[sl] = kn[t], vn[t]
    np.testing.assert_array_equal(k2.reshape(-1, hkv, d), kf)
    np.testing.assert_array_equal(v2.reshape(-1, hkv, d), vf)
    # page/offset view: slot 23 = page 5, offset 3; slot 9 = page 2, offset 1
    np.testing.assert_array_equal(k2[5, 3], kn[1])
    np.testing.assert_array_equal(v2[2, 1], vn[3])


def test_append_counts_out_of_pool_slots():
    kp = np.zeros((2, 4, 1, 8), np.uint16)
    kn = np.ones((2, 1, 8), np.uint16)
    k2, _, bad = oracle.kv_append(kn, kn, np.array([8, 3], np.int32), kp, kp)
    assert bad == 1
    assert (k2.reshape(-1, 8)[3] == 1).all()
    assert k2.reshape(-1, 8).sum() == 8


def test_workload_append_fills_the_last_position():
    wl = W.continuous_mix(batch=16)
    assert ((wl.context_lens - 1) % 16 != 0).all()
    kp, vp, bad = oracle.kv_append(wl.k_new, wl.v_new, wl.slot_mapping,
                                   wl.k_pool, wl.v_pool)
    assert bad == 0
    for s in range(wl.num_seqs):
        pos = int(wl.context_lens[s]) - 1
        page = wl.block_tables[s, pos // 16]
        np.testing.assert_array_equal(kp[page, pos % 16], wl.k_new[s])
        # the append landed in a page already holding earlier tokens
        assert not np.isnan(W.bf16_to_f64(wl.k_pool[page, 0])).any()



# ---- RoPE on K (oracle.rope) ---------------------------------------------------

def _rope_table(angles):
    """cos_sin [positions][2][half] float32 from fp64 angles [positions][half]."""
    a = np.asarray(angles, dtype=np.float64)
    return np.stack([np.cos(a), np.sin(a)], axis=1).astype(np.float32)


def _bf16_rows(rng, shape):
    return W.bf16_bits(rng.standard_normal(shape).astype(np.float32))


def test_rope_golden_pairs_worked_by_hand():
    path = os.path.join(os.path.dirname(__file__), "golden", "rope_example.txt")
    for line in open(path):
        line = line.split("#")[0].split()
        if not line:
            continue
        x1, x2, c, s, y1, y2 = line
        d = 64
        rows = np.zeros((1, 1, d), np.uint16)
        rows[0, 0, 5], rows[0, 0, 5 + d // 2] = int(x1, 16), int(x2, 16)
        cs = np.zeros((1, 2, d // 2), np.float32)
        cs[0, 0, :], cs[0, 1, :] = 1.0, 0.0
        cs[0, 0, 5], cs[0, 1, 5] = float(c), float(s)
        out, bad = oracle.rope(rows, np.array([0], np.int32), cs)
        assert bad == 0
        assert (int(out[0, 0, 5]), int(out[0, 0, 5 + d // 2])) == \
            (int(y1, 16), int(y2, 16))
        # every other pair sees angle 0: unchanged
        keep = np.ones(d, bool)
        keep[[5, 5 + d // 2]] = False
        np.testing.assert_array_equal(out[0, 0, keep], rows[0, 0, keep])


def test_rope_exact_turns():
    rng = np.random.default_rng(61)
    rows = _bf16_rows(rng, (5, 8, 64))
    pos = np.arange(5, dtype=np.int32)
    # 0, a quarter, half and three quarters of a turn, for every pair
    cs = np.zeros((5, 2, 32), np.float32)
    cs[0, 0], cs[0, 1] = 1, 0
    cs[1, 0], cs[1, 1] = 0, 1
    cs[2, 0], cs[2, 1] = -1, 0
    cs[3, 0], cs[3, 1] = 0, -1
    cs[4, 0], cs[4, 1] = 1, 0
    out, bad = oracle.rope(rows, pos, cs)
    assert bad == 0
    x1, x2 = rows[..., :32], rows[..., 32:]
    neg = lambda b: b ^ np.uint16(0x8000)
    np.testing.assert_array_equal(out[0], rows[0])
    np.testing.assert_array_equal(out[1, :, :32], neg(x2[1]))
    np.testing.assert_array_equal(out[1, :, 32:], x1[1])
    np.testing.assert_array_equal(out[2, :, :32], neg(x1[2]))
    np.testing.assert_array_equal(out[2, :, 32:], neg(x2[2]))
    np.testing.assert_array_equal(out[3, :, :32], x2[3])
    np.testing.assert_array_equal(out[3, :, 32:], neg(x1[3]))


def test_rope_matches_the_fp64_rotation_within_rounding():
    """Against a rotation in fp64 of the same bf16 inputs by the same
    (float32) cos/sin: the binary32 steps err by at most 2^-23 of the
    products' magnitude, the bf16 rounding by half an ulp (at most 2^-8 of
    the result, at the bottom of a binade)."""
    rng = np.random.default_rng(62)
    n, hkv, d = 40, 8, 64
    rows = _bf16_rows(rng, (n, hkv, d))
    theta = 10000.0 ** (-np.arange(d // 2) / (d // 2))
    cs = _rope_table(np.arange(300)[:, None] * theta[None, :])
    pos = rng.integers(0, 300, n).astype(np.int32)
    out, bad = oracle.rope(rows, pos, cs)
    assert bad == 0
    x = W.bf16_to_f64(rows)
    c = cs[pos, 0].astype(np.float64)[:, None, :]
    s = cs[pos, 1].astype(np.float64)[:, None, :]
    x1, x2 = x[..., :32], x[..., 32:]
    y = np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)
    mag = np.concatenate([np.abs(x1 * c) + np.abs(x2 * s),
                          np.abs(x2 * c) + np.abs(x1 * s)], axis=-1)
    got = W.bf16_to_f64(out)
    assert (np.abs(got - y) <= 2.0 ** -8 * np.abs(y) + 2.0 ** -22 * mag).all()
    # and not looser than that: some elements need more than a quarter ulp
    assert (np.abs(got - y) > 2.0 ** -10 * np.abs(y)).any()
    # a rotation keeps the length of every pair (up to the same rounding)
    n_in = x1 ** 2 + x2 ** 2
    n_out = got[..., :32] ** 2 + got[..., 32:] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=2.0 ** -6, atol=1e-6)


def test_rope_positions_outside_the_table_are_left_alone_and_counted():
    rng = np.random.default_rng(63)
    rows = _bf16_rows(rng, (3, 2, 64))
    cs = _rope_table(rng.random((4, 32)))
    out, bad = oracle.rope(rows, np.array([-1, 2, 4], np.int32), cs)
    assert bad == 2
    np.testing.assert_array_equal(out[0], rows[0])
    np.testing.assert_array_equal(out[2], rows[2])
    assert not np.array_equal(out[1], rows[1])


def test_kv_append_rope_rotates_k_and_not_v():
    rng = np.random.default_rng(64)
    wl = W.decode_workload([5, 40], seed=65)
    cs = _rope_table(rng.random((64, 32)) * 6.0)
    pos = (wl.context_lens - 1).astype(np.int32)
    kp, vp, bad, bad_pos = oracle.kv_append_rope(
        wl.k_new, wl.v_new, wl.slot_mapping, pos, cs, wl.k_pool, wl.v_pool)
    assert bad == 0 and bad_pos == 0
    k_rot, _ = oracle.rope(wl.k_new, pos, cs)
    kp2, vp2, _ = oracle.kv_append(k_rot, wl.v_new, wl.slot_mapping,
                                   wl.k_pool, wl.v_pool)
    np.testing.assert_array_equal(kp, kp2)
    np.testing.assert_array_equal(vp, vp2)
    _, vp3, _ = oracle.kv_append(wl.k_new, wl.v_new, wl.slot_mapping,
                                 wl.k_pool, wl.v_pool)
    np.testing.assert_array_equal(vp, vp3)
