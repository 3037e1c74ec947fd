"""Independent float64 brute force used to pin the oracle.

Nothing here is paged: attention is computed on *contiguous* per-sequence
K/V arrays by materialising the whole score matrix, and pools are built from
those arrays by copying whole pages (blocks) into shuffled physical page ids.
It shares no code with ``oracle/`` (which walks a block table token by token)
nor with the CUDA library.
"""
from __future__ import annotations

import numpy as np

BF16_NAN = 0x7FC0


def bits_to_f64(bits):
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def f32_to_bf16_bits(x):
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def random_bf16(rng, shape, sigma=1.0):
    return f32_to_bf16_bits(
        (rng.standard_normal(int(np.prod(shape))) * sigma).astype(np.float32)
    ).reshape(shape)


def attention(q, k, v, visible, scale):
    """q [nq][Hq][D], k/v [nk][Hkv][D] (float64), visible [nq][nk] bool.
    Returns [nq][Hq][D]: softmax over the visible keys of scale * q.k,
    materialised as a full matrix per head; GQA by repeating KV heads."""
    nq, hq, d = q.shape
    hkv = k.shape[1]
    g = hq // hkv
    kk = np.repeat(k, g, axis=1)          # [nk][Hq][D]
    vv = np.repeat(v, g, axis=1)
    s = np.einsum("qhd,khd->hqk", q, kk) * scale
    s = np.where(visible[None, :, :], s, -np.inf)
    m = s.max(axis=2, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(s - m)
    denom = w.sum(axis=2, keepdims=True)
    p = np.divide(w, denom, out=np.zeros_like(w), where=denom > 0)
    return np.einsum("hqk,khd->qhd", p, vv)


def paginate(seqs, page_size, num_pages, rng):
    """Place each contiguous [n_s][Hkv][D] uint16 array into a pool of
    ``num_pages`` pages at shuffled page ids, one whole page at a time.
    Returns (pool [NP][PS][Hkv][D] uint16 (unused slots NaN), block_tables
    [B][MB] int32 (-1 padded))."""
    hkv, d = seqs[0].shape[1:]
    pool = np.full((num_pages, page_size, hkv, d), BF16_NAN, dtype=np.uint16)
    nblocks = [-(-len(x) // page_size) for x in seqs]
    mb = max(1, max(nblocks))
    bt = np.full((len(seqs), mb), -1, dtype=np.int32)
    ids = rng.permutation(num_pages)
    cur = 0
    for s, x in enumerate(seqs):
        for b in range(nblocks[s]):
            page = int(ids[cur])
            cur += 1
            bt[s, b] = page
            chunk = x[b * page_size:(b + 1) * page_size]
            pool[page, :len(chunk)] = chunk
    return pool, bt


def paginate_pair(k_seqs, v_seqs, page_size, num_pages, rng):
    """paginate() for K and V with the same page assignment."""
    state = rng.bit_generator.state
    kp, bt = paginate(k_seqs, page_size, num_pages, rng)
    rng.bit_generator.state = state
    vp, bt2 = paginate(v_seqs, page_size, num_pages, rng)
    assert (bt == bt2).all()
    return kp, vp, bt
