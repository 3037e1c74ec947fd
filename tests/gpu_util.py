"""Helpers shared by the GPU parity tests."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from paged_kv_cache_376_b200 import _lib, build
from paged_kv_cache_376_b200.device import bf16_bits, upload  # noqa: F401
from paged_kv_cache_376_b200.workloads import bf16_to_f64

# Parity bound for attention outputs (fp32 accumulation, bf16 output):
#   |gpu - oracle| <= 2^-7 * |oracle| + 1e-3, elementwise.
REL = 2.0 ** -7
ABS = 1e-3


def require_gpu():
    """GPU tests fail loudly (never skip) when CUDA or the library is
    missing, so a broken box cannot look green."""
    assert torch.cuda.is_available(), "CUDA device required"
    build.build()
    _lib.load()


def to_f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return bf16_to_f64(bf16_bits(t))
    return t.detach().cpu().double().numpy()


def assert_parity(gpu, ref, what="", rel=REL, abs_=ABS):
    g = to_f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    # a NaN reference would make every comparison below vacuously true
    assert np.isfinite(ref).all(), f"{what}: non-finite oracle output"
    err = np.abs(g - ref)
    bound = rel * np.abs(ref) + abs_
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements out of bound; "
            f"max err {err.max():.3e}; first {idx.tolist()} "
            f"gpu {g[tuple(idx[0])]:.6f} ref {ref[tuple(idx[0])]:.6f}")


def oracle_after_append(wl):
    """Oracle pools after the workload's append."""
    kp, vp, bad = oracle.kv_append(wl.k_new, wl.v_new, wl.slot_mapping,
                                   wl.k_pool, wl.v_pool)
    assert bad == 0
    return kp, vp


def gpu_append(db, stream=None):
    _lib.tv_kv_append(db.k_new, db.v_new, db.slot_mapping, db.k_pool,
                      db.v_pool, err=db.err, stream=stream)


def gpu_decode(db, scale):
    out = torch.empty_like(db.q)
    _lib.tv_paged_decode(out, db.q, db.k_pool, db.v_pool, db.block_tables,
                         db.context_lens, scale, err=db.err)
    return out


def gpu_split(db, scale, partition_tokens, max_partitions):
    b, hq, d = db.q.shape
    po = torch.empty((b, hq, max_partitions, d), dtype=torch.float32,
                     device=db.q.device)
    pl = torch.empty((b, hq, max_partitions), dtype=torch.float32,
                     device=db.q.device)
    _lib.tv_paged_decode_split(po, pl, db.q, db.k_pool, db.v_pool,
                               db.block_tables, db.context_lens, scale,
                               partition_tokens, err=db.err)
    return po, pl


def gpu_merge(db, po, pl, partition_tokens):
    b, hq, _, d = po.shape
    out = torch.empty((b, hq, d), dtype=torch.bfloat16, device=po.device)
    _lib.tv_split_merge(out, po, pl, db.context_lens, partition_tokens)
    return out


def gpu_prefill(db, scale, max_query_len):
    out = torch.empty_like(db.q)
    _lib.tv_paged_prefill(out, db.q, db.query_start_loc, db.k_pool, db.v_pool,
                          db.block_tables, db.context_lens, scale,
                          max_query_len, err=db.err)
    return out


def err_word(db) -> int:
    torch.cuda.synchronize()
    return int(db.err.item()) & 0xFFFFFFFF


def grow_keys(wl, step=128, max_shift=6):
    """Multiply the key row at position j of every sequence by
    2^min(j // step, max_shift) (a power of two: exact in bf16), so the row
    maxima of the scores climb along the context and the running offset of
    the online softmax has to move again and again, far past the 2^8 the
    kernels let it lag.  Cached keys are changed in the pool, the new
    tokens' keys in k_new; stale slots keep their NaN poison."""
    from paged_kv_cache_376_b200 import workloads as W
    ps = wl.k_pool.shape[1]
    new = np.diff(wl.query_start_loc)
    cached = wl.context_lens - new
    kp = wl.k_pool.reshape(-1, *wl.k_pool.shape[2:]).copy()
    kn = wl.k_new.copy()

    def scaled(bits, shift):
        f = W.bf16_to_f64(bits) * (2.0 ** shift)[:, None, None]
        return W.bf16_bits(f.astype(np.float32))

    for s in range(wl.num_seqs):
        pos = np.arange(int(cached[s]))
        shift = np.minimum(pos // step, max_shift)
        if len(pos):
            slots = wl.block_tables[s, pos // ps].astype(np.int64) * ps + pos % ps
            kp[slots] = scaled(kp[slots], shift)
        q0 = int(wl.query_start_loc[s])
        pos = int(cached[s]) + np.arange(int(new[s]))
        if len(pos):
            shift = np.minimum(pos // step, max_shift)
            kn[q0:q0 + len(pos)] = scaled(kn[q0:q0 + len(pos)], shift)
    wl.k_pool = kp.reshape(wl.k_pool.shape)
    wl.k_new = kn
    return wl
