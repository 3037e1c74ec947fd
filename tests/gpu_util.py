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
