"""Double-precision CPU oracle for paged attention over a block-table KV cache.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product library never imports it.

The arithmetic lives in ``oracle.c`` (plain C, fp64, OpenMP over rows); this
module only builds that file with gcc and marshals numpy arrays.  bf16 tensors
cross as ``uint16`` arrays of raw bit patterns.  Every function states which
passage of the source pages it follows in ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libtv_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into oracle/_build/libtv_oracle.so with gcc."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    # binary32 steps stay unfused (the RoPE reading fixes each rounding)
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.oracle_set_threads.argtypes = [i32]
    lib.oracle_set_threads.restype = None
    lib.oracle_max_threads.argtypes = []
    lib.oracle_max_threads.restype = i32
    lib.oracle_kv_append.argtypes = [P, P, P, i64, P, P, i64, i32, i32, i32]
    lib.oracle_kv_append.restype = i64
    lib.oracle_paged_decode_rows.argtypes = [
        P, P, P, P, i64, P, P, P, P, i32, P, i32, i32, i32, i32, i64, dbl]
    lib.oracle_paged_decode_rows.restype = i64
    lib.oracle_paged_decode_partials.argtypes = [
        P, P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64, dbl, i32, i32]
    lib.oracle_paged_decode_partials.restype = i64
    lib.oracle_split_merge.argtypes = [P, P, P, P, i32, i32, i32, i32, i32]
    lib.oracle_split_merge.restype = None
    lib.oracle_paged_prefill_rows.argtypes = [
        P, P, P, i64, P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i64, dbl]
    lib.oracle_paged_prefill_rows.restype = i64
    lib.oracle_rope_rows.argtypes = [P, P, i64, i32, i32, P, i32]
    lib.oracle_rope_rows.restype = i64
    _lib = lib
    return lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def kv_append(k_new, v_new, slot_mapping, k_pool, v_pool):
    """Return copies of (k_pool, v_pool) after writing token t's rows into slot
    slot_mapping[t] (negative = skipped).  Pools are uint16
    [num_pages][page_size][num_kv_heads][head_dim]; k_new/v_new are uint16
    [T][num_kv_heads][head_dim].  Also returns the count of out-of-pool slots."""
    lib = _load()
    kp = np.array(k_pool, dtype=np.uint16, copy=True, order="C")
    vp = np.array(v_pool, dtype=np.uint16, copy=True, order="C")
    kn, vn = _c(k_new, np.uint16), _c(v_new, np.uint16)
    sm = _c(slot_mapping, np.int32)
    num_pages, page_size, hkv, d = kp.shape
    bad = lib.oracle_kv_append(_ptr(kn), _ptr(vn), _ptr(sm), sm.shape[0],
                               _ptr(kp), _ptr(vp), num_pages, hkv, d,
                               page_size)
    return kp, vp, int(bad)


def rope(rows, positions, cos_sin):
    """RoPE of K rows (oracle.c: oracle_rope_rows): a rotated copy of the
    uint16 bf16 rows [T][num_kv_heads][head_dim] at the given positions, with
    angles from cos_sin float32 [max_position][2][head_dim // 2] (cos row,
    then sin row).  Also returns the count of rows whose position is outside
    the table (left unrotated)."""
    lib = _load()
    out = np.array(rows, dtype=np.uint16, copy=True, order="C")
    pos = _c(positions, np.int32)
    cs = _c(cos_sin, np.float32)
    t, hkv, d = out.shape
    if cs.ndim != 3 or cs.shape[1:] != (2, d // 2):
        raise ValueError("cos_sin must be [max_position][2][head_dim // 2]")
    bad = lib.oracle_rope_rows(_ptr(out), _ptr(pos), t, hkv, d, _ptr(cs),
                               cs.shape[0])
    return out, int(bad)


def kv_append_rope(k_new, v_new, slot_mapping, positions, cos_sin, k_pool,
                   v_pool):
    """kv_append with each new K row rotated at its position first (V is not
    rotated)."""
    k_rot, bad_pos = rope(k_new, positions, cos_sin)
    kp, vp, bad = kv_append(k_rot, v_new, slot_mapping, k_pool, v_pool)
    return kp, vp, bad, bad_pos


def paged_decode_rows(q, k_pool, v_pool, block_tables, context_lens, scale,
                      seq_idx, head_idx, with_lse=False, allow_bad=False):
    """Decode attention for selected (sequence, q-head) rows; float64 [n][D].
    Keys whose page id is outside the pool are left out; that raises unless
    ``allow_bad``."""
    lib = _load()
    q = _c(q, np.uint16)
    kp, vp = _c(k_pool, np.uint16), _c(v_pool, np.uint16)
    bt, cl = _c(block_tables, np.int32), _c(context_lens, np.int32)
    si, hi = _c(seq_idx, np.int32), _c(head_idx, np.int32)
    num_pages, page_size, hkv, d = kp.shape
    hq = q.shape[1]
    out = np.zeros((si.shape[0], d), dtype=np.float64)
    lse = np.zeros((si.shape[0],), dtype=np.float64)
    bad = lib.oracle_paged_decode_rows(
        _ptr(out), _ptr(lse), _ptr(si), _ptr(hi), si.shape[0], _ptr(q),
        _ptr(kp), _ptr(vp), _ptr(bt), bt.shape[1], _ptr(cl), hq, hkv, d,
        page_size, num_pages, float(scale))
    if bad and not allow_bad:
        raise ValueError(f"{bad} keys referenced pages outside the pool")
    return (out, lse) if with_lse else out


def paged_decode(q, k_pool, v_pool, block_tables, context_lens, scale,
                 with_lse=False, allow_bad=False):
    """Decode attention for every (sequence, q-head): float64 [B][Hq][D]."""
    b, hq, d = q.shape
    seq_idx = np.repeat(np.arange(b, dtype=np.int32), hq)
    head_idx = np.tile(np.arange(hq, dtype=np.int32), b)
    res = paged_decode_rows(q, k_pool, v_pool, block_tables, context_lens,
                            scale, seq_idx, head_idx, with_lse=True,
                            allow_bad=allow_bad)
    out = res[0].reshape(b, hq, d)
    return (out, res[1].reshape(b, hq)) if with_lse else out


def paged_decode_partials(q, k_pool, v_pool, block_tables, context_lens,
                          scale, partition_tokens, max_partitions):
    """Per-partition normalised outputs [B][Hq][P][D] and natural-log
    sum-exp [B][Hq][P] (float64), -inf for empty partitions."""
    lib = _load()
    q = _c(q, np.uint16)
    kp, vp = _c(k_pool, np.uint16), _c(v_pool, np.uint16)
    bt, cl = _c(block_tables, np.int32), _c(context_lens, np.int32)
    num_pages, page_size, hkv, d = kp.shape
    b, hq, _ = q.shape
    o_p = np.zeros((b, hq, max_partitions, d), dtype=np.float64)
    lse_p = np.zeros((b, hq, max_partitions), dtype=np.float64)
    bad = lib.oracle_paged_decode_partials(
        _ptr(o_p), _ptr(lse_p), _ptr(q), _ptr(kp), _ptr(vp), _ptr(bt),
        bt.shape[1], _ptr(cl), b, hq, hkv, d, page_size, num_pages,
        float(scale), int(partition_tokens), int(max_partitions))
    if bad:
        raise ValueError(f"{bad} keys referenced pages outside the pool")
    return o_p, lse_p


def split_merge(o_p, lse_p, context_lens, partition_tokens):
    """Log-sum-exp merge of partials: float64 [B][Hq][D]."""
    lib = _load()
    o_p = _c(o_p, np.float64)
    lse_p = _c(lse_p, np.float64)
    cl = _c(context_lens, np.int32)
    b, hq, maxp, d = o_p.shape
    out = np.zeros((b, hq, d), dtype=np.float64)
    lib.oracle_split_merge(_ptr(out), _ptr(o_p), _ptr(lse_p), _ptr(cl), b,
                           hq, d, int(partition_tokens), maxp)
    return out


def paged_prefill_rows(q, query_start_loc, k_pool, v_pool, block_tables,
                       context_lens, scale, tok_idx, head_idx, allow_bad=False):
    """Chunked-prefill attention for selected (query row, q-head) pairs.
    Keys whose page id is outside the pool are left out; that raises unless
    ``allow_bad``."""
    lib = _load()
    q = _c(q, np.uint16)
    qsl = _c(query_start_loc, np.int32)
    kp, vp = _c(k_pool, np.uint16), _c(v_pool, np.uint16)
    bt, cl = _c(block_tables, np.int32), _c(context_lens, np.int32)
    ti, hi = _c(tok_idx, np.int32), _c(head_idx, np.int32)
    num_pages, page_size, hkv, d = kp.shape
    hq = q.shape[1]
    out = np.zeros((ti.shape[0], d), dtype=np.float64)
    bad = lib.oracle_paged_prefill_rows(
        _ptr(out), _ptr(ti), _ptr(hi), ti.shape[0], _ptr(q), _ptr(qsl),
        _ptr(kp), _ptr(vp), _ptr(bt), bt.shape[1], _ptr(cl),
        cl.shape[0], hq, hkv, d, page_size, num_pages, float(scale))
    if bad and not allow_bad:
        raise ValueError(f"{bad} keys referenced pages outside the pool")
    return out


def paged_prefill(q, query_start_loc, k_pool, v_pool, block_tables,
                  context_lens, scale, allow_bad=False):
    """Chunked-prefill attention for every row: float64 [rows][Hq][D]."""
    rows, hq, d = q.shape
    tok_idx = np.repeat(np.arange(rows, dtype=np.int32), hq)
    head_idx = np.tile(np.arange(hq, dtype=np.int32), rows)
    out = paged_prefill_rows(q, query_start_loc, k_pool, v_pool, block_tables,
                             context_lens, scale, tok_idx, head_idx,
                             allow_bad=allow_bad)
    return out.reshape(rows, hq, d)
