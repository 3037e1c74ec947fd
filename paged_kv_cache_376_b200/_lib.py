"""ctypes binding of libtv (include/tv.h).

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of libtv.so.  Functions keep the C names and take torch tensors that
already live on the GPU; they check dtype/shape/device, pass raw pointers and
the current CUDA stream, and raise on a non-OK status.  There is no CPU or
eager fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtv.so")

TV_OK = 0
STATUS = {0: "TV_OK", 1: "TV_ERR_INVALID_ARG", 2: "TV_ERR_UNSUPPORTED",
          3: "TV_ERR_CUDA", 4: "TV_ERR_SCRATCH_LIMIT"}
TV_ERR_SCRATCH_LIMIT = 4
STATIC_SCRATCH_FLOATS = 1 << 23   # TV_STATIC_SCRATCH_FLOATS in include/tv.h
DEVERR_BAD_SLOT = 1 << 0
DEVERR_BAD_PAGE = 1 << 1
DEVERR_BAD_CONTEXT = 1 << 2
DEVERR_TIMEOUT = 1 << 3
DEVERR_BAD_QUERY = 1 << 4
DEVERR_POOL_EMPTY = 1 << 5
DEVERR_BAD_SEQ = 1 << 6
DEVERR_BAD_POSITION = 1 << 7

# (name, restype, argtypes) of every symbol include/tv.h declares
_P, _I, _I64, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
SIGNATURES = {
    "tv_status_string": (ctypes.c_char_p, [_I]),
    "tv_last_cuda_error": (_I, []),
    "tv_version": (_I, []),
    "tv_kv_append": (_I, [_P, _P, _P, _I64, _P, _P, _I64, _I, _I, _I, _P,
                          _P]),
    "tv_kv_append_rope": (_I, [_P, _P, _P, _P, _I64, _P, _P, _I64, _I, _I,
                               _I, _P, _I, _P, _P]),
    "tv_paged_decode": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I,
                             _I64, _F, _P, _P]),
    "tv_paged_decode_append_rope": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P,
                                         _I, _I, _I, _I, _I, _I64, _F, _P, _I,
                                         _P, _P]),
    "tv_paged_decode_append": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _I,
                                    _I, _I, _I, _I, _I64, _F, _P, _P]),
    "tv_paged_decode_split": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _I, _I,
                                   _I, _I, _I, _I64, _F, _I, _I, _P, _P]),
    "tv_split_merge": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "tv_paged_prefill": (_I, [_P, _P, _I64, _P, _P, _P, _P, _I, _P, _I, _I,
                              _I, _I, _I, _I, _I64, _F, _P, ctypes.c_size_t,
                              _P, _P]),
    "tv_prefill_workspace_size": (_I, [_I, _I,
                                       ctypes.POINTER(ctypes.c_size_t)]),
    "tv_paged_decode_split_static": (_I, [_P, _P, _P, _P, _P, _I, _P, _I, _I,
                                          _I, _I, _I, _I64, _F, _I, _I, _P,
                                          _P]),
    "tv_decode_workspace_size": (_I, [_I, _I, _I, _I,
                                      ctypes.POINTER(ctypes.c_size_t)]),
    "tv_paged_decode_balanced": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _P, _I,
                                      _I, _I, _I, _I, _I64, _F, _P,
                                      ctypes.c_size_t, _P, _P]),
    "tv_selftest_wait_timeout": (_I, [_P, _I64, _P, _P]),
    "tv_pool_init": (_I, [_P, _I64, _I, _P, _I, _P, _I, _P, _P]),
    "tv_pool_append_slots": (_I, [_P, _I64, _P, _I, _P, _P, _I, _P, _P, _P,
                                  _I, _I, _I, _P, _P]),
    "tv_pool_fork": (_I, [_P, _I64, _P, _I, _P, _I, _P, _P, _I, _P, _P]),
    "tv_pool_release": (_I, [_P, _I64, _P, _I, _P, _I, _P, _I, _P, _P]),
    "tv_decode_step": (_I, [_P, _I64, _P, _P, _P, _P, _P, _P, _P, _I, _P, _I,
                            _I, _I, _I, _I, _F, _P, ctypes.c_size_t, _P,
                            _P]),
}

_lib = None


class TVError(RuntimeError):
    pass


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libtv.so; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise TVError(
            f"{path} is missing: build it with "
            "`python -m paged_kv_cache_376_b200.build` (there is no fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int, what: str) -> None:
    if status != TV_OK:
        lib = load()
        extra = ""
        if status == 3:
            extra = f" (CUDA error {lib.tv_last_cuda_error()})"
        raise TVError(f"{what}: {STATUS.get(status, status)}{extra}")


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _cuda(t: torch.Tensor, dtype, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def tv_kv_append(k_new, v_new, slot_mapping, k_pool, v_pool, err=None,
                 stream=None):
    """Scatter k_new/v_new [T][Hkv][D] (bf16) into pool slots
    slot_mapping [T] (int32) of k_pool/v_pool [NP][PS][Hkv][D] in place."""
    lib = load()
    bf = torch.bfloat16
    _cuda(k_new, bf, "k_new"), _cuda(v_new, bf, "v_new")
    _cuda(k_pool, bf, "k_pool"), _cuda(v_pool, bf, "v_pool")
    _cuda(slot_mapping, torch.int32, "slot_mapping")
    if err is not None:
        _cuda(err, torch.int32, "err")
    num_pages, page_size, hkv, d = k_pool.shape
    if v_pool.shape != k_pool.shape or k_new.shape != v_new.shape:
        raise ValueError("K/V shape mismatch")
    if k_new.shape[1:] != (hkv, d) or slot_mapping.shape != k_new.shape[:1]:
        raise ValueError("k_new must be [T][Hkv][D] with slot_mapping [T]")
    _check(lib.tv_kv_append(_ptr(k_new), _ptr(v_new), _ptr(slot_mapping),
                            k_new.shape[0], _ptr(k_pool), _ptr(v_pool),
                            num_pages, hkv, d, page_size, _ptr(err),
                            _stream(stream)), "tv_kv_append")


def _rope_table(cos_sin, d):
    _cuda(cos_sin, torch.float32, "rope_cos_sin")
    if cos_sin.dim() != 3 or tuple(cos_sin.shape[1:]) != (2, d // 2):
        raise ValueError("rope_cos_sin must be [max_position][2][head_dim//2]")
    return cos_sin.shape[0]


def tv_kv_append_rope(k_new, v_new, slot_mapping, positions, k_pool, v_pool,
                      cos_sin, err=None, stream=None):
    """tv_kv_append with each K row rotated at positions[t] (RoPE, angles
    from cos_sin [max_position][2][D/2] fp32: cos row, sin row)."""
    lib = load()
    bf = torch.bfloat16
    _cuda(k_new, bf, "k_new"), _cuda(v_new, bf, "v_new")
    _cuda(k_pool, bf, "k_pool"), _cuda(v_pool, bf, "v_pool")
    _cuda(slot_mapping, torch.int32, "slot_mapping")
    _cuda(positions, torch.int32, "positions")
    if err is not None:
        _cuda(err, torch.int32, "err")
    num_pages, page_size, hkv, d = k_pool.shape
    if v_pool.shape != k_pool.shape or k_new.shape != v_new.shape:
        raise ValueError("K/V shape mismatch")
    if k_new.shape[1:] != (hkv, d) or slot_mapping.shape != k_new.shape[:1] \
            or positions.shape != slot_mapping.shape:
        raise ValueError("k_new must be [T][Hkv][D] with slot_mapping and "
                         "positions [T]")
    max_pos = _rope_table(cos_sin, d)
    _check(lib.tv_kv_append_rope(
        _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), _ptr(positions),
        k_new.shape[0], _ptr(k_pool), _ptr(v_pool), num_pages, hkv, d,
        page_size, _ptr(cos_sin), max_pos, _ptr(err), _stream(stream)),
        "tv_kv_append_rope")


def tv_paged_decode_append_rope(out, q, k_new, v_new, k_pool, v_pool,
                                block_tables, context_lens, scale, cos_sin,
                                err=None, stream=None):
    """tv_paged_decode_append with each sequence's new K row rotated at its
    position context_len-1 (RoPE, table as tv_kv_append_rope)."""
    lib = load()
    bf = torch.bfloat16
    for n, t in (("out", out), ("q", q), ("k_new", k_new), ("v_new", v_new),
                 ("k_pool", k_pool), ("v_pool", v_pool)):
        _cuda(t, bf, n)
    _cuda(block_tables, torch.int32, "block_tables")
    _cuda(context_lens, torch.int32, "context_lens")
    if err is not None:
        _cuda(err, torch.int32, "err")
    num_pages, page_size, hkv, d = k_pool.shape
    b, hq, _ = q.shape
    if out.shape != q.shape or block_tables.shape[0] != b or \
            k_new.shape != (b, hkv, d) or v_new.shape != k_new.shape:
        raise ValueError("shape mismatch")
    max_pos = _rope_table(cos_sin, d)
    _check(lib.tv_paged_decode_append_rope(
        _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool),
        _ptr(v_pool), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), b, hq, hkv, d, page_size, num_pages, float(scale),
        _ptr(cos_sin), max_pos, _ptr(err), _stream(stream)),
        "tv_paged_decode_append_rope")


def tv_paged_decode(out, q, k_pool, v_pool, block_tables, context_lens,
                    scale, err=None, stream=None):
    """out[B][Hq][D] (bf16) = paged decode attention of q[B][Hq][D]."""
    lib = load()
    bf = torch.bfloat16
    for n, t in (("out", out), ("q", q), ("k_pool", k_pool),
                 ("v_pool", v_pool)):
        _cuda(t, bf, n)
    _cuda(block_tables, torch.int32, "block_tables")
    _cuda(context_lens, torch.int32, "context_lens")
    if err is not None:
        _cuda(err, torch.int32, "err")
    num_pages, page_size, hkv, d = k_pool.shape
    b, hq, _ = q.shape
    if out.shape != q.shape or block_tables.shape[0] != b:
        raise ValueError("shape mismatch")
    _check(lib.tv_paged_decode(
        _ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), b, hq, hkv, d, page_size,
        num_pages, float(scale), _ptr(err), _stream(stream)),
        "tv_paged_decode")


def tv_paged_decode_append(out, q, k_new, v_new, k_pool, v_pool,
                           block_tables, context_lens, scale, err=None,
                           stream=None):
    """Fused decode step: append k_new/v_new [B][Hkv][D] at position
    context_len-1 of each sequence (slot from the block table) and write the
    attention of q[B][Hq][D] over the cache into out[B][Hq][D]."""
    lib = load()
    bf = torch.bfloat16
    for n, t in (("out", out), ("q", q), ("k_new", k_new), ("v_new", v_new),
                 ("k_pool", k_pool), ("v_pool", v_pool)):
        _cuda(t, bf, n)
    _cuda(block_tables, torch.int32, "block_tables")
    _cuda(context_lens, torch.int32, "context_lens")
    if err is not None:
        _cuda(err, torch.int32, "err")
    num_pages, page_size, hkv, d = k_pool.shape
    b, hq, _ = q.shape
    if out.shape != q.shape or block_tables.shape[0] != b or \
            k_new.shape != (b, hkv, d) or v_new.shape != k_new.shape:
        raise ValueError("shape mismatch")
    _check(lib.tv_paged_decode_append(
        _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool),
        _ptr(v_pool), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), b, hq, hkv, d, page_size, num_pages, float(scale),
        _ptr(err), _stream(stream)), "tv_paged_decode_append")


def tv_paged_decode_split(partial_out, partial_lse, q, k_pool, v_pool,
                          block_tables, context_lens, scale,
                          partition_tokens, err=None, stream=None):
    """Per-partition fp32 partials: partial_out [B][Hq][P][D], partial_lse
    [B][Hq][P] with P = partial_out.shape[2] partitions."""
    lib = load()
    bf = torch.bfloat16
    _cuda(q, bf, "q"), _cuda(k_pool, bf, "k_pool"), _cuda(v_pool, bf, "v_pool")
    _cuda(partial_out, torch.float32, "partial_out")
    _cuda(partial_lse, torch.float32, "partial_lse")
    _cuda(block_tables, torch.int32, "block_tables")
    _cuda(context_lens, torch.int32, "context_lens")
    if err is not None:
        _cuda(err, torch.int32, "err")
    num_pages, page_size, hkv, d = k_pool.shape
    b, hq, _ = q.shape
    maxp = partial_out.shape[2]
    if partial_out.shape != (b, hq, maxp, d) or \
            partial_lse.shape != (b, hq, maxp):
        raise ValueError("partials must be [B][Hq][P][D] and [B][Hq][P]")
    _check(lib.tv_paged_decode_split(
        _ptr(partial_out), _ptr(partial_lse), _ptr(q), _ptr(k_pool),
        _ptr(v_pool), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), b, hq, hkv, d, page_size, num_pages, float(scale),
        int(partition_tokens), maxp, _ptr(err), _stream(stream)),
        "tv_paged_decode_split")


def tv_split_merge(out, partial_out, partial_lse, context_lens,
                   partition_tokens, stream=None):
    """out[B][Hq][D] (bf16) = log-sum-exp merge of the partials."""
    lib = load()
    _cuda(out, torch.bfloat16, "out")
    _cuda(partial_out, torch.float32, "partial_out")
    _cuda(partial_lse, torch.float32, "partial_lse")
    _cuda(context_lens, torch.int32, "context_lens")
    b, hq, maxp, d = partial_out.shape
    if out.shape != (b, hq, d):
        raise ValueError("out must be [B][Hq][D]")
    _check(lib.tv_split_merge(
        _ptr(out), _ptr(partial_out), _ptr(partial_lse), _ptr(context_lens),
        b, hq, d, int(partition_tokens), maxp, _stream(stream)),
        "tv_split_merge")


def tv_prefill_workspace_size(num_seqs, max_query_len):
    n = ctypes.c_size_t(0)
    _check(load().tv_prefill_workspace_size(int(num_seqs), int(max_query_len),
                                            ctypes.byref(n)),
           "tv_prefill_workspace_size")
    return n.value


def prefill_workspace(num_seqs, max_query_len, device="cuda"):
    """Device workspace for the cost-ordered prefill dispatch (no initial
    contents needed)."""
    n = tv_prefill_workspace_size(num_seqs, max_query_len)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def tv_paged_prefill(out, q, query_start_loc, k_pool, v_pool, block_tables,
                     context_lens, scale, max_query_len, err=None,
                     stream=None, workspace=None, ordered=True):
    """out[rows][Hq][D] (bf16) = chunked-prefill attention of q[rows][Hq][D]
    over the paged cache (chunk K/V already appended).  With ordered=True
    the blocks run costliest first, through ``workspace`` (allocated here
    when None); ordered=False keeps grid order (same results)."""
    lib = load()
    bf = torch.bfloat16
    for n, t in (("out", out), ("q", q), ("k_pool", k_pool),
                 ("v_pool", v_pool)):
        _cuda(t, bf, n)
    _cuda(query_start_loc, torch.int32, "query_start_loc")
    _cuda(block_tables, torch.int32, "block_tables")
    _cuda(context_lens, torch.int32, "context_lens")
    if err is not None:
        _cuda(err, torch.int32, "err")
    num_pages, page_size, hkv, d = k_pool.shape
    rows, hq, _ = q.shape
    b = context_lens.shape[0]
    if out.shape != q.shape or query_start_loc.shape != (b + 1,):
        raise ValueError("shape mismatch")
    ws, ws_bytes = None, 0
    if ordered:
        if workspace is None:
            workspace = prefill_workspace(b, max_query_len, q.device)
        _cuda(workspace, workspace.dtype, "workspace")
        ws, ws_bytes = workspace, workspace.numel() * workspace.element_size()
    _check(lib.tv_paged_prefill(
        _ptr(out), _ptr(q), rows, _ptr(query_start_loc), _ptr(k_pool),
        _ptr(v_pool), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), b, int(max_query_len), hq, hkv, d, page_size,
        num_pages, float(scale), _ptr(ws), ws_bytes, _ptr(err),
        _stream(stream)), "tv_paged_prefill")


def tv_paged_decode_split_static(out, q, k_pool, v_pool, block_tables,
                                 context_lens, scale, partition_tokens,
                                 max_partitions, err=None, stream=None):
    """Split-KV decode + merge into out[B][Hq][D] (bf16) without any
    caller-side scratch: the partials live in the library's fixed device
    array (for callers that cannot allocate on the decode path).  Raises
    TVError with TV_ERR_SCRATCH_LIMIT when B * Hq * max_partitions * (D + 1)
    exceeds STATIC_SCRATCH_FLOATS."""
    lib = load()
    bf = torch.bfloat16
    for n, t in (("out", out), ("q", q), ("k_pool", k_pool),
                 ("v_pool", v_pool)):
        _cuda(t, bf, n)
    _cuda(block_tables, torch.int32, "block_tables")
    _cuda(context_lens, torch.int32, "context_lens")
    if err is not None:
        _cuda(err, torch.int32, "err")
    num_pages, page_size, hkv, d = k_pool.shape
    b, hq, _ = q.shape
    if out.shape != q.shape or block_tables.shape[0] != b:
        raise ValueError("shape mismatch")
    _check(lib.tv_paged_decode_split_static(
        _ptr(out), _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), b, hq, hkv, d, page_size,
        num_pages, float(scale), int(partition_tokens), int(max_partitions),
        _ptr(err), _stream(stream)), "tv_paged_decode_split_static")


def tv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads,
                             head_dim=64):
    """Bytes of workspace tv_paged_decode_balanced needs on the current
    device for up to num_seqs sequences."""
    lib = load()
    out = ctypes.c_size_t(0)
    _check(lib.tv_decode_workspace_size(int(num_seqs), int(num_q_heads),
                                        int(num_kv_heads), int(head_dim),
                                        ctypes.byref(out)),
           "tv_decode_workspace_size")
    return out.value


def decode_workspace(num_seqs, num_q_heads, num_kv_heads, device=None):
    """A zero-filled uint8 workspace of the size tv_decode_workspace_size
    gives (the balanced decode leaves it zero-filled after every call)."""
    n = tv_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def tv_paged_decode_balanced(out, q, k_pool, v_pool, block_tables,
                             context_lens, scale, workspace, k_new=None,
                             v_new=None, err=None, stream=None):
    """Work-balanced decode (fused with the append when k_new/v_new are
    given): out[B][Hq][D] as tv_paged_decode / tv_paged_decode_append."""
    lib = load()
    bf = torch.bfloat16
    for n, t in (("out", out), ("q", q), ("k_pool", k_pool),
                 ("v_pool", v_pool)):
        _cuda(t, bf, n)
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if k_new is not None:
        _cuda(k_new, bf, "k_new"), _cuda(v_new, bf, "v_new")
    _cuda(block_tables, torch.int32, "block_tables")
    _cuda(context_lens, torch.int32, "context_lens")
    _cuda(workspace, torch.uint8, "workspace")
    if err is not None:
        _cuda(err, torch.int32, "err")
    num_pages, page_size, hkv, d = k_pool.shape
    b, hq, _ = q.shape
    if out.shape != q.shape or block_tables.shape[0] != b or (
            k_new is not None and (k_new.shape != (b, hkv, d) or
                                   v_new.shape != k_new.shape)):
        raise ValueError("shape mismatch")
    _check(lib.tv_paged_decode_balanced(
        _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pool),
        _ptr(v_pool), _ptr(block_tables), block_tables.shape[1],
        _ptr(context_lens), b, hq, hkv, d, page_size, num_pages, float(scale),
        _ptr(workspace), workspace.numel(), _ptr(err), _stream(stream)),
        "tv_paged_decode_balanced")


# ---- device page pool --------------------------------------------------------

POOL_MAX_SEQS = 1024   # TV_POOL_MAX_SEQS


def pool_state_ints(num_pages):
    """TV_POOL_STATE_INTS(num_pages) of include/tv.h."""
    return 4 + 4 * int(num_pages) + POOL_MAX_SEQS


def pool_state(num_pages, device=None):
    """An (uninitialised) pool state array for tv_pool_init."""
    return torch.zeros(pool_state_ints(num_pages), dtype=torch.int32,
                       device=device or "cuda")


def _pool_tables(block_tables, context_lens):
    _cuda(block_tables, torch.int32, "block_tables")
    _cuda(context_lens, torch.int32, "context_lens")
    if block_tables.shape[0] != context_lens.shape[0]:
        raise ValueError("block_tables and context_lens disagree on num_seqs")
    return block_tables.shape[1], block_tables.shape[0]


def _pool_pages(state):
    _cuda(state, torch.int32, "pool_state")
    n = state.numel() - 4 - POOL_MAX_SEQS
    if n <= 0 or n % 4:
        raise ValueError("pool_state must hold TV_POOL_STATE_INTS(num_pages)"
                         " = 4 + 4 * num_pages + 1024 ints")
    return n // 4


def tv_pool_init(state, block_tables=None, context_lens=None, err=None,
                 stream=None, page_size=16):
    lib = load()
    num_pages = _pool_pages(state)
    mb, b = (_pool_tables(block_tables, context_lens)
             if block_tables is not None else (0, 0))
    if err is not None:
        _cuda(err, torch.int32, "err")
    _check(lib.tv_pool_init(_ptr(state), num_pages, int(page_size),
                            _ptr(block_tables), mb,
                            _ptr(context_lens), b, _ptr(err),
                            _stream(stream)), "tv_pool_init")


def tv_pool_append_slots(state, block_tables, context_lens, k_pool, v_pool,
                         num_new_tokens=None, slot_mapping=None, err=None,
                         stream=None):
    lib = load()
    num_pages = _pool_pages(state)
    mb, b = _pool_tables(block_tables, context_lens)
    _cuda(k_pool, torch.bfloat16, "k_pool"), _cuda(v_pool, torch.bfloat16,
                                                   "v_pool")
    if k_pool.shape[0] != num_pages:
        raise ValueError("pool_state and k_pool disagree on num_pages")
    for n, t in (("num_new_tokens", num_new_tokens),
                 ("slot_mapping", slot_mapping), ("err", err)):
        if t is not None:
            _cuda(t, torch.int32, n)
    _, ps, hkv, d = k_pool.shape
    _check(lib.tv_pool_append_slots(
        _ptr(state), num_pages, _ptr(block_tables), mb, _ptr(context_lens),
        _ptr(num_new_tokens), b, _ptr(slot_mapping), _ptr(k_pool),
        _ptr(v_pool), hkv, d, ps, _ptr(err), _stream(stream)),
        "tv_pool_append_slots")


def tv_pool_fork(state, block_tables, context_lens, src_seqs, dst_seqs,
                 err=None, stream=None):
    lib = load()
    num_pages = _pool_pages(state)
    mb, b = _pool_tables(block_tables, context_lens)
    _cuda(src_seqs, torch.int32, "src_seqs"), _cuda(dst_seqs, torch.int32,
                                                    "dst_seqs")
    if src_seqs.shape != dst_seqs.shape:
        raise ValueError("src_seqs and dst_seqs differ in length")
    if err is not None:
        _cuda(err, torch.int32, "err")
    _check(lib.tv_pool_fork(_ptr(state), num_pages, _ptr(block_tables), mb,
                            _ptr(context_lens), b, _ptr(src_seqs),
                            _ptr(dst_seqs), src_seqs.numel(), _ptr(err),
                            _stream(stream)), "tv_pool_fork")


def tv_pool_release(state, block_tables, context_lens, seqs, err=None,
                    stream=None):
    lib = load()
    num_pages = _pool_pages(state)
    mb, b = _pool_tables(block_tables, context_lens)
    _cuda(seqs, torch.int32, "seqs")
    if err is not None:
        _cuda(err, torch.int32, "err")
    _check(lib.tv_pool_release(_ptr(state), num_pages, _ptr(block_tables), mb,
                               _ptr(context_lens), b, _ptr(seqs), seqs.numel(),
                               _ptr(err), _stream(stream)), "tv_pool_release")


def tv_decode_step(state, out, q, k_new, v_new, k_pool, v_pool, block_tables,
                   context_lens, scale, workspace=None, err=None, stream=None):
    """Room for one new token per live sequence, then the fused append +
    decode (two launches, no host synchronisation); with a workspace the
    decode runs on the work-balanced grid."""
    lib = load()
    num_pages = _pool_pages(state)
    mb, b = _pool_tables(block_tables, context_lens)
    bf = torch.bfloat16
    for n, t in (("out", out), ("q", q), ("k_new", k_new), ("v_new", v_new),
                 ("k_pool", k_pool), ("v_pool", v_pool)):
        _cuda(t, bf, n)
    if err is not None:
        _cuda(err, torch.int32, "err")
    if workspace is not None:
        _cuda(workspace, torch.uint8, "workspace")
    _, ps, hkv, d = k_pool.shape
    hq = q.shape[1]
    if out.shape != q.shape or q.shape[0] != b or k_new.shape != (b, hkv, d):
        raise ValueError("shape mismatch")
    _check(lib.tv_decode_step(
        _ptr(state), num_pages, _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new),
        _ptr(k_pool), _ptr(v_pool), _ptr(block_tables), mb,
        _ptr(context_lens), b, hq, hkv, d, ps, float(scale), _ptr(workspace),
        workspace.numel() if workspace is not None else 0, _ptr(err),
        _stream(stream)), "tv_decode_step")


def tv_selftest_wait_timeout(err, limit_ns, waited_ns=None, stream=None):
    """Run the bounded-wait self-test (see include/tv.h)."""
    lib = load()
    _cuda(err, torch.int32, "err")
    if waited_ns is not None:
        _cuda(waited_ns, torch.int64, "waited_ns")
    _check(lib.tv_selftest_wait_timeout(_ptr(err), int(limit_ns),
                                        _ptr(waited_ns), _stream(stream)),
           "tv_selftest_wait_timeout")
