"""Seeded synthetic inputs for the paged-attention hot path.

This module only *builds inputs*: lengths, a shuffled page assignment (the
block tables), the matching slot mapping for the tokens to append, and bf16
values drawn from N(0, 1).  It holds none of the attention arithmetic.  Both
the CUDA path and the CPU oracle are fed from here.

Shapes follow the Llama-3.2-1B attention layer the source pages use
("tiny-vllm：从零构建高性能LLM推理引擎的完整指南", sec. "Llama 3.2 1B架构拆解":
32 query heads sharing 8 KV heads; head_dim 64) and the 16-token page of
"Tiny-vLLM 实战：用 C++/CUDA 手写高性能 LLM 推理引擎", sec. "内存池管理".

Recipe (all arrays numpy; bf16 travels as uint16 bit patterns):
  * rng = numpy.random.Generator(PCG64(seed));
  * lengths as stated per workload;
  * physical pages: perm = rng.permutation(num_pages); sequence s takes the
    next ceil(len_s / page_size) ids of perm, in order, as its block-table
    row; unused table entries are -1;
  * values: float32 standard normals rounded to bf16 (nearest even), in
    (sequence, position) order, one stream per tensor (tag 0 = cached K,
    1 = cached V, 2 = q, 3 = k_new, 4 = v_new); chunk i of 2^22 values of
    stream t comes from PCG64(SeedSequence(seed, spawn_key=(t, i)));
  * every pool slot that holds no cached token is bf16 NaN (0x7FC0), so a
    kernel that reads a slot it must not read produces NaN.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field

import numpy as np

NUM_Q_HEADS = 32
NUM_KV_HEADS = 8
HEAD_DIM = 64
PAGE_SIZE = 16
SCALE = 1.0 / 8.0
BF16_NAN = np.uint16(0x7FC0)
SEED_BASE = 376_000


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest even) and return the uint16 bits.
    Inputs are finite normals, so no NaN/Inf handling is needed."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns as float64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


_CHUNK = 1 << 22


def _normal_bf16(seed: int, tag: int, shape) -> np.ndarray:
    """bf16 N(0,1) values for stream ``tag``: chunk i of 2^22 values comes
    from PCG64(SeedSequence(seed, spawn_key=(tag, i))), so chunks are
    independent and are drawn on several host threads."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)

    def fill(i):
        g = np.random.Generator(np.random.PCG64(
            np.random.SeedSequence(seed, spawn_key=(tag, i))))
        lo = i * _CHUNK
        m = min(_CHUNK, n - lo)
        out[lo:lo + m] = bf16_bits(g.standard_normal(m, dtype=np.float32))

    nchunks = -(-n // _CHUNK)
    if nchunks <= 1:
        for i in range(nchunks):
            fill(i)
    else:
        from concurrent.futures import ThreadPoolExecutor
        workers = min(16, os.cpu_count() or 1, nchunks)
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, range(nchunks)))
    return out.reshape(shape)


@dataclass
class Workload:
    """One batch of inputs.  ``k_pool``/``v_pool`` hold the cache *before* the
    append; ``context_lens`` counts tokens *after* it."""
    name: str
    seed: int
    q: np.ndarray                 # [rows][Hq][D] uint16
    k_pool: np.ndarray            # [NP][PS][Hkv][D] uint16
    v_pool: np.ndarray
    block_tables: np.ndarray      # [B][MB] int32, -1 = unused
    context_lens: np.ndarray      # [B] int32, after the append
    k_new: np.ndarray             # [T][Hkv][D] uint16
    v_new: np.ndarray
    slot_mapping: np.ndarray      # [T] int32
    query_start_loc: np.ndarray   # [B+1] int32 (rows of q per sequence)
    scale: float = SCALE
    partition_tokens: int = 0     # split-KV partition size (0 = unsplit)
    kind: str = "decode"          # "decode" or "prefill"
    info: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_pages(self) -> int:
        return int(self.k_pool.shape[0])

    @property
    def page_size(self) -> int:
        return int(self.k_pool.shape[1])

    @property
    def num_kv_heads(self) -> int:
        return int(self.k_pool.shape[2])

    @property
    def head_dim(self) -> int:
        return int(self.k_pool.shape[3])

    @property
    def num_q_heads(self) -> int:
        return int(self.q.shape[1])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    def max_partitions(self) -> int:
        if not self.partition_tokens:
            return 1
        return max(1, -(-int(self.context_lens.max()) // self.partition_tokens))

    def kv_bytes_read(self) -> int:
        """Algorithmic K+V bytes one attention pass reads: every cached
        token's row for every KV head, once for K and once for V."""
        per_tok = 2 * self.num_kv_heads * self.head_dim * 2
        return int(self.context_lens.astype(np.int64).sum()) * per_tok

    def append_bytes(self) -> int:
        """Bytes the append moves: read k_new+v_new, write the same."""
        t = int((self.slot_mapping >= 0).sum())
        return 2 * 2 * t * self.num_kv_heads * self.head_dim * 2

    def prefill_flops(self) -> int:
        """Causal algorithmic flops: 4*D per (query row, head, visible key)."""
        ctx = self.context_lens.astype(np.int64)
        qsl = self.query_start_loc.astype(np.int64)
        total = 0
        for s in range(self.num_seqs):
            t = int(qsl[s + 1] - qsl[s])
            p = int(ctx[s]) - t
            keys = t * p + t * (t + 1) // 2
            total += keys
        return 4 * self.head_dim * self.num_q_heads * total


def _assign_pages(rng, lengths, num_pages, page_size):
    blocks = [-(-int(n) // page_size) for n in lengths]
    need = sum(blocks)
    if need > num_pages:
        raise ValueError(f"pool of {num_pages} pages cannot hold {need}")
    mb = max(1, max(blocks) if blocks else 1)
    perm = rng.permutation(num_pages).astype(np.int32)
    bt = np.full((len(lengths), mb), -1, dtype=np.int32)
    cur = 0
    for s, nb in enumerate(blocks):
        bt[s, :nb] = perm[cur:cur + nb]
        cur += nb
    return bt


def _slots(block_tables, seq, positions, page_size):
    pos = np.asarray(positions, dtype=np.int64)
    return (block_tables[seq, pos // page_size].astype(np.int64) * page_size
            + pos % page_size)


def _build(name, seed, cached_lens, new_lens, num_pages, *, kind,
           num_q_heads=NUM_Q_HEADS, num_kv_heads=NUM_KV_HEADS,
           head_dim=HEAD_DIM, page_size=PAGE_SIZE, scale=SCALE,
           partition_tokens=0, rng=None, extra_blocks=0):
    """Cache holds ``cached_lens[s]`` tokens of sequence s; ``new_lens[s]``
    tokens are appended (and are the query rows).  Context after the append
    is their sum."""
    rng = rng if rng is not None else np.random.Generator(np.random.PCG64(seed))
    cached = np.asarray(cached_lens, dtype=np.int64)
    new = np.asarray(new_lens, dtype=np.int64)
    ctx = cached + new
    b = ctx.shape[0]
    bt = _assign_pages(rng, ctx, num_pages, page_size)
    if extra_blocks:
        bt = np.concatenate(
            [bt, np.full((b, extra_blocks), -1, dtype=np.int32)], axis=1)
    row = num_kv_heads * head_dim
    k_pool = np.full((num_pages * page_size, row), BF16_NAN, dtype=np.uint16)
    v_pool = np.full((num_pages * page_size, row), BF16_NAN, dtype=np.uint16)
    n_cached = int(cached.sum())
    if n_cached:
        seq_of = np.repeat(np.arange(b), cached)
        pos_of = np.concatenate([np.arange(c) for c in cached])
        slots = _slots(bt, seq_of, pos_of, page_size)
        k_pool[slots] = _normal_bf16(seed, 0, (n_cached, row))
        v_pool[slots] = _normal_bf16(seed, 1, (n_cached, row))
    n_new = int(new.sum())
    q = _normal_bf16(seed, 2, (n_new, num_q_heads, head_dim))
    k_new = _normal_bf16(seed, 3, (n_new, num_kv_heads, head_dim))
    v_new = _normal_bf16(seed, 4, (n_new, num_kv_heads, head_dim))
    if n_new:
        seq_of = np.repeat(np.arange(b), new)
        pos_of = np.concatenate(
            [np.arange(c, c + n) for c, n in zip(cached, new)])
        slot_mapping = _slots(bt, seq_of, pos_of, page_size).astype(np.int32)
    else:
        slot_mapping = np.zeros((0,), dtype=np.int32)
    qsl = np.zeros((b + 1,), dtype=np.int32)
    qsl[1:] = np.cumsum(new)
    return Workload(
        name=name, seed=seed, q=q,
        k_pool=k_pool.reshape(num_pages, page_size, num_kv_heads, head_dim),
        v_pool=v_pool.reshape(num_pages, page_size, num_kv_heads, head_dim),
        block_tables=bt, context_lens=ctx.astype(np.int32),
        k_new=k_new, v_new=v_new, slot_mapping=slot_mapping,
        query_start_loc=qsl, scale=scale, partition_tokens=partition_tokens,
        kind=kind)


def decode_workload(context_lens, num_pages=None, seed=SEED_BASE, name=None,
                    partition_tokens=0, **kw):
    """Decode batch: one new token per sequence (appended at position
    context_len - 1, then attended from there)."""
    ctx = np.asarray(context_lens, dtype=np.int64)
    if (ctx < 1).any():
        raise ValueError("decode contexts include the appended token (>= 1)")
    ps = kw.get("page_size", PAGE_SIZE)
    if num_pages is None:
        num_pages = int(sum(-(-int(n) // ps) for n in ctx))
    return _build(name or f"decode-b{len(ctx)}", seed, ctx - 1,
                  np.ones_like(ctx), num_pages, kind="decode",
                  partition_tokens=partition_tokens, **kw)


def prefill_workload(prefix_lens, chunk_lens, num_pages=None,
                     seed=SEED_BASE, name=None, **kw):
    """Chunked prefill: ``chunk_lens[s]`` new tokens appended after a cached
    prefix of ``prefix_lens[s]`` tokens; the new tokens are the queries."""
    pre = np.asarray(prefix_lens, dtype=np.int64)
    chunk = np.asarray(chunk_lens, dtype=np.int64)
    ps = kw.get("page_size", PAGE_SIZE)
    if num_pages is None:
        num_pages = int(sum(-(-int(n) // ps) for n in pre + chunk))
    return _build(name or f"prefill-b{len(pre)}", seed, pre, chunk,
                  num_pages, kind="prefill", **kw)


# --- the five named workloads ---------------------------------------------

def tiny_decode() -> Workload:
    """4 sequences, contexts {1, 17, 33, 100} after the append, a 64-page
    shuffled pool (13 pages used, the rest NaN)."""
    return decode_workload([1, 17, 33, 100], num_pages=64,
                           seed=SEED_BASE + 1, name="tiny-decode")


def _ps_tag(page_size: int) -> str:
    return "" if page_size == PAGE_SIZE else f"-ps{page_size}"


def llama_decode(batch: int = 64, context: int = 2048,
                 num_pages: int = 16384, page_size: int = PAGE_SIZE
                 ) -> Workload:
    """Llama-3.2-1B-shaped decode: 64 sequences x 2048 tokens, a shuffled
    pool twice the size of the cache (16384 pages of 16 tokens)."""
    num_pages = num_pages * PAGE_SIZE // page_size
    return decode_workload([context] * batch, num_pages=num_pages,
                           seed=SEED_BASE + 2, page_size=page_size,
                           name=f"llama3.2-1b-decode-b{batch}-ctx{context}"
                                + _ps_tag(page_size))


def continuous_mix(batch: int = 256, page_size: int = PAGE_SIZE) -> Workload:
    """Continuous-batching mix: contexts log-uniform in [16, 8192]; a context
    whose appended token would open a new page is bumped by one, so every
    append lands in a partly filled last page."""
    seed = SEED_BASE + 3
    rng = np.random.Generator(np.random.PCG64(seed))
    ctx = np.rint(np.exp(rng.uniform(math.log(16), math.log(8192),
                                     size=batch))).astype(np.int64)
    ctx = np.where((ctx - 1) % PAGE_SIZE == 0, ctx + 1, ctx)
    num_pages = int(sum(-(-int(n) // page_size) for n in ctx))
    return _build(f"continuous-mix-b{batch}" + _ps_tag(page_size), seed,
                  ctx - 1, np.ones_like(ctx), num_pages, kind="decode",
                  rng=rng, page_size=page_size)


def long_split(batch: int = 8, context: int = 131072,
               partition_tokens: int = 512, page_size: int = PAGE_SIZE
               ) -> Workload:
    """Long-context split-KV decode: 8 x 131072 tokens, 512-token
    partitions merged by log-sum-exp."""
    num_pages = batch * context // page_size
    return decode_workload([context] * batch, num_pages=num_pages,
                           seed=SEED_BASE + 4, page_size=page_size,
                           name=f"long-split-b{batch}-ctx{context}"
                                + _ps_tag(page_size),
                           partition_tokens=partition_tokens)


def chunked_prefill(batch: int = 16, chunk: int = 512,
                    max_prefix: int = 4096, page_size: int = PAGE_SIZE
                    ) -> Workload:
    """Chunked prefill: 16 sequences, 512 new tokens each over a cached
    prefix drawn uniformly from {0 .. 4096}."""
    seed = SEED_BASE + 5
    rng = np.random.Generator(np.random.PCG64(seed))
    pre = rng.integers(0, max_prefix + 1, size=batch).astype(np.int64)
    chunks = np.full((batch,), chunk, dtype=np.int64)
    num_pages = int(sum(-(-int(n) // page_size) for n in pre + chunks))
    return _build(f"chunked-prefill-b{batch}-chunk{chunk}"
                  + _ps_tag(page_size), seed, pre, chunks, num_pages,
                  kind="prefill", rng=rng, page_size=page_size)


NAMED = {
    "tiny": tiny_decode,
    "llama": llama_decode,
    "mix": continuous_mix,
    "long": long_split,
    "prefill": chunked_prefill,
}
