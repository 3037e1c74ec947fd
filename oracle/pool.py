"""Sequential model of the KV page pool: free pages, per-page reference counts,
on-demand allocation, copy-on-write sharing and release.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``): the tests and the
benchmark's CPU-baseline leg are the only callers; the product library never
imports it.

What it follows.  "Tiny-vLLM 实战：用 C++/CUDA 手写高性能 LLM 推理引擎",
sec. 内存池管理: the KV cache is cut into fixed-size pages; when a request
produces a new token a page is allocated on demand; when a request ends its
pages go back to the free pool; different requests may share the same pages
(prefix caching); the pool's core structure is a list of free pages.
"tiny-vllm：从零构建高性能LLM推理引擎的完整指南", sec. PagedAttention：从操作系统
借来的智慧: pages are allocated only when needed, and sharing is made safe with
copy-on-write.

Where the pages stop, the readings taken (each also listed in the design
notes):
  * the free list is a LIFO stack: ``stack[0 .. top)``; a pop takes
    ``stack[top - 1]``.  ``init`` stacks the free pages in descending id
    order, so a fresh pool hands out pages 0, 1, 2, ...
  * a page's reference count is the number of block-table rows that hold it.
  * ``append_slots`` (room for ``n[s]`` new tokens at positions
    ``ctx .. ctx + n - 1`` of every sequence, in batch order): a sequence first
    copies-on-write the partly filled page it will write into when that page
    is shared (reference count > 1 at its turn), then takes one new page for
    every page boundary it crosses; it is served all-or-nothing, and once one
    sequence cannot be served (too few free pages) no later one in the batch
    is (the needs are reserved in batch order).  Pops go in batch order, the
    copy before the new pages.  ``context_lens[s] += n[s]`` for served
    sequences; ``slot_mapping`` lists the slots of the new tokens in batch
    order.
  * ``release``: every page reference of the listed sequences is dropped;
    pages whose count reaches zero return to the stack in ascending page id
    order; the rows become empty (context 0, entries -1).
  * ``fork``: the destination (empty) sequence takes the source's pages and
    context; every shared page's count grows by one.
"""
from __future__ import annotations

import numpy as np

PAGE = 16


def pages_for(ctx: int, page_size: int = PAGE) -> int:
    return (int(ctx) + page_size - 1) // page_size


class PagePool:
    """Free-page stack and reference counts of a pool of ``num_pages``."""

    def __init__(self, num_pages: int, block_tables=None, context_lens=None,
                 page_size: int = PAGE):
        self.num_pages = int(num_pages)
        self.ps = int(page_size)
        self.ref = np.zeros(self.num_pages, np.int64)
        if block_tables is not None:
            for s, ctx in enumerate(np.asarray(context_lens)):
                for b in range(pages_for(ctx, self.ps)):
                    self.ref[int(block_tables[s][b])] += 1
        free = [p for p in range(self.num_pages) if self.ref[p] == 0]
        self.stack = list(reversed(free))     # top of stack = smallest id

    @property
    def top(self) -> int:
        return len(self.stack)

    def _pop(self) -> int:
        return self.stack.pop()

    def append_slots(self, block_tables, context_lens, n_new, k_pool=None,
                     v_pool=None):
        """Make room for n_new[s] tokens per sequence (in place on the
        tables, lengths and pools).  Returns (slot_mapping, served mask)."""
        bt, ctx = block_tables, context_lens
        ps = self.ps
        n_new = np.asarray(n_new, np.int64)
        # needs, reserved in batch order (all-or-nothing per sequence)
        ref_seen = self.ref.copy()     # counts as each sequence sees them
        need = np.zeros(len(ctx), np.int64)
        cow = np.zeros(len(ctx), bool)
        for s in range(len(ctx)):
            c, n = int(ctx[s]), int(n_new[s])
            if n <= 0:
                continue
            if c % ps:
                p = int(bt[s][c // ps])
                if ref_seen[p] > 1:
                    cow[s] = True
                    ref_seen[p] -= 1
            need[s] = int(cow[s]) + pages_for(c + n, ps) - pages_for(c, ps)
        served = np.zeros(len(ctx), bool)
        used = 0
        for s in range(len(ctx)):
            if used + need[s] > self.top:
                break
            served[s] = True
            used += need[s]
        slots = []
        for s in range(len(ctx)):
            c, n = int(ctx[s]), int(n_new[s])
            if n <= 0 or not served[s]:
                continue
            if cow[s]:
                old = int(bt[s][c // ps])
                new = self._pop()
                self.ref[old] -= 1
                self.ref[new] = 1
                bt[s][c // ps] = new
                if k_pool is not None:
                    k_pool[new] = k_pool[old]
                    v_pool[new] = v_pool[old]
            for b in range(pages_for(c, ps), pages_for(c + n, ps)):
                new = self._pop()
                self.ref[new] = 1
                bt[s][b] = new
            for t in range(c, c + n):
                slots.append(int(bt[s][t // ps]) * ps + t % ps)
            ctx[s] = c + n
        return np.array(slots, np.int32), served

    def release(self, block_tables, context_lens, seqs):
        """Drop every page reference of the sequences ``seqs``."""
        freed = set()
        for s in seqs:
            for b in range(pages_for(context_lens[s], self.ps)):
                p = int(block_tables[s][b])
                self.ref[p] -= 1
                if self.ref[p] == 0:
                    freed.add(p)
            block_tables[s][:] = -1
            context_lens[s] = 0
        for p in sorted(freed):
            self.stack.append(p)

    def fork(self, block_tables, context_lens, pairs):
        """For every (src, dst): dst (empty) shares src's pages."""
        for src, dst in pairs:
            n = pages_for(context_lens[src], self.ps)
            block_tables[dst][:] = -1
            block_tables[dst][:n] = block_tables[src][:n]
            for b in range(n):
                self.ref[int(block_tables[src][b])] += 1
            context_lens[dst] = context_lens[src]
