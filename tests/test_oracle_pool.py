"""Pins of the page-pool model (oracle/pool.py).

The pool is pinned against things it does not compute itself:
  * a contiguous-cache model: every sequence also keeps its own list of K/V
    rows; after every operation, the rows gathered through its block table
    must equal that list (sharing and copy-on-write never let one sequence
    see another's writes);
  * conservation: free pages + referenced pages = the pool, and each page's
    count equals the number of table rows that hold it;
  * small cases worked out by hand from the stated rules (pop order, the
    all-or-nothing batch order, the push order of released pages).
"""
import numpy as np
import pytest

from oracle.pool import PAGE, PagePool, pages_for

H, D = 2, 4   # a small pool: 2 KV heads x 4 dims per row


def _fresh(num_pages, batch, max_blocks, page_size=PAGE):
    bt = np.full((batch, max_blocks), -1, np.int64)
    ctx = np.zeros(batch, np.int64)
    kp = np.zeros((num_pages, page_size, H, D), np.int64)
    return (PagePool(num_pages, page_size=page_size), bt, ctx, kp,
            kp.copy())


def _check_conservation(pool, bt, ctx):
    held = np.zeros(pool.num_pages, np.int64)
    for s in range(len(ctx)):
        for b in range(pages_for(ctx[s], pool.ps)):
            held[bt[s][b]] += 1
    np.testing.assert_array_equal(held, pool.ref)
    assert len(set(pool.stack)) == pool.top
    assert all(pool.ref[p] == 0 for p in pool.stack)
    assert pool.top + int((held > 0).sum()) == pool.num_pages


def _gather(kp, bt, s, ctx):
    ps = kp.shape[1]
    return [kp[bt[s][t // ps], t % ps].copy() for t in range(ctx)]


def test_fresh_pool_hands_out_pages_in_order_and_maps_slots():
    pool, bt, ctx, kp, vp = _fresh(8, 3, 4)
    slots, served = pool.append_slots(bt, ctx, [1, 17, 16], kp, vp)
    assert served.all()
    assert bt[0][:1].tolist() == [0]
    assert bt[1][:2].tolist() == [1, 2]
    assert bt[2][:1].tolist() == [3]
    assert ctx.tolist() == [1, 17, 16]
    want = [0] + list(range(16, 32)) + [32] + list(range(48, 64))
    assert slots.tolist() == want
    assert pool.stack == [7, 6, 5, 4]          # next pop: 4
    _check_conservation(pool, bt, ctx)


def test_batch_order_all_or_nothing_when_the_pool_runs_out():
    pool, bt, ctx, kp, vp = _fresh(4, 3, 4)
    # needs 1, 3, 1 pages with 4 free: seq 0 and 1 are served, 2 is not
    _, served = pool.append_slots(bt, ctx, [5, 40, 1], kp, vp)
    assert served.tolist() == [True, True, False]
    assert ctx.tolist() == [5, 40, 0]
    # needs 5 then 1: the first cannot be served, so neither is the second
    pool, bt, ctx, kp, vp = _fresh(4, 2, 8)
    _, served = pool.append_slots(bt, ctx, [70, 1], kp, vp)
    assert served.tolist() == [False, False]
    assert pool.top == 4 and ctx.tolist() == [0, 0]


def test_released_pages_return_in_ascending_order():
    pool, bt, ctx, kp, vp = _fresh(10, 2, 4)
    pool.append_slots(bt, ctx, [33, 16], kp, vp)   # seq 0: 0,1,2; seq 1: 3
    pool.release(bt, ctx, [0])
    assert pool.stack == [9, 8, 7, 6, 5, 4, 0, 1, 2]   # next pop: 2
    assert ctx[0] == 0 and (bt[0] == -1).all()
    _check_conservation(pool, bt, ctx)


def test_fork_then_both_append_copies_on_write_once():
    pool, bt, ctx, kp, vp = _fresh(8, 2, 4)
    pool.append_slots(bt, ctx, [20, 0], kp, vp)     # pages 0, 1; page 1 partial
    pool.fork(bt, ctx, [(0, 1)])
    assert pool.ref[0] == 2 and pool.ref[1] == 2
    pool.append_slots(bt, ctx, [1, 1], kp, vp)
    # seq 0 (first in batch order) copies the shared partial page; seq 1,
    # now its only holder, writes into page 1 in place
    assert bt[0][:2].tolist() == [0, 2] and bt[1][:2].tolist() == [0, 1]
    assert pool.ref[[0, 1, 2]].tolist() == [2, 1, 1]
    _check_conservation(pool, bt, ctx)


def test_fork_then_only_the_child_appends():
    pool, bt, ctx, kp, vp = _fresh(8, 2, 4)
    pool.append_slots(bt, ctx, [20, 0], kp, vp)
    pool.fork(bt, ctx, [(0, 1)])
    pool.append_slots(bt, ctx, [0, 1], kp, vp)
    assert bt[0][:2].tolist() == [0, 1] and bt[1][:2].tolist() == [0, 2]
    _check_conservation(pool, bt, ctx)


def test_page_size_32_pops_and_slots():
    pool, bt, ctx, kp, vp = _fresh(8, 2, 4, page_size=32)
    slots, _ = pool.append_slots(bt, ctx, [33, 32], kp, vp)
    assert bt[0][:2].tolist() == [0, 1] and bt[1][:1].tolist() == [2]
    assert slots.tolist() == list(range(0, 33)) + list(range(64, 96))
    _check_conservation(pool, bt, ctx)


def test_full_shared_pages_are_not_copied():
    pool, bt, ctx, kp, vp = _fresh(8, 2, 4)
    pool.append_slots(bt, ctx, [32, 0], kp, vp)     # two full pages
    pool.fork(bt, ctx, [(0, 1)])
    pool.append_slots(bt, ctx, [1, 1], kp, vp)      # both open a new page
    assert bt[0][:3].tolist() == [0, 1, 2] and bt[1][:3].tolist() == [0, 1, 3]
    assert pool.ref[[0, 1]].tolist() == [2, 2]
    _check_conservation(pool, bt, ctx)


@pytest.mark.parametrize("seed,page_size", [(1, 16), (2, 16), (3, 32)])
def test_random_operations_match_a_contiguous_cache(seed, page_size):
    rng = np.random.default_rng(seed)
    batch, max_blocks, num_pages = 12, 24, 200
    pool, bt, ctx, kp, vp = _fresh(num_pages, batch, max_blocks, page_size)
    model = [[] for _ in range(batch)]      # contiguous K rows per sequence
    counter = 1
    for step in range(120):
        op = rng.random()
        if op < 0.6:
            n = np.where(rng.random(batch) < 0.7,
                         rng.integers(1, 40, batch), 0)
            n = np.minimum(n, max_blocks * page_size - ctx)
            before = ctx.copy()
            slots, served = pool.append_slots(bt, ctx, n, kp, vp)
            # write the new rows through the slot mapping
            k = 0
            for s in range(batch):
                if not served[s] or n[s] <= 0:
                    continue
                for t in range(before[s], before[s] + n[s]):
                    row = np.full((H, D), counter, np.int64)
                    counter += 1
                    sl = slots[k]
                    k += 1
                    assert sl == (bt[s][t // page_size] * page_size +
                                  t % page_size)
                    kp[sl // page_size, sl % page_size] = row
                    model[s].append(row)
            assert k == len(slots)
        elif op < 0.8:
            live = [s for s in range(batch) if ctx[s] > 0]
            empty = [s for s in range(batch) if ctx[s] == 0]
            if live and empty:
                src, dst = int(rng.choice(live)), int(rng.choice(empty))
                pool.fork(bt, ctx, [(src, dst)])
                model[dst] = [r.copy() for r in model[src]]
        else:
            live = [s for s in range(batch) if ctx[s] > 0]
            if live:
                rel = sorted(rng.choice(live, size=min(2, len(live)),
                                        replace=False).tolist())
                pool.release(bt, ctx, rel)
                for s in rel:
                    model[s] = []
        _check_conservation(pool, bt, ctx)
        for s in range(batch):
            got = _gather(kp, bt, s, int(ctx[s]))
            assert len(got) == len(model[s])
            for a, b in zip(got, model[s]):
                np.testing.assert_array_equal(a, b)
