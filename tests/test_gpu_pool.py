"""Device page pool (tv_pool_*) and the graph-captured decode step against
the sequential pool model (oracle/pool.py) and the attention oracle.

Allocation is deterministic by construction (scans in batch order), so the
GPU's block tables, reference counts, free stack, slot mappings and pools
must equal the model's bit for bit after every call.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, bf16_bits, err_word, require_gpu
from oracle.pool import PAGE, PagePool
from paged_kv_cache_376_b200 import _lib
from paged_kv_cache_376_b200 import workloads as W

pytestmark = pytest.mark.gpu

HKV, D = 8, 64


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _i32(a):
    return torch.tensor(np.asarray(a, np.int32), device="cuda")


def _bits(a):
    return torch.tensor(np.asarray(a, np.int16).view(np.int16),
                        device="cuda").view(torch.bfloat16)


class Both:
    """The same pool on the GPU and in the model."""

    def __init__(self, num_pages, batch, max_blocks, seed, hkv=HKV):
        rng = np.random.default_rng(seed)
        self.hkv = hkv
        self.np_, self.b, self.mb = num_pages, batch, max_blocks
        self.bt = np.full((batch, max_blocks), -1, np.int64)
        self.ctx = np.zeros(batch, np.int64)
        # pools start as random bf16 bit patterns (no NaN: exponent < 255)
        kp = rng.integers(0, 0x7F00, (num_pages, PAGE, hkv, D)).astype(np.uint16)
        vp = rng.integers(0, 0x7F00, (num_pages, PAGE, hkv, D)).astype(np.uint16)
        self.kp, self.vp = kp, vp
        self.pool = PagePool(num_pages)
        self.g_state = _lib.pool_state(num_pages)
        self.g_bt = _i32(self.bt)
        self.g_ctx = _i32(self.ctx)
        self.g_kp = _bits(kp.view(np.int16))
        self.g_vp = _bits(vp.view(np.int16))
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        # growth marks: 1 where the last append call gave a sequence tokens
        self.grown = np.zeros(batch, np.int32)
        _lib.tv_pool_init(self.g_state, err=self.err)

    def check(self):
        torch.cuda.synchronize()
        np.testing.assert_array_equal(self.g_bt.cpu().numpy(), self.bt)
        np.testing.assert_array_equal(self.g_ctx.cpu().numpy(), self.ctx)
        st = self.g_state.cpu().numpy()
        top = int(st[0])
        assert top == self.pool.top
        np.testing.assert_array_equal(st[4:4 + top], self.pool.stack)
        n = self.np_
        np.testing.assert_array_equal(st[4 + n:4 + 2 * n], self.pool.ref)
        # the scratch words are back at zero
        assert not st[4 + 2 * n:4 + 4 * n].any()
        np.testing.assert_array_equal(st[4 + 4 * n:4 + 4 * n + self.b],
                                      self.grown)
        np.testing.assert_array_equal(bf16_bits(self.g_kp), self.kp)
        np.testing.assert_array_equal(bf16_bits(self.g_vp), self.vp)

    def append(self, n_new, rng=None):
        before = self.ctx.copy()
        slots, served = self.pool.append_slots(self.bt, self.ctx, n_new,
                                               self.kp, self.vp)
        g_slots = torch.full((int(np.maximum(n_new, 0).sum()) + 1,), -7,
                             dtype=torch.int32, device="cuda")
        _lib.tv_pool_append_slots(self.g_state, self.g_bt, self.g_ctx,
                                  self.g_kp, self.g_vp,
                                  num_new_tokens=_i32(n_new),
                                  slot_mapping=g_slots, err=self.err)
        torch.cuda.synchronize()
        self.grown = (served & (np.asarray(n_new) > 0)).astype(np.int32)
        assert int(self.g_state[2]) == len(slots)
        np.testing.assert_array_equal(g_slots[:len(slots)].cpu().numpy(),
                                      slots)
        if rng is not None and len(slots):
            # write new rows through the slot mapping on both sides
            kn = rng.integers(0, 0x7F00,
                              (len(slots), self.hkv, D)).astype(np.uint16)
            vn = rng.integers(0, 0x7F00,
                              (len(slots), self.hkv, D)).astype(np.uint16)
            self.kp, self.vp, bad = oracle.kv_append(kn, vn, slots, self.kp,
                                                     self.vp)
            assert bad == 0
            _lib.tv_kv_append(_bits(kn.view(np.int16)),
                              _bits(vn.view(np.int16)),
                              _i32(slots), self.g_kp, self.g_vp, err=self.err)
        return served, before

    def fork(self, pairs):
        self.pool.fork(self.bt, self.ctx, pairs)
        src = _i32([a for a, _ in pairs])
        dst = _i32([b for _, b in pairs])
        _lib.tv_pool_fork(self.g_state, self.g_bt, self.g_ctx, src, dst,
                          err=self.err)

    def release(self, seqs):
        self.pool.release(self.bt, self.ctx, seqs)
        _lib.tv_pool_release(self.g_state, self.g_bt, self.g_ctx, _i32(seqs),
                             err=self.err)


def test_fresh_pool_append_matches_the_model():
    p = Both(64, 5, 8, seed=1)
    p.check()
    p.append([1, 17, 16, 0, 33], np.random.default_rng(2))
    p.check()
    assert err_word(p) == 0


def test_fork_then_both_append_copies_on_write():
    p = Both(32, 3, 8, seed=3)
    rng = np.random.default_rng(4)
    p.append([20, 0, 45], rng)
    p.fork([(0, 1)])
    p.check()
    p.append([1, 1, 1], rng)       # seq 0 copies the shared partial page
    p.check()
    assert err_word(p) == 0


def test_pool_exhaustion_is_flagged_in_batch_order():
    p = Both(6, 3, 8, seed=5)
    served, _ = p.append([40, 70, 1])   # needs 3, 5, 1 of 6 pages
    assert served.tolist() == [True, False, False]
    p.check()
    assert err_word(p) & _lib.DEVERR_POOL_EMPTY


def test_init_from_existing_tables():
    wl = W.decode_workload([70, 513, 16, 200], num_pages=80, seed=6)
    bt = torch.tensor(wl.block_tables, device="cuda")
    ctx = torch.tensor(wl.context_lens, device="cuda")
    st = _lib.pool_state(wl.num_pages)
    _lib.tv_pool_init(st, bt, ctx)
    pool = PagePool(wl.num_pages, wl.block_tables, wl.context_lens)
    got = st.cpu().numpy()
    assert int(got[0]) == pool.top
    np.testing.assert_array_equal(got[4:4 + pool.top], pool.stack)
    n = wl.num_pages
    np.testing.assert_array_equal(got[4 + n:4 + 2 * n], pool.ref)


def test_release_of_more_pages_than_the_sorted_list_holds():
    # 8500 pages freed at once: past the 8192-entry list, the kernel scans
    # the whole pool instead; the push order must not change
    p = Both(9000, 3, 8600, seed=7, hkv=1)
    p.append([8500 * PAGE - 3, 40, 0])
    p.fork([(1, 2)])
    p.release([0, 1])
    p.check()
    p.append([0, 0, 1])
    p.check()
    assert err_word(p) == 0


@pytest.mark.parametrize("seed", [11, 12])
def test_random_operations_match_the_model(seed):
    rng = np.random.default_rng(seed)
    batch, mb = 40, 24
    p = Both(300, batch, mb, seed=seed)
    for step in range(40):
        op = rng.random()
        if op < 0.6:
            n = np.where(rng.random(batch) < 0.6,
                         rng.integers(1, 40, batch), 0)
            n = np.minimum(n, mb * PAGE - p.ctx)
            p.append(n, rng)
        elif op < 0.8:
            live = [s for s in range(batch) if p.ctx[s] > 0]
            empty = [s for s in range(batch) if p.ctx[s] == 0]
            k = min(3, len(live), len(empty))
            if k:
                src = rng.choice(live, size=k).tolist()
                dst = rng.choice(empty, size=k, replace=False).tolist()
                p.fork(list(zip(src, dst)))
        else:
            live = [s for s in range(batch) if p.ctx[s] > 0]
            if live:
                rel = rng.choice(live, size=min(3, len(live)),
                                 replace=False).tolist()
                p.release(rel)
        p.check()
    assert (err_word(p) & ~_lib.DEVERR_POOL_EMPTY) == 0


@pytest.mark.parametrize("balanced", [False, True],
                         ids=["per-pair", "balanced"])
def test_graph_captured_decode_steps_match_the_oracle(balanced):
    """A decode loop: every step is tv_decode_step (room for the token, then
    the fused append + attention) replayed from one CUDA graph with new
    inputs copied into its buffers; a fork in the middle makes the next
    step copy-on-write a shared page."""
    lens = [5, 16, 17, 100, 31, 1, 64, 0]
    batch, mb, steps = len(lens), 16, 12
    rng = np.random.default_rng(21)
    # the workload caches n tokens of each sequence (position n, where this
    # step appends, is the workload's own unfilled slot)
    wl = W.decode_workload([n + 1 for n in lens], num_pages=120, seed=22)
    bt = np.full((batch, mb), -1, np.int64)
    bt[:, :wl.block_tables.shape[1]] = wl.block_tables
    ctx = np.asarray(lens, np.int64)
    bt[7, :] = -1
    kp, vp = wl.k_pool.copy(), wl.v_pool.copy()
    pool = PagePool(wl.num_pages, bt, ctx)

    g = dict(bt=_i32(bt), ctx=_i32(ctx), kp=_bits(kp.view(np.int16)),
             vp=_bits(vp.view(np.int16)),
             q=torch.empty((batch, 32, D), dtype=torch.bfloat16, device="cuda"),
             kn=torch.empty((batch, HKV, D), dtype=torch.bfloat16,
                            device="cuda"),
             vn=torch.empty((batch, HKV, D), dtype=torch.bfloat16,
                            device="cuda"),
             out=torch.empty((batch, 32, D), dtype=torch.bfloat16,
                             device="cuda"))
    st = _lib.pool_state(wl.num_pages)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.tv_pool_init(st, g["bt"], g["ctx"])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    ws = _lib.decode_workspace(batch, 32, HKV) if balanced else None
    with torch.cuda.graph(graph, stream=side):
        _lib.tv_decode_step(st, g["out"], g["q"], g["kn"], g["vn"], g["kp"],
                            g["vp"], g["bt"], g["ctx"], wl.scale,
                            workspace=ws, err=err)
    torch.cuda.synchronize()

    def draw(shape):
        f = rng.standard_normal(shape).astype(np.float32)
        return W.bf16_bits(f)

    for step in range(steps):
        if step == 5:
            # seq 7 (idle) becomes a fork of seq 3; both then write into the
            # shared last page, so seq 3 copies it on its next step
            pool.fork(bt, ctx, [(3, 7)])
            _lib.tv_pool_fork(st, g["bt"], g["ctx"], _i32([3]), _i32([7]))
        q, kn, vn = draw((batch, 32, D)), draw((batch, HKV, D)), \
            draw((batch, HKV, D))
        g["q"].copy_(_bits(q.view(np.int16)))
        g["kn"].copy_(_bits(kn.view(np.int16)))
        g["vn"].copy_(_bits(vn.view(np.int16)))
        graph.replay()
        torch.cuda.synchronize()
        # the model: room for one token per live sequence, append, attend
        live = (ctx > 0).astype(np.int64)
        before = ctx.copy()
        slots, served = pool.append_slots(bt, ctx, live, kp, vp)
        assert served[live > 0].all()
        sl = np.full(batch, -1, np.int32)
        for s in range(batch):
            if live[s]:
                t = ctx[s] - 1
                sl[s] = bt[s][t // PAGE] * PAGE + t % PAGE
        kp, vp, bad = oracle.kv_append(kn, vn, sl, kp, vp)
        assert bad == 0
        ref = oracle.paged_decode(q, kp, vp, bt.astype(np.int32),
                                  ctx.astype(np.int32), wl.scale)
        np.testing.assert_array_equal(g["bt"].cpu().numpy(), bt)
        np.testing.assert_array_equal(g["ctx"].cpu().numpy(), ctx)
        np.testing.assert_array_equal(bf16_bits(g["kp"]), kp)
        np.testing.assert_array_equal(bf16_bits(g["vp"]), vp)
        assert_parity(g["out"], ref, f"decode step {step}")
    assert int(err.item()) == 0


@pytest.mark.parametrize("balanced", [False, True],
                         ids=["per-pair", "balanced"])
def test_exhausted_pool_leaves_unserved_sequences_untouched(balanced):
    """An exhausted pool inside graph-replayed decode steps: a sequence that
    gets no room for its token (and every later one in batch order) is idle
    for the step -- its cached rows, its context and the pages it shares
    with a fork stay bit for bit as they were, and its output row is zero --
    while the served ones append and attend as the oracle says.  Pages are
    released between steps until everyone is served again.

    Sequences (batch order): A (16 cached tokens: its next token opens a
    page), B = fork of A, D (20 cached: its next token goes into a partly
    filled page that E shares, so D must copy it first), E = fork of D.  The
    pool has one free page."""
    batch, mb = 4, 8
    # the workload caches 16 and 20 tokens of A and D (its own append slot
    # at position 16 / 20 is not used here)
    wl = W.decode_workload([17, 21], num_pages=4, seed=31)
    bt = np.full((batch, mb), -1, np.int64)
    ctx = np.zeros(batch, np.int64)
    bt[0, :1] = wl.block_tables[0, :1]
    bt[2, :2] = wl.block_tables[1, :2]
    ctx[0], ctx[2] = 16, 20
    kp, vp = wl.k_pool.copy(), wl.v_pool.copy()
    pool = PagePool(wl.num_pages, bt, ctx)
    assert pool.top == 1
    g = dict(bt=_i32(bt), ctx=_i32(ctx), kp=_bits(kp.view(np.int16)),
             vp=_bits(vp.view(np.int16)),
             q=torch.empty((batch, 32, D), dtype=torch.bfloat16, device="cuda"),
             kn=torch.empty((batch, HKV, D), dtype=torch.bfloat16,
                            device="cuda"),
             vn=torch.empty((batch, HKV, D), dtype=torch.bfloat16,
                            device="cuda"),
             out=torch.empty((batch, 32, D), dtype=torch.bfloat16,
                             device="cuda"))
    st = _lib.pool_state(wl.num_pages)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _lib.tv_pool_init(st, g["bt"], g["ctx"])
    pool.fork(bt, ctx, [(0, 1), (2, 3)])
    _lib.tv_pool_fork(st, g["bt"], g["ctx"], _i32([0, 2]), _i32([1, 3]))

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    ws = _lib.decode_workspace(batch, 32, HKV) if balanced else None
    with torch.cuda.graph(graph, stream=side):
        _lib.tv_decode_step(st, g["out"], g["q"], g["kn"], g["vn"], g["kp"],
                            g["vp"], g["bt"], g["ctx"], wl.scale,
                            workspace=ws, err=err)
    torch.cuda.synchronize()
    rng = np.random.default_rng(32)

    def draw(shape):
        return W.bf16_bits(rng.standard_normal(shape).astype(np.float32))

    # (sequences released before the step, sequences served by the step)
    plan = [([], [0]), ([0], [1]), ([1], [2, 3]), ([], [2, 3])]
    for step, (release, want_served) in enumerate(plan):
        if release:
            pool.release(bt, ctx, release)
            _lib.tv_pool_release(st, g["bt"], g["ctx"], _i32(release))
        q, kn, vn = draw((batch, 32, D)), draw((batch, HKV, D)), \
            draw((batch, HKV, D))
        g["q"].copy_(_bits(q.view(np.int16)))
        g["kn"].copy_(_bits(kn.view(np.int16)))
        g["vn"].copy_(_bits(vn.view(np.int16)))
        g["out"].fill_(float("nan"))
        err.zero_()
        graph.replay()
        torch.cuda.synchronize()
        live = (ctx > 0).astype(np.int64)
        before = ctx.copy()
        _, served = pool.append_slots(bt, ctx, live, kp, vp)
        grown = served & (live > 0)
        assert np.flatnonzero(grown).tolist() == want_served, step
        sl = np.full(batch, -1, np.int32)
        for s in np.flatnonzero(grown):
            t = ctx[s] - 1
            sl[s] = bt[s][t // PAGE] * PAGE + t % PAGE
        kp, vp, bad = oracle.kv_append(kn, vn, sl, kp, vp)
        assert bad == 0
        att_ctx = np.where(grown, ctx, 0).astype(np.int32)
        ref = oracle.paged_decode(q, kp, vp, bt.astype(np.int32), att_ctx,
                                  wl.scale)
        np.testing.assert_array_equal(g["bt"].cpu().numpy(), bt)
        np.testing.assert_array_equal(g["ctx"].cpu().numpy(), ctx)
        # cached rows of every sequence, shared pages included, bit-exact
        np.testing.assert_array_equal(bf16_bits(g["kp"]), kp)
        np.testing.assert_array_equal(bf16_bits(g["vp"]), vp)
        n = wl.num_pages
        np.testing.assert_array_equal(
            st.cpu().numpy()[4 + 4 * n:4 + 4 * n + batch], grown)
        out = g["out"].cpu().float().numpy()
        for s in range(batch):
            if not grown[s]:
                assert (out[s] == 0).all(), (step, s)
        assert_parity(g["out"][torch.tensor(grown, device="cuda")],
                      ref[grown], f"served rows, step {step}")
        want_err = _lib.DEVERR_POOL_EMPTY if step < 2 else 0
        assert int(err.item()) == want_err, step
