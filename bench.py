#!/usr/bin/env python3
"""Benchmark of the paged-attention hot path (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tv|reference]
                    [--workload llama|mix|long|prefill|tiny]

A step is one pass of the hot path over one batch:
  llama / tiny       : the decode step -- append one token per sequence and
                       attend over the whole paged context -- as one launch
                       of tv_paged_decode_append (one CTA per sequence and KV
                       head: equal lengths fill the GPU evenly);
  mix                : the same step as one launch of tv_paged_decode_balanced
                       with k_new/v_new (the work-balanced grid: mixed lengths
                       would leave the one-CTA-per-pair grid with a long
                       tail);
                       --balanced / --per-pair pick either kernel for any
                       decode workload, --unfused runs tv_kv_append +
                       tv_paged_decode;
  long               : tv_kv_append, tv_paged_decode_split (512-token
                       partitions), tv_split_merge;
  prefill            : tv_kv_append of the 512-token chunks, then
                       tv_paged_prefill on the tensor cores.
The default is the Llama-3.2-1B-shaped decode (64 sequences x 2048 tokens).
Single-launch steps are timed as CUDA-graph replays of the K steps (chunks
of up to 200 launches, back to back on one stream; --eager: one host launch
per step with events around it); the end-to-end leg always launches from
the host through the C ABI.
Under torchrun every rank runs its own replica of the batch (sequences are
independent; no collective touches the data path) and the whole-job value
is the units of all ranks over the slowest rank's device time.

--impl reference times the CPU oracle (double precision, the repository's
correctness reference) on a bounded sample of the same workload; only rank 0
runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("paged decode KV-read GB/s (% of B200 HBM peak) and "
          "sequence-steps/s")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# timed regions at least this long are compared with the sustained tensor
# peak (the GPU reaches its power cap within seconds), shorter ones with the
# burst peak
SUSTAINED_S = 1.0


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return (float(p["hbm_gbs"]), float(p["bf16_tflops"]),
                float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "measured")
    except (OSError, KeyError, ValueError):
        return (FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS,
                "fallback")


def _traffic(kernel, workload_name):
    """DRAM bytes per launch of `kernel` on this workload from the committed
    ncu capture (profiles/traffic.json), or None when there is none or when a
    source file of the kernel has changed since the counters were taken."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            entry = json.load(f).get(f"{kernel}@{workload_name}")
        if not entry:
            return None
        for path, digest in entry["sources"].items():
            with open(os.path.join(ROOT, path), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        return int(entry["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        return None


def _roofline_peak(unit, wall_s, hbm, tfl_burst, tfl_sustained):
    """(peak, bound, MEASURED_PEAKS key) for the dominant kernel: HBM for
    byte-bound work; for tensor-bound work the sustained GEMM figure when the
    timed region lasted SUSTAINED_S or more (it then runs under the 1 kW power
    cap, as that figure was measured), else the burst figure."""
    if unit == "GB/s":
        return hbm, "hbm", "hbm_gbs"
    if wall_s >= SUSTAINED_S:
        return tfl_sustained, "tensor", "bf16_tflops_sustained"
    return tfl_burst, "tensor", "bf16_tflops"


def _workload(name, page_size=16):
    from paged_kv_cache_376_b200 import workloads as W
    if name == "tiny":
        if page_size != 16:
            raise SystemExit("the tiny configuration has 16-token pages")
        return W.tiny_decode()
    return {"llama": W.llama_decode, "mix": W.continuous_mix,
            "long": W.long_split, "prefill": W.chunked_prefill}[name](
                page_size=page_size)


def _default_kind(name):
    return {"prefill": "prefill", "long": "split",
            "mix": "balanced"}.get(name, "fused")


def _config(wl, name, kind=None, engine=False):
    kind = kind or _default_kind(name)
    cfg = {"workload": wl.name, "batch": wl.num_seqs,
           "q_heads": wl.num_q_heads, "kv_heads": wl.num_kv_heads,
           "head_dim": wl.head_dim, "page_size": wl.page_size,
           "num_pages": wl.num_pages,
           "context_tokens": int(wl.context_lens.sum())}
    if name in ("llama", "mix", "tiny"):
        cfg["step"] = {
            "decode": "tv_kv_append + tv_paged_decode",
            "fused": "tv_paged_decode_append (fused append + decode, one "
                     "CTA per sequence and KV head)",
            "split": "tv_kv_append + tv_paged_decode_split + "
                     "tv_split_merge",
        }.get(kind, "tv_paged_decode_balanced (fused append + decode, "
                    "work-balanced persistent grid)")
    elif name == "long":
        cfg["step"] = ("tv_kv_append + tv_paged_decode_split + "
                       "tv_split_merge")
        cfg["partition_tokens"] = wl.partition_tokens
    else:
        cfg["step"] = ("tv_kv_append (512-token chunks) + tv_paged_prefill "
                       "(cost-ordered dispatch)")
        cfg["query_rows"] = int(wl.q.shape[0])
    if engine:
        cfg["step"] = ("tv_decode_step: device page pool slot reservation, "
                       "then " + cfg["step"])
        cfg["engine_state"] = (
            "cache one token short of the workload; tables, lengths and "
            f"pool state restored every {TVRunner.ENGINE_ROUND} steps by 3 "
            "device copies inside the timed region, so contexts grow by up "
            f"to {TVRunner.ENGINE_ROUND - 1} tokens within a round")
    kvb = wl.kv_bytes_read()
    cfg["l2"] = (f"inputs larger than L2: {kvb / 1e6:.0f} MB of K/V read per "
                 "step, streamed with an L2 evict-first policy"
                 if not flushes_l2(wl) else
                 f"working set ({working_set_bytes(wl) / 1e6:.0f} MB) under "
                 "2x L2: L2 flushed before every timed step by writing 2x "
                 "the L2 size, outside the step's CUDA events; the step time "
                 "is the mean of the event-timed steps")
    return cfg


L2_BYTES = 126 * 1024 * 1024     # B200; bench.py reads the device's own figure


def working_set_bytes(wl):
    """Bytes a step touches at least once: the cached K/V rows it attends
    over plus q and out."""
    return wl.kv_bytes_read() + 2 * int(wl.q.nbytes)


def flushes_l2(wl, l2_bytes=None):
    """Steps whose working set could stay in L2 from one step to the next
    are timed one by one with L2 flushed in between."""
    return working_set_bytes(wl) < 2 * (l2_bytes or L2_BYTES)


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
             "sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.gpu_index = gpu_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]),
                             float(parts[3]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return None
        busy = [r for r in rows if r[2] >= 50] or rows
        reasons = sorted({self.NAMES[i] for r in busy
                          for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in busy),
                "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(busy)}


# ------------------------------------------------------------------ tv arm --

class TVRunner:
    """Device buffers and the calls of one step, marshalled once so that the
    host submits a step in a few microseconds."""

    ENGINE_ROUND = 64   # engine mode: steps between state restores

    def __init__(self, wl, name, device, unfused=False, split_tokens=0,
                 per_pair=False, balanced=False, engine=False):
        import torch
        from paged_kv_cache_376_b200 import _lib
        from paged_kv_cache_376_b200.device import upload
        self.torch = torch
        self.lib = _lib.load()
        self.wl, self.name, self.device = wl, name, device
        self.db = db = upload(wl, device)
        self.out = torch.empty_like(db.q)
        self.kind = ("prefill" if name == "prefill" else
                     "split" if name == "long" or split_tokens else
                     "decode" if unfused else
                     "fused" if per_pair else
                     "balanced" if balanced else _default_kind(name))
        if self.kind == "balanced":
            self.ws = _lib.decode_workspace(wl.num_seqs, wl.num_q_heads,
                                            wl.num_kv_heads, device)
        if self.kind == "split":
            if split_tokens:
                wl.partition_tokens = split_tokens
            maxp = wl.max_partitions()
            b, hq, d = db.q.shape
            self.po = torch.empty((b, hq, maxp, d), dtype=torch.float32,
                                  device=device)
            self.pl = torch.empty((b, hq, maxp), dtype=torch.float32,
                                  device=device)
            self.maxp = maxp
        self.maxq = int(np.diff(wl.query_start_loc).max())
        if self.kind == "prefill":
            self.pws = _lib.prefill_workspace(wl.num_seqs, self.maxq, device)
        self.stream = torch.cuda.current_stream(device)
        self.engine = engine
        if engine:
            self._setup_engine()

    def _setup_engine(self):
        """Engine mode: the step is tv_decode_step on a device page pool.
        The cache starts one token short of the workload (the step appends
        it); the pools and tables get room for one round of growth, and the
        tables, lengths and pool state are restored after every round so
        each round repeats the same work."""
        torch, db, wl = self.torch, self.db, self.wl
        from paged_kv_cache_376_b200 import _lib
        if self.kind not in ("fused", "balanced"):
            raise SystemExit("--engine needs a decode workload")
        b = wl.num_seqs
        grow = self.ENGINE_ROUND // db.k_pool.shape[1] + 2
        shape = (b * grow,) + tuple(db.k_pool.shape[1:])
        db.k_pool = torch.cat([db.k_pool, torch.zeros(
            shape, dtype=db.k_pool.dtype, device=self.device)])
        db.v_pool = torch.cat([db.v_pool, torch.zeros(
            shape, dtype=db.v_pool.dtype, device=self.device)])
        db.block_tables = torch.cat([db.block_tables, torch.full(
            (b, grow), -1, dtype=torch.int32, device=self.device)], dim=1)
        db.context_lens = (db.context_lens - 1).clamp_(min=0)
        self.pool = _lib.pool_state(db.k_pool.shape[0], self.device)
        _lib.tv_pool_init(self.pool, db.block_tables, db.context_lens,
                          page_size=db.k_pool.shape[1])
        self.saved = (db.block_tables.clone(), db.context_lens.clone(),
                      self.pool.clone())
        self.since_restore = 0
        torch.cuda.synchronize(self.device)

    def restore(self):
        """Engine mode: back to the state at the start of a round."""
        db = self.db
        with self.torch.cuda.stream(self.stream):
            db.block_tables.copy_(self.saved[0])
            db.context_lens.copy_(self.saved[1])
            self.pool.copy_(self.saved[2])
        self.since_restore = 0

    def _p(self, t):
        import ctypes
        return ctypes.c_void_p(t.data_ptr())

    def step(self, timing=None):
        """Launch one step on the current stream.  ``timing`` = (start, end)
        events recorded around the dominant kernel."""
        lib, db, wl = self.lib, self.db, self.wl
        s = self.stream.cuda_stream
        num_pages, ps, hkv, d = db.k_pool.shape
        b, hq = db.context_lens.shape[0], db.q.shape[1]
        mb = db.block_tables.shape[1]
        if self.engine:
            ws = self.ws if self.kind == "balanced" else None
            if timing is not None:
                timing[0].record(self.stream)
            st = lib.tv_decode_step(
                self._p(self.pool), num_pages, self._p(self.out),
                self._p(db.q), self._p(db.k_new), self._p(db.v_new),
                self._p(db.k_pool), self._p(db.v_pool),
                self._p(db.block_tables), mb, self._p(db.context_lens), b, hq,
                hkv, d, ps, wl.scale, self._p(ws) if ws is not None else None,
                ws.numel() if ws is not None else 0, self._p(db.err), s)
            assert st == 0, st
            if timing is not None:
                timing[1].record(self.stream)
            self.since_restore += 1
            if self.since_restore == self.ENGINE_ROUND:
                self.restore()
            return
        if self.kind == "balanced":
            if timing is not None:
                timing[0].record(self.stream)
            st = lib.tv_paged_decode_balanced(
                self._p(self.out), self._p(db.q), self._p(db.k_new),
                self._p(db.v_new), self._p(db.k_pool), self._p(db.v_pool),
                self._p(db.block_tables), mb, self._p(db.context_lens), b, hq,
                hkv, d, ps, num_pages, wl.scale, self._p(self.ws),
                self.ws.numel(), self._p(db.err), s)
            assert st == 0, st
            if timing is not None:
                timing[1].record(self.stream)
            return
        if self.kind == "fused":
            if timing is not None:
                timing[0].record(self.stream)
            st = lib.tv_paged_decode_append(
                self._p(self.out), self._p(db.q), self._p(db.k_new),
                self._p(db.v_new), self._p(db.k_pool), self._p(db.v_pool),
                self._p(db.block_tables), mb, self._p(db.context_lens), b, hq,
                hkv, d, ps, num_pages, wl.scale, self._p(db.err), s)
            assert st == 0, st
            if timing is not None:
                timing[1].record(self.stream)
            return
        st = lib.tv_kv_append(
            self._p(db.k_new), self._p(db.v_new), self._p(db.slot_mapping),
            db.k_new.shape[0], self._p(db.k_pool), self._p(db.v_pool),
            num_pages, hkv, d, ps, self._p(db.err), s)
        assert st == 0, st
        if timing is not None:
            timing[0].record(self.stream)
        if self.kind == "decode":
            st = lib.tv_paged_decode(
                self._p(self.out), self._p(db.q), self._p(db.k_pool),
                self._p(db.v_pool), self._p(db.block_tables), mb,
                self._p(db.context_lens), b, hq, hkv, d, ps, num_pages,
                wl.scale, self._p(db.err), s)
        elif self.kind == "split":
            st = lib.tv_paged_decode_split(
                self._p(self.po), self._p(self.pl), self._p(db.q),
                self._p(db.k_pool), self._p(db.v_pool),
                self._p(db.block_tables), mb, self._p(db.context_lens), b, hq,
                hkv, d, ps, num_pages, wl.scale, wl.partition_tokens,
                self.maxp, self._p(db.err), s)
        else:
            st = lib.tv_paged_prefill(
                self._p(self.out), self._p(db.q), db.q.shape[0],
                self._p(db.query_start_loc), self._p(db.k_pool),
                self._p(db.v_pool), self._p(db.block_tables), mb,
                self._p(db.context_lens), b, self.maxq, hq, hkv, d, ps,
                num_pages, wl.scale, self._p(self.pws), self.pws.numel(),
                self._p(db.err), s)
        assert st == 0, st
        if timing is not None:
            timing[1].record(self.stream)
        if self.kind == "split":
            st = lib.tv_split_merge(
                self._p(self.out), self._p(self.po), self._p(self.pl),
                self._p(db.context_lens), b, hq, d, wl.partition_tokens,
                self.maxp, s)
            assert st == 0, st

    def launches_per_step(self):
        if self.engine:
            return 2
        # prefill: append, the dispatch-order kernel, attention
        return {"split": 3, "fused": 1, "balanced": 1,
                "prefill": 3}.get(self.kind, 2)

    def graph_timed(self):
        """Steps timed by CUDA-graph replay: one launch per step, or the
        engine's two launches with its restores."""
        return self.engine or self.launches_per_step() == 1

    def graphs(self, steps, chunk=200):
        """CUDA graphs that replay exactly ``steps`` steps: a list of
        graphs, each captured from ``chunk`` (or fewer) consecutive steps
        (engine mode: rounds of ENGINE_ROUND steps, each ending with the
        state restore)."""
        torch = self.torch
        if self.engine:
            chunk = self.ENGINE_ROUND
            self.restore()
        cap = torch.cuda.Stream(self.device)
        cap.wait_stream(torch.cuda.current_stream(self.device))
        home, self.stream = self.stream, cap
        made, plan = {}, []
        try:
            left = steps
            while left:
                n = min(chunk, left)
                if n not in made:
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=cap):
                        for _ in range(n):
                            self.step()
                    made[n] = g
                plan.append(made[n])
                left -= n
        finally:
            self.stream = home
        torch.cuda.current_stream(self.device).wait_stream(cap)
        if self.engine:
            self.since_restore = 0
        return plan

    # -- end to end: host inputs in, host result out, through the C ABI ------
    def setup_e2e(self):
        torch = self.torch
        db = self.db
        self.h_in = {}
        if self.engine:
            # the engine's tables, lengths and pool stay on the device
            self.restore()
            names = ("q", "k_new", "v_new")
        else:
            names = None
        names = names or {"fused": ("q", "k_new", "v_new", "block_tables",
                           "context_lens"),
                 "prefill": ("q", "k_new", "v_new", "slot_mapping",
                             "block_tables", "context_lens",
                             "query_start_loc")}.get(
            self.kind, ("q", "k_new", "v_new", "slot_mapping",
                        "block_tables", "context_lens"))
        for name in names:
            t = getattr(db, name)
            self.h_in[name] = torch.empty(t.shape, dtype=t.dtype,
                                          pin_memory=True).copy_(t.cpu())
        self.h_out = torch.empty(self.out.shape, dtype=self.out.dtype,
                                 pin_memory=True)

    def e2e_bytes(self):
        h2d = sum(t.numel() * t.element_size() for t in self.h_in.values())
        d2h = self.h_out.numel() * self.h_out.element_size()
        return h2d, d2h

    def e2e_step(self):
        """Serial end-to-end step: copies in, the step, result out, all on the
        step's stream."""
        db = self.db
        for name, h in self.h_in.items():
            getattr(db, name).copy_(h, non_blocking=True)
        self.step()
        self.h_out.copy_(self.out, non_blocking=True)

    def setup_e2e_pipelined(self):
        """Two device buffer sets, each holding one step's inputs packed into
        one staging buffer (so a step's inputs arrive in one host-to-device
        copy) and its result; inputs are copied on one side stream and
        results read back on another, so the copies of the neighbouring
        steps overlap this step's kernels.  Pools, tables held on the
        device, workspaces and the error word are shared."""
        import dataclasses
        torch = self.torch
        align = 256
        offs, total = {}, 0
        for name, h in self.h_in.items():
            offs[name] = total
            total += -(-h.numel() * h.element_size() // align) * align
        h_stage = torch.empty(total, dtype=torch.uint8, pin_memory=True)
        for name, h in self.h_in.items():
            n = h.numel() * h.element_size()
            h_stage[offs[name]:offs[name] + n].copy_(
                h.reshape(-1).view(torch.uint8))
        self.h_stage = h_stage
        self.e2e_sets = []
        for _ in range(2):
            d_stage = torch.empty(total, dtype=torch.uint8, device=self.device)
            views = {}
            for name, h in self.h_in.items():
                n = h.numel() * h.element_size()
                views[name] = d_stage[offs[name]:offs[name] + n].view(
                    h.dtype).view(h.shape)
            self.e2e_sets.append((d_stage, dataclasses.replace(self.db, **views),
                                  torch.empty_like(self.out),
                                  torch.empty(self.out.shape,
                                              dtype=self.out.dtype,
                                              pin_memory=True)))
        self.s_in = torch.cuda.Stream(self.device)
        self.s_out = torch.cuda.Stream(self.device)
        mk = lambda: [torch.cuda.Event(), torch.cuda.Event()]
        self.ev_in, self.ev_k, self.ev_out = mk(), mk(), mk()
        self.e2e_i = 0

    def e2e_step_pipelined(self):
        torch = self.torch
        k = self.e2e_i & 1
        d_stage, dbk, outk, h_outk = self.e2e_sets[k]
        # inputs: buffer k is free once the step two back has run
        self.s_in.wait_event(self.ev_k[k])
        with torch.cuda.stream(self.s_in):
            d_stage.copy_(self.h_stage, non_blocking=True)
        self.ev_in[k].record(self.s_in)
        # the step: after its inputs, and after the result two back is read
        self.stream.wait_event(self.ev_in[k])
        self.stream.wait_event(self.ev_out[k])
        home = (self.db, self.out)
        self.db, self.out = dbk, outk
        try:
            self.step()
        finally:
            self.db, self.out = home
        self.ev_k[k].record(self.stream)
        # result back on the other side stream
        self.s_out.wait_event(self.ev_k[k])
        with torch.cuda.stream(self.s_out):
            h_outk.copy_(outk, non_blocking=True)
        self.ev_out[k].record(self.s_out)
        self.e2e_i += 1

    def e2e_join(self):
        """The step's stream waits for the last result reads."""
        for ev in self.ev_out:
            self.stream.wait_event(ev)


def _units(wl, name):
    """(metric value numerator per step, unit, seq-steps per step)."""
    if name == "prefill":
        return wl.prefill_flops() / 1e12, "TFLOP/s", wl.num_seqs
    return wl.kv_bytes_read() / 1e9, "GB/s", wl.num_seqs


def run_tv(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    wl = _workload(args.workload, args.page_size)
    runner = TVRunner(wl, args.workload, device, unfused=args.unfused,
                      split_tokens=args.split_tokens, per_pair=args.per_pair,
                      balanced=args.balanced, engine=args.engine)
    l2_bytes = torch.cuda.get_device_properties(device).L2_cache_size
    flush = None
    if flushes_l2(wl, l2_bytes):
        flush = torch.empty(2 * l2_bytes // 4, dtype=torch.int32,
                            device=device)
    use_graph = runner.graph_timed() and not args.eager and flush is None
    per_step, unit, seqs = _units(wl, args.workload)
    hbm, tfl, tfl_sus, peak_src = _peaks()
    K, Wm = args.steps, args.warmup

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local_rank])
        torch.cuda.synchronize(device)

    for _ in range(Wm):
        runner.step()
    plan = runner.graphs(K) if use_graph else None
    if plan:
        plan[0].replay()          # untimed: uploads the graph
    barrier()

    # ---- device-timed region ------------------------------------------------
    ev = [(torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sev = [(torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    gpu_index = _gpu_index(local_rank)
    clocks = ClockSampler(gpu_index) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    barrier()
    wall0 = time.perf_counter()
    t0.record()
    if plan:
        for g in plan:
            g.replay()
    else:
        for i in range(K):
            if flush is not None:
                flush.fill_(i)       # evicts the previous step's lines
            sev[i][0].record()
            runner.step(ev[i])
            sev[i][1].record()
    t1.record()
    barrier()
    wall = time.perf_counter() - wall0
    clock_info = clocks.stop() if clocks else None
    ms = (t0.elapsed_time(t1) if flush is None else
          sum(a.elapsed_time(b) for a, b in sev))
    # one launch per step under a graph: the kernel's share is the step
    kern_ms = (ms / K if plan else
               statistics.fmean(a.elapsed_time(b) for a, b in ev))
    ms_max = _max_over_ranks(ms, world, device)
    kern_ms_max = _max_over_ranks(kern_ms, world, device)
    err = int(runner.db.err.item())

    # ---- end to end through the C ABI with host buffers -----------------------
    runner.setup_e2e()
    for _ in range(Wm):
        runner.e2e_step()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K):
        runner.e2e_step()
    e1.record()
    barrier()
    e2e_serial_ms = _max_over_ranks(e0.elapsed_time(e1), world, device)
    h2d, d2h = runner.e2e_bytes()
    # the same, with the copies of neighbouring steps overlapping each step
    runner.setup_e2e_pipelined()
    h2d = runner.h_stage.numel()        # the packed copy, alignment included
    for _ in range(Wm):
        runner.e2e_step_pipelined()
    runner.e2e_join()
    barrier()
    e0.record()
    for _ in range(K):
        runner.e2e_step_pipelined()
    runner.e2e_join()
    e1.record()
    barrier()
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1), world, device)

    value = whole_job_rate(per_step, K, ms_max, world)
    step_ms = ms_max / K
    kern_per_launch = per_step / (kern_ms_max / 1e3)     # GB/s or TFLOP/s
    kernel_name = {"decode": "tv_paged_decode", "split":
                   "tv_paged_decode_split", "prefill": "tv_paged_prefill",
                   "fused": "tv_paged_decode_append",
                   "balanced": "tv_paged_decode_balanced"}[runner.kind]
    if runner.engine:
        kernel_name = "tv_decode_step"
    peak, bound, key = _roofline_peak(unit, wall, hbm, tfl, tfl_sus)
    res = {
        "metric": METRIC if args.workload != "prefill" else
        "chunked prefill causal attention TFLOP/s (% of B200 bf16 peak)",
        "value": round(value, 3), "unit": unit, "n_gpus": world,
        "steps": K, "warmup": Wm, "ms_per_step": round(step_ms, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16, shuffled "
        "page pool)",
        "config": dict(_config(wl, args.workload, runner.kind,
                               runner.engine),
                       parallelism=f"replicas{world}" if world > 1
                       else "single GPU",
                       launch=("CUDA graphs of up to 200 steps, replayed "
                               "back to back" if plan else
                               "one host launch per step")),
        "seq_steps_per_s": round(whole_job_rate(seqs, K, ms_max, world), 1),
        "hbm_frac" if unit == "GB/s" else "tensor_frac":
            round(value / world / peak, 4),
        "roofline": {
            "bound": bound, "achieved": round(kern_per_launch, 2),
            "peak": peak, "unit": unit, "frac": round(kern_per_launch / peak,
                                                      4),
            "peak_source": (f"{peak_src} ({key})" if peak_src == "measured"
                            or bound == "hbm" else
                            f"{peak_src} (bf16 burst figure; the fallback "
                            "has no sustained one)"),
            "kernel": kernel_name,
            "kernel_ms": round(kern_ms_max, 6),
            "traffic": _traffic(kernel_name, wl.name),
            "traffic_unit": "bytes per launch (ncu dram read + write)",
        },
        "e2e": {"value": round(whole_job_rate(per_step, K, e2e_ms, world), 3),
                "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "mode": "every step copies its inputs from pinned host memory "
                        "(one packed copy) and reads its result back; two "
                        "device buffer sets and two copy streams let the "
                        "copies of neighbouring steps overlap each step",
                "serial_value": round(whole_job_rate(per_step, K,
                                                     e2e_serial_ms, world), 3)},
        "gpu_launches": K * runner.launches_per_step(),
        "clocks": clock_info,
        "device_error_word": err,
        "wall_s_timed_region": round(wall, 3),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl, args.workload, budget_s=12.0)
    return res


def _gpu_index(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


def _max_over_ranks(x, world, device):
    """The slowest rank's time: every rank calls this with its own device
    time; the result is the same on all ranks (a host-side timing reduction,
    not part of the data path)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step_per_rank, steps, ms_max, world):
    """Whole-job throughput: every rank runs its own replica of the batch,
    so the job processes world x units per step; time is the slowest rank's."""
    return world * units_per_step_per_rank * steps / (ms_max / 1e3)


# ------------------------------------------------------------ oracle arm --

def _oracle_step(wl, name, seqs):
    """One oracle pass over the sequences ``seqs`` of the workload."""
    import oracle
    seqs = np.asarray(seqs)
    if name == "prefill":
        qsl = wl.query_start_loc
        tok = np.concatenate([np.arange(qsl[s], qsl[s + 1]) for s in seqs])
        sl = wl.slot_mapping[tok]
        kp, vp, _ = oracle.kv_append(wl.k_new[tok], wl.v_new[tok], sl,
                                     wl.k_pool, wl.v_pool)
        hq = wl.num_q_heads
        ti = np.repeat(tok, hq).astype(np.int32)
        hi = np.tile(np.arange(hq), len(tok)).astype(np.int32)
        oracle.paged_prefill_rows(wl.q, qsl, kp, vp, wl.block_tables,
                                  wl.context_lens, wl.scale, ti, hi)
        return
    kp, vp, _ = oracle.kv_append(wl.k_new[seqs], wl.v_new[seqs],
                                 wl.slot_mapping[seqs], wl.k_pool, wl.v_pool)
    hq = wl.num_q_heads
    si = np.repeat(seqs, hq).astype(np.int32)
    hi = np.tile(np.arange(hq), len(seqs)).astype(np.int32)
    if name == "long":
        o_p, lse = oracle.paged_decode_partials(
            wl.q[seqs], kp, vp, wl.block_tables[seqs], wl.context_lens[seqs],
            wl.scale, wl.partition_tokens, wl.max_partitions())
        oracle.split_merge(o_p, lse, wl.context_lens[seqs],
                           wl.partition_tokens)
    else:
        oracle.paged_decode_rows(wl.q, kp, vp, wl.block_tables,
                                 wl.context_lens, wl.scale, si, hi)


def _sample_work(wl, name, seqs):
    if name == "prefill":
        sub = 0
        qsl, ctx = wl.query_start_loc, wl.context_lens
        for s in seqs:
            t = int(qsl[s + 1] - qsl[s])
            p = int(ctx[s]) - t
            sub += t * p + t * (t + 1) // 2
        return 4 * wl.head_dim * wl.num_q_heads * sub / 1e12
    per_tok = 2 * wl.num_kv_heads * wl.head_dim * 2
    return float(wl.context_lens[np.asarray(seqs)].astype(np.int64).sum()
                 * per_tok / 1e9)


def _calibrate(wl, name, target_s):
    """Smallest prefix of sequences whose oracle pass takes >= target_s
    (or the whole batch)."""
    n = 1
    while True:
        t = time.perf_counter()
        _oracle_step(wl, name, range(n))
        dt = time.perf_counter() - t
        if dt >= target_s or n >= wl.num_seqs:
            return n, dt
        n = min(wl.num_seqs, max(n + 1, int(n * min(8.0, target_s /
                                                     max(dt, 1e-3)))))


def _timed_oracle(wl, name, budget_s, max_reps):
    """Oracle throughput on the smallest prefix of the batch that takes
    about budget_s / 4: (value, sequences sampled, passes, seconds)."""
    n, _ = _calibrate(wl, name, budget_s / 4)
    reps, total, t_all = 0, 0.0, time.perf_counter()
    while reps < 1 or (time.perf_counter() - t_all < budget_s and
                       reps < max_reps):
        t = time.perf_counter()
        _oracle_step(wl, name, range(n))
        total += time.perf_counter() - t
        reps += 1
    work = _sample_work(wl, name, range(n))
    return work * reps / total, n, reps, total


def cpu_baseline(wl, name, budget_s=12.0):
    """The oracle on every host core; for the decode configurations also on
    one core (the all-core figure depends on the host's core count)."""
    import oracle
    cores = oracle.max_threads()
    value, n, reps, total = _timed_oracle(wl, name, budget_s, 5)
    unit = "TFLOP/s" if name == "prefill" else "GB/s"
    res = {"value": round(value, 6), "unit": unit,
           "cores": cores, "kind": "oracle",
           "sample": f"{n} of {wl.num_seqs} sequences (all heads), "
                     f"append + attention, {reps} pass(es), "
                     f"{total:.1f} s of CPU time"}
    if name in ("llama", "tiny"):
        oracle.set_threads(1)
        try:
            value1, n1, reps1, total1 = _timed_oracle(wl, name,
                                                      budget_s / 3, 3)
        finally:
            oracle.set_threads(cores)
        res["single_core"] = {
            "value": round(value1, 6), "unit": unit, "cores": 1,
            "sample": f"{n1} of {wl.num_seqs} sequences (all heads), "
                      f"append + attention, {reps1} pass(es), "
                      f"{total1:.1f} s of CPU time"}
    return res


def run_reference(args):
    import oracle
    wl = _workload(args.workload, args.page_size)
    cores = oracle.max_threads()
    K, Wm = args.steps, args.warmup
    # size the per-step sample so the whole run takes about two minutes
    n, dt = _calibrate(wl, args.workload, 0.5)
    per_seq = dt / n
    n = int(max(1, min(wl.num_seqs, 120.0 / max(1, K + Wm) / per_seq)))
    seqs = range(n)
    for _ in range(Wm):
        _oracle_step(wl, args.workload, seqs)
    t = time.perf_counter()
    for _ in range(K):
        _oracle_step(wl, args.workload, seqs)
    el = time.perf_counter() - t
    work = _sample_work(wl, args.workload, seqs)
    unit = "TFLOP/s" if args.workload == "prefill" else "GB/s"
    value = work * K / el
    sample = (f"{n} of {wl.num_seqs} sequences (all heads) per step, "
              "append + attention")
    return {
        "metric": METRIC if args.workload != "prefill" else
        "chunked prefill causal attention TFLOP/s (% of B200 bf16 peak)",
        "value": round(value, 6), "unit": unit, "n_gpus": 1, "steps": K,
        "warmup": Wm, "ms_per_step": round(el / K * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded N(0,1) bf16, shuffled "
        "page pool)", "config": _config(wl, args.workload),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": unit,
                         "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": unit,
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["tv", "reference"], default="tv")
    ap.add_argument("--workload", default="llama",
                    choices=["llama", "mix", "long", "prefill", "tiny"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="decode step as tv_kv_append + tv_paged_decode")
    ap.add_argument("--per-pair", action="store_true",
                    help="decode step as tv_paged_decode_append (one CTA "
                         "per sequence and KV head)")
    ap.add_argument("--balanced", action="store_true",
                    help="decode step as tv_paged_decode_balanced (the "
                         "work-balanced grid) with the append fused")
    ap.add_argument("--page-size", type=int, default=16, choices=[16, 32],
                    help="tokens per KV page (the workloads keep their "
                         "contexts and pool bytes)")
    ap.add_argument("--engine", action="store_true",
                    help="decode step as tv_decode_step on a device page "
                         "pool (host-free, graph-captured engine step)")
    ap.add_argument("--eager", action="store_true",
                    help="launch every timed step from the host (no graph)")
    ap.add_argument("--split-tokens", type=int, default=0,
                    help="decode step as tv_kv_append + tv_paged_decode_split "
                         "(partitions of this many tokens) + tv_split_merge")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    from paged_kv_cache_376_b200 import build as _build
    _build.build()
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(
            seconds=120), device_id=torch.device("cuda", local_rank))
    try:
        res = run_tv(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
