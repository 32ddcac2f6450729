#!/usr/bin/env python
"""Benchmark of the PBSA hot path on B200.

Default workload (N=1): one single-layer decode step shaped like a 1.3B video
DiT -- B1 H12 D128 bf16, 128-token blocks, a 4680-token query chunk (37
blocks), a cache of 5 chunks (185 blocks), persistent budget 24, window of 2
chunks, local top-16 -- run as score -> update memory -> select -> attend.
A step is one pass of that path over the chunk; the memory starts empty each
step (snapshot semantics) and the pooled keys of older blocks are cached, so
the step pools only the current chunk's Q and K.

Reported (one JSON line on rank 0):
  value          attended forward TFLOP/s over the whole step (all ranks)
  ms_per_step    per-chunk latency of the step (device time, max over ranks)
  roofline       the attention kernel against the measured bf16 peak
  e2e            the same metric through the public API with pinned host
                 inputs copied in and the output copied out every step
  cpu_baseline   the CPU oracle timed on a bounded sample on the host cores
  --impl reference  times the CPU oracle itself as the reference arm.

Multi-GPU (torchrun): every rank runs its own decode problem (independent
layers/sequences), no data-path collective; scaling is weak.  --shard heads
instead splits one rollout layer's heads over the ranks and all-gathers the
output every step (strong scaling).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) of one attn_fwd launch on the decode step, from a
# one-launch ncu capture of this workload, keyed by a hash of the kernel's
# sources: a changed kernel reports null until it is captured again.
ATTN_TRAFFIC_SOURCES = ["attn_fwd.cu", "tc_sm100.cuh", "common.cuh", "launch.h", "tmap.h"]
ATTN_TRAFFIC = {"91216dbb2101212aa8fc26523cbd2ce2c3da31d391134e9960edeac56176a14a": 95695104}


def attn_traffic():
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_attention_39_b200", "csrc")
    for f in ATTN_TRAFFIC_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return ATTN_TRAFFIC.get(h.hexdigest())
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="pbsa", choices=["pbsa", "reference"])
    ap.add_argument("--workload", default="decode", choices=["decode", "train", "hbm"],
                    help="decode: the decode step (default); train: forward + backward of "
                         "the trainable shape on its P32 + top-16 lists; hbm: the score and "
                         "update calls on bandwidth-sized work")
    ap.add_argument("--shard", default="none", choices=["none", "heads"],
                    help="heads: one rollout layer split by heads over the ranks, the output "
                         "all-gathered every step (strong scaling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the trainable-path, dense-comparator and rollout measurements")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ----------------------------------------------------------------- distributed
def init_dist(n):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The max of x over all ranks (the step time a job is held to)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank, ms_max, world):
    """Weak scaling: every rank processes its own problem of flops_per_rank;
    the job's throughput is all ranks' work over the slowest rank's time."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def rank_workload(rank):
    """The decode workload of one rank: same shapes, its own seed."""
    import pbsa_inputs as PI
    w = PI.WORKLOADS["decode"]
    return PI.variant(w, seed=w.seed + 1000 * rank) if rank else w


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- decode
class DecodeRunner:
    """One decode-step problem resident on the device, captured as a CUDA graph."""

    def __init__(self, seed_offset=0):
        import torch

        import pbsa_inputs as PI
        from block_sparse_attention_39_b200.engine import PbsaLayer
        self.torch = torch
        w = rank_workload(seed_offset)
        self.w = w
        chunks = PI.snapshot_chunks(w)
        self.chunks = chunks
        L = PbsaLayer(w)
        self.lay = L.layout
        dev = torch.device("cuda")

        def st(x):
            return torch.from_numpy(np.ascontiguousarray(x)).to(dev).to(torch.bfloat16)
        for t, (_, k, v) in chunks.items():
            L.write_chunk(t, st(k), st(v))
        self.t = w.n_chunks - 1
        L.q.copy_(st(chunks[self.t][0]))
        self.L = L
        # pooled keys of every cached block (older blocks stay cached)
        L.score(self.t, pool_ids=L.all_ids())
        L.reset_memory()
        self.cand = L.candidates(self.t)
        L.window_ids(self.t)
        L.chunk_ids(self.t)
        torch.cuda.synchronize()
        self.flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        # the headline schedule: the routing call (one dependency-driven kernel for
        # score -> update -> select) then attention; the per-call path (five
        # kernels chained by programmatic dependent launch) is timed beside it
        self.fused = True

    @property
    def launches_per_step(self):
        # route_kernel + attention, or pool, score, plan, apply, select + attention
        return 2 if self.fused else 6

    def step(self, ev=None, fused=None, appended=False):
        """One step.  fused: the routing call (pbsa_route_step) then attention;
        otherwise the per-call path (score, update, select, attention).  `ev`
        records an event between the calls.  appended: the chunk came in through
        pbsa_append_chunk, so its keys are pooled already."""
        L = self.L
        if fused is None:
            fused = self.fused
        pids = L.no_ids if appended else None
        calls = ([lambda: L.route(self.t, appended=appended)] if fused else
                 [lambda: L.score(self.t, pool_ids=pids), lambda: L.update(*self.cand),
                  lambda: L.select(self.t)])
        calls.append(lambda: L.attend(self.t))
        for k, c in enumerate(calls):
            if ev is not None:
                ev[k].record()
            c()
        if ev is not None:
            ev[len(calls)].record()

    def chunk_kv(self):
        """The step's chunk as the [B,H,T_c,D] K and V a caller appends."""
        torch = self.torch
        _, k, v = self.chunks[self.t]
        return (torch.from_numpy(np.ascontiguousarray(k)).to(torch.bfloat16),
                torch.from_numpy(np.ascontiguousarray(v)).to(torch.bfloat16))

    def prologue(self):
        self.L.reset_memory()
        self.flush_buf.zero_()

    def flops(self):
        L = self.L
        idx = L.idx.cpu().numpy()
        cnt = L.cnt.cpu().numpy()
        bl = L.blk_len.cpu().numpy()
        lens = np.array(self.lay.block_lens(), dtype=np.int64)
        total = 0
        for b in range(self.w.B):
            for h in range(self.w.H):
                for i in range(L.nQB):
                    ids = idx[b, h, i, :cnt[b, h, i]]
                    total += 4 * int(lens[i]) * int(bl[b, h, ids].astype(np.int64).sum()) * self.w.D
        return total

    def hbm_bytes(self):
        """Algorithmic HBM bytes of the score and update calls of one step: each
        input element read once, each output written once (the q_bar re-read by
        the scoring kernel is an intermediate and is not counted)."""
        w, L = self.w, self.L
        BH = w.B * w.H
        el = 2
        rows_q = w.chunk_tokens
        rows_k = sum(self.lay.block_lens())                # new chunk's valid key rows
        NB, nb_c = L.NB, self.lay.nb_c
        score = BH * (rows_q * w.D * el + rows_k * w.D * el          # Q and new K read
                      + L.nQB * w.D * 4 + nb_c * w.D * 4           # q_bar, new k_bar written
                      + (NB - nb_c) * w.D * 4                      # older k_bar read
                      + L.nQB * NB * 4 + NB * 4)                   # S and m written
        src = L.slot_src.cpu().numpy()
        written = int((src >= 0).sum())                            # slots (re)written this step
        upd = written * (w.bs * w.D * el * 2 * 2 + w.D * 4 * 2)    # K+V read+write, k_bar copy
        return score, upd

    def capture(self, n_graphs, breakdown=False, fused=None):
        """Capture n_graphs copies of [prologue, e0, step, e_last], each with its own
        timing events (event-record graph nodes).  With `breakdown`, events also
        sit between the calls; they split the step for the per-call report but
        add their own cost and stop the next call's kernels from launching early
        (programmatic dependent launch), so the headline uses graphs without them."""
        torch = self.torch
        if fused is None:
            fused = self.fused
        s = torch.cuda.Stream()
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            for _ in range(3):                   # eager warm-up before capture
                self.prologue()
                self.step(fused=fused)
        torch.cuda.synchronize()
        pool = torch.cuda.graph_pool_handle()
        graphs, evs = [], []
        n_ev = (2 if fused else 4) + 1
        for _ in range(n_graphs):
            ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_ev)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, pool=pool, stream=s):
                self.prologue()
                if breakdown:
                    self.step(ev, fused=fused)
                else:
                    ev[0].record()
                    self.step(fused=fused)
                    ev[-1].record()
            graphs.append(g)
            evs.append(ev)
        torch.cuda.synchronize()
        return graphs, evs, s

    def e2e(self, steps, warmup):
        """Through the public API with host buffers, as a decode loop runs it: every
        step copies its Q and new-chunk K/V [B,H,T_c,D] from pinned host memory,
        appends the chunk to the cache (pbsa_append_chunk, which pools its keys),
        runs the step and reads its O and LSE back.  The copies of step t+1's
        inputs and of step t-1's outputs run on their own streams while step t
        computes (double-buffered device staging); the time is the whole loop's
        device time over the steps."""
        torch = self.torch
        L, w = self.L, self.w
        hq = torch.from_numpy(self.chunks[self.t][0]).to(torch.bfloat16).pin_memory()
        ck, cv = self.chunk_kv()
        hk, hv = ck.pin_memory(), cv.pin_memory()
        ho = [torch.empty(L.o.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        hl = [torch.empty(L.lse.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
        q_st = [torch.empty_like(L.q) for _ in range(2)]
        k_st = [torch.empty(hk.shape, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        v_st = [torch.empty(hv.shape, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        o_st = [torch.empty_like(L.o) for _ in range(2)]
        l_st = [torch.empty_like(L.lse) for _ in range(2)]
        h2d = hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2
        d2h = ho[0].numel() * 2 + hl[0].numel() * 4
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        n = warmup + steps
        ev_in, ev_used, ev_cmp, ev_out = [None] * n, [None] * n, [None] * n, [None] * n
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()

        def mark(stream):
            e = torch.cuda.Event()
            e.record(stream)
            return e
        for it in range(n):
            b = it % 2
            if it == warmup:
                start.record(s_in)
            with torch.cuda.stream(s_in):
                if it >= 2:
                    s_in.wait_event(ev_used[it - 2])     # staging buffer b is free
                q_st[b].copy_(hq, non_blocking=True)
                k_st[b].copy_(hk, non_blocking=True)
                v_st[b].copy_(hv, non_blocking=True)
                ev_in[it] = mark(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[it])
                L.reset_memory()                       # each step starts from empty memory
                L.q.copy_(q_st[b])
                L.append(self.t, k_st[b], v_st[b])
                ev_used[it] = mark(s_cmp)
                self.step(appended=True)
                if it >= 2:
                    s_cmp.wait_event(ev_out[it - 2])   # output staging b is free
                o_st[b].copy_(L.o)
                l_st[b].copy_(L.lse)
                ev_cmp[it] = mark(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[it])
                ho[b].copy_(o_st[b], non_blocking=True)
                hl[b].copy_(l_st[b], non_blocking=True)
                ev_out[it] = mark(s_out)
        end.record(s_out)
        torch.cuda.synchronize()
        ms = start.elapsed_time(end) / steps
        return ms, h2d, d2h


# ----------------------------------------------------------------- extras
def _timed(torch, fn, reps, flush=None):
    """Mean device time (ms) of fn() over reps, L2 flushed before each."""
    s = torch.cuda.current_stream()
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        fn()
        b.record(s)
        ts.append((a, b))
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in ts]))


def _graph_timed(torch, fn, reps, pre=None):
    """Mean device time (ms) of fn() captured in CUDA graphs with its timing
    events inside the graph, so host launch overhead is not timed; pre() (if
    given) runs in the same graph before the first event."""
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        for _ in range(2):
            if pre is not None:
                pre()
            fn()
    torch.cuda.synchronize()
    graphs = []
    for _ in range(reps):
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            if pre is not None:
                pre()
            ev[0].record()
            fn()
            ev[1].record()
        graphs.append((g, ev))
    with torch.cuda.stream(s):
        for g, _ in graphs:          # first replays upload the graphs: untimed
            g.replay()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        for g, _ in graphs:
            g.replay()
    torch.cuda.synchronize()
    ms = float(np.mean([ev[0].elapsed_time(ev[1]) for _, ev in graphs]))
    del graphs
    return ms


def _pair_flops(idx, cnt, blk_len, q_lens, D, per_pair):
    total = 0
    B, H, nQB = cnt.shape
    for b in range(B):
        for h in range(H):
            for i in range(nQB):
                ids = idx[b, h, i, :cnt[b, h, i]]
                total += per_pair * int(q_lens[i]) * int(blk_len[b, h, ids].astype(np.int64).sum()) * D
    return total


def bench_train(torch, flush, reps=5):
    """Trainable-path shape: forward and backward of the one-shot lists, and the
    density sweep (the d = 1 lists are dense block-causal attention)."""
    import pbsa_inputs as PI
    from block_sparse_attention_39_b200.engine import PbsaTrain
    w = PI.WORKLOADS["train"]
    T = PbsaTrain(w)
    g = torch.Generator(device="cuda").manual_seed(w.seed)
    for t in (T.q, T.dO):
        t.copy_(torch.randn(t.shape, generator=g, device="cuda").bfloat16())
    for t in (T.kpool, T.vpool):
        t.copy_(torch.randn(t.shape, generator=g, device="cuda").bfloat16())
    T.set_meta()
    lens = np.array([n for c in range(w.n_chunks) for n in T.layout.block_lens()], dtype=np.int64)
    bl = T.blk_len.cpu().numpy()
    out = {"shape": f"B{w.B} H{w.H} D{w.D} bf16, {w.n_chunks} chunks x {w.chunk_tokens} tokens "
                    f"= {T.T} tokens, {T.NB} blocks of {w.bs}, chunk-causal"}
    runs = [("lists P32+k16", None)] + [(f"density {int(d * 100)}%", d) for d in PI.TRAIN_DENSITIES]
    dense_fwd = dense_bwd = None
    rows = {}
    for name, dens in runs:
        T.lists(density=dens)
        torch.cuda.synchronize()
        idx, cnt = T.idx.cpu().numpy(), T.cnt.cpu().numpy()
        ffl = _pair_flops(idx, cnt, bl, lens, w.D, 4)
        T.fwd()
        ms_f = _timed(torch, T.fwd, reps, flush)
        ms_b = _timed(torch, T.bwd, reps, flush)
        rows[name] = {"attended_blocks_per_query_block": round(float(cnt.mean()), 2),
                      "fwd_ms": round(ms_f, 4), "fwd_tflops": round(ffl / ms_f / 1e9, 1),
                      "bwd_ms": round(ms_b, 4), "bwd_tflops": round(2.5 * ffl / ms_b / 1e9, 1)}
        if dens == 1.0:
            dense_fwd, dense_bwd = ms_f, ms_b
    for name, r in rows.items():
        r["fwd_speedup_vs_dense"] = round(dense_fwd / r["fwd_ms"], 2)
        r["bwd_speedup_vs_dense"] = round(dense_bwd / r["bwd_ms"], 2)
    out["runs"] = rows
    out["flop_count"] = "fwd 4*len_q*len_k*D, bwd 10*len_q*len_k*D per attended block pair"
    del T
    torch.cuda.empty_cache()
    return out


def bench_dense_comparators(torch, runner, flush, reps=10):
    """The decode inputs through the same attention kernel with full lists:
    the whole cache (185 blocks) and the sliding window alone (last 2 chunks)."""
    from block_sparse_attention_39_b200 import pbsa as K
    L, w, lay = runner.L, runner.w, runner.lay
    out = {}
    for name, chunks in (("dense_full_cache", list(range(w.n_chunks))),
                         ("dense_sliding_window", lay.window_chunks(w.n_chunks - 1))):
        ids = [p for c in chunks for p in lay.chunk_phys_ids(c)]
        idx = torch.tensor(ids, dtype=torch.int32, device="cuda").expand(
            w.B, w.H, L.nQB, len(ids)).contiguous()
        cnt = torch.full((w.B, w.H, L.nQB), len(ids), dtype=torch.int32, device="cuda")
        fn = lambda: K.attn_fwd(L.dbf, L.q, w.chunk_tokens, runner.t * w.chunk_tokens, L.kpool,
                                L.vpool, L.NB, L.blk_len, L.blk_pos, idx, cnt, len(ids), w.mask,
                                L.o, L.lse)
        fn()
        ms = _timed(torch, fn, reps, flush)
        lens = np.array(lay.block_lens(), dtype=np.int64)
        fl = 4 * int(lens.sum()) * int(lens.sum()) * len(chunks) * w.D * w.B * w.H
        out[name] = {"blocks": len(ids), "ms": round(ms, 4), "tflops": round(fl / ms / 1e9, 1)}
    return out


def layer_bytes(L):
    """Library-owned device bytes of one layer's PBSA state (pool, metadata,
    pooled keys, slots, workspace)."""
    ts = [L.kpool, L.vpool, L.blk_len, L.blk_pos, L.k_bar, L.slot_src, L.slot_w, L.ws]
    return int(sum(t.numel() * t.element_size() for t in ts))


def _pct(xs):
    xs = np.asarray(xs, dtype=np.float64)
    return {"mean": round(float(xs.mean()), 4), "p50": round(float(np.percentile(xs, 50)), 4),
            "p90": round(float(np.percentile(xs, 90)), 4), "max": round(float(xs.max()), 4)}


def _dense_attend(K, torch, d, q, Tc, pos0, kp, vp, NB, bl, bp, ids, nQB, o, lse, parts_o,
                  parts_lse, max_list):
    """Dense attention of a query chunk over the blocks `ids` with the library's
    attention kernel; lists longer than the kernel's shared-memory list limit
    run as parts whose outputs are merged by their log-sum-exps."""
    parts = [ids[i:i + max_list] for i in range(0, len(ids), max_list)]
    B, H = d.B, d.H
    outs = []
    for pi, part in enumerate(parts):
        idx = part.expand(B, H, nQB, part.numel()).contiguous()
        cnt = torch.full((B, H, nQB), part.numel(), dtype=torch.int32, device="cuda")
        oo, ll = (o, lse) if len(parts) == 1 else (parts_o[pi], parts_lse[pi])
        K.attn_fwd(d, q, Tc, pos0, kp, vp, NB, bl, bp, idx, cnt, part.numel(), 0, oo, ll)
        outs.append((oo, ll))
    if len(parts) > 1:
        m = torch.stack([ll for _, ll in outs]).amax(0)
        wsum = sum(torch.exp(ll - m) for _, ll in outs)
        acc = sum(oo.float() * (torch.exp(ll - m) / wsum).unsqueeze(-1) for oo, ll in outs)
        o.copy_(acc)
        lse.copy_(m + torch.log(wsum))


def bench_rollouts(torch):
    """The rollout workloads as stated: every chunk step of the 20-second rollout
    (27 steps, 1 layer) and of the 1-minute rollout (80 steps x 30 layers), each
    step score -> update -> select -> attend per layer, on device-drawn seeded
    inputs with the workloads' salience structure; per-step latency and its
    percentiles; the same inputs through the library's attention kernel as the
    dense comparators (every chunk so far, and the last W chunks); library KV
    bytes against a dense cache, and the allocator's peak."""
    import pbsa_inputs as PI
    from block_sparse_attention_39_b200 import pbsa as K
    from block_sparse_attention_39_b200.engine import PbsaLayer
    out = {}
    for name in ("rollout20s", "rollout1min"):
        w = PI.WORKLOADS[name]
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        base = torch.cuda.memory_allocated()
        torch.cuda.reset_peak_memory_stats()
        layers = [PbsaLayer(w) for _ in range(w.layers)]
        state_alloc = torch.cuda.memory_allocated() - base
        gs = torch.cuda.Stream()
        pbsa_ms = []
        for t in range(w.n_chunks):
            for li, L in enumerate(layers):
                q, k, v = PI.chunk_tensors_device(w, t, li)
                L.write_chunk(t, k, v)
                L.q.copy_(q)
                L.candidates(t)                 # id lists built outside the timed region
                L.window_ids(t)
                L.chunk_ids(t)
            del q, k, v
            torch.cuda.synchronize()
            # each step: a CUDA graph of every layer's score -> update -> select ->
            # attend with the timing events inside it (host launch cost not timed)
            ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=gs):
                ev[0].record()
                for L in layers:
                    L.step(t)
                ev[1].record()
            with torch.cuda.stream(gs):
                graph.replay()
            torch.cuda.synchronize()
            pbsa_ms.append(ev[0].elapsed_time(ev[1]))
            del graph
        peak_alloc = torch.cuda.max_memory_allocated() - base
        kv = sum(layer_bytes(L) for L in layers)
        lay = layers[0].layout
        nb_c = lay.nb_c
        del layers
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        base = torch.cuda.memory_allocated()
        torch.cuda.reset_peak_memory_stats()
        # dense comparators: per layer a cache of every chunk so far, filled by
        # pbsa_append_chunk with the same (layer, t) inputs; one layer's cache
        # lives at a time, the per-step time is summed over the layers
        NBd = w.n_chunks * nb_c
        d = K.dims(w.B, w.H, w.D, w.bs, 1.0 / math.sqrt(w.D), torch.bfloat16)
        dense_full = np.zeros(w.n_chunks)
        dense_win = np.zeros(w.n_chunks)
        max_list = 2048
        Tc = w.chunk_tokens
        kp = torch.zeros(w.B, w.H, NBd, w.bs, w.D, dtype=torch.bfloat16, device="cuda")
        vp = torch.zeros_like(kp)
        bl = torch.zeros(w.B, w.H, NBd, dtype=torch.int32, device="cuda")
        bp = torch.zeros_like(bl)
        kb = torch.zeros(w.B, w.H, NBd, w.D, dtype=torch.float32, device="cuda")
        o = torch.empty(w.B, w.H, Tc, w.D, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(w.B, w.H, Tc, dtype=torch.float32, device="cuda")
        n_parts = -(-NBd // max_list)
        parts_o = [torch.empty_like(o) for _ in range(n_parts)]
        parts_lse = [torch.empty_like(lse) for _ in range(n_parts)]
        all_ids = torch.arange(NBd, dtype=torch.int32, device="cuda")
        dense_peak = 0
        for li in range(w.layers):
            bl.zero_()
            for t in range(w.n_chunks):
                q, k, v = PI.chunk_tensors_device(w, t, li)
                blk = all_ids[t * nb_c:(t + 1) * nb_c]
                K.append_chunk(d, k, v, Tc, t * Tc, kp, vp, NBd, blk, bl, bp, kb)
                for kind, ids in (("full", all_ids[:(t + 1) * nb_c]),
                                  ("win", all_ids[max(0, t + 1 - w.W) * nb_c:(t + 1) * nb_c])):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record()
                    _dense_attend(K, torch, d, q, Tc, t * Tc, kp, vp, NBd, bl, bp, ids, nb_c, o,
                                  lse, parts_o, parts_lse, max_list)
                    e1.record()
                    torch.cuda.synchronize()
                    (dense_full if kind == "full" else dense_win)[t] += e0.elapsed_time(e1)
            dense_peak = max(dense_peak, torch.cuda.max_memory_allocated() - base)
        dense_kv_last = NBd * w.bs * w.D * 2 * 2 * w.B * w.H * w.layers
        del kp, vp, bl, bp, kb, o, lse, parts_o, parts_lse
        torch.cuda.empty_cache()
        pb = np.array(pbsa_ms)
        out[name] = {
            "layers": w.layers, "P": w.P, "policy": "merge_mean" if w.policy else "evict",
            "steps": w.n_chunks,
            "inputs": "device-drawn per (layer, step), N(0,1) with the workload's salient blocks "
                      "(N(0,2) offsets), the same draws for PBSA and the dense comparators",
            "pbsa_ms_per_step": _pct(pb),
            "pbsa_ms_steps": [round(float(x), 4) for x in pb],
            "dense_full_cache_ms_per_step": _pct(dense_full),
            "dense_full_cache_ms_steps": [round(float(x), 4) for x in dense_full],
            "dense_sliding_window_ms_per_step": _pct(dense_win),
            "speedup_vs_dense_full_cache": {
                "whole_rollout": round(float(dense_full.sum() / pb.sum()), 3),
                "last_step": round(float(dense_full[-1] / pb[-1]), 3)},
            "kv_bytes_library": kv,
            "allocator_bytes_pbsa_state": int(state_alloc),
            "allocator_peak_bytes_pbsa_rollout": int(peak_alloc),
            "dense_full_cache_kv_bytes_at_last_step": dense_kv_last,
            "allocator_peak_bytes_dense_one_layer": int(dense_peak),
            "kv_reduction": round(1 - kv / dense_kv_last, 4),
            "dense_note": "PBSA step = score + update + select + attend per layer; dense = the "
                          "attention kernel over every chunk so far (lists over 2048 blocks run "
                          "as parts merged by log-sum-exp) or the last W chunks; per step summed "
                          "over the layers"}
    return out


def bench_select_hier(torch, runner, reps=20):
    """The two-level (frame -> block) selection against the one-level local
    selection on the decode step's scores (both per-call, CUDA graphs)."""
    L, t = runner.L, runner.t
    out = {}
    runner.step()
    torch.cuda.synchronize()
    out["select_local_ms"] = round(_graph_timed(torch, lambda: L.select(t), reps), 5)
    for F in (2, 4):
        out[f"select_hier_F{F}_ms"] = round(
            _graph_timed(torch, lambda: L.select_hier(t, F, 1560), reps), 5)
    out["frames"] = "1560-token frames: 3 per chunk, 6 in the 2-chunk window; top-k 16 inside"
    return out


def bench_rollout_backward(torch):
    """The recurrent trainable path on the 20-second rollout shape (B1 H12 D128,
    27 chunk steps, merge policy, P48): the forward steps recorded, then the
    backward of sum_t <O_t, dO_t> back through every step's attention and
    memory update; per-step time, the attention backward's TF/s over attended
    blocks (10 len_q len_k D per pair) and the memory update's backward."""
    import pbsa_inputs as PI
    from block_sparse_attention_39_b200 import pbsa as K
    from block_sparse_attention_39_b200.engine import PbsaLayer, PbsaRolloutTrain
    w = PI.WORKLOADS["rollout20s"]
    L = PbsaLayer(w)
    tr = PbsaRolloutTrain(L)
    dOs = []
    g = torch.Generator(device="cuda").manual_seed(11)
    for t in range(w.n_chunks):
        q, k, v = PI.chunk_tensors_device(w, t)
        tr.step(t, q, k, v)
        dOs.append(torch.randn(q.shape, generator=g, device="cuda").bfloat16())
    torch.cuda.synchronize()
    tr.backward(dOs)                        # warm-up
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    tr.backward(dOs)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    lens = np.array(L.layout.block_lens(), dtype=np.int64)
    fl = sum(_pair_flops(r["idx"].cpu().numpy(), r["cnt"].cpu().numpy(),
                         r["blk_len"].cpu().numpy(), lens, w.D, 10) for r in tr.steps)
    # one memory-update backward on its own
    rec = [r for r in tr.steps if r["plan"] is not None][-1]
    dk = torch.zeros(w.B, w.H, L.NB, w.bs, w.D, dtype=torch.float32, device="cuda")
    dv = torch.zeros_like(dk)
    upd_ms = _graph_timed(torch, lambda: K.update_memory_bwd(L.d, L.NB, L.P, rec["n_cand"],
                                                             rec["plan"], dk, dv, tr.upd_ws), 20)
    merged = int((L.slot_w.cpu().numpy() > 1).sum())
    out = {"shape": "B1 H12 D128 bf16, 27 steps, P48 merge_mean",
           "backward_ms_whole_rollout": round(ms, 3),
           "backward_ms_per_step": round(ms / w.n_chunks, 4),
           "attn_bwd_tflops_over_attended": round(fl / (ms * 1e-3) / 1e12, 1),
           "update_memory_bwd_ms": round(upd_ms, 5),
           "slots_holding_merges_at_end": merged,
           "note": "includes the per-chunk gradient accumulation (torch adds) and the "
                   "slot-gradient carry between steps"}
    del tr, L, dOs
    torch.cuda.empty_cache()
    return out


def append_traffic(BH, Tc, nb, bs, D):
    """Algorithmic HBM bytes of pbsa_append_chunk (bf16): K and V rows read
    once, their blocks (padding included) written once, the pooled keys and the
    two metadata words of each block written."""
    return BH * (2 * Tc * D * 2 + 2 * nb * bs * D * 2 + nb * D * 4 + nb * 8)


def bench_hbm_at_scale(torch, flush, pk, reps=5):
    """The HBM-bound calls on bandwidth-sized work, beside the latency-bound
    decode step: score_blocks pooling and scoring the whole trainable shape
    (every query and key block of 32 760 tokens, B2 H12), update_memory
    filling 128 slots per head from 111 candidate blocks (B2 H12), and
    append_chunk placing a 32 760-token chunk (B2 H12, 805 MB moved)."""
    import pbsa_inputs as PI
    from block_sparse_attention_39_b200 import pbsa as K
    from block_sparse_attention_39_b200.engine import PbsaLayer, PbsaTrain
    out = {}
    w = PI.WORKLOADS["train"]
    T = PbsaTrain(w)
    g = torch.Generator(device="cuda").manual_seed(5)
    for t in (T.q, T.kpool):
        t.copy_(torch.randn(t.shape, generator=g, device="cuda").bfloat16())
    T.set_meta()
    fn = lambda: K.score_blocks(T.d, T.q, T.T, T.kpool, T.NB, T.blk_len, T.all_ids, T.NB,
                                T.q_bar, T.k_bar, T.scores, T.mem)
    fn()
    # inputs (415 MB) exceed the 126 MB L2, so no flush between repetitions: a
    # flush leaves dirty lines whose write-back would land in the timed call
    ms = _graph_timed(torch, fn, reps)
    BH = w.B * w.H
    byt = (BH * T.T * w.D * 2 * 2                    # Q and every key row read
           + BH * (T.nQB + T.NB) * w.D * 4           # q_bar, k_bar written
           + BH * T.nQB * T.NB * 4 + BH * T.G * T.NB * 4)   # S and m written
    out["score_blocks, trainable shape"] = {
        "bytes": byt, "ms": round(ms, 4), "gbs": round(byt / ms / 1e6, 1),
        "frac": round(byt / ms / 1e6 / pk["hbm_gbs"], 4)}
    del T
    torch.cuda.empty_cache()
    wv = PI.variant(PI.WORKLOADS["decode"], B=2, P=128)
    L = PbsaLayer(wv)
    for t in (L.kpool, L.vpool):
        t.copy_(torch.randn(t.shape, generator=g, device="cuda").bfloat16())
    for c in range(wv.n_chunks):
        L.set_chunk_meta(c)
    L.score(wv.n_chunks - 1, pool_ids=L.all_ids())
    ci, cs = L.candidates(wv.n_chunks - 1)

    L.reset_memory()
    L.update(ci, cs)
    torch.cuda.synchronize()
    kept = int((L.slot_src >= 0).sum().item())
    # the update call alone, the memory reset before it in the same graph (the
    # 352 MB it moves exceed L2, so no flush)
    ms = _graph_timed(torch, lambda: L.update(ci, cs), reps, pre=L.reset_memory)
    byt = kept * (wv.bs * wv.D * 2 * 2 * 2 + wv.D * 4 * 2)
    out["update_memory, 128 slots from 111 candidates, B2 H12"] = {
        "bytes": byt, "ms": round(ms, 4), "gbs": round(byt / ms / 1e6, 1),
        "frac": round(byt / ms / 1e6 / pk["hbm_gbs"], 4)}
    del L
    torch.cuda.empty_cache()
    # bandwidth-sized: inputs and pool (805 MB) exceed L2, no flush
    B, H, D, bs, Tc = 2, 12, 128, 128, 32760
    nb = -(-Tc // bs)
    d = K.dims(B, H, D, bs, 1 / math.sqrt(D), torch.bfloat16)
    g = torch.Generator(device="cuda").manual_seed(9)
    kb = torch.randn(B, H, Tc, D, generator=g, device="cuda").bfloat16()
    vb = torch.randn(B, H, Tc, D, generator=g, device="cuda").bfloat16()
    kp = torch.empty(B, H, nb, bs, D, dtype=torch.bfloat16, device="cuda")
    vp = torch.empty_like(kp)
    bl = torch.empty(B, H, nb, dtype=torch.int32, device="cuda")
    bp = torch.empty_like(bl)
    kbar = torch.empty(B, H, nb, D, dtype=torch.float32, device="cuda")
    ids = torch.randperm(nb, generator=torch.Generator().manual_seed(3)).int().cuda()
    fn = lambda: K.append_chunk(d, kb, vb, Tc, 0, kp, vp, nb, ids, bl, bp, kbar)
    ms = _graph_timed(torch, fn, reps)
    byt = append_traffic(B * H, Tc, nb, bs, D)
    out["append_chunk, 32 760-token chunk, B2 H12"] = {
        "bytes": byt, "ms": round(ms, 4), "gbs": round(byt / ms / 1e6, 1),
        "frac": round(byt / ms / 1e6 / pk["hbm_gbs"], 4)}
    del kb, vb, kp, vp, bl, bp, kbar
    torch.cuda.empty_cache()
    out["peak_gbs"] = pk["hbm_gbs"]
    out["l2"] = "not flushed: every input is larger than the 126 MB L2"
    out["timed"] = "CUDA graphs with the timing events inside, device time of the call"
    return out


def bench_append(torch, runner, pk, reps=20):
    """pbsa_append_chunk, the KV append with the keys' block pooling fused in,
    on the decode step's chunk (B1 H12, 4680 tokens); after it the step's score
    call pools only the queries.  The bandwidth-sized case is in
    bench_hbm_at_scale."""
    L, w, t = runner.L, runner.w, runner.t
    flush = runner.flush_buf
    k, v = (x.cuda() for x in runner.chunk_kv())

    def entry(byt, ms):
        return {"bytes": int(byt), "ms": round(ms, 5), "gbs": round(byt / ms / 1e6, 1),
                "frac": round(byt / ms / 1e6 / pk["hbm_gbs"], 4)}
    out = {}
    # decode chunk: 29 MB of inputs fit L2, so the graph flushes it first (as the step does)
    ms = _graph_timed(torch, lambda: L.append(t, k, v), reps, pre=flush.zero_)
    out["append_chunk, decode chunk"] = entry(append_traffic(w.B * w.H, w.chunk_tokens,
                                                             L.layout.nb_c, w.bs, w.D), ms)
    out["score_blocks, keys pooled by the append (queries only)"] = {
        "ms": round(_graph_timed(torch, lambda: L.score(t, pool_ids=L.no_ids), reps,
                                 pre=flush.zero_), 5)}
    out["score_blocks, pooling the chunk's keys itself"] = {
        "ms": round(_graph_timed(torch, lambda: L.score(t), reps, pre=flush.zero_), 5)}
    out["peak_gbs"] = pk["hbm_gbs"]
    out["timed"] = "CUDA graphs with the timing events inside, device time of the call"
    return out


# ----------------------------------------------------------------- CPU oracle
def cpu_oracle_sample(w, chunks, n_heads=2, n_qblocks=None):
    """Time the oracle on a bounded sample of the decode step: its own layer
    state for the sampled heads (every chunk written through its own
    placement), the full score/update/select, and attention on their first
    query blocks.  Returns (attended FLOPs of the sample, seconds,
    description)."""
    import oracle as O
    import pbsa_inputs as PI
    H = n_heads
    orc = O.OracleLayer.of(PI.variant(w, H=H))
    for t, (_, k, v) in chunks.items():
        orc.write_chunk(t, k[:, :H], v[:, :H])
    t_cur = w.n_chunks - 1
    q = chunks[t_cur][0][:, :H]
    all_ids = [p for c in range(w.n_chunks) for p in orc.place.chunk_ids(c)]
    t0 = time.perf_counter()
    res = orc.step(t_cur, q, pool_ids=all_ids, attend=False)
    idx, cnt = res["idx"], res["cnt"]
    nq = idx.shape[2] if n_qblocks is None else n_qblocks
    lens = np.array([n for _, n in orc.place.blocks], dtype=np.int64)
    O.attention_fwd(q[:, :, :int(lens[:nq].sum())], orc.kp, orc.vp, orc.bl, orc.bp,
                    idx[:, :, :nq], cnt[:, :, :nq], orc.scale, w.mask, t_cur * w.chunk_tokens)
    dt = time.perf_counter() - t0
    fl = 0
    for h in range(H):
        for i in range(nq):
            ids = idx[0, h, i, :cnt[0, h, i]]
            fl += 4 * int(lens[i]) * int(orc.bl[0, h, ids].astype(np.int64).sum()) * w.D
    return fl, dt, f"{H} of {w.H} heads, {nq} of {idx.shape[2]} query blocks, full score/update/select"


def cores_used():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def config_of(w):
    nb_c = -(-w.chunk_tokens // w.bs)
    return {"workload": (f"decode step: B{w.B} H{w.H} D{w.D} bf16, {w.bs}-token blocks, "
                         f"query chunk {w.chunk_tokens} tokens ({nb_c} blocks), cache "
                         f"{w.n_chunks} chunks ({w.n_chunks * nb_c} blocks), P{w.P} "
                         f"W{w.W} chunks k{w.k}, evict"),
            "global_batch": w.B, "seq_len": w.chunk_tokens,
            "cache_tokens": w.n_chunks * w.chunk_tokens,
            "l2": "flushed between steps (256 MiB device write outside the timed events)",
            "parallelism": "replicas"}


# ----------------------------------------------------------------- main
def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "train":
        return run_train(args)
    if args.workload == "hbm":
        return run_hbm(args)
    if args.shard == "heads":
        return run_sharded(args)
    import torch
    rank, world, local = init_dist(args.gpus)
    pk, pk_kind = peaks()
    runner = DecodeRunner(seed_offset=rank)
    w = runner.w

    def timed_steps(fused, steps, clocks=None):
        """Mean device time of `steps` whole steps (graphs with events only at the
        step's start and end), after the warm-up."""
        n_graphs = max(1, min(64, steps))
        graphs, evs, s = runner.capture(n_graphs, fused=fused)
        with torch.cuda.stream(s):
            for i in range(args.warmup):
                graphs[i % n_graphs].replay()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        if clocks is not None:
            clocks.start()
        wall0 = time.perf_counter()
        times = []
        done = 0
        while done < steps:
            n = min(n_graphs, steps - done)
            with torch.cuda.stream(s):
                for i in range(n):
                    graphs[i].replay()
            torch.cuda.synchronize()
            times += [evs[i][0].elapsed_time(evs[i][-1]) for i in range(n)]
            done += n
        wall = time.perf_counter() - wall0
        barrier(world)
        clk = clocks.stop() if clocks is not None else None
        del graphs
        return float(np.mean(times)), wall, clk

    clocks = ClockSampler(local)
    ms_step, wall, clk = timed_steps(runner.fused, args.steps, clocks)
    # the other schedule, timed the same way on fewer steps (reported beside)
    ms_other, _, _ = timed_steps(not runner.fused, min(args.steps, 200))

    def breakdown(fused):
        """Per-call times from separate graphs with events between the calls."""
        n_bd = max(1, min(64, args.steps))
        gbd, ebd, sbd = runner.capture(n_bd, breakdown=True, fused=fused)
        with torch.cuda.stream(sbd):
            for i in range(args.warmup):
                gbd[i % n_bd].replay()
        torch.cuda.synchronize()
        rows = []
        for _ in range(max(1, min(args.steps, 256) // n_bd)):
            with torch.cuda.stream(sbd):
                for i in range(n_bd):
                    gbd[i].replay()
            torch.cuda.synchronize()
            rows += [[ebd[i][k].elapsed_time(ebd[i][k + 1]) for k in range(len(ebd[i]) - 1)]
                     for i in range(n_bd)]
        return np.array(rows)

    per = breakdown(True)                 # ms: routing call, attention
    per_unfused = breakdown(False)        # ms: score, update, select, attention
    ms_attn = float(per[:, 1].mean())
    ms_step_max = max_over_ranks(ms_step, world)
    flops = runner.flops()
    value = whole_job_tflops(flops, ms_step_max, world)
    attn_tflops = flops / (ms_attn * 1e-3) / 1e12
    peak = pk["bf16_tflops"]
    b_score, b_upd = runner.hbm_bytes()
    hbm = {}
    t_route = float(per[:, 0].mean()) * 1e-3
    for name, b, t in (("route_step (score + update + select)", b_score + b_upd, t_route),
                       ("score_blocks (per-call path)", b_score, float(per_unfused[:, 0].mean()) * 1e-3),
                       ("update_memory (per-call path)", b_upd, float(per_unfused[:, 1].mean()) * 1e-3)):
        hbm[name] = {"bytes": int(b), "ms": round(t * 1e3, 5), "gbs": round(b / t / 1e9, 1),
                     "frac": round(b / t / 1e9 / pk["hbm_gbs"], 4)}
    hbm["peak_gbs"] = pk["hbm_gbs"]
    hbm["peak_kind"] = f"hbm_gbs copy, {pk_kind}"
    hbm["timed"] = "call boundary to call boundary (CUDA events in the graph)"
    # HBM view of the HBM-bound calls: algorithmic bytes of score (read Q chunk +
    # new K blocks, write q_bar/k_bar/scores/mem) and of the update (copy 24 blocks)
    line = {
        "metric": "PBSA fwd effective TFLOP/s (attended blocks) & per-chunk latency",
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step_max, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/K/V, salience offsets N(0,2) on 10% of key blocks)",
        "config": config_of(w),
        "ms_per_step_by_schedule": {
            "routing kernel + attention": round(ms_step if runner.fused else ms_other, 5),
            "per-call path + attention": round(ms_other if runner.fused else ms_step, 5),
            "headline": "routing kernel + attention" if runner.fused else "per-call path + attention"},
        "per_call_ms": {"route_step": round(float(per[:, 0].mean()), 5),
                        "attn_fwd": round(ms_attn, 5),
                        "per_call_path": {
                            "score_blocks": round(float(per_unfused[:, 0].mean()), 5),
                            "update_memory": round(float(per_unfused[:, 1].mean()), 5),
                            "select_local": round(float(per_unfused[:, 2].mean()), 5),
                            "attn_fwd": round(float(per_unfused[:, 3].mean()), 5)},
                        "note": "separate graphs with events between the calls (each event "
                                "adds its own cost, so the sums exceed ms_per_step)"},
        "attended_gflop_per_step": round(flops / 1e9, 3),
        "roofline": {"kernel": "attn_fwd_kernel (D=128, bs=128)", "bound": "tensor",
                     "achieved": round(attn_tflops, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(attn_tflops / peak, 4), "traffic": attn_traffic(),
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "peak_kind": f"bf16_tflops burst, {pk_kind}"},
        "hbm": hbm,
        "gpu_launches": runner.launches_per_step * args.steps,
        "clocks": clk,
        "wall_s_timed_region": round(wall, 3),
    }
    if not args.no_e2e:
        e2e_ms, h2d, d2h = runner.e2e(steps=min(args.steps, 50), warmup=5)
        e2e_ms = max_over_ranks(e2e_ms, world)
        line["e2e"] = {"value": round(whole_job_tflops(flops, e2e_ms, world), 3), "unit": "TFLOP/s",
                       "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h,
                       "schedule": "pipelined decode loop: step t+1's inputs upload and step "
                                   "t-1's outputs download while step t computes (own "
                                   "streams, double-buffered staging); no L2 flush"}
    if world == 1 and not args.no_extras:
        extras = {"dense_comparators_on_decode_inputs": bench_dense_comparators(torch, runner,
                                                                                 runner.flush_buf)}
        extras["train"] = bench_train(torch, runner.flush_buf)
        extras["rollouts"] = bench_rollouts(torch)
        extras["hbm_at_scale"] = bench_hbm_at_scale(torch, runner.flush_buf, pk)
        extras["append_chunk"] = bench_append(torch, runner, pk)
        extras["select_hier"] = bench_select_hier(torch, runner)
        extras["rollout_backward"] = bench_rollout_backward(torch)
        line["extras"] = extras
    if rank == 0 and not args.no_cpu:
        fl, dt, desc = cpu_oracle_sample(w, runner.chunks)
        line["cpu_baseline"] = {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s",
                                "cores": cores_used(), "kind": "oracle", "sample": desc,
                                "seconds": round(dt, 2)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_train(args):
    """Forward + backward of the trainable shape (B2 H12 D128, 32 760 tokens) on
    the lists the library builds (persistent top-32 + local top-16).  One step
    is one forward and one backward; the metric counts 4 (forward) + 10
    (backward) x len_q x len_k x D FLOP per attended pair."""
    import torch
    import pbsa_inputs as PI
    from block_sparse_attention_39_b200.engine import PbsaTrain
    rank, world, local = init_dist(args.gpus)
    w = PI.WORKLOADS["train"]
    T = PbsaTrain(w)
    g = torch.Generator(device="cuda").manual_seed(w.seed + 1000 * rank)
    for t in (T.q, T.dO, T.kpool, T.vpool):
        t.copy_(torch.randn(t.shape, generator=g, device="cuda").bfloat16())
    T.set_meta()
    T.lists()
    torch.cuda.synchronize()
    lens = np.array([n for c in range(w.n_chunks) for n in T.layout.block_lens()], dtype=np.int64)
    ffl = _pair_flops(T.idx.cpu().numpy(), T.cnt.cpu().numpy(), T.blk_len.cpu().numpy(), lens,
                      w.D, 4)
    flops = ffl * (4 + 10) // 4
    for _ in range(args.warmup):
        T.fwd()
        T.bwd()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    for e in ev:
        e[0].record(s)
        T.fwd()
        e[1].record(s)
        T.bwd()
        e[2].record(s)
    torch.cuda.synchronize()
    barrier(world)
    ms_f = float(np.mean([a.elapsed_time(b) for a, b, _ in ev]))
    ms_b = float(np.mean([b.elapsed_time(c) for _, b, c in ev]))
    ms = max_over_ranks(ms_f + ms_b, world)
    if rank == 0:
        line = {"metric": "PBSA fwd+bwd effective TFLOP/s (trainable shape)",
                "value": round(whole_job_tflops(flops, ms, world), 3), "unit": "TFLOP/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1))",
                "config": {"workload": f"trainable shape B{w.B} H{w.H} D{w.D}, {T.T} tokens, "
                                       f"lists P{w.P} + top-{w.k}", "parallelism": "replicas"},
                "fwd_ms": round(ms_f, 4), "bwd_ms": round(ms_b, 4),
                "fwd_tflops": round(ffl / ms_f / 1e9, 1),
                "bwd_tflops": round(2.5 * ffl / ms_b / 1e9, 1),
                "gpu_launches": args.steps * 5}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_hbm(args):
    """The HBM-bound calls on bandwidth-sized work (see bench_hbm_at_scale)."""
    import torch
    rank, world, local = init_dist(args.gpus)
    pk, pk_kind = peaks()
    res = bench_hbm_at_scale(torch, None, pk, reps=max(1, args.steps))
    if rank == 0:
        best = min(v["frac"] for k, v in res.items() if isinstance(v, dict))
        line = {"metric": "PBSA HBM-bound calls: achieved HBM bandwidth at bandwidth scale "
                          "(lowest of the calls)",
                "value": round(best, 4), "unit": "fraction of measured HBM copy GB/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic (seeded N(0,1))",
                "config": {"workload": "score_blocks on the trainable shape; update_memory "
                                       "filling 128 slots of B2 H12; append_chunk of a "
                                       "32 760-token chunk, B2 H12", "parallelism": "replicas"},
                "calls": res, "peak_kind": pk_kind}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_sharded(args):
    """--shard heads: one layer of the 20-second rollout (B1 H12 D128 bf16, P48
    merge, window 2 chunks, top-16) split by heads over the ranks, strong
    scaling.  Every step each rank appends the chunk's K/V for its heads, runs
    score -> update -> select -> attend on them and all-gathers O over the
    ranks (NCCL), so every rank ends the step with the whole layer's output.
    Timed per step with CUDA events on the launching stream (no graphs: the
    step is the API call a caller makes), max over ranks; the FLOPs are the
    attended pairs of all heads.  L2 is not flushed: the step's pool and
    chunk tensors (about 330 MB for 12 heads) exceed the 126 MB L2."""
    import torch
    import pbsa_inputs as PI
    from block_sparse_attention_39_b200.shard import ShardedLayer
    rank, world, local = init_dist(args.gpus)
    warm = max(3, args.warmup, PI.WORKLOADS["rollout20s"].W + 2)
    steps = max(1, args.steps)
    w = PI.variant(PI.WORKLOADS["rollout20s"], n_chunks=warm + steps)
    S = ShardedLayer(w, world, rank)
    L = S.layer
    q_lens = np.array(L.layout.block_lens(), dtype=np.int64)
    ms, flops = [], 0
    for t in range(warm + steps):
        q, k, v = PI.chunk_tensors_device(w, t)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
        e0.record()
        S.step(t, q, k, v)
        e1.record()
        torch.cuda.synchronize()
        if t >= warm:
            ms.append(e0.elapsed_time(e1))
            flops += _pair_flops(L.idx.cpu().numpy(), L.cnt.cpu().numpy(),
                                 L.blk_len.cpu().numpy(), q_lens, w.D, 4)
    ms_step = max_over_ranks(float(np.mean(ms)), world)
    if world > 1:
        import torch.distributed as dist
        ft = torch.tensor([float(flops)], dtype=torch.float64, device="cuda")
        dist.all_reduce(ft)
        flops = ft.item()
    value = flops / steps / (ms_step * 1e-3) / 1e12
    if rank == 0:
        line = {"metric": "PBSA fwd effective TFLOP/s (attended blocks) & per-chunk latency",
                "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": steps,
                "warmup": warm, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded N(0,1) Q/K/V drawn on the device, salient blocks)",
                "config": {"workload": f"one layer of the 20-second rollout, B{w.B} H{w.H} "
                                       f"D{w.D} bf16, P{w.P} merge, W{w.W} chunks, k{w.k}, "
                                       f"steps {warm}..{warm + steps - 1}",
                           "global_batch": w.B, "seq_len": w.chunk_tokens,
                           "l2": "not flushed: the step's data exceed the 126 MB L2",
                           "parallelism": f"heads{world}"},
                "timed": "one step per pair of CUDA events: append, score, update, select, "
                         "attend and the all-gather of O"}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    """Reference arm: the CPU oracle, as it stands, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import pbsa_inputs as PI
    w = PI.WORKLOADS["decode"]
    chunks = PI.snapshot_chunks(w)
    times, fls = [], []
    desc = ""
    # keep the whole run to a few minutes: smaller samples when many steps are asked
    nq = 8 if args.warmup + args.steps <= 100 else 1
    for it in range(args.warmup + args.steps):
        fl, dt, desc = cpu_oracle_sample(w, chunks, n_heads=1, n_qblocks=nq)
        if it >= args.warmup:
            times.append(dt)
            fls.append(fl)
    ms = float(np.mean(times)) * 1e3
    value = float(np.mean(fls)) / (ms * 1e-3) / 1e12
    line = {"impl": "reference", "metric": "PBSA fwd effective TFLOP/s (attended blocks) & per-chunk latency",
            "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores_used(),
                             "kind": "oracle", "sample": "each step: " + desc},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
