#!/usr/bin/env python
"""Benchmark of block-compressed attention on B200.

One step = one decode step of the whole hot path for every sequence of the
workload: append the new raw token (ring write, running pooling softmax, and
pooling + finalisation of a block when it completes) and decode its query
(RoPE / RMSNorm of the query, scores over the visible pooled entries and the
raw window, softmax with sink, weighted values, split merge).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU, each rank
decodes its own sequences (weak scaling, no collective on the data path); the
step time is the max over ranks.  The inputs of the workload are resident in
HBM before timing.  Steps rotate over enough independent cache replicas
(more than 3x the L2 in total) that every step reads cold data, as the caches
of a model's layers and sequences are at every decode step; the K timed steps
are replayed back to back from one CUDA graph.  ``e2e`` repeats the steps
through the public API with each step's inputs copied from pinned host memory
and its output copied back inside the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode µs/token"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="ragged_gqa_decode_append",
                    help="the decode workload of the headline line (default: the largest single-GPU one)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--leg", default="decode", choices=["decode", "prefill", "pool", "csa", "backward", "chain"],
                    help="decode: the decode-step benchmark (default, with the other decode workloads, the "
                         "prefill and the pool legs appended under 'also' at one GPU); prefill / pool: that leg "
                         "alone (one JSON line)")
    ap.add_argument("--prefill", default="gqa_prefill_16k", help="workload of --leg prefill")
    ap.add_argument("--pool", default=next(iter(POOL_CASES)), choices=list(POOL_CASES), help="case of --leg pool")
    ap.add_argument("--no-also", action="store_true", help="the headline line alone")
    return ap.parse_args()


def peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------- clocks ----
class ClockSampler:
    """nvidia-smi samples (200 ms) of the benchmarked GPU during the timed region."""
    Q = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 10 and (self.uuid is None or self.uuid in f[1]):
                self.rows.append(f)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        rows = self.rows
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[6 + i] and "Not" not in r[6 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------- workload ----
def bytes_per_decode(w, lens):
    """Algorithmic HBM bytes of one decode launch: every visible pooled and raw
    entry read once (K and V, or the shared entry), the queries read and the
    outputs written once."""
    esize = 2 if w.dtype == "bf16" else 4
    series = 1 if w.shared_kv else 2
    total = 0
    for L in lens:
        L = int(L)
        P = max(0, (L - w.n_win) // w.block_m)
        total += (P + (L - P * w.block_m)) * w.n_kv_heads * w.head_dim * esize * series
    total += 2 * len(lens) * w.n_q_heads * w.head_dim * esize
    return total


class DecodeBench:
    """Decode workload state on one GPU: NR replicas of the workload's cache,
    each advanced by its own steps.  Steps rotate over the replicas so that
    the data of each step has been evicted from L2 by the other replicas'
    traffic (the replicas together hold more than 3x the L2 size), the way the
    caches of a model's many layers and sequences are cold at every step."""

    def __init__(self, w, rank, min_steps):
        import torch

        from block_compressed_long_b200 import lbca as L
        from block_compressed_long_b200 import ranks, synth
        self.L, self.torch = L, torch
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        base = synth.scaled(w, steps=1)
        lens0 = synth.contexts(base)
        step_bytes = bytes_per_decode(base, lens0 + 1)
        self.NR = max(1, -(-3 * l2 // step_bytes))
        self.local_steps = -(-min_steps // self.NR) + 1
        self.w = synth.scaled(ranks.rank_workload(w, rank), steps=self.local_steps)
        self.inp = synth.make(self.w)
        w = self.w
        self.cfg = L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win,
                            w.rope_dims, w.rmsnorm, w.rope_theta, dtype=w.dtype)
        B = w.batch
        self.B = B
        self.max_ctx = int(self.inp.lens.max()) + self.local_steps
        d = lambda t: None if t is None else t.cuda()  # noqa: E731
        k, v, zk, zv = (d(t) for t in (self.inp.k, self.inp.v, self.inp.zk, self.inp.zv))
        self.bpk, self.bpv, self.sink = d(self.inp.bpos_k), d(self.inp.bpos_v), d(self.inp.sink)
        self.q = d(self.inp.q)
        c0 = L.Cache.allocate(self.cfg, B, self.max_ctx)
        per = c0.pool_state.numel() // B
        ws0 = torch.zeros(16, dtype=torch.uint8, device="cuda")
        for b in range(B):  # build each sequence's cache with the prefill path (cache only)
            Lb = int(self.inp.lens[b])
            sc = L.Cache(self.cfg, 1, c0.max_blocks, c0.ring_slots, c0.pooled_k[b:b + 1],
                         None if c0.pooled_v is None else c0.pooled_v[b:b + 1], c0.ring_k[b:b + 1],
                         None if c0.ring_v is None else c0.ring_v[b:b + 1], c0.pool_state[b * per:(b + 1) * per],
                         c0.seq_lens[b:b + 1])
            s = lambda t: None if t is None else t[b:b + 1, :Lb]  # noqa: E731
            L.lbca_prefill(self.cfg, None, s(k), s(v), s(zk), s(zv), self.bpk, self.bpv,
                           None, None, None, None, sc, ws0, batch=1, T=Lb)
        cl = lambda t: None if t is None else t.clone()  # noqa: E731
        self.caches = [c0] + [L.Cache(self.cfg, B, c0.max_blocks, c0.ring_slots, cl(c0.pooled_k), cl(c0.pooled_v),
                                      cl(c0.ring_k), cl(c0.ring_v), cl(c0.pool_state), cl(c0.seq_lens))
                              for _ in range(self.NR - 1)]
        del k, v, zk, zv
        torch.cuda.synchronize()
        torch.cuda.empty_cache()  # the raw token history is no longer needed: hand its memory back
        wsb = max(L.lbca_decode_step_workspace_bytes(self.cfg, B, self.max_ctx), 16)
        self.step_ws = [torch.zeros(wsb, dtype=torch.uint8, device="cuda") for _ in range(self.NR)]
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.launches = L.lbca_decode_step_launches(self.cfg, B, self.max_ctx)
        self.form = L.lbca_decode_step_form(self.cfg, B, self.max_ctx)
        self.dec_ws = []
        if self.launches == 2:
            dwb = max(L.lbca_decode_workspace_bytes(self.cfg, B, self.max_ctx), 16)
            self.dec_ws = [torch.zeros(dwb, dtype=torch.uint8, device="cuda") for _ in range(self.NR)]
        # per-step token inputs, gathered once: [local_steps, B, G, D]
        ar = torch.arange(B)
        pos = torch.as_tensor(self.inp.lens)
        tok = lambda t: None if t is None else torch.stack(  # noqa: E731
            [t[ar, pos + i] for i in range(self.local_steps)]).cuda()
        self.tk, self.tv, self.tzk, self.tzv = (tok(t) for t in (self.inp.k, self.inp.v, self.inp.zk, self.inp.zv))
        self.outs = [torch.empty(B, w.n_q_heads, w.head_dim, dtype=L.torch_dtype(self.cfg), device="cuda")
                     for _ in range(self.NR)]
        self.i = 0  # global step counter; step i uses replica i % NR, local step i // NR

    def lens_at(self, i):
        return self.inp.lens + i // self.NR + 1

    def launch_decode(self, i):
        """Enqueue only the decode launch of global step i (replica i % NR, at
        the replica's current lengths): times the attention kernel of a step
        that runs as append + decode."""
        L = self.L
        rep, j = i % self.NR, i // self.NR
        L.lbca_decode(self.cfg, self.q[j], self.caches[rep], self.sink, None, None, self.outs[rep], self.dec_ws[rep],
                      self.max_ctx, self.status)

    def launch(self, i, q=None, tok=None):
        """Enqueue global step i (lbca_decode_step on replica i % NR)."""
        L = self.L
        rep, j = i % self.NR, i // self.NR
        g = lambda t: None if t is None else t[j]  # noqa: E731
        k, v, zk, zv = tok if tok is not None else (g(self.tk), g(self.tv), g(self.tzk), g(self.tzv))
        q = self.q[j] if q is None else q
        L.lbca_decode_step(self.cfg, k, v, zk, zv, self.bpk, self.bpv, None, q, self.caches[rep], self.sink, None,
                           self.outs[rep], self.step_ws[rep], self.max_ctx, self.status)


def run_ours(args, w, rank, world, reps=3):
    """Decode steps of workload `w` on this GPU: W warm-up steps, then K steps
    replayed back to back from one CUDA graph, `reps` times (median taken, the
    clock sampler running throughout); then the end-to-end loop (e2e_loop).
    Returns (JSON line, bench)."""
    import torch
    import torch.distributed as dist

    from block_compressed_long_b200 import ranks

    K, W = args.steps, args.warmup
    # steps each replica must hold: warm-up, reps graph replays, decode-only
    # timing of a two-launch step, e2e warm-up and steps
    bench = DecodeBench(w, rank, W + 2 * reps * K + (W + K) + (W + K))
    L = bench.L
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    cap = torch.cuda.Stream()

    def graph_of(first, n, body):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=cap):
            for i in range(first, first + n):
                body(i)
        return gr

    # warm-up (eager, sets kernel attributes), then K steps captured in one graph
    for _ in range(W):
        bench.launch(bench.i)
        bench.i += 1
    torch.cuda.synchronize()
    nbytes = sum(bytes_per_decode(bench.w, bench.lens_at(i)) for i in range(bench.i, bench.i + K))
    uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    # Consecutive steps run on different cache replicas (as a model's layers
    # follow each other), which is the contract of LBCA_CACHE_OVERLAP_PREV:
    # timed with the replicas flagged (each step starts and reads its cache
    # while the previous one drains) and without.
    medians = {}
    for flags in (L.LBCA_CACHE_OVERLAP_PREV, 0):
        for c in bench.caches:
            c.flags = flags
        g_main = graph_of(bench.i, K, bench.launch)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        times = []
        for _ in range(reps):  # each replay appends K more tokens per replica: the cache holds them
            e0, e1 = E(), E()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            e0.record()
            g_main.replay()
            e1.record()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            times.append(e0.elapsed_time(e1) / K)
        medians[flags] = statistics.median(times)
        del g_main
    for c in bench.caches:
        c.flags = 0
    step_ms = medians[L.LBCA_CACHE_OVERLAP_PREV]
    serial_ms = medians[0]
    bench.i += K
    kernel_ms = step_ms  # one fused kernel per step: the step is the kernel
    if bench.launches == 2:
        # append + decode: time the decode launches alone (same replicas, same rotation)
        for i in range(bench.i, bench.i + W):
            bench.launch_decode(i)
        g_dec = graph_of(bench.i, K, bench.launch_decode)
        torch.cuda.synchronize()
        e0, e1 = E(), E()
        e0.record()
        g_dec.replay()
        e1.record()
        torch.cuda.synchronize()
        kernel_ms = e0.elapsed_time(e1) / K
        del g_dec
    e2e_ms, h2d, d2h = e2e_loop(bench, K, W)
    clocks = sampler.stop()
    status = int(bench.status.item())
    if status:
        raise RuntimeError(f"device status {L.lbca_status_string(status)}")

    step_ms, e2e_ms, kernel_ms, serial_ms = ranks.max_over_ranks([step_ms, e2e_ms, kernel_ms, serial_ms],
                                                                 device="cuda")
    hbm, src = peaks()
    achieved = nbytes / K / (kernel_ms * 1e-3) / 1e9
    w_ = bench.w
    line = {
        "metric": METRIC, "value": ranks.job_us_per_token(step_ms, bench.B, world), "unit": "µs/token",
        "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": step_ms, "serial_ms_per_step": serial_ms,
        "serial_value": ranks.job_us_per_token(serial_ms, bench.B, world), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": w_.dtype, "data": "synthetic",
        "config": {"workload": w_.name, "batch_per_gpu": w_.batch, "context": [int(w_.ctx[0]), int(w_.ctx[1])],
                   "n_q_heads": w_.n_q_heads, "n_kv_heads": w_.n_kv_heads, "head_dim": w_.head_dim,
                   "block_m": w_.block_m, "n_win": w_.n_win, "rope_dims": w_.rope_dims,
                   "shared_kv": w_.shared_kv, "parallelism": f"dp{world}",
                   "l2": (f"inputs larger than L2: steps rotate over {bench.NR} cache replicas "
                          f"(>= 3x L2 of data in total), each step's data cold"),
                   "launch": (f"K steps of lbca_decode_step ({bench.launches} kernel launch"
                              f"{'es' if bench.launches > 1 else ''} each), back to back from one CUDA graph, "
                              f"median of {reps} replays, the replicas flagged LBCA_CACHE_OVERLAP_PREV (each step "
                              "reads its cache while the previous step, on another replica, drains); "
                              "serial_value: the same graph without the flag; "
                              "e2e: an eager host loop of lbca_decode_step calls "
                              "(host-side validation and launch every step), each step's inputs uploaded from "
                              "pinned host memory and its output read back on copy streams beside the kernels, "
                              "timed as the longer of the device events and the host wall clock")},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "peak_source": src,
                     "kernel": ({L.LBCA_STEP_CLUSTER: "decode_step_kernel (cluster form)",
                                 L.LBCA_STEP_PERSISTENT: "decode_flat_kernel (persistent evenly split form)",
                                 L.LBCA_STEP_SHARED_TC: "decode_mqa_tc_kernel (shared-entry tensor-core form, "
                                                        "append fused)"}
                                .get(bench.form, "the decode launch of the step (timed alone over the same replicas)")),
                     "bytes_per_launch": nbytes / K, "launch_us": kernel_ms * 1e3,
                     "traffic": load_traffic(w_.name)},
        "e2e": {"value": ranks.job_us_per_token(e2e_ms, bench.B, world), "unit": "µs/token",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": K * bench.launches,
        "clocks": clocks,
    }
    return line, bench


class _Driver:
    """The few CUDA driver calls the end-to-end loop issues per step (one
    asynchronous copy each way, event record and stream wait), called through
    ctypes: a fraction of the host time of the same operations through the
    torch dispatcher.  Streams are torch's (their handles are driver streams)."""

    def __init__(self):
        import ctypes
        d = ctypes.CDLL("libcuda.so.1")
        u64, vp, sz = ctypes.c_uint64, ctypes.c_void_p, ctypes.c_size_t
        d.cuMemcpyHtoDAsync_v2.argtypes = [u64, vp, sz, vp]
        d.cuMemcpyDtoHAsync_v2.argtypes = [vp, u64, sz, vp]
        d.cuEventCreate.argtypes = [ctypes.POINTER(vp), ctypes.c_uint]
        d.cuEventRecord.argtypes = [vp, vp]
        d.cuStreamWaitEvent.argtypes = [vp, vp, ctypes.c_uint]
        d.cuEventDestroy_v2.argtypes = [vp]
        self.d, self.ct = d, ctypes
        self.events = []

    def _ok(self, r, what):
        if r != 0:
            raise RuntimeError(f"{what} failed with CUresult {r}")

    def event(self):
        ev = self.ct.c_void_p()
        self._ok(self.d.cuEventCreate(self.ct.byref(ev), 2), "cuEventCreate")  # CU_EVENT_DISABLE_TIMING
        self.events.append(ev)
        return ev

    def h2d(self, dst, src, n, stream):
        self._ok(self.d.cuMemcpyHtoDAsync_v2(dst, src, n, stream), "cuMemcpyHtoDAsync")

    def d2h(self, dst, src, n, stream):
        self._ok(self.d.cuMemcpyDtoHAsync_v2(dst, src, n, stream), "cuMemcpyDtoHAsync")

    def record(self, ev, stream):
        self._ok(self.d.cuEventRecord(ev, stream), "cuEventRecord")

    def wait(self, stream, ev):
        self._ok(self.d.cuStreamWaitEvent(stream, ev, 0), "cuStreamWaitEvent")

    def close(self):
        for ev in self.events:
            self.d.cuEventDestroy_v2(ev)
        self.events = []


def e2e_loop(bench, K, W):
    """The decode steps end to end through the public API, eagerly: each step
    is one lbca_decode_step call from the host (argument validation and launch
    included), its inputs (q and the new token's k, v, z_k, z_v, packed in one
    pinned host buffer) cross with one copy and its output comes back with one
    copy.  As in a serving loop the copies run on streams of their own beside
    the kernels (step i+1's upload overlaps step i's kernel, step i's download
    overlaps step i+1's; two staging slots; every step waits for its own
    upload, every download for its own step); copies and events go to the
    driver directly (`_Driver`).  Returns (ms per step = the longer of the
    device-event span and the host wall clock, H2D bytes and D2H bytes per
    step)."""
    import torch

    parts = [bench.q] + [t for t in (bench.tk, bench.tv, bench.tzk, bench.tzv) if t is not None]
    sizes = [t[0].numel() * t[0].element_size() for t in parts]
    offs = np.cumsum([0] + sizes)
    nloc = bench.q.shape[0]
    hstage = torch.empty(nloc, int(offs[-1]), dtype=torch.uint8).pin_memory()
    for pi, t in enumerate(parts):
        hstage[:, offs[pi]:offs[pi + 1]] = t.cpu().contiguous().view(nloc, -1).view(torch.uint8)
    NS = 2  # staging slots
    dstage = [torch.empty(int(offs[-1]), dtype=torch.uint8, device="cuda") for _ in range(NS)]
    dq, dtok = [], []
    for sl in range(NS):
        views = [dstage[sl][offs[pi]:offs[pi + 1]].view(parts[pi].dtype).view(parts[pi][0].shape)
                 for pi in range(len(parts))]
        it = iter(views[1:])
        dq.append(views[0])
        dtok.append([None if t is None else next(it) for t in (bench.tk, bench.tv, bench.tzk, bench.tzv)])
    hout = [torch.empty(bench.outs[0].shape, dtype=bench.outs[0].dtype).pin_memory() for _ in range(NS)]
    h2d = int(offs[-1])
    d2h = hout[0].numel() * hout[0].element_size()
    drv = _Driver()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    h_in, h_out, h_cur = s_in.cuda_stream, s_out.cuda_stream, torch.cuda.current_stream().cuda_stream
    ev_in = [drv.event() for _ in range(NS)]          # slot's upload done
    ev_run = [drv.event() for _ in range(NS)]         # the step that read the slot is done
    ev_down = [drv.event() for _ in range(bench.NR)]  # download of an output replica done
    ev_join = drv.event()
    dst_in = [t.data_ptr() for t in dstage]
    src_out = [t.data_ptr() for t in bench.outs]
    dst_out = [t.data_ptr() for t in hout]
    row = hstage.stride(0)

    def steps(first, n):
        base = hstage.data_ptr()
        for j, i in enumerate(range(first, first + n)):
            sl, rep = j % NS, i % bench.NR
            if j >= NS:
                drv.wait(h_in, ev_run[sl])       # the step two back has read this slot
            drv.h2d(dst_in[sl], base + (i // bench.NR) * row, h2d, h_in)
            drv.record(ev_in[sl], h_in)
            drv.wait(h_cur, ev_in[sl])
            if j >= bench.NR:
                drv.wait(h_cur, ev_down[rep])    # this output replica has been read back
            bench.launch(i, q=dq[sl], tok=dtok[sl])
            drv.record(ev_run[sl], h_cur)
            drv.wait(h_out, ev_run[sl])
            drv.d2h(dst_out[sl], src_out[rep], d2h, h_out)
            drv.record(ev_down[rep], h_out)
        for h in (h_in, h_out):  # join both copy streams back
            drv.record(ev_join, h)
            drv.wait(h_cur, ev_join)

    steps(bench.i, W)
    bench.i += W
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    e0.record()
    steps(bench.i, K)
    e1.record()
    torch.cuda.synchronize()
    wall_ms = (time.perf_counter() - t0) * 1e3
    bench.i += K
    drv.close()
    return max(e0.elapsed_time(e1), wall_ms) / K, h2d, d2h


def decode_also(args, name):
    """One more decode workload at N = 1 (its own line under "also"), with the
    oracle beside it."""
    import gc

    import torch

    from block_compressed_long_b200 import synth
    line, bench = run_ours(args, synth.WORKLOADS[name], 0, 1)
    del bench
    gc.collect()
    torch.cuda.empty_cache()
    for k in ("n_gpus", "steps", "warmup", "scaling", "vs_baseline", "data"):
        line.pop(k, None)
    line = {"workload": name, **line}
    us, n, cores, desc = oracle_decode_timing(synth.WORKLOADS[name])
    line["cpu_baseline"] = {"value": us, "unit": "µs/token", "cores": cores, "kind": "oracle", "sample": desc}
    return line


def peak_tflops():
    try:
        with open(PEAKS_PATH) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (bf16 burst; fp16 has the same dense rate)"
    except Exception:
        return 1590.0, "fallback"


# FP32 CUDA-core peak of one B200: 148 SMs x 128 FP32 lanes x 2 flops per FMA x
# 1965 MHz (the SM clock the machine's GPUs run at under load) = 74.4 TFLOP/s.
F32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def prefill_pairs(w, rows=None):
    """Visible (query, entry) pairs of the rows (all T by default), per head
    and sequence."""
    m, n = w.block_m, w.n_win
    rows = range(w.seq_len) if rows is None else rows
    pairs = 0
    for t in rows:
        L = t + 1
        P = max(0, (L - n) // m)
        pairs += P + (L - P * m)
    return pairs


def prefill_flops(w, rows=None):
    """Algorithmic FLOPs: 4 D Hq per visible (query, entry) pair."""
    return 4.0 * w.head_dim * w.n_q_heads * prefill_pairs(w, rows) * w.batch


def timed(run, reps, warm, uuid=None):
    """Median over `reps` CUDA-event-timed calls of run() (ms), after `warm`
    untimed calls, with the clock sampler running."""
    import torch
    for _ in range(warm):
        run()
    torch.cuda.synchronize()
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts), sampler.stop()


def prefill_leg(name="gqa_prefill_16k", reps=10, warm=3, baseline=True):
    """lbca_prefill of a prefill workload (pool pass, RoPE table, finalised
    keys, attention), inputs resident in HBM (larger than L2 for the 16K
    layer), CUDA events; the oracle on a bounded sample beside it."""
    import torch

    from block_compressed_long_b200 import lbca as L
    from block_compressed_long_b200 import synth
    w = synth.WORKLOADS[name]
    inp = synth.make(w)
    cfg = L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   w.rmsnorm, w.rope_theta, dtype=w.dtype)
    d = lambda t: None if t is None else t.cuda()  # noqa: E731
    q, k, v, zk, zv, bpk, bpv, sink = (d(t) for t in (inp.q, inp.k, inp.v, inp.zk, inp.zv, inp.bpos_k, inp.bpos_v,
                                                      inp.sink))
    out = torch.empty_like(q)
    ws = torch.zeros(max(L.lbca_prefill_workspace_bytes(cfg, w.batch, w.seq_len, False), 16), dtype=torch.uint8,
                     device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    ms, clocks = timed(lambda: L.lbca_prefill(cfg, q, k, v, zk, zv, bpk, bpv, sink, None, None, out, None, ws,
                                              d_status=st), reps, warm, uuid)
    if int(st.item()):
        raise RuntimeError(f"prefill device status {L.lbca_status_string(int(st.item()))}")
    fl = prefill_flops(w)
    tf = fl / (ms * 1e-3) / 1e12
    if w.dtype == "bf16":
        pk, src = peak_tflops()
        roof = {"bound": "tensor", "achieved": tf, "peak": pk, "unit": "TFLOP/s", "frac": tf / pk,
                "peak_source": src, "kernel": "prefill_tc_kernel (whole lbca_prefill call timed)"}
        dt = "bf16 I/O, fp16 tensor-core operands, f32 accumulate"
    else:
        roof = {"bound": "alu", "achieved": tf, "peak": F32_ALU_TFLOPS, "unit": "TFLOP/s",
                "frac": tf / F32_ALU_TFLOPS, "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 x 1965 MHz",
                "kernel": "prefill_simt_kernel (whole lbca_prefill call timed)"}
        dt = "f32 I/O and arithmetic (CUDA cores, no TF32)"
    roof["flops_per_call"] = fl
    line = {"workload": name, "metric": "prefill TFLOP/s", "value": tf, "unit": "TFLOP/s", "ms_per_call": ms,
            "dtype": dt, "roofline": roof, "clocks": clocks}
    del q, k, v, zk, zv, out, ws
    torch.cuda.empty_cache()
    if baseline:
        line["cpu_baseline"] = oracle_prefill_timing(w, inp)
    return line


def backward_leg(T=2048, reps=5, warm=2):
    """lbca_prefill_backward of a T-token GQA layer (the 16K prefill layer's
    shapes, m = 16): all gradients in f32 on the CUDA cores.  Algorithmic
    flops: 10 D Hq per visible (query, entry) pair (the scores recomputed, and
    the products giving dP, dQ, dK and dV)."""
    import torch

    from block_compressed_long_b200 import lbca as L
    from block_compressed_long_b200 import synth
    w = synth.scaled(synth.WORKLOADS["gqa_prefill_16k"], seq_len=T)
    inp = synth.make(w)
    cfg = L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   w.rmsnorm, w.rope_theta, dtype=w.dtype)
    d = lambda t: None if t is None else t.cuda()  # noqa: E731
    q, k, v, zk, zv, bpk, bpv = (d(t) for t in (inp.q, inp.k, inp.v, inp.zk, inp.zv, inp.bpos_k, inp.bpos_v))
    dout = d(synth.normal(w.seed, "dout", tuple(inp.q.shape), dtype=w.dtype))
    f = lambda *sh: torch.empty(*sh, dtype=torch.float32, device="cuda")  # noqa: E731
    G, D, m = w.n_kv_heads, w.head_dim, w.block_m
    grads = {"dq": f(*q.shape), "dk": f(*k.shape), "dv": f(*k.shape), "dzk": f(*k.shape), "dzv": f(*k.shape),
             "dbk": f(m, G * D), "dbv": f(m, G * D)}
    ws = torch.zeros(L.lbca_prefill_backward_workspace_bytes(cfg, w.batch, T), dtype=torch.uint8, device="cuda")
    uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    ms, clocks = timed(lambda: L.lbca_prefill_backward(cfg, q, k, v, zk, zv, bpk, bpv, None, None, None, dout, grads,
                                                       ws), reps, warm, uuid)
    fl = 2.5 * prefill_flops(w)
    tf = fl / (ms * 1e-3) / 1e12
    return {"workload": f"gqa_prefill_16k shapes, T = {T}: prefill backward", "metric": "backward TFLOP/s",
            "value": tf, "unit": "TFLOP/s", "ms_per_call": ms, "dtype": "bf16 inputs, f32 arithmetic and gradients",
            "roofline": {"bound": "alu", "achieved": tf, "peak": F32_ALU_TFLOPS, "unit": "TFLOP/s",
                         "frac": tf / F32_ALU_TFLOPS, "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 x 1965 MHz",
                         "flops_per_call": fl,
                         "kernel": "pool_fwd, finalise, row_lse, dq, dkv, key_bwd, pool_bwd kernels (call timed)"},
            "clocks": clocks}


POOL_CASES = {
    "csa_sparse_decode_64k (4 x 65536 tokens, D = 512, m = 4, dual overlapped a/b series: RMSNorm and RoPE "
    "epilogue)": ("csa_sparse_decode_64k", 65536, 4, (0,)),
    # name: (workload, tokens, batch, series)
    "gqa_decode_32k prefix (32768 tokens, K and V series)": ("gqa_decode_32k", 32768, 1, (0, 1)),
    "gqa_prefill_16k (16384 tokens, m = 16, K and V series)": ("gqa_prefill_16k", 16384, 1, (0, 1)),
    "hca_mqa_decode_128k (8 x 131072 tokens, D = 512, shared entries: RMSNorm and RoPE epilogue)":
        ("hca_mqa_decode_128k", 131072, 8, (0,)),
}


def pool_leg(label, reps=10, warm=3, baseline=True):
    """Pooling of every complete block of a workload's raw K/V (or C): both
    series of the GQA form in one lbca_pool_kv launch, the shared form's one
    series by lbca_pool (HBM-bound: X and Z read once, entries written)."""
    import torch

    from block_compressed_long_b200 import lbca as L
    from block_compressed_long_b200 import synth
    name, T, B, series = POOL_CASES[label]
    # the raw series of T tokens per sequence (no queries are drawn: steps = 0)
    w = synth.scaled(synth.WORKLOADS[name], kind="decode", ctx=(T, T), seq_len=T, batch=B, steps=0, index_heads=0)
    inp = synth.make(w)
    cfg = L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   w.rmsnorm, w.rope_theta, dtype=w.dtype)
    d = lambda t: None if t is None else t.cuda()  # noqa: E731
    srcs = [(d(inp.k), d(inp.zk), d(inp.bpos_k))] + ([] if w.shared_kv else [(d(inp.v), d(inp.zv), d(inp.bpos_v))])
    nb = T // w.block_m
    outs = [torch.empty(B, w.n_kv_heads, nb, w.head_dim, dtype=L.torch_dtype(cfg), device="cuda") for _ in srcs]

    dual = w.dual
    if dual:  # the b-series of the dual overlapped form
        xb, zb, bpb = d(inp.csa["kb"]), d(inp.csa["zkb"]), d(inp.csa["bpos_kb"])

    def run():
        if len(srcs) == 2:
            (k, zk, bpk), (v, zv, bpv) = srcs
            L.lbca_pool_kv(cfg, k, v, zk, zv, bpk, bpv, None, outs[0], outs[1])
            return
        for s, (x, z, bp) in zip(series, srcs):
            if dual:
                L.lbca_pool_dual(cfg, s, x, z, xb, zb, bp, bpb, None, outs[s])
            else:
                L.lbca_pool(cfg, s, x, z, bp, None, outs[s])

    uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    ms, clocks = timed(run, reps, warm, uuid)
    esz = 2 if w.dtype == "bf16" else 4
    nbytes = sum((4 if dual else 2) * x.numel() * esz + o.numel() * esz for (x, _, _), o in zip(srcs, outs))
    gbs = nbytes / (ms * 1e-3) / 1e9
    hbm, src = peaks()
    line = {"workload": label, "metric": "pool GB/s", "value": gbs, "unit": "GB/s", "ms_per_call": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "peak_source": src, "kernel": "pool_kernel" + (" (dual overlapped form)" if dual else ""),
                         "bytes_per_call": nbytes,
                         "launches_per_call": 1},
            "clocks": clocks}
    del srcs, outs
    if dual:
        del xb, zb, bpb
    torch.cuda.empty_cache()
    if baseline:
        line["cpu_baseline"] = oracle_pool_timing(w, inp, series)
    return line


def layer_chain_leg(NL=14, K=20, W=3, reps=3):
    """One token through NL LBCA layers of the 32K GQA shape (the README's
    retrofit replaces 14 of the 3B model's 28 layers): layer l's query is layer
    l-1's output, so the steps form a true dependency chain, each layer with
    its own cache, K tokens back to back from one CUDA graph.  Timed twice:
    with the caches flagged LBCA_CACHE_OVERLAP_PREV (each layer's step starts
    and reads its cache while the previous layer's kernel drains; programmatic
    dependent launch) and without.  Chains rotate over replicas holding more
    than 3x the L2 of cache, so every step reads cold data."""
    import gc

    import torch

    from block_compressed_long_b200 import lbca as L
    from block_compressed_long_b200 import synth
    w = synth.WORKLOADS["gqa_decode_32k"]
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    lens0 = synth.contexts(w)
    per_layer = bytes_per_decode(w, lens0 + 1)
    NR = max(1, -(-3 * l2 // (per_layer * NL)))
    total_steps = W + 2 * reps * K + W
    local = -(-total_steps // NR) + 1
    ws_ = synth.scaled(w, steps=local)
    inp = synth.make(ws_)
    cfg = L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   w.rmsnorm, w.rope_theta, dtype=w.dtype)
    max_ctx = int(inp.lens.max()) + local
    c0 = L.Cache.allocate(cfg, 1, max_ctx)
    d = lambda t: None if t is None else t.cuda()  # noqa: E731
    n0 = int(inp.lens[0])
    L.lbca_prefill(cfg, None, d(inp.k[:, :n0]), d(inp.v[:, :n0]), d(inp.zk[:, :n0]), d(inp.zv[:, :n0]),
                   d(inp.bpos_k), d(inp.bpos_v), None, None, None, None, c0,
                   torch.zeros(16, dtype=torch.uint8, device="cuda"), batch=1, T=n0)
    cl = lambda t: None if t is None else t.clone()  # noqa: E731
    chains = [[L.Cache(cfg, 1, c0.max_blocks, c0.ring_slots, cl(c0.pooled_k), cl(c0.pooled_v), cl(c0.ring_k),
                       cl(c0.ring_v), cl(c0.pool_state), cl(c0.seq_lens)) for _ in range(NL)] for _ in range(NR)]
    del c0
    wsb = max(L.lbca_decode_step_workspace_bytes(cfg, 1, max_ctx), 16)
    wss = [[torch.zeros(wsb, dtype=torch.uint8, device="cuda") for _ in range(NL)] for _ in range(NR)]
    outs = [[torch.empty(1, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda") for _ in range(NL)]
            for _ in range(NR)]
    tok = [d(t[:, n0:n0 + local].transpose(0, 1).contiguous()) for t in (inp.k, inp.v, inp.zk, inp.zv)]
    q0 = d(inp.q[:, 0].contiguous())
    bpk, bpv = d(inp.bpos_k), d(inp.bpos_v)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    launches = L.lbca_decode_step_launches(cfg, 1, max_ctx)

    def token(i, flags):
        r, j = i % NR, (i // NR) % local
        q = q0[j]
        for layer in range(NL):
            c = chains[r][layer]
            c.flags = flags
            L.lbca_decode_step(cfg, tok[0][j], tok[1][j], tok[2][j], tok[3][j], bpk, bpv, None, q, c, None, None,
                               outs[r][layer], wss[r][layer], max_ctx, status)
            q = outs[r][layer]  # the next layer attends with this layer's output

    i = 0
    for _ in range(W):
        token(i, 0)
        i += 1
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    res = {}
    uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    for name, flags in (("overlap", L.LBCA_CACHE_OVERLAP_PREV), ("serial", 0)):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=cap):
            for ii in range(i, i + K):
                token(ii, flags)
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record()
            gr.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) / K)
        i += K
        res[name] = statistics.median(ts)
        del gr
    clocks = sampler.stop()
    st = int(status.item())
    if st:
        raise RuntimeError(f"layer chain device status {L.lbca_status_string(st)}")
    ms = res["overlap"]
    hbm, src = peaks()
    nbytes = NL * per_layer
    gbs = nbytes / (ms * 1e-3) / 1e9
    del chains, wss, outs, tok
    gc.collect()
    torch.cuda.empty_cache()
    return {"workload": f"layer chain: {NL} LBCA layers of gqa_decode_32k, one token, each layer's query the "
                        "previous layer's output", "metric": "decode µs/token (all layers)", "value": ms * 1e3,
            "unit": "µs/token", "serial_us_per_token": res["serial"] * 1e3, "per_layer_us": ms * 1e3 / NL,
            "config": {"layers": NL, "launches_per_layer": launches,
                       "l2": f"chains rotate over {NR} replicas of {NL} caches (>= 3x L2), each step's data cold",
                       "launch": (f"{K} tokens x {NL} lbca_decode_step calls back to back from one CUDA graph, "
                                  f"median of {reps}; caches flagged LBCA_CACHE_OVERLAP_PREV (programmatic "
                                  "dependent launch); serial_us_per_token: the same graph without the flag")},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "peak_source": src, "bytes_per_token": nbytes,
                         "kernel": "decode_step_kernel (cluster form) x layers"},
            "gpu_launches": K * NL * launches, "clocks": clocks}


class CsaBench:
    """The CSA workload's decode state on one GPU, built through the C ABI:
    dual-pooled finalised entries, dual-pooled indexer keys, the raw window
    and the lengths, cloned into NR replicas that together hold more than 3x
    the L2 so that every step reads cold data.  A step, for every sequence:
    lightning-indexer relevance and top-k (lbca_indexer_topk), then the
    sparse attention over the selected entries and the window
    (lbca_decode_sparse); the cache is not advanced (no append)."""

    def __init__(self, w, steps):
        import torch

        from block_compressed_long_b200 import lbca as L
        from block_compressed_long_b200 import synth
        self.L, self.w = L, w
        ws = synth.scaled(w, steps=steps)
        inp = synth.make(ws)
        self.inp = inp
        B = w.batch
        self.cfg = L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                            w.rmsnorm, w.rope_theta, dtype=w.dtype)
        icfg = L.config(1, 1, w.index_dim, True, w.block_m, w.n_win, 0, False, dtype=w.dtype)
        lens = np.asarray(inp.lens, dtype=np.int64)
        c0 = L.Cache.allocate(self.cfg, B, int(lens.max()) + 1)
        nb = c0.max_blocks
        kidx = torch.zeros(B, 1, nb, w.index_dim, dtype=torch.bfloat16, device="cuda")
        c = inp.csa
        d = lambda t: t.contiguous().cuda()  # noqa: E731
        for b in range(B):
            n = int(lens[b])
            sl = lambda t: d(t[b:b + 1, :n])  # noqa: E731
            L.lbca_pool_dual(self.cfg, L.LBCA_KEY, sl(inp.k), sl(inp.zk), sl(c["kb"]), sl(c["zkb"]), d(inp.bpos_k),
                             d(c["bpos_kb"]), None, c0.pooled_k[b:b + 1], nb)
            L.lbca_pool_dual(icfg, L.LBCA_VALUE, sl(c["ika"]), sl(c["izka"]), sl(c["ikb"]), sl(c["izkb"]),
                             d(c["ibpa"]), d(c["ibpb"]), None, kidx[b:b + 1], nb)
            R = c0.ring_slots
            rows = torch.arange(max(0, n - R), n)
            c0.ring_k[b, 0, rows % R] = inp.k[b, rows, 0].cuda()
        c0.seq_lens.copy_(torch.as_tensor(lens, dtype=torch.int32))
        kidx = kidx[:, 0].contiguous()
        torch.cuda.synchronize()
        self.nvis = np.minimum(lens // w.block_m, nb)
        self.step_bytes = self.bytes_per_step()
        l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
        self.NR = max(1, -(-3 * l2 // self.step_bytes))
        cl = lambda t: None if t is None else t.clone()  # noqa: E731
        self.caches = [c0] + [L.Cache(self.cfg, B, nb, c0.ring_slots, cl(c0.pooled_k), None, cl(c0.ring_k), None,
                                      cl(c0.pool_state), cl(c0.seq_lens)) for _ in range(self.NR - 1)]
        self.kidx = [kidx] + [kidx.clone() for _ in range(self.NR - 1)]
        self.iq = c["iq"].cuda()
        self.iw = c["iw"].cuda()
        self.q = inp.q.cuda()
        self.sink = inp.sink.cuda()
        self.sel = [torch.empty(B, w.top_k, dtype=torch.int32, device="cuda") for _ in range(self.NR)]
        self.outs = [torch.empty(B, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
                     for _ in range(self.NR)]
        self.ws = torch.zeros(L.lbca_indexer_workspace_bytes(B, nb), dtype=torch.uint8, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.steps = steps

    def bytes_per_step(self):
        """Algorithmic HBM bytes of one step: the visible indexer keys, the
        indexer queries and weights, the selected entries and the window rows,
        the queries and the outputs, each once."""
        w = self.w
        nsel = np.minimum(self.nvis, w.top_k)
        nwin = np.minimum(np.asarray(self.inp.lens), w.n_win)
        b = int(self.nvis.sum()) * w.index_dim * 2 + w.batch * w.index_heads * (w.index_dim * 2 + 4)
        b += int((nsel + nwin).sum()) * w.head_dim * 2 + 2 * w.batch * w.n_q_heads * w.head_dim * 2
        return b

    def flops_per_step(self):
        w = self.w
        nsel = np.minimum(self.nvis, w.top_k)
        nwin = np.minimum(np.asarray(self.inp.lens), w.n_win)
        return (2.0 * int(self.nvis.sum()) * w.index_heads * w.index_dim +
                4.0 * int((nsel + nwin).sum()) * w.n_q_heads * w.head_dim)

    def launch(self, i):
        L, rep, j = self.L, i % self.NR, (i // self.NR) % self.steps
        L.lbca_indexer_topk(self.iq[j], self.iw[j], self.kidx[rep], self.caches[rep].seq_lens, self.w.block_m,
                            self.sel[rep], None, self.ws, self.status)
        L.lbca_decode_sparse(self.cfg, self.q[j], self.caches[rep], self.sel[rep], self.sink, None, None,
                             self.outs[rep], self.status)


def csa_leg(K=20, W=5, reps=3):
    """The CSA sparse decode step (indexer relevance + top-k + sparse
    attention) of the 4 x 64K workload, K steps replayed from one CUDA graph,
    median of `reps` replays; the oracle on one sequence beside it."""
    import gc

    import torch

    from block_compressed_long_b200 import synth
    w = synth.WORKLOADS["csa_sparse_decode_64k"]
    bench = CsaBench(w, steps=8)
    for i in range(W):
        bench.launch(i)
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr, stream=cap):
        for i in range(W, W + K):
            bench.launch(i)
    uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record()
        gr.replay()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) / K)
    clocks = sampler.stop()
    st = int(bench.status.item())
    if st:
        raise RuntimeError(f"CSA step device status {bench.L.lbca_status_string(st)}")
    ms = statistics.median(ts)
    hbm, src = peaks()
    gbs = bench.step_bytes / (ms * 1e-3) / 1e9
    line = {"workload": w.name, "metric": METRIC, "value": ms * 1e3 / w.batch, "unit": "µs/token",
            "ms_per_step": ms, "dtype": "bf16 I/O; indexer bf16 tensor-core products, f32 accumulate; "
                                        "attention fp16 tensor-core operands",
            "config": {"batch": w.batch, "context": w.ctx[0], "block_m": w.block_m, "n_win": w.n_win,
                       "n_q_heads": w.n_q_heads, "head_dim": w.head_dim, "index_heads": w.index_heads,
                       "index_dim": w.index_dim, "top_k": w.top_k,
                       "l2": f"steps rotate over {bench.NR} cache replicas (>= 3x L2), each step's data cold",
                       "launch": f"{K} steps (3 kernels each) back to back from one CUDA graph, median of {reps}"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "peak_source": src, "bytes_per_step": bench.step_bytes,
                         "flops_per_step": bench.flops_per_step(),
                         "kernel": "indexer_score_kernel + topk_kernel + decode_mqa_tc_kernel (whole step timed)"},
            "gpu_launches": 3 * K, "clocks": clocks}
    inp = bench.inp
    del bench, gr
    gc.collect()
    torch.cuda.empty_cache()
    line["cpu_baseline"] = oracle_csa_timing(w, inp)
    return line


def oracle_csa_timing(w, inp):
    """The fp64 oracle's CSA decode step for the first sequence (indexer
    relevance over its complete blocks, top-k, sparse attention), the
    sequence's pooled entries and indexer keys computed beforehand (untimed,
    as the GPU leg's cache is built beforehand)."""
    from block_compressed_long_b200 import synth
    from oracle import oracle as orc
    f64 = synth.f64
    c = inp.csa
    n = int(inp.lens[0])
    oc = orc.Config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                    w.rmsnorm, w.rope_theta)
    ic = orc.Config(1, 1, w.index_dim, True, w.block_m, w.n_win)
    ek = orc.pool_dual(oc, orc.KEY, f64(inp.k[:1, :n]), f64(inp.zk[:1, :n]), f64(c["kb"][:1, :n]),
                       f64(c["zkb"][:1, :n]), f64(inp.bpos_k), f64(c["bpos_kb"]))
    kx = orc.pool_dual(ic, orc.VALUE, *(f64(c[t][:1, :n]) for t in ("ika", "izka", "ikb", "izkb")),
                       f64(c["ibpa"]), f64(c["ibpb"]))[:, :, 0]
    hist = f64(inp.k[:1, :n])
    per = []
    for j in range(3):
        t0 = time.perf_counter()
        sc = orc.indexer_scores(f64(c["iq"][j, :1]), f64(c["iw"][j, :1]), kx, [kx.shape[1]])
        sel = orc.topk_blocks(sc, [kx.shape[1]], w.top_k)
        orc.attend_sparse(oc, f64(inp.q[j, :1]), ek, sel, hist, [n], f64(inp.sink))
        per.append(time.perf_counter() - t0)
    med = statistics.median(per)
    return {"value": med * 1e6, "unit": "µs/token", "cores": _cores(), "kind": "oracle",
            "sample": f"3 decode steps of sequence 0 of {w.name} (context {n}), fp64 C oracle; median step"}


def load_traffic(workload):
    """DRAM bytes per decode launch from a committed ncu capture, if the
    decode source has not changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(p))[workload]
    except Exception:
        return None
    src = os.path.join(ROOT, "block_compressed_long_b200", "csrc", rec["source"])
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return rec["bytes"] if rec.get("source_sha256_16") == h else None


# ----------------------------------------------------- oracle (CPU) timing ----
def _cores():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def oracle_decode_timing(w, budget_s=12.0, max_steps=None):
    """The fp64 oracle as it stands, driven step by step on the host cores:
    each step appends one token per sequence (pooling a block when it
    completes) and attends its query.  Each step is timed on its own and the
    median step is reported (a few steps that pool a block take longer).
    Returns (µs/token, tokens, cores, description)."""
    from block_compressed_long_b200 import synth
    from oracle import oracle as orc
    f64 = synth.f64
    nb = max_steps or 64
    # a bounded sample: the workload's first (at most) 4 sequences, drawn alone
    # (every sequence has its own random streams, so they equal those of the
    # whole batch)
    nseq = min(w.batch, 4)
    ws = synth.scaled(w, steps=nb, batch=nseq)
    inp = synth.make(ws, lens=synth.contexts(w)[:nseq])
    c = orc.Config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   w.rmsnorm, w.rope_theta)
    seqs = list(range(nseq))
    streams = []
    for b in seqs:
        Lb = int(inp.lens[b])
        st = orc.Stream(c, f64(inp.bpos_k), f64(inp.bpos_v))
        st.extend(f64(inp.k[b, :Lb]), f64(inp.zk[b, :Lb]), None if w.shared_kv else f64(inp.v[b, :Lb]),
                  None if w.shared_kv else f64(inp.zv[b, :Lb]))
        streams.append(st)
    sink = f64(inp.sink)
    t_start = time.perf_counter()
    per_step = []
    n = 0
    while n < nb and (time.perf_counter() - t_start) < budget_s:
        t0 = time.perf_counter()
        for st, b in zip(streams, seqs):
            p = int(inp.lens[b]) + n
            st.extend(f64(inp.k[b, p:p + 1]), f64(inp.zk[b, p:p + 1]),
                      None if w.shared_kv else f64(inp.v[b, p:p + 1]),
                      None if w.shared_kv else f64(inp.zv[b, p:p + 1]))
            st.query(f64(inp.q[n, b]), sink)
        per_step.append(time.perf_counter() - t0)
        n += 1
    med = statistics.median(per_step)
    desc = (f"{n} decode steps of {len(seqs)} sequence(s) of {w.name} (contexts "
            f"{[int(inp.lens[b]) for b in seqs]}), fp64 C oracle, cache of pooled entries kept between steps; "
            f"median step {med * 1e3:.2f} ms (min {min(per_step) * 1e3:.2f}, max {max(per_step) * 1e3:.2f})")
    return med * 1e6 / len(seqs), n * len(seqs), _cores(), desc


def oracle_prefill_timing(w, inp, n_rows=48):
    """The fp64 oracle's prefill of the same inputs on the host cores: the
    pooling of every complete block timed in full, the attention of a bounded
    sample of query rows (spread over the sequence) timed and scaled to all T
    rows by their share of the visible pairs.  Returns a cpu_baseline record
    in the leg's unit (TFLOP/s of the algorithmic flops)."""
    from block_compressed_long_b200 import synth
    from oracle import oracle as orc
    f64 = synth.f64
    c = orc.Config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   w.rmsnorm, w.rope_theta)
    T = w.seq_len
    k, v, zk, zv = f64(inp.k), f64(inp.v), f64(inp.zk), f64(inp.zv)
    t0 = time.perf_counter()
    nbk = T // w.block_m * w.block_m
    ek = orc.pool(c, orc.KEY, k[:, :nbk], zk[:, :nbk], f64(inp.bpos_k))
    ev = None if w.shared_kv else orc.pool(c, orc.VALUE, v[:, :nbk], zv[:, :nbk], f64(inp.bpos_v))
    t_pool = time.perf_counter() - t0
    rows = np.unique(np.linspace(0, T - 1, min(n_rows, T)).astype(np.int64))
    q = f64(inp.q[:, rows])
    t0 = time.perf_counter()
    orc.attend(c, q, np.broadcast_to(rows, (w.batch, len(rows))), ek, ev, k, None if w.shared_kv else v,
               np.full(w.batch, T), f64(inp.sink))
    t_att = time.perf_counter() - t0
    t_total = t_pool + t_att * prefill_pairs(w) / max(1, prefill_pairs(w, rows))
    return {"value": prefill_flops(w) / t_total / 1e12, "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
            "sample": (f"{w.name}: fp64 C oracle, pooling of all {T // w.block_m} blocks timed ({t_pool:.2f} s), "
                       f"attention of {len(rows)} of {T} query rows timed ({t_att:.2f} s) and scaled by visible "
                       f"pairs to all rows: {t_total:.1f} s per prefill")}


def oracle_pool_timing(w, inp, series, max_tokens=8192):
    """The fp64 oracle's pooling of a bounded sample (the first blocks, at most
    max_tokens tokens of every sequence) on the host cores, in GB/s of the same
    algorithmic bytes the GPU leg counts."""
    from block_compressed_long_b200 import synth
    from oracle import oracle as orc
    f64 = synth.f64
    c = orc.Config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   w.rmsnorm, w.rope_theta)
    n = min(w.seq_len, max_tokens) // w.block_m * w.block_m
    srcs = [(orc.KEY, inp.k, inp.zk, inp.bpos_k)] + ([] if w.shared_kv else [(orc.VALUE, inp.v, inp.zv, inp.bpos_v)])
    xs = [(s, f64(x[:, :n]), f64(z[:, :n]), f64(bp)) for s, x, z, bp in srcs]
    if w.dual:
        xb, zb, bpb = f64(inp.csa["kb"][:, :n]), f64(inp.csa["zkb"][:, :n]), f64(inp.csa["bpos_kb"])
    t0 = time.perf_counter()
    for s, x, z, bp in xs:
        if w.dual:
            orc.pool_dual(c, s, x, z, xb, zb, bp, bpb)
        else:
            orc.pool(c, s, x, z, bp)
    dt = time.perf_counter() - t0
    esz = 2 if w.dtype == "bf16" else 4
    nbytes = len(xs) * w.batch * n * w.n_kv_heads * w.head_dim * esz * ((4 if w.dual else 2) + 1.0 / w.block_m)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": _cores(), "kind": "oracle",
            "sample": (f"fp64 C oracle pooling the first {n} tokens of each of {w.batch} sequence(s), "
                       f"{len(xs)} series ({dt:.2f} s)")}


def main():
    args = parse()
    from block_compressed_long_b200 import ranks, synth
    rank, world, local_rank = ranks.from_env()
    w = synth.WORKLOADS[args.workload]
    if w.kind != "decode":
        raise SystemExit("bench.py times decode workloads; prefill is timed by its own leg")

    if args.impl == "reference":
        if rank != 0:
            return
        budget = min(60.0, max(5.0, 0.5 * (args.warmup + args.steps)))
        us, n, cores, desc = oracle_decode_timing(w, budget_s=budget, max_steps=args.warmup + args.steps)
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": us, "unit": "µs/token", "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "higher_is_better": False, "scaling": "weak",
                          "dtype": "f64", "data": "synthetic", "config": {"workload": w.name},
                          "cpu_baseline": {"value": us, "unit": "µs/token", "cores": cores, "kind": "oracle",
                                           "sample": desc},
                          "e2e": {"value": us, "unit": "µs/token", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
              flush=True)
        return

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    import __graft_entry__
    __graft_entry__.build()
    if args.leg != "decode":  # one leg alone, on this GPU
        if rank == 0:
            if args.leg == "prefill":
                out = prefill_leg(args.prefill, reps=args.steps, warm=args.warmup, baseline=False)
            elif args.leg == "pool":
                out = pool_leg(args.pool, reps=args.steps, warm=args.warmup, baseline=False)
            elif args.leg == "csa":
                out = csa_leg(K=args.steps, W=args.warmup)
            elif args.leg == "backward":
                out = backward_leg(reps=args.steps, warm=args.warmup)
            else:
                out = layer_chain_leg(K=args.steps, W=args.warmup)
            print(json.dumps(out), flush=True)
        return
    line, bench = run_ours(args, w, rank, world)
    del bench
    if world == 1 and not args.no_also:
        import gc
        gc.collect()
        torch.cuda.empty_cache()
        also = [decode_also(args, n) for n in ("gqa_decode_32k", "hca_mqa_decode_128k") if n != w.name]
        also += [layer_chain_leg(), csa_leg(), backward_leg()]
        also += [prefill_leg("gqa_prefill_16k"), prefill_leg("tiny_f32_prefill")]
        also += [pool_leg(label) for label in POOL_CASES]
        line["also"] = also
    if rank == 0 and world == 1:
        us, n, cores, desc = oracle_decode_timing(w)
        line["cpu_baseline"] = {"value": us, "unit": "µs/token", "cores": cores, "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
