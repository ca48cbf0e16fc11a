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
    ap.add_argument("--workload", default="gqa_decode_32k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--leg", default="decode", choices=["decode", "prefill", "pool"],
                    help="decode: the decode-step benchmark (default, with the prefill and pool legs appended); "
                         "prefill / pool: that leg alone (one JSON line)")
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
        L.lbca_decode(self.cfg, self.q[j], self.caches[rep], self.sink, None, self.outs[rep], self.dec_ws[rep],
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


def run_ours(args, w, rank, world):
    import torch
    import torch.distributed as dist

    from block_compressed_long_b200 import ranks

    K, W = args.steps, args.warmup
    bench = DecodeBench(w, rank, 2 * (W + K))
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
    g_main = graph_of(bench.i, K, bench.launch)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
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
    step_ms = e0.elapsed_time(e1) / K
    bench.i += K
    del g_main
    kernel_ms = step_ms  # one fused kernel per step: the step is the kernel
    if bench.launches == 2:
        # append + decode: time the decode launches alone (same replicas, same rotation)
        for i in range(bench.i, bench.i + W):
            bench.launch_decode(i)
        g_dec = graph_of(bench.i, K, bench.launch_decode)
        torch.cuda.synchronize()
        e0.record()
        g_dec.replay()
        e1.record()
        torch.cuda.synchronize()
        kernel_ms = e0.elapsed_time(e1) / K
        del g_dec

    # ---- end to end through the public API: pinned host inputs and output ----
    # each step's inputs (q and the new token's k, v, z_k, z_v) sit packed in
    # one pinned host buffer and cross with one copy; the output comes back
    # with one copy.  As in a serving loop, the copies run on streams of their
    # own beside the kernels: step i+1's upload overlaps step i's kernel and
    # step i's download overlaps step i+1's (two staging slots; every step
    # waits for its own upload, every download for its own step).
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
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(NS)]        # slot's upload done
    ev_run = [torch.cuda.Event() for _ in range(NS)]       # the step that read the slot is done
    ev_down = [torch.cuda.Event() for _ in range(bench.NR)]  # download of an output replica done

    def e2e_steps(first, n):
        cur = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(cur)
        s_in.wait_event(fork)
        s_out.wait_event(fork)
        for j, i in enumerate(range(first, first + n)):
            sl, rep = j % NS, i % bench.NR
            if j >= NS:
                s_in.wait_event(ev_run[sl])       # the step two back has read this slot
            with torch.cuda.stream(s_in):
                dstage[sl].copy_(hstage[i // bench.NR], non_blocking=True)
                ev_in[sl].record(s_in)
            cur.wait_event(ev_in[sl])
            if j >= bench.NR:
                cur.wait_event(ev_down[rep])     # this output replica has been read back
            bench.launch(i, q=dq[sl], tok=dtok[sl])
            ev_run[sl].record(cur)
            s_out.wait_event(ev_run[sl])
            with torch.cuda.stream(s_out):
                hout[sl].copy_(bench.outs[rep], non_blocking=True)
                ev_down[rep].record(s_out)
        for st in (s_in, s_out):  # join both copy streams back
            ev = torch.cuda.Event()
            ev.record(st)
            cur.wait_event(ev)

    e2e_steps(bench.i, W)
    bench.i += W
    torch.cuda.synchronize()
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=cap):
        e2e_steps(bench.i, K)
    torch.cuda.synchronize()
    e0.record()
    g_e2e.replay()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / K
    bench.i += K
    del g_e2e
    clocks = sampler.stop()
    status = int(bench.status.item())
    if status:
        raise RuntimeError(f"device status {L.lbca_status_string(status)}")

    step_ms, e2e_ms, kernel_ms = ranks.max_over_ranks([step_ms, e2e_ms, kernel_ms], device="cuda")
    hbm, src = peaks()
    achieved = nbytes / K / (kernel_ms * 1e-3) / 1e9
    w_ = bench.w
    line = {
        "metric": METRIC, "value": ranks.job_us_per_token(step_ms, bench.B, world), "unit": "µs/token",
        "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": step_ms, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": w_.dtype, "data": "synthetic",
        "config": {"workload": w_.name, "batch_per_gpu": w_.batch, "context": [int(w_.ctx[0]), int(w_.ctx[1])],
                   "n_q_heads": w_.n_q_heads, "n_kv_heads": w_.n_kv_heads, "head_dim": w_.head_dim,
                   "block_m": w_.block_m, "n_win": w_.n_win, "rope_dims": w_.rope_dims,
                   "shared_kv": w_.shared_kv, "parallelism": f"dp{world}",
                   "l2": (f"inputs larger than L2: steps rotate over {bench.NR} cache replicas "
                          f"(>= 3x L2 of data in total), each step's data cold"),
                   "launch": (f"K steps of lbca_decode_step ({bench.launches} kernel launch"
                              f"{'es' if bench.launches > 1 else ''} each), back to back from one CUDA graph; "
                              "e2e: each step's upload and download on copy streams beside the kernels "
                              "(uploads one step ahead, downloads one step behind), all inside the timed graph")},
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
                "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": K * bench.launches,
        "clocks": clocks,
    }
    return line, bench


def peak_tflops():
    try:
        with open(PEAKS_PATH) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (bf16 burst; fp16 has the same dense rate)"
    except Exception:
        return 1590.0, "fallback"


def prefill_flops(w):
    """Algorithmic FLOPs: 4 D Hq per visible (query, entry) pair."""
    T, m, n = w.seq_len, w.block_m, w.n_win
    pairs = 0
    for L in range(1, T + 1):
        P = max(0, (L - n) // m)
        pairs += P + (L - P * m)
    return 4.0 * w.head_dim * w.n_q_heads * pairs * w.batch


def extra_prefill(reps=10, warm=3):
    """lbca_prefill of the 16K-token GQA layer (pool pass, RoPE table, finalised
    keys, tensor-core attention), inputs resident (> L2), CUDA events."""
    import torch

    from block_compressed_long_b200 import lbca as L
    from block_compressed_long_b200 import synth
    w = synth.WORKLOADS["gqa_prefill_16k"]
    inp = synth.make(w)
    cfg = L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   w.rmsnorm, w.rope_theta, dtype=w.dtype)
    d = lambda t: None if t is None else t.cuda()  # noqa: E731
    q, k, v, zk, zv, bpk, bpv = (d(t) for t in (inp.q, inp.k, inp.v, inp.zk, inp.zv, inp.bpos_k, inp.bpos_v))
    out = torch.empty_like(q)
    ws = torch.zeros(L.lbca_prefill_workspace_bytes(cfg, w.batch, w.seq_len, False), dtype=torch.uint8,
                     device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(warm):
        L.lbca_prefill(cfg, q, k, v, zk, zv, bpk, bpv, None, None, None, out, None, ws, d_status=st)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        L.lbca_prefill(cfg, q, k, v, zk, zv, bpk, bpv, None, None, None, out, None, ws, d_status=st)
    e1.record()
    torch.cuda.synchronize()
    if int(st.item()):
        raise RuntimeError(f"prefill device status {L.lbca_status_string(int(st.item()))}")
    ms = e0.elapsed_time(e1) / reps
    fl = prefill_flops(w)
    tf = fl / (ms * 1e-3) / 1e12
    pk, src = peak_tflops()
    return {"workload": w.name, "metric": "prefill TFLOP/s", "value": tf, "unit": "TFLOP/s", "ms_per_call": ms,
            "dtype": "bf16 I/O, fp16 tensor-core operands, f32 accumulate",
            "roofline": {"bound": "tensor", "achieved": tf, "peak": pk, "unit": "TFLOP/s", "frac": tf / pk,
                         "peak_source": src, "kernel": "prefill_tc_kernel (whole lbca_prefill call timed)",
                         "flops_per_call": fl}}


def extra_pool(reps=10, warm=3):
    """lbca_pool of both series of the 32K-token GQA prefix (HBM-bound)."""
    import torch

    from block_compressed_long_b200 import lbca as L
    from block_compressed_long_b200 import synth
    w = synth.scaled(synth.WORKLOADS["gqa_decode_32k"], kind="prefill", seq_len=32768)
    inp = synth.make(w)
    cfg = L.config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   dtype=w.dtype)
    d = lambda t: t.cuda()  # noqa: E731
    k, v, zk, zv, bpk, bpv = (d(t) for t in (inp.k, inp.v, inp.zk, inp.zv, inp.bpos_k, inp.bpos_v))
    nb = w.seq_len // w.block_m
    ok_ = torch.empty(1, w.n_kv_heads, nb, w.head_dim, dtype=torch.bfloat16, device="cuda")
    ov_ = torch.empty_like(ok_)

    def run():
        L.lbca_pool(cfg, L.LBCA_KEY, k, zk, bpk, None, ok_)
        L.lbca_pool(cfg, L.LBCA_VALUE, v, zv, bpv, None, ov_)

    for _ in range(warm):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = 2 * (2 * k.numel() * 2 + ok_.numel() * 2)  # K and V series: read X and Z, write entries
    gbs = nbytes / (ms * 1e-3) / 1e9
    hbm, src = peaks()
    return {"workload": "gqa_decode_32k prefix (32768 tokens, K and V series)", "metric": "pool GB/s", "value": gbs,
            "unit": "GB/s", "ms_per_call": ms,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "peak_source": src, "kernel": "pool_kernel", "bytes_per_call": nbytes}}


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
def oracle_decode_timing(w, budget_s=12.0, max_steps=None):
    """The fp64 oracle as it stands, driven step by step on the host cores:
    each step appends one token per sequence (pooling a block when it
    completes) and attends its query.  Returns (µs/token, steps, cores, desc)."""
    from block_compressed_long_b200 import synth
    from oracle import oracle as orc
    f64 = synth.f64
    nb = max_steps or 64
    ws = synth.scaled(w, steps=nb)
    inp = synth.make(ws)
    c = orc.Config(w.n_q_heads, w.n_kv_heads, w.head_dim, w.shared_kv, w.block_m, w.n_win, w.rope_dims,
                   w.rmsnorm, w.rope_theta)
    seqs = list(range(min(ws.batch, 4)))  # bounded sample of sequences
    streams = []
    for b in seqs:
        Lb = int(inp.lens[b])
        st = orc.Stream(c, f64(inp.bpos_k), f64(inp.bpos_v))
        st.extend(f64(inp.k[b, :Lb]), f64(inp.zk[b, :Lb]), None if w.shared_kv else f64(inp.v[b, :Lb]),
                  None if w.shared_kv else f64(inp.zv[b, :Lb]))
        streams.append(st)
    sink = f64(inp.sink)
    t0 = time.perf_counter()
    n = 0
    while n < nb and (time.perf_counter() - t0) < budget_s:
        for st, b in zip(streams, seqs):
            p = int(inp.lens[b]) + n
            st.extend(f64(inp.k[b, p:p + 1]), f64(inp.zk[b, p:p + 1]),
                      None if w.shared_kv else f64(inp.v[b, p:p + 1]),
                      None if w.shared_kv else f64(inp.zv[b, p:p + 1]))
            st.query(f64(inp.q[n, b]), sink)
        n += 1
    dt = time.perf_counter() - t0
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    desc = (f"{n} decode steps of {len(seqs)} sequence(s) of {w.name} (contexts "
            f"{[int(inp.lens[b]) for b in seqs]}), fp64 C oracle, cache of pooled entries kept between steps")
    return dt * 1e6 / (n * len(seqs)), n * len(seqs), cores, desc


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
        us, n, cores, desc = oracle_decode_timing(w, budget_s=max(5.0, 0.5 * args.steps), max_steps=args.warmup + args.steps)
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
            leg = extra_prefill if args.leg == "prefill" else extra_pool
            print(json.dumps(leg(reps=args.steps, warm=args.warmup)), flush=True)
        return
    line, _ = run_ours(args, w, rank, world)
    if world == 1 and args.workload == "gqa_decode_32k":
        line["also"] = [extra_prefill(), extra_pool()]
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
