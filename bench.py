#!/usr/bin/env python
"""Decode-step benchmark of the quantized KV cache (libkvq.so, one process per GPU).

A step is one decode step of the whole batch through kvq_append_decode: the
new token enters the residual window (a flush quantizes G tokens when due) and
the attention runs over the packed cache, in one kernel launch on steps that
do not flush.  Metric: packed-KV bytes read by the decode attention per
second (GB/s), with tokens/s alongside.  The default workload is the
Llama-3.1-70B-shaped 128K-token context at 2 bits.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config 70b] [--impl kivi|reference]

Timing: the K timed steps are captured into one CUDA graph (library calls
through the C ABI) and replayed once between CUDA events on the launching
stream, bracketed by a barrier and torch.cuda.synchronize(); the max over ranks
is reported.  Each step targets the next of several identical cache replicas
whose total size is over 3x the L2, so every step streams its cache from HBM.
The decode kernel is also timed launch by launch (at least 100 single-launch
graph replays, replicas rotated: the cold-L2 median; the same replica again
and again: the warm-L2 median), and the launch overhead is reported apart:
the host cost of one library call and the device gap a separately launched
graph adds.  The e2e figure calls the public API step by step with host
buffers: one pinned host-to-device copy of the step's inputs and one
device-to-host copy of its output per step, each on its own stream into
double-buffered device rows, so a step's copies overlap its neighbours'
kernels as in a serving loop (events keep every buffer's reuse in order).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-KV decode attn: packed-KV GB/s (% of HBM peak), tokens/s"
HBM_FALLBACK_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # the B200 HBM3e peak as usually quoted (DGX figure)


def _profiled_traffic(kernel: str, source: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, or None when there is none or the kernel source has changed
    since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.md")
    if not os.path.exists(p):
        return None
    m = re.search(r"traffic_bytes_per_launch=(\d+) source_sha256_16=([0-9a-f]+)", open(p).read())
    if not m:
        return None
    src = open(os.path.join(ROOT, "quantized_kv_cache_18_b200", "csrc", source), "rb").read()
    return int(m.group(1)) if hashlib.sha256(src).hexdigest()[:16] == m.group(2) else None


class CudaRt:
    """The e2e loop's copies and stream orderings, issued as plain CUDA runtime
    calls (the system libcudart through ctypes): the torch equivalents cost
    several microseconds of host time each, which bounds a ~40 us step.
    Events per buffer b: in[b] (inputs on the device), done[b] (the kernel that
    read row b ended), read[b] (output buffer b copied back)."""

    H2D, D2H, NO_TIMING = 1, 2, 2

    def __init__(self, compute, s_h2d, s_d2h):
        self.lib = None
        for name in ("libcudart.so.12", "/usr/local/cuda/lib64/libcudart.so.12"):
            try:
                self.lib = ctypes.CDLL(name)
                break
            except OSError:
                continue
        if self.lib is None:
            raise RuntimeError("the CUDA runtime library (libcudart.so.12) is needed for the e2e copies")
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        self.lib.cudaMemcpyAsync.argtypes = [vp, vp, sz, ctypes.c_int, vp]
        self.lib.cudaEventRecord.argtypes = [vp, vp]
        self.lib.cudaStreamWaitEvent.argtypes = [vp, vp, ctypes.c_uint]
        self.lib.cudaEventCreateWithFlags.argtypes = [ctypes.POINTER(vp), ctypes.c_uint]
        self.lib.cudaEventDestroy.argtypes = [vp]

        def make():
            e = vp()
            self._chk(self.lib.cudaEventCreateWithFlags(ctypes.byref(e), self.NO_TIMING), "cudaEventCreateWithFlags")
            return e
        self.ev = {k: [make(), make()] for k in ("in", "done", "read")}
        self.sp = {k: vp(st.cuda_stream) for k, st in (("c", compute), ("h", s_h2d), ("d", s_d2h))}

    @staticmethod
    def _chk(r, what):
        if r != 0:
            raise RuntimeError(f"{what} failed ({r})")

    def _wait(self, stream_key, ev):
        self._chk(self.lib.cudaStreamWaitEvent(self.sp[stream_key], ev, 0), "cudaStreamWaitEvent")

    def _record(self, ev, stream_key):
        self._chk(self.lib.cudaEventRecord(ev, self.sp[stream_key]), "cudaEventRecord")

    def _copy(self, dst, src, n, kind, stream_key):
        self._chk(self.lib.cudaMemcpyAsync(ctypes.c_void_p(dst), ctypes.c_void_p(src), n, kind, self.sp[stream_key]),
                  "cudaMemcpyAsync")

    def h2d(self, dst, src, n, b, wait_done):
        if wait_done:
            self._wait("h", self.ev["done"][b])
        self._copy(dst, src, n, self.H2D, "h")
        self._record(self.ev["in"][b], "h")

    def before_kernel(self, b, wait_read):
        self._wait("c", self.ev["in"][b])
        if wait_read:
            self._wait("c", self.ev["read"][b])

    def after_kernel(self, b):
        self._record(self.ev["done"][b], "c")

    def d2h(self, dst, src, n, b):
        self._wait("d", self.ev["done"][b])
        self._copy(dst, src, n, self.D2H, "d")
        self._record(self.ev["read"][b], "d")

    def finish(self, b):
        self._wait("c", self.ev["read"][b])

    def close(self):
        for evs in self.ev.values():
            for e in evs:
                self.lib.cudaEventDestroy(e)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return HBM_FALLBACK_GBS, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = max(mx, float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- ranks
# Weak scaling: every rank owns an independent batch of sequences (its own
# seeded inputs and caches); there is no exchange on the data path.  The only
# collectives are the barriers around the timed region and these reductions.
def rank_seed(w, rank: int) -> int:
    return 1000 + w.seed + 7919 * rank


def combine_ranks(ms: float, units: float, world: int, device) -> tuple:
    """(max of ms over ranks, sum of units over ranks)."""
    if world == 1:
        return ms, units
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


# ---------------------------------------------------------------- inputs on the device
def device_inputs(w, device, steps_total, rank: int = 0):
    """Seeded synthetic inputs with the workload's recipe, drawn on the device
    (standard normal, K outlier channels x20, 2% of V tokens per batch row x10);
    each rank draws its own batch."""
    import torch
    from quantized_kv_cache_18_b200 import workloads as W
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float16
    g = torch.Generator(device=device)
    g.manual_seed(rank_seed(w, rank))
    shape = (w.batch, w.num_kv_heads, w.seq_len, w.head_dim)
    ch = torch.as_tensor(W.k_outlier_channels(w), device=device)
    K = torch.randn(shape, generator=g, device=device)
    K[..., ch] *= w.k_outlier_scale
    K = K.to(dt)
    V = torch.randn(shape, generator=g, device=device)
    if w.v_channel_outliers:
        V[..., ch] *= w.k_outlier_scale
    for b in range(w.batch):
        vt = torch.as_tensor(W.v_outlier_tokens(w, b), device=device)
        if vt.numel():
            V[b, :, vt, :] *= w.v_outlier_scale
    V = V.to(dt)
    q = torch.randn((steps_total, w.batch, w.num_q_heads, w.head_dim), generator=g, device=device).to(dt)
    kn = torch.randn((steps_total, w.batch, w.num_kv_heads, w.head_dim), generator=g, device=device)
    kn[..., ch] *= w.k_outlier_scale
    vn = torch.randn((steps_total, w.batch, w.num_kv_heads, w.head_dim), generator=g, device=device)
    hit = torch.rand((steps_total, w.batch), generator=g, device=device) < w.v_outlier_frac
    vn[hit] *= w.v_outlier_scale
    return K, V, q, kn.to(dt), vn.to(dt)


def step_bytes(cache) -> int:
    """Packed bytes one decode attention reads: every group record, every
    window token (key and value rows: 16-bit, or FP8 rows in the mixed cache)
    and the mixed cache's FP8 anchor rows."""
    c, lay = cache.cfg, cache.layout
    rows = c.batch * c.num_kv_heads
    return rows * (cache.quantized_len // c.group * lay.record_bytes +
                   (cache.window_len + c.anchor_tokens) * 2 * lay.token_row_bytes)


# ---------------------------------------------------------------- GPU arm
def run_gpu(args, w, rank, world):
    import torch
    from quantized_kv_cache_18_b200 import build as kbuild
    from quantized_kv_cache_18_b200 import _lib as L
    from quantized_kv_cache_18_b200.cache import (QuantizedKVCache, config_from_workload, launch_count, layout,
                                                   turbo_setup_from_workload)

    kbuild.build()
    device = torch.device("cuda", torch.cuda.current_device())
    steps_total = args.warmup + args.steps
    max_seq = w.seq_len + steps_total + 1
    cfg = config_from_workload(w, max_seq)
    P = args.page_records
    if P > 0:
        # paged caches: a pool with exactly the pages the rows need, each row's
        # block table a random slice of a permutation of the pool
        gpr = layout(cfg).groups_per_row
        ppr = (gpr + P - 1) // P
        rows = w.batch * w.num_kv_heads
        cfg = config_from_workload(w, max_seq, P, rows * ppr)
        tables = []

    def new_cache():
        c = QuantizedKVCache(cfg, device=device)
        if P > 0:
            g = torch.Generator().manual_seed(rank_seed(w, rank) + len(tables))
            perm = (torch.randperm(rows * ppr, generator=g) if args.page_order == "shuffled"
                    else torch.arange(rows * ppr))
            t = perm.to(torch.int32).view(rows, ppr).to(device)
            tables.append(t)
            c.set_page_table(t)
        return c

    K, V, q, kn, vn = device_inputs(w, device, steps_total, rank)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    probe = new_cache()
    n_rep = max(2, math.ceil(3 * l2 / probe.nbytes) + 1)
    caches = [probe] + [new_cache() for _ in range(n_rep - 1)]
    turbo = w.scheme == "turbo"
    for c in caches:
        if turbo:
            turbo_setup_from_workload(c, w)
        c.prefill(K, V)
    del K, V
    torch.cuda.synchronize()
    out = torch.empty((w.batch, w.num_q_heads, w.head_dim), dtype=torch.float32, device=device)
    lib = L.load()
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    scale = ctypes.c_float(w.scale)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    qp = [ptr(q[i]) for i in range(steps_total)]
    knp = [ptr(kn[i]) for i in range(steps_total)]
    vnp = [ptr(vn[i]) for i in range(steps_total)]
    outp = ptr(out)

    # one decode step = append the new token + attend (kvq_append_decode: one
    # launch, or quantize + attend on a step that flushes the window)
    def one_step(i):
        c = caches[i % n_rep]
        L.check(lib.kvq_append_decode(c.handle, knp[i], vnp[i], qp[i], outp, scale, ptr(c.ws), c.ws.numel(), sp),
                "append_decode")
        return step_bytes(c)

    for i in range(args.warmup):
        one_step(i)
    torch.cuda.synchronize()

    # The timed steps run as one CUDA graph: capturing enqueues nothing, and the
    # host-side cache counters advance during capture exactly as the replay
    # advances the device state, so one replay performs the K steps.  This keeps
    # Python launch overhead out of a ~20 us step.
    graph = torch.cuda.CUDAGraph()
    cap_stream = torch.cuda.Stream()
    launches0 = launch_count()
    total_bytes = 0
    with torch.cuda.stream(cap_stream):
        csp = ctypes.c_void_p(cap_stream.cuda_stream)
        with torch.cuda.graph(graph, stream=cap_stream):
            for j in range(args.steps):
                i = args.warmup + j
                c = caches[i % n_rep]
                L.check(lib.kvq_append_decode(c.handle, knp[i], vnp[i], qp[i], outp, scale, ptr(c.ws),
                                              c.ws.numel(), csp), "append_decode")
                total_bytes += step_bytes(c)
    launches = launch_count() - launches0
    # attention-only graphs over the same replicas: one graph of K launches
    # (the mean launch time) and one single-launch graph per replica (launch
    # by launch medians); attention does not change the cache, so replays are
    # idempotent
    agraph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap_stream):
        with torch.cuda.graph(agraph, stream=cap_stream):
            for j in range(args.steps):
                c = caches[j % n_rep]
                L.check(lib.kvq_decode_attention(c.handle, qp[j], outp, scale, ptr(c.ws), c.ws.numel(), csp),
                        "attention")
    # (at most 64 of them: a workload whose cache is tiny has thousands of
    # replicas, and its launches are L2-resident whatever the rotation)
    single = []
    for i in range(min(n_rep, 64)):
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.stream(cap_stream):
            with torch.cuda.graph(g1, stream=cap_stream):
                c = caches[i]
                L.check(lib.kvq_decode_attention(c.handle, qp[i % steps_total], outp, scale, ptr(c.ws),
                                                 c.ws.numel(), csp), "attention")
        single.append(g1)
    attn_bytes = sum(step_bytes(caches[j % n_rep]) for j in range(args.steps))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # clocks are sampled while the GPU runs this workload: attention-only graph
    # replays (idempotent) surround the single timed replay of the step graph
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        tl = time.time()
        while time.time() - tl < 0.4:
            agraph.replay()
            torch.cuda.synchronize()
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        tl = time.time()
        while time.time() - tl < 0.2:
            agraph.replay()
            torch.cuda.synchronize()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    agraph.replay()
    a1.record(stream)
    torch.cuda.synchronize()
    attn_ms = [a0.elapsed_time(a1) / args.steps] * args.steps

    def per_launch(order):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in order]
        for (e0, e1), i in zip(ev, order):
            e0.record(stream)
            single[i].replay()
            e1.record(stream)
        torch.cuda.synchronize()
        return [e0.elapsed_time(e1) for e0, e1 in ev]

    n_med = max(100, args.steps)
    cold = per_launch([j % len(single) for j in range(n_med)])
    warm = per_launch([0] * (n_med + 1))[1:]   # the first launch brings replica 0 into L2
    # host cost of one library call (argument checks, partition, launch), no graph
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    n_host = 100
    for j in range(n_host):
        c = caches[j % n_rep]
        lib.kvq_decode_attention(c.handle, qp[j % steps_total], outp, scale, ptr(c.ws), c.ws.numel(), sp)
    host_us = (time.perf_counter() - h0) / n_host * 1e6
    torch.cuda.synchronize()
    kernel = {"mean_us": statistics.mean(attn_ms) * 1e3, "median_cold_us": statistics.median(cold) * 1e3,
              "median_warm_us": statistics.median(warm) * 1e3, "launches_timed": len(cold),
              "host_call_us": host_us,
              "graph_launch_gap_us": (statistics.median(cold) - statistics.mean(attn_ms)) * 1e3}
    del graph, agraph, single
    for c in caches:
        if c.status():
            raise RuntimeError("device status word set during the bench")
    ms, total_bytes = combine_ranks(ms, total_bytes, world, device)

    # end-to-end through the public API with host buffers: each step's q,
    # k_new and v_new sit in one pinned host row and cross in one host-to-device
    # copy; the output comes back in one device-to-host copy
    nq, nk = q[0].numel(), kn[0].numel()
    row_elems = nq + 2 * nk
    h_in = torch.empty((args.steps, row_elems), dtype=q.dtype).pin_memory()
    for j in range(args.steps):
        i = args.warmup + j
        h_in[j, :nq].copy_(q[i].reshape(-1))
        h_in[j, nq:nq + nk].copy_(kn[i].reshape(-1))
        h_in[j, nq + nk:].copy_(vn[i].reshape(-1))
    h_out = torch.empty((args.steps,) + tuple(out.shape), dtype=torch.float32).pin_memory()
    # two device input rows and two output buffers: step j uses buffer j % 2, so
    # the copy of step j + 1's inputs and the read of step j's output can run
    # on their own streams while step j + 1 (or j) computes
    d_in = [torch.empty(row_elems, dtype=q.dtype, device=device) for _ in range(2)]
    d_out = [torch.empty_like(out) for _ in range(2)]
    esz = d_in[0].element_size()
    d_ptrs = [(ctypes.c_void_p(t.data_ptr()), ctypes.c_void_p(t.data_ptr() + nq * esz),
               ctypes.c_void_p(t.data_ptr() + (nq + nk) * esz)) for t in d_in]
    e_caches = [new_cache() for _ in range(n_rep)]
    K, V, _, _, _ = device_inputs(w, device, 1, rank)
    if turbo:
        for c in e_caches:
            turbo_setup_from_workload(c, w)
    # prefill (quantize + window copy) of the replicas, timed on the device:
    # bytes = the K/V inputs read plus the packed records and window written
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(stream)
    for c in e_caches:
        c.prefill(K, V)
    p1.record(stream)
    torch.cuda.synchronize()
    prefill_ms = p0.elapsed_time(p1) / n_rep
    prefill_bytes = int(K.numel() * 2 + V.numel() * 2) + step_bytes(e_caches[0])
    del K, V
    e_args = [(c.handle, ptr(c.ws), c.ws.numel()) for c in e_caches]
    e_bytes = 0
    torch.cuda.synchronize()
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
    rt = CudaRt(stream, s_h2d, s_d2h)
    in_bytes, out_bytes = int(row_elems * esz), int(out.numel() * 4)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_h2d.wait_event(e0)
    for j in range(args.steps):
        b = j % 2
        hnd, wsp, wsn = e_args[j % n_rep]
        # inputs of step j into row b once the kernel that last read it (step j - 2) is done
        rt.h2d(d_in[b].data_ptr(), h_in[j].data_ptr(), in_bytes, b, wait_done=j >= 2)
        d_q, d_kn, d_vn = d_ptrs[b]
        rt.before_kernel(b, wait_read=j >= 2)
        L.check(lib.kvq_append_decode(hnd, d_kn, d_vn, d_q, ptr(d_out[b]), scale, wsp, wsn, sp), "append_decode")
        rt.after_kernel(b)
        rt.d2h(h_out[j].data_ptr(), d_out[b].data_ptr(), out_bytes, b)
        e_bytes += step_bytes(e_caches[j % n_rep])
    rt.finish((args.steps - 1) % 2)
    e1.record(stream)
    torch.cuda.synchronize()
    rt.close()
    e_ms = e0.elapsed_time(e1)
    e_ms, e_bytes = combine_ranks(e_ms, e_bytes, world, device)

    res = dict(ms=ms, bytes=total_bytes, attn_ms=attn_ms, launches=launches, clocks=clk.summary(),
               e2e_ms=e_ms, e2e_bytes=e_bytes, n_rep=n_rep, splits=caches[0].decode_splits,
               h2d=int(row_elems * esz), d2h=int(out.numel() * 4), kernel=kernel,
               step_bytes_last=attn_bytes // args.steps, prefill_ms=prefill_ms, prefill_bytes=prefill_bytes)
    return res


# ---------------------------------------------------------------- oracle (CPU) timing
def oracle_sample(w, budget_s: float, steps: int = 1):
    """Times the float64 oracle on a bounded sample of (batch, kv-head) rows:
    the prefill quantization of each sampled row, then its decode steps
    (append + attention over the dequantized cache), the latter once with
    numpy's thread pool as it is and once limited to one thread.  Rows are
    processed one after another; a step's attention is numpy matrix products,
    the only part the thread pool spreads over cores."""
    import copy

    import numpy as np
    from threadpoolctl import threadpool_info, threadpool_limits
    from oracle import attention as oatt
    from oracle import turbo, turbo_cache
    from oracle.cache import KiviRow
    from oracle.numerics import decode16
    from quantized_kv_cache_18_b200 import workloads as W

    if w.scheme == "turbo":
        tq_params = (turbo.rotation_wht(w.head_dim) if w.rotation == "wht"
                     else turbo.rotation(W.gaussian_matrix(w, "rot", w.head_dim, w.head_dim)),
                     W.gaussian_matrix(w, "qjl", w.qjl_dim, w.head_dim).astype(np.float64),
                     *turbo.deployed_codebook(w.head_dim))
        rec_bytes = turbo_cache.TB_BYTES
    else:
        rec_bytes = w.group * w.head_dim * w.bits // 4 + 4 * w.head_dim + 4 * w.group

    def decode_steps(row, b, h):
        """Seconds and packed bytes of `steps` append + attention steps."""
        t_sum, nbytes = 0.0, 0
        for s in range(1, steps + 1):
            kn, vn = W.decode_token(w, s)
            q = W.query(w, s)[b, h * w.gqa:(h + 1) * w.gqa]
            t = time.perf_counter()
            row.append(kn[b, h], vn[b, h])
            if w.scheme == "turbo":
                row.attention(q, w.scale)
            else:
                Kd, Vd = row.dequantized()
                oatt.attention(decode16(q, w.dtype), Kd, Vd, w.scale)
            t_sum += time.perf_counter() - t
            nbytes += (row.tq // w.group) * rec_bytes + row.r * 4 * w.head_dim
        return t_sum, nbytes

    acc = dict(pre_s=0.0, pre_bytes=0, multi_s=0.0, multi_bytes=0, single_s=0.0, single_bytes=0)
    rows = 0
    b, h = 0, 0
    wall0 = time.time()
    while acc["multi_s"] + acc["single_s"] + acc["pre_s"] < budget_s and time.time() - wall0 < 3 * budget_s + 15:
        k, v = W.prefill_row(w, b, h)
        if w.scheme == "turbo":
            row = turbo_cache.TurboRow(w.head_dim, w.residual, w.dtype, *tq_params, G=w.group)
        else:
            row = KiviRow(w.head_dim, w.bits, w.group, w.residual, w.dtype)
        t = time.perf_counter()
        row.prefill(k, v)
        acc["pre_s"] += time.perf_counter() - t
        acc["pre_bytes"] += int(k.nbytes + v.nbytes) + (row.tq // w.group) * rec_bytes + row.r * 4 * w.head_dim
        single_row = copy.deepcopy(row)
        ts, nb = decode_steps(row, b, h)
        acc["multi_s"] += ts
        acc["multi_bytes"] += nb
        with threadpool_limits(limits=1):
            ts, nb = decode_steps(single_row, b, h)
        acc["single_s"] += ts
        acc["single_bytes"] += nb
        rows += 1
        h += 1
        if h == w.num_kv_heads:
            h, b = 0, (b + 1) % w.batch
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return dict(value=acc["multi_bytes"] / acc["multi_s"] / 1e9, seconds=acc["multi_s"], rows=rows, steps=steps,
                cores=threads, single_value=acc["single_bytes"] / acc["single_s"] / 1e9,
                single_seconds=acc["single_s"], prefill_value=acc["pre_bytes"] / acc["pre_s"] / 1e9,
                prefill_seconds=acc["pre_s"])


def _sig4(v: float) -> float:
    """v to four significant digits (a slow oracle's GB/s can be far below 1e-4)."""
    return float(f"{v:.4g}")


def cpu_baseline_obj(samp, w):
    return {"value": _sig4(samp["value"]), "unit": "GB/s", "cores": samp["cores"], "kind": "oracle",
            "sample": f"{samp['rows']} (batch, kv-head) rows of {w.name}, {samp['steps']} append + attention "
                      f"step(s) each after the row's prefill, {samp['seconds']:.1f} s; rows one after another, "
                      f"numpy's {samp['cores']}-thread pool in the attention products",
            "single_thread": {"value": _sig4(samp["single_value"]), "unit": "GB/s", "cores": 1,
                              "seconds": round(samp["single_seconds"], 2)},
            "prefill_quantize": {"value": _sig4(samp["prefill_value"]), "unit": "GB/s (inputs read + "
                                 "records and window written)", "seconds": round(samp["prefill_seconds"], 2)}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="70b")
    ap.add_argument("--impl", default="kivi", choices=["kivi", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--page-records", type=int, default=0,
                    help="paged caches: records per page (block tables are random permutations of the pool)")
    ap.add_argument("--page-order", default="shuffled", choices=["shuffled", "in-order"],
                    help="paged caches: pool pages handed out at random or in order")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"

    from quantized_kv_cache_18_b200 import workloads as W
    w = W.WORKLOADS[args.config]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    cfg_desc = {"workload": f"{w.name}: B{w.batch} Hkv{w.num_kv_heads} Hq{w.num_q_heads} d{w.head_dim} "
                            f"S{w.seq_len} {w.scheme} {w.bits}-bit G{w.group} R{w.residual}",
                "global_batch": w.batch * world, "seq_len": w.seq_len, "parallelism": f"dp{world}",
                "l2": "cache replicas > 3x L2, rotated per step"}
    if args.page_records > 0:
        cfg_desc["paged"] = f"{args.page_records} records per page, {args.page_order} block tables"

    if args.impl == "reference":
        if rank != 0:
            return
        samp = oracle_sample(w, args.cpu_budget, steps=max(1, args.steps // 10))
        # the oracle times a bounded sample of rows: a full step's time is
        # projected from its rate over the packed bytes of the first decode step
        rows = w.batch * w.num_kv_heads
        A = w.anchor_tokens if w.scheme == "turbo" else 0
        tq = w.group * (max(0, w.seq_len - A - w.residual) // w.group)
        rec = 4032 if w.scheme == "turbo" else w.group * w.head_dim * w.bits // 4 + 4 * w.head_dim + 4 * w.group
        tokb = 2 * 144 if w.fp8_recent else 4 * w.head_dim
        full_bytes = rows * ((tq // w.group) * rec + (w.seq_len - tq + 1) * tokb)
        value = _sig4(samp["value"])   # the cpu_baseline object's rounding, so the two agree
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(full_bytes / (value * 1e9) * 1e3, 3),
                "ms_per_step_kind": "projected: one full step at the sampled rate", "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg_desc,
                "cpu_baseline": cpu_baseline_obj(samp, w),
                "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_gpu(args, w, rank, world)
    hbm, peak_kind = _peaks()
    value = res["bytes"] / (res["ms"] * 1e-3) / 1e9          # all ranks' bytes / max time
    attn_mean = statistics.mean(res["attn_ms"])
    if w.scheme == "turbo":
        kern, kern_src = "tq_decode_kernel", "tq_attn.cu"
        kern_desc = "tq_decode_kernel (after tq_query_prep_kernel; both inside the timed attention call)"
    else:
        kern, kern_src = "kivi_decode_kernel", "kivi_attn.cu"
        kern_desc = "kivi_decode_kernel (one launch per decode attention)"
    achieved = res["step_bytes_last"] / (attn_mean * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(res["ms"] / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": ("f16 mma (fp32 accumulate) over 3-bit codes + 1-bit sketch" if w.scheme == "turbo"
                  else "f16 mma (fp32 accumulate) over int2/int4 codes"),
        "data": "synthetic", "config": cfg_desc,
        "tokens_per_s": round(w.batch * world * args.steps / (res["ms"] * 1e-3), 1),
        "pct_of_nominal_8tbs_hbm": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "roofline": {"bound": "hbm", "kernel": kern_desc,
                     "achieved": round(achieved, 1), "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4),
                     "traffic": _profiled_traffic(kern, kern_src, w.name),
                     "bytes_per_launch": res["step_bytes_last"], "mean_launch_us": round(attn_mean * 1e3, 2)},
        "e2e": {"value": round(res["e2e_bytes"] / (res["e2e_ms"] * 1e-3) / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]},
        "kernel_timing": {k: round(v, 2) if isinstance(v, float) else v for k, v in res["kernel"].items()},
        "gpu_launches": res["launches"], "clocks": res["clocks"], "replicas": res["n_rep"],
        "decode_splits": res["splits"],
        # secondary: the prefill (quantize kernel + window copy) of one replica,
        # algorithmic bytes = K/V inputs read + packed records and window written
        "prefill": {"us": round(res["prefill_ms"] * 1e3, 1), "bytes": res["prefill_bytes"],
                    "achieved": round(res["prefill_bytes"] / (res["prefill_ms"] * 1e-3) / 1e9, 1), "unit": "GB/s",
                    "frac": round(res["prefill_bytes"] / (res["prefill_ms"] * 1e-3) / 1e9 / hbm, 4),
                    "kernel": "kivi_quantize_kernel" if w.scheme != "turbo" else "tq_quantize_tc_kernel"},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_obj(oracle_sample(w, args.cpu_budget), w)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))


if __name__ == "__main__":
    main()
