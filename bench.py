#!/usr/bin/env python
"""Benchmark of the column-sparse cross-step delta hot path on B200.

One step is one sparse-delta step of a HunyuanVideo-shaped DiT layer (720x1280
video, 129 frames -> 33x90x160 latent, 2x2 patches -> T = 118800 tokens;
d_model 3072, MLP hidden 12288, 24 heads x 128): the MLP delta (gathered
up-projection with GELU / delta / cache writeback, then the gathered sparse-K
down-projection into the fp32 output cache; 70% column sparsity, k = 3686 per
128-token block) and the attention delta (top 7% keys per 128-query block,
k = 8316, merged with the cached complement partial). Selections and caches
come from a dense refresh of the previous step run with the same library.
Steps alternate between two drifted inputs so every step changes the caches.

Printed: one JSON line (rank 0). ``value`` is microseconds per layer-step for
the whole job (max over ranks / number of GPUs); the other hot-path rows (the
FLUX.1-dev layers at 1280x768 and 2304x1280, top-k, dense refresh, cache
gather / scatter, dense layer at k = all, the 10-step schedule) are timed in
the same run and reported under ``rows``.

``--impl reference`` times the C++ fp64 CPU oracle instead, on a bounded sample
of the same workload, extrapolated to one layer-step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "µs/layer & useful TFLOP/s (% B200 bf16 peak) for sparse-delta MLP/attn"
UNIT = "us/layer"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# FLUX.1-dev at 1280x768: 80x48 latent patches (2x2) = 3840 image tokens + 512 text tokens
FLUX = dict(T=4352, D=3072, H=12288, heads=24, d=128, Bt=128, mlp_permille=300, attn_permille=165, sigma=0.03,
            key="flux_1280x768",
            name="FLUX.1-dev 1280x768 DiT layer, sparse-delta step (MLP 70% + attention 83.5% sparse)")
# HunyuanVideo at 720x1280, 129 frames: 33 x 45 x 80 latent patches = 118800 tokens; attention 93% sparse
HUNYUAN = dict(FLUX, T=118800, attn_permille=70, key="hunyuan_720x1280x129",
               name="HunyuanVideo 720x1280x129 DiT layer, sparse-delta step (MLP 70% + attention 93% sparse)")
W = HUNYUAN


def k_of(n, permille):
    return n * permille // 1000


def flops_step(w):
    """Useful FLOPs of one sparse step: selected columns / keys only."""
    T, D, kc = w["T"], w["D"], k_of(w["H"], w["mlp_permille"])
    kk = k_of(w["T"], w["attn_permille"])
    up = 2 * T * D * kc
    down = 2 * T * kc * D
    attn = 4 * T * kk * w["d"] * w["heads"]
    return up, down, attn


def max_over_ranks(x, device=None):
    """Maximum of a per-rank float over all ranks of the default process group (x when there is none)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_us_per_layer(ms_step_max, world):
    """Whole-job microseconds per layer-step: every rank processes one layer per step (weak scaling)."""
    return ms_step_max * 1e3 / world


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS if k in p}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", self.gpu_id], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")
        sm = [num(r[1]) for r in rows]
        mx = [num(r[2]) for r in rows]
        pw = [num(r[3]) for r in rows]
        loaded = [s for s, p in zip(sm, pw) if p > 250.0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded), "power_w_max": max(pw)}


# ---------------------------------------------------------------- CPU oracle sample

class OracleSample:
    """A bounded sample of one sparse layer-step for the C++ fp64 oracle (``oracle/``), with seeded
    synthetic inputs of the layer's shapes: the MLP delta on ``mlp_blocks`` token blocks (the short
    last block among them) and the attention delta on ``attn_tiles`` (head, query-block) tiles of
    at most two heads. With ``whole`` the sample is the whole layer-step (every block, every tile of
    every head). ``time_step`` runs the sample once and returns its wall time and that time
    extrapolated linearly to one layer-step (the two agree when ``whole``)."""

    def __init__(self, w, mlp_blocks=32, attn_tiles=48, seed=0, whole=False):
        import numpy as np
        import oracle
        self.O = oracle.default()
        self.cores = self.O.threads()
        g = np.random.default_rng(seed)
        T, D, H, h, d, Bt = w["T"], w["D"], w["H"], w["heads"], w["d"], w["Bt"]
        self.w, self.whole = w, whole
        self.nb = nb = (T + Bt - 1) // Bt
        kc, kk = k_of(H, w["mlp_permille"]), k_of(T, w["attn_permille"])
        # MLP: the sampled blocks' rows, laid end to end (the short last block last)
        blocks = list(range(nb)) if whole else sorted(set(g.choice(nb - 1, mlp_blocks - 1, replace=False).tolist())
                                                      | {nb - 1})
        rows = sum(min(Bt, T - b * Bt) for b in blocks)
        self.mlp_blocks = len(blocks)
        self.x = g.standard_normal((rows, D))
        self.w1t = g.standard_normal((H, D)) / math.sqrt(D)   # W1 transposed: passed as its .T view, no copy
        self.b1 = 0.02 * g.standard_normal(H)
        self.W2 = g.standard_normal((H, D)) / math.sqrt(H)
        self.A = np.abs(g.standard_normal((rows, H))) * 0.5
        self.Y = g.standard_normal((rows, D))
        self.idx = np.sort(np.stack([g.choice(H, kc, replace=False) for _ in blocks]), axis=1).astype(np.int32)
        # attention: all heads when whole, else two heads with the sampled tiles spread over them
        self.heads = h if whole else min(h, 2)
        self.q = g.standard_normal((self.heads, T, d))
        self.k = g.standard_normal((self.heads, T, d))
        self.v = g.standard_normal((self.heads, T, d))
        # selected keys: spread over the whole sequence, a random offset per (head, block)
        stride = T // max(kk, 1)
        off = g.integers(0, stride, (self.heads, nb, 1))
        self.aidx = (np.arange(kk)[None, None, :] * stride + off).astype(np.int32)
        self.m_c = g.standard_normal((self.heads, T))
        self.l_c = 1.0 + g.random((self.heads, T)) * 100
        self.acc_c = g.standard_normal((self.heads, T, d))
        if whole:
            self.tiles = None
            self.ntiles = h * nb
        else:
            per = max(1, attn_tiles // self.heads)
            self.tiles = [(hh, int(b)) for hh in range(self.heads)
                          for b in sorted(set(g.choice(nb - 1, per - 1, replace=False).tolist()) | {nb - 1})]
            self.ntiles = len(self.tiles)

    def time_step(self):
        """(wall seconds of the sample, microseconds extrapolated to one layer-step)."""
        w = self.w
        t0 = time.perf_counter()
        self.O.mlp_delta(self.x, self.w1t.T, self.b1, self.W2, self.idx, self.A, self.Y, w["Bt"])
        t1 = time.perf_counter()
        self.O.attn_delta(self.q, self.k, self.v, self.aidx, self.m_c, self.l_c, self.acc_c, 1.0 / math.sqrt(w["d"]),
                          w["Bt"], tiles=self.tiles)
        t2 = time.perf_counter()
        us = ((t1 - t0) * self.nb / self.mlp_blocks + (t2 - t1) * (w["heads"] * self.nb) / self.ntiles) * 1e6
        return t2 - t0, us

    def describe(self, runs):
        if self.whole:
            return (f"C++ fp64 oracle ({self.cores} threads): the whole sparse layer-step (MLP delta on all "
                    f"{self.nb} token blocks, attention delta on all {self.ntiles} (head, query-block) tiles), "
                    f"{runs} run(s)")
        return (f"C++ fp64 oracle ({self.cores} threads): MLP delta on {self.mlp_blocks} of {self.nb} token blocks "
                f"and attention delta on {self.ntiles} of {self.w['heads'] * self.nb} (head, query-block) tiles, "
                f"{runs} run(s), extrapolated linearly to one layer-step")

    def info(self, runs):
        return {"kind": "oracle", "cores": int(self.cores), "sample": self.describe(runs)}


def cpu_baseline(w):
    """The oracle on the host cores: a sample of the headline layer-step (extrapolated), and the
    whole FLUX.1-dev 1280x768 layer-step timed as it is."""
    smp = OracleSample(w)
    runs = [smp.time_step() for _ in range(2)]
    info = smp.info(len(runs))
    info["value"] = round(statistics.median(us for _, us in runs), 1)
    info["unit"] = UNIT
    info["sample_wall_s"] = round(statistics.median(s for s, _ in runs), 2)
    del smp
    flux = OracleSample(FLUX, whole=True)
    s, us = flux.time_step()
    info["flux_1280x768_whole_step"] = {"value": round(us, 1), "unit": UNIT, "wall_s": round(s, 2),
                                        "sample": flux.describe(1)}
    return info


# ---------------------------------------------------------------- GPU arm

class Layer:
    """Device-resident layer of the workload `w`: weights, two drifted inputs, caches and selections.
    With keep_mass the attention refresh also keeps the mass [h][nb][T] (the standalone top-k rows use it)."""

    def __init__(self, w, dev, seed, keep_mass=False):
        import torch
        from dynamic_column_sparse_b200 import chipmunk as cm
        self.w, self.dev, self.cm = w, dev, cm
        T, D, H, h, d, Bt = w["T"], w["D"], w["H"], w["heads"], w["d"], w["Bt"]
        g = torch.Generator(device=dev).manual_seed(seed)

        def rn(shape, std=1.0):
            return (torch.randn(shape, generator=g, device=dev) * std).to(torch.bfloat16)

        def drift(t):
            return (t.float() + w["sigma"] * torch.randn(t.shape, generator=g, device=dev)).to(torch.bfloat16)

        self.nb = (T + Bt - 1) // Bt
        self.kc, self.kk = k_of(H, w["mlp_permille"]), k_of(T, w["attn_permille"])
        self.w1t, self.b1 = rn((H, D), 1 / math.sqrt(D)), rn((H,), 0.02)
        self.w2, self.b2 = rn((H, D), 1 / math.sqrt(H)), rn((D,), 0.02)
        x_prev = rn((T, D))
        self.xs = [drift(x_prev)]
        self.xs.append(drift(self.xs[0]))
        qkv_prev = [rn((T, h, d)) for _ in range(3)]
        self.qkvs = [[drift(t) for t in qkv_prev]]
        self.qkvs.append([drift(t) for t in self.qkvs[0]])
        f32, i32 = torch.float32, torch.int32
        self.a_cache = torch.empty((self.nb, H, Bt), dtype=torch.bfloat16, device=dev)
        self.y_cache = torch.empty((T, D), dtype=f32, device=dev)
        self.out = torch.empty((T, D), dtype=torch.bfloat16, device=dev)
        self.idx = torch.empty((self.nb, self.kc), dtype=i32, device=dev)
        self.mlp_scores = torch.empty((self.nb, H), dtype=f32, device=dev)
        self.aidx = torch.empty((h, self.nb, self.kk), dtype=i32, device=dev)
        self.m_c = torch.empty((h, T), dtype=f32, device=dev)
        self.l_c = torch.empty((h, T), dtype=f32, device=dev)
        self.acc_c = torch.empty((h, T, d), dtype=f32, device=dev)
        self.o = torch.empty((T, h, d), dtype=torch.bfloat16, device=dev)
        self.mass = torch.empty((h, self.nb, T), dtype=f32, device=dev) if keep_mass else None
        self.ws = torch.empty(cm.mlp_workspace_bytes(T, H, self.kc, Bt), dtype=torch.uint8, device=dev)
        self.attn_ws = torch.empty(cm.attn_refresh_workspace_bytes(T, h, self.kk, keep_mass), dtype=torch.uint8,
                                   device=dev)
        self.x_prev, self.qkv_prev = x_prev, qkv_prev
        self.refresh()

    def refresh(self, first=True):
        cm, w = self.cm, self.w
        cm.mlp_refresh(self.x_prev, self.w1t, self.b1, self.w2, self.b2, self.a_cache, self.y_cache, self.idx,
                       self.mlp_scores, self.out, Bt=w["Bt"], first_step=first)
        q, k, v = self.qkv_prev
        cm.attn_refresh(q, k, v, self.aidx, self.m_c, self.l_c, self.acc_c, self.o, self.mass,
                        scale=1 / math.sqrt(w["d"]), workspace=self.attn_ws)

    def mlp_up(self, i):
        self.cm.mlp_delta(self.xs[i % 2], self.w1t, self.b1, self.w2, self.idx, self.a_cache, self.y_cache, self.out,
                          Bt=self.w["Bt"], workspace=self.ws, part="up")

    def mlp_down(self, i):
        self.cm.mlp_delta(self.xs[i % 2], self.w1t, self.b1, self.w2, self.idx, self.a_cache, self.y_cache, self.out,
                          Bt=self.w["Bt"], workspace=self.ws, part="down")

    def attn(self, i):
        q, k, v = self.qkvs[i % 2]
        self.cm.attn_delta(q, k, v, self.aidx, self.m_c, self.l_c, self.acc_c, self.o, scale=1 / math.sqrt(self.w["d"]))


def time_events(fn, reps, flush, torch):
    """Median device time (ms) of fn() over reps runs, L2 flushed before each."""
    ts = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def source_sha(files):
    h = hashlib.sha1()
    for f in files:
        with open(os.path.join(ROOT, "dynamic_column_sparse_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


KERNEL_SOURCES = {"mlp_up": ["mlp.cu", "ptx.cuh"], "mlp_down": ["mlp.cu", "ptx.cuh"], "attn_delta": ["attn.cu", "ptx.cuh"]}


def traffic_for(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary of this kernel at this workload, if the
    kernel source is unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(f"{kernel}@{workload}")
    if not e or e.get("source_sha1") != source_sha(KERNEL_SOURCES[kernel]):
        return None
    return e.get("dram_bytes_per_launch")


def run_gpu(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} needs {args.gpus} ranks (launch with torchrun); WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    from dynamic_column_sparse_b200 import chipmunk as cm
    cm.load_library()
    w = dict(W)
    L = Layer(w, dev, seed=1234 + rank)
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0, "device status set during set-up"
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.zero_()

    def step(i, ev=None):
        if ev:
            ev[0].record()
        L.mlp_up(i)
        if ev:
            ev[1].record()
        L.mlp_down(i)
        if ev:
            ev[2].record()
        L.attn(i)
        if ev:
            ev[3].record()

    for i in range(args.warmup):
        flush()
        step(i)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush()
        step(i, evs[i])
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    tot = [e[0].elapsed_time(e[3]) for e in evs]
    t_up = [e[0].elapsed_time(e[1]) for e in evs]
    t_down = [e[1].elapsed_time(e[2]) for e in evs]
    t_attn = [e[2].elapsed_time(e[3]) for e in evs]
    ms_step = max_over_ranks(statistics.mean(tot), dev)
    status = cm.read_device_status()
    assert status == 0, f"device status {status}"

    # End to end through the public API, every step's inputs copied in from pinned host memory
    # and its outputs copied back, pipelined over three streams: step i + 1's inputs go up and
    # step i - 1's outputs come down while step i computes (device inputs and outputs double
    # buffered, events order the reuse; the caches update in place on the compute stream, step
    # after step). The per-step working set (weights, caches, inputs: about 450 MB) is larger
    # than L2, so the steps are not flushed in between. Per step = the whole run / steps.
    x_h = [x.cpu().pin_memory() for x in L.xs]
    qkv_h = [[t.cpu().pin_memory() for t in qkv] for qkv in L.qkvs]
    out_h = torch.empty(L.out.shape, dtype=L.out.dtype).pin_memory()
    o_h = torch.empty(L.o.shape, dtype=L.o.dtype).pin_memory()
    x_d = [torch.empty_like(L.xs[0]) for _ in range(2)]
    qkv_d = [[torch.empty_like(t) for t in L.qkvs[0]] for _ in range(2)]
    out_d = [torch.empty_like(L.out) for _ in range(2)]
    o_d = [torch.empty_like(L.o) for _ in range(2)]
    s_cmp = torch.cuda.current_stream()
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
    w_ = L.w

    def e2e_run(nsteps):
        ev = lambda: torch.cuda.Event(enable_timing=True)
        ev_h, ev_c, ev_d = [ev() for _ in range(nsteps)], [ev() for _ in range(nsteps)], [ev() for _ in range(nsteps)]
        start, end = ev(), ev()
        start.record(s_h2d)
        for i in range(nsteps):
            b = i % 2
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(ev_c[i - 2])       # step i - 2 has read this input buffer
                x_d[b].copy_(x_h[i % 2], non_blocking=True)
                for dst, src in zip(qkv_d[b], qkv_h[i % 2]):
                    dst.copy_(src, non_blocking=True)
                ev_h[i].record(s_h2d)
            s_cmp.wait_event(ev_h[i])
            if i >= 2:
                s_cmp.wait_event(ev_d[i - 2])           # step i - 2's outputs are downloaded
            cm.mlp_delta(x_d[b], L.w1t, L.b1, L.w2, L.idx, L.a_cache, L.y_cache, out_d[b], Bt=w_["Bt"],
                         workspace=L.ws, stream=s_cmp)
            cm.attn_delta(*qkv_d[b], L.aidx, L.m_c, L.l_c, L.acc_c, o_d[b], scale=1 / math.sqrt(w_["d"]),
                          stream=s_cmp)
            ev_c[i].record(s_cmp)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_c[i])
                out_h.copy_(out_d[b], non_blocking=True)
                o_h.copy_(o_d[b], non_blocking=True)
                ev_d[i].record(s_d2h)
        end.record(s_d2h)
        end.synchronize()
        torch.cuda.synchronize()
        return start.elapsed_time(end) / nsteps

    e2e_run(max(args.warmup, 3))
    barrier()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e2e_run(args.steps), dev)
    barrier()
    h2d = x_d[0].numel() * 2 + sum(t.numel() * 2 for t in qkv_d[0])
    d2h = out_h.numel() * 2 + o_h.numel() * 2

    peaks, peak_src = load_peaks()
    f_up, f_down, f_attn = flops_step(w)
    flops = f_up + f_down + f_attn
    kern = {}
    for name, ts, fl in (("mlp_up", t_up, f_up), ("mlp_down", t_down, f_down), ("attn_delta", t_attn, f_attn)):
        ms = statistics.mean(ts)
        kern[name] = {"us": round(ms * 1e3, 2), "tflops": round(fl / (ms * 1e-3) / 1e12, 1),
                      "frac_bf16_peak": round(fl / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4)}
    dom = max(kern, key=lambda k: kern[k]["us"])
    dom_flops = {"mlp_up": f_up, "mlp_down": f_down, "attn_delta": f_attn}[dom]
    achieved = dom_flops / (kern[dom]["us"] * 1e-6) / 1e12
    tr = traffic_for(dom, w["key"])
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "traffic": tr, "peak_source": f"{peak_src} bf16 dense (burst)"}
    if "bf16_tflops_sustained" in peaks:
        roofline["frac_of_sustained"] = round(achieved / peaks["bf16_tflops_sustained"], 4)
        roofline["sustained_peak"] = peaks["bf16_tflops_sustained"]

    us_layer = job_us_per_layer(ms_step, world)
    res = {
        "metric": METRIC, "value": round(us_layer, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded device Philox normals with the layer recipe's distributions (no model weights)",
        "config": {"workload": w["name"],
                   "T": w["T"], "d_model": w["D"], "mlp_hidden": w["H"], "heads": w["heads"], "head_dim": w["d"],
                   "block": w["Bt"], "mlp_k": L.kc, "attn_k": L.kk, "global_batch": world, "seq_len": w["T"],
                   "l2": "flushed before every timed step (write of a 2x L2 buffer, outside the step's events)",
                   "parallelism": f"independent layer per GPU x{world} (no collective)"},
        "useful_tflops": round(flops * world / (ms_step * 1e-3) / 1e12, 1),
        "pct_bf16_peak": round(100 * flops / (ms_step * 1e-3) / 1e12 / peaks["bf16_tflops"], 2),
        "kernels": kern, "roofline": roofline,
        "e2e": {"value": round(job_us_per_layer(e2e_ms, world), 2), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h),
                "overlap": "step i+1 inputs up and step i-1 outputs down while step i computes (3 streams)"},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_rows:
        groups = set(ROW_GROUPS) if args.rows == "all" else set(args.rows.split(","))
        res["rows"] = extra_rows(L, w, peaks, flush, torch, cm, groups)
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(res), flush=True)
    del L
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def step_rows(Lx, w, reps, flush, torch):
    """Per-kernel device time and useful TFLOP/s of one sparse step of layer Lx."""
    T, D, H, h, d = w["T"], w["D"], w["H"], w["heads"], w["d"]
    out = {"T": T, "mlp_k": Lx.kc, "attn_k": Lx.kk}
    flops = {"mlp_up": 2 * T * D * Lx.kc, "mlp_down": 2 * T * D * Lx.kc, "attn_delta": 4 * T * Lx.kk * d * h}
    total = 0.0
    for name, fn in (("mlp_up", Lx.mlp_up), ("mlp_down", Lx.mlp_down), ("attn_delta", Lx.attn)):
        it = [0]

        def call():
            it[0] += 1
            fn(it[0])
        call()
        ms = time_events(call, reps, flush, torch)
        total += ms
        out[name] = {"us": round(ms * 1e3, 1), "tflops": round(flops[name] / (ms * 1e-3) / 1e12, 1)}
    out["step_us"] = round(total * 1e3, 1)
    return out


ROW_GROUPS = ("topk", "cols", "refresh", "dense", "sweep", "compact", "workloads", "fp8", "cublas")


def fp8_rows(Lx, w, reps, flush, torch, cm, peaks):
    """The FP8 form of the sparse MLP step on layer Lx: x quantised per token (timed on its own), then
    the gathered e4m3 GEMMs (chipmunk_mlp_delta_fp8). The weights are quantised once, outside the
    timing; the deltas use a static scale that covers |delta| <= 0.5."""
    T, D, H = w["T"], w["D"], w["H"]
    w1t8, s1 = cm.quantize_e4m3_rows(Lx.w1t)
    w2_8, s2 = cm.quantize_e4m3_rows(Lx.w2)
    s_delta = float(s2.max().item()) * 0.5 / 448.0
    g2 = (s2 / s_delta).float().contiguous()
    x8 = torch.empty((T, D), dtype=torch.uint8, device=Lx.dev)
    sx = torch.empty((T,), dtype=torch.float32, device=Lx.dev)
    ws = torch.empty(cm.mlp_fp8_workspace_bytes(T, H, Lx.kc), dtype=torch.uint8, device=Lx.dev)
    it = [0]

    def quant():
        cm.quantize_e4m3_rows(Lx.xs[it[0] % 2], x8, sx)

    def step():
        it[0] += 1
        cm.mlp_delta_fp8(x8, sx, w1t8, s1, Lx.b1, w2_8, g2, s_delta, Lx.idx, Lx.a_cache, Lx.y_cache, Lx.out,
                         workspace=ws)
    quant()
    step()
    ms_q = time_events(quant, reps, flush, torch)
    ms_s = time_events(step, reps, flush, torch)
    flops = 4 * T * D * Lx.kc
    fp8_peak = 2.0 * peaks["bf16_tflops"]   # the measured bf16 peak times the nominal fp8 / bf16 ratio
    return {"T": T, "mlp_k": Lx.kc, "quantize_x_us": round(ms_q * 1e3, 1), "mlp_fp8_us": round(ms_s * 1e3, 1),
            "tflops": round(flops / (ms_s * 1e-3) / 1e12, 1),
            "frac_fp8_peak": round(flops / (ms_s * 1e-3) / 1e12 / fp8_peak, 4),
            "peak_note": "fp8 peak = 2 x measured bf16 burst (nominal ratio)"}


def extra_rows(L, w, peaks, flush, torch, cm, groups=frozenset(ROW_GROUPS)):
    """The other rows of the hot path, timed with CUDA events (median of several runs, L2 flushed).

    ``L`` is the headline (HunyuanVideo) layer; the FLUX.1-dev rows build their own layer."""
    hbm = peaks["hbm_gbs"]
    rows = {}

    def gbs(nbytes, ms):
        return {"us": round(ms * 1e3, 2), "GB/s": round(nbytes / (ms * 1e-3) / 1e9, 1),
                "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4)}

    if "workloads" in groups:
        hunyuan_refresh_rows(L, w, rows, gbs, flush, torch, cm)
    wf = dict(FLUX)
    LF = Layer(wf, L.dev, seed=77, keep_mass=True)
    T, D, H, h = wf["T"], wf["D"], wf["H"], wf["heads"]
    if "workloads" in groups:
        # the same sparse step at the pages' two FLUX.1-dev workloads: 1280x768 (80 x 48 latent
        # patches + 512 text tokens) and 2304x1280 (144 x 80 latent patches + 512 text tokens)
        rows["flux_1280x768_step"] = step_rows(LF, wf, 10, flush, torch)
        w2 = dict(wf, T=144 * 80 + 512)
        L2 = Layer(w2, L.dev, seed=99)
        rows["flux_2304x1280_step"] = step_rows(L2, w2, 5, flush, torch)
        del L2
        torch.cuda.empty_cache()
    if "fp8" in groups:
        rows["fp8_mlp_flux_1280x768"] = fp8_rows(LF, wf, 10, flush, torch, cm, peaks)
        rows["fp8_mlp_hunyuan"] = fp8_rows(L, w, 3, flush, torch, cm, peaks)
    if "topk" in groups:
        topk_rows(LF, wf, rows, gbs, flush, torch, cm)
    if "cols" in groups:
        cols_rows(LF, wf, rows, gbs, flush, torch, cm)
    dense_mlp_f = 4 * T * D * H
    dense_attn_f = 4 * T * T * wf["d"] * h
    if "refresh" in groups:
        refresh_rows(LF, wf, rows, flush, torch, cm, dense_mlp_f, dense_attn_f)
    lib_dense_us = None
    if "cublas" in groups:
        lib_dense_us = library_dense_rows(LF, wf, rows, flush, torch)
    if "dense" in groups or "sweep" in groups:
        dense_us = dense_rows(LF, wf, rows, flush, torch, cm, dense_mlp_f, dense_attn_f)
        if "sweep" in groups:
            sweep_rows(LF, wf, rows, flush, torch, dense_us, lib_dense_us)
    if "compact" in groups:
        compact_rows(LF, wf, rows, flush, torch, hbm)
    del LF
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    return rows


def hunyuan_refresh_rows(L, w, rows, gbs, flush, torch, cm):
    """a5 at the HunyuanVideo layer: the dense MLP refresh, and the attention refresh (dense pass, the
    attention mass with its top-k in one kernel, complement pass). For comparison the attention refresh
    is also timed keeping the mass in HBM, and the standalone top-k over that kept mass."""
    T, D, H, h, d = w["T"], w["D"], w["H"], w["heads"], w["d"]
    ms_mlp = time_events(lambda: cm.mlp_refresh(L.x_prev, L.w1t, L.b1, L.w2, L.b2, L.a_cache, L.y_cache, L.idx,
                                                L.mlp_scores, L.out, Bt=w["Bt"]), 3, flush, torch)
    q, k, v = L.qkv_prev
    ms_attn = time_events(lambda: cm.attn_refresh(q, k, v, L.aidx, L.m_c, L.l_c, L.acc_c, L.o, None,
                                                  scale=1 / math.sqrt(d), workspace=L.attn_ws), 3, flush, torch)
    mass = torch.empty((h, L.nb, T), dtype=torch.float32, device=L.dev)
    ws_kept = torch.empty(cm.attn_refresh_workspace_bytes(T, h, L.kk, True), dtype=torch.uint8, device=L.dev)
    ms_kept = time_events(lambda: cm.attn_refresh(q, k, v, L.aidx, L.m_c, L.l_c, L.acc_c, L.o, mass,
                                                  scale=1 / math.sqrt(d), workspace=ws_kept), 2, flush, torch)
    aidx2 = torch.empty((h * L.nb, L.kk), dtype=torch.int32, device=L.dev)
    ms_topk = time_events(lambda: cm.topk_cols(mass.view(h * L.nb, T), L.kk, out=aidx2), 3, flush, torch)
    del mass, ws_kept, aidx2
    dense_attn_f = 4 * T * T * d * h
    rows["hunyuan_refresh"] = {
        "mlp_us": round(ms_mlp * 1e3, 1), "mlp_tflops": round(4 * T * D * H / (ms_mlp * 1e-3) / 1e12, 1),
        "attn_us": round(ms_attn * 1e3, 1), "attn_passes": "dense + fused mass/top-k + complement",
        "attn_tflops_mma": round(2.5 * dense_attn_f / (ms_attn * 1e-3) / 1e12, 1),
        "attn_us_mass_kept": round(ms_kept * 1e3, 1),
        "mass_bytes_not_written": h * L.nb * T * 4,
        "standalone_topk_on_kept_mass": dict(rows=h * L.nb, n=T, k=L.kk, **gbs(h * L.nb * (T + L.kk) * 4, ms_topk)),
        "us": round((ms_mlp + ms_attn) * 1e3, 1)}


def topk_rows(L, w, rows, gbs, flush, torch, cm):
    """a1: top-k over the layer's score rows, and over HunyuanVideo-length attention rows."""
    T, H, h = w["T"], w["H"], w["heads"]
    reps = 10
    ms = time_events(lambda: cm.topk_cols(L.mlp_scores, L.kc, out=L.idx), reps, flush, torch)
    rows["topk_flux_mlp"] = dict(rows=L.nb, n=H, k=L.kc, **gbs(L.nb * (H + L.kc) * 4, ms))
    mass2 = L.mass.view(h * L.nb, T)
    aidx2 = L.aidx.view(h * L.nb, L.kk)
    ms = time_events(lambda: cm.topk_cols(mass2, L.kk, out=aidx2), reps, flush, torch)
    rows["topk_flux_attn"] = dict(rows=h * L.nb, n=T, k=L.kk, **gbs(h * L.nb * (T + L.kk) * 4, ms))
    g = torch.Generator(device=L.dev).manual_seed(7)
    hn, hk, hr = 118800, 8316, 148 * 20
    hs = torch.rand((hr, hn), generator=g, device=L.dev) ** 4
    hidx = torch.empty((hr, hk), dtype=torch.int32, device=L.dev)
    ms = time_events(lambda: cm.topk_cols(hs, hk, out=hidx), 3, flush, torch)
    rows["topk_hunyuan_attn_rows"] = dict(rows=hr, n=hn, k=hk, note="2960 of 22296 HunyuanVideo mass rows",
                                          **gbs(hr * (hn + hk) * 4, ms))
    del hs, hidx


def cols_rows(L, w, rows, gbs, flush, torch, cm):
    """a6: cache column gather / scatter (FLUX and HunyuanVideo-sized caches)."""
    H, Bt = w["H"], w["Bt"]
    reps = 10
    g = torch.Generator(device=L.dev).manual_seed(8)
    packed = torch.empty((L.nb, L.kc, Bt), dtype=torch.bfloat16, device=L.dev)
    nbytes = 2 * L.nb * L.kc * Bt * 2
    ms = time_events(lambda: cm.gather_cols(L.a_cache, L.idx, packed), reps, flush, torch)
    rows["gather_flux"] = gbs(nbytes, ms)
    ms = time_events(lambda: cm.scatter_cols(packed, L.idx, L.a_cache), reps, flush, torch)
    rows["scatter_flux"] = gbs(nbytes, ms)
    del packed
    nbh = (118800 + 127) // 128
    cache_h = torch.zeros((nbh, H, Bt), dtype=torch.bfloat16, device=L.dev)
    idx_h = torch.sort(torch.rand((nbh, H), generator=g, device=L.dev).argsort(dim=1)[:, :L.kc], dim=1)[0]
    idx_h = idx_h.to(torch.int32).contiguous()
    packed_h = torch.empty((nbh, L.kc, Bt), dtype=torch.bfloat16, device=L.dev)
    nbytes = 2 * nbh * L.kc * Bt * 2
    ms = time_events(lambda: cm.gather_cols(cache_h, idx_h, packed_h), 5, flush, torch)
    rows["gather_hunyuan"] = gbs(nbytes, ms)
    ms = time_events(lambda: cm.scatter_cols(packed_h, idx_h, cache_h), 5, flush, torch)
    rows["scatter_hunyuan"] = gbs(nbytes, ms)
    del cache_h, idx_h, packed_h


def refresh_rows(L, w, rows, flush, torch, cm, dense_mlp_f, dense_attn_f):
    """a5: dense refresh of the layer."""
    Bt = w["Bt"]
    ms_mlp = time_events(lambda: cm.mlp_refresh(L.x_prev, L.w1t, L.b1, L.w2, L.b2, L.a_cache, L.y_cache, L.idx,
                                                L.mlp_scores, L.out, Bt=Bt), 5, flush, torch)
    q, k, v = L.qkv_prev
    ws = torch.empty(cm.attn_refresh_workspace_bytes(w["T"], w["heads"], L.kk, False), dtype=torch.uint8, device=L.dev)
    ms_attn = time_events(lambda: cm.attn_refresh(q, k, v, L.aidx, L.m_c, L.l_c, L.acc_c, L.o, None,
                                                  scale=1 / math.sqrt(w["d"]), workspace=ws), 5, flush, torch)
    rows["refresh_mlp"] = {"us": round(ms_mlp * 1e3, 1),
                           "tflops": round(dense_mlp_f / (ms_mlp * 1e-3) / 1e12, 1)}
    rows["refresh_attn"] = {"us": round(ms_attn * 1e3, 1), "passes": "dense + fused mass/top-k + complement",
                            "tflops_mma": round(2.5 * dense_attn_f / (ms_attn * 1e-3) / 1e12, 1)}


def dense_rows(L, w, rows, flush, torch, cm, dense_mlp_f, dense_attn_f):
    """The dense layer at the same shape with the same kernels (k = all columns, all keys)."""
    T, H, h, Bt = w["T"], w["H"], w["heads"], w["Bt"]
    q, k, v = L.qkv_prev
    idx_all = torch.arange(H, dtype=torch.int32, device=L.dev).repeat(L.nb, 1).contiguous()
    ws_all = torch.empty(cm.mlp_workspace_bytes(T, H, H, Bt), dtype=torch.uint8, device=L.dev)
    aidx_all = torch.arange(T, dtype=torch.int32, device=L.dev).repeat(h, L.nb, 1).contiguous()
    m0 = torch.full((h, T), float("-inf"), device=L.dev)
    l0 = torch.zeros((h, T), device=L.dev)
    a0 = torch.zeros((h, T, w["d"]), device=L.dev)
    ms_dm = time_events(lambda: cm.mlp_delta(L.xs[0], L.w1t, L.b1, L.w2, idx_all, L.a_cache, L.y_cache, L.out,
                                             Bt=Bt, workspace=ws_all), 5, flush, torch)
    ms_da = time_events(lambda: cm.attn_delta(q, k, v, aidx_all, m0, l0, a0, L.o, scale=1 / math.sqrt(w["d"])), 5,
                        flush, torch)
    rows["dense_layer_k_all"] = {"us": round((ms_dm + ms_da) * 1e3, 1), "mlp_us": round(ms_dm * 1e3, 1),
                                 "attn_us": round(ms_da * 1e3, 1),
                                 "tflops": round((dense_mlp_f + dense_attn_f) / ((ms_dm + ms_da) * 1e-3) / 1e12, 1)}
    return (ms_dm + ms_da) * 1e3


def library_dense_rows(L, w, rows, flush, torch):
    """Context only: the dense FLUX layer with library kernels, torch.matmul (cuBLAS) + GELU for the MLP and
    torch's scaled_dot_product_attention for the attention. Returns the layer's us."""
    T, h, d = w["T"], w["heads"], w["d"]
    xw, w1 = L.xs[0], L.w1t.t()
    ms_mlp = time_events(lambda: torch.matmul(torch.nn.functional.gelu(torch.matmul(xw, w1), approximate="tanh"),
                                              L.w2), 5, flush, torch)
    q, k, v = (t.view(1, T, h, d).transpose(1, 2) for t in L.qkvs[0])
    ms_attn = time_events(lambda: torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=d ** -0.5), 5,
                          flush, torch)
    rows["dense_mlp_torch_context"] = {"us": round(ms_mlp * 1e3, 1), "T": T,
                                       "note": "torch.matmul (cuBLAS) + GELU at the FLUX 1280x768 shape, context only"}
    rows["dense_attn_torch_sdpa_context"] = {"us": round(ms_attn * 1e3, 1), "T": T, "heads": h,
                                             "note": "torch scaled_dot_product_attention at the FLUX 1280x768 shape, "
                                                     "context only"}
    return (ms_mlp + ms_attn) * 1e3


def compact_rows(L, w, rows, flush, torch, hbm):
    """Attention delta step with the complement cached as fp32 (m, l, acc) or compact (lse fp32, o_c bf16)."""
    from dynamic_column_sparse_b200.layer import SparseDeltaAttention
    T, h, d = w["T"], w["heads"], w["d"]
    out = {}
    for name, compact in (("partial_fp32", False), ("compact_lse_bf16", True)):
        att = SparseDeltaAttention(T, h, L.dev, w["attn_permille"], compact=compact)
        att.refresh(*L.qkv_prev)
        it = [0]

        def step():
            it[0] += 1
            att.step(*L.qkvs[it[0] % 2])
        step()
        ms = time_events(step, 10, flush, torch)
        cache_bytes = h * T * (4 + d * 2) if compact else h * T * (8 + d * 4)
        nbytes = 4 * T * h * d * 2 + cache_bytes + h * att.nb * att.k * 4
        out[name] = {"us": round(ms * 1e3, 1), "tflops": round(4 * T * att.k * d * h / (ms * 1e-3) / 1e12, 1),
                     "algorithmic_MB": round(nbytes / 1e6, 1),
                     "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4)}
        del att
    rows["attn_delta_cache_forms"] = out


def sweep_rows(L, w, rows, flush, torch, dense_us, lib_dense_us=None):
    """Multi-step schedule (10 steps, dense at 0 and 5) across sparsity levels, through the layer API.
    The speed-ups are against this library's own dense layer (k = all) and, when timed, against the
    faster of that and the library-kernel dense layer (cuBLAS MLP + torch attention)."""
    from dynamic_column_sparse_b200.layer import Schedule, SparseDeltaAttention, SparseDeltaMLP
    T, h, Bt = w["T"], w["heads"], w["Bt"]
    reps = 10
    sweep = {}
    for mp, ap in ((500, 500), (300, 165), (150, 150), (70, 70)):
        mlp = SparseDeltaMLP(L.w1t, L.b1, L.w2, L.b2, T, Bt, mp)
        att = SparseDeltaAttention(T, h, L.dev, ap)
        mlp.refresh(L.x_prev)
        att.refresh(*L.qkv_prev)
        ms_ref = time_events(lambda: (mlp.refresh(L.x_prev), att.refresh(*L.qkv_prev)), 3, flush, torch)
        it = [0]

        def sparse_step():
            i = it[0] = it[0] + 1
            mlp.step(L.xs[i % 2])
            att.step(*L.qkvs[i % 2])
        ms_sp = time_events(sparse_step, reps, flush, torch)
        sched = Schedule((0, 5))
        n_dense = sum(sched.is_dense(s) for s in range(10))
        amort = (n_dense * ms_ref + (10 - n_dense) * ms_sp) / 10 * 1e3
        sweep[f"mlp{100 - mp // 10}_attn{round(100 - ap / 10, 1)}"] = {
            "mlp_k": mlp.k, "attn_k": att.k, "sparse_step_us": round(ms_sp * 1e3, 1),
            "refresh_us": round(ms_ref * 1e3, 1), "loop10_us_per_layer_step": round(amort, 1),
            "speedup_vs_dense_k_all": round(dense_us / (ms_sp * 1e3), 2)}
        if lib_dense_us is not None:
            best = min(dense_us, lib_dense_us)
            sweep[f"mlp{100 - mp // 10}_attn{round(100 - ap / 10, 1)}"].update(
                speedup_vs_fastest_dense=round(best / (ms_sp * 1e3), 2),
                loop10_speedup_vs_fastest_dense=round(best / amort, 2))
        del mlp, att
    rows["loop_sweep"] = sweep


# ---------------------------------------------------------------- reference arm

def run_reference(args):
    """The oracle as it stands, on the host cores: each step runs a bounded sample of the headline
    layer-step (2 token blocks of the MLP delta, 8 (head, query-block) tiles of the attention delta).
    ``ms_per_step`` is the sample's own wall time; ``value`` extrapolates it linearly to one whole
    layer-step, the metric's unit."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = dict(W)
    smp = OracleSample(w, mlp_blocks=2, attn_tiles=8)
    for _ in range(args.warmup):
        smp.time_step()
    runs = [smp.time_step() for _ in range(args.steps)]
    us = statistics.mean(u for _, u in runs)
    wall_ms = statistics.mean(s for s, _ in runs) * 1e3
    info = smp.info(args.steps)
    info["value"] = round(us, 1)
    info["unit"] = UNIT
    res = {"impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(wall_ms, 3), "higher_is_better": False,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic: seeded numpy normals with the layer recipe's shapes",
           "config": {"workload": w["name"], "T": w["T"], "d_model": w["D"], "mlp_hidden": w["H"],
                      "heads": w["heads"], "head_dim": w["d"], "block": w["Bt"],
                      "ms_per_step": "wall time of one step's sample; value is that sample extrapolated to a layer-step"},
           "cpu_baseline": info,
           "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


PROFILE_CASES = ("attn_delta", "mass_select", "mass_kept", "mlp", "topk_long")


def run_profile_case(args):
    """Runs one kernel's workload at a size an ncu capture of many passes can hold (a few GB at most,
    inputs larger than L2), `--steps` times, and prints what ran. Not a bench line.
      attn_delta, mass_select, mass_kept: the HunyuanVideo attention (T = 118800, k = 8316) on 2 of
        its 24 heads (heads are independent, so per-launch traffic scales by 12). attn_delta runs the
        sparse step; mass_select the refresh without a mass tensor (the fused mass/top-k kernel keeps
        the rows in its L2 row buffers), mass_kept the refresh writing the mass [h][nb][T] to HBM.
      mlp: the sparse MLP step (mlp_up, mlp_down) of the FLUX.1-dev 2304x1280 layer (T = 12032).
      topk_long: the top-k (k = 8316) of 2960 HunyuanVideo-length rows (118800) drawn as u^4, the bench's
        `topk_hunyuan_attn_rows` row (1.41 GB)."""
    import torch
    from dynamic_column_sparse_b200 import chipmunk as cm
    cm.load_library()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.profile_case == "topk_long":
        g = torch.Generator(device=dev).manual_seed(7)
        hn, hk, hr = 118800, 8316, 148 * 20
        hs = torch.rand((hr, hn), generator=g, device=dev) ** 4
        for _ in range(args.steps):
            cm.topk_cols(hs, hk)
        info = {"rows": hr, "n": hn, "k": hk}
    elif args.profile_case == "mlp":
        w = dict(FLUX, T=144 * 80 + 512, key="flux_2304x1280")
        L = Layer(w, dev, seed=99)
        for i in range(args.steps):
            L.mlp_up(i)
            L.mlp_down(i)
        info = {"T": w["T"], "mlp_k": L.kc}
    else:
        w = dict(HUNYUAN, heads=2)
        T, h, d = w["T"], w["heads"], w["d"]
        kk, nb = k_of(T, w["attn_permille"]), (T + 127) // 128
        g = torch.Generator(device=dev).manual_seed(5)
        q, k, v = ((torch.randn((T, h, d), generator=g, device=dev)).to(torch.bfloat16) for _ in range(3))
        idx = torch.empty((h, nb, kk), dtype=torch.int32, device=dev)
        m_c, l_c = (torch.empty((h, T), dtype=torch.float32, device=dev) for _ in range(2))
        acc_c = torch.empty((h, T, d), dtype=torch.float32, device=dev)
        o = torch.empty((T, h, d), dtype=torch.bfloat16, device=dev)
        keep = args.profile_case == "mass_kept"
        mass = torch.empty((h, nb, T), dtype=torch.float32, device=dev) if keep else None
        ws = torch.empty(cm.attn_refresh_workspace_bytes(T, h, kk, keep), dtype=torch.uint8, device=dev)
        refresh = lambda: cm.attn_refresh(q, k, v, idx, m_c, l_c, acc_c, o, mass, scale=d ** -0.5, workspace=ws)
        refresh()
        for _ in range(args.steps):
            if args.profile_case == "attn_delta":
                cm.attn_delta(q, k, v, idx, m_c, l_c, acc_c, o, scale=d ** -0.5)
            else:
                refresh()
        info = {"T": T, "heads": h, "attn_k": kk}
    torch.cuda.synchronize()
    assert cm.read_device_status() == 0
    print(json.dumps({"profile_case": args.profile_case, "launches": args.steps, **info}), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-rows", action="store_true", help="skip the extra hot-path rows")
    ap.add_argument("--rows", default="all",
                    help="comma list of extra row groups: " + ",".join(ROW_GROUPS) + " (default: all)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", choices=PROFILE_CASES,
                    help="run one kernel's workload at a size for an ncu capture, --steps times (no bench line)")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
