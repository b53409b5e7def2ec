#!/usr/bin/env python
"""Benchmark of the streaming chunk-attention hot path on B200.

One bench step = one block of a rollout through the model's attention layers:
for every denoising step and every layer, one fd_block_attention call with
that step's q/k/v, then one batched fd_cache_commit of the last step's k/v
into every layer's ring buffer.  The cache is full (steady state) before the
timed region, so every call attends to sinks + the whole window + the block.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fd|reference]
                    [--workload 480p|tiny|large|long|ragged|multiview|gqa|d64]

N > 1 runs one independent replica per GPU (the path has no exchange step):
value = work of all ranks / max-over-ranks time ("scaling": "weak").
`--impl reference` times the CPU oracle (the reference arm of this method)
on a bounded sample of the same workload.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("chunk-attention TFLOP/s & latent-frames/s per layer; "
          "% of bf16 tensor/HBM roofline")
PROFILE = os.path.join(ROOT, "profiles", "attn_bf16_d128_sm100.480p.md")
_CSRC = os.path.join(ROOT, "streaming_autoregressive_video_b200", "csrc")
# a kernel's source files: the .cu and the package headers it includes (the
# summaries record the sha256 of their bytes concatenated in this order)
KERNEL_SRCS = [os.path.join(_CSRC, f)
               for f in ("attn_sm100.cu", "attn_sched.cuh", "sm100.cuh", "fd_internal.h")]
COMMIT_PROFILE = os.path.join(ROOT, "profiles", "commit_copy_kernel.480p_l30.md")
COMMIT_SRCS = [os.path.join(_CSRC, f) for f in ("cache_kernels.cu", "fd_internal.h")]


def workloads():
    from streaming_autoregressive_video_b200 import workloads as wl
    return {"480p": wl.SINGLE_480P, "tiny": wl.TINY_F32, "large": wl.LARGE_ACTIONS,
            "long": wl.LONG_ROLLOUT, "ragged": wl.BATCHED_RAGGED,
            "multiview": wl.MULTIVIEW_4, "gqa": wl.GQA_480P, "d64": wl.D64_480P}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["fd", "reference"], default="fd")
    ap.add_argument("--workload", default="480p")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the finalize-overlap and other-workload measurements")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the layer count (small profiling cases only)")
    return ap.parse_args()


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------
def attn_flops(w, nkeys_per_rollout):
    """Algorithmic FLOPs of one call: QK^T + PV over the valid keys only."""
    return sum(4.0 * w.heads * w.head_dim * w.queries * nk for nk in nkeys_per_rollout)


def attn_bytes(w, nkeys_per_rollout, esz=2):
    """Q + block K/V + valid cache K/V read once + O written once (queries and
    outputs carry H heads, keys and values Hkv)."""
    per_q = w.heads * w.head_dim * esz
    per_kv = w.hkv * w.head_dim * esz
    b = 0
    for nk in nkeys_per_rollout:
        b += 2 * w.queries * per_q + 2 * nk * per_kv
    return float(b)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
            "bf16_tflops_sustained": 1400.0}, "fallback"


def sources_sha256(sources):
    h = hashlib.sha256()
    for path in sources:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _traffic_from(profile, sources):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (sha256 recorded in the summary)."""
    try:
        text = open(profile).read()
        src = sources_sha256(sources)
    except OSError:
        return None
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_tr or m_sha.group(1) != src:
        return None
    return float(m_tr.group(1))


def profile_traffic():
    return _traffic_from(PROFILE, KERNEL_SRCS)


def commit_traffic():
    return _traffic_from(COMMIT_PROFILE, COMMIT_SRCS)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd_, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd_)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r[2] > 250.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[3])
                          if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in load),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(load),
                "power_w_max": max(r[2] for r in rows)}


# --------------------------------------------------------------------------
# Workload description (both arms print the same config)
# --------------------------------------------------------------------------
def prefill_frames(w, rank):
    """Frames committed per rollout before the timed block: the window is
    filled (steady state), or for a ragged workload each rollout's fill is
    drawn from the replica's seed."""
    from streaming_autoregressive_video_b200 import synth
    if w.ragged_window:
        lo, hi = w.ragged_window
        return [int(x) for x in
                synth.ragged_fill(synth.seed_of(replica_seed_base(rank), 3), w.rollouts, lo, hi)]
    return [w.block_frames * (-(-w.slots // w.block_frames) + 1)] * w.rollouts


def keys_per_rollout(w, frames):
    """Keys of one attention call per rollout: valid cache frames (sinks,
    then at most W window frames) plus the block, Tf tokens each."""
    S, W = w.sink_frames, w.window_frames
    return [(min(n, S) + min(max(n - S, 0), W) + w.block_frames) * w.frame_tokens
            for n in frames]


def workload_config(w, world, rank=0):
    nk = keys_per_rollout(w, prefill_frames(w, rank))
    return {"workload": w.name, "rollouts_per_gpu": w.rollouts, "layers": w.layers,
            "heads": w.heads, "kv_heads": w.hkv, "head_dim": w.head_dim,
            "views": w.views, "grid": f"{w.grid_h}x{w.grid_w}",
            "action_tokens": w.action_tokens, "block_frames": w.block_frames,
            "sink_frames": w.sink_frames, "window_frames": w.window_frames,
            "denoise_steps": w.steps, "keys_per_rollout": nk[0] if len(set(nk)) == 1 else nk,
            "l2": "inputs larger than L2: every step reads all layers' caches and "
                  "fresh q/k/v per (step, layer)",
            "parallelism": f"replicas x{world}"}


# --------------------------------------------------------------------------
# CPU oracle timings (baseline / reference arm)
# --------------------------------------------------------------------------
def oracle_call_setup(w, heads):
    import oracle
    from streaming_autoregressive_video_b200 import synth
    dt = w.dtype
    c = oracle.RolloutCache(w.sink_frames, w.window_frames, w.frame_tokens, w.hkv,
                            w.head_dim, dt)
    ks = (w.block_frames, w.frame_tokens, w.hkv, w.head_dim)
    n_commits = -(-w.slots // w.block_frames) + 1
    for b in range(n_commits):
        c.commit(synth.normal(synth.seed_of(7, b, 0), ks, dt, w.value_scale),
                 synth.normal(synth.seed_of(7, b, 1), ks, dt, w.value_scale))
    q = synth.normal(synth.seed_of(7, 99, 0), (w.queries, w.heads, w.head_dim), dt, w.value_scale)
    k = synth.normal(synth.seed_of(7, 99, 1), (w.block_frames * w.frame_tokens, w.hkv, w.head_dim), dt, w.value_scale)
    v = synth.normal(synth.seed_of(7, 99, 2), (w.block_frames * w.frame_tokens, w.hkv, w.head_dim), dt, w.value_scale)
    nk = (c.valid_slots() + w.block_frames) * w.frame_tokens

    def call():
        oracle.block_attention(c, q, k, v, tokens=w.tokens, grid_w=w.grid_w,
                               theta=w.theta, heads=heads, view_tokens=w.view_tokens)
    return call, 4.0 * len(heads) * w.head_dim * w.queries * nk


def cpu_model():
    """Model name of the host CPU (first entry of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_threads():
    try:
        import threadpoolctl
        return max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


# --------------------------------------------------------------------------
# Replicas (N > 1): the host-side rank logic, tested with gloo on the CPU
# --------------------------------------------------------------------------
def replica_seed_base(rank):
    """Each replica draws its own inputs (same shapes and distributions)."""
    return 1000 * rank


def max_over_ranks(values, world, device="cpu"):
    """Element-wise max over ranks: the job lasts as long as its slowest rank.
    Every rank calls this the same number of times, in the same order."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_rate(work_per_rank, world, ms_max):
    """Whole-job throughput: the work of all ranks over the slowest rank's time
    (per second)."""
    return work_per_rank * world / (ms_max * 1e-3)


def cpu_baseline(w):
    heads = list(range(w.heads))
    call, flops = oracle_call_setup(w, heads)
    t0 = time.perf_counter()
    call()
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle_threads(),
            "kind": "oracle", "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"one full attention call ({w.heads} heads x {w.queries} queries, "
                      f"cache full) in fp64 numpy, {dt:.1f} s"}


def run_reference(args, w, rank):
    if rank != 0:
        return
    heads = [0, 1]
    call, flops = oracle_call_setup(w, heads)
    for _ in range(args.warmup):
        call()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        call()
    dt = (time.perf_counter() - t0) / args.steps
    val = flops / dt / 1e12
    sample = (f"per step: {len(heads)} of {w.heads} heads of one attention call "
              f"({w.queries} queries, cache full), fp64 numpy oracle")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus), "cpu_baseline": {
            "value": val, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(), "sample": sample},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


# --------------------------------------------------------------------------
# CUDA path
# --------------------------------------------------------------------------
class Rollout:
    """One workload on the device: a cache prefilled to steady state (or to
    its ragged fill), and fresh q/k/v per (denoising step, layer)."""

    def __init__(self, w, dev, rank):
        import torch
        from streaming_autoregressive_video_b200 import binding as fd
        from streaming_autoregressive_video_b200 import synth

        self.w, self.dev = w, dev
        L, R, S = w.layers, w.rollouts, w.steps
        F, Tf, H, d = w.block_frames, w.frame_tokens, w.heads, w.head_dim
        self.desc = fd.make_desc(w)
        self.cache_bytes = fd.fd_cache_bytes(self.desc)
        raw = torch.empty(self.cache_bytes + 1024, dtype=torch.uint8, device=dev)
        off = (-raw.data_ptr()) % 1024
        self.cache = fd.fd_cache_create(self.desc, raw[off:off + self.cache_bytes])
        self.esz = 2 if w.dtype == "bf16" else 4
        tdt = torch.int16 if w.dtype == "bf16" else torch.float32

        def gen(seed, shape):
            t = synth.normal_device(seed, shape, w.dtype, dev, w.value_scale)
            return t.view(torch.int16) if w.dtype == "bf16" else t

        self.qshape = (R, w.queries, H, d)
        self.kshape = (R, F * Tf, w.hkv, d)
        base = replica_seed_base(rank)
        self._pk = [gen(synth.seed_of(base, 1, l), self.kshape) for l in range(L)]
        self._pv = [gen(synth.seed_of(base, 2, l), self.kshape) for l in range(L)]
        self.fill = prefill_frames(w, rank)
        self.stream = torch.cuda.current_stream(dev)
        self._prefill()
        torch.cuda.synchronize()
        # the library's own frame counters agree with the described prefill
        assert [fd.fd_cache_frames(self.cache, 0, r) for r in range(R)] == self.fill
        # a ragged workload keeps its prefill keys to restore its fill before
        # every timed block (each block's commit advances every rollout's fill)
        self.ragged = bool(w.ragged_window)
        if not self.ragged:
            del self._pk, self._pv
        self.q = [[gen(synth.seed_of(base, 10, s, l), self.qshape) for l in range(L)]
                  for s in range(S)]
        self.k = [[gen(synth.seed_of(base, 11, s, l), self.kshape) for l in range(L)]
                  for s in range(S)]
        self.v = [[gen(synth.seed_of(base, 12, s, l), self.kshape) for l in range(L)]
                  for s in range(S)]
        self.outs = [torch.empty(self.qshape, dtype=tdt, device=dev) for _ in range(L)]
        self.nk = keys_per_rollout(w, self.fill)
        self.flops_call = attn_flops(w, self.nk)
        self.bytes_call = attn_bytes(w, self.nk, self.esz)
        self.kv_bytes = 2 * w.layers * w.rollouts * w.slots * Tf * w.hkv * d * self.esz
        # one block's commit: read k, v; write K, V and the rotated K
        self.commit_bytes = 5.0 * L * R * F * Tf * w.hkv * d * self.esz

    def _prefill(self):
        from streaming_autoregressive_video_b200 import binding as fd
        w = self.w
        left = list(self.fill)
        while max(left) > 0:
            fr = [min(w.block_frames, x) for x in left]
            fd.fd_cache_commit(self.cache, 0, w.layers, w.rollouts, self._pk, self._pv,
                               frames=fr, stream=self.stream)
            left = [a - b for a, b in zip(left, fr)]

    def restore_fill(self):
        """Back to the described ragged fill (reset every rollout, commit the
        prefill again), so the next block's calls see the same key counts
        as the first; a no-op for steady-state workloads, whose window stays
        full as blocks are committed."""
        from streaming_autoregressive_video_b200 import binding as fd
        if not self.ragged:
            return
        fd.fd_cache_reset(self.cache, list(range(self.w.rollouts)), stream=self.stream)
        self._prefill()

    def _timed(self, fn, evs):
        import torch
        if evs is None:
            fn()
            return
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(self.stream)
        fn()
        b.record(self.stream)
        evs.append((a, b))

    def step(self, evs=None, cevs=None):
        """One block: every denoising step through every layer, then one
        batched commit of the last step's k/v into every layer."""
        from streaming_autoregressive_video_b200 import binding as fd
        w, c = self.w, self.cache
        L, R, S = w.layers, w.rollouts, w.steps
        for s in range(S):
            for l in range(L):
                self._timed(lambda: fd.fd_block_attention(
                    c, l, R, self.q[s][l], self.k[s][l], self.v[s][l], self.outs[l],
                    stream=self.stream), evs)
        self._timed(lambda: fd.fd_cache_commit(c, 0, L, R, self.k[S - 1], self.v[S - 1],
                                               stream=self.stream), cevs)

    def step_side_commits(self, aux, attn_done, commit_done):
        """The same block with finalize() in the background: layer l's commit
        runs on stream `aux` once its last-step attention is done, and the next
        block's first call on layer l waits for it."""
        from streaming_autoregressive_video_b200 import binding as fd
        w, c = self.w, self.cache
        L, R, S = w.layers, w.rollouts, w.steps
        for s in range(S):
            for l in range(L):
                if s == 0:
                    self.stream.wait_event(commit_done[l])
                fd.fd_block_attention(c, l, R, self.q[s][l], self.k[s][l], self.v[s][l],
                                      self.outs[l], stream=self.stream)
                if s == S - 1:
                    attn_done[l].record(self.stream)
                    aux.wait_event(attn_done[l])
                    fd.fd_cache_commit(c, l, l + 1, R, [self.k[s][l]], [self.v[s][l]],
                                       stream=aux)
                    commit_done[l].record(aux)

    def check(self):
        from streaming_autoregressive_video_b200 import binding as fd
        err = fd.fd_get_device_error(self.cache)
        assert err == 0, f"device error word {err:#x}"


def time_steps(ro, steps, warmup, world=1, barrier=None):
    """Device time of `steps` blocks after `warmup` untimed ones: (ms per
    step, mean ms per attention call, mean ms per commit).  A ragged
    workload's fill is restored before every block, and its step time is
    the sum of the blocks' own intervals (the restores are not timed)."""
    import torch
    for _ in range(warmup):
        ro.restore_fill()
        ro.step()
    torch.cuda.synchronize()
    if barrier:
        barrier()
    torch.cuda.synchronize()
    evs, cevs, sevs = [], [], []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(ro.stream)
    for _ in range(steps):
        ro.restore_fill()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(ro.stream)
        ro.step(evs, cevs)
        b.record(ro.stream)
        sevs.append((a, b))
    e1.record(ro.stream)
    torch.cuda.synchronize()
    if barrier:
        barrier()
    ms_step = (sum(a.elapsed_time(b) for a, b in sevs) if ro.ragged
               else e0.elapsed_time(e1)) / steps
    attn_ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    commit_ms = sum(a.elapsed_time(b) for a, b in cevs) / len(cevs)
    return ms_step, attn_ms, commit_ms


def finalize_overlap(ro, steps):
    """Step time with one batched commit after the block (serial) and with
    each layer's commit on a second stream right after its last attention
    call (finalize() in the background)."""
    import torch
    serial = time_steps(ro, steps, 2)[0]
    aux = torch.cuda.Stream(ro.dev)
    L = ro.w.layers
    attn_done = [torch.cuda.Event() for _ in range(L)]
    commit_done = [torch.cuda.Event() for _ in range(L)]
    for e in commit_done:
        e.record(ro.stream)
    for _ in range(2):
        ro.step_side_commits(aux, attn_done, commit_done)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(ro.stream)
    for _ in range(steps):
        ro.step_side_commits(aux, attn_done, commit_done)
    for e in commit_done:
        ro.stream.wait_event(e)
    e1.record(ro.stream)
    torch.cuda.synchronize()
    ro.check()
    return {"ms_per_step_batched_commit": serial,
            "ms_per_step_side_stream_commits": e0.elapsed_time(e1) / steps,
            "steps": steps, "layers": L,
            "how": "per-layer fd_cache_commit on a second stream after the layer's "
                   "last-step attention (event-ordered), against one batched commit "
                   "after the block on the same stream"}


# secondary workloads timed in the default run: name -> (workload key,
# layers, steps); layers > 1 give each call its own cache so the K/V come
# from HBM rather than from L2 (each call has the workload's shape)
OTHER_CONFIGS = {"tiny": ("tiny", 1, 40), "large": ("large", 4, 4),
                 "long": ("long", 8, 10), "ragged": ("ragged", 1, 10),
                 "d64": ("d64", 4, 4), "gqa": ("gqa", 8, 4),
                 "multiview": ("multiview", 2, 2)}


def other_configs(dev, rank):
    """Per-call time, TFLOP/s and roofline fraction of the other workloads,
    each with the clocks seen while it ran."""
    import gc
    import torch
    peaks, src = measured_peaks()
    res = {}
    for name, (key, layers, steps) in OTHER_CONFIGS.items():
        w = workloads()[key]
        if layers != w.layers:
            w = w.scaled(layers=layers, name=f"{w.name}-L{layers}")
        ro = Rollout(w, dev, rank)
        sampler = ClockSampler(dev.index or 0)
        sampler.start()
        ms_step, attn_ms, commit_ms = time_steps(ro, steps, 3)
        clocks = sampler.stop()
        ro.check()
        tf = ro.flops_call / (attn_ms * 1e-3) / 1e12
        gbs = ro.bytes_call / (attn_ms * 1e-3) / 1e9
        entry = {"workload": w.name, "dtype": w.dtype, "steps": steps, "layers": layers,
                 "ms_per_call": attn_ms, "ms_per_step": ms_step, "commit_ms": commit_ms,
                 "tflops_per_call": tf, "hbm_gbs_per_call": gbs,
                 "latent_frames_per_s_per_layer":
                     w.rollouts * w.block_frames * w.layers / (ms_step * 1e-3),
                 "frac_of_burst_bf16": tf / peaks["bf16_tflops"],
                 "frac_of_hbm": gbs / peaks["hbm_gbs"],
                 "commit_frac_of_hbm": ro.commit_bytes / (commit_ms * 1e-3) / 1e9
                                       / peaks["hbm_gbs"],
                 "cache_bytes": ro.cache_bytes, "kv_bytes": ro.kv_bytes,
                 "clocks": clocks}
        if w.dtype != "bf16":
            entry["bound"] = "latency (CUDA-core fp32 kernel, launch-sized work)"
            entry["us_per_call"] = attn_ms * 1e3
        res[name] = entry
        del ro
        gc.collect()
        torch.cuda.empty_cache()
    res["long"]["rollout"] = whole_rollout(workloads()["long"], dev, rank)
    return res


def whole_rollout(w, dev, rank):
    """The one-frame-per-block workload's whole rollout as the workload states
    it (its layers, its blocks: 10,000 blocks through the ring), timed on the
    device from the first block to the last: every block runs its denoising
    steps and commits, so the ring wraps about 1,250 times.  The device
    memory the process holds is compared before and after (the cache and the
    inputs are allocated once)."""
    import torch
    ro = Rollout(w, dev, rank)
    ro.step()
    torch.cuda.synchronize()
    mem0 = torch.cuda.memory_allocated(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(ro.stream)
    for _ in range(w.blocks):
        ro.step()
    e1.record(ro.stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    ro.check()
    out = {"blocks": w.blocks, "layers": w.layers, "steps": w.steps, "ms_total": ms,
           "ms_per_block": ms / w.blocks,
           "tflops": ro.flops_call * w.steps * w.layers * w.blocks / (ms * 1e-3) / 1e12,
           "device_bytes_constant": torch.cuda.memory_allocated(dev) == mem0,
           "note": "one layer: consecutive blocks read the same layer's cache, "
                   "partly from L2"}
    del ro
    torch.cuda.empty_cache()
    return out


def run_fd(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from streaming_autoregressive_video_b200 import binding as fd

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    fd.load(build_if_missing=(rank == 0))
    ro = Rollout(w, dev, rank)
    L, R, S, F = w.layers, w.rollouts, w.steps, w.block_frames

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        ro.restore_fill()
        ro.step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    sampler.start()
    launches0 = fd.fd_launch_count()
    ms_step, attn_ms, commit_ms = time_steps(ro, args.steps, 0, world, barrier)
    launches = fd.fd_launch_count() - launches0
    clocks = sampler.stop()
    ms_step, attn_ms, commit_ms = max_over_ranks([ms_step, attn_ms, commit_ms], world, dev)
    ro.check()

    flops_step = ro.flops_call * S * L
    value = job_rate(flops_step, world, ms_step) / 1e12
    frames_per_s_layer = job_rate(R * F * L, world, ms_step)

    # ---------------- end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, ro.cache, dev, ro.stream, ro.q, ro.k, ro.v, ro.outs,
                      flops_step, world, restore=ro.restore_fill)
    overlap = None
    if not args.no_extra and world == 1 and not ro.ragged:
        overlap = finalize_overlap(ro, 5)

    if rank != 0:
        return
    peaks, src = measured_peaks()
    dtype = "bf16" if w.dtype == "bf16" else "f32"
    line_extra = {}
    if w.dtype == "bf16":
        # the attention kernel runs for a step of tens of ms between host
        # syncs, not for seconds: its fraction is quoted against the burst
        # bf16 figure, and against the sustained one for context
        peak = peaks["bf16_tflops"]
        achieved = ro.flops_call / (attn_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak,
                # the committed ncu capture is of the 480p call
                "traffic": profile_traffic() if w.name == workloads()["480p"].name else None,
                "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peak),
                "kernel": f"attn_bf16_d{w.head_dim}_sm100",
                "peak_source": f"{src} bf16_tflops (burst)",
                "algorithmic_bytes_per_launch": ro.bytes_call,
                "flops_per_launch": ro.flops_call, "launch_ms": attn_ms,
                "launch_covers": "fd_block_attention call: RoPE pass over the block's "
                                 "queries and keys + attention kernel + fold of the "
                                 "split query-tile pairs"}
    else:
        achieved = ro.bytes_call / (attn_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                "kernel": "attn_cuda_core_kernel", "peak_source": f"{src} hbm_gbs",
                "algorithmic_bytes_per_launch": ro.bytes_call, "launch_ms": attn_ms,
                "note": "fp32 CUDA-core kernel on a launch-sized call: latency bound",
                "us_per_call": attn_ms * 1e3}
    # batched commit of all layers: read k, v; write K, V and rotated K
    commit_gbs = ro.commit_bytes / (commit_ms * 1e-3) / 1e9
    commit_roof = {"bound": "hbm", "achieved": commit_gbs, "peak": peaks["hbm_gbs"],
                   "unit": "GB/s", "frac": commit_gbs / peaks["hbm_gbs"],
                   "traffic": commit_traffic() if w.name == workloads()["480p"].name else None,
                   "frac_4stream": 0.8 * commit_gbs / peaks["hbm_gbs"],
                   "kernel": "commit_copy_kernel + commit_meta_kernel",
                   "peak_source": f"{src} hbm_gbs",
                   "algorithmic_bytes_per_launch": ro.commit_bytes,
                   "bytes_counted": "read k, v; write K, V, rotated K (5 element streams); "
                                    "frac_4stream counts only read k, v + write K, V",
                   "launch_ms": commit_ms, "layers_per_launch": L}
    cfg = workload_config(w, world, rank)
    cfg.update(cache_bytes=ro.cache_bytes, kv_bytes=ro.kv_bytes)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype, "data": "synthetic",
        "config": cfg,
        "latent_frames_per_s_per_layer": frames_per_s_layer,
        "roofline": roof,
        "commit_roofline": commit_roof,
        "gpu_launches": launches,
        "clocks": clocks,
        "e2e": e2e,
    }
    line.update(line_extra)
    if overlap is not None:
        line["finalize_overlap"] = overlap
    if world == 1 and not args.no_extra and args.workload == "480p":
        del ro
        line["other_configs"] = other_configs(dev, rank)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)


def run_e2e(args, w, cache, dev, stream, q, k, v, outs, flops_step, world, restore=None):
    """Same steps through the C ABI with the q/k/v of every call copied from
    pinned host memory and every output copied back, inside the timed region.
    Copies run on their own streams so they overlap the kernels.  The host
    buffers hold the first denoising step's q/k/v of every layer and are sent
    again at every step and block: the copies move the bytes of fresh inputs,
    which is what the end-to-end figure measures."""
    import torch
    import torch.distributed as dist
    from streaming_autoregressive_video_b200 import binding as fd

    L, R, S = w.layers, w.rollouts, w.steps
    hq = [t.cpu().pin_memory() for t in q[0]]
    hk = [t.cpu().pin_memory() for t in k[0]]
    hv = [t.cpu().pin_memory() for t in v[0]]
    hout = [torch.empty(outs[0].shape, dtype=outs[0].dtype).pin_memory() for _ in range(L)]
    nbuf = 2
    dq = [torch.empty_like(q[0][0]) for _ in range(nbuf)]
    dk = [torch.empty_like(k[0][0]) for _ in range(nbuf)]
    dv = [torch.empty_like(v[0][0]) for _ in range(nbuf)]
    dout = [torch.empty_like(outs[0]) for _ in range(nbuf)]
    klast = [torch.empty_like(k[0][0]) for _ in range(L)]
    vlast = [torch.empty_like(v[0][0]) for _ in range(L)]
    h2d = torch.cuda.Stream(dev)
    d2h = torch.cuda.Stream(dev)
    ready = [torch.cuda.Event() for _ in range(nbuf)]
    done = [torch.cuda.Event() for _ in range(nbuf)]
    freed = [torch.cuda.Event() for _ in range(nbuf)]
    for e in freed:
        e.record(d2h)
    h2d_bytes = d2h_bytes = 0

    def step():
        nonlocal h2d_bytes, d2h_bytes
        if restore is not None:
            # a ragged workload's fill before every block (timed with it: the
            # end-to-end figure of that workload is slightly pessimistic)
            restore()
        i = 0
        for s in range(S):
            last = s == S - 1
            for l in range(L):
                b = i % nbuf
                kd = klast[l] if last else dk[b]
                vd = vlast[l] if last else dv[b]
                h2d.wait_event(freed[b])
                with torch.cuda.stream(h2d):
                    dq[b].copy_(hq[l], non_blocking=True)
                    kd.copy_(hk[l], non_blocking=True)
                    vd.copy_(hv[l], non_blocking=True)
                ready[b].record(h2d)
                stream.wait_event(ready[b])
                fd.fd_block_attention(cache, l, R, dq[b], kd, vd, dout[b], stream=stream)
                done[b].record(stream)
                d2h.wait_event(done[b])
                with torch.cuda.stream(d2h):
                    hout[l].copy_(dout[b], non_blocking=True)
                freed[b].record(d2h)
                h2d_bytes += sum(t.numel() * t.element_size() for t in (hq[l], hk[l], hv[l]))
                d2h_bytes += hout[l].numel() * hout[l].element_size()
                i += 1
        fd.fd_cache_commit(cache, 0, L, R, klast, vlast, stream=stream)

    for _ in range(max(2, min(3, args.warmup))):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    h2d_bytes = d2h_bytes = 0
    steps = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    fin = torch.cuda.Event()
    fin.record(d2h)
    stream.wait_event(fin)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks([e0.elapsed_time(e1) / steps], world, dev)[0]
    return {"value": job_rate(flops_step, world, ms) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d_bytes // steps, "d2h_bytes_per_step": d2h_bytes // steps,
            "ms_per_step": ms}


def main():
    args = parse_args()
    w = workloads()[args.workload]
    if args.layers:
        w = w.scaled(layers=args.layers, name=w.name + f"-L{args.layers}")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_fd(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
