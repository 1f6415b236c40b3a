"""Benchmark of the Monarch video-attention forward on B200.

One step = one full forward call (every refinement iteration, every kernel)
over one batch of seeded synthetic input.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference]

--impl reference times the fp64 CPU oracle (the only reference that exists
for this method here) on a bounded sample of the same workload.

Multi-GPU: one process per GPU (torchrun); (batch, head) units are
independent, so every rank runs its own full copy of the workload with no
collective on the data path (weak scaling); the timed region is bracketed by
barriers and the max over ranks is reported.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from structured_sparse_attention_grid_b200.workloads import WORKLOADS, make_cotangent, make_inputs  # noqa: E402

METRIC = "Monarch-attn ms/call & effective TFLOP/s, bf16, N=4680–32760; % roofline"
DEFAULT_WORKLOAD = "chunk_4680_bf16"
L2_BYTES = 126 * 2**20
# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of a
# workload's dominant kernel from an ncu capture of the current kernel code,
# scaled to the workload's heads where the capture used fewer (profiles/);
# a kernel without a capture of its current code reports null.
NCU_TRAFFIC = {
    ("chunk_4680_bf16", "r_step"): 48.13e6,     # mean of the call's two launches (30.15 and 66.11 MB)
    ("chunk_4680_bf16", "l_lsecol"): 44.82e6,
    ("chunk_4680_bf16", "l_out"): 76.24e6,
    ("full_32760_bf16", "l_col"): 897.1e6,      # 299.03 MB (mean of two launches) at 8 heads x 3
    ("full_32760_bf16", "l_out"): 1341.4e6,     # 447.13 MB at 8 heads x 3
}
# FP32 FMA ceiling of the CUDA cores: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz
ALU_F32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# Algorithmic work of one call (no recompute counted).
def geometry(w):
    P = (w.H // w.th) * (w.W // w.tw)
    return dict(P=P, b2=w.th * w.tw, b1q=w.T * P, b1k=w.Tkey * P)


def visible_fraction(w):
    """Fraction of (query tile, key tile) pairs inside the frame-chunk causal
    mask (1 without it): the L step only works on those."""
    if not w.chunk_frames or w.chunk_frames >= w.T or w.Tkey != w.T:
        return 1.0
    g = geometry(w)
    cq = w.chunk_frames * g["P"]
    seen = sum(min(g["b1k"], (a1 // cq + 1) * cq) for a1 in range(g["b1q"]))
    return seen / (g["b1q"] * g["b1k"])


def work_model(w):
    g = geometry(w)
    BH = w.B * w.heads
    fv = visible_fraction(w)
    FL = 2.0 * g["b2"] * g["b1q"] * g["b1k"] * w.d * fv  # one L-sized contraction (visible pairs), per head
    FR = 2.0 * g["b1k"] * g["b2"] ** 2 * w.d        # one R-sized contraction, per head
    es = 4 if w.dtype == "f32" else 2
    nq, nk = w.Nq * w.d * es * BH, w.Nk * w.d * es * BH  # bytes of q and of k (= v)
    no = w.Nq * w.d * 4 * BH                                # f32 output
    flops_total = BH * (2 * w.iters * FL + (2 * w.iters + 1) * FR)
    # per-phase algorithmic FLOPs and compulsory bytes of ONE launch
    lse = BH * g["b2"] * g["b1q"] * 4
    hb = BH * g["b2"] * g["b1k"] * 4
    phases = {
        "l_out": dict(flops=BH * 2 * FL, bytes=nq + 2 * nk + hb + no),   # q, k~, z, h -> out
        "l_lse": dict(flops=BH * FL, bytes=nq + nk + hb + lse),          # q, k~, h -> lse
        "l_col": dict(flops=BH * FL, bytes=nq + nk + hb + lse + nk),     # q, k~, h, lse -> q~
        # q~ (or q), k in and k~ out, plus v in and z out in the final
        # launch; h out every launch.  Mean over the call's `iters` launches.
        "r_step": dict(flops=BH * (2 * w.iters + 1) * FR / w.iters,
                       bytes=(3 * (w.iters - 1) * nk + 5 * nk) / w.iters + hb),
        "qbar": dict(flops=0.0, bytes=nq),
        # one refinement step in one kernel: R step (scores, k~, z) and output
        # pass; its compulsory bytes are the call's q, k, v in and out
        "onestep": dict(flops=BH * (3 * FR + 2 * FL), bytes=nq + 2 * nk + no),
        # LSE and column passes in one kernel: q, k~, h in; q~ out
        "l_lsecol": dict(flops=BH * 2 * FL, bytes=nq + nk + hb + nk),
    }
    # compulsory call bytes: Q, K, V in and O out, all in the input dtype
    # (the output is written as f32 by default, which adds nq bytes; the
    # roofline keeps the smaller count)
    return dict(flops=flops_total, io_bytes=2 * nq + 2 * nk, io_bytes_f32_out=nq + 2 * nk + no,
                dense_flops=4.0 * BH * w.Nq * w.Nk * w.d * fv,
                phases=phases, FL=FL, FR=FR, visible_fraction=fv)


def call_roofline(w, model, peaks, ms):
    """Whole-call roofline: the slower of the Monarch FLOPs at the measured
    bf16 tensor peak and the compulsory Q/K/V/O bytes at the measured HBM
    bandwidth; frac = that time / the measured time."""
    t_flop = model["flops"] / (peaks["bf16_tflops"] * 1e12)
    t_hbm = model["io_bytes"] / (peaks["hbm_gbs"] * 1e9)
    roof_ms = 1e3 * max(t_flop, t_hbm)
    return {"roofline_ms": roof_ms, "frac": roof_ms / ms, "bound": "tensor" if t_flop >= t_hbm else "hbm",
            "flop_ms": 1e3 * t_flop, "hbm_ms": 1e3 * t_hbm, "io_bytes": model["io_bytes"],
            "peak_source": peaks["source"]}


def backward_work_model(w):
    """Algorithmic FLOPs of the backward of the one-step forward (gradient
    contractions only, the forward recompute not counted): L step dL, dq, dk~,
    dz (4 F_L); R step dR (2 F_R), dk (2 F_R), dv and dq (2 F_R).  Per kernel,
    the algorithmic work of what it computes (recompute included) and its
    bound: tensor-core kernels against the bf16 tensor peak, CUDA-core ones
    against the FP32 FMA ceiling."""
    m = work_model(w)
    FL, FR, BH = m["FL"], m["FR"], w.B * w.heads
    if w.dtype == "f32":
        phases = {"bwd_prep": (BH * 2 * FL, "alu"), "bwd_dq": (BH * 3 * FL, "alu"), "bwd_dkv": (BH * 4 * FL, "alu"),
                  "bwd_r": (BH * 5 * FR, "alu"), "r_step": (BH * 3 * FR, "alu")}
    else:
        phases = {"bwd_dq": (BH * 3 * FL, "tensor"),        # S, dP, dq
                  "bwd_dkv": (BH * 4 * FL, "tensor"),       # S^T, dP^T, dz, dk~
                  "l_out": (BH * 2 * FL, "tensor"),         # recompute: S, y
                  "r_step": (BH * 3 * FR, "tensor"),        # recompute: scores, k~, z
                  "bwd_r": (BH * 5 * FR, "alu"),            # R-step backward (CUDA cores)
                  "bwd_prep": (0.0, "hbm")}
    return dict(flops=BH * (4 * FL + 6 * FR), phases=phases)


# ---------------------------------------------------------------------------
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons in the background."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None
        self.mark = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        threading.Thread(target=self._read, daemon=True).start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def begin(self):
        self.mark = time.time()

    def end(self):
        self.stop_t = time.time()

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = [r for t, r in self.rows if self.mark and self.mark - 0.15 <= t <= self.stop_t + 0.15]
        if not rows:
            rows = [r for _, r in self.rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(rows[0][2]), "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max((num(r[3]) or 0.0) for r in rows)}


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest value over the ranks (for a time: the slowest rank); the
    value itself on one rank.  device: where the reduction tensor lives (the
    rank's GPU under NCCL, None = host under gloo)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
_INPUT_CACHE = {}


def inputs_of(w):
    """Seeded inputs of a workload; workloads that differ only in name,
    iterations or mask share one draw."""
    key = (w.B, w.heads, w.T, w.H, w.W, w.d, w.dtype, w.seed, w.kind, w.Tk, w.planted)
    if key not in _INPUT_CACHE:
        _INPUT_CACHE.clear()
        _INPUT_CACHE[key] = make_inputs(w)
    return _INPUT_CACHE[key]


def time_forward(m, w, qd, kd, vd, out, steps, warmup, stream, flush, world=1, clocks=None):
    """Per-step device times (ms) of `steps` forward calls after `warmup`
    untimed ones, each bracketed by CUDA events on the launching stream, with
    an L2 flush before every call when `flush` is given.  Returns the list and
    the number of library kernels launched in the timed region."""
    def step():
        m.monarch_attn_fwd(qd, kd, vd, out, w.T, w.H, w.W, w.th, w.tw, w.iters, stream=stream,
                           chunk_frames=w.chunk_frames)

    for _ in range(warmup):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = m.launch_count()
    if clocks:
        clocks.begin()
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    if clocks:
        clocks.end()
    launches = m.launch_count() - launches0
    if world > 1:
        torch.distributed.barrier()
    return [a.elapsed_time(b) for a, b in zip(starts, ends)], launches, step


def keep_loaded(step, timed_ms, device, clocks, at_least_ms=1000.0):
    """If the timed steps were short, keep the same calls running (untimed)
    so that the clock sampler sees the GPU under that load for about a
    second; the sampled window then ends here."""
    if timed_ms < at_least_ms:
        t_end = time.time() + (at_least_ms - timed_ms) / 1e3
        while time.time() < t_end:
            step()
        torch.cuda.synchronize(device)
        clocks.end()


# Every configuration the headline metric covers (N = 4680 to 32760), timed in
# the same run as the headline: the toy, the KV-cache step, the shape sweep, the
# full sequence, and the one-step and chunk-causal training forms (the three
# full-sequence workloads share one input draw, so they run back to back).
EXTRA_WORKLOADS = ["toy_256_f32", "kvcache_4680x32760_bf16", "sweep_2048_f16", "sweep_8192_f16",
                   "sweep_32768_f16", "chunk_4680_bf16_1step", "full_32760_bf16", "full_32760_bf16_1step",
                   "train_32760_bf16_causal"]


def extra_configs(m, args, device, stream, flush_buf, peaks, world, clocks=None):
    """ms per call (median of CUDA-event-timed steps), effective TFLOP/s and
    the whole-call roofline fraction of every other configuration, with dense
    SDPA on the same tensors as context, and the SM clocks sampled while each
    one ran (a 1000 W part settles lower under the long full-sequence calls)."""
    res = {}
    for name in EXTRA_WORKLOADS:
        if name == args.workload:
            continue
        w = WORKLOADS[name]
        model = work_model(w)
        q, k, v = inputs_of(w)
        qd, kd, vd = (t.to(device) for t in (q, k, v))
        out = torch.empty(qd.shape, dtype=torch.float32, device=device)
        flush = flush_buf if model["io_bytes"] < 4 * L2_BYTES else None
        steps = max(5, min(args.steps, 20 if model["flops"] > 5e11 else 50))
        times, _, step = time_forward(m, w, qd, kd, vd, out, steps, args.warmup, stream, flush, world, clocks)
        if clocks:
            keep_loaded(step, sum(times), device, clocks)
        ms = max_over_ranks(statistics.median(times), world, device)
        rec = {"ms_per_call": ms, "mean_ms": statistics.fmean(times), "steps": steps,
               "value": world * model["flops"] / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "monarch_gflop_per_call": model["flops"] / 1e9, "dtype": w.dtype,
               "config": {"B": w.B, "heads": w.heads, "grid": [w.T, w.H, w.W], "kv_frames": w.Tkey,
                          "head_dim": w.d, "tile": [w.th, w.tw], "iters": w.iters,
                          "chunk_frames": w.chunk_frames},
               "call_roofline": call_roofline(w, model, peaks, ms),
               "l2": "flushed between steps" if flush is not None else "inputs larger than L2"}
        if clocks:
            rec["clocks"] = clocks.summary()
        rec["dense_context"] = dense_context(qd, kd, vd, model, flush, stream, ms)
        res[name] = rec
        del qd, kd, vd, out
        torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, device):
    import structured_sparse_attention_grid_b200 as m
    w = WORKLOADS[args.workload]
    model = work_model(w)
    peaks = load_peaks()
    q, k, v = inputs_of(w)
    qd, kd, vd = (t.to(device) for t in (q, k, v))
    out = torch.empty(qd.shape, dtype=torch.float32, device=device)  # the library's default f32 output
    stream = torch.cuda.current_stream(device)
    io_bytes = model["io_bytes"]
    flush_buf = torch.empty(int(2 * L2_BYTES), dtype=torch.uint8, device=device)
    flush_l2 = io_bytes < 4 * L2_BYTES  # inputs smaller than ~4x L2: flush between steps
    flush = flush_buf if flush_l2 else None

    clocks = ClockSampler(torch.cuda.current_device() if device.index is None else device.index)
    clocks.start()
    time.sleep(0.3)
    per_step, launches, step = time_forward(m, w, qd, kd, vd, out, args.steps, args.warmup, stream, flush,
                                            world, clocks)
    ms = statistics.median(per_step)
    keep_loaded(step, sum(per_step), device, clocks)
    head_clocks = clocks.summary()

    ms = max_over_ranks(ms, world, device)
    mean_ms = max_over_ranks(statistics.fmean(per_step), world, device)

    # Per-kernel times: the same step, with CUDA events around every launch.
    m.profile_enable(True)
    m.profile_read(reset=True)
    nprof = max(3, min(args.steps, 20))
    for _ in range(nprof):
        if flush_l2:
            flush_buf.zero_()
        step()
    torch.cuda.synchronize(device)
    prof = m.profile_read(reset=True)
    m.profile_enable(False)
    dom = max((p for p in prof if prof[p][1] > 0), key=lambda p: prof[p][0])
    dom_ms = prof[dom][0] / prof[dom][1]
    ph = model["phases"][dom]
    t_flop = ph["flops"] / (peaks["bf16_tflops"] * 1e12)
    t_hbm = ph["bytes"] / (peaks["hbm_gbs"] * 1e9)
    if t_flop >= t_hbm and w.dtype != "f32":
        roof = {"bound": "tensor", "achieved": ph["flops"] / (dom_ms * 1e-3) / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": ph["bytes"] / (dom_ms * 1e-3) / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = NCU_TRAFFIC.get((w.name, dom))
    roof["traffic_unit"] = "bytes per launch (ncu DRAM read + write)"
    roof["kernel"] = dom
    roof["launch_ms"] = dom_ms
    roof["algorithmic_per_launch"] = ph["bytes"] if roof["bound"] == "hbm" else ph["flops"]
    roof["peak_source"] = peaks["source"]

    dense = dense_context(qd, kd, vd, model, flush, stream, ms)
    backward = backward_line(m, w, qd, kd, vd, flush, stream)

    # End to end (copies inside the timed region): the host-buffer entry point
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty(q.shape, dtype=torch.float32).pin_memory()

    def e2e_call():
        m.monarch_attn_fwd_host(qh, kh, vh, oh, w.T, w.H, w.W, w.th, w.tw, w.iters, stream=stream,
                                chunk_frames=w.chunk_frames)

    for _ in range(2):
        e2e_call()
    e2e_n = max(3, min(args.steps, 10))
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    e2e_times = []
    for _ in range(e2e_n):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_call()
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_times.append(e0.elapsed_time(e1))
    e2e_ms = max_over_ranks(statistics.median(e2e_times), world, device)
    del qh, kh, vh, oh

    # the per-configuration timings are single-GPU figures: one run (N = 1) gives them
    configs = extra_configs(m, args, device, stream, flush_buf, peaks, world, clocks) \
        if (world == 1 and not args.no_configs) else {}
    clocks.stop()

    es = q.element_size()
    rec = {
        "metric": METRIC,
        "value": world * model["flops"] / (ms * 1e-3) / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "ms_per_step_mean": mean_ms,
        "timing": "median of per-step CUDA-event times on the launching stream; max over ranks",
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded; positional + planted-pair structure, see workloads.py)",
        "config": {"workload": w.name, "B": w.B, "heads": w.heads, "grid": [w.T, w.H, w.W],
                   "kv_frames": w.Tkey, "head_dim": w.d, "tile": [w.th, w.tw], "iters": w.iters,
                   "Nq": w.Nq, "Nk": w.Nk, "chunk_frames": w.chunk_frames, "parallelism": f"replicas{world}",
                   "l2": "flushed between steps" if flush_l2 else "inputs larger than L2"},
        "monarch_gflop_per_call": model["flops"] / 1e9,
        "dense_gflop_per_call": model["dense_flops"] / 1e9,
        "call_roofline": call_roofline(w, model, peaks, ms),
        "roofline": roof,
        "kernels": {p: {"ms_per_launch": prof[p][0] / prof[p][1], "launches_per_step": prof[p][1] / nprof}
                    for p in prof if prof[p][1] > 0},
        "e2e": {"value": world * model["flops"] / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_call": e2e_ms,
                "h2d_bytes_per_step": (q.numel() + k.numel() + v.numel()) * es,
                "d2h_bytes_per_step": q.numel() * 4},
        "gpu_launches": launches,
        "clocks": head_clocks,
        "dense_context": dense,
        "backward": backward,
        "configs": configs,
    }
    return rec, (q, k, v, w)


def backward_line(m, w, qd, kd, vd, flush, stream):
    """The backward of the one-step forward (the finetuned regime) on the same
    q, k, v with a seeded cotangent and f32 gradients: ms per call, effective
    TFLOP/s of its algorithmic FLOPs and the roofline of its dominant kernel,
    all from CUDA events on the launching stream."""
    if w.Tkey != w.T:
        return {"impl": "not defined: the backward is for self-attention"}
    bm = backward_work_model(w)
    dy = make_cotangent(w, "f32").to(qd.device)
    dq, dk, dv = (torch.empty_like(dy) for _ in range(3))

    def call():
        m.monarch_attn_bwd(qd, kd, vd, dy, dq, dk, dv, w.T, w.H, w.W, w.th, w.tw, stream=stream,
                           chunk_frames=w.chunk_frames)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    n = 3 if bm["flops"] > 2e11 else 10
    times = []
    for _ in range(n):
        if flush is not None:
            flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    ms = statistics.median(times)
    m.profile_enable(True)
    m.profile_read(reset=True)
    if flush is not None:
        flush.zero_()
    call()
    torch.cuda.synchronize()
    prof = m.profile_read(reset=True)
    m.profile_enable(False)
    kernels = {p: prof[p][0] / prof[p][1] for p in prof if prof[p][1] > 0}
    totals = {p: prof[p][0] for p in prof if prof[p][1] > 0}
    dom = max(totals, key=totals.get)
    flops, bound = bm["phases"][dom]
    achieved = flops / (totals[dom] * 1e-3) / 1e12
    peaks = load_peaks()
    if bound == "tensor":
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                "peak_source": peaks["source"]}
    else:
        roof = {"bound": "alu", "kernel": dom, "achieved": achieved, "peak": ALU_F32_TFLOPS,
                "unit": "TFLOP/s", "frac": achieved / ALU_F32_TFLOPS, "traffic": None,
                "peak_source": "FP32 FMA: 148 SMs x 128 lanes x 2 x 1.965 GHz"}
    saved = None
    if w.dtype != "f32":
        # the training pair: the forward keeps out and the row LSE, the
        # backward takes them instead of recomputing the output pass
        out = torch.empty(qd.shape, dtype=torch.float32, device=qd.device)
        lse = torch.empty(m.lse_numel(w.B, w.heads, w.T, w.H, w.W, w.d, w.th, w.tw), dtype=torch.float32,
                          device=qd.device)
        m.monarch_attn_fwd_train(qd, kd, vd, out, lse, w.T, w.H, w.W, w.th, w.tw, stream=stream,
                                 chunk_frames=w.chunk_frames)

        def call_saved():
            m.monarch_attn_bwd_saved(qd, kd, vd, out, lse, dy, dq, dk, dv, w.T, w.H, w.W, w.th, w.tw,
                                     stream=stream, chunk_frames=w.chunk_frames)

        for _ in range(3):
            call_saved()
        torch.cuda.synchronize()
        st = []
        for _ in range(n):
            if flush is not None:
                flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call_saved()
            b.record(stream)
            torch.cuda.synchronize()
            st.append(a.elapsed_time(b))
        sms = statistics.median(st)
        saved = {"entry": "monarch_attn_bwd_saved (out and row LSE kept by monarch_attn_fwd_train)",
                 "ms_per_call": sms, "value": bm["flops"] / (sms * 1e-3) / 1e12, "unit": "TFLOP/s"}
    return {"workload": w.name, "iters": 1, "grad_dtype": "f32", "ms_per_call": ms,
            "saved_state": saved,
            "value": bm["flops"] / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "gflop_per_call": bm["flops"] / 1e9,
            "kernels_ms": kernels, "launches": {p: prof[p][1] for p in prof if prof[p][1] > 0},
            "roofline": roof}


def dense_context(qd, kd, vd, model, flush, stream, monarch_ms):
    """Context only, not the product: dense softmax attention over the same
    q, k, v with torch's scaled_dot_product_attention (flash / cuDNN kernels),
    i.e. the N x N attention that the Monarch factorisation replaces."""
    import torch.nn.functional as F
    if qd.dtype == torch.float32:
        return {"impl": "not timed for f32 inputs"}
    if model.get("visible_fraction", 1.0) < 1.0:
        return {"impl": "not timed: the frame-chunk mask is not a kernel-native SDPA mask"}
    try:
        F.scaled_dot_product_attention(qd, kd, vd)
        torch.cuda.synchronize()
        n = 3 if model["dense_flops"] > 2e12 else 10
        times = []
        for _ in range(n):
            if flush is not None:
                flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            F.scaled_dot_product_attention(qd, kd, vd)
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms = sorted(times)[len(times) // 2]
        return {"impl": "torch.nn.functional.scaled_dot_product_attention (backend chosen by torch)",
                "ms_per_call": ms, "tflops": model["dense_flops"] / (ms * 1e-3) / 1e12,
                "dense_over_monarch_time": ms / monarch_ms}
    except Exception as e:  # context only: never fail the bench line over it
        return {"impl": "unavailable", "error": str(e)[:200]}


def cpu_baseline(w, q, k, v, budget_s: float):
    """Times the fp64 oracle on the host on whole (batch, head) units until
    about budget_s seconds of CPU work; returns the record and the throughput
    in the metric's unit."""
    from oracle import monarch as om
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        blas = 1
    g = om.Grid(w.T, w.H, w.W, w.th, w.tw, Tk=w.Tkey if w.Tk else None)
    model = work_model(w)
    per_head = model["flops"] / (w.B * w.heads)
    done, t0 = 0, time.perf_counter()
    units = [(b, h) for b in range(w.B) for h in range(w.heads)]
    while True:
        b, h = units[done % len(units)]
        qn, kn, vn = (t[b:b + 1, h:h + 1].double().numpy() for t in (q, k, v))
        om.monarch_attention(qn, kn, vn, g, w.iters)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or done >= len(units):
            break
    value = done * per_head / el / 1e12
    return {"value": value, "unit": "TFLOP/s", "cores": blas, "host_cpus": os.cpu_count(),
            "kind": "oracle", "sample": f"{done} of {len(units)} (batch, head) units of {w.name}, "
                                        f"{el:.1f} s fp64 numpy"}, el / done


def run_reference(args, rank, world):
    """The oracle, as it stands, on the host cores: a bounded sample of the
    workload per step (whole (batch, head) units)."""
    w = WORKLOADS[args.workload]
    q, k, v = make_inputs(w)
    from oracle import monarch as om
    g = om.Grid(w.T, w.H, w.W, w.th, w.tw, Tk=w.Tkey if w.Tk else None)
    model = work_model(w)
    per_head = model["flops"] / (w.B * w.heads)
    units = [(b, h) for b in range(w.B) for h in range(w.heads)]
    # size the per-step sample so warm-up + steps stay within ~2 minutes
    t0 = time.perf_counter()
    qn, kn, vn = (t[0:1, 0:1].double().numpy() for t in (q, k, v))
    om.monarch_attention(qn, kn, vn, g, w.iters)
    t_unit = time.perf_counter() - t0
    per_step = max(1, min(len(units), int(120.0 / max(1e-3, t_unit) / max(1, args.steps + args.warmup))))
    times = []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        for j in range(per_step):
            b, h = units[(s * per_step + j) % len(units)]
            qn, kn, vn = (t[b:b + 1, h:h + 1].double().numpy() for t in (q, k, v))
            om.monarch_attention(qn, kn, vn, g, w.iters)
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = per_step * per_head / sec / 1e12
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        blas = 1
    sample = f"{per_step} of {len(units)} (batch, head) units of {w.name} per step, fp64 numpy"
    return {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
        "config": {"workload": w.name, "B": w.B, "heads": w.heads, "grid": [w.T, w.H, w.W],
                   "kv_frames": w.Tkey, "head_dim": w.d, "tile": [w.th, w.tw], "iters": w.iters,
                   "parallelism": "host"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "kind": "oracle", "cores": blas, "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def profile_calls(args):
    """A bare run of the workload for profiler captures: no timing, no bench
    line.  --profile-pass bwd runs the backward (f32 gradients) instead."""
    import structured_sparse_attention_grid_b200 as m
    w = WORKLOADS[args.workload]
    q, k, v = (t.cuda() for t in make_inputs(w))
    if args.profile_pass == "bwd":
        dy = make_cotangent(w, "f32").cuda()
        dq, dk, dv = (torch.empty_like(dy) for _ in range(3))
        for _ in range(args.profile_calls):
            m.monarch_attn_bwd(q, k, v, dy, dq, dk, dv, w.T, w.H, w.W, w.th, w.tw, chunk_frames=w.chunk_frames)
    else:
        out = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        for _ in range(args.profile_calls):
            m.monarch_attn_fwd(q, k, v, out, w.T, w.H, w.W, w.th, w.tw, w.iters, chunk_frames=w.chunk_frames)
    torch.cuda.synchronize()
    err = m.device_error()
    print(f"profile case {w.name} ({args.profile_pass}) B={w.B} heads={w.heads} calls={args.profile_calls} "
          f"device_error={err}")
    if err:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-configs", action="store_true",
                    help="time only --workload (skip the per-configuration timings of the other workloads)")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiler cases)")
    ap.add_argument("--heads", type=int, default=0, help="override the workload's head count (profiler cases)")
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="run this many forward calls of the workload and exit (for ncu); no timing")
    ap.add_argument("--profile-pass", default="fwd", choices=["fwd", "bwd"],
                    help="which pass --profile-calls runs")
    args = ap.parse_args()
    if args.batch or args.heads:
        import dataclasses
        base = WORKLOADS[args.workload]
        WORKLOADS[args.workload] = dataclasses.replace(base, B=args.batch or base.B, heads=args.heads or base.heads)
    if args.profile_calls:
        return profile_calls(args)
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    rec, (q, k, v, w) = run_ours(args, rank, world, device)
    if rank == 0:
        if world == 1:
            cb, _ = cpu_baseline(w, q, k, v, args.cpu_budget)
            rec["cpu_baseline"] = cb
        print(json.dumps(rec), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
