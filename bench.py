#!/usr/bin/env python
"""Benchmark of the B200 MSDeformAttn core: queries/s and achieved HBM GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

One step = one pass of the whole hot path over one batch: the forward
(msda_forward) and the training backward (msda_backward) of the encoder
training workload -- B=4, M=8, D=32, K=4, L=4, levels (100,150),(50,75),
(25,38),(13,19), S = Lq = 19947, float32 -- on seeded synthetic inputs.  The
unit is a query (one (b, q) pair), so a step processes B*Lq = 79,788 queries.

Timing: inputs are resident in HBM; L2 (126 MB) is flushed by a 256 MiB write
before every step, outside the timed events; each step is bracketed by CUDA
events on the launching stream; W untimed warm-up steps come first.  With
N > 1 (torchrun, one process per GPU) every rank runs the same workload on its
own GPU -- the operator has no exchange step, so ranks are replicas ("weak"
scaling) -- and the step time is the max over ranks.

Printed (rank 0, one JSON line): the contract keys, plus
  roofline       the dominant launch: algorithmic bytes / its mean event time,
                 against the measured HBM copy bandwidth of this machine's B200s;
  forward_encoder the encoder self-attention forward (B=2, S=Lq=19947), timed
                 alone the same way, with its own roofline;
  e2e            the same metric through the public API with host buffers: the
                 H2D copy of every input and the D2H copy of every result are
                 inside the timed region; consecutive steps are pipelined over
                 upload / compute / download streams;
  cpu_baseline   the float64 CPU oracle on a bounded sample (rank 0, N=1);
  clocks         SM clocks and throttle reasons sampled during the timed region.

``--impl reference`` times the float64 oracle instead (the deliberately slow
reference arm; rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import threading
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from scale_deformable_attention_backward_b200 import workloads as W  # noqa: E402

STEP_WORKLOAD = "encoder_train_fp32"
FORWARD_WORKLOAD = "encoder_fp32"
METRIC = "MSDeformAttn fwd/bwd queries/sec and achieved HBM GB/s vs B200 peak (1 GPU)"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
# msda_backward without a workspace (the timed path): zero grad_value, backward.
BACKWARD_LAUNCHES = 2
KERNEL_SOURCES = os.path.join(ROOT, "scale_deformable_attention_backward_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


# ---------------------------------------------------------------------------
# algorithmic bytes (compulsory HBM traffic) per launch
# ---------------------------------------------------------------------------

def algorithmic_bytes(cfg: W.Config, inp: W.Inputs) -> dict:
    """Compulsory bytes: every input read once and every output written once."""
    B, S, M, D = inp.value.shape
    _, Lq, _, L, K, _ = inp.sampling_locations.shape
    vbytes = 2 if cfg.dtype == "bf16" else 4
    value = B * S * M * D * vbytes
    loc = B * Lq * M * L * K * 2 * 4
    attn = B * Lq * M * L * K * 4
    out = B * Lq * M * D * vbytes
    fwd = value + loc + attn + out
    # backward reads value, loc, attn, grad_output; writes grad_value, grad_loc, grad_attn
    bwd = value + loc + attn + B * Lq * M * D * 4 + B * S * M * D * 4 + loc + attn
    return {"forward": fwd, "backward": bwd}


def grad_value_adds(inp: W.Inputs) -> int:
    """Float adds the backward's grad_value scatter performs: D per corner inside
    the map, i.e. one vector atomic per lane and corner (host count from the
    inputs, float64 pixel mapping)."""
    B, S, M, D = inp.value.shape
    ss = inp.spatial_shapes.astype(np.float64)
    loc = inp.sampling_locations.astype(np.float64)            # [B,Lq,M,L,K,2]
    W_ = ss[:, 1][None, None, None, :, None]
    H_ = ss[:, 0][None, None, None, :, None]
    x0 = np.floor(loc[..., 0] * W_ - 0.5)
    y0 = np.floor(loc[..., 1] * H_ - 0.5)
    vx = (x0 >= 0) & (x0 <= W_ - 1)
    vx1 = (x0 + 1 >= 0) & (x0 + 1 <= W_ - 1)
    vy = (y0 >= 0) & (y0 <= H_ - 1)
    vy1 = (y0 + 1 >= 0) & (y0 + 1 <= H_ - 1)
    corners = (vx & vy).sum() + (vx1 & vy).sum() + (vx & vy1).sum() + (vx1 & vy1).sum()
    return int(corners) * D


def source_digest(files) -> str:
    """Digest of the kernel sources a recorded measurement depends on."""
    h = hashlib.sha256()
    for name in sorted(files):
        with open(os.path.join(KERNEL_SOURCES, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(key: str):
    """ncu DRAM bytes per launch recorded in profiles/traffic.json for `key`, or
    None when there is no record or the kernel's sources changed since."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f).get(key)
        if not rec or rec.get("source_digest") != source_digest(rec["files"]):
            return None
    except (OSError, ValueError, KeyError):
        return None
    return rec.get("dram_bytes_per_launch")


FALLBACK_BF16_TFLOPS = 1590.0


def measured_bf16_peak():
    """Dense bf16 GEMM burst peak in TF/s: MEASURED_PEAKS.json's, else the pool's
    earlier measurement (fallback)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, ValueError, KeyError):
        return FALLBACK_BF16_TFLOPS, "fallback"


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "25"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            # Wait (up to 10 s) for the first sample, taken before the timed
            # region and not counted, so that the sampler is running when the
            # region starts.
            first = threading.Thread(target=self.proc.stdout.readline, daemon=True)
            first.start()
            first.join(timeout=10.0)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, v in enumerate(flags)
                          if v.lower() == "active"})
        top = max(r[0] for r in rows)
        loaded = [r[0] for r in rows if r[0] >= 0.5 * top] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# the CPU oracle on a bounded sample (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(cfg: W.Config, target_s: float = 12.0, per_step_target_s=None):
    """Time the float64 oracle (single thread, as it stands) on the first n
    queries of every image of ``cfg``, forward + backward, with n grown until the
    timed call takes about ``target_s``.  Returns (queries/s, description)."""
    import oracle  # test infrastructure: used here only for the CPU baseline
    inp = W.make_inputs(cfg, seed=0, with_grad=True)
    orc = oracle.default()
    n = 64
    while True:
        sub = W.select_queries(inp, np.arange(n))
        t0 = time.perf_counter()
        orc.forward(sub.value, sub.spatial_shapes, sub.level_start_index,
                    sub.sampling_locations, sub.attention_weights)
        orc.backward(sub.value, sub.spatial_shapes, sub.level_start_index,
                     sub.sampling_locations, sub.attention_weights, sub.grad_output)
        dt = time.perf_counter() - t0
        target = per_step_target_s if per_step_target_s is not None else target_s
        if dt >= 0.5 * target or n >= cfg.queries:
            break
        n = min(cfg.queries, max(2 * n, int(n * 0.8 * target / max(dt, 1e-3))))
    queries = cfg.B * n
    desc = (f"{cfg.name}: forward + backward of the first {n} of {cfg.queries} queries of "
            f"each of the B={cfg.B} images (value over all {cfg.S} tokens), float64 oracle, "
            f"single thread, {dt:.2f} s")
    return queries / dt, desc, dt


def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def host_cpu() -> dict:
    """CPU model and core counts of the host (from /proc/cpuinfo)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "logical_cpus": os.cpu_count(), "usable_cpus": host_threads()}


def oracle_threaded(cfg: W.Config, n: int, threads: int):
    """The same sample as oracle_sample (the first n queries of every image),
    forward + backward, split into `threads` runs of consecutive queries that
    call the float64 oracle at once from `threads` host threads (the oracle's
    plain loops, unchanged; the foreign calls release the GIL).  Each run keeps
    its own grad_value, and the runs' grad_values are added at the end.
    Returns (queries/s, description)."""
    inp = W.select_queries(W.make_inputs(cfg, seed=0, with_grad=True), np.arange(n))
    step, parts = threaded_oracle_step(inp, threads)
    t0 = time.perf_counter()
    step()
    dt = time.perf_counter() - t0
    desc = (f"{cfg.name}: the same {n} queries of each of the B={cfg.B} images, in "
            f"{parts} runs (one image, a range of its queries) on {threads} host threads "
            f"(private grad_value per run, added per image), float64 oracle, {dt:.2f} s")
    return cfg.B * n / dt, desc


def threaded_oracle_step(inp, threads: int):
    """A callable that runs the float64 oracle's forward + backward on `inp` from
    `threads` host threads: the work is cut into runs of (one image, a range of its
    queries), each run keeps its own grad_value of its image, and the runs'
    grad_values are added per image at the end.  The oracle's C loops are
    unchanged; its foreign calls release the GIL.  Returns (step, number of runs)."""
    import dataclasses
    import oracle  # test infrastructure: used here only for the CPU baseline
    from concurrent.futures import ThreadPoolExecutor
    orc = oracle.default()
    B = inp.value.shape[0]
    n = inp.sampling_locations.shape[1]
    per_image = max(1, -(-threads // B))
    bounds = np.linspace(0, n, per_image + 1).astype(int)
    runs = []
    for b in range(B):
        img = dataclasses.replace(
            inp, value=inp.value[b:b + 1], sampling_locations=inp.sampling_locations[b:b + 1],
            attention_weights=inp.attention_weights[b:b + 1],
            grad_output=inp.grad_output[b:b + 1])
        for lo, hi in zip(bounds[:-1], bounds[1:]):
            if hi > lo:
                runs.append((b, W.select_queries(img, np.arange(lo, hi))))

    def run(item):
        b, sub = item
        orc.forward(sub.value, sub.spatial_shapes, sub.level_start_index,
                    sub.sampling_locations, sub.attention_weights)
        gv, _, _ = orc.backward(sub.value, sub.spatial_shapes, sub.level_start_index,
                                sub.sampling_locations, sub.attention_weights,
                                sub.grad_output)
        return b, gv

    def step():
        with ThreadPoolExecutor(max_workers=threads) as pool:
            total = {}
            for b, gv in pool.map(run, runs):
                if b in total:
                    total[b] += gv
                else:
                    total[b] = gv
        return total

    return step, len(runs)


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, units_per_rank: int, steps: int, total_ms_max: float) -> float:
    """Whole-job units/s of `world` independent replicas (weak scaling): every rank
    processes `units_per_rank` per step, and the job takes the slowest rank's time."""
    return world * units_per_rank * steps / (total_ms_max / 1e3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# the B200 arm
# ---------------------------------------------------------------------------

def _device_inputs(inp, device):
    import torch

    def bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)

    d = {
        "value": (bf16(inp.value_bf16_bits) if inp.value_bf16_bits is not None
                  else torch.from_numpy(inp.value).to(device)),
        "spatial_shapes": torch.from_numpy(inp.spatial_shapes).to(device),
        "level_start_index": torch.from_numpy(inp.level_start_index).to(device),
        "sampling_locations": torch.from_numpy(inp.sampling_locations).to(device),
        "attention_weights": torch.from_numpy(inp.attention_weights).to(device),
    }
    if inp.grad_output_bf16_bits is not None:
        d["grad_output"] = bf16(inp.grad_output_bf16_bits)
    elif inp.grad_output is not None:
        d["grad_output"] = torch.from_numpy(inp.grad_output).to(device)
    return d


def run_b200(args, world, rank, local):
    import torch
    from scale_deformable_attention_backward_b200 import binding

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    cfg = W.CONFIGS[STEP_WORKLOAD]
    inp = W.make_inputs(cfg, seed=0)
    d = _device_inputs(inp, device)
    B, S, M, D = inp.value.shape
    _, Lq, _, L, K, _ = inp.sampling_locations.shape
    out = torch.empty((B, Lq, M * D), dtype=torch.float32, device=device)
    gv = torch.empty_like(d["value"])
    gl = torch.empty_like(d["sampling_locations"])
    ga = torch.empty_like(d["attention_weights"])
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    ws = torch.empty(binding.workspace_size(B, S, M, D, Lq, L, K), dtype=torch.uint8,
                     device=device)

    def step():
        binding.forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                        d["sampling_locations"], d["attention_weights"], output=out)

    def step_bwd(workspace=None):
        binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                         d["sampling_locations"], d["attention_weights"], d["grad_output"],
                         grad_value=gv, grad_sampling_locations=gl, grad_attention_weights=ga,
                         workspace=workspace)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
        step_bwd()
    torch.cuda.synchronize()

    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e2 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.fill_(float(i))
            e0[i].record(stream)
            step()
            e1[i].record(stream)
            step_bwd()
            e2[i].record(stream)
        torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    barrier(world)
    fwd_ms = [a.elapsed_time(b) for a, b in zip(e0, e1)]
    bwd_ms = [a.elapsed_time(b) for a, b in zip(e1, e2)]
    total_ms = sum(f + b for f, b in zip(fwd_ms, bwd_ms))
    total_ms_max = max_over_ranks(total_ms, world, device)
    ms_per_step = total_ms_max / args.steps
    queries = B * Lq
    value = replica_throughput(world, queries, args.steps, total_ms_max)
    step_median_ms = max_over_ranks(statistics.median(f + b for f, b in zip(fwd_ms, bwd_ms)),
                                    world, device)
    # Warm: steps back to back with no L2 flush between them (context only; the
    # flushed figure above is the metric).
    warm_n = max(3, min(args.steps, 50))
    ws0, ws1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step()
    step_bwd()
    ws0.record(stream)
    for _ in range(warm_n):
        step()
        step_bwd()
    ws1.record(stream)
    torch.cuda.synchronize()
    step_warm_ms = max_over_ranks(ws0.elapsed_time(ws1) / warm_n, world, device)

    peak, peak_kind = measured_peak()
    algo = algorithmic_bytes(cfg, inp)
    f_ms, b_ms = statistics.mean(fwd_ms), statistics.mean(bwd_ms)
    dom, dom_ms = ("backward", b_ms) if b_ms >= f_ms else ("forward", f_ms)
    achieved = algo[dom] / (dom_ms * 1e-3) / 1e9
    roofline = {
        "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
        "frac": round(achieved / peak, 4), "traffic": recorded_traffic(f"{STEP_WORKLOAD}.{dom}"),
        "kernel": ("msda_backward without workspace: zero_kernel + backward_kernel"
                   if dom == "backward" else "msda_forward: forward_kernel"),
        "algorithmic_bytes": algo[dom], "mean_ms": round(dom_ms, 4),
        "peak_source": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                       if peak_kind == "measured" else "fallback 6.65 TB/s",
        "other": {
            "forward": {"mean_ms": round(f_ms, 4), "algorithmic_bytes": algo["forward"],
                        "achieved_gbs": round(algo["forward"] / (f_ms * 1e-3) / 1e9, 1),
                        "frac": round(algo["forward"] / (f_ms * 1e-3) / 1e9 / peak, 4),
                        "traffic": recorded_traffic(f"{STEP_WORKLOAD}.forward")},
            "backward": {"mean_ms": round(b_ms, 4), "algorithmic_bytes": algo["backward"],
                         "achieved_gbs": round(algo["backward"] / (b_ms * 1e-3) / 1e9, 1),
                         "frac": round(algo["backward"] / (b_ms * 1e-3) / 1e9 / peak, 4),
                         "traffic": recorded_traffic(f"{STEP_WORKLOAD}.backward")},
        },
    }

    # The backward's real ceiling: L2 float atomics (a probe on this pool measured
    # about 1.5e12 float adds/s for 16-byte vector reductions).
    adds = grad_value_adds(inp)
    roofline["other"]["backward"]["atomic_adds"] = adds
    roofline["other"]["backward"]["atomic_adds_per_s"] = round(adds / (b_ms * 1e-3), 1)
    roofline["other"]["backward"]["atomic_note"] = (
        "bound by L2 float atomics; a throughput probe on this pool measured about 1.5e12 "
        "float adds/s for 16-byte vector reductions")

    # The cell-sorted backward (with a workspace), timed alone for reference.
    for _ in range(args.warmup):
        flush.fill_(1.0)
        step_bwd(ws)
    se0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    se1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(float(i))
        se0[i].record(stream)
        step_bwd(ws)
        se1[i].record(stream)
    torch.cuda.synchronize()
    sorted_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(se0, se1))
    roofline["other"]["backward_sorted"] = {
        "mean_ms": round(sorted_ms, 4),
        "achieved_gbs": round(algo["backward"] / (sorted_ms * 1e-3) / 1e9, 1),
        "note": "cell-sorted path (msda_backward with a workspace), not the timed step"}

    # The op fused with the step before it (softmax of the logits, locations from
    # reference points and offsets), one training step on the same workload, against
    # that step written with torch ops around msda_forward / msda_backward.
    fz = W.make_fused_inputs(cfg, seed=0)
    fzd = {k: torch.from_numpy(getattr(fz, k)).to(device) for k in
           ("value", "spatial_shapes", "level_start_index", "reference_points",
            "sampling_offsets", "attention_logits", "grad_output")}
    norm = fzd["spatial_shapes"].flip(-1).to(torch.float32)[None, None, None, :, None, :]

    def fused_step():
        binding.fused_forward(fzd["value"], fzd["spatial_shapes"], fzd["level_start_index"],
                              fzd["reference_points"], fzd["sampling_offsets"],
                              fzd["attention_logits"], output=out)
        binding.fused_backward(fzd["value"], fzd["spatial_shapes"], fzd["level_start_index"],
                               fzd["reference_points"], fzd["sampling_offsets"],
                               fzd["attention_logits"], fzd["grad_output"],
                               reference_grad=False)

    def unfused_step():
        A = torch.softmax(fzd["attention_logits"], -1)
        loc = fzd["reference_points"][:, :, None, :, None, :] + fzd["sampling_offsets"] / norm
        Av = A.view(B, Lq, M, L, K)
        binding.forward(fzd["value"], fzd["spatial_shapes"], fzd["level_start_index"], loc, Av,
                        output=out)
        _, g_loc, g_a = binding.backward(fzd["value"], fzd["spatial_shapes"],
                                         fzd["level_start_index"], loc, Av, fzd["grad_output"])
        g_off = g_loc / norm
        g_a = g_a.view(B, Lq, M, L * K)
        g_z = A * (g_a - (A * g_a).sum(-1, keepdim=True))
        return g_off, g_z

    def time_steps(fn, n):
        for _ in range(args.warmup):
            flush.fill_(1.0)
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        torch.cuda.synchronize()
        for i in range(n):
            flush.fill_(float(i))
            ev[i][0].record(stream)
            fn()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ev)

    n_fused = max(3, min(args.steps, 50))
    fused_ms = max_over_ranks(time_steps(fused_step, n_fused), world, device)
    unfused_ms = max_over_ranks(time_steps(unfused_step, n_fused), world, device)
    fused = {
        "workload": cfg.description + "; inputs are reference points, offsets (pixels) and "
                                      "softmax logits",
        "step": "msda_fused_forward + msda_fused_backward (reference points detached)",
        "ms_per_step": round(fused_ms, 4),
        "queries_per_s": round(world * queries / (fused_ms * 1e-3), 1),
        "unfused_ms_per_step": round(unfused_ms, 4),
        "unfused": "torch softmax and offset normaliser, msda_forward + msda_backward, "
                   "torch chain rule (offset scaling, softmax Jacobian)",
        "steps": n_fused,
    }

    # The deterministic backward (exact integer accumulation of grad_value) on the
    # step's workload, with its workspace allocated once.
    dws = torch.empty(binding.deterministic_workspace_size(B, S, M, D, Lq, L, K),
                      dtype=torch.uint8, device=device)

    def det_bwd():
        binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                         d["sampling_locations"], d["attention_weights"], d["grad_output"],
                         grad_value=gv, grad_sampling_locations=gl, grad_attention_weights=ga,
                         workspace=dws, deterministic=True)

    det_ms = max_over_ranks(time_steps(det_bwd, n_fused), world, device)
    roofline["other"]["backward_deterministic"] = {
        "mean_ms": round(det_ms, 4),
        "achieved_gbs": round(algo["backward"] / (det_ms * 1e-3) / 1e9, 1),
        "note": "msda_backward_deterministic (bit-identical grad_value), not the timed step"}

    # The output projection after the op (Linear 256 -> 256 on the tensor cores,
    # tcgen05 kind::tf32) on the step's forward output.
    prng = np.random.default_rng(1)
    pw = torch.from_numpy((prng.standard_normal((M * D, M * D)) /
                           np.sqrt(M * D)).astype(np.float32)).to(device)
    pb = torch.from_numpy(prng.standard_normal(M * D).astype(np.float32)).to(device)
    px = out.reshape(-1, M * D)
    py = torch.empty_like(px)

    def proj_step():
        binding.output_projection(px, pw, pb, out=py)

    proj_ms = max_over_ranks(time_steps(proj_step, n_fused), world, device)

    def proj_f32_step():
        binding.output_projection(px, pw, pb, out=py, precise=True)

    proj_f32_ms = max_over_ranks(time_steps(proj_f32_step, n_fused), world, device)
    proj_rows = B * Lq
    proj_bytes = proj_rows * M * D * 4 * 2 + M * D * M * D * 4 + M * D * 4
    proj_flops = 2.0 * proj_rows * (M * D) * (M * D)
    bf16_peak, bf16_source = measured_bf16_peak()
    tf32_peak = bf16_peak * 1.1 / 2.25
    proj_gbs = proj_bytes / (proj_ms * 1e-3) / 1e9
    projection = {
        "workload": f"output_proj Linear {M * D}->{M * D} on the step's forward output "
                    f"({proj_rows} rows)",
        "kernel": "proj_kernel: TMA loads/stores, tcgen05.mma kind::tf32, accumulators in tensor memory",
        "mean_ms": round(proj_ms, 4),
        "roofline": {"bound": "hbm", "achieved": round(proj_gbs, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(proj_gbs / peak, 4),
                     "algorithmic_bytes": proj_bytes},
        "tensor": {"achieved_tflops": round(proj_flops / (proj_ms * 1e-3) / 1e12, 1),
                   "tf32_peak_tflops": round(tf32_peak, 1),
                   "peak_source": f"{bf16_source} bf16 burst x nominal tf32/bf16 ratio "
                                  f"1.1/2.25"},
        "precise": {"kernel": "proj_kernel<true>: float32 accuracy from 3 x TF32 MMAs, operands "
                              "split into TF32 heads and float32 remainders in shared memory",
                    "mean_ms": round(proj_f32_ms, 4),
                    "achieved_gbs": round(proj_bytes / (proj_f32_ms * 1e-3) / 1e9, 1),
                    "achieved_tflops_3x": round(3 * proj_flops / (proj_f32_ms * 1e-3) / 1e12, 1)},
    }

    # The bfloat16 training step (value and grad_output bf16; float32 arithmetic and
    # gradients) on the bf16 encoder geometry.
    bcfg = W.CONFIGS["encoder_train_bf16"]
    binp = W.make_inputs(bcfg, seed=0)
    bd = _device_inputs(binp, device)
    bout = torch.empty((bcfg.B, bcfg.queries, bcfg.M * bcfg.D), dtype=torch.bfloat16,
                       device=device)
    bgv = torch.empty(binp.value.shape, dtype=torch.float32, device=device)
    bgl = torch.empty_like(bd["sampling_locations"])
    bga = torch.empty_like(bd["attention_weights"])

    def bf16_step():
        binding.forward(bd["value"], bd["spatial_shapes"], bd["level_start_index"],
                        bd["sampling_locations"], bd["attention_weights"], output=bout)
        binding.backward(bd["value"], bd["spatial_shapes"], bd["level_start_index"],
                         bd["sampling_locations"], bd["attention_weights"], bd["grad_output"],
                         grad_value=bgv, grad_sampling_locations=bgl, grad_attention_weights=bga)

    bf16_ms = max_over_ranks(time_steps(bf16_step, n_fused), world, device)

    # The same bf16 step through the fused op (raw reference points, offsets and
    # logits; bf16 value and grad_output).
    bfz = W.make_fused_inputs(bcfg, seed=0)
    bfd = {k: torch.from_numpy(getattr(bfz, k)).to(device) for k in
           ("spatial_shapes", "level_start_index", "reference_points", "sampling_offsets",
            "attention_logits")}
    bfd["value"] = bd["value"]
    bfd["grad_output"] = bd["grad_output"]

    def bf16_fused_step():
        binding.fused_forward(bfd["value"], bfd["spatial_shapes"], bfd["level_start_index"],
                              bfd["reference_points"], bfd["sampling_offsets"],
                              bfd["attention_logits"], output=bout)
        binding.fused_backward(bfd["value"], bfd["spatial_shapes"], bfd["level_start_index"],
                               bfd["reference_points"], bfd["sampling_offsets"],
                               bfd["attention_logits"], bfd["grad_output"],
                               reference_grad=False)

    bf16_fused_ms = max_over_ranks(time_steps(bf16_fused_step, n_fused), world, device)
    bq = bcfg.B * bcfg.queries
    bf16_train = {
        "workload": bcfg.description, "step": "msda_forward + msda_backward, bf16 value and "
                                              "grad_output",
        "ms_per_step": round(bf16_ms, 4),
        "queries_per_s": round(world * bq / (bf16_ms * 1e-3), 1),
        "fused_ms_per_step": round(bf16_fused_ms, 4),
        "fused_step": "msda_fused_forward + msda_fused_backward on the same workload's raw "
                      "reference points, offsets and logits (reference points detached)",
        "steps": n_fused,
    }

    # The decoder cross-attention workloads (a few hundred queries over the
    # encoder's whole value): forward of decoder_fp32, backward of
    # decoder_box_train_fp32.  Their compulsory bytes count the whole value
    # tensor, which the gathers touch only in part (latency / random-access bound).
    decoder = {}
    for dname, passes in (("decoder_fp32", ("forward",)),
                          ("decoder_box_train_fp32", ("forward", "backward"))):
        dcfg = W.CONFIGS[dname]
        dinp = W.make_inputs(dcfg, seed=0, with_grad=True)
        dd = _device_inputs(dinp, device)
        dout = torch.empty((dcfg.B, dcfg.queries, dcfg.M * dcfg.D), dtype=torch.float32,
                           device=device)
        dgv = torch.empty(dinp.value.shape, dtype=torch.float32, device=device)
        dgl = torch.empty_like(dd["sampling_locations"])
        dga = torch.empty_like(dd["attention_weights"])
        dalgo = algorithmic_bytes(dcfg, dinp)
        entry = {"workload": dcfg.description}
        for pas in passes:
            if pas == "forward":
                fn = lambda: binding.forward(dd["value"], dd["spatial_shapes"],
                                             dd["level_start_index"], dd["sampling_locations"],
                                             dd["attention_weights"], output=dout)
            else:
                fn = lambda: binding.backward(dd["value"], dd["spatial_shapes"],
                                              dd["level_start_index"],
                                              dd["sampling_locations"],
                                              dd["attention_weights"], dd["grad_output"],
                                              grad_value=dgv, grad_sampling_locations=dgl,
                                              grad_attention_weights=dga)
            t_ms = max_over_ranks(time_steps(fn, n_fused), world, device)
            gbs = dalgo[pas] / (t_ms * 1e-3) / 1e9
            entry[pas] = {"mean_us": round(t_ms * 1e3, 2),
                          "queries_per_s": round(world * dcfg.B * dcfg.queries / (t_ms * 1e-3), 1),
                          "achieved_gbs_whole_value": round(gbs, 1),
                          "frac_whole_value": round(gbs / peak, 4)}
        entry["note"] = ("bytes count the whole value tensor (and for the backward the "
                         "whole grad_value, zeroed in the call); the gathers read only "
                         "the lines their points touch, as random 128-byte lines")
        decoder[dname] = entry

    # The encoder self-attention forward alone (B=2), the spec workload.
    fcfg = W.CONFIGS[FORWARD_WORKLOAD]
    finp = W.make_inputs(fcfg, seed=0)
    fd = _device_inputs(finp, device)
    fout = torch.empty((fcfg.B, fcfg.queries, fcfg.M * fcfg.D), dtype=torch.float32,
                       device=device)

    def fstep():
        binding.forward(fd["value"], fd["spatial_shapes"], fd["level_start_index"],
                        fd["sampling_locations"], fd["attention_weights"], output=fout)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        fstep()
    fe0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    fe1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(float(i))
        fe0[i].record(stream)
        fstep()
        fe1[i].record(stream)
    torch.cuda.synchronize()
    fms_all = [a.elapsed_time(b) for a, b in zip(fe0, fe1)]
    fms = max_over_ranks(statistics.mean(fms_all), world, device)
    fms_median = max_over_ranks(statistics.median(fms_all), world, device)
    # Warm: the same launches back to back with no flush between them, so the
    # inputs are partly L2-resident (the cold figures above are the contract's).
    warm_n = max(3, min(args.steps, 50))
    we0, we1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fstep()
    we0.record(stream)
    for _ in range(warm_n):
        fstep()
    we1.record(stream)
    torch.cuda.synchronize()
    fms_warm = max_over_ranks(we0.elapsed_time(we1) / warm_n, world, device)
    fbytes = algorithmic_bytes(fcfg, finp)["forward"]
    fach = fbytes / (fms * 1e-3) / 1e9
    forward_encoder = {
        "workload": fcfg.description, "queries": fcfg.B * fcfg.queries,
        "ms": round(fms, 4), "queries_per_s": round(fcfg.B * fcfg.queries / (fms * 1e-3), 1),
        "median_ms": round(fms_median, 4),
        "warm_ms": round(fms_warm, 4),
        "warm_note": "back-to-back launches with no L2 flush between them (inputs partly "
                     "L2-resident); ms is the L2-flushed figure",
        "roofline": {"bound": "hbm", "achieved": round(fach, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(fach / peak, 4),
                     "traffic": recorded_traffic(f"{FORWARD_WORKLOAD}.forward"),
                     "algorithmic_bytes": fbytes},
    }

    # End to end through the public API with host buffers.  Every step uploads
    # its inputs from pinned host memory, runs forward + backward and downloads
    # the output and the three gradients.  Steps are independent, so they are
    # pipelined over three streams (upload, compute, download) with two device
    # buffer sets: step i's upload overlaps step i-1's compute and step i-2's
    # download.  PCIe carries host->device and device->host at once.
    pin = {k: torch.from_numpy(getattr(inp, k)).pin_memory() for k in
           ("value", "sampling_locations", "attention_weights", "grad_output")}
    pin["spatial_shapes"] = torch.from_numpy(inp.spatial_shapes).pin_memory()
    pin["level_start_index"] = torch.from_numpy(inp.level_start_index).pin_memory()
    n_buf = 2
    dev_in = [{k: torch.empty(t.shape, dtype=t.dtype, device=device) for k, t in pin.items()}
              for _ in range(n_buf)]
    out_shapes = (("out", out), ("gv", gv), ("gl", gl), ("ga", ga))
    dev_out = [{k: torch.empty(t.shape, dtype=t.dtype, device=device) for k, t in out_shapes}
               for _ in range(n_buf)]
    host_out = [{k: torch.empty(t.shape, dtype=t.dtype).pin_memory() for k, t in out_shapes}
                for _ in range(n_buf)]
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
    s_up, s_run, s_down = (torch.cuda.Stream(device) for _ in range(3))
    ev_up = [torch.cuda.Event() for _ in range(n_buf)]
    ev_run = [torch.cuda.Event() for _ in range(n_buf)]
    ev_down = [torch.cuda.Event() for _ in range(n_buf)]
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step(i):
        b = i % n_buf
        di, do, ho = dev_in[b], dev_out[b], host_out[b]
        with torch.cuda.stream(s_up):
            if i >= n_buf:
                s_up.wait_event(ev_run[b])      # step i - 2 no longer reads di
            for k, t in pin.items():
                di[k].copy_(t, non_blocking=True)
            ev_up[b].record(s_up)
        with torch.cuda.stream(s_run):
            s_run.wait_event(ev_up[b])
            if i >= n_buf:
                s_run.wait_event(ev_down[b])    # step i - 2's results have left do
            binding.forward(di["value"], di["spatial_shapes"], di["level_start_index"],
                            di["sampling_locations"], di["attention_weights"],
                            output=do["out"])
            binding.backward(di["value"], di["spatial_shapes"], di["level_start_index"],
                             di["sampling_locations"], di["attention_weights"],
                             di["grad_output"], grad_value=do["gv"],
                             grad_sampling_locations=do["gl"], grad_attention_weights=do["ga"])
            ev_run[b].record(s_run)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev_run[b])
            for k in ho:
                ho[k].copy_(do[k], non_blocking=True)
            ev_down[b].record(s_down)

    for i in range(2 * n_buf):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    ee0 = torch.cuda.Event(enable_timing=True)
    ee1 = torch.cuda.Event(enable_timing=True)
    ee0.record(s_up)
    for i in range(e2e_steps):
        e2e_step(i)
    # The last download is ordered after every earlier upload, launch and download.
    ee1.record(s_down)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ee0.elapsed_time(ee1), world, device) / e2e_steps
    barrier(world)
    # The pipeline returns what one plain call on the device-resident inputs
    # returns (the output, grad_sampling_locations and grad_attention_weights do
    # not depend on the order of atomics, so they must match bit for bit).
    ref_out = binding.forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                              d["sampling_locations"], d["attention_weights"])
    _, ref_gl, ref_ga = binding.backward(d["value"], d["spatial_shapes"],
                                         d["level_start_index"], d["sampling_locations"],
                                         d["attention_weights"], d["grad_output"])
    last = host_out[(e2e_steps - 1) % n_buf]
    if not (torch.equal(last["out"], ref_out.cpu()) and torch.equal(last["gl"], ref_gl.cpu())
            and torch.equal(last["ga"], ref_ga.cpu())):
        raise RuntimeError("end-to-end pipeline results differ from a plain call's")
    del ref_out, ref_gl, ref_ga
    # The link's floor for these bytes: the same uploads and downloads alone, on
    # two streams at once (no kernels).
    def link_copies():
        with torch.cuda.stream(s_up):
            for k, t in pin.items():
                dev_in[0][k].copy_(t, non_blocking=True)
        with torch.cuda.stream(s_down):
            for k in host_out[0]:
                host_out[0][k].copy_(dev_out[0][k], non_blocking=True)

    link_copies()
    torch.cuda.synchronize()
    le0, le1, le2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    link_reps = 5
    le0.record(s_up)
    s_down.wait_event(le0)
    for _ in range(link_reps):
        link_copies()
    le1.record(s_up)
    le2.record(s_down)
    torch.cuda.synchronize()
    link_ms = max(le0.elapsed_time(le1), le0.elapsed_time(le2)) / link_reps
    link_ms = max_over_ranks(link_ms, world, device)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded numpy; no dataset)",
        "config": {"workload": cfg.description, "step": "msda_forward + msda_backward",
                   "queries_per_step_per_gpu": queries, "parallelism": f"replicas x{world}",
                   "l2": "flushed before every step by a 256 MiB write (outside the timed events)",
                   "timing": "CUDA events per step on the launching stream, max over ranks"},
        "roofline": roofline,
        "step_timing": {"mean_ms": round(ms_per_step, 4), "median_ms": round(step_median_ms, 4),
                        "warm_ms": round(step_warm_ms, 4),
                        "warm_note": "steps back to back with no L2 flush between them"},
        "forward_encoder": forward_encoder,
        "fused": fused,
        "bf16_train": bf16_train,
        "decoder": decoder,
        "projection": projection,
        "e2e": {"value": round(world * queries / (e2e_ms * 1e-3), 1), "unit": "queries/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h),
                "pipeline": "upload / compute / download on three streams, two buffer sets",
                "link_floor_ms": round(link_ms, 3),
                "frac_of_link_floor": round(link_ms / e2e_ms, 4),
                "link_note": "link_floor_ms: the same uploads and downloads alone, concurrently "
                             "on two streams, no kernels (host link, both directions at once)",
                "api": "the Python binding of the C ABI (msda_forward, msda_backward) with torch "
                       "tensors as memory; host buffers are pinned torch CPU tensors"},
        "gpu_launches": (1 + BACKWARD_LAUNCHES) * args.steps,
        "clocks": clocks.summary(),
        "wall_s_timed_region": round(wall, 3),
        "cpu_baseline": None,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        qps, desc, dt = oracle_sample(cfg)
        n = int(round(qps * dt / cfg.B))
        threads = host_threads()
        mt_qps, mt_desc = oracle_threaded(cfg, n, threads)
        result["cpu_baseline"] = {"value": round(qps, 2), "unit": "queries/s", "cores": 1,
                                  "kind": "oracle", "sample": desc, "host": host_cpu(),
                                  "threaded": {"value": round(mt_qps, 2), "unit": "queries/s",
                                               "cores": threads, "sample": mt_desc}}
    return result


CASES = ("step", "forward", "forward_encoder", "backward", "backward_sorted", "fused_forward",
         "fused_backward", "projection", "projection_f32", "decoder_forward", "decoder_backward")


def case_workload(case: str) -> str:
    """The workload a single-launch case (--case) runs on."""
    if case == "forward_encoder":
        return FORWARD_WORKLOAD
    if case == "decoder_forward":
        return "decoder_fp32"
    if case == "decoder_backward":
        return "decoder_box_train_fp32"
    return STEP_WORKLOAD


def run_case(args, local):
    """One launch type alone (for profiler captures): W + K launches with an L2
    flush before each, and a one-line JSON with the mean event time."""
    import torch
    from scale_deformable_attention_backward_b200 import binding

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = W.CONFIGS[case_workload(args.case)]
    if args.case.startswith("fused"):
        fz = W.make_fused_inputs(cfg, seed=0)
        d = {k: torch.from_numpy(getattr(fz, k)).to(device) for k in
             ("value", "spatial_shapes", "level_start_index", "reference_points",
              "sampling_offsets", "attention_logits", "grad_output")}
    else:
        inp = W.make_inputs(cfg, seed=0,
                            with_grad=args.case.startswith("backward") or
                            args.case == "decoder_backward")
        d = _device_inputs(inp, device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    if args.case.startswith("projection"):
        # output_proj on the op's output, with the weights the full bench uses.
        px = binding.forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                             d["sampling_locations"], d["attention_weights"])
        C = px.shape[-1]
        px = px.reshape(-1, C)
        prng = np.random.default_rng(1)
        pw = torch.from_numpy((prng.standard_normal((C, C)) / np.sqrt(C)).astype(
            np.float32)).to(device)
        pb = torch.from_numpy(prng.standard_normal(C).astype(np.float32)).to(device)
        py = torch.empty_like(px)
    fused_args = ("value", "spatial_shapes", "level_start_index", "reference_points",
                  "sampling_offsets", "attention_logits")

    def launch():
        if args.case == "projection":
            binding.output_projection(px, pw, pb, out=py)
        elif args.case == "projection_f32":
            binding.output_projection(px, pw, pb, out=py, precise=True)
        elif args.case == "fused_forward":
            binding.fused_forward(*[d[k] for k in fused_args])
        elif args.case == "fused_backward":
            binding.fused_backward(*[d[k] for k in fused_args], d["grad_output"],
                                   reference_grad=False)
        elif args.case.startswith("backward") or args.case == "decoder_backward":
            binding.backward(d["value"], d["spatial_shapes"], d["level_start_index"],
                             d["sampling_locations"], d["attention_weights"], d["grad_output"],
                             workspace="auto" if args.case == "backward_sorted" else None)
        else:
            binding.forward(d["value"], d["spatial_shapes"], d["level_start_index"],
                            d["sampling_locations"], d["attention_weights"])

    times = []
    for i in range(args.warmup + args.steps):
        flush.fill_(float(i))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        launch()
        b.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(a.elapsed_time(b))
    return {"case": args.case, "workload": cfg.description,
            "ms": round(statistics.mean(times), 4), "launches": args.warmup + args.steps}


def run_reference(args):
    """The reference arm: the float64 oracle as it stands, on all the host's cores
    (threaded_oracle_step).  Each step is the whole workload when the run fits the
    time budget, else the first n queries of every image."""
    cfg = W.CONFIGS[STEP_WORKLOAD]
    budget = 150.0
    threads = host_threads()
    per_step = max(0.5, min(10.0, budget / max(1, args.steps + args.warmup)))
    # Calibrate on a sample: single-thread rate times the threads is the estimate.
    qps1, _, _ = oracle_sample(cfg, target_s=2.0)
    n = min(cfg.queries, max(64, int(qps1 * threads * 0.7 * per_step / cfg.B)))
    inp = W.select_queries(W.make_inputs(cfg, seed=0, with_grad=True), np.arange(n))
    step, _ = threaded_oracle_step(inp, threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    total = time.perf_counter() - t0
    ms = total / args.steps * 1e3
    value = cfg.B * n / (ms * 1e-3)
    what = ("the whole workload" if n == cfg.queries else
            f"the first {n} of {cfg.queries} queries of each of the B={cfg.B} images")
    sample = (f"{cfg.name}: forward + backward of {what} per step, float64 oracle on {threads} "
              f"host threads (runs of one image and a range of its queries, private grad_value "
              f"per run)")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "queries/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded numpy; no dataset)",
        "config": {"workload": cfg.description, "step": "oracle forward + backward",
                   "queries_per_step": cfg.B * n, "whole_workload": n == cfg.queries},
        "cpu_baseline": {"value": round(value, 3), "unit": "queries/s", "cores": threads,
                         "kind": "oracle", "sample": sample, "host": host_cpu()},
        "e2e": {"value": round(value, 3), "unit": "queries/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["b200", "reference"], default="b200")
    p.add_argument("--no-cpu-baseline", action="store_true",
                   help="skip the CPU oracle timing (it takes ~10-20 s)")
    p.add_argument("--case", choices=list(CASES),
                   default="step",
                   help="time one launch type alone (for profiler captures) instead of "
                        "the full benchmark")
    args = p.parse_args(argv)
    if args.warmup < 3:
        p.error("--warmup must be at least 3")
    if args.steps < 1:
        p.error("--steps must be at least 1")
    return args


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = dist_env()
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    if args.case != "step":
        print(json.dumps(run_case(args, local)), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        result = run_b200(args, world, rank, local)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
