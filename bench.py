"""Benchmark of the VSA forward pass on B200 (one JSON line on rank 0).

Workload: 61,440 tokens (grid 16x48x80, 960 cubes), B=1, 12 heads, D=128,
top-K = 32, seeded synthetic cube-correlated bf16 inputs (trainable_block_sparse_cube_b200.synth,
workload "long61k_k32"). One step = one full forward pass (gather + pool,
coarse attention + selection, fine attention + gated combine).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the fp64 CPU oracle, rank 0 only)

Metric: sparse TFLOP/s of the forward pass, counting executed FLOPs only:
fine 4*64*(64*n_i)*D per query cube (QK^T and PV), coarse 4*C^2*D per head.
ms_per_step is the device time of one call (the metric's ms/call).
Multi-GPU runs are independent replicas (every (batch, head) is independent;
there is no exchange step), so scaling is weak and value sums all ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from trainable_block_sparse_cube_b200 import replicas, synth  # noqa: E402

METRIC = "VSA fwd ms/call & sparse TFLOP/s (% bf16 TC peak) at 61,440 tokens, K=32"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
FINE_SOURCES = ["fine.cu", "sm100_ptx.cuh", "vsa_common.cuh"]
PROFILE = os.path.join(ROOT, "profiles", "fine_attention_long61k_k32.md")


def flops(wl, counts=None):
    D, C, BH = wl.D, wl.C, wl.B * wl.heads
    n_sum = BH * C * wl.topk if counts is None else int(np.asarray(counts, dtype=np.int64).sum())
    fine = 4.0 * 64 * 64 * D * n_sum
    coarse = 4.0 * C * C * D * BH
    return fine, coarse


def workload_desc(wl):
    sel = f"top-K={wl.topk}" if wl.topk > 0 else f"top-p={wl.top_p} clamp [{wl.kmin},{wl.kmax}]"
    return (f"{wl.name}: B={wl.B}, heads={wl.heads}, D={wl.D}, T x H x W = {wl.T}x{wl.H}x{wl.W} "
            f"({wl.N} tokens, {wl.C} cubes), {sel}, generator {wl.gen} seed {wl.seed}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def fine_traffic():
    """dram bytes per launch of the fine kernel from the committed ncu summary,
    if it was taken on the current kernel source; else None."""
    if not os.path.exists(PROFILE):
        return None
    h = hashlib.sha256()
    for f in FINE_SOURCES:
        h.update(open(os.path.join(ROOT, "trainable_block_sparse_cube_b200", "csrc", f), "rb").read())
    sha = h.hexdigest()
    vals = {}
    for line in open(PROFILE):
        if ":" in line and line.strip().startswith(("traffic_bytes_per_launch", "kernel_source_sha256")):
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256") == sha and "traffic_bytes_per_launch" in vals:
        return float(vals["traffic_bytes_per_launch"])
    return None


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        # raw samples go to VSA_BENCH_LOG_DIR (default: the temp directory)
        log_dir = os.environ.get("VSA_BENCH_LOG_DIR") or tempfile.gettempdir()
        os.makedirs(log_dir, exist_ok=True)
        self.path = os.path.join(log_dir, f"clocks_gpu{self.gpu}.csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

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
                rows.append(dict(sm=float(parts[1]), max=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hw_thermal=parts[6], sw_thermal=parts[7], sw_power=parts[8]))
            except ValueError:
                continue
        if not rows:
            return None
        loaded = [r for r in rows if r["power"] > 250.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                              ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded), "sm_max_mhz": max(r["max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r["power"] for r in rows)}


def oracle_sample(wl, seconds, q=None, k=None, v=None, gc=None, gf=None, first_cube=0):
    """Times the fp64 oracle on a bounded sample of the workload: the coarse
    stage of head 0 and the fine stage of as many query cubes as fit in
    `seconds` (chunks of 16). Returns (flops, elapsed_s, description)."""
    import oracle  # test infrastructure; used here only for the CPU baseline

    if q is None:
        q, k, v, gc, gf = synth.head_inputs(wl, 0, 0)
    qd, kd, vd = (x.double().numpy() for x in (q, k, v))
    t0 = time.perf_counter()
    perm = oracle.cube_perm(wl.T, wl.H, wl.W)
    pooled = [oracle.pool_cubes(x, perm) for x in (qd, kd, vd)]
    s, P, Oc = oracle.coarse_attention(*pooled)
    if wl.topk > 0:
        lists = oracle.select_topk(s, wl.topk)
        counts = np.full(wl.C, wl.topk)
    else:
        lists, counts = oracle.select_topp(s, P, wl.top_p, wl.kmin, wl.kmax)
    f = 4.0 * wl.C * wl.C * wl.D
    done = 0
    c = first_cube
    while time.perf_counter() - t0 < seconds and done < wl.C:
        cubes = [(c + j) % wl.C for j in range(16)]
        Of = oracle.fine_attention(qd, kd, vd, perm, lists, counts, cubes)
        oracle.gated_combine(Oc, Of, gc.double().numpy(), gf.double().numpy(), perm)
        f += sum(4.0 * 64 * 64 * wl.D * counts[x] for x in cubes)
        done += 16
        c += 16
    el = time.perf_counter() - t0
    return f, el, f"head 0: coarse stage of all {wl.C} cubes + fine stage and combine of {done} query cubes"


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads") for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(n[0])
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    q, k, v, gc, gf = synth.head_inputs(wl, 0, 0)
    per_step = max(0.5, min(8.0, 120.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        oracle_sample(wl, per_step, q, k, v, gc, gf, first_cube=16 * i)
    tot_f = tot_t = 0.0
    desc = ""
    for i in range(args.steps):
        f, t, desc = oracle_sample(wl, per_step, q, k, v, gc, gf, first_cube=16 * (i + args.warmup))
        tot_f += f
        tot_t += t
    val = tot_f / tot_t / 1e12
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_desc(wl)},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"per step: {desc} (fp64 numpy, {per_step:.1f} s budget)"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="long61k_k32", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = synth.WORKLOADS[args.workload]
    if args.heads:
        wl = wl.with_(heads=args.heads)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, wl, rank, world)

    from trainable_block_sparse_cube_b200 import vsa

    torch.cuda.set_device(local)
    rep = replicas.from_env("nccl")
    barrier = rep.barrier

    q, k, v, gc, gf = synth.make_inputs(wl)
    dq, dk, dv, dgc, dgf = (t.cuda() for t in (q, k, v, gc, gf))
    plan = vsa.Plan(wl.B, wl.heads, wl.T, wl.H, wl.W, wl.D, wl.topk, wl.top_p, wl.kmin, wl.kmax)
    out = torch.empty_like(dq)
    idx = torch.empty((wl.B, wl.heads, wl.C, wl.kcap), dtype=torch.int32, device=dq.device)
    cnt = torch.empty((wl.B, wl.heads, wl.C), dtype=torch.int32, device=dq.device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dq.device)   # > L2 (126 MB)
    stream = torch.cuda.current_stream()
    plan.set_stage_timing(True)

    for _ in range(args.warmup):
        plan.run(dq, dk, dv, dgc, dgf, out, idx, cnt)
    plan.check()
    counts = cnt.cpu().numpy()
    f_fine, f_coarse = flops(wl, counts)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    for _ in range(20):  # keep the GPU busy while the sampler starts
        plan.run(dq, dk, dv, dgc, dgf, out, idx, cnt)
    barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    stage = np.zeros(3)
    for i in range(args.steps):
        flush.zero_()                       # L2 flush, outside the timed interval
        ev[i][0].record(stream)
        plan.run(dq, dk, dv, dgc, dgf, out, idx, cnt)
        ev[i][1].record(stream)
        stage += np.array(plan.stage_times()) if (i % 10 == 0 or i == args.steps - 1) else 0
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    # stage split: re-time a subset of steps (stage_times syncs, so sampled steps only)
    n_stage = len(range(0, args.steps, 10)) + (0 if (args.steps - 1) % 10 == 0 else 1)
    stage_ms = stage / n_stage
    plan.check()
    t_max = rep.max_over_ranks(float(sum(step_ms)))
    ms_per_step = t_max / args.steps
    value = rep.job_throughput((f_fine + f_coarse) * args.steps, t_max * 1e-3) / 1e12

    # e2e through the C ABI's host-buffer entry point (vsa_run_host): pinned host
    # inputs -> device, forward, output + index lists -> host, all timed; the
    # library pipelines the copies per (batch, head) slice against the compute.
    hq, hk, hv, hgc, hgf = (t.pin_memory() for t in (q, k, v, gc, gf))
    hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    hidx = torch.empty(idx.shape, dtype=idx.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hgc, hgf))
    d2h = hout.numel() * hout.element_size() + hidx.numel() * hidx.element_size()
    e2e_ms = []
    for i in range(args.e2e_steps + 2 if args.e2e_steps > 0 else 0):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        plan.run_host(hq, hk, hv, hgc, hgf, hout, hidx)
        b.record(stream)
        b.synchronize()
        if i >= 2:
            e2e_ms.append(a.elapsed_time(b))
    e2e_t = rep.max_over_ranks(sum(e2e_ms) if e2e_ms else float("nan"))
    e2e_val = rep.job_throughput((f_fine + f_coarse) * len(e2e_ms), e2e_t * 1e-3) / 1e12 if e2e_ms else None
    plan.check()

    peaks, peak_src = load_peaks()
    fine_ms = float(stage_ms[2])
    achieved = f_fine / (fine_ms * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    BH, N, D, C = wl.B * wl.heads, wl.N, wl.D, wl.C
    gather_bytes = 2.0 * 3 * BH * N * D * 2 + 3.0 * BH * C * D * 4
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(wl), "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "inputs (566 MB) larger than L2; 256 MB L2 flush write between timed steps",
                   "flops_per_step": {"fine": f_fine, "coarse": f_coarse}},
        "roofline": {"bound": "tensor", "kernel": "fine_attention_kernel<128>", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "traffic": fine_traffic(),
                     "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                     "frac_of_datasheet_2250": achieved / 2250.0},
        "stages_ms": {"gather_pool": float(stage_ms[0]), "coarse": float(stage_ms[1]), "fine": fine_ms},
        "gather_pool_gbs": gather_bytes / (stage_ms[0] * 1e-3) / 1e9,
        "gather_pool_frac_hbm": gather_bytes / (stage_ms[0] * 1e-3) / 1e9 / hbm,
        "coarse_share": float(stage_ms[1]) / float(stage_ms.sum()),
        # coarse stage: its FLOPs (two C x C x D products per head) and the bytes it
        # must move (three-term means in, scores and three-term P written and read
        # back, lists, coarse output), over its event-timed duration
        "coarse_tflops": f_coarse / (stage_ms[1] * 1e-3) / 1e12,
        "coarse_gbs": (9.0 * BH * C * D * 2 + 2.0 * BH * C * C * 4 + 2.0 * 3 * BH * C * ((C + 7) // 8 * 8) * 2
                       + BH * C * wl.kcap * 4 + BH * C * D * 4) / (stage_ms[1] * 1e-3) / 1e9,
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_t / len(e2e_ms) if e2e_ms else None},
        "gpu_launches": vsa.load().vsa_kernels_per_run() * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, el, desc = oracle_sample(wl, args.cpu_seconds, q[0, 0], k[0, 0], v[0, 0], gc[0, 0], gf[0, 0])
        line["cpu_baseline"] = {"value": f / el / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"{desc}; {el:.1f} s fp64 numpy"}
    if rep.is_reporter:
        print(json.dumps(line), flush=True)
    rep.close()


if __name__ == "__main__":
    main()
