"""Throughput of the ButterflyMoE expert-layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config headline]
                    [--impl ours|reference]

A step is one pass of the whole layer (top-k routing, bucketing, gather,
input butterflies, the ternary contraction, output butterflies, gate-weighted
combine) over one batch of T synthetic tokens resident in HBM.  The metric is
routed tokens per second (T / step time, summed over ranks); the layer
roofline fraction is t_roof / t_step with t_roof = max(2 T k d^2 / peak
tensor, B_min / peak HBM), B_min = x + y + d^2/4 + 2 N (d/2) log2 d * 4 +
T N * 4 bytes.

Timing: W warm-up steps, then K steps replayed from a CUDA graph, bracketed
by a barrier and a device synchronise, timed with CUDA events on the
launching stream; the max over ranks is reported.  Inputs rotate over
enough batches (x, logits, y) to exceed the 126 MB L2, so every step reads
its activations from HBM.  With N > 1 (torchrun) every rank runs an
independent replica on its own tokens: the layer has no exchange step.

--impl reference times the fp64 CPU oracle (the only other implementation)
on the host cores over a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from ternary_moe_butterfly_b200 import workloads as wl  # noqa: E402

L2_BYTES = 126 * 2**20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def kernel_sources_hash() -> str:
    import glob
    import hashlib
    src = sorted(glob.glob(os.path.join(ROOT, "ternary_moe_butterfly_b200", "csrc", "*")))
    return hashlib.sha256(b"".join(open(f, "rb").read() for f in src)).hexdigest()[:16]


def profiled_traffic(workload: str) -> dict:
    """DRAM bytes per launch from profiles/traffic.txt, if it was captured on
    the current kernel sources and this workload (else empty)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return {}
    meta, vals = {}, {}
    for line in open(p):
        parts = line.split()
        if len(parts) == 3 and parts[0] == "#":
            meta[parts[1]] = parts[2]
        elif len(parts) == 2 and not line.startswith("#"):
            vals[parts[0]] = int(parts[1])
    if meta.get("source_hash") != kernel_sources_hash() or meta.get("workload") != workload:
        return {}
    return vals


def layer_model(w: wl.Workload):
    d, N, k, T, L = w.d, w.N, w.k, w.T, w.L
    xb = 2 if w.dtype == "bf16" else 4
    flops = 2.0 * T * k * d * d
    bmin = T * d * xb * 2 + d * d / 4 + 2 * N * (d // 2) * L * 4 + T * N * 4
    return flops, bmin


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), ws, int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(x: float, device=None) -> float:
    """The largest of the ranks' values (every rank takes part); x itself
    without an initialised process group of more than one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(w: wl.Workload, rank: int) -> int:
    """Each rank routes its own tokens (weak scaling: replicas of the layer,
    disjoint synthetic token shards)."""
    return w.seed + 1000 * rank


def job_tokens_per_s(world: int, T: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank's T tokens per step over the slowest
    rank's step time."""
    return world * T / (ms_per_step * 1e-3)


# ----------------------------------------------------------------- reference

def cpu_oracle_rate(w: wl.Workload, target_s: float, inp=None, max_tokens=None, nthreads: int = 0):
    """tokens/s of the fp64 oracle on the host cores over a bounded sample
    (nthreads OpenMP threads; 0: all the runtime offers)."""
    import oracle
    inp = inp or wl.make_inputs(w.name, T=min(w.T, 64))
    threads = nthreads if nthreads > 0 else oracle.max_threads()
    n = min(16, inp.x.shape[0])
    t0 = time.perf_counter()
    oracle.forward(inp.x[:n], inp.logits[:n], w.k, inp.w_base, inp.alpha, inp.theta, inp.phi, nthreads=threads)
    per_tok = max((time.perf_counter() - t0) / n, 1e-6)
    n2 = int(max(n, min(1 << 20 if max_tokens is None else max_tokens, target_s / per_tok)))
    reps = max(1, int(math.ceil(n2 / inp.x.shape[0])))
    xs = np.concatenate([inp.x] * reps)[:n2]
    ls = np.concatenate([inp.logits] * reps)[:n2]
    t0 = time.perf_counter()
    oracle.forward(xs, ls, w.k, inp.w_base, inp.alpha, inp.theta, inp.phi, nthreads=threads)
    dt = time.perf_counter() - t0
    return n2 / dt, threads, n2, dt


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    inp = wl.make_inputs(w.name, T=min(w.T, 256))
    per_step = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_oracle_rate(w, min(per_step, 2.0), inp)
    rates = []
    for _ in range(args.steps):
        r, threads, n, dt = cpu_oracle_rate(w, per_step, inp)
        rates.append((r, n, dt))
    value = statistics.median(r for r, _, _ in rates)
    n = rates[0][1]
    line = {
        "impl": "reference", "metric": "ButterflyMoE layer routed tokens/s (d=%d,N=%d,top-%d)" % (w.d, w.N, w.k),
        "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * w.T / value, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "d": w.d, "N": w.N, "k": w.k, "T": w.T, "x": w.dtype},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n} tokens of the {w.name} workload per step (fp64 C oracle, OpenMP)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- ours

def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import ternary_moe_butterfly_b200 as bf
    from ternary_moe_butterfly_b200 import build as bfbuild

    rank, world, local = dist_env()
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    if rank == 0:
        bfbuild.build()
    if world > 1:
        dist.barrier()
    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.Stream(device)
    peaks = load_peaks()

    inp = wl.make_inputs(w.name, seed=rank_seed(w, rank))
    d, N, k, T = w.d, w.N, w.k, w.T
    xdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    xb = 2 if w.dtype == "bf16" else 4
    set_bytes = T * d * xb * 2 + T * N * 4
    nsets = max(2, int(math.ceil(1.5 * L2_BYTES / set_bytes)))
    g = torch.Generator(device="cpu").manual_seed(1234 + rank)
    x0 = torch.from_numpy(inp.x).to(xdt)
    l0 = torch.from_numpy(inp.logits)
    xs, ls, ys = [], [], []
    for s in range(nsets):
        p = torch.arange(T) if s == 0 else torch.randperm(T, generator=g)
        xs.append(x0[p].contiguous().to(device))
        ls.append(l0[p].contiguous().to(device))
        ys.append(torch.empty((T, d), dtype=xdt, device=device))
    packed = bf.pack_base(torch.from_numpy(inp.w_base).to(device), inp.alpha)
    theta = torch.from_numpy(inp.theta).to(device)
    phi = torch.from_numpy(inp.phi).to(device)
    ws = bf.forward_workspace(T, d, N, k, device)

    def step(s):
        bf.forward(xs[s], ls[s], k, packed, theta, phi, ws=ws, out=ys[s], stream=stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i % nsets)
    st = bf.sync_status(ws, stream)
    if st != bf.OK:
        raise RuntimeError(f"warm-up status {bf.status_string(st)}")

    # exactly K timed steps, cycling through the input sets, in one graph
    K = args.steps
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            for i in range(K):
                step(i % nsets)
        graph.replay()
    stream.synchronize()

    # clocks: sample through a soak of back-to-back replays and the timed
    # region that follows it
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_id = vis.split(",")[local].strip() if vis else str(device.index)
    sampler = ClockSampler(smi_id)
    sampler.start()
    with torch.cuda.stream(stream):
        t_end = time.perf_counter() + args.soak_seconds
        while time.perf_counter() < t_end:
            graph.replay()
            stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1) / K
    ksteps = K
    st = bf.sync_status(ws, stream)
    if st != bf.OK:
        raise RuntimeError(f"timed status {bf.status_string(st)}")
    ms = max_over_ranks(ms, device)

    # per-kernel durations (events between the launches of one step)
    prof = {}
    nprof = args.profile_steps
    with torch.cuda.stream(stream):
        for i in range(nprof):
            r = bf.forward_profile(xs[i % nsets], ls[i % nsets], k, packed, theta, phi, ws, ys[i % nsets],
                                   stream=stream)
            for key, v in r.items():
                prof[key] = prof.get(key, 0.0) + v / nprof

    # end to end through the public API from pinned host buffers
    hx = [xs[s].cpu().pin_memory() for s in range(nsets)]
    hl = [ls[s].cpu().pin_memory() for s in range(nsets)]
    hy = [torch.empty((T, d), dtype=xdt).pin_memory() for _ in range(nsets)]
    dx = torch.empty_like(xs[0])
    dl = torch.empty_like(ls[0])
    dy = torch.empty_like(ys[0])

    def e2e_step(s):
        dx.copy_(hx[s], non_blocking=True)
        dl.copy_(hl[s], non_blocking=True)
        bf.forward(dx, dl, k, packed, theta, phi, ws=ws, out=dy, stream=stream)
        hy[s].copy_(dy, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 1)):
            e2e_step(i % nsets)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g2, stream=stream):
            for i in range(K):
                e2e_step(i % nsets)
        g2.replay()
    stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        g2.replay()
        f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / K, device)
    if bf.sync_status(ws, stream) != bf.OK:
        raise RuntimeError("e2e status")

    flops, bmin = layer_model(w)
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = bmin / (peaks["hbm_gbs"] * 1e9)
    t_roof = max(t_tensor, t_hbm)
    value = job_tokens_per_s(world, T, ms)

    # dominant kernel and its roofline
    R, Rp, L = T * k, (T * k + 127) // 128 * 128, w.L
    rot = R * L * (d // 2)  # Givens rotations per butterfly pass over all rows
    sm_mhz = (clocks or {}).get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)
    alu_peak = 148 * 128 * sm_mhz * 1e6 / 1e12  # FP32 lane-instructions, Tops/s
    models = {
        "contract": ("tensor", 2.0 * R * d * d, "TFLOP/s"),
        "expert_in": ("alu", 4.0 * rot, "Tops/s"),
        "combine": ("hbm", R * d * 2 + T * d * xb + R * 4, "GB/s"),
        "route": ("hbm", T * N * 4 + T * k * 12, "GB/s"),
    }
    dom = max(prof, key=prof.get) if prof else None
    # rows per expert of the last forward on this workspace (skewed loads show here)
    _, _, _, offs = bf.forward_routing(ws, T, d, N, k)
    sizes = np.diff(offs.cpu().numpy().astype(np.int64))
    buckets = {"max": int(sizes.max()), "min": int(sizes.min()), "empty": int((sizes == 0).sum())}
    roof = None
    if dom in models:
        bound, amount, unit = models[dom]
        sec = prof[dom] * 1e-3
        if bound == "tensor":
            achieved = amount / sec / 1e12
            peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        elif bound == "alu":
            achieved = amount / sec / 1e12
            peak = alu_peak
        else:
            achieved = amount / sec / 1e9
            peak = peaks["hbm_gbs"]
        roof = {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": profiled_traffic(w.name).get(dom),
                "peak_source": peaks["source"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r, threads, n, dt = cpu_oracle_rate(w, args.cpu_seconds)
        cpu = {"value": r, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n} tokens of the {w.name} workload, fp64 C oracle with OpenMP, {dt:.1f} s"}
        if w.name in ("tiny", "headline"):
            r1, _, n1, dt1 = cpu_oracle_rate(w, min(2.0, args.cpu_seconds / 4), nthreads=1)
            cpu["single_thread_value"] = r1
            cpu["single_thread_sample"] = f"{n1} tokens, 1 thread, {dt1:.1f} s"

    if rank == 0:
        line = {
            "metric": "ButterflyMoE layer routed tokens/s (d=%d,N=%d,top-%d)" % (d, N, k),
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": ksteps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": w.name, "d": d, "N": N, "k": k, "T": T, "x": w.dtype,
                       "parallelism": f"replicas x{world}", "l2": f"inputs rotate over {nsets} sets "
                       f"({nsets * set_bytes / 2**20:.0f} MiB > L2)", "graph": "CUDA graph replay"},
            "routed_rows_per_s": world * T * k / (ms * 1e-3),
            "layer_roofline": {"t_roof_us": t_roof * 1e6, "t_step_us": ms * 1e3, "frac": t_roof / (ms * 1e-3),
                               "bound": "tensor" if t_tensor >= t_hbm else "hbm",
                               "t_tensor_us": t_tensor * 1e6, "t_hbm_us": t_hbm * 1e6,
                               "frac_sustained": max(flops / (peaks.get("bf16_tflops_sustained",
                                                                        peaks["bf16_tflops"]) * 1e12),
                                                     t_hbm) / (ms * 1e-3),
                               "peaks": f"{peaks['bf16_tflops']} TF bf16 burst, "
                                        f"{peaks.get('bf16_tflops_sustained', peaks['bf16_tflops'])} TF sustained, "
                                        f"{peaks['hbm_gbs']} GB/s ({peaks['source']})"},
            "buckets": buckets,
            "roofline": roof,
            "kernels_ms": prof,
            "gpu_launches": len(prof) * ksteps if prof else None,
            "cpu_baseline": cpu,
            "e2e": {"value": job_tokens_per_s(world, T, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(xs[0].numel() * xs[0].element_size() + ls[0].numel() * 4),
                    "d2h_bytes_per_step": int(ys[0].numel() * ys[0].element_size()), "ms_per_step": e2e_ms},
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    del graph, g2
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--profile-steps", type=int, default=20)
    ap.add_argument("--config", default="headline", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--soak-seconds", type=float, default=1.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    w = wl.WORKLOADS[args.config]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
