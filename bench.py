#!/usr/bin/env python
"""Throughput of the Sign-Muon optimizer step on B200.

A step is one pass of the whole hot path over one ResNet-50 layer set
(53 conv weights reshaped C_out x C_in*k_h*k_w, 23,454,912 parameters) with
M = 4 simulated workers: momentum update + Frobenius normalisation + one
quintic Newton-Schulz step per worker and layer (212 matrices, tcgen05), then
the fused sign / int8-sum vote / update of the 53 weight matrices.

Prints one JSON line (rank 0). `value` is layer-set steps per second over all
ranks (each rank updates its own layer set: weak scaling, no data-path
collective). `--impl reference` times the CPU oracle on the same workload.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
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

import workloads as WL  # noqa: E402

WORKLOAD = "c2_resnet50"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--graph", action="store_true", help="replay the step as a CUDA graph")
    p.add_argument("--no-graph-compare", dest="graph_compare", action="store_false",
                   help="skip the extra CUDA-graph replay measurement")
    p.add_argument("--e2e-steps", type=int, default=30)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-ns4096", dest="ns4096", action="store_false",
                   help="skip the extra 4096x4096 Newton-Schulz measurement")
    p.add_argument("--only-ns4096", action="store_true",
                   help="run only the 4096x4096 Newton-Schulz measurement (for profiling)")
    p.add_argument("--cachemuon", nargs="*", metavar="RxC:GAMMA",
                   help="CacheMuon sweep instead of the Sign-Muon step, e.g. 4096x4096:2 8192x8192:15 "
                        "(no value: the three large shapes x gamma in {2, 15}); --steps sets the schedule length")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ oracle timing
def oracle_step_sample(cfg, W, grads, layer_ids):
    """One Sign-Muon step of the CPU oracle over the given layers."""
    import oracle as O
    Ws = [W[i] for i in layer_ids]
    Ms = [[np.zeros(cfg.shapes[i]) for _ in range(cfg.workers)] for i in layer_ids]
    Gs = [grads[i] for i in layer_ids]
    return O.sign_muon_step(Ws, Ms, Gs, cfg.beta, cfg.coeffs, cfg.iters, cfg.eta, cfg.w_dtype,
                            cfg.tie_value, cfg.vote)


def layer_cost(shape, cfg):
    r, c = shape
    m, n = min(r, c), max(r, c)
    return cfg.workers * (4 * m * m * n + 2 * m ** 3) * cfg.iters


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [os.cpu_count() or 1])
    except Exception:
        return os.cpu_count() or 1


_ORACLE_INPUTS = {}


def time_oracle(cfg, budget_s):
    """Times the oracle on a bounded sample of the layer set (largest layers
    first until the time budget is used), scaled to layer-set steps/s by the
    sampled share of the Newton-Schulz work."""
    if cfg.name not in _ORACLE_INPUTS:
        _ORACLE_INPUTS[cfg.name] = (WL.weights(cfg.shapes, cfg.w_init, cfg.w_dtype),
                                    WL.GradientStreams(cfg.shapes, cfg.workers, cfg.grad_sigma).next_step())
    W, grads = _ORACLE_INPUTS[cfg.name]
    costs = np.array([layer_cost(s, cfg) for s in cfg.shapes], dtype=np.float64)
    order = list(np.argsort(-costs))
    ids, t_used = [], 0.0
    t_start = time.perf_counter()
    for i in order:
        ids.append(int(i))
        oracle_step_sample(cfg, W, grads, [int(i)])
        t_used = time.perf_counter() - t_start
        if t_used > budget_s:
            break
    share = costs[ids].sum() / costs.sum()
    t_full = t_used / share
    return 1.0 / t_full, ids, share, t_used


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.device_index = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            import torch
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.device_index).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((ts, float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1] or rows
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


# ------------------------------------------------------------------ multi-rank host logic
def rank_seed_base(rank: int) -> int:
    """Each rank updates its own layer set: its gradient streams are seeded
    1000 * rank + worker, so no two ranks share a stream."""
    return 1000 * rank


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(steps: int, ms_max: float, world: int) -> float:
    """Whole-job layer-set steps per second: every rank ran `steps` steps of its
    own layer set within the slowest rank's time."""
    return world * steps / (ms_max / 1000.0)


# ------------------------------------------------------------------ Newton-Schulz on one large matrix
def measure_ns_square(S, torch, peaks, n, iters, reps=10):
    """Five quintic Newton-Schulz steps on one n x n matrix (plain BF16 mode),
    as in a CacheMuon fresh solve without the transform. Issued and nominal
    TFLOP/s of the GEMM stages, and the whole call's time."""
    gen = torch.Generator(device="cuda").manual_seed(4242)
    M = torch.randn((n, n), device="cuda", generator=gen)
    U = torch.empty((n, n), dtype=torch.bfloat16, device="cuda")
    plan = S.NsPlan([M], [U], *WL.QUINTIC, iters)
    for _ in range(3):
        plan.run()
    torch.cuda.synchronize()
    S.trace_enable(True)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        plan.run()
    e1.record()
    torch.cuda.synchronize()
    S.trace_enable(False)
    recs = [r for r in S.trace_read() if r["name"].startswith("k_gemm")]
    stage_ms = {}
    for r in recs:
        stage_ms[r["name"]] = stage_ms.get(r["name"], 0.0) + r["ms"] / reps
    ms_call = e0.elapsed_time(e1) / reps
    t = sum(r["ms"] for r in recs) / 1e3
    issued = sum(r["work"] for r in recs) / t / 1e12
    nominal = sum(r["nominal"] for r in recs) / t / 1e12
    return {"ms_per_call": ms_call, "gemm_ms_per_call_by_stage": stage_ms,
            "gemm_tflops_issued": issued, "gemm_tflops_nominal": nominal,
            "frac_of_peak": issued / peaks["bf16_tflops_sustained"], "nominal_tflop_per_call": 6 * n ** 3 * iters / 1e12}


# ------------------------------------------------------------------ CacheMuon sweep
def run_cachemuon(S, torch, shape, gamma, steps, iters=5):
    """M_0 ~ N(0,1); M_{t+1} = M_t + 0.01 N(0,1); every step probes the cached
    transform on the device and runs the fresh solve only when the residual
    exceeds gamma. Reports the hit rate and the orthogonalisation flops saved
    against a fresh five-step quintic solve every step (nominal counts: Gram
    2m^2n, A^2 2m^3, B X 2m^2n per step; Q accumulation 2m^3 for steps 2..K;
    reuse Q X and probe D D^T 2m^2n each)."""
    m, n = min(shape), max(shape)
    gen = torch.Generator(device="cuda").manual_seed(4242)
    M = torch.randn(shape, device="cuda", generator=gen)
    D = torch.empty(shape, device="cuda")
    cm = S.CacheMuon(M, D, gamma, WL.QUINTIC, iters)
    noise = torch.empty_like(M)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for t in range(steps):
        if t:
            noise.normal_(generator=gen)
            M.add_(noise, alpha=0.01)
        cm.step()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    c = cm.counters()
    f_muon = iters * (4 * m * m * n + 2 * m ** 3)
    f_q = (iters - 1) * 2 * m ** 3
    f_probe = 4 * m * m * n
    fresh = c["misses"]
    cost = fresh * (f_muon + f_q) + c["probes"] * f_probe
    return {"workload": "cachemuon", "shape": list(shape), "gamma": gamma, "steps": steps,
            "hits": c["hits"], "misses": c["misses"], "hit_rate": c["hits"] / steps,
            "orth_flops_saved_vs_fresh": 1.0 - cost / (steps * f_muon),
            "ms_per_step": ms / steps, "note": "momentum drift generated on the device inside the timed loop"}


# ------------------------------------------------------------------ reference arm
def run_reference(args, rank):
    cfg = WL.SIGN_MUON_WORKLOADS[WORKLOAD]
    if rank != 0:
        return
    budget = max(0.05, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        time_oracle(cfg, budget)
    vals = []
    info = None
    for _ in range(args.steps):
        v, ids, share, used = time_oracle(cfg, budget)
        vals.append(v)
        info = (ids, share, used)
    value = float(np.median(vals))
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": "Muon steps/s per layer set", "value": value, "unit": "steps/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Gaussian gradients, He-normal weights)",
        "config": {"workload": "resnet50_conv_set_53_layers_M4_quintic1_int8_vote", "global_batch": None,
                   "seq_len": None, "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {len(info[0])} largest layers x 4 workers "
                                   f"({100 * info[1]:.1f}% of the NS flops), scaled to the full set"},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist

    import matrix_aware_sign_b200 as S

    torch.cuda.set_device(local)
    if args.cachemuon is not None:
        cases = args.cachemuon or [f"{r}x{c}:{g}" for (r, c) in ((4096, 4096), (8192, 8192), (4096, 16384))
                                   for g in (2, 15)]
        for case in cases:
            shp, gam = case.split(":")
            r, c = (int(x) for x in shp.split("x"))
            print(json.dumps(run_cachemuon(S, torch, (r, c), float(gam), args.steps)), flush=True)
        return
    if args.only_ns4096:
        peaks, _ = load_peaks()
        print(json.dumps({"ns_4096sq_quintic5": measure_ns_square(S, torch, peaks, 4096, 5, reps=args.steps)}))
        return
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    cfg = WL.SIGN_MUON_WORKLOADS[WORKLOAD]
    M = cfg.workers
    shapes = cfg.shapes
    L = len(shapes)
    # --- inputs, resident in HBM (two gradient sets, so consecutive steps read different data)
    W = WL.weights(shapes, cfg.w_init, cfg.w_dtype)
    streams = WL.GradientStreams(shapes, M, cfg.grad_sigma, seed_base=rank_seed_base(rank))
    gsets = [streams.next_step(), streams.next_step()]
    Wd = [torch.from_numpy(w).cuda() for w in W]
    Md = [torch.zeros(s, device="cuda") for s in shapes for _ in range(M)]
    Ud = [torch.zeros(s, dtype=torch.bfloat16, device="cuda") for s in shapes for _ in range(M)]
    Gd = [[torch.from_numpy(g).cuda() for layer in gs for g in layer] for gs in gsets]
    Ul = [Ud[l * M:(l + 1) * M] for l in range(L)]
    ws = S.workspace(S.smuon_ns_workspace_bytes(Md, cfg.iters, 0))
    n_params = sum(r * c for r, c in shapes)
    g_bytes = n_params * M * 4
    w_bytes = n_params * 4

    # prepared calls (plan handles): each plan's descriptors are uploaded once into its workspace
    ws2 = S.workspace(ws.numel())
    ws_e2e = S.workspace(ws.numel()) if args.e2e_steps > 0 else None
    ns_plans = [S.NsPlan(Md, Ud, *cfg.coeffs, cfg.iters, G=Gd[j], beta=cfg.beta, ws=[ws, ws2][j]) for j in range(2)]
    upd_plan = S.UpdatePlan(Wd, cfg.eta, U=Ul, M=M, tie_value=cfg.tie_value, vote_kind=S.VOTE_INT8)

    def step(i, G=None):
        if G is None:
            ns_plans[i & 1].run()
            upd_plan.run()
        else:  # end to end: the one-shot public calls (own workspace, the plans keep theirs)
            S.smuon_ns(Md, Ud, *cfg.coeffs, cfg.iters, G=G, beta=cfg.beta, ws=ws_e2e)
            S.smuon_update(Wd, cfg.eta, U=Ul, M=M, tie_value=cfg.tie_value, vote_kind=S.VOTE_INT8)

    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    graph = None
    if args.graph:
        graph = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
        side = torch.cuda.Stream()
        with torch.cuda.stream(side):
            for j in range(2):
                with torch.cuda.graph(graph[j], stream=side):
                    step(j)
        torch.cuda.synchronize()

    # --- timed region
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    S.trace_enable(not args.graph)
    n0 = S.launch_count()
    barrier()
    torch.cuda.synchronize()
    t_wall0 = time.perf_counter()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(args.steps):
        if graph is not None:
            graph[i & 1].replay()
        else:
            step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    t_wall1 = time.perf_counter()
    launches = S.launch_count() - n0
    S.trace_enable(False)
    recs = S.trace_read()
    time.sleep(0.3)
    sampler.stop()
    ms = reduce_max(ev0.elapsed_time(ev1), world, device="cuda")
    if graph is not None:
        launches = launches or 8 * args.steps  # graph replays launch the captured kernels
    ms_per_step = ms / args.steps
    value = job_throughput(args.steps, ms, world)

    # --- roofline of the dominant kernel (from the library's event trace)
    peaks, peak_src = load_peaks()
    by, stages = {}, {}
    for r in recs:
        kname = r["name"].split(".")[0]  # stage-qualified names ("k_gemm_tc.axpy") roll up into their kernel
        for key, table in ((kname, by), (r["name"], stages)):
            d = table.setdefault(key, {"ms": 0.0, "work": 0.0, "nominal": 0.0, "n": 0, "kind": r["kind"]})
            d["ms"] += max(r["ms"], 0.0)
            d["work"] += r["work"]
            d["nominal"] += r["nominal"]
            d["n"] += 1
    roofline = None
    kernels = {}
    total_ms = sum(d["ms"] for d in by.values()) or 1.0
    for name, d in by.items():
        per_launch_ms = d["ms"] / max(d["n"], 1)
        if d["kind"] == S.WORK_FLOPS:
            ach = d["work"] / (d["ms"] / 1e3) / 1e12 if d["ms"] > 0 else 0.0
            unit, peak = "TFLOP/s", peaks["bf16_tflops_sustained"]
        else:
            ach = d["work"] / (d["ms"] / 1e3) / 1e9 if d["ms"] > 0 else 0.0
            unit, peak = "GB/s", peaks["hbm_gbs"]
        kernels[name] = {"launches": d["n"], "share": d["ms"] / total_ms, "ms_per_launch": per_launch_ms,
                         "achieved": ach, "unit": unit, "frac": ach / peak}
    stage_detail = {k: {"launches": d["n"], "ms_per_launch": d["ms"] / max(d["n"], 1),
                        "tflops_issued": d["work"] / (d["ms"] / 1e3) / 1e12 if d["ms"] > 0 else 0.0}
                    for k, d in stages.items() if "." in k}
    if by:
        dom = max(by, key=lambda k: by[k]["ms"])
        kd = kernels[dom]
        traffic = None
        tf = os.path.join(ROOT, "profiles", "traffic.json")
        if os.path.exists(tf):
            try:
                import hashlib
                with open(tf) as f:
                    tj = json.load(f)
                ent = tj.get(dom)
                if ent:  # valid only while the kernel's sources are the ones the counters were taken on
                    hs = hashlib.sha256()
                    for f in ent["sources"]:
                        hs.update(open(os.path.join(ROOT, "matrix_aware_sign_b200", "csrc", f), "rb").read())
                    if hs.hexdigest() == ent["sha256"]:
                        traffic = ent["bytes_per_launch"]
            except Exception:
                traffic = None
        roofline = {"bound": "tensor" if kd["unit"] == "TFLOP/s" else "hbm", "kernel": dom,
                    "achieved": kd["achieved"], "peak": peaks["bf16_tflops_sustained"] if kd["unit"] == "TFLOP/s"
                    else peaks["hbm_gbs"], "unit": kd["unit"], "frac": kd["frac"], "traffic": traffic,
                    "peak_source": f"{peak_src} ({'bf16 sustained' if kd['unit'] == 'TFLOP/s' else 'HBM copy'})"}

    # --- the same step replayed as a CUDA graph (launch overhead removed), reported beside `value`
    graph_value = None
    if graph is None and args.graph_compare and world == 1:
        g2 = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
        side = torch.cuda.Stream()
        with torch.cuda.stream(side):
            for j in range(2):
                with torch.cuda.graph(g2[j], stream=side):
                    step(j)
        torch.cuda.synchronize()
        for j in range(4):
            g2[j & 1].replay()
        torch.cuda.synchronize()
        q0 = torch.cuda.Event(enable_timing=True)
        q1 = torch.cuda.Event(enable_timing=True)
        q0.record(stream)
        for i in range(args.steps):
            g2[i & 1].replay()
        q1.record(stream)
        torch.cuda.synchronize()
        graph_value = args.steps / (q0.elapsed_time(q1) / 1000.0)
        del g2

    # --- end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0:
        hostG = [[torch.from_numpy(g).pin_memory() for layer in gs for g in layer] for gs in gsets]
        hostW = [torch.empty(w.shape, dtype=torch.float32).pin_memory() for w in W]
        devG = [torch.empty_like(g) for g in Gd[0]]
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.e2e_steps):
            for d, h in zip(devG, hostG[i & 1]):
                d.copy_(h, non_blocking=True)
            step(i, devG)
            for h, d in zip(hostW, Wd):
                h.copy_(d, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems = reduce_max(e0.elapsed_time(e1), world, device="cuda")
        e2e = {"value": job_throughput(args.e2e_steps, ems, world), "unit": "steps/s",
               "h2d_bytes_per_step": g_bytes, "d2h_bytes_per_step": w_bytes}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, ids, share, used = time_oracle(cfg, budget_s=15.0)
        cpu = {"value": v, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{len(ids)} largest of 53 layers x 4 workers ({100 * share:.1f}% of the NS flops, "
                         f"{used:.1f} s), scaled to the full layer set"}

    ns = [k for k in kernels if k.startswith("k_gemm")]
    summary = {}
    if ns:
        fl = sum(by[k]["work"] for k in ns)
        nom = sum(by[k]["nominal"] for k in ns)
        t = sum(by[k]["ms"] for k in ns)
        summary["ns_tflops"] = fl / (t / 1e3) / 1e12
        summary["ns_tflops_nominal"] = nom / (t / 1e3) / 1e12
        summary["ns_frac_of_peak"] = summary["ns_tflops"] / peaks["bf16_tflops_sustained"]
    if rank == 0 and world == 1 and args.ns4096:
        summary["ns_4096sq_quintic5"] = measure_ns_square(S, torch, peaks, 4096, 5)
    vk = [k for k in kernels if k.startswith("k_vote_update")]
    if vk:
        summary["vote_gbs"] = kernels[vk[0]]["achieved"]
        summary["vote_frac_of_hbm"] = kernels[vk[0]]["frac"]

    if rank == 0:
        clocks = sampler.summary(t_wall0, t_wall1)
        line = {
            "metric": "Muon steps/s per layer set", "value": value, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Gaussian gradients N(0,1e-4), He-normal weights)",
            "config": {"workload": "resnet50_conv_set_53_layers_M4_quintic1_int8_vote", "layers": L,
                       "params": n_params, "workers": M, "ns_iters": cfg.iters, "vote": "int8 sum",
                       "global_batch": None, "seq_len": None, "parallelism": f"replicas x{world}",
                       "launch": "cuda_graph" if graph is not None else "eager",
                       "l2": "inputs larger than L2: 375 MB of gradients per step, two resident sets alternate"},
            "roofline": roofline, "kernels": kernels, "gemm_stages": stage_detail, **summary,
            "steps_per_s_cuda_graph": graph_value,
            "clocks": clocks, "e2e": e2e,
            "gpu_launches": launches, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
