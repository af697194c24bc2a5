#!/usr/bin/env python
"""Throughput of the Sign-Muon / LionMuon optimizer step on B200.

Headline (the default): the GPT-2-Large layer set under the LionMuon schedule
(36 blocks x {1280x3840, 1280x1280, 1280x5120, 5120x1280}, 144 matrices,
707,788,800 parameters, bf16 weights) with M = 16 simulated workers and period
P = 4: three Lion sign steps (the workers' sign(G_hat) in a 1-bit majority vote)
and one Muon step (five quintic Newton-Schulz steps on the worker mean of G_hat,
split-BF16 tensor-core operands) per period. A step is one step of the schedule;
the timed region covers whole periods when --steps is a multiple of 4.

Beside it, under "extra", each with its own roofline: the ResNet-50 layer set
(53 convolutions, M = 4, one quintic step, int8 sum vote), the GPT-2-small set
(48 matrices, M = 8, five quintic steps, 1-bit popcount vote) and five quintic
Newton-Schulz steps on one 4096 x 4096 matrix.

Prints one JSON line (rank 0). `value` is layer-set steps per second. With N
ranks the layer set is split by layer (every matrix with all its workers on one
rank, longest first onto the least loaded rank) and `value` counts whole
layer-set steps in the slowest rank's time. `--impl reference` times the CPU
oracle on the same workload.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
import heapq
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

WORKLOAD = "c5_gpt2l"
WORKLOAD_CHOICES = ["c5_gpt2l", "c2_resnet50", "c3_gpt2s", "resnet18", "llama124m", "llama355m", "llama720m"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
BURST_REGION_S = 1.0  # a timed region shorter than this is compared with the burst tensor peak
DEFAULT_PLAIN_LEAD = 2  # leading Newton-Schulz steps with plain BF16 operands in split mode (the GPT-2 sets'
                        # Gaussian momenta meet the tolerances with two; smaller matrices take one)


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=40)
    p.add_argument("--warmup", type=int, default=8)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--graph", action="store_true", help="replay the step as a CUDA graph")
    p.add_argument("--no-graph-compare", dest="graph_compare", action="store_false",
                   help="skip the extra CUDA-graph replay measurement")
    p.add_argument("--e2e-steps", type=int, default=8)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extras", dest="extras", action="store_false",
                   help="headline only: skip the ResNet-50, GPT-2-small and 4096^2 measurements")
    p.add_argument("--only-ns4096", action="store_true",
                   help="run only the 4096x4096 Newton-Schulz measurement (for profiling)")
    p.add_argument("--workload", choices=WORKLOAD_CHOICES, default=WORKLOAD,
                   help="layer set: GPT-2-Large LionMuon (M=16, P=4; default), ResNet-50 Sign-Muon (M=4, int8 "
                        "vote, 1 quintic step), GPT-2-small Sign-Muon (M=8, popcount vote, 5 quintic steps); "
                        "ResNet-18 with the ResNet-50 set's settings, LLaMA-style 124M/355M/720M sets with the "
                        "GPT-2-small set's")
    p.add_argument("--ns-mode", choices=["plain", "split"], default=None,
                   help="Newton-Schulz operand precision (default: plain for one quintic step, split BF16 for "
                        "five, the mode that meets the tolerances there)")
    p.add_argument("--plain-lead", type=int, default=None,
                   help="split mode: run this many leading Newton-Schulz steps with plain BF16 operands "
                        "(SMUON_NS_PLAIN_LEAD; default 2; matrices with a smaller side under 512 take one)")
    p.add_argument("--one-sm", action="store_true",
                   help="tensor-core stages on single-SM 128x256 tiles (SMUON_NS_ONE_SM) instead of the SM pairs "
                        "(256x256 tiles over clusters of two CTAs) that batches of matrices with a smaller side "
                        ">= 256 use by default")
    p.add_argument("--grad-source", choices=["hbm", "counter"], default="hbm",
                   help="LionMuon set: read a resident 45 GB gradient set (default), or draw the workers' "
                        "gradients inside the kernels from the counter-based streams (no gradient bytes, more ALU)")
    p.add_argument("--period", type=int, default=None,
                   help="LionMuon set: period P (default 4; 1 = Muon steps only, 0 = never a Muon step)")
    p.add_argument("--beta2", type=float, default=None,
                   help="LionMuon set: EMA rate beta2 (default 0.99; beta2 = beta1 = 0.9 gives Signum-type sign steps)")
    p.add_argument("--layers", type=int, default=0,
                   help="use only the first LAYERS matrices of the set (a smaller case for profiler captures)")
    p.add_argument("--local-polar", action="store_true",
                   help="GPT-2-small set: orthogonalise the voted matrix before the update")
    p.add_argument("--sign-out", choices=["i8", "bf16", "bits"], default="i8",
                   help="ResNet sets: the NS epilogue writes the int8 signs (default) or bf16 U for the vote "
                        "kernel; GPT-2-small set: 'bits' has the NS epilogue write the 1-bit messages")
    p.add_argument("--spectral", action="store_true",
                   help="Sign-Muon sets: normalise by the spectral norm (SMUON_NS_SPECTRAL, Lanczos estimate on "
                        "the device) instead of the Frobenius norm")
    p.add_argument("--gram-only", action="store_true",
                   help="CacheMuon sweep: fresh solves iterated on the m x m Gram (SMUON_NS_GRAM_ONLY)")
    p.add_argument("--diagnose", action="store_true",
                   help="CacheMuon sweep: every step also runs a fresh solve and records the residual beside the "
                        "cached/fresh agreement")
    p.add_argument("--drift", type=float, default=0.01,
                   help="CacheMuon sweep: momentum drift per step, M_{t+1} = M_t + drift * N(0,1) (default 0.01)")
    p.add_argument("--cachemuon", nargs="*", metavar="RxC:GAMMA",
                   help="CacheMuon sweep instead of the Sign-Muon step, e.g. 4096x4096:2 8192x8192:15 "
                        "(no value: the three large shapes x gamma in {2, 15}); --steps sets the schedule length")
    return p.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def tensor_peak(peaks, region_s):
    """The dense bf16 peak a contraction timed over `region_s` seconds is
    compared with: the burst figure for a region shorter than about a second,
    the sustained (power-capped) one for longer regions."""
    if region_s < BURST_REGION_S:
        return peaks["bf16_tflops"], "bf16 burst"
    return peaks["bf16_tflops_sustained"], "bf16 sustained"


# ------------------------------------------------------------------ oracle timing
def oracle_step_sample(cfg, W, grads, layer_ids):
    """One Sign-Muon step of the CPU oracle over the given layers."""
    import oracle as O
    Ws = [W[i] for i in layer_ids]
    Ms = [[np.zeros(cfg.shapes[i]) for _ in range(cfg.workers)] for i in layer_ids]
    Gs = [grads[i] for i in layer_ids]
    return O.sign_muon_step(Ws, Ms, Gs, cfg.beta, cfg.coeffs, cfg.iters, cfg.eta, cfg.w_dtype,
                            cfg.tie_value, cfg.vote, spectral=_SPECTRAL[0])


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
_SPECTRAL = [False]  # --spectral: both arms normalise by the spectral norm


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
        for ts, line in list(self.lines):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((ts, float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        if not inside:  # a region shorter than the sampling period: the samples around it
            near = sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))
            inside = near[:3]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


# ------------------------------------------------------------------ multi-rank host logic
def partition_layers(costs, world: int):
    """Splits one layer set across `world` ranks by whole layers (every matrix
    with all its simulated workers on one rank): layers in decreasing cost
    (ties in index order), each onto the rank with the least cost so far
    (ties: lowest rank). Returns one sorted list of layer indices per rank."""
    order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
    heap = [(0.0, r) for r in range(world)]
    owned = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        owned[r].append(i)
        heapq.heappush(heap, (load + float(costs[i]), r))
    return [sorted(o) for o in owned]


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def layer_set_rate(steps: int, ms_max: float) -> float:
    """Whole-job layer-set steps per second: the ranks together updated every
    layer of the set `steps` times within the slowest rank's time."""
    return steps / (ms_max / 1000.0)


# ------------------------------------------------------------------ Newton-Schulz on one large matrix
def measure_ns_square(S, torch, peaks, n, iters, flags, reps=10):
    """Five quintic Newton-Schulz steps on one n x n matrix, as in a CacheMuon
    fresh solve without the transform, timed alone (so against the burst peak).
    The rate that counts is the method's nominal flops (per step 2n^3 for the
    Gram, 2n^3 for A^2, 2n^3 for B X) over the GEMM stages' event-timed
    duration; the tensor cores' issued flops (the symmetric stages compute only
    their upper tile triangle; split mode issues three products) are given
    beside it."""
    gen = torch.Generator(device="cuda").manual_seed(4242)
    M = torch.randn((n, n), device="cuda", generator=gen)
    U = torch.empty((n, n), dtype=torch.bfloat16, device="cuda")
    plan = S.NsPlan([M], [U], *WL.QUINTIC, iters, flags=flags)
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
    del plan, M, U
    return {"ms_per_call": ms_call, "gemm_ms_per_call": t * 1e3 / reps, "gemm_ms_per_call_by_stage": stage_ms,
            "gemm_tflops_nominal": nominal, "frac_of_burst_peak": nominal / peaks["bf16_tflops"],
            "gemm_tflops_issued": issued, "issued_frac_of_burst_peak": issued / peaks["bf16_tflops"],
            "nominal_tflop_per_call": 6 * n ** 3 * iters / 1e12}


# ------------------------------------------------------------------ CacheMuon sweep
def cachemuon_flop_counts(m, n, iters, gram_only):
    """Nominal orthogonalisation flops per event of the sweep: a fresh Muon
    solve (per step Gram 2m^2n, A^2 2m^3, B X 2m^2n), the accumulation of Q
    (2m^3 for steps 2..K), a probe (reuse Q X and D D^T, 2m^2n each), and the
    Gram-only fresh solve (X_0 X_0^T and Q_K X_0 once, per step A^2 and, but
    for the last step, Q and the two A updates). The symmetric-aware counts
    take the Gram, A^2, D D^T and A-update products at half their size."""
    f_muon = iters * (4 * m * m * n + 2 * m ** 3)
    f_q = (iters - 1) * 2 * m ** 3
    f_probe = 4 * m * m * n
    f_gram_only = 4 * m * m * n + iters * 2 * m ** 3 + (iters - 1) * 3 * 2 * m ** 3
    sym = {"muon": iters * (3 * m * m * n + m ** 3), "q": f_q, "probe": 3 * m * m * n,
           "gram_only": 3 * m * m * n + iters * m ** 3 + (iters - 1) * (2 * m ** 3 + 2 * m ** 3)}
    return {"muon": f_muon, "q": f_q, "probe": f_probe, "gram_only": f_gram_only}, sym


def cachemuon_saved(counts, hits, misses, probes, steps, gram_only):
    """1 - (issued orthogonalisation flops) / (a fresh solve every step)."""
    fresh = counts["gram_only"] if gram_only else counts["muon"] + counts["q"]
    cost = misses * fresh + probes * counts["probe"]
    return 1.0 - cost / (steps * counts["muon"])


def run_cachemuon(S, torch, shape, gamma, steps, iters=5, gram_only=False, diagnose=False, drift=0.01,
                  one_sm=False):
    """M_0 ~ N(0,1); M_{t+1} = M_t + drift N(0,1); every step probes the cached
    transform on the device and runs the fresh solve only when the residual
    exceeds gamma. Reports the hit rate and the orthogonalisation flops saved
    against a fresh five-step quintic solve every step, on nominal and on
    symmetric-aware counts. With `diagnose`, every step also runs a fresh solve
    into a second buffer (outside the schedule's counters) and records the
    probe's residual beside the cached/fresh agreement."""
    m, n = min(shape), max(shape)
    gen = torch.Generator(device="cuda").manual_seed(4242)
    M = torch.randn(shape, device="cuda", generator=gen)
    D = torch.empty(shape, device="cuda")
    flags = S.NS_SPLIT_BF16 | (S.NS_GRAM_ONLY if gram_only else 0) | (S.NS_ONE_SM if one_sm else 0)
    cm = S.CacheMuon(M, D, gamma, WL.QUINTIC, iters, flags=flags)
    noise = torch.empty_like(M)
    rows = []
    if diagnose:
        D_fresh = torch.empty(shape, device="cuda")
        fresh = S.NsPlan([M], [D_fresh], *WL.QUINTIC, iters, flags=S.NS_SPLIT_BF16)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for t in range(steps):
        if t:
            noise.normal_(generator=gen)
            M.add_(noise, alpha=drift)
        if not diagnose:
            cm.step()
            continue
        # the candidate D_hat of this step's probe against a fresh solve of the same momentum, before the
        # schedule's own fresh solve (skipped on a hit) overwrites D; kept on the device until the end
        fresh.run()
        cm.probe()
        if t:
            rel = torch.linalg.vector_norm(D - D_fresh) / torch.linalg.vector_norm(D_fresh)
            agree = ((D >= 0) == (D_fresh >= 0)).float().mean()
            rows.append(torch.stack([cm.err[0], rel, agree, cm.accept[0].float()]))
        cm.refresh()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    c = cm.counters()
    counts, sym = cachemuon_flop_counts(m, n, iters, gram_only)
    out = {"workload": "cachemuon", "shape": list(shape), "gamma": gamma, "steps": steps, "drift": drift,
           "hits": c["hits"], "misses": c["misses"], "hit_rate": c["hits"] / steps,
           "orth_flops_saved_vs_fresh": cachemuon_saved(counts, c["hits"], c["misses"], c["probes"], steps, gram_only),
           "orth_flops_saved_vs_fresh_symmetric_aware": cachemuon_saved(sym, c["hits"], c["misses"], c["probes"],
                                                                        steps, gram_only),
           "ms_per_step": ms / steps, "fresh_solve": "gram_only" if gram_only else "x_iteration",
           "fresh_solve_tiles": "single_sm" if one_sm else "sm_pairs",
           "note": "momentum drift generated on the device inside the timed loop"}
    if diagnose:
        vals = torch.stack(rows).cpu().tolist() if rows else []
        out["diagnostic"] = [{"step": t + 1, "err": e, "rel_diff_cached_vs_fresh": r, "sign_agreement": a,
                              "accepted": bool(acc)} for t, (e, r, a, acc) in enumerate(vals)]
        out["note"] += "; with the diagnostic the timed loop also runs a fresh solve every step"
    return out


# ------------------------------------------------------------------ oracle timing of the other layer sets
_LION_INPUTS = {}


def time_oracle_lion(cfg, budget_s):
    """Oracle steps/s of the LionMuon schedule, from two bounded samples on one
    transformer block (the blocks are identical): a sign step on the first rows
    of the block's four matrices (elementwise: scaled by the entries), and a
    Muon step on a square slice of the 1280 x 1280 matrix (scaled by the
    Newton-Schulz flops of the block). Period time = (P-1) sign steps + one
    Muon step."""
    import oracle as O
    block = cfg.shapes[:4]
    n_blocks = len(cfg.shapes) // 4
    if cfg.name not in _LION_INPUTS:
        rng = np.random.default_rng(7)
        W = WL.weights(block, "normal002", cfg.w_dtype)
        G = [[rng.standard_normal(s, dtype=np.float32) for _ in range(cfg.workers)] for s in block]
        _LION_INPUTS[cfg.name] = (W, G)
    W, G = _LION_INPUTS[cfg.name]
    args = (cfg.period, cfg.beta1, cfg.beta2, cfg.eta, cfg.coeffs, cfg.iters, cfg.w_dtype, cfg.tie_value)

    def timed(t, Ws, Gs):
        Ms = [[np.zeros(w.shape, np.float32) for _ in range(cfg.workers)] for w in Ws]
        t0 = time.perf_counter()
        O.lionmuon_step(t, Ws, Ms, Gs, *args)
        return time.perf_counter() - t0

    def sign_sample(rows):
        return timed(1, [w[:rows] for w in W], [[g[:rows] for g in gl] for gl in G])

    probe = sign_sample(16)
    rows = int(min(1280, max(16, 16 * 0.5 * budget_s / max(probe, 1e-6))))
    t_rows = sign_sample(rows)
    frac = sum(min(rows, r) * c for r, c in block) / sum(r * c for r, c in block)
    t_sign = t_rows / frac
    side = 1280 if budget_s >= 4.0 else 320
    t_sq = timed(cfg.period, [W[1][:side, :side]], [[g[:side, :side] for g in G[1]]])
    ns = lambda m, n: 4 * m * m * n + 2 * m ** 3
    t_muon = t_sq * sum(ns(min(r, c), max(r, c)) for r, c in block) / ns(side, side)
    period = (cfg.period - 1) * t_sign + t_muon
    return cfg.period / (period * n_blocks), rows, side, probe + t_rows + t_sq


def oracle_rate(name, budget_s):
    """(steps/s of the oracle, sample description) for a layer set."""
    if name in WL.LION_MUON_WORKLOADS:
        cfg = WL.LION_MUON_WORKLOADS[name]
        v, rows, side, used = time_oracle_lion(cfg, budget_s)
        return v, (f"one transformer block x {cfg.workers} workers: a sign step on the first {rows} rows, a Muon "
                   f"step on a {side}x{side} slice ({used:.1f} s); period = {cfg.period - 1} sign + 1 Muon, "
                   f"scaled by entries and NS flops to the {len(cfg.shapes) // 4} identical blocks")
    cfg = WL.SIGN_MUON_WORKLOADS[name]
    v, ids, share, used = time_oracle(cfg, budget_s)
    return v, (f"{len(ids)} largest of {len(cfg.shapes)} layers x {cfg.workers} workers ({100 * share:.1f}% of "
               f"the NS flops, {used:.1f} s), scaled to the full layer set")


# ------------------------------------------------------------------ reference arm
def run_reference(args, rank):
    if rank != 0:
        return
    _SPECTRAL[0] = args.spectral
    mode = default_ns_mode(args)
    desc = describe(args.workload, mode, args.local_polar, args.spectral, plain_lead_of(args) if mode == "split" else 0,
                    args.sign_out)
    budget = max(0.05, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_rate(args.workload, budget)
    vals = []
    sample = None
    for _ in range(args.steps):
        v, sample = oracle_rate(args.workload, budget)
        vals.append(v)
    value = float(np.median(vals))
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": "Muon steps/s per layer set", "value": value, "unit": "steps/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 / value,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Gaussian gradients and weights of the same distributions, drawn on the host)",
        "config": {"workload": desc["workload"], "global_batch": None, "seq_len": None, "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the layer sets
def default_ns_mode(args):
    if args.ns_mode:
        return args.ns_mode
    return "plain" if args.workload in ("c2_resnet50", "resnet18") else "split"


def plain_lead_of(args):
    """Plain leading steps of the split mode: the default two, none with spectral scaling (its s_max = 1 start
    leaves no step whose B X term is small), or --plain-lead as given."""
    if args.plain_lead is not None:
        if args.plain_lead and getattr(args, "spectral", False):
            raise SystemExit("--plain-lead does not combine with --spectral")
        return args.plain_lead
    return 0 if getattr(args, "spectral", False) else DEFAULT_PLAIN_LEAD


def describe(name, ns_mode, local_polar, spectral=False, plain_lead=0, sign_out="i8"):
    d = _describe(name, ns_mode, local_polar)
    if ns_mode == "split" and plain_lead:
        d["workload"] += f"_plain_lead{plain_lead}"
    if sign_out == "bits" and name not in ("c2_resnet50", "resnet18", "c5_gpt2l"):
        d["workload"] += "_ns_bits"
    if spectral:
        d["workload"] += "_spectral_norm"
    return d


def _describe(name, ns_mode, local_polar):
    if name == "c2_resnet50":
        return {"workload": "resnet50_conv_set_53_layers_M4_quintic1_int8_vote",
                "data": "synthetic (seeded Gaussian gradients N(0,1e-4), He-normal weights)"}
    if name == "c3_gpt2s":
        return {"workload": "gpt2_small_set_48_matrices_M8_quintic5_popcount_vote"
                            + ("_local_polar" if local_polar else "") + f"_{ns_mode}_bf16",
                "data": "synthetic (seeded Gaussian gradients N(0,1) drawn on the device, weights N(0,0.02^2) bf16)"}
    if name == "resnet18":
        return {"workload": "resnet18_conv_set_20_layers_M4_quintic1_int8_vote",
                "data": "synthetic (seeded Gaussian gradients N(0,1e-4), He-normal weights)"}
    if name.startswith("llama"):
        n = len(WL.SIGN_MUON_WORKLOADS[name].shapes)
        return {"workload": f"{name}_style_set_{n}_matrices_M8_quintic5_popcount_vote"
                            + ("_local_polar" if local_polar else "") + f"_{ns_mode}_bf16",
                "data": "synthetic (seeded Gaussian gradients N(0,1) drawn on the device, weights N(0,0.02^2) bf16)"}
    return {"workload": f"gpt2_large_set_144_matrices_M16_lionmuon_P4_quintic5_{ns_mode}_bf16",
            "data": "synthetic (seeded Gaussian gradients N(0,1) resident on the device, or with --grad-source "
                    "counter drawn in-kernel from Philox4x32-10 streams; weights N(0,0.02^2) bf16)"}


def set_shapes(name):
    if name in WL.LION_MUON_WORKLOADS:
        return WL.LION_MUON_WORKLOADS[name].shapes
    return WL.SIGN_MUON_WORKLOADS[name].shapes


def set_costs(name, shapes):
    """Per-layer cost used to split a set across ranks: the Newton-Schulz
    flops of all its workers (Sign-Muon sets) or of its Muon step plus the
    elementwise entries (LionMuon, where the sign steps are bandwidth-bound)."""
    if name in WL.LION_MUON_WORKLOADS:
        cfg = WL.LION_MUON_WORKLOADS[name]
        return [(4 * min(r, c) ** 2 * max(r, c) + 2 * min(r, c) ** 3) * cfg.iters + 2e4 * r * c * cfg.workers
                for r, c in shapes]
    cfg = WL.SIGN_MUON_WORKLOADS[name]
    return [layer_cost(s, cfg) for s in shapes]


def rank_layers(name, layers, rank, world):
    """Indices (into the set) of the layers this rank updates: the first
    `layers` of the set when given, split by layer across the ranks."""
    shapes = set_shapes(name)
    ids = list(range(len(shapes) if layers <= 0 else min(layers, len(shapes))))
    if world <= 1:
        return ids
    parts = partition_layers(set_costs(name, [shapes[i] for i in ids]), world)
    return [ids[j] for j in parts[rank]]


def setup_c2(S, torch, ids, ns_flags, e2e, name="c2_resnet50", sign_out="i8"):
    """ResNet layer sets, M = 4: momentum + one quintic NS step (prepared
    plans on two resident gradient sets) + int8-sum vote / update. With
    sign_out = "i8" the NS epilogue writes the workers' int8 sign matrices
    (no U in memory) and the vote kernel sums them; with "bf16" it writes U
    and the vote kernel takes the signs."""
    cfg = WL.SIGN_MUON_WORKLOADS[name]
    M = cfg.workers
    shapes = [cfg.shapes[i] for i in ids]
    L = len(shapes)
    W = WL.weights(shapes, cfg.w_init, cfg.w_dtype)
    streams = WL.GradientStreams(shapes, M, cfg.grad_sigma)
    gsets = [streams.next_step(), streams.next_step()]
    Wd = [torch.from_numpy(w).cuda() for w in W]
    Md = [torch.zeros(s, device="cuda") for s in shapes for _ in range(M)]
    u_dtype = torch.int8 if sign_out == "i8" else torch.bfloat16
    Ud = [torch.zeros(s, dtype=u_dtype, device="cuda") for s in shapes for _ in range(M)]
    Gd = [[torch.from_numpy(g).cuda() for layer in gs for g in layer] for gs in gsets]
    Ul = [Ud[l * M:(l + 1) * M] for l in range(L)]
    nbytes = S.smuon_ns_workspace_bytes(Md, cfg.iters, ns_flags)
    wss = [S.workspace(nbytes), S.workspace(nbytes)]
    ws_e2e = S.workspace(nbytes) if e2e else None
    ns_plans = [S.NsPlan(Md, Ud, *cfg.coeffs, cfg.iters, G=Gd[j], beta=cfg.beta, flags=ns_flags, ws=wss[j])
                for j in range(2)]
    upd_plan = S.UpdatePlan(Wd, cfg.eta, U=Ul, M=M, tie_value=cfg.tie_value, vote_kind=S.VOTE_INT8)
    n_params = sum(r * c for r, c in shapes)

    def step(i):
        ns_plans[i & 1].run()
        upd_plan.run()

    def e2e_io():
        hostG = [[torch.from_numpy(g).pin_memory() for layer in gs for g in layer] for gs in gsets]
        hostW = [torch.empty(w.shape, dtype=torch.float32).pin_memory() for w in W]
        return hostG, [torch.empty_like(g) for g in Gd[0]], hostW, Wd

    def e2e_ns(G):  # the one-shot public calls (own workspace; the prepared plans keep theirs)
        S.smuon_ns(Md, Ud, *cfg.coeffs, cfg.iters, G=G, beta=cfg.beta, flags=ns_flags, ws=ws_e2e)

    def e2e_tail():
        S.smuon_update(Wd, cfg.eta, U=Ul, M=M, tie_value=cfg.tie_value, vote_kind=S.VOTE_INT8)

    return {"step": step, "graphable": True, "e2e_io": e2e_io if e2e else None, "e2e_ns": e2e_ns, "e2e_tail": e2e_tail,
            "g_bytes": n_params * M * 4, "w_bytes": n_params * 4,
            "stage_bytes": gemm_stage_bytes(shapes, M, cfg.iters, cfg.coeffs[2], bool(ns_flags & S.NS_SPLIT_BF16),
                                            1 if sign_out == "i8" else 2),
            "config": {"layers": L, "params": n_params, "workers": M, "ns_iters": cfg.iters, "vote": "int8 sum",
                       "ns_output": "int8 signs from the NS epilogue" if sign_out == "i8" else "bf16 U",
                       "l2": f"inputs larger than L2: {n_params * M * 4 / 1e6:.0f} MB of gradients per step, "
                             "two resident sets alternate"}}


def setup_c3(S, torch, ids, ns_flags, e2e, local_polar, name="c3_gpt2s", sign_out="bf16"):
    """GPT-2-small layer set, M = 8: momentum + five quintic NS steps (prepared
    plans on two resident gradient sets), then either the fused sign / 1-bit
    pack / popcount vote / update with the packed payload written out, or
    (local polar step) sign-pack + popcount vote, NS on the 48 voted matrices
    and the dense update. With sign_out = "bits" the last NS epilogue writes
    each worker's 1-bit message (no U in memory) and the vote kernel reads
    only the messages and W."""
    cfg = WL.SIGN_MUON_WORKLOADS[name]
    M = cfg.workers
    shapes = [cfg.shapes[i] for i in ids]
    L = len(shapes)
    Wd = [torch.from_numpy(w).to(torch.bfloat16).cuda() for w in WL.weights(shapes, cfg.w_init, cfg.w_dtype)]
    gen = torch.Generator(device="cuda").manual_seed(3)
    n_params = sum(r * c for r, c in shapes)
    # two resident gradient sets alternate while they are small; one set (and one
    # workspace) once a set alone is far larger than L2
    n_sets = 2 if n_params * M * 4 <= 4e9 else 1
    Gd = [[torch.randn(s, device="cuda", generator=gen) * cfg.grad_sigma for s in shapes for _ in range(M)]
          for _ in range(n_sets)]
    Md = [torch.zeros(s, device="cuda") for s in shapes for _ in range(M)]
    bits = sign_out == "bits" and not local_polar
    if bits:
        Ud = [S.Bits(torch.zeros(S.packed_words(r * c), dtype=torch.int32, device="cuda"), r, c)
              for r, c in shapes for _ in range(M)]
    else:
        Ud = [torch.zeros(s, dtype=torch.bfloat16, device="cuda") for s in shapes for _ in range(M)]
    Ul = [Ud[l * M:(l + 1) * M] for l in range(L)]
    nbytes = S.smuon_ns_workspace_bytes(Md, cfg.iters, ns_flags)
    wss = [S.workspace(nbytes) for _ in range(n_sets)]
    ns_plans = [S.NsPlan(Md, Ud, *cfg.coeffs, cfg.iters, G=Gd[j], beta=cfg.beta, flags=ns_flags, ws=wss[j])
                for j in range(n_sets)]
    packed = [torch.zeros((M, S.packed_words(r * c)), dtype=torch.int32, device="cuda") for r, c in shapes]
    vote_plan = None
    if bits:
        upd = S.UpdatePlan(Wd, cfg.eta, U=Ul, M=M, tie_value=cfg.tie_value, vote_kind=S.VOTE_POPCOUNT)
        vote_plan = upd
        vote_bytes = n_params * (M / 8 + 2 * 2)

        def tail():
            upd.run()
    elif not local_polar:
        upd = S.UpdatePlan(Wd, cfg.eta, U=Ul, M=M, tie_value=cfg.tie_value, vote_kind=S.VOTE_POPCOUNT,
                           packed_out=packed)
        vote_plan = upd
        vote_bytes = n_params * (M * 2 + 2 * 2 + M / 8)

        def tail():
            upd.run()
    else:
        votes = [torch.zeros(s, dtype=torch.int8, device="cuda") for s in shapes]
        dirs = [torch.zeros(s, device="cuda") for s in shapes]
        # one fused launch for the signs, the packed message and the votes of every layer (no W)
        signs_votes = S.UpdatePlan(None, 0.0, U=Ul, M=M, tie_value=cfg.tie_value, vote_kind=S.VOTE_POPCOUNT,
                                   packed_out=packed, vote_out=votes)
        polar = S.NsPlan(votes, dirs, *cfg.coeffs, cfg.iters, flags=ns_flags)
        upd = S.UpdatePlan(Wd, cfg.eta, dense=dirs)
        vote_bytes = n_params * (M * 2 + M / 8 + 1)

        def tail():
            signs_votes.run()
            polar.run()
            upd.run()
    ws_e2e = S.workspace(nbytes) if e2e else None

    def step(i):
        ns_plans[i % n_sets].run()
        tail()

    def e2e_io():
        hostG = [[g.cpu().pin_memory() for g in Gd[0]]]
        hostW = [torch.empty(w.shape, dtype=torch.bfloat16).pin_memory() for w in Wd]
        return hostG, [torch.empty_like(g) for g in Gd[0]], hostW, Wd

    def e2e_ns(G):
        S.smuon_ns(Md, Ud, *cfg.coeffs, cfg.iters, G=G, beta=cfg.beta, flags=ns_flags, ws=ws_e2e)

    u_bytes = 1 / 8 if bits else 2
    return {"step": step, "graphable": True, "e2e_io": e2e_io if e2e else None, "e2e_ns": e2e_ns, "e2e_tail": tail,
            "g_bytes": n_params * M * 4, "w_bytes": n_params * 2,
            "vote_alone": (vote_plan, vote_bytes) if vote_plan is not None else None,
            "stage_bytes": gemm_stage_bytes(shapes, M, cfg.iters, cfg.coeffs[2], bool(ns_flags & S.NS_SPLIT_BF16),
                                            u_bytes),
            "config": {"layers": L, "params": n_params, "workers": M, "ns_iters": cfg.iters,
                       "vote": "1-bit packed, popcount" + (", local polar step" if local_polar else ""),
                       "ns_output": "1-bit messages from the NS epilogue" if bits else "bf16 U",
                       "payload_bytes_per_worker": {"one_bit": n_params / 8, "int8": n_params, "f32": n_params * 4},
                       "l2": f"inputs larger than L2: {n_params * M * 4 / 1e9:.1f} GB of gradients per step"
                             + (", two resident sets alternate" if n_sets == 2 else "")}}


def setup_c5(S, torch, ids, ns_flags, grad_source="hbm", period=None, beta2=None):
    """GPT-2-Large LionMuon, M = 16, P = 4: three sign steps (vote of the
    workers' sign(G_hat)) and one Muon step (NS of the worker mean) per period.
    Gradients: one resident 45 GB set read every step (each layer's drawn from
    its own seed, so a rank's layers do not depend on the number of ranks), or
    drawn inside the kernels from the counter-based streams (new numbers every
    step)."""
    cfg = WL.LION_MUON_WORKLOADS["c5_gpt2l"]
    P = cfg.period if period is None else period
    b2 = cfg.beta2 if beta2 is None else beta2
    M = cfg.workers
    shapes = [cfg.shapes[i] for i in ids]
    n_params = sum(r * c for r, c in shapes)
    gen = torch.Generator(device="cuda")
    Wd = []
    for i, s in zip(ids, shapes):
        gen.manual_seed(5000 + i)
        Wd.append((torch.randn(s, device="cuda", generator=gen) * 0.02).to(torch.bfloat16))
    mom = [[torch.zeros(s, device="cuda") for _ in range(M)] for s in shapes]
    if grad_source == "hbm":
        G = []
        for i, s in zip(ids, shapes):
            gen.manual_seed(7000 + i)
            G.append([torch.randn(s, device="cuda", generator=gen) for _ in range(M)])
        opt = S.LionMuon(Wd, mom)
    else:
        G = None
        opt = S.LionMuon(Wd, mom, grad=S.GradStream(0, 0, 1.0, 0))
    ws = S.workspace(opt.workspace_bytes(cfg.iters, ns_flags))

    def step(i):
        S.lionmuon_step(opt, G, P, cfg.beta1, b2, cfg.eta, *cfg.coeffs, cfg.iters,
                        tie_value=cfg.tie_value, ns_flags=ns_flags, ws=ws)

    def e2e_steps(n, stream):
        """End to end through lionmuon_step: the workers' gradients drawn inside
        the kernels from the counter-based streams (the simulated workers live on
        the GPU, so no gradient crosses PCIe), and every step's updated weights
        read back into pinned host memory. The read of step i overlaps step
        i + 1: the weights are first copied into one of two device snapshots."""
        opt2 = S.LionMuon(Wd, mom, grad=S.GradStream(0, 0, 1.0, 0))
        flat = [torch.empty(n_params, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        host = torch.empty(n_params, dtype=torch.bfloat16).pin_memory()
        d2h = torch.cuda.Stream()
        ev_snap = [torch.cuda.Event(), torch.cuda.Event()]
        ev_read = [torch.cuda.Event(), torch.cuda.Event()]
        offs = np.cumsum([0] + [r * c for r, c in shapes])
        for _ in range(2):
            S.lionmuon_step(opt2, None, P, cfg.beta1, b2, cfg.eta, *cfg.coeffs, cfg.iters,
                            tie_value=cfg.tie_value, ns_flags=ns_flags, ws=ws)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            b = i & 1
            S.lionmuon_step(opt2, None, P, cfg.beta1, b2, cfg.eta, *cfg.coeffs, cfg.iters,
                            tie_value=cfg.tie_value, ns_flags=ns_flags, ws=ws)
            if i >= 2:
                stream.wait_event(ev_read[b])  # the read of step i - 2 has left this snapshot
            for j, w in enumerate(Wd):
                flat[b][offs[j]:offs[j + 1]].copy_(w.view(-1), non_blocking=True)
            ev_snap[b].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_snap[b])
                host.copy_(flat[b], non_blocking=True)
                ev_read[b].record(d2h)
        stream.wait_event(ev_read[(n - 1) & 1])
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    return {"step": step, "graphable": False, "e2e_io": None, "e2e_run": e2e_steps,
            "g_bytes": 0, "w_bytes": n_params * 2, "period": P,
            "config": {"layers": len(shapes), "params": n_params, "workers": M, "ns_iters": cfg.iters,
                       "period": P, "beta1": cfg.beta1, "beta2": b2, "vote": "1-bit majority on sign steps",
                       "gradients": grad_source,
                       "l2": "inputs larger than L2: 45 GB of EMA (and 45 GB of gradients when read) per step"}}


def rollup(S, recs, peaks, t_peak):
    """Per-kernel time, work and roofline fraction from the library's trace.
    A contraction's rate is the method's nominal flops (2 M N K per product,
    full symmetric products, one product per GEMM in split mode) over its
    event-timed duration, compared with `t_peak`; the tensor cores' issued
    flops are given beside it. A bandwidth-bound kernel's rate is its
    algorithmic bytes over its duration, compared with the HBM copy peak."""
    by, stages = {}, {}
    for r in recs:
        kname = r["name"].split(".")[0]  # stage-qualified names ("k_gemm_tc.axpy") roll up into their kernel
        for key, table in ((kname, by), (r["name"], stages)):
            d = table.setdefault(key, {"ms": 0.0, "work": 0.0, "nominal": 0.0, "n": 0, "kind": r["kind"],
                                       "ms_known": 0.0, "n_known": 0})
            d["ms"] += max(r["ms"], 0.0)
            d["work"] += r["work"]
            d["nominal"] += r["nominal"]
            d["n"] += 1
            if r["work"] > 0:  # launches whose work the library states (a later Lanczos step's is data-dependent)
                d["ms_known"] += max(r["ms"], 0.0)
                d["n_known"] += 1
    kernels = {}
    total_ms = sum(d["ms"] for d in by.values()) or 1.0
    for name, d in by.items():
        secs = d["ms"] / 1e3
        e = {"launches": d["n"], "share": d["ms"] / total_ms, "ms_per_launch": d["ms"] / max(d["n"], 1)}
        if d["kind"] == S.WORK_FLOPS:
            e.update(achieved=d["nominal"] / secs / 1e12 if secs > 0 else 0.0, unit="TFLOP/s",
                     achieved_issued=d["work"] / secs / 1e12 if secs > 0 else 0.0)
            e["frac"] = e["achieved"] / t_peak
            e["frac_issued"] = e["achieved_issued"] / t_peak
        else:
            rated = d["ms"]
            if 0 < d["n_known"] < d["n"]:  # rate only the launches whose bytes are known
                rated = d["ms_known"]
                e["rated_launches"] = d["n_known"]
            e.update(achieved=d["work"] / (rated / 1e3) / 1e9 if rated > 0 else 0.0, unit="GB/s")
            e["frac"] = e["achieved"] / peaks["hbm_gbs"]
        kernels[name] = e
    stage_detail = {k: {"launches": d["n"], "ms_per_launch": d["ms"] / max(d["n"], 1),
                        "tflops_nominal": d["nominal"] / (d["ms"] / 1e3) / 1e12 if d["ms"] > 0 else 0.0,
                        "tflops_issued": d["work"] / (d["ms"] / 1e3) / 1e12 if d["ms"] > 0 else 0.0}
                    for k, d in stages.items() if "." in k}
    return by, kernels, stage_detail


def roofline_of(by, kernels, peaks, peak_src, t_peak, t_peak_name):
    """The dominant kernel (most event-timed time) and its roofline entry."""
    if not by:
        return None
    dom = max(by, key=lambda k: by[k]["ms"])
    kd = kernels[dom]
    tensor = kd["unit"] == "TFLOP/s"
    out = {"bound": "tensor" if tensor else "hbm", "kernel": dom, "achieved": kd["achieved"],
           "peak": t_peak if tensor else peaks["hbm_gbs"], "unit": kd["unit"], "frac": kd["frac"],
           "traffic": load_traffic(dom),
           "peak_source": f"{peak_src} ({t_peak_name if tensor else 'HBM copy'})"}
    if tensor:
        out["work"] = "nominal flops of the method (2MNK per product); issued tensor-core flops beside"
        out["achieved_issued"] = kd["achieved_issued"]
        out["frac_issued"] = kd["frac_issued"]
    return out


def gemm_stage_bytes(shapes, workers, iters, c, split, u_bytes):
    """Algorithmic HBM bytes per launch of each Newton-Schulz GEMM stage
    (averaged over the iterations), from the shapes alone: every operand read
    once, the epilogue's source read and its outputs written once. X is the
    wide m x n form; operands are bf16 (hi and lo parts in split mode); A is
    kept in f32 beside its operand in plain mode and as its hi and lo parts
    alone in split mode, X likewise between steps (4 bytes read back as the
    next step's source either way); the first step's X source is the f32
    momentum, the last step writes U (u_bytes per entry). B's lo part, which a
    plain leading step does not write, is counted as written."""
    op = 4 if split else 2
    tot = {"gram": 0.0, "poly": 0.0, "axpy": 0.0}
    for r, cc in shapes:
        m, n = min(r, cc), max(r, cc)
        for k in range(iters):
            last = k == iters - 1
            # A as f32 plus its operand (split mode: its hi + lo parts alone), or B = b A directly when c = 0
            tot["gram"] += workers * (op * m * n + ((0 if split else 4 * m * m) + op * m * m if c != 0 else op * m * m))
            if c != 0:
                tot["poly"] += workers * (op * m * m + 4 * m * m + op * m * m)
            out = u_bytes * m * n if last else (op if split else 4 + op) * m * n
            tot["axpy"] += workers * (op * m * m + op * m * n + 4 * m * n + out)
    return {k: v / iters for k, v in tot.items()}


def load_traffic(dom):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, valid
    only while the kernel's sources are the ones the counters were taken on."""
    tf = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(tf):
        return None
    try:
        import hashlib
        with open(tf) as f:
            ent = json.load(f).get(dom)
        if not ent:
            return None
        hs = hashlib.sha256()
        for f in ent["sources"]:
            hs.update(open(os.path.join(ROOT, "matrix_aware_sign_b200", "csrc", f), "rb").read())
        return ent["bytes_per_launch"] if hs.hexdigest() == ent["sha256"] else None
    except Exception:
        return None


def ns_flags_for(S, name, args):
    """Newton-Schulz flags of a layer set: split BF16 for five quintic steps (the
    mode that meets the tolerances there), plain BF16 for one step."""
    if args.ns_mode and name == args.workload:
        mode = args.ns_mode
    else:
        mode = "plain" if name in ("c2_resnet50", "resnet18") else "split"
    flags = S.NS_SPLIT_BF16 if mode == "split" else 0
    lead = plain_lead_of(args)
    if mode == "split" and lead:
        flags |= S.ns_plain_lead(lead)
    if args.spectral and name not in WL.LION_MUON_WORKLOADS:
        flags |= S.NS_SPECTRAL
    if args.one_sm:
        flags |= S.NS_ONE_SM
    return mode, flags, lead if mode == "split" else 0


def setup_workload(S, torch, name, ids, ns_flags, args, e2e, headline):
    if name in ("c2_resnet50", "resnet18"):
        return setup_c2(S, torch, ids, ns_flags, e2e, name, args.sign_out if args.sign_out != "bits" else "i8")
    if name == "c3_gpt2s" or name.startswith("llama"):
        sign_out = args.sign_out if headline else "bits"
        return setup_c3(S, torch, ids, ns_flags, e2e and name == "c3_gpt2s", args.local_polar and headline, name,
                        "bits" if sign_out == "bits" else "bf16")
    return setup_c5(S, torch, ids, ns_flags, args.grad_source, args.period, args.beta2)


def time_steps(S, torch, step, steps, warmup, stream, barrier, graph=False):
    """W untimed steps, then exactly `steps` steps between CUDA events on the
    launching stream, bracketed by a barrier and a device synchronisation on
    both sides. Returns (ms, trace records, launches, wall-clock window)."""
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    g = None
    if graph:
        g = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
        side = torch.cuda.Stream()
        with torch.cuda.stream(side):
            for j in range(2):
                with torch.cuda.graph(g[j], stream=side):
                    step(j)
        torch.cuda.synchronize()
    S.trace_enable(g is None)
    n0 = S.launch_count()
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(steps):
        if g is not None:
            g[i & 1].replay()
        else:
            step(warmup + i)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    t1 = time.perf_counter()
    launches = S.launch_count() - n0
    S.trace_enable(False)
    recs = S.trace_read()
    return ev0.elapsed_time(ev1), recs, launches, (t0, t1), g


def graph_rate(torch, step, steps, stream):
    """The same step replayed as a CUDA graph (launch overhead removed)."""
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
    for i in range(steps):
        g2[i & 1].replay()
    q1.record(stream)
    torch.cuda.synchronize()
    return steps / (q0.elapsed_time(q1) / 1000.0)


def e2e_copy_loop(torch, wl, n, stream, barrier):
    """End to end through the public calls with host buffers: every step copies
    its gradients from pinned host memory and reads the updated weights back;
    the copies run on their own streams, double-buffered, so that step i+1's
    gradients cross PCIe while step i computes and step i's weights come back
    while step i+1's Newton-Schulz runs."""
    hostG, devG0, hostW, Wd = wl["e2e_io"]()
    devG = [devG0, [torch.empty_like(g) for g in devG0]]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev_copied = [torch.cuda.Event(), torch.cuda.Event()]
    ev_free = [torch.cuda.Event(), torch.cuda.Event()]
    ev_done, ev_read = torch.cuda.Event(), torch.cuda.Event()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h2d.wait_stream(stream)
    with torch.cuda.stream(h2d):
        for d, hg in zip(devG[0], hostG[0]):
            d.copy_(hg, non_blocking=True)
        ev_copied[0].record(h2d)
    for i in range(n):
        b = i & 1
        if i + 1 < n:
            with torch.cuda.stream(h2d):
                if i >= 1:
                    h2d.wait_event(ev_free[1 - b])  # step i-1's Newton-Schulz has read that buffer
                for d, hg in zip(devG[1 - b], hostG[(i + 1) % len(hostG)]):
                    d.copy_(hg, non_blocking=True)
                ev_copied[1 - b].record(h2d)
        stream.wait_event(ev_copied[b])
        wl["e2e_ns"](devG[b])
        ev_free[b].record(stream)
        if i >= 1:
            stream.wait_event(ev_read)  # step i-1's weights are on the host before W changes again
        wl["e2e_tail"]()
        ev_done.record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_done)
            for hw, d in zip(hostW, Wd):
                hw.copy_(d, non_blocking=True)
            ev_read.record(d2h)
    stream.wait_event(ev_read)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1)


def vote_alone(torch, wl, peaks, stream):
    """The fused vote / update kernel of a layer set timed alone (burst), next
    to its in-step rate, which runs at the clocks the tensor-core stages leave
    under the power cap."""
    plan, vb = wl["vote_alone"]
    for _ in range(3):
        plan.run()
    torch.cuda.synchronize()
    v0 = torch.cuda.Event(enable_timing=True)
    v1 = torch.cuda.Event(enable_timing=True)
    v0.record(stream)
    for _ in range(20):
        plan.run()
    v1.record(stream)
    torch.cuda.synchronize()
    vms = v0.elapsed_time(v1) / 20
    return {"ms_per_call": vms, "gbs": vb / (vms / 1e3) / 1e9, "frac_of_hbm": vb / (vms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "bytes_per_call": vb}


def measure_set(S, torch, name, ids, args, peaks, peak_src, stream, barrier, world, steps, warmup, headline,
                sampler=None):
    """Sets up a layer set and times it; returns the pieces of a bench entry."""
    ns_mode, ns_flags, lead = ns_flags_for(S, name, args)
    desc = describe(name, ns_mode, args.local_polar and headline, args.spectral and name not in WL.LION_MUON_WORKLOADS,
                    lead, args.sign_out if headline else ("bits" if name == "c3_gpt2s" else "i8"))
    e2e_on = headline and args.e2e_steps > 0
    wl = setup_workload(S, torch, name, ids, ns_flags, args, e2e_on, headline)
    ms, recs, launches, (tw0, tw1), graph = time_steps(S, torch, wl["step"], steps, warmup, stream, barrier,
                                                       graph=headline and args.graph and wl["graphable"])
    ms = reduce_max(ms, world, device="cuda")
    region_s = ms / 1e3
    t_peak, t_peak_name = tensor_peak(peaks, region_s)
    by, kernels, stage_detail = rollup(S, recs, peaks, t_peak)
    if "stage_bytes" in wl:  # the GEMM stages of small matrices move bytes more than flops: their HBM view
        for sname, d in stage_detail.items():
            b = wl["stage_bytes"].get(sname.split(".")[1])
            if b and d["ms_per_launch"] > 0:
                d["gbs_algorithmic"] = b / (d["ms_per_launch"] / 1e3) / 1e9
                d["frac_of_hbm"] = d["gbs_algorithmic"] / peaks["hbm_gbs"]
    entry = {"workload": desc["workload"] + (f"_first_{args.layers}_matrices" if args.layers > 0 else ""),
             "value": layer_set_rate(steps, ms), "unit": "steps/s", "steps": steps, "warmup": warmup,
             "ms_per_step": ms / steps, "timed_region_s": region_s, "ns_mode": ns_mode,
             "roofline": roofline_of(by, kernels, peaks, peak_src, t_peak, t_peak_name),
             "kernels": kernels, "gemm_stages": stage_detail, "config": wl["config"]}
    if sampler is not None:
        entry["clocks"] = sampler.summary(tw0, tw1)
    ns = [k for k in kernels if k.startswith("k_gemm")]
    if ns:
        fl = sum(by[k]["work"] for k in ns)
        nom = sum(by[k]["nominal"] for k in ns)
        t = sum(by[k]["ms"] for k in ns) / 1e3
        entry["ns_tflops_nominal"] = nom / t / 1e12
        entry["ns_frac_of_peak"] = entry["ns_tflops_nominal"] / t_peak
        entry["ns_tflops_issued"] = fl / t / 1e12
        entry["ns_peak"] = f"{peak_src} {t_peak_name}"
    vk = [k for k in kernels if k.startswith("k_vote_update") or k == "k_lion_sign"]
    if vk:
        entry["vote_kernel"] = vk[0]
        entry["vote_gbs"] = kernels[vk[0]]["achieved"]
        entry["vote_frac_of_hbm"] = kernels[vk[0]]["frac"]
    if wl.get("vote_alone") and world == 1:
        entry["vote_alone"] = vote_alone(torch, wl, peaks, stream)
    return wl, entry, launches, graph, desc


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
    peaks, peak_src = load_peaks()
    if args.cachemuon is not None:
        cases = args.cachemuon or [f"{r}x{c}:{g}" for (r, c) in ((4096, 4096), (8192, 8192), (4096, 16384))
                                   for g in (2, 15)]
        for case in cases:
            shp, gam = case.split(":")
            r, c = (int(x) for x in shp.split("x"))
            print(json.dumps(run_cachemuon(S, torch, (r, c), float(gam), args.steps, gram_only=args.gram_only,
                                           diagnose=args.diagnose, drift=args.drift, one_sm=args.one_sm)),
                  flush=True)
        return
    if args.only_ns4096:
        flags = S.NS_SPLIT_BF16 if (args.ns_mode or "split") == "split" else 0
        if flags and args.plain_lead:
            flags |= S.ns_plain_lead(args.plain_lead)
        if args.one_sm:
            flags |= S.NS_ONE_SM
        print(json.dumps({"ns_4096sq_quintic5": measure_ns_square(S, torch, peaks, 4096, 5, flags,
                                                                   reps=args.steps)}))
        return
    if args.spectral and args.workload == "c5_gpt2l":
        raise SystemExit("--spectral applies to the Sign-Muon sets")
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    _SPECTRAL[0] = args.spectral
    stream = torch.cuda.current_stream()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)

    # --- the 4096^2 solve first: it is a burst of a few ms compared with the burst peak, so it is timed before
    # the long workloads heat the GPU into its power cap
    extras_on = args.extras and world == 1 and args.layers <= 0 and args.workload == WORKLOAD
    ns4096 = None
    if extras_on:
        ns4096 = {  # the mode that meets the criteria fastest first
            "split_bf16_plain_lead2": measure_ns_square(S, torch, peaks, 4096, 5,
                                                        S.NS_SPLIT_BF16 | S.ns_plain_lead(2)),
            "split_bf16": measure_ns_square(S, torch, peaks, 4096, 5, S.NS_SPLIT_BF16),
            "plain_bf16": measure_ns_square(S, torch, peaks, 4096, 5, 0),
            "split_bf16_plain_lead2_one_sm": measure_ns_square(S, torch, peaks, 4096, 5,
                                                               S.NS_SPLIT_BF16 | S.ns_plain_lead(2) | S.NS_ONE_SM),
            "note": "timed alone, before the other workloads: compared with the burst peak; plain BF16 misses the "
                    "sign criterion at five quintic steps, split BF16 (also with two plain leading steps) meets "
                    "it; SM pairs (256x256 tiles) unless the key says one_sm (128x256 tiles on single SMs)"}
        torch.cuda.empty_cache()

    # --- headline: this rank's share of the layer set
    ids = rank_layers(args.workload, args.layers, rank, world)
    wl, head, launches, graph, desc = measure_set(S, torch, args.workload, ids, args, peaks, peak_src, stream,
                                                  barrier, world, args.steps, args.warmup, True, sampler)
    if graph is not None:
        launches = launches or 8 * args.steps  # graph replays launch the captured kernels
    graph_value = None
    if graph is None and args.graph_compare and world == 1 and wl["graphable"]:
        graph_value = graph_rate(torch, wl["step"], args.steps, stream)

    # --- end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0 and wl.get("e2e_run") is not None:
        ems = reduce_max(wl["e2e_run"](args.e2e_steps, stream), world, device="cuda")
        e2e = {"value": layer_set_rate(args.e2e_steps, ems), "unit": "steps/s",
               "h2d_bytes_per_step": wl["g_bytes"], "d2h_bytes_per_step": wl["w_bytes"],
               "note": "lionmuon_step with the simulated workers' gradients drawn inside the kernels from their "
                       "counter-based streams (no gradient input crosses PCIe); every step's bf16 weights are read "
                       "back into pinned host memory, overlapping the next step"}
    elif args.e2e_steps > 0 and wl.get("e2e_io") is not None:
        ems = reduce_max(e2e_copy_loop(torch, wl, args.e2e_steps, stream, barrier), world, device="cuda")
        e2e = {"value": layer_set_rate(args.e2e_steps, ems), "unit": "steps/s",
               "h2d_bytes_per_step": wl["g_bytes"], "d2h_bytes_per_step": wl["w_bytes"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample = oracle_rate(args.workload, 15.0)
        cpu = {"value": v, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle", "sample": sample}

    # --- the other layer sets and the 4096^2 solve, each timed alone with its own roofline (one GPU)
    extra = {}
    if extras_on:
        del wl
        torch.cuda.empty_cache()
        for name, steps, warm in (("c2_resnet50", 200, 20), ("c3_gpt2s", 20, 5)):
            ids_x = rank_layers(name, 0, 0, 1)
            wlx, ex, _, _, _ = measure_set(S, torch, name, ids_x, args, peaks, peak_src, stream, barrier, 1,
                                           steps, warm, False, sampler)
            extra[name] = ex
            del wlx
            torch.cuda.empty_cache()
        extra["ns_4096sq_quintic5"] = ns4096
    sampler.stop()

    if rank == 0:
        config = {"workload": head["workload"], **head["config"], "ns_mode": head["ns_mode"],
                  "global_batch": None, "seq_len": None,
                  "parallelism": "by layer" + (f" over {world} ranks" if world > 1 else ""),
                  "launch": "cuda_graph" if graph is not None else "eager"}
        line = {
            "metric": "Muon steps/s per layer set", "value": head["value"], "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": desc["data"], "config": config, "roofline": head["roofline"],
            "timed_region_s": head["timed_region_s"], "kernels": head["kernels"],
            "gemm_stages": head["gemm_stages"],
            **{k: head[k] for k in ("ns_tflops_nominal", "ns_frac_of_peak", "ns_tflops_issued", "ns_peak",
                                    "vote_kernel", "vote_gbs", "vote_frac_of_hbm", "vote_alone") if k in head},
            "steps_per_s_cuda_graph": graph_value,
            "clocks": head.get("clocks"), "e2e": e2e,
            "gpu_launches": launches, "cpu_baseline": cpu,
            "extra": extra or None,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
