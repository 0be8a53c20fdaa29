#!/usr/bin/env python
"""Throughput of the partial-recompute denoising step on B200.

Workload: one 8B-shape bidirectional layer (d=4096, 32 heads x 128, SwiGLU
F=12288), N=1024 tokens, batch 1, active fraction M/N = 0.25 (256 rows), as in
the SureLock page's setting ("Stopping Computation for Converged Tokens in
Masked Diffusion-LM Decoding", Sec. 4: LLaDA-8B).  One step is the whole hot
path: S1 drift score (rank-128 singular proxy, L2), S2/S3 top-k selection and
compaction, S4-S10 partial layer step, S10 proxy refresh.  The 256 perturbed
rows are exactly the ones the top-k picks; the proxy cache is restored between
steps (untimed) so that every step does the same work.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl plk|reference]

Prints one JSON line (rank 0).  --impl reference times the CPU oracle instead.
Multi-GPU: one process per GPU under torchrun; every rank runs its own
replica (independent sequences, no collective on the data path), time is the
max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "active-token-layers/sec at 8B-shape, M/N=0.25; % of bf16 tensor peak"
UNIT = "active-token-layers/s"
PROFILE_TXT = os.path.join(ROOT, "profiles", "gemm_tc_8b_quarter.txt")
GEMM_SRC = os.path.join(ROOT, "partial_recompute_kv_b200", "csrc", "gemm_tc.cu")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# workload (seeded synthetic inputs shared by both arms)
# ---------------------------------------------------------------------------
class Workload:
    def __init__(self, frac=0.25, rank=128, seed=0, share=None):
        """share: another Workload of the same seed and rank whose weights, X and U are reused."""
        import synth
        self.D = synth.LAYER_8B
        self.frac, self.r = frac, rank
        self.M = synth.active_count(self.D.N, frac)
        if share is not None:
            self.W, self.X, self.Ut = share.W, share.X, share.Ut
        else:
            self.W = synth.layer_weights(self.D, synth.LAYER_8B_WSTD, seed=seed)
            self.X = synth.hidden_states(self.D, seed=seed)
            self.Ut = synth.proxy_basis(self.D.d, rank, seed=seed)
        self.pos = synth.layer_8b_positions(self.D.N, frac, seed=seed)
        mask = np.zeros((self.D.B, self.D.N), bool)
        mask[0, self.pos] = True
        noise = synth.step_noise((self.D.B, self.D.N, self.D.d), 0.01, seed=seed)
        self.Xp = synth.perturb_rows(self.X, noise, mask, "bf16")

    def flops_per_row(self):
        D = self.D
        return 8 * D.d * D.d + 6 * D.d * D.F + 4 * D.N * D.d

    def gemm_flops_per_row(self):
        D = self.D
        return 8 * D.d * D.d + 6 * D.d * D.F

    def weight_bytes(self):
        D = self.D
        return 2 * (4 * D.d * D.d + 3 * D.d * D.F)

    def gemm_bytes(self):
        """Algorithmic DRAM bytes of the four projections of one step: every weight once, the
        activations read once as bf16, the fp32 sums written once."""
        D, M = self.D, self.M
        return self.weight_bytes() + M * (2 * (3 * D.d + D.F) + 4 * (5 * D.d + 2 * D.F))

    def config(self, l2="stream"):
        D = self.D
        return {"workload": (f"single 8B-shape layer, d={D.d}, {D.H} heads x {D.hd}, SwiGLU F={D.F}, "
                             f"N={D.N}, batch {D.B}, M/N={self.frac} ({self.M} active rows); step = drift "
                             f"score (rank-{self.r} proxy, L2) + top-k select + partial layer step + "
                             f"proxy refresh"),
                "B": D.B, "N": D.N, "d": D.d, "heads": D.H, "head_dim": D.hd, "F": D.F,
                "active_rows": self.M, "proxy_rank": self.r,
                "l2": ("flushed before every timed step (256 MiB write)" if l2 == "flush" else
                       f"not flushed: inputs larger than L2 -- every step streams the layer's "
                       f"{self.weight_bytes() / 2**20:.0f} MiB of weights through the 126 MB L2"),
                "inputs": "resident in HBM for value; host pinned buffers for e2e"}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------
def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except Exception:
        return dict(FALLBACK_PEAKS)


def gemm_traffic_per_launch():
    """dram read+write bytes per GEMM launch from the committed ncu summary, or None
    when the summary is missing or was taken on a different kernel source."""
    try:
        src_hash = hashlib.sha256(open(GEMM_SRC, "rb").read()).hexdigest()[:16]
        kv = {}
        for line in open(PROFILE_TXT):
            if ":" in line:
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if kv.get("kernel_source_sha256_16") != src_hash:
            return None
        return float(kv["dram_bytes_per_launch_avg"])
    except Exception:
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    def __init__(self, device_index, period=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop = period, threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            pass

    def _run(self):
        nv = self.nv
        names = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
                 "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for n, bit in names.items():
                    if r & bit:
                        self.reasons.add(n)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def aggregate(dist, value_local, device=None):
    """Max of a float over ranks (identity when not distributed)."""
    if dist is None or not dist.is_initialized():
        return value_local
    import torch
    t = torch.tensor([value_local], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline of the GPU arm, and the reference arm)
# ---------------------------------------------------------------------------
class OracleRunner:
    """The CPU oracle on the same workload: caches from a full step (untimed), then
    partial steps.  A step on `rows` active rows is a complete partial-recompute
    step with that active set (S1 for all N rows, S2 top-k, S3, S4-S10, proxy refresh)."""

    def __init__(self, wl):
        import oracle
        self.o, self.wl = oracle, wl
        D = wl.D
        self.base = oracle.full_layer_step(D, wl.W, wl.X, "bf16")
        x = wl.X.reshape(-1, D.d).astype(np.float64)
        self.pc = oracle.to_f32(oracle.proxy_project(x, wl.Ut.astype(np.float64))).reshape(D.B, D.N, -1)
        self.Utd = wl.Ut.astype(np.float64)

    def step(self, rows):
        o, wl, D = self.o, self.wl, self.wl.D
        # only the chosen `rows` of the perturbed positions differ from the cached proxies
        keep = np.zeros((D.B, D.N), bool)
        keep[0, wl.pos[:rows]] = True
        Xs = np.where(keep[..., None], wl.Xp, wl.X)
        score, p = o.score_drift(Xs.astype(np.float64), self.Utd, self.pc, "l2")
        lock = o.lock_topk(score, np.zeros((D.B, D.N), np.uint8), rows, True)
        idx, seg = o.compact(lock)
        o.layer_step_partial(D, wl.W, Xs, idx, seg, self.base, "bf16")
        o.proxy_commit(self.pc, p, idx)
        return int(idx.size)


def run_reference(args, wl):
    cfg = wl.config(args.l2)
    run = OracleRunner(wl)
    # complete steps of the workload itself (all wl.M active rows) when they fit the budget
    # (about 150 s for the whole run); otherwise steps on fewer rows, said so in `sample`
    t0 = time.perf_counter()
    run.step(wl.M)
    t_full = time.perf_counter() - t0
    budget = 150.0
    n_steps = max(args.steps + args.warmup, 1)
    rows = wl.M if n_steps * t_full <= budget else int(max(1, wl.M * budget / (n_steps * t_full)))
    for _ in range(args.warmup):
        run.step(rows)
    t0 = time.perf_counter()
    units = 0
    for _ in range(args.steps):
        units += run.step(rows)
    el = time.perf_counter() - t0
    value = units / el
    sample = (f"{args.steps} complete oracle steps of this workload ({rows} active rows each)" if rows == wl.M else
              f"{args.steps} oracle steps of the same layer and cache state with {rows} of the "
              f"{wl.M} active rows per step (complete partial steps at that active count)")
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline(wl, budget_s=15.0, run=None):
    run = run or OracleRunner(wl)
    t0 = time.perf_counter()
    units, steps = 0, 0
    while True:
        units += run.step(wl.M)
        steps += 1
        if time.perf_counter() - t0 > budget_s or steps >= 20:
            break
    el = time.perf_counter() - t0
    return {"value": units / el, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{steps} complete oracle steps of this workload ({wl.M} active rows each), "
                      f"caches from an untimed oracle full step"}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_gpu(args, wl, dist, rank, world, local_rank):
    import torch
    import partial_recompute_kv_b200 as plk

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    D, r, M = wl.D, wl.r, wl.M
    bf = torch.bfloat16
    up = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(dt)
    dm = plk.dims(D.B, D.N, D.d, D.H, D.hd, D.F, D.eps, plk.BF16)
    W = {k: up(v, bf) for k, v in wl.W.items()}
    pw = plk.weights(W)
    X, Xp, Ut = up(wl.X, bf), up(wl.Xp, bf), up(wl.Ut, bf)
    K = torch.zeros((D.B, D.N, D.d), dtype=bf, device=dev)
    V, Y = torch.zeros_like(K), torch.zeros_like(K)
    ws = plk.alloc_workspace(dm, device=dev)
    score = torch.empty((D.B, D.N), dtype=torch.float32, device=dev)
    pnew = torch.empty((D.B, D.N, r), dtype=torch.float32, device=dev)
    pc = torch.zeros_like(pnew)
    lock_in = torch.zeros((D.B, D.N), dtype=torch.uint8, device=dev)
    lock = torch.empty_like(lock_in)
    idx = torch.empty(D.B * D.N, dtype=torch.int32, device=dev)
    seg = torch.empty(D.B + 1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if args.l2 == "flush" else None

    # state: caches from a full step on X, cached proxies of X
    plk.full_layer_step(dm, pw, X, K, V, Y, ws)
    plk.score_drift(dm, X, Ut, r, pc, plk.METRIC_L2, score, proxy_out=pnew)
    pc0 = pnew.clone()
    pc.copy_(pc0)

    sws = plk.alloc_step_workspace(dm, r, device=dev)
    lock_s = torch.zeros_like(lock_in)  # the whole-step call locks in place

    def step(xin):  # one call: score, select, layer step with the proxy refresh folded in
        plk.denoise_step(dm, pw, Ut, r, plk.METRIC_L2, plk.SEL_TOPK_LARGEST, 0.0, M, pc, lock_s, K, V, Y, xin, sws)

    def prep():
        pc.copy_(pc0)
        lock_s.zero_()
        if flush is not None:
            flush.zero_()

    prep()
    step(Xp)
    st = plk.get_status()
    if st != plk.OK:
        raise RuntimeError(f"device status {plk.error_string(st)}")
    got = np.flatnonzero(lock_s.cpu().numpy().reshape(-1) == 0)
    if got.size != M or not np.array_equal(got, np.sort(wl.pos)):
        raise RuntimeError("the top-k did not select the perturbed rows")
    if args.profile:
        for _ in range(args.steps):
            prep()
            step(Xp)
        torch.cuda.synchronize()
        return None
    for _ in range(args.warmup):
        prep()
        step(Xp)
    torch.cuda.synchronize()

    K_ = args.steps
    E = lambda: torch.cuda.Event(enable_timing=True)
    ev = [(E(), E()) for _ in range(K_)]
    if dist is not None:
        dist.barrier(device_ids=[local_rank])
    torch.cuda.synchronize()
    graph = None
    if args.graph:
        # the whole step (score, select, layer step, commit) as one CUDA graph: every call is
        # capture-safe (no allocation, no host synchronisation, launch attributes kept)
        graph = torch.cuda.CUDAGraph()
        prep()
        with torch.cuda.graph(graph):
            step(Xp)
        torch.cuda.synchronize()
        for _ in range(3):
            prep()
            graph.replay()
        torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        h0 = time.perf_counter()
        for i in range(K_):
            prep()
            ev[i][0].record()
            if graph is not None:
                graph.replay()
            else:
                step(Xp)
            ev[i][1].record()
        h1 = time.perf_counter()
        torch.cuda.synchronize()
    host_us = (h1 - h0) / K_ * 1e6
    if dist is not None:
        dist.barrier(device_ids=[local_rank])
    st = plk.get_status()
    if st != plk.OK:
        raise RuntimeError(f"device status {plk.error_string(st)}")
    step_ms = [a.elapsed_time(b) for a, b in ev]

    # per-kernel breakdown: separate, untimed-for-value steps with an event between
    # every kernel (the events themselves add a little time to each gap)
    nb = min(K_, 20)
    bev = [[E() for _ in range(15)] for _ in range(nb)]  # 0 start, 1 score, 2 select, 3..13 layer, 14 end
    for i in range(nb):
        prep()
        e = bev[i]
        plk.trace_events(e[3:14])
        e[0].record()
        plk.score_drift(dm, Xp, Ut, r, pc, plk.METRIC_L2, score, proxy_out=pnew)
        e[1].record()
        plk.select_active(dm, score, lock_in, lock, plk.SEL_TOPK_LARGEST, 0.0, M, idx, seg)
        e[2].record()
        plk.layer_step_partial(dm, pw, Xp, idx, seg, K, V, Y, ws)
        plk.proxy_commit(dm, r, idx, seg, pnew, pc)
        e[14].record()
    torch.cuda.synchronize()
    plk.trace_events([])
    names = ["score", "select", "rmsnorm1", "gemm_qkv", "finish_qkv", "attention", "gemm_o", "rmsnorm2",
             "gemm_gu", "finish_gu", "gemm_down", "finish_y", "proxy_commit"]
    bounds = [(0, 1), (1, 2)] + [(i, i + 1) for i in range(3, 14)]
    per = {n: statistics.mean(e[a].elapsed_time(e[b]) for e in bev) * 1e3 for n, (a, b) in zip(names, bounds)}
    per["traced_step"] = statistics.mean(e[0].elapsed_time(e[14]) for e in bev) * 1e3
    total_ms = sum(step_ms)
    total_ms_max = aggregate(dist, total_ms, dev)
    ms_per_step = total_ms_max / K_
    value = world * M * K_ / (total_ms_max / 1e3)

    # roofline of the dominant kernel: the tcgen05 GEMM (4 launches per step)
    pk = peaks()
    gemm_us = per["gemm_qkv"] + per["gemm_o"] + per["gemm_gu"] + per["gemm_down"]
    gemm_flops_launch = M * wl.gemm_flops_per_row() / 4
    achieved = gemm_flops_launch / (gemm_us / 4 * 1e-6) / 1e12
    peak = float(pk["bf16_tflops"])
    traffic = gemm_traffic_per_launch()
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "kernel": "gemm_tc_kernel",
                "launches_per_step": 4, "peak_source": f"{pk.get('source')} bf16_tflops (burst)",
                "frac_of_sustained": achieved / float(pk.get("bf16_tflops_sustained", peak)),
                "issued_frac": 2 * achieved / peak,
                "issued_note": "the activations enter as bf16 hi/lo pairs: the tensor cores issue twice the "
                               "algorithmic FLOP"}

    # the memory-bound kernels: algorithmic bytes / traced time against the measured HBM copy rate
    d_, F_, r_, BN = D.d, D.F, r, D.B * D.N
    alg_bytes = {"score": 2 * BN * d_ + 8 * BN * r_ + 2 * d_ * r_,
                 "select": 6 * BN + 4 * M,
                 # x in (bf16), the hi/lo pair and the fp32 residual out
                 "rmsnorm1": 10 * M * d_,
                 # the fp32 q, k and v sums in, q as a hi/lo pair and the K/V rows (bf16) out
                 "finish_qkv": 20 * M * d_,
                 "rmsnorm2": 8 * M * d_,  # h in (fp32), the hi/lo pair out
                 "finish_gu": 12 * M * F_,  # gate and up sums in, silu(g) u as a hi/lo pair out
                 "finish_y": 6 * M * d_, "proxy_commit": 8 * M * r_}
    hbm = float(pk["hbm_gbs"])
    hbm_kernels = {k: {"bytes": v, "GB/s": v / (per[k] * 1e-6) / 1e9, "frac": v / (per[k] * 1e-6) / 1e9 / hbm}
                   for k, v in alg_bytes.items()}

    # e2e through the public API with host buffers, every step's X copied in from pinned host memory
    # and its output cache Y copied back out inside the timed region.  Headline: one
    # plk_denoise_steps_host call over e2e_steps consecutive steps (step t + 1's upload and step
    # t's download run on two copy streams while the neighbouring steps compute).  Also reported:
    # the same steps as one plk_denoise_step_host call each (copies in line with the compute).
    e2e_steps = min(K_, 50)
    Xp_host = torch.from_numpy(np.ascontiguousarray(wl.Xp)).to(bf).pin_memory()
    Y_pair = [torch.empty(Y.shape, dtype=bf).pin_memory() for _ in range(2)]
    lock_e = torch.empty_like(lock_in)
    ee = [(E(), E()) for _ in range(e2e_steps)]
    torch.cuda.synchronize()
    for i in range(e2e_steps):
        prep()
        lock_e.zero_()
        ee[i][0].record()
        plk.denoise_step_host(dm, pw, Ut, r, plk.METRIC_L2, plk.SEL_TOPK_LARGEST, 0.0, M, pc, lock_e, K, V, Y,
                              Xp_host, Y_pair[i & 1], sws)
        ee[i][1].record()
    torch.cuda.synchronize()
    if plk.get_status() != plk.OK:
        raise RuntimeError("device status after the host-buffer steps")
    single_ms = aggregate(dist, sum(a.elapsed_time(b) for a, b in ee), dev) / e2e_steps
    # pipelined: the first step of the call selects the M rows (top-M of N), the later ones keep
    # those M rows (the only unlocked candidates, k = M): every step recomputes M rows
    mws = plk.alloc_steps_workspace(dm, r, device=dev)
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    X_hosts = [Xp_host] * e2e_steps
    Y_hosts = [Y_pair[t & 1] for t in range(e2e_steps)]

    def steps_call(T):
        prep()
        lock_e.zero_()
        plk.denoise_steps_host(dm, pw, Ut, r, plk.METRIC_L2, plk.SEL_TOPK_LARGEST, 0.0, M, pc, lock_e, K, V, Y,
                               X_hosts[:T], Y_hosts[:T], mws, up, down)

    steps_call(3)  # warm-up
    torch.cuda.synchronize()
    pa, pb = E(), E()
    with ClockSampler(local_rank) as clk_e2e:  # a short run: its clocks may differ from the value's
        pa.record()
        steps_call(e2e_steps)
        pb.record()
        torch.cuda.synchronize()
    if plk.get_status() != plk.OK:
        raise RuntimeError("device status after the pipelined host-buffer steps")
    if int((lock_e == 0).sum()) != M:
        raise RuntimeError("the pipelined steps did not keep M active rows")
    e2e_ms = aggregate(dist, pa.elapsed_time(pb), dev) / e2e_steps
    e2e = {"value": world * M / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": Xp_host.numel() * Xp_host.element_size(),
           "d2h_bytes_per_step": Y_pair[0].numel() * Y_pair[0].element_size(), "ms_per_step": e2e_ms,
           "api": f"plk_denoise_steps_host over {e2e_steps} consecutive steps (host X in, host Y out every "
                  "step; the copies overlap the neighbouring steps' compute)", "clocks": clk_e2e.summary(),
           "single_call_per_step": {"value": world * M / (single_ms / 1e3), "ms_per_step": single_ms,
                                    "api": "plk_denoise_step_host, one call per step (copies in line)"}}
    step_flops = M * wl.flops_per_row()
    return {"value": value, "ms_per_step": ms_per_step, "per_kernel_us": per, "roofline": roofline,
            "host_enqueue_us_per_step": host_us, "hbm_kernels": hbm_kernels,
            "ms_per_step_median": statistics.median(step_ms),
            "e2e": e2e, "clocks": clk.summary(), "step_tflops": step_flops / (ms_per_step * 1e-3) / 1e12,
            "peaks": pk}


# ---------------------------------------------------------------------------
# the KL lock rule (SureLock's locking condition) on its own: not part of the
# headline step, measured with --kernel kl_lock
# ---------------------------------------------------------------------------
def run_kl_lock(args):
    import torch
    import partial_recompute_kv_b200 as plk
    import oracle
    import synth

    B, N, V, M = 1, 1024, synth.VOCAB_8B, 256
    dev = torch.device("cuda", 0)
    zt, zp = synth.logits_pair(B, N, V, seed=0, drift=(0.0, 0.3), dtype="bf16")
    lock0 = np.ones((B, N), np.uint8)
    lock0[0, synth.layer_8b_positions(N, M / N)] = 0
    bf = torch.bfloat16
    Zt = torch.from_numpy(zt).to(dev).to(bf)
    Zp = torch.from_numpy(zp).to(dev).to(bf)
    lk0 = torch.from_numpy(lock0).to(dev)
    lk = torch.empty_like(lk0)
    kl = torch.empty((B, N), dtype=torch.float32, device=dev)
    dm = plk.dims(B, N, 256, 2, 128, 512, dtype=plk.BF16)
    eps = 1e-3
    call = lambda: plk.kl_lock(dm, V, Zt, Zp, lk0, lk, eps, math.inf, kl_out=kl)
    for _ in range(max(args.warmup, 3)):
        call()
    torch.cuda.synchronize()
    E = lambda: torch.cuda.Event(enable_timing=True)
    ev = [(E(), E()) for _ in range(args.steps)]
    with ClockSampler(0) as clk:
        for a, b in ev:
            a.record()
            call()
            b.record()
        torch.cuda.synchronize()
    st = plk.get_status()
    if st != plk.OK:
        raise RuntimeError(f"device status {plk.error_string(st)}")
    us = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3
    pk = peaks()
    alg = 2 * M * V * 2  # both steps' bf16 logits of the active rows, read once
    gbs = alg / (us * 1e-6) / 1e9
    # cpu baseline: the oracle on 8 of the active rows
    rows = np.flatnonzero(lock0[0] == 0)[:8]
    t0 = time.perf_counter()
    oracle.kl_lock(zt[:, rows], zp[:, rows], np.zeros((1, rows.size), np.uint8), eps)
    cpu_s = time.perf_counter() - t0
    line = {"metric": "KL-lock rows/s (8B vocabulary, bf16 logits)", "value": M / (us * 1e-6),
            "unit": "rows/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "us_per_call": us,
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"kl_lock, B={B}, N={N}, V={V}, {M} active rows, eps={eps}, gate off"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": float(pk["hbm_gbs"]), "unit": "GB/s",
                         "frac": gbs / float(pk["hbm_gbs"]), "traffic": None,
                         "kernel": "kl_lock_kernel", "alg_bytes_per_call": alg},
            "clocks": clk.summary(),
            "cpu_baseline": {"value": rows.size / cpu_s, "unit": "rows/s", "cores": os.cpu_count(),
                             "kind": "oracle", "sample": f"{rows.size} active rows of the same workload"}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# kernels at the configurations where their rooflines are judged (not the
# headline): scoring at the 8 x 4096 scoring shape (HBM-bound), and the layer
# step with every row active at B = 4, N = 2048 (step 0 of the 32-layer stack:
# compute-bound GEMMs and attention, the K/V scatter kernel moving 671 MB)
# ---------------------------------------------------------------------------
def _timed(torch, fn, steps, warmup):
    """Device time of one call of fn: `reps` calls captured in a CUDA graph (so host launch
    time is not measured), the graph replayed with events around every replay; median."""
    for _ in range(max(warmup, 3)):
        fn()
    torch.cuda.synchronize()
    reps = max(1, min(steps, 20))
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for _ in range(reps):
            fn()
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    E = lambda: torch.cuda.Event(enable_timing=True)
    ev = [(E(), E()) for _ in range(max(3, steps // reps))]
    for a, b in ev:
        a.record()
        graph.replay()
        b.record()
    torch.cuda.synchronize()
    del graph
    return statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3 / reps


def run_kernel_configs(args, scoring_only=False):
    import torch
    import partial_recompute_kv_b200 as plk
    import synth

    clk = ClockSampler(0).__enter__()  # SM clock and throttle reasons over every config below

    dev = torch.device("cuda", 0)
    bf = torch.bfloat16
    pk = peaks()
    hbm, tfl = float(pk["hbm_gbs"]), float(pk["bf16_tflops"])
    up = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(dt)
    out = []
    # scoring shape: X [8, 4096, 4096] bf16, rank 128, L2; top-k 10% per sequence
    D, r = synth.SCORE_8B, synth.PROXY_RANK_8B
    dm = plk.dims(D.B, D.N, D.d, D.H, D.hd, D.F, D.eps, plk.BF16)
    X = torch.randn((D.B, D.N, D.d), device=dev).to(bf)
    Ut = up(synth.proxy_basis(D.d, r, seed=0), bf)
    pc = torch.randn((D.B, D.N, r), device=dev)
    pnew, score = torch.empty_like(pc), torch.empty((D.B, D.N), device=dev)
    us = _timed(torch, lambda: plk.score_drift(dm, X, Ut, r, pc, plk.METRIC_L2, score, proxy_out=pnew),
                args.steps, args.warmup)
    by = 2 * D.B * D.N * D.d + 8 * D.B * D.N * r + 2 * D.d * r
    out.append({"kernel": "score_tc_kernel", "config": f"B={D.B} N={D.N} d={D.d} r={r} L2", "us": us,
                "GB/s": by / (us * 1e-6) / 1e9, "frac_of_hbm": by / (us * 1e-6) / 1e9 / hbm})
    score_us = us
    lk_in = torch.zeros((D.B, D.N), dtype=torch.uint8, device=dev)
    lk, idx = torch.empty_like(lk_in), torch.empty(D.B * D.N, dtype=torch.int32, device=dev)
    seg = torch.empty(D.B + 1, dtype=torch.int32, device=dev)
    for pct in synth.SCORE_PCTS:  # the per-layer budget k = {5, 10, 20}% of N (SPA-Cache part 2)
        k = D.N * pct // 100
        us = _timed(torch, lambda: plk.select_active(dm, score, lk_in, lk, plk.SEL_TOPK_LARGEST, 0.0, k, idx, seg),
                    args.steps, args.warmup)
        by = 6 * D.B * D.N + 4 * D.B * k
        out.append({"kernel": "select_active (top-k decide + compaction)", "config": f"B={D.B} N={D.N} k={k} ({pct}% of N)", "us": us,
                    "GB/s": by / (us * 1e-6) / 1e9, "frac_of_hbm": by / (us * 1e-6) / 1e9 / hbm,
                    "scoring_layer_us": score_us + us,
                    "scoring_32_layers_us": 32 * (score_us + us)})
    del X, pc, pnew
    if scoring_only:
        return _configs_done(torch, plk, clk, out)
    # stack step 0: B = 4, N = 2048, every row active
    D = synth.STACK_8B
    dm = plk.dims(D.B, D.N, D.d, D.H, D.hd, D.F, D.eps, plk.BF16)
    W = {kk: (torch.randn(sh, device=dev) * 0.02).to(bf) if len(sh) == 2 else torch.ones(sh, device=dev).to(bf)
         for kk, sh in (("g1", (D.d,)), ("w_qkv", (3 * D.d, D.d)), ("w_o", (D.d, D.d)), ("g2", (D.d,)),
                        ("w_gu", (2 * D.F, D.d)), ("w_down", (D.d, D.F)))}
    pw = plk.weights(W)
    X = torch.randn((D.B, D.N, D.d), device=dev).to(bf)
    K, V, Y = (torch.zeros((D.B, D.N, D.d), dtype=bf, device=dev) for _ in range(3))
    M = D.B * D.N
    idx = torch.arange(M, dtype=torch.int32, device=dev)
    seg = torch.tensor([b * D.N for b in range(D.B + 1)], dtype=torch.int32, device=dev)
    ws = plk.alloc_workspace(dm, device=dev)
    step = lambda: plk.layer_step_partial(dm, pw, X, idx, seg, K, V, Y, ws)
    us_step = _timed(torch, step, max(args.steps // 10, 5), args.warmup)
    E = lambda: torch.cuda.Event(enable_timing=True)
    tr = [[E() for _ in range(11)] for _ in range(5)]
    for e in tr:
        plk.trace_events(e)
        step()
    torch.cuda.synchronize()
    plk.trace_events([])
    names = ["rmsnorm1", "gemm_qkv", "finish_qkv", "attention", "gemm_o", "rmsnorm2", "gemm_gu", "finish_gu",
             "gemm_down", "finish_y"]
    per = {n: statistics.median(e[i].elapsed_time(e[i + 1]) for e in tr) * 1e3 for i, n in enumerate(names)}
    gemm_flops = M * (8 * D.d * D.d + 6 * D.d * D.F)
    gemm_us = per["gemm_qkv"] + per["gemm_o"] + per["gemm_gu"] + per["gemm_down"]
    att_flops = 4 * D.B * D.N * D.N * D.d  # QK^T and PV over every (query, key) pair of a sequence
    scat = 20 * M * D.d  # the fp32 q, k and v sums in; q (hi/lo) and the K/V rows out
    out.append({"kernel": "layer step, every row active", "config": f"B={D.B} N={D.N} (stack step 0)",
                "us": us_step, "active_token_layers_per_s": M / (us_step * 1e-6),
                "gemm_tc_kernel": {"us": gemm_us, "TFLOP/s": gemm_flops / (gemm_us * 1e-6) / 1e12,
                                   "frac_of_peak": gemm_flops / (gemm_us * 1e-6) / 1e12 / tfl},
                "attn_tc_kernel": {"us": per["attention"], "TFLOP/s": att_flops / (per["attention"] * 1e-6) / 1e12,
                                   "frac_of_peak": att_flops / (per["attention"] * 1e-6) / 1e12 / tfl},
                "finish_qkv_kernel (K/V scatter)": {"us": per["finish_qkv"], "GB/s": scat / (per["finish_qkv"] * 1e-6) / 1e9,
                                                    "frac_of_hbm": scat / (per["finish_qkv"] * 1e-6) / 1e9 / hbm},
                "per_kernel_us_traced": per})
    del W, pw, X, K, V, Y, ws
    # grouped-query layer variant at a 7B-class shape (28 query heads, 4 K/V heads of 128,
    # SwiGLU 18944), N = 1024, 256 active rows
    d_, H_, Hkv_, F_, N_, M_ = 3584, 28, 4, 18944, 1024, 256
    dkv_ = Hkv_ * 128
    dm = plk.dims(1, N_, d_, H_, 128, F_, 1e-6, plk.BF16, 0.0, Hkv_)
    W = {kk: (torch.randn(sh, device=dev) * 0.02).to(bf) if len(sh) == 2 else torch.ones(sh, device=dev).to(bf)
         for kk, sh in (("g1", (d_,)), ("w_qkv", (d_ + 2 * dkv_, d_)), ("w_o", (d_, d_)), ("g2", (d_,)),
                        ("w_gu", (2 * F_, d_)), ("w_down", (d_, F_)))}
    pw = plk.weights(W)
    X = torch.randn((1, N_, d_), device=dev).to(bf)
    K, V = (torch.randn((1, N_, dkv_), device=dev).to(bf) for _ in range(2))
    Y = torch.zeros((1, N_, d_), dtype=bf, device=dev)
    rows = np.sort(np.random.default_rng(0).choice(N_, M_, replace=False)).astype(np.int32)
    idx = torch.from_numpy(rows).to(dev)
    seg = torch.tensor([0, M_], dtype=torch.int32, device=dev)
    ws = plk.alloc_workspace(dm, device=dev)
    us_g = _timed(torch, lambda: plk.layer_step_partial(dm, pw, X, idx, seg, K, V, Y, ws), args.steps, args.warmup)
    fl = M_ * (2 * d_ * (d_ + 2 * dkv_) + 2 * d_ * d_ + 6 * d_ * F_) + 4 * M_ * N_ * d_
    out.append({"kernel": "layer step, grouped-query attention", "config": f"d={d_} H={H_} Hkv={Hkv_} F={F_} "
                f"N={N_} M={M_}", "us": us_g, "active_token_layers_per_s": M_ / (us_g * 1e-6),
                "TFLOP/s": fl / (us_g * 1e-6) / 1e12, "frac_of_peak": fl / (us_g * 1e-6) / 1e12 / tfl})
    return _configs_done(torch, plk, clk, out)


def _configs_done(torch, plk, clk, out):
    st = plk.get_status()
    if st != plk.OK:
        raise RuntimeError(f"device status {plk.error_string(st)}")
    clk.__exit__(None, None, None)
    for o in out:
        o["clocks_over_all_configs"] = clk.summary()
        print(json.dumps(o), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the SlowFast span policy on its own (one call per decoding step), measured with
# --kernel slowfast over whole decoding trajectories at the 32-layer stack's
# batch (4 x 2048, 1024 generated) and the long-context sequence (1 x 8192, 256
# generated), with K_max = 8, W_hist = 2, variance threshold 1.0
# ---------------------------------------------------------------------------
SF_SHAPES = ((4, 2048, 1024), (1, 8192, 7936))
SF_PARAMS = dict(k=2, tau_conv=0.7, tau_high=0.9, var_stable=1.0, w_hist=2, k_max=8)


def run_slowfast(args):
    import torch
    import partial_recompute_kv_b200 as plk
    import oracle
    import synth

    dev = torch.device("cuda", 0)
    pk = peaks()
    hbm = float(pk["hbm_gbs"])
    params, op = plk.sf_params(**SF_PARAMS), oracle.SpanParams(**SF_PARAMS)
    lines = []
    for B, N, prompt in SF_SHAPES:
        dm = plk.dims(B, N, 64, 4, 16, 64, dtype=plk.F32)
        m0 = torch.from_numpy(synth.generation_mask(B, N, prompt)).to(dev)
        m, st = torch.empty_like(m0), plk.sf_state(B, device=dev)
        un, lk = torch.empty_like(m0), torch.empty_like(m0)
        confs = [torch.from_numpy(synth.span_confidences(B, N, t, seed=1, prompt=prompt)).to(dev)
                 for t in range(N - prompt)]

        def trajectory():
            for c in confs:
                plk.slowfast_step(dm, params, c, m, st, un, lk)

        def reset():
            m.copy_(m0)
            st.zero_()

        # the decode is over once nothing is masked; time the calls up to that step
        reset()
        T = 0
        for c in confs:
            plk.slowfast_step(dm, params, c, m, st, un, lk)
            T += 1
            if not bool(m.any()):
                break
        confs = confs[:T]
        # host cost of one call (ctypes marshalling and the launch), GPU left to run behind
        reset()
        torch.cuda.synchronize()
        h0 = time.perf_counter()
        trajectory()
        host_us = (time.perf_counter() - h0) / T * 1e6
        torch.cuda.synchronize()
        # device time: the whole decode captured as one CUDA graph and replayed, so the
        # calls run back to back as they would inside a captured decoding loop
        graph = torch.cuda.CUDAGraph()
        reset()
        with torch.cuda.graph(graph):
            trajectory()
        for _ in range(max(args.warmup, 3)):
            reset()
            graph.replay()
        torch.cuda.synchronize()
        E = lambda: torch.cuda.Event(enable_timing=True)
        reps = max(5, min(50, args.steps // max(T, 1) + 1))
        us = []
        with ClockSampler(0) as clk:
            for _ in range(reps):
                reset()
                a, b_ = E(), E()
                a.record()
                graph.replay()
                b_.record()
                torch.cuda.synchronize()
                us.append(a.elapsed_time(b_) * 1e3 / T)
        assert not bool(m.any()), "trajectory did not finish"
        del graph
        us_mean = statistics.mean(us)
        alg = 8 * B * N  # conf 4 B, masked read + write, unmask and lock 1 B each per position
        gbs = alg / (us_mean * 1e-6) / 1e9
        # cpu baseline: the oracle over the first steps of the same trajectory (about 10 s at most)
        mo = synth.generation_mask(B, N, prompt)
        so = [oracle.SpanState() for _ in range(B)]
        t0, n = time.perf_counter(), 0
        for c in confs:
            mo, _, _, so = oracle.slowfast_step(c.cpu().numpy(), mo, so, op)
            n += 1
            if time.perf_counter() - t0 > 10.0:
                break
        cpu_s = (time.perf_counter() - t0) / n
        lines.append({"metric": "SlowFast policy steps/s", "value": 1e6 / us_mean, "unit": "steps/s",
                      "n_gpus": 1, "steps": reps * T, "warmup": args.warmup, "us_per_call": us_mean,
                      "us_per_call_median": statistics.median(us), "host_enqueue_us_per_call": host_us,
                      "timing": "CUDA events around graph replays of whole decodes (calls back to back)",
                      "higher_is_better": True, "dtype": "f32",
                      "data": "synthetic",
                      "config": {"workload": f"slowfast_step, B={B}, N={N}, {N - prompt} generated, "
                                             f"{T} steps per decode, {reps} decodes",
                                 **{kk: v for kk, v in SF_PARAMS.items()}},
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                                   "frac": gbs / hbm, "traffic": None, "kernel": "slowfast_kernel",
                                   "alg_bytes_per_call": alg,
                                   "note": "one CTA per sequence: launch- and latency-bound at these sizes"},
                      "clocks": clk.summary(),
                      "cpu_baseline": {"value": 1.0 / cpu_s, "unit": "steps/s", "cores": 1, "kind": "oracle",
                                       "sample": f"the first {n} steps of the same decode"}})
    s_ = plk.get_status()
    if s_ != plk.OK:
        raise RuntimeError(f"device status {plk.error_string(s_)}")
    for ln in lines:
        print(json.dumps(ln), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the 32-layer stack over a whole decode (--kernel stack): B = 4 sequences of
# N = 2048, 32 independently drawn 8B-shape layers, 256 steps of the linear
# active-count schedule M_t = N - floor(t (N - floor(N/20)) / 255).  Per step
# and layer: drift score (rank 128, L2) -> the M_t most drifted rows among those
# not yet locked stay active, the rest lock for good -> partial layer step ->
# proxy refresh; each layer's output cache is the next layer's input.  The
# layer-0 input takes N(0, 0.01) noise on its active rows every step (outside
# the timed region).
# ---------------------------------------------------------------------------
STACK_LAYERS, STACK_STEPS, STACK_RANK = 32, 256, 128


def _stack_state(torch, plk, D, dev, seed):
    import synth

    bf = torch.bfloat16
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    rnd = lambda shape, std: (torch.randn(shape, generator=g, device=dev) * std).to(bf)
    d, F, r = D.d, D.F, STACK_RANK
    layers = []
    for l in range(STACK_LAYERS):
        W = {"g1": torch.ones(d, device=dev, dtype=bf), "w_qkv": rnd((3 * d, d), 0.02), "w_o": rnd((d, d), 0.02),
             "g2": torch.ones(d, device=dev, dtype=bf), "w_gu": rnd((2 * F, d), 0.02), "w_down": rnd((d, F), 0.02)}
        layers.append({"W": W, "pw": plk.weights(W),
                       "Ut": torch.from_numpy(synth.proxy_basis(d, r, seed=l)).to(dev).to(bf),
                       "pc": torch.zeros((D.B, D.N, r), device=dev), "pn": torch.empty((D.B, D.N, r), device=dev),
                       "K": torch.zeros((D.B, D.N, d), device=dev, dtype=bf),
                       "V": torch.zeros((D.B, D.N, d), device=dev, dtype=bf),
                       "Y": torch.zeros((D.B, D.N, d), device=dev, dtype=bf),
                       "lock": torch.zeros((D.B, D.N), device=dev, dtype=torch.uint8)})
    X0 = rnd((D.B, D.N, d), 1.0)
    noise = [torch.randn((D.B, D.N, d), generator=g, device=dev) * 0.1 for _ in range(4)]
    return layers, X0, noise


def _stack_reset(layers, X0, X0_init):
    for Ly in layers:
        Ly["pc"].zero_()
        Ly["K"].zero_()
        Ly["V"].zero_()
        Ly["Y"].zero_()
        Ly["lock"].zero_()
    X0.copy_(X0_init)


def run_stack(args):
    import torch
    import partial_recompute_kv_b200 as plk
    import oracle
    import synth

    dev = torch.device("cuda", 0)
    D = synth.STACK_8B
    B, N, d, F, r = D.B, D.N, D.d, D.F, STACK_RANK
    dm = plk.dims(B, N, d, D.H, D.hd, F, D.eps, plk.BF16)
    layers, X0, noise = _stack_state(torch, plk, D, dev, seed=0)
    X0_init = X0.clone()
    ws = plk.alloc_workspace(dm, device=dev)
    score = torch.empty((B, N), device=dev)
    idx = torch.empty(B * N, dtype=torch.int32, device=dev)
    seg = torch.empty(B + 1, dtype=torch.int32, device=dev)
    sched = synth.linear_schedule(N, STACK_STEPS)

    def step(t):
        M = int(sched[t])
        X = X0
        for Ly in layers:
            plk.score_drift(dm, X, Ly["Ut"], r, Ly["pc"], plk.METRIC_L2, score, proxy_out=Ly["pn"])
            plk.select_active(dm, score, Ly["lock"], Ly["lock"], plk.SEL_TOPK_LARGEST, 0.0, M, idx, seg)
            plk.layer_step_partial(dm, Ly["pw"], X, idx, seg, Ly["K"], Ly["V"], Ly["Y"], ws)
            plk.proxy_commit(dm, r, idx, seg, Ly["pn"], Ly["pc"])
            X = Ly["Y"]

    def perturb(t):  # the layer-0 input process: noise on the rows still active at layer 0
        act0 = (layers[0]["lock"] == 0).unsqueeze(-1)
        X0.copy_((X0.float() + noise[t % len(noise)] * act0).to(torch.bfloat16))

    warm = max(args.warmup, 3)
    for t in range(warm):
        perturb(t)
        step(t)
    torch.cuda.synchronize()
    _stack_reset(layers, X0, X0_init)
    E = lambda: torch.cuda.Event(enable_timing=True)
    ev = [(E(), E()) for _ in range(STACK_STEPS)]
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        for t in range(STACK_STEPS):
            perturb(t)
            ev[t][0].record()
            step(t)
            ev[t][1].record()
        torch.cuda.synchronize()
    st_ = plk.get_status()
    if st_ != plk.OK:
        raise RuntimeError(f"device status {plk.error_string(st_)}")
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_s = sum(step_ms) * 1e-3
    # every layer ends with B * M_255 active rows: the schedule was followed
    M_last = int(sched[-1])
    for Ly in layers:
        assert int((Ly["lock"] == 0).sum()) == B * M_last, "schedule not followed"
    atl = int(sched.sum()) * B * STACK_LAYERS
    flops = sum(int(m) * B * (8 * d * d + 6 * d * F + 4 * N * d) for m in sched) * STACK_LAYERS
    pk = peaks()
    tf = flops / total_s / 1e12
    # cpu baseline: the oracle on one layer at the schedule's last step (B * M_255 active rows),
    # extrapolated to the run by FLOP count
    Dn = synth.Dims(B=B, N=N, d=d, H=D.H, hd=D.hd, F=F, eps=D.eps, dtype="bf16")
    Wn = synth.layer_weights(Dn, 0.02, seed=0)
    Xn = synth.hidden_states(Dn, seed=0)
    rng = np.random.default_rng(0)
    lock = np.ones((B, N), np.uint8)
    for b in range(B):
        lock[b, rng.choice(N, M_last, replace=False)] = 0
    oidx, oseg = oracle.compact(lock)
    zeros = np.zeros((B, N, d))
    stn = oracle.LayerState(zeros, zeros.copy(), zeros.copy())
    t0 = time.perf_counter()
    oracle.layer_step_partial(Dn, Wn, Xn, oidx, oseg, stn, "bf16")
    cpu_s = time.perf_counter() - t0
    cpu_flops = B * M_last * (8 * d * d + 6 * d * F + 4 * N * d)
    cpu_steps_per_s = (cpu_flops / cpu_s) / (flops / STACK_STEPS)
    line = {"metric": "decode steps/s, 32-layer stack, B=4 x N=2048, linear 100%->5% active schedule",
            "value": STACK_STEPS / total_s, "unit": "steps/s", "n_gpus": 1, "steps": STACK_STEPS,
            "warmup": warm, "ms_per_step": total_s * 1e3 / STACK_STEPS,
            "ms_per_step_first_last": [step_ms[0], step_ms[-1]],
            "active_token_layers_per_s": atl / total_s, "active_token_layers_per_run": atl,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (random-init weights, N(0,1) layer-0 input + N(0,0.01) noise per step)",
            "config": {"workload": f"32-layer 8B-shape stack, B={B}, N={N}, d={d}, F={F}, rank-{r} L2 drift, "
                                   f"top-M_t among unlocked rows (permanent), M_t from {int(sched[0])} to {M_last}, "
                                   f"{STACK_STEPS} steps", "l2": "weights 14 GB, streamed every step"},
            "roofline": {"bound": "tensor", "achieved": tf, "peak": float(pk["bf16_tflops_sustained"]),
                         "unit": "TFLOP/s", "frac": tf / float(pk["bf16_tflops_sustained"]), "traffic": None,
                         "kernel": "whole step (all kernels): algorithmic FLOP of the run / run time, against "
                                   "the sustained bf16 peak"},
            "clocks": clk.summary(),
            "cpu_baseline": {"value": cpu_steps_per_s, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"one oracle layer step with {B * M_last} active rows (the last step), "
                                       f"extrapolated to the run by FLOP count"}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# long context (--kernel long): one 8B-shape layer, N = 8192 (7936 prompt rows),
# 8 block steps of 32 generated rows; block step i recomputes its 32 rows and
# M_i - 32 earlier positions drawn uniformly, M_i = 32 + min(G, 480),
# G ~ Geometric(1/64).  Caches come from one untimed full step.  Reports block
# steps/s (the 8 steps captured as one CUDA graph) and the attention roofline
# of each block (its K/V read of 2 N d bf16 values is what bounds it).
# ---------------------------------------------------------------------------
def run_long(args):
    import torch
    import partial_recompute_kv_b200 as plk
    import oracle
    import synth

    dev = torch.device("cuda", 0)
    bf = torch.bfloat16
    D = synth.LONG_8B
    N, d, F, prompt, nblk = D.N, D.d, D.F, 7936, 8
    dm = plk.dims(1, N, d, D.H, D.hd, F, D.eps, plk.BF16)
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    rnd = lambda shape, std: (torch.randn(shape, generator=g, device=dev) * std).to(bf)
    W = {"g1": torch.ones(d, device=dev, dtype=bf), "w_qkv": rnd((3 * d, d), 0.02), "w_o": rnd((d, d), 0.02),
         "g2": torch.ones(d, device=dev, dtype=bf), "w_gu": rnd((2 * F, d), 0.02), "w_down": rnd((d, F), 0.02)}
    pw = plk.weights(W)
    X = rnd((1, N, d), 1.0)
    K, V, Y = (torch.zeros((1, N, d), device=dev, dtype=bf) for _ in range(3))
    ws = plk.alloc_workspace(dm, device=dev)
    plk.full_layer_step(dm, pw, X, K, V, Y, ws)
    Ms = [int(m) for m in synth.geometric_block_m(nblk)]
    blocks = []
    for blk, M in enumerate(Ms):
        b0 = prompt + 32 * blk
        rows = np.concatenate([synth.uniform_positions(0, b0, M - 32, tag=100 + blk), np.arange(b0, b0 + 32)])
        blocks.append((M, torch.from_numpy(np.sort(rows).astype(np.int32)).to(dev),
                       torch.tensor([0, M], dtype=torch.int32, device=dev)))

    def decode():
        for M, idx, seg in blocks:
            plk.layer_step_partial(dm, pw, X, idx, seg, K, V, Y, ws)

    for _ in range(max(args.warmup, 3)):
        decode()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        decode()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    E = lambda: torch.cuda.Event(enable_timing=True)
    reps = max(5, min(100, args.steps // nblk))
    ev = [(E(), E()) for _ in range(reps)]
    with ClockSampler(0) as clk:
        for a, b in ev:
            a.record()
            graph.replay()
            b.record()
        torch.cuda.synchronize()
    del graph
    dec_ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    # traced pass: the attention kernel of every block (events between the library's kernels)
    att_us = []
    for M, idx, seg in blocks:
        samples = []
        for _ in range(5):
            tr = [E() for _ in range(11)]
            plk.trace_events(tr)
            plk.layer_step_partial(dm, pw, X, idx, seg, K, V, Y, ws)
            plk.trace_events([])
            torch.cuda.synchronize()
            samples.append(tr[3].elapsed_time(tr[4]) * 1e3)
        att_us.append(statistics.median(samples))
    st_ = plk.get_status()
    if st_ != plk.OK:
        raise RuntimeError(f"device status {plk.error_string(st_)}")
    pk = peaks()
    hbm, tfl = float(pk["hbm_gbs"]), float(pk["bf16_tflops"])
    att = []
    for (M, _, _), us in zip(blocks, att_us):
        by = 2 * N * d * 2 + 2 * M * d * 2  # K and V of the sequence, q in and a out
        att.append({"M": M, "us": us, "GB/s": by / (us * 1e-6) / 1e9, "frac_of_hbm": by / (us * 1e-6) / 1e9 / hbm,
                    "TFLOP/s": 4 * M * N * d / (us * 1e-6) / 1e12})
    gbs_mean = statistics.mean(a["GB/s"] for a in att)
    # cpu baseline: the oracle on block 0's step from zero caches
    Dn = synth.Dims(B=1, N=N, d=d, H=D.H, hd=D.hd, F=F, eps=D.eps, dtype="bf16")
    Wn = synth.layer_weights(Dn, 0.02, seed=0)
    Xn = synth.hidden_states(Dn, seed=0)
    lock = np.ones((1, N), np.uint8)
    lock[0, blocks[0][1].cpu().numpy()] = 0
    oidx, oseg = oracle.compact(lock)
    zeros = np.zeros((1, N, d))
    t0 = time.perf_counter()
    oracle.layer_step_partial(Dn, Wn, Xn, oidx, oseg, oracle.LayerState(zeros, zeros.copy(), zeros.copy()), "bf16")
    cpu_s = time.perf_counter() - t0
    line = {"metric": "block steps/s, long context (8B layer, N=8192, 8 blocks of 32, geometric M)",
            "value": nblk / (dec_ms * 1e-3), "unit": "steps/s", "n_gpus": 1, "steps": reps * nblk,
            "warmup": max(args.warmup, 3), "ms_per_step": dec_ms / nblk, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (random-init weights, N(0,1) input)",
            "config": {"workload": f"long context, B=1, N={N}, prompt {prompt}, {nblk} blocks of 32, M per block "
                                   f"{Ms}, one layer d={d} F={F}, the {nblk} block steps as one CUDA graph"},
            "active_token_layers_per_s": sum(Ms) / (dec_ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": gbs_mean, "peak": hbm, "unit": "GB/s", "frac": gbs_mean / hbm,
                         "traffic": None, "kernel": "attn_tc_kernel (mean over the 8 blocks, traced pass)",
                         "per_block": att},
            "clocks": clk.summary(),
            "cpu_baseline": {"value": 1.0 / cpu_s, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"one oracle block step (block 0, M={Ms[0]}) from zero caches"}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the active-fraction sweep (--kernel sweep): the headline step at every active
# fraction of the 8B-shape layer, M/N in {1, 1/2, 1/4, 1/10, 1/20} (SureLock page,
# Sec. 2 "Algorithmic Complexity": the per-step work falls with the active count
# M_t <= N); one JSON line per fraction with the projections' roofline taken
# against the tensor peak where their arithmetic intensity is above the ridge
# and against HBM below it, and the CPU oracle beside it
# ---------------------------------------------------------------------------
def run_sweep(args):
    import synth

    base = Workload(frac=synth.LAYER_8B_FRACTIONS[0])
    oracle_base = None
    for frac in synth.LAYER_8B_FRACTIONS:
        wl = Workload(frac=frac, share=base)
        res = run_gpu(args, wl, None, 0, 1, 0)
        pk = res["peaks"]
        per = res["per_kernel_us"]
        gemm_us = per["gemm_qkv"] + per["gemm_o"] + per["gemm_gu"] + per["gemm_down"]
        flops, by = wl.M * wl.gemm_flops_per_row(), wl.gemm_bytes()
        tfl, hbm = float(pk["bf16_tflops"]), float(pk["hbm_gbs"])
        ridge = tfl * 1e12 / (hbm * 1e9)
        t_achieved = flops / (gemm_us * 1e-6) / 1e12
        b_achieved = by / (gemm_us * 1e-6) / 1e9
        if flops / by >= ridge:
            roof = {"bound": "tensor", "achieved": t_achieved, "peak": tfl, "unit": "TFLOP/s", "frac": t_achieved / tfl}
        else:
            roof = {"bound": "hbm", "achieved": b_achieved, "peak": hbm, "unit": "GB/s", "frac": b_achieved / hbm}
        roof.update({"kernel": "gemm_tc_kernel (4 launches)", "intensity_flop_per_byte": flops / by, "ridge": ridge,
                     "tensor_frac": t_achieved / tfl, "hbm_frac": b_achieved / hbm, "alg_flops": flops,
                     "alg_bytes": by, "peak_source": pk.get("source"), "traffic": None})
        if oracle_base is None:
            oracle_base = OracleRunner(wl)
        run = OracleRunner.__new__(OracleRunner)
        run.__dict__.update(oracle_base.__dict__)
        run.wl, run.pc = wl, oracle_base.pc.copy()
        line = {"metric": f"active-token-layers/sec at 8B-shape, M/N={frac}", "value": res["value"], "unit": UNIT,
                "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
                "decode_steps_per_s": 1e3 / res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": wl.config(args.l2),
                "roofline": roof, "step_tflops": res["step_tflops"], "per_kernel_us": per,
                "e2e": res["e2e"], "clocks": res["clocks"],
                "cpu_baseline": cpu_baseline(wl, budget_s=6.0, run=run)}
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["plk", "reference"], default="plk")
    ap.add_argument("--l2", choices=["stream", "flush"], default="stream",
                    help="stream: no flush between steps (the weights alone are 3.5x L2); "
                         "flush: write 256 MiB before every step")
    ap.add_argument("--graph", dest="graph", action="store_true", default=True,
                    help="replay the step as one captured CUDA graph (default)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="enqueue the step's library calls directly every step")
    ap.add_argument("--frac", type=float, default=0.25,
                    help="active fraction M/N of the headline step (the metric is quoted at 0.25)")
    ap.add_argument("--kernel", choices=["step", "sweep", "kl_lock", "slowfast", "configs", "scoring", "stack",
                                         "long"],
                    default="step",
                    help="step: the headline layer step; sweep: the step at every active fraction 1, 1/2, 1/4, "
                         "1/10, 1/20; kl_lock: the KL lock rule alone; slowfast: the SlowFast "
                         "span policy over whole decodes; configs: scoring and the all-active stack step at the "
                         "shapes where their rooflines are judged; scoring: the first of those alone (score and "
                         "top-k at 8 x 4096); stack: the 32-layer stack over the 256-step "
                         "schedule; long: the long-context block decode at N = 8192")
    ap.add_argument("--profile", action="store_true",
                    help="set up and run --steps steps without timing or output (for ncu)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3) if not args.profile else args.warmup

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.kernel == "kl_lock":
        return run_kl_lock(args) if rank == 0 else 0
    if args.kernel == "slowfast":
        return run_slowfast(args) if rank == 0 else 0
    if args.kernel == "stack":
        return run_stack(args) if rank == 0 else 0
    if args.kernel == "long":
        return run_long(args) if rank == 0 else 0
    if args.kernel in ("configs", "scoring"):
        return run_kernel_configs(args, scoring_only=args.kernel == "scoring") if rank == 0 else 0
    if args.kernel == "sweep":
        return run_sweep(args) if rank == 0 else 0
    if args.impl == "reference":
        if rank != 0:
            return 0
        run_reference(args, Workload(frac=args.frac))
        return 0

    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    wl = Workload(frac=args.frac)
    try:
        res = run_gpu(args, wl, dist, rank, world, local_rank)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    if res is None or rank != 0:
        return 0
    launches_per_step = 1 + 1 + 10  # score, select (B = 1: one launch), layer step (proxy refresh folded in)
    metric = METRIC if args.frac == 0.25 else f"active-token-layers/sec at 8B-shape, M/N={args.frac}"
    line = {"metric": metric, "value": res["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(wl.config(args.l2), parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
            "roofline": res["roofline"],
            "step_tflops": res["step_tflops"],
            "step_frac_of_bf16_peak": res["step_tflops"] / float(res["peaks"]["bf16_tflops"]),
            "per_kernel_us": res["per_kernel_us"], "host_enqueue_us_per_step": res["host_enqueue_us_per_step"],
            "ms_per_step_median": res["ms_per_step_median"], "hbm_kernels": res["hbm_kernels"],
            "launch": "cuda graph" if args.graph else "stream",
            "e2e": res["e2e"], "gpu_launches": launches_per_step * args.steps, "clocks": res["clocks"]}
    if world == 1:
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
