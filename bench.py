"""Benchmark of one DSpark round (drafting, confidence, Algorithm-1 scheduling,
verification) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload headline]
    python bench.py --impl reference ...     # the fp64 CPU oracle, timed on host cores

A step is one round over one batch of synthetic requests (the headline
workload: B=256, G=5, V=129280, r=256, d=4096, bf16).  The round is captured
once in a CUDA graph and replayed; L2 is flushed (a 256 MiB write) before
every timed replay, outside the timed events.  Under torchrun every rank runs
its own engine on its own batch (weak scaling, no collective on the data
path); the reported time is the max over ranks.

Prints one JSON line: value = verified draft tokens/s (sum over ranks of the
admitted draft tokens per round / round time), plus the round's fraction of
the HBM roofline, the dominant stage's roofline, the oracle's CPU baseline,
an end-to-end number through host buffers and the clocks seen.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "verified draft tokens/s, B=256 γ=5 V=129280, as % of HBM roofline"
UNIT = "verified draft tokens/s"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


def _workload(name):
    from speculative_decoding_draft_rank_b200 import workloads as wl
    table = {"tiny": wl.tiny, "qwen_vocab": wl.qwen_vocab, "headline": wl.headline,
             "saturated": wl.saturated}
    if name.startswith("long_block_g"):
        return wl.long_block(int(name[len("long_block_g"):]))
    return table[name]()


def algorithmic_bytes(w, ell_sum):
    """Bytes a round must move at least once: draft logits, the transition
    factor W once, the gathered U rows, the hidden states, and the target
    rows of the admitted prefixes plus one bonus/final row per request."""
    es = 2 if w.dtype == "bf16" else 4
    B, G, V, r, d = w.B, w.G, w.V, w.r, w.d
    parts = {
        "draft_logits": B * G * V * es,
        "transition_W": r * V * es,
        "U_rows": B * G * r * es,
        "hidden": B * G * d * es,
        "target_rows": (ell_sum + B) * V * es,
    }
    return parts


class ClockSampler:
    """SM clock and throttle reasons sampled every 5 ms by an NVML reader
    thread while the timed region runs (read-only queries)."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.gpu]) if vis else self.gpu
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nv = pynvml
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self._nv = None
            return self
        self._stop = threading.Event()

        def run():
            nv = self._nv
            while not self._stop.is_set():
                try:
                    self.samples.append(float(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)))
                    get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                        nv.nvmlDeviceGetCurrentClocksThrottleReasons
                    mask = get(self._h)
                    for name, bit in self.REASONS.items():
                        if mask & bit:
                            self.reasons.add(name)
                except Exception:
                    pass
                self._stop.wait(0.005)

        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        if self._stop is not None:
            self._stop.set()
            self._t.join(timeout=2)
        return False

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml, 5 ms"}


# The sources the drafting kernel is built from (kernel, its device helpers,
# its host launcher): profile counters are valid only for the code they were
# taken on.
DRAFT_KERNEL_SOURCES = ("draft_tc.cu", "draft_pair.cu", "finalize.cuh", "tc.cuh", "common.cuh", "kernels.cuh",
                        "draft.cu")


def kernel_sources_digest():
    import hashlib
    h = hashlib.sha256()
    for name in DRAFT_KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "speculative_decoding_draft_rank_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload_name):
    """DRAM bytes per round of the drafting stage from the committed ncu
    summary, or None when the kernels changed since it was taken."""
    p = os.path.join(ROOT, "profiles", f"draft_stage_traffic_{workload_name}.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    return d["dram_bytes_per_round"] if d.get("sources_digest") == kernel_sources_digest() else None


def oracle_sample(w, inp, n_req, seed=0, A=None):
    """Time the fp64 oracle (as it stands, one thread) on a bounded sample of
    the round: confidence and scheduling for the whole batch, drafting and
    verification for n_req requests.  Returns (verified tokens in the sample,
    seconds)."""
    from oracle import oracle
    from speculative_decoding_draft_rank_b200 import synth
    rng = np.random.default_rng(seed)
    idx = np.sort(rng.choice(w.B, size=min(n_req, w.B), replace=False))
    sub = synth.select_requests(inp, idx)
    oracle._load()                   # library load outside the timed region
    t0 = time.perf_counter()
    c0 = time.process_time()
    _, S = oracle.confidence(inp.h, inp.w, inp.bias)
    sch = oracle.schedule(S, w.knots_n, w.knots_t, w.budget, w.mode)
    dr = oracle.draft(sub.L, sub.U, sub.W, sub.x0, sub.temp, sub.u_draft.astype(np.float64), A=A)
    oracle.verify(sub.Tlog, sub.L, sub.U, sub.W, sub.x0, dr.x, sub.temp, sub.u_accept.astype(np.float64),
                  sub.u_final.astype(np.float64), sch.ell[idx], A=A)
    dt = time.perf_counter() - t0
    oracle_sample.cpu_s = time.process_time() - c0   # CPU time of every thread in the region
    return int(sch.ell[idx].sum()), dt, len(idx)


def run_reference(args):
    """The reference arm: the oracle on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = _workload(args.workload)
    inp = w.inputs()
    n_req = args.reference_requests
    for _ in range(args.warmup):
        oracle_sample(w, inp, max(1, n_req // 8), seed=1)
    toks, secs, cpu = 0, 0.0, 0.0
    for s in range(args.steps):
        t, dt, n = oracle_sample(w, inp, n_req, seed=100 + s)
        toks += t
        secs += dt
        cpu += oracle_sample.cpu_s
    value = toks / secs if secs > 0 else 0.0
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "G": w.G, "V": w.V, "r": w.r, "d": w.d},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": max(1, round(cpu / secs)) if secs > 0 else 1,
                         "kind": "oracle",
                         "sample": f"{n_req} requests per step (draft+verify), whole-batch confidence+schedule, "
                                   f"{secs:.1f} s wall, {cpu:.1f} s CPU"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def run_sharded(args):
    """The request-sharded round: each rank drafts, scores and verifies its
    own headline-sized batch; the survivals are all-gathered (NCCL) and every
    rank runs the same admission over the whole batch (profile knots scaled
    by the rank count).  Eager launches per round (the collective sits
    between library calls); device time per round is the max over ranks."""
    import datetime
    import torch
    import torch.distributed as dist
    from speculative_decoding_draft_rank_b200.round import DeviceRound
    from speculative_decoding_draft_rank_b200.sharded import ShardedRound

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if dist.is_available() and not dist.is_initialized():
        if "MASTER_ADDR" not in os.environ:
            os.environ["MASTER_ADDR"] = "127.0.0.1"
            os.environ["MASTER_PORT"] = "29511"
        dist.init_process_group("nccl", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    w = _workload(args.workload)
    w.seed = rank
    inp = w.inputs()
    kn = np.asarray(w.knots_n, np.int64) * world
    dr = DeviceRound(inp, w.knots_n, w.knots_t, w.budget, w.mode, device=dev)
    sh = ShardedRound(dr, kn.astype(np.int32), w.knots_t, w.budget * world if w.budget >= 0 else -1, w.mode)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            sh.run(stream)
    torch.cuda.synchronize()
    dist.barrier()
    times = []
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            flush.zero_()
            e0.record(stream)
            sh.run(stream)
            e1.record(stream)
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
    torch.cuda.synchronize()
    dist.barrier()
    ms = statistics.mean(times)
    ell_sum = int(dr.o["ell"].sum().item())
    tt = torch.tensor([ms, float(ell_sum)], device=dev, dtype=torch.float64)
    gathered = [torch.zeros_like(tt) for _ in range(world)]
    dist.all_gather(gathered, tt)
    ms = max(float(g[0]) for g in gathered)
    ell_tot = sum(float(g[1]) for g in gathered)
    if dr.device_status() != 0:
        raise RuntimeError("device status word set")
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": ell_tot / (ms * 1e-3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded generator, one batch per rank)",
            "config": {"workload": w.name, "B_per_rank": w.B, "G": w.G, "V": w.V, "r": w.r, "d": w.d,
                       "l2_flush": "256 MiB write before every timed round", "graph_replay": False,
                       "parallelism": f"{world} ranks, request-sharded, survivals all-gathered (NCCL)"},
            "round": {"admitted_draft_tokens": ell_tot, "n_adm_global": int(sh.n_adm.item())}}))
    dist.destroy_process_group()
    return 0


# The sources of the calibration kernels: their fp64 counters are valid only
# for the code they were taken on.
STS_KERNEL_SOURCES = ("calibration.cu", "calibration.cuh", "common.cuh")


def sts_sources_digest():
    import hashlib
    h = hashlib.sha256()
    for name in STS_KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "speculative_decoding_draft_rank_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def profiled_sts_fp64(workload_name):
    """fp64 FLOPs of one fit (all positions) and DRAM bytes from the committed
    ncu summary, or None when the kernels changed since it was taken."""
    p = os.path.join(ROOT, "profiles", f"sts_position_fp64_{workload_name}.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    return d if d.get("sources_digest") == sts_sources_digest() else None


# fp64 peak: 64 fp64 lanes per SM (one fused multiply-add each per clock, the
# half rate of the 128 fp32 lanes), 148 SMs.
FP64_LANES_PER_SM = 64
SMS = 148


def run_sts(args):
    """Sequential temperature scaling fit of the confidence head (one step =
    one fit over N labelled blocks: every grid temperature at every position,
    left to right) and the survivals' ROC-AUC, on one GPU per rank (replicas:
    every rank fits its own seeded set; time = max over ranks)."""
    import datetime
    import torch
    import torch.distributed as dist
    from speculative_decoding_draft_rank_b200 import _lib, workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    w = wl.calibration_headline()
    metric = f"STS fit candidate evaluations/s, N={w.N} γ={w.G} K={w.K} M={w.M}"
    unit = "candidate evaluations/s"
    evals = w.N * (w.K + 1) * w.G          # every grid entry plus the raw chain, every position

    if args.impl == "reference":
        if rank != 0:
            return 0
        from oracle import calibration as C
        cs = w.inputs()
        grid = w.grid()
        times = []
        for _ in range(max(1, args.warmup)):
            C.sts_fit(cs.z, cs.acc, grid, w.M)
        c0 = time.process_time()
        for _ in range(args.steps):
            t0 = time.perf_counter()
            C.sts_fit(cs.z, cs.acc, grid, w.M)
            times.append(time.perf_counter() - t0)
        cpu = time.process_time() - c0
        ms = 1e3 * statistics.mean(times)
        v = evals / (ms * 1e-3)
        cores = max(1, round(cpu / sum(times)))
        print(json.dumps({"impl": "reference", "metric": metric, "value": v, "unit": unit, "n_gpus": 1,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                          "config": {"workload": w.name, "N": w.N, "G": w.G, "K": w.K, "M": w.M},
                          "cpu_baseline": {"value": v, "unit": unit, "cores": cores, "kind": "oracle",
                                           "sample": f"the whole fit, every step ({cpu:.2f} s CPU)"},
                          "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return 0

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    w.seed = rank
    cs = w.inputs()
    grid = w.grid()
    f32, f64 = dict(dtype=torch.float32, device=dev), dict(dtype=torch.float64, device=dev)
    z = torch.from_numpy(cs.z).to(dev)
    acc = torch.from_numpy(cs.acc).to(dev)
    g = torch.from_numpy(grid).to(dev)
    z_h = torch.from_numpy(cs.z).pin_memory()
    acc_h = torch.from_numpy(cs.acc).pin_memory()
    ws = torch.zeros(_lib.dspark_sts_workspace_size(w.N, w.G, w.K, w.M), dtype=torch.uint8, device=dev)
    tau = torch.zeros(w.G, **f32)
    tau_h = torch.zeros(w.G, dtype=torch.float32).pin_memory()
    e_raw, e_fit = torch.zeros(w.G, **f64), torch.zeros(w.G, **f64)
    S = torch.zeros((w.N, w.G), **f32)
    twice = torch.zeros(w.G, dtype=torch.int64, device=dev)
    pairs = torch.zeros(w.G, dtype=torch.int64, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def fit():
        _lib.dspark_sts_fit(z, acc, g, w.M, ws, tau, e_raw, e_fit, None, S)

    def auc():
        _lib.dspark_survival_auc(S, acc, twice, pairs)

    with torch.cuda.stream(stream):
        fit()
        auc()
    torch.cuda.synchronize()
    g_fit, g_auc = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_fit, stream=stream):
        fit()
    with torch.cuda.graph(g_auc, stream=stream):
        auc()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            g_fit.replay()
            g_auc.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    fit_ms, auc_ms = [], []
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                flush.zero_()
                e0.record(stream)
                g_fit.replay()
                e1.record(stream)
                e1.synchronize()
                fit_ms.append(e0.elapsed_time(e1))
        torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.steps // 4)):
            flush.zero_()
            e0.record(stream)
            g_auc.replay()
            e1.record(stream)
            e1.synchronize()
            auc_ms.append(e0.elapsed_time(e1))
        # End to end: the labelled set from pinned host memory, the fit, the
        # temperatures back to pinned host memory.
        e2e_ms = []
        for i in range(max(2, args.steps // 4) + 1):
            e0.record(stream)
            z.copy_(z_h, non_blocking=True)
            acc.copy_(acc_h, non_blocking=True)
            fit()
            tau_h.copy_(tau, non_blocking=True)
            e1.record(stream)
            e1.synchronize()
            if i > 0:
                e2e_ms.append(e0.elapsed_time(e1))
    torch.cuda.synchronize()
    status = _lib.dspark_get_device_status(ws)
    if status != 0:
        raise RuntimeError(f"device status word {status:#x}")
    ms, a_ms, e2e = statistics.mean(fit_ms), statistics.mean(auc_ms), statistics.mean(e2e_ms)
    if world > 1:
        tt = torch.tensor([ms, a_ms, e2e], device=dev, dtype=torch.float64)
        gathered = [torch.zeros_like(tt) for _ in range(world)]
        dist.all_gather(gathered, tt)
        ms, a_ms, e2e = (max(float(x[j]) for x in gathered) for j in range(3))
    tw, pr = twice.cpu().numpy(), pairs.cpu().numpy()
    clocks = clk.summary()
    mhz = clocks["sm_mhz"] or 1965.0
    peak_tflops = SMS * FP64_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
    prof = profiled_sts_fp64(w.name)
    roof = {"kernel": f"sts_position ({w.G} launches per fit)", "bound": "alu", "unit": "TFLOP/s",
            "peak": peak_tflops, "peak_source": f"derived: {SMS} SMs x {FP64_LANES_PER_SM} fp64 lanes x 2 x "
                                                f"{mhz:.0f} MHz (median SM clock of the timed region)",
            "achieved": None, "frac": None, "traffic": None, "ms": ms, "launches": w.G}
    if prof is not None:
        ach = prof["fp64_flops_per_fit"] / (ms * 1e-3) / 1e12
        roof.update(achieved=ach, frac=ach / peak_tflops, traffic=prof["dram_bytes_per_fit"],
                    fp64_flops_per_fit=prof["fp64_flops_per_fit"])
    line = {
        "metric": metric, "value": world * evals / (ms * 1e-3), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded calibration sets, one per rank)",
        "config": {"workload": w.name, "N": w.N, "G": w.G, "K": w.K, "M": w.M,
                   "l2_flush": "256 MiB write before every timed fit", "graph_replay": True,
                   "parallelism": f"{world} independent fits"},
        "fit": {"tau": [float(x) for x in tau.cpu()], "ece_raw": [float(x) for x in e_raw.cpu()],
                "ece_fit": [float(x) for x in e_fit.cpu()]},
        "auc": {"ms": a_ms, "pairs_per_s": float(pr.sum()) / (a_ms * 1e-3),
                "auc_fit": [float(tw[i]) / (2.0 * float(pr[i])) if pr[i] else None for i in range(w.G)]},
        "roofline": roof,
        "e2e": {"value": world * evals / (e2e * 1e-3), "unit": unit,
                "h2d_bytes_per_step": z_h.numel() * 4 + acc_h.numel() * 4, "d2h_bytes_per_step": w.G * 4,
                "ms_per_step": e2e},
        "gpu_launches": (w.G + 1) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import calibration as C
        n, t0, c0 = 0, time.perf_counter(), time.process_time()
        while n == 0 or time.perf_counter() - t0 < 10.0:
            C.sts_fit(cs.z, cs.acc, grid, w.M)
            n += 1
        secs, cpu = time.perf_counter() - t0, time.process_time() - c0
        line["cpu_baseline"] = {"value": n * evals / secs, "unit": unit, "cores": max(1, round(cpu / secs)),
                                "kind": "oracle", "sample": f"{n} whole fits, {secs:.1f} s wall, {cpu:.1f} s CPU"}
    if rank == 0:
        print(json.dumps(line))
    g_fit.reset()
    g_auc.reset()
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_production(args):
    """The headline round with the production scheduler: the capacity from the
    previous round's survivals (global search, side stream, overlapping
    drafting) and the dynamic top-K of the current survivals.  One graph per
    round (the fork to the side stream and the join are in it), replayed with
    L2 flushed before each; one GPU per rank (replicas)."""
    import datetime
    import torch
    import torch.distributed as dist
    from speculative_decoding_draft_rank_b200 import _lib
    from speculative_decoding_draft_rank_b200.production import ProductionRound, ProductionScheduler
    from speculative_decoding_draft_rank_b200.round import DeviceRound

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    w = _workload(args.workload)
    w.seed = rank
    inp = w.inputs()
    dr = DeviceRound(inp, w.knots_n, w.knots_t, w.budget, w.mode, device=dev)
    ps = ProductionScheduler(w.B, w.G, w.knots_n, w.knots_t, w.budget, device=dev)
    pr = ProductionRound(dr, ps)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        pr.run(stream)          # round 0: Algorithm 1's own count, no history
        pr.run(stream)          # round 1: capacity from round 0
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        pr.run(stream)
    # The selection alone (the stage that replaces Algorithm 1 on the round's
    # critical path) in its own graph.
    o = dr.o
    sel = torch.cuda.CUDAGraph()
    with torch.cuda.graph(sel, stream=stream):
        _lib.dspark_schedule_topk(o["S"], ps.capacity, ps.budget, ps.ws_sel, o["ell"], o["n_adm"], o["order"],
                                  stream)
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    step_ms, sel_ms = [], []
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                flush.zero_()
                e0.record(stream)
                graph.replay()
                e1.record(stream)
                e1.synchronize()
                step_ms.append(e0.elapsed_time(e1))
        torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.steps // 4)):
            flush.zero_()
            e0.record(stream)
            sel.replay()
            e1.record(stream)
            e1.synchronize()
            sel_ms.append(e0.elapsed_time(e1))
    torch.cuda.synchronize()
    status = dr.device_status() | ps.device_status()
    if status != 0:
        raise RuntimeError(f"device status word {status:#x}")
    ms = statistics.mean(step_ms)
    ell_sum = int(o["ell"].sum().item())
    if world > 1:
        tt = torch.tensor([ms, float(ell_sum)], device=dev, dtype=torch.float64)
        gathered = [torch.zeros_like(tt) for _ in range(world)]
        dist.all_gather(gathered, tt)
        ms = max(float(g[0]) for g in gathered)
        ell_tot = sum(float(g[1]) for g in gathered)
    else:
        ell_tot = float(ell_sum)
    line = {
        "metric": METRIC, "value": ell_tot / (ms * 1e-3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded generator, one batch per rank)",
        "config": {"workload": w.name, "B": w.B, "G": w.G, "V": w.V, "r": w.r, "d": w.d,
                   "scheduler": "production: capacity from the previous round (global search, side stream), "
                                "dynamic top-K of the current survivals",
                   "l2_flush": "256 MiB write before every timed round", "graph_replay": True,
                   "parallelism": f"{world} independent engines"},
        "round": {"admitted_draft_tokens": ell_sum, "capacity": int(ps.capacity.item()),
                  "selection_ms": statistics.mean(sel_ms)},
        "gpu_launches": (1 + 1 + 1 + 1 + 5) * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line))
    graph.reset()
    sel.reset()
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="headline")
    ap.add_argument("--oracle-requests", type=int, default=64,
                    help="requests drafted+verified by the oracle for the CPU baseline leg")
    ap.add_argument("--reference-requests", type=int, default=8,
                    help="requests per step of the reference arm (the oracle)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--head", default="markov", choices=["markov", "rnn"],
                    help="sequential draft head: the Markov head (the headline path) or the RNN head")
    ap.add_argument("--mode", default="replicas", choices=["replicas", "sharded", "sts", "production"],
                    help="replicas: every rank an independent engine (default); sharded: one engine over all "
                         "ranks' requests, survivals all-gathered for one global admission; sts: the "
                         "confidence head's sequential temperature scaling fit; production: the round with "
                         "the production scheduler (capacity from the previous round, dynamic top-K)")
    args = ap.parse_args()
    if args.mode == "sts":
        return run_sts(args)
    if args.mode == "production" and args.impl == "native":
        return run_production(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.mode == "sharded":
        return run_sharded(args)

    import torch
    import torch.distributed as dist
    from speculative_decoding_draft_rank_b200.round import DeviceRound

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    w = _workload(args.workload)
    w.seed = rank  # every engine drafts its own batch
    inp = w.inputs()
    Arec = None
    if args.head == "rnn":
        from speculative_decoding_draft_rank_b200 import synth
        Arec = synth.bf16_to_f32(synth.bf16_bits(synth.rnn_matrix(w.r, seed=rank))).reshape(w.r, w.r)
    dr = DeviceRound(inp, w.knots_n, w.knots_t, w.budget, w.mode, device=dev, pinned_host=True, Arec=Arec)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    # Warm up eagerly once (library attributes, lazy module loads), then capture.
    with torch.cuda.stream(stream):
        dr.run(stream)
    torch.cuda.synchronize()
    from speculative_decoding_draft_rank_b200 import _lib
    t, o = dr.t, dr.o
    stages = [
        lambda: dr.draft(),
        lambda: _lib.dspark_confidence(t["h"], t["w"], float(inp.bias), t["tau"], o["c"], o["S"]),
        lambda: _lib.dspark_schedule(o["S"], t["knots_n"], t["knots_t"], dr.budget, dr.mode, dr.ws, o["ell"],
                                     o["n_adm"], o["theta"], o["order"]),
        lambda: dr.verify(),
    ]
    graph = torch.cuda.CUDAGraph()          # the whole round: the timed unit
    with torch.cuda.graph(graph, stream=stream):
        dr.run(stream)                      # confidence forked to a side stream, joined before scheduling
    stage_graphs = []                       # one graph per stage: the breakdown
    for f in stages:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            f()
        stage_graphs.append(g)

    launches_per_round = (1 if w.dtype == "bf16" else 2 * w.G) + 1 + 1 + 5

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            graph.replay()
    torch.cuda.synchronize()
    barrier()

    step_ms, stage_ms = [], [[] for _ in range(4)]
    ell_sum = int(dr.o["ell"].sum().item())
    nout_sum = int(dr.o["nout"].sum().item())
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    _lib.dspark_clear_device_status(dr.ws, stream)
    with ClockSampler(local) as clk:
        torch.cuda.synchronize()
        barrier()
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                flush.zero_()
                e0.record(stream)
                graph.replay()
                e1.record(stream)
                e1.synchronize()
                step_ms.append(e0.elapsed_time(e1))
        torch.cuda.synchronize()
        barrier()
    # Decisions within 1e-5 of their threshold, as the kernels counted them
    # over the timed rounds (the same inputs every round).
    ties_d, ties_v = _lib.dspark_get_near_ties(dr.ws, stream)
    # Stage breakdown (not the headline): each stage's graph between events.
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.steps // 2)):
            flush.zero_()
            for j, g in enumerate(stage_graphs):
                ev[j].record(stream)
                g.replay()
            ev[4].record(stream)
            ev[4].synchronize()
            for j in range(4):
                stage_ms[j].append(ev[j].elapsed_time(ev[j + 1]))
    torch.cuda.synchronize()
    status = dr.device_status()
    if status != 0:
        raise RuntimeError(f"device status word {status:#x}")

    ms = statistics.mean(step_ms)
    if world > 1:
        tt = torch.tensor([ms, float(ell_sum), float(nout_sum)], device=dev, dtype=torch.float64)
        gathered = [torch.zeros_like(tt) for _ in range(world)]
        dist.all_gather(gathered, tt)
        ms = max(float(g[0]) for g in gathered)
        ell_tot = sum(float(g[1]) for g in gathered)
        nout_tot = sum(float(g[2]) for g in gathered)
    else:
        ell_tot, nout_tot = float(ell_sum), float(nout_sum)
    value = ell_tot / (ms * 1e-3)

    # End to end through the public API (DeviceRound.run_from_host): the
    # round's draft-side inputs from pinned host memory, drafting, confidence
    # and scheduling, the target rows verification reads (rows 0..ell_b per
    # request, pulled from pinned host memory by one kernel that reads ell on
    # the device), verification, and the emitted tokens, counts and lengths
    # back to pinned host memory.
    e2e_ms = []
    h2d = d2h = 0
    with torch.cuda.stream(stream):
        for i in range(max(2, args.steps // 2) + 1):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            dr.run_from_host(stream)
            e1.record(stream)
            stream.synchronize()
            h2d, d2h = dr.host_round_bytes()
            if i > 0:
                e2e_ms.append(e0.elapsed_time(e1))
    e2e = statistics.mean(e2e_ms)
    if world > 1:
        tt = torch.tensor([e2e], device=dev, dtype=torch.float64)
        gathered = [torch.zeros_like(tt) for _ in range(world)]
        dist.all_gather(gathered, tt)
        e2e = max(float(g[0]) for g in gathered)

    hbm_gbs, bf16_tf, peak_kind = _peaks()
    parts = algorithmic_bytes(w, ell_sum)
    round_bytes = sum(parts.values())
    stage_means = [statistics.mean(s) for s in stage_ms]
    dom = int(np.argmax(stage_means))
    stage_names = ["draft", "confidence", "schedule", "verify"]
    stage_bytes = [parts["draft_logits"] + parts["transition_W"] + parts["U_rows"], parts["hidden"],
                   w.B * w.G * 8, parts["target_rows"]]
    ach = stage_bytes[dom] / (stage_means[dom] * 1e-3) / 1e9
    # bf16 drafting is one persistent launch for every position (timed alone
    # in its stage graph); fp32 rounds launch a tile and a finalize kernel per
    # position.
    bf16 = w.dtype == "bf16"
    pair = bf16 and (w.B > 128 or args.head == "rnn")
    draft_kernel = ("markov_pair_tc (drafting on CTA pairs, all positions in one launch)" if pair else
                    "markov_tile_tc (drafting, all positions in one launch)") if bf16 else "draft stage"
    stage_kernels = [draft_kernel, "confidence_kernel", "schedule_kernel", "verify stage"]
    stage_launches = [1 if bf16 else 2 * w.G, 1, 1, 5]
    draft_flops = 2.0 * w.B * w.G * w.r * w.V
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded generator, one batch per rank)",
        "config": {"workload": w.name, "B": w.B, "G": w.G, "V": w.V, "r": w.r, "d": w.d,
                   "head": args.head,
                   "l2_flush": "256 MiB write before every timed round", "graph_replay": True,
                   "parallelism": f"{world} independent engines"},
        "round": {"admitted_draft_tokens": ell_sum, "emitted_tokens": nout_sum,
                  "rounds_per_s": world * 1e3 / ms, "emitted_tokens_per_s": nout_tot / (ms * 1e-3),
                  "algorithmic_bytes": round_bytes,
                  "hbm_roofline_frac": (round_bytes / (ms * 1e-3) / 1e9) / hbm_gbs,
                  "stage_ms": dict(zip(stage_names, stage_means)),
                  "near_ties_per_round": {"draft": ties_d / max(1, args.steps),
                                          "verify": ties_v / max(1, args.steps)}},
        "roofline": {"kernel": stage_kernels[dom], "bound": "hbm", "achieved": ach,
                     "peak": hbm_gbs, "unit": "GB/s", "frac": ach / hbm_gbs,
                     "traffic": profiled_traffic(w.name) if dom == 0 else None,
                     "algorithmic_bytes": stage_bytes[dom], "ms": stage_means[dom],
                     "launches": stage_launches[dom],
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)",
                     "tensor": ({"flops": draft_flops, "achieved_tflops": draft_flops / (stage_means[0] * 1e-3) / 1e12,
                                 "peak_tflops": bf16_tf, "frac": draft_flops / (stage_means[0] * 1e-3) / 1e12 / bf16_tf}
                                if dom == 0 else None)},
        "e2e": {"value": ell_tot / (e2e * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e},
        "gpu_launches": launches_per_round * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        t, secs, n = oracle_sample(w, inp, args.oracle_requests, A=Arec)
        cores = max(1, round(oracle_sample.cpu_s / secs))
        line["cpu_baseline"] = {"value": t / secs, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"{n} of {w.B} requests drafted+verified, whole-batch "
                                          f"confidence+schedule, {secs:.1f} s wall, "
                                          f"{oracle_sample.cpu_s:.1f} s CPU"}
    if rank == 0:
        print(json.dumps(line))
    graph.reset()
    for g in stage_graphs:
        g.reset()
    del graph, stage_graphs
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
