"""Benchmark: one blocked-Shampoo optimizer step on B200 (blocks/s, ms/step).

python bench.py [--gpus N] [--steps K] [--warmup W] [--config transformer]
                [--dtype fp32] [--impl ours|reference]

A step is the whole hot path on one batch of synthetic gradients: gather the
gradient blocks into stacks, update the statistics, compute every inverse
fourth root (Newton-DB after power-iteration scaling), precondition, graft
onto Adam and update the weights.  Inputs are seeded synthetic data already
resident in HBM; they are larger than L2 (no flush needed).  Rank 0 prints
one JSON line.  Under torchrun each rank runs its own independent copy of the
workload (weak scaling, no collective on the data path).

`--impl reference` times the float64 CPU oracle on the host cores on a
bounded sample of the same workload (the reference arm); only rank 0 runs.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

# ---------------------------------------------------------------- workloads --

CONFIGS = {
    # 8 transformer layers, d = 1024, FFN 4096, blocked at 1024: 96 blocks.
    "transformer": dict(kind="transformer", workload="transformer_8x1024_ffn4096_b1024", shapes="transformer", block_size=1024,
                        beta2=0.999, alpha=1.0, eps=1e-6, method="ndb", iters=20, scaling="power",
                        graft="adam", lr=1e-3, weight_decay=0.0),
    # 256 blocks of 128 x 128 (each block its own layer).
    "lowrank_stack": dict(kind="lowrank_stack", workload="stack_256x128x128", shapes=[(128, 128)] * 256, block_size=128,
                          beta2=0.999, alpha=1.0, eps=1e-6, method="ndb", iters=15, scaling="frobenius",
                          graft="adam", lr=1e-3, weight_decay=0.0),
    # 32 blocks of 2048 x 2048.
    "large_blocks": dict(kind="large_blocks", workload="stack_32x2048x2048", shapes=[(2048, 2048)] * 32, block_size=2048,
                         beta2=0.999, alpha=1.0, eps=1e-6, method="ndb", iters=20, scaling="frobenius",
                         graft="adam", lr=1e-3, weight_decay=0.01),
    # one 256 x 256 weight in 16 blocks of 64 x 64
    "tiny_dense": dict(kind="tiny_dense", workload="dense_256x256_b64", shapes=[(256, 256)], block_size=64, beta2=1.0, alpha=1.0,
                       eps=1e-6, method="ndb", iters=20, scaling="frobenius", graft="sgd", lr=0.1,
                       weight_decay=0.0),
}


def shapes_of(cfg):
    from matrix_roots_b200 import workloads as W
    return W.transformer_shapes() if cfg["shapes"] == "transformer" else list(cfg["shapes"])


def make_grads(shapes, seed, kind="transformer"):
    """One gradient per layer with the workload's value distribution."""
    from matrix_roots_b200 import workloads as W
    if kind == "lowrank_stack":
        g = W.lowrank_stack_grads(steps=1, blocks=len(shapes), n=shapes[0][0], seed=seed)[0]
        return [g[i] for i in range(len(shapes))]
    if kind == "large_blocks":
        g = W.large_block_grads(steps=1, blocks=len(shapes), n=shapes[0][0], seed=seed)[0]
        return [g[i] for i in range(len(shapes))]
    if kind == "tiny_dense":
        return [W.tiny_dense_grads(steps=1, rows=m, cols=n, seed=seed)[0] for (m, n) in shapes]
    return W.transformer_grads(shapes, seed=seed)


# DRAM bytes per launch of the FP32 GEMM on the transformer workload: mean
# over the 121 launches of the ncu launch list in
# profiles/launches_transformer_step.txt (current kernel)
GEMM_DRAM_BYTES_PER_LAUNCH = 3482.4e6


def root_flops(n, count, method, iters, scaling, pi_vectors, pi_iters, dense=False):
    """Algorithmic FLOPs of one shampoo_inv_root call: 2 n^3 per product of
    the coupled iterations; the Chebyshev products are computed as symmetric
    matrices, so their algorithmic work is that of the n(n+1)/2 distinct
    entries, n^2 (n+1) flops (``dense`` counts 2 n^3 for them too)."""
    if method == "ndb":
        mm = 2 * (3 * iters - 3) if iters >= 2 else 2
    elif method == "cn":
        mm = 4 * iters - 4 if iters >= 2 else 0
    else:
        mm = max(iters - 1, 0)
    f = mm * (n * n * (n + 1.0) if (method == "cheb" and not dense) else 2.0 * n ** 3)
    if scaling == "power":
        f += (pi_iters + 1) * 2.0 * n * n * pi_vectors
    return f * count


# ------------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------- distributed --

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local):
    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))


def barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x, world):
    import torch
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ peaks ----

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"], "bf16_sust": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sust": 1400.0, "source": "fallback"}


# ----------------------------------------------------------- cpu baseline ----

def cpu_threads():
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count()
    blas = None
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        blas = max((i.get("num_threads", 0) for i in info), default=None)
    except Exception:
        pass
    return cores, blas


def oracle_blocks_per_s(cfg, shapes, sample_blocks, seed=0):
    """Times the oracle's step on `sample_blocks` gradient blocks of the workload."""
    import oracle as O
    from matrix_roots_b200 import workloads as W
    B = cfg["block_size"]
    sub = []
    for (m, n) in shapes:
        sub.append((min(m, B), min(n, B)))
        if len(sub) >= sample_blocks:
            break
    grads = make_grads(sub, seed, kind=cfg["kind"])
    st = O.ShampooState(sub, B, cfg["graft"])
    Wt = [np.zeros(s) for s in sub]
    starts = None
    if cfg["scaling"] == "power":
        starts = W.power_iteration_starts(min(B, max(max(s) for s in sub)), 16)
    t0 = time.perf_counter()
    O.shampoo_step(st, Wt, grads, beta2=cfg["beta2"], alpha=cfg["alpha"], eps=cfg["eps"], method=cfg["method"],
                   iters=cfg["iters"], scaling=cfg["scaling"], graft=cfg["graft"], lr=cfg["lr"],
                   wd=cfg["weight_decay"], pi_starts=starts, pi_iters=10)
    dt = time.perf_counter() - t0
    nblocks = len(O.plan_blocks(sub, B)["blocks"])
    return nblocks / dt, dt, nblocks


def arm_config(cfg, n_blocks, n_factors, world):
    """The `config` object both arms print for a workload."""
    return {"workload": cfg["workload"], "blocks_per_gpu": int(n_blocks), "factors_per_gpu": int(n_factors),
            "method": cfg["method"], "iters": cfg["iters"], "scaling": cfg["scaling"], "graft": cfg["graft"],
            "l2": "inputs larger than L2 (no flush)", "parallelism": f"replicas x{world}"}


def oracle_one_core(cfg, shapes):
    """The oracle's step on one block with the BLAS pool limited to one thread."""
    try:
        import threadpoolctl
        with threadpoolctl.threadpool_limits(limits=1):
            rate, dt, nb = oracle_blocks_per_s(cfg, shapes, 1)
        return {"value": rate, "cores": 1, "sample": f"{nb} gradient block, one oracle step ({dt:.1f} s)"}
    except Exception:  # threadpoolctl missing or no BLAS pool to limit
        return None


# ------------------------------------------------------------------ arms -----

def plan_counts(cfg, shapes):
    """Gradient blocks and factors of the workload on one GPU (oracle planner)."""
    import oracle as O
    plan = O.plan_blocks(shapes, cfg["block_size"])
    return len(plan["blocks"]), int(sum(int(c) for _, c in plan["f_buckets"]))


def run_reference(args, cfg):
    world, rank, local = dist_env()
    if rank != 0:
        return
    shapes = shapes_of(cfg)
    cores, blas = cpu_threads()
    for _ in range(args.warmup):
        oracle_blocks_per_s(cfg, shapes, 1)
    times, nb = [], 0
    for _ in range(args.steps):
        _, dt, nb = oracle_blocks_per_s(cfg, shapes, 1)
        times.append(dt)
    ms = 1000 * statistics.median(times)
    value = nb / (ms / 1000)
    sample = f"{nb} gradient block(s) of {cfg['workload']} per step (oracle float64 step: stats, eigen-replayed " \
             f"{cfg['method']} roots, direction, graft)"
    out = {"metric": "shampoo optimizer step throughput", "value": value, "unit": "blocks/s", "impl": "reference",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": arm_config(cfg, *plan_counts(cfg, shapes), world),
           "cpu_baseline": {"value": value, "unit": "blocks/s", "cores": blas or cores, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": "blocks/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_ours(args, cfg):
    import torch
    from matrix_roots_b200 import binding as B
    from matrix_roots_b200 import build
    from matrix_roots_b200.optimizer import BlockedShampoo, ShampooConfig

    world, rank, local = dist_env()
    build.build()
    init_dist(world, local)
    dev = torch.device("cuda", local)
    shapes = shapes_of(cfg)
    scfg = ShampooConfig(block_size=cfg["block_size"], beta2=cfg["beta2"], alpha=cfg["alpha"], eps=cfg["eps"],
                         method=cfg["method"], iters=cfg["iters"], dtype=args.dtype, stats_dtype=args.dtype,
                         precond_dtype=args.dtype, scaling=cfg["scaling"], graft=cfg["graft"], lr=cfg["lr"],
                         weight_decay=cfg["weight_decay"], graph=args.graph, layerwise=args.layerwise)
    opt = BlockedShampoo(shapes, scfg, dev)
    grads_np = make_grads(shapes, seed=rank, kind=args.config)
    G = [torch.from_numpy(g).to(dev) for g in grads_np]
    W = [torch.zeros(s, dtype=torch.float32, device=dev) for s in shapes]
    stream = torch.cuda.current_stream(dev)
    n_blocks = opt.plan.n_blocks

    # root timing hooks: events around every inv_root call of the timed steps
    root_events = []

    c = scfg
    ws = opt.workspace

    def part_stats():
        B.stack_blocks(opt.plan, G, opt.g_stacks)
        B.update_stats(opt.plan, opt.g_stacks, opt.factors, c.beta2, c.alpha, c.stats_dtype, ws)

    def part_root(fb):
        n = int(opt.tables["f_buckets"][fb][0])
        B.inv_root(opt.factors[fb], c.eps, c.method, c.iters, c.dtype, c.scaling, 4, c.pi_vectors, c.pi_iters,
                   opt.pi_starts.get(n), opt.roots[fb], opt.scales[fb], opt.status[fb], ws)

    def part_precond():
        B.precondition(opt.plan, opt.roots, opt.g_stacks, opt.d_stacks, opt.dnorm2, c.precond_dtype, ws)

    def root_flops_of(fbs):
        return sum(root_flops(int(opt.tables["f_buckets"][fb][0]), int(opt.tables["f_buckets"][fb][1]), c.method,
                              c.iters, c.scaling, c.pi_vectors, c.pi_iters) for fb in fbs)

    buckets = list(range(len(opt.tables["f_buckets"])))
    graphs = {}

    def run_part(name, fn):
        if name in graphs:
            graphs[name][0].replay()
            opt.graph_launches += graphs[name][1]
        else:
            fn()

    def step(timed):
        opt.t += 1
        run_part("stats", part_stats)
        if graphs:  # all root calls replay as one graph
            if timed:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            run_part("roots", None)
            if timed:
                e1.record(stream)
                root_events.append((e0, e1, root_flops_of(buckets)))
        else:
            for fb in buckets:
                if timed:
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                part_root(fb)
                if timed:
                    e1.record(stream)
                    root_events.append((e0, e1, root_flops_of([fb])))
        run_part("precond", part_precond)
        B.graft_step(opt.plan, W, G, opt.d_stacks, opt.dnorm2, opt.m, opt.v, c.graft, c.lr, c.beta1,
                     c.graft_beta2, c.graft_eps, c.weight_decay, opt.t, c.graft_per_block, ws)

    for _ in range(args.warmup):
        step(False)
    if args.graph:  # capture after the eager warm-up; the graft step stays direct (its step count changes)
        torch.cuda.synchronize(dev)
        for name, fn in (("stats", part_stats), ("roots", lambda: [part_root(fb) for fb in buckets]),
                         ("precond", part_precond)):
            gr = torch.cuda.CUDAGraph()
            before = B.launch_count()
            with torch.cuda.graph(gr):
                fn()
            graphs[name] = (gr, B.launch_count() - before)
        step(False)
    barrier(world)
    assert B.device_error() == 0, "a kernel reported a barrier timeout during warm-up"
    for s in opt.status:
        assert int(s.abs().sum()) == 0, "non-finite root during warm-up"

    l0, g0 = B.launch_count(), opt.graph_launches
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier(world)
        t0.record(stream)
        for _ in range(args.steps):
            step(True)
        t1.record(stream)
        barrier(world)
    launches = B.launch_count() - l0 + (opt.graph_launches - g0)  # graph replays count their kernels
    ms_total = t0.elapsed_time(t1)
    ms_max = max_over_ranks(ms_total, world)
    ms_step = ms_max / args.steps
    value = world * n_blocks * args.steps / (ms_max / 1000.0)

    # roofline of the dominant kernel (the tcgen05 GEMM engine inside inv_root)
    root_ms = sum(a.elapsed_time(b) for a, b, _ in root_events) / args.steps
    flops = sum(f for _, _, f in root_events) / args.steps
    peaks = load_peaks()
    # MMA work per algorithmic flop, in units of the dense fp16/bf16 rate:
    # FP32 = three fp16 passes (hi*hi, lo*hi, hi*lo); TF32 runs at half rate
    passes = {"fp32": 3.0, "tf32": 2.0, "fp16": 1.0, "bf16": 1.0}[args.dtype]
    peak = peaks["bf16_sust"] / passes
    achieved = flops / (root_ms / 1000.0) / 1e12
    # DRAM bytes per launch of the FP32 GEMM on this workload (ncu launch
    # list of the transformer step); other workloads / dtypes not captured
    traffic = GEMM_DRAM_BYTES_PER_LAUNCH if (args.config == "transformer" and args.dtype == "fp32") else None
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": traffic, "traffic_unit": "DRAM bytes per launch (read + write)",
                "kernel": "gemm_kernel (all launches inside shampoo_inv_root)",
                "peak_note": f"{peaks['source']} sustained bf16 rate / {passes:g} (fp16-rate MMA work per "
                             f"algorithmic flop, {args.dtype})",
                "root_ms_per_step": root_ms, "root_tflop_per_step": flops / 1e12}

    # end to end through the public API with host-resident gradients and weights
    e2e = None
    if not args.no_e2e:
        G_host = [g.cpu().pin_memory() for g in G]
        W_host = [torch.empty(s, dtype=torch.float32).pin_memory() for s in shapes]
        h2d = sum(g.numel() * 4 for g in G_host)
        d2h = sum(w.numel() * 4 for w in W_host)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        e0.record(stream)
        for _ in range(args.steps):
            for gd, gh in zip(G, G_host):
                gd.copy_(gh, non_blocking=True)
            step(False)
            for wh, wd in zip(W_host, W):
                wh.copy_(wd, non_blocking=True)
        e1.record(stream)
        barrier(world)
        e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": world * n_blocks * args.steps / (e_ms / 1000.0), "unit": "blocks/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms / args.steps}

    out = None
    if rank == 0:
        out = {"metric": "shampoo optimizer step throughput", "value": value, "unit": "blocks/s",
               "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
               "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
               "dtype": {"fp32": "f32 (3 fp16 tensor-core passes on a scaled hi/lo split)", "tf32": "tf32",
                         "fp16": "f16", "bf16": "bf16"}[args.dtype],
               "data": "synthetic",
               "config": dict(arm_config(cfg, n_blocks, sum(int(c) for _, c in opt.tables["f_buckets"]), world),
                              cuda_graph=bool(args.graph), stacking="layerwise" if args.layerwise else "global"),
               "roofline": roofline, "e2e": e2e, "gpu_launches": launches,
               "clocks": clocks.summary()}
        if world == 1 and not args.no_cpu:
            cores, blas = cpu_threads()
            rate, dt, nb = oracle_blocks_per_s(cfg, shapes, args.cpu_blocks)
            out["cpu_baseline"] = {"value": rate, "unit": "blocks/s", "cores": blas or cores, "kind": "oracle",
                                   "sample": f"{nb} of the {n_blocks} gradient blocks, one oracle step "
                                             f"({dt:.1f} s)", "one_core": oracle_one_core(cfg, shapes)}
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


SPD_METHODS = [("cheb", 32, "fp32"), ("cheb", 32, "fp16"), ("ndb", 20, "fp32"), ("cn", 20, "fp16"),
               ("cn", 20, "bf16")]


def run_spd(args):
    """Ill-conditioned roots: 512 SPD 256^2 matrices Q diag(lam) Q^T, lam
    log-uniform in [1e-6, 1], eps = 1e-8, Frobenius scaling; every method and
    precision of the workload timed as shampoo_inv_root calls on
    device-resident inputs (CUDA events; each call streams 3-5 work stacks
    of 128 MB, larger than L2).  value = NDB-20 FP32 matrices/s; all
    methods under "methods"."""
    import torch
    from matrix_roots_b200 import binding as B
    from matrix_roots_b200 import build
    from matrix_roots_b200 import workloads as W
    build.build()
    A32, _, _ = W.spd_stack(512, 256, seed=0)
    A = torch.from_numpy(A32).cuda()
    count, n = A.shape[0], A.shape[1]
    peaks = load_peaks()
    rows = {}
    l0 = B.launch_count()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        run_spd_methods(A, count, n, args, peaks, rows)
    launches = B.launch_count() - l0
    ref = rows["ndb20_fp32"]
    out = {"metric": "inverse-root throughput (ill-conditioned SPD stack)", "value": ref["matrices_per_s"],
           "unit": "matrices/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ref["ms"],
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 (3 fp16 passes)",
           "data": "synthetic",
           "config": {"workload": "spd_512x256_logunif_1e-6_1", "eps": 1e-8, "scaling": "frobenius",
                      "l2": "workspace larger than L2 (no flush)"},
           "roofline": {"bound": "tensor", "achieved": ref["tflops_algorithmic"],
                        "peak": peaks["bf16_sust"] / 3.0, "unit": "TFLOP/s", "frac": ref["frac"], "traffic": None,
                        "kernel": "gemm_kernel (NDB-20 FP32)"},
           "methods": rows, "gpu_launches": launches, "clocks": clocks.summary()}
    print(json.dumps(out), flush=True)


def run_spd_methods(A, count, n, args, peaks, rows):
    import torch
    from matrix_roots_b200 import binding as B
    for method, iters, dtype in SPD_METHODS:
        ws = torch.empty(B.inv_root_workspace_bytes(count, n, method, dtype, "frobenius"), dtype=torch.uint8,
                         device="cuda")
        for _ in range(args.warmup):
            B.inv_root(A, 1e-8, method, iters, dtype, "frobenius", workspace=ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            B.inv_root(A, 1e-8, method, iters, dtype, "frobenius", workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        fl = root_flops(n, count, method, iters, "frobenius", 0, 0)
        passes = {"fp32": 3.0, "tf32": 2.0, "fp16": 1.0, "bf16": 1.0}[dtype]
        rows[f"{method}{iters}_{dtype}"] = {"ms": ms, "matrices_per_s": count / (ms / 1000.0),
                                           "tflops_algorithmic": fl / (ms / 1000.0) / 1e12,
                                           "frac": fl / (ms / 1000.0) / 1e12 / (peaks["bf16_sust"] / passes)}
        del ws


EVD_HEURISTIC_NAMES = ["corrected", "shifted_relu", "abs_add", "shmp"]


def evd_fp64_flops(n, sweeps) -> float:
    """Float64 work of the Jacobi solves: per sweep n(n-1)/2 rotations, each
    updating two rows and two columns of A (n element pairs each, 2 fused
    multiply-adds per element: 8 flops per pair)."""
    return float(np.sum(sweeps)) * (n * (n - 1) / 2) * 16.0 * n


def run_evd(args):
    """EVD roots against the iterative ones on C2's factor shape: 512 SPD
    128^2 matrices Q diag(lam) Q^T, lam log-uniform in [1e-6, 1], eps = 1e-8.
    Times shampoo_inv_root_evd for each dampening heuristic and, on the same
    stack, Newton-DB-20 and coupled Newton-20 in FP32 (CUDA events, inputs
    resident).  value = EVD (corrected spectrum) matrices/s; the roofline is
    the float64 ALU work of the sweeps the solver reports, against the
    float64 FMA rate of 148 SMs x 64 lanes at the sampled SM clock."""
    import torch
    from matrix_roots_b200 import binding as B
    from matrix_roots_b200 import build
    from matrix_roots_b200 import workloads as W
    build.build()
    A32, _, _ = W.spd_stack(512, 128, seed=0)
    A = torch.from_numpy(A32).cuda()
    count, n = A.shape[0], A.shape[1]
    peaks = load_peaks()
    rows = {}
    X = torch.empty_like(A)
    st = torch.empty(count, dtype=torch.int32, device="cuda")
    l0 = B.launch_count()
    with ClockSampler(torch.cuda.current_device()) as clocks:
        for h in EVD_HEURISTIC_NAMES:
            for _ in range(args.warmup):
                B.inv_root_evd(A, 1e-8, h, out=X, status_out=st)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(args.steps):
                B.inv_root_evd(A, 1e-8, h, out=X, status_out=st)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / args.steps
            s_np = st.cpu().numpy()
            sweeps = s_np >> 8
            rows[f"evd_{h}"] = {"ms": ms, "matrices_per_s": count / (ms / 1000.0),
                                "sweeps_mean": float(sweeps.mean()), "sweeps_max": int(sweeps.max()),
                                "unconverged": int(((s_np & 0xff) != 0).sum()),
                                "fp64_tflops": evd_fp64_flops(n, sweeps) / (ms / 1000.0) / 1e12}
        for method in ("ndb", "cn"):
            ws = torch.empty(B.inv_root_workspace_bytes(count, n, method, "fp32", "frobenius"), dtype=torch.uint8,
                             device="cuda")
            for _ in range(args.warmup):
                B.inv_root(A, 1e-8, method, 20, "fp32", "frobenius", workspace=ws)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(args.steps):
                B.inv_root(A, 1e-8, method, 20, "fp32", "frobenius", workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / args.steps
            rows[f"{method}20_fp32"] = {"ms": ms, "matrices_per_s": count / (ms / 1000.0)}
    launches = B.launch_count() - l0
    cs = clocks.summary()
    ref = rows["evd_corrected"]
    mhz = cs.get("sm_mhz") or 1965.0
    peak = 148 * 64 * 2 * mhz * 1e6 / 1e12
    out = {"metric": "inverse-root throughput, EVD (SPD stack)", "value": ref["matrices_per_s"],
           "unit": "matrices/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ref["ms"],
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f64 Jacobi rotations, f32 eigenvectors and roots", "data": "synthetic",
           "config": {"workload": "spd_512x128_logunif_1e-6_1", "eps": 1e-8,
                      "l2": "inputs 32 MB, resident in L2 (one CTA per matrix reads it once)"},
           "roofline": {"bound": "alu", "achieved": ref["fp64_tflops"], "peak": peak, "unit": "TFLOP/s (fp64)",
                        "frac": ref["fp64_tflops"] / peak, "traffic": None,
                        "kernel": "evd_root_kernel (corrected spectrum)",
                        "peak_note": "148 SMs x 64 fp64 FMA lanes x 2 x sampled SM clock"},
           "methods": rows, "gpu_launches": launches, "clocks": cs}
    print(json.dumps(out), flush=True)


def run_root_stack(args):
    """Small fixed case of the dominant kernel for profilers: Newton-DB-20
    on `args.root_stack` factors L = G G^T of transformer gradient blocks
    (1024^2), two shampoo_inv_root calls; prints one JSON line."""
    import torch
    from matrix_roots_b200 import binding as B
    from matrix_roots_b200 import build
    from matrix_roots_b200 import workloads as W
    build.build()
    k = args.root_stack
    g = W.transformer_grads([(1024, 1024)] * k, seed=0)
    L = np.stack([(x.astype(np.float64) @ x.astype(np.float64).T).astype(np.float32) for x in g])
    A = torch.from_numpy(L).cuda()
    ws = torch.empty(B.inv_root_workspace_bytes(k, 1024, "ndb", args.dtype, "frobenius"), dtype=torch.uint8,
                     device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    B.inv_root(A, 1e-6, "ndb", 20, args.dtype, "frobenius", workspace=ws)
    e0.record()
    X, s, st = B.inv_root(A, 1e-6, "ndb", 20, args.dtype, "frobenius", workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    assert B.device_error() == 0 and int(st.abs().sum()) == 0
    print(json.dumps({"case": f"ndb20_{args.dtype}_{k}x1024", "ms": e0.elapsed_time(e1)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--root-stack", type=int, default=0,
                    help="profile case: Newton-DB roots of this many 1024^2 factors, then exit")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="transformer", choices=sorted(CONFIGS) + ["spd_stack", "evd_stack"])
    ap.add_argument("--dtype", default="fp32", choices=["fp32", "tf32", "fp16", "bf16"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layerwise", action="store_true",
                    help="stack blocks per layer (DASH-LAYERWISE) instead of across all layers")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step's launches before the graft step as a CUDA graph")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-blocks", type=int, default=4)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.root_stack:
        run_root_stack(args)
        return
    if args.config == "spd_stack":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm covers the optimizer-step "
                                                                  "workloads; spd_stack times inverse roots only"}))
            return
        run_spd(args)
        return
    if args.config == "evd_stack":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the reference arm covers the optimizer-step "
                                                                  "workloads; evd_stack times inverse roots only"}))
            return
        run_evd(args)
        return
    cfg = CONFIGS[args.config]
    if args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
