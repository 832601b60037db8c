#!/usr/bin/env python3
"""Benchmark: log-domain Sinkhorn half-iterations on B200, in cost-entries/s.

One step = the whole hot path over one synthetic problem, inputs resident in
HBM: fs_create (centring / packing / norms / log-weights), fs_solve for the
workload's iteration count (2 streamed LSE passes per iteration), then the
fused measurements fs_marginal_err and fs_ot_cost.  The metric counts n*m
cost entries per half-iteration of the solve (the three measurement passes
are timed but not counted).

    python bench.py [--gpus N --steps K --warmup W] [--workload highdim]
    python bench.py --impl reference      # the CPU oracle, timed on host cores

Multi-GPU (torchrun, one process per GPU): every rank solves its own replica
of the workload (no data-path collective); value = all ranks' entries / the
slowest rank's device time ("scaling": "weak").
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from log_domain_sinkhorn_updates_b200.workloads import WORKLOADS, make_problem  # noqa: E402

METRIC = "Sinkhorn cost-entries/s (n·m per half-iter) at n=m=65536,d=128; % of roofline"
UNIT = "cost-entries/s"
MUFU_EX2_PER_CLK_PER_SM = 16  # special-function-unit exp2 results per clock per SM
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "lse_tc_highdim_ncu.md")
PROFILE_TRAFFIC_APPLY = os.path.join(ROOT, "profiles", "apply_tc_highdim_ncu.md")
PROFILE_TRAFFIC_APPLY_Q2 = os.path.join(ROOT, "profiles", "apply_q2_highdim_ncu.md")
PROFILE_TRAFFIC_APPLY_Q2S = os.path.join(ROOT, "profiles", "apply_q2s_highdim_ncu.md")
# the transport kernels by the path the handle reports: (ncu summary, source file, description)
APPLY_KERNELS = {
    "tc_q2": (PROFILE_TRAFFIC_APPLY_Q2, "fs_apply_tc_q2.cu",
              "apply_q2_kernel (two 128-row blocks per CTA: S = Q K^T, P~ back into TMEM, O += P~ V~)"),
    "tc": (PROFILE_TRAFFIC_APPLY, "fs_apply_tc.cu", "apply_tc_kernel (S = Q K^T, then O += P~ V~)"),
    "tc_2s": (PROFILE_TRAFFIC_APPLY_Q2S, "fs_apply_tc_q2.cu",
              "apply_q2_kernel, one row block per CTA (both groups on alternate tiles, P~ in TMEM): the whole "
              "row blocks, then the column parts of those past the last full wave, then their merge; "
              "traffic per application"),
    "tc_pair": (None, "fs_apply_tc2.cu", "apply_tc2_kernel (CTA pairs: S = Q K^T, then O += P~ V~)"),
    "simt": (None, "fs_apply.cu", "apply_simt_kernel (CUDA cores)"),
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="highdim")
    ap.add_argument("--iters", type=int, default=None, help="override the workload's iteration count")
    ap.add_argument("--n", type=int, default=None, help="override n (profiling / small cases)")
    ap.add_argument("--m", type=int, default=None, help="override m")
    ap.add_argument("--batch", type=int, default=None, help="override the batch")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU-baseline sample duration")
    ap.add_argument("--shard", choices=["replicas", "rows"], default="replicas",
                    help="multi-GPU mode of --op solve: replicas (each rank solves its own copy of the workload, "
                         "weak scaling) or rows (one problem, rows and columns split over the ranks, the "
                         "potentials all-gathered after every half-iteration; strong scaling)")
    ap.add_argument("--op", choices=["solve", "transport", "hvp"], default="solve",
                    help="solve: the Sinkhorn solve (the headline); transport: the barycentric map at the "
                         "converged potentials (transport application, tensor-core kernel); hvp: the streaming "
                         "Hessian-vector product of the EOT cost in X at the converged potentials (batch 1)")
    return ap.parse_args()


def workload_config(prob, iters, extra=None):
    cfg = {
        "workload": (f"{prob.name}: batch={prob.batch}, n={prob.n}, m={prob.m}, d={prob.d}, {prob.dtype} inputs, "
                     f"eps={prob.eps}, {iters} alternating iterations from f=g=0"),
        "batch": prob.batch, "n": prob.n, "m": prob.m, "d": prob.d, "eps": prob.eps, "iters": iters,
        "half_iters_per_step": 2 * iters,
        "step": f"fs_create + fs_solve({iters}) + fs_marginal_err + fs_ot_cost",
        "l2": "flushed between steps (256 MiB write outside the timed events)",
        "seed": prob.seed,
    }
    if extra:
        cfg.update(extra)
    return cfg


# ----------------------------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ----------------------------------------------------------------------------------------------
def oracle_rows_timer(prob):
    import oracle
    X, Y, loga, logb = oracle.problem_arrays(prob, 0)
    g = np.zeros(prob.m)

    def run(rows):
        idx = np.arange(rows) % prob.n
        t0 = time.perf_counter()
        oracle.update_f_rows(idx, X, Y, logb, g, prob.eps)
        return time.perf_counter() - t0

    return run, oracle.num_threads()


def calibrated_rows(run, prob, seconds):
    probe = max(8, min(prob.n, 32))
    dt = run(probe)
    rate = probe * prob.m / max(dt, 1e-6)
    return int(max(8, min(prob.n, rate * seconds / prob.m))), rate


def cpu_baseline(prob, seconds):
    run, threads = oracle_rows_timer(prob)
    rows, _ = calibrated_rows(run, prob, seconds)
    dt = run(rows)
    return {"value": rows * prob.m / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": (f"fp64 C oracle f-update of {rows} rows x {prob.m} columns (d={prob.d}) of the {prob.name} "
                       f"workload, {dt:.1f} s on {threads} threads")}


def max_over_ranks(values, device=None):
    """Element-wise maximum of per-rank timings over all ranks of the default process group
    (identity on one process): every multi-GPU number is the slowest rank's."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def replica_throughput(world, steps, units_per_step, total_ms):
    """Whole-job throughput of `world` independent replicas: every rank processes
    units_per_step per step, timed as the slowest rank's total over `steps` steps."""
    return world * steps * units_per_step / (total_ms / 1e3)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    prob = make_problem(args.workload, n=args.n, m=args.m, batch=args.batch)
    iters = args.iters or prob.iters
    run, threads = oracle_rows_timer(prob)
    # each step: a bounded sample (~4 s) of the same half-iteration
    rows, _ = calibrated_rows(run, prob, 4.0)
    for _ in range(args.warmup):
        run(rows)
    times = [run(rows) for _ in range(args.steps)]
    total = sum(times)
    value = args.steps * rows * prob.m / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(prob, iters, {"step": f"oracle f-update of {rows} rows (bounded sample)",
                                                "half_iters_per_step": round(rows / prob.n, 6),
                                                "l2": "not applicable: host CPU oracle"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{rows} rows x {prob.m} columns per step, d={prob.d}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
            if self.gpu_id is not None:
                cmd += ["-i", str(self.gpu_id)]
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(", ") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], [], set()
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for name, flag in zip(self.NAMES, r[5:9]):
                if flag.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_identifier(torch, dev):
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return None


def profile_traffic(profile=PROFILE_TRAFFIC, source="fs_lse_tc.cu"):
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu summary, if the kernel
    source has not changed since the capture (else None)."""
    import hashlib
    try:
        txt = open(profile).read()
    except OSError:
        return None
    fields = dict(line.split(":", 1) for line in txt.splitlines() if line.startswith(("dram_bytes_per_launch:",
                                                                                       "kernel_source_sha256:")))
    src = os.path.join(ROOT, "log_domain_sinkhorn_updates_b200", "csrc", source)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if fields.get("kernel_source_sha256", "").strip() != sha:
        return None
    try:
        return float(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return json.load(fh), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


# ----------------------------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------------------------
def run_transport(args):
    """Barycentric map sum_j P_ij y_j / sum_j P_ij at the workload's converged potentials: one
    application per step, timed with CUDA events; roofline against the tensor pipe."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import log_domain_sinkhorn_updates_b200 as fs
    prob = make_problem(args.workload, n=args.n, m=args.m, batch=args.batch)
    B, n, m, d = prob.batch, prob.n, prob.m, prob.d
    if prob.dtype == "bf16":
        X = torch.from_numpy(prob.X_dev.view(np.int16)).view(torch.bfloat16).to(dev)
        Y = torch.from_numpy(prob.Y_dev.view(np.int16)).view(torch.bfloat16).to(dev)
    else:
        X, Y = torch.from_numpy(prob.X_dev).to(dev), torch.from_numpy(prob.Y_dev).to(dev)
    a = None if prob.a_dev is None else torch.from_numpy(prob.a_dev).to(dev)
    b = None if prob.b_dev is None else torch.from_numpy(prob.b_dev).to(dev)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    f = torch.zeros(B, n, device=dev)
    g = torch.zeros(B, m, device=dev)
    fs.fs_solve(h, f, g, args.iters or prob.iters)
    out = torch.empty(B, n, d, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush.zero_()
        fs.fs_barycentric_map(h, f, g, Y, out)
    fs.fs_sync(h)
    sampler = ClockSampler(gpu_identifier(torch, dev))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    launches0 = fs.fs_kernel_launches()
    tot = 0.0
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fs.fs_barycentric_map(h, f, g, Y, out)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        tot += e0.elapsed_time(e1)
    fs.fs_sync(h)
    launches = fs.fs_kernel_launches() - launches0
    clocks = sampler.stop()
    tot = max_over_ranks([tot], dev)[0]
    info = fs.fs_get_info(h)
    entries = B * n * m
    app_s = tot / 1e3 / args.steps
    # S = Q K^T in the handle's precision, then P~ (hi + lo) times V~ (one bf16 plane for bf16 Y, two else)
    npass_s = 3 if info["prec"] in ("3xtf32", "3xf16") else 1
    npass_o = 2 if prob.dtype == "bf16" else 3
    flops = 2.0 * entries * (d * npass_s + d * npass_o)
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", 1590.0))
    kprof, ksrc, kdesc = APPLY_KERNELS.get(info["last_apply_path"], (None, None, str(info["last_apply_path"])))
    line = {
        "metric": "transport application (barycentric map) cost-entries/s at the converged potentials",
        "value": replica_throughput(world, args.steps, entries, tot), "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if info["prec"] == "bf16" else "f32", "data": "synthetic",
        "config": workload_config(prob, args.iters or prob.iters, {
            "op": "fs_barycentric_map", "dv": d, "precision": info["prec"], "parallelism": f"replicas x{world}",
            "step": f"fs_barycentric_map at the potentials of fs_solve({args.iters or prob.iters}) (solve untimed)",
            "half_iters_per_step": 0}),
        "roofline": {"bound": "tensor", "achieved": flops / app_s / 1e12, "peak": peak, "unit": "TFLOP/s",
                     "frac": flops / app_s / 1e12 / peak,
                     # the committed capture is of the full highdim workload
                     "traffic": profile_traffic(kprof, ksrc)
                     if kprof and (args.workload, args.n, args.m, args.batch) == ("highdim", None, None, None)
                     else None,
                     "peak_source": peak_src,
                     "kernel": kdesc,
                     "flops_per_launch": flops},
        "cpu_baseline": None, "e2e": None, "clocks": clocks, "gpu_launches": int(launches),
    }
    fs.fs_destroy(h)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_hvp(args):
    """fs_hvp_x at the workload's converged potentials in a seeded direction, conjugate
    gradients to a relative residual of 1e-6: one product per step, timed with CUDA events
    (the product synchronises once per CG step; its host waits are inside the timed region)."""
    import torch
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    import log_domain_sinkhorn_updates_b200 as fs
    prob = make_problem(args.workload, n=args.n, m=args.m, batch=1)
    n, m, d = prob.n, prob.m, prob.d
    if prob.dtype == "bf16":
        X = torch.from_numpy(prob.X_dev.view(np.int16)).view(torch.bfloat16).to(dev)
        Y = torch.from_numpy(prob.Y_dev.view(np.int16)).view(torch.bfloat16).to(dev)
    else:
        X, Y = torch.from_numpy(prob.X_dev).to(dev), torch.from_numpy(prob.Y_dev).to(dev)
    a = None if prob.a_dev is None else torch.from_numpy(prob.a_dev).to(dev)
    b = None if prob.b_dev is None else torch.from_numpy(prob.b_dev).to(dev)
    h = fs.fs_create(X, Y, a, b, eps=prob.eps)
    f = torch.zeros(1, n, device=dev)
    g = torch.zeros(1, m, device=dev)
    fs.fs_solve(h, f, g, args.iters or prob.iters)
    V = torch.from_numpy(np.random.default_rng(200).standard_normal((1, n, d)).astype(np.float32)).to(dev)
    out = torch.empty(1, n, d, device=dev)
    stream = torch.cuda.current_stream(dev)
    its = 0
    for _ in range(args.warmup):
        its = fs.fs_hvp_x(h, f, g, X, Y, V, out, max_cg_iters=500, cg_rtol=1e-6)
    fs.fs_sync(h)
    sampler = ClockSampler(gpu_identifier(torch, dev))
    torch.cuda.synchronize(dev)
    sampler.start()
    launches0 = fs.fs_kernel_launches()
    tot = 0.0
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        its = fs.fs_hvp_x(h, f, g, X, Y, V, out, max_cg_iters=500, cg_rtol=1e-6)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        tot += e0.elapsed_time(e1)
    launches = fs.fs_kernel_launches() - launches0
    clocks = sampler.stop()
    info = fs.fs_get_info(h)
    line = {
        "metric": "streaming Hessian-vector product of the EOT cost in X (ms per product, CG to 1e-6)",
        "value": tot / args.steps, "unit": "ms", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot / args.steps, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if info["prec"] == "bf16" else "f32", "data": "synthetic",
        "config": workload_config(prob, args.iters or prob.iters, {
            "op": "fs_hvp_x", "cg_steps": int(its), "fused_term": bool(info["last_hvp_fused"]),
            "precision": info["prec"], "step": "fs_hvp_x at the potentials of the solve (solve untimed)",
            "half_iters_per_step": 0, "l2": "not flushed (a product is tens of passes over the same operands)"}),
        "cpu_baseline": None, "e2e": None, "clocks": clocks, "gpu_launches": int(launches),
    }
    fs.fs_destroy(h)
    print(json.dumps(line), flush=True)
    return 0


def run_row_sharded(args):
    """One problem per job, its rows split over the ranks (log_domain_sinkhorn_updates_b200.sharded):
    each rank updates its share of f, then of g, and the slices are all-gathered (NCCL) after
    every half-iteration.  value = the problem's entries per half-iteration x 2 iters / the
    slowest rank's device time ("scaling": "strong")."""
    import torch
    import torch.distributed as dist
    from log_domain_sinkhorn_updates_b200.sharded import DistGather, FsShard, LocalGather, shard_ranges, \
        solve_row_sharded
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import log_domain_sinkhorn_updates_b200 as fs
    prob = make_problem(args.workload, n=args.n, m=args.m, batch=args.batch)
    iters = args.iters or prob.iters
    B, n, m = prob.batch, prob.n, prob.m
    if prob.dtype == "bf16":
        X = torch.from_numpy(prob.X_dev.view(np.int16)).view(torch.bfloat16).to(dev)
        Y = torch.from_numpy(prob.Y_dev.view(np.int16)).view(torch.bfloat16).to(dev)
    else:
        X, Y = torch.from_numpy(prob.X_dev).to(dev), torch.from_numpy(prob.Y_dev).to(dev)
    a = None if prob.a_dev is None else torch.from_numpy(prob.a_dev).to(dev)
    b = None if prob.b_dev is None else torch.from_numpy(prob.b_dev).to(dev)
    rr, _ = shard_ranges(n, world)
    cc, _ = shard_ranges(m, world)
    shard = FsShard(X, Y, a, b, prob.eps, rr[rank], cc[rank])
    gather = DistGather() if world > 1 else LocalGather()
    for _ in range(args.warmup):
        solve_row_sharded([shard], gather, n, m, B, world, 2, device=dev)
    sampler = ClockSampler(gpu_identifier(torch, dev))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    launches0 = fs.fs_kernel_launches()
    stream = torch.cuda.current_stream(dev)
    tot = 0.0
    f = g = None
    for _ in range(args.steps):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        f, g = solve_row_sharded([shard], gather, n, m, B, world, iters, device=dev)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        tot += e0.elapsed_time(e1)
    launches = fs.fs_kernel_launches() - launches0
    clocks = sampler.stop()
    tot = max_over_ranks([tot], dev)[0]
    value = args.steps * 2 * iters * B * n * m / (tot / 1e3)
    shard.close()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot / args.steps, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": prob.dtype, "data": "synthetic",
        "config": workload_config(prob, iters, {
            "step": f"row-sharded fs_update_f / fs_update_g x {iters}, all-gather after every half-iteration",
            "parallelism": f"rows x{world}", "l2": "not flushed (the shards stay resident)"}),
        "cpu_baseline": None, "e2e": None, "clocks": clocks, "gpu_launches": int(launches),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.shard == "rows" and args.op == "solve":
        return run_row_sharded(args)
    if args.op == "transport":
        return run_transport(args)
    if args.op == "hvp":
        return run_hvp(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    import log_domain_sinkhorn_updates_b200 as fs
    from log_domain_sinkhorn_updates_b200 import binding

    prob = make_problem(args.workload, n=args.n, m=args.m, batch=args.batch)
    iters = args.iters or prob.iters
    B, n, m, d = prob.batch, prob.n, prob.m, prob.d
    if prob.dtype == "bf16":
        Xh = torch.from_numpy(prob.X_dev.view(np.int16)).view(torch.bfloat16)
        Yh = torch.from_numpy(prob.Y_dev.view(np.int16)).view(torch.bfloat16)
    else:
        Xh = torch.from_numpy(prob.X_dev)
        Yh = torch.from_numpy(prob.Y_dev)
    X, Y = Xh.to(dev), Yh.to(dev)
    a = None if prob.a_dev is None else torch.from_numpy(prob.a_dev).to(dev)
    b = None if prob.b_dev is None else torch.from_numpy(prob.b_dev).to(dev)
    f = torch.zeros(B, n, device=dev)
    g = torch.zeros(B, m, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    results = {}

    def step(ev=None):
        g.zero_()
        h = fs.fs_create(X, Y, a, b, eps=prob.eps)
        if ev:
            ev[0].record(stream)
        fs.fs_solve(h, f, g, iters)
        if ev:
            ev[1].record(stream)
        er, ec = fs.fs_marginal_err(h, f, g)
        dual, primal = fs.fs_ot_cost(h, f, g)
        results.update(err_row=er.tolist(), err_col=ec.tolist(), dual=dual.tolist(), primal=primal.tolist(),
                       info=fs.fs_get_info(h))
        fs.fs_destroy(h)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(gpu_identifier(torch, dev))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    launches0 = fs.fs_kernel_launches()
    evs = []
    for _ in range(args.steps):
        flush.zero_()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record(stream)
        step((e[1], e[2]))
        e[3].record(stream)
        evs.append(e)
    torch.cuda.synchronize(dev)
    launches = fs.fs_kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()

    step_ms = sum(e[0].elapsed_time(e[3]) for e in evs)
    solve_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    step_ms, solve_ms = max_over_ranks([step_ms, solve_ms], dev)

    entries_per_half = B * n * m
    half_per_step = 2 * iters
    value = replica_throughput(world, args.steps, half_per_step * entries_per_half, step_ms)

    # ---- roofline of the dominant kernel (the streamed LSE pass) ----
    peaks, peak_src = load_peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    pass_s = solve_ms / 1e3 / (args.steps * half_per_step)  # one bias launch per solve is included
    ex2_rate = entries_per_half / pass_s
    ex2_peak = sms * MUFU_EX2_PER_CLK_PER_SM * sm_max * 1e6
    flops = 2.0 * entries_per_half * d * (3 if results["info"]["prec"] == "3xtf32" else 1)
    roofline = {
        "bound": "alu", "achieved": ex2_rate / 1e9, "peak": ex2_peak / 1e9, "unit": "Gexp2/s",
        "frac": ex2_rate / ex2_peak, "traffic": profile_traffic(),
        "kernel": "lse_tc_kernel (streamed LSE pass)", "pass_ms": pass_s * 1e3,
        "peak_basis": f"{sms} SMs x {MUFU_EX2_PER_CLK_PER_SM} ex2/clk x {sm_max:.0f} MHz (MUFU)",
        "tensor": {"achieved": flops / pass_s / 1e12, "peak": float(peaks.get("bf16_tflops", 1590.0)),
                   "unit": "TFLOP/s", "frac": flops / pass_s / 1e12 / float(peaks.get("bf16_tflops", 1590.0)),
                   "peak_source": peak_src},
        # per point: its operand row, norm, log-weight and potential, and its 32-byte bias row
        "algorithmic_bytes_per_launch": (n + m) * B * (d * (2 if prob.dtype == "bf16" else 4) + 44),
    }
    if clocks and clocks.get("sm_mhz"):
        roofline["frac_at_median_clock"] = ex2_rate / (sms * MUFU_EX2_PER_CLK_PER_SM * clocks["sm_mhz"] * 1e6)

    # ---- end to end through the host entry point (pinned host buffers) ----
    e2e = None
    if not args.no_e2e:
        Xp = Xh.pin_memory()
        Yp = Yh.pin_memory()
        ap = None if prob.a_dev is None else torch.from_numpy(prob.a_dev).pin_memory()
        bp = None if prob.b_dev is None else torch.from_numpy(prob.b_dev).pin_memory()
        g0 = torch.zeros(B, m).pin_memory()
        fo = torch.empty(B, n).pin_memory()
        go = torch.empty(B, m).pin_memory()
        xn = Xp.view(torch.int16).numpy() if prob.dtype == "bf16" else Xp.numpy()
        yn = Yp.view(torch.int16).numpy() if prob.dtype == "bf16" else Yp.numpy()

        def host_step():
            binding.fs_solve_host(xn, yn, None if ap is None else ap.numpy(), None if bp is None else bp.numpy(),
                                  g0.numpy(), prob.eps, iters, dtype=prob.dtype, stream=stream,
                                  out=(fo.numpy(), go.numpy()))

        for _ in range(max(1, args.warmup)):
            host_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        tot = 0.0
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            host_step()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            tot += e0.elapsed_time(e1)
        tot = max_over_ranks([tot], dev)[0]
        h2d = Xh.numel() * Xh.element_size() + Yh.numel() * Yh.element_size() + g0.numel() * 4
        h2d += 0 if ap is None else ap.numel() * 4
        h2d += 0 if bp is None else bp.numel() * 4
        d2h = (fo.numel() + go.numel()) * 4 + 4 * B * 8
        e2e = {"value": replica_throughput(world, args.steps, half_per_step * entries_per_half, tot), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": tot / args.steps,
               "api": "fs_solve_host (C ABI, pinned host buffers)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(prob, args.cpu_seconds)

    info = results["info"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if info["prec"] == "bf16" else ("tf32" if "tf32" in info["prec"] else "f32"),
        "data": "synthetic",
        "config": workload_config(prob, iters, {
            "precision": info["prec"], "accumulate": "f32", "splits_f": info["splits_f"],
            "splits_g": info["splits_g"], "stages": info["stages"], "parallelism": f"replicas x{world}"}),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "gpu_launches": int(launches),
        "results": {k: results[k] for k in ("err_row", "err_col", "dual", "primal")},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
