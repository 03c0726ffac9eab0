"""Benchmark of the on-the-fly equivariant attention hot path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole path on one batch: the cell-list CSR build plus the
fused attention forward (projections, edge geometry, Wigner-D, logits,
online softmax, SO(2) block products, back-rotation, accumulation).
Workload: 256 drug-like molecules of 20-60 atoms (N = 10,304 atoms, about
395k directed edges within r_c = 6 A), L_max = 4, C = 128, 8 heads, bf16
storage with fp32 accumulation; synthetic, seeded inputs.  Each rank runs
its own batch (weak scaling, no collective on the data path).

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA
events on the working stream; L2 is flushed (256 MiB write) between steps,
outside the step events; barrier + synchronize around the timed region,
the max over ranks is reported.  `value` = edges processed by all ranks /
that time.  `e2e` repeats the measurement through the public API with the
inputs copied from pinned host memory and the output copied back inside
every step.  The dominant kernel (the fused attention kernel) is timed live
with CUDA events recorded by the library on its stream.

`--impl reference` times the fp64 CPU oracle on the host cores instead
(rank 0 only; bounded samples of the same workload per step).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD_CFG = 1
WORKLOAD_DESC = ("256 drug-like molecules, 20-60 atoms each, open boundaries, r_c = 6 A; "
                 "L_max = 4, C = 128, H = 8; bf16 storage / fp32 accumulate")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_FLUSH_BYTES = 256 << 20


def so2_flops_per_edge(L: int, C: int) -> int:
    """Algorithmic FLOPs of the SO(2) block products per edge:
    2 n0^2 + sum_{m>=1} 8 n_m^2 with n_m = (L - m + 1) C."""
    n = [(L - m + 1) * C for m in range(L + 1)]
    return 2 * n[0] ** 2 + sum(8 * n[m] ** 2 for m in range(1, L + 1))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------
# distributed plumbing (also exercised by the CPU tests with gloo)
# ----------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def reduce_max(value: float, dist, device) -> float:
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, dist, device) -> float:
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch of molecules (weak scaling)."""
    from atomistic_mlip_b200 import workloads as w
    return w.BASE_SEED + WORKLOAD_CFG + 1000 * rank


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # wait (up to 5 s) for the first sample, so the timed region is covered
        t0 = time.time()
        while time.time() - t0 < 5.0:
            self.fh.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
def kernel_traffic(peaks_kernel: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if the kernel source has not changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    src = os.path.join(ROOT, d.get("source", ""))
    if not os.path.exists(src):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if sha != d.get("source_sha256") or d.get("kernel") != peaks_kernel:
        return None
    return d.get("dram_bytes_per_launch")


def run_ours(args):
    import torch
    from atomistic_mlip_b200 import e2f
    from atomistic_mlip_b200 import workloads as w

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    e2f.lib()

    wl = w.make_workload(WORKLOAD_CFG, seed=rank_seed(rank))
    L, C, H = wl.L, wl.C, wl.H
    pos_h = torch.from_numpy(wl.pos).pin_memory()
    x_h = torch.from_numpy(wl.x).to(torch.bfloat16).pin_memory()
    pos = pos_h.to(dev)
    x = x_h.to(dev)
    dw = e2f.DeviceWeights.from_workload(wl, dev)
    Q = (L + 1) ** 2
    out = torch.empty((wl.N, Q, C), dtype=torch.float32, device=dev)
    out_h = torch.empty((wl.N, Q, C), dtype=torch.float32).pin_memory()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    cap = 64 * wl.N
    row_ptr = torch.empty(wl.N + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(cap, dtype=torch.int32, device=dev)

    def step():
        nl = e2f.build_neighbors(pos, None, wl.r_c, row_ptr=row_ptr, col_idx=col_idx)
        e2f.attention_forward(x, pos, nl, dw, out=out)
        return nl.n_edges

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()

    clocks = ClockSampler(local)
    clocks.start()
    launches0 = e2f.kernel_launches()
    e2f.profile_enable(True)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    edges = 0
    for k in range(args.steps):
        flush.zero_()
        evs[k][0].record(stream)
        edges += step()
        evs[k][1].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e2f.profile_enable(False)
    n_attn, attn_ms = e2f.profile_read()
    launches = e2f.kernel_launches() - launches0
    clk = clocks.stop()
    t_ms = sum(a.elapsed_time(b) for a, b in evs)

    # e2e through the public API with host buffers
    e2e_evs = []
    for k in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        a.record(stream)
        pos.copy_(pos_h, non_blocking=True)
        x.copy_(x_h, non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)
        b.record(stream)
        if k >= args.warmup:
            e2e_evs.append((a, b))
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_evs)

    t_max = reduce_max(t_ms, dist, dev)
    e2e_max = reduce_max(e2e_ms, dist, dev)
    edges_all = reduce_sum(float(edges), dist, dev)
    e2e_edges_all = edges_all  # same batches
    peaks, peak_src = load_peaks()
    F = so2_flops_per_edge(L, C)
    E_rank = edges // args.steps
    avg_attn_ms = attn_ms / max(n_attn, 1)
    achieved = F * E_rank / (avg_attn_ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return

    cpu = cpu_baseline(wl) if world == 1 else None
    line = {
        "metric": "edges/s of fused SO(2) equivariant attention fwd; % bf16 tensor-pipe peak",
        "value": edges_all / (t_max * 1e-3),
        "unit": "edges/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded generator; no dataset)",
        "config": {"workload": WORKLOAD_DESC, "N_atoms_per_rank": wl.N, "edges_per_step_rank0": E_rank,
                   "l2": "flushed between steps (256 MiB write outside the step events)",
                   "step": "e2f_build_neighbors + e2f_attention_forward", "parallelism": f"dp{world} (independent batches)"},
        "node_updates_per_s": wl.N * world * args.steps / (t_max * 1e-3),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_source": f"bf16_tflops burst, {peak_src}",
                     "kernel": "fused attention", "flops_per_edge": F, "launches": n_attn,
                     "avg_launch_ms": avg_attn_ms,
                     "traffic": kernel_traffic("attention")},
        "e2e": {"value": e2e_edges_all / (e2e_max * 1e-3), "unit": "edges/s",
                "h2d_bytes_per_step": int(pos_h.numel() * 4 + x_h.numel() * 2),
                "d2h_bytes_per_step": int(out_h.numel() * 4)},
        "gpu_launches": int(launches),
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


# ----------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)
# ----------------------------------------------------------------------------
def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample_step(wl, csr, nodes):
    """One oracle pass over a sample: brute-force CSR of the whole batch and
    the attention of the sampled destination rows; returns edges done."""
    from oracle import attention as oa
    from oracle import neighbors as nb
    rp, col = nb.neighbors(wl.pos, wl.box, wl.r_c)
    oa.attention_workload(wl, nodes=nodes, csr=(rp, col))
    return int(sum(rp[i + 1] - rp[i] for i in nodes))


def cpu_baseline(wl, budget_s: float = 15.0, chunk: int = 64):
    """Oracle edges/s on the host cores over a bounded sample of rows."""
    from threadpoolctl import threadpool_limits
    from oracle import attention as oa
    from oracle import neighbors as nb
    cores = _cores()
    with threadpool_limits(limits=cores):
        rp, col = nb.neighbors(wl.pos, wl.box, wl.r_c)
        order = np.random.default_rng(7).permutation(wl.N)
        t0 = time.perf_counter()
        edges, rows, k = 0, 0, 0
        while time.perf_counter() - t0 < budget_s and k < wl.N:
            nodes = np.sort(order[k:k + chunk])
            oa.attention_workload(wl, nodes=nodes, csr=(rp, col))
            edges += int(sum(rp[i + 1] - rp[i] for i in nodes))
            rows += len(nodes)
            k += chunk
        dt = time.perf_counter() - t0
    return {"value": edges / dt, "unit": "edges/s", "cores": cores, "kind": "oracle",
            "sample": f"{rows} random destination rows ({edges} edges) of the benchmark batch, fp64 NumPy, {dt:.1f} s"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from threadpoolctl import threadpool_limits
    from atomistic_mlip_b200 import workloads as w
    wl = w.make_workload(WORKLOAD_CFG, seed=rank_seed(0))
    cores = _cores()
    rows_per_step = 48
    order = np.random.default_rng(11).permutation(wl.N)
    times, edges = [], 0
    with threadpool_limits(limits=cores):
        for k in range(args.warmup + args.steps):
            nodes = np.sort(order[(k * rows_per_step) % wl.N:][:rows_per_step])
            t0 = time.perf_counter()
            e = oracle_sample_step(wl, None, nodes)
            dt = time.perf_counter() - t0
            if k >= args.warmup:
                times.append(dt)
                edges += e
    total = sum(times)
    value = edges / total
    line = {
        "impl": "reference",
        "metric": "edges/s of fused SO(2) equivariant attention fwd; % bf16 tensor-pipe peak",
        "value": value, "unit": "edges/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator; no dataset)",
        "config": {"workload": WORKLOAD_DESC, "N_atoms_per_rank": wl.N,
                   "sample_per_step": f"brute-force CSR of the batch + attention of {rows_per_step} rows"},
        "cpu_baseline": {"value": value, "unit": "edges/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows_per_step} destination rows per step, fp64 NumPy oracle"},
        "e2e": {"value": value, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# per-row measurements (one JSON line per hot-path row and workload)
# ----------------------------------------------------------------------------
def run_rows(args):
    """Each row of the hot path against its own roofline, on every workload:
    the neighbour build (HBM: algorithmic bytes 12N + 4(N+1) + 4E, the
    positions read, row_ptr and col_idx written) and the fused attention
    (tensor: F(L, C) FLOP per edge), plus peak device memory against N on the
    water-box sweep.  Times are CUDA events on the working stream, median of
    `--steps` calls after `--warmup`; the neighbour build's time includes its
    two host read-backs (bounding box, edge count)."""
    import torch
    from atomistic_mlip_b200 import e2f
    from atomistic_mlip_b200 import workloads as w

    if not torch.cuda.is_available():
        raise SystemExit("bench.py --rows needs a CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    e2f.lib()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)

    def timed(fn, reps):
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    def one(cfg, n_target=None, attention=True, reps=None):
        steps = args.steps if reps is None else reps
        warm = args.warmup if reps is None else 1
        wl = w.make_workload(cfg, n_target=n_target)
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats(dev)
        e2f.scratch_high_water(reset=True)
        pos = torch.from_numpy(wl.pos).to(dev)
        x = torch.from_numpy(wl.x).to(dev, torch.bfloat16 if wl.precision == "bf16" else torch.float32)
        dw = e2f.DeviceWeights.from_workload(wl, dev)
        box = None if wl.box is None else [float(b) for b in wl.box]
        nl = e2f.build_neighbors(pos, box, wl.r_c)
        cap = nl.n_edges
        row_ptr = torch.empty(wl.N + 1, dtype=torch.int32, device=dev)
        col_idx = torch.empty(max(1, cap), dtype=torch.int32, device=dev)

        def nb():
            e2f.build_neighbors(pos, box, wl.r_c, row_ptr=row_ptr, col_idx=col_idx)
        for _ in range(warm):
            nb()
        t_nb = timed(nb, steps)
        E = nl.n_edges
        nb_bytes = 12 * wl.N + 4 * (wl.N + 1) + 4 * E
        out = {"row": "A1-A3 neighbour build", "workload": wl.cfg_name if hasattr(wl, "cfg_name") else f"cfg{cfg}",
               "N": wl.N, "E": E, "ms": t_nb,
               "roofline": {"bound": "hbm", "algorithmic_bytes": nb_bytes,
                            "achieved": nb_bytes / (t_nb * 1e-3) / 1e9, "peak": float(peaks["hbm_gbs"]),
                            "unit": "GB/s", "frac": nb_bytes / (t_nb * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
                            "peak_source": f"hbm_gbs, {peak_src}"}}
        print(json.dumps(out), flush=True)
        if not attention:
            return
        o = torch.empty((wl.N, (wl.L + 1) ** 2, wl.C), dtype=torch.float32, device=dev)

        def att():
            e2f.attention_forward(x, pos, nl, dw, out=o)
        for _ in range(warm):
            att()
        e2f.profile_enable(True)
        t_call = timed(att, steps)
        e2f.profile_enable(False)
        n_k, k_ms = e2f.profile_read()
        k_ms = k_ms / max(n_k, 1)
        F = so2_flops_per_edge(wl.L, wl.C)
        peak = float(peaks["bf16_tflops"])
        out = {"row": "A4-A11 attention forward (projections + fused kernel)", "workload": f"cfg{cfg}",
               "N": wl.N, "E": E, "L": wl.L, "C": wl.C, "H": wl.H, "precision": wl.precision,
               "call_ms": t_call, "fused_kernel_ms": k_ms,
               "edges_per_s": E / (t_call * 1e-3), "node_updates_per_s": wl.N / (t_call * 1e-3),
               "roofline": {"bound": "tensor", "flops_per_edge": F, "achieved": F * E / (k_ms * 1e-3) / 1e12,
                            "peak": peak, "unit": "TFLOP/s", "frac": F * E / (k_ms * 1e-3) / 1e12 / peak,
                            "peak_source": f"bf16_tflops burst, {peak_src}",
                            "path": "tcgen05" if (wl.precision == "bf16" and wl.C == 128 and 1 <= wl.L <= 6) else "SIMT"},
               "peak_device_bytes": {"torch": int(torch.cuda.max_memory_allocated(dev)),
                                     "library_scratch": int(e2f.scratch_high_water())}}
        print(json.dumps(out), flush=True)
        del o

    if args.rows_what == "neighbors":
        one(4, attention=False)
        return
    for cfg in (1, 2, 4):
        one(cfg)
    for n in (10002, 30000):   # memory sweep of the water box (cfg4 is the 100k point)
        one(4, n_target=n)
    one(3)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--rows", action="store_true", help="per-row measurements on every workload (one GPU)")
    ap.add_argument("--rows-what", choices=["all", "neighbors"], default="all",
                    help="with --rows: every row, or the neighbour build of the 100k-atom water box only")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.rows:
        run_rows(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
