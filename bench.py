"""Benchmark of the on-the-fly equivariant attention hot path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole path on one system: the cell-list CSR build plus the
fused attention forward (projections, edge geometry, Wigner-D, logits,
online softmax, SO(2) block products, back-rotation, accumulation).
Headline workload: the 100,002-atom periodic water box (33,334 rigid
waters in a 100.0007 A cube, r_c = 6 A, about 8.7 M directed edges),
L_max = 4, C = 128, 8 heads, bf16 storage with fp32 accumulation;
synthetic, seeded inputs.  Each rank runs its own system (weak scaling, no
collective on the data path).

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA
events on the working stream; L2 is flushed (256 MiB write) between steps,
outside the step events; barrier + synchronize around the timed region,
the max over ranks is reported.  `value` = edges processed by all ranks /
that time.  `e2e` repeats the measurement through the public API with the
inputs copied from pinned host memory and the output copied back for every
step, the copies on their own streams overlapping the neighbouring steps'
compute (double-buffered), timed as one interval.  The dominant kernel (the fused attention kernel) is timed live
with CUDA events recorded by the library on its stream.

At one GPU the same line also carries `workloads` (every other workload:
the 256-molecule batch, the 3,000-atom water box, the 30,000-atom
protein-in-water box at L_max = 6; each row against its own roofline) and
`memory_sweep` (peak device memory and edges/s of the water box at 10k,
30k and 100k atoms, with a linear fit in N).

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

WORKLOAD_CFG = 4
WORKLOAD_DESC = ("periodic water box, 100,002 atoms (33,334 rigid waters) in a 100.0007 A cube, "
                 "minimum image, r_c = 6 A; L_max = 4, C = 128, H = 8; bf16 storage / fp32 accumulate")
EXTRA_DESC = {1: "256 drug-like molecules, 20-60 atoms each, open boundaries, r_c = 6 A; L=4, C=128, H=8, bf16",
              2: "periodic water box, 3,000 atoms in a 31 A cube, r_c = 6 A; L=4, C=128, H=8, bf16",
              3: ("30,000-atom box: 3,000-atom compact chain + 9,000 waters in a 66.94 A cube, r_c = 6 A; "
                  "L=6, C=128, H=8, bf16"),
              4: "periodic water box, 100,002 atoms, r_c = 6 A; L=4, C=128, H=8, bf16"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_FLUSH_BYTES = 256 << 20


def so2_flops_per_edge(L: int, C: int) -> int:
    """Algorithmic FLOPs of the SO(2) block products per edge:
    2 n0^2 + sum_{m>=1} 8 n_m^2 with n_m = (L - m + 1) C."""
    n = [(L - m + 1) * C for m in range(L + 1)]
    return 2 * n[0] ** 2 + sum(8 * n[m] ** 2 for m in range(1, L + 1))


def cg_eaas_flops_per_edge(L: int, C: int) -> int:
    """Algorithmic FLOPs per edge of the re-indexed CG convolution (2 per
    multiply-add, per channel): z rotations in and out (4 per (l, m >= 1)
    pair each), the y blocks in and out (sum over l >= 1 of (l+1)^2 + l^2
    each), the coupling ((L+1)^2 + 4 sum_{m>=1} (L-m+1)^2) and the m = 0
    accumulation (L + 1)."""
    z = 2 * L * (L + 1)
    y = sum((l + 1) ** 2 + l ** 2 for l in range(1, L + 1))
    coup = (L + 1) ** 2 + 4 * sum((L - m + 1) ** 2 for m in range(1, L + 1))
    return 2 * C * (2 * z + 2 * y + coup + (L + 1))


def cg_dense_flops_per_edge(L: int, C: int) -> int:
    """The same convolution as a dense contraction in the global frame:
    2 (2l1+1)(2l2+1)(2l3+1) per path and channel (harmonics not counted)."""
    n = 0
    for l1 in range(L + 1):
        for l2 in range(L + 1):
            for l3 in range(abs(l1 - l2), min(L, l1 + l2) + 1):
                n += (2 * l1 + 1) * (2 * l2 + 1) * (2 * l3 + 1)
    return 2 * C * n


def fp32_alu_peak_tflops(dev) -> float:
    """FP32 multiply-add peak: SMs x 128 lanes x 2 FLOP x the maximum SM clock
    (nvidia-smi clocks.max.sm; 1965 MHz if unavailable)."""
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = 1965.0
    try:
        q = subprocess.run(["nvidia-smi", "--query-gpu=clocks.max.sm", "--format=csv,noheader,nounits", "-i",
                            str(dev.index or 0)], capture_output=True, text=True, timeout=10)
        mhz = float(q.stdout.strip().splitlines()[0])
    except Exception:
        pass
    return sms * 128 * 2 * mhz * 1e6 / 1e12


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
    """Each rank draws its own system (weak scaling); rank 0's is the seeded
    workload itself."""
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


def _box_list(wl):
    return None if wl.box is None else [float(b) for b in wl.box]


def measure_workload(cfg, dev, peaks, peak_src, reps=5, warm=2, n_target=None, wl=None, attention=True):
    """One workload against its rooflines: the neighbour build (HBM:
    algorithmic bytes 12N + 4(N+1) + 4E) and the fused attention kernel
    (tensor: F(L, C) FLOP per edge over the kernel's own event time), plus
    the whole attention call and peak device memory.  Median of `reps`
    calls after `warm`; CUDA events on the working stream."""
    import torch
    from atomistic_mlip_b200 import e2f
    from atomistic_mlip_b200 import workloads as w
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    if wl is None:
        wl = w.make_workload(cfg, n_target=n_target)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats(dev)
    e2f.scratch_high_water(reset=True)
    pos = torch.from_numpy(wl.pos).to(dev)
    x = torch.from_numpy(wl.x).to(dev, torch.bfloat16 if wl.precision == "bf16" else torch.float32)
    dw = e2f.DeviceWeights.from_workload(wl, dev)
    box = _box_list(wl)
    nl = e2f.build_neighbors(pos, box, wl.r_c)
    E = nl.n_edges
    row_ptr = torch.empty(wl.N + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(max(1, E), dtype=torch.int32, device=dev)

    def nb():
        e2f.build_neighbors(pos, box, wl.r_c, row_ptr=row_ptr, col_idx=col_idx)
    for _ in range(warm):
        nb()
    t_nb = timed(nb)
    nb_bytes = 12 * wl.N + 4 * (wl.N + 1) + 4 * E
    nb_row = {"ms": t_nb, "algorithmic_bytes": nb_bytes, "achieved_gbs": nb_bytes / (t_nb * 1e-3) / 1e9,
              "frac_hbm": nb_bytes / (t_nb * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
              "note": "whole call, including its host read-backs"}
    if not attention:
        return {"workload": EXTRA_DESC.get(cfg, f"cfg{cfg}"), "N": wl.N, "E": E, "neighbour_build": nb_row}
    o = torch.empty((wl.N, (wl.L + 1) ** 2, wl.C), dtype=torch.float32, device=dev)

    def att():
        e2f.attention_forward(x, pos, nl, dw, out=o)
    for _ in range(warm):
        att()
    e2f.profile_enable(True)
    t_call = timed(att)
    e2f.profile_enable(False)
    n_k, k_ms = e2f.profile_read()
    k_ms = k_ms / max(n_k, 1)
    F = so2_flops_per_edge(wl.L, wl.C)
    peak = float(peaks["bf16_tflops"])
    res = {"workload": EXTRA_DESC.get(cfg, f"cfg{cfg}") if n_target is None else
           f"periodic water box, {wl.N} atoms, r_c = 6 A; L=4, C=128, H=8, bf16",
           "N": wl.N, "E": E, "L": wl.L,
           "neighbour_build": nb_row,
           "attention": {"call_ms": t_call, "fused_kernel_ms": k_ms,
                         "edges_per_s": E / (t_call * 1e-3), "node_updates_per_s": wl.N / (t_call * 1e-3),
                         "achieved_tflops": F * E / (k_ms * 1e-3) / 1e12,
                         "frac": F * E / (k_ms * 1e-3) / 1e12 / peak, "flops_per_edge": F},
           "peak_device_bytes": {"torch": int(torch.cuda.max_memory_allocated(dev)),
                                 "library_scratch": int(e2f.scratch_high_water())}}
    del o, x, pos, dw, nl, row_ptr, col_idx
    torch.cuda.empty_cache()
    return res


def measure_forces(cfg, dev, peaks, reps=3, warm=1, wl=None):
    """The backward of the attention (dL/dx and dL/dpos, forces = -dL/dpos)
    on a workload: whole-call time (CUDA events), edges/s, and the SO(2)
    block products it recomputes and transposes (2 F(L, C) FLOP per edge)
    as achieved TFLOP/s against the bf16 peak."""
    import torch
    from atomistic_mlip_b200 import e2f
    from atomistic_mlip_b200 import workloads as w
    stream = torch.cuda.current_stream(dev)
    if wl is None:
        wl = w.make_workload(cfg)
    pos = torch.from_numpy(wl.pos).to(dev)
    x = torch.from_numpy(wl.x).to(dev, torch.bfloat16)
    dw = e2f.DeviceWeights.from_workload(wl, dev)
    nl = e2f.build_neighbors(pos, _box_list(wl), wl.r_c)
    G = torch.randn((wl.N, (wl.L + 1) ** 2, wl.C), dtype=torch.float32, device=dev,
                    generator=torch.Generator(device=dev).manual_seed(7))
    for _ in range(warm):
        e2f.attention_backward(x, pos, nl, dw, G)
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        _, gp = e2f.attention_backward(x, pos, nl, dw, G)
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    t = statistics.median(ts)
    F2 = 2 * so2_flops_per_edge(wl.L, wl.C)
    res = {"workload": EXTRA_DESC.get(cfg, f"cfg{cfg}"), "N": wl.N, "E": nl.n_edges, "ms": t,
           "edges_per_s": nl.n_edges / (t * 1e-3),
           "so2_tflops": F2 * nl.n_edges / (t * 1e-3) / 1e12,
           "frac_of_bf16_peak": F2 * nl.n_edges / (t * 1e-3) / 1e12 / float(peaks["bf16_tflops"]),
           "net_force_over_max": float(gp.sum(0).abs().max() / gp.abs().max().clamp_min(1e-30)),
           "what": "e2f_attention_backward: dL/dx and dL/dpos (forces = -dL/dpos), bf16 storage"}
    del x, pos, dw, nl, G, gp
    torch.cuda.empty_cache()
    return res


def measure_cg(cfg, dev, reps=3, warm=1, wl=None):
    """The re-indexed CG convolution (x (x) Y(rhat) with channel-wise path
    weights, evaluated in the edge frame) on a workload's features: call
    time (CUDA events), edges/s and achieved FP32 TFLOP/s of its algorithmic
    FLOPs against the FP32 multiply-add peak (the kernel runs on the CUDA
    cores: the coupling is channel-wise, not a contraction)."""
    import torch
    from atomistic_mlip_b200 import e2f
    from atomistic_mlip_b200 import workloads as w
    stream = torch.cuda.current_stream(dev)
    if wl is None:
        wl = w.make_workload(cfg)
    pos = torch.from_numpy(wl.pos).to(dev)
    x = torch.from_numpy(wl.x).to(dev, torch.bfloat16)
    W = torch.from_numpy(w.make_cg_weights(wl.L, wl.C, 77)).to(dev)
    nl = e2f.build_neighbors(pos, _box_list(wl), wl.r_c)
    for _ in range(warm):
        e2f.cg_conv_forward(x, pos, nl, W, wl.L)
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2f.cg_conv_forward(x, pos, nl, W, wl.L)
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    t = statistics.median(ts)
    F = cg_eaas_flops_per_edge(wl.L, wl.C)
    peak = fp32_alu_peak_tflops(dev)
    res = {"workload": EXTRA_DESC.get(cfg, f"cfg{cfg}"), "N": wl.N, "E": nl.n_edges, "L": wl.L, "C": wl.C,
           "ms": t, "edges_per_s": nl.n_edges / (t * 1e-3), "flops_per_edge": F,
           "dense_cg_flops_per_edge": cg_dense_flops_per_edge(wl.L, wl.C),
           "achieved_tflops": F * nl.n_edges / (t * 1e-3) / 1e12, "fp32_peak_tflops": peak,
           "frac_of_fp32_peak": F * nl.n_edges / (t * 1e-3) / 1e12 / peak,
           "what": "e2f_cg_conv_forward: channel-wise CG convolution x (x) Y(rhat), edge-frame re-indexing, "
                   "bf16 features, fp32 arithmetic"}
    del x, pos, W, nl
    torch.cuda.empty_cache()
    return res


def measure_multifocus(cfg, dev, peaks, F=4, reps=3, warm=1, wl=None):
    """The multi-focus attention (F streams, per-stream SO(2) stacks, cross-
    focus softmax) on a workload: call time, fused-kernel time and edges/s.
    The kernel runs the full C x C block products with the cross-stream
    entries packed as zero, so its tensor-pipe work is that of the plain
    operator (reported against the bf16 peak); the useful part is 1/F of it."""
    import torch
    from atomistic_mlip_b200 import e2f
    from atomistic_mlip_b200 import workloads as w
    stream = torch.cuda.current_stream(dev)
    if wl is None:
        wl = w.make_workload(cfg)
    pos = torch.from_numpy(wl.pos).to(dev)
    x = torch.from_numpy(wl.x).to(dev, torch.bfloat16)
    dw = e2f.DeviceWeights.from_workload(wl, dev)
    a = torch.randn(wl.C, device=dev, generator=torch.Generator(device=dev).manual_seed(5)) * 2.0
    nl = e2f.build_neighbors(pos, _box_list(wl), wl.r_c)
    for _ in range(warm):
        e2f.attention_forward_multifocus(x, pos, nl, dw, F, a)
    e2f.profile_enable(True)
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2f.attention_forward_multifocus(x, pos, nl, dw, F, a)
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    kern = e2f.profile_read()
    e2f.profile_enable(False)
    t = statistics.median(ts)
    kt = kern[1] / max(kern[0], 1)
    Fx = so2_flops_per_edge(wl.L, wl.C)
    res = {"workload": EXTRA_DESC.get(cfg, f"cfg{cfg}"), "N": wl.N, "E": nl.n_edges, "F": F, "call_ms": t,
           "fused_kernel_ms": kt, "edges_per_s": nl.n_edges / (kt * 1e-3),
           "executed_tflops": Fx * nl.n_edges / (kt * 1e-3) / 1e12,
           "frac_of_bf16_peak": Fx * nl.n_edges / (kt * 1e-3) / 1e12 / float(peaks["bf16_tflops"]),
           "useful_flops_per_edge": Fx // F,
           "what": "e2f_attention_forward_multifocus: F focus streams, cross-focus softmax, bf16"}
    del x, pos, dw, nl, a
    torch.cuda.empty_cache()
    return res


def measure_block(cfg, dev, n_layers=1, reps=3, warm=1, wl=None):
    """n_layers E2Former-V2 blocks (merged RMS norm, attention, scalar-gated
    FFN with Hd = 4C, residuals) on a workload: time per block, and the
    attention kernel's share of it."""
    import torch
    from atomistic_mlip_b200 import e2f
    from atomistic_mlip_b200 import workloads as w
    stream = torch.cuda.current_stream(dev)
    if wl is None:
        wl = w.make_workload(cfg)
    pos = torch.from_numpy(wl.pos).to(dev)
    x = torch.from_numpy(np.ascontiguousarray(wl.x, np.float32)).to(dev)
    nl = e2f.build_neighbors(pos, _box_list(wl), wl.r_c)
    layers = [e2f.DeviceBlockWeights.from_layer(w.make_layer_weights(wl.L, wl.C, wl.H, "bf16", 900 + k), dev)
              for k in range(n_layers)]
    for _ in range(warm):
        e2f.model_forward(x, pos, nl, layers)
    e2f.profile_enable(True)
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2f.model_forward(x, pos, nl, layers)
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    e2f.profile_enable(False)
    n_k, k_ms = e2f.profile_read()
    t = statistics.median(ts)
    Q = (wl.L + 1) ** 2
    ffn_flops = 2 * wl.N * wl.C * 4 * wl.C * (1 + 2 * Q)   # gate + up (all rows) + down
    res = {"workload": EXTRA_DESC.get(cfg, f"cfg{cfg}"), "N": wl.N, "E": nl.n_edges, "layers": n_layers,
           "ms_per_forward": t, "ms_per_block": t / n_layers,
           "attention_kernel_share": (k_ms / max(n_k, 1)) * n_layers / t,
           "node_updates_per_s": wl.N * n_layers / (t * 1e-3), "ffn_flops_per_block": ffn_flops,
           "what": "e2f_block_forward x layers: Norm -> attention -> residual -> Norm -> FFN(Hd = 4C) -> residual, bf16"}
    del x, pos, nl, layers
    torch.cuda.empty_cache()
    return res


def linear_fit(ns, ys):
    """Least-squares y = a + b N and its R^2."""
    A = np.stack([np.ones(len(ns)), np.asarray(ns, float)], 1)
    coef, *_ = np.linalg.lstsq(A, np.asarray(ys, float), rcond=None)
    pred = A @ coef
    ss_res = float(np.sum((np.asarray(ys) - pred) ** 2))
    ss_tot = float(np.sum((np.asarray(ys) - np.mean(ys)) ** 2)) or 1.0
    return {"intercept_bytes": float(coef[0]), "bytes_per_atom": float(coef[1]), "r2": 1.0 - ss_res / ss_tot}


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
    box = _box_list(wl)
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
    cap = 128 * wl.N
    row_ptr = torch.empty(wl.N + 1, dtype=torch.int32, device=dev)
    col_idx = torch.empty(cap, dtype=torch.int32, device=dev)

    def step():
        nl = e2f.build_neighbors(pos, box, wl.r_c, row_ptr=row_ptr, col_idx=col_idx)
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

    # e2e through the public API with host buffers: every step copies its
    # inputs from pinned host memory and its output back, as a caller that
    # overlaps transfers with compute would -- the copies in of step k + 1
    # and out of step k - 1 run on their own streams while step k computes
    # (double-buffered device inputs and outputs; the inputs exceed L2, so no
    # flush).  One interval from the first copy in to the last copy out.
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    pos_d = [pos, torch.empty_like(pos)]
    x_d = [x, torch.empty_like(x)]
    out_d = [out, torch.empty_like(out)]
    nl_rp = [row_ptr, torch.empty_like(row_ptr)]
    nl_ci = [col_idx, torch.empty_like(col_idx)]
    ev = lambda: torch.cuda.Event(enable_timing=False)

    def e2e_run(n_steps):
        h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(h2d_s)
        for k in range(n_steps):
            bb = k % 2
            with torch.cuda.stream(h2d_s):
                if k >= 2:
                    h2d_s.wait_event(comp_done[bb])
                pos_d[bb].copy_(pos_h, non_blocking=True)
                x_d[bb].copy_(x_h, non_blocking=True)
                h2d_done[bb].record(h2d_s)
            stream.wait_event(h2d_done[bb])
            if k >= 2:
                stream.wait_event(d2h_done[bb])
            nl = e2f.build_neighbors(pos_d[bb], box, wl.r_c, row_ptr=nl_rp[bb], col_idx=nl_ci[bb])
            e2f.attention_forward(x_d[bb], pos_d[bb], nl, dw, out=out_d[bb])
            comp_done[bb].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(comp_done[bb])
                out_h.copy_(out_d[bb], non_blocking=True)
                d2h_done[bb].record(d2h_s)
        d2h_s.wait_stream(h2d_s)
        t1.record(d2h_s)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(args.warmup)
    e2e_ms = e2e_run(args.steps)
    # release the e2e buffers (the lists and the closure hold references)
    del e2e_run
    for lst in (pos_d, x_d, out_d, nl_rp, nl_ci):
        lst.clear()
    h2d_bytes = int(pos_h.numel() * 4 + x_h.numel() * 2)
    d2h_bytes = int(out_h.numel() * 4)

    t_max = reduce_max(t_ms, dist, dev)
    e2e_max = reduce_max(e2e_ms, dist, dev)
    edges_all = reduce_sum(float(edges), dist, dev)
    e2e_edges_all = edges_all  # same systems
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

    extras = {}
    if world == 1 and not args.headline_only:
        # free the headline's buffers before the other workloads
        del out, out_h, x, pos, flush, row_ptr, col_idx, dw, pos_h, x_h
        torch.cuda.empty_cache()
        rows = [measure_workload(cfg, dev, peaks, peak_src) for cfg in (1, 2, 3)]
        sweep = [measure_workload(4, dev, peaks, peak_src, n_target=n) for n in (10002, 30000)]
        sweep.append(measure_workload(4, dev, peaks, peak_src, wl=wl))
        ns = [r["N"] for r in sweep]
        tot = [r["peak_device_bytes"]["torch"] + r["peak_device_bytes"]["library_scratch"] for r in sweep]
        extras["workloads"] = rows + [sweep[-1]]
        extras["forces"] = [measure_forces(2, dev, peaks), measure_forces(4, dev, peaks, reps=2, wl=wl)]
        extras["block"] = [measure_block(4, dev, n_layers=1, wl=wl), measure_block(2, dev, n_layers=2)]
        extras["cg_conv"] = [measure_cg(4, dev, wl=wl), measure_cg(2, dev)]
        extras["multifocus"] = [measure_multifocus(4, dev, peaks, F=4, wl=wl)]
        extras["memory_sweep"] = {
            "N": ns, "peak_device_bytes": tot,
            "edges_per_s": [r["attention"]["edges_per_s"] for r in sweep],
            "frac": [r["attention"]["frac"] for r in sweep],
            "fit": linear_fit(ns, tot),
            "what": "torch.cuda.max_memory_allocated + the library pool's high-water mark, per attention call"}

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
                   "l2": "flushed between steps (256 MiB write outside the step events); inputs exceed L2",
                   "step": "e2f_build_neighbors + e2f_attention_forward", "parallelism": f"dp{world} (independent systems)"},
        "node_updates_per_s": wl.N * world * args.steps / (t_max * 1e-3),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_source": f"bf16_tflops burst, {peak_src}",
                     "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                     "kernel": "fused attention", "flops_per_edge": F, "launches": n_attn,
                     "avg_launch_ms": avg_attn_ms,
                     "traffic": kernel_traffic("attention")},
        "e2e": {"value": e2e_edges_all / (e2e_max * 1e-3), "unit": "edges/s",
                "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                "how": "per step: pinned H2D of positions and x, e2f_build_neighbors + e2f_attention_forward, "
                       "D2H of o; copies on two extra streams overlapping the adjacent steps' compute"},
        "gpu_launches": int(launches),
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    line.update(extras)
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


def oracle_sample_step(wl, nodes):
    """One oracle pass over a sample of destination rows: their brute-force
    neighbour rows, then their attention; returns the edges done."""
    from oracle import attention as oa
    from oracle import neighbors as nb
    rp, col = nb.neighbor_rows(wl.pos, wl.box, wl.r_c, nodes)
    oa.attention_workload(wl, nodes=nodes, csr=(rp, col))
    return int(sum(rp[i + 1] - rp[i] for i in nodes))


def cpu_baseline(wl, budget_s: float = 15.0, chunk: int = 64):
    """Oracle edges/s on the host cores over a bounded sample of rows of the
    seeded 1,000-node subset (brute-force rows + attention, both timed)."""
    from threadpoolctl import threadpool_limits
    cores = _cores()
    order = np.random.default_rng(7).permutation(wl.subset)
    with threadpool_limits(limits=cores):
        t0 = time.perf_counter()
        edges, rows, k = 0, 0, 0
        while time.perf_counter() - t0 < budget_s and k < len(order):
            nodes = np.sort(order[k:k + chunk])
            edges += oracle_sample_step(wl, nodes)
            rows += len(nodes)
            k += chunk
        dt = time.perf_counter() - t0
    return {"value": edges / dt, "unit": "edges/s", "cores": cores, "kind": "oracle",
            "sample": (f"{rows} rows of the seeded 1,000-node subset ({edges} edges) of the benchmark system: "
                       f"brute-force neighbour rows + attention, fp64 NumPy, {dt:.1f} s")}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from threadpoolctl import threadpool_limits
    from atomistic_mlip_b200 import workloads as w
    wl = w.make_workload(WORKLOAD_CFG, seed=rank_seed(0))
    cores = _cores()
    rows_per_step = 24
    order = np.random.default_rng(11).permutation(wl.subset)
    times, edges = [], 0
    with threadpool_limits(limits=cores):
        for k in range(args.warmup + args.steps):
            nodes = np.sort(np.resize(np.roll(order, -k * rows_per_step), rows_per_step))
            t0 = time.perf_counter()
            e = oracle_sample_step(wl, nodes)
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
                   "sample_per_step": f"brute-force neighbour rows + attention of {rows_per_step} destination rows"},
        "cpu_baseline": {"value": value, "unit": "edges/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows_per_step} destination rows per step, fp64 NumPy oracle"},
        "e2e": {"value": value, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# per-row measurements (one JSON line per workload)
# ----------------------------------------------------------------------------
def run_rows(args):
    """Each workload against its rooflines, one JSON line each (the same
    measurement the default line carries under `workloads`)."""
    import torch
    from atomistic_mlip_b200 import e2f
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --rows needs a CUDA device")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    e2f.lib()
    peaks, peak_src = load_peaks()
    what = args.rows_what
    if what == "forces":
        print(json.dumps(measure_forces(2, dev, peaks, reps=args.steps, warm=args.warmup)), flush=True)
        return
    if what == "block":
        print(json.dumps(measure_block(4, dev, reps=args.steps, warm=args.warmup)), flush=True)
        return
    if what == "multifocus":
        for cfg in (1, 4):
            print(json.dumps(measure_multifocus(cfg, dev, peaks, F=4, reps=args.steps, warm=args.warmup)), flush=True)
        return
    if what == "cg":
        for cfg in (2, 4):
            print(json.dumps(measure_cg(cfg, dev, reps=args.steps, warm=args.warmup)), flush=True)
        return
    cfgs = {"all": (1, 2, 4, 3), "neighbors": (4,), "molecules": (1,), "water3k": (2,), "protein": (3,),
            "water100k": (4,)}[what]
    for cfg in cfgs:
        print(json.dumps(measure_workload(cfg, dev, peaks, peak_src, reps=args.steps, warm=args.warmup,
                                          attention=what != "neighbors")), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the other workloads and the memory sweep (profiling runs)")
    ap.add_argument("--rows", action="store_true", help="one JSON line per workload (one GPU)")
    ap.add_argument("--rows-what", choices=["all", "neighbors", "molecules", "water3k", "protein", "water100k",
                                            "forces", "block", "cg", "multifocus"], default="all")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    _, world, _ = dist_env()
    if args.gpus != world:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE = {world}; launch N > 1 ranks with "
                         f"torchrun (--nproc-per-node N), one process per GPU")
    if args.rows:
        run_rows(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
