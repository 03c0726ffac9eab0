"""Helpers shared by the GPU parity tests: move a workload to the device,
run the library, and compare with the oracle under the error measure the
tests use (max |gpu - ref| / max |ref| over the compared rows)."""
from __future__ import annotations

import functools

import numpy as np

from atomistic_mlip_b200 import workloads as wlmod


def rel_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    scale = float(np.max(np.abs(ref)))
    if scale == 0.0:
        return float(np.max(np.abs(gpu)))
    return float(np.max(np.abs(gpu - ref))) / scale


def to_device(wl, precision=None):
    import torch
    from atomistic_mlip_b200 import e2f
    prec = precision or wl.precision
    dt = torch.float32 if prec == "fp32" else torch.bfloat16
    pos = torch.from_numpy(np.ascontiguousarray(wl.pos, np.float32)).cuda()
    x = torch.from_numpy(np.ascontiguousarray(wl.x, np.float32)).to("cuda", dt)
    w = e2f.DeviceWeights.from_workload(wl, "cuda", prec)
    box = None if wl.box is None else [float(b) for b in wl.box]
    return pos, x, w, box


def gpu_forward(wl, precision=None):
    """(out [N,Q,C] float64 numpy, NeighborList) from the CUDA path."""
    import torch
    from atomistic_mlip_b200 import e2f
    pos, x, w, box = to_device(wl, precision)
    nl = e2f.build_neighbors(pos, box, wl.r_c)
    out = e2f.attention_forward(x, pos, nl, w)
    torch.cuda.synchronize()
    assert e2f.stream_status() == 0
    return out.double().cpu().numpy(), nl


@functools.lru_cache(maxsize=None)
def oracle_csr(cfg: int):
    from oracle import neighbors as nb
    wl = cached_workload(cfg, "bf16" if cfg else "fp32")
    return nb.neighbors(wl.pos, wl.box, wl.r_c)


@functools.lru_cache(maxsize=None)
def cached_workload(cfg: int, precision: str):
    return wlmod.make_workload(cfg, precision=precision)
