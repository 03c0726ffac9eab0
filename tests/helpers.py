"""Helpers shared by the GPU parity tests: move a workload to the device,
run the library, and compare with the oracle under the error measure the
tests use (max |gpu - ref| / max |ref| over the compared rows)."""
from __future__ import annotations

import dataclasses
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


def local_rows(pos, box, r_c, rows):
    """(U, (row_ptr, col), idx) for sampled rows of a large system: the atoms
    U that the radius-graph rows `rows` read (the rows' own atoms and their
    neighbours, sorted), the CSR over U that lists exactly those rows in
    full (every other row empty), and idx mapping a global atom index to its
    place in U (-1 outside).  An operator whose output row i reads only atom
    i and its neighbours gives the same rows on this subsystem."""
    from oracle import neighbors as nb
    rows = np.unique(np.asarray(rows, np.int64))
    rp, col = nb.neighbor_rows(pos, box, r_c, rows)
    U = np.unique(np.concatenate([rows, col.astype(np.int64)]))
    idx = -np.ones(len(pos), np.int64)
    idx[U] = np.arange(len(U))
    lrp = np.zeros(len(U) + 1, np.int64)
    np.cumsum(np.diff(rp)[U], out=lrp[1:])
    lcol = np.concatenate([idx[col[rp[u]:rp[u + 1]]] for u in U]).astype(np.int32)
    return U, (lrp, lcol), idx


def local_gradients(wl, nodes, G):
    """Oracle (dL/dpos, dL/dx) of the atoms `nodes` of a large system, from
    the outputs that depend on them: the rows of the nodes and of their
    neighbours, over the atoms those rows read; every other output row is
    left out (it does not depend on the sampled atoms)."""
    from oracle import attention_grad as ag
    from oracle import neighbors as nb
    col1 = nb.neighbor_rows(wl.pos, wl.box, wl.r_c, nodes)[1]
    S = np.unique(np.concatenate([np.asarray(nodes, np.int64), col1.astype(np.int64)]))
    U, csr, idx = local_rows(wl.pos, wl.box, wl.r_c, S)
    local = dataclasses.replace(wl, pos=wl.pos[U], x=wl.x[U])
    ref = ag.gradients(local, csr, G[U])
    return ref["pos"][idx[nodes]], ref["x"][idx[nodes]]
