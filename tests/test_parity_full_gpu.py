"""Parity where the kernels are least exercised: full-size workloads on
seeded 1,000-node subsets at both precisions, every node at a boundary of
the fused kernel's per-CTA edge ranges and in each CTA's last tile, and
rotation equivariance on periodic boxes.

Error measure as everywhere: max |gpu - ref| / max |ref| over the compared
rows; <= 1e-4 with fp32 storage, <= 2e-2 with bf16 storage and fp32
accumulation ("E2Former-V2 ..." summary §2.2: the streaming, online-softmax
kernel reaches the plain edge-by-edge definition up to rounding order).
The oracle's neighbour rows for the compared nodes come from its own
brute-force predicate (oracle.neighbors.neighbor_rows).
"""
import copy

import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from oracle import attention as oa
from oracle import neighbors as nb
from oracle import sh
from tests import helpers

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}
TE = {l: (32 if l >= 5 else 64) for l in range(7)}   # edges per tile of the tensor-core kernel
S = 4                                                 # destination nodes per tile


def _oracle_rows(wl, nodes):
    csr = nb.neighbor_rows(wl.pos, wl.box, wl.r_c, nodes)
    return oa.attention_workload(wl, nodes=nodes, csr=csr), csr


def _check_rows(wl, out, nl, nodes, tol):
    ref, (rp, col) = _oracle_rows(wl, nodes)
    # the device CSR agrees with the brute force on the compared rows
    grp = nl.row_ptr.cpu().numpy()
    gcol = nl.col_idx[: nl.n_edges].cpu().numpy()
    for i in nodes:
        assert np.array_equal(gcol[grp[i]:grp[i + 1]], col[rp[i]:rp[i + 1]]), i
    err = helpers.rel_err(out[nodes], ref)
    assert err <= tol, err
    return err


@pytest.mark.parametrize("cfg", [3, 4])
def test_fp32_full_size_subset(cuda_ok, cfg):
    """fp32 storage (the SIMT path) on the 30k protein-in-water box (L = 6)
    and the 100k water box, compared on the workload's seeded 1,000-node
    subset with full neighbour rows."""
    wl = wlmod.make_workload(cfg, precision="fp32")
    out, nl = helpers.gpu_forward(wl)
    assert np.all(np.isfinite(out))
    _check_rows(wl, out, nl, wl.subset, TOL["fp32"])


def test_bf16_protein_box_1000_rows(cuda_ok):
    """bf16 tensor-core path at L = 6 (32-edge tiles, the padding unit) on the
    30k protein-in-water box: the seeded 1,000-node subset."""
    wl = helpers.cached_workload(3, "bf16")
    out, nl = helpers.gpu_forward(wl)
    assert np.all(np.isfinite(out))
    _check_rows(wl, out, nl, wl.subset, TOL["bf16"])


def kernel_partition(row_ptr, E, L, n_sm):
    """The fused kernel's work split: G = min(#SM, ceil(E / TE)) CTAs; CTA b
    owns the nodes [n_b, n_{b+1}) (n_0 = 0, n_G = N, otherwise the first
    node whose row starts at or after E b / G); its edges are walked in tiles
    of <= TE edges covering <= 4 nodes.  Returns, per CTA, its node range
    and the nodes of its first and last tile."""
    N = len(row_ptr) - 1
    te = TE[L]
    G = max(1, min(n_sm, -(-E // te)))
    bounds = [0] + [int(np.searchsorted(row_ptr, E * b // G, side="left")) for b in range(1, G)] + [N]
    out = []
    for b in range(G):
        nlo, nhi = bounds[b], bounds[b + 1]
        e0, eend = int(row_ptr[nlo]), int(row_ptr[nhi])
        tiles = []
        if e0 < eend:
            n0 = nlo
            while row_ptr[n0 + 1] <= e0:
                n0 += 1
            while True:
                nlim = min(n0 + S, N)
                e1 = min(e0 + te, eend, int(row_ptr[nlim]))
                last = n0
                while row_ptr[last + 1] < e1:
                    last += 1
                tiles.append((n0, last))
                e0 = e1
                if e0 >= eend:
                    break
                while row_ptr[n0 + 1] <= e0:
                    n0 += 1
        out.append((nlo, nhi, tiles[:1] + tiles[-1:]))
    return out


@pytest.mark.parametrize("cfg", [1, 4])
def test_cta_boundary_and_last_tile_rows(cuda_ok, cfg):
    """Every node next to a boundary between two CTAs' edge ranges, and every
    node of each CTA's first and last tile (nodes spanning tiles, ragged last
    tiles), on the molecule batch and the 100k water box (bf16, tensor
    cores)."""
    import torch
    wl = helpers.cached_workload(cfg, "bf16")
    out, nl = helpers.gpu_forward(wl)
    assert np.all(np.isfinite(out))
    rp = nl.row_ptr.cpu().numpy().astype(np.int64)
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    part = kernel_partition(rp, nl.n_edges, wl.L, n_sm)
    rows = set()
    for nlo, nhi, tiles in part:
        rows.update([nlo, nhi - 1, max(nlo - 1, 0), min(nhi, wl.N - 1)])
        for n0, n1 in tiles:
            rows.update(range(n0, n1 + 1))
    rows = np.array(sorted(r for r in rows if 0 <= r < wl.N and rp[r + 1] > rp[r]), np.int64)
    assert len(rows) >= len(part)
    _check_rows(wl, out, nl, rows, TOL["bf16"])


def _cube_transform(wl, out_unused, Q, t):
    """Positions Q p + t wrapped into the box, features D(Q) x (float64)."""
    w2 = copy.deepcopy(wl)
    p = wl.pos.astype(np.float64) @ Q.T + t[None, :]
    w2.pos = wlmod.wrap_into_box(p, wl.box.astype(np.float64))
    D = [sh.wigner_d_fit(l, Q) for l in range(wl.L + 1)]
    xr = np.empty(wl.x.shape, np.float64)
    for l in range(wl.L + 1):
        s_ = slice(l * l, (l + 1) ** 2)
        xr[:, s_, :] = D[l] @ wl.x[:, s_, :].astype(np.float64)
    return w2, xr, D


def _rotate_out(out, D, L):
    o = np.empty_like(out)
    for l in range(L + 1):
        s_ = slice(l * l, (l + 1) ** 2)
        o[:, s_, :] = D[l] @ out[:, s_, :]
    return o


def test_periodic_equivariance_fp32(cuda_ok):
    """C20 on the GPU: 3,000-atom periodic water box (L = 4, C = 32, H = 2,
    fp32): a proper rotation of the cube plus a translation, wrapped back
    into the box, rotates the output by D(Q), to <= 1e-5."""
    wl = wlmod.make_workload(2, precision="fp32", C=32, H=2)
    out, _ = helpers.gpu_forward(wl)
    rng = np.random.default_rng(23)
    rots = wlmod.cube_rotations()
    for k in rng.choice(len(rots), size=3, replace=False):
        Q = rots[k]
        t = rng.uniform(0, wl.box[0], 3)
        w2, xr, D = _cube_transform(wl, out, Q, t)
        w2.x = xr.astype(np.float32)
        out2, _ = helpers.gpu_forward(w2)
        err = helpers.rel_err(out2, _rotate_out(out, D, wl.L))
        assert err <= 1e-5, (k, err)


def test_periodic_equivariance_bf16_tensor_cores(cuda_ok):
    """The bf16 tensor-core path on the 3,000-atom water box (L = 4, C = 128,
    H = 8): the rotated features are rounded to bf16 again, so the bound is
    the bf16 parity tolerance; the rotated system itself is also checked
    against the oracle on sampled rows."""
    wl = helpers.cached_workload(2, "bf16")
    out, _ = helpers.gpu_forward(wl)
    rng = np.random.default_rng(29)
    rots = wlmod.cube_rotations()
    k = int(rng.integers(1, len(rots)))
    Q = rots[k]
    t = rng.uniform(0, wl.box[0], 3)
    w2, xr, D = _cube_transform(wl, out, Q, t)
    w2.x = wlmod.round_to(xr, "bf16")
    out2, nl2 = helpers.gpu_forward(w2)
    err = helpers.rel_err(out2, _rotate_out(out, D, wl.L))
    assert err <= TOL["bf16"], err
    nodes = np.sort(rng.choice(wl.N, size=100, replace=False))
    _check_rows(w2, out2, nl2, nodes, TOL["bf16"])
