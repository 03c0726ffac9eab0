"""Attention parity: the CUDA path against the fp64 oracle on the same
seeded inputs.

Error measure: max |gpu - ref| / max |ref| over the compared rows.
Tolerances: <= 1e-4 with fp32 storage, <= 2e-2 with bf16 storage and fp32
accumulation; rotation equivariance of the fp32 path <= 1e-5.
Full-size workloads are compared on a seeded subset of destination rows
(each full row of the CSR), the rest of the output being checked finite.
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


def _compare(wl, nodes=None, tol=None):
    out, nl = helpers.gpu_forward(wl)
    csr = nb.neighbors(wl.pos, wl.box, wl.r_c) if wl.N <= 20000 else helpers.oracle_csr(wl.cfg)
    ref = oa.attention_workload(wl, nodes=nodes, csr=csr)
    got = out if nodes is None else out[nodes]
    assert np.all(np.isfinite(out))
    err = helpers.rel_err(got, ref)
    assert err <= (tol or TOL[wl.precision]), err
    return out, err


def test_cfg0_fp32_full(cuda_ok):
    _compare(wlmod.make_workload(0))


def test_cfg0_fp32_equivariance(cuda_ok):
    """P7 on the GPU: f(Q p, D(Q) x) = D(Q) f(p, x) within 1e-5 (fp32)."""
    wl = wlmod.make_workload(0)
    out, _ = helpers.gpu_forward(wl)
    rng = np.random.default_rng(17)
    for _ in range(3):
        Q = wlmod.haar_rotation(rng)
        w2 = copy.deepcopy(wl)
        w2.pos = (wl.pos.astype(np.float64) @ Q.T).astype(np.float32)
        D = [sh.wigner_d_fit(l, Q) for l in range(wl.L + 1)]
        xr = np.empty_like(wl.x)
        orot = np.empty_like(out)
        for l in range(wl.L + 1):
            s_ = slice(l * l, (l + 1) ** 2)
            xr[:, s_, :] = (D[l] @ wl.x[:, s_, :].astype(np.float64)).astype(np.float32)
            orot[:, s_, :] = D[l] @ out[:, s_, :]
        w2.x = xr
        out2, _ = helpers.gpu_forward(w2)
        assert helpers.rel_err(out2, orot) <= 1e-5


def test_reduced_width_full_graph_fp32(cuda_ok):
    """cfg2 geometry, L=4, C=32, H=2: every row of a 3,000-atom periodic box."""
    wl = wlmod.make_workload(2, precision="fp32", C=32, H=2)
    _compare(wl, nodes=np.arange(0, wl.N, 3))


@pytest.mark.parametrize("L", [0, 1, 3, 5, 6])
def test_degrees_small_width(cuda_ok, L):
    wl = wlmod.make_workload(0, L=L, C=16, H=2)
    _compare(wl)


@pytest.mark.parametrize("cfg,prec,n", [(1, "bf16", 300), (1, "fp32", 150), (2, "bf16", 200),
                                        (2, "fp32", 100), (3, "bf16", 60), (4, "bf16", 150)])
def test_full_size_sampled_rows(cuda_ok, cfg, prec, n):
    wl = helpers.cached_workload(cfg, "bf16") if prec == "bf16" else wlmod.make_workload(cfg, precision="fp32")
    nodes = np.sort(np.random.default_rng(100 + cfg).choice(wl.N, size=n, replace=False))
    _compare(wl, nodes=nodes)


@pytest.mark.parametrize("L", [1, 2, 3, 4, 5, 6])
def test_tensor_core_path_small(cuda_ok, L):
    """bf16, C = 128, H = 8 takes the tcgen05 kernel: 24-atom cluster (7 edge
    tiles of 64, or 14 of 32 for L >= 5; ragged last tile) for every degree
    but L = 3, which the library routes to the CUDA-core kernel (its
    tensor-core build is not instantiated)."""
    wl0 = wlmod.make_workload(0)
    wl = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=L, C=128, H=8, precision="bf16", seed=3 + L)
    _compare(wl)


@pytest.mark.parametrize("H", [4, 16])
def test_tensor_core_path_head_counts(cuda_ok, H):
    """The smallest and largest head counts the tcgen05 kernel takes (32 and
    8 channels per head: head sums over four blocks, or one)."""
    wl0 = wlmod.make_workload(0)
    wl = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=4, C=128, H=H, precision="bf16", seed=20 + H)
    _compare(wl)


def test_tensor_core_path_isolated_and_low_degree(cuda_ok):
    """Isolated atoms (empty rows), degree-1 rows and a dense clump in one
    batch: tiles bounded by the node-slot limit, nodes spanning tiles."""
    rng = np.random.default_rng(8)
    clump = rng.uniform(0, 4.0, (90, 3))
    pairs = np.array([[20, 20, 20], [21, 20, 20], [40, 40, 40], [60, 5, 5]], float)
    chain = np.stack([np.arange(12) * 1.4 + 80, np.full(12, 80.0), np.full(12, 80.0)], 1)
    pos = np.concatenate([clump, pairs, chain]).astype(np.float32)
    wl = wlmod.make_custom(pos, None, 5.0, L=4, C=128, H=4, precision="bf16", seed=9)
    out, _ = _compare(wl)
    assert np.all(out[92] == 0) and np.all(out[93] == 0)


def test_isolated_atoms_and_coincident(cuda_ok):
    pos = np.array([[0, 0, 0], [50, 50, 50], [1.0, 0.5, 0.2], [1.0, 0.5, 0.2], [0.3, 1.2, 2.0]], np.float32)
    wl = wlmod.make_custom(pos, None, 3.0, L=3, C=16, H=4, precision="fp32", seed=4)
    out, _ = _compare(wl)
    assert np.all(out[1] == 0)


def test_single_atom(cuda_ok):
    wl = wlmod.make_custom(np.array([[1.0, 2.0, 3.0]], np.float32), None, 3.0, L=2, C=8, H=1, seed=1)
    out, _ = helpers.gpu_forward(wl)
    assert out.shape == (1, 9, 8) and np.all(out == 0)


def test_neighbour_order_invariance(cuda_ok):
    """P8 on the GPU: a permuted CSR row gives the same output (fp32)."""
    import torch
    from atomistic_mlip_b200 import e2f
    wl = wlmod.make_workload(0)
    pos, x, w, box = helpers.to_device(wl)
    nl = e2f.build_neighbors(pos, box, wl.r_c)
    o1 = e2f.attention_forward(x, pos, nl, w).double().cpu().numpy()
    rp = nl.row_ptr.cpu().numpy()
    col = nl.col_idx[: nl.n_edges].cpu().numpy().copy()
    rng = np.random.default_rng(3)
    for i in range(wl.N):
        seg = col[rp[i]:rp[i + 1]]
        rng.shuffle(seg)
    nl2 = e2f.NeighborList(nl.row_ptr, torch.from_numpy(col).cuda(), nl.n_edges, nl.box, nl.r_c)
    o2 = e2f.attention_forward(x, pos, nl2, w).double().cpu().numpy()
    assert helpers.rel_err(o2, o1) <= 1e-5


def test_tensor_core_path_large_logits(cuda_ok):
    """Features scaled by 2 (exact in bf16) spread each node's logits by about
    20, so later tiles of a node exceed its reference maximum by more than
    the margin of 8 and the online softmax rescales the node's earlier sums.
    (Much larger scales make the comparison measure the bf16 rounding of q
    and k, amplified by the logit size, rather than the kernel.)"""
    wl0 = wlmod.make_workload(0)
    wl = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=4, C=128, H=8, precision="bf16", seed=31)
    wl.x = (wl.x * 2.0).astype(np.float32)
    _compare(wl)
