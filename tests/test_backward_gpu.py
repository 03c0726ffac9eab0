"""Backward of the attention on the GPU (e2f_attention_backward): dL/dx and
dL/dpos of L = sum(G * o) against the gradient oracle
(oracle/attention_grad.py: autograd of the fp64 restatement of the operator,
itself pinned to finite differences of oracle/attention.py).

Error measure: max |gpu - ref| / max |ref| per gradient; <= 1e-4 with fp32
storage, <= 3e-2 with bf16 storage (the gradient passes through the bf16
rotated features and SO(2) products twice).  Forces sum to zero: every edge
adds opposite vectors to its two atoms.

The two water boxes the forces are timed on (3,000 and 100,002 atoms) are
checked on sampled atoms: dL/dpos_i and dL/dx_i depend only on the outputs of
atom i and of its neighbours, so the oracle evaluates exactly those outputs
(full neighbour rows) over the atoms they read."""
import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from oracle import attention_grad as ag
from oracle import neighbors as nb
from tests import helpers

pytestmark = pytest.mark.gpu


def _gpu_grads(wl, G, prec):
    import torch
    from atomistic_mlip_b200 import e2f
    pos, x, w, box = helpers.to_device(wl, prec)
    nl = e2f.build_neighbors(pos, box, wl.r_c)
    g = torch.from_numpy(np.ascontiguousarray(G, np.float32)).cuda()
    gx, gp = e2f.attention_backward(x, pos, nl, w, g)
    torch.cuda.synchronize()
    assert e2f.stream_status() == 0
    return gx.double().cpu().numpy(), gp.double().cpu().numpy()


def _check(wl, prec, tol, seed=5):
    G = np.random.default_rng(seed).standard_normal(wl.x.shape)
    csr = nb.neighbors(wl.pos, wl.box, wl.r_c)
    ref = ag.gradients(wl, csr, G)
    gx, gp = _gpu_grads(wl, G, prec)
    ex = helpers.rel_err(gx, ref["x"])
    ep = helpers.rel_err(gp, ref["pos"])
    assert ex <= tol and ep <= tol, (ex, ep)
    # Newton's third law: the force contributions of each edge cancel
    assert np.max(np.abs(gp.sum(axis=0))) <= 1e-5 * np.max(np.abs(gp)) * max(1, wl.N) ** 0.5
    return ex, ep


@pytest.mark.parametrize("cfg", [2, 4])
def test_backward_water_sampled(cuda_ok, cfg):
    """The 3,000-atom (cfg 2) and 100,002-atom (cfg 4) periodic water boxes,
    L = 4, C = 128, H = 8, bf16: the full-size backward launch, two sampled
    atoms against the oracle's local gradients."""
    wl = helpers.cached_workload(cfg, "bf16")
    rng = np.random.default_rng(400 + cfg)
    G = rng.standard_normal(wl.x.shape).astype(np.float32)
    gx, gp = _gpu_grads(wl, G, "bf16")
    nodes = np.sort(rng.choice(wl.N, size=2, replace=False))
    ref_p, ref_x = helpers.local_gradients(wl, nodes, G)
    assert helpers.rel_err(gp[nodes], ref_p) <= 3e-2
    assert helpers.rel_err(gx[nodes], ref_x) <= 3e-2


def test_backward_fp32_cluster(cuda_ok):
    """24-atom cluster, L = 2, C = 8, one head (fp32)."""
    _check(wlmod.make_workload(0), "fp32", 1e-4)


@pytest.mark.parametrize("L", [0, 1, 3, 4, 6])
def test_backward_fp32_degrees(cuda_ok, L):
    """C = 16 (the per-row dL/dD form, C a multiple of 16), every tile shape
    of the degree loop up to the largest L."""
    wl = wlmod.make_workload(0, L=L, C=16, H=2)
    _check(wl, "fp32", 1e-4, seed=10 + L)


def test_backward_fp32_periodic(cuda_ok):
    """Minimum-image edges across the faces of a periodic box."""
    rng = np.random.default_rng(3)
    box = np.full(3, 11.0, np.float32)
    pos = rng.uniform(0, 11.0, (40, 3)).astype(np.float32)
    wl = wlmod.make_custom(pos, box, 4.0, L=2, C=8, H=2, precision="fp32", seed=4)
    _check(wl, "fp32", 1e-4)


def test_backward_bf16_full_width(cuda_ok):
    """C = 128, H = 8, L = 4 (bf16 storage, fp32 accumulation) on the
    24-atom cluster."""
    wl0 = wlmod.make_workload(0)
    wl = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=4, C=128, H=8, precision="bf16", seed=8)
    _check(wl, "bf16", 3e-2)


def test_backward_isolated_atoms_and_no_edges(cuda_ok):
    """Isolated atoms get zero gradients; a system with no edge at all gives
    zero dL/dx and dL/dpos (every chunk is empty)."""
    pos = np.array([[0, 0, 0], [1.1, 0.4, -0.3], [40, 40, 40], [80, 0, 0]], np.float32)
    wl = wlmod.make_custom(pos, None, 3.0, L=2, C=16, H=2, precision="fp32", seed=500)
    ex, ep = _check(wl, "fp32", 1e-4, seed=501)
    G = np.random.default_rng(502).standard_normal(wl.x.shape)
    gx, gp = _gpu_grads(wl, G, "fp32")
    assert np.all(gx[2:] == 0) and np.all(gp[2:] == 0)
    far = wlmod.make_custom(pos[2:], None, 3.0, L=2, C=16, H=2, precision="fp32", seed=503)
    gx, gp = _gpu_grads(far, np.random.default_rng(504).standard_normal(far.x.shape), "fp32")
    assert np.all(gx == 0) and np.all(gp == 0)
