"""Unit parity: the device Wigner-D generator and the q/k/v projections
against the oracle."""
import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from oracle import attention as oa
from oracle import sh
from tests import helpers

pytestmark = pytest.mark.gpu


def test_wigner_blocks_match_oracle(cuda_ok):
    import torch
    from atomistic_mlip_b200 import e2f
    rng = np.random.default_rng(5)
    R = np.stack([wlmod.haar_rotation(rng) for _ in range(300)])
    # include the two poles of the edge frame
    R[0] = np.eye(3)
    R[1] = np.diag([1.0, -1.0, -1.0])
    D = e2f.wigner_d(torch.from_numpy(R.astype(np.float32)).cuda(), 6).cpu().numpy()
    off = 0
    for l in range(7):
        w = 2 * l + 1
        ref = sh.wigner_d_fit(l, R.astype(np.float32).astype(np.float64))
        got = D[:, off:off + w * w].reshape(-1, w, w)
        off += w * w
        assert np.max(np.abs(got - ref)) < 2e-6, l


def _check_projection(wl, prec):
    import torch
    from atomistic_mlip_b200 import e2f
    _, x, w, _ = helpers.to_device(wl, prec)
    q, k, v = e2f.project_qkv(x, w)
    torch.cuda.synchronize()
    for got, W in ((q, wl.Wq), (k, wl.Wk), (v, wl.Wv)):
        ref = oa.project(wl.x, W, wl.L)
        g = got.double().cpu().numpy()
        if prec == "fp32":
            assert helpers.rel_err(g, ref) < 1e-5
        else:
            # one rounding to bf16 of an fp32-accumulated value
            assert np.all(np.abs(g - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * np.max(np.abs(ref)))


@pytest.mark.parametrize("prec,C,H", [("fp32", 64, 4), ("bf16", 64, 4), ("bf16", 128, 8)])
def test_projection_matches_oracle(cuda_ok, prec, C, H):
    """C = 128 bf16 takes the tensor-core kernel (3,000 nodes: every degree
    ends in a ragged 128-row tile, and each CTA walks tiles of several
    degrees); the others the SIMT kernel."""
    _check_projection(wlmod.make_workload(2, precision=prec, C=C, H=H), prec)


@pytest.mark.parametrize("n,L", [(1, 0), (5, 6), (300, 2)])
def test_projection_tensor_core_few_tiles(cuda_ok, n, L):
    """The tensor-core projection with fewer tiles than SMs: one node, one
    partial tile per degree up to L = 6, and a few hundred rows."""
    rng = np.random.default_rng(40 + n)
    pos = rng.uniform(0.0, 8.0, (n, 3)).astype(np.float32)
    _check_projection(wlmod.make_custom(pos, None, 3.0, L=L, C=128, H=8, precision="bf16", seed=11 + L), "bf16")
