"""Re-indexed CG convolution on the GPU (e2f_cg_conv_forward, edge frame)
against the dense global-frame oracle (oracle/cg.py) on the same seeded
inputs.  Error measure: max |gpu - ref| / max |ref| over the compared rows.
The GPU reads x in its storage type and computes in fp32; the oracle gets
the same stored values (bf16-rounded where the GPU stores bf16), so both
precisions are held to the fp32 bound 2e-5.  Rotation equivariance of the
fp32 path: <= 1e-5."""
import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from oracle import cg
from oracle import neighbors as nb
from oracle import sh
from tests import helpers

pytestmark = pytest.mark.gpu

TOL = 2e-5


def _gpu(pos, box, r_c, x, W, L, prec):
    import torch
    from atomistic_mlip_b200 import e2f
    dt = torch.float32 if prec == "fp32" else torch.bfloat16
    p = torch.from_numpy(np.ascontiguousarray(pos, np.float32)).cuda()
    xt = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to("cuda", dt)
    Wt = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    nl = e2f.build_neighbors(p, None if box is None else [float(b) for b in box], r_c)
    out = e2f.cg_conv_forward(xt, p, nl, Wt, L)
    torch.cuda.synchronize()
    assert e2f.stream_status() == 0
    return out.double().cpu().numpy()


def _stored(x, prec):
    return wlmod.round_to(np.asarray(x, np.float32), prec)


def _check(pos, box, r_c, x, W, L, prec, nodes=None):
    xs = _stored(x, prec)
    got = _gpu(pos, box, r_c, xs, W, L, prec)
    rp, col = nb.neighbors(pos, box, r_c)[:2] if nodes is None else nb.neighbor_rows(pos, box, r_c, nodes)[:2]
    ref = cg.cg_conv(pos, box, r_c, rp, col, xs, W, L, nodes=nodes)
    if nodes is not None:
        got = got[nodes]
    assert np.all(np.isfinite(got))
    err = helpers.rel_err(got, ref)
    assert err <= TOL, err
    return got


@pytest.mark.parametrize("L", [0, 1, 2, 3, 4, 5, 6])
def test_cg_conv_cluster_fp32(cuda_ok, L):
    """24-atom open cluster, C = 8 (four threads per node), every degree."""
    wl = wlmod.make_workload(0, L=L, C=8, H=1)
    _check(wl.pos, wl.box, wl.r_c, wl.x, wlmod.make_cg_weights(L, 8, 100 + L), L, "fp32")


@pytest.mark.parametrize("L", [2, 4])
def test_cg_conv_cluster_bf16_full_width(cuda_ok, L):
    """C = 128 (64 threads per node, two channels each), bf16 storage."""
    wl0 = wlmod.make_workload(0)
    wl = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=L, C=128, H=8, precision="bf16", seed=110 + L)
    _check(wl.pos, wl.box, wl.r_c, wl.x, wlmod.make_cg_weights(L, 128, 120 + L), L, "bf16")


def test_cg_conv_periodic_water_sampled(cuda_ok):
    """The 3,000-atom periodic water box (minimum-image edges), L = 4, C = 32,
    bf16 storage, 100 sampled rows."""
    wl = helpers.cached_workload(2, "bf16")
    rng = np.random.default_rng(131)
    x = rng.standard_normal((wl.N, 25, 32)).astype(np.float32)
    nodes = np.sort(rng.choice(wl.N, size=100, replace=False))
    _check(wl.pos, wl.box, wl.r_c, x, wlmod.make_cg_weights(4, 32, 132), 4, "bf16", nodes=nodes)


def test_cg_conv_empty_rows_and_coincident(cuda_ok):
    """Isolated atoms give exact zeros; two coincident atoms (r = 0) take the
    frame of +z on both sides."""
    pos = np.array([[0, 0, 0], [0, 0, 0], [1.2, 0.3, -0.4], [30, 30, 30], [50, 2, 2]], np.float32)
    rng = np.random.default_rng(140)
    x = rng.standard_normal((5, 16, 6)).astype(np.float32)
    got = _check(pos, None, 3.0, x, wlmod.make_cg_weights(3, 6, 141), 3, "fp32")
    assert np.all(got[3] == 0) and np.all(got[4] == 0)


def test_cg_conv_equivariance_fp32(cuda_ok):
    L, C = 4, 16
    wl = wlmod.make_workload(0, L=L, C=C, H=1)
    W = wlmod.make_cg_weights(L, C, 150)
    out = _gpu(wl.pos, None, wl.r_c, wl.x, W, L, "fp32")
    Q = wlmod.haar_rotation(np.random.default_rng(151))
    D = [sh.wigner_d_fit(l, Q) for l in range(L + 1)]
    pos2 = (wl.pos.astype(np.float64) @ Q.T).astype(np.float32)
    x2 = np.empty_like(wl.x)
    orot = np.empty_like(out)
    for l in range(L + 1):
        s_ = slice(l * l, (l + 1) ** 2)
        x2[:, s_, :] = (D[l] @ wl.x[:, s_, :].astype(np.float64)).astype(np.float32)
        orot[:, s_, :] = D[l] @ out[:, s_, :]
    assert helpers.rel_err(_gpu(pos2, None, wl.r_c, x2, W, L, "fp32"), orot) <= 1e-5


def test_cg_num_paths_matches_oracle(cuda_ok):
    from atomistic_mlip_b200 import e2f
    for L in range(7):
        assert e2f.cg_num_paths(L) == len(cg.paths(L)) == wlmod.cg_num_paths(L)


@pytest.mark.parametrize("cfg", [2, 4])
def test_cg_conv_water_timed_configs(cuda_ok, cfg):
    """The configurations the convolution is timed on: the 3,000- and
    100,002-atom water boxes, L = 4, C = 128, the workload's bf16 features,
    40 sampled rows of the full-size launch against the oracle's brute-force
    rows."""
    wl = helpers.cached_workload(cfg, "bf16")
    W = wlmod.make_cg_weights(4, 128, 77)
    got = _gpu(wl.pos, wl.box, wl.r_c, wl.x, W, 4, "bf16")
    assert np.all(np.isfinite(got))
    nodes = np.sort(np.random.default_rng(160 + cfg).choice(wl.N, size=40, replace=False))
    rp, col = nb.neighbor_rows(wl.pos, wl.box, wl.r_c, nodes)[:2]
    ref = cg.cg_conv(wl.pos, wl.box, wl.r_c, rp, col, _stored(wl.x, "bf16"), W, 4, nodes=nodes)
    assert helpers.rel_err(got[nodes], ref) <= TOL


@pytest.mark.parametrize("L", [4, 6])
def test_cg_conv_cluster_fp32_full_width(cuda_ok, L):
    """C = 128 in fp32 storage (two channels per thread), L = 4 and the
    largest degree, on the 24-atom cluster."""
    wl0 = wlmod.make_workload(0)
    rng = np.random.default_rng(170 + L)
    x = rng.standard_normal((wl0.N, (L + 1) ** 2, 128)).astype(np.float32)
    _check(wl0.pos, wl0.box, wl0.r_c, x, wlmod.make_cg_weights(L, 128, 171 + L), L, "fp32")
