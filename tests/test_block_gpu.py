"""E2Former-V2 block (merged RMS norm, attention, scalar-gated FFN, residuals)
on the GPU against the block oracle (oracle/block.py), on the same seeded
inputs.  Error measure: max |gpu - ref| / max |ref| over the compared rows;
<= 1e-4 with fp32 storage, <= 2e-2 with bf16 storage (the oracle then
rounds the normalised features to bf16 like the GPU stores them)."""
import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from oracle import block as ob
from oracle import neighbors as nb
from oracle import sh
from tests import helpers

pytestmark = pytest.mark.gpu


def _run(wl, layers, prec):
    import torch
    from atomistic_mlip_b200 import e2f
    pos = torch.from_numpy(wl.pos).cuda()
    x = torch.from_numpy(np.ascontiguousarray(wl.x, np.float32)).cuda()
    box = None if wl.box is None else [float(b) for b in wl.box]
    nl = e2f.build_neighbors(pos, box, wl.r_c)
    bws = [e2f.DeviceBlockWeights.from_layer(lw, "cuda", prec) for lw in layers]
    out = e2f.model_forward(x, pos, nl, bws)
    torch.cuda.synchronize()
    assert e2f.stream_status() == 0
    return out.double().cpu().numpy()


def test_block_fp32_cluster(cuda_ok):
    """24-atom cluster, L = 2, C = 8, one head, Hd = 32: CUDA-core GEMMs."""
    wl = wlmod.make_workload(0)
    lw = wlmod.make_layer_weights(wl.L, wl.C, wl.H, "fp32", 31)
    got = _run(wl, [lw], "fp32")
    ref = ob.block_forward(wl.pos, wl.box, wl.r_c, nb.neighbors(wl.pos, wl.box, wl.r_c), wl.x, lw)
    assert helpers.rel_err(got, ref) <= 1e-4


def test_two_layer_model_fp32(cuda_ok):
    wl = wlmod.make_workload(0, C=16, H=2, L=3)
    layers = [wlmod.make_layer_weights(wl.L, wl.C, wl.H, "fp32", s) for s in (41, 42)]
    got = _run(wl, layers, "fp32")
    ref = ob.model_forward(wl.pos, wl.box, wl.r_c, nb.neighbors(wl.pos, wl.box, wl.r_c), wl.x, layers)
    assert helpers.rel_err(got, ref) <= 1e-4


def test_block_fp32_equivariance(cuda_ok):
    """The whole block on the GPU rotates with the system (fp32, <= 1e-5)."""
    wl = wlmod.make_workload(0)
    lw = wlmod.make_layer_weights(wl.L, wl.C, wl.H, "fp32", 32)
    out = _run(wl, [lw], "fp32")
    Q = wlmod.haar_rotation(np.random.default_rng(33))
    D = [sh.wigner_d_fit(l, Q) for l in range(wl.L + 1)]
    w2 = wlmod.make_workload(0)
    w2.pos = (wl.pos.astype(np.float64) @ Q.T).astype(np.float32)
    xr = np.empty_like(wl.x)
    orot = np.empty_like(out)
    for l in range(wl.L + 1):
        s_ = slice(l * l, (l + 1) ** 2)
        xr[:, s_, :] = (D[l] @ wl.x[:, s_, :].astype(np.float64)).astype(np.float32)
        orot[:, s_, :] = D[l] @ out[:, s_, :]
    w2.x = xr
    assert helpers.rel_err(_run(w2, [lw], "fp32"), orot) <= 1e-5


@pytest.mark.parametrize("L", [2, 4])
def test_block_bf16_tensor_cores(cuda_ok, L):
    """C = 128, H = 8, Hd = 512, bf16: the tensor-core attention and the
    tensor-core FFN GEMMs (gate, up with gate, down into the residual)."""
    wl0 = wlmod.make_workload(0)
    wl = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=L, C=128, H=8, precision="fp32", seed=50 + L)
    lw = wlmod.make_layer_weights(L, 128, 8, "bf16", 60 + L)
    got = _run(wl, [lw], "bf16")
    ref = ob.block_forward(wl.pos, wl.box, wl.r_c, nb.neighbors(wl.pos, wl.box, wl.r_c), wl.x, lw,
                           round_bf16=True)
    assert helpers.rel_err(got, ref) <= 2e-2


def test_block_bf16_water_box_sampled(cuda_ok):
    """The 3,000-atom periodic water box at full width (bf16), 120 sampled rows."""
    wl = helpers.cached_workload(2, "bf16")
    lw = wlmod.make_layer_weights(wl.L, wl.C, wl.H, "bf16", 70)
    got = _run(wl, [lw], "bf16")
    assert np.all(np.isfinite(got))
    nodes = np.sort(np.random.default_rng(71).choice(wl.N, size=120, replace=False))
    csr = nb.neighbor_rows(wl.pos, wl.box, wl.r_c, nodes)
    ref = ob.block_forward(wl.pos, wl.box, wl.r_c, csr, wl.x, lw, nodes=nodes, round_bf16=True)
    assert helpers.rel_err(got[nodes], ref) <= 2e-2


def test_block_bf16_water100k_sampled(cuda_ok):
    """The 100,002-atom water box, one block (the configuration the block is
    timed on), 40 sampled rows of the full-size call against the oracle on
    the rows' local subsystem (the rows' atoms and their neighbours)."""
    wl = helpers.cached_workload(4, "bf16")
    lw = wlmod.make_layer_weights(wl.L, wl.C, wl.H, "bf16", 72)
    got = _run(wl, [lw], "bf16")
    nodes = np.sort(np.random.default_rng(73).choice(wl.N, size=40, replace=False))
    U, csr, idx = helpers.local_rows(wl.pos, wl.box, wl.r_c, nodes)
    ref = ob.block_forward(wl.pos[U], wl.box, wl.r_c, csr, wl.x[U], lw, nodes=idx[nodes], round_bf16=True)
    assert np.all(np.isfinite(got[nodes]))
    assert helpers.rel_err(got[nodes], ref) <= 2e-2


def test_two_layer_model_water_box_sampled(cuda_ok):
    """Two blocks on the 3,000-atom water box (bf16, as timed), 8 sampled
    rows: the second block's rows read the first block's outputs at the rows
    and their neighbours, which the oracle computes on their own local
    subsystem first."""
    wl = helpers.cached_workload(2, "bf16")
    layers = [wlmod.make_layer_weights(wl.L, wl.C, wl.H, "bf16", s) for s in (74, 75)]
    got = _run(wl, layers, "bf16")
    nodes = np.sort(np.random.default_rng(76).choice(wl.N, size=8, replace=False))
    U1, csr2, idx1 = helpers.local_rows(wl.pos, wl.box, wl.r_c, nodes)
    U2, csr1, idx2 = helpers.local_rows(wl.pos, wl.box, wl.r_c, U1)
    x1 = ob.block_forward(wl.pos[U2], wl.box, wl.r_c, csr1, wl.x[U2], layers[0], nodes=idx2[U1],
                          round_bf16=True)
    ref = ob.block_forward(wl.pos[U1], wl.box, wl.r_c, csr2, x1, layers[1], nodes=idx1[nodes], round_bf16=True)
    assert helpers.rel_err(got[nodes], ref) <= 2e-2
