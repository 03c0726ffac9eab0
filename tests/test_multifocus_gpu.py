"""Multi-focus attention on the GPU (e2f_attention_forward_multifocus, the
tensor-core kernel with per-stream SO(2) stacks and the cross-focus softmax)
against the oracle's multi-focus variant (oracle/attention.py, F1-F3) on the
same seeded inputs.  Error measure and bound as for the bf16 tensor-core
path: max |gpu - ref| / max |ref| <= 2e-2."""
import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from oracle import attention as oa
from oracle import neighbors as nb
from tests import helpers

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _gpu(wl, F, a):
    import torch
    from atomistic_mlip_b200 import e2f
    pos, x, w, box = helpers.to_device(wl, "bf16")
    nl = e2f.build_neighbors(pos, box, wl.r_c)
    at = torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    out = e2f.attention_forward_multifocus(x, pos, nl, w, F, at)
    torch.cuda.synchronize()
    assert e2f.stream_status() == 0
    return out.double().cpu().numpy(), nl


def _focus(C, seed, scale=2.0):
    return (scale * np.random.default_rng(seed).standard_normal(C)).astype(np.float32)


@pytest.mark.parametrize("L,F", [(2, 2), (4, 4), (4, 8)])
def test_multifocus_cluster(cuda_ok, L, F):
    """24-atom cluster, C = 128, H = 8, bf16."""
    wl0 = wlmod.make_workload(0)
    wl = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=L, C=128, H=8, precision="bf16", seed=200 + L + F)
    a = _focus(128, 210 + F)
    got, _ = _gpu(wl, F, a)
    ref = oa.attention_workload(wl, focus=(F, a.astype(np.float64)))
    assert np.all(np.isfinite(got))
    assert helpers.rel_err(got, ref) <= TOL


def test_single_stream_equals_plain_attention(cuda_ok):
    """F = 1 through the multi-focus entry is the plain operator (the same
    kernel; the two runs differ only by the order of the float atomics that
    sum each tile's softmax weights)."""
    wl0 = wlmod.make_workload(0)
    wl = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=4, C=128, H=8, precision="bf16", seed=220)
    got, _ = _gpu(wl, 1, np.zeros(128, np.float32))
    plain, _ = helpers.gpu_forward(wl)
    assert helpers.rel_err(got, plain) <= 1e-6


def test_multifocus_molecules_sampled(cuda_ok):
    """The 256-molecule batch (10,304 atoms), L = 4, F = 4, 150 sampled rows."""
    wl = helpers.cached_workload(1, "bf16")
    a = _focus(wl.C, 230)
    got, nl = _gpu(wl, 4, a)
    assert np.all(np.isfinite(got))
    rng = np.random.default_rng(231)
    nodes = np.sort(rng.choice(wl.N, size=150, replace=False))
    csr = helpers.oracle_csr(1)
    ref = oa.attention_workload(wl, nodes=nodes, csr=csr, focus=(4, a.astype(np.float64)))
    assert helpers.rel_err(got[nodes], ref) <= TOL


def test_multifocus_water100k_sampled(cuda_ok):
    """The benchmark configuration: the 100,002-atom water box, L = 4, F = 4,
    40 sampled rows of the full-size launch."""
    wl = helpers.cached_workload(4, "bf16")
    a = _focus(wl.C, 240)
    got, _ = _gpu(wl, 4, a)
    assert np.all(np.isfinite(got))
    nodes = np.sort(np.random.default_rng(241).choice(wl.N, size=40, replace=False))
    csr = nb.neighbor_rows(wl.pos, wl.box, wl.r_c, nodes)
    ref = oa.attention_workload(wl, nodes=nodes, csr=csr, focus=(4, a.astype(np.float64)))
    assert helpers.rel_err(got[nodes], ref) <= TOL
