"""The step-by-step backward of tests/backward_plan.py (the derivation a
tiled backward kernel follows, in the two-angle gauge) against autograd of
the plain definition (oracle.attention_grad)."""
import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from oracle import attention as oa
from oracle import attention_grad as ag
from oracle import neighbors as nb
from tests import backward_plan as bp


def _system(periodic: bool, L: int, seed: int):
    rng = np.random.default_rng(seed)
    if periodic:
        b = 9.0
        pos = rng.uniform(0.0, b, (16, 3)).astype(np.float32)
        wl = wlmod.make_custom(pos, np.array([b, b, b], np.float32), 4.0, L=L, C=8, H=2, seed=seed)
    else:
        pos = rng.uniform(0.0, 7.0, (14, 3)).astype(np.float32)
        wl = wlmod.make_custom(pos, None, 4.0, L=L, C=8, H=2, seed=seed)
    return wl, nb.neighbors(wl.pos, wl.box, wl.r_c)


def _rel(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b))) / max(np.max(np.abs(np.asarray(b))), 1e-30))


@pytest.mark.parametrize("periodic,L", [(False, 3), (True, 2), (False, 1)])
def test_backward_plan_matches_autograd(periodic, L):
    wl, csr = _system(periodic, L, seed=50 + L)
    G = np.random.default_rng(51).standard_normal((wl.N, (L + 1) ** 2, wl.C))
    got = bp.backward(wl, csr, G)
    # the two-angle gauge gives the same output as the oracle's minimal rotation
    assert _rel(got["o"], oa.attention_workload(wl, csr=csr)) < 1e-12
    ref = ag.gradients(wl, csr, G)
    for key in ("pos", "x", "W0", "rad_W1", "rad_W2"):
        assert _rel(got[key], ref[key]) < 1e-8, key
    for key in ("Wq", "Wk", "Wv"):
        for l in range(L + 1):
            assert _rel(got[key][l], ref[key][l]) < 1e-8, (key, l)
    for key in ("Wr", "Wi"):
        for m in range(1, L + 1):
            assert _rel(got[key][m], ref[key][m]) < 1e-8, (key, m)
