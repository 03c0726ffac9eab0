"""The seeded workload generators produce the systems they describe."""
import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as w
from oracle import neighbors as nb


def test_deterministic_and_bf16_exact():
    a, b = w.make_workload(0), w.make_workload(0)
    np.testing.assert_array_equal(a.pos, b.pos)
    np.testing.assert_array_equal(a.x, b.x)
    c = w.make_workload(0, precision="bf16")
    bits = w.f32_to_bf16_bits(c.x)
    np.testing.assert_array_equal(w.bf16_bits_to_f32(bits), c.x)
    np.testing.assert_array_equal(w.bf16_bits_to_f32(w.f32_to_bf16_bits(c.W0)), c.W0)
    assert c.rad_W1.dtype == np.float32


def test_cfg0_cluster():
    wl = w.make_workload(0)
    assert wl.N == 24 and wl.box is None and wl.L == 2 and wl.C == 8 and wl.H == 1
    assert np.all(wl.pos >= 0) and np.all(wl.pos < 6)
    d = np.linalg.norm(wl.pos[:, None].astype(np.float64) - wl.pos[None], axis=-1)
    assert np.min(d + 100 * np.eye(24)) >= 0.9 - 1e-6


def test_cfg1_molecules_are_disconnected():
    wl = w.make_workload(1, C=8, L=1, H=1)
    sizes = wl.meta["mol_sizes"]
    assert len(sizes) == 256 and sizes.min() >= 20 and sizes.max() <= 60
    assert wl.N == sizes.sum()
    mol = np.repeat(np.arange(256), sizes)
    rp, col = nb.neighbors(wl.pos, None, wl.r_c)
    src = np.repeat(np.arange(wl.N), np.diff(rp))
    assert np.all(mol[src] == mol[col])
    assert 30 < len(col) / wl.N < 50


def test_cfg2_water_box():
    wl = w.make_workload(2, C=8, L=1, H=1)
    assert wl.N == 3000 and np.all(wl.box == np.float32(31.0))
    assert np.all(wl.pos >= 0) and np.all(wl.pos < wl.box)
    oh = np.linalg.norm(wl.pos[1::3].astype(np.float64) - wl.pos[0::3], axis=1)
    oh = np.minimum(oh, np.linalg.norm(((wl.pos[1::3].astype(np.float64) - wl.pos[0::3] + 15.5) % 31) - 15.5, axis=1))
    np.testing.assert_allclose(oh, 0.96, atol=1e-4)


@pytest.mark.parametrize("cfg,n", [(3, 30000), (4, 100002)])
def test_large_positions(cfg, n):
    rng = np.random.default_rng(w.BASE_SEED + cfg)
    p, box, _ = w.make_positions(cfg, rng)
    pos = w.wrap_into_box(p, box)
    assert pos.shape == (n, 3)
    assert np.all(pos >= 0) and np.all(pos < box.astype(np.float32))
    np.testing.assert_allclose(n / np.prod(box), 0.1, rtol=1e-3)


def test_sweep_sizes():
    for target, n in ((10000, 10002), (30000, 30000), (100000, 100002)):
        units, N, b = w.water_box_size(target)
        assert N == n and abs(N / b ** 3 - 0.1) < 1e-9
