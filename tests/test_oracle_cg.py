"""Pins of the dense Clebsch-Gordan oracle (oracle/cg.py) to what does not
depend on it: a library routine (SymPy's exact Clebsch-Gordan values), the
closed forms of the l2 = 1 coupling table, orthogonality, the intertwining of
the real Wigner matrices built by the Euler / Wigner small-d route, the
product of two harmonics at one point (Gaunt relation), and closed forms of
the convolution (l = 0 only; the l1 = l2 = 1 -> 1 path as a cross product)."""
import math

import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from oracle import cg
from oracle import neighbors as nb
from oracle import sh


def _rand_rot(rng):
    q = rng.standard_normal(4)
    a, b, c, d = q / np.linalg.norm(q)
    return np.array([[a * a + b * b - c * c - d * d, 2 * (b * c - a * d), 2 * (b * d + a * c)],
                     [2 * (b * c + a * d), a * a - b * b + c * c - d * d, 2 * (c * d - a * b)],
                     [2 * (b * d - a * c), 2 * (c * d + a * b), a * a - b * b - c * c + d * d]])


def test_racah_matches_sympy():
    from sympy.physics.quantum.cg import CG
    worst = 0.0
    for l1 in range(4):
        for l2 in range(4):
            for l3 in range(abs(l1 - l2), l1 + l2 + 1):
                for m1 in range(-l1, l1 + 1):
                    for m2 in range(-l2, l2 + 1):
                        m3 = m1 + m2
                        if abs(m3) > l3:
                            continue
                        ref = float(CG(l1, m1, l2, m2, l3, m3).doit())
                        worst = max(worst, abs(cg.cg_complex(l1, m1, l2, m2, l3, m3) - ref))
    assert worst < 1e-14


@pytest.mark.parametrize("j", [1, 2, 3, 5])
def test_l2_one_closed_forms(j):
    """<j m-1; 1 1 | j+1 m>, <j m; 1 0 | j+1 m>, <j m; 1 0 | j m> and
    <j m; 1 0 | j-1 m> from the standard j2 = 1 table."""
    for m in range(-j, j + 1):
        if abs(m - 1) <= j:
            ref = math.sqrt((j + m) * (j + m + 1) / ((2 * j + 1) * (2 * j + 2)))
            assert abs(cg.cg_complex(j, m - 1, 1, 1, j + 1, m) - ref) < 1e-14
        ref = math.sqrt((j - m + 1) * (j + m + 1) / ((2 * j + 1) * (j + 1)))
        assert abs(cg.cg_complex(j, m, 1, 0, j + 1, m) - ref) < 1e-14
        ref = m / math.sqrt(j * (j + 1))
        assert abs(cg.cg_complex(j, m, 1, 0, j, m) - ref) < 1e-14
        if abs(m) <= j - 1:
            ref = -math.sqrt((j - m) * (j + m) / (j * (2 * j + 1)))
            assert abs(cg.cg_complex(j, m, 1, 0, j - 1, m) - ref) < 1e-14


def test_orthogonality():
    for l1 in range(4):
        for l2 in range(4):
            rows = []
            for l3 in range(abs(l1 - l2), l1 + l2 + 1):
                T = cg.cg_complex_tensor(l1, l2, l3).reshape(-1, 2 * l3 + 1)
                assert np.allclose(T.T @ T, np.eye(2 * l3 + 1), atol=1e-13)
                rows.append(T)
                R = cg.real_cg(l1, l2, l3).reshape(-1, 2 * l3 + 1)
                assert np.allclose(R.T @ R, np.eye(2 * l3 + 1), atol=1e-13)
            full = np.concatenate(rows, axis=1)   # unitary change of basis
            assert np.allclose(full @ full.T, np.eye(full.shape[0]), atol=1e-13)


def test_real_coupling_intertwines_wigner_d():
    rng = np.random.default_rng(1)
    for _ in range(3):
        R = _rand_rot(rng)
        for (l1, l2, l3) in cg.paths(4):
            D1, D2, D3 = (sh.wigner_d_euler(l, R) for l in (l1, l2, l3))
            a = rng.standard_normal((2 * l1 + 1, 3))
            b = rng.standard_normal(2 * l2 + 1)
            lhs = cg.tensor_product(D1 @ a, D2 @ b, l1, l2, l3)
            rhs = D3 @ cg.tensor_product(a, b, l1, l2, l3)
            assert np.max(np.abs(lhs - rhs)) < 1e-12, (l1, l2, l3)


def test_gaunt_product_of_harmonics():
    """(Y_l1(u) (x) Y_l2(u))^l3 = sqrt((2l1+1)(2l2+1) / (4 pi (2l3+1)))
    <l1 0; l2 0 | l3 0> Y_l3(u): zero for odd l1 + l2 + l3."""
    rng = np.random.default_rng(2)
    u = rng.standard_normal((5, 3))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    for (l1, l2, l3) in cg.paths(4):
        Y1, Y2, Y3 = (sh.real_sh(l, u) for l in (l1, l2, l3))
        got = np.einsum("xyz,ex,ey->ez", cg.real_cg(l1, l2, l3), Y1, Y2)
        g = math.sqrt((2 * l1 + 1) * (2 * l2 + 1) / (4 * math.pi * (2 * l3 + 1))) * cg.cg_complex(l1, 0, l2, 0, l3, 0)
        assert np.max(np.abs(got - g * Y3)) < 1e-13, (l1, l2, l3)


def test_scalar_path_is_identity():
    for l in range(5):
        C = cg.real_cg(l, 0, l)
        assert np.allclose(C[:, 0, :], np.eye(2 * l + 1), atol=1e-14)


def test_vector_cross_product_path():
    """l1 = l2 = l3 = 1 couples two vectors into their cross product (real
    l = 1 harmonics are (y, z, x)): (a (x) b)^1 = s / sqrt(2) (a x b), with one
    sign s for every a, b."""
    rng = np.random.default_rng(3)
    signs = set()
    for _ in range(4):
        a3, b3 = rng.standard_normal(3), rng.standard_normal(3)
        a = np.empty(3); b = np.empty(3)
        a[[0, 1, 2]] = a3[[1, 2, 0]]
        b[[0, 1, 2]] = b3[[1, 2, 0]]
        got = cg.tensor_product(a[:, None], b, 1, 1, 1)[:, 0]
        cr = np.cross(a3, b3)
        ref = np.array([cr[1], cr[2], cr[0]]) / math.sqrt(2.0)
        s = 1.0 if np.dot(got, ref) > 0 else -1.0
        signs.add(s)
        assert np.max(np.abs(got - s * ref)) < 1e-14
    assert len(signs) == 1


def _cluster(L=2, C=4, seed=5):
    wl = wlmod.make_workload(0, L=L, C=C, H=1)
    W = wlmod.make_cg_weights(L, C, seed)
    row_ptr, col = nb.neighbors(wl.pos, wl.box, wl.r_c)[:2]
    return wl, W, row_ptr, col


def test_conv_scalar_only_closed_form():
    """L = 0: o_i = sum_j u(r_ij) W x_j / sqrt(4 pi)."""
    wl, W, rp, col = _cluster(L=0, C=3)
    out = cg.cg_conv(wl.pos, wl.box, wl.r_c, rp, col, wl.x, W, 0)
    for i in range(wl.N):
        ref = np.zeros(3)
        for e in range(rp[i], rp[i + 1]):
            j = col[e]
            r = np.linalg.norm(wl.pos[j].astype(np.float64) - wl.pos[i])
            u = 0.5 * (math.cos(math.pi * r / wl.r_c) + 1.0)
            ref += u * W[0].astype(np.float64) * wl.x[j, 0].astype(np.float64) / math.sqrt(4 * math.pi)
        assert np.allclose(out[i, 0], ref, rtol=1e-12, atol=1e-14)


def test_conv_equivariant_and_translation_invariant():
    wl, W, rp, col = _cluster(L=3, C=2)
    out = cg.cg_conv(wl.pos, wl.box, wl.r_c, rp, col, wl.x, W, 3)
    Q = _rand_rot(np.random.default_rng(9))
    D = [sh.wigner_d_euler(l, Q) for l in range(4)]
    pos2 = wl.pos.astype(np.float64) @ Q.T + np.array([1.5, -2.0, 0.25])
    x2 = np.empty_like(wl.x, dtype=np.float64)
    orot = np.empty_like(out)
    for l in range(4):
        s_ = slice(l * l, (l + 1) ** 2)
        x2[:, s_, :] = np.einsum("ab,nbc->nac", D[l], wl.x[:, s_, :].astype(np.float64))
        orot[:, s_, :] = np.einsum("ab,nbc->nac", D[l], out[:, s_, :])
    out2 = cg.cg_conv(pos2, None, wl.r_c, rp, col, x2, W, 3)
    assert np.max(np.abs(out2 - orot)) < 1e-12 * max(1.0, np.max(np.abs(out)))


def test_conv_node_subset_matches_full():
    wl, W, rp, col = _cluster(L=2, C=3)
    full = cg.cg_conv(wl.pos, wl.box, wl.r_c, rp, col, wl.x, W, 2)
    nodes = np.array([0, 5, 7, 23])
    sub = cg.cg_conv(wl.pos, wl.box, wl.r_c, rp, col, wl.x, W, 2, nodes=nodes)
    assert np.array_equal(sub, full[nodes])
