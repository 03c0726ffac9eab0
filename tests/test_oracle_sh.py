"""Pins of the oracle's real spherical harmonics and Wigner-D matrices.

Each test checks the oracle against something other than itself: textbook
closed forms, group properties, or the second independent construction.
"""
import math

import numpy as np
import pytest

from atomistic_mlip_b200.workloads import haar_rotation
from oracle import sh

RNG = np.random.default_rng(2024)


def _units(n):
    u = RNG.standard_normal((n, 3))
    return u / np.linalg.norm(u, axis=1, keepdims=True)


def test_real_sh_textbook_l_le_2():
    """Standard table of real harmonics (no Condon-Shortley phase) for l <= 2."""
    u = _units(50)
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    pi = math.pi
    exp = {
        (0, 0): np.full_like(x, 0.5 * math.sqrt(1 / pi)),
        (1, -1): math.sqrt(3 / (4 * pi)) * y,
        (1, 0): math.sqrt(3 / (4 * pi)) * z,
        (1, 1): math.sqrt(3 / (4 * pi)) * x,
        (2, -2): 0.5 * math.sqrt(15 / pi) * x * y,
        (2, -1): 0.5 * math.sqrt(15 / pi) * y * z,
        (2, 0): 0.25 * math.sqrt(5 / pi) * (3 * z * z - 1),
        (2, 1): 0.5 * math.sqrt(15 / pi) * x * z,
        (2, 2): 0.25 * math.sqrt(15 / pi) * (x * x - y * y),
    }
    for (l, m), v in exp.items():
        np.testing.assert_allclose(sh.real_sh(l, u)[:, l + m], v, atol=1e-14)


@pytest.mark.parametrize("L", [6])
def test_real_sh_orthonormal(L):
    """<Y_lm, Y_l'm'> = delta by Gauss-Legendre x uniform-phi quadrature
    (exact for these band-limited products)."""
    nt, nphi = 2 * L + 2, 4 * L + 4
    xg, wg = np.polynomial.legendre.leggauss(nt)
    phi = 2 * np.pi * np.arange(nphi) / nphi
    ct = np.repeat(xg, nphi)
    st = np.sqrt(1 - ct ** 2)
    ph = np.tile(phi, nt)
    u = np.stack([st * np.cos(ph), st * np.sin(ph), ct], 1)
    w = np.repeat(wg, nphi) * (2 * np.pi / nphi)
    Y = sh.real_sh_all(L, u)
    G = (Y * w[:, None]).T @ Y
    np.testing.assert_allclose(G, np.eye((L + 1) ** 2), atol=1e-12)


@pytest.mark.parametrize("l", range(7))
def test_wigner_orthogonal_and_fit_equals_euler(l):
    """P1: D D^T = I.  P5: fit construction == Euler/small-d construction."""
    for _ in range(4):
        R = haar_rotation(RNG)
        A = sh.wigner_d_fit(l, R)
        B = sh.wigner_d_euler(l, R)
        np.testing.assert_allclose(A @ A.T, np.eye(2 * l + 1), atol=1e-13)
        np.testing.assert_allclose(A, B, atol=1e-12)


def test_wigner_l1_is_rotation_in_yzx_order():
    """P2: D^1(R) = Pi R Pi^T with Pi: (x, y, z) -> (y, z, x)."""
    perm = [1, 2, 0]
    for _ in range(5):
        R = haar_rotation(RNG)
        np.testing.assert_allclose(sh.wigner_d_fit(1, R), R[perm][:, perm], atol=1e-13)
        np.testing.assert_allclose(sh.wigner_d_euler(1, R), R[perm][:, perm], atol=1e-13)


@pytest.mark.parametrize("l", [2, 4, 6])
def test_wigner_homomorphism(l):
    """P3: D(R1 R2) = D(R1) D(R2)."""
    R1, R2 = haar_rotation(RNG), haar_rotation(RNG)
    np.testing.assert_allclose(sh.wigner_d_fit(l, R1 @ R2),
                               sh.wigner_d_fit(l, R1) @ sh.wigner_d_fit(l, R2), atol=1e-12)


def test_small_d_textbook_l1():
    """Sakurai's table of d^1(beta), rows/cols m = -1, 0, 1."""
    b = 0.7
    c, s = math.cos(b), math.sin(b)
    exp = np.array([[(1 + c) / 2, s / math.sqrt(2), (1 - c) / 2],
                    [-s / math.sqrt(2), c, s / math.sqrt(2)],
                    [(1 - c) / 2, -s / math.sqrt(2), (1 + c) / 2]])
    np.testing.assert_allclose(sh.small_d(1, b), exp, atol=1e-15)


def test_d_z_matches_azimuth_shift():
    """D of Rz(a) acting on Y equals Y at the azimuth-shifted points."""
    a = 0.37
    u = _units(20)
    for l in range(5):
        Ru = u @ sh.rot_z(a).T
        np.testing.assert_allclose(sh.real_sh(l, Ru), sh.real_sh(l, u) @ sh.d_z(l, a).T, atol=1e-13)


@pytest.mark.parametrize("L", [2, 4, 6])
def test_lemma_axis_aligned_sparsity(L):
    """P4 (E2Former-V2 summary §2.1, Lemma 4.1): in the edge frame the
    harmonics of the edge direction vanish except at m = 0, and the m = 0
    row of D^l(R_ij) is sqrt(4 pi / (2l+1)) Y_l(rhat), whatever the gauge."""
    u = _units(30)
    R = sh.edge_frame(u)
    np.testing.assert_allclose(np.einsum("eab,eb->ea", R, u), np.tile([0, 0, 1.0], (30, 1)), atol=1e-14)
    for l in range(L + 1):
        D = sh.wigner_d_fit(l, R)
        y = np.einsum("eab,eb->ea", D, sh.real_sh(l, u))
        mask = np.ones(2 * l + 1, bool)
        mask[l] = False
        if l > 0:
            assert np.max(np.abs(y[:, mask])) <= 1e-13
        np.testing.assert_allclose(y[:, l], math.sqrt((2 * l + 1) / (4 * math.pi)), atol=1e-13)
        np.testing.assert_allclose(D[:, l, :], math.sqrt(4 * math.pi / (2 * l + 1)) * sh.real_sh(l, u),
                                   atol=1e-13)
        # gauge freedom: an extra z-rotation leaves the m = 0 row unchanged
        Dg = sh.wigner_d_fit(l, sh.rot_z(1.1)[None] @ R)
        np.testing.assert_allclose(Dg[:, l, :], D[:, l, :], atol=1e-13)


def test_edge_frame_poles():
    """rhat = +z -> identity; rhat = -z -> rotation by pi about x."""
    R = sh.edge_frame(np.array([[0, 0, 1.0], [0, 0, -1.0]]))
    np.testing.assert_allclose(R[0], np.eye(3))
    np.testing.assert_allclose(R[1], np.diag([1.0, -1.0, -1.0]), atol=1e-15)


def test_edge_frame_is_minimal_rotation():
    """The frame rotates about rhat x z by exactly the angle between rhat and z."""
    u = _units(10)
    R = sh.edge_frame(u)
    for e in range(10):
        ang = math.acos(np.clip((np.trace(R[e]) - 1) / 2, -1, 1))
        np.testing.assert_allclose(ang, math.acos(u[e, 2]), atol=1e-12)
        axis = np.cross(u[e], [0, 0, 1.0])
        np.testing.assert_allclose(R[e] @ axis, axis, atol=1e-13)
        np.testing.assert_allclose(np.linalg.det(R[e]), 1.0, atol=1e-13)
