"""Real spherical harmonics and real Wigner-D matrices, fp64.

Test infrastructure only (see the package docstring).

Convention (the plainest standard one; the pages fix only that the frame
rotation makes the harmonics of the edge direction axis-aligned, E2Former-V2
summary §2.1, "Lemma 4.1"):

  * index (l, m) -> l*l + l + m, m = -l..l;
  * Y_l^0 = N_l0 P_l(cos t); Y_l^m = sqrt(2) N_lm P_l^m(cos t) cos(m p) for
    m > 0 and sqrt(2) N_l|m| P_l^|m|(cos t) sin(|m| p) for m < 0, with P_l^m
    WITHOUT the Condon-Shortley phase and N_lm = sqrt((2l+1)/(4 pi) (l-m)!/(l+m)!);
    so l = 1 is (y, z, x) * sqrt(3 / (4 pi));
  * D^l(R) is the matrix with Y_l(R u) = D^l(R) Y_l(u) for every unit u.

D^l is built two independent ways:
  (i)  ``wigner_d_fit``: least squares on random unit vectors,
       D = Y(R U) pinv(Y(U));
  (ii) ``wigner_d_euler``: z-y-z Euler angles, D_z(a) D_y(b) D_z(g), with
       D_y(b) from Wigner's explicit small-d sum conjugated by the unitary
       between complex (Condon-Shortley) and real harmonics.
"""
from __future__ import annotations

import math
from functools import lru_cache

import numpy as np
from scipy.special import lpmv


def sh_index(l: int, m: int) -> int:
    return l * l + l + m


def real_sh(l: int, u: np.ndarray) -> np.ndarray:
    """Real SH of degree l at unit vectors u [..., 3] -> [..., 2l+1] (fp64)."""
    u = np.asarray(u, dtype=np.float64)
    x, y, z = u[..., 0], u[..., 1], u[..., 2]
    ct = np.clip(z, -1.0, 1.0)
    phi = np.arctan2(y, x)
    out = np.empty(u.shape[:-1] + (2 * l + 1,), dtype=np.float64)
    for m in range(0, l + 1):
        # scipy's lpmv carries the Condon-Shortley phase (-1)^m; remove it.
        plm = ((-1.0) ** m) * lpmv(m, l, ct)
        nlm = math.sqrt((2 * l + 1) / (4.0 * math.pi)
                        * math.factorial(l - m) / math.factorial(l + m))
        if m == 0:
            out[..., l] = nlm * plm
        else:
            out[..., l + m] = math.sqrt(2.0) * nlm * plm * np.cos(m * phi)
            out[..., l - m] = math.sqrt(2.0) * nlm * plm * np.sin(m * phi)
    return out


def real_sh_all(L: int, u: np.ndarray) -> np.ndarray:
    """Concatenated real SH for l = 0..L -> [..., (L+1)^2]."""
    return np.concatenate([real_sh(l, u) for l in range(L + 1)], axis=-1)


# ---------------------------------------------------------------------------
# (i) least-squares fit
# ---------------------------------------------------------------------------
@lru_cache(maxsize=None)
def _fit_points(l: int):
    rng = np.random.default_rng(1000 + l)
    n = 4 * (2 * l + 1)
    u = rng.standard_normal((n, 3))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    Y = real_sh(l, u).T                       # [2l+1, n]
    return u, np.linalg.pinv(Y)               # pinv: [n, 2l+1]


def wigner_d_fit(l: int, R: np.ndarray) -> np.ndarray:
    """D^l(R) by least squares; R [..., 3, 3] -> [..., 2l+1, 2l+1]."""
    R = np.asarray(R, dtype=np.float64)
    u, pinv = _fit_points(l)
    ru = np.einsum("...ab,nb->...na", R, u)   # rotated points
    Yr = np.swapaxes(real_sh(l, ru), -1, -2)  # [..., 2l+1, n]
    return Yr @ pinv


# ---------------------------------------------------------------------------
# (ii) Euler angles + Wigner small-d
# ---------------------------------------------------------------------------
def rot_z(a: float) -> np.ndarray:
    c, s = math.cos(a), math.sin(a)
    return np.array([[c, -s, 0.0], [s, c, 0.0], [0.0, 0.0, 1.0]])


def rot_y(b: float) -> np.ndarray:
    c, s = math.cos(b), math.sin(b)
    return np.array([[c, 0.0, s], [0.0, 1.0, 0.0], [-s, 0.0, c]])


def rot_x(a: float) -> np.ndarray:
    c, s = math.cos(a), math.sin(a)
    return np.array([[1.0, 0.0, 0.0], [0.0, c, -s], [0.0, s, c]])


def euler_zyz(R: np.ndarray):
    """(a, b, g) with R = Rz(a) Ry(b) Rz(g)."""
    b = math.acos(max(-1.0, min(1.0, R[2, 2])))
    if abs(math.sin(b)) < 1e-12:
        g = 0.0
        if R[2, 2] > 0:
            a = math.atan2(R[1, 0], R[0, 0])
        else:
            a = math.atan2(-R[1, 0], -R[0, 0])
        return a, b, g
    a = math.atan2(R[1, 2], R[0, 2])
    g = math.atan2(R[2, 1], -R[2, 0])
    return a, b, g


def small_d(l: int, beta: float) -> np.ndarray:
    """Wigner's small-d matrix d^l_{m'm}(beta) (Sakurai's convention),
    rows m' = -l..l, columns m = -l..l, from the explicit sum formula."""
    f = math.factorial
    c, s = math.cos(beta / 2.0), math.sin(beta / 2.0)
    d = np.zeros((2 * l + 1, 2 * l + 1))
    for mp in range(-l, l + 1):
        for m in range(-l, l + 1):
            pref = math.sqrt(f(l + m) * f(l - m) * f(l + mp) * f(l - mp))
            acc = 0.0
            for k in range(0, 2 * l + 1):
                a1, a2, a3 = l + m - k, l - k - mp, k - m + mp
                if a1 < 0 or a2 < 0 or a3 < 0:
                    continue
                acc += ((-1.0) ** (k - m + mp) * pref / (f(a1) * f(k) * f(a2) * f(a3))
                        * c ** (2 * l - 2 * k + m - mp) * s ** (2 * k - m + mp))
            d[mp + l, m + l] = acc
    return d


def complex_to_real(l: int) -> np.ndarray:
    """Unitary U with Y_real = U Y_complex (complex Y with Condon-Shortley)."""
    U = np.zeros((2 * l + 1, 2 * l + 1), dtype=np.complex128)
    r2 = 1.0 / math.sqrt(2.0)
    U[l, l] = 1.0
    for m in range(1, l + 1):
        sgn = (-1.0) ** m
        U[l + m, l + m] = sgn * r2
        U[l + m, l - m] = r2
        U[l - m, l - m] = 1j * r2
        U[l - m, l + m] = -1j * sgn * r2
    return U


def d_z(l: int, a: float) -> np.ndarray:
    """Real-basis D^l of Rz(a): on each (+m, -m) pair
    [[cos m a, -sin m a], [sin m a, cos m a]], 1 at m = 0."""
    D = np.zeros((2 * l + 1, 2 * l + 1))
    D[l, l] = 1.0
    for m in range(1, l + 1):
        c, s = math.cos(m * a), math.sin(m * a)
        D[l + m, l + m] = c
        D[l + m, l - m] = -s
        D[l - m, l + m] = s
        D[l - m, l - m] = c
    return D


def d_y(l: int, b: float) -> np.ndarray:
    """Real-basis D^l of Ry(b) = U conj(d^l(b)) U^dagger."""
    U = complex_to_real(l)
    Dc = np.conj(small_d(l, b))
    D = U @ Dc @ U.conj().T
    assert np.max(np.abs(D.imag)) < 1e-12
    return D.real


def wigner_d_euler(l: int, R: np.ndarray) -> np.ndarray:
    """D^l(R) through z-y-z Euler angles; R [3, 3] -> [2l+1, 2l+1]."""
    a, b, g = euler_zyz(np.asarray(R, dtype=np.float64))
    return d_z(l, a) @ d_y(l, b) @ d_z(l, g)


def wigner_d_blocks(L: int, R: np.ndarray):
    """[D^0(R), ..., D^L(R)] for a batch R [..., 3, 3] (fit construction)."""
    return [wigner_d_fit(l, R) for l in range(L + 1)]


# ---------------------------------------------------------------------------
# Edge frame
# ---------------------------------------------------------------------------
def edge_frame(rhat: np.ndarray) -> np.ndarray:
    """Minimal rotation R with R rhat = +z: rotation about rhat x z by the
    angle between them (Rodrigues); identity at rhat = +z and a rotation by
    pi about x at rhat = -z.  rhat [..., 3] -> [..., 3, 3]."""
    rhat = np.asarray(rhat, dtype=np.float64)
    out = np.empty(rhat.shape[:-1] + (3, 3))
    flat_r = rhat.reshape(-1, 3)
    flat_o = out.reshape(-1, 3, 3)
    for e in range(flat_r.shape[0]):
        x, y, z = flat_r[e]
        axis = np.array([y, -x, 0.0])          # rhat x z
        s = float(np.linalg.norm(axis))
        if s == 0.0:
            flat_o[e] = np.eye(3) if z > 0 else rot_x(math.pi)
            continue
        k = axis / s
        K = np.array([[0.0, -k[2], k[1]], [k[2], 0.0, -k[0]], [-k[1], k[0], 0.0]])
        c = z
        flat_o[e] = np.eye(3) + s * K + (1.0 - c) * (K @ K)
    return out
