"""Clebsch-Gordan coupling and the x (x) Y(rhat) convolution, dense, fp64.

Test infrastructure only (see the package docstring).

What it computes.  "E2Former-V2 ..." summary §2.1 ("Axis-aligned
equivariant sparsification (EAAS)", "Re-indexing operator"): a standard
SO(3) tensor contraction is a dense sum over Clebsch-Gordan coefficients;
EAAS rotates into the edge-aligned frame, where the harmonics of the edge
direction have only their m = 0 component (Lemma 4.1), so the contraction
collapses into a block-sparse re-indexing.  This module is the DENSE side
only -- the plain definition, in the global frame, with no rotation:

  G1  complex CG <l1 m1; l2 m2 | l3 m3> by the Racah formula, in exact
      rational arithmetic, then one square root;
  G2  real-basis coupling tensor (the real harmonics of oracle.sh, U the
      complex -> real unitary, Y_real = U Y_complex):
          K[m1, m2, m3] = sum_{M1 M2 M3} U3[m3, M3] CG[M1, M2, M3]
                                         conj(U1[m1, M1]) conj(U2[m2, M2]);
      K is real when l1 + l2 + l3 is even and purely imaginary when it is
      odd; the real tensor is C = Re K (even) or C = Im K (odd);
  G3  product (a (x) b)^{l3}_{m3} = sum_{m1, m2} C[m1, m2, m3] a_{m1} b_{m2};
  G4  paths: every (l1, l2, l3) with 0 <= l1, l2, l3 <= L and
      |l1 - l2| <= l3 <= l1 + l2, in lexicographic (l1, l2, l3) order;
  G5  convolution, per destination i and channel c:
          o_i[(l3, m3), c] = sum_{j in N(i)} u(r_ij)
              sum_{paths p = (l1, l2, l3)} W[p, c] (x_j^{l1}[., c] (x) Y^{l2}(rhat_ij))^{l3}_{m3}
      with r_ij = p_j - p_i (minimum image), Y the orthonormal real
      harmonics of oracle.sh, u the cosine envelope of oracle.attention.

Readings (the pages print neither Eq. 13 nor the weight structure): the
weights are one scalar per (path, channel) -- channel-wise ("depthwise")
path weights, the plainest learnable form of x (x) Y(rhat); the only radial
dependence is the envelope; the sign of the odd-parity real tensors is the
one G2 fixes.
"""
from __future__ import annotations

import math
from fractions import Fraction
from functools import lru_cache
from typing import List, Optional, Tuple

import numpy as np

from . import sh
from .attention import envelope
from .neighbors import min_image


# ---------------------------------------------------------------------------
# G1  complex Clebsch-Gordan coefficients (Racah formula)
# ---------------------------------------------------------------------------
def cg_complex(l1: int, m1: int, l2: int, m2: int, l3: int, m3: int) -> float:
    """<l1 m1; l2 m2 | l3 m3> (Condon-Shortley phase convention)."""
    if m1 + m2 != m3:
        return 0.0
    if not (abs(l1 - l2) <= l3 <= l1 + l2):
        return 0.0
    if abs(m1) > l1 or abs(m2) > l2 or abs(m3) > l3:
        return 0.0
    f = math.factorial
    # the squared prefactor, exact
    pre = Fraction((2 * l3 + 1) * f(l1 + l2 - l3) * f(l1 - l2 + l3) * f(-l1 + l2 + l3), f(l1 + l2 + l3 + 1))
    pre *= f(l1 + m1) * f(l1 - m1) * f(l2 + m2) * f(l2 - m2) * f(l3 + m3) * f(l3 - m3)
    s = Fraction(0)
    kmin = max(0, l2 - l3 - m1, l1 - l3 + m2)
    kmax = min(l1 + l2 - l3, l1 - m1, l2 + m2)
    for k in range(kmin, kmax + 1):
        den = (f(k) * f(l1 + l2 - l3 - k) * f(l1 - m1 - k) * f(l2 + m2 - k)
               * f(l3 - l2 + m1 + k) * f(l3 - l1 - m2 + k))
        s += Fraction((-1) ** k, den)
    if s == 0:
        return 0.0
    # sqrt(pre) * s = sign(s) sqrt(pre s^2), one rounding
    val = math.sqrt(float(pre * s * s))
    return val if s > 0 else -val


@lru_cache(maxsize=None)
def cg_complex_tensor(l1: int, l2: int, l3: int) -> np.ndarray:
    """[2l1+1, 2l2+1, 2l3+1], index m + l."""
    T = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
    for m1 in range(-l1, l1 + 1):
        for m2 in range(-l2, l2 + 1):
            m3 = m1 + m2
            if abs(m3) <= l3:
                T[m1 + l1, m2 + l2, m3 + l3] = cg_complex(l1, m1, l2, m2, l3, m3)
    return T


# ---------------------------------------------------------------------------
# G2  real coupling tensor
# ---------------------------------------------------------------------------
@lru_cache(maxsize=None)
def real_cg(l1: int, l2: int, l3: int) -> np.ndarray:
    """C[m1, m2, m3] (index m + l) in the real harmonics of oracle.sh."""
    U1, U2, U3 = sh.complex_to_real(l1), sh.complex_to_real(l2), sh.complex_to_real(l3)
    K = np.einsum("ZM,abM,xa,yb->xyZ", U3, cg_complex_tensor(l1, l2, l3), np.conj(U1), np.conj(U2))
    if (l1 + l2 + l3) % 2 == 0:
        assert np.max(np.abs(K.imag)) < 1e-12
        return np.ascontiguousarray(K.real)
    assert np.max(np.abs(K.real)) < 1e-12
    return np.ascontiguousarray(K.imag)


# ---------------------------------------------------------------------------
# G3, G4
# ---------------------------------------------------------------------------
def tensor_product(a: np.ndarray, b: np.ndarray, l1: int, l2: int, l3: int) -> np.ndarray:
    """(a (x) b)^{l3}: a [..., 2l1+1, C], b [..., 2l2+1] -> [..., 2l3+1, C]."""
    return np.einsum("xyz,...xc,...y->...zc", real_cg(l1, l2, l3), a, b)


def paths(L: int) -> List[Tuple[int, int, int]]:
    return [(l1, l2, l3) for l1 in range(L + 1) for l2 in range(L + 1) for l3 in range(L + 1)
            if abs(l1 - l2) <= l3 <= l1 + l2]


# ---------------------------------------------------------------------------
# G5  convolution
# ---------------------------------------------------------------------------
def cg_conv(pos: np.ndarray, box: Optional[np.ndarray], r_c: float, row_ptr: np.ndarray, col: np.ndarray,
            x: np.ndarray, W: np.ndarray, L: int, nodes: Optional[np.ndarray] = None,
            max_edges_per_chunk: int = 8192) -> np.ndarray:
    """o_i for i in `nodes` (default all) -> [len(nodes), (L+1)^2, C] fp64.

    x [N, (L+1)^2, C]; W [len(paths(L)), C]."""
    N = np.asarray(pos).shape[0]
    Q = (L + 1) ** 2
    x = np.asarray(x)
    C = x.shape[2]
    W = np.asarray(W, np.float64)
    P = paths(L)
    assert W.shape == (len(P), C)
    row_ptr = np.asarray(row_ptr, np.int64)
    col = np.asarray(col, np.int64)
    nodes = np.arange(N) if nodes is None else np.asarray(nodes, np.int64)
    out = np.zeros((len(nodes), Q, C))
    sl = [slice(l * l, (l + 1) * (l + 1)) for l in range(L + 1)]
    start = 0
    deg = row_ptr[nodes + 1] - row_ptr[nodes]
    while start < len(nodes):
        stop, tot = start, 0
        while stop < len(nodes) and (stop == start or tot + deg[stop] <= max_edges_per_chunk):
            tot += deg[stop]
            stop += 1
        dst, e_ids = [], []
        for t in range(start, stop):
            i = nodes[t]
            e = np.arange(row_ptr[i], row_ptr[i + 1])
            e_ids.append(e)
            dst.append(np.full(len(e), t))
        e_ids = np.concatenate(e_ids)
        if len(e_ids):
            dst = np.concatenate(dst)
            i_g, j_g = nodes[dst], col[e_ids]
            rij = min_image(pos, box, i_g, j_g)
            r = np.linalg.norm(rij, axis=1)
            rhat = np.where(r[:, None] > 0, rij / np.where(r > 0, r, 1.0)[:, None], np.array([0.0, 0.0, 1.0]))
            u = envelope(r, r_c)
            Y = [sh.real_sh(l, rhat) for l in range(L + 1)]                  # [E, 2l+1]
            xe = np.asarray(x[j_g], np.float64)                                # [E, Q, C]
            msg = np.zeros((len(e_ids), Q, C))
            for p, (l1, l2, l3) in enumerate(P):
                msg[:, sl[l3], :] += W[p][None, None, :] * tensor_product(xe[:, sl[l1], :], Y[l2], l1, l2, l3)
            msg *= u[:, None, None]
            np.add.at(out, dst, msg)
        start = stop
    return out
