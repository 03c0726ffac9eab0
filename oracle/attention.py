"""The on-the-fly equivariant attention operator, edge by edge, in fp64.

Test infrastructure only (see the package docstring).

What it computes (the method is exact: the streaming / online-softmax
kernel reaches the same value as this two-pass, fully materialised
evaluation up to rounding order -- "E2Former-V2 ..." summary §2.2, "Online
softmax" and "No edge materialisation"):

For every destination atom i and every neighbour j in N(i) (CSR row i):
  O2  r_ij = p_j - p_i (minimum image), r = |r_ij|, rhat = r_ij / r.
  O3  R_ij = minimal rotation with R_ij rhat = +z (SO(3) -> SO(2) change of
      basis, summary §2.1).
  O5  D_ij = blockdiag_l D^l(R_ij) (real Wigner-D, oracle.sh).
  O6  q, k, v = per-degree C x C linear maps of x (out x in, no bias); the
      pages call these projections "invariant scalar projections" (Eq. 6,
      not printed) -- invariance comes from using the edge-frame m = 0 rows.
  O7  qt = D_ij q_i, kt = D_ij k_j, vt = D_ij v_j.
  O8  s^h = (1/sqrt(d)) sum_l sum_{c in head h} qt[(l,0),c] kt[(l,0),c],
      d = (L+1) C_h  (the m = 0 rows are the only non-zero harmonics of the
      edge direction in this frame, "Lemma 4.1").
  O9  radial MLP: phi_k(r) = exp(-(r - mu_k)^2 / (2 sigma^2)), mu_k = k r_c / 7,
      sigma = 0.5, k = 0..7; h = SiLU(W1 phi); g = W2 h, g_{m,l} in
      lexicographic (m, l) order, m = 0..L, l = m..L.
  O10 SO(2) mix per m: stack vt[(l, +m), c] for l = m..L (l-major, then c)
      into v+ (length n_m = (L-m+1) C), likewise v-;
      m = 0: y0 = W0 v0;  m >= 1: y+ = Wr v+ - Wi v-,  y- = Wi v+ + Wr v-;
      then y[(l, +-m), c] *= g_{m,l}(r).
  O11 envelope u(r) = (cos(pi r / r_c) + 1) / 2 (EquiformerV3 summary §2B.3:
      the envelope enters numerator and denominator of the softmax).
  O12 alpha^h_ij = u_ij exp(s^h_ij) / sum_j' u_ij' exp(s^h_ij'), two-pass
      (max subtracted, then normalised).
  O13 o_i = sum_j alpha^{h(c)}_ij D_ij^T y_ij;  o_i = 0 when N(i) is empty.

Multi-focus variant ("DPA4 ...", §2.1 A2: the hidden channels split into F
focus streams, each with its own SO(2) stack, re-weighted by a cross-focus
softmax computed from the l = 0 section), optional (``focus=(F, a)``):
  F1  stream f owns channels [f C/F, (f+1) C/F); its SO(2) stack is the
      diagonal block of W0 / Wr / Wi between its own input and output
      channels (for every pair of degrees); cross-stream entries are dropped;
  F2  z^f_ij = (F / C)^(1/2) sum_{c in f} a_c y_ij[(0,0), c] (the l = 0 section
      of the edge message after the radial scale), beta_ij = softmax_f z_ij;
  F3  y_ij[., c] *= beta^{f(c)}_ij, then O13 as above.
Readings: the pages name neither the focus logits' form nor their source
beyond "the l = 0 section of the edge features"; the edge message's own
l = 0 section with one learned vector a (one weight per channel) is the
plainest choice that keeps the re-weighting invariant.
"""
from __future__ import annotations

import math
from typing import Callable, List, Optional, Sequence

import numpy as np

from . import sh
from .neighbors import min_image

N_RBF = 8
RBF_SIGMA = 0.5
N_HIDDEN = 16


# ---------------------------------------------------------------------------
# small pieces (each used by the tests on its own)
# ---------------------------------------------------------------------------
def pair_list(L: int):
    """(m, l) pairs of the radial output, m = 0..L then l = m..L."""
    return [(m, l) for m in range(L + 1) for l in range(m, L + 1)]


def radial_basis(r: np.ndarray, r_c: float) -> np.ndarray:
    mu = np.arange(N_RBF, dtype=np.float64) * (r_c / (N_RBF - 1))
    return np.exp(-((np.asarray(r, np.float64)[..., None] - mu) ** 2) / (2.0 * RBF_SIGMA ** 2))


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def radial_mlp(r: np.ndarray, r_c: float, W1: np.ndarray, W2: np.ndarray) -> np.ndarray:
    """g(r) -> [..., P]."""
    phi = radial_basis(r, r_c)
    h = silu(phi @ np.asarray(W1, np.float64).T)
    return h @ np.asarray(W2, np.float64).T


def envelope(r: np.ndarray, r_c: float) -> np.ndarray:
    return 0.5 * (np.cos(math.pi * np.asarray(r, np.float64) / r_c) + 1.0)


def project(x: np.ndarray, W: Sequence[np.ndarray], L: int) -> np.ndarray:
    """Per-degree linear map: out[n, (l,m), :] = W[l] @ x[n, (l,m), :]."""
    x = np.asarray(x, np.float64)
    out = np.empty_like(x)
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) * (l + 1))
        out[:, sl, :] = x[:, sl, :] @ np.asarray(W[l], np.float64).T
    return out


def rotate(D: List[np.ndarray], f: np.ndarray, L: int, transpose: bool = False) -> np.ndarray:
    """Apply blockdiag_l D^l (or its transpose) to f [E, Q, C]."""
    out = np.empty_like(f)
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) * (l + 1))
        Dl = np.swapaxes(D[l], -1, -2) if transpose else D[l]
        out[:, sl, :] = Dl @ f[:, sl, :]
    return out


def stack_m(f: np.ndarray, L: int, m: int) -> np.ndarray:
    """[E, Q, C] -> [E, n_m]: entries (l, m) for l = |m|..L, l-major then c."""
    parts = [f[:, sh.sh_index(l, m), :] for l in range(abs(m), L + 1)]
    return np.concatenate(parts, axis=-1)


def unstack_m(y: np.ndarray, out: np.ndarray, L: int, m: int, C: int) -> None:
    for t, l in enumerate(range(abs(m), L + 1)):
        out[:, sh.sh_index(l, m), :] = y[:, t * C:(t + 1) * C]


def so2_mix(vt: np.ndarray, g: np.ndarray, L: int, C: int, W0, Wr, Wi) -> np.ndarray:
    """O10 with the radial scale: vt [E, Q, C], g [E, P] -> y [E, Q, C]."""
    y = np.zeros_like(vt)
    gi = {ml: p for p, ml in enumerate(pair_list(L))}
    v0 = stack_m(vt, L, 0)
    unstack_m(v0 @ np.asarray(W0, np.float64).T, y, L, 0, C)
    for m in range(1, L + 1):
        vp, vm = stack_m(vt, L, m), stack_m(vt, L, -m)
        wr, wi = np.asarray(Wr[m], np.float64), np.asarray(Wi[m], np.float64)
        unstack_m(vp @ wr.T - vm @ wi.T, y, L, m, C)
        unstack_m(vp @ wi.T + vm @ wr.T, y, L, -m, C)
    for (m, l), p in gi.items():
        for mm in ((m, -m) if m else (0,)):
            y[:, sh.sh_index(l, mm), :] *= g[:, p][:, None]
    return y


def focus_mask(W: np.ndarray, C: int, F: int) -> np.ndarray:
    """F1: keep the entries of a stacked SO(2) matrix (rows and columns
    l-major, then channel) whose output and input channels share a stream."""
    W = np.asarray(W, np.float64)
    Cf = C // F
    fr = (np.arange(W.shape[0]) % C) // Cf
    fc = (np.arange(W.shape[1]) % C) // Cf
    return np.where(fr[:, None] == fc[None, :], W, 0.0)


def cross_focus(y: np.ndarray, F: int, a: np.ndarray) -> np.ndarray:
    """F2, F3: y [E, Q, C] -> y with each stream scaled by its softmax weight."""
    E, Q, C = y.shape
    Cf = C // F
    y00 = y[:, 0, :] * np.asarray(a, np.float64)[None, :]
    z = y00.reshape(E, F, Cf).sum(axis=2) / math.sqrt(Cf)
    z = z - z.max(axis=1, keepdims=True)
    beta = np.exp(z)
    beta /= beta.sum(axis=1, keepdims=True)
    return y * np.repeat(beta, Cf, axis=1)[:, None, :]


# ---------------------------------------------------------------------------
# the operator
# ---------------------------------------------------------------------------
def attention(pos: np.ndarray, box: Optional[np.ndarray], r_c: float,
              row_ptr: np.ndarray, col: np.ndarray,
              x: np.ndarray, Wq, Wk, Wv, W0, Wr, Wi, rad_W1, rad_W2,
              L: int, C: int, H: int,
              nodes: Optional[np.ndarray] = None,
              gauge: Optional[Callable[[np.ndarray], np.ndarray]] = None,
              g_override: Optional[float] = None,
              max_edges_per_chunk: int = 4096,
              focus: Optional[tuple] = None) -> np.ndarray:
    """o_i for i in `nodes` (default: all) -> [len(nodes), Q, C] fp64.

    `gauge(e_ids)` may return per-edge angles gamma (radians); the frame is
    then R_z(gamma) R_ij (test hook: the output must not change).
    `g_override` replaces the radial MLP output by a constant (test hook).
    `focus=(F, a)` selects the multi-focus variant (F1-F3)."""
    N = np.asarray(pos).shape[0]
    Q = (L + 1) ** 2
    Ch = C // H
    d = (L + 1) * Ch
    row_ptr = np.asarray(row_ptr, np.int64)
    col = np.asarray(col, np.int64)
    nodes = np.arange(N) if nodes is None else np.asarray(nodes, np.int64)
    out = np.zeros((len(nodes), Q, C))
    if len(nodes) == 0:
        return out

    # projections of the rows that are needed (q of destinations, k/v of sources)
    need_src = np.unique(np.concatenate([col[row_ptr[i]:row_ptr[i + 1]] for i in nodes]
                                        + [np.zeros(0, np.int64)]))
    # (only the rows used are widened to fp64; the widening is exact)
    x_src = np.asarray(np.asarray(x)[need_src], np.float64)
    q_rows = project(np.asarray(np.asarray(x)[nodes], np.float64), Wq, L)
    src_map = {int(j): t for t, j in enumerate(need_src)}
    k_rows = project(x_src, Wk, L) if len(need_src) else np.zeros((0, Q, C))
    v_rows = project(x_src, Wv, L) if len(need_src) else np.zeros((0, Q, C))

    if focus is not None:   # F1
        F = int(focus[0])
        W0 = focus_mask(W0, C, F)
        Wr = [None] + [focus_mask(Wr[m], C, F) for m in range(1, L + 1)]
        Wi = [None] + [focus_mask(Wi[m], C, F) for m in range(1, L + 1)]

    # chunks of destination nodes with a bounded number of edges
    deg = row_ptr[nodes + 1] - row_ptr[nodes]
    start = 0
    while start < len(nodes):
        stop, tot = start, 0
        while stop < len(nodes) and (stop == start or tot + deg[stop] <= max_edges_per_chunk):
            tot += deg[stop]
            stop += 1
        _chunk(out, start, stop, nodes, row_ptr, col, pos, box, r_c, q_rows, k_rows, v_rows,
               src_map, W0, Wr, Wi, rad_W1, rad_W2, L, C, H, Ch, d, gauge, g_override, focus)
        start = stop
    return out


def _chunk(out, start, stop, nodes, row_ptr, col, pos, box, r_c, q_rows, k_rows, v_rows,
           src_map, W0, Wr, Wi, rad_W1, rad_W2, L, C, H, Ch, d, gauge, g_override, focus=None):
    dst_local, e_ids = [], []
    for t in range(start, stop):
        i = nodes[t]
        e = np.arange(row_ptr[i], row_ptr[i + 1])
        e_ids.append(e)
        dst_local.append(np.full(len(e), t))
    e_ids = np.concatenate(e_ids)
    if len(e_ids) == 0:
        return
    dst_local = np.concatenate(dst_local)
    i_glob = nodes[dst_local]
    j_glob = col[e_ids]
    # O2
    rij = min_image(pos, box, i_glob, j_glob)
    r = np.linalg.norm(rij, axis=1)
    rhat = np.where(r[:, None] > 0, rij / np.where(r > 0, r, 1.0)[:, None], np.array([0.0, 0.0, 1.0]))
    # O3, O5
    R = sh.edge_frame(rhat)
    if gauge is not None:
        gam = np.asarray(gauge(e_ids), np.float64)
        Rz = np.zeros((len(gam), 3, 3))
        Rz[:, 0, 0] = np.cos(gam); Rz[:, 0, 1] = -np.sin(gam)
        Rz[:, 1, 0] = np.sin(gam); Rz[:, 1, 1] = np.cos(gam)
        Rz[:, 2, 2] = 1.0
        R = Rz @ R
    D = sh.wigner_d_blocks(L, R)
    # O7
    srcs = np.array([src_map[int(j)] for j in j_glob], dtype=np.int64)
    qt = rotate(D, q_rows[dst_local], L)
    kt = rotate(D, k_rows[srcs], L)
    vt = rotate(D, v_rows[srcs], L)
    # O8
    m0 = [sh.sh_index(l, 0) for l in range(L + 1)]
    prod = qt[:, m0, :] * kt[:, m0, :]                       # [E, L+1, C]
    s = prod.sum(axis=1).reshape(-1, H, Ch).sum(axis=2) / math.sqrt(d)   # [E, H]
    # O9
    if g_override is None:
        g = radial_mlp(r, r_c, rad_W1, rad_W2)
    else:
        g = np.full((len(r), (L + 1) * (L + 2) // 2), float(g_override))
    # O10
    y = so2_mix(vt, g, L, C, W0, Wr, Wi)
    if focus is not None:   # F2, F3
        y = cross_focus(y, int(focus[0]), focus[1])
    # O13 (per-edge message in the global frame)
    z = rotate(D, y, L, transpose=True)
    # O11, O12 (two-pass softmax per destination and head)
    u = envelope(r, r_c)
    for t in range(start, stop):
        sel = np.nonzero(dst_local == t)[0]
        if len(sel) == 0:
            continue
        st = s[sel]                                          # [k, H]
        smax = st.max(axis=0, keepdims=True)
        w = u[sel][:, None] * np.exp(st - smax)
        alpha = w / w.sum(axis=0, keepdims=True)             # [k, H]
        a_c = np.repeat(alpha, Ch, axis=1)                   # [k, C]
        out[t] = np.einsum("kc,kqc->qc", a_c, z[sel])


def attention_workload(wl, nodes=None, csr=None, **kw) -> np.ndarray:
    """Convenience wrapper for an atomistic_mlip_b200.workloads.Workload."""
    if csr is None:
        from .neighbors import neighbors
        csr = neighbors(wl.pos, wl.box, wl.r_c)
    row_ptr, col = csr
    return attention(wl.pos, wl.box, wl.r_c, row_ptr, col, wl.x, wl.Wq, wl.Wk, wl.Wv,
                     wl.W0, wl.Wr, wl.Wi, wl.rad_W1, wl.rad_W2, wl.L, wl.C, wl.H,
                     nodes=nodes, **kw)
