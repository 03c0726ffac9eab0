"""Gradients of the attention operator, fp64, through PyTorch CPU autograd.

Test infrastructure only (see the package docstring).

The backward of the path -- gradients of a scalar of the outputs with
respect to the features x, the weights and the atom positions, i.e.
conservative forces ("E2Former-V2 ..." summary §4, the conservative variant
timed at 100k atoms) -- is checked against this module.  It restates the
operator of ``oracle.attention`` (steps O2-O13 there, same conventions) in
plain PyTorch CPU ops so that autograd differentiates it:

  * real spherical harmonics as polynomials in (x, y, z): for a unit vector,
    P_l^m(z) cos(m phi) = Q_l^m(z) Re((x + i y)^m) with Q_l^m = P_l^m / (1 -
    z^2)^(m/2) a polynomial (no Condon-Shortley phase), so the harmonics and
    their derivatives are smooth at the poles;
  * D^l(R) by the same least-squares fit as ``oracle.sh.wigner_d_fit`` (the
    same sample points and pseudo-inverse, used as constants);
  * the minimal edge rotation (Rodrigues) written as R = I + A + A^2 / (1 + z)
    with A the cross-product matrix of rhat x z, equal to the oracle's form
    away from rhat = -z (where both are singular and tests keep away).

The forward is pinned to ``oracle.attention`` and the gradients to central
finite differences of it (``tests/test_oracle_grad.py``).  Small systems
only: everything is materialised edge by edge.
"""
from __future__ import annotations

import math
from typing import Dict, Optional

import numpy as np
import torch

from . import sh as osh
from .attention import N_RBF, RBF_SIGMA, pair_list

DT = torch.float64


def real_sh_t(l: int, u: torch.Tensor) -> torch.Tensor:
    """Real SH of degree l at unit vectors u [E, 3] -> [E, 2l+1] (torch, fp64),
    the convention of ``oracle.sh.real_sh``."""
    x, y, z = u[:, 0], u[:, 1], u[:, 2]
    out = [None] * (2 * l + 1)
    # Re / Im of (x + i y)^m, m = 0..l
    re, im = [torch.ones_like(x)], [torch.zeros_like(x)]
    for m in range(1, l + 1):
        re.append(re[-1] * x - im[-1] * y)
        im.append(re[-2] * y + im[-1] * x)
    for m in range(0, l + 1):
        # Q_l^m(z) by the three-term recursion in l, from Q_m^m = (2m-1)!!
        q_prev = torch.full_like(z, float(np.prod(np.arange(1, 2 * m, 2))) if m > 0 else 1.0)
        if l == m:
            q = q_prev
        else:
            q_cur = z * (2 * m + 1) * q_prev
            for ll in range(m + 2, l + 1):
                q_prev, q_cur = q_cur, ((2 * ll - 1) * z * q_cur - (ll + m - 1) * q_prev) / (ll - m)
            q = q_cur
        nlm = math.sqrt((2 * l + 1) / (4.0 * math.pi) * math.factorial(l - m) / math.factorial(l + m))
        if m == 0:
            out[l] = nlm * q
        else:
            out[l + m] = math.sqrt(2.0) * nlm * q * re[m]
            out[l - m] = math.sqrt(2.0) * nlm * q * im[m]
    return torch.stack(out, dim=-1)


def wigner_blocks_t(L: int, R: torch.Tensor):
    """[D^0, ..., D^L] of rotations R [E, 3, 3] by the oracle's least-squares fit."""
    blocks = []
    for l in range(L + 1):
        u, pinv = osh._fit_points(l)
        ut = torch.as_tensor(u, dtype=DT)
        ru = torch.einsum("eab,nb->ena", R, ut)                       # [E, n, 3]
        Yr = real_sh_t(l, ru.reshape(-1, 3)).reshape(R.shape[0], -1, 2 * l + 1)
        blocks.append(Yr.transpose(1, 2) @ torch.as_tensor(pinv, dtype=DT))
    return blocks


def edge_frame_t(rhat: torch.Tensor) -> torch.Tensor:
    """Minimal rotation with R rhat = +z, as R = I + A + A^2 / (1 + z)."""
    x, y, z = rhat[:, 0], rhat[:, 1], rhat[:, 2]
    zero = torch.zeros_like(x)
    # cross-product matrix of a = rhat x z = (y, -x, 0)
    A = torch.stack([torch.stack([zero, zero, -x], -1),
                     torch.stack([zero, zero, -y], -1),
                     torch.stack([x, y, zero], -1)], -2)
    eye = torch.eye(3, dtype=DT).expand_as(A)
    return eye + A + (A @ A) / (1.0 + z)[:, None, None]


def _project(x: torch.Tensor, W, L: int) -> torch.Tensor:
    parts = [x[:, l * l:(l + 1) * (l + 1), :] @ W[l].T for l in range(L + 1)]
    return torch.cat(parts, dim=1)


def _rotate(D, f: torch.Tensor, L: int, transpose: bool = False) -> torch.Tensor:
    parts = []
    for l in range(L + 1):
        Dl = D[l].transpose(1, 2) if transpose else D[l]
        parts.append(Dl @ f[:, l * l:(l + 1) * (l + 1), :])
    return torch.cat(parts, dim=1)


def _so2_mix(vt: torch.Tensor, g: torch.Tensor, L: int, C: int, W0, Wr, Wi) -> torch.Tensor:
    E = vt.shape[0]
    rows = {}
    def stack(m):
        return torch.cat([vt[:, osh.sh_index(l, m), :] for l in range(abs(m), L + 1)], dim=-1)
    def put(yv, m):
        for t, l in enumerate(range(abs(m), L + 1)):
            rows[osh.sh_index(l, m)] = yv[:, t * C:(t + 1) * C]
    put(stack(0) @ W0.T, 0)
    for m in range(1, L + 1):
        vp, vm = stack(m), stack(-m)
        put(vp @ Wr[m].T - vm @ Wi[m].T, m)
        put(vp @ Wi[m].T + vm @ Wr[m].T, -m)
    gi = {ml: p for p, ml in enumerate(pair_list(L))}
    for (m, l), p in gi.items():
        for mm in ((m, -m) if m else (0,)):
            rows[osh.sh_index(l, mm)] = rows[osh.sh_index(l, mm)] * g[:, p][:, None]
    return torch.stack([rows[k] for k in range((L + 1) ** 2)], dim=1).reshape(E, (L + 1) ** 2, C)


def forward_t(pos: torch.Tensor, box: Optional[np.ndarray], r_c: float, row_ptr: np.ndarray,
              col: np.ndarray, x: torch.Tensor, P: Dict[str, object], L: int, C: int, H: int,
              parts: Optional[dict] = None) -> torch.Tensor:
    """o [N, Q, C] of every node (steps O2-O13 of ``oracle.attention``), in torch.
    P holds the weights as fp64 tensors: Wq, Wk, Wv (lists by l), W0, Wr, Wi
    (lists by m, index 0 unused), rad_W1, rad_W2.  If `parts` is a dict it
    receives the per-edge logits "s" [E, H] (with their gradient retained),
    weights "alpha" [E, H] and global-frame messages "z" [E, Q, C]."""
    N = pos.shape[0]
    Q = (L + 1) ** 2
    Ch = C // H
    d = (L + 1) * Ch
    row_ptr = np.asarray(row_ptr, np.int64)
    col = np.asarray(col, np.int64)
    E = int(row_ptr[-1])
    dst = torch.as_tensor(np.repeat(np.arange(N), np.diff(row_ptr)), dtype=torch.long)
    src = torch.as_tensor(col[:E], dtype=torch.long)
    out = torch.zeros((N, Q, C), dtype=DT)
    if E == 0:
        return out
    # O2: minimum image with the oracle's > b/2 / < -b/2 rule
    rij = pos[src] - pos[dst]
    if box is not None:
        shift = []
        for k in range(3):
            b = float(box[k])
            dk = rij[:, k].detach()
            if b > 0:
                s = torch.where(dk > 0.5 * b, -b, 0.0) + torch.where(dk < -0.5 * b, b, 0.0)
            else:
                s = torch.zeros_like(dk)
            shift.append(s)
        rij = rij + torch.stack(shift, dim=-1).to(DT)
    r = torch.linalg.norm(rij, dim=1)
    rhat = rij / r[:, None]
    # O3, O5
    D = wigner_blocks_t(L, edge_frame_t(rhat))
    # O6, O7
    q = _project(x, P["Wq"], L)
    k = _project(x, P["Wk"], L)
    v = _project(x, P["Wv"], L)
    qt, kt, vt = _rotate(D, q[dst], L), _rotate(D, k[src], L), _rotate(D, v[src], L)
    # O8
    m0 = [osh.sh_index(l, 0) for l in range(L + 1)]
    s = (qt[:, m0, :] * kt[:, m0, :]).sum(dim=1).reshape(E, H, Ch).sum(dim=2) / math.sqrt(d)
    # O9
    mu = torch.arange(N_RBF, dtype=DT) * (r_c / (N_RBF - 1))
    phi = torch.exp(-((r[:, None] - mu) ** 2) / (2.0 * RBF_SIGMA ** 2))
    hdn = phi @ P["rad_W1"].T
    g = (hdn / (1.0 + torch.exp(-hdn))) @ P["rad_W2"].T
    # O10, O13 (message in the global frame)
    z = _rotate(D, _so2_mix(vt, g, L, C, P["W0"], P["Wr"], P["Wi"]), L, transpose=True)
    # O11, O12: two-pass softmax per destination and head
    u = 0.5 * (torch.cos(math.pi * r / r_c) + 1.0)
    if parts is not None:
        s.retain_grad()
        parts["s"], parts["z"], parts["alpha"] = s, z, []
    rows = []
    for i in range(N):
        a0, a1 = int(row_ptr[i]), int(row_ptr[i + 1])
        if a1 == a0:
            rows.append(torch.zeros((Q, C), dtype=DT))
            continue
        st = s[a0:a1]
        w = u[a0:a1, None] * torch.exp(st - st.max(dim=0, keepdim=True).values)
        alpha = w / w.sum(dim=0, keepdim=True)
        if parts is not None:
            parts["alpha"].append(alpha)
        a_c = alpha.repeat_interleave(Ch, dim=1)               # [k, C]
        rows.append(torch.einsum("kc,kqc->qc", a_c, z[a0:a1]))
    return torch.stack(rows, dim=0)


def params_t(wl, requires_grad: bool = False) -> Dict[str, object]:
    """The weights of a workload as fp64 tensors (lists kept as lists)."""
    def t(a):
        return torch.tensor(np.asarray(a, np.float64), dtype=DT, requires_grad=requires_grad)
    P = {"Wq": [t(w) for w in wl.Wq], "Wk": [t(w) for w in wl.Wk], "Wv": [t(w) for w in wl.Wv],
         "W0": t(wl.W0),
         "Wr": [None] + [t(w) for w in wl.Wr[1:]], "Wi": [None] + [t(w) for w in wl.Wi[1:]],
         "rad_W1": t(wl.rad_W1), "rad_W2": t(wl.rad_W2)}
    return P


def gradients(wl, csr, G: np.ndarray, pos: Optional[np.ndarray] = None, x: Optional[np.ndarray] = None):
    """Gradients of sum(G * o) with respect to positions, features and weights.

    Returns a dict of fp64 arrays: "pos" [N, 3], "x" [N, Q, C], "W0", "rad_W1",
    "rad_W2" and the per-degree lists "Wq", "Wk", "Wv", "Wr", "Wi"."""
    row_ptr, col = csr
    pos_t = torch.tensor(np.asarray(wl.pos if pos is None else pos, np.float64), dtype=DT, requires_grad=True)
    x_t = torch.tensor(np.asarray(wl.x if x is None else x, np.float64), dtype=DT, requires_grad=True)
    P = params_t(wl, requires_grad=True)
    o = forward_t(pos_t, wl.box, wl.r_c, row_ptr, col, x_t, P, wl.L, wl.C, wl.H)
    (o * torch.as_tensor(np.asarray(G, np.float64))).sum().backward()
    def gnp(v):
        return None if v is None else (np.zeros(tuple(v.shape)) if v.grad is None else v.grad.numpy().copy())
    out = {"pos": gnp(pos_t), "x": gnp(x_t), "W0": gnp(P["W0"]),
           "rad_W1": gnp(P["rad_W1"]), "rad_W2": gnp(P["rad_W2"])}
    for key in ("Wq", "Wk", "Wv", "Wr", "Wi"):
        out[key] = [gnp(v) for v in P[key]]
    return out


def logit_gradient(wl, csr, G: np.ndarray):
    """d sum(G o) / d s [E, H] two ways: autograd, and the recompute form a
    backward kernel uses, alpha (<G_i, z_e>_h - Delta_ih) with
    Delta_ih = <G_i, o_i>_h (sums over the channels of head h)."""
    row_ptr, col = csr
    parts: dict = {}
    P = params_t(wl, requires_grad=True)
    o = forward_t(torch.tensor(np.asarray(wl.pos, np.float64), dtype=DT), wl.box, wl.r_c, row_ptr, col,
                  torch.tensor(np.asarray(wl.x, np.float64), dtype=DT), P, wl.L, wl.C, wl.H, parts=parts)
    Gt = torch.as_tensor(np.asarray(G, np.float64))
    (o * Gt).sum().backward()
    auto = parts["s"].grad.numpy().copy()
    Ch = wl.C // wl.H
    alpha = torch.cat(parts["alpha"], dim=0).detach().numpy()
    z = parts["z"].detach().numpy()
    on = o.detach().numpy()
    rp = np.asarray(row_ptr, np.int64)
    dst = np.repeat(np.arange(wl.N), np.diff(rp))
    Gn = np.asarray(G, np.float64)
    gz = np.einsum("eqc,eqc->ec", Gn[dst], z).reshape(-1, wl.H, Ch).sum(axis=2)      # [E, H]
    delta = np.einsum("iqc,iqc->ic", Gn, on).reshape(-1, wl.H, Ch).sum(axis=2)       # [N, H]
    formula = alpha * (gz - delta[dst])
    return auto, formula
