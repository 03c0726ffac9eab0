"""The backward of the attention written out step by step, the way a tiled
kernel would compute it (recompute per edge, no autograd), in fp64 NumPy.

Test helper: ``tests/test_backward_plan.py`` checks every gradient it gives
against ``oracle.attention_grad`` (autograd of the plain definition).  What
it pins is the derivation a backward kernel follows:

  * the edge frame in the two-angle gauge R = Ry(-theta) Rz(-phi), which
    takes rhat to +z; D^l = d_y(-theta) d_z(-phi) (the output does not
    depend on the gauge, but the chain through D does);
  * the softmax backward per head, ds = alpha (<G_i, z_e>_h - Delta_ih);
  * the envelope enters like the logits (alpha ~ u exp(s)), so its gradient
    is sum_h exp(s - M)/den (dalpha - Delta) with no division by u;
  * the SO(2) block products backward: transposed blocks for the input, and
    outer products summed over edges for the weights;
  * dL/dD per degree from the three places D enters (rotate in, back
    rotation, the m = 0 rows in the logits), carried to the two angles by the
    rotation generators: d/db d_y(l, b) = d_y(l, b) J_y^l, d/da d_z(l, a) =
    d_z(l, a) J_z^l;
  * the angles and the radius carried to the edge vector, and from there to
    both atoms.
"""
from __future__ import annotations

import math
from functools import lru_cache

import numpy as np

from oracle import attention as oa
from oracle import sh
from oracle.neighbors import min_image


@lru_cache(maxsize=None)
def _gen_y(l: int) -> np.ndarray:
    """J_y^l = d/db d_y(l, b) at b = 0 (central difference of the exact
    small-d construction; d_y is entire in b, the error is O(eps^2))."""
    eps = 1e-5
    return (sh.d_y(l, eps) - sh.d_y(l, -eps)) / (2 * eps)


def _gen_z(l: int) -> np.ndarray:
    """J_z^l = d/da d_z(l, a) at a = 0: [[0, -m], [m, 0]] on each (+m, -m) pair."""
    J = np.zeros((2 * l + 1, 2 * l + 1))
    for m in range(1, l + 1):
        J[l + m, l - m] = -m
        J[l - m, l + m] = m
    return J


def backward(wl, csr, G):
    """Gradients of sum(G o): dict with "pos", "x", "Wq", "Wk", "Wv", "W0",
    "Wr", "Wi", "rad_W1", "rad_W2" (the layout of oracle.attention_grad)."""
    L, C, H = wl.L, wl.C, wl.H
    Q, Ch = (L + 1) ** 2, C // H
    d = (L + 1) * Ch
    N = wl.N
    row_ptr, col = (np.asarray(a, np.int64) for a in csr)
    E = int(row_ptr[-1])
    dst = np.repeat(np.arange(N), np.diff(row_ptr))
    src = col[:E]
    G = np.asarray(G, np.float64)
    x = np.asarray(wl.x, np.float64)
    Wq = [np.asarray(w, np.float64) for w in wl.Wq]
    Wk = [np.asarray(w, np.float64) for w in wl.Wk]
    Wv = [np.asarray(w, np.float64) for w in wl.Wv]
    W0 = np.asarray(wl.W0, np.float64)
    Wr = [None] + [np.asarray(w, np.float64) for w in wl.Wr[1:]]
    Wi = [None] + [np.asarray(w, np.float64) for w in wl.Wi[1:]]
    W1, W2 = np.asarray(wl.rad_W1, np.float64), np.asarray(wl.rad_W2, np.float64)
    blocks = [slice(l * l, (l + 1) ** 2) for l in range(L + 1)]

    # ---- forward recompute, per edge, in the two-angle gauge
    rij = min_image(np.asarray(wl.pos, np.float64), wl.box, dst, src)
    r = np.linalg.norm(rij, axis=1)
    rho = np.hypot(rij[:, 0], rij[:, 1])
    theta = np.arctan2(rho, rij[:, 2])
    phi = np.arctan2(rij[:, 1], rij[:, 0])
    Ay = [[sh.d_y(l, -t) for t in theta] for l in range(L + 1)]
    Bz = [[sh.d_z(l, -p) for p in phi] for l in range(L + 1)]
    D = [np.stack([Ay[l][e] @ Bz[l][e] for e in range(E)]) for l in range(L + 1)]
    q = oa.project(x, Wq, L)
    k = oa.project(x, Wk, L)
    v = oa.project(x, Wv, L)
    qt, kt, vt = oa.rotate(D, q[dst], L), oa.rotate(D, k[src], L), oa.rotate(D, v[src], L)
    m0 = [sh.sh_index(l, 0) for l in range(L + 1)]
    s = (qt[:, m0, :] * kt[:, m0, :]).sum(axis=1).reshape(E, H, Ch).sum(axis=2) / math.sqrt(d)
    mu = np.arange(oa.N_RBF) * (wl.r_c / (oa.N_RBF - 1))
    phi_r = np.exp(-((r[:, None] - mu) ** 2) / (2 * oa.RBF_SIGMA ** 2))
    hdn = phi_r @ W1.T
    sig = 1.0 / (1.0 + np.exp(-hdn))
    hid = hdn * sig
    g = hid @ W2.T
    wmix = oa.so2_mix(vt, np.ones_like(g), L, C, W0, Wr, Wi)     # SO(2) products, unscaled
    gi = {ml: p for p, ml in enumerate(oa.pair_list(L))}
    row_p = np.zeros(Q, np.int64)                                 # pair index of each row
    for (m, l), p in gi.items():
        for mm in ((m, -m) if m else (0,)):
            row_p[sh.sh_index(l, mm)] = p
    y = wmix * g[:, row_p][:, :, None]
    z = oa.rotate(D, y, L, transpose=True)
    u = 0.5 * (np.cos(math.pi * r / wl.r_c) + 1.0)
    M = np.full((N, H), -np.inf)
    np.maximum.at(M, dst, s)
    ex = np.exp(s - M[dst])                                       # e^(s - M)
    den = np.zeros((N, H))
    np.add.at(den, dst, u[:, None] * ex)
    alpha = u[:, None] * ex / den[dst]
    a_c = np.repeat(alpha, Ch, axis=1)
    o = np.zeros((N, Q, C))
    np.add.at(o, dst, a_c[:, None, :] * z)

    # ---- backward
    # softmax, per head
    dalpha = (G[dst] * z).sum(axis=1).reshape(E, H, Ch).sum(axis=2)
    delta = (G * o).sum(axis=1).reshape(N, H, Ch).sum(axis=2)
    ds = alpha * (dalpha - delta[dst])
    du = (ex / den[dst] * (dalpha - delta[dst])).sum(axis=1)     # d/du, no division by u
    # messages
    dz = a_c[:, None, :] * G[dst]
    dy = oa.rotate(D, dz, L)                                      # z = D^T y  ->  dy = D dz
    dg = np.zeros_like(g)
    np.add.at(dg.T, row_p, (dy * wmix).sum(axis=2).T)
    dw = dy * g[:, row_p][:, :, None]
    # SO(2) block products
    dvt = np.zeros_like(vt)
    dW0 = np.zeros_like(W0)
    dWr = [None] + [np.zeros_like(w) for w in Wr[1:]]
    dWi = [None] + [np.zeros_like(w) for w in Wi[1:]]
    v0, dw0 = oa.stack_m(vt, L, 0), oa.stack_m(dw, L, 0)
    oa.unstack_m(dw0 @ W0, dvt, L, 0, C)
    dW0 += dw0.T @ v0
    for m in range(1, L + 1):
        vp, vm = oa.stack_m(vt, L, m), oa.stack_m(vt, L, -m)
        dp, dmn = oa.stack_m(dw, L, m), oa.stack_m(dw, L, -m)
        oa.unstack_m(dp @ Wr[m] + dmn @ Wi[m], dvt, L, m, C)
        oa.unstack_m(-dp @ Wi[m] + dmn @ Wr[m], dvt, L, -m, C)
        dWr[m] += dp.T @ vp + dmn.T @ vm
        dWi[m] += -dp.T @ vm + dmn.T @ vp
    # logits (m = 0 rows of the rotated q, k)
    dsc = np.repeat(ds, Ch, axis=1) / math.sqrt(d)               # [E, C]
    dqt0 = dsc[:, None, :] * kt[:, m0, :]                         # [E, L+1, C]
    dkt0 = dsc[:, None, :] * qt[:, m0, :]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dD = [np.zeros_like(Dl) for Dl in D]
    for l in range(L + 1):
        b_ = blocks[l]
        Dl = D[l]
        row0 = Dl[:, l, :]                                        # m = 0 row, [E, 2l+1]
        dq_e = row0[:, :, None] * dqt0[:, l, None, :]             # D^T e_0 dqt0
        dk_e = row0[:, :, None] * dkt0[:, l, None, :]
        tmpq = np.zeros((N, 2 * l + 1, C))
        np.add.at(tmpq, dst, dq_e)
        dq[:, b_, :] += tmpq
        tmpk = np.zeros((N, 2 * l + 1, C))
        np.add.at(tmpk, src, dk_e)
        dk[:, b_, :] += tmpk
        tmpv = np.zeros((N, 2 * l + 1, C))
        np.add.at(tmpv, src, np.swapaxes(Dl, 1, 2) @ dvt[:, b_, :])
        dv[:, b_, :] += tmpv
        # dL/dD^l: rotate in, back rotation, logits (row 0)
        dD[l] += dvt[:, b_, :] @ np.swapaxes(v[src][:, b_, :], 1, 2)
        dD[l] += y[:, b_, :] @ np.swapaxes(dz[:, b_, :], 1, 2)
        dD[l][:, l, :] += (dqt0[:, l, None, :] * q[dst][:, b_, :]).sum(axis=2)
        dD[l][:, l, :] += (dkt0[:, l, None, :] * k[src][:, b_, :]).sum(axis=2)
    # D^l = d_y(-theta) d_z(-phi): d/dtheta = -d_y(-t) J_y d_z(-p), d/dphi = -d_y(-t) d_z(-p) J_z
    dtheta = np.zeros(E)
    dphi = np.zeros(E)
    for l in range(L + 1):
        Jy, Jz = _gen_y(l), _gen_z(l)
        for e in range(E):
            dtheta[e] -= np.sum(dD[l][e] * (Ay[l][e] @ Jy @ Bz[l][e]))
            dphi[e] -= np.sum(dD[l][e] * (Ay[l][e] @ Bz[l][e] @ Jz))
    # radius: radial MLP and envelope
    dhid = dg @ W2
    dW2 = dg.T @ hid
    dhdn = dhid * (sig * (1.0 + hdn * (1.0 - sig)))
    dW1 = dhdn.T @ phi_r
    dphi_r = dhdn @ W1
    dr = (dphi_r * phi_r * (-(r[:, None] - mu) / oa.RBF_SIGMA ** 2)).sum(axis=1)
    dr += du * (-0.5 * math.pi / wl.r_c) * np.sin(math.pi * r / wl.r_c)
    # to the edge vector: theta = atan2(rho, z), phi = atan2(y, x)
    xx, yy, zz = rij[:, 0], rij[:, 1], rij[:, 2]
    r2 = r * r
    drij = dr[:, None] * rij / r[:, None]
    drij[:, 0] += dtheta * xx * zz / (rho * r2) - dphi * yy / (rho * rho)
    drij[:, 1] += dtheta * yy * zz / (rho * r2) + dphi * xx / (rho * rho)
    drij[:, 2] += -dtheta * rho / r2
    dpos = np.zeros((N, 3))
    np.add.at(dpos, src, drij)
    np.add.at(dpos, dst, -drij)
    # projections
    dx = np.zeros_like(x)
    dWq, dWk, dWv = [], [], []
    for l in range(L + 1):
        b_ = blocks[l]
        dx[:, b_, :] += dq[:, b_, :] @ Wq[l] + dk[:, b_, :] @ Wk[l] + dv[:, b_, :] @ Wv[l]
        dWq.append(np.einsum("nmo,nmi->oi", dq[:, b_, :], x[:, b_, :]))
        dWk.append(np.einsum("nmo,nmi->oi", dk[:, b_, :], x[:, b_, :]))
        dWv.append(np.einsum("nmo,nmi->oi", dv[:, b_, :], x[:, b_, :]))
    return {"pos": dpos, "x": dx, "Wq": dWq, "Wk": dWk, "Wv": dWv, "W0": dW0, "Wr": dWr, "Wi": dWi,
            "rad_W1": dW1, "rad_W2": dW2, "o": o}
