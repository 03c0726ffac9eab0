"""Pins of the multi-focus variant of the attention oracle (oracle/attention.py,
F1-F3): one stream is the plain operator; a zero focus vector weights every
stream 1/F, so F times the output equals the plain operator on block-diagonal
weights built here (which pins the stream masking); the re-weighting keeps
the output equivariant; and on a single edge the stream weights are the
softmax of the scaled l = 0 sums, computed here by hand."""
import math

import numpy as np

from atomistic_mlip_b200 import workloads as wlmod
from oracle import attention as oa
from oracle import neighbors as nb
from oracle import sh


def _wl(C=16, H=2, L=2, seed=3):
    return wlmod.make_workload(0, L=L, C=C, H=H, seed=seed)


def _run(wl, focus=None, W=None):
    rp, col = nb.neighbors(wl.pos, wl.box, wl.r_c)[:2]
    W0, Wr, Wi = (wl.W0, wl.Wr, wl.Wi) if W is None else W
    return oa.attention(wl.pos, wl.box, wl.r_c, rp, col, wl.x, wl.Wq, wl.Wk, wl.Wv, W0, Wr, Wi,
                        wl.rad_W1, wl.rad_W2, wl.L, wl.C, wl.H, focus=focus)


def _blockdiag(W, C, F):
    """Zero every entry whose output and input channels (index mod C) lie in
    different streams of C / F channels, by explicit loops."""
    W = np.array(W, np.float64)
    Cf = C // F
    for r in range(W.shape[0]):
        for c in range(W.shape[1]):
            if (r % C) // Cf != (c % C) // Cf:
                W[r, c] = 0.0
    return W


def test_single_stream_is_plain_operator():
    wl = _wl()
    a = np.random.default_rng(1).standard_normal(wl.C)
    assert np.array_equal(_run(wl, focus=(1, a)), _run(wl))


def test_zero_focus_vector_weights_streams_equally():
    wl = _wl()
    F = 4
    bd = (_blockdiag(wl.W0, wl.C, F), [None] + [_blockdiag(wl.Wr[m], wl.C, F) for m in range(1, wl.L + 1)],
          [None] + [_blockdiag(wl.Wi[m], wl.C, F) for m in range(1, wl.L + 1)])
    got = _run(wl, focus=(F, np.zeros(wl.C)))
    ref = _run(wl, W=bd)
    assert np.max(np.abs(F * got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_multifocus_equivariant():
    wl = _wl(L=3, C=8, H=2)
    F = 2
    a = np.random.default_rng(2).standard_normal(wl.C) * 3.0
    out = _run(wl, focus=(F, a))
    Q = wlmod.haar_rotation(np.random.default_rng(4))
    D = [sh.wigner_d_euler(l, Q) for l in range(wl.L + 1)]
    w2 = _wl(L=3, C=8, H=2)
    w2.pos = wl.pos.astype(np.float64) @ Q.T
    xr = np.empty_like(wl.x, dtype=np.float64)
    orot = np.empty_like(out)
    for l in range(wl.L + 1):
        s_ = slice(l * l, (l + 1) ** 2)
        xr[:, s_, :] = np.einsum("ab,nbc->nac", D[l], wl.x[:, s_, :].astype(np.float64))
        orot[:, s_, :] = np.einsum("ab,nbc->nac", D[l], out[:, s_, :])
    w2.x = xr
    assert np.max(np.abs(_run(w2, focus=(F, a)) - orot)) <= 1e-10 * np.max(np.abs(out))


def test_single_edge_stream_weights_by_hand():
    """Two atoms: node 0 has one neighbour, so alpha = 1 and o_0 = D^T (beta y)."""
    L, C, H, F = 2, 8, 2, 4
    pos = np.array([[0.0, 0.0, 0.0], [0.7, -1.1, 1.9]], np.float32)
    wl = wlmod.make_custom(pos, None, 4.0, L=L, C=C, H=H, precision="fp32", seed=11)
    a = np.random.default_rng(12).standard_normal(C)
    rp = np.array([0, 1, 2]); col = np.array([1, 0])
    got = oa.attention(wl.pos, None, wl.r_c, rp, col, wl.x, wl.Wq, wl.Wk, wl.Wv, wl.W0, wl.Wr, wl.Wi,
                       wl.rad_W1, wl.rad_W2, L, C, H, nodes=np.array([0]), focus=(F, a))[0]
    # the same edge through the oracle's pieces, stream weights by hand
    r = pos[1].astype(np.float64) - pos[0]
    R = sh.edge_frame((r / np.linalg.norm(r))[None])
    D = sh.wigner_d_blocks(L, R)
    v = oa.project(wl.x.astype(np.float64), wl.Wv, L)[1:2]
    vt = oa.rotate(D, v, L)
    g = oa.radial_mlp(np.array([np.linalg.norm(r)]), wl.r_c, wl.rad_W1, wl.rad_W2)
    W0 = oa.focus_mask(wl.W0, C, F)
    Wr = [None] + [oa.focus_mask(wl.Wr[m], C, F) for m in range(1, L + 1)]
    Wi = [None] + [oa.focus_mask(wl.Wi[m], C, F) for m in range(1, L + 1)]
    y = oa.so2_mix(vt, g, L, C, W0, Wr, Wi)[0]
    Cf = C // F
    z = [sum(a[c] * y[0, c] for c in range(f * Cf, (f + 1) * Cf)) / math.sqrt(Cf) for f in range(F)]
    ez = [math.exp(t - max(z)) for t in z]
    beta = [t / sum(ez) for t in ez]
    yb = y.copy()
    for c in range(C):
        yb[:, c] *= beta[c // Cf]
    ref = oa.rotate(D, yb[None], L, transpose=True)[0]
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))
