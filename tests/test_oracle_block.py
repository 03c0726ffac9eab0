"""Pins of the block oracle (oracle/block.py): the merged RMS norm, the
scalar-gated FFN and the pre-norm residual block, each against what the
mathematics fixes (library routine, closed forms, invariants, special
cases), not against a retyping of its own formula."""
import math

import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from oracle import attention as oa
from oracle import block as ob
from oracle import neighbors as nb
from oracle import sh


def _rotate_blocks(x, Q_rot, L):
    D = [sh.wigner_d_fit(l, Q_rot) for l in range(L + 1)]
    out = np.empty_like(x)
    for l in range(L + 1):
        s_ = slice(l * l, (l + 1) ** 2)
        out[:, s_, :] = D[l] @ x[:, s_, :]
    return out


def test_norm_equals_library_rms_norm():
    """The merged norm is torch's RMS norm over the node's flattened (l, m, c)
    entries with the gain of each entry's (degree, channel) -- for L = 0 the
    textbook RMSNorm over channels."""
    import torch
    rng = np.random.default_rng(1)
    for L, C in ((0, 16), (3, 8)):
        Q = (L + 1) ** 2
        x = rng.standard_normal((7, Q, C)) * rng.uniform(0.1, 10, (7, 1, 1))
        gamma = rng.uniform(0.5, 1.5, (L + 1, C))
        g_full = np.concatenate([np.repeat(gamma[l][None, :], 2 * l + 1, 0) for l in range(L + 1)]).reshape(-1)
        ref = torch.nn.functional.rms_norm(torch.from_numpy(x.reshape(7, Q * C)), (Q * C,),
                                           weight=torch.from_numpy(g_full), eps=ob.RMS_EPS).numpy()
        got = ob.merged_rms_norm(x, gamma, L).reshape(7, Q * C)
        assert np.max(np.abs(got - ref)) < 1e-12


def test_norm_closed_form_and_invariants():
    rng = np.random.default_rng(2)
    L, C = 2, 5
    x = rng.standard_normal((4, 9, C))
    y = ob.merged_rms_norm(x, np.ones((L + 1, C)), L)
    ms = np.mean(x * x, axis=(1, 2))
    # mean square of the output = ms / (ms + eps)
    assert np.allclose(np.mean(y * y, axis=(1, 2)), ms / (ms + ob.RMS_EPS), rtol=0, atol=1e-14)
    # scale invariance (eps = 0) and one statistic for all degrees: scaling
    # only the l = 2 block changes the l = 0 output
    assert np.allclose(ob.merged_rms_norm(3.7 * x, np.ones((L + 1, C)), L, eps=0.0),
                       ob.merged_rms_norm(x, np.ones((L + 1, C)), L, eps=0.0), atol=1e-14)
    x2 = x.copy()
    x2[:, 4:9, :] *= 5.0
    assert not np.allclose(ob.merged_rms_norm(x2, np.ones((L + 1, C)), L)[:, 0, :], y[:, 0, :])
    # equivariance: rotating every degree block commutes with the norm
    Qr = wlmod.haar_rotation(rng)
    g = rng.uniform(0.5, 1.5, (L + 1, C))
    assert np.max(np.abs(ob.merged_rms_norm(_rotate_blocks(x, Qr, L), g, L)
                         - _rotate_blocks(ob.merged_rms_norm(x, g, L), Qr, L))) < 1e-12


def test_silu_values():
    assert ob.silu(np.array(0.0)) == 0.0
    assert abs(ob.silu(np.array(1.0)) - 0.7310585786300049) < 1e-15   # 1 / (1 + e^-1)
    assert abs(ob.silu(np.array(-40.0))) < 1e-15 and abs(ob.silu(np.array(40.0)) - 40.0) < 1e-15


def test_ffn_hand_computed_example():
    """C = 1, Hd = 1, L = 1: out_(0,0) = d silu(a x0) b x0, out_(1,m) = d silu(a x0) b x_(1,m);
    with a = 0.5, b = 3, d = 0.25, x0 = 2: silu(1) 3 2 0.25 = 1.0965878679450074."""
    x = np.array([[[2.0], [1.0], [-2.0], [0.5]]])
    out = ob.ffn(x, np.array([[0.5]]), [np.array([[3.0]])] * 2, [np.array([[0.25]])] * 2, 1)
    s1 = 0.7310585786300049
    assert abs(out[0, 0, 0] - 1.0965878679450074) < 1e-14
    assert np.allclose(out[0, 1:, 0], s1 * 3.0 * 0.25 * np.array([1.0, -2.0, 0.5]), atol=1e-15)


def test_ffn_structure():
    """Equivariance; the gate depends only on the l = 0 features; for fixed
    x_0 the l >= 1 outputs are linear in x_l; zero gate weights give zero."""
    rng = np.random.default_rng(3)
    L, C, Hd = 3, 6, 24
    Q = (L + 1) ** 2
    Wa = rng.standard_normal((Hd, C))
    Wb = [rng.standard_normal((Hd, C)) for _ in range(L + 1)]
    Wd = [rng.standard_normal((C, Hd)) for _ in range(L + 1)]
    x = rng.standard_normal((5, Q, C))
    f = ob.ffn(x, Wa, Wb, Wd, L)
    Qr = wlmod.haar_rotation(rng)
    assert np.max(np.abs(ob.ffn(_rotate_blocks(x, Qr, L), Wa, Wb, Wd, L) - _rotate_blocks(f, Qr, L))) < 1e-11
    x2 = x.copy()
    x2[:, 1:, :] = rng.standard_normal((5, Q - 1, C))
    assert np.max(np.abs(ob.ffn(x2, Wa, Wb, Wd, L)[:, 0, :] - f[:, 0, :])) < 1e-13
    xa, xb = x.copy(), x.copy()
    xb[:, 1:, :] = rng.standard_normal((5, Q - 1, C))
    xs = x.copy()
    xs[:, 1:, :] = 2.0 * xa[:, 1:, :] - 3.0 * xb[:, 1:, :]
    fa, fb, fs = (ob.ffn(z, Wa, Wb, Wd, L) for z in (xa, xb, xs))
    assert np.max(np.abs(fs[:, 1:, :] - (2.0 * fa[:, 1:, :] - 3.0 * fb[:, 1:, :]))) < 1e-11
    assert np.all(ob.ffn(x, np.zeros_like(Wa), Wb, Wd, L) == 0.0)


def _zero_layer(lw):
    z = dict(lw)
    z["W0"] = np.zeros_like(lw["W0"])
    z["Wr"] = [None] + [np.zeros_like(w) for w in lw["Wr"][1:]]
    z["Wi"] = [None] + [np.zeros_like(w) for w in lw["Wi"][1:]]
    z["Wd"] = [np.zeros_like(w) for w in lw["Wd"]]
    return z


def test_block_residual_identity_and_equivariance():
    wl = wlmod.make_workload(0)
    lw = wlmod.make_layer_weights(wl.L, wl.C, wl.H, "fp32", 11)
    csr = nb.neighbors(wl.pos, wl.box, wl.r_c)
    # zero SO(2) blocks and zero FFN output maps: the block is the identity
    assert np.array_equal(ob.block_forward(wl.pos, wl.box, wl.r_c, csr, wl.x, _zero_layer(lw)),
                          wl.x.astype(np.float64))
    out = ob.block_forward(wl.pos, wl.box, wl.r_c, csr, wl.x, lw)
    rng = np.random.default_rng(4)
    Qr = wlmod.haar_rotation(rng)
    pos2 = (wl.pos.astype(np.float64) @ Qr.T)
    out2 = ob.block_forward(pos2, None, wl.r_c, csr, _rotate_blocks(wl.x.astype(np.float64), Qr, wl.L), lw)
    err = np.max(np.abs(out2 - _rotate_blocks(out, Qr, wl.L))) / np.max(np.abs(out))
    assert err < 1e-10
    # translation invariance
    out3 = ob.block_forward(wl.pos.astype(np.float64) + np.array([3.0, -1.0, 7.5]), None, wl.r_c, csr, wl.x, lw)
    assert np.max(np.abs(out3 - out)) / np.max(np.abs(out)) < 1e-12


def test_block_degree_zero_is_a_scalar_transformer_block():
    """L = 0: the block is a pre-norm transformer block on scalars --
    RMSNorm, envelope-weighted softmax attention with value map g00 W0 Wv,
    residual, RMSNorm, SwiGLU MLP, residual -- checked with torch's rms_norm
    and an independent edge loop."""
    import torch
    wl0 = wlmod.make_workload(0)
    L, C, H = 0, 8, 2
    wl = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=L, C=C, H=H, seed=6)
    lw = wlmod.make_layer_weights(L, C, H, "fp32", 12)
    rp, col = nb.neighbors(wl.pos, None, wl.r_c)
    got = ob.block_forward(wl.pos, None, wl.r_c, (rp, col), wl.x, lw)

    x = wl.x[:, 0, :].astype(np.float64)
    def rms(v, g):
        return torch.nn.functional.rms_norm(torch.from_numpy(v), (C,), weight=torch.from_numpy(
            np.asarray(g, np.float64)), eps=ob.RMS_EPS).numpy()
    xn = rms(x, lw["gamma1"][0])
    q, k, v = (xn @ np.asarray(lw[n][0], np.float64).T for n in ("Wq", "Wk", "Wv"))
    att = np.zeros_like(x)
    Ch = C // H
    for i in range(wl.N):
        js = col[rp[i]:rp[i + 1]]
        if len(js) == 0:
            continue
        r = np.linalg.norm(wl.pos[js].astype(np.float64) - wl.pos[i].astype(np.float64), axis=1)
        u = 0.5 * (np.cos(math.pi * r / wl.r_c) + 1.0)
        g00 = oa.radial_mlp(r, wl.r_c, lw["rad_W1"], lw["rad_W2"])[:, 0]
        msg = (v[js] @ np.asarray(lw["W0"], np.float64).T) * g00[:, None]
        for h in range(H):
            c = slice(h * Ch, (h + 1) * Ch)
            logit = (k[js][:, c] @ q[i, c]) / math.sqrt(Ch) + np.log(u)
            w = np.exp(logit - logit.max())
            att[i, c] = (w / w.sum()) @ msg[:, c]
    x1 = x + att
    yn = rms(x1, lw["gamma2"][0])
    gate = yn @ np.asarray(lw["Wa"], np.float64).T
    hid = gate / (1.0 + np.exp(-gate)) * (yn @ np.asarray(lw["Wb"][0], np.float64).T)
    ref = x1 + hid @ np.asarray(lw["Wd"][0], np.float64).T
    assert np.max(np.abs(got[:, 0, :] - ref)) < 1e-12


def test_model_forward_is_blocks_in_turn():
    wl = wlmod.make_workload(0)
    csr = nb.neighbors(wl.pos, wl.box, wl.r_c)
    layers = [wlmod.make_layer_weights(wl.L, wl.C, wl.H, "fp32", s) for s in (21, 22)]
    two = ob.model_forward(wl.pos, wl.box, wl.r_c, csr, wl.x, layers)
    one = ob.block_forward(wl.pos, wl.box, wl.r_c, csr, wl.x, layers[0])
    assert np.array_equal(two, ob.block_forward(wl.pos, wl.box, wl.r_c, csr, one, layers[1]))
