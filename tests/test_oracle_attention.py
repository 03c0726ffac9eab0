"""Pins of the attention oracle (P6-P12, P14 and special cases).

Each check compares the oracle with something it does not compute itself:
an invariant of the operator (gauge, rotation, translation, relabelling,
neighbour order), a reduction to textbook scalar attention, a special
geometry whose rotation matrices are known in closed form, the complex-
number form of the SO(2) blocks, or closed-form facts about the radial
basis and envelope.
"""
import copy
import math

import numpy as np
import pytest
from scipy.special import expit

from atomistic_mlip_b200 import workloads as wlmod
from oracle import attention as oa
from oracle import neighbors as nb
from oracle import sh


def _run(wl, csr=None, **kw):
    csr = csr if csr is not None else nb.neighbors(wl.pos, wl.box, wl.r_c)
    return oa.attention_workload(wl, csr=csr, **kw), csr


def _rotate_nodes(o, Q, L):
    D = [sh.wigner_d_fit(l, Q) for l in range(L + 1)]
    out = np.empty_like(o)
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) ** 2)
        out[:, sl, :] = D[l] @ o[:, sl, :]
    return out


@pytest.fixture(scope="module")
def cfg0():
    return wlmod.make_workload(0)


@pytest.fixture(scope="module")
def small_l4():
    """cfg0 geometry with L = 4, C = 16, H = 2 (more SO(2) blocks)."""
    wl0 = wlmod.make_workload(0)
    return wlmod.make_custom(wl0.pos, None, wl0.r_c, L=4, C=16, H=2, seed=11)


def test_gauge_invariance(cfg0, small_l4):
    """P6: an arbitrary extra z-rotation of every edge frame changes nothing
    (SO(2) blocks commute with z-rotations, m = 0 rows are z-invariant)."""
    for wl in (cfg0, small_l4):
        o, csr = _run(wl)
        g = _run(wl, csr=csr, gauge=lambda e: np.random.default_rng(5).uniform(0, 2 * np.pi, len(e)))[0]
        assert np.max(np.abs(g - o)) <= 1e-12 * np.max(np.abs(o))


def test_rotation_equivariance_open(cfg0, small_l4):
    """P7: positions -> Q p, features -> D(Q) x gives outputs D(Q) o."""
    rng = np.random.default_rng(99)
    for wl in (cfg0, small_l4):
        o, csr = _run(wl)
        for _ in range(2):
            Q = wlmod.haar_rotation(rng)
            w2 = copy.deepcopy(wl)
            w2.pos = wl.pos.astype(np.float64) @ Q.T
            w2.x = _rotate_nodes(wl.x.astype(np.float64), Q, wl.L)
            o2 = oa.attention_workload(w2, csr=csr)
            err = np.max(np.abs(o2 - _rotate_nodes(o, Q, wl.L))) / np.max(np.abs(o))
            assert err <= 1e-10


def test_rotation_equivariance_periodic():
    """P7 on a periodic box: a cube rotation plus a translation, wrapped."""
    rng = np.random.default_rng(3)
    box = np.array([12.0, 12.0, 12.0], np.float32)
    pos = (rng.uniform(0, 12.0, (40, 3))).astype(np.float32)
    wl = wlmod.make_custom(pos, box, 4.0, L=3, C=8, H=2, seed=5)
    o, csr = _run(wl)
    Q = wlmod.cube_rotations()[7]
    shift = np.array([3.0, 5.0, 1.0])
    w2 = copy.deepcopy(wl)
    w2.pos = np.mod(pos.astype(np.float64) @ Q.T + shift, 12.0)
    w2.x = _rotate_nodes(wl.x.astype(np.float64), Q, wl.L)
    o2 = oa.attention_workload(w2, csr=csr)
    assert np.max(np.abs(o2 - _rotate_nodes(o, Q, wl.L))) <= 1e-10 * np.max(np.abs(o))


def test_translation_relabel_and_column_order(small_l4):
    """P8: translation invariance; relabelling atoms permutes outputs;
    permuting the columns of a CSR row leaves the output unchanged."""
    wl = small_l4
    o, (rp, col) = _run(wl)
    w2 = copy.deepcopy(wl)
    w2.pos = wl.pos.astype(np.float64) + np.array([1.5, -2.0, 7.25])
    o2 = oa.attention_workload(w2, csr=(rp, col))
    assert np.max(np.abs(o2 - o)) <= 1e-12 * np.max(np.abs(o))
    # relabel
    perm = np.random.default_rng(1).permutation(wl.N)
    inv = np.argsort(perm)
    w3 = copy.deepcopy(wl)
    w3.pos, w3.x = wl.pos[perm], wl.x[perm]
    o3, _ = _run(w3)
    assert np.max(np.abs(o3 - o[perm])) <= 1e-12 * np.max(np.abs(o))
    # shuffle within rows
    col2 = col.copy()
    rng = np.random.default_rng(2)
    for i in range(wl.N):
        seg = col2[rp[i]:rp[i + 1]]
        rng.shuffle(seg)
    o4 = oa.attention_workload(wl, csr=(rp, col2))
    assert np.max(np.abs(o4 - o)) <= 1e-12 * np.max(np.abs(o))
    _ = inv


def test_l0_reduces_to_scalar_attention():
    """P9: with L = 0 the operator is plain scalar softmax attention with an
    envelope: o_i = sum_j softmax_j(log u + q_i.k_j / sqrt(C_h)) g00(r) W0 v_j."""
    wl0 = wlmod.make_workload(0)
    wl = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=0, C=12, H=3, seed=21)
    o, (rp, col) = _run(wl)
    x = wl.x[:, 0, :].astype(np.float64)
    q, k, v = x @ wl.Wq[0].T, x @ wl.Wk[0].T, x @ wl.Wv[0].T
    Ch = wl.C // wl.H
    p = wl.pos.astype(np.float64)
    ref = np.zeros((wl.N, wl.C))
    for i in range(wl.N):
        js = col[rp[i]:rp[i + 1]]
        if len(js) == 0:
            continue
        r = np.linalg.norm(p[js] - p[i], axis=1)
        u = 0.5 * (np.cos(np.pi * r / wl.r_c) + 1)
        mu = np.linspace(0, wl.r_c, 8)
        phi = np.exp(-(r[:, None] - mu) ** 2 / (2 * 0.25))
        hid = phi @ wl.rad_W1.T.astype(np.float64)
        g = (hid * expit(hid)) @ wl.rad_W2.T.astype(np.float64)      # P = 1
        msg = g[:, :1] * (v[js] @ wl.W0.T.astype(np.float64))
        for h in range(wl.H):
            cs = slice(h * Ch, (h + 1) * Ch)
            logits = np.log(u) + (q[i, cs] * k[js][:, cs]).sum(1) / math.sqrt(Ch)
            a = np.exp(logits - logits.max())
            a /= a.sum()
            ref[i, cs] = a @ msg[:, cs]
    np.testing.assert_allclose(o[:, 0, :], ref, atol=1e-13 * np.max(np.abs(ref)))


def test_identity_weights_average_values(small_l4):
    """P10: W0 = I, Wr = I, Wi = 0, g = 1  =>  o_i = sum_j alpha_ij v_j
    (rotate-in / rotate-out round trip and the +-m stacking)."""
    wl = copy.deepcopy(small_l4)
    wl.W0 = np.eye(wl.n_m(0))
    wl.Wr = [None] + [np.eye(wl.n_m(m)) for m in range(1, wl.L + 1)]
    wl.Wi = [None] + [np.zeros((wl.n_m(m), wl.n_m(m))) for m in range(1, wl.L + 1)]
    o, (rp, col) = _run(wl, g_override=1.0)
    v = oa.project(wl.x, wl.Wv, wl.L)
    # alpha from a run whose values are a constant one-hot feature
    # (independent check: outputs must be convex combinations of v_j with
    # the same per-head weights; verify by reconstructing alpha from l=0).
    for i in range(wl.N):
        js = col[rp[i]:rp[i + 1]]
        if len(js) == 0:
            assert np.all(o[i] == 0)
            continue
        # solve for alpha per head from the l=0 channel block (overdetermined)
        Ch = wl.C // wl.H
        for h in range(wl.H):
            cs = slice(h * Ch, (h + 1) * Ch)
            A = v[js][:, :, cs].reshape(len(js), -1).T             # [(Q*Ch), k]
            b = o[i][:, cs].reshape(-1)
            a, *_ = np.linalg.lstsq(A, b, rcond=None)
            assert np.all(a > 0) and abs(a.sum() - 1) < 1e-10
            np.testing.assert_allclose(A @ a, b, atol=1e-12)


def test_so2_block_is_complex_multiplication():
    """For m >= 1 the block [[Wr, -Wi], [Wi, Wr]] acting on (v+, v-) is the
    complex product (Wr + i Wi)(v+ + i v-)."""
    rng = np.random.default_rng(4)
    L, C = 3, 5
    Q = (L + 1) ** 2
    vt = rng.standard_normal((6, Q, C))
    W0 = rng.standard_normal(((L + 1) * C,) * 2)
    Wr = [None] + [rng.standard_normal(((L - m + 1) * C,) * 2) for m in range(1, L + 1)]
    Wi = [None] + [rng.standard_normal(((L - m + 1) * C,) * 2) for m in range(1, L + 1)]
    y = oa.so2_mix(vt, np.ones((6, (L + 1) * (L + 2) // 2)), L, C, W0, Wr, Wi)
    for m in range(1, L + 1):
        vp = np.concatenate([vt[:, l * l + l + m, :] for l in range(m, L + 1)], 1)
        vm = np.concatenate([vt[:, l * l + l - m, :] for l in range(m, L + 1)], 1)
        z = (vp + 1j * vm) @ (Wr[m] + 1j * Wi[m]).T
        yp = np.concatenate([y[:, l * l + l + m, :] for l in range(m, L + 1)], 1)
        ym = np.concatenate([y[:, l * l + l - m, :] for l in range(m, L + 1)], 1)
        np.testing.assert_allclose(yp, z.real, atol=1e-12)
        np.testing.assert_allclose(ym, z.imag, atol=1e-12)
    v0 = np.concatenate([vt[:, l * l + l, :] for l in range(L + 1)], 1)
    y0 = np.concatenate([y[:, l * l + l, :] for l in range(L + 1)], 1)
    np.testing.assert_allclose(y0, v0 @ W0.T, atol=1e-12)


def test_one_neighbour_along_z_and_minus_z():
    """P11 + closed-form frames.  Atom 0 has one neighbour at +z (frame = I):
    o_0 = g * SO2(v_1) directly in the global frame.  Atom 2's neighbour
    lies at -z (frame = rotation by pi about x, a diagonal sign matrix on
    the real harmonics: (-1)^(l+m) for m >= 0, (-1)^(l+|m|+1) for m < 0)."""
    pos = np.array([[0, 0, 0], [0, 0, 1.7], [20, 0, 3.0], [20, 0, 1.1]], np.float32)
    wl = wlmod.make_custom(pos, None, 2.5, L=3, C=8, H=2, seed=8)
    o, (rp, col) = _run(wl)
    L, C = wl.L, wl.C
    v = oa.project(wl.x, wl.Wv, L)
    for (i, j, signs) in ((0, 1, None), (2, 3, True)):
        r = float(np.linalg.norm(pos[j].astype(np.float64) - pos[i]))
        g = oa.radial_mlp(np.array([r]), wl.r_c, wl.rad_W1, wl.rad_W2)
        S = np.ones((L + 1) ** 2)
        if signs:
            for l in range(L + 1):
                for m in range(-l, l + 1):
                    S[l * l + l + m] = (-1) ** (l + m) if m >= 0 else (-1) ** (l - m + 1)
        vt = (S[:, None] * v[j])[None]
        y = oa.so2_mix(vt, g, L, C, wl.W0, wl.Wr, wl.Wi)[0]
        np.testing.assert_allclose(o[i], S[:, None] * y, atol=1e-12)


def test_logit_orientation_two_neighbours():
    """Logits with neighbours at +z and -z only involve the m = 0 entries of
    q_i = Wq[l] x_i and k_j = Wk[l] x_j (signs (-1)^l at -z); checks the
    out x in orientation of Wq / Wk for every degree."""
    pos = np.array([[0, 0, 0], [0, 0, 1.3], [0, 0, -1.9]], np.float32)
    wl = wlmod.make_custom(pos, None, 2.5, L=3, C=8, H=1, seed=31)
    wl.W0 = np.eye(wl.n_m(0))
    wl.Wr = [None] + [np.eye(wl.n_m(m)) for m in range(1, wl.L + 1)]
    wl.Wi = [None] + [np.zeros((wl.n_m(m),) * 2) for m in range(1, wl.L + 1)]
    o, _ = _run(wl, g_override=1.0)
    x = wl.x.astype(np.float64)
    d = (wl.L + 1) * wl.C
    s = []
    for j, sgn in ((1, 1.0), (2, -1.0)):
        tot = 0.0
        for l in range(wl.L + 1):
            qi = wl.Wq[l] @ x[0, l * l + l]
            kj = wl.Wk[l] @ x[j, l * l + l]
            tot += (sgn ** l) ** 2 * qi @ kj
        s.append(tot / math.sqrt(d))
    r1, r2, rc = float(np.float32(1.3)), float(np.float32(1.9)), float(np.float32(2.5))
    u = [0.5 * (math.cos(math.pi * r1 / rc) + 1), 0.5 * (math.cos(math.pi * r2 / rc) + 1)]
    w = np.array(u) * np.exp(np.array(s) - max(s))
    a = w / w.sum()
    # identity mixing and g = 1: o_0 = sum_j a_j v_j (frame round trip)
    v = oa.project(wl.x, wl.Wv, wl.L)
    np.testing.assert_allclose(o[0], a[0] * v[1] + a[1] * v[2], atol=1e-12)


def test_online_softmax_chunks_equal_two_pass():
    """P12: the streaming update (running max M, denominator l, accumulator
    rescaled by exp(M_old - M_new)) over random chunkings equals two-pass."""
    rng = np.random.default_rng(12)
    s = rng.standard_normal(97) * 4
    u = rng.uniform(0.01, 1, 97)
    z = rng.standard_normal((97, 5))
    ref = (u * np.exp(s - s.max()))[:, None] * z
    ref = ref.sum(0) / (u * np.exp(s - s.max())).sum()
    for _ in range(5):
        cuts = np.sort(rng.choice(np.arange(1, 97), size=6, replace=False))
        M, den, acc = -np.inf, 0.0, np.zeros(5)
        for a, b in zip(np.r_[0, cuts], np.r_[cuts, 97]):
            Mn = max(M, s[a:b].max())
            scale = math.exp(M - Mn) if M > -np.inf else 0.0
            w = u[a:b] * np.exp(s[a:b] - Mn)
            den = den * scale + w.sum()
            acc = acc * scale + w @ z[a:b]
            M = Mn
        np.testing.assert_allclose(acc / den, ref, rtol=1e-14, atol=1e-14)


def test_radial_basis_and_envelope_closed_forms():
    rc = 6.0
    mu = np.arange(8) * rc / 7
    phi = oa.radial_basis(mu, rc)
    np.testing.assert_allclose(np.diag(phi), 1.0)
    np.testing.assert_allclose(oa.radial_basis(mu + 0.5, rc)[np.arange(8), np.arange(8)], math.exp(-0.5))
    z = np.linspace(-5, 5, 11)
    np.testing.assert_allclose(oa.silu(z), z * expit(z), rtol=1e-15)
    np.testing.assert_allclose(oa.envelope(np.array([0.0, rc / 2, rc]), rc), [1.0, 0.5, 0.0], atol=1e-15)
    # one-hot MLP: W1 picks phi_3, W2 picks hidden unit 0 for output p = 2
    W1 = np.zeros((16, 8)); W1[0, 3] = 1.0
    W2 = np.zeros((6, 16)); W2[2, 0] = 1.0
    r = np.array([2.0])
    p3 = math.exp(-(2.0 - 3 * rc / 7) ** 2 / 0.5)
    g = oa.radial_mlp(r, rc, W1, W2)
    np.testing.assert_allclose(g[0], [0, 0, p3 * expit(p3), 0, 0, 0], rtol=1e-14)
    assert oa.pair_list(2) == [(0, 0), (0, 1), (0, 2), (1, 1), (1, 2), (2, 2)]


def test_envelope_continuity_at_cutoff():
    """P14: an atom crossing r_c changes the output by O((r_c - r)^2)."""
    base = np.array([[0, 0, 0], [1.2, 0.3, -0.4], [-0.8, 1.1, 0.5]], np.float32)
    diffs = []
    for eps in (0.2, 0.1, 0.05):
        pos = np.vstack([base, [[0.0, 0.0, 3.0 - eps]]]).astype(np.float32)
        wl = wlmod.make_custom(pos, None, 3.0, L=2, C=8, H=2, seed=3)
        o_in, _ = _run(wl)
        wl_out = copy.deepcopy(wl)
        wl_out.pos = wl.pos.copy()
        wl_out.pos[3] = [0.0, 0.0, 3.5]
        o_out, _ = _run(wl_out)
        diffs.append(np.max(np.abs(o_in[0] - o_out[0])))
    # halving the distance to the cutoff divides the jump by ~4
    assert diffs[1] / diffs[0] < 0.35 and diffs[2] / diffs[1] < 0.35


def test_empty_neighbourhood_is_zero():
    pos = np.array([[0, 0, 0], [10, 0, 0], [10.5, 0, 0]], np.float32)
    wl = wlmod.make_custom(pos, None, 2.0, L=2, C=8, H=2, seed=1)
    o, _ = _run(wl)
    assert np.all(o[0] == 0) and np.any(o[1] != 0)
