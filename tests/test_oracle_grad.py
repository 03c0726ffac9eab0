"""Pins of the gradient oracle (oracle.attention_grad): the torch restatement
of the operator equals oracle.attention, and its autograd gradients equal
central finite differences of oracle.attention; forces sum to zero and
rotate with the system."""
import numpy as np
import pytest
import torch

from atomistic_mlip_b200 import workloads as wlmod
from oracle import attention as oa
from oracle import attention_grad as ag
from oracle import neighbors as nb
from oracle import sh


def _system(periodic: bool, L: int, seed: int):
    rng = np.random.default_rng(seed)
    if periodic:
        b = 9.0
        pos = rng.uniform(0.0, b, (16, 3)).astype(np.float32)
        wl = wlmod.make_custom(pos, np.array([b, b, b], np.float32), 4.0, L=L, C=8, H=2, seed=seed)
    else:
        pos = rng.uniform(0.0, 7.0, (14, 3)).astype(np.float32)
        wl = wlmod.make_custom(pos, None, 4.0, L=L, C=8, H=2, seed=seed)
    return wl, nb.neighbors(wl.pos, wl.box, wl.r_c)


def _loss_np(wl, csr, G, pos=None, x=None, **w):
    kw = dict(Wq=wl.Wq, Wk=wl.Wk, Wv=wl.Wv, W0=wl.W0, Wr=wl.Wr, Wi=wl.Wi, rad_W1=wl.rad_W1, rad_W2=wl.rad_W2)
    kw.update(w)
    o = oa.attention(wl.pos.astype(np.float64) if pos is None else pos, wl.box, wl.r_c, csr[0], csr[1],
                     wl.x if x is None else x, kw["Wq"], kw["Wk"], kw["Wv"], kw["W0"], kw["Wr"], kw["Wi"],
                     kw["rad_W1"], kw["rad_W2"], wl.L, wl.C, wl.H)
    return float((o * G).sum())


def test_real_sh_polynomial_form():
    rng = np.random.default_rng(1)
    u = rng.standard_normal((200, 3))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    u[0], u[1] = [0.0, 0.0, 1.0], [0.0, 0.0, -1.0]
    for l in range(7):
        got = ag.real_sh_t(l, torch.tensor(u)).numpy()
        assert np.max(np.abs(got - sh.real_sh(l, u))) < 1e-13, l


@pytest.mark.parametrize("periodic,L", [(False, 3), (True, 2), (False, 0)])
def test_forward_matches_oracle(periodic, L):
    wl, csr = _system(periodic, L, seed=5 + L)
    ref = oa.attention_workload(wl, csr=csr)
    got = ag.forward_t(torch.tensor(wl.pos.astype(np.float64)), wl.box, wl.r_c, csr[0], csr[1],
                       torch.tensor(wl.x.astype(np.float64)), ag.params_t(wl), wl.L, wl.C, wl.H).numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


@pytest.mark.parametrize("periodic", [False, True])
def test_gradients_match_finite_differences(periodic):
    """d/dh sum(G o) along random directions of positions, features and
    several weights, central differences (h = 1e-5, truncation ~ h^2)."""
    wl, csr = _system(periodic, 3 if not periodic else 2, seed=11)
    rng = np.random.default_rng(12)
    G = rng.standard_normal((wl.N, (wl.L + 1) ** 2, wl.C))
    gr = ag.gradients(wl, csr, G)
    h = 1e-5

    def check(ad, fp, fm):
        fd = (fp - fm) / (2 * h)
        assert abs(fd - ad) <= 1e-6 * max(abs(ad), 1e-3), (fd, ad)

    p0 = wl.pos.astype(np.float64)
    for _ in range(3):
        d = rng.standard_normal(p0.shape)
        check(float((gr["pos"] * d).sum()), _loss_np(wl, csr, G, pos=p0 + h * d), _loss_np(wl, csr, G, pos=p0 - h * d))
    x0 = wl.x.astype(np.float64)
    d = rng.standard_normal(x0.shape)
    check(float((gr["x"] * d).sum()), _loss_np(wl, csr, G, x=x0 + h * d), _loss_np(wl, csr, G, x=x0 - h * d))
    for key, idx in (("W0", None), ("rad_W1", None), ("rad_W2", None), ("Wq", 1), ("Wk", wl.L), ("Wv", 0),
                     ("Wr", 1), ("Wi", wl.L)):
        base = getattr(wl, key)
        w0 = np.asarray(base if idx is None else base[idx], np.float64)
        d = rng.standard_normal(w0.shape)
        ad = float(((gr[key] if idx is None else gr[key][idx]) * d).sum())

        def with_w(delta):
            if idx is None:
                return {key: w0 + delta}
            lst = [np.asarray(a, np.float64) for a in base]
            lst[idx] = w0 + delta
            return {key: lst}

        check(ad, _loss_np(wl, csr, G, **with_w(h * d)), _loss_np(wl, csr, G, **with_w(-h * d)))


def test_forces_sum_to_zero():
    """sum(G o) depends on positions through differences only."""
    for periodic in (False, True):
        wl, csr = _system(periodic, 2, seed=21)
        G = np.random.default_rng(22).standard_normal((wl.N, (wl.L + 1) ** 2, wl.C))
        g = ag.gradients(wl, csr, G)["pos"]
        assert np.max(np.abs(g.sum(axis=0))) <= 1e-12 * np.max(np.abs(g))


def test_forces_rotate_with_the_system():
    """With a readout of the l = 0 rows only (an invariant of the output),
    rotating positions and features rotates the position gradient."""
    wl, csr = _system(False, 3, seed=31)
    rng = np.random.default_rng(32)
    Q = (wl.L + 1) ** 2
    G = np.zeros((wl.N, Q, wl.C))
    G[:, 0, :] = rng.standard_normal((wl.N, wl.C))
    g0 = ag.gradients(wl, csr, G)["pos"]
    Rq = wlmod.haar_rotation(rng)
    pos_r = wl.pos.astype(np.float64) @ Rq.T
    x_r = np.empty((wl.N, Q, wl.C))
    for l in range(wl.L + 1):
        s_ = slice(l * l, (l + 1) ** 2)
        x_r[:, s_, :] = sh.wigner_d_fit(l, Rq) @ wl.x[:, s_, :].astype(np.float64)
    g1 = ag.gradients(wl, csr, G, pos=pos_r, x=x_r)["pos"]
    assert np.max(np.abs(g1 - g0 @ Rq.T)) <= 1e-10 * np.max(np.abs(g0))


def test_logit_gradient_recompute_form():
    """The softmax backward a tiled kernel uses (per head: alpha times the
    message-gradient product minus the node's Delta) equals autograd."""
    for periodic in (False, True):
        wl, csr = _system(periodic, 2, seed=41)
        G = np.random.default_rng(42).standard_normal((wl.N, (wl.L + 1) ** 2, wl.C))
        auto, formula = ag.logit_gradient(wl, csr, G)
        assert np.max(np.abs(auto - formula)) <= 1e-12 * np.max(np.abs(auto))


def test_local_gradients_equal_full_gradients():
    """The sampled form used on large systems (tests.helpers.local_gradients:
    only the outputs of an atom and of its neighbours, over the atoms those
    rows read) gives the atom's full dL/dpos and dL/dx: pinned against the
    gradients of the whole system on a periodic box where the local region is
    a strict subset of the atoms."""
    from tests import helpers
    rng = np.random.default_rng(21)
    b = 16.0
    pos = rng.uniform(0.0, b, (120, 3)).astype(np.float32)
    wl = wlmod.make_custom(pos, np.array([b, b, b], np.float32), 3.5, L=2, C=8, H=2, seed=22)
    G = rng.standard_normal(wl.x.shape)
    full = ag.gradients(wl, nb.neighbors(wl.pos, wl.box, wl.r_c), G)
    nodes = np.array([3, 57, 101])
    gp, gx = helpers.local_gradients(wl, nodes, G)
    assert np.max(np.abs(gp - full["pos"][nodes])) <= 1e-12 * np.max(np.abs(full["pos"][nodes]))
    assert np.max(np.abs(gx - full["x"][nodes])) <= 1e-12 * np.max(np.abs(full["x"][nodes]))
    assert np.max(np.abs(full["pos"][nodes])) > 0


def test_local_rows_reproduce_the_attention_rows():
    """tests.helpers.local_rows: the attention oracle on the subsystem of
    some rows (their atoms and neighbours, only those rows listed) gives the
    same rows as on the whole periodic system."""
    from tests import helpers
    rng = np.random.default_rng(23)
    b = 16.0
    pos = rng.uniform(0.0, b, (120, 3)).astype(np.float32)
    wl = wlmod.make_custom(pos, np.array([b, b, b], np.float32), 3.5, L=2, C=8, H=2, seed=24)
    rp, col = nb.neighbors(wl.pos, wl.box, wl.r_c)[:2]
    args = (wl.Wq, wl.Wk, wl.Wv, wl.W0, wl.Wr, wl.Wi, wl.rad_W1, wl.rad_W2, wl.L, wl.C, wl.H)
    full = oa.attention(wl.pos, wl.box, wl.r_c, rp, col, wl.x, *args)
    nodes = np.array([5, 60, 99])
    U, csr, idx = helpers.local_rows(wl.pos, wl.box, wl.r_c, nodes)
    assert len(U) < wl.N
    loc = oa.attention(wl.pos[U], wl.box, wl.r_c, csr[0], csr[1], wl.x[U], *args, nodes=idx[nodes])
    assert np.max(np.abs(loc - full[nodes])) <= 1e-12 * np.max(np.abs(full[nodes]))
