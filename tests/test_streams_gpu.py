"""Calls on different streams from different host threads are independent:
two threads, each on its own CUDA stream, run the neighbour build, the
forward and the backward (cuBLAS products included) on two different
systems at the same time, three times over; every result equals the one the
same call gives alone on the default stream: the CSR bit for bit; the
forward output to 1e-6 and the gradients to 1e-5 of their largest entry
(float atomics sum each tile's softmax weights and the backward's
scatter, so the order of those sums may change between runs)."""
import threading

import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from tests import helpers

pytestmark = pytest.mark.gpu


def _inputs(wl, seed):
    import torch
    pos, x, w, box = helpers.to_device(wl, "bf16")
    G = torch.from_numpy(np.random.default_rng(seed).standard_normal(wl.x.shape).astype(np.float32)).cuda()
    return pos, x, w, box, G


def _run(wl, inp):
    from atomistic_mlip_b200 import e2f
    pos, x, w, box, G = inp
    nl = e2f.build_neighbors(pos, box, wl.r_c)
    out = e2f.attention_forward(x, pos, nl, w)
    gx, gp = e2f.attention_backward(x, pos, nl, w, G)
    return (nl.n_edges, nl.row_ptr, nl.col_idx), out, gx, gp


def _graph(g):
    E, rp, ci = g
    return E, rp.cpu().numpy(), ci[:E].cpu().numpy()


def test_two_threads_two_streams(cuda_ok):
    import torch
    from atomistic_mlip_b200 import e2f
    wl_a = helpers.cached_workload(2, "bf16")
    wl0 = wlmod.make_workload(0)
    wl_b = wlmod.make_custom(wl0.pos, None, wl0.r_c, L=4, C=128, H=8, precision="bf16", seed=300)
    wls = [wl_a, wl_b]
    inps = [_inputs(wl_a, 301), _inputs(wl_b, 302)]
    ref = []
    for wl, inp in zip(wls, inps):
        g, out, gx, gp = _run(wl, inp)
        torch.cuda.synchronize()
        ref.append((_graph(g), out.cpu().numpy(), gx.cpu().numpy(), gp.cpu().numpy()))
    assert e2f.stream_status() == 0

    got = [[], []]
    errors = []

    def worker(k):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(3):
                    g, out, gx, gp = _run(wls[k], inps[k])
                    s.synchronize()
                    got[k].append((_graph(g), out.cpu().numpy(), gx.cpu().numpy(), gp.cpu().numpy()))
        except Exception as exc:   # reported on the main thread
            errors.append(exc)

    threads = [threading.Thread(target=worker, args=(k,)) for k in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    torch.cuda.synchronize()
    assert e2f.stream_status() == 0
    for k in range(2):
        E, out, gx, gp = ref[k]
        assert len(got[k]) == 3
        for E2, out2, gx2, gp2 in got[k]:
            assert E2[0] == E[0] and np.array_equal(E2[1], E[1]) and np.array_equal(E2[2], E[2])
            assert np.max(np.abs(out2 - out)) <= 1e-6 * np.max(np.abs(out))
            assert np.max(np.abs(gx2 - gx)) <= 1e-5 * np.max(np.abs(gx))
            assert np.max(np.abs(gp2 - gp)) <= 1e-5 * np.max(np.abs(gp))
