"""The C-ABI library loads, exports every entry point include/e2f.h
declares, and rejects bad arguments on the host (no GPU needed: these calls
return before any CUDA work)."""
import ctypes
import os
import re

import pytest

from atomistic_mlip_b200 import build as build_mod
from atomistic_mlip_b200 import e2f

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"E2F_API\s+[\w\s\*]+?\b(e2f_\w+)\s*\(", txt)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return e2f.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
        assert n in e2f.SIGNATURES, f"{n} missing from the binding"


def test_status_strings(lib):
    assert lib.e2f_status_string(0) == b"ok"
    assert b"capacity" in lib.e2f_status_string(3)


def test_build_neighbors_validation(lib):
    n_e = ctypes.c_int64(0)
    dummy = ctypes.c_void_p(16)
    f = lib.e2f_build_neighbors
    assert f(dummy, -1, None, 1.0, dummy, dummy, 10, ctypes.byref(n_e), None, None) == 1
    assert f(dummy, 10, None, 0.0, dummy, dummy, 10, ctypes.byref(n_e), None, None) == 1
    assert f(dummy, 10, None, float("nan"), dummy, dummy, 10, ctypes.byref(n_e), None, None) == 1
    assert f(None, 10, None, 1.0, dummy, dummy, 10, ctypes.byref(n_e), None, None) == 1
    box = (ctypes.c_float * 3)(10.0, 10.0, 10.0)
    assert f(dummy, 10, box, 5.0, dummy, dummy, 10, ctypes.byref(n_e), None, None) == 2
    box = (ctypes.c_float * 3)(10.0, -1.0, 10.0)
    assert f(dummy, 10, box, 1.0, dummy, dummy, 10, ctypes.byref(n_e), None, None) == 1


def _weights(L=2, C=8, H=2, dtype=0, fill=True):
    w = e2f.Weights()
    w.L_max, w.C, w.H, w.dtype = L, C, H, dtype
    p = 64
    if fill:
        for l in range(min(L, 6) + 1):
            w.Wq[l] = w.Wk[l] = w.Wv[l] = p
        w.W0 = p
        for m in range(1, min(L, 6) + 1):
            w.Wr[m] = w.Wi[m] = p
        w.rad_W1 = w.rad_W2 = p
    return w


def test_attention_validation(lib):
    csr = e2f.Csr()
    csr.row_ptr = 64; csr.col_idx = 64; csr.n_nodes = 4; csr.n_edges = 4; csr.r_c = 1.0
    f = lib.e2f_attention_forward
    d = ctypes.c_void_p(64)
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights(L=7)), d, None) == 1
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights(C=8, H=3)), d, None) == 4
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights(dtype=5)), d, None) == 4
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights(fill=False)), d, None) == 1
    assert f(d, None, ctypes.byref(csr), ctypes.byref(_weights()), d, None) == 1
    csr.box[0] = 1.5
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights()), d, None) == 2
    csr.box[0] = 0.0
    csr.n_nodes = 0
    assert f(None, None, ctypes.byref(csr), ctypes.byref(_weights()), None, None) == 0


def test_unit_entry_validation(lib):
    d = ctypes.c_void_p(64)
    assert lib.e2f_wigner_d(d, 5, 7, d, None) == 1
    assert lib.e2f_wigner_d(None, 0, 3, None, None) == 0
    assert lib.e2f_project_qkv(d, -1, ctypes.byref(_weights()), d, d, d, None) == 1
    assert lib.e2f_profile_read(None, None) == 1


def test_misaligned_pointers_rejected(lib):
    """Feature and weight pointers are read as 16-byte vectors: a pointer
    that is not 16-byte aligned is rejected on the host."""
    csr = e2f.Csr()
    csr.row_ptr = 64; csr.col_idx = 64; csr.n_nodes = 4; csr.n_edges = 4; csr.r_c = 1.0
    f = lib.e2f_attention_forward
    d, odd = ctypes.c_void_p(64), ctypes.c_void_p(72)
    assert f(odd, d, ctypes.byref(csr), ctypes.byref(_weights()), d, None) == 1
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights()), odd, None) == 1
    w = _weights()
    w.Wr[1] = 72
    assert f(d, d, ctypes.byref(csr), ctypes.byref(w), d, None) == 1
    assert lib.e2f_project_qkv(d, 4, ctypes.byref(_weights()), d, odd, d, None) == 1


def test_validation_from_two_host_threads(lib):
    """The entry points keep no state while validating arguments: two host
    threads calling them at once each get the status of their own call."""
    import threading
    errors = []

    def worker(seed):
        n_e = ctypes.c_int64(0)
        d = ctypes.c_void_p(64)
        csr = e2f.Csr()
        csr.row_ptr = 64; csr.col_idx = 64; csr.n_nodes = 4; csr.n_edges = 4; csr.r_c = 1.0
        box = (ctypes.c_float * 3)(10.0, 10.0, 10.0)
        for it in range(2000):
            k = (it + seed) % 4
            if k == 0:
                got, want = lib.e2f_build_neighbors(d, -1, None, 1.0, d, d, 10, ctypes.byref(n_e), None, None), 1
            elif k == 1:
                got, want = lib.e2f_build_neighbors(d, 10, box, 5.0, d, d, 10, ctypes.byref(n_e), None, None), 2
            elif k == 2:
                got, want = lib.e2f_attention_forward(d, d, ctypes.byref(csr), ctypes.byref(_weights(C=8, H=3)),
                                                      d, None), 4
            else:
                got, want = lib.e2f_attention_forward(d, d, ctypes.byref(csr), ctypes.byref(_weights(L=7)),
                                                      d, None), 1
            if got != want:
                errors.append((seed, it, got, want))

    ts = [threading.Thread(target=worker, args=(s,)) for s in (0, 1)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors[:5]


def test_multifocus_and_cg_validation(lib):
    """Host-side checks of the multi-focus attention and the CG convolution
    (no GPU work: every call below returns before any CUDA call)."""
    csr = e2f.Csr()
    csr.row_ptr = 64; csr.col_idx = 64; csr.n_nodes = 4; csr.n_edges = 4; csr.r_c = 1.0
    f = lib.e2f_attention_forward_multifocus
    d, odd = ctypes.c_void_p(64), ctypes.c_void_p(72)
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights()), 3, d, d, None) == 1       # F not 1, 2, 4, 8
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights(C=128, H=8, dtype=1, L=3)), 4, d, d, None) == 4
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights(C=128, H=8, dtype=0, L=4)), 4, d, d, None) == 4
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights(C=128, H=8, dtype=1, L=4)), 4, odd, d, None) == 1
    assert f(d, d, ctypes.byref(csr), ctypes.byref(_weights(C=128, H=8, dtype=1, L=4)), 4, None, d, None) == 1
    g = lib.e2f_cg_conv_forward
    assert lib.e2f_cg_num_paths(7) == -1 and lib.e2f_cg_num_paths(-1) == -1
    assert [lib.e2f_cg_num_paths(L) for L in range(4)] == [1, 5, 15, 34]
    assert g(d, 0, d, ctypes.byref(csr), 7, 8, d, d, None) == 4      # L out of range
    assert g(d, 2, d, ctypes.byref(csr), 2, 8, d, d, None) == 4      # dtype
    assert g(d, 0, d, ctypes.byref(csr), 2, 7, d, d, None) == 1      # odd C
    assert g(d, 0, d, ctypes.byref(csr), 2, 258, d, d, None) == 1    # C too large
    assert g(odd, 0, d, ctypes.byref(csr), 2, 8, d, d, None) == 1    # misaligned x
    assert g(d, 0, d, ctypes.byref(csr), 2, 8, None, d, None) == 1   # no weights
