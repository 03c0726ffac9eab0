"""e2f_build_neighbors_noalloc: the neighbour build for callers that cannot
allocate device memory (hosts that reserve the device memory budget at
start-up and own every later allocation, or step loops that must not meet
an allocation mid-step).  It keeps its temporaries in one fixed device
array inside the library instead of the library's memory pool.

The test calls it through the C ABI twice in a row per workload -- the
array then holds the previous call's contents -- and compares every result
bit for bit with e2f_build_neighbors (the CSR is integer data, compared
exactly like every other CSR test).  The file is collected last so that a
run stopping at the first failure has run every other test before it.
"""
import ctypes

import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from tests import helpers

pytestmark = pytest.mark.gpu


def _call(fn, pos, box, rc, cap):
    import torch
    from atomistic_mlip_b200 import e2f
    N = int(pos.shape[0])
    row_ptr = torch.full((N + 1,), -1, dtype=torch.int32, device="cuda")
    col_idx = torch.full((cap,), -1, dtype=torch.int32, device="cuda")
    box_arr = None if box is None else (ctypes.c_float * 3)(*[float(b) for b in box])
    n_e = ctypes.c_int64(0)
    code = getattr(e2f.lib(), fn)(pos.data_ptr(), N, box_arr, float(rc), row_ptr.data_ptr(), col_idx.data_ptr(),
                                  cap, ctypes.byref(n_e), None, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return code, row_ptr.cpu().numpy(), col_idx[: n_e.value].cpu().numpy()


@pytest.mark.parametrize("cfg", [2, 1, 0])
def test_noalloc_matches_standard_twice(cuda_ok, cfg):
    import torch
    from atomistic_mlip_b200 import e2f
    wl = helpers.cached_workload(cfg, "bf16" if cfg else "fp32")
    pos = torch.from_numpy(wl.pos).cuda()
    cap = 128 * wl.N
    code, rp_ref, col_ref = _call("e2f_build_neighbors", pos, wl.box, wl.r_c, cap)
    assert code == 0
    e2f.scratch_high_water(reset=True)
    for _ in range(2):
        code, rp, col = _call("e2f_build_neighbors_noalloc", pos, wl.box, wl.r_c, cap)
        assert code == 0
        np.testing.assert_array_equal(rp, rp_ref)
        np.testing.assert_array_equal(col, col_ref)
    # nothing was taken from the library's memory pool
    assert e2f.scratch_high_water() == 0


def test_noalloc_limits(cuda_ok):
    import torch
    big = torch.zeros((131073, 3), dtype=torch.float32, device="cuda")
    code, _, _ = _call("e2f_build_neighbors_noalloc", big, None, 1.0, 16)
    assert code == 8
    # a sparse open system needs more than the cell limit before coarsening
    rng = np.random.default_rng(4)
    pos_np = rng.uniform(-3e3, 3e3, (20000, 3)).astype(np.float32)
    pos = torch.from_numpy(pos_np).cuda()
    c1, rp1, col1 = _call("e2f_build_neighbors", pos, None, 60.0, 1 << 20)
    c2, rp2, col2 = _call("e2f_build_neighbors_noalloc", pos, None, 60.0, 1 << 20)
    assert c1 == 0 and c2 == 0
    np.testing.assert_array_equal(rp1, rp2)
    np.testing.assert_array_equal(col1, col2)


def test_noalloc_sparse_periodic_box(cuda_ok):
    """A sparse periodic box whose natural cell grid (166^3 cells) is far
    above the fixed scratch's cell limit: the no-allocation build coarsens
    every periodic dimension at once and still gives the brute-force CSR,
    bit for bit, and the same CSR as the standard build."""
    import torch
    from oracle import neighbors as nb
    rng = np.random.default_rng(12)
    box = np.full(3, 1000.0, np.float32)
    pos_np = rng.uniform(0, 1000.0, (10000, 3)).astype(np.float32)
    # a few close pairs so that the graph is not empty
    pos_np[1::50] = np.mod(pos_np[0::50] + rng.uniform(-3, 3, pos_np[0::50].shape), 1000.0).astype(np.float32)
    pos_np[pos_np >= 1000.0] = 0.0
    pos = torch.from_numpy(pos_np).cuda()
    rp_o, col_o = nb.neighbors(pos_np, box, 6.0)
    assert rp_o[-1] > 0
    c1, rp1, col1 = _call("e2f_build_neighbors", pos, box, 6.0, 1 << 16)
    for _ in range(2):
        c2, rp2, col2 = _call("e2f_build_neighbors_noalloc", pos, box, 6.0, 1 << 16)
        assert c1 == 0 and c2 == 0
        np.testing.assert_array_equal(rp2, rp_o)
        np.testing.assert_array_equal(col2, col_o)
        np.testing.assert_array_equal(rp2, rp1)
        np.testing.assert_array_equal(col2, col1)


def test_noalloc_water_100k_vs_oracle(cuda_ok):
    """The 100,002-atom periodic water box (below the 131,072-atom limit)
    against the oracle's all-pairs CSR, twice in a row."""
    import torch
    wl = helpers.cached_workload(4, "bf16")
    rp_o, col_o = helpers.oracle_csr(4)
    pos = torch.from_numpy(wl.pos).cuda()
    for _ in range(2):
        code, rp, col = _call("e2f_build_neighbors_noalloc", pos, wl.box, wl.r_c, 128 * wl.N)
        assert code == 0
        np.testing.assert_array_equal(rp, rp_o)
        np.testing.assert_array_equal(col, col_o)
