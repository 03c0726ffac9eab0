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
