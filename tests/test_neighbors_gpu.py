"""GPU cell-list CSR == brute-force oracle, bit for bit (P13), on all five
workloads and on the edge cases of the builder."""
import numpy as np
import pytest

from oracle import neighbors as nb
from tests import helpers

pytestmark = pytest.mark.gpu


def _gpu_csr(pos, box, rc, capacity=None):
    import torch
    from atomistic_mlip_b200 import e2f
    p = torch.from_numpy(np.ascontiguousarray(pos, np.float32)).cuda()
    nl = e2f.build_neighbors(p, None if box is None else [float(b) for b in box], rc, capacity=capacity)
    torch.cuda.synchronize()
    rp = nl.row_ptr.cpu().numpy().astype(np.int64)
    col = nl.col_idx[: nl.n_edges].cpu().numpy()
    return rp, col


def _assert_same(pos, box, rc, capacity=None):
    rp, col = _gpu_csr(pos, box, rc, capacity)
    rp_o, col_o = nb.neighbors(pos, box, rc)
    np.testing.assert_array_equal(rp, rp_o)
    np.testing.assert_array_equal(col, col_o)
    return rp, col


@pytest.mark.parametrize("cfg", [0, 1, 2, 3, 4])
def test_workload_csr_bit_exact(cuda_ok, cfg):
    wl = helpers.cached_workload(cfg, "bf16" if cfg else "fp32")
    rp, col = _gpu_csr(wl.pos, wl.box, wl.r_c)
    rp_o, col_o = helpers.oracle_csr(cfg)
    np.testing.assert_array_equal(rp, rp_o)
    np.testing.assert_array_equal(col, col_o)


def test_empty_and_single(cuda_ok):
    rp, col = _gpu_csr(np.zeros((0, 3), np.float32), None, 2.0)
    assert list(rp) == [0] and len(col) == 0
    rp, col = _gpu_csr(np.ones((1, 3), np.float32), [5.0, 5.0, 5.0], 2.0)
    assert list(rp) == [0, 0]


def test_coincident_and_cell_faces(cuda_ok):
    # atoms exactly on multiples of the cutoff (cell faces) and duplicates
    g = np.arange(0, 24, 3.0, dtype=np.float32)
    pos = np.stack(np.meshgrid(g, g, g, indexing="ij"), -1).reshape(-1, 3)
    pos = np.concatenate([pos, pos[:7]]).astype(np.float32)
    _assert_same(pos, [24.0, 24.0, 24.0], 3.0)
    _assert_same(pos, None, 3.0)
    _assert_same(pos, None, 3.0000002)


def test_cutoff_close_to_half_box_and_small_grid(cuda_ok):
    rng = np.random.default_rng(0)
    pos = (rng.uniform(0, 1, (400, 3)) * [12.1, 14.0, 30.0]).astype(np.float32)
    _assert_same(pos, [12.1, 14.0, 30.0], 6.0)
    _assert_same(pos, [12.1, 0.0, 30.0], 6.0)      # mixed periodic / open


def test_sparse_open_system(cuda_ok):
    rng = np.random.default_rng(1)
    pos = (rng.uniform(-1e4, 1e4, (300, 3))).astype(np.float32)
    pos[:50] = rng.uniform(0, 5, (50, 3))
    _assert_same(pos, None, 2.5)


def test_long_rows_fallback(cuda_ok):
    """Rows longer than the shared-memory row buffer take the in-place sort."""
    rng = np.random.default_rng(2)
    pos = rng.uniform(0, 4.0, (900, 3)).astype(np.float32)
    rp, _ = _assert_same(pos, None, 6.0)
    assert np.max(np.diff(rp)) > 512


def test_capacity_overflow(cuda_ok):
    import ctypes
    import torch
    from atomistic_mlip_b200 import e2f
    wl = helpers.cached_workload(0, "fp32")
    p = torch.from_numpy(wl.pos).cuda()
    rp = torch.empty(wl.N + 1, dtype=torch.int32, device="cuda")
    guard = torch.full((64,), -7, dtype=torch.int32, device="cuda")
    n_e = ctypes.c_int64(0)
    code = e2f.lib().e2f_build_neighbors(p.data_ptr(), wl.N, None, wl.r_c, rp.data_ptr(), guard.data_ptr(),
                                         10, ctypes.byref(n_e), None,
                                         torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert code == 3 and n_e.value == helpers.oracle_csr(0)[0][-1]
    assert torch.all(guard == -7)          # nothing written when E > capacity
    # the binding retries with the reported size
    _assert_same(wl.pos, None, wl.r_c, capacity=10)


def test_domain_error(cuda_ok):
    import torch
    from atomistic_mlip_b200 import e2f
    pos = torch.tensor([[1.0, 1.0, 1.0], [10.5, 1.0, 1.0]], device="cuda")
    with pytest.raises(e2f.E2FError) as ei:
        e2f.build_neighbors(pos, [10.0, 10.0, 10.0], 2.0)
    assert ei.value.code == 7
