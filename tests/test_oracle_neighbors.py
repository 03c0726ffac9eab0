"""Pins of the brute-force neighbour oracle (P13): three independent
evaluations of the same predicate agree, and the CSR has the structure the
definition forces (symmetric, no self edges, ascending rows)."""
import numpy as np
import pytest

from atomistic_mlip_b200 import workloads as wlmod
from oracle import neighbors as nb


def _python_pairs(pos, box, rc):
    """Pure-Python double loop with numpy float32 scalars (tiny inputs)."""
    f = np.float32
    n = len(pos)
    rows = []
    for i in range(n):
        row = []
        for j in range(n):
            if i == j:
                continue
            d = [f(pos[j, k]) - f(pos[i, k]) for k in range(3)]
            if box is not None:
                for k in range(3):
                    b = f(box[k])
                    if d[k] > f(0.5) * b:
                        d[k] = d[k] - b
                    elif d[k] < -(f(0.5) * b):
                        d[k] = d[k] + b
            r2 = (d[0] * d[0] + d[1] * d[1]) + d[2] * d[2]
            if r2 < f(rc) * f(rc):
                row.append(j)
        rows.append(row)
    return rows


def _check_csr_structure(row_ptr, col, n):
    assert row_ptr[0] == 0 and row_ptr[-1] == len(col)
    assert np.all(np.diff(row_ptr) >= 0)
    pairs = set()
    for i in range(n):
        row = col[row_ptr[i]:row_ptr[i + 1]]
        assert np.all(np.diff(row) > 0), "rows ascending, no duplicates"
        assert i not in row
        pairs.update((i, int(j)) for j in row)
    assert all((j, i) in pairs for (i, j) in pairs), "symmetric"


@pytest.mark.parametrize("periodic", [False, True])
def test_tiny_random_three_ways(periodic):
    rng = np.random.default_rng(7)
    box = np.array([7.0, 8.0, 9.0], np.float32) if periodic else None
    pos = (rng.uniform(0, 1, (60, 3)) * (box if periodic else 8.0)).astype(np.float32)
    rc = 3.1
    rp_a, col_a = nb.neighbors_numpy(pos, box, rc)
    rp_b, col_b = nb.neighbors_c(pos, box, rc)
    rows = _python_pairs(pos, box, rc)
    np.testing.assert_array_equal(rp_a, rp_b)
    np.testing.assert_array_equal(col_a, col_b)
    for i in range(60):
        assert list(col_a[rp_a[i]:rp_a[i + 1]]) == rows[i]
    _check_csr_structure(rp_a, col_a, 60)


def test_strict_cutoff_and_exact_rounding():
    """A pair exactly at r_c is excluded; one just inside (in fp32) is kept."""
    rc = np.float32(2.0)
    inside = np.nextafter(np.float32(2.0), np.float32(0))
    pos = np.array([[0, 0, 0], [2.0, 0, 0], [0, inside, 0], [10, 10, 10]], np.float32)
    rp, col = nb.neighbors_numpy(pos, None, float(rc))
    assert list(col[rp[0]:rp[1]]) == [2]
    assert list(col[rp[3]:rp[4]]) == []


def test_minimum_image_wraps():
    box = np.array([10.0, 10.0, 10.0], np.float32)
    pos = np.array([[0.2, 5, 5], [9.9, 5, 5], [5, 5, 5]], np.float32)
    rp, col = nb.neighbors_numpy(pos, box, 1.0)
    assert list(col[rp[0]:rp[1]]) == [1]
    assert list(col[rp[1]:rp[2]]) == [0]
    assert rp[3] - rp[2] == 0


def test_empty_and_single():
    rp, col = nb.neighbors_numpy(np.zeros((0, 3), np.float32), None, 1.0)
    assert list(rp) == [0] and len(col) == 0
    rp, col = nb.neighbors_numpy(np.zeros((1, 3), np.float32), None, 1.0)
    assert list(rp) == [0, 0] and len(col) == 0


def test_coincident_atoms_are_neighbours():
    pos = np.array([[1, 1, 1], [1, 1, 1]], np.float32)
    rp, col = nb.neighbors_numpy(pos, None, 1.0)
    assert list(col) == [1, 0]


@pytest.mark.parametrize("cfg", [0, 2])
def test_workload_graphs_c_equals_numpy(cfg):
    wl = wlmod.make_workload(cfg)
    a = nb.neighbors_numpy(wl.pos, wl.box, wl.r_c)
    b = nb.neighbors_c(wl.pos, wl.box, wl.r_c)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])
    _check_csr_structure(*a, wl.N)
    if cfg == 2:
        # ~90 neighbours per atom at 0.1 atoms/A^3 and r_c = 6 A
        assert 80 < len(a[1]) / wl.N < 95


def test_neighbor_rows_match_full_brute_force():
    """The sampled-rows CSR lists, for every sampled row, exactly the full
    brute-force row (open and periodic), and nothing for the other rows."""
    from atomistic_mlip_b200 import workloads as w
    for cfg in (0, 2):
        wl = w.make_workload(cfg, C=8, L=1, H=1)
        rp, col = nb.neighbors(wl.pos, wl.box, wl.r_c)
        rows = np.random.default_rng(3).choice(wl.N, size=min(17, wl.N), replace=False)
        rp2, col2 = nb.neighbor_rows(wl.pos, wl.box, wl.r_c, rows)
        for i in range(wl.N):
            got = col2[rp2[i]:rp2[i + 1]]
            if i in set(rows.tolist()):
                assert np.array_equal(got, col[rp[i]:rp[i + 1]])
            else:
                assert len(got) == 0
