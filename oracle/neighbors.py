"""Brute-force radius graph (CSR), exact fp32 predicate.

Test infrastructure only.  Every pair (i, j), i != j, is tested; there is
no cell list, so nothing is shared with the GPU builder.  The predicate
(minimum image in fp32, r2 = (dx*dx + dy*dy) + dz*dz rounded after each
operation, strict r2 < r_c*r_c) is the rounding rule this project fixes for
the neighbour set j in N(i) that E2Former-V2's attention streams over
("E2Former-V2 ..." summary, §2.2 "Streaming reduction"; the pages give the
set, not its rounding).  NumPy float32 element-wise operations round each
result, exactly like the C loop compiled with -ffp-contract=off.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "neighbors_bf.c")
_LIB = os.path.join(_HERE, "_neighbors_bf.so")


def build_c_oracle(force: bool = False) -> str:
    """Compile the plain-C all-pairs loop (gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", _LIB, _SRC])
    return _LIB


def _box_args(box: Optional[np.ndarray]):
    if box is None:
        return np.ones(3, np.float32), np.zeros(3, np.int32)
    b = np.asarray(box, dtype=np.float32)
    return b, (b > 0).astype(np.int32)


def _pair_mask(pos: np.ndarray, rows: np.ndarray, box: Optional[np.ndarray], r_c: float):
    """Boolean [len(rows), N] adjacency for the given rows (float32 ops)."""
    b, per = _box_args(box)
    half = np.float32(0.5) * b
    d = pos[None, :, :] - pos[rows][:, None, :]          # float32 - float32
    for k in range(3):
        if per[k]:
            dk = d[..., k]
            hi = dk > half[k]
            lo = dk < -half[k]
            dk[hi] = dk[hi] - b[k]
            dk[lo] = dk[lo] + b[k]
    sq = d * d
    r2 = (sq[..., 0] + sq[..., 1]) + sq[..., 2]
    rc = np.float32(r_c)
    mask = r2 < rc * rc
    mask[np.arange(len(rows)), rows] = False
    return mask


def neighbors_numpy(pos: np.ndarray, box: Optional[np.ndarray], r_c: float,
                    block: int = 2048) -> Tuple[np.ndarray, np.ndarray]:
    """All-pairs CSR in NumPy (rows of `block` at a time)."""
    pos = np.ascontiguousarray(pos, dtype=np.float32)
    n = pos.shape[0]
    cols, degs = [], []
    for r0 in range(0, n, block):
        rows = np.arange(r0, min(n, r0 + block))
        m = _pair_mask(pos, rows, box, r_c)
        degs.append(m.sum(axis=1))
        cols.append(np.nonzero(m)[1].astype(np.int32))   # row-major: ascending j per row
    deg = np.concatenate(degs) if degs else np.zeros(0, np.int64)
    row_ptr = np.zeros(n + 1, np.int64)
    np.cumsum(deg, out=row_ptr[1:])
    col = np.concatenate(cols) if cols else np.zeros(0, np.int32)
    return row_ptr, col


def neighbors_c(pos: np.ndarray, box: Optional[np.ndarray], r_c: float) -> Tuple[np.ndarray, np.ndarray]:
    """All-pairs CSR through the plain-C loop (for large N)."""
    lib = ctypes.CDLL(build_c_oracle())
    pos = np.ascontiguousarray(pos, dtype=np.float32)
    n = pos.shape[0]
    b, per = _box_args(box)
    fp = ctypes.POINTER(ctypes.c_float)
    ip = ctypes.POINTER(ctypes.c_int)
    lp = ctypes.POINTER(ctypes.c_int64)
    deg = np.zeros(n, np.int64)
    lib.oracle_bf_count(pos.ctypes.data_as(fp), ctypes.c_int64(n), b.ctypes.data_as(fp),
                        per.ctypes.data_as(ip), ctypes.c_float(r_c), deg.ctypes.data_as(lp))
    row_ptr = np.zeros(n + 1, np.int64)
    np.cumsum(deg, out=row_ptr[1:])
    col = np.zeros(int(row_ptr[-1]), np.int32)
    lib.oracle_bf_fill(pos.ctypes.data_as(fp), ctypes.c_int64(n), b.ctypes.data_as(fp),
                       per.ctypes.data_as(ip), ctypes.c_float(r_c), row_ptr.ctypes.data_as(lp),
                       col.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
    return row_ptr, col


def neighbor_rows(pos: np.ndarray, box: Optional[np.ndarray], r_c: float,
                  rows: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Brute-force CSR that lists only the given rows (every other row is
    empty): row i of it equals row i of the full radius graph for i in
    `rows`.  For sampled destination rows of a large system."""
    pos = np.ascontiguousarray(pos, dtype=np.float32)
    n = pos.shape[0]
    rows = np.unique(np.asarray(rows, np.int64))
    deg = np.zeros(n, np.int64)
    cols = []
    for r0 in range(0, len(rows), 256):
        rr = rows[r0:r0 + 256]
        m = _pair_mask(pos, rr, box, r_c)
        deg[rr] = m.sum(axis=1)
        cols.append(np.nonzero(m)[1].astype(np.int32))
    row_ptr = np.zeros(n + 1, np.int64)
    np.cumsum(deg, out=row_ptr[1:])
    col = np.concatenate(cols) if cols else np.zeros(0, np.int32)
    return row_ptr, col


def neighbors(pos, box, r_c):
    """CSR (row_ptr int64 [N+1], col int32 [E]); C loop above 4096 atoms."""
    if np.asarray(pos).shape[0] > 4096:
        return neighbors_c(pos, box, r_c)
    return neighbors_numpy(pos, box, r_c)


def min_image(pos: np.ndarray, box: Optional[np.ndarray], i: np.ndarray, j: np.ndarray) -> np.ndarray:
    """r_ij = p_j - p_i in fp64 from the fp32 positions, minimum-imaged with
    the same > b/2 / < -b/2 rule as the predicate."""
    p = np.asarray(pos, dtype=np.float64)
    d = p[j] - p[i]
    if box is not None:
        b = np.asarray(box, dtype=np.float64)
        for k in range(3):
            if b[k] > 0:
                dk = d[..., k]
                dk[dk > 0.5 * b[k]] -= b[k]
                dk[dk < -0.5 * b[k]] += b[k]
    return d
