"""Seeded synthetic workloads for the on-the-fly equivariant attention path.

This module only *draws inputs*: atom positions, node features and weight
matrices, rounded once to the storage precision.  It holds none of the
operator's arithmetic and is shared by the CUDA path, the oracle, the tests
and the benchmark, so that both sides see the very same numbers.

Workloads (shapes follow the systems the E2Former-V2 summaries talk about:
drug-like molecules, liquid water, a ~30k-atom solvated protein and the
100k-atom scaling claim -- "E2Former-V2: On-the-Fly Equivariant Attention
with Linear Activation Memory", §4 "Experimental results"):

  0  24 random atoms in a 6 A cube (min distance 0.9 A), open, r_c = 5,
     L=2, C=8, H=1                                      (correctness case)
  1  256 tree-grown molecules of 20-60 atoms on a separated grid, open,
     r_c = 6, L=4, C=128, H=8                           (benchmark case)
  2  1,000 rigid waters in a 31 A periodic box, r_c = 6, L=4, C=128, H=8
  3  3,000-atom compact chain + 9,000 waters in a 66.94 A periodic box,
     r_c = 6, L=6, C=128, H=8
  4  33,334 waters in a 100.0007 A periodic box (N = 100,002), r_c = 6,
     L=4, C=128, H=8; plus the same recipe at 10k / 30k atoms for the
     memory sweep.

Random draw order per workload (numpy PCG64, seed 12345 + k): positions;
x; (Wq, Wk, Wv) for l = 0..L; W0; (Wr_m, Wi_m) for m = 1..L; rad_W1;
rad_W2; the 1,000-node subset.  x ~ N(0, 1); every weight ~ N(0, 1/fan_in)
with fan_in = C (q/k/v), n0 (W0), 2 n_m (Wr_m, Wi_m), 8 (rad_W1),
16 (rad_W2), where n_m = (L - m + 1) C.

Storage precision: 'fp32' rounds the float64 draws to float32 (RN);
'bf16' rounds to float32 then to bfloat16 (RN-even) for x, Wq/Wk/Wv, W0,
Wr, Wi, while positions and the radial MLP stay float32.  The stored values
are the inputs of both the GPU path and the oracle.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

BASE_SEED = 12345
WATER_OH = 0.96              # A
WATER_HOH_DEG = 104.5        # degrees
DENSITY = 0.1                # atoms / A^3


# ----------------------------------------------------------------------------
# bf16 storage helpers (bit manipulation only)
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even) and
    return the 16-bit patterns as uint16.  Inf/NaN do not occur in the draws."""
    u = np.array(a, dtype=np.float32, copy=True).view(np.uint32)
    lsb = (u >> 16) & 1
    u += np.uint32(0x7FFF)
    u += lsb
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def round_to(a: np.ndarray, precision: str) -> np.ndarray:
    """float64 draws -> the stored value, returned as float32 (exact)."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    if precision == "fp32":
        return f
    if precision == "bf16":
        return bf16_bits_to_f32(f32_to_bf16_bits(f))
    raise ValueError(f"unknown precision {precision!r}")


# ----------------------------------------------------------------------------
# Random rotations (input generation for the equivariance tests)
# ----------------------------------------------------------------------------
def haar_rotation(rng: np.random.Generator) -> np.ndarray:
    """Uniform (Haar) random proper rotation: QR of a Gaussian 3x3 with the
    sign of R's diagonal fixed, then det forced to +1."""
    g = rng.standard_normal((3, 3))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q


def cube_rotations() -> List[np.ndarray]:
    """The 24 proper rotations of the cube (signed axis permutations, det +1)."""
    out = []
    for perm in ([0, 1, 2], [0, 2, 1], [1, 0, 2], [1, 2, 0], [2, 0, 1], [2, 1, 0]):
        for sx in (1, -1):
            for sy in (1, -1):
                for sz in (1, -1):
                    m = np.zeros((3, 3))
                    for row, (col, s) in enumerate(zip(perm, (sx, sy, sz))):
                        m[row, col] = s
                    if np.linalg.det(m) > 0:
                        out.append(m)
    return out


def wrap_into_box(p: np.ndarray, box: np.ndarray) -> np.ndarray:
    """float64 positions -> float32 positions in [0, b) per periodic axis."""
    b32 = box.astype(np.float32)
    q = np.mod(p, box[None, :]).astype(np.float32)
    for k in range(3):
        col = q[:, k]
        col[col >= b32[k]] -= b32[k]
        col[col < 0] = 0.0
    return q


# ----------------------------------------------------------------------------
# Geometry generators
# ----------------------------------------------------------------------------
def _random_unit(rng: np.random.Generator) -> np.ndarray:
    v = rng.standard_normal(3)
    return v / np.linalg.norm(v)


def gen_random_cluster(rng, n=24, edge=6.0, dmin=0.9) -> np.ndarray:
    """n points uniform in [0, edge)^3, sequential rejection to min distance."""
    pts: List[np.ndarray] = []
    while len(pts) < n:
        c = rng.uniform(0.0, edge, size=3)
        if all(np.linalg.norm(c - p) >= dmin for p in pts):
            pts.append(c)
    return np.array(pts)


def gen_molecule(rng, n_atoms, bond=(1.0, 1.6), dmin=1.0) -> np.ndarray:
    """Tree-grown molecule: each new atom hangs off a uniformly chosen parent
    at a uniform direction and a U(1.0, 1.6) A bond; rejected if it comes
    within dmin of any placed atom."""
    pts = [np.zeros(3)]
    while len(pts) < n_atoms:
        parent = pts[rng.integers(len(pts))]
        c = parent + rng.uniform(*bond) * _random_unit(rng)
        arr = np.array(pts)
        if np.min(np.linalg.norm(arr - c[None, :], axis=1)) >= dmin:
            pts.append(c)
    return np.array(pts)


def gen_molecule_batch(rng, n_mol=256, n_range=(20, 60), r_c=6.0):
    """Molecules centred at their centroids and placed on a cubic grid
    (site k -> (k mod 7, k//7 mod 7, k//49)) with spacing = max bounding-
    sphere diameter + r_c + 1 A, so no pair of atoms from different molecules
    is within r_c."""
    mols = [gen_molecule(rng, int(rng.integers(n_range[0], n_range[1] + 1)))
            for _ in range(n_mol)]
    mols = [m - m.mean(axis=0, keepdims=True) for m in mols]
    extent = 2.0 * max(float(np.max(np.linalg.norm(m, axis=1))) for m in mols)
    spacing = extent + r_c + 1.0
    out = []
    for k, m in enumerate(mols):
        site = np.array([k % 7, (k // 7) % 7, k // 49], dtype=np.float64)
        out.append(m + (site + 0.5) * spacing)
    sizes = np.array([len(m) for m in mols])
    return np.concatenate(out, axis=0), sizes, spacing


def _water_sites(rng, n_side, box):
    a = box / n_side
    idx = np.stack(np.meshgrid(np.arange(n_side), np.arange(n_side),
                               np.arange(n_side), indexing="ij"), -1).reshape(-1, 3)
    centres = (idx + 0.5) * a
    jitter = rng.uniform(-0.2 * a, 0.2 * a, size=centres.shape)
    return centres + jitter


def _water_atoms(rng, oxygens):
    """O, H, H for each oxygen; Haar-random orientation per unit (one batched
    draw of Gaussian 3x3 matrices, QR with the sign of R's diagonal fixed,
    det forced to +1)."""
    ang = math.radians(WATER_HOH_DEG)
    n = len(oxygens)
    g = rng.standard_normal((n, 3, 3))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diagonal(r, axis1=1, axis2=2))[:, None, :]
    neg = np.linalg.det(q) < 0
    q[neg, :, 0] = -q[neg, :, 0]
    e1 = np.array([1.0, 0.0, 0.0])
    e2 = np.array([math.cos(ang), math.sin(ang), 0.0])
    out = np.empty((n, 3, 3))
    out[:, 0] = oxygens
    out[:, 1] = oxygens + WATER_OH * (q @ e1)
    out[:, 2] = oxygens + WATER_OH * (q @ e2)
    return out.reshape(3 * n, 3)


def gen_water_box(rng, n_units, box):
    """Jittered cubic lattice with ceil(units^(1/3)) sites per side, a seeded
    subset of n_units sites, one rigid water per site."""
    n_side = int(math.ceil(round(n_units ** (1.0 / 3.0), 9)))
    while n_side ** 3 < n_units:
        n_side += 1
    sites = _water_sites(rng, n_side, box)
    if len(sites) > n_units:
        sites = sites[np.sort(rng.permutation(len(sites))[:n_units])]
    return _water_atoms(rng, sites)


def gen_solvated_chain(rng, n_chain=3000, n_water=9000, box=None,
                       step=1.5, dmin=1.2, max_tries=1000):
    """Compact self-avoiding chain in a core sphere plus lattice waters.

    Chain: starts at the box centre; 1.5 A steps in uniform directions;
    a step is rejected if it lands within 1.2 A of an earlier atom or outside
    the core sphere R = (3 n_chain / (4 pi rho))^(1/3); after max_tries
    rejections the last atom is removed (backtrack).
    Waters: jittered cubic lattice over the box; sites whose O lies within
    R + 1.5 A of the centre are dropped; the lattice is refined (one more
    site per side) until at least n_water sites remain; n_water sites are
    chosen by seeded permutation."""
    centre = box / 2.0
    radius = (3.0 * n_chain / (4.0 * math.pi * DENSITY)) ** (1.0 / 3.0)
    chain = [centre.copy()]
    tries = 0
    while len(chain) < n_chain:
        c = chain[-1] + step * _random_unit(rng)
        arr = np.array(chain)
        ok = (np.linalg.norm(c - centre) <= radius and
              np.min(np.linalg.norm(arr - c[None, :], axis=1)) >= dmin)
        if ok:
            chain.append(c)
            tries = 0
        else:
            tries += 1
            if tries >= max_tries and len(chain) > 1:
                chain.pop()
                tries = 0
    chain = np.array(chain)
    n_side = int(math.ceil(round(n_water ** (1.0 / 3.0), 9)))
    while True:
        sites = _water_sites(rng, n_side, box)
        keep = np.linalg.norm(sites - centre[None, :], axis=1) > radius + 1.5
        if keep.sum() >= n_water:
            break
        n_side += 1
    sites = sites[keep]
    sites = sites[np.sort(rng.permutation(len(sites))[:n_water])]
    return np.concatenate([chain, _water_atoms(rng, sites)], axis=0)


# ----------------------------------------------------------------------------
# Workload container
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class Workload:
    name: str
    cfg: int
    precision: str
    pos: np.ndarray                 # float32 [N, 3]
    box: Optional[np.ndarray]       # float32 [3] (periodic) or None (open)
    r_c: float                      # stored as a float32 value
    L: int
    C: int
    H: int
    x: np.ndarray                   # float32 [N, Q, C] (values exact in the storage type)
    Wq: List[np.ndarray]            # float32 [C, C] per l, out x in
    Wk: List[np.ndarray]
    Wv: List[np.ndarray]
    W0: np.ndarray                  # [n0, n0]
    Wr: List[Optional[np.ndarray]]  # index m = 1..L, [n_m, n_m]; Wr[0] is None
    Wi: List[Optional[np.ndarray]]
    rad_W1: np.ndarray              # float32 [16, 8]
    rad_W2: np.ndarray              # float32 [P, 16]
    subset: np.ndarray              # int64 sorted node subset (oracle sampling)
    seed: int
    meta: Dict

    @property
    def N(self) -> int:
        return int(self.pos.shape[0])

    @property
    def Q(self) -> int:
        return (self.L + 1) ** 2

    @property
    def P(self) -> int:
        return (self.L + 1) * (self.L + 2) // 2

    def n_m(self, m: int) -> int:
        return (self.L - m + 1) * self.C


def _normal_rows(rng, shape, precision, rows_per_chunk=4096):
    """rng.standard_normal(shape) rounded to the storage type, drawn in row
    chunks (the same numbers as one draw) to bound host memory."""
    out = np.empty(shape, dtype=np.float32)
    for r0 in range(0, shape[0], rows_per_chunk):
        r1 = min(shape[0], r0 + rows_per_chunk)
        out[r0:r1] = round_to(rng.standard_normal((r1 - r0,) + tuple(shape[1:])), precision)
    return out


def _draw_features_and_weights(rng, N, L, C, precision):
    Q = (L + 1) ** 2
    x = _normal_rows(rng, (N, Q, C), precision)
    Wq, Wk, Wv = [], [], []
    for _ in range(L + 1):
        for lst in (Wq, Wk, Wv):
            lst.append(round_to(rng.standard_normal((C, C)) / math.sqrt(C), precision))
    n0 = (L + 1) * C
    W0 = round_to(rng.standard_normal((n0, n0)) / math.sqrt(n0), precision)
    Wr: List[Optional[np.ndarray]] = [None]
    Wi: List[Optional[np.ndarray]] = [None]
    for m in range(1, L + 1):
        n = (L - m + 1) * C
        Wr.append(round_to(rng.standard_normal((n, n)) / math.sqrt(2 * n), precision))
        Wi.append(round_to(rng.standard_normal((n, n)) / math.sqrt(2 * n), precision))
    P = (L + 1) * (L + 2) // 2
    rad_W1 = rng.standard_normal((16, 8)).astype(np.float64) / math.sqrt(8)
    rad_W2 = rng.standard_normal((P, 16)).astype(np.float64) / math.sqrt(16)
    return (x, Wq, Wk, Wv, W0, Wr, Wi,
            rad_W1.astype(np.float32), rad_W2.astype(np.float32))


CONFIG_SPECS = {
    0: dict(L=2, C=8, H=1, r_c=5.0, precision="fp32"),
    1: dict(L=4, C=128, H=8, r_c=6.0, precision="bf16"),
    2: dict(L=4, C=128, H=8, r_c=6.0, precision="bf16"),
    3: dict(L=6, C=128, H=8, r_c=6.0, precision="bf16"),
    4: dict(L=4, C=128, H=8, r_c=6.0, precision="bf16"),
}


def water_box_size(n_atoms_target: int):
    units = -(-n_atoms_target // 3)
    n = 3 * units
    return units, n, (n / DENSITY) ** (1.0 / 3.0)


def make_positions(cfg: int, rng, n_target: Optional[int] = None):
    """Positions (float64) and box for a workload; the rng is advanced."""
    meta: Dict = {}
    if cfg == 0:
        return gen_random_cluster(rng), None, meta
    if cfg == 1:
        p, sizes, spacing = gen_molecule_batch(rng)
        meta.update(mol_sizes=sizes, spacing=spacing)
        return p, None, meta
    if cfg == 2:
        box = np.full(3, 31.0)
        return gen_water_box(rng, 1000, 31.0), box, meta
    if cfg == 3:
        b = (30000 / DENSITY) ** (1.0 / 3.0)
        box = np.full(3, b)
        return gen_solvated_chain(rng, box=box), box, meta
    if cfg == 4:
        units, _, b = water_box_size(n_target or 100000)
        box = np.full(3, b)
        return gen_water_box(rng, units, b), box, meta
    raise ValueError(cfg)


def make_workload(cfg: int, precision: Optional[str] = None, seed: Optional[int] = None,
                  n_target: Optional[int] = None, C: Optional[int] = None,
                  L: Optional[int] = None, H: Optional[int] = None,
                  subset_size: int = 1000) -> Workload:
    """Build workload `cfg` (0..4).  `n_target` picks the size of the water
    box for the memory sweep (cfg 4).  C/L/H overrides give reduced-width
    variants of the same geometry for fast tests."""
    spec = dict(CONFIG_SPECS[cfg])
    prec = precision or spec["precision"]
    Lv = spec["L"] if L is None else L
    Cv = spec["C"] if C is None else C
    Hv = spec["H"] if H is None else H
    sd = BASE_SEED + cfg if seed is None else seed
    rng = np.random.default_rng(sd)
    p64, box64, meta = make_positions(cfg, rng, n_target)
    if box64 is None:
        pos = p64.astype(np.float32)
        box = None
    else:
        pos = wrap_into_box(p64, box64)
        box = box64.astype(np.float32)
    N = pos.shape[0]
    (x, Wq, Wk, Wv, W0, Wr, Wi, w1, w2) = _draw_features_and_weights(rng, N, Lv, Cv, prec)
    k = min(subset_size, N)
    subset = np.sort(rng.choice(N, size=k, replace=False)).astype(np.int64)
    return Workload(name=f"cfg{cfg}", cfg=cfg, precision=prec, pos=pos, box=box,
                    r_c=float(np.float32(spec["r_c"])), L=Lv, C=Cv, H=Hv, x=x,
                    Wq=Wq, Wk=Wk, Wv=Wv, W0=W0, Wr=Wr, Wi=Wi, rad_W1=w1, rad_W2=w2,
                    subset=subset, seed=sd, meta=meta)


def make_layer_weights(L: int, C: int, H: int, precision: str, seed: int, hidden_mult: int = 4) -> Dict:
    """Weights of one E2Former-V2 block: the attention's (drawn as in
    make_workload) plus the two merged-norm gains (float32, 1 + 0.1 N(0, 1)
    per (degree, channel)) and the FFN maps Wa [Hd][C], Wb[l] [Hd][C],
    Wd[l] [C][Hd] (Hd = hidden_mult C, N(0, 1/fan_in)), seeded."""
    rng = np.random.default_rng(seed)
    (_, Wq, Wk, Wv, W0, Wr, Wi, w1, w2) = _draw_features_and_weights(rng, 0, L, C, precision)
    Hd = hidden_mult * C
    g1 = (1.0 + 0.1 * rng.standard_normal((L + 1, C))).astype(np.float32)
    g2 = (1.0 + 0.1 * rng.standard_normal((L + 1, C))).astype(np.float32)
    Wa = round_to(rng.standard_normal((Hd, C)) / math.sqrt(C), precision)
    Wb = [round_to(rng.standard_normal((Hd, C)) / math.sqrt(C), precision) for _ in range(L + 1)]
    Wd = [round_to(rng.standard_normal((C, Hd)) / math.sqrt(Hd), precision) for _ in range(L + 1)]
    return dict(L=L, C=C, H=H, precision=precision, Wq=Wq, Wk=Wk, Wv=Wv, W0=W0, Wr=Wr, Wi=Wi, rad_W1=w1,
                rad_W2=w2, gamma1=g1, gamma2=g2, Wa=Wa, Wb=Wb, Wd=Wd)


def cg_num_paths(L: int) -> int:
    """Coupling paths (l1, l2, l3) with 0 <= l1, l2, l3 <= L and
    |l1 - l2| <= l3 <= l1 + l2 (the row count of the CG-convolution weights)."""
    return sum(1 for l1 in range(L + 1) for l2 in range(L + 1) for l3 in range(L + 1)
               if abs(l1 - l2) <= l3 <= l1 + l2)


def make_cg_weights(L: int, C: int, seed: int) -> np.ndarray:
    """Channel-wise path weights of the CG convolution, float32
    [cg_num_paths(L)][C], N(0, 1) / sqrt(number of paths), seeded."""
    rng = np.random.default_rng(seed)
    n = cg_num_paths(L)
    return (rng.standard_normal((n, C)) / math.sqrt(n)).astype(np.float32)


def make_custom(pos: np.ndarray, box: Optional[np.ndarray], r_c: float, L: int, C: int,
                H: int, precision: str = "fp32", seed: int = 0) -> Workload:
    """Features and weights for caller-given positions (edge-case tests)."""
    rng = np.random.default_rng(seed)
    pos = np.asarray(pos, dtype=np.float32)
    N = pos.shape[0]
    (x, Wq, Wk, Wv, W0, Wr, Wi, w1, w2) = _draw_features_and_weights(rng, N, L, C, precision)
    return Workload(name="custom", cfg=-1, precision=precision, pos=pos,
                    box=None if box is None else np.asarray(box, np.float32),
                    r_c=float(np.float32(r_c)), L=L, C=C, H=H, x=x, Wq=Wq, Wk=Wk, Wv=Wv,
                    W0=W0, Wr=Wr, Wi=Wi, rad_W1=w1, rad_W2=w2,
                    subset=np.arange(min(N, 1000), dtype=np.int64), seed=seed, meta={})
