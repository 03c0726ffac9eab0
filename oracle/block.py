"""The E2Former-V2 block around the attention, fp64: merged equivariant RMS
layer norm, node feed-forward network with a scalar-gated (SwiGLU-style)
activation, and pre-norm residual connections.

Test infrastructure only (see the package docstring).

What the pages fix and the readings taken where they do not:

* Merged layer norm ("EquiformerV3 ..." technical summary §2B.1,
  "Normalización de Capa Equivariante Fusionada"): one root-mean-square
  statistic shared by all degrees l >= 0 instead of one per degree.  Reading:
  the mean of x^2 over all (l, m, c) entries of the node, eps = 1e-6 inside
  the root, then a learnable gain per (degree, channel) and no bias (a bias
  on l >= 1 would break equivariance; none is used on l = 0 either).

      rms_n = sqrt(mean_{l,m,c} x[n,(l,m),c]^2 + eps)
      y[n,(l,m),c] = gamma[l,c] * x[n,(l,m),c] / rms_n

* Node FFN (§2B.2: hidden width 4x the channel width; §2C SwiGLU-S2: the
  non-linear gate acts on the scalar (l = 0) features only).  The spherical
  grid half of SwiGLU-S2 (projection to S^2 and bilinear products there) is
  out of scope; the reading kept is its scalar gate: with Hd = 4 C,

      gate[n]      = SiLU(Wa x[n,(0,0)])                      (Hd, invariant)
      h[n,(l,m)]   = gate[n] * (Wb[l] x[n,(l,m)])             (Hd, every l, m)
      out[n,(l,m)] = Wd[l] h[n,(l,m)]                         (C)

  Wa: [Hd][C], Wb[l]: [Hd][C], Wd[l]: [C][Hd], out x in, no biases.  Every
  degree is mixed only along channels and scaled by an invariant, so the
  map is equivariant.

* Block (pre-norm, residual): x1 = x + Attn(Norm1(x));  x2 = x1 + FFN(Norm2(x1)),
  with Attn the on-the-fly attention of ``oracle.attention`` (its own
  weights) on the positions' radius graph.  A multi-layer forward applies
  blocks with independent weights in turn; positions and graph are fixed.
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import numpy as np

from . import attention as oa

RMS_EPS = 1e-6


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def merged_rms_norm(x: np.ndarray, gamma: np.ndarray, L: int, eps: float = RMS_EPS) -> np.ndarray:
    """x [N, Q, C], gamma [L+1, C] -> [N, Q, C] (fp64)."""
    x = np.asarray(x, np.float64)
    ms = np.mean(x * x, axis=(1, 2))
    inv = 1.0 / np.sqrt(ms + eps)
    out = np.empty_like(x)
    g = np.asarray(gamma, np.float64)
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) * (l + 1))
        out[:, sl, :] = x[:, sl, :] * inv[:, None, None] * g[l][None, None, :]
    return out


def ffn(x: np.ndarray, Wa: np.ndarray, Wb: Sequence[np.ndarray], Wd: Sequence[np.ndarray], L: int) -> np.ndarray:
    """Scalar-gated node FFN: x [N, Q, C] -> [N, Q, C] (fp64)."""
    x = np.asarray(x, np.float64)
    gate = silu(x[:, 0, :] @ np.asarray(Wa, np.float64).T)          # [N, Hd]
    out = np.empty_like(x)
    for l in range(L + 1):
        sl = slice(l * l, (l + 1) * (l + 1))
        h = (x[:, sl, :] @ np.asarray(Wb[l], np.float64).T) * gate[:, None, :]
        out[:, sl, :] = h @ np.asarray(Wd[l], np.float64).T
    return out


def block_forward(pos, box, r_c, csr, x, lw: Dict, nodes=None, round_bf16: bool = False) -> np.ndarray:
    """One block: x [N, Q, C] -> x2 (fp64), rows ``nodes`` (default all).

    ``lw`` holds the layer's attention weights (Wq, Wk, Wv, W0, Wr, Wi,
    rad_W1, rad_W2, L, C, H) and block weights (gamma1, gamma2, Wa, Wb, Wd).
    With ``nodes`` the attention runs on those destination rows only (its
    inputs are the normalised features of every node).  ``round_bf16``
    rounds the two normalised feature tensors to bfloat16, the storage
    precision of the bf16 path (both sides then consume the same values)."""
    L, C, H = lw["L"], lw["C"], lw["H"]
    x = np.asarray(x, np.float64)
    xn = merged_rms_norm(x, lw["gamma1"], L)
    if round_bf16:
        xn = _round_bf16(xn)
    a = oa.attention(pos, box, r_c, csr[0], csr[1], xn, lw["Wq"], lw["Wk"], lw["Wv"], lw["W0"], lw["Wr"],
                     lw["Wi"], lw["rad_W1"], lw["rad_W2"], L, C, H, nodes=nodes)
    rows = np.arange(x.shape[0]) if nodes is None else np.asarray(nodes)
    x1 = x[rows] + a
    yn = merged_rms_norm(x1, lw["gamma2"], L)
    if round_bf16:
        yn = _round_bf16(yn)
    return x1 + ffn(yn, lw["Wa"], lw["Wb"], lw["Wd"], L)


def _round_bf16(a: np.ndarray) -> np.ndarray:
    """Round to bfloat16 (nearest, ties to even), returned as float64: the
    storage precision the bf16 path keeps the normalised features in."""
    f = np.asarray(a, np.float64).astype(np.float32)
    u = f.view(np.uint32).copy()
    u += np.uint32(0x7FFF) + ((u >> 16) & 1)
    return ((u >> 16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def model_forward(pos, box, r_c, csr, x, layers: List[Dict], round_bf16: bool = False) -> np.ndarray:
    """Blocks applied in turn (every row)."""
    for lw in layers:
        x = block_forward(pos, box, r_c, csr, x, lw, round_bf16=round_bf16)
    return x
