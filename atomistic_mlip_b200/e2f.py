"""Thin Python binding of libe2f (include/e2f.h) through ctypes.

Argument marshalling only: tensors are passed as raw device pointers and
the current torch CUDA stream as a cudaStream_t; every step of the path runs
in the library's kernels.  PyTorch is used for device memory and streams.

The library must have been built (``python -m atomistic_mlip_b200.build``);
loading raises if it is missing -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import List, Optional, Sequence

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libe2f.so")
MAX_L = 6
F32, BF16 = 0, 1

STATUS = {0: "ok", 1: "invalid argument", 2: "cutoff too large", 3: "capacity",
          4: "unsupported", 5: "CUDA error", 6: "timeout", 7: "domain", 8: "scratch limit"}


class E2FError(RuntimeError):
    def __init__(self, code: int, what: str, detail: str = ""):
        super().__init__(f"{what}: {STATUS.get(code, code)} ({code}) {detail}".rstrip())
        self.code = code


class Csr(ctypes.Structure):
    _fields_ = [("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p),
                ("n_nodes", ctypes.c_int64), ("n_edges", ctypes.c_int64),
                ("box", ctypes.c_float * 3), ("r_c", ctypes.c_float)]


_P7 = ctypes.c_void_p * (MAX_L + 1)


class Weights(ctypes.Structure):
    _fields_ = [("L_max", ctypes.c_int32), ("C", ctypes.c_int32), ("H", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("Wq", _P7), ("Wk", _P7), ("Wv", _P7),
                ("W0", ctypes.c_void_p), ("Wr", _P7), ("Wi", _P7),
                ("rad_W1", ctypes.c_void_p), ("rad_W2", ctypes.c_void_p)]


class BlockWeights(ctypes.Structure):
    _fields_ = [("attn", Weights), ("hidden", ctypes.c_int32), ("gamma1", ctypes.c_void_p),
                ("gamma2", ctypes.c_void_p), ("Wa", ctypes.c_void_p), ("Wb", _P7), ("Wd", _P7)]


# name -> (restype, argtypes); must match include/e2f.h
SIGNATURES = {
    "e2f_status_string": (ctypes.c_char_p, [ctypes.c_int32]),
    "e2f_last_cuda_error": (ctypes.c_char_p, []),
    "e2f_build_neighbors": (ctypes.c_int32, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                             ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(Csr),
                                             ctypes.c_void_p]),
    "e2f_build_neighbors_noalloc": (ctypes.c_int32, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                                     ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                                     ctypes.c_int64, ctypes.POINTER(ctypes.c_int64),
                                                     ctypes.POINTER(Csr), ctypes.c_void_p]),
    "e2f_attention_forward": (ctypes.c_int32, [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(Csr),
                                               ctypes.POINTER(Weights), ctypes.c_void_p, ctypes.c_void_p]),
    "e2f_attention_backward": (ctypes.c_int32, [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(Csr),
                                                ctypes.POINTER(Weights), ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p]),
    "e2f_block_forward": (ctypes.c_int32, [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(Csr),
                                           ctypes.POINTER(BlockWeights), ctypes.c_void_p, ctypes.c_void_p]),
    "e2f_attention_forward_multifocus": (ctypes.c_int32, [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(Csr),
                                                          ctypes.POINTER(Weights), ctypes.c_int32, ctypes.c_void_p,
                                                          ctypes.c_void_p, ctypes.c_void_p]),
    "e2f_cg_num_paths": (ctypes.c_int64, [ctypes.c_int32]),
    "e2f_cg_conv_forward": (ctypes.c_int32, [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.POINTER(Csr),
                                             ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_void_p]),
    "e2f_stream_status": (ctypes.c_int32, [ctypes.c_void_p]),
    "e2f_wigner_d": (ctypes.c_int32, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p,
                                      ctypes.c_void_p]),
    "e2f_project_qkv": (ctypes.c_int32, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(Weights),
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "e2f_kernel_launches": (ctypes.c_int64, []),
    "e2f_profile_enable": (ctypes.c_int32, [ctypes.c_int32]),
    "e2f_profile_read": (ctypes.c_int32, [ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_double)]),
    "e2f_scratch_high_water": (ctypes.c_int32, [ctypes.POINTER(ctypes.c_int64), ctypes.c_int32]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libe2f.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"libe2f.so not found at {_LIB_PATH}; build it with "
                              "`python -m atomistic_mlip_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code: int, what: str):
    if code != 0:
        detail = ""
        if code == 5:
            detail = lib().e2f_last_cuda_error().decode()
        raise E2FError(code, what, detail)


def _torch():
    import torch
    return torch


def _stream_ptr(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


# ----------------------------------------------------------------------------
# neighbour list
# ----------------------------------------------------------------------------
@dataclasses.dataclass
class NeighborList:
    row_ptr: "object"       # torch.int32 [N+1] cuda
    col_idx: "object"       # torch.int32 [capacity] cuda (first n_edges valid)
    n_edges: int
    box: Optional[Sequence[float]]
    r_c: float

    @property
    def n_nodes(self) -> int:
        return int(self.row_ptr.numel()) - 1

    def csr(self) -> Csr:
        c = Csr()
        c.row_ptr = self.row_ptr.data_ptr()
        c.col_idx = self.col_idx.data_ptr() if self.col_idx.numel() else None
        c.n_nodes = self.n_nodes
        c.n_edges = self.n_edges
        for k in range(3):
            c.box[k] = float(self.box[k]) if self.box is not None else 0.0
        c.r_c = self.r_c
        return c


def build_neighbors(pos, box: Optional[Sequence[float]], r_c: float, capacity: Optional[int] = None,
                    stream=None, row_ptr=None, col_idx=None) -> NeighborList:
    """CSR radius graph of `pos` (torch float32 [N, 3] on a CUDA device).

    Allocates row_ptr / col_idx with torch unless given; if col_idx is too
    small the call is repeated once with the exact size the library reports."""
    torch = _torch()
    N = int(pos.shape[0])
    dev = pos.device
    if row_ptr is None:
        row_ptr = torch.empty(N + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        cap = capacity if capacity is not None else max(1024, 128 * N)
        col_idx = torch.empty(cap, dtype=torch.int32, device=dev)
    box_arr = None
    if box is not None:
        box_arr = (ctypes.c_float * 3)(*[float(b) for b in box])
    n_e = ctypes.c_int64(0)
    s = _stream_ptr(stream)
    code = lib().e2f_build_neighbors(_ptr(pos), N, box_arr, float(r_c), _ptr(row_ptr),
                                     _ptr(col_idx) if col_idx.numel() else None, int(col_idx.numel()),
                                     ctypes.byref(n_e), None, s)
    if code == 3:
        col_idx = torch.empty(max(1, n_e.value), dtype=torch.int32, device=dev)
        code = lib().e2f_build_neighbors(_ptr(pos), N, box_arr, float(r_c), _ptr(row_ptr), _ptr(col_idx),
                                         int(col_idx.numel()), ctypes.byref(n_e), None, s)
    _check(code, "e2f_build_neighbors")
    return NeighborList(row_ptr, col_idx, int(n_e.value), None if box is None else list(box), float(r_c))


# ----------------------------------------------------------------------------
# weights
# ----------------------------------------------------------------------------
class DeviceWeights:
    """Device copies of the attention weights plus the e2f_weights struct."""

    def __init__(self, L: int, C: int, H: int, dtype: int, Wq: List, Wk: List, Wv: List, W0, Wr: List,
                 Wi: List, rad_W1, rad_W2):
        self.L, self.C, self.H, self.dtype = L, C, H, dtype
        self.tensors = dict(Wq=Wq, Wk=Wk, Wv=Wv, W0=W0, Wr=Wr, Wi=Wi, rad_W1=rad_W1, rad_W2=rad_W2)
        w = Weights()
        w.L_max, w.C, w.H, w.dtype = L, C, H, dtype
        for l in range(L + 1):
            w.Wq[l], w.Wk[l], w.Wv[l] = Wq[l].data_ptr(), Wk[l].data_ptr(), Wv[l].data_ptr()
        w.W0 = W0.data_ptr()
        for m in range(1, L + 1):
            w.Wr[m], w.Wi[m] = Wr[m].data_ptr(), Wi[m].data_ptr()
        w.rad_W1, w.rad_W2 = rad_W1.data_ptr(), rad_W2.data_ptr()
        self.struct = w

    @classmethod
    def from_workload(cls, wl, device="cuda", dtype: Optional[str] = None) -> "DeviceWeights":
        torch = _torch()
        prec = dtype or wl.precision
        td = torch.float32 if prec == "fp32" else torch.bfloat16
        code = F32 if prec == "fp32" else BF16

        def up(a, t=td):
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device, dtype=t)

        return cls(wl.L, wl.C, wl.H, code, [up(a) for a in wl.Wq], [up(a) for a in wl.Wk],
                   [up(a) for a in wl.Wv], up(wl.W0), [None] + [up(a) for a in wl.Wr[1:]],
                   [None] + [up(a) for a in wl.Wi[1:]], up(wl.rad_W1, torch.float32),
                   up(wl.rad_W2, torch.float32))

    @property
    def torch_dtype(self):
        torch = _torch()
        return torch.float32 if self.dtype == F32 else torch.bfloat16


# ----------------------------------------------------------------------------
# attention and unit entry points
# ----------------------------------------------------------------------------
def attention_forward(x, pos, nl: NeighborList, w: DeviceWeights, out=None, stream=None):
    """o = on-the-fly equivariant attention (float32 [N, Q, C])."""
    torch = _torch()
    N = int(pos.shape[0])
    Q = (w.L + 1) ** 2
    if out is None:
        out = torch.empty((N, Q, w.C), dtype=torch.float32, device=pos.device)
    csr = nl.csr()
    code = lib().e2f_attention_forward(_ptr(x), _ptr(pos), ctypes.byref(csr), ctypes.byref(w.struct),
                                       _ptr(out), _stream_ptr(stream))
    _check(code, "e2f_attention_forward")
    return out


def attention_forward_multifocus(x, pos, nl: NeighborList, w: DeviceWeights, F: int, focus_a, out=None,
                                 stream=None):
    """Multi-focus attention: F streams with their own SO(2) stacks,
    re-weighted per edge by a softmax over the streams (float32 [N, Q, C])."""
    torch = _torch()
    N = int(pos.shape[0])
    Q = (w.L + 1) ** 2
    if out is None:
        out = torch.empty((N, Q, w.C), dtype=torch.float32, device=pos.device)
    csr = nl.csr()
    code = lib().e2f_attention_forward_multifocus(_ptr(x), _ptr(pos), ctypes.byref(csr), ctypes.byref(w.struct),
                                                  int(F), _ptr(focus_a) if focus_a is not None else None,
                                                  _ptr(out), _stream_ptr(stream))
    _check(code, "e2f_attention_forward_multifocus")
    return out


def cg_num_paths(L: int) -> int:
    """Rows of the CG-convolution weights for degree L."""
    n = int(lib().e2f_cg_num_paths(int(L)))
    if n < 0:
        raise E2FError(1, "e2f_cg_num_paths", f"L = {L} out of range")
    return n


def cg_conv_forward(x, pos, nl: NeighborList, W, L: int, out=None, stream=None):
    """Re-indexed CG convolution of x (float32 or bfloat16 [N, (L+1)^2, C])
    with the harmonics of the edge directions; W float32 [cg_num_paths(L), C].
    Returns float32 [N, (L+1)^2, C]."""
    torch = _torch()
    N, Q, C = int(x.shape[0]), int(x.shape[1]), int(x.shape[2])
    if Q != (L + 1) ** 2:
        raise ValueError(f"x has {Q} components, L = {L} needs {(L + 1) ** 2}")
    dtype = F32 if x.dtype == torch.float32 else BF16
    if out is None:
        out = torch.empty((N, Q, C), dtype=torch.float32, device=pos.device)
    csr = nl.csr()
    code = lib().e2f_cg_conv_forward(_ptr(x), dtype, _ptr(pos), ctypes.byref(csr), int(L), C, _ptr(W), _ptr(out),
                                     _stream_ptr(stream))
    _check(code, "e2f_cg_conv_forward")
    return out


class DeviceBlockWeights:
    """Device copies of one block's weights (attention + merged norms + FFN)
    and the e2f_block_weights struct."""

    def __init__(self, attn: DeviceWeights, gamma1, gamma2, Wa, Wb: List, Wd: List):
        self.attn = attn
        self.tensors = dict(gamma1=gamma1, gamma2=gamma2, Wa=Wa, Wb=Wb, Wd=Wd)
        b = BlockWeights()
        b.attn = attn.struct
        b.hidden = int(Wa.shape[0])
        b.gamma1, b.gamma2, b.Wa = gamma1.data_ptr(), gamma2.data_ptr(), Wa.data_ptr()
        for l in range(attn.L + 1):
            b.Wb[l], b.Wd[l] = Wb[l].data_ptr(), Wd[l].data_ptr()
        self.struct = b

    @classmethod
    def from_layer(cls, lw: dict, device="cuda", dtype: Optional[str] = None) -> "DeviceBlockWeights":
        """From a layer-weights dict (atomistic_mlip_b200.workloads.make_layer_weights)."""
        torch = _torch()
        prec = dtype or lw["precision"]
        td = torch.float32 if prec == "fp32" else torch.bfloat16

        def up(a, t=td):
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device=device, dtype=t)

        L = lw["L"]
        attn = DeviceWeights(L, lw["C"], lw["H"], F32 if prec == "fp32" else BF16,
                             [up(a) for a in lw["Wq"]], [up(a) for a in lw["Wk"]], [up(a) for a in lw["Wv"]],
                             up(lw["W0"]), [None] + [up(a) for a in lw["Wr"][1:]],
                             [None] + [up(a) for a in lw["Wi"][1:]], up(lw["rad_W1"], torch.float32),
                             up(lw["rad_W2"], torch.float32))
        return cls(attn, up(lw["gamma1"], torch.float32), up(lw["gamma2"], torch.float32), up(lw["Wa"]),
                   [up(a) for a in lw["Wb"]], [up(a) for a in lw["Wd"]])


def block_forward(x, pos, nl: NeighborList, bw: DeviceBlockWeights, out=None, stream=None):
    """One E2Former-V2 block on the fp32 residual stream x [N, Q, C]."""
    torch = _torch()
    if out is None:
        out = torch.empty_like(x)
    csr = nl.csr()
    code = lib().e2f_block_forward(_ptr(x), _ptr(pos), ctypes.byref(csr), ctypes.byref(bw.struct), _ptr(out),
                                   _stream_ptr(stream))
    _check(code, "e2f_block_forward")
    return out


def model_forward(x, pos, nl: NeighborList, layers: List[DeviceBlockWeights], stream=None):
    """Blocks in turn; two ping-pong buffers for the residual stream."""
    torch = _torch()
    a, b = x, torch.empty_like(x)
    for i, bw in enumerate(layers):
        block_forward(a, pos, nl, bw, out=b, stream=stream)
        a, b = b, (torch.empty_like(x) if i == 0 else a)
    return a


def attention_backward(x, pos, nl: NeighborList, w: DeviceWeights, grad_out, stream=None):
    """(dL/dx, dL/dpos) for L = sum(grad_out * attention_forward(x, pos, nl, w));
    the forces of an energy are -dL/dpos."""
    torch = _torch()
    N = int(pos.shape[0])
    gx = torch.empty(grad_out.shape, dtype=torch.float32, device=pos.device)
    gp = torch.empty((N, 3), dtype=torch.float32, device=pos.device)
    csr = nl.csr()
    code = lib().e2f_attention_backward(_ptr(x), _ptr(pos), ctypes.byref(csr), ctypes.byref(w.struct),
                                        _ptr(grad_out), _ptr(gx), _ptr(gp), _stream_ptr(stream))
    _check(code, "e2f_attention_backward")
    return gx, gp


def project_qkv(x, w: DeviceWeights, stream=None):
    torch = _torch()
    q, k, v = (torch.empty_like(x) for _ in range(3))
    code = lib().e2f_project_qkv(_ptr(x), int(x.shape[0]), ctypes.byref(w.struct), _ptr(q), _ptr(k), _ptr(v),
                                 _stream_ptr(stream))
    _check(code, "e2f_project_qkv")
    return q, k, v


def wigner_size(L: int) -> int:
    return sum((2 * l + 1) ** 2 for l in range(L + 1))


def wigner_d(R, L: int, stream=None):
    """Real Wigner-D blocks for rotations R (float32 [n, 3, 3] cuda) -> [n, S]."""
    torch = _torch()
    n = int(R.shape[0])
    D = torch.empty((n, wigner_size(L)), dtype=torch.float32, device=R.device)
    _check(lib().e2f_wigner_d(_ptr(R), n, L, _ptr(D), _stream_ptr(stream)), "e2f_wigner_d")
    return D


def stream_status(stream=None) -> int:
    return int(lib().e2f_stream_status(_stream_ptr(stream)))


def kernel_launches() -> int:
    return int(lib().e2f_kernel_launches())


def profile_enable(on: bool = True):
    _check(lib().e2f_profile_enable(1 if on else 0), "e2f_profile_enable")


def profile_read():
    n = ctypes.c_int64(0)
    ms = ctypes.c_double(0.0)
    _check(lib().e2f_profile_read(ctypes.byref(n), ctypes.byref(ms)), "e2f_profile_read")
    return int(n.value), float(ms.value)


def scratch_high_water(reset: bool = False) -> int:
    b = ctypes.c_int64(0)
    _check(lib().e2f_scratch_high_water(ctypes.byref(b), 1 if reset else 0), "e2f_scratch_high_water")
    return int(b.value)
