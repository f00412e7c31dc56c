"""fp64 CPU oracle for Lightweight DC attention (ctypes wrapper of dc_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by __graft_entry__.smoke() and
by the CPU-baseline leg of bench.py.  The product (the CUDA library and its
Python binding) never imports it.

Every function takes plain numpy / torch CPU arrays in any float dtype; values
are widened to float64 exactly (bf16 and fp32 are subsets of fp64), so the
oracle sees the same numbers the GPU sees.  The arithmetic itself lives in
dc_oracle.c; see its header for the definition and the derivation of the
backward pass.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dc_oracle.c")
_SRC_CG = os.path.join(_HERE, "cg_oracle.c")
_LIB = os.path.join(_HERE, "libdcoracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile dc_oracle.c and cg_oracle.c into libdcoracle.so next to them (gcc, -O2, OpenMP)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_CG))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", tmp, _SRC, _SRC_CG, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        d = ctypes.POINTER(ctypes.c_double)
        i32 = ctypes.POINTER(ctypes.c_int32)
        common = [ctypes.c_int64, ctypes.c_int, i32, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_double]
        lib.dc_oracle_fwd.argtypes = common + [d] * 5 + [d] * 3
        lib.dc_oracle_fwd.restype = ctypes.c_int
        lib.dc_oracle_bwd.argtypes = common + [d] * 6 + [d] * 5
        lib.dc_oracle_bwd.restype = ctypes.c_int
        lib.dc_oracle_num_threads.argtypes = []
        lib.dc_oracle_num_threads.restype = ctypes.c_int
        lib.dc_oracle_cg_fwd.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int] + [d] * 5
        lib.dc_oracle_cg_fwd.restype = ctypes.c_int
        lib.dc_oracle_cg_bwd.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int] + [d] * 7
        lib.dc_oracle_cg_bwd.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (any float dtype, CPU)
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _cu(cu_seqlens) -> np.ndarray:
    if hasattr(cu_seqlens, "detach"):
        cu_seqlens = cu_seqlens.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))


def num_threads() -> int:
    return int(_load().dc_oracle_num_threads())


def forward(q, k, v, c, g, cu_seqlens, window: int, scale: float):
    """Returns (o [N,H,d], lse [N,H], pmap [N,W]) as float64 numpy arrays."""
    q, k, v, c, g = map(_f64, (q, k, v, c, g))
    cu = _cu(cu_seqlens)
    N, H, d = q.shape
    o = np.empty((N, H, d))
    lse = np.empty((N, H))
    pmap = np.empty((N, window))
    rc = _load().dc_oracle_fwd(N, len(cu) - 1, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                               H, d, int(window), float(scale), _ptr(q), _ptr(k), _ptr(v),
                               _ptr(c), _ptr(g), _ptr(o), _ptr(lse), _ptr(pmap))
    if rc != 0:
        raise ValueError(f"dc_oracle_fwd rejected its arguments (rc={rc})")
    return o, lse, pmap


def backward(q, k, v, c, g, dO, cu_seqlens, window: int, scale: float):
    """Returns (dq, dk, dv [N,H,d], dc, dg [N,H]) as float64 numpy arrays."""
    q, k, v, c, g, dO = map(_f64, (q, k, v, c, g, dO))
    cu = _cu(cu_seqlens)
    N, H, d = q.shape
    dq = np.empty((N, H, d))
    dk = np.empty((N, H, d))
    dv = np.empty((N, H, d))
    dc = np.empty((N, H))
    dg = np.empty((N, H))
    rc = _load().dc_oracle_bwd(N, len(cu) - 1, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                               H, d, int(window), float(scale), _ptr(q), _ptr(k), _ptr(v),
                               _ptr(c), _ptr(g), _ptr(dO), _ptr(dq), _ptr(dk), _ptr(dv),
                               _ptr(dc), _ptr(dg))
    if rc != 0:
        raise ValueError(f"dc_oracle_bwd rejected its arguments (rc={rc})")
    return dq, dk, dv, dc, dg


def cg_forward(x, w, b):
    """The assumed producer of c and g (see cg_oracle.c): x [N, D], w [D, 2H], b [2H].
    Returns (c [N, H], g [N, H]) as float64 numpy arrays."""
    x, w, b = map(_f64, (x, w, b))
    N, D = x.shape
    H = w.shape[1] // 2
    if w.shape != (D, 2 * H) or b.shape != (2 * H,):
        raise ValueError("cg_forward: w must be [D, 2H] and b [2H]")
    c = np.empty((N, H))
    g = np.empty((N, H))
    rc = _load().dc_oracle_cg_fwd(N, D, H, _ptr(x), _ptr(w), _ptr(b), _ptr(c), _ptr(g))
    if rc != 0:
        raise ValueError(f"dc_oracle_cg_fwd rejected its arguments (rc={rc})")
    return c, g


def cg_backward(x, w, dc, dg):
    """Gradients of cg_forward for dL/dc = dc, dL/dg = dg.  Returns (dx [N, D], dw [D, 2H],
    db [2H]) as float64 numpy arrays."""
    x, w, dc, dg = map(_f64, (x, w, dc, dg))
    N, D = x.shape
    H = w.shape[1] // 2
    dx = np.empty((N, D))
    dw = np.empty((D, 2 * H))
    db = np.empty(2 * H)
    rc = _load().dc_oracle_cg_bwd(N, D, H, _ptr(x), _ptr(w), _ptr(dc), _ptr(dg), _ptr(dx), _ptr(dw), _ptr(db))
    if rc != 0:
        raise ValueError(f"dc_oracle_cg_bwd rejected its arguments (rc={rc})")
    return dx, dw, db
