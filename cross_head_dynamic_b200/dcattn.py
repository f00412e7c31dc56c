"""Python binding of libdcattn (ctypes).  Argument marshalling only: every step
of the computation runs in the CUDA kernels behind include/dcattn.h.

Functions carry the C entry points' names and take torch CUDA tensors; torch is
used for device memory and the current stream, nothing else.  There is no CPU
path: a missing library or a CPU tensor raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdcattn.so")

DC_OK, DC_ERR_INVALID_ARG, DC_ERR_UNSUPPORTED, DC_ERR_CUDA, DC_ERR_DEVICE = range(5)
DC_F32, DC_BF16 = 0, 1
IMPLS = {"auto": 0, "simt": 1, "tcgen05": 2}
IMPL_NAMES = {v: k for k, v in IMPLS.items()}
DC_DEVERR_SEQLENS = 0x1
DC_DEVERR_TIMEOUT = 0x2

EXPORTED = ("dc_attn_fwd", "dc_attn_bwd_workspace_size", "dc_attn_bwd_query", "dc_attn_bwd_key",
            "dc_attn_bwd", "dc_attn_resolve_impl", "dc_attn_device_status", "dc_attn_status_string",
            "dc_attn_last_launch_count", "dc_attn_bwd_noalloc", "dc_attn_halo_add", "dc_attn_set_wait_limit",
            "dc_attn_inject_missing_load", "dc_attn_cg_fwd", "dc_attn_cg_bwd_workspace_size", "dc_attn_cg_bwd",
            "dc_attn_cg_resolve_impl", "dc_attn_cg_prepare_size", "dc_attn_cg_prepare")


class DCAttnError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {msg} (status {code})")
        self.code = code


class Params(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("impl", ctypes.c_int32), ("total_tokens", ctypes.c_int64),
                ("num_docs", ctypes.c_int32), ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("window", ctypes.c_int32), ("softmax_scale", ctypes.c_float), ("reserved", ctypes.c_int32),
                ("cu_seqlens", ctypes.c_void_p), ("stride_qkv", ctypes.c_int64), ("stride_dqkv", ctypes.c_int64),
                ("stride_o", ctypes.c_int64)]


class CgParams(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("model_dim", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("impl", ctypes.c_int32), ("num_tokens", ctypes.c_int64), ("stride_x", ctypes.c_int64),
                ("stride_dx", ctypes.c_int64), ("weight_splits", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libdcattn.so and declare its signatures.  Raises if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libdcattn.so is not built ({path}); run `python -m cross_head_dynamic_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(Params)
    vp = ctypes.c_void_p
    st = ctypes.c_int
    lib.dc_attn_fwd.argtypes = [P] + [vp] * 9
    lib.dc_attn_fwd.restype = st
    lib.dc_attn_bwd_workspace_size.argtypes = [P]
    lib.dc_attn_bwd_workspace_size.restype = ctypes.c_size_t
    lib.dc_attn_bwd_query.argtypes = [P] + [vp] * 12 + [ctypes.c_size_t, vp]
    lib.dc_attn_bwd_query.restype = st
    lib.dc_attn_bwd_key.argtypes = [P] + [vp] * 11 + [ctypes.c_size_t, vp]
    lib.dc_attn_bwd_key.restype = st
    lib.dc_attn_bwd.argtypes = [P] + [vp] * 14 + [ctypes.c_size_t, vp]
    lib.dc_attn_bwd.restype = st
    lib.dc_attn_resolve_impl.argtypes = [P]
    lib.dc_attn_resolve_impl.restype = ctypes.c_int32
    lib.dc_attn_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32]
    lib.dc_attn_device_status.restype = st
    lib.dc_attn_status_string.argtypes = [st]
    lib.dc_attn_status_string.restype = ctypes.c_char_p
    lib.dc_attn_bwd_noalloc.argtypes = [P] + [vp] * 14
    lib.dc_attn_bwd_noalloc.restype = st
    lib.dc_attn_last_launch_count.argtypes = []
    lib.dc_attn_last_launch_count.restype = ctypes.c_int32
    lib.dc_attn_halo_add.argtypes = [vp, vp, ctypes.c_int64, ctypes.c_int32, vp]
    lib.dc_attn_halo_add.restype = st
    lib.dc_attn_set_wait_limit.argtypes = [ctypes.c_uint32]
    lib.dc_attn_set_wait_limit.restype = st
    lib.dc_attn_inject_missing_load.argtypes = []
    lib.dc_attn_inject_missing_load.restype = st
    CP = ctypes.POINTER(CgParams)
    lib.dc_attn_cg_fwd.argtypes = [CP] + [vp] * 6
    lib.dc_attn_cg_fwd.restype = st
    lib.dc_attn_cg_bwd_workspace_size.argtypes = [CP]
    lib.dc_attn_cg_bwd_workspace_size.restype = ctypes.c_size_t
    lib.dc_attn_cg_bwd.argtypes = [CP] + [vp] * 8 + [ctypes.c_size_t, vp]
    lib.dc_attn_cg_bwd.restype = st
    lib.dc_attn_cg_resolve_impl.argtypes = [CP]
    lib.dc_attn_cg_resolve_impl.restype = ctypes.c_int32
    lib.dc_attn_cg_prepare_size.argtypes = [CP]
    lib.dc_attn_cg_prepare_size.restype = ctypes.c_size_t
    lib.dc_attn_cg_prepare.argtypes = [CP, vp, vp, vp]
    lib.dc_attn_cg_prepare.restype = st
    _lib = lib
    return lib


def _check(fn: str, code: int):
    if code != DC_OK:
        msg = load_library().dc_attn_status_string(code).decode()
        raise DCAttnError(fn, code, msg)


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dev(x: torch.Tensor, name: str, dtype=None, rows: bool = False):
    """Device pointer of x.  With rows=True, x is [N, H, d] with each token's H * d
    elements contiguous (tokens may be further apart: a view of a fused tensor)."""
    if not isinstance(x, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libdcattn has no CPU path)")
    if rows:
        if x.dim() != 3 or x.stride(2) != 1 or x.stride(1) != x.shape[2]:
            raise ValueError(f"{name} must be [N, H, d] with each token's H * d elements contiguous")
    elif not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and x.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {x.dtype}")
    return x.data_ptr()


def _row_stride(name: str, *xs) -> int:
    """The common token stride of the [N, H, d] tensors xs (None entries ignored)."""
    st = {int(x.stride(0)) for x in xs if x is not None and x.shape[0] > 1}
    if len(st) > 1:
        raise ValueError(f"{name} must share one token stride, got {sorted(st)}")
    return st.pop() if st else 0


def _opt(x, name, dtype=None):
    return None if x is None else _dev(x, name, dtype)


def make_params(q: torch.Tensor, cu_seqlens: torch.Tensor, window: int, scale: float,
                impl: str = "auto", stride_qkv: int = 0, stride_dqkv: int = 0, stride_o: int = 0) -> Params:
    if q.dim() != 3:
        raise ValueError("q must be [N, H, d]")
    N, H, d = q.shape
    if q.dtype == torch.float32:
        dt = DC_F32
    elif q.dtype == torch.bfloat16:
        dt = DC_BF16
    else:
        raise TypeError(f"unsupported dtype {q.dtype}")
    return Params(dtype=dt, impl=IMPLS[impl], total_tokens=N, num_docs=cu_seqlens.numel() - 1,
                  num_heads=H, head_dim=d, window=int(window), softmax_scale=float(scale), reserved=0,
                  cu_seqlens=_dev(cu_seqlens, "cu_seqlens", torch.int32), stride_qkv=stride_qkv,
                  stride_dqkv=stride_dqkv, stride_o=stride_o)


def dc_attn_resolve_impl(q, cu_seqlens, window, scale, impl="auto") -> str:
    p = make_params(q, cu_seqlens, window, scale, impl)
    r = load_library().dc_attn_resolve_impl(ctypes.byref(p))
    if r < 0:
        raise DCAttnError("dc_attn_resolve_impl", DC_ERR_INVALID_ARG, "invalid parameters")
    return IMPL_NAMES[r]


def dc_attn_fwd(q, k, v, c, g, cu_seqlens, window: int, scale: float, *, o=None, lse=None, pmap=None,
                need_backward: bool = True, impl: str = "auto", stream=None):
    """Forward pass; returns (o, lse, pmap).  lse/pmap are None when need_backward
    is False and none were passed in."""
    N, H, d = q.shape
    if o is None:
        o = torch.empty(q.shape, device=q.device, dtype=q.dtype)
    p = make_params(q, cu_seqlens, window, scale, impl, stride_qkv=_row_stride("q, k, v", q, k, v),
                    stride_o=_row_stride("o", o))
    if need_backward:
        if lse is None:
            lse = torch.empty(N, H, device=q.device, dtype=torch.float32)
        if pmap is None:
            pmap = torch.empty(N, int(window), device=q.device, dtype=q.dtype)
    code = load_library().dc_attn_fwd(
        ctypes.byref(p), _dev(q, "q", q.dtype, True), _dev(k, "k", q.dtype, True), _dev(v, "v", q.dtype, True),
        _dev(c, "c", torch.float32), _dev(g, "g", torch.float32), _dev(o, "o", q.dtype, True),
        _opt(lse, "lse", torch.float32), _opt(pmap, "pmap", q.dtype), _stream_handle(stream))
    _check("dc_attn_fwd", code)
    return o, lse, pmap


def dc_attn_bwd_workspace_size(q, cu_seqlens, window, scale, impl="auto") -> int:
    p = make_params(q, cu_seqlens, window, scale, impl)
    return int(load_library().dc_attn_bwd_workspace_size(ctypes.byref(p)))


def _workspace(q, cu_seqlens, window, scale, impl, workspace):
    need = dc_attn_bwd_workspace_size(q, cu_seqlens, window, scale, impl)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    return workspace


def dc_attn_bwd_query(q, k, v, c, g, dO, lse, pmap, cu_seqlens, window, scale, *, dq=None, dc=None,
                      dg=None, workspace=None, impl="auto", stream=None):
    """Query side of the backward; returns (dq, dc, dg, workspace)."""
    N, H, d = q.shape
    dq = torch.empty(q.shape, device=q.device, dtype=q.dtype) if dq is None else dq
    dc = torch.empty(N, H, device=q.device, dtype=torch.float32) if dc is None else dc
    dg = torch.empty(N, H, device=q.device, dtype=torch.float32) if dg is None else dg
    p = make_params(q, cu_seqlens, window, scale, impl, stride_qkv=_row_stride("q, k, v", q, k, v),
                    stride_dqkv=_row_stride("dq", dq), stride_o=_row_stride("dO", dO))
    workspace = _workspace(q, cu_seqlens, window, scale, impl, workspace)
    code = load_library().dc_attn_bwd_query(
        ctypes.byref(p), _dev(q, "q", q.dtype, True), _dev(k, "k", q.dtype, True), _dev(v, "v", q.dtype, True),
        _dev(c, "c", torch.float32), _dev(g, "g", torch.float32), _dev(dO, "dO", q.dtype, True),
        _dev(lse, "lse", torch.float32), _dev(pmap, "pmap", q.dtype), _dev(dq, "dq", q.dtype, True),
        _dev(dc, "dc", torch.float32), _dev(dg, "dg", torch.float32), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _check("dc_attn_bwd_query", code)
    return dq, dc, dg, workspace


def dc_attn_bwd_key(q, k, c, g, dO, lse, pmap, dc, workspace, cu_seqlens, window, scale, *, dk=None, dv=None,
                    impl="auto", stream=None):
    """Key side of the backward (after dc_attn_bwd_query); returns (dk, dv)."""
    dk = torch.empty(q.shape, device=q.device, dtype=q.dtype) if dk is None else dk
    dv = torch.empty(q.shape, device=q.device, dtype=q.dtype) if dv is None else dv
    p = make_params(q, cu_seqlens, window, scale, impl, stride_qkv=_row_stride("q, k", q, k),
                    stride_dqkv=_row_stride("dk, dv", dk, dv), stride_o=_row_stride("dO", dO))
    code = load_library().dc_attn_bwd_key(
        ctypes.byref(p), _dev(q, "q", q.dtype, True), _dev(k, "k", q.dtype, True), _dev(c, "c", torch.float32),
        _dev(g, "g", torch.float32), _dev(dO, "dO", q.dtype, True), _dev(lse, "lse", torch.float32),
        _dev(pmap, "pmap", q.dtype), _dev(dc, "dc", torch.float32), _dev(dk, "dk", q.dtype, True),
        _dev(dv, "dv", q.dtype, True), _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream_handle(stream))
    _check("dc_attn_bwd_key", code)
    return dk, dv


def dc_attn_bwd(q, k, v, c, g, dO, lse, pmap, cu_seqlens, window, scale, *, dq=None, dk=None, dv=None,
                dc=None, dg=None, workspace=None, impl="auto", stream=None):
    """Full backward; returns (dq, dk, dv, dc, dg)."""
    N, H, d = q.shape
    dq = torch.empty(q.shape, device=q.device, dtype=q.dtype) if dq is None else dq
    dk = torch.empty(q.shape, device=q.device, dtype=q.dtype) if dk is None else dk
    dv = torch.empty(q.shape, device=q.device, dtype=q.dtype) if dv is None else dv
    p = make_params(q, cu_seqlens, window, scale, impl, stride_qkv=_row_stride("q, k, v", q, k, v),
                    stride_dqkv=_row_stride("dq, dk, dv", dq, dk, dv), stride_o=_row_stride("dO", dO))
    dc = torch.empty(N, H, device=q.device, dtype=torch.float32) if dc is None else dc
    dg = torch.empty(N, H, device=q.device, dtype=torch.float32) if dg is None else dg
    workspace = _workspace(q, cu_seqlens, window, scale, impl, workspace)
    code = load_library().dc_attn_bwd(
        ctypes.byref(p), _dev(q, "q", q.dtype, True), _dev(k, "k", q.dtype, True), _dev(v, "v", q.dtype, True),
        _dev(c, "c", torch.float32), _dev(g, "g", torch.float32), _dev(dO, "dO", q.dtype, True),
        _dev(lse, "lse", torch.float32), _dev(pmap, "pmap", q.dtype), _dev(dq, "dq", q.dtype, True),
        _dev(dk, "dk", q.dtype, True), _dev(dv, "dv", q.dtype, True), _dev(dc, "dc", torch.float32),
        _dev(dg, "dg", torch.float32), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _check("dc_attn_bwd", code)
    return dq, dk, dv, dc, dg


def dc_attn_bwd_noalloc(q, k, v, c, g, dO, lse, pmap, cu_seqlens, window, scale, *, dq=None, dk=None, dv=None,
                        dc=None, dg=None, impl="auto", stream=None):
    """Full backward without a workspace, for callers that cannot allocate scratch
    (plugin-style interfaces that pass an op only its inputs and outputs, or
    processes that reserve all device memory up front).  The library's static
    32 MiB scratch array serves as the workspace, so N * W * 4 must not exceed
    32 MiB; overlapping calls on one device race on that array.  Returns
    (dq, dk, dv, dc, dg)."""
    N, H, d = q.shape
    dq = torch.empty(q.shape, device=q.device, dtype=q.dtype) if dq is None else dq
    dk = torch.empty(q.shape, device=q.device, dtype=q.dtype) if dk is None else dk
    dv = torch.empty(q.shape, device=q.device, dtype=q.dtype) if dv is None else dv
    p = make_params(q, cu_seqlens, window, scale, impl, stride_qkv=_row_stride("q, k, v", q, k, v),
                    stride_dqkv=_row_stride("dq, dk, dv", dq, dk, dv), stride_o=_row_stride("dO", dO))
    dc = torch.empty(N, H, device=q.device, dtype=torch.float32) if dc is None else dc
    dg = torch.empty(N, H, device=q.device, dtype=torch.float32) if dg is None else dg
    code = load_library().dc_attn_bwd_noalloc(
        ctypes.byref(p), _dev(q, "q", q.dtype, True), _dev(k, "k", q.dtype, True), _dev(v, "v", q.dtype, True),
        _dev(c, "c", torch.float32), _dev(g, "g", torch.float32), _dev(dO, "dO", q.dtype, True),
        _dev(lse, "lse", torch.float32), _dev(pmap, "pmap", q.dtype), _dev(dq, "dq", q.dtype, True),
        _dev(dk, "dk", q.dtype, True), _dev(dv, "dv", q.dtype, True), _dev(dc, "dc", torch.float32),
        _dev(dg, "dg", torch.float32), _stream_handle(stream))
    _check("dc_attn_bwd_noalloc", code)
    return dq, dk, dv, dc, dg


def dc_attn_device_status(reset: bool = True, stream=None) -> int:
    """Synchronize and return the device status word (DC_DEVERR_* bits)."""
    out = ctypes.c_uint32(0)
    code = load_library().dc_attn_device_status(_stream_handle(stream), ctypes.byref(out), int(reset))
    _check("dc_attn_device_status", code)
    return int(out.value)


def dc_attn_last_launch_count() -> int:
    return int(load_library().dc_attn_last_launch_count())


def dc_attn_halo_add(dst, src, stream=None):
    """dst += src in place (same shape, bf16 or fp32; fp32 sum rounded once), on the GPU."""
    if dst.shape != src.shape or dst.dtype != src.dtype:
        raise ValueError("dc_attn_halo_add: dst and src differ in shape or dtype")
    dt = {torch.float32: DC_F32, torch.bfloat16: DC_BF16}.get(dst.dtype)
    if dt is None:
        raise ValueError(f"dc_attn_halo_add: unsupported dtype {dst.dtype}")
    code = load_library().dc_attn_halo_add(_dev(dst, "dst", dst.dtype), _dev(src, "src", dst.dtype), dst.numel(),
                                           dt, _stream_handle(stream))
    _check("dc_attn_halo_add", code)
    return dst


def dc_attn_set_wait_limit(ns: int = 0):
    """Limit (nanoseconds) of the tcgen05 kernels' bounded waits for later calls; 0 = default 2 s."""
    _check("dc_attn_set_wait_limit", load_library().dc_attn_set_wait_limit(int(ns)))


def dc_attn_inject_missing_load():
    """Test hook: the next one-piece tcgen05 forward leaves out its first CTA's head-0 loads."""
    _check("dc_attn_inject_missing_load", load_library().dc_attn_inject_missing_load())


def _token_rows(x: torch.Tensor, name: str, dtype=None) -> int:
    """Token stride of x [N, D] whose rows are contiguous (x may be a column slice)."""
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError(f"{name} must be a [N, D] torch tensor")
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libdcattn has no CPU path)")
    if x.shape[1] > 1 and x.stride(1) != 1:
        raise ValueError(f"{name} must have contiguous rows")
    if dtype is not None and x.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {x.dtype}")
    return int(x.stride(0)) if x.shape[0] > 1 else 0


def make_cg_params(x: torch.Tensor, num_heads: int, dx=None, impl: str = "auto", weight_splits=None) -> CgParams:
    dt = {torch.float32: DC_F32, torch.bfloat16: DC_BF16}.get(x.dtype)
    if dt is None:
        raise TypeError(f"unsupported dtype {x.dtype}")
    sx = _token_rows(x, "x")
    sdx = 0 if dx is None else _token_rows(dx, "dx", x.dtype)
    return CgParams(dtype=dt, model_dim=int(x.shape[1]), num_heads=int(num_heads), impl=IMPLS[impl],
                    num_tokens=int(x.shape[0]), stride_x=sx, stride_dx=sdx,
                    weight_splits=None if weight_splits is None else _dev(weight_splits, "weight_splits"))


def dc_attn_cg_prepare(weight, *, splits=None, stream=None):
    """The weight [2H, D] fp32 as the tensor-core kernels read it (bf16 splits in their
    shared-memory layout); pass the result as weight_splits= to the producer's calls while
    the weight is unchanged.  Returns the image (uint8 device tensor)."""
    H, D = weight.shape[0] // 2, weight.shape[1]
    probe = torch.empty(0, D, device=weight.device, dtype=torch.bfloat16)
    p = make_cg_params(probe, H)
    n = int(load_library().dc_attn_cg_prepare_size(ctypes.byref(p)))
    if n == 0:
        raise DCAttnError("dc_attn_cg_prepare_size", DC_ERR_INVALID_ARG, "invalid parameters")
    splits = torch.empty(n, device=weight.device, dtype=torch.uint8) if splits is None else splits
    code = load_library().dc_attn_cg_prepare(ctypes.byref(p), _dev(weight, "weight", torch.float32),
                                             _dev(splits, "splits"), _stream_handle(stream))
    _check("dc_attn_cg_prepare", code)
    return splits


def dc_attn_cg_resolve_impl(x, num_heads: int, impl: str = "auto") -> str:
    """Kernel family of the c/g forward for x and H ('simt' or 'tcgen05')."""
    r = load_library().dc_attn_cg_resolve_impl(ctypes.byref(make_cg_params(x, num_heads, impl=impl)))
    if r < 0:
        raise DCAttnError("dc_attn_cg_resolve_impl", DC_ERR_UNSUPPORTED, "invalid or unsupported parameters")
    return IMPL_NAMES[r]


def dc_attn_cg_fwd(x, weight, bias, *, c=None, g=None, impl: str = "auto", weight_splits=None, stream=None):
    """c, g [N, H] fp32 from the hidden state x [N, D] (per-token affine maps; weight
    [2H, D] fp32 in a linear layer's layout, bias [2H] fp32).  Returns (c, g)."""
    H = weight.shape[0] // 2
    N = x.shape[0]
    c = torch.empty(N, H, device=x.device, dtype=torch.float32) if c is None else c
    g = torch.empty(N, H, device=x.device, dtype=torch.float32) if g is None else g
    p = make_cg_params(x, H, impl=impl, weight_splits=weight_splits)
    code = load_library().dc_attn_cg_fwd(ctypes.byref(p), x.data_ptr(), _dev(weight, "weight", torch.float32),
                                         _dev(bias, "bias", torch.float32), _dev(c, "c", torch.float32),
                                         _dev(g, "g", torch.float32), _stream_handle(stream))
    _check("dc_attn_cg_fwd", code)
    return c, g


def dc_attn_cg_bwd_workspace_size(x, num_heads: int) -> int:
    p = make_cg_params(x, num_heads)
    return int(load_library().dc_attn_cg_bwd_workspace_size(ctypes.byref(p)))


def dc_attn_cg_bwd(x, weight, dc, dg, *, dx=None, dweight=None, dbias=None, workspace=None, impl: str = "auto",
                   weight_splits=None, stream=None):
    """Gradients of the c/g producer for dL/dc = dc, dL/dg = dg.  Returns
    (dx, dweight, dbias); dweight and dbias are bitwise reproducible for a given N.
    `impl` chooses the kernel family of dx."""
    H = weight.shape[0] // 2
    dx = torch.empty(x.shape, device=x.device, dtype=x.dtype) if dx is None else dx
    dweight = torch.empty(weight.shape, device=x.device, dtype=torch.float32) if dweight is None else dweight
    dbias = torch.empty(2 * H, device=x.device, dtype=torch.float32) if dbias is None else dbias
    p = make_cg_params(x, H, dx, impl=impl, weight_splits=weight_splits)
    if workspace is None:
        workspace = torch.empty(max(dc_attn_cg_bwd_workspace_size(x, H), 16), device=x.device, dtype=torch.uint8)
    code = load_library().dc_attn_cg_bwd(
        ctypes.byref(p), x.data_ptr(), _dev(weight, "weight", torch.float32), _dev(dc, "dc", torch.float32),
        _dev(dg, "dg", torch.float32), dx.data_ptr(), _dev(dweight, "dweight", torch.float32),
        _dev(dbias, "dbias", torch.float32), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _check("dc_attn_cg_bwd", code)
    return dx, dweight, dbias
