"""Host-side checks of the C ABI: the library builds/loads, exports every
function include/dcattn.h declares, and rejects bad arguments on the host
before any CUDA call (so these run without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from cross_head_dynamic_b200 import build as dcbuild
from cross_head_dynamic_b200 import dcattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dcattn.h")


@pytest.fixture(scope="module")
def lib():
    dcbuild.build()
    return dcattn.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dc_attn_\w+)\s*\(", text)))


def test_header_declares_expected_api():
    names = declared_functions()
    assert set(dcattn.EXPORTED) <= set(names), names
    assert set(names) <= set(dcattn.EXPORTED), names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", dcattn.LIB_PATH]).decode()
    exported = set(re.findall(r"\bT (dc_attn_\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_library_has_no_oracle_dependency(lib):
    out = subprocess.check_output(["nm", "-D", dcattn.LIB_PATH]).decode()
    assert "dc_oracle" not in out
    ldd = subprocess.check_output(["ldd", dcattn.LIB_PATH]).decode()
    assert "dcoracle" not in ldd


def test_status_strings(lib):
    for code in range(5):
        assert lib.dc_attn_status_string(code)
    assert lib.dc_attn_status_string(99) == b"unknown status"


def _params(**kw):
    base = dict(dtype=dcattn.DC_BF16, impl=0, total_tokens=256, num_docs=1, num_heads=6, head_dim=128,
                window=112, softmax_scale=0.088, reserved=0, cu_seqlens=0x1000)
    base.update(kw)
    return dcattn.Params(**base)


def _fwd(lib, p, ptr=0x2000):
    return lib.dc_attn_fwd(ctypes.byref(p), ptr, ptr, ptr, ptr, ptr, ptr, None, None, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(dtype=7), dcattn.DC_ERR_INVALID_ARG),
    (dict(impl=9), dcattn.DC_ERR_INVALID_ARG),
    (dict(reserved=1), dcattn.DC_ERR_INVALID_ARG),
    (dict(total_tokens=-1), dcattn.DC_ERR_INVALID_ARG),
    (dict(num_heads=0), dcattn.DC_ERR_INVALID_ARG),
    (dict(num_heads=17), dcattn.DC_ERR_INVALID_ARG),
    (dict(window=0), dcattn.DC_ERR_INVALID_ARG),
    (dict(num_docs=0), dcattn.DC_ERR_INVALID_ARG),
    (dict(num_docs=258), dcattn.DC_ERR_INVALID_ARG),
    (dict(cu_seqlens=0), dcattn.DC_ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), dcattn.DC_ERR_INVALID_ARG),
    (dict(head_dim=48), dcattn.DC_ERR_UNSUPPORTED),
    (dict(head_dim=256), dcattn.DC_ERR_UNSUPPORTED),
    (dict(window=5000), dcattn.DC_ERR_UNSUPPORTED),
    (dict(dtype=dcattn.DC_F32, impl=2), dcattn.DC_ERR_UNSUPPORTED),
])
def test_bad_params_rejected_on_host(lib, kw, expect):
    assert _fwd(lib, _params(**kw)) == expect


def test_null_and_misaligned_pointers_rejected(lib):
    p = _params(dtype=dcattn.DC_F32)
    assert _fwd(lib, p, ptr=0) == dcattn.DC_ERR_INVALID_ARG
    assert _fwd(lib, p, ptr=0x2008) == dcattn.DC_ERR_INVALID_ARG


def test_halo_add_rejects_bad_arguments_on_host(lib):
    ok = 0x4000
    assert lib.dc_attn_halo_add(ok, ok, 16, 7, None) == dcattn.DC_ERR_INVALID_ARG          # dtype
    assert lib.dc_attn_halo_add(ok, ok, -1, dcattn.DC_BF16, None) == dcattn.DC_ERR_INVALID_ARG
    assert lib.dc_attn_halo_add(0, ok, 16, dcattn.DC_BF16, None) == dcattn.DC_ERR_INVALID_ARG   # null
    assert lib.dc_attn_halo_add(ok, 0x4008, 16, dcattn.DC_F32, None) == dcattn.DC_ERR_INVALID_ARG  # misaligned
    assert lib.dc_attn_halo_add(0, 0, 0, dcattn.DC_F32, None) == dcattn.DC_OK                # n = 0: no-op


def test_empty_problem_is_a_noop(lib):
    p = _params(total_tokens=0, num_docs=0, cu_seqlens=0)
    assert _fwd(lib, p, ptr=0) == dcattn.DC_OK
    assert lib.dc_attn_bwd_workspace_size(ctypes.byref(p)) == 0


def test_workspace_size_and_check(lib):
    p = _params(dtype=dcattn.DC_F32, total_tokens=1000, num_docs=3, window=112)
    need = lib.dc_attn_bwd_workspace_size(ctypes.byref(p))
    assert need == 4 * 1000 * 112
    a = 0x4000
    args = [a] * 12
    rc = lib.dc_attn_bwd_query(ctypes.byref(p), *args, need - 1, None)
    assert rc == dcattn.DC_ERR_INVALID_ARG


def test_resolve_impl(lib):
    assert lib.dc_attn_resolve_impl(ctypes.byref(_params(dtype=dcattn.DC_F32))) == 1
    assert lib.dc_attn_resolve_impl(ctypes.byref(_params(impl=1))) == 1
    assert lib.dc_attn_resolve_impl(ctypes.byref(_params(window=0))) == -1


def test_resolve_impl_tcgen05_range(lib):
    # bf16 with d in {64, 128} and 1 <= W <= 256 runs on tcgen05 (W > 129 as two window
    # segments), other bf16 shapes on SIMT; more than 16 heads is refused on every path
    tc, simt = dcattn.IMPLS["tcgen05"], dcattn.IMPLS["simt"]
    for W, d, H, want in ((1, 128, 6, tc), (112, 128, 6, tc), (129, 128, 4, tc), (130, 64, 2, tc),
                          (256, 128, 6, tc), (257, 128, 6, simt), (64, 64, 16, tc), (64, 96, 6, simt),
                          (64, 64, 17, -1)):
        p = _params(dtype=dcattn.DC_BF16, window=W, head_dim=d, num_heads=H)
        assert lib.dc_attn_resolve_impl(ctypes.byref(p)) == want, (W, d, H)


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(4, 1, 32)
    with pytest.raises(ValueError):
        dcattn.dc_attn_fwd(q, q, q, torch.zeros(4, 1), torch.zeros(4, 1), torch.tensor([0, 4], dtype=torch.int32),
                           4, 1.0)


def test_wait_limit_hook_validates_on_the_host(lib):
    assert lib.dc_attn_set_wait_limit(50) == dcattn.DC_ERR_INVALID_ARG      # below 0.1 ms
    assert lib.dc_attn_set_wait_limit(99999) == dcattn.DC_ERR_INVALID_ARG
    assert lib.dc_attn_set_wait_limit(5_000_000) == dcattn.DC_OK
    assert lib.dc_attn_set_wait_limit(0) == dcattn.DC_OK                    # back to the default


@pytest.mark.parametrize("field", ["stride_qkv", "stride_dqkv", "stride_o"])
@pytest.mark.parametrize("value", [767, 772, -768])
def test_rejects_bad_row_strides(lib, field, value):
    """A row stride below H * d (768 here), or one that is not a multiple of 16 bytes, is
    refused on the host before anything runs."""
    p = _params(**{field: value})
    assert _fwd(lib, p) == dcattn.DC_ERR_INVALID_ARG


def test_accepts_fused_projection_strides(lib):
    """3 * H * d (q, k, v as views of one [N][3][H][d] projection) passes the host checks; the
    call then stops at the device pointers, which are not real (N = 0 would skip them)."""
    p = _params(stride_qkv=3 * 768, stride_dqkv=3 * 768, stride_o=2 * 768, total_tokens=0)
    assert _fwd(lib, p) == dcattn.DC_OK


def _cg(**kw):
    base = dict(dtype=dcattn.DC_BF16, model_dim=768, num_heads=6, impl=0, num_tokens=1000, stride_x=0,
                stride_dx=0)
    base.update(kw)
    return dcattn.CgParams(**base)


@pytest.mark.parametrize("kw, expect", [
    (dict(dtype=7), dcattn.DC_ERR_INVALID_ARG),
    (dict(model_dim=767), dcattn.DC_ERR_INVALID_ARG),      # D must be even
    (dict(model_dim=0), dcattn.DC_ERR_INVALID_ARG),
    (dict(num_heads=0), dcattn.DC_ERR_INVALID_ARG),
    (dict(num_tokens=-1), dcattn.DC_ERR_INVALID_ARG),
    (dict(stride_x=770 + 1), dcattn.DC_ERR_INVALID_ARG),   # odd stride
    (dict(stride_x=766), dcattn.DC_ERR_INVALID_ARG),       # below D
    (dict(stride_dx=-768), dcattn.DC_ERR_INVALID_ARG),
    (dict(num_heads=17), dcattn.DC_ERR_UNSUPPORTED),
    (dict(model_dim=4332), dcattn.DC_ERR_UNSUPPORTED),     # weight + partial sums above 227 KB
    (dict(model_dim=4332, dtype=dcattn.DC_F32), dcattn.DC_ERR_UNSUPPORTED),
    (dict(num_heads=16, model_dim=1562), dcattn.DC_ERR_UNSUPPORTED),
    (dict(impl=3), dcattn.DC_ERR_INVALID_ARG),
])
def test_cg_bad_params_rejected_on_host(lib, kw, expect):
    p = _cg(**kw)
    a = 0x4000
    assert lib.dc_attn_cg_fwd(ctypes.byref(p), a, a, a, a, a, None) == expect
    assert lib.dc_attn_cg_bwd(ctypes.byref(p), a, a, a, a, a, a, a, a, 1 << 30, None) == expect
    assert lib.dc_attn_cg_bwd_workspace_size(ctypes.byref(p)) == 0


def test_cg_limits_accepted(lib):
    """The largest shapes inside the limits pass the host checks (N = 0: nothing runs)."""
    for D, H, dt in ((4330, 6, dcattn.DC_BF16), (4330, 6, dcattn.DC_F32), (1560, 16, dcattn.DC_BF16), (2, 1, 0),
                     (6752, 4, dcattn.DC_BF16), (3376, 8, dcattn.DC_BF16)):
        p = _cg(model_dim=D, num_heads=H, num_tokens=0, dtype=dt)
        assert lib.dc_attn_cg_fwd(ctypes.byref(p), 0, 0, 0, 0, 0, None) == dcattn.DC_OK, (D, H, dt)


def test_cg_workspace_and_pointer_checks(lib):
    p = _cg()
    need = lib.dc_attn_cg_bwd_workspace_size(ctypes.byref(p))
    assert need == 4 * 16 * (12 * 768 + 12)            # ceil(1000 / 64) records of dweight + dbias
    p_big = _cg(num_tokens=10 ** 7)
    assert lib.dc_attn_cg_bwd_workspace_size(ctypes.byref(p_big)) == 4 * 148 * (12 * 768 + 12)
    a = 0x4000
    assert lib.dc_attn_cg_bwd(ctypes.byref(p), a, a, a, a, a, a, a, a, need - 1, None) == dcattn.DC_ERR_INVALID_ARG
    assert lib.dc_attn_cg_fwd(ctypes.byref(p), a + 8, a, a, a, a, None) == dcattn.DC_ERR_INVALID_ARG
    assert lib.dc_attn_cg_fwd(ctypes.byref(p), a, a, a, 0, a, None) == dcattn.DC_ERR_INVALID_ARG
    p0 = _cg(num_tokens=0)
    assert lib.dc_attn_cg_bwd_workspace_size(ctypes.byref(p0)) == 0
    assert lib.dc_attn_cg_fwd(ctypes.byref(p0), 0, 0, 0, 0, 0, None) == dcattn.DC_OK
    # N = 0 still writes dweight and dbias (zeros), so those two must be valid
    assert lib.dc_attn_cg_bwd(ctypes.byref(p0), 0, 0, 0, 0, 0, 0, 0, 0, 0, None) == dcattn.DC_ERR_INVALID_ARG


def test_cg_resolve_impl(lib):
    """bf16 x with TMA-addressable rows, a full 128-token tile, D >= 64 and the weight splits
    within shared memory runs on tcgen05; everything else on SIMT; forcing tcgen05 where it
    is not possible is refused."""
    tc, simt = dcattn.IMPLS["tcgen05"], dcattn.IMPLS["simt"]
    for kw, want in ((dict(), tc), (dict(dtype=dcattn.DC_F32), simt), (dict(num_tokens=127), simt),
                     (dict(stride_x=770), simt), (dict(stride_x=776), tc), (dict(model_dim=62), simt),
                     (dict(model_dim=2048, num_heads=8), tc), (dict(model_dim=2050, num_heads=8), simt),
                     (dict(model_dim=1024, num_heads=16), tc), (dict(model_dim=1026, num_heads=16), simt),
                     (dict(impl=simt), simt), (dict(impl=tc, dtype=dcattn.DC_F32), -1), (dict(impl=tc), tc),
                     (dict(impl=7), -1)):
        p = _cg(**kw)
        assert lib.dc_attn_cg_resolve_impl(ctypes.byref(p)) == want, kw
    p = _cg(impl=tc, dtype=dcattn.DC_F32)
    a = 0x4000
    assert lib.dc_attn_cg_fwd(ctypes.byref(p), a, a, a, a, a, None) == dcattn.DC_ERR_UNSUPPORTED


def test_cg_prepare_size_and_alignment(lib):
    """The weight image holds the three bf16 splits (3 x R rows x 128 bytes per 64 columns,
    R = 16 outputs per split for 2H <= 16, else 32), read by the forward and by dx; a
    misaligned image pointer is refused on the host."""
    p = _cg()
    assert lib.dc_attn_cg_prepare_size(ctypes.byref(p)) == 12 * 48 * 128
    p16 = _cg(num_heads=16, model_dim=1024)
    assert lib.dc_attn_cg_prepare_size(ctypes.byref(p16)) == 16 * 96 * 128
    a = 0x4000
    pm = _cg(weight_splits=a + 8)
    assert lib.dc_attn_cg_fwd(ctypes.byref(pm), a, a, a, a, a, None) == dcattn.DC_ERR_INVALID_ARG
    assert lib.dc_attn_cg_prepare(ctypes.byref(_cg()), a, a + 4, None) == dcattn.DC_ERR_INVALID_ARG
