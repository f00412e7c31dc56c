"""Row strides: q, k, v (and dq, dk, dv) as views of one fused [N, 3, H, d] tensor, o and dO
as views of wider buffers.  The same kernels run on the same values, so every output must be
bit-identical to the call on contiguous copies; the gaps between the views must be left
untouched.  Covers the ds-tile backward (W = 112), the ds band (W = 64), window segments
(W = 200) and the SIMT kernels (fp32)."""
import pytest
import torch

from cross_head_dynamic_b200 import dcattn
from cross_head_dynamic_b200.inputs import random_problem
from parity_util import to_cuda

pytestmark = pytest.mark.gpu

SENTINEL = -7.0


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cross_head_dynamic_b200 import build
    build.build()
    dcattn.load_library()
    dcattn.dc_attn_device_status(reset=True)
    yield
    assert dcattn.dc_attn_device_status(reset=True) == 0


CASES = [
    ("tiles_w112", [700, 45, 300], 6, 128, 112, "bf16"),
    ("band_w64", [500, 77], 6, 128, 64, "bf16"),
    ("segments_w200", [600, 90], 4, 64, 200, "bf16"),
    ("simt_fp32", [300, 41], 4, 64, 40, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_strided_views_match_contiguous(case):
    _, lens, H, d, W, dtype = case
    x = to_cuda(random_problem(51, lens, H, d, W, dtype=dtype))
    N = x["q"].shape[0]
    dt = x["q"].dtype
    sc, cu = x["scale"], x["cu_seqlens"]
    # contiguous reference
    o0, lse0, pm0 = dcattn.dc_attn_fwd(x["q"], x["k"], x["v"], x["c"], x["g"], cu, W, sc)
    ref = dcattn.dc_attn_bwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["dO"], lse0, pm0, cu, W, sc)
    # fused views: qkv [N, 3, H, d], o and dO in [N, 2, H, d], dq/dk/dv into [N, 3, H, d]
    qkv = torch.stack([x["q"], x["k"], x["v"]], dim=1).contiguous()
    q, k, v = qkv[:, 0], qkv[:, 1], qkv[:, 2]
    obuf = torch.full((N, 2, H, d), SENTINEL, device="cuda", dtype=dt)
    dobuf = torch.full((N, 2, H, d), SENTINEL, device="cuda", dtype=dt)
    dobuf[:, 1] = x["dO"]
    dqkv = torch.full((N, 3, H, d), SENTINEL, device="cuda", dtype=dt)
    assert q.stride(0) == 3 * H * d and obuf[:, 0].stride(0) == 2 * H * d
    o, lse, pm = dcattn.dc_attn_fwd(q, k, v, x["c"], x["g"], cu, W, sc, o=obuf[:, 0])
    got = dcattn.dc_attn_bwd(q, k, v, x["c"], x["g"], dobuf[:, 1], lse, pm, cu, W, sc,
                             dq=dqkv[:, 0], dk=dqkv[:, 1], dv=dqkv[:, 2])
    torch.cuda.synchronize()
    assert torch.equal(o, o0) and torch.equal(lse, lse0) and torch.equal(pm, pm0)
    for name, a, b in zip(("dq", "dk", "dv", "dc", "dg"), got, ref):
        assert torch.equal(a, b), name
    assert bool((obuf[:, 1] == SENTINEL).all())          # the gap next to o is untouched
    assert torch.equal(dobuf[:, 1], x["dO"])              # dO is an input
    assert torch.equal(qkv[:, 0], x["q"]) and torch.equal(qkv[:, 2], x["v"])
