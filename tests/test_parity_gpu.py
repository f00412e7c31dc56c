"""GPU parity: libdcattn (through the C ABI) against the fp64 oracle on seeded inputs.

Metric per output tensor: max|gpu - oracle| / max|oracle|; bound 1e-5 for fp32
storage and 1.5e-2 for bf16 storage (fp32 accumulation on the GPU in both).
Every workload, the full-size ones included, is compared on every token of
every output tensor: each document boundary of the packed varlen batch falls
at its own offset inside a query block, and all of them are checked.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from cross_head_dynamic_b200 import dcattn
from cross_head_dynamic_b200.inputs import CONFIGS, generate, random_problem
from parity_util import BWD_OUT, FWD_OUT, TOL, compare, run_gpu, run_oracle, to_cuda

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


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


def test_tiny_fp32_parity():
    inp = generate(CONFIGS["tiny_fp32"])
    gpu = run_gpu(inp, impl="auto")
    rows, ref = run_oracle(inp)
    compare(gpu, rows, ref, TOL["f32"])


def test_worked_example_on_gpu():
    """The hand-derived example (d = 1) embedded in d = 32 with zero padding."""
    ex = json.load(open(GOLDEN))
    T, H, W = ex["T"], ex["H"], ex["W"]
    d = 32
    ln3 = math.log(3.0)
    pad = lambda a: torch.nn.functional.pad(torch.tensor(a, dtype=torch.float32).reshape(T, H, 1), (0, d - 1))
    q, k, v, dO = pad(ex["q"]), pad(np.array(ex["k_coef_ln3"]) * ln3), pad(ex["v"]), pad(ex["dO"])
    x = to_cuda(dict(q=q, k=k, v=v, dO=dO, c=torch.tensor(ex["c"], dtype=torch.float32),
                     g=torch.tensor(ex["g"], dtype=torch.float32),
                     cu_seqlens=torch.tensor(ex["cu_seqlens"], dtype=torch.int32)))
    o, lse, pmap = dcattn.dc_attn_fwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["cu_seqlens"], W, 1.0)
    dq, dk, dv, dc, dg = dcattn.dc_attn_bwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["dO"], lse, pmap,
                                            x["cu_seqlens"], W, 1.0)
    e = ex["expect"]
    tol = 1e-6
    np.testing.assert_allclose(o[:, :, 0].cpu(), e["o"], atol=tol)
    assert float(o[:, :, 1:].abs().max()) == 0.0
    np.testing.assert_allclose(lse.cpu(), np.log(np.array(e["lse_ln"], dtype=np.float64)), atol=tol)
    np.testing.assert_allclose(pmap.cpu(), e["pmap"], atol=tol)
    np.testing.assert_allclose(dg.cpu(), e["dg"], atol=tol)
    np.testing.assert_allclose(dc.cpu(), e["dc"], atol=tol)
    np.testing.assert_allclose(dv[:, :, 0].cpu(), e["dv"], atol=tol)
    np.testing.assert_allclose(dk[:, :, 0].cpu(), e["dk"], atol=tol)
    np.testing.assert_allclose(dq[:, :, 0].cpu(), np.array(e["dq_coef_ln3"]) * ln3, atol=tol)


EDGE_CASES = [
    # id, doc lengths, H, d, W, dtype
    ("ragged_tail", [300, 77], 4, 64, 112, "f32"),
    ("single_tokens", [1] * 40, 3, 64, 8, "f32"),
    ("empty_doc", [50, 0, 90], 2, 32, 16, "f32"),
    ("w1", [130], 2, 64, 1, "f32"),
    ("w_ge_T", [200], 2, 64, 256, "f32"),
    ("n1", [1], 1, 32, 112, "f32"),
    ("h16_d96", [70, 61], 16, 96, 20, "f32"),
    ("bf16_ragged", [333, 1, 250], 6, 128, 112, "bf16"),
    ("bf16_d64_h12", [400, 129], 12, 64, 64, "bf16"),
    ("bf16_w1", [260], 6, 128, 1, "bf16"),
    ("bf16_short_docs", [5, 17, 3, 200, 9], 6, 128, 112, "bf16"),
    ("bf16_h1", [300, 50], 1, 128, 112, "bf16"),
    # the widest window the tcgen05 kernels take in one piece (7 chunks of 8 columns per
    # thread), the most heads, and the first window past it
    ("bf16_w129", [700, 45], 4, 128, 129, "bf16"),
    # windows of 97-113 keys hand ds from the query side to the key side as whole tiles
    # (key tile starting 112 keys before the block): the smallest and largest such window,
    # one in between with d = 64 and twelve heads, documents starting inside blocks
    ("bf16_w97_tiles", [333, 90, 1], 6, 128, 97, "bf16"),
    ("bf16_w113_tiles", [400, 2, 300], 3, 128, 113, "bf16"),
    ("bf16_w100_d64_tiles", [500, 37, 260], 12, 64, 100, "bf16"),
    ("bf16_w120_h16_d64", [520], 16, 64, 120, "bf16"),
    # W > 129: a near segment of 128 keys and a far one of W - 128 (2 keys at W = 130); documents
    # shorter than the near segment (far segment empty), windows past the document start,
    # segment offsets that are not multiples of 8 (W = 200, 250), one head, sixteen heads
    ("bf16_w130", [300], 2, 64, 130, "bf16"),
    ("bf16_w256_docs", [700, 45, 200, 3, 130], 6, 128, 256, "bf16"),
    ("bf16_w200_h12_d64", [600, 90], 12, 64, 200, "bf16"),
    ("bf16_w250_h16_d64", [520], 16, 64, 250, "bf16"),
    ("bf16_w256_h1", [1100], 1, 128, 256, "bf16"),
    ("bf16_w256_short", [100, 60], 4, 128, 256, "bf16"),
    # SIMT kernels: key tiles of 4 consecutive keys (N >= 16 keys per SM) with a ragged last
    # tile and documents ending inside tiles; a window past the tcgen05 range; a forward
    # whose scores (H * W floats) do not fit the shared-memory budget and are recomputed
    ("simt_key_tiles", [1500, 3, 1100], 6, 64, 112, "f32"),
    ("bf16_simt_key_tiles", [2500, 1, 99], 6, 128, 112, "bf16"),
    ("w300", [700, 500], 4, 64, 300, "f32"),
    ("w1100_h16_scores_recomputed", [1200], 16, 32, 1100, "f32"),
]


@pytest.mark.parametrize("case", EDGE_CASES, ids=[c[0] for c in EDGE_CASES])
@pytest.mark.parametrize("impl", ["auto", "simt"])
def test_edge_cases(case, impl):
    _, lens, H, d, W, dtype = case
    inp = random_problem(21, lens, H, d, W, dtype=dtype)
    gpu = run_gpu(inp, impl=impl)
    rows, ref = run_oracle(inp)
    compare(gpu, rows, ref, TOL[dtype])


CONFIG_NAMES = [n for n in CONFIGS if n != "tiny_fp32"]


@pytest.mark.parametrize("name", CONFIG_NAMES)
def test_config_parity(name):
    """Full-size workload in the launch configuration the benchmark times, every row."""
    cfg = CONFIGS[name]
    inp = generate(cfg)
    gpu = run_gpu(inp, backward=cfg.backward)
    rows, ref = run_oracle(inp, backward=cfg.backward)
    assert len(rows) == cfg.total_tokens
    compare(gpu, rows, ref, TOL[cfg.dtype])


def test_bf16_impls_agree_with_oracle_on_same_rows():
    """tcgen05 path (when AUTO picks it) and SIMT path on the same bf16 input."""
    inp = random_problem(5, [1000, 600, 448], 6, 128, 112, dtype="bf16")
    rows, ref = run_oracle(inp)
    for impl in ("auto", "simt"):
        compare(run_gpu(inp, impl=impl), rows, ref, TOL["bf16"])


def test_deterministic():
    inp = random_problem(6, [700, 324], 6, 128, 112, dtype="bf16")
    a = run_gpu(inp)
    b = run_gpu(inp)
    for n in FWD_OUT + BWD_OUT:
        assert np.array_equal(a[n], b[n]), n


@pytest.mark.parametrize("W", [112, 256])
def test_guard_bands_untouched(W):
    """Outputs written into the middle of larger buffers: sentinels around them survive
    (W = 256: the window-segment kernels, which add into o, dq, dk and dv)."""
    inp = to_cuda(random_problem(7, [257, 130], 6, 128, W, dtype="bf16"))
    N, H, d = inp["q"].shape
    W = inp["window"]
    G = 4096

    def guarded(numel, dtype):
        buf = torch.full((numel + 2 * G,), 7.0, device="cuda", dtype=dtype)
        return buf, buf[G:G + numel]

    bo, o = guarded(N * H * d, torch.bfloat16)
    bl, lse = guarded(N * H, torch.float32)
    bp, pm = guarded(N * W, torch.bfloat16)
    dcattn.dc_attn_fwd(inp["q"], inp["k"], inp["v"], inp["c"], inp["g"], inp["cu_seqlens"], W, inp["scale"],
                       o=o.view(N, H, d), lse=lse.view(N, H), pmap=pm.view(N, W))
    bufs = {}
    for nm, numel, dt in (("dq", N * H * d, torch.bfloat16), ("dk", N * H * d, torch.bfloat16),
                          ("dv", N * H * d, torch.bfloat16), ("dc", N * H, torch.float32),
                          ("dg", N * H, torch.float32)):
        bufs[nm] = guarded(numel, dt)
    ws_need = dcattn.dc_attn_bwd_workspace_size(inp["q"], inp["cu_seqlens"], W, inp["scale"])
    bws, ws = guarded(ws_need, torch.uint8)
    dcattn.dc_attn_bwd(inp["q"], inp["k"], inp["v"], inp["c"], inp["g"], inp["dO"], lse.view(N, H), pm.view(N, W),
                       inp["cu_seqlens"], W, inp["scale"], dq=bufs["dq"][1].view(N, H, d),
                       dk=bufs["dk"][1].view(N, H, d), dv=bufs["dv"][1].view(N, H, d),
                       dc=bufs["dc"][1].view(N, H), dg=bufs["dg"][1].view(N, H), workspace=ws)
    torch.cuda.synchronize()
    for buf in [bo, bl, bp, bws] + [b for b, _ in bufs.values()]:
        assert bool((buf[:G] == 7).all()) and bool((buf[-G:] == 7).all())


@pytest.mark.parametrize("W", [112, 129])
def test_backward_with_band_sized_workspace(W):
    """A workspace of only N * W * 4 bytes (the dP band) is too small for the ds band, so
    the key side recomputes ds from S^T; both backward pairs must match the oracle."""
    inp = random_problem(10, [700, 45, 300], 6, 128, W, dtype="bf16")
    x = to_cuda(inp)
    N = x["q"].shape[0]
    o, lse, pmap = dcattn.dc_attn_fwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["cu_seqlens"], W, x["scale"])
    ws = torch.empty(N * W * 4, device="cuda", dtype=torch.uint8)
    assert ws.numel() < dcattn.dc_attn_bwd_workspace_size(x["q"], x["cu_seqlens"], W, x["scale"])
    dq, dk, dv, dc, dg = dcattn.dc_attn_bwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["dO"], lse, pmap,
                                            x["cu_seqlens"], W, x["scale"], workspace=ws)
    torch.cuda.synchronize()
    gpu = {n: t.double().cpu().numpy() for n, t in dict(dq=dq, dk=dk, dv=dv, dc=dc, dg=dg).items()}
    rows, ref = run_oracle(inp)
    compare(gpu, rows, ref, TOL["bf16"], names=list(gpu))


def test_segmented_forward_without_lse():
    """W > 129 without an lse buffer: AUTO serves it on the SIMT kernels, an explicit
    tcgen05 request is refused before any launch."""
    inp = to_cuda(random_problem(9, [300], 2, 64, 200, dtype="bf16"))
    args = (inp["q"], inp["k"], inp["v"], inp["c"], inp["g"], inp["cu_seqlens"], 200, inp["scale"])
    o, lse, pmap = dcattn.dc_attn_fwd(*args, need_backward=False)
    assert lse is None and pmap is None
    o_ref, _, _ = dcattn.dc_attn_fwd(*args, impl="simt")
    assert torch.equal(o, o_ref)
    with pytest.raises(dcattn.DCAttnError):
        dcattn.dc_attn_fwd(*args, need_backward=False, impl="tcgen05")


def test_malformed_seqlens_flagged_not_faulting():
    """Non-monotonic cu_seqlens: the call completes, the status word says so."""
    inp = to_cuda(random_problem(8, [64, 64], 2, 64, 16, dtype="bf16"))
    bad = torch.tensor([0, 100, 40, 128], dtype=torch.int32, device="cuda")
    dcattn.dc_attn_device_status(reset=True)
    o, lse, pmap = dcattn.dc_attn_fwd(inp["q"], inp["k"], inp["v"], inp["c"], inp["g"], bad, 16, inp["scale"])
    dcattn.dc_attn_bwd(inp["q"], inp["k"], inp["v"], inp["c"], inp["g"], inp["dO"], lse, pmap, bad, 16,
                       inp["scale"])
    st = dcattn.dc_attn_device_status(reset=True)
    assert st & dcattn.DC_DEVERR_SEQLENS
    bad2 = torch.tensor([0, 64, 127], dtype=torch.int32, device="cuda")   # does not end at N
    dcattn.dc_attn_fwd(inp["q"], inp["k"], inp["v"], inp["c"], inp["g"], bad2, 16, inp["scale"])
    assert dcattn.dc_attn_device_status(reset=True) & dcattn.DC_DEVERR_SEQLENS
    dcattn.dc_attn_fwd(inp["q"], inp["k"], inp["v"], inp["c"], inp["g"], inp["cu_seqlens"], 16, inp["scale"])
    assert dcattn.dc_attn_device_status(reset=True) == 0
