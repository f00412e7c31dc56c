"""The backward entry point that allocates nothing (dc_attn_bwd_noalloc).

It exists for callers that cannot give the backward a scratch buffer: plugin
interfaces that hand an op only its inputs and outputs, and processes whose
device memory is reserved by their own pool at start-up so that no cudaMalloc
may follow.  Its scratch is a fixed 32 MiB array inside the library.  These
tests call it through the C ABI and compare it with dc_attn_bwd given a
caller-owned workspace of the same size, on the same inputs: both then run the
same kernels, so the results must be bit-identical.  Every problem runs twice
in a row and problems of different sizes follow one another, so whatever an
earlier call left in the shared array is there when the next one starts.
This file is collected last so a stop-at-first-failure run has already run
everything else.
"""
import ctypes

import pytest
import torch

from cross_head_dynamic_b200 import dcattn
from cross_head_dynamic_b200.inputs import CONFIGS, generate, random_problem
from parity_util import TOL, compare, run_oracle, to_cuda

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 32 << 20
NAMES = ("dq", "dk", "dv", "dc", "dg")


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


def _forward(x, impl):
    return dcattn.dc_attn_fwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["cu_seqlens"], x["window"], x["scale"],
                              impl=impl)


def _check_against_workspace_backward(pb, impl, ws_bytes=SCRATCH_BYTES, calls=2):
    """dc_attn_bwd_noalloc, `calls` times in a row, against dc_attn_bwd with a caller
    workspace of `ws_bytes` (the array's size unless a test wants a specific route)."""
    x = to_cuda(pb)
    o, lse, pmap = _forward(x, impl)
    args = (x["q"], x["k"], x["v"], x["c"], x["g"], x["dO"], lse, pmap, x["cu_seqlens"], x["window"], x["scale"])
    ws = torch.empty(ws_bytes, device="cuda", dtype=torch.uint8)
    ref = dcattn.dc_attn_bwd(*args, impl=impl, workspace=ws)
    torch.cuda.synchronize()
    got = None
    for _ in range(calls):
        got = dcattn.dc_attn_bwd_noalloc(*args, impl=impl)
        torch.cuda.synchronize()
        for name, a, b in zip(NAMES, got, ref):
            assert torch.equal(a, b), name
    assert dcattn.dc_attn_device_status(reset=True) == 0
    return {n: t.double().cpu().numpy() for n, t in zip(NAMES, got)}


@pytest.mark.parametrize("impl", ["auto", "simt"])
def test_noalloc_matches_workspace_backward_on_consecutive_calls(impl):
    problems = [random_problem(31, [1000, 600, 448], 6, 128, 112, dtype="bf16"),
                random_problem(32, [257, 3, 700], 6, 128, 112, dtype="bf16")]
    for pb in problems:               # the second problem is smaller: stale array contents must not leak
        got = _check_against_workspace_backward(pb, impl)
        rows, ref = run_oracle(pb)
        compare(got, rows, ref, TOL["bf16"], names=list(NAMES))


def test_noalloc_recomputing_key_pass_in_the_array():
    """65536 tokens, H6 x d128, W112 (the packed varlen batch): the dP band (N*W*4 =
    29.4 MB) fits the array but the ds band (H*N*272 = 107 MB) does not, so the key pass
    recomputes ds inside the array.  Checked against dc_attn_bwd given a band-sized
    workspace (the same route), and against the oracle on every token."""
    cfg = CONFIGS["varlen"]
    pb = generate(cfg)
    N, W = cfg.total_tokens, cfg.window
    assert N * W * 4 <= SCRATCH_BYTES < cfg.heads * N * 136 * 2
    got = _check_against_workspace_backward(pb, "auto", ws_bytes=N * W * 4)
    rows, ref = run_oracle(pb)
    compare(got, rows, ref, TOL["bf16"], names=list(NAMES))


def test_noalloc_window_segments_after_other_problems():
    """W = 256 (two window segments, dP band only) following the problems above, then a
    smaller one that leaves most of the array as the previous call wrote it."""
    for pb in (random_problem(34, [1500, 40, 700], 6, 128, 256, dtype="bf16"),
               random_problem(35, [300, 9], 6, 128, 256, dtype="bf16")):
        got = _check_against_workspace_backward(pb, "auto")
        rows, ref = run_oracle(pb)
        compare(got, rows, ref, TOL["bf16"], names=list(NAMES))


def test_noalloc_rejects_problems_beyond_the_scratch_array():
    x = to_cuda(random_problem(33, [64], 2, 64, 16, dtype="bf16"))
    lib = dcattn.load_library()
    W = 128
    N = SCRATCH_BYTES // (4 * W) + 1          # band of N * W fp32 entries just above 32 MiB
    p = dcattn.Params(dtype=dcattn.DC_BF16, impl=0, total_tokens=N, num_docs=1, num_heads=2, head_dim=64,
                      window=W, softmax_scale=0.125, reserved=0, cu_seqlens=x["cu_seqlens"].data_ptr())
    ptr = x["q"].data_ptr()
    rc = lib.dc_attn_bwd_noalloc(ctypes.byref(p), *([ptr] * 13), None)
    assert rc == dcattn.DC_ERR_UNSUPPORTED
    p.total_tokens = SCRATCH_BYTES // (4 * W)  # band exactly at the limit: accepted by the size check
    # the workspace size asked for also holds the ds band (H * N * 136 bf16, a faster key pass);
    # the no-alloc entry point needs only the band and falls back to the recomputing key pass
    assert lib.dc_attn_bwd_workspace_size(ctypes.byref(p)) == max(SCRATCH_BYTES, 2 * p.total_tokens * 136 * 2)
