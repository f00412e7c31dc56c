"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait of a tcgen05 kernel on one of its own pipeline stages has a time limit;
when it runs out the CTA records DC_DEVERR_TIMEOUT in the device status word, skips
the rest of its work and exits normally.  Here the wait is made to run out on purpose:
the library is asked to leave out one tile load (one that is never issued, so nothing
is in flight when the CTA exits) with a 2 ms limit.  The call must return, the status
word must say what happened, and the next call on the same context must be correct.
"""
import time

import pytest
import torch

from cross_head_dynamic_b200 import dcattn
from cross_head_dynamic_b200.inputs import random_problem
from parity_util import TOL, compare, run_gpu, run_oracle, to_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cross_head_dynamic_b200 import build
    build.build()
    dcattn.load_library()
    dcattn.dc_attn_device_status(reset=True)
    yield
    dcattn.dc_attn_set_wait_limit(0)
    assert dcattn.dc_attn_device_status(reset=True) == 0


def test_missing_load_times_out_and_context_stays_usable():
    inp = random_problem(41, [700, 300], 6, 128, 112, dtype="bf16")
    x = to_cuda(inp)
    assert dcattn.dc_attn_resolve_impl(x["q"], x["cu_seqlens"], x["window"], x["scale"]) == "tcgen05"
    args = (x["q"], x["k"], x["v"], x["c"], x["g"], x["cu_seqlens"], x["window"], x["scale"])
    dcattn.dc_attn_fwd(*args)                   # warm: module loaded, first-launch costs paid
    assert dcattn.dc_attn_device_status(reset=True) == 0
    dcattn.dc_attn_set_wait_limit(2_000_000)    # 2 ms
    try:
        dcattn.dc_attn_inject_missing_load()
        t = time.perf_counter()
        dcattn.dc_attn_fwd(*args)
        status = dcattn.dc_attn_device_status(reset=True)   # synchronizes the stream
        elapsed = time.perf_counter() - t
    finally:
        dcattn.dc_attn_set_wait_limit(0)
    assert status & dcattn.DC_DEVERR_TIMEOUT, status
    assert elapsed < 1.0, elapsed               # the 2 ms limit, not the 2 s default
    # the hook was one-shot and the context is intact: the same problem is right again
    gpu = run_gpu(inp)
    rows, ref = run_oracle(inp)
    compare(gpu, rows, ref, TOL["bf16"])
    assert dcattn.dc_attn_device_status(reset=True) == 0
