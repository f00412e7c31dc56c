"""Token-range sharding with libdcattn on one GPU: the shards of one sequence run one
after another in this process (the halo rows and the returned dk, dv partials are
handed over as tensors instead of over NCCL), and together must match the oracle on
every token.  The multi-rank exchange itself is covered on CPU (test_sharded.py).
"""
import numpy as np
import pytest
import torch

from cross_head_dynamic_b200 import dcattn, sharded
from cross_head_dynamic_b200.inputs import random_problem
from parity_util import TOL, compare, run_oracle, to_cuda

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
    assert dcattn.dc_attn_device_status(reset=True) == 0


@pytest.mark.parametrize("W", [112, 256])
def test_shards_in_sequence_match_oracle(W):
    inp = random_problem(12, [700, 45, 600, 155], 6, 128, W, dtype="bf16")
    x = to_cuda(inp)
    bounds = [(0, 500), (500, 1100), (1100, 1500)]
    sharded.check_bounds(bounds, W)
    ops = sharded.DcAttnOps()
    scale = x["scale"]
    rows = lambda t, a, b: t[a:b].contiguous()
    o_parts, ctxs = [], []
    for a, b in bounds:
        h = sharded.halo_len(a, W)
        halo = torch.stack([x["k"][a - h:a], x["v"][a - h:a]]).contiguous() if h else None
        cu = sharded.extended_seqlens(inp["cu_seqlens"], a - h, b).cuda()
        o, ctx = sharded.forward_local(ops, rows(x["q"], a, b), rows(x["k"], a, b), rows(x["v"], a, b),
                                       rows(x["c"], a, b), rows(x["g"], a, b), halo, cu, W, scale)
        o_parts.append(o)
        ctxs.append(ctx)
    grads = [list(sharded.backward_local(ops, ctx, rows(x["dO"], a, b))) for ctx, (a, b) in zip(ctxs, bounds)]
    for r in range(1, len(bounds)):   # each shard's halo partials go to its left neighbour's last rows
        part = grads[r][5]
        h = part.shape[1]
        ops.add_(grads[r - 1][1][-h:], part[0].contiguous())
        ops.add_(grads[r - 1][2][-h:], part[1].contiguous())
    torch.cuda.synchronize()
    cat = lambda i: torch.cat([g[i] for g in grads]).double().cpu().numpy()
    gpu = dict(o=torch.cat(o_parts).double().cpu().numpy(), dq=cat(0), dk=cat(1), dv=cat(2), dc=cat(3), dg=cat(4))
    rows_all, ref = run_oracle(inp)
    compare(gpu, rows_all, ref, TOL["bf16"], names=list(gpu))


def test_halo_add():
    a = torch.randn(1000, 6, 128, device="cuda").to(torch.bfloat16)
    b = torch.randn(1000, 6, 128, device="cuda").to(torch.bfloat16)
    want = (a.float() + b.float()).to(torch.bfloat16)
    dcattn.dc_attn_halo_add(a, b)
    assert torch.equal(a, want)
    f = torch.randn(333, device="cuda")
    f0 = f.clone()
    g = torch.randn(333, device="cuda")
    dcattn.dc_attn_halo_add(f, g)
    assert torch.equal(f, f0 + g)
