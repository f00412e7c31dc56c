"""Token-range sharding (cross_head_dynamic_b200/sharded.py) on CPU: two and three gloo
ranks, each running the fp64 oracle on its extended range, must reproduce the
unsharded oracle on their own rows (documents crossing range boundaries included).
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from cross_head_dynamic_b200 import sharded  # noqa: E402


class OracleOps:
    """A shard's compute on the host: the fp64 oracle (test infrastructure)."""

    def __init__(self):
        import oracle
        self.oracle = oracle

    def fwd(self, q, k, v, c, g, cu, window, scale):
        o, lse, pmap = self.oracle.forward(q, k, v, c, g, cu, window, scale)
        return torch.from_numpy(o), torch.from_numpy(lse), torch.from_numpy(pmap)

    def bwd(self, q, k, v, c, g, dO, lse, pmap, cu, window, scale):
        return tuple(torch.from_numpy(x) for x in self.oracle.backward(q, k, v, c, g, dO, cu, window, scale))

    def add_(self, dst, src):
        dst += src


def _problem(seed, lens, H, d):
    gen = torch.Generator().manual_seed(seed)
    N = sum(lens)
    r = lambda *s: torch.randn(*s, generator=gen, dtype=torch.float64)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return dict(q=r(N, H, d), k=r(N, H, d), v=r(N, H, d), c=0.5 * r(N, H),
                g=0.5 + torch.rand(N, H, generator=gen, dtype=torch.float64), dO=r(N, H, d), cu=cu)


CASES = {
    # name: (doc lengths, window, rank bounds or None for an even split)
    "even_w9": ([30, 5, 50, 1, 34], 9, None),
    "uneven_w16": ([70, 3, 47], 16, [(0, 20), (20, 90), (90, 120)]),
    "one_doc_w16": ([96], 16, None),
    "w1_no_halo": ([40, 1, 39], 1, None),
    # four ranges, the middle ones exactly as long as the halo their right neighbour needs
    "min_ranges_w16": ([20, 45, 2, 33], 16, [(0, 40), (40, 55), (55, 70), (70, 100)]),
}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lens, W, bounds = CASES[case]
        x = _problem(3, lens, 2, 8)
        N = int(x["cu"][-1])
        bounds = bounds if bounds and len(bounds) == world else sharded.even_bounds(N, world)
        a, b = bounds[rank]
        ops, comm = OracleOps(), sharded.NeighbourComm()
        loc = {n: x[n][a:b].contiguous() for n in ("q", "k", "v", "c", "g", "dO")}
        o, ctx = sharded.sharded_forward(ops, comm, bounds, loc["q"], loc["k"], loc["v"], loc["c"], loc["g"],
                                         x["cu"], W, 0.3)
        grads = sharded.sharded_backward(ops, comm, bounds, ctx, loc["dO"])
        ref_o, _, _ = ops.fwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["cu"], W, 0.3)
        ref_g = ops.bwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["dO"], None, None, x["cu"], W, 0.3)
        errs = {"o": float((o - ref_o[a:b]).abs().max())}
        for n, got, ref in zip(("dq", "dk", "dv", "dc", "dg"), grads, ref_g):
            errs[n] = float((got - ref[a:b]).abs().max())
        out[rank] = errs
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("case", list(CASES))
def test_sharded_matches_unsharded_oracle(case, world):
    if world == 4 and case != "min_ranges_w16":
        pytest.skip("four ranks run on the case built for them")
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_main, args=(world, port, case, out), nprocs=world, join=True)
    for r in range(world):
        for n, e in out[r].items():
            assert e < 1e-12, (r, n, e)


def test_extended_seqlens():
    cu = [0, 30, 35, 85, 86, 120]
    assert sharded.extended_seqlens(cu, 0, 40).tolist() == [0, 30, 35, 40]
    assert sharded.extended_seqlens(cu, 32, 80).tolist() == [0, 3, 48]
    assert sharded.extended_seqlens(cu, 85, 120).tolist() == [0, 1, 35]


def test_bounds_checked():
    sharded.check_bounds([(0, 20), (20, 90), (90, 120)], 16)
    sharded.check_bounds([(0, 10), (10, 120)], 16)   # range 1 needs only the 10 tokens before it
    with pytest.raises(ValueError):   # range 1 (10 tokens) cannot supply the 15 halo rows of range 2
        sharded.check_bounds([(0, 30), (30, 40), (40, 120)], 16)
    with pytest.raises(ValueError):   # not contiguous
        sharded.check_bounds([(0, 50), (60, 120)], 16)
    assert sharded.even_bounds(10, 3) == [(0, 4), (4, 8), (8, 10)]
