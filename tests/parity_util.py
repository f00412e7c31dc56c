"""Helpers for GPU-vs-oracle parity tests (test infrastructure)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from cross_head_dynamic_b200 import dcattn

TOL = {"f32": 1e-5, "bf16": 1.5e-2}
FWD_OUT = ("o", "lse", "pmap")
BWD_OUT = ("dq", "dk", "dv", "dc", "dg")


def rel_err(got, ref) -> float:
    """max |got - ref| / max |ref| (absolute error when ref is all zero)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    den = float(np.max(np.abs(ref)))
    num = float(np.max(np.abs(got - ref)))
    if not np.isfinite(num):
        return float("inf")
    return num / den if den > 0 else num


def to_cuda(inp: dict) -> dict:
    out = {}
    for key, val in inp.items():
        out[key] = val.cuda() if isinstance(val, torch.Tensor) else val
    return out


def run_gpu(inp: dict, impl: str = "auto", backward: bool = True) -> dict:
    x = to_cuda(inp)
    o, lse, pmap = dcattn.dc_attn_fwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["cu_seqlens"], x["window"],
                                      x["scale"], impl=impl)
    res = dict(o=o, lse=lse, pmap=pmap)
    if backward:
        dq, dk, dv, dc, dg = dcattn.dc_attn_bwd(x["q"], x["k"], x["v"], x["c"], x["g"], x["dO"], lse, pmap,
                                                x["cu_seqlens"], x["window"], x["scale"], impl=impl)
        res.update(dq=dq, dk=dk, dv=dv, dc=dc, dg=dg)
    torch.cuda.synchronize()
    return {k2: v2.double().cpu().numpy() for k2, v2 in res.items()}


def doc_token_ranges(cu, docs):
    cu = [int(x) for x in cu]
    return [(cu[i], cu[i + 1]) for i in docs]


def run_oracle(inp: dict, docs=None, backward: bool = True):
    """Oracle outputs on all tokens, or only on the whole documents `docs`.

    Documents are independent, so the oracle run on a subset of complete
    documents gives the exact expected values for their tokens.  Returns
    (rows, outputs) with rows the token indices covered."""
    cu = inp["cu_seqlens"].numpy()
    if docs is None:
        rows = np.arange(int(cu[-1]))
        sub_cu = cu
    else:
        ranges = doc_token_ranges(cu, docs)
        rows = np.concatenate([np.arange(a, b) for a, b in ranges])
        lens = [b - a for a, b in ranges]
        sub_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    take = lambda t: t[torch.from_numpy(rows)] if t is not None else None
    q, k, v, c, g, dO = (take(inp[n]) for n in ("q", "k", "v", "c", "g", "dO"))
    o, lse, pmap = oracle.forward(q, k, v, c, g, sub_cu, inp["window"], inp["scale"])
    out = dict(o=o, lse=lse, pmap=pmap)
    if backward:
        dq, dk, dv, dc, dg = oracle.backward(q, k, v, c, g, dO, sub_cu, inp["window"], inp["scale"])
        out.update(dq=dq, dk=dk, dv=dv, dc=dc, dg=dg)
    return rows, out


def compare(gpu: dict, rows, ref: dict, tol: float, names=None):
    names = names or list(ref.keys())
    errs = {n: rel_err(gpu[n][rows], ref[n]) for n in names}
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, f"parity failed (tol {tol:g}): {errs}"
    return errs
