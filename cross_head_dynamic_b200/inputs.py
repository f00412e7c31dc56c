"""Seeded synthetic inputs for Lightweight DC attention.

This module is the only code shared by the CUDA path's tests/bench and the
fp64 oracle's tests: it draws random numbers and lays them out, and it holds
none of the attention arithmetic.

Workloads (the five problem settings of the "Lightweight DC" description on the
m.aitntnews.com blog post, section "第二刀-砍层内": 112-token local window,
GPT-2-small attention shape with d_model 768 split into 6 heads of 128):

  tiny_fp32     B1  T256   H4  d64  W112, fp32, q drawn N(0,1) then divided by
                sqrt(d) (softmax scale 1), single document
  gpt2_fwd      B8  T2048  H6  d128 W112, bf16, one document per row
  gpt2_fwdbwd   same shape, plus dO (the headline fwd+bwd workload)
  varlen        B1  T65536 H6  d128 W112, bf16, packed documents with lengths
                ~ Geometric(mean 900) clipped to [16, 8192]
  sweep_*       B4  T16384, W in {32,64,112,256} x (H,d) in {(6,128),(12,64)},
                bf16, one document per row, seed 100 + point index (W-major)

Value recipe: q, k, v, dO ~ N(0,1); c ~ N(0, 0.5^2) (signed composition
weights); g ~ U(0.5, 1.5) (per-token head scale).  Draw order from one
torch CPU generator seeded with the config seed: q, k, v, c, g, dO.  Document
lengths come from numpy.random.default_rng(seed).  bf16 configs draw in fp32
and round to bf16 (round-to-nearest-even, torch's conversion); c and g stay
fp32.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class DCConfig:
    name: str
    batch: int
    seqlen: int
    heads: int
    head_dim: int
    window: int
    dtype: str            # "f32" or "bf16": storage/arithmetic type of q, k, v, o, dO, dq, dk, dv
    docs: str             # "rows": one document per batch row; "geometric": packed varlen
    seed: int
    q_prescaled: bool = False   # q already divided by sqrt(d); softmax scale 1
    backward: bool = True

    @property
    def total_tokens(self) -> int:
        return self.batch * self.seqlen

    @property
    def softmax_scale(self) -> float:
        return 1.0 if self.q_prescaled else 1.0 / math.sqrt(self.head_dim)

    def replace(self, **kw) -> "DCConfig":
        return dataclasses.replace(self, **kw)


SWEEP_WINDOWS = (32, 64, 112, 256)
SWEEP_HEADS = ((6, 128), (12, 64))


def _sweep_configs():
    out = {}
    idx = 0
    for w in SWEEP_WINDOWS:
        for (h, d) in SWEEP_HEADS:
            name = f"sweep_W{w}_H{h}_d{d}"
            out[name] = DCConfig(name, 4, 16384, h, d, w, "bf16", "rows", 100 + idx)
            idx += 1
    return out


CONFIGS = {
    "tiny_fp32": DCConfig("tiny_fp32", 1, 256, 4, 64, 112, "f32", "rows", 0, q_prescaled=True),
    "gpt2_fwd": DCConfig("gpt2_fwd", 8, 2048, 6, 128, 112, "bf16", "rows", 0, backward=False),
    "gpt2_fwdbwd": DCConfig("gpt2_fwdbwd", 8, 2048, 6, 128, 112, "bf16", "rows", 0),
    "varlen": DCConfig("varlen", 1, 65536, 6, 128, 112, "bf16", "geometric", 0),
    **_sweep_configs(),
}

GEOM_MEAN = 900
GEOM_MIN = 16
GEOM_MAX = 8192


def geometric_doc_lengths(seqlen: int, rng: np.random.Generator) -> list[int]:
    """Document lengths for one packed row of `seqlen` tokens.

    Lengths ~ Geometric(p = 1/900) (support >= 1, mean 900), clipped to
    [16, 8192].  The last document is cut so the row ends exactly at `seqlen`;
    a cut remainder shorter than 16 tokens is merged into the previous document.
    """
    lens: list[int] = []
    total = 0
    while total < seqlen:
        n = int(np.clip(rng.geometric(1.0 / GEOM_MEAN), GEOM_MIN, GEOM_MAX))
        n = min(n, seqlen - total)
        lens.append(n)
        total += n
    if len(lens) > 1 and lens[-1] < GEOM_MIN:
        last = lens.pop()
        lens[-1] += last
    return lens


def cu_seqlens_for(cfg: DCConfig) -> torch.Tensor:
    """int32 prefix sums of document lengths over the packed [B*T] token axis."""
    if cfg.docs == "rows":
        lens = [cfg.seqlen] * cfg.batch
    elif cfg.docs == "geometric":
        rng = np.random.default_rng(cfg.seed)
        lens = []
        for _ in range(cfg.batch):
            lens.extend(geometric_doc_lengths(cfg.seqlen, rng))
    else:
        raise ValueError(f"unknown document recipe {cfg.docs!r}")
    cu = np.zeros(len(lens) + 1, dtype=np.int64)
    np.cumsum(np.asarray(lens, dtype=np.int64), out=cu[1:])
    return torch.from_numpy(cu.astype(np.int32))


def generate(cfg: DCConfig) -> dict:
    """All inputs of one workload as CPU tensors.

    Returns q, k, v, dO as [N, H, d] (fp32 or bf16), c, g as [N, H] fp32,
    cu_seqlens int32 [num_docs + 1], and the scalars window/scale.
    """
    N, H, d = cfg.total_tokens, cfg.heads, cfg.head_dim
    gen = torch.Generator().manual_seed(cfg.seed)
    q = torch.randn(N, H, d, generator=gen)
    k = torch.randn(N, H, d, generator=gen)
    v = torch.randn(N, H, d, generator=gen)
    c = torch.randn(N, H, generator=gen) * 0.5
    g = torch.rand(N, H, generator=gen) + 0.5
    dO = torch.randn(N, H, d, generator=gen) if cfg.backward else None
    if cfg.q_prescaled:
        q = q / math.sqrt(d)
    if cfg.dtype == "bf16":
        q, k, v = q.bfloat16(), k.bfloat16(), v.bfloat16()
        if dO is not None:
            dO = dO.bfloat16()
    elif cfg.dtype != "f32":
        raise ValueError(f"unknown dtype {cfg.dtype!r}")
    return dict(q=q, k=k, v=v, c=c.contiguous(), g=g.contiguous(), dO=dO,
                cu_seqlens=cu_seqlens_for(cfg), window=cfg.window,
                scale=cfg.softmax_scale)


def random_problem(seed: int, doc_lens, heads: int, head_dim: int, window: int,
                   dtype: str = "f32", scale: float | None = None,
                   c_std: float = 0.5) -> dict:
    """A small ad-hoc problem with explicit document lengths (tests, edge cases)."""
    lens = [int(x) for x in doc_lens]
    N = sum(lens)
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(N, heads, head_dim, generator=gen)
    k = torch.randn(N, heads, head_dim, generator=gen)
    v = torch.randn(N, heads, head_dim, generator=gen)
    c = torch.randn(N, heads, generator=gen) * c_std
    g = torch.rand(N, heads, generator=gen) + 0.5
    dO = torch.randn(N, heads, head_dim, generator=gen)
    if dtype == "bf16":
        q, k, v, dO = q.bfloat16(), k.bfloat16(), v.bfloat16(), dO.bfloat16()
    cu = np.zeros(len(lens) + 1, dtype=np.int64)
    if lens:
        np.cumsum(np.asarray(lens, dtype=np.int64), out=cu[1:])
    return dict(q=q, k=k, v=v, c=c, g=g, dO=dO,
                cu_seqlens=torch.from_numpy(cu.astype(np.int32)), window=window,
                scale=(1.0 / math.sqrt(head_dim)) if scale is None else scale)


def cg_problem(seed: int, n_tokens: int, model_dim: int, heads: int, dtype: str = "bf16") -> dict:
    """Seeded inputs for the producer of c and g (random numbers only): x [N, D] ~ N(0,1)
    in `dtype` (bf16 rounded from fp32, or fp32); w [D, 2H] fp32 ~ N(0, 0.25 / D), so that
    the projected c has a standard deviation near 0.5; b [2H] fp32 with the c half ~ N(0, 0.1)
    and the g half 1 + N(0, 0.1); dc, dg [N, H] fp32 ~ N(0, 1).  Draw order: x, w, b, dc, dg."""
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(n_tokens, model_dim, generator=gen)
    w = torch.randn(model_dim, 2 * heads, generator=gen) * math.sqrt(0.25 / model_dim)
    b = torch.randn(2 * heads, generator=gen) * 0.1
    b[heads:] += 1.0
    dc = torch.randn(n_tokens, heads, generator=gen)
    dg = torch.randn(n_tokens, heads, generator=gen)
    if dtype == "bf16":
        x = x.to(torch.bfloat16)
    elif dtype != "f32":
        raise ValueError(f"unknown dtype {dtype!r}")
    return dict(x=x, w=w, b=b, dc=dc, dg=dg)
