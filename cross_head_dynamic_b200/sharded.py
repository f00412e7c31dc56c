"""Token-range sharding of one long packed token sequence over ranks, one GPU each.

Rank r holds the tokens [start_r, end_r) of q, k, v, c, g (and of dO in the backward).
A query sees keys up to W - 1 tokens back, so the first queries of a range need keys
that the left neighbour holds:

- forward: the left neighbour sends the k and v rows of its last h_r = min(W - 1,
  start_r) tokens (the halo); the rank runs the kernels on the extended range
  [start_r - h_r, end_r) with q, c and g zero on the halo rows and keeps the outputs
  of its own rows only;
- backward: the kernels run on the same extended range with dO zero on the halo rows,
  so the halo queries contribute nothing; the dk and dv rows computed for the halo
  keys are partial sums (this rank's queries only) and go back to the left
  neighbour, which adds them to its last rows.

Documents may cross range boundaries; the extended range's cu_seqlens are the
global boundaries that fall inside it.  Every range except the last must hold at
least min(W - 1, its end) tokens, since only the immediate neighbour sends a halo.
The exchange is point to point (torch.distributed isend/irecv: NCCL between GPUs);
the arithmetic runs in libdcattn (the kernels, and dc_attn_halo_add for the partial
sums).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


def halo_len(start: int, window: int) -> int:
    """Halo rows of a range starting at token `start`."""
    return min(window - 1, start)


def even_bounds(n_tokens: int, world: int) -> list:
    """[start, end) of each rank for an even split of n_tokens."""
    per = -(-n_tokens // world)
    return [(min(r * per, n_tokens), min((r + 1) * per, n_tokens)) for r in range(world)]


def check_bounds(bounds, window: int) -> None:
    """The ranges tile [0, N) in order and each can send its right neighbour's halo."""
    if not bounds or bounds[0][0] != 0:
        raise ValueError("ranges must start at token 0")
    for r, (a, b) in enumerate(bounds):
        if b < a or (r > 0 and a != bounds[r - 1][1]):
            raise ValueError("ranges must be contiguous and in rank order")
        if r + 1 < len(bounds) and b - a < halo_len(b, window):
            raise ValueError(f"range {r} holds {b - a} tokens, fewer than the {halo_len(b, window)} "
                             "halo rows its right neighbour needs")


def extended_seqlens(cu_global, a: int, b: int) -> torch.Tensor:
    """cu_seqlens (int32, CPU) of the token range [a, b): the global document
    boundaries inside it, shifted to start at 0."""
    cu = [int(x) for x in cu_global]
    inner = sorted({x for x in cu if a < x < b})
    return torch.tensor([0] + [x - a for x in inner] + [b - a], dtype=torch.int32)


class DcAttnOps:
    """The compute of a shard on its GPU: libdcattn's kernels."""

    def __init__(self, impl: str = "auto"):
        from cross_head_dynamic_b200 import dcattn
        self.dcattn = dcattn
        self.impl = impl

    def fwd(self, q, k, v, c, g, cu, window, scale):
        return self.dcattn.dc_attn_fwd(q, k, v, c, g, cu, window, scale, impl=self.impl)

    def bwd(self, q, k, v, c, g, dO, lse, pmap, cu, window, scale):
        return self.dcattn.dc_attn_bwd(q, k, v, c, g, dO, lse, pmap, cu, window, scale, impl=self.impl)

    def add_(self, dst, src):
        self.dcattn.dc_attn_halo_add(dst, src)


@dataclass
class ShardContext:
    """What the backward of a shard needs from its forward."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    c: torch.Tensor
    g: torch.Tensor
    lse: torch.Tensor
    pmap: torch.Tensor
    cu: torch.Tensor
    halo: int
    window: int
    scale: float


def _with_halo(x: torch.Tensor, halo_rows) -> torch.Tensor:
    """x with `halo_rows` (a tensor, or an int number of zero rows) in front."""
    if isinstance(halo_rows, int):
        if halo_rows == 0:
            return x
        halo_rows = torch.zeros((halo_rows,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    return torch.cat([halo_rows, x], dim=0)


def forward_local(ops, q, k, v, c, g, halo_kv, cu_ext, window: int, scale: float):
    """Forward of one range given its halo (k and v rows stacked as [2, h, H, d], or
    None when h = 0).  Returns (o of the range's own rows, context for the backward)."""
    h = 0 if halo_kv is None else int(halo_kv.shape[1])
    q_e, c_e, g_e = _with_halo(q, h), _with_halo(c, h), _with_halo(g, h)
    k_e = _with_halo(k, halo_kv[0]) if h else k
    v_e = _with_halo(v, halo_kv[1]) if h else v
    o, lse, pmap = ops.fwd(q_e, k_e, v_e, c_e, g_e, cu_ext, window, scale)
    ctx = ShardContext(q_e, k_e, v_e, c_e, g_e, lse, pmap, cu_ext, h, window, scale)
    return o[h:], ctx


def backward_local(ops, ctx: ShardContext, dO):
    """Backward of one range.  Returns (dq, dk, dv, dc, dg) of its own rows and the dk, dv
    partials of the halo keys stacked as [2, h, H, d] (None when h = 0)."""
    h = ctx.halo
    dO_e = _with_halo(dO, h)
    dq, dk, dv, dc, dg = ops.bwd(ctx.q, ctx.k, ctx.v, ctx.c, ctx.g, dO_e, ctx.lse, ctx.pmap, ctx.cu, ctx.window,
                                 ctx.scale)
    halo_grad = torch.stack([dk[:h], dv[:h]]).contiguous() if h else None
    return dq[h:], dk[h:].contiguous(), dv[h:].contiguous(), dc[h:], dg[h:], halo_grad


class NeighbourComm:
    """Point-to-point exchange with the left and right neighbour over torch.distributed."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def _run(self, ops):
        if ops:
            for req in self.dist.batch_isend_irecv(ops):
                req.wait()

    def shift_right(self, send, recv_shape, dtype, device):
        """Send `send` to rank + 1 (when there is one and send is not None) and receive a
        tensor of recv_shape from rank - 1 (when recv_shape has rows).  Returns it or None."""
        d, ops, out = self.dist, [], None
        if send is not None and self.rank + 1 < self.world:
            ops.append(d.P2POp(d.isend, send.contiguous(), self.rank + 1, self.group))
        if recv_shape is not None and self.rank > 0:
            out = torch.empty(recv_shape, dtype=dtype, device=device)
            ops.append(d.P2POp(d.irecv, out, self.rank - 1, self.group))
        self._run(ops)
        return out

    def shift_left(self, send, recv_shape, dtype, device):
        """Send `send` to rank - 1 and receive a tensor of recv_shape from rank + 1."""
        d, ops, out = self.dist, [], None
        if send is not None and self.rank > 0:
            ops.append(d.P2POp(d.isend, send.contiguous(), self.rank - 1, self.group))
        if recv_shape is not None and self.rank + 1 < self.world:
            out = torch.empty(recv_shape, dtype=dtype, device=device)
            ops.append(d.P2POp(d.irecv, out, self.rank + 1, self.group))
        self._run(ops)
        return out


def sharded_forward(ops, comm, bounds, q, k, v, c, g, cu_global, window: int, scale: float):
    """Forward of this rank's range (bounds[comm.rank]); q, k, v, c, g hold its rows.
    Returns (o of its rows, context for sharded_backward)."""
    check_bounds(bounds, window)
    a, b = bounds[comm.rank]
    h = halo_len(a, window)
    h_right = halo_len(b, window) if comm.rank + 1 < comm.world else 0
    send = torch.stack([k[len(k) - h_right:], v[len(v) - h_right:]]) if h_right else None
    recv_shape = (2, h) + tuple(k.shape[1:]) if h else None
    halo_kv = comm.shift_right(send, recv_shape, k.dtype, k.device)
    cu_ext = extended_seqlens(cu_global, a - h, b).to(q.device)
    return forward_local(ops, q, k, v, c, g, halo_kv, cu_ext, window, scale)


def sharded_backward(ops, comm, bounds, ctx: ShardContext, dO):
    """Backward of this rank's range.  Returns (dq, dk, dv, dc, dg) of its rows, with the
    right neighbour's partials for its last rows already added to dk and dv."""
    dq, dk, dv, dc, dg, halo_grad = backward_local(ops, ctx, dO)
    a, b = bounds[comm.rank]
    h_right = halo_len(b, ctx.window) if comm.rank + 1 < comm.world else 0
    recv_shape = (2, h_right) + tuple(dk.shape[1:]) if h_right else None
    part = comm.shift_left(halo_grad, recv_shape, dk.dtype, dk.device)
    if part is not None:
        ops.add_(dk[len(dk) - h_right:], part[0].contiguous())
        ops.add_(dv[len(dv) - h_right:], part[1].contiguous())
    return dq, dk, dv, dc, dg
