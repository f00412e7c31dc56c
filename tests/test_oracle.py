"""Pins for the fp64 oracle, each against something other than the oracle itself.

- a hand-derived worked example (tests/golden/worked_example.*),
- brute force on tiny inputs: dense T x T score matrices with an explicit
  window/document/causal mask, and torch autograd of that dense form for the
  gradients,
- library routines the method reduces to in special cases (torch's
  scaled_dot_product_attention with a causal or banded mask),
- closed forms and invariants (softmax rows sum to 1, locality, constant V,
  gradient identities from homogeneity and shift invariance, scale folding, W=1),
- central finite differences for every input element.

The definition being pinned is the Lightweight DC paragraph of the
m.aitntnews.com blog post (section 第二刀-砍层内); see oracle/dc_oracle.c.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from cross_head_dynamic_b200.inputs import random_problem

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


# ----------------------------------------------------------------------------
# brute force: dense matrices, explicit masks (independent of the oracle code)
# ----------------------------------------------------------------------------

def dense_mask(cu, N, W):
    cu = np.asarray(cu)
    doc = np.searchsorted(cu, np.arange(N), side="right") - 1
    t = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    return (j <= t) & (j >= t - W + 1) & (doc[:, None] == doc[None, :])


def dense_forward_torch(q, k, v, c, g, cu, W, scale):
    """o via full [H, N, N] score tensors, -inf outside the mask, dense softmax."""
    N = q.shape[0]
    mask = torch.from_numpy(dense_mask(cu, N, W))
    S = scale * torch.einsum("thd,jhd->htj", q, k)
    S = S.masked_fill(~mask, float("-inf"))
    p = torch.softmax(S, dim=-1)
    P = torch.einsum("th,htj->tj", c, p)
    o = g[:, :, None] * torch.einsum("tj,jhd->thd", P, v)
    lse = torch.logsumexp(S, dim=-1).T
    return o, lse, P


def as64(x):
    return x.detach().double().clone()


def band_of(P, W):
    N = P.shape[0]
    out = np.zeros((N, W))
    for t in range(N):
        for w in range(W):
            j = t - W + 1 + w
            if j >= 0:
                out[t, w] = P[t, j]
    return out


def max_rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.max(np.abs(b)) if b.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(a - b))) if a.size else 0.0
    return float(np.max(np.abs(a - b)) / den)


# ----------------------------------------------------------------------------
# worked example
# ----------------------------------------------------------------------------

def test_worked_example(oracle_mod):
    ex = json.load(open(GOLDEN))
    ln3 = math.log(3.0)
    T, H, d, W = ex["T"], ex["H"], ex["d"], ex["W"]
    q = np.array(ex["q"], dtype=np.float64).reshape(T, H, d)
    k = (np.array(ex["k_coef_ln3"], dtype=np.float64) * ln3).reshape(T, H, d)
    v = np.array(ex["v"], dtype=np.float64).reshape(T, H, d)
    c = np.array(ex["c"], dtype=np.float64)
    g = np.array(ex["g"], dtype=np.float64)
    dO = np.array(ex["dO"], dtype=np.float64).reshape(T, H, d)
    cu = ex["cu_seqlens"]
    e = ex["expect"]
    o, lse, pmap = oracle_mod.forward(q, k, v, c, g, cu, W, ex["scale"])
    np.testing.assert_allclose(o.reshape(T, H), e["o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.log(np.array(e["lse_ln"], dtype=np.float64)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(pmap, e["pmap"], rtol=0, atol=1e-12)
    dq, dk, dv, dc, dg = oracle_mod.backward(q, k, v, c, g, dO, cu, W, ex["scale"])
    np.testing.assert_allclose(dg, e["dg"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dc, e["dc"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv.reshape(T, H), e["dv"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk.reshape(T, H), e["dk"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dq.reshape(T, H), np.array(e["dq_coef_ln3"]) * ln3, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# brute force forward + autograd backward on tiny problems
# ----------------------------------------------------------------------------

BRUTE_CASES = [
    # doc lengths, H, d, W, scale
    ([16], 3, 5, 4, 0.7),
    ([5, 11], 3, 5, 4, 0.7),
    ([1, 6, 1, 8], 2, 3, 3, 1.3),
    ([7, 9], 4, 2, 16, 0.5),       # W >= every document: full causal attention per document
    ([12], 2, 4, 1, 1.0),          # W = 1: only the query itself
    ([3, 0, 9], 2, 3, 5, 0.9),     # an empty document in cu_seqlens
]


@pytest.mark.parametrize("lens,H,d,W,scale", BRUTE_CASES)
def test_brute_force_forward(oracle_mod, lens, H, d, W, scale):
    pb = random_problem(11, lens, H, d, W, scale=scale, c_std=0.8)
    q, k, v, c, g = (as64(pb[n]) for n in ("q", "k", "v", "c", "g"))
    cu = pb["cu_seqlens"].numpy()
    o_ref, lse_ref, P_ref = dense_forward_torch(q, k, v, c, g, cu, W, scale)
    o, lse, pmap = oracle_mod.forward(q, k, v, c, g, cu, W, scale)
    assert max_rel(o, o_ref.numpy()) < 1e-12
    assert max_rel(lse, lse_ref.numpy()) < 1e-12
    assert max_rel(pmap, band_of(P_ref.numpy(), W)) < 1e-12


@pytest.mark.parametrize("lens,H,d,W,scale", BRUTE_CASES)
def test_autograd_backward(oracle_mod, lens, H, d, W, scale):
    pb = random_problem(12, lens, H, d, W, scale=scale, c_std=0.8)
    ins = {n: as64(pb[n]).requires_grad_(True) for n in ("q", "k", "v", "c", "g")}
    dO = as64(pb["dO"])
    cu = pb["cu_seqlens"].numpy()
    o_ref, _, _ = dense_forward_torch(ins["q"], ins["k"], ins["v"], ins["c"], ins["g"], cu, W, scale)
    (o_ref * dO).sum().backward()
    got = oracle_mod.backward(*(ins[n].detach() for n in ("q", "k", "v", "c", "g")), dO, cu, W, scale)
    for name, val in zip(("q", "k", "v", "c", "g"), got):
        assert max_rel(val, ins[name].grad.numpy()) < 1e-11, name


# ----------------------------------------------------------------------------
# special cases that reduce to a library routine
# ----------------------------------------------------------------------------

def _onehot_c(N, H, h0):
    c = torch.zeros(N, H, dtype=torch.float64)
    c[:, h0] = 1.0
    return c


def test_full_causal_reduces_to_sdpa(oracle_mod):
    """W >= T, one-hot c on head h0, g = 1: head h's output is causal softmax
    attention with head h0's scores applied to head h's values."""
    N, H, d = 40, 3, 8
    pb = random_problem(3, [N], H, d, N)
    q, k, v = (as64(pb[n]) for n in ("q", "k", "v"))
    g = torch.ones(N, H, dtype=torch.float64)
    scale = 1 / math.sqrt(d)
    for h0 in range(H):
        c = _onehot_c(N, H, h0)
        o, _, _ = oracle_mod.forward(q, k, v, c, g, [0, N], N + 5, scale)
        for h in range(H):
            ref = torch.nn.functional.scaled_dot_product_attention(
                q[:, h0][None, None], k[:, h0][None, None], v[:, h][None, None],
                is_causal=True, scale=scale)[0, 0]
            assert max_rel(o[:, h], ref.numpy()) < 1e-12


def test_onehot_window_reduces_to_banded_sdpa(oracle_mod):
    """One-hot c, g = 1: standard per-head sliding-window attention (boolean band mask)."""
    lens = [37, 25]
    N, H, d, W = sum(lens), 4, 8, 9
    pb = random_problem(4, lens, H, d, W)
    q, k, v = (as64(pb[n]) for n in ("q", "k", "v"))
    cu = pb["cu_seqlens"].numpy()
    g = torch.ones(N, H, dtype=torch.float64)
    mask = torch.from_numpy(dense_mask(cu, N, W))
    for h0 in range(H):
        o, _, _ = oracle_mod.forward(q, k, v, _onehot_c(N, H, h0), g, cu, W, pb["scale"])
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[:, h0][None, None], k[:, h0][None, None], v[:, h0][None, None],
            attn_mask=mask[None, None], scale=pb["scale"])[0, 0]
        assert max_rel(o[:, h0], ref.numpy()) < 1e-12


# ----------------------------------------------------------------------------
# closed forms and invariants
# ----------------------------------------------------------------------------

def test_shared_map_rows_sum_to_sum_of_c(oracle_mod):
    """Each p_h row sums to 1, so each row of P sums to sum_h c[t,h]."""
    pb = random_problem(5, [50, 1, 30], 5, 16, 12)
    o, lse, pmap = oracle_mod.forward(pb["q"], pb["k"], pb["v"], pb["c"], pb["g"],
                                      pb["cu_seqlens"], 12, pb["scale"])
    np.testing.assert_allclose(pmap.sum(1), pb["c"].double().numpy().sum(1), rtol=0, atol=1e-13)


def test_locality(oracle_mod):
    """Keys/values outside a query's window or document do not change its output
    (bit-identical); a key inside the window does."""
    lens = [20, 30]
    N, H, d, W = 50, 2, 4, 6
    pb = random_problem(6, lens, H, d, W)
    q, k, v, c, g = (pb[n].double().numpy().copy() for n in ("q", "k", "v", "c", "g"))
    cu = pb["cu_seqlens"].numpy()
    o0, _, _ = oracle_mod.forward(q, k, v, c, g, cu, W, pb["scale"])
    t = 24                      # document [20, 50): window of t=24 is [20, 24]
    k2, v2 = k.copy(), v.copy()
    for j in list(range(0, 20)) + list(range(25, 50)):
        k2[j] += 3.0
        v2[j] -= 2.0
    o1, _, _ = oracle_mod.forward(q, k2, v2, c, g, cu, W, pb["scale"])
    assert np.array_equal(o0[t], o1[t])
    t = 40                      # window [35, 40]
    k3 = k.copy()
    for j in list(range(0, 35)) + list(range(41, 50)):
        k3[j] *= -1.5
    o2, _, _ = oracle_mod.forward(q, k3, v, c, g, cu, W, pb["scale"])
    assert np.array_equal(o0[t], o2[t])
    k4 = k.copy()
    k4[36] += 1.0
    o3, _, _ = oracle_mod.forward(q, k4, v, c, g, cu, W, pb["scale"])
    assert not np.array_equal(o0[t], o3[t])


def test_constant_values(oracle_mod):
    """v_h(j) = v0_h for all j gives o_h(t) = g[t,h] * (sum_h' c[t,h']) * v0_h."""
    lens = [17, 23]
    N, H, d, W = 40, 3, 6, 7
    pb = random_problem(7, lens, H, d, W)
    v0 = np.random.default_rng(0).normal(size=(H, d))
    v = np.broadcast_to(v0, (N, H, d)).copy()
    c = pb["c"].double().numpy()
    g = pb["g"].double().numpy()
    o, _, _ = oracle_mod.forward(pb["q"], pb["k"], v, c, g, pb["cu_seqlens"], W, pb["scale"])
    ref = g[:, :, None] * c.sum(1)[:, None, None] * v0[None]
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-13)


def test_window_one(oracle_mod):
    """W = 1: o_h(t) = g[t,h] * (sum_h' c[t,h']) * v_h(t); the scores do not matter."""
    pb = random_problem(8, [9, 14], 3, 5, 1)
    c = pb["c"].double().numpy()
    g = pb["g"].double().numpy()
    v = pb["v"].double().numpy()
    o, lse, pmap = oracle_mod.forward(pb["q"], pb["k"], v, c, g, pb["cu_seqlens"], 1, pb["scale"])
    np.testing.assert_allclose(o, g[:, :, None] * c.sum(1)[:, None, None] * v, rtol=0, atol=1e-13)
    qk = (pb["q"].double() * pb["k"].double()).sum(-1).numpy() * pb["scale"]
    np.testing.assert_allclose(lse, qk, rtol=0, atol=1e-13)


def test_scale_folding(oracle_mod):
    """(alpha * q, sigma / alpha) gives the same result as (q, sigma)."""
    pb = random_problem(9, [33], 2, 8, 10)
    q = pb["q"].double().numpy()
    args = (pb["k"], pb["v"], pb["c"], pb["g"], pb["cu_seqlens"], 10)
    o1, l1, p1 = oracle_mod.forward(q, *args, 0.25)
    o2, l2, p2 = oracle_mod.forward(q * 0.125, *args, 2.0)
    assert max_rel(o2, o1) < 1e-13 and max_rel(p2, p1) < 1e-13 and max_rel(l2, l1) < 1e-13


def test_gradient_identities(oracle_mod):
    """Homogeneity and shift invariance give closed-form sums of the gradients:
    sum_h g dg = sum_h <dO, o> = sum_h c dc per token; sum_j dk = 0 and
    sum_j dv_h = sum_t (sum_h' c[t,h']) g[t,h] dO_h(t) per document and head."""
    lens = [21, 1, 40]
    N, H, d, W = sum(lens), 3, 5, 9
    pb = random_problem(10, lens, H, d, W)
    q, k, v, c, g, dO = (pb[n].double().numpy() for n in ("q", "k", "v", "c", "g", "dO"))
    cu = pb["cu_seqlens"].numpy()
    o, _, _ = oracle_mod.forward(q, k, v, c, g, cu, W, pb["scale"])
    dq, dk, dv, dc, dg = oracle_mod.backward(q, k, v, c, g, dO, cu, W, pb["scale"])
    lhs = (g * dg).sum(1)
    np.testing.assert_allclose(lhs, (dO * o).sum((1, 2)), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lhs, (c * dc).sum(1), rtol=1e-12, atol=1e-12)
    for a, b in zip(cu[:-1], cu[1:]):
        np.testing.assert_allclose(dk[a:b].sum(0), 0.0, atol=1e-12)
        ref = (c[a:b].sum(1)[:, None, None] * g[a:b, :, None] * dO[a:b]).sum(0)
        np.testing.assert_allclose(dv[a:b].sum(0), ref, rtol=1e-12, atol=1e-12)


def test_finite_differences(oracle_mod):
    """Central differences of L = sum dO * o for every element of q, k, v, c, g."""
    lens = [13, 19]
    H, d, W = 2, 3, 6
    pb = random_problem(13, lens, H, d, W, c_std=1.0)
    base = {n: pb[n].double().numpy().copy() for n in ("q", "k", "v", "c", "g")}
    dO = pb["dO"].double().numpy()
    cu = pb["cu_seqlens"].numpy()
    sc = pb["scale"]
    grads = dict(zip(("q", "k", "v", "c", "g"),
                     oracle_mod.backward(*(base[n] for n in ("q", "k", "v", "c", "g")), dO, cu, W, sc)))

    def loss(x):
        o, _, _ = oracle_mod.forward(x["q"], x["k"], x["v"], x["c"], x["g"], cu, W, sc)
        return float((o * dO).sum())

    eps = 1e-6
    for name in ("q", "k", "v", "c", "g"):
        arr = base[name]
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            x = dict(base)
            a = arr.copy()
            a[idx] += eps
            x[name] = a
            lp = loss(x)
            a[idx] -= 2 * eps
            lm = loss(x)
            fd[idx] = (lp - lm) / (2 * eps)
        assert max_rel(grads[name], fd) < 1e-6, name


# ----------------------------------------------------------------------------
# argument handling and degenerate inputs
# ----------------------------------------------------------------------------

def test_rejects_bad_cu_seqlens(oracle_mod):
    pb = random_problem(1, [8], 1, 2, 3)
    for bad in ([0, 7], [1, 8], [0, 5, 3, 8]):
        with pytest.raises(ValueError):
            oracle_mod.forward(pb["q"], pb["k"], pb["v"], pb["c"], pb["g"], bad, 3, 1.0)


def test_single_token_documents(oracle_mod):
    """Every document of length 1: o_h(t) = g (sum c) v_h(t), gradients of q, k vanish."""
    N, H, d = 10, 2, 4
    pb = random_problem(2, [1] * N, H, d, 5)
    q, k, v, c, g, dO = (pb[n].double().numpy() for n in ("q", "k", "v", "c", "g", "dO"))
    cu = pb["cu_seqlens"].numpy()
    o, _, pmap = oracle_mod.forward(q, k, v, c, g, cu, 5, pb["scale"])
    np.testing.assert_allclose(o, g[:, :, None] * c.sum(1)[:, None, None] * v, atol=1e-13)
    dq, dk, dv, dc, dg = oracle_mod.backward(q, k, v, c, g, dO, cu, 5, pb["scale"])
    assert np.abs(dq).max() < 1e-13 and np.abs(dk).max() < 1e-13
