"""Pins of the fp64 oracle for the producer of c and g (oracle/cg_oracle.c).

The form is an assumption (the pages give none; see the oracle's header): per-token
affine maps c = x Wc + bc, g = x Wg + bg.  None of these checks re-types that formula:
the forward is pinned by what it must give on basis vectors and by affinity, the
backward by central finite differences of the pinned forward and by closed forms.
"""
import numpy as np
import pytest

import oracle
from cross_head_dynamic_b200.inputs import cg_problem


@pytest.fixture(scope="module", autouse=True)
def _build():
    oracle.build()


def test_basis_vectors_give_weight_rows_plus_bias():
    """x = identity: token k selects row k of w.  A transposed w, a dropped bias or c and g
    swapped all fail here."""
    D, H = 7, 3
    p = cg_problem(1, 4, D, H, "f32")
    w, b = p["w"].double().numpy(), p["b"].double().numpy()
    c, g = oracle.cg_forward(np.eye(D), w, b)
    np.testing.assert_allclose(c, w[:, :H] + b[:H], rtol=0, atol=1e-15)
    np.testing.assert_allclose(g, w[:, H:] + b[H:], rtol=0, atol=1e-15)


def test_zero_input_gives_the_bias():
    p = cg_problem(2, 3, 10, 4, "f32")
    c, g = oracle.cg_forward(np.zeros((3, 10)), p["w"], p["b"])
    b = p["b"].double().numpy()
    assert np.array_equal(c, np.tile(b[:4], (3, 1))) and np.array_equal(g, np.tile(b[4:], (3, 1)))


def test_affine_in_x():
    """f(a x1 + (1 - a) x2) = a f(x1) + (1 - a) f(x2): catches any nonlinearity."""
    p = cg_problem(3, 6, 12, 2, "f32")
    q = cg_problem(4, 6, 12, 2, "f32")
    x1, x2 = p["x"].double().numpy(), q["x"].double().numpy()
    a = 0.3
    c, g = oracle.cg_forward(a * x1 + (1 - a) * x2, p["w"], p["b"])
    c1, g1 = oracle.cg_forward(x1, p["w"], p["b"])
    c2, g2 = oracle.cg_forward(x2, p["w"], p["b"])
    np.testing.assert_allclose(c, a * c1 + (1 - a) * c2, atol=1e-13)
    np.testing.assert_allclose(g, a * g1 + (1 - a) * g2, atol=1e-13)


def _loss(x, w, b, dc, dg):
    c, g = oracle.cg_forward(x, w, b)
    return float((c * dc).sum() + (g * dg).sum())


def test_backward_matches_central_differences():
    """Every element of dx, dw and db against central differences of the (pinned) forward
    for L = <dc, c> + <dg, g>.  The maps are affine, so the differences are exact up to
    rounding."""
    N, D, H = 5, 6, 2
    p = cg_problem(5, N, D, H, "f32")
    x, w, b = (p[n].double().numpy() for n in ("x", "w", "b"))
    dc, dg = p["dc"].double().numpy(), p["dg"].double().numpy()
    dx, dw, db = oracle.cg_backward(x, w, dc, dg)
    eps = 1e-4
    for arr, grad in ((x, dx), (w, dw), (b, db)):
        fd = np.empty_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + eps
            lp = _loss(x, w, b, dc, dg)
            arr[idx] = old - eps
            lm = _loss(x, w, b, dc, dg)
            arr[idx] = old
            fd[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, fd, rtol=1e-8, atol=1e-9)


def test_backward_closed_forms():
    """db holds the column sums of (dc | dg); with x = identity, dw row k is token k's
    (dc | dg); zero upstream gradients give zero everywhere."""
    D, H = 5, 3
    p = cg_problem(6, D, D, H, "f32")
    w = p["w"].double().numpy()
    dc, dg = p["dc"].double().numpy(), p["dg"].double().numpy()
    dx, dw, db = oracle.cg_backward(np.eye(D), w, dc, dg)
    np.testing.assert_allclose(db, np.concatenate([dc.sum(0), dg.sum(0)]), atol=1e-14)
    np.testing.assert_allclose(dw, np.concatenate([dc, dg], axis=1), atol=1e-15)
    z = np.zeros_like(dc)
    dx0, dw0, db0 = oracle.cg_backward(p["x"], w, z, z)
    assert not dx0.any() and not dw0.any() and not db0.any()
