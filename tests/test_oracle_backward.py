"""Pins of the oracle's gradients: central finite differences of the oracle forward itself.

L(x) = sum(dout * out(x)) + aux_coef * aux(x).  The routing decision is constant near the seeded inputs (no
near-ties), so L is smooth there and its central difference with step 1e-6 agrees with the analytic gradient to
about 1e-8.  A dropped term (the gates' own derivative, the softmax through the router, the renormalisation,
the statistic, the shared expert) or a wrong sign in any of them moves dx by far more.  The weight gradients
(every routed expert's W13 and W2, the shared expert's, W_r) are pinned the same way, entry by entry.
"""

import numpy as np
import pytest

import oracle as O


def _problem(T, d, E, k, H, H_s, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    w_r = rng.standard_normal((E, d)) * 0.5
    bias = rng.standard_normal(E) * 0.2
    w13 = rng.standard_normal((E, 2 * H, d)) * d ** -0.5
    w2 = rng.standard_normal((E, d, H)) * H ** -0.5
    w13_sh = rng.standard_normal((1, 2 * H_s, d)) * d ** -0.5 if H_s else None
    w2_sh = rng.standard_normal((1, d, H_s)) * H_s ** -0.5 if H_s else None
    dout = rng.standard_normal((T, d))
    return x, w_r, bias, w13, w2, w13_sh, w2_sh, dout


def _loss(x, w_r, bias, w13, w2, w13_sh, w2_sh, dout, k, act, renorm, cap, aux_coef):
    fw = O.moe_forward(x, w_r, bias, w13, w2, k=k, act=act, renorm=renorm, cap=cap, w13_sh=w13_sh, w2_sh=w2_sh)
    return float(np.sum(dout * fw["out"])) + aux_coef * fw["aux"]


def _fd(f, x, h=1e-6):
    g = np.zeros_like(x)
    for i in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[i] += h
        xm[i] -= h
        g[i] = (f(xp) - f(xm)) / (2 * h)
    return g


@pytest.mark.parametrize("act,renorm,cap,H_s,aux_coef", [(O.ACT_SWIGLU, True, 0, 0, 0.0),
                                                         (O.ACT_GEGLU, False, 0, 4, 0.0),
                                                         (O.ACT_SWIGLU, True, 0, 4, 0.3),
                                                         (O.ACT_SWIGLU, False, 2, 0, 0.1),
                                                         (O.ACT_GEGLU, True, 2, 4, 0.05)])
def test_backward_matches_finite_differences(act, renorm, cap, H_s, aux_coef):
    T, d, E, k, H = 6, 5, 4, 2, 3
    x, w_r, bias, w13, w2, w13_sh, w2_sh, dout = _problem(T, d, E, k, H, H_s, seed=3)
    r = O.route(x, w_r, bias, k, renorm)
    assert O.topk_margin(r["z"], k).min() > 1e-3          # the routing is constant under the differences
    if cap:
        assert O.permute(r["idx"], E, cap)["drop"].any()    # the capacity drops something
    got = O.moe_backward(x, w_r, bias, w13, w2, dout, k=k, act=act, renorm=renorm, cap=cap, w13_sh=w13_sh,
                           w2_sh=w2_sh, aux_coef=aux_coef)["dx"]
    fd = _fd(lambda xx: _loss(xx, w_r, bias, w13, w2, w13_sh, w2_sh, dout, k, act, renorm, cap, aux_coef), x)
    np.testing.assert_allclose(got, fd, rtol=1e-6, atol=1e-7)


def test_activation_derivatives_match_finite_differences():
    z = np.linspace(-6.0, 6.0, 101)
    h = 1e-6
    np.testing.assert_allclose(O.silu_grad(z), (O.silu(z + h) - O.silu(z - h)) / (2 * h), rtol=1e-7, atol=1e-9)
    np.testing.assert_allclose(O.gelu_erf_grad(z), (O.gelu_erf(z + h) - O.gelu_erf(z - h)) / (2 * h), rtol=1e-7,
                               atol=1e-9)
    # closed values: silu'(0) = 1/2, GELU'(0) = 1/2
    assert O.silu_grad(0.0) == 0.5 and O.gelu_erf_grad(0.0) == 0.5


def test_single_expert_layer_reduces_to_the_expert_gradient():
    # E = k = 1: every gate is 1 and the softmax has one entry, so the router passes no gradient and dx is the
    # expert's own input gradient
    x, w_r, bias, w13, w2, _, _, dout = _problem(4, 5, 1, 1, 3, 0, seed=9)
    got = O.moe_backward(x, w_r, bias, w13, w2, dout, k=1)["dx"]
    np.testing.assert_allclose(got, O.expert_ffn_backward_x(x, w13[0], w2[0], O.ACT_SWIGLU, dout), rtol=1e-12)


@pytest.mark.parametrize("act,renorm,cap,H_s,aux_coef", [(O.ACT_SWIGLU, True, 0, 4, 0.3),
                                                         (O.ACT_GEGLU, False, 2, 4, 0.05),
                                                         (O.ACT_SWIGLU, False, 2, 0, 0.0)])
def test_weight_gradients_match_finite_differences(act, renorm, cap, H_s, aux_coef):
    T, d, E, k, H = 6, 5, 4, 2, 3
    x, w_r, bias, w13, w2, w13_sh, w2_sh, dout = _problem(T, d, E, k, H, H_s, seed=5)
    r = O.route(x, w_r, bias, k, renorm)
    assert O.topk_margin(r["z"], k).min() > 1e-3
    g = O.moe_backward(x, w_r, bias, w13, w2, dout, k=k, act=act, renorm=renorm, cap=cap, w13_sh=w13_sh,
                       w2_sh=w2_sh, aux_coef=aux_coef)
    L = lambda **kw: _loss(kw.get("x", x), kw.get("w_r", w_r), bias, kw.get("w13", w13), kw.get("w2", w2),
                           kw.get("w13_sh", w13_sh), kw.get("w2_sh", w2_sh), dout, k, act, renorm, cap, aux_coef)
    checks = [("dw13", w13, "w13"), ("dw2", w2, "w2"), ("dw_router", w_r, "w_r")]
    if H_s:
        checks += [("dw13_sh", w13_sh, "w13_sh"), ("dw2_sh", w2_sh, "w2_sh")]
    for key, w0, name in checks:
        fd = _fd(lambda ww: L(**{name: ww}), w0)
        np.testing.assert_allclose(g[key], fd, rtol=1e-6, atol=1e-7, err_msg=key)
    if cap:   # an expert's dropped rows add nothing: every expert still gets a gradient from its kept rows
        assert O.permute(r["idx"], E, cap)["drop"].any()
    assert g["dw13_sh"] is None if not H_s else g["dw13_sh"].shape == (1, 2 * H_s, d)


def test_expert_weight_gradients_single_row_closed_form():
    # one row, H = 1: y = act(g) u w2 with g = <w1, x>, u = <w3, x>; dW2 = dy act(g) u, dW1 = <dy, w2> u act'(g) x,
    # dW3 = <dy, w2> act(g) x
    x = np.array([[0.3, -1.2, 0.7]])
    w13 = np.array([[0.5, 0.1, -0.4], [-0.2, 0.9, 0.3]])
    w2 = np.array([[1.5], [-0.5], [0.25]])
    dy = np.array([[0.4, -1.0, 2.0]])
    g, u = float(w13[0] @ x[0]), float(w13[1] @ x[0])
    s = 1.0 / (1.0 + np.exp(-g))
    a, da = g * s, s * (1.0 + g * (1.0 - s))
    c = float(dy[0] @ w2[:, 0])
    dw13, dw2 = O.expert_ffn_backward_weights(x, w13, w2, O.ACT_SWIGLU, dy)
    np.testing.assert_allclose(dw2[:, 0], dy[0] * a * u, rtol=1e-14)
    np.testing.assert_allclose(dw13[0], c * u * da * x[0], rtol=1e-14)
    np.testing.assert_allclose(dw13[1], c * a * x[0], rtol=1e-14)
