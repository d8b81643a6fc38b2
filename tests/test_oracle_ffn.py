"""Pins of the oracle's expert FFN and of the whole layer on a hand-worked example.

Activations are pinned to tabulated values (``tests/golden``); the gated FFN
orientation (gate vs up half of w13, [out, in] layouts) to structured weights
with closed-form outputs; the whole layer (route -> group -> FFN -> combine ->
shared expert, with and without capacity) to a two-token example worked out
by hand from the definitions in moe_stream.py ``MoEFFN.forward`` and the Kvasir
"Backbone x worker" step ``combine(p, partials) + shared(cur)``.
"""

import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
L3 = math.log(3.0)


def _table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                a, b = line.split()
                rows.append((float(a), float(b)))
    return rows


def test_silu_matches_logistic_table():
    for z, sig in _table("logistic.txt"):
        assert abs(O.silu(np.array([z]))[0] - z * sig) <= 1e-15 * max(1.0, abs(z))


def test_gelu_is_exact_erf_form():
    for z, phi in _table("normal_cdf.txt"):
        assert abs(O.gelu_erf(np.array([z]))[0] - z * phi) < 1e-10 * max(1.0, z)
        assert abs(O.gelu_erf(np.array([-z]))[0] - (-z) * (1.0 - phi)) < 1e-10 * max(1.0, z)
    # the tanh approximation differs from the erf form by ~1.5e-4 at z = 1
    tanh_form = 0.5 * (1 + math.tanh(math.sqrt(2 / math.pi) * (1 + 0.044715)))
    assert abs(O.gelu_erf(np.array([1.0]))[0] - tanh_form) > 1e-4


def test_glu_orientation_closed_form():
    # W1 = I (gate), W3 = 2I (up), W2 = P (y_o = sum_i P[o,i] h_i), x = (ln3, 0, -ln3):
    # h = silu(x) * 2x = (1.5 L^2, 0, 0.5 L^2), y = P h = (h1, h2, h0).
    x = np.array([[L3, 0.0, -L3]])
    w13 = np.concatenate([np.eye(3), 2 * np.eye(3)])
    P = np.array([[0, 1, 0], [0, 0, 1], [1, 0, 0]], float)
    h = O.glu_hidden(x, w13, O.ACT_SWIGLU)
    np.testing.assert_allclose(h, [[1.5 * L3 ** 2, 0.0, 0.5 * L3 ** 2]], rtol=1e-15, atol=1e-300)
    y = O.expert_ffn(x, w13, P, O.ACT_SWIGLU)
    np.testing.assert_allclose(y, [[0.0, 0.5 * L3 ** 2, 1.5 * L3 ** 2]], rtol=1e-15, atol=1e-300)


def _worked_layer(act):
    """T=2, d=2, E=3, k=2, H=1; see the module docstring and the comments below."""
    x = np.array([[1.0, 0.0], [0.0, 1.0]])
    w_router = np.array([[0.0, math.log(4.0)], [math.log(2.0), 0.0], [L3, 0.0]])
    g = L3 if act == O.ACT_SWIGLU else 1.0
    w13 = np.array([[[g, g], [e + 1.0, 2.0 * (e + 1.0)]] for e in range(3)])     # [E, 2H, d]
    w2 = np.array([[[1.0], [-(e + 1.0)]] for e in range(3)])                     # [E, d, H]
    w13_sh = np.array([[[g, g], [1.0, 1.0]]])
    w2_sh = np.array([[[1.0], [1.0]]])
    return x, w_router, w13, w2, w13_sh, w2_sh


@pytest.mark.parametrize("act", [O.ACT_SWIGLU, O.ACT_GEGLU])
def test_worked_layer_example(act):
    # gate activation a = silu(ln3) = 0.75 ln3 (SwiGLU) or gelu(1) = Phi(1) (GeGLU), same for all rows.
    # expert e: h(x0) = a (e+1), h(x1) = 2 a (e+1), y = h (1, -(e+1)).
    # token 0 -> experts (2, 1), gates (0.6, 0.4); token 1 -> experts (0, 1), gates (0.8, 0.2).
    a = 0.75 * L3 if act == O.ACT_SWIGLU else dict(_table("normal_cdf.txt"))[1.0]
    x, w_router, w13, w2, w13_sh, w2_sh = _worked_layer(act)
    r = O.moe_forward(x, w_router, None, w13, w2, k=2, act=act, renorm=True)
    want = np.array([a * np.array([2.6, -7.0]), 2 * a * np.array([1.2, -1.6])])
    tol = 1e-14 if act == O.ACT_SWIGLU else 1e-10
    np.testing.assert_allclose(r["out"], want, rtol=tol)
    # shared expert at weight one: y_s = a (1, 1) for both tokens
    r = O.moe_forward(x, w_router, None, w13, w2, k=2, act=act, renorm=True, w13_sh=w13_sh, w2_sh=w2_sh)
    np.testing.assert_allclose(r["out"], want + a, rtol=tol)
    # capacity 1: token 1's slot on expert 1 (rank 1) is dropped; its other gate is not renormalised
    r = O.moe_forward(x, w_router, None, w13, w2, k=2, act=act, renorm=True, cap=1)
    assert r["drop"].tolist() == [[0, 0], [0, 1]]
    np.testing.assert_allclose(r["out"], [want[0], 2 * a * np.array([0.8, -0.8])], rtol=tol)


def test_grouped_ffn_leaves_padding_rows_zero():
    rng = np.random.default_rng(0)
    x_perm = rng.standard_normal((10, 4))
    w13 = rng.standard_normal((2, 6, 4))
    w2 = rng.standard_normal((2, 4, 3))
    y = O.grouped_ffn(x_perm, np.array([0, 5, 10]), np.array([2, 3]), w13, w2, O.ACT_SWIGLU)
    assert (y[2:5] == 0).all() and (y[8:] == 0).all()
    np.testing.assert_allclose(y[5:8], O.expert_ffn(x_perm[5:8], w13[1], w2[1], O.ACT_SWIGLU))
