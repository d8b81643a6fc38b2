"""Pins of the oracle's whole routed layer against independent evaluations.

* Routed == dense: every expert on every token, mixed by the masked gate
  matrix (kieve-moe "Tests": dense <-> parallel MoE equivalence; the Kvasir
  wiki reports sharded == monolithic to max|delta| = 3.6e-12, an exact
  regrouping).  Bar here: 1e-12 relative.
* Special cases that reduce to textbook routines: one expert with k=1 is a
  plain gated FFN; k = E without renormalisation is the full softmax mixture.
"""

import numpy as np
import pytest

from oracle import moe_oracle as O


def _layer(rng, T=64, d=16, E=6, H=8, Hs=0):
    x = rng.standard_normal((T, d))
    w_router = rng.standard_normal((E, d)) / np.sqrt(d)
    w13 = rng.standard_normal((E, 2 * H, d)) / np.sqrt(d)
    w2 = rng.standard_normal((E, d, H)) / np.sqrt(H)
    sh = (None, None)
    if Hs:
        sh = (rng.standard_normal((1, 2 * Hs, d)) / np.sqrt(d), rng.standard_normal((1, d, Hs)) / np.sqrt(Hs))
    return x, w_router, w13, w2, sh


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("k,cap,Hs,act,renorm", [(2, 0, 0, O.ACT_SWIGLU, True), (2, 10, 0, O.ACT_SWIGLU, True),
                                                 (3, 0, 5, O.ACT_GEGLU, False), (3, 12, 5, O.ACT_SWIGLU, True),
                                                 (1, 4, 0, O.ACT_GEGLU, True)])
def test_routed_equals_dense(k, cap, Hs, act, renorm):
    rng = np.random.default_rng(k * 100 + cap)
    x, w_router, w13, w2, (w13s, w2s) = _layer(rng, Hs=Hs)
    bias = -1.2 * np.log(np.arange(6) + 1.0)
    r = O.moe_forward(x, w_router, bias, w13, w2, k=k, act=act, renorm=renorm, cap=cap,
                      w13_sh=w13s, w2_sh=w2s)
    if cap:
        assert r["drop"].sum() > 0           # the case really drops
    dense = O.dense_moe_forward(x, w13, w2, r["idx"], r["w"], r["drop"], act=act, w13_sh=w13s, w2_sh=w2s)
    assert _rel(r["out"], dense) < 1e-12


def test_single_expert_is_a_plain_gated_ffn():
    rng = np.random.default_rng(3)
    x, w_router, w13, w2, _ = _layer(rng, E=1)
    r = O.moe_forward(x, w_router, None, w13, w2, k=1, renorm=True)
    assert (r["w"] == 1.0).all()
    np.testing.assert_allclose(r["out"], O.expert_ffn(x, w13[0], w2[0], O.ACT_SWIGLU), rtol=1e-13)
    # the shared expert adds at weight one
    r2 = O.moe_forward(x, w_router, None, w13, w2, k=1, renorm=True, w13_sh=w13[:1], w2_sh=w2[:1])
    np.testing.assert_allclose(r2["out"], 2 * r["out"], rtol=1e-13)


def test_all_experts_without_renorm_is_the_softmax_mixture():
    rng = np.random.default_rng(4)
    E = 5
    x, w_router, w13, w2, _ = _layer(rng, E=E)
    r = O.moe_forward(x, w_router, None, w13, w2, k=E, renorm=False)
    p = O.softmax(x @ w_router.T)
    mix = sum(p[:, e:e + 1] * O.expert_ffn(x, w13[e], w2[e], O.ACT_SWIGLU) for e in range(E))
    assert _rel(r["out"], mix) < 1e-13


def test_fully_dropped_token_gets_only_the_shared_expert():
    rng = np.random.default_rng(5)
    x, w_router, w13, w2, (w13s, w2s) = _layer(rng, T=40, E=4, Hs=3)
    r = O.moe_forward(x, w_router, None, w13, w2, k=2, cap=3, w13_sh=w13s, w2_sh=w2s)
    gone = np.nonzero(r["drop"].sum(1) == 2)[0]
    assert gone.size > 0
    np.testing.assert_allclose(r["out"][gone], r["y_shared"][gone], rtol=0, atol=0)
