"""Pins of the oracle's router: softmax, top-k order and tie-break, gates, load-balance statistic.

Each check compares the oracle with something other than itself: a closed
form, a brute-force sort, or an invariant the MoE-Stream ``MoEFFN.forward``
definition fixes (softmax -> top-k -> renormalise; batch-local load balance).
"""

import math

import numpy as np
import pytest

from oracle import moe_oracle as O


def test_topk_equal_logits_take_lowest_indices():
    z = np.full((5, 7), 0.25)
    for k in range(1, 8):
        assert (O.topk_select(z, k) == np.arange(k)[None, :]).all()


def test_topk_signed_zero_ties_go_to_lower_index():
    z = np.array([[-0.0, 0.0, -1.0], [0.0, -0.0, -1.0], [-1.0, -0.0, 0.0]])
    assert O.topk_select(z, 1)[:, 0].tolist() == [0, 0, 1]
    assert O.topk_select(z, 2).tolist() == [[0, 1], [0, 1], [1, 2]]


@pytest.mark.parametrize("seed", range(5))
def test_topk_matches_brute_force_sort(seed):
    rng = np.random.default_rng(seed)
    z = rng.integers(-3, 3, size=(8, 6)) * 0.5          # many ties
    for k in range(1, 7):
        got = O.topk_select(z, k)
        for t in range(8):
            want = sorted(range(6), key=lambda e: (-z[t, e], e))[:k]
            assert got[t].tolist() == want


def test_topk_of_logits_equals_topk_of_probabilities_when_distinct():
    # moe_stream.py runs torch.topk on softmax probabilities; softmax is monotone.
    rng = np.random.default_rng(1)
    z = rng.standard_normal((50, 16))
    p = O.softmax(z)
    assert (O.topk_select(z, 4) == np.argsort(-p, axis=1)[:, :4]).all()


def test_softmax_closed_form():
    z = np.array([[0.0, math.log(2.0), math.log(3.0)]])
    np.testing.assert_allclose(O.softmax(z), [[1 / 6, 2 / 6, 3 / 6]], rtol=1e-15)
    # shift invariance of the definition
    np.testing.assert_allclose(O.softmax(z + 100.0), [[1 / 6, 2 / 6, 3 / 6]], rtol=1e-14)


def test_worked_routing_example():
    # token 0: z = (0, ln2, ln3) -> p = (1,2,3)/6 -> top-2 = (2, 1), w = (1/2, 1/3) -> renorm (3/5, 2/5)
    # token 1: z = (ln4, 0, 0)   -> p = (4,1,1)/6 -> top-2 = (0, 1) (tie 1 vs 2 -> 1), w -> (4/5, 1/5)
    z = np.array([[0.0, math.log(2.0), math.log(3.0)], [math.log(4.0), 0.0, 0.0]])
    r = O.route_from_logits(z, 2, renorm=True)
    assert r["idx"].tolist() == [[2, 1], [0, 1]]
    np.testing.assert_allclose(r["w"], [[0.6, 0.4], [0.8, 0.2]], rtol=1e-15)
    r0 = O.route_from_logits(z, 2, renorm=False)
    np.testing.assert_allclose(r0["w"], [[0.5, 1 / 3], [4 / 6, 1 / 6]], rtol=1e-15)
    assert r["counts"].tolist() == [1, 2, 1]
    # f = counts/T, P = mean p, aux = E * sum f P
    f = np.array([0.5, 1.0, 0.5])
    P = np.array([(1 / 6 + 4 / 6) / 2, (2 / 6 + 1 / 6) / 2, (3 / 6 + 1 / 6) / 2])
    np.testing.assert_allclose(r["f"], f, rtol=1e-15)
    np.testing.assert_allclose(r["P"], P, rtol=1e-15)
    assert abs(r["aux"] - 3 * float(f @ P)) < 1e-15


def test_router_logits_orientation_and_bias():
    # W_r is [E, d] (a bias-free Linear(d, E)); z[t,e] = x[t] . W_r[e] + bias[e]
    x = np.array([[1.0, 2.0]])
    W = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    bias = np.array([0.5, -0.5, 0.0])
    assert O.router_logits(x, W, bias).tolist() == [[1.5, 1.5, 3.0]]


def test_renormalised_gates_sum_to_one_and_invariants():
    rng = np.random.default_rng(2)
    T, E, k = 300, 12, 3
    z = rng.standard_normal((T, E))
    r = O.route_from_logits(z, k, renorm=True)
    np.testing.assert_allclose(r["w"].sum(1), 1.0, rtol=1e-14)
    assert (np.diff(r["w"], axis=1) <= 0).all()           # larger first
    assert r["counts"].sum() == T * k
    np.testing.assert_allclose(r["f"].sum(), k, rtol=1e-14)
    np.testing.assert_allclose(r["P"].sum(), 1.0, rtol=1e-14)
    for t in range(T):
        assert len(set(r["idx"][t].tolist())) == k


def test_balanced_routing_gives_aux_equal_to_k():
    # Uniform softmax and every expert chosen by the same number of tokens:
    # f_e = k/E, P_e = 1/E, so aux = E * E * (k/E) * (1/E) = k.
    E, k = 6, 2
    T = 3 * E
    z = np.zeros((T, E))
    # nudge so that token t picks experts (t mod E, t+1 mod E) while softmax stays ~uniform
    for t in range(T):
        z[t, t % E] = 1e-9
        z[t, (t + 1) % E] = 5e-10
    r = O.route_from_logits(z, k, renorm=True)
    np.testing.assert_allclose(r["f"], k / E, rtol=0)
    np.testing.assert_allclose(r["aux"], k, rtol=1e-8)


def test_topk_margin():
    z = np.array([[3.0, 1.0, 2.0, 2.0]])
    assert O.topk_margin(z, 1)[0] == 1.0
    assert O.topk_margin(z, 2)[0] == 0.0
    assert O.topk_margin(z, 3)[0] == 1.0
    assert O.topk_margin(z, 4)[0] == np.inf
