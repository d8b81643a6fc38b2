"""Pins of the oracle's hierarchical ("fractal") router, ``route_tree``.

Reading (kieve-moe Features, "Fractal tiling routing"): expert e is the leaf reached by its base-branch digits,
most significant first; level l has its own router W_l shared by the nodes of the level, and the leaf
probability is the product of the level softmaxes along the path.  Pinned by: a hand-worked two-level tree,
an explicit loop over the digits (a least-significant-first digit order or swapped level routers fail it),
the one-level tree equal to the flat router, the factorisation (rows sum to one; the top-1 leaf is the
per-level argmax), and the exactness of the beam search a kernel can use for the top-k.
"""

import math

import numpy as np
import pytest

import oracle as O


def test_two_level_hand_example():
    # branch 2, levels 2, d = 1, x = 1: q0 = softmax(ln 3, 0) = (3/4, 1/4), q1 = softmax(0, ln 2) = (1/3, 2/3)
    x = np.array([[1.0]])
    w = np.array([[math.log(3.0)], [0.0], [0.0], [math.log(2.0)]])
    r = O.route_tree(x, w, None, 2, 2, 2, renorm=False)
    np.testing.assert_allclose(r["p"][0], [1 / 4, 1 / 2, 1 / 12, 1 / 6], rtol=1e-14)
    assert r["idx"][0].tolist() == [1, 0]
    np.testing.assert_allclose(r["w"][0], [1 / 2, 1 / 4], rtol=1e-14)
    rn = O.route_tree(x, w, None, 2, 2, 2, renorm=True)
    np.testing.assert_allclose(rn["w"][0], [2 / 3, 1 / 3], rtol=1e-14)
    # a bias (ln 2, 0) on level 1 evens its split: logits (ln 2, ln 2), q1 = (1/2, 1/2)
    rb = O.route_tree(x, w, np.array([0.0, 0.0, math.log(2.0), 0.0]), 2, 2, 1, renorm=False)
    np.testing.assert_allclose(rb["p"][0], [3 / 8, 3 / 8, 1 / 8, 1 / 8], rtol=1e-14)
    assert rb["idx"][0].tolist() == [0]   # equal leaves 0 and 1: the lower index


def test_leaf_probability_matches_an_explicit_digit_loop():
    rng = np.random.default_rng(4)
    T, d, B, L = 5, 6, 3, 3
    x = rng.standard_normal((T, d))
    w = rng.standard_normal((L * B, d))
    bias = rng.standard_normal(L * B) * 0.3
    r = O.route_tree(x, w, bias, B, L, 4, renorm=True)
    for t in range(T):
        for a in range(B):
            for b in range(B):
                for c in range(B):
                    q = []
                    for l, dig in enumerate((a, b, c)):
                        z = x[t] @ w[l * B:(l + 1) * B].T + bias[l * B:(l + 1) * B]
                        ez = np.exp(z - z.max())
                        q.append(ez[dig] / ez.sum())
                    assert abs(r["p"][t, a * B * B + b * B + c] - q[0] * q[1] * q[2]) < 1e-15
    np.testing.assert_allclose(r["p"].sum(axis=1), 1.0, rtol=1e-14)


def test_one_level_tree_is_the_flat_router():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((16, 8))
    w = rng.standard_normal((12, 8))
    bias = rng.standard_normal(12) * 0.2
    t = O.route_tree(x, w, bias, 12, 1, 3, renorm=True)
    f = O.route(x, w, bias, 3, True)
    assert (t["idx"] == f["idx"]).all()
    np.testing.assert_allclose(t["w"], f["w"], rtol=1e-13)
    np.testing.assert_allclose(t["p"], f["p"], rtol=1e-13)
    np.testing.assert_allclose(t["aux"], f["aux"], rtol=1e-13)


def test_top1_leaf_is_the_per_level_argmax():
    rng = np.random.default_rng(6)
    B, L = 4, 3
    x = rng.standard_normal((64, 10))
    w = rng.standard_normal((L * B, 10))
    r = O.route_tree(x, w, None, B, L, 1, renorm=False)
    digits = np.stack([np.argmax(r["z"][:, l * B:(l + 1) * B], axis=1) for l in range(L)], axis=1)
    assert (r["idx"][:, 0] == digits @ (B ** np.arange(L - 1, -1, -1))).all()
    assert (O.tree_digits(r["idx"][:, 0], B, L) == digits).all()


def _beam_topk(q, k):
    """k-best paths level by level, keeping (value desc, index asc) after each level."""
    L, B = q.shape
    beam = [(1.0, 0)]
    for l in range(L):
        cand = [(v * q[l, c], i * B + c) for v, i in beam for c in range(B)]
        cand.sort(key=lambda vi: (-vi[0], vi[1]))
        beam = cand[:k]
    return [i for _, i in beam]


@pytest.mark.parametrize("B,L,k", [(2, 4, 3), (4, 3, 8), (8, 2, 5), (3, 3, 27)])
def test_beam_search_reaches_the_global_topk(B, L, k):
    # the product of per-level probabilities is monotone in each factor, so pruning every level to the k
    # best partial paths keeps the k best leaves
    rng = np.random.default_rng(7)
    x = rng.standard_normal((40, 6))
    w = rng.standard_normal((L * B, 6)) * 1.5
    r = O.route_tree(x, w, None, B, L, k, renorm=False)
    for t in range(x.shape[0]):
        assert _beam_topk(r["q"][t], k) == r["idx"][t].tolist()
