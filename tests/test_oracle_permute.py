"""Pins of the oracle's grouping step: brute force, invariants, capacity drops.

The grouping keeps each (token, top-k slot) identity (ExpertMesh README,
"Activation grouping that preserves token and top-k slot identity"); with a
capacity factor (MoEEvolve README, static-shape capacity dispatch) overflow is
dropped in token order.
"""

import numpy as np
import pytest

from oracle import moe_oracle as O


def _random_idx(rng, T, E, k, skew=0.0):
    wts = (np.arange(E) + 1.0) ** (-skew)
    wts /= wts.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=wts) for _ in range(T)]).astype(np.int32)


def _brute_force(idx, E, cap):
    """Explicit loops: rank by scanning earlier tokens, rows laid out group by group."""
    T, k = len(idx), len(idx[0])
    counts = [0] * E
    for t in range(T):
        for j in range(k):
            counts[idx[t][j]] += 1
    kept = [min(c, cap) if cap else c for c in counts]
    if cap:
        offsets = [e * cap for e in range(E + 1)]
    else:
        offsets = [0]
        for e in range(E):
            offsets.append(offsets[-1] + counts[e])
    slot = [[-1] * k for _ in range(T)]
    for t in range(T):
        for j in range(k):
            e = idx[t][j]
            rank = sum(1 for t2 in range(t) for j2 in range(k) if idx[t2][j2] == e)
            if not cap or rank < cap:
                slot[t][j] = offsets[e] + rank
    return counts, kept, offsets, slot


@pytest.mark.parametrize("seed,T,E,k,cap", [(0, 8, 4, 2, 0), (1, 8, 6, 3, 0), (2, 10, 4, 2, 3),
                                            (3, 12, 5, 1, 2), (4, 9, 3, 3, 4), (5, 7, 6, 6, 1)])
def test_permute_matches_brute_force(seed, T, E, k, cap):
    rng = np.random.default_rng(seed)
    idx = _random_idx(rng, T, E, k, skew=1.0)
    g = O.permute(idx, E, cap)
    counts, kept, offsets, slot = _brute_force(idx.tolist(), E, cap)
    assert g["counts"].tolist() == counts
    assert g["kept"].tolist() == kept
    assert g["offsets"].tolist() == offsets
    assert g["slot_pos"].tolist() == slot
    assert g["drop"].tolist() == [[int(s < 0) for s in row] for row in slot]


@pytest.mark.parametrize("cap", [0, 20, 60])
def test_permute_invariants(cap):
    rng = np.random.default_rng(7)
    T, E, k = 500, 16, 4
    idx = _random_idx(rng, T, E, k, skew=1.2)
    g = O.permute(idx, E, cap)
    slot, drop, row_src = g["slot_pos"], g["drop"], g["row_src"]
    assert g["counts"].sum() == T * k
    assert g["kept"].sum() == T * k - drop.sum()
    if cap:
        assert (g["kept"] <= cap).all()
        assert (drop == (g["rank"] >= cap)).all()      # drops exactly where rank >= C
    else:
        assert drop.sum() == 0
    # bijection of kept (t,j) onto the rows [offsets_e, offsets_e + kept_e)
    kept_rows = slot[slot >= 0]
    assert len(set(kept_rows.tolist())) == kept_rows.size
    for e in range(E):
        rows = sorted(slot[(idx == e) & (slot >= 0)].tolist())
        a = int(g["offsets"][e])
        assert rows == list(range(a, a + int(g["kept"][e])))
        # token order inside a group
        src = row_src[a:a + int(g["kept"][e])]
        assert (np.diff(src // k) > 0).all()
    # row_src is the inverse of slot_pos
    for t in range(T):
        for j in range(k):
            if slot[t, j] >= 0:
                assert row_src[slot[t, j]] == t * k + j
    assert (row_src >= 0).sum() == kept_rows.size


def test_capacity_hand_example():
    # five tokens, all on expert 0, capacity 2: tokens 0 and 1 kept, later ones dropped
    idx = np.zeros((5, 1), np.int32)
    g = O.permute(idx, 2, 2)
    assert g["slot_pos"][:, 0].tolist() == [0, 1, -1, -1, -1]
    assert g["offsets"].tolist() == [0, 2, 4]
    assert g["row_src"].tolist() == [0, 1, -1, -1]
    assert g["kept"].tolist() == [2, 0]
    assert g["counts"].tolist() == [5, 0]


def test_capacity_formula():
    # C = ceil(cf * T * k / E): 1.25 * 32768 * 4 / 192 = 853.33 -> 854
    assert O.capacity(32768, 4, 192, 1.25) == 854
    assert O.capacity(256, 2, 8, 0.5) == 32
    assert O.capacity(256, 2, 8, 1.0) == 64
    assert O.capacity(256, 2, 8, 0.0) == 0


def test_gather_rows():
    x = np.arange(6.0).reshape(3, 2)
    row_src = np.array([4, -1, 1])          # k = 2: rows from tokens 2, none, 0
    np.testing.assert_array_equal(O.gather_rows(x, row_src, 2), [[4, 5], [0, 0], [0, 1]])
