"""Hierarchical ("fractal") router on the GPU against the float64 oracle's ``route_tree``.

The oracle decides on float64 level logits, the library on the tensor-core screen's fp32 ones (a two-term bf16
split of W_tree, within gamma |x_t| |w_r| of the exact logits).  A token whose top k+1 leaf probabilities are
all at least TREE_BAND apart (relative) must get the same experts in the same order; every other token must pick
leaves no further than the band below the oracle's k-th.  Gates: 1e-3 relative (the logit error moves a leaf
probability by a few 1e-5 relative).
"""

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import assert_out_close, np64, npi

pytestmark = pytest.mark.gpu
DEV = "cuda"
TREE_BAND = 1e-3


def _shape(moe, T, d, E, k, renorm):
    return moe.MoeShape(T=T, d=d, E=E, k=k, H=16, renorm=int(renorm))


def _check_routing(got_idx, got_w, r, k):
    p = r["p"]
    srt = -np.sort(-p, axis=1)[:, :k + 1]
    gaps = (srt[:, :-1] - srt[:, 1:]) / srt[:, :-1] if srt.shape[1] > k else np.full((p.shape[0], k), np.inf)
    clear = gaps.min(axis=1) >= TREE_BAND
    assert clear.mean() > 0.5, f"only {clear.mean():.2f} of the tokens are clear of the band"
    assert (got_idx[clear] == r["idx"][clear]).all()
    np.testing.assert_allclose(got_w[clear], r["w"][clear], rtol=1e-3, atol=1e-7)
    # every token: distinct leaves in range, each within the band below the oracle's k-th
    assert (got_idx >= 0).all() and (got_idx < p.shape[1]).all()
    assert all(len(set(row)) == k for row in got_idx.tolist())
    pk = srt[:, k - 1]
    picked = np.take_along_axis(p, got_idx.astype(np.int64), axis=1)
    assert (picked >= pk[:, None] * (1 - 2 * TREE_BAND)).all()
    return clear


@pytest.mark.parametrize("T,d,B,L,k,renorm,bias", [(256, 64, 4, 2, 2, True, False),
                                                   (1024, 256, 8, 3, 4, True, True),
                                                   (2048, 768, 16, 3, 8, False, False),
                                                   (512, 128, 2, 8, 3, True, False),
                                                   (300, 64, 32, 1, 4, True, True),
                                                   (256, 768, 16, 4, 16, True, False)])
def test_tree_router_matches_oracle(lib, T, d, B, L, k, renorm, bias):
    moe = lib
    E = B ** L
    inp = synth.draw_tree_router(T, d, B, L, seed=3, device=DEV)
    b = (torch.linspace(-0.5, 0.5, B * L, device=DEV, dtype=torch.float32) if bias else None)
    s = _shape(moe, T, d, E, k, renorm)
    got = moe.moe_route_tree(s, B, L, inp["x"], inp["w_tree"], b, counts=True, logits=True)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    x64, w64 = np64(inp["x"]), np64(inp["w_tree"])
    r = O.route_tree(x64, w64, np64(b) if bias else None, B, L, k, renorm)
    # level logits within the screening bound of the exact ones
    gamma = (2.0 ** -16 + (2 * d + 2) * 2.0 ** -23) * (1 + 2.0 ** -7)
    bound = gamma * np.linalg.norm(x64, axis=1)[:, None] * np.linalg.norm(w64, axis=1)[None, :]
    assert (np.abs(np64(got["level_logits"]) - r["z"]) <= bound + 1e-6).all()
    idx, w = npi(got["topk_idx"]), np64(got["topk_w"])
    clear = _check_routing(idx, w, r, k)
    assert (npi(got["counts"]) == np.bincount(idx.ravel(), minlength=E)).all()
    print(f"B={B} L={L} E={E} k={k}: {clear.mean():.4f} of tokens clear of the band, all of them equal")


def test_tree_router_errors(lib):
    moe = lib
    x = torch.zeros(8, 64, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(8, 64, dtype=torch.float32, device=DEV)
    with pytest.raises(moe.MoeError):   # E != branch^levels
        moe.moe_route_tree(_shape(moe, 8, 64, 15, 2, True), 4, 2, x, w)
    with pytest.raises(moe.MoeError):   # branch above 32
        moe.moe_route_tree(_shape(moe, 8, 64, 64 * 64, 2, True), 64, 2, x, torch.zeros(128, 64, device=DEV))


def test_tree_routed_layer_matches_oracle(lib):
    # tree routing, then the library's grouping, grouped expert FFN and combine: E = 4^3 = 64 experts
    moe = lib
    B, L, k = 4, 3, 2
    E = B ** L
    wl = synth.get_workload("tiny").replace(E=E, k=k, T=512)
    inp = synth.make_inputs(wl, seed=8, device=DEV)
    tr = synth.draw_tree_router(wl.T, wl.d, B, L, seed=8, device=DEV)
    s = moe.MoeShape(T=wl.T, d=wl.d, E=E, k=k, H=wl.H, renorm=1)
    rt = moe.moe_route_tree(s, B, L, inp["x"], tr["w_tree"])
    p = moe.moe_permute(s, inp["x"], rt["topk_idx"])
    _, y = moe.moe_expert_ffn(s, p["x_perm"], inp["w13"], inp["w2"], hidden=wl.H, group_start=p["offsets"][:E],
                              group_rows=p["kept"])
    out = moe.moe_combine(s, y, p["slot_pos"], rt["topk_w"])
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    x64 = np64(inp["x"])
    r = O.route_tree(x64, np64(tr["w_tree"]), None, B, L, k, True)
    clear = _check_routing(npi(rt["topk_idx"]), np64(rt["topk_w"]), r, k)
    fw = O.moe_forward(x64, None, None, np64(inp["w13"]), np64(inp["w2"]), k=k, act=wl.act, routing=r)
    assert_out_close(np64(out)[clear], fw["out"][clear], "tree-routed layer")
