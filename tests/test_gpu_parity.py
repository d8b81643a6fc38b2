"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Routing, grouping and quantised codes must match bit for bit; float outputs
must meet the layer tolerance (relative Frobenius <= 5e-3, max|delta| <= 3e-2)
or the per-step tolerances derived in each test.  Inputs are drawn by
``synth`` with fixed seeds; the oracle never receives a value computed by the
CUDA path.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synth
from helpers import MARGIN, assert_bf16_rounded, assert_out_close, glu_accum_scale, np64, npi, rel_frob, shape_of

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _shape(moe, T, E, k, d=16, H=16, H_s=0, cap=0, act=0, renorm=1, wfmt=0):
    return moe.MoeShape(T=T, d=d, E=E, k=k, H=H, H_s=H_s, capacity=cap, act=act, wfmt=wfmt, renorm=renorm)


# ---------------------------------------------------------------- router


@pytest.mark.parametrize("T,E,k,renorm,mode", [(300, 8, 2, 1, "normal"), (1000, 192, 4, 1, "coarse"),
                                               (257, 384, 8, 0, "signed_zero"), (64, 33, 5, 1, "equal"),
                                               (130, 512, 16, 1, "normal"), (5, 3, 3, 0, "coarse"),
                                               (129, 1, 1, 1, "normal")])
def test_route_from_logits_bit_exact(lib, T, E, k, renorm, mode):
    moe = lib
    z = synth.draw_logits(T, E, seed=T + E, mode=mode)
    s = _shape(moe, T, E, k, renorm=renorm)
    r = moe.moe_route_from_logits(s, z.to(DEV), aux=True)
    torch.cuda.synchronize()
    z64 = z.double().numpy()
    ref = O.route_from_logits(z64, k, bool(renorm))
    assert (npi(r["topk_idx"]) == ref["idx"]).all()
    assert (npi(r["counts"]) == ref["counts"]).all()
    # fp32 softmax with expf and an E-term sum: relative error well inside 2e-5
    np.testing.assert_allclose(np64(r["topk_w"]), ref["w"], rtol=2e-5, atol=1e-30)
    np.testing.assert_allclose(np64(r["aux_f"]), ref["f"], rtol=1e-7)
    np.testing.assert_allclose(np64(r["aux_p"]), ref["P"], rtol=2e-5, atol=1e-12)
    np.testing.assert_allclose(np64(r["aux"])[0], ref["aux"], rtol=2e-5)


def _route_case(moe, wl, T, seed):
    wl = wl.replace(T=T)
    inp = synth.make_inputs(wl, seed=seed, device="cpu", with_expert_weights=False)
    s = shape_of(moe, wl)
    bias = inp["bias"].to(DEV) if inp["bias"] is not None else None
    r = moe.moe_route(s, inp["x"].to(DEV), inp["w_router"].to(DEV), bias, logits=True, aux=True)
    torch.cuda.synchronize()
    x64 = np64(inp["x"])
    W64 = np64(inp["w_router"])
    b64 = np64(inp["bias"]) if inp["bias"] is not None else None
    ref = O.route(x64, W64, b64, wl.k, bool(wl.renorm))
    return wl, inp, r, ref, x64, W64, b64


# Router paths: lane-per-token router for E <= 16 (tiny, small, E = 13), shared-memory router for
# 16 < E <= 256 with a small W_r (geglu's E = 32, E = 64), certified tensor-core router (skewed, granular shapes),
# weight-streaming decode router (decode_int4; T <= 256: one token, a ragged token block with E = 200
# and a ragged last input slice with d = 784), split-K CUDA-core router (E = 200, which is neither a
# multiple of 16 nor small enough for the shared-memory router).
@pytest.mark.parametrize("name,T,over", [("tiny", 256, {}), ("small", 4096, {}), ("tiny", 300, {"E": 13}),
                                         ("small", 1000, {"E": 64, "k": 4}), ("skewed", 3000, {}),
                                         ("geglu", 2000, {}), ("decode_int4", 64, {}), ("decode_int4", 1, {}),
                                         ("granular", 37, {"E": 200, "d": 784}),
                                         ("granular", 1000, {"E": 200}), ("decode_int4", 300, {"E": 96})])
def test_route_matches_oracle(lib, name, T, over):
    wl, inp, r, ref, x64, W64, b64 = _route_case(lib, synth.get_workload(name).replace(**over), T, seed=1)
    # Logits.  Every logit is within the bound of the tensor-core screening pass: the two-term bf16 split of
    # W_r (representation error 2^-16 |w|) plus an fp32 accumulation of 2d products in any rounding direction;
    # the logits of the chosen experts are plain fp32 FMA dot products, within the round-to-nearest bound
    # gamma_{d+2} * sum|x_i w_i| (+ |bias|).
    zg = np64(r["logits"])
    mag = np.abs(x64) @ np.abs(W64).T + (np.abs(b64) if b64 is not None else 0)
    assert (np.abs(zg - ref["z"]) <= (2.0 ** -16 + (2 * wl.d + 2) * 2.0 ** -23) * 1.01 * mag + 1e-7).all()
    sel = np.take_along_axis(np.abs(zg - ref["z"]) - (wl.d + 2) * 2.0 ** -24 * mag, npi(r["topk_idx"]).astype(np.int64),
                             axis=1)
    assert (sel <= 0).all()
    # top-k: bit-exact where the oracle's k-th/(k+1)-th margin is >= 1e-5; inside the band any choice
    # within the band is valid
    margin = O.topk_margin(ref["z"], wl.k)
    amb = margin < MARGIN
    idx = npi(r["topk_idx"])
    assert (idx[~amb] == ref["idx"][~amb]).all()
    for t in np.nonzero(amb)[0]:
        kth = np.sort(ref["z"][t])[::-1][wl.k - 1]
        assert len(set(idx[t].tolist())) == wl.k
        assert (ref["z"][t, idx[t]] >= kth - MARGIN).all()
    if not amb.any():
        assert (npi(r["counts"]) == ref["counts"]).all()
        np.testing.assert_allclose(np64(r["topk_w"]), ref["w"], rtol=5e-5)
        np.testing.assert_allclose(np64(r["aux_p"]), ref["P"], rtol=5e-5)
        np.testing.assert_allclose(np64(r["aux"])[0], ref["aux"], rtol=5e-5)


# Tensor-core router with the certified selection kernels (taken when neither logits nor the load-balance
# statistic is requested): every k up to 16, column tiles of 64 (E = 48: 16 padding columns), 128, 192 and
# 256, single-CTA screening tiles (batches below a wave of 128-row tiles) and CTA-pair tiles (the full granular
# batch; 20000 tokens: a ragged last 256-row tile), the largest input width it takes (d = 2048), a skew bias,
# and tokens whose input row is zero (every logit equal, more candidates than the selection keeps: those tokens
# are finished from exact logits of every expert, lowest indices first).
@pytest.mark.parametrize("name,T,over,zero_rows", [("skewed", 3000, {}, 0), ("granular", 32768, {}, 0),
                                                   ("granular", 1100, {"E": 256, "k": 8, "d": 1024}, 0),
                                                   ("granular", 2100, {"E": 64, "k": 2, "d": 2048}, 0),
                                                   ("skewed", 20000, {"E": 48, "k": 3}, 0),
                                                   ("granular", 19500, {"E": 128, "k": 4, "d": 512}, 0),
                                                   ("granular", 2000, {"k": 16}, 0),
                                                   ("granular", 2000, {}, 37)])
def test_route_select_path_matches_oracle(lib, name, T, over, zero_rows):
    moe = lib
    wl = synth.get_workload(name).replace(T=T, **over)
    inp = synth.make_inputs(wl, seed=2, device="cpu", with_expert_weights=False)
    x = inp["x"].clone()
    if zero_rows:
        x[5:5 + zero_rows] = 0
    s = shape_of(moe, wl)
    assert T * wl.E * wl.d >= 1 << 28 and wl.E % 16 == 0        # the tensor-core router's range
    bias = inp["bias"].to(DEV) if inp["bias"] is not None else None
    r = moe.moe_route(s, x.to(DEV), inp["w_router"].to(DEV), bias)                 # selection path
    full = moe.moe_route(s, x.to(DEV), inp["w_router"].to(DEV), bias, logits=True)  # logits path
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    # both certify the same exact fp32 decisions
    assert (npi(r["topk_idx"]) == npi(full["topk_idx"])).all()
    assert (npi(r["counts"]) == npi(full["counts"])).all()
    np.testing.assert_allclose(np64(r["topk_w"]), np64(full["topk_w"]), rtol=2e-6, atol=1e-9)
    x64 = np64(x)
    b64 = np64(inp["bias"]) if inp["bias"] is not None else None
    ref = O.route(x64, np64(inp["w_router"]), b64, wl.k, bool(wl.renorm))
    amb = O.topk_margin(ref["z"], wl.k) < MARGIN
    idx = npi(r["topk_idx"])
    assert (idx[~amb] == ref["idx"][~amb]).all()
    for t in np.nonzero(amb)[0]:
        kth = np.sort(ref["z"][t])[::-1][wl.k - 1]
        assert len(set(idx[t].tolist())) == wl.k
        assert (ref["z"][t, idx[t]] >= kth - MARGIN).all()
    if zero_rows:
        # all logits equal the bias (none here): the k lowest expert indices, equal gates
        assert (idx[5:5 + zero_rows] == np.arange(wl.k)[None, :]).all()
        np.testing.assert_allclose(np64(r["topk_w"])[5:5 + zero_rows], 1.0 / wl.k, rtol=1e-6)
    ok = ~amb
    np.testing.assert_allclose(np64(r["topk_w"])[ok], ref["w"][ok], rtol=5e-5)
    if not amb.any():
        assert (npi(r["counts"]) == ref["counts"]).all()


# ---------------------------------------------------------------- grouping


@pytest.mark.parametrize("T,E,k,cap,skew,d", [(256, 8, 2, 0, 0.0, 64), (256, 8, 2, 32, 0.0, 64),
                                              (1000, 192, 4, 0, 1.2, 768), (1000, 192, 4, 27, 1.2, 768),
                                              (70, 384, 8, 0, 0.0, 256), (129, 5, 5, 0, 0.0, 16),
                                              (4096, 32, 2, 300, 1.2, 128), (1, 4, 2, 1, 0.0, 32),
                                              (300, 512, 16, 0, 0.5, 48)])
def test_permute_bit_exact(lib, T, E, k, cap, skew, d):
    moe = lib
    idx = synth.draw_topk_idx(T, E, k, seed=T * 7 + E, skew=skew)
    g = torch.Generator().manual_seed(T)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    s = _shape(moe, T, E, k, d=d, cap=cap)
    r = moe.moe_permute(s, x.to(DEV), idx.to(DEV))
    torch.cuda.synchronize()
    ref = O.permute(npi(idx), E, cap)
    for key in ("slot_pos", "counts", "kept", "offsets", "row_src"):
        assert (npi(r[key]) == ref[key]).all(), key
    assert (npi(r["drop_mask"]) == ref["drop"]).all()
    rs = ref["row_src"]
    filled = rs >= 0
    xp = npi(r["x_perm"].view(torch.int16))
    xs = npi(x.view(torch.int16))
    assert (xp[filled] == xs[rs[filled] // k]).all()          # bit-exact row moves


@pytest.mark.parametrize("cap", [854, 0])
def test_permute_bit_exact_full_size(lib, cap):
    """The granular/skewed grouping at full size (T=32768, E=192, top-4; 1024 chunks of 32 tokens), Zipf-like
    skew 1.2, with the workload's capacity C = 854 (heavy drops on the popular experts) and without a capacity."""
    moe = lib
    T, E, k, d = 32768, 192, 4, 768
    idx = synth.draw_topk_idx(T, E, k, seed=4242, skew=1.2)
    g = torch.Generator().manual_seed(77)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    s = _shape(moe, T, E, k, d=d, cap=cap)
    r = moe.moe_permute(s, x.to(DEV), idx.to(DEV))
    torch.cuda.synchronize()
    ref = O.permute(npi(idx), E, cap)
    for key in ("slot_pos", "counts", "kept", "offsets", "row_src"):
        assert (npi(r[key]) == ref[key]).all(), key
    assert (npi(r["drop_mask"]) == ref["drop"]).all()
    if cap:
        assert ref["drop"].sum() > 0
    rs = ref["row_src"]
    filled = rs >= 0
    xp = npi(r["x_perm"].view(torch.int16))
    xs = npi(x.view(torch.int16))
    assert (xp[filled] == xs[rs[filled] // k]).all()


# ---------------------------------------------------------------- grouped expert FFN


@pytest.mark.parametrize("E,d,H,act,max_rows,cap", [(4, 64, 128, 0, 300, 0), (8, 256, 1024, 0, 200, 0),
                                                    (6, 768, 256, 1, 400, 300), (3, 128, 64, 0, 130, 0),
                                                    (2, 64, 32, 1, 100, 0), (1, 96, 48, 0, 200, 0),
                                                    (5, 256, 4096, 1, 140, 0)])
def test_expert_ffn_matches_oracle(lib, E, d, H, act, max_rows, cap):
    moe = lib
    start, rows, R = synth.draw_groups(E, max_rows, seed=E * d + H, cap=cap)
    wl = synth.Workload("t", T=1, d=d, E=E, k=1, H=H, act=act)
    w13 = torch.stack([synth.expert_weights_f32(wl, 3, e)[0] for e in range(E)]).to(torch.bfloat16)
    w2 = torch.stack([synth.expert_weights_f32(wl, 3, e)[1] for e in range(E)]).to(torch.bfloat16)
    g = torch.Generator().manual_seed(E + d)
    xg = torch.randn(R, d, generator=g).to(torch.bfloat16)
    s = _shape(moe, 1, E, 1, d=d, H=H, act=act)
    h, y = moe.moe_expert_ffn(s, xg.to(DEV), w13.to(DEV), w2.to(DEV), hidden=H, group_start=start.to(DEV),
                              group_rows=rows.to(DEV))
    torch.cuda.synchronize()
    x64, w13_64, w2_64 = np64(xg), np64(w13), np64(w2)
    hg, yg = np64(h), np64(y)
    for e in range(E):
        a, n = int(start[e]), int(rows[e])
        if n == 0:
            continue
        h_ref = O.glu_hidden(x64[a:a + n], w13_64[e], act)
        y_ref = h_ref @ w2_64[e].T
        assert_bf16_rounded(hg[a:a + n], h_ref, glu_accum_scale(x64[a:a + n], w13_64[e], act), f"h[e={e}]")
        assert_bf16_rounded(yg[a:a + n], y_ref, np.abs(h_ref) @ np.abs(w2_64[e]).T, f"y[e={e}]")
        assert rel_frob(yg[a:a + n], y_ref) <= 5e-3


# CTA-pair tiles (256 rows, tcgen05 cta_group::2) against the oracle and against the single-CTA kernel on the
# same inputs: ragged groups (an empty one, tails shorter than the second CTA's 128 rows), gated SwiGLU and GeGLU
# GEMMs and a plain down GEMM wide enough for 256-column tiles.
@pytest.mark.parametrize("d,H,act,rows", [(256, 2048, 0, [1000, 0, 1001]), (512, 1024, 1, [1500, 129]),
                                          (1024, 512, 0, [1500, 1500])])
def test_expert_ffn_pair_tiles(lib, d, H, act, rows):
    moe = lib
    E = len(rows)
    rows_t = torch.tensor(rows, dtype=torch.int32)
    start = torch.cumsum(torch.tensor([0] + rows[:-1]), 0).to(torch.int32)
    R = int(sum(rows))
    wl = synth.Workload("t", T=1, d=d, E=E, k=1, H=H, act=act)
    w13 = torch.stack([synth.expert_weights_f32(wl, 4, e)[0] for e in range(E)]).to(torch.bfloat16)
    w2 = torch.stack([synth.expert_weights_f32(wl, 4, e)[1] for e in range(E)]).to(torch.bfloat16)
    g = torch.Generator().manual_seed(d + H)
    xg = torch.randn(R, d, generator=g).to(torch.bfloat16)
    outs = {}
    for pair in (True, False):
        s = moe.MoeShape(T=1, d=d, E=E, k=1, H=H, act=act, flags=0 if pair else moe.FLAG_SINGLE_CTA_GEMM)
        h, y = moe.moe_expert_ffn(s, xg.to(DEV), w13.to(DEV), w2.to(DEV), hidden=H, group_start=start.to(DEV),
                                  group_rows=rows_t.to(DEV))
        torch.cuda.synchronize()
        outs[pair] = (np64(h), np64(y))
    x64, w13_64, w2_64 = np64(xg), np64(w13), np64(w2)
    for pair, (hg, yg) in outs.items():
        for e in range(E):
            a, n = int(start[e]), int(rows[e])
            if n == 0:
                continue
            h_ref = O.glu_hidden(x64[a:a + n], w13_64[e], act)
            y_ref = h_ref @ w2_64[e].T
            assert_bf16_rounded(hg[a:a + n], h_ref, glu_accum_scale(x64[a:a + n], w13_64[e], act), f"h[e={e}, pair={pair}]")
            assert_bf16_rounded(yg[a:a + n], y_ref, np.abs(h_ref) @ np.abs(w2_64[e]).T, f"y[e={e}, pair={pair}]")
            assert rel_frob(yg[a:a + n], y_ref) <= 5e-3
    same_h = np.array_equal(outs[True][0], outs[False][0])
    same_y = np.array_equal(outs[True][1], outs[False][1])
    print(f"pair vs single: h identical={same_h} y identical={same_y}")


# Fused gate/up -> down kernel (h kept in shared memory; moe_expert_ffn with h = NULL): hidden 128 and 256,
# SwiGLU and GeGLU, CTA pairs (groups averaging >= 192 rows) and single CTAs (the flag, or small groups), an
# empty group, groups shorter than one tile, a model width that leaves a partial 256-column down chunk (320) and
# one below a single chunk (64); y against the oracle and against the unfused kernels on the same inputs.
@pytest.mark.parametrize("E,d,H,act,max_rows,single", [(6, 768, 256, 0, 900, False), (6, 768, 256, 1, 900, True),
                                                       (5, 320, 128, 0, 700, False), (4, 64, 256, 1, 300, False),
                                                       (7, 256, 128, 1, 150, False), (3, 768, 256, 0, 60, False)])
def test_expert_ffn_fused_matches_oracle(lib, E, d, H, act, max_rows, single):
    moe = lib
    start, rows, R = synth.draw_groups(E, max_rows, seed=E * d + H + 1)
    rows[1] = 0                                                   # an empty group
    start = torch.cumsum(torch.cat([torch.zeros(1, dtype=rows.dtype), rows[:-1]]), 0).to(torch.int32)
    R = int(rows.sum())
    wl = synth.Workload("t", T=1, d=d, E=E, k=1, H=H, act=act)
    w13 = torch.stack([synth.expert_weights_f32(wl, 6, e)[0] for e in range(E)]).to(torch.bfloat16)
    w2 = torch.stack([synth.expert_weights_f32(wl, 6, e)[1] for e in range(E)]).to(torch.bfloat16)
    g = torch.Generator().manual_seed(E + d + H)
    xg = torch.randn(R, d, generator=g).to(torch.bfloat16)
    s = moe.MoeShape(T=1, d=d, E=E, k=1, H=H, act=act, flags=moe.FLAG_SINGLE_CTA_GEMM if single else 0)
    args = (s, xg.to(DEV), w13.to(DEV), w2.to(DEV))
    kw = dict(hidden=H, group_start=start.to(DEV), group_rows=rows.to(DEV))
    h0, y_fused = moe.moe_expert_ffn(*args, want_h=False, **kw)
    h_ref_gpu, y_unfused = moe.moe_expert_ffn(*args, **kw)
    torch.cuda.synchronize()
    assert h0 is None and moe.moe_get_status()[0] == 0
    x64, w13_64, w2_64 = np64(xg), np64(w13), np64(w2)
    yg = np64(y_fused)
    for e in range(E):
        a, n = int(start[e]), int(rows[e])
        if n == 0:
            continue
        h_ref = O.glu_hidden(x64[a:a + n], w13_64[e], act)
        y_ref = h_ref @ w2_64[e].T
        # h rounded to bf16 once (as in the unfused kernel): y inherits |h| |W2|^T 2^-8 plus the bf16 y rounding
        assert_bf16_rounded(yg[a:a + n], y_ref, np.abs(h_ref) @ np.abs(w2_64[e]).T, f"y[e={e}]")
        assert rel_frob(yg[a:a + n], y_ref) <= 5e-3
    assert_bf16_rounded(yg, np64(y_unfused), 1e-3 * np.abs(np64(y_unfused)), "fused vs unfused")
    print(f"fused vs unfused y identical: {torch.equal(y_fused, y_unfused)}")


@pytest.mark.parametrize("act", [0, 1])
def test_glu_activation_grid(lib, act):
    """The epilogue activation alone: one-hot inputs make g = W1[:, 0] (a grid over [-8, 8] in bf16) and u = 1,
    so h = act(g) to within one bf16 rounding.  Pins SiLU and the exact-erf GELU (the oracle's scipy erf)."""
    moe = lib
    H, d, R = 2048, 64, 128
    g = torch.linspace(-8, 8, H).to(torch.bfloat16)
    w13 = torch.zeros(1, 2 * H, d)
    w13[0, :H, 0] = g.float()
    w13[0, H:, 0] = 1.0
    w2 = torch.zeros(1, d, H)
    x = torch.zeros(R, d)
    x[:, 0] = 1.0
    s = _shape(moe, R, 1, 1, d=d, H=H, act=act)
    h, _ = moe.moe_expert_ffn(s, x.to(torch.bfloat16).to(DEV), w13.to(torch.bfloat16).to(DEV),
                              w2.to(torch.bfloat16).to(DEV), hidden=H)
    torch.cuda.synchronize()
    g64 = np64(g)
    want = O.silu(g64) if act == 0 else O.gelu_erf(g64)
    got = np64(h)
    assert (np.abs(got - want[None, :]) <= 2.0 ** -8 * np.abs(want)[None, :] + 1e-6).all()


def test_expert_ffn_single_dense_group(lib):
    moe = lib
    wl = synth.Workload("t", T=1000, d=256, E=1, k=1, H=512)
    w13, w2 = synth.expert_weights_f32(wl, 5, 0)
    g = torch.Generator().manual_seed(9)
    x = torch.randn(1000, 256, generator=g).to(torch.bfloat16)
    s = _shape(moe, 1000, 1, 1, d=256, H=512)
    h, y = moe.moe_expert_ffn(s, x.to(DEV), w13.to(torch.bfloat16)[None].to(DEV),
                              w2.to(torch.bfloat16)[None].to(DEV), hidden=512)
    torch.cuda.synchronize()
    ref = O.expert_ffn(np64(x), np64(w13.to(torch.bfloat16)), np64(w2.to(torch.bfloat16)), 0)
    assert_out_close(np64(y), ref)


# ---------------------------------------------------------------- combine


@pytest.mark.parametrize("T,E,k,cap,d,shared", [(256, 8, 2, 0, 64, False), (500, 16, 4, 100, 256, True),
                                                (64, 384, 8, 0, 7168, True), (33, 4, 3, 5, 16, False)])
def test_combine_matches_oracle(lib, T, E, k, cap, d, shared):
    moe = lib
    idx = synth.draw_topk_idx(T, E, k, seed=11, skew=1.0)
    g = torch.Generator().manual_seed(T + d)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    s = _shape(moe, T, E, k, d=d, cap=cap)
    p = moe.moe_permute(s, x.to(DEV), idx.to(DEV))
    ref = O.permute(npi(idx), E, cap)
    R = s.R
    y_perm = torch.randn(R, d, generator=g).to(torch.bfloat16)
    w = torch.rand(T, k, generator=g)
    ysh = torch.randn(T, d, generator=g).to(torch.bfloat16) if shared else None
    out = moe.moe_combine(s, y_perm.to(DEV), p["slot_pos"], w.to(DEV), ysh.to(DEV) if shared else None)
    torch.cuda.synchronize()
    assert (npi(p["slot_pos"]) == ref["slot_pos"]).all()
    want = O.combine(np64(y_perm), ref["slot_pos"], np64(w), np64(ysh) if shared else None)
    # fp32 sum of <= k+1 terms, one bf16 rounding: |delta| <= 2^-8 |out| + k * 2^-23 sum|terms|
    got = np64(out)
    bound = 2.0 ** -8 * np.abs(want) + 1e-6 * (np.abs(want) + 1)
    assert (np.abs(got - want) <= bound).all()


# ---------------------------------------------------------------- whole layer


def _forward_case(moe, wl, seed=0, device="cpu"):
    inp = synth.make_inputs(wl, seed=seed, device=device)
    s = shape_of(moe, wl)
    d_ = {k_: (v.to(DEV) if v is not None else None) for k_, v in inp.items()}
    r = moe.moe_forward(s, d_["x"], d_["w_router"], d_["w13"], d_["w2"], bias=d_["bias"],
                        w13_sh=d_.get("w13_sh"), w2_sh=d_.get("w2_sh"), routing=True, aux=wl.aux)
    torch.cuda.synchronize()
    st, site = moe.moe_get_status()
    assert st == 0, (st, hex(site))
    return inp, s, r


def _check_forward(wl, inp, s, r, sample=None):
    """Compare a GPU forward with the oracle; returns (n_excluded, rel, maxabs)."""
    x64 = np64(inp["x"])
    b64 = np64(inp["bias"]) if inp["bias"] is not None else None
    ref_r = O.route(x64, np64(inp["w_router"]), b64, wl.k, bool(wl.renorm))
    idx_g = npi(r["topk_idx"])
    amb = O.topk_margin(ref_r["z"], wl.k) < MARGIN
    assert (idx_g[~amb] == ref_r["idx"][~amb]).all()
    flipped = np.nonzero((idx_g != ref_r["idx"]).any(1))[0]
    cap = s.capacity
    perm = O.permute(ref_r["idx"], wl.E, cap)
    excl = np.zeros(wl.T, bool)
    excl[flipped] = True
    if cap and flipped.size:
        # A flipped token shifts by one the ranks of later tokens on the experts it moved between; drop
        # decisions can then differ only on those experts that reach the capacity in either routing.
        cnt_g = npi(r["counts"])
        aff = set()
        for t in flipped:
            aff |= set(idx_g[t].tolist()) ^ set(ref_r["idx"][t].tolist())
        aff = [e for e in aff if max(cnt_g[e], ref_r["counts"][e]) > cap]
        if aff:
            later = np.arange(wl.T) > flipped.min()
            excl |= later & np.isin(ref_r["idx"], aff).any(1)
            excl |= later & np.isin(idx_g, aff).any(1)
    assert (npi(r["drop_mask"])[~excl] == perm["drop"][~excl]).all()
    if not flipped.size:
        assert (npi(r["counts"]) == ref_r["counts"]).all()
    toks = np.arange(wl.T) if sample is None else np.asarray(sample)
    toks = toks[~excl[toks]]
    w13 = inp["w13"]
    w2 = inp["w2"]
    out_ref = np.zeros((toks.size, wl.d))
    for n, t in enumerate(toks):
        for j in range(wl.k):
            if perm["drop"][t, j]:
                continue
            e = int(ref_r["idx"][t, j])
            out_ref[n] += ref_r["w"][t, j] * O.expert_ffn(x64[t:t + 1], np64(w13[e]), np64(w2[e]), wl.act)[0]
    if wl.H_s:
        out_ref += O.expert_ffn(x64[toks], np64(inp["w13_sh"][0]), np64(inp["w2_sh"][0]), wl.act)
    got = np64(r["out"])[toks]
    rel, mx = assert_out_close(got, out_ref)
    if wl.aux:
        np.testing.assert_allclose(np64(r["aux"])[0], ref_r["aux"], rtol=5e-5)
    print(f"{wl.name}: T={wl.T} ambiguous={int(amb.sum())} flipped={flipped.size} excluded={int(excl.sum())} "
          f"compared={toks.size} rel={rel:.2e} max={mx:.2e}")
    return int(flipped.size), rel, mx


@pytest.mark.parametrize("name,over", [("tiny", {}), ("small", {}), ("tiny", {"capacity_factor": 0.5}),
                                       ("tiny", {"H_s": 64, "act": 1, "skew": 1.2}),
                                       ("tiny", {"renorm": 0, "k": 3}),
                                       ("granular", {"T": 2048}), ("skewed", {"T": 2048}),
                                       ("geglu", {"T": 512}),
                                       ("granular", {"T": 1024, "skew": 1.2, "capacity_factor": 1.25})])
def test_forward_matches_oracle(lib, name, over):
    wl = synth.get_workload(name).replace(**over)
    inp, s, r = _forward_case(lib, wl)
    n_flip, rel, mx = _check_forward(wl, inp, s, r)
    assert n_flip <= max(2, wl.T // 5000)
    if over.get("capacity_factor") == 0.5:
        assert npi(r["drop_mask"]).sum() > 0


@pytest.mark.parametrize("name", ["granular", "skewed", "geglu"])
def test_forward_full_size_sampled(lib, name):
    """Full workload size, the launch configuration the benchmark times; oracle on sampled tokens."""
    wl = synth.get_workload(name)
    inp, s, r = _forward_case(lib, wl, device=DEV)
    inp = {k_: (v.cpu() if v is not None else None) for k_, v in inp.items()}
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([rng.choice(wl.T, 96, replace=False), [0, wl.T - 1]]))
    n_flip, rel, mx = _check_forward(wl, inp, s, r, sample=sample)
    assert n_flip <= max(2, wl.T // 5000)


# ---------------------------------------------------------------- INT4 quantiser


@pytest.mark.parametrize("rows,K", [(7, 128), (300, 7168), (4096, 256)])
def test_quantize_int4_bit_exact(lib, rows, K):
    moe = lib
    g = torch.Generator().manual_seed(rows + K)
    w = torch.randn(rows, K, generator=g) / math.sqrt(K)
    w[0, :128] = 0.0                   # an all-zero group
    w[1, :6] = torch.tensor([7.0, 0.5, 1.5, 2.5, -0.5, -7.0]) * 0.01
    q, sc = moe.moe_quantize_int4(w.to(DEV))
    torch.cuda.synchronize()
    q_ref, s_ref = O.quantize_int4_g128(w.numpy())
    assert (npi(q) == O.pack_int4(q_ref)).all()
    assert (npi(sc.view(torch.int16)) == (s_ref.view(np.uint32) >> 16).astype(np.int16)).all()


# ---------------------------------------------------------------- failure detection


def test_bounded_wait_reports_timeout(lib):
    moe = lib
    L = moe.load()
    assert moe.moe_get_status()[0] == 0
    assert L.moe_set_wait_limit_ns(20_000_000) == 0           # 20 ms
    try:
        assert L.moe_selftest_wait_timeout(None) == 0
        st, site = moe.moe_get_status(torch.cuda.default_stream())
        assert st == 5                                         # MOE_DEVICE_TIMEOUT
        assert site == 0x7F01
        assert moe.moe_get_status()[0] == 0                    # read clears it
    finally:
        L.moe_set_wait_limit_ns(2_000_000_000)
    # the context is still usable
    x = torch.ones(4, device=DEV)
    assert float(x.sum()) == 4.0


# ---------------------------------------------------------------- INT4 expert path


@pytest.mark.parametrize("E,d,H,act,max_rows", [(6, 256, 256, 0, 12), (3, 1024, 512, 1, 20), (4, 128, 128, 0, 3)])
def test_expert_ffn_int4_matches_oracle(lib, E, d, H, act, max_rows):
    from helpers import int4_expert_weights, oracle_int4_expert
    moe = lib
    wl = synth.Workload("t", T=1, d=d, E=E, k=1, H=H, act=act, wfmt=1)
    start, rows, R = synth.draw_groups(E, max_rows, seed=E + d)
    W = int4_expert_weights(moe, wl, seed=4, device=DEV)
    g = torch.Generator().manual_seed(d)
    xg = torch.randn(max(R, 1), d, generator=g).to(torch.bfloat16)[:R]
    s = _shape(moe, 1, E, 1, d=d, H=H, act=act, wfmt=1)
    h, y = moe.moe_expert_ffn(s, xg.to(DEV), W["w13"], W["w2"], s13=W["s13"], s2=W["s2"], hidden=H,
                              group_start=start.to(DEV), group_rows=rows.to(DEV))
    torch.cuda.synchronize()
    x64, hg, yg = np64(xg), np64(h), np64(y)
    for e in range(E):
        a, n = int(start[e]), int(rows[e])
        if n == 0:
            continue
        w13e, w2e = oracle_int4_expert(wl, 4, e, DEV)
        h_ref = O.glu_hidden(x64[a:a + n], w13e, act)
        assert_bf16_rounded(hg[a:a + n], h_ref, glu_accum_scale(x64[a:a + n], w13e, act), f"h[e={e}]")
        assert_bf16_rounded(yg[a:a + n], h_ref @ w2e.T, np.abs(h_ref) @ np.abs(w2e).T, f"y[e={e}]")


def _int4_forward(moe, wl, seed=0):
    from helpers import int4_expert_weights
    inp = synth.make_inputs(wl, seed=seed, device=DEV, with_expert_weights=False)
    W = int4_expert_weights(moe, wl, seed=seed, device=DEV)
    s = shape_of(moe, wl)
    r = moe.moe_forward(s, inp["x"], inp["w_router"], W["w13"], W["w2"], bias=inp["bias"], s13=W["s13"],
                        s2=W["s2"], w13_sh=W.get("w13_sh"), s13_sh=W.get("s13_sh"), w2_sh=W.get("w2_sh"),
                        s2_sh=W.get("s2_sh"), routing=True)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    return inp, r


def _check_int4_forward(wl, inp, r, sample, seed=0, cap=0):
    """Oracle output of the sampled tokens, one expert at a time: each touched expert's fp32 draw is quantised
    and dequantised by the oracle, applied to the sampled tokens that chose it, then released (the whole
    decode layer in float64 would not fit in host memory).  The oracle work of several experts runs on a thread
    pool (numpy releases the GIL); the fp32 draws come from the device generator in the calling thread."""
    from concurrent.futures import ThreadPoolExecutor

    from helpers import oracle_int4_from_f32
    x64 = np64(inp["x"])
    b64 = np64(inp["bias"]) if inp["bias"] is not None else None
    ref = O.route(x64, np64(inp["w_router"]), b64, wl.k, bool(wl.renorm))
    idx = npi(r["topk_idx"])
    amb = O.topk_margin(ref["z"], wl.k) < MARGIN
    assert (idx[~amb] == ref["idx"][~amb]).all()
    drop = np.zeros((wl.T, wl.k), bool)
    if cap:
        # with a capacity every later drop decision depends on every routing decision: the seeded cases
        # have no near-ties, so the whole routing must agree, and then the drops bit for bit
        assert (idx == ref["idx"]).all()
        drop = O.permute(ref["idx"], wl.E, cap)["drop"].astype(bool)
        assert (npi(r["drop_mask"]).astype(bool) == drop).all()
        assert drop.any()
    toks = np.array([t for t in sample if (idx[t] == ref["idx"][t]).all()], np.int64)
    sel = ref["idx"][toks]                                  # [n, k]
    users = {}                                              # expert -> [(row in toks, slot j)]
    for n in range(toks.size):
        for j in range(wl.k):
            if not drop[toks[n], j]:
                users.setdefault(int(sel[n, j]), []).append((n, j))
    if wl.H_s:
        users[wl.E] = [(n, -1) for n in range(toks.size)]   # the shared expert, weight one

    def job(e, a, b):
        w13e, w2e = oracle_int4_from_f32(a, b)
        rows = np.array([n for n, _ in users[e]], np.int64)
        gate = np.array([1.0 if j < 0 else ref["w"][toks[n], j] for n, j in users[e]])
        return rows, gate[:, None] * O.expert_ffn(x64[toks[rows]], w13e, w2e, wl.act)

    out_ref = np.zeros((toks.size, wl.d))
    import os
    with ThreadPoolExecutor(max_workers=max(1, min(8, len(os.sched_getaffinity(0)) // 2))) as pool:
        futs = []
        for e in sorted(users):
            a, b = synth.expert_weights_f32(wl, seed, e, DEV)
            futs.append(pool.submit(job, e, a.cpu().numpy(), b.cpu().numpy()))
            if len(futs) >= 16:                             # bound the host memory in flight
                rows, y = futs.pop(0).result()
                np.add.at(out_ref, rows, y)
        for f in futs:
            rows, y = f.result()
            np.add.at(out_ref, rows, y)
    assert_out_close(np64(r["out"])[toks], out_ref)
    return toks.size


# Reduced decode layers: batches of 64 (two 32-row blocks of the dense shared-expert kernel), 100 (a ragged
# last row block) and 7 rows; every token against the oracle.
@pytest.mark.parametrize("T", [64, 100, 7])
def test_forward_int4_reduced(lib, T):
    wl = synth.get_workload("decode_int4").replace(T=T, d=1024, E=48, H=256, H_s=256)
    inp, r = _int4_forward(lib, wl)
    _check_int4_forward(wl, inp, r, sample=list(range(wl.T)))


# Capacity drops (the grouped activation copy skips dropped slots) and hidden widths above d (the shared
# expert's activation copy sits past the routed rows of the widest reduction), every token against the oracle.
@pytest.mark.parametrize("over", [{"T": 100, "d": 1024, "E": 48, "H": 256, "H_s": 256, "capacity_factor": 0.5},
                                  {"T": 64, "d": 512, "E": 32, "H": 1024, "H_s": 1024}])
def test_forward_int4_capacity_and_wide_hidden(lib, over):
    wl = synth.get_workload("decode_int4").replace(**over)
    cap = O.capacity(wl.T, wl.k, wl.E, wl.capacity_factor) if wl.capacity_factor else 0
    inp, r = _int4_forward(lib, wl)
    _check_int4_forward(wl, inp, r, sample=list(range(wl.T)), cap=cap)


def test_forward_int4_full_size(lib):
    """The decode workload at full size (8.7 GB of INT4 experts), every one of the 64 tokens against the oracle
    (about 285 touched experts, each dequantised by the oracle once)."""
    wl = synth.get_workload("decode_int4")
    inp, r = _int4_forward(lib, wl)
    n = _check_int4_forward(wl, inp, r, sample=list(range(wl.T)))
    assert n >= wl.T - 2


# ---------------------------------------------------------------- expert parallelism


@pytest.mark.parametrize("name,over", [("tiny", {}), ("granular", {"T": 2048, "skew": 1.2, "capacity_factor": 0.0}),
                                       ("small", {}), ("tiny", {"capacity_factor": 0.5}),
                                       ("granular", {"T": 2048, "skew": 1.2, "capacity_factor": 1.0})])
def test_expert_parallel_single_rank_equals_forward(lib, name, over):
    """moe_forward_ep on one NCCL rank (the exchanges are identities) runs the same kernels on the same grouped
    rows as moe_forward, so the outputs agree bit for bit; the two-rank exchange is covered on gloo (CPU).  With a
    capacity the static-shape exchange also runs the padding rows through the experts, which changes no kept
    row's output."""
    import socket
    from datetime import timedelta

    import torch.distributed as dist

    from sparse_mixture_experts_expert_b200.ep import moe_forward_ep
    moe = lib
    own = not dist.is_initialized()
    if own:
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
        sk.close()
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=timedelta(seconds=60),
                                device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        _ep_single_rank_case(moe, moe_forward_ep, name, over)
    finally:
        if own:
            dist.destroy_process_group()


def test_expert_parallel_static_shapes_capture_in_a_graph(lib):
    """With a capacity, moe_forward_ep has static shapes and no host synchronisation: one NCCL rank captures it
    in a CUDA graph, and the replay gives the eager output."""
    import socket
    from datetime import timedelta

    import torch.distributed as dist

    from sparse_mixture_experts_expert_b200.ep import moe_forward_ep
    moe = lib
    own = not dist.is_initialized()
    if own:
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
        sk.close()
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=timedelta(seconds=60),
                                device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        wl = synth.get_workload("tiny").replace(H_s=64, capacity_factor=0.5)
        inp = synth.make_inputs(wl, seed=5, device=DEV)
        s = shape_of(moe, wl)
        kw = dict(bias=inp["bias"], w13_sh=inp["w13_sh"], w2_sh=inp["w2_sh"])
        eager = moe_forward_ep(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], **kw)[0]
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            out = moe_forward_ep(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], **kw)[0]
        g.replay()
        torch.cuda.synchronize()
        assert moe.moe_get_status()[0] == 0
        assert torch.equal(out, eager)
        del g
    finally:
        if own:
            dist.destroy_process_group()


def _ep_single_rank_case(moe, moe_forward_ep, name, over):
    wl = synth.get_workload(name).replace(**over)
    inp = synth.make_inputs(wl, seed=5, device=DEV)
    s = shape_of(moe, wl)
    assert (s.capacity > 0) == (wl.capacity_factor > 0)
    ref = moe.moe_forward(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], bias=inp["bias"],
                          w13_sh=inp.get("w13_sh"), w2_sh=inp.get("w2_sh"), routing=True)
    out, idx, w = moe_forward_ep(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], bias=inp["bias"],
                                 w13_sh=inp.get("w13_sh"), w2_sh=inp.get("w2_sh"))
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    assert torch.equal(idx, ref["topk_idx"])
    assert torch.equal(out, ref["out"])


# ---------------------------------------------------------------- backward (input gradient)

# rel-Frobenius bound of dx: the expert steps round dy, dh, the recomputed [g | u], [dg | du] and the grouped dx
# to bf16 (each about 2^-9 / sqrt(3) = 1.1e-3 relative, independent), and the router's dz W_r rounds both
# operands: about 2.5e-3 in quadrature, bounded here at 1e-2.
BWD_REL_FROB = 1e-2


@pytest.mark.parametrize("name,over,aux_coef", [("tiny", {}, 0.0),
                                                ("tiny", {"H_s": 64, "act": 1, "capacity_factor": 0.5}, 0.1),
                                                ("small", {}, 0.05),
                                                ("granular", {"T": 1024, "skew": 1.2}, 0.0),
                                                ("geglu", {"T": 512}, 0.0)])
def test_backward_x_matches_oracle(lib, name, over, aux_coef):
    moe = lib
    wl = synth.get_workload(name).replace(**over)
    inp = synth.make_inputs(wl, seed=6, device=DEV)
    s = shape_of(moe, wl)
    g = torch.Generator(device=DEV).manual_seed(17)
    dout = torch.randn(wl.T, wl.d, generator=g, device=DEV).to(torch.bfloat16)
    dx = moe.moe_backward_x(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], dout, bias=inp["bias"],
                            w13_sh=inp.get("w13_sh"), w2_sh=inp.get("w2_sh"), aux_coef=aux_coef)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    b64 = np64(inp["bias"]) if inp["bias"] is not None else None
    ref = O.moe_backward(np64(inp["x"]), np64(inp["w_router"]), b64, np64(inp["w13"]), np64(inp["w2"]),
                           np64(dout), k=wl.k, act=wl.act, renorm=bool(wl.renorm), cap=s.capacity,
                           w13_sh=np64(inp["w13_sh"]) if wl.H_s else None,
                           w2_sh=np64(inp["w2_sh"]) if wl.H_s else None, aux_coef=aux_coef)
    # the routing must agree (the seeded cases have no near-ties): the gradient is taken at the same decision
    r = moe.moe_route(s, inp["x"], inp["w_router"], inp["bias"])
    assert (npi(r["topk_idx"]) == ref["forward"]["idx"]).all()
    got, want = np64(dx), ref["dx"]
    rel = rel_frob(got, want)
    print(f"{name}: rel-Frobenius {rel:.2e}, max|d| {np.abs(got - want).max():.2e}, max|dx| {np.abs(want).max():.2e}")
    assert rel <= BWD_REL_FROB
    assert np.isfinite(got).all()
    # each part of dx is far above the bound, so dropping one would fail: the router (dz W_r) and the shared expert
    router = ref["dz"] @ np64(inp["w_router"])
    assert rel_frob(want - router, want) > 5 * BWD_REL_FROB
    if wl.H_s:
        sh = O.expert_ffn_backward_x(np64(inp["x"]), np64(inp["w13_sh"])[0], np64(inp["w2_sh"])[0], wl.act, np64(dout))
        assert rel_frob(want - sh, want) > 5 * BWD_REL_FROB


# The load-balance term alone (dout = 0, so L = aux_coef * aux): dx = W_r^T dz with dp = aux_coef E f_e / T; a
# uniform f has no effect through the softmax, so the routing is skewed.
@pytest.mark.parametrize("name,over", [("tiny", {"skew": 1.2}), ("granular", {"T": 1024, "skew": 1.2})])
def test_backward_x_load_balance_term_alone(lib, name, over):
    moe = lib
    wl = synth.get_workload(name).replace(**over)
    inp = synth.make_inputs(wl, seed=6, device=DEV)
    s = shape_of(moe, wl)
    dout = torch.zeros(wl.T, wl.d, dtype=torch.bfloat16, device=DEV)
    dx = moe.moe_backward_x(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], dout, bias=inp["bias"],
                            w13_sh=inp.get("w13_sh"), w2_sh=inp.get("w2_sh"), aux_coef=1.0)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    b64 = np64(inp["bias"]) if inp["bias"] is not None else None
    ref = O.moe_backward(np64(inp["x"]), np64(inp["w_router"]), b64, np64(inp["w13"]), np64(inp["w2"]),
                           np64(dout), k=wl.k, act=wl.act, renorm=bool(wl.renorm), cap=s.capacity,
                           w13_sh=np64(inp["w13_sh"]) if wl.H_s else None,
                           w2_sh=np64(inp["w2_sh"]) if wl.H_s else None, aux_coef=1.0)
    r = moe.moe_route(s, inp["x"], inp["w_router"], inp["bias"])
    assert (npi(r["topk_idx"]) == ref["forward"]["idx"]).all()
    want = ref["dx"]
    assert np.abs(want).max() > 0
    rel = rel_frob(np64(dx), want)
    print(f"{name}: load-balance term alone, rel-Frobenius {rel:.2e}")
    assert rel <= BWD_REL_FROB


# Weight gradients: each a bf16 GEMM with fp32 accumulation down the rows, of operands rounded once to bf16
# ([dg | du], w h, dz; x and dout are exact), so about 2^-9 / sqrt(3) relative per term: bounded at 1e-2 in
# rel-Frobenius per tensor, 3e-2 per expert (an expert's few rows average less).  skewed at 4096 tokens has
# three experts above 2048 rows (3770, 2932, 2180), whose gradients are summed from 2048-row chunks.  The tiny
# cases add a ragged token count (300: a partial 8-token block, a partial 64-row reduction step of the dense
# gradients) and gates without renormalisation; the last case has widths that are no multiple of 64 (d = 80,
# H = 48, H_s = 32: partial TMA boxes in every GEMM and weight gradient), E = 6 and k = 3.
@pytest.mark.parametrize("name,over,aux_coef", [("tiny", {"H_s": 64, "act": 1, "capacity_factor": 0.5}, 0.1),
                                                ("tiny", {"T": 300, "H_s": 64}, 0.05),
                                                ("tiny", {"T": 200, "renorm": 0}, 0.1),
                                                ("small", {}, 0.05),
                                                ("granular", {"T": 1024, "skew": 1.2}, 0.0),
                                                ("skewed", {"T": 4096}, 0.0),
                                                ("geglu", {"T": 512, "H": 1024}, 0.0),
                                                ("tiny", {"T": 77, "d": 80, "E": 6, "k": 3, "H": 48, "H_s": 32,
                                                          "act": 1, "skew": 0.5}, 0.2)])
def test_backward_weights_match_oracle(lib, name, over, aux_coef):
    moe = lib
    wl = synth.get_workload(name).replace(**over)
    inp = synth.make_inputs(wl, seed=6, device=DEV)
    s = shape_of(moe, wl)
    g = torch.Generator(device=DEV).manual_seed(17)
    dout = torch.randn(wl.T, wl.d, generator=g, device=DEV).to(torch.bfloat16)
    kw = dict(bias=inp["bias"], w13_sh=inp.get("w13_sh"), w2_sh=inp.get("w2_sh"), aux_coef=aux_coef)
    got = moe.moe_backward(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], dout, **kw)
    dx_only = moe.moe_backward_x(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], dout, **kw)
    side = moe.moe_backward(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], dout, side_stream=torch.cuda.Stream(),
                            **kw)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    assert torch.equal(got["dx"], dx_only)   # the weight gradients leave the input gradient's path unchanged
    for key, v in got.items():               # the shared expert's chain on a second stream: the same results
        assert (v is None and side[key] is None) or torch.equal(v, side[key]), key
    b64 = np64(inp["bias"]) if inp["bias"] is not None else None
    ref = O.moe_backward(np64(inp["x"]), np64(inp["w_router"]), b64, np64(inp["w13"]), np64(inp["w2"]),
                         np64(dout), k=wl.k, act=wl.act, renorm=bool(wl.renorm), cap=s.capacity,
                         w13_sh=np64(inp["w13_sh"]) if wl.H_s else None,
                         w2_sh=np64(inp["w2_sh"]) if wl.H_s else None, aux_coef=aux_coef)
    r = moe.moe_route(s, inp["x"], inp["w_router"], inp["bias"])
    assert (npi(r["topk_idx"]) == ref["forward"]["idx"]).all()
    keys = ["dx", "dw13", "dw2", "dw_router"] + (["dw13_sh", "dw2_sh"] if wl.H_s else [])
    for key in keys:
        a, b = np64(got[key]), ref[key]
        rel = rel_frob(a, b)
        print(f"{name} {key}: rel-Frobenius {rel:.2e}")
        assert np.isfinite(a).all() and rel <= BWD_REL_FROB, key
    kept = ref["forward"]["kept"]
    for key in ("dw13", "dw2"):
        a, b = np64(got[key]), ref[key]
        for e in range(wl.E):
            if kept[e] == 0:
                assert not a[e].any(), f"{key}[{e}]: an expert without rows has a zero gradient"
            else:
                assert rel_frob(a[e], b[e]) <= 3 * BWD_REL_FROB, f"{key}[{e}] ({kept[e]} rows)"
    if not wl.H_s:
        assert got["dw13_sh"] is None and got["dw2_sh"] is None


# The shared expert on a second stream (moe_forward's side_stream) changes nothing in the output: the same kernels
# on the same inputs, joined before the combine.
@pytest.mark.parametrize("name,over", [("granular", {"T": 4096}), ("tiny", {"H_s": 64}), ("small", {})])
def test_forward_side_stream_is_bit_identical(lib, name, over):
    moe = lib
    wl = synth.get_workload(name).replace(**over)
    inp = synth.make_inputs(wl, seed=5, device=DEV)
    s = shape_of(moe, wl)
    kw = dict(bias=inp["bias"], w13_sh=inp.get("w13_sh"), w2_sh=inp.get("w2_sh"), routing=True)
    a = moe.moe_forward(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], **kw)
    side = torch.cuda.Stream()
    b = moe.moe_forward(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], side_stream=side, **kw)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    for key in ("out", "topk_idx", "topk_w", "counts", "drop_mask"):
        assert torch.equal(a[key], b[key]), key
    # and inside a captured graph, replayed
    g = torch.cuda.CUDAGraph()
    out = torch.empty_like(a["out"])
    with torch.cuda.graph(g):
        moe.moe_forward(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], bias=inp["bias"],
                        w13_sh=inp.get("w13_sh"), w2_sh=inp.get("w2_sh"), out=out, side_stream=side)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, a["out"])
    del g


# The autograd wrapper: gradients of loss = sum(dout * out) through torch.autograd equal moe_backward's (cast to
# the parameters' dtypes), and the output equals moe_forward's.
def test_autograd_layer_matches_the_entry_points(lib):
    from sparse_mixture_experts_expert_b200.autograd import moe_layer
    moe = lib
    wl = synth.get_workload("tiny").replace(H_s=64, skew=0.5)
    inp = synth.make_inputs(wl, seed=9, device=DEV)
    s = shape_of(moe, wl)
    g = torch.Generator(device=DEV).manual_seed(3)
    dout = torch.randn(wl.T, wl.d, generator=g, device=DEV).to(torch.bfloat16)
    leaves = {k: inp[k].clone().requires_grad_(True) for k in ("x", "w_router", "w13", "w2", "w13_sh", "w2_sh")}
    out, aux = moe_layer(s, leaves["x"], leaves["w_router"], leaves["w13"], leaves["w2"], bias=inp["bias"],
                         w13_sh=leaves["w13_sh"], w2_sh=leaves["w2_sh"], aux_coef=0.1, return_aux=True)
    (out.float() * dout.float()).sum().backward()
    ref_out = moe.moe_forward(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], bias=inp["bias"],
                              w13_sh=inp["w13_sh"], w2_sh=inp["w2_sh"])
    ref = moe.moe_backward(s, inp["x"], inp["w_router"], inp["w13"], inp["w2"], dout, bias=inp["bias"],
                           w13_sh=inp["w13_sh"], w2_sh=inp["w2_sh"], aux_coef=0.1)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    assert torch.equal(out, ref_out) and not aux.requires_grad
    pairs = [("x", "dx"), ("w_router", "dw_router"), ("w13", "dw13"), ("w2", "dw2"), ("w13_sh", "dw13_sh"),
             ("w2_sh", "dw2_sh")]
    for leaf, key in pairs:
        assert leaves[leaf].grad is not None and leaves[leaf].grad.dtype == leaves[leaf].dtype, leaf
        assert torch.equal(leaves[leaf].grad, ref[key].to(leaves[leaf].dtype)), leaf
