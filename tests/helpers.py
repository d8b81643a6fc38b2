"""Shared test helpers: shape construction, tensor conversion, the output tolerance."""

import numpy as np
import torch

# Output tolerance of the layer (bf16 inputs, fp32 accumulation, bf16 h / y / out):
# relative Frobenius error <= 5e-3 and max |delta| <= 3e-2 against the float64 oracle.
REL_FROB = 5e-3
MAX_ABS = 3e-2
# Tokens whose k-th vs (k+1)-th logit margin is below this are excluded from
# routing and output comparisons (fp32 logits may order them either way).
MARGIN = 1e-5


def np64(t) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def npi(t) -> np.ndarray:
    return t.detach().to("cpu").numpy()


def shape_of(moe, wl, T=None, capacity=None):
    import oracle
    T = wl.T if T is None else T
    if capacity is None:
        capacity = oracle.capacity(T, wl.k, wl.E, wl.capacity_factor)
    return moe.MoeShape(T=T, d=wl.d, E=wl.E, k=wl.k, H=wl.H, H_s=wl.H_s, capacity=capacity, act=wl.act,
                        wfmt=wl.wfmt, renorm=wl.renorm)


def rel_frob(a, b) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_out_close(got, want, what="out", rel=REL_FROB, atol=MAX_ABS):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    r = rel_frob(got, want)
    m = float(np.abs(got - want).max()) if got.size else 0.0
    assert r <= rel and m <= atol, f"{what}: rel Frobenius {r:.3e} (<= {rel}), max|d| {m:.3e} (<= {atol})"
    return r, m


def assert_bf16_rounded(got, want, scale, what="value"):
    """Elementwise bound for a bf16-rounded intermediate: |got - want| <= 2^-8 * (|want| + scale).

    ``scale`` carries the propagated error of bf16-rounded inputs (e.g. |h| @ |W2|^T for y = h W2^T);
    one bf16 rounding is at most 2^-9 relative, the factor 2 covers fp32 accumulation and the
    approximate exp of the activation.
    """
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    bound = 2.0 ** -8 * (np.abs(want) + scale) + 1e-6
    bad = np.abs(got - want) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements outside the bf16 bound, worst " \
        f"{float((np.abs(got - want) / bound).max()):.2f}x"


def glu_accum_scale(x, w13, act):
    """Propagated fp32 accumulation error of h = act(x W1^T) * (x W3^T), as a ``scale`` for assert_bf16_rounded.

    Each of g = x W1^T and u = x W3^T is a d-term fp32 dot product, off by at most d * 2^-24 * |x| @ |W|^T
    (recursive summation); |act'| <= 1.13 for SiLU and exact-erf GELU, so
    |dh| <= gamma_d * (1.13 * (|x| @ |W1|^T) * |u| + |act(g)| * (|x| @ |W3|^T)).  At points where g or u
    cancels to nearly zero this term, not the bf16 rounding of h, dominates.
    """
    import oracle
    x = np.asarray(x, np.float64)
    w13 = np.asarray(w13, np.float64)
    H = w13.shape[0] // 2
    d = x.shape[1]
    g, u = x @ w13[:H].T, x @ w13[H:].T
    a = oracle.silu(g) if act == 0 else oracle.gelu_erf(g)
    gam = 1.01 * d * 2.0 ** -24
    err = gam * (1.13 * (np.abs(x) @ np.abs(w13[:H]).T) * np.abs(u) + np.abs(a) * (np.abs(x) @ np.abs(w13[H:]).T))
    return err * 2.0 ** 8


def int4_expert_weights(moe, wl, seed=0, device="cuda", experts=None):
    """Draw every expert's fp32 weights with synth (on ``device``) and pack them with the library's INT4 quantiser.

    Returns dict w13 [E,2H,d/2] u8, s13 [E,2H,d/128] bf16, w2 [E,d,H/2] u8, s2 [E,d,H/128] bf16 and, when
    H_s > 0, the shared expert's w13_sh, s13_sh, w2_sh, s2_sh with a leading dim of 1.
    """
    import synth
    E, d, H = wl.E, wl.d, wl.H
    out = dict(w13=torch.empty(E, 2 * H, d // 2, dtype=torch.uint8, device=device),
               s13=torch.empty(E, 2 * H, d // 128, dtype=torch.bfloat16, device=device),
               w2=torch.empty(E, d, H // 2, dtype=torch.uint8, device=device),
               s2=torch.empty(E, d, H // 128, dtype=torch.bfloat16, device=device))
    for e in range(E):
        a, b = synth.expert_weights_f32(wl, seed, e, device)
        moe.moe_quantize_int4(a, q=out["w13"][e], scales=out["s13"][e])
        moe.moe_quantize_int4(b, q=out["w2"][e], scales=out["s2"][e])
    if wl.H_s:
        a, b = synth.expert_weights_f32(wl, seed, E, device)
        q13, s13 = moe.moe_quantize_int4(a)
        q2, s2 = moe.moe_quantize_int4(b)
        out.update(w13_sh=q13[None], s13_sh=s13[None], w2_sh=q2[None], s2_sh=s2[None])
    return out


def oracle_int4_from_f32(a, b):
    """float64 (w13, w2) after the oracle's own quantise -> pack -> dequantise of fp32 draws (numpy arrays)."""
    import oracle as O
    qa, sa = O.quantize_int4_g128(a)
    qb, sb = O.quantize_int4_g128(b)
    return (O.dequantize_int4_g128(O.pack_int4(qa), sa), O.dequantize_int4_g128(O.pack_int4(qb), sb))


def oracle_int4_expert(wl, seed, e, device="cuda"):
    """float64 (w13, w2) of expert e after the oracle's own quantise -> dequantise of the same fp32 draws."""
    import synth
    a, b = synth.expert_weights_f32(wl, seed, e, device)
    return oracle_int4_from_f32(a.cpu().numpy(), b.cpu().numpy())
