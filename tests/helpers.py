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
