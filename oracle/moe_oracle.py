"""Float64 CPU oracle of the top-k routed Mixture-of-Experts FFN forward pass.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline legs of ``bench.py`` may import this module.  The CUDA library never
imports it, and it imports nothing from the library: the two share no code.
Inputs come from ``synth`` (seeded draws) as numpy arrays holding the exact
bf16 / fp32 input values; everything here widens them to float64.

What it computes, and where each step is defined on the pages it follows:

1. Router logits z = x W_r^T (+ bias_e): the router of "Sharding d'experts"
   (Kvasir wiki), section "Backbone x worker" (``cur @ router``), and
   ``MoEFFN.forward`` in moe_stream.py (``self.gate`` is a bias-free Linear
   [E, d]; the per-expert exploration bias is added to the logits before the
   softmax).
2. p = softmax(z) over experts; top-k experts in order of decreasing z, lowest
   expert index first among equal logits (softmax is monotone, so this is the
   top-k of p); w_j = p[idx_j], optionally renormalised to sum to one
   (``MoEFFN.forward``: softmax, topk, divide by the sum).  The renormalising
   denominator carries no epsilon here (reading: the sum is at least k/E > 0).
3. Load-balance statistic: f_e = counts_e / T, P_e = sum_t p[t,e] / T,
   aux = E * sum_e f_e P_e (``MoEFFN.forward``, "Load balancing loss", batch
   local fractions).
4. Grouping by expert with each (token, slot) identity kept (ExpertMesh
   README: "Activation grouping that preserves token and top-k slot
   identity"; flowchart "Group activations by expert owner").  Groups are in
   expert order; inside a group, rows are in token order.  With a capacity C
   (MoEEvolve README: capacity-factor dispatch with static shapes), group e
   occupies rows [e*C, (e+1)*C) and an assignment whose in-group rank is >= C
   is dropped (reading: ranks counted in token order).
5. Expert FFN, gated: h = act(x W1^T) * (x W3^T), y = h W2^T, with SwiGLU
   (act = SiLU) or GeGLU (act = exact-erf GELU, the torch ``nn.GELU`` default
   used by moe_stream.py) -- MoEEvolve README ("SwiGLU hidden 256"), the
   Kvasir worker's "3 mat-muls", kieve-moe ("top-k GeGLU MoE").
6. Weighted top-k reduction back to token order plus an always-on shared
   expert at weight one: out_t = sum_j w_j y_{e_j}(x_t) + y_shared(x_t)
   (Kvasir "Backbone x worker": ``combine(p, partials) + shared(cur)``;
   ExpertMesh flowchart "Weighted top-k reduction"; ``MoEFFN.forward``:
   ``out[mask] += w * expert_out``).  No residual and no norm.
7. Group-scaled signed INT4 weights (ExpertMesh README: HIP routed-expert
   kernel for group-scaled signed INT4 weights; layout [expert, output,
   packed_input]): one scale per 128 consecutive inputs of an output row,
   s = bf16(max|w| / 7), q = clamp(rint(w / s), -8, 7), two nibbles per byte
   with the even input index in the low nibble; dequantised exactly as q*s.
   The float decisions (max, division, rounding to bf16, rint) are taken in
   fp32, the precision the library's quantiser uses.

Parity pins: every function here is checked by ``tests/test_oracle_*.py``
against closed forms, textbook values (``tests/golden``), brute force on tiny
inputs, the dense compute-all-experts-then-mask evaluation (kieve-moe "Tests":
dense <-> parallel equivalence; Kvasir "Mesure": sharded == monolithic), and
invariants.  Absolute output values of random full-size layers rest on this
independent float64 evaluation (no page prints a worked example).
"""

from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

ACT_SWIGLU = 0
ACT_GEGLU = 1
GROUP = 128   # inputs per INT4 scale group


# ---------------------------------------------------------------- bf16 / fp32 helpers

def bf16_round(a) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even), returned as float32."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).reshape(f.shape)


# ---------------------------------------------------------------- step 1-3: router

def router_logits(x, w_router, bias=None) -> np.ndarray:
    """z[t,e] = sum_i x[t,i] * W_r[e,i] (+ bias[e]), float64."""
    z = np.asarray(x, np.float64) @ np.asarray(w_router, np.float64).T
    if bias is not None:
        z = z + np.asarray(bias, np.float64)[None, :]
    return z


def softmax(z) -> np.ndarray:
    z = np.asarray(z, np.float64)
    m = z.max(axis=1, keepdims=True)
    ez = np.exp(z - m)
    return ez / ez.sum(axis=1, keepdims=True)


def topk_select(z, k: int) -> np.ndarray:
    """Indices [T,k] of the k largest entries per row, larger first, lower index first on ties.

    A stable sort of -z keeps equal keys in index order; -0.0 and +0.0 compare
    equal, so the index decides between them.
    """
    z = np.asarray(z)
    order = np.argsort(-z, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def topk_margin(z, k: int) -> np.ndarray:
    """Gap between the k-th and (k+1)-th largest logit of each row (inf when k == E)."""
    z = np.asarray(z, np.float64)
    if k >= z.shape[1]:
        return np.full(z.shape[0], np.inf)
    s = -np.sort(-z, axis=1)
    return s[:, k - 1] - s[:, k]


def gate_weights(p, idx, renorm: bool) -> np.ndarray:
    w = np.take_along_axis(np.asarray(p, np.float64), np.asarray(idx, np.int64), axis=1)
    if renorm:
        w = w / w.sum(axis=1, keepdims=True)
    return w


def expert_counts(idx, E: int) -> np.ndarray:
    """counts[e] = number of tokens that selected e (before any capacity drop)."""
    return np.bincount(np.asarray(idx, np.int64).ravel(), minlength=E).astype(np.int64)


def load_balance(counts, p, T: int, E: int):
    """(f, P, aux): f_e = counts_e/T, P_e = mean_t p[t,e], aux = E * sum_e f_e P_e."""
    f = np.asarray(counts, np.float64) / T
    P = np.asarray(p, np.float64).sum(axis=0) / T
    return f, P, E * float(np.sum(f * P))


def route(x, w_router, bias, k: int, renorm: bool):
    """Steps 1-3 on float64 logits.  Returns dict(z, p, idx, w, counts, f, P, aux)."""
    z = router_logits(x, w_router, bias)
    return route_from_logits(z, k, renorm)


def route_from_logits(z, k: int, renorm: bool):
    z = np.asarray(z, np.float64)
    T, E = z.shape
    p = softmax(z)
    idx = topk_select(z, k)
    w = gate_weights(p, idx, renorm)
    counts = expert_counts(idx, E)
    f, P, aux = load_balance(counts, p, T, E)
    return dict(z=z, p=p, idx=idx, w=w, counts=counts, f=f, P=P, aux=aux)


# ---------------------------------------------------------------- hierarchical ("fractal") router
# kieve-moe Features, "Fractal tiling routing": self-similar hierarchical routing over a branch^levels expert tree,
# a cheap router for very large expert pools.  The page names it without the rule; the reading taken here:
# expert e is the leaf whose base-`branch` digits (most significant first) d_0 .. d_{L-1} give the child taken
# at each level; every level l has its own router W_l [branch, d] (and bias), shared by all nodes of the level
# (the same split repeated at every node: the self-similarity); the level probabilities q_l = softmax(x W_l^T)
# multiply along the path, p(e) = prod_l q_l[d_l], a distribution over the E = branch^levels leaves that costs
# levels * branch logits per token instead of E.  Top-k, gates, renormalisation and the load-balance statistic
# then follow the flat router on p (lower expert index first among equal p).

def tree_digits(e, branch: int, levels: int) -> np.ndarray:
    """Base-branch digits of the expert indices e, most significant first: [..., levels]."""
    e = np.asarray(e, np.int64)
    return np.stack([(e // branch ** (levels - 1 - l)) % branch for l in range(levels)], axis=-1)


def route_tree(x, w_tree, bias_tree, branch: int, levels: int, k: int, renorm: bool):
    """Tree routing on float64 level logits.  w_tree [levels * branch, d] stacks W_0 .. W_{L-1}; bias_tree
    [levels * branch] or None.  Returns dict(z, q, p, idx, w, counts, f, P, aux) with z [T, L*B] the level
    logits, q [T, L, B] the level probabilities and p [T, B^L] the leaf probabilities."""
    z = router_logits(x, w_tree, bias_tree)
    T = z.shape[0]
    E = branch ** levels
    q = np.stack([softmax(z[:, l * branch:(l + 1) * branch]) for l in range(levels)], axis=1)
    dig = tree_digits(np.arange(E), branch, levels)                 # [E, L]
    p = np.ones((T, E))
    for l in range(levels):
        p = p * q[:, l, dig[:, l]]
    idx = topk_select(p, k)
    w = gate_weights(p, idx, renorm)
    counts = expert_counts(idx, E)
    f, P, aux = load_balance(counts, p, T, E)
    return dict(z=z, q=q, p=p, idx=idx, w=w, counts=counts, f=f, P=P, aux=aux)


def tree_topk_margin(p, k: int) -> np.ndarray:
    """Relative gap between the k-th and (k+1)-th largest leaf probability of each row (inf when k == E)."""
    p = np.asarray(p, np.float64)
    if k >= p.shape[1]:
        return np.full(p.shape[0], np.inf)
    s = -np.sort(-p, axis=1)
    return (s[:, k - 1] - s[:, k]) / s[:, k - 1]


# ---------------------------------------------------------------- step 4: grouping

def capacity(T: int, k: int, E: int, factor: float) -> int:
    """C = ceil(factor * T * k / E); 0 when no capacity limit is set."""
    if not factor:
        return 0
    from fractions import Fraction
    return int(math.ceil(Fraction(factor).limit_denominator(10**6) * T * k / E))


def permute(idx, E: int, cap: int = 0):
    """Group the (token, slot) assignments by expert.

    Returns dict with
      counts [E]    tokens that chose e;
      kept   [E]    rows of group e actually filled (min(counts, C) with a capacity);
      offsets [E+1] first row of each group (e*C with a capacity, else an exclusive
                    prefix sum of counts) and the row total R at [E];
      rank  [T,k]   position of (t,j) among the tokens that chose idx[t,j], in token order;
      slot_pos [T,k] row of (t,j) in the grouped buffer, -1 if dropped;
      drop  [T,k]   1 where dropped;
      row_src [R]   t*k + j of the assignment in each row, -1 for unfilled rows.
    """
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    flat = idx.ravel()                               # token-major order t*k + j
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    order = np.argsort(flat, kind="stable")          # grouped by expert, token order inside
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]])
    rank_sorted = np.arange(flat.size) - np.repeat(starts, counts)
    rank = np.empty(flat.size, np.int64)
    rank[order] = rank_sorted
    if cap > 0:
        kept = np.minimum(counts, cap)
        offsets = np.arange(E + 1, dtype=np.int64) * cap
        keep = rank < cap
    else:
        kept = counts.copy()
        offsets = np.concatenate([[0], np.cumsum(counts)])
        keep = np.ones(flat.size, bool)
    slot = np.where(keep, offsets[flat] + rank, -1)
    R = int(offsets[E])
    row_src = np.full(R, -1, np.int64)
    row_src[slot[keep]] = np.nonzero(keep)[0]
    return dict(counts=counts, kept=kept, offsets=offsets, rank=rank.reshape(T, k),
                slot_pos=slot.reshape(T, k), drop=(~keep).astype(np.uint8).reshape(T, k),
                row_src=row_src)


def gather_rows(x, row_src, k: int) -> np.ndarray:
    """x_perm[r] = x[row_src[r] // k]; unfilled rows are zero."""
    x = np.asarray(x, np.float64)
    out = np.zeros((row_src.size, x.shape[1]))
    m = row_src >= 0
    out[m] = x[row_src[m] // k]
    return out


# ---------------------------------------------------------------- step 5: expert FFN

def silu(z):
    z = np.asarray(z, np.float64)
    return z / (1.0 + np.exp(-z))


def gelu_erf(z):
    z = np.asarray(z, np.float64)
    return 0.5 * z * (1.0 + _erf(z / math.sqrt(2.0)))


def glu_hidden(x, w13, act: int) -> np.ndarray:
    """h = act(x W1^T) * (x W3^T) with w13 = [W1; W3] stacked as [2H, d]."""
    w13 = np.asarray(w13, np.float64)
    H = w13.shape[0] // 2
    xz = np.asarray(x, np.float64) @ w13.T
    g, u = xz[:, :H], xz[:, H:]
    a = silu(g) if act == ACT_SWIGLU else gelu_erf(g)
    return a * u


def expert_ffn(x, w13, w2, act: int) -> np.ndarray:
    """One expert: y = (act(x W1^T) * (x W3^T)) W2^T, w2 = [d, H]."""
    return glu_hidden(x, w13, act) @ np.asarray(w2, np.float64).T


def grouped_ffn(x_perm, offsets, kept, w13, w2, act: int) -> np.ndarray:
    """Apply expert e to rows [offsets[e], offsets[e] + kept[e]); other rows stay zero."""
    x_perm = np.asarray(x_perm, np.float64)
    y = np.zeros((x_perm.shape[0], np.asarray(w2).shape[1]))
    for e in range(len(kept)):
        n = int(kept[e])
        if n == 0:
            continue
        a = int(offsets[e])
        y[a:a + n] = expert_ffn(x_perm[a:a + n], w13[e], w2[e], act)
    return y


# ---------------------------------------------------------------- step 6: combine

def combine(y_perm, slot_pos, w, y_shared=None) -> np.ndarray:
    """out[t] = sum_j w[t,j] * y_perm[slot_pos[t,j]] over kept slots, plus y_shared[t]."""
    slot_pos = np.asarray(slot_pos, np.int64)
    T, k = slot_pos.shape
    y_perm = np.asarray(y_perm, np.float64)
    out = np.zeros((T, y_perm.shape[1]))
    for j in range(k):
        m = slot_pos[:, j] >= 0
        out[m] += np.asarray(w, np.float64)[m, j, None] * y_perm[slot_pos[m, j]]
    if y_shared is not None:
        out += np.asarray(y_shared, np.float64)
    return out


# ---------------------------------------------------------------- the whole layer

def moe_forward(x, w_router, bias, w13, w2, *, k: int, act: int = ACT_SWIGLU, renorm: bool = True,
                cap: int = 0, w13_sh=None, w2_sh=None, routing=None):
    """Routed layer: route -> group -> expert FFN -> combine (+ shared expert).

    ``routing`` may carry a precomputed ``route()`` result.  Returns a dict with
    ``out`` and every intermediate.
    """
    E = np.asarray(w_router).shape[0] if w_router is not None else len(w13)
    r = routing if routing is not None else route(x, w_router, bias, k, renorm)
    g = permute(r["idx"], E, cap)
    x_perm = gather_rows(x, g["row_src"], k)
    y_perm = grouped_ffn(x_perm, g["offsets"], g["kept"], w13, w2, act)
    y_sh = None
    if w13_sh is not None:
        y_sh = expert_ffn(x, np.asarray(w13_sh)[0], np.asarray(w2_sh)[0], act)
    out = combine(y_perm, g["slot_pos"], r["w"], y_sh)
    res = dict(r)
    res.update(g)
    res.update(x_perm=x_perm, y_perm=y_perm, y_shared=y_sh, out=out)
    return res


# ---------------------------------------------------------------- backward: input and weight gradients
# Training is the setting of p1 (kieve-moe Features: the load-balancing auxiliary loss), p2 (MoEEvolve
# Architecture) and p5 (MoEFFN.forward, "Load balancing loss").  The gradients of
# L = sum(dout * out) + aux_coef * aux follow the forward above by the chain rule.  The routing decision (the
# top-k and the capacity drops) is piecewise constant in x and passes no gradient; the gate values and the
# softmax do.  The count fractions f_e of the statistic are counts, also constant.

def silu_grad(z):
    """d/dz of z sigmoid(z) = sigmoid(z) (1 + z (1 - sigmoid(z)))."""
    z = np.asarray(z, np.float64)
    s = 1.0 / (1.0 + np.exp(-z))
    return s * (1.0 + z * (1.0 - s))


def gelu_erf_grad(z):
    """d/dz of z Phi(z) = Phi(z) + z phi(z), with the standard normal cdf Phi and density phi."""
    z = np.asarray(z, np.float64)
    return 0.5 * (1.0 + _erf(z / math.sqrt(2.0))) + z * np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)


def expert_ffn_backward_x(x, w13, w2, act: int, dy) -> np.ndarray:
    """dL/dx of y = (act(x W1^T) * (x W3^T)) W2^T given dy = dL/dy; x, dy [n, d], w13 [2H, d], w2 [d, H]."""
    x = np.asarray(x, np.float64)
    w13 = np.asarray(w13, np.float64)
    H = w13.shape[0] // 2
    w1, w3 = w13[:H], w13[H:]
    g, u = x @ w1.T, x @ w3.T
    dh = np.asarray(dy, np.float64) @ np.asarray(w2, np.float64)
    a = silu(g) if act == ACT_SWIGLU else gelu_erf(g)
    da = silu_grad(g) if act == ACT_SWIGLU else gelu_erf_grad(g)
    return (dh * u * da) @ w1 + (dh * a) @ w3


def expert_ffn_backward_weights(x, w13, w2, act: int, dy):
    """Weight gradients of y = (act(x W1^T) * (x W3^T)) W2^T given dy = dL/dy, summed over the rows:
    dW2 = dy^T h [d, H] with h = act(g) u; dW1 = (dh u act'(g))^T x and dW3 = (dh act(g))^T x, stacked as
    dW13 [2H, d] like w13.  x, dy [n, d], w13 [2H, d], w2 [d, H]."""
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    w13 = np.asarray(w13, np.float64)
    H = w13.shape[0] // 2
    g, u = x @ w13[:H].T, x @ w13[H:].T
    a = silu(g) if act == ACT_SWIGLU else gelu_erf(g)
    da = silu_grad(g) if act == ACT_SWIGLU else gelu_erf_grad(g)
    dh = dy @ np.asarray(w2, np.float64)
    dw2 = dy.T @ (a * u)
    dw13 = np.concatenate([(dh * u * da).T @ x, (dh * a).T @ x], axis=0)
    return dw13, dw2


def moe_backward(x, w_router, bias, w13, w2, dout, *, k: int, act: int = ACT_SWIGLU, renorm: bool = True,
                 cap: int = 0, w13_sh=None, w2_sh=None, aux_coef: float = 0.0):
    """Gradients of L = sum(dout * out) + aux_coef * aux for the layer of moe_forward: dx [T, d] and the
    weight gradients dw13 [E, 2H, d], dw2 [E, d, H], dw13_sh [1, 2H_s, d], dw2_sh [1, d, H_s] (None without a
    shared expert) and dw_router [E, d].  The exploration bias added to the logits is taken as a constant.

    Parts of dx: the routed experts (each kept slot: w_tj times the expert's input gradient of dout_t), the
    shared expert, and the router: dw_tj = <dout_t, y_{e_tj}(x_t)> on kept slots -> the gate derivative
    (renorm: w_j = p_j / S) -> dp on the selected experts, plus aux_coef E f_e / T on every expert
    (P_e = mean_t p) -> through the softmax, dz = p (dp - <p, dp>) -> dz W_r.  Each expert's weight gradient
    sums its kept rows with dy = w_tj dout_t; dW_r = dz^T x.  Returns a dict with these and the intermediates.
    """
    x = np.asarray(x, np.float64)
    dout = np.asarray(dout, np.float64)
    fw = moe_forward(x, w_router, bias, w13, w2, k=k, act=act, renorm=renorm, cap=cap, w13_sh=w13_sh,
                     w2_sh=w2_sh)
    T = x.shape[0]
    E = np.asarray(w_router).shape[0]
    idx, w, p, slot = fw["idx"], fw["w"], fw["p"], fw["slot_pos"]
    dx = np.zeros_like(x)
    dw = np.zeros((T, k))
    dw13 = np.zeros(np.shape(w13), np.float64)
    dw2 = np.zeros(np.shape(w2), np.float64)
    for e in range(E):
        tj = np.argwhere((idx == e) & (slot >= 0))
        if tj.size == 0:
            continue
        t, j = tj[:, 0], tj[:, 1]
        dy_e = w[t, j, None] * dout[t]
        dx_e = expert_ffn_backward_x(x[t], np.asarray(w13[e]), np.asarray(w2[e]), act, dy_e)
        np.add.at(dx, t, dx_e)
        dw13[e], dw2[e] = expert_ffn_backward_weights(x[t], w13[e], w2[e], act, dy_e)
        dw[t, j] = np.sum(dout[t] * fw["y_perm"][slot[t, j]], axis=1)
    dw13_sh = dw2_sh = None
    if w13_sh is not None:
        dx += expert_ffn_backward_x(x, np.asarray(w13_sh)[0], np.asarray(w2_sh)[0], act, dout)
        g13, g2 = expert_ffn_backward_weights(x, np.asarray(w13_sh)[0], np.asarray(w2_sh)[0], act, dout)
        dw13_sh, dw2_sh = g13[None], g2[None]
    psel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    if renorm:
        S = psel.sum(axis=1, keepdims=True)
        dpsel = (dw - np.sum(dw * w, axis=1, keepdims=True)) / S
    else:
        dpsel = dw
    dp = np.zeros((T, E))
    np.add.at(dp, (np.repeat(np.arange(T), k), idx.astype(np.int64).ravel()), dpsel.ravel())
    if aux_coef:
        f = fw["counts"] / T
        dp += aux_coef * E * f[None, :] / T
    dz = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
    dx += dz @ np.asarray(w_router, np.float64)
    return dict(dx=dx, dw13=dw13, dw2=dw2, dw13_sh=dw13_sh, dw2_sh=dw2_sh, dw_router=dz.T @ x, dw=dw, dz=dz,
                forward=fw)


def dense_moe_forward(x, w13, w2, idx, w, drop=None, *, act: int = ACT_SWIGLU, w13_sh=None, w2_sh=None):
    """Dense evaluation: every expert on every token, mixed by the masked gate matrix.

    G[t,e] = w[t,j] where idx[t,j] = e and (t,j) is kept, else 0;
    out = sum_e G[:,e] * FFN_e(x) (+ shared).  Equal to the routed layer by
    construction of the grouping (kieve-moe "Tests": dense <-> parallel MoE
    equivalence).
    """
    x = np.asarray(x, np.float64)
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    E = len(w13)
    G = np.zeros((T, E))
    for j in range(k):
        keep = np.ones(T, bool) if drop is None else (np.asarray(drop)[:, j] == 0)
        G[np.arange(T)[keep], idx[keep, j]] += np.asarray(w, np.float64)[keep, j]
    out = np.zeros((T, np.asarray(w2).shape[1]))
    for e in range(E):
        if np.any(G[:, e] != 0):
            out += G[:, e:e + 1] * expert_ffn(x, w13[e], w2[e], act)
    if w13_sh is not None:
        out += expert_ffn(x, np.asarray(w13_sh)[0], np.asarray(w2_sh)[0], act)
    return out


# ---------------------------------------------------------------- step 7: INT4 weights

def quantize_int4_g128(w):
    """Symmetric signed INT4 with one bf16 scale per 128 inputs.

    w [..., N, K] (float32 values, K % 128 == 0) -> (q int8 [..., N, K] in
    [-8, 7], s float32 [..., N, K/128] holding bf16 values).  Decisions in fp32:
    s = bf16(max|w_g| / 7), q = clamp(rint(w / s), -8, 7), q = 0 where s == 0.
    """
    w = np.asarray(w, np.float32)
    *lead, N, K = w.shape
    assert K % GROUP == 0
    wg = w.reshape(*lead, N, K // GROUP, GROUP)
    amax = np.abs(wg).max(axis=-1)
    s = bf16_round(amax / np.float32(7.0))
    safe = np.where(s == 0, np.float32(1.0), s).astype(np.float32)
    q = np.rint(wg / safe[..., None])
    q = np.where(s[..., None] == 0, 0.0, q)
    q = np.clip(q, -8, 7).astype(np.int8)
    return q.reshape(*lead, N, K), s.astype(np.float32)


def pack_int4(q) -> np.ndarray:
    """Two signed nibbles per byte: input index 2i in the low nibble, 2i+1 in the high one."""
    q = np.asarray(q, np.int8)
    lo = (q[..., 0::2].astype(np.int16) & 0xF)
    hi = (q[..., 1::2].astype(np.int16) & 0xF)
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(packed) -> np.ndarray:
    b = np.asarray(packed, np.uint8).astype(np.int16)
    lo = b & 0xF
    hi = (b >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def dequantize_int4_g128(packed, scales) -> np.ndarray:
    """Exact float64 weights q * s from packed nibbles [..., N, K/2] and scales [..., N, K/128]."""
    q = unpack_int4(packed).astype(np.float64)
    *lead, N, K = q.shape
    s = np.asarray(scales, np.float64)
    return (q.reshape(*lead, N, K // GROUP, GROUP) * s[..., None]).reshape(*lead, N, K)
