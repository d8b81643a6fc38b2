"""Workload shapes and seeded input generators.

Shapes follow the five workloads of the routed-MoE study this library is
measured on:

* ``tiny``      T=256, d=64, E=8, top-2, SwiGLU hidden 128.
* ``small``     T=4096 (batch 4 x seq 1024), d=256, E=8, top-2, SwiGLU hidden
                1024, renormalised gates, load-balance statistic returned
                (the MoE-Stream ``MoEStreamConfig`` defaults: n_embd 256,
                8 experts, top-2, hidden 4 x n_embd).
* ``granular``  T=32768 (batch 64 x seq 512), d=768, 192 experts SwiGLU hidden
                256, top-4, one shared expert hidden 512, capacity factor 1.25
                (the MoEEvolve README, "Architecture": 192 granular experts,
                top-4, one coarse shared expert of hidden 512, capacity-factor
                static-shape dispatch).
* ``skewed``    granular shapes, router logits offset by a per-expert bias so
                popularity is Zipf-like, no capacity limit.
* ``geglu``     T=8192, d=768, E=32, top-2, GeGLU hidden 4096 (kieve-moe,
                "Features": top-k GeGLU MoE, I=4096, E=32), same bias.
* ``decode_int4`` T=64, d=7168, E=384, top-8, one shared expert, SwiGLU hidden
                2048, experts stored as signed INT4 with one bf16 scale per 128
                inputs (ExpertMesh README: group-scaled signed INT4 routed
                experts in an [expert, output, packed_input] layout).

Distributions: x ~ N(0,1) rounded to bf16; router weight ~ N(0, 1/d) in fp32;
expert weights ~ N(0, 1/fan_in) rounded to bf16 (fan_in = d for the gate/up
matrix, H for the down matrix).  INT4 workloads draw the expert weights in
fp32 one expert at a time; quantising them is the library's (and the
oracle's) job, not this module's.

Every tensor comes from its own ``torch.Generator`` seeded with
``seed * 10**6 + stream`` so one expert can be regenerated alone.  CPU and CUDA
generators give different numbers: a test draws on one device and copies.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch

ACT_SWIGLU = 0
ACT_GEGLU = 1
WFMT_BF16 = 0
WFMT_INT4_G128 = 1

_STREAM_X = 1
_STREAM_ROUTER = 2
_STREAM_TOPK = 3
_STREAM_LOGITS = 4
_STREAM_TREE = 5
_STREAM_EXPERT0 = 1000        # expert e uses 1000 + e; the shared expert uses 1000 + E


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    H: int
    H_s: int = 0                 # shared expert hidden (0 = none)
    capacity_factor: float = 0.0 # 0 = unbounded groups
    act: int = ACT_SWIGLU
    wfmt: int = WFMT_BF16
    renorm: int = 1
    skew: float = 0.0            # bias_e = -skew * ln(e + 1) added to the logits
    aux: bool = False            # load-balance statistic requested
    description: str = ""

    def replace(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)

    @property
    def has_bias(self) -> bool:
        return self.skew != 0.0

    def flops_tc(self, kept: int | None = None) -> float:
        """Algorithmic expert flops: 6*d*H per kept (token, slot) plus 6*d*H_s per token."""
        kept = self.T * self.k if kept is None else kept
        return 6.0 * self.d * self.H * kept + 6.0 * self.d * self.H_s * self.T

    def flops_router(self) -> float:
        return 2.0 * self.T * self.d * self.E


WORKLOADS = {
    "tiny": Workload("tiny", T=256, d=64, E=8, k=2, H=128,
                     description="tiny routed MoE layer, T=256 d=64 E=8 top-2 SwiGLU H=128"),
    "small": Workload("small", T=4096, d=256, E=8, k=2, H=1024, aux=True,
                      description="small dense-token MoE FFN, T=4096 d=256 E=8 top-2 SwiGLU H=1024 + aux"),
    "granular": Workload("granular", T=32768, d=768, E=192, k=4, H=256, H_s=512, capacity_factor=1.25,
                         description="granular experts, T=32768 d=768 E=192 top-4 H=256 + shared 512, cf 1.25"),
    "skewed": Workload("skewed", T=32768, d=768, E=192, k=4, H=256, H_s=512, skew=1.2,
                       description="Zipf-skewed routing, granular shapes, no capacity"),
    "geglu": Workload("geglu", T=8192, d=768, E=32, k=2, H=4096, act=ACT_GEGLU, skew=1.2,
                      description="GeGLU variant, T=8192 d=768 E=32 top-2 H=4096, skew bias"),
    "decode_int4": Workload("decode_int4", T=64, d=7168, E=384, k=8, H=2048, H_s=2048,
                            wfmt=WFMT_INT4_G128, renorm=0,
                            description="INT4 decode, T=64 d=7168 E=384 top-8 H=2048 + shared 2048, g128 bf16 scales"),
}


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 10**6 + stream)
    return g


def expert_weights_f32(wl: Workload, seed: int, e: int, device="cpu", hidden: int | None = None):
    """fp32 draws of one expert: (w13 [2H, d], w2 [d, H]) with std 1/sqrt(fan_in).

    ``e == wl.E`` is the shared expert (hidden H_s unless ``hidden`` is given).
    """
    H = hidden if hidden is not None else (wl.H_s if e == wl.E else wl.H)
    g = _gen(seed, _STREAM_EXPERT0 + e, device)
    w13 = torch.randn(2 * H, wl.d, generator=g, device=device, dtype=torch.float32) / math.sqrt(wl.d)
    w2 = torch.randn(wl.d, H, generator=g, device=device, dtype=torch.float32) / math.sqrt(H)
    return w13, w2


def make_inputs(wl: Workload, seed: int = 0, device="cpu", with_expert_weights: bool = True):
    """Draw the layer inputs.

    Returns a dict: ``x`` [T,d] bf16, ``w_router`` [E,d] fp32, ``bias`` [E] fp32
    or None, and for bf16 workloads ``w13`` [E,2H,d], ``w2`` [E,d,H] bf16 plus,
    when H_s > 0, ``w13_sh`` [1,2H_s,d] and ``w2_sh`` [1,d,H_s] bf16.  INT4
    workloads get no expert tensors here: call :func:`expert_weights_f32` per
    expert.
    """
    out = {}
    g = _gen(seed, _STREAM_X, device)
    out["x"] = torch.randn(wl.T, wl.d, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    g = _gen(seed, _STREAM_ROUTER, device)
    out["w_router"] = torch.randn(wl.E, wl.d, generator=g, device=device, dtype=torch.float32) / math.sqrt(wl.d)
    if wl.skew != 0.0:
        e = torch.arange(wl.E, device=device, dtype=torch.float64)
        out["bias"] = (-wl.skew * torch.log(e + 1.0)).to(torch.float32)
    else:
        out["bias"] = None
    if with_expert_weights and wl.wfmt == WFMT_BF16:
        w13 = torch.empty(wl.E, 2 * wl.H, wl.d, device=device, dtype=torch.bfloat16)
        w2 = torch.empty(wl.E, wl.d, wl.H, device=device, dtype=torch.bfloat16)
        for e in range(wl.E):
            a, b = expert_weights_f32(wl, seed, e, device)
            w13[e].copy_(a)
            w2[e].copy_(b)
        out["w13"], out["w2"] = w13, w2
        if wl.H_s > 0:
            a, b = expert_weights_f32(wl, seed, wl.E, device)
            out["w13_sh"] = a.to(torch.bfloat16).unsqueeze(0).contiguous()
            out["w2_sh"] = b.to(torch.bfloat16).unsqueeze(0).contiguous()
    return out


def draw_tree_router(T: int, d: int, branch: int, levels: int, seed: int = 0, device="cpu"):
    """Inputs of a hierarchical router over branch**levels experts: ``x`` [T, d] bf16 (the same draw as
    :func:`make_inputs` for these T, d and seed) and ``w_tree`` [levels * branch, d] fp32 with std 1/sqrt(d),
    so that every level's logits are about unit normal."""
    g = _gen(seed, _STREAM_X, device)
    x = torch.randn(T, d, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    g = _gen(seed, _STREAM_TREE, device)
    w = torch.randn(levels * branch, d, generator=g, device=device, dtype=torch.float32) / math.sqrt(d)
    return dict(x=x, w_tree=w)


def draw_topk_idx(T: int, E: int, k: int, seed: int = 0, skew: float = 0.0, device="cpu") -> torch.Tensor:
    """Random routing [T,k] int32: k distinct experts per token.

    With ``skew > 0`` expert e is drawn with weight (e+1)^-skew (Zipf-like).
    """
    g = _gen(seed, _STREAM_TOPK, device)
    wts = torch.ones(E, dtype=torch.float64, device=device)
    if skew:
        wts = (torch.arange(E, dtype=torch.float64, device=device) + 1.0) ** (-skew)
    probs = wts.expand(T, E).contiguous()
    idx = torch.multinomial(probs, k, replacement=False, generator=g)
    return idx.to(torch.int32)


def draw_logits(T: int, E: int, seed: int = 0, mode: str = "normal", device="cpu") -> torch.Tensor:
    """Random fp32 router logits [T,E].

    ``normal``: N(0,1).  ``coarse``: multiples of 0.25 in [-1, 1), so ties are
    frequent.  ``signed_zero``: coarse values with every zero given a random
    sign bit, to exercise +0.0 / -0.0 ties.  ``equal``: all logits equal.
    """
    g = _gen(seed, _STREAM_LOGITS, device)
    if mode == "normal":
        return torch.randn(T, E, generator=g, device=device, dtype=torch.float32)
    if mode in ("coarse", "signed_zero"):
        z = torch.randint(-4, 4, (T, E), generator=g, device=device).to(torch.float32) * 0.25
        if mode == "signed_zero":
            sign = torch.randint(0, 2, (T, E), generator=g, device=device).bool()
            z = torch.where((z == 0) & sign, torch.full_like(z, -0.0), z)
        return z
    if mode == "equal":
        return torch.full((T, E), 0.5, device=device, dtype=torch.float32)
    raise ValueError(mode)


def draw_groups(n_groups: int, max_rows: int, seed: int = 0, cap: int = 0, device="cpu"):
    """Random group table for grouped-FFN tests: (start [G] int32, rows [G] int32, R).

    Sizes are drawn in [0, max_rows] with some empty groups and some larger
    than one 128-row tile.  ``cap > 0`` lays groups out as fixed slabs of
    ``cap`` rows (sizes clipped to cap), else back to back.
    """
    g = _gen(seed, 5, "cpu")
    rows = torch.randint(0, max_rows + 1, (n_groups,), generator=g)
    if n_groups >= 4:
        rows[torch.randint(0, n_groups, (n_groups // 4,), generator=g)] = 0
    rows[0] = max(int(rows[0]), 1)
    if cap > 0:
        rows = rows.clamp(max=cap)
        start = torch.arange(n_groups) * cap
        R = n_groups * cap
    else:
        start = torch.cumsum(rows, 0) - rows
        R = int(rows.sum())
    return start.to(torch.int32).to(device), rows.to(torch.int32).to(device), R
