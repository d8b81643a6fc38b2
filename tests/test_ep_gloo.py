"""Expert-parallel orchestration (``sparse_mixture_experts_expert_b200.ep``) on two gloo ranks on CPU.

The per-rank steps (route, grouping, expert FFN, combine) run on the float64 oracle, the exchanges on
torch.distributed all-to-all; every rank's output must equal the single-process oracle layer on its tokens.
Cases: a balanced routing, an odd token split with three experts per rank and a skew, and a routing that sends
every row to rank 0's experts (rank 1 receives nothing).  With a capacity C (static shapes: equal all-to-all
splits, padding rows included) every rank's output must equal the oracle layer with capacity C on its own
tokens, drops included.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class OracleOps:
    """The per-rank steps of moe_forward_ep on the float64 oracle (CPU tensors)."""

    def __init__(self, O, torch):
        self.O, self.torch = O, torch

    def route(self, shape, x, w_router, bias):
        r = self.O.route(x.numpy(), w_router.numpy(), None if bias is None else bias.numpy(), shape.k,
                         bool(shape.renorm))
        return self.torch.from_numpy(r["idx"].astype(np.int32)), self.torch.from_numpy(r["w"])

    def permute(self, shape, x, topk_idx):
        p = self.O.permute(topk_idx.numpy(), shape.E, shape.capacity)
        rs = p["row_src"]
        x_perm = np.zeros((shape.R, shape.d))
        x_perm[rs >= 0] = x.numpy()[rs[rs >= 0] // shape.k]
        t = lambda a: self.torch.from_numpy(np.ascontiguousarray(a).astype(np.int32))
        return dict(x_perm=self.torch.from_numpy(x_perm), slot_pos=t(p["slot_pos"]), counts=t(p["counts"]),
                    kept=t(p["kept"]), offsets=t(p["offsets"]))

    def expert_ffn(self, shape, xg, w13, w2, hidden, group_start=None, group_rows=None, s13=None, s2=None, y=None):
        xg = xg.numpy()
        yy = np.zeros((xg.shape[0], shape.d))
        groups = [(0, xg.shape[0])] if group_start is None else zip(group_start.tolist(), group_rows.tolist())
        for g, (a, n) in enumerate(groups):
            if n:
                yy[a:a + n] = self.O.expert_ffn(xg[a:a + n], w13[g].numpy(), w2[g].numpy(), shape.act)
        if y is not None:   # the caller's rows (a view of a larger buffer)
            y.copy_(self.torch.from_numpy(yy))
            return y
        return self.torch.from_numpy(yy)

    def combine(self, shape, y_perm, slot_pos, w, y_shared=None):
        return self.torch.from_numpy(self.O.combine(y_perm.numpy(), slot_pos.numpy(), w.numpy(),
                                                    None if y_shared is None else y_shared.numpy()))


def _problem(case):
    T, d, E, k, H, H_s, mode = case
    rng = np.random.default_rng(11)
    x = rng.standard_normal((T, d))
    w_r = rng.standard_normal((E, d)) * 0.3
    bias = np.zeros(E)
    if mode == "skew":
        bias = -0.5 * np.log1p(np.arange(E))
    elif mode == "rank0":
        bias[: E // 2] = 50.0   # every token's k picks are rank 0's experts
    w13 = rng.standard_normal((E, 2 * H, d)) * d ** -0.5
    w2 = rng.standard_normal((E, d, H)) * H ** -0.5
    w13_sh = rng.standard_normal((1, 2 * H_s, d)) * d ** -0.5 if H_s else None
    w2_sh = rng.standard_normal((1, d, H_s)) * H_s ** -0.5 if H_s else None
    return x, w_r, bias, w13, w2, w13_sh, w2_sh


def _reference(case):
    """The single-process oracle layer on all tokens."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    T, d, E, k, H, H_s, mode = case
    x, w_r, bias, w13, w2, w13_sh, w2_sh = _problem(case)
    r = O.route(x, w_r, bias, k, True)
    out = np.zeros((T, d))
    for t in range(T):
        for j in range(k):
            e = int(r["idx"][t, j])
            out[t] += r["w"][t, j] * O.expert_ffn(x[t:t + 1], w13[e], w2[e], 0)[0]
    if H_s:
        out += O.expert_ffn(x, w13_sh[0], w2_sh[0], 0)
    return out, r["idx"]


def _worker(rank, world, port, case, q, cap=0):
    import sys
    from datetime import timedelta

    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle as O
    import sparse_mixture_experts_expert_b200 as moe
    from sparse_mixture_experts_expert_b200.ep import moe_forward_ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        T, d, E, k, H, H_s, mode = case
        x, w_r, bias, w13, w2, w13_sh, w2_sh = _problem(case)
        toks = np.arange(rank, T, world)             # an interleaved token split (odd T: uneven shares)
        E_loc = E // world
        mine = slice(rank * E_loc, (rank + 1) * E_loc)
        f = torch.from_numpy
        shape = moe.MoeShape(T=len(toks), d=d, E=E, k=k, H=H, H_s=H_s, capacity=cap, act=0, wfmt=0, renorm=1)
        out, idx, _ = moe_forward_ep(shape, f(x[toks].copy()), f(w_r), f(w13[mine].copy()), f(w2[mine].copy()),
                                     bias=f(bias), w13_sh=None if w13_sh is None else f(w13_sh),
                                     w2_sh=None if w2_sh is None else f(w2_sh), ops=OracleOps(O, torch))
        q.put((rank, toks, out.numpy(), idx.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [(40, 32, 8, 2, 32, 16, "plain"), (33, 32, 6, 3, 16, 0, "skew"),
                                  (24, 16, 8, 2, 16, 16, "rank0")])
def test_expert_parallel_two_ranks_matches_the_single_process_layer(case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    ref, ref_idx = _reference(case)
    for rank, toks, out, idx in got:
        assert (idx == ref_idx[toks]).all()
        np.testing.assert_allclose(out, ref[toks], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("case,cap", [((40, 32, 8, 2, 32, 16, "skew"), 6), ((33, 32, 6, 3, 16, 0, "skew"), 4),
                                      ((24, 16, 8, 2, 16, 16, "rank0"), 3)])
def test_expert_parallel_static_capacity_matches_the_per_rank_layer(case, cap):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, case, q, cap)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    T, d, E, k, H, H_s, mode = case
    x, w_r, bias, w13, w2, w13_sh, w2_sh = _problem(case)
    dropped = 0
    for rank, toks, out, idx in got:
        ref = O.moe_forward(x[toks], w_r, bias, w13, w2, k=k, act=0, renorm=True, cap=cap, w13_sh=w13_sh,
                            w2_sh=w2_sh)
        dropped += int(ref["drop"].sum())
        assert (idx == ref["idx"]).all()
        np.testing.assert_allclose(out, ref["out"], rtol=1e-10, atol=1e-12)
    assert dropped > 0   # the capacity binds somewhere


@pytest.mark.parametrize("cap", [0, 4])
def test_expert_parallel_four_ranks(cap):
    # four ranks of two experts each, an uneven token split (37 tokens), with and without a capacity
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle as O
    case = (37, 16, 8, 2, 16, 16, "skew")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 4, port, case, q, cap)) for r in range(4)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in range(4)]
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    T, d, E, k, H, H_s, mode = case
    x, w_r, bias, w13, w2, w13_sh, w2_sh = _problem(case)
    for rank, toks, out, idx in got:
        ref = O.moe_forward(x[toks], w_r, bias, w13, w2, k=k, act=0, renorm=True, cap=cap, w13_sh=w13_sh,
                            w2_sh=w2_sh)
        assert (idx == ref["idx"]).all()
        np.testing.assert_allclose(out, ref["out"], rtol=1e-10, atol=1e-12)
