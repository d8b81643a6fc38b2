"""Expert-parallel forward: every rank of a process group holds E / G of the routed experts and its own tokens.

kieve-moe *Features* (tokens routed to the rank that owns their selected experts), the Kvasir wiki's
*Backbone × worker* (each worker owns a slice of the experts) and the ExpertMesh README's feature list
("activation grouping that preserves token and top-k slot identity") describe this layout.

Per rank r of G ranks, owning experts [r * E_loc, (r + 1) * E_loc) with E_loc = E / G:

1. route the local tokens over all E experts (``moe_route``, the full W_r on every rank);
2. group the (token, slot) pairs by global expert (``moe_permute``, no capacity), so that the rows bound for
   rank q are the contiguous groups of q's experts;
3. exchange the per-expert row counts (``all_to_all``), then the rows (``all_to_all`` with the counts as
   splits);
4. run the local experts on the received rows where they lie: each source's rows are its groups of this
   rank's experts in expert order, so ``moe_expert_ffn`` takes each source's block as E_loc groups (sizes from
   the exchanged counts) and writes the outputs in place;
5. send the outputs back (``all_to_all``);
6. the weighted top-k reduction in token order plus the shared expert on the local tokens (``moe_combine``).

Each (token, slot) row gets the expert output the single-GPU forward gives it, and the reduction runs in the
same slot order, so with bf16 experts the output equals ``moe_forward`` on the rank's tokens bit for bit.

The row counts reach the host as the splits of the exchanges: one device synchronisation per forward.

With a capacity (``shape.capacity = C > 0``, the same C on every rank: the MoEEvolve README's capacity-factor
dispatch with static shapes) the exchange has static shapes instead.  Each rank groups its own tokens with
capacity C (ranks counted in its token order, as ``moe_forward`` with capacity C on those tokens), so the rows for
rank q are always E_loc * C rows, kept ones first in each expert's C-row block.  Both exchanges then use equal
splits, the kept counts travel as a small device tensor, and the local experts run on each source's blocks where
they lie (groups at e * C), so nothing reaches the host and the whole forward can be captured in a CUDA graph.
The price is the padding rows crossing the exchange; the experts skip them.  Output: ``moe_forward`` with
capacity C on the rank's tokens.

The exchanges are NCCL all-to-all calls (``torch.distributed``), not fused with the expert GEMMs.
"""

from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import MoeShape, moe_combine, moe_expert_ffn, moe_permute, moe_route


class KernelOps:
    """The per-rank steps on this library's kernels (device tensors)."""

    def route(self, shape, x, w_router, bias):
        r = moe_route(shape, x, w_router, bias)
        return r["topk_idx"], r["topk_w"]

    def permute(self, shape, x, topk_idx):
        p = moe_permute(shape, x, topk_idx)
        return dict(x_perm=p["x_perm"], slot_pos=p["slot_pos"], counts=p["counts"], kept=p["kept"],
                    offsets=p["offsets"])

    def expert_ffn(self, shape, x_grouped, w13, w2, hidden, group_start=None, group_rows=None, s13=None, s2=None,
                   y=None):
        _, y = moe_expert_ffn(shape, x_grouped, w13, w2, hidden=hidden, group_start=group_start,
                              group_rows=group_rows, s13=s13, s2=s2, y=y)
        return y

    def combine(self, shape, y_perm, slot_pos, topk_w, y_shared=None):
        return moe_combine(shape, y_perm, slot_pos, topk_w, y_shared)


def _shape(like: MoeShape, T: int, E: int, k: int, H_s: int) -> MoeShape:
    return MoeShape(T=T, d=like.d, E=E, k=k, H=like.H, H_s=H_s, capacity=0, act=like.act, wfmt=like.wfmt,
                    renorm=like.renorm, flags=like.flags)


def moe_forward_ep(shape: MoeShape, x, w_router, w13_local, w2_local, *, bias=None, s13_local=None,
                   s2_local=None, w13_sh=None, s13_sh=None, w2_sh=None, s2_sh=None, group=None, ops=None):
    """Expert-parallel layer forward on this rank's tokens.

    shape       the layer (E = all routed experts across the group; T = this rank's tokens; capacity 0 for
                the exchange of exact counts, or C > 0, the same on every rank, for static shapes)
    x           [T, d] this rank's tokens
    w_router    [E, d] fp32, the same on every rank
    w13_local, w2_local (s13_local, s2_local)   this rank's E / G experts, layout as for moe_forward
    w13_sh ...  the shared expert (every rank holds it), or None when shape.H_s == 0
    Returns out [T, d] and the routing (topk_idx, topk_w).
    """
    ops = ops if ops is not None else KernelOps()
    G = dist.get_world_size(group)
    E, k, T, d = shape.E, shape.k, shape.T, shape.d
    if E % G != 0 or w13_local.shape[0] != E // G:
        raise ValueError(f"moe_forward_ep: {E} experts do not split into {G} ranks of {w13_local.shape[0]}")
    E_loc = E // G
    if shape.capacity > 0:
        return _forward_ep_static(shape, x, w_router, w13_local, w2_local, bias, s13_local, s2_local, w13_sh,
                                  s13_sh, w2_sh, s2_sh, group, ops, G, E_loc)
    s_route = _shape(shape, T, E, k, 0)

    # 1-2. route over all experts, group the (token, slot) pairs by global expert
    topk_idx, topk_w = ops.route(s_route, x, w_router, bias)
    p = ops.permute(s_route, x, topk_idx)
    x_perm = p["x_perm"]                                 # [T k, d]: rank-major, then expert, then token order

    # 3. per-expert counts to the owners, then the rows
    cnt_send = p["counts"].to(torch.int32)
    cnt_recv = torch.empty_like(cnt_send)                # [G, E_loc]: rows from rank q for local expert e
    dist.all_to_all_single(cnt_recv, cnt_send, group=group)
    cs = cnt_send.cpu().numpy().reshape(G, E_loc)
    cr = cnt_recv.cpu().numpy().reshape(G, E_loc)
    send_split = [int(v) for v in cs.sum(1)]
    recv_split = [int(v) for v in cr.sum(1)]
    n_recv = int(sum(recv_split))
    x_recv = x_perm.new_empty((n_recv, d))
    dist.all_to_all_single(x_recv, x_perm, output_split_sizes=recv_split, input_split_sizes=send_split,
                           group=group)

    # 4-5. the local experts on the received rows where they lie: source q's rows are its groups of my experts in
    # expert order (counts cr[q]), so each source's block runs as E_loc groups, outputs written in place
    y_recv = x_perm.new_empty((n_recv, d))
    base = 0
    for q in range(G):
        nq = int(cr[q].sum())
        if nq > 0:
            starts = np.concatenate([[0], np.cumsum(cr[q])[:-1]]).astype(np.int32)
            dev = topk_idx.device
            s_blk = _shape(shape, nq, E_loc, 1, 0)
            ops.expert_ffn(s_blk, x_recv[base:base + nq], w13_local, w2_local, shape.H,
                           group_start=torch.from_numpy(starts).to(dev),
                           group_rows=torch.from_numpy(cr[q].astype(np.int32)).to(dev), s13=s13_local, s2=s2_local,
                           y=y_recv[base:base + nq])
        base += nq
    y_back = x_perm.new_empty((T * k, d))
    dist.all_to_all_single(y_back, y_recv, output_split_sizes=send_split, input_split_sizes=recv_split,
                           group=group)

    # 6. shared expert on the local tokens, weighted top-k reduction in slot order
    y_sh = None
    if shape.H_s > 0:   # one dense group of the T local tokens
        y_sh = ops.expert_ffn(s_route, x, w13_sh, w2_sh, shape.H_s, s13=s13_sh, s2=s2_sh)
    out = ops.combine(s_route, y_back, p["slot_pos"], topk_w, y_sh)
    return out, topk_idx, topk_w


def _forward_ep_static(shape, x, w_router, w13_local, w2_local, bias, s13_local, s2_local, w13_sh, s13_sh, w2_sh,
                       s2_sh, group, ops, G, E_loc):
    """moe_forward_ep with capacity C: equal all-to-all splits, no host synchronisation.

    Source rank q's rows arrive as its E_loc blocks of C rows, kept rows first, one block per local expert, so the
    local experts run on each source's blocks where they lie (groups at e C with the exchanged kept counts) and
    write their outputs in place: no regrouping, no restoring copy, and the padding rows are skipped.
    """
    E, k, T, d, C = shape.E, shape.k, shape.T, shape.d, shape.capacity
    s_route = MoeShape(T=T, d=d, E=E, k=k, H=shape.H, H_s=0, capacity=C, act=shape.act, wfmt=shape.wfmt,
                       renorm=shape.renorm, flags=shape.flags)
    topk_idx, topk_w = ops.route(s_route, x, w_router, bias)
    p = ops.permute(s_route, x, topk_idx)
    x_perm = p["x_perm"]                       # [E C, d]: expert e's block at rows [e C, (e + 1) C), kept rows first
    kept = p["kept"][:E].to(torch.int32).contiguous()
    kept_recv = torch.empty_like(kept)         # [G][E_loc]: kept rows of my experts from each source rank
    dist.all_to_all_single(kept_recv, kept, group=group)
    x_recv = x_perm.new_empty((E * C, d))      # [G][E_loc][C]
    dist.all_to_all_single(x_recv, x_perm, group=group)
    y_recv = x_perm.new_empty((E * C, d))
    starts = torch.arange(E_loc, dtype=torch.int32, device=kept.device) * C
    s_blk = _shape(shape, E_loc * C, E_loc, 1, 0)
    for q in range(G):
        blk = slice(q * E_loc * C, (q + 1) * E_loc * C)
        ops.expert_ffn(s_blk, x_recv[blk], w13_local, w2_local, shape.H, group_start=starts,
                       group_rows=kept_recv[q * E_loc:(q + 1) * E_loc], s13=s13_local, s2=s2_local, y=y_recv[blk])
    y_back = torch.empty_like(y_recv)
    dist.all_to_all_single(y_back, y_recv, group=group)
    y_sh = None
    if shape.H_s > 0:
        y_sh = ops.expert_ffn(_shape(shape, T, E, k, 0), x, w13_sh, w2_sh, shape.H_s, s13=s13_sh, s2=s2_sh)
    out = ops.combine(s_route, y_back, p["slot_pos"], topk_w, y_sh)
    return out, topk_idx, topk_w
