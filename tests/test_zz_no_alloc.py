"""The allocation-free grouping entry point against the workspace one.

``moe_permute_noalloc`` serves callers that cannot allocate device scratch
(for example code running where the device allocator is owned by someone else
or must not be called): it keeps its scratch in a fixed array inside the
library instead of a caller workspace.  Its results must be identical to
``moe_permute`` -- bit for bit, grouping is integer work -- on consecutive
calls that reuse the same scratch, and it must reject shapes whose scratch
would not fit.  This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _shape(moe, T, E, k, d, cap):
    return moe.MoeShape(T=T, d=d, E=E, k=k, H=16, capacity=cap)


def _case(T, E, k, d, cap, skew, seed):
    idx = synth.draw_topk_idx(T, E, k, seed=seed, skew=skew)
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    return x.to(DEV), idx.to(DEV)


def _same(a, b):
    for key in ("slot_pos", "drop_mask", "counts", "kept", "offsets", "row_src"):
        assert torch.equal(a[key], b[key]), key
    assert torch.equal(a["x_perm"].view(torch.int16), b["x_perm"].view(torch.int16))


def _same_as_oracle(got, idx, E, k, cap, x):
    ref = O.permute(idx.cpu().numpy(), E, cap)
    for key in ("slot_pos", "kept", "offsets", "row_src"):
        assert (got[key].cpu().numpy() == ref[key]).all(), key
    assert (got["drop_mask"].cpu().numpy() == ref["drop"]).all()
    if got.get("counts") is not None:
        assert (got["counts"].cpu().numpy() == ref["counts"]).all()
    rs = ref["row_src"]
    filled = rs >= 0
    xp = got["x_perm"].view(torch.int16).cpu().numpy()
    assert (xp[filled] == x.view(torch.int16).cpu().numpy()[rs[filled] // k]).all()


def test_noalloc_permute_matches_workspace_permute_twice(lib):
    moe = lib
    cases = [(1000, 192, 4, 768, 27, 1.2, 1), (300, 8, 2, 64, 0, 0.0, 2)]
    for T, E, k, d, cap, skew, seed in cases:            # two calls in a row, different shapes
        s = _shape(moe, T, E, k, d, cap)
        x, idx = _case(T, E, k, d, cap, skew, seed)
        want = moe.moe_permute(s, x, idx)
        got = moe.moe_permute_noalloc(s, x, idx)
        torch.cuda.synchronize()
        _same(got, want)
        _same_as_oracle(got, idx, E, k, cap, x)
    assert moe.moe_get_status()[0] == 0


def test_noalloc_permute_without_counts_buffer(lib):
    """counts = NULL: the per-expert counts then live in the tail of the fixed scratch array.  Called through
    the C ABI directly, twice in a row with a capacity (drops) and without, against the oracle."""
    moe = lib
    L = moe.load()
    for T, E, k, d, cap, skew, seed in [(777, 24, 3, 128, 60, 1.2, 3), (2049, 64, 4, 64, 0, 0.5, 4)]:
        s = _shape(moe, T, E, k, d, cap)
        x, idx = _case(T, E, k, d, cap, skew, seed)
        R = s.R
        out = dict(slot_pos=torch.empty(T, k, dtype=torch.int32, device=DEV),
                   drop_mask=torch.empty(T, k, dtype=torch.uint8, device=DEV),
                   kept=torch.empty(E, dtype=torch.int32, device=DEV),
                   offsets=torch.empty(E + 1, dtype=torch.int32, device=DEV),
                   row_src=torch.full((R,), -1, dtype=torch.int32, device=DEV),
                   x_perm=torch.zeros(R, d, dtype=torch.bfloat16, device=DEV))
        P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        rc = L.moe_permute_noalloc(ctypes.byref(s), P(x), P(idx), P(out["slot_pos"]), P(out["drop_mask"]), None,
                                   P(out["kept"]), P(out["offsets"]), P(out["row_src"]), P(out["x_perm"]),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0
        torch.cuda.synchronize()
        _same_as_oracle(out, idx, E, k, cap, x)
        if cap:
            assert int(out["drop_mask"].sum()) > 0
    assert moe.moe_get_status()[0] == 0


def test_noalloc_permute_rejects_shapes_beyond_its_scratch(lib):
    moe = lib
    L = moe.load()
    s = _shape(moe, 32 * 513, 512, 2, 16, 0)               # ceil(T/32) * E = 262656 > 262144
    fake = ctypes.c_void_p(4096)                            # never dereferenced: the size check fails first
    rc = L.moe_permute_noalloc(ctypes.byref(s), fake, fake, fake, None, None, fake, fake, None, fake, None)
    assert rc == 2                                          # MOE_UNSUPPORTED_SHAPE
