"""Python binding of the B200 routed MoE FFN forward library (``libmoe_b200.so``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels, enqueued on the current torch CUDA stream.  torch provides device
memory (outputs, workspace) and streams.  There is no CPU fallback: if the
library is missing or no CUDA device is present, calls raise.

The entry points mirror the C ABI in ``include/moe_b200.h``:
``moe_route``, ``moe_route_from_logits``, ``moe_permute``, ``moe_expert_ffn``,
``moe_combine``, ``moe_forward``, ``moe_quantize_int4``, plus
``moe_workspace_size``, ``moe_capacity``, ``moe_get_status``.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

ACT_SWIGLU, ACT_GEGLU = 0, 1
WFMT_BF16, WFMT_INT4_G128 = 0, 1
FLAG_SINGLE_CTA_GEMM = 1
STATUS = {0: "MOE_OK", 1: "MOE_INVALID_ARGUMENT", 2: "MOE_UNSUPPORTED_SHAPE", 3: "MOE_WORKSPACE_TOO_SMALL",
          4: "MOE_CUDA_ERROR", 5: "MOE_DEVICE_TIMEOUT"}

EXPORTED = ["moe_grouped_rows", "moe_capacity", "moe_workspace_size", "moe_route", "moe_route_from_logits",
            "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward", "moe_quantize_int4", "moe_get_status",
            "moe_set_wait_limit_ns", "moe_selftest_wait_timeout", "moe_launch_count", "moe_status_string",
            "moe_permute_noalloc", "moe_transpose_experts", "moe_backward_workspace_size", "moe_backward_x",
            "moe_backward", "moe_route_tree_workspace_size", "moe_route_tree"]


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("H", ctypes.c_int32), ("H_s", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("act", ctypes.c_int32), ("wfmt", ctypes.c_int32), ("renorm", ctypes.c_int32),
                ("flags", ctypes.c_int32)]

    def __init__(self, T, d, E, k, H, H_s=0, capacity=0, act=ACT_SWIGLU, wfmt=WFMT_BF16, renorm=1, flags=0):
        super().__init__(T, d, E, k, H, H_s, capacity, act, wfmt, renorm, flags)

    @property
    def R(self) -> int:
        return self.E * self.capacity if self.capacity > 0 else self.T * self.k

    def __repr__(self):
        return "MoeShape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


_lib = None
_P = ctypes.c_void_p


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (built by ``__graft_entry__.build()``); raises if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing (run __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    S = ctypes.POINTER(MoeShape)
    i32, i64, u64, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    sig = {
        "moe_grouped_rows": (i64, [S]),
        "moe_capacity": (ctypes.c_int, [i64, i32, i32, ctypes.c_double, ctypes.POINTER(i32)]),
        "moe_workspace_size": (ctypes.c_int, [S, ctypes.POINTER(sz)]),
        "moe_route": (ctypes.c_int, [S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
        "moe_route_from_logits": (ctypes.c_int, [S, _P, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
        "moe_permute": (ctypes.c_int, [S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, sz, _P]),
        "moe_expert_ffn": (ctypes.c_int, [S, i32, i32, i64, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "moe_combine": (ctypes.c_int, [S, _P, _P, _P, _P, _P, _P]),
        "moe_forward": (ctypes.c_int, [S] + [_P] * 20 + [sz, _P, _P]),
        "moe_quantize_int4": (ctypes.c_int, [_P, i64, i32, _P, _P, _P]),
        "moe_get_status": (ctypes.c_int, [_P, ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_uint32)]),
        "moe_set_wait_limit_ns": (ctypes.c_int, [u64]),
        "moe_selftest_wait_timeout": (ctypes.c_int, [_P]),
        "moe_launch_count": (u64, []),
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_permute_noalloc": (ctypes.c_int, [S, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
        "moe_transpose_experts": (ctypes.c_int, [_P, i64, i32, i32, _P, _P]),
        "moe_backward_workspace_size": (ctypes.c_int, [S, ctypes.POINTER(sz)]),
        "moe_backward_x": (ctypes.c_int, [S] + [_P] * 10 + [ctypes.c_float, _P, _P, sz, _P]),
        "moe_backward": (ctypes.c_int, [S] + [_P] * 10 + [ctypes.c_float] + [_P] * 7 + [sz, _P, _P]),
        "moe_route_tree_workspace_size": (ctypes.c_int, [S, i32, i32, ctypes.POINTER(sz)]),
        "moe_route_tree": (ctypes.c_int, [S, i32, i32] + [_P] * 8 + [sz, _P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _L():
    return _lib if _lib is not None else load()


def _check(code: int, where: str):
    if code != 0:
        raise MoeError(code, where)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensor expected")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _want(t, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


_ws_cache: dict = {}


def moe_workspace_size(shape: MoeShape) -> int:
    n = ctypes.c_size_t(0)
    _check(_L().moe_workspace_size(ctypes.byref(shape), ctypes.byref(n)), "moe_workspace_size")
    return int(n.value)


def workspace(shape: MoeShape, device=None) -> torch.Tensor:
    """A cached device buffer of moe_workspace_size(shape) bytes (grown on demand, per device)."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    need = moe_workspace_size(shape)
    buf = _ws_cache.get(dev)
    if buf is None or buf.numel() < need:
        buf = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
        _ws_cache[dev] = buf
    return buf


def moe_capacity(T: int, k: int, E: int, factor: float) -> int:
    c = ctypes.c_int32(0)
    _check(_L().moe_capacity(T, k, E, float(factor), ctypes.byref(c)), "moe_capacity")
    return int(c.value)


def moe_route(shape: MoeShape, x, w_router, bias=None, *, logits=False, aux=False, ws=None, stream=None):
    T, d, E, k = shape.T, shape.d, shape.E, shape.k
    _want(x, torch.bfloat16, (T, d), "x")
    _want(w_router, torch.float32, (E, d), "w_router")
    dev = x.device
    out = dict(topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
               topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
               counts=torch.empty(E, dtype=torch.int32, device=dev))
    if logits:
        out["logits"] = torch.empty(T, E, dtype=torch.float32, device=dev)
    if aux:
        out["aux_f"] = torch.empty(E, dtype=torch.float32, device=dev)
        out["aux_p"] = torch.empty(E, dtype=torch.float32, device=dev)
        out["aux"] = torch.empty(1, dtype=torch.float32, device=dev)
    ws = ws if ws is not None else workspace(shape, dev)
    rc = _L().moe_route(ctypes.byref(shape), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(out.get("logits")),
                        _ptr(out["topk_idx"]), _ptr(out["topk_w"]), _ptr(out["counts"]), _ptr(out.get("aux_f")),
                        _ptr(out.get("aux_p")), _ptr(out.get("aux")), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "moe_route")
    return out


def moe_route_from_logits(shape: MoeShape, logits, *, aux=False, ws=None, stream=None):
    T, E, k = shape.T, shape.E, shape.k
    _want(logits, torch.float32, (T, E), "logits")
    dev = logits.device
    out = dict(topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
               topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
               counts=torch.empty(E, dtype=torch.int32, device=dev))
    if aux:
        out["aux_f"] = torch.empty(E, dtype=torch.float32, device=dev)
        out["aux_p"] = torch.empty(E, dtype=torch.float32, device=dev)
        out["aux"] = torch.empty(1, dtype=torch.float32, device=dev)
    ws = ws if ws is not None else workspace(shape, dev)
    rc = _L().moe_route_from_logits(ctypes.byref(shape), _ptr(logits), _ptr(out["topk_idx"]), _ptr(out["topk_w"]),
                                    _ptr(out["counts"]), _ptr(out.get("aux_f")), _ptr(out.get("aux_p")),
                                    _ptr(out.get("aux")), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "moe_route_from_logits")
    return out


def permute_outputs(shape: MoeShape, device):
    """Output buffers of moe_permute: row_src = -1 and x_perm = 0 in the rows the call leaves unfilled."""
    T, d, E, k, R = shape.T, shape.d, shape.E, shape.k, shape.R
    return dict(slot_pos=torch.empty(T, k, dtype=torch.int32, device=device),
                drop_mask=torch.empty(T, k, dtype=torch.uint8, device=device),
                counts=torch.empty(E, dtype=torch.int32, device=device),
                kept=torch.empty(E, dtype=torch.int32, device=device),
                offsets=torch.empty(E + 1, dtype=torch.int32, device=device),
                row_src=torch.full((R,), -1, dtype=torch.int32, device=device),
                x_perm=torch.zeros(R, d, dtype=torch.bfloat16, device=device))


def moe_permute(shape: MoeShape, x, topk_idx, *, ws=None, stream=None, out=None):
    """Grouping by expert.  `out` (from permute_outputs) reuses buffers: rows this call leaves unfilled keep
    what they held, and nothing is allocated or filled here."""
    T, d, E, k = shape.T, shape.d, shape.E, shape.k
    _want(x, torch.bfloat16, (T, d), "x")
    _want(topk_idx, torch.int32, (T, k), "topk_idx")
    dev = x.device
    if out is None:
        out = permute_outputs(shape, dev)
    else:
        _want(out["x_perm"], torch.bfloat16, (shape.R, d), "out['x_perm']")
        _want(out["row_src"], torch.int32, (shape.R,), "out['row_src']")
        _want(out["slot_pos"], torch.int32, (T, k), "out['slot_pos']")
    ws = ws if ws is not None else workspace(shape, dev)
    rc = _L().moe_permute(ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(out["slot_pos"]),
                          _ptr(out["drop_mask"]), _ptr(out["counts"]), _ptr(out["kept"]), _ptr(out["offsets"]),
                          _ptr(out["row_src"]), _ptr(out["x_perm"]), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "moe_permute")
    return out


def moe_permute_noalloc(shape: MoeShape, x, topk_idx, *, stream=None):
    """moe_permute without a workspace: the library's fixed scratch array is used instead.

    For callers that cannot allocate device scratch; the outputs here are still
    torch tensors.  Calls that overlap on the GPU race on the shared scratch.
    """
    T, d, E, k = shape.T, shape.d, shape.E, shape.k
    _want(x, torch.bfloat16, (T, d), "x")
    _want(topk_idx, torch.int32, (T, k), "topk_idx")
    dev = x.device
    R = shape.R
    out = dict(slot_pos=torch.empty(T, k, dtype=torch.int32, device=dev),
               drop_mask=torch.empty(T, k, dtype=torch.uint8, device=dev),
               counts=torch.empty(E, dtype=torch.int32, device=dev),
               kept=torch.empty(E, dtype=torch.int32, device=dev),
               offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
               row_src=torch.full((R,), -1, dtype=torch.int32, device=dev),
               x_perm=torch.zeros(R, d, dtype=torch.bfloat16, device=dev))
    rc = _L().moe_permute_noalloc(ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(out["slot_pos"]),
                                  _ptr(out["drop_mask"]), _ptr(out["counts"]), _ptr(out["kept"]),
                                  _ptr(out["offsets"]), _ptr(out["row_src"]), _ptr(out["x_perm"]), _stream(stream))
    _check(rc, "moe_permute_noalloc")
    return out


def moe_expert_ffn(shape: MoeShape, x_grouped, w13, w2, *, hidden=None, group_start=None, group_rows=None,
                   s13=None, s2=None, h=None, y=None, want_h=True, stream=None):
    """Grouped gated expert FFN.  Returns (h, y); with ``want_h=False`` (bf16 experts of hidden 128 or 256) h
    stays on chip in the fused kernel and None is returned in its place."""
    hidden = shape.H if hidden is None else hidden
    R = x_grouped.shape[0]
    n_groups = w13.shape[0]
    dev = x_grouped.device
    if h is None and want_h:
        h = torch.empty(R, hidden, dtype=torch.bfloat16, device=dev)
    if y is None:
        y = torch.empty(R, shape.d, dtype=torch.bfloat16, device=dev)
    rc = _L().moe_expert_ffn(ctypes.byref(shape), n_groups, hidden, R, _ptr(x_grouped), _ptr(group_start),
                             _ptr(group_rows), _ptr(w13), _ptr(s13), _ptr(w2), _ptr(s2), _ptr(h), _ptr(y),
                             _stream(stream))
    _check(rc, "moe_expert_ffn")
    return h, y


def moe_combine(shape: MoeShape, y_perm, slot_pos, topk_w, y_shared=None, *, out=None, stream=None):
    if out is None:
        out = torch.empty(shape.T, shape.d, dtype=torch.bfloat16, device=y_perm.device)
    rc = _L().moe_combine(ctypes.byref(shape), _ptr(y_perm), _ptr(slot_pos), _ptr(topk_w), _ptr(y_shared),
                          _ptr(out), _stream(stream))
    _check(rc, "moe_combine")
    return out


def moe_forward(shape: MoeShape, x, w_router, w13, w2, *, bias=None, s13=None, s2=None, w13_sh=None, s13_sh=None,
                w2_sh=None, s2_sh=None, out=None, routing=False, aux=False, ws=None, stream=None, side_stream=None):
    """The whole layer.  Returns ``out`` [T, d] bf16, or a dict with routing outputs when asked.
    ``side_stream`` (a torch.cuda.Stream) lets a bf16 shared expert overlap the routing and routed experts."""
    T, d, E, k = shape.T, shape.d, shape.E, shape.k
    _want(x, torch.bfloat16, (T, d), "x")
    dev = x.device
    if out is None:
        out = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    r = {}
    if routing:
        r = dict(topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
                 topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
                 counts=torch.empty(E, dtype=torch.int32, device=dev),
                 drop_mask=torch.empty(T, k, dtype=torch.uint8, device=dev))
    if aux:
        r.update(aux_f=torch.empty(E, dtype=torch.float32, device=dev),
                 aux_p=torch.empty(E, dtype=torch.float32, device=dev),
                 aux=torch.empty(1, dtype=torch.float32, device=dev))
    ws = ws if ws is not None else workspace(shape, dev)
    rc = _L().moe_forward(ctypes.byref(shape), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w13), _ptr(s13), _ptr(w2),
                          _ptr(s2), _ptr(w13_sh), _ptr(s13_sh), _ptr(w2_sh), _ptr(s2_sh), _ptr(out),
                          _ptr(r.get("topk_idx")), _ptr(r.get("topk_w")), _ptr(r.get("counts")),
                          _ptr(r.get("drop_mask")), _ptr(r.get("aux_f")), _ptr(r.get("aux_p")), _ptr(r.get("aux")),
                          _ptr(ws), ws.numel(), _stream(stream),
                          ctypes.c_void_p(side_stream.cuda_stream) if side_stream is not None else None)
    _check(rc, "moe_forward")
    if r:
        r["out"] = out
        return r
    return out


def moe_transpose_experts(w, *, out=None, stream=None):
    """[n, rows, cols] bf16 -> [n, cols, rows] bf16 (the transposed expert weights moe_backward_x takes)."""
    n, rows, cols = w.shape
    _want(w, torch.bfloat16, (n, rows, cols), "w")
    if out is None:
        out = torch.empty(n, cols, rows, dtype=torch.bfloat16, device=w.device)
    _check(_L().moe_transpose_experts(_ptr(w), n, rows, cols, _ptr(out), _stream(stream)), "moe_transpose_experts")
    return out


def _backward(shape, x, w_router, w13, w2, dout, bias, w13t, w2t, w13_sh, w2_sh, w13t_sh, w2t_sh, aux_coef, ws,
              stream, weights, side_stream=None):
    T, d, E, H, Hs = shape.T, shape.d, shape.E, shape.H, shape.H_s
    _want(x, torch.bfloat16, (T, d), "x")
    _want(dout, torch.bfloat16, (T, d), "dout")
    w13t = w13t if w13t is not None else moe_transpose_experts(w13, stream=stream)
    w2t = w2t if w2t is not None else moe_transpose_experts(w2, stream=stream)
    if Hs:
        w13t_sh = w13t_sh if w13t_sh is not None else moe_transpose_experts(w13_sh, stream=stream)
        w2t_sh = w2t_sh if w2t_sh is not None else moe_transpose_experts(w2_sh, stream=stream)
    if ws is None:
        n = ctypes.c_size_t(0)
        _check(_L().moe_backward_workspace_size(ctypes.byref(shape), ctypes.byref(n)), "moe_backward_workspace_size")
        ws = torch.empty(int(n.value), dtype=torch.uint8, device=x.device)
    f32 = dict(dtype=torch.float32, device=x.device)
    g = dict(dx=torch.empty(T, d, **f32))
    head = [ctypes.byref(shape), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w13), _ptr(w13t), _ptr(w2t),
            _ptr(w13_sh), _ptr(w13t_sh), _ptr(w2t_sh), _ptr(dout), float(aux_coef), _ptr(g["dx"])]
    tail = [_ptr(ws), ws.numel(), _stream(stream)]
    if not weights:
        _check(_L().moe_backward_x(*head, *tail), "moe_backward_x")
        return g
    g.update(dw13=torch.empty(E, 2 * H, d, **f32), dw2=torch.empty(E, d, H, **f32),
             dw13_sh=torch.empty(1, 2 * Hs, d, **f32) if Hs else None,
             dw2_sh=torch.empty(1, d, Hs, **f32) if Hs else None, dw_router=torch.empty(E, d, **f32))
    side = ctypes.c_void_p(side_stream.cuda_stream) if side_stream is not None else None
    _check(_L().moe_backward(*head, _ptr(g["dw13"]), _ptr(g["dw2"]), _ptr(g["dw13_sh"]), _ptr(g["dw2_sh"]),
                             _ptr(g["dw_router"]), *tail, side), "moe_backward")
    return g


def moe_backward_x(shape: MoeShape, x, w_router, w13, w2, dout, *, bias=None, w13t=None, w2t=None, w13_sh=None,
                   w2_sh=None, w13t_sh=None, w2t_sh=None, aux_coef=0.0, ws=None, stream=None):
    """Input gradient dL/dx [T, d] fp32 of L = sum(dout * out) + aux_coef * aux (bf16 experts).  The transposed
    weights are made here when not given (moe_transpose_experts); the down projections enter only transposed."""
    return _backward(shape, x, w_router, w13, w2, dout, bias, w13t, w2t, w13_sh, w2_sh, w13t_sh, w2t_sh, aux_coef,
                     ws, stream, False)["dx"]


def moe_backward(shape: MoeShape, x, w_router, w13, w2, dout, *, bias=None, w13t=None, w2t=None, w13_sh=None,
                 w2_sh=None, w13t_sh=None, w2t_sh=None, aux_coef=0.0, ws=None, stream=None, side_stream=None):
    """All gradients of L = sum(dout * out) + aux_coef * aux: a dict of fp32 tensors dx [T, d], dw13 [E, 2H, d],
    dw2 [E, d, H], dw13_sh [1, 2H_s, d] and dw2_sh [1, d, H_s] (None without a shared expert), dw_router [E, d].
    ``side_stream`` (a torch.cuda.Stream) lets the shared expert's chain overlap the routed one."""
    return _backward(shape, x, w_router, w13, w2, dout, bias, w13t, w2t, w13_sh, w2_sh, w13t_sh, w2t_sh, aux_coef,
                     ws, stream, True, side_stream)


def moe_route_tree(shape: MoeShape, branch: int, levels: int, x, w_tree, bias_tree=None, *, counts=False,
                   logits=False, ws=None, stream=None):
    """Hierarchical router over E = branch**levels experts (shape.E).  w_tree [levels * branch, d] fp32 stacks
    the levels' routers.  Returns dict(topk_idx [T, k] int32, topk_w [T, k] fp32, counts [E] int32 or None,
    level_logits [T, levels * branch] fp32 or None)."""
    T, d, E, k = shape.T, shape.d, shape.E, shape.k
    n = branch * levels
    _want(x, torch.bfloat16, (T, d), "x")
    _want(w_tree, torch.float32, (n, d), "w_tree")
    if bias_tree is not None:
        _want(bias_tree, torch.float32, (n,), "bias_tree")
    dev = x.device
    if ws is None:
        nb = ctypes.c_size_t(0)
        _check(_L().moe_route_tree_workspace_size(ctypes.byref(shape), branch, levels, ctypes.byref(nb)),
               "moe_route_tree_workspace_size")
        ws = torch.empty(int(nb.value), dtype=torch.uint8, device=dev)
    out = dict(topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
               topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
               counts=torch.empty(E, dtype=torch.int32, device=dev) if counts else None,
               level_logits=torch.empty(T, n, dtype=torch.float32, device=dev) if logits else None)
    rc = _L().moe_route_tree(ctypes.byref(shape), branch, levels, _ptr(x), _ptr(w_tree), _ptr(bias_tree),
                             _ptr(out["topk_idx"]), _ptr(out["topk_w"]), _ptr(out["counts"]),
                             _ptr(out["level_logits"]), _ptr(ws), ws.numel(), _stream(stream))
    _check(rc, "moe_route_tree")
    return out


def moe_quantize_int4(w, *, q=None, scales=None, stream=None):
    """w [..., K] fp32 -> (q [..., K/2] uint8, scales [..., K/128] bf16)."""
    K = w.shape[-1]
    rows = w.numel() // K
    if q is None:
        q = torch.empty(*w.shape[:-1], K // 2, dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(*w.shape[:-1], K // 128, dtype=torch.bfloat16, device=w.device)
    rc = _L().moe_quantize_int4(_ptr(w), rows, K, _ptr(q), _ptr(scales), _stream(stream))
    _check(rc, "moe_quantize_int4")
    return q, scales


def moe_get_status(stream=None):
    st, site = ctypes.c_int32(0), ctypes.c_uint32(0)
    _check(_L().moe_get_status(_stream(stream), ctypes.byref(st), ctypes.byref(site)), "moe_get_status")
    return int(st.value), int(site.value)


def moe_launch_count() -> int:
    return int(_L().moe_launch_count())
