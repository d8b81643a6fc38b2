"""Host-side checks of the C ABI (no GPU needed): the library builds, loads,
exports every entry point its header declares, and rejects bad arguments with
the documented status codes before touching the device."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from sparse_mixture_experts_expert_b200 import _build
    _build.build()
    import sparse_mixture_experts_expert_b200 as moe
    return moe.load()


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(moe_[a-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 12, names
    for n in names:
        assert hasattr(L, n), n
    import sparse_mixture_experts_expert_b200 as moe
    assert sorted(moe.EXPORTED) == names


def _declared_arity():
    """Number of parameters of every declared entry point (from the header's prototypes)."""
    out = {}
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            for m in re.finditer(r"(moe_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src, flags=re.S):
                params = m.group(2).strip()
                out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header(L):
    # every ctypes prototype the binding sets takes as many arguments as the header declares
    arity = _declared_arity()
    for name in arity:
        f = getattr(L, name)
        assert f.argtypes is not None, name
        assert len(f.argtypes) == arity[name], (name, len(f.argtypes), arity[name])


def _shape(moe, **kw):
    base = dict(T=256, d=64, E=8, k=2, H=128)
    base.update(kw)
    return moe.MoeShape(**base)


def test_status_strings(L):
    assert L.moe_status_string(0) == b"ok"
    assert L.moe_status_string(3) == b"workspace too small"
    assert L.moe_status_string(99) == b"unknown status"


def test_capacity_and_rows(L):
    import sparse_mixture_experts_expert_b200 as moe
    assert moe.moe_capacity(32768, 4, 192, 1.25) == 854
    assert moe.moe_capacity(256, 2, 8, 0.5) == 32
    assert moe.moe_capacity(256, 2, 8, 0.0) == 0
    s = _shape(moe, capacity=32)
    assert L.moe_grouped_rows(ctypes.byref(s)) == 8 * 32
    s = _shape(moe)
    assert L.moe_grouped_rows(ctypes.byref(s)) == 512


@pytest.mark.parametrize("kw,code", [({"k": 9}, 1), ({"d": 60}, 2), ({"H": 0}, 2), ({"E": 513}, 2),
                                     ({"T": 0}, 2), ({"act": 7}, 1), ({"wfmt": 1, "d": 64}, 2),
                                     ({"renorm": 2}, 1), ({"capacity": -1}, 1), ({"flags": 2}, 1),
                                     ({"flags": -1}, 1), ({"flags": 1}, 0)])
def test_shape_validation(L, kw, code):
    import sparse_mixture_experts_expert_b200 as moe
    s = _shape(moe, **kw)
    n = ctypes.c_size_t(0)
    assert L.moe_workspace_size(ctypes.byref(s), ctypes.byref(n)) == code


def test_workspace_size_grows_with_shape(L):
    import sparse_mixture_experts_expert_b200 as moe
    a = moe.moe_workspace_size(_shape(moe))
    b = moe.moe_workspace_size(_shape(moe, T=4096))
    assert 0 < a < b
    assert a % 256 == 0


def test_null_and_workspace_errors_return_before_device_work(L):
    import sparse_mixture_experts_expert_b200 as moe
    s = _shape(moe)
    P = ctypes.c_void_p
    fake = P(4096)            # never dereferenced: the checks fail first
    rc = L.moe_route(ctypes.byref(s), None, fake, None, None, fake, fake, fake, None, None, None, fake, 1 << 30, None)
    assert rc == 1
    rc = L.moe_route(ctypes.byref(s), fake, fake, None, None, fake, fake, fake, None, None, None, fake, 16, None)
    assert rc == 3
    rc = L.moe_route(ctypes.byref(s), P(4097), fake, None, None, fake, fake, fake, None, None, None, fake, 1 << 30,
                     None)
    assert rc == 1            # misaligned x
    rc = L.moe_forward(ctypes.byref(s), fake, fake, None, fake, None, fake, None, None, None, None, None, fake,
                       None, None, None, None, None, None, None, fake, 16, None, None)
    assert rc == 3
    rc = L.moe_quantize_int4(fake, 4, 100, fake, fake, None)
    assert rc == 1            # K % 128 != 0
    assert L.moe_set_wait_limit_ns(0) == 1


@pytest.mark.parametrize("kw,branch,levels,code", [({"E": 4096}, 16, 3, 0), ({"E": 4095}, 16, 3, 1),
                                                   ({"E": 2 ** 20}, 32, 4, 0), ({"E": 33 ** 2}, 33, 2, 2),
                                                   ({"E": 27}, 3, 3, 2), ({"E": 16, "k": 17}, 16, 1, 2),
                                                   ({"E": 4, "k": 3}, 2, 2, 0), ({"E": 4, "k": 5}, 4, 1, 1), ({"E": 2}, 2, 1, 2),
                                                   ({"E": 2 ** 21}, 2, 21, 2), ({"E": 16, "renorm": 3}, 4, 2, 1)])
def test_tree_router_shape_validation(L, kw, branch, levels, code):
    # E = branch^levels; branch 2..32; branch * levels a multiple of 4 and <= 256; E <= 2^20; k <= min(16, E)
    import sparse_mixture_experts_expert_b200 as moe
    s = _shape(moe, **kw)
    n = ctypes.c_size_t(0)
    assert L.moe_route_tree_workspace_size(ctypes.byref(s), branch, levels, ctypes.byref(n)) == code
    if code == 0:
        assert n.value > 0 and n.value % 256 == 0


def test_tree_router_errors_return_before_device_work(L):
    import sparse_mixture_experts_expert_b200 as moe
    s = _shape(moe, E=16)
    P = ctypes.c_void_p
    fake = P(4096)
    n = ctypes.c_size_t(0)
    assert L.moe_route_tree_workspace_size(ctypes.byref(s), 4, 2, ctypes.byref(n)) == 0
    args = lambda x, ws, nb: (ctypes.byref(s), 4, 2, x, fake, None, fake, fake, None, None, ws, nb, None)
    assert L.moe_route_tree(*args(None, fake, n.value)) == 1            # x missing
    assert L.moe_route_tree(*args(P(4098), fake, n.value)) == 1         # misaligned x
    assert L.moe_route_tree(*args(fake, fake, n.value - 256)) == 3      # workspace too small
    assert L.moe_route_tree(*args(fake, P(4096 + 16), n.value)) == 1    # workspace not 256-byte aligned


def test_backward_workspace_and_errors(L):
    import sparse_mixture_experts_expert_b200 as moe
    s = _shape(moe, H_s=64)
    n, f = ctypes.c_size_t(0), ctypes.c_size_t(0)
    assert L.moe_backward_workspace_size(ctypes.byref(s), ctypes.byref(n)) == 0
    assert L.moe_workspace_size(ctypes.byref(s), ctypes.byref(f)) == 0
    assert n.value > f.value        # the forward's regions plus the backward's own
    P = ctypes.c_void_p
    fake = P(4096)
    head = lambda sh: [ctypes.byref(sh), fake, fake, None, fake, fake, fake, fake, fake, fake, fake,
                       ctypes.c_float(0.0), fake]
    assert L.moe_backward_x(*head(s), fake, n.value - 256, None) == 3  # workspace too small
    assert L.moe_backward(*head(s), None, None, None, None, None, fake, n.value - 256, None, None) == 3
    assert L.moe_backward(*head(s), P(4100), None, None, None, None, fake, n.value, None, None) == 1  # misaligned dw13
    sh = _shape(moe, H_s=64)
    sh.wfmt = 1
    assert L.moe_backward_x(*head(sh), fake, n.value, None) == 2       # INT4 experts: no backward
    s0 = _shape(moe, H_s=64)
    args = head(s0)
    args[7] = None                                                      # shared expert without its weights
    assert L.moe_backward_x(*args, fake, n.value, None) == 1
