"""Host logic of the autograd wrapper (``sparse_mixture_experts_expert_b200.autograd``) on CPU, with the two
entry points replaced by stand-ins that record their arguments: which tensors reach moe_forward and
moe_backward, that the returned aux takes no gradient, that each gradient reaches its own input (the exploration
bias none), and that a layer without a shared expert passes None through."""

import torch

import sparse_mixture_experts_expert_b200 as moe
import sparse_mixture_experts_expert_b200.autograd as ag


def _fakes(calls):
    def fwd(shape, x, w_router, w13, w2, *, bias=None, w13_sh=None, w2_sh=None, aux=False):
        calls["fwd"] = dict(bias=bias, w13_sh=w13_sh, aux=aux)
        return dict(out=(x.float() * 2).to(x.dtype), aux=torch.tensor([1.5]))

    def bwd(shape, x, w_router, w13, w2, dout, *, bias=None, w13_sh=None, w2_sh=None, aux_coef=0.0):
        calls["bwd"] = dict(bias=bias, w13_sh=w13_sh, aux_coef=aux_coef, dout=dout.clone())
        f = lambda t, v: torch.full(t.shape, v, dtype=torch.float32)
        return dict(dx=dout.float() * 2, dw_router=f(w_router, 3.0), dw13=f(w13, 4.0), dw2=f(w2, 5.0),
                    dw13_sh=f(w13_sh, 6.0) if w13_sh is not None else None,
                    dw2_sh=f(w2_sh, 7.0) if w2_sh is not None else None)
    return fwd, bwd


def _inputs(shared):
    T, d, E, H = 4, 8, 3, 16
    g = torch.Generator().manual_seed(0)
    t = lambda *sh, dt=torch.bfloat16: torch.randn(*sh, generator=g).to(dt).requires_grad_(True)
    x, wr, w13, w2 = t(T, d), t(E, d, dt=torch.float32), t(E, 2 * H, d), t(E, d, H)
    w13s, w2s = (t(1, 2 * 16, d), t(1, d, 16)) if shared else (None, None)
    return moe.MoeShape(T=T, d=d, E=E, k=2, H=H, H_s=16 if shared else 0), x, wr, w13, w2, w13s, w2s


def test_gradients_reach_their_inputs(monkeypatch):
    calls = {}
    fwd, bwd = _fakes(calls)
    monkeypatch.setattr(ag, "moe_forward", fwd)
    monkeypatch.setattr(ag, "moe_backward", bwd)
    s, x, wr, w13, w2, w13s, w2s = _inputs(True)
    bias = torch.zeros(3)
    out, aux = ag.moe_layer(s, x, wr, w13, w2, bias=bias, w13_sh=w13s, w2_sh=w2s, aux_coef=0.25, return_aux=True)
    assert calls["fwd"]["aux"] and calls["fwd"]["bias"] is bias and calls["fwd"]["w13_sh"] is w13s
    assert not aux.requires_grad and float(aux) == 1.5
    out.float().sum().backward()
    b = calls["bwd"]
    assert b["aux_coef"] == 0.25 and b["bias"] is not None and b["w13_sh"] is not None
    assert b["dout"].dtype == torch.bfloat16 and torch.equal(b["dout"], torch.ones(4, 8, dtype=torch.bfloat16))
    assert x.grad.dtype == torch.bfloat16 and torch.equal(x.grad, torch.full((4, 8), 2.0, dtype=torch.bfloat16))
    for leaf, v in ((wr, 3.0), (w13, 4.0), (w2, 5.0), (w13s, 6.0), (w2s, 7.0)):
        assert leaf.grad.dtype == leaf.dtype and bool((leaf.grad.float() == v).all())


def test_layer_without_a_shared_expert(monkeypatch):
    calls = {}
    fwd, bwd = _fakes(calls)
    monkeypatch.setattr(ag, "moe_forward", fwd)
    monkeypatch.setattr(ag, "moe_backward", bwd)
    s, x, wr, w13, w2, _, _ = _inputs(False)
    out = ag.moe_layer(s, x, wr, w13, w2)
    assert calls["fwd"]["w13_sh"] is None and calls["fwd"]["bias"] is None
    out.float().sum().backward()
    assert calls["bwd"]["w13_sh"] is None and calls["bwd"]["bias"] is None and calls["bwd"]["aux_coef"] == 0.0
    assert x.grad is not None and w13.grad is not None
