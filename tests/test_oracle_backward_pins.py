"""Pins for the oracle's gradients: with respect to the inputs and routing weights
(experts frozen) and with respect to the expert weights.

* central finite differences of the oracle forward (itself pinned by
  tests/test_oracle_pins.py): L = sum_t,o out[t, o] * dout[t, o], each element of x
  and of topk_weights moved both ways, in fp64 on fp32 inputs;
* torch autograd of a dense fp64 formulation sum_e R[t, e] * MLP_e(x_t) (a
  different loop structure: a routing matrix instead of slots, the library's
  differentiation instead of the hand-written chain rule);
* special cases: an out-of-range id contributes nothing and its weight gets a
  zero gradient; strided views read the same values as contiguous copies.
"""

import pytest
import torch

import oracle
from mixture_experts_layer_46_b200 import workloads as wl


def _case(T=3, H=16, I=8, E=3, k=2, seed=5):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, H, generator=g)
    gate = torch.randn(E, I, H, generator=g) / H ** 0.5
    up = torch.randn(E, I, H, generator=g) / H ** 0.5
    w2 = torch.randn(E, H, I, generator=g) / I ** 0.5
    ids, wts = wl.route_softmax_topk(T, E, k, seed=seed + 1)
    dout = torch.randn(T, H, generator=g)
    return x, gate, up, w2, ids, wts.float(), dout


def _loss(x, gate, up, w2, ids, wts, dout):
    out, _ = oracle.moe_forward(x, gate, up, w2, ids, wts)
    return float((out * dout.double()).sum())


def test_gradient_matches_central_finite_differences():
    x, gate, up, w2, ids, wts, dout = _case()
    dx, dw = oracle.moe_backward_input(x, gate, up, w2, ids, wts, dout)
    d = 1e-3
    num_dx = torch.zeros_like(dx)
    for t in range(x.shape[0]):
        for h in range(x.shape[1]):
            xp, xm = x.clone(), x.clone()
            xp[t, h] += d
            xm[t, h] -= d
            step = float(xp[t, h].double() - xm[t, h].double())  # the fp32 values' real distance
            num_dx[t, h] = (_loss(xp, gate, up, w2, ids, wts, dout) -
                            _loss(xm, gate, up, w2, ids, wts, dout)) / step
    num_dw = torch.zeros_like(dw)
    for t in range(wts.shape[0]):
        for j in range(wts.shape[1]):
            wp, wm = wts.clone(), wts.clone()
            wp[t, j] += d
            wm[t, j] -= d
            step = float(wp[t, j].double() - wm[t, j].double())
            num_dw[t, j] = (_loss(x, gate, up, w2, ids, wp, dout) -
                            _loss(x, gate, up, w2, ids, wm, dout)) / step
    assert (dx - num_dx).abs().max() <= 1e-5 * dx.abs().max()
    assert (dw - num_dw).abs().max() <= 1e-5 * dw.abs().max()


def test_gradient_matches_autograd_of_dense_formulation():
    x, gate, up, w2, ids, wts, dout = _case(T=5, H=24, I=12, E=4, k=3, seed=9)
    xd = x.double().requires_grad_(True)
    wd = wts.double().requires_grad_(True)
    E = gate.shape[0]
    R = torch.zeros(x.shape[0], E, dtype=torch.float64).index_put(
        (torch.arange(x.shape[0]).repeat_interleave(ids.shape[1]), ids.long().reshape(-1)),
        wd.reshape(-1), accumulate=True)
    out = torch.zeros(x.shape[0], x.shape[1], dtype=torch.float64)
    for e in range(E):
        hmid = torch.nn.functional.silu(xd @ gate[e].double().T) * (xd @ up[e].double().T)
        out = out + R[:, e:e + 1] * (hmid @ w2[e].double().T)
    out.backward(dout.double())
    dx, dw = oracle.moe_backward_input(x, gate, up, w2, ids, wts, dout)
    assert torch.allclose(dx, xd.grad, rtol=1e-10, atol=1e-12)
    assert torch.allclose(dw, wd.grad, rtol=1e-10, atol=1e-12)


def test_out_of_range_id_contributes_nothing():
    x, gate, up, w2, ids, wts, dout = _case(T=4, H=16, I=8, E=3, k=2, seed=3)
    bad = ids.clone()
    bad[1, 0] = 7
    zero_w = wts.clone()
    zero_w[1, 0] = 0.0
    dx_bad, dw_bad = oracle.moe_backward_input(x, gate, up, w2, bad, wts, dout)
    dx_zero, _ = oracle.moe_backward_input(x, gate, up, w2, ids, zero_w, dout)
    assert dw_bad[1, 0] == 0.0
    assert torch.equal(dx_bad, dx_zero)


def test_strided_views_read_like_contiguous_copies():
    x, gate, up, w2, ids, wts, dout = _case(T=4, H=16, I=8, E=3, k=2, seed=4)
    w13 = torch.cat([gate, up], dim=1)  # packed [E, 2I, H]: gate and up are strided views
    dwide = torch.zeros(dout.shape[0], 2 * dout.shape[1])
    dwide[:, ::2] = dout
    a = oracle.moe_backward_input(x, w13[:, :8], w13[:, 8:], w2, ids, wts, dwide[:, ::2])
    b = oracle.moe_backward_input(x, gate, up, w2, ids, wts, dout)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_token_subset_rows_match_full_run():
    x, gate, up, w2, ids, wts, dout = _case(T=6, H=16, I=8, E=3, k=2, seed=6)
    full = oracle.moe_backward_input(x, gate, up, w2, ids, wts, dout)
    toks = torch.tensor([4, 1])
    part = oracle.moe_backward_input(x, gate, up, w2, ids, wts, dout, tokens=toks)
    assert torch.equal(part[0], full[0][toks]) and torch.equal(part[1], full[1][toks])


def test_weight_gradient_matches_central_finite_differences():
    x, gate, up, w2, ids, wts, dout = _case(T=3, H=8, I=4, E=2, k=2, seed=12)
    dg, du, dw2 = oracle.moe_backward_weights(x, gate, up, w2, ids, wts, dout)
    d = 1e-3
    for name, tensor, grad in (("gate", gate, dg), ("up", up, du), ("w2", w2, dw2)):
        num = torch.zeros_like(grad)
        for idx in range(tensor.numel()):
            p, m = tensor.clone(), tensor.clone()
            p.view(-1)[idx] += d
            m.view(-1)[idx] -= d
            step = float(p.view(-1)[idx].double() - m.view(-1)[idx].double())
            args = dict(gate=gate, up=up, w2=w2)
            lp = _loss(x, **{**args, name: p}, ids=ids, wts=wts, dout=dout)
            lm = _loss(x, **{**args, name: m}, ids=ids, wts=wts, dout=dout)
            num.view(-1)[idx] = (lp - lm) / step
        assert (grad - num).abs().max() <= 1e-5 * grad.abs().max(), name


def test_weight_gradient_matches_autograd_of_dense_formulation():
    x, gate, up, w2, ids, wts, dout = _case(T=5, H=24, I=12, E=4, k=3, seed=19)
    g_ = gate.double().requires_grad_(True)
    u_ = up.double().requires_grad_(True)
    d_ = w2.double().requires_grad_(True)
    xd = x.double()
    E = gate.shape[0]
    R = torch.zeros(x.shape[0], E, dtype=torch.float64).index_put(
        (torch.arange(x.shape[0]).repeat_interleave(ids.shape[1]), ids.long().reshape(-1)),
        wts.double().reshape(-1), accumulate=True)
    out = torch.zeros(x.shape[0], x.shape[1], dtype=torch.float64)
    for e in range(E):
        hmid = torch.nn.functional.silu(xd @ g_[e].T) * (xd @ u_[e].T)
        out = out + R[:, e:e + 1] * (hmid @ d_[e].T)
    out.backward(dout.double())
    dg, du, dw2 = oracle.moe_backward_weights(x, gate, up, w2, ids, wts, dout)
    assert torch.allclose(dg, g_.grad, rtol=1e-10, atol=1e-12)
    assert torch.allclose(du, u_.grad, rtol=1e-10, atol=1e-12)
    assert torch.allclose(dw2, d_.grad, rtol=1e-10, atol=1e-12)


def test_unrouted_expert_gets_zero_weight_gradient():
    x, gate, up, w2, ids, wts, dout = _case(T=4, H=16, I=8, E=4, k=1, seed=2)
    ids = torch.zeros_like(ids)  # every token on expert 0
    dg, du, dw2 = oracle.moe_backward_weights(x, gate, up, w2, ids, wts, dout)
    assert dg[1:].abs().max() == 0 and du[1:].abs().max() == 0 and dw2[1:].abs().max() == 0
    assert dg[0].abs().max() > 0
