"""GPU parity of the router (moe_router_topk) against the fp64 oracle router.

Bars: the chosen experts are bit-exact (the kernel compares fp32 logits; the
oracle orders fp64 softmax probabilities of the same values, and softmax is
monotonic, so both take the same decision), ties going to the lower index;
weights within a relative 1e-5: each weight is exp(l - l_max) / sum in fp32,
whose error is at most (|spread| + 40) * 2^-24 relative for a logit spread
|spread| (the fp32 subtraction, expf's 2 ulp, and at most 37 fp32 additions per
sum), i.e. below 1e-5 for the spreads below 100 used here.

The routing feeds the forward with no copy: the router writes the per-layer
slice of a [T, layers, k] routing tensor (prime-rl PR #2860, "Problem") and the
shared-expert column of the 513/11 convention (aiter PR #3859, "Summary").
"""

import pytest
import torch

import mixture_experts_layer_46_b200 as moe
import oracle
from mixture_experts_layer_46_b200 import workloads as wl

pytestmark = pytest.mark.gpu

W_RTOL = 1e-5


def check(logits_cpu, k, renorm, shared, ids, wts):
    rid, rw = oracle.router_topk(logits_cpu, k, renormalize=renorm, shared_expert=shared)
    got_ids = ids.cpu().to(torch.int32)
    assert torch.equal(got_ids, rid)
    got_w = wts.cpu().double()
    assert torch.all((got_w - rw).abs() <= W_RTOL * rw.abs())


@pytest.mark.parametrize("T,E,k,shared,renorm,ldt,idt", [
    (64, 8, 2, False, True, torch.float32, torch.int32),       # tiny layer's routing
    (4096, 128, 8, False, True, torch.float32, torch.int32),   # Qwen3-235B-shaped layer
    (257, 512, 10, True, True, torch.float32, torch.int32),    # 513/11 shared-expert-fused
    (33, 512, 10, False, False, torch.bfloat16, torch.int64),  # unrenormalised, bf16 logits
    (5, 1024, 32, False, True, torch.float32, torch.int32),    # widest expert count, k = 32
    (100, 40, 31, True, True, torch.bfloat16, torch.int32),    # 32 output columns
    (3, 6, 6, False, True, torch.float32, torch.int32),        # k = E
])
def test_router_matches_oracle(T, E, k, shared, renorm, ldt, idt):
    g = torch.Generator().manual_seed(T + E + k)
    logits = (torch.randn(T, E, generator=g) * 3.0).to(ldt)
    ids, wts = moe.router_topk(logits.cuda(), k, renormalize=renorm, shared_expert=shared,
                               id_dtype=idt)
    torch.cuda.synchronize()
    assert ids.dtype == idt
    check(logits, k, renorm, shared, ids, wts)


def test_router_exact_ties_and_nan():
    g = torch.Generator().manual_seed(3)
    # few distinct values: many exact ties, including -0.0 against +0.0
    logits = torch.round(torch.randn(300, 64, generator=g) * 2.0) / 2.0
    logits[logits == 0] = -0.0
    logits[::7, 5] = 0.0
    ids, wts = moe.router_topk(logits.cuda(), 8)
    torch.cuda.synchronize()
    check(logits, 8, True, False, ids, wts)
    # NaN ranks below every number: never chosen while numbers remain
    ln = torch.randn(16, 32, generator=g)
    ln[:, ::2] = float("nan")
    ids, _ = moe.router_topk(ln.cuda(), 8)
    assert bool((ids.cpu() % 2 == 1).all())


def test_router_strided_inputs_and_replay_slice_outputs():
    T, E, k, L, layer = 1000, 128, 8, 46, 23
    g = torch.Generator().manual_seed(7)
    logits_t = torch.randn(E, T, generator=g) * 2.0
    logits = logits_t.t()                              # strides (1, T): column-major
    ids_all = torch.full((T, L, k), -5, dtype=torch.int32, device="cuda")
    w_all = torch.full((T, L, k), -5.0, dtype=torch.float32, device="cuda")
    ids, wts = ids_all[:, layer, :], w_all[:, layer, :]
    assert ids.stride() == (L * k, 1)
    moe.router_topk(logits_t.cuda().t(), k, topk_ids=ids, topk_weights=wts)
    torch.cuda.synchronize()
    check(logits.contiguous(), k, True, False, ids, wts)
    # nothing outside the slice is touched
    assert bool((ids_all[:, :layer] == -5).all()) and bool((ids_all[:, layer + 1:] == -5).all())
    assert bool((w_all[:, :layer] == -5.0).all())


def test_router_then_forward_on_the_same_stream_decode():
    # the ids are written by the kernel just before the forward; at these sizes
    # GEMM1 requests weights from the ids before align has finished, and must
    # still use align's experts: outputs equal the unprefetched forward bit for bit
    H, I, E, k = 512, 384, 64, 8
    w13, w2 = wl.make_weights_bf16(E, I, H, seed=4, device="cuda")
    v = moe.w13_from_packed(w13)
    moe.device_errors()
    for trial in range(24):
        T = 1 + trial % 4
        x = wl.make_x(T, H, seed=100 + trial, device="cuda")
        logits = torch.randn(T, E, generator=torch.Generator().manual_seed(trial)).cuda() * 2.0
        ids = torch.zeros(T, k, dtype=torch.int32, device="cuda")
        wts = torch.zeros(T, k, dtype=torch.float32, device="cuda")
        outs = {}
        for name, flags in (("prefetch", dict(prefetch=1, fused=0)),
                            ("no-prefetch", dict(prefetch=0, fused=0)),
                            ("one-kernel", dict(fused=1, split=1))):
            with moe.config_override((T, H, I, E, k), **flags):
                ids.fill_(0)                     # stale routing the prefetch could see
                moe.router_topk(logits, k, topk_ids=ids, topk_weights=wts)
                outs[name] = moe.forward(x, v, w2, ids, wts)
                torch.cuda.synchronize()
        assert torch.equal(outs["prefetch"], outs["no-prefetch"]), trial
        assert torch.equal(outs["one-kernel"], outs["no-prefetch"]), trial
        outs[1] = outs["prefetch"]
        if trial < 4:
            rid, rw = oracle.router_topk(logits.cpu(), k)
            gate, up = wl.gate_up_views(w13.cpu())
            ref, _ = oracle.moe_forward(x.cpu(), gate, up, w2.cpu(), rid, rw.float())
            err = (outs[1].double().cpu() - ref).abs().max() / ref.abs().max()
            assert err <= 1e-2
    nbad, nto = moe.device_errors()
    assert nbad == 0 and nto == 0
