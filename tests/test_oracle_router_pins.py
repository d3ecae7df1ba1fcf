"""Pins for the oracle's router (softmax over the experts, the k most probable,
renormalised; the shared-expert-fused convention of aiter PR #3859, "Summary":
expert=513 / topk=11 next to the unfused expert=512 / topk=10).

Each pin checks the oracle against something other than itself:
* torch's softmax and stable sort (library routines) on random logits;
* a brute-force Python selection on tiny inputs (every k-subset scored);
* exact ties resolved to the lower expert index;
* invariants: adding a constant to a row's logits changes nothing, renormalised
  weights sum to one, unrenormalised weights are the softmax probabilities;
* the seeded routing generator every other test uses (workloads.route_softmax_topk
  and route_shared_expert) agrees with the oracle on the generator's own logits.
"""

import itertools
import math

import pytest
import torch

import oracle
from mixture_experts_layer_46_b200 import workloads as wl


def _torch_router(logits, k, renormalize=True):
    p = torch.softmax(logits.double(), dim=1)
    order = torch.sort(-p, dim=1, stable=True).indices[:, :k]
    w = torch.gather(p, 1, order)
    if renormalize:
        w = w / w.sum(dim=1, keepdim=True)
    return order.to(torch.int32), w


@pytest.mark.parametrize("T,E,k", [(64, 8, 2), (33, 128, 8), (7, 512, 10), (3, 1024, 32), (5, 6, 6)])
@pytest.mark.parametrize("renorm", [True, False])
def test_router_matches_torch_softmax_and_stable_sort(T, E, k, renorm):
    g = torch.Generator().manual_seed(T * E + k)
    logits = torch.randn(T, E, generator=g) * 3.0
    ids, w = oracle.router_topk(logits, k, renormalize=renorm)
    rid, rw = _torch_router(logits, k, renorm)
    assert torch.equal(ids, rid)
    assert torch.allclose(w, rw, rtol=1e-12, atol=0)


def test_router_brute_force_subsets():
    g = torch.Generator().manual_seed(5)
    for trial in range(20):
        E, k = 6, 3
        logits = torch.randn(1, E, generator=g)
        ids, w = oracle.router_topk(logits, k)
        z = sum(math.exp(float(v)) for v in logits[0])
        p = [math.exp(float(v)) / z for v in logits[0]]
        # the best subset maximises the summed probability; order inside it is by p
        best = max(itertools.combinations(range(E), k), key=lambda s: sum(p[i] for i in s))
        want = sorted(best, key=lambda i: (-p[i], i))
        assert ids[0].tolist() == want
        tot = sum(p[i] for i in want)
        for j, i in enumerate(want):
            assert abs(float(w[0, j]) - p[i] / tot) < 1e-12


def test_router_ties_go_to_the_lower_index():
    logits = torch.tensor([[1.0, 3.0, 3.0, 0.5, 3.0, -2.0],
                           [0.0, 0.0, 0.0, 0.0, 0.0, 0.0]])
    ids, w = oracle.router_topk(logits, 4)
    assert ids[0].tolist() == [1, 2, 4, 0]
    assert ids[1].tolist() == [0, 1, 2, 3]
    assert torch.allclose(w[1], torch.full((4,), 0.25, dtype=torch.float64), rtol=0, atol=1e-15)


def test_router_invariants():
    g = torch.Generator().manual_seed(9)
    # multiples of 2^-12 below 16 in magnitude: adding 7.25 is exact in fp32
    logits = torch.round(torch.randn(40, 64, generator=g) * 4096.0) / 4096.0
    ids, w = oracle.router_topk(logits, 8)
    ids2, w2 = oracle.router_topk(logits + 7.25, 8)  # shift invariance
    assert torch.equal(ids, ids2)
    assert torch.allclose(w, w2, rtol=1e-12, atol=0)
    assert torch.allclose(w.sum(1), torch.ones(40, dtype=torch.float64), rtol=0, atol=1e-12)
    _, wp = oracle.router_topk(logits, 8, renormalize=False)
    p = torch.softmax(logits.double(), 1)
    assert torch.allclose(wp, torch.gather(p, 1, ids.long()), rtol=1e-12, atol=0)
    assert bool((w[:, :-1] >= w[:, 1:]).all())   # descending weights


def test_router_strided_and_bf16_logits():
    g = torch.Generator().manual_seed(11)
    big = torch.randn(30, 3, 128, generator=g)
    view = big[:, 1, :]                      # token stride 384
    a = oracle.router_topk(view, 8)
    b = oracle.router_topk(view.contiguous(), 8)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    lb = view.to(torch.bfloat16)
    c = oracle.router_topk(lb, 8)
    d = _torch_router(lb.double(), 8)
    assert torch.equal(c[0], d[0]) and torch.allclose(c[1], d[1], rtol=1e-12, atol=0)


def test_router_shared_expert_column():
    g = torch.Generator().manual_seed(13)
    logits = torch.randn(17, 512, generator=g)
    ids, w = oracle.router_topk(logits, 10, shared_expert=True)
    base_ids, base_w = oracle.router_topk(logits, 10)
    assert ids.shape == (17, 11)
    assert torch.all(ids[:, 10] == 512) and torch.all(w[:, 10] == 1.0)
    assert torch.equal(ids[:, :10], base_ids) and torch.equal(w[:, :10], base_w)


def test_router_agrees_with_the_seeded_routing_generator():
    # the generator draws its logits from this seeded stream and routes them itself
    T, E, k, seed = 64, 8, 2, 2
    logits = torch.randn(T, E, generator=torch.Generator().manual_seed(seed))
    gi, gw = wl.route_softmax_topk(T, E, k, seed=seed)
    ids, w = oracle.router_topk(logits, k)
    assert torch.equal(ids, gi)
    assert torch.allclose(w.float(), gw, rtol=0, atol=1e-7)
    si, sw = wl.route_shared_expert(20, 512, 10, seed=3)
    l2 = torch.randn(20, 512, generator=torch.Generator().manual_seed(3))
    ids2, w2 = oracle.router_topk(l2, 10, shared_expert=True)
    assert torch.equal(ids2, si)
    assert torch.allclose(w2.float(), sw, rtol=0, atol=1e-7)


def test_router_rejects_k_above_E():
    with pytest.raises(ValueError):
        oracle.router_topk(torch.zeros(2, 4), 5)
