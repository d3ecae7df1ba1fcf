"""Pins for the fp64 oracle, each against something other than the oracle itself.

* brute force: a dense numpy formulation sum_e R[t, e] * MLP_e(x_t) with a
  routing matrix R (different loop structure, matrix products, no slots);
* special case: top_k = 1 with one expert is the textbook SwiGLU MLP
  (silu(x Wg^T) * (x Wu^T)) Wd^T, computed with torch's own silu and matmul;
* invariants: packed strided w13 equals the .contiguous() copy (Liger-Kernel
  PR #1377, "Problems"), token permutation permutes rows, linearity in the
  routing weights, zero-weight and out-of-range slots contribute nothing, and
  the shared-expert-fused routing (aiter PR #3859, "Summary") equals the routed
  output plus the shared expert's dense MLP;
* align: Python's sorted() by (expert, slot).
"""

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_46_b200 import workloads as wl


def _bf16(t):
    return t.to(torch.bfloat16)


def _dense_reference(x, gate, up, w2, ids, weights):
    """sum_e R[t,e] * (silu(x Wg_e^T) * (x Wu_e^T)) Wd_e^T with numpy fp64."""
    X = x.double().numpy()
    G, U, D = gate.double().numpy(), up.double().numpy(), w2.double().numpy()
    T = X.shape[0]
    E = G.shape[0]
    R = np.zeros((T, E))
    idn, wn = ids.long().numpy(), weights.double().numpy()
    for t in range(T):
        for j in range(idn.shape[1]):
            if 0 <= idn[t, j] < E:
                R[t, idn[t, j]] += wn[t, j]
    out = np.zeros((T, X.shape[1]))
    for e in range(E):
        g = X @ G[e].T
        u = X @ U[e].T
        a = g / (1.0 + np.exp(-g)) * u
        out += R[:, e:e + 1] * (a @ D[e].T)
    return out


def _tiny_inputs(T=6, H=64, I=32, E=4, k=2, seed=11):
    torch.manual_seed(seed)
    x = _bf16(torch.randn(T, H))
    w13 = _bf16(torch.randn(E, 2 * I, H) / H ** 0.5)
    w2 = _bf16(torch.randn(E, H, I) / I ** 0.5)
    ids, wts = wl.route_softmax_topk(T, E, k, seed=seed + 1)
    return x, w13, w2, ids, wts


def test_dense_formulation_matches():
    x, w13, w2, ids, wts = _tiny_inputs()
    gate, up = wl.gate_up_views(w13)
    got, nbad = oracle.moe_forward(x, gate, up, w2, ids, wts)
    ref = _dense_reference(x, gate, up, w2, ids, wts)
    assert nbad == 0
    assert np.max(np.abs(got.numpy() - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_dense_formulation_strided_everything():
    # x stored transposed (stride (1, T)), ids int64 read from a [T, L, k] slice,
    # weights from a [T, L, k] slice, w2 with a padded expert stride.
    T, H, I, E, k, L = 5, 64, 32, 3, 2, 4
    torch.manual_seed(3)
    x = _bf16(torch.randn(H, T)).t()
    assert x.stride() == (1, T)
    w13 = _bf16(torch.randn(E, 2 * I, H) / 8)
    w2big = _bf16(torch.randn(E, H + 3, I) / 6)
    w2 = w2big[:, 1:H + 1, :]
    ids_all = torch.randint(0, E, (T, L, k), dtype=torch.int64)
    w_all = torch.rand(T, L, k, dtype=torch.float32)
    ids, wts = ids_all[:, 2, :], w_all[:, 2, :]
    assert ids.stride() == (L * k, 1)
    gate, up = wl.gate_up_views(w13)
    got, _ = oracle.moe_forward(x, gate, up, w2, ids, wts)
    ref = _dense_reference(x.contiguous(), gate.contiguous(), up.contiguous(), w2.contiguous(),
                           ids.contiguous(), wts.contiguous())
    assert np.max(np.abs(got.numpy() - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_one_expert_is_dense_swiglu_mlp():
    T, H, I = 7, 64, 48
    torch.manual_seed(5)
    x = _bf16(torch.randn(T, H))
    w13 = _bf16(torch.randn(1, 2 * I, H) / 8)
    w2 = _bf16(torch.randn(1, H, I) / 7)
    ids = torch.zeros(T, 1, dtype=torch.int32)
    wts = torch.ones(T, 1, dtype=torch.float32)
    gate, up = wl.gate_up_views(w13)
    got, _ = oracle.moe_forward(x, gate, up, w2, ids, wts)
    xd = x.double()
    ref = (torch.nn.functional.silu(xd @ gate[0].double().T) * (xd @ up[0].double().T)) @ w2[0].double().T
    assert torch.max(torch.abs(got - ref)).item() <= 1e-12 * torch.max(torch.abs(ref)).item()


def test_packed_view_equals_contiguous_copy_bit_identical():
    x, w13, w2, ids, wts = _tiny_inputs(seed=21)
    gate, up = wl.gate_up_views(w13)
    assert not gate.is_contiguous() and gate.stride(0) == 2 * gate.shape[1] * gate.shape[2]
    a, _ = oracle.moe_forward(x, gate, up, w2, ids, wts)
    b, _ = oracle.moe_forward(x, gate.contiguous(), up.contiguous(), w2, ids, wts)
    assert torch.equal(a, b)


def test_swapping_gate_and_up_changes_result():
    # the gate/up halves are not interchangeable: silu is applied to rows [:I] only
    x, w13, w2, ids, wts = _tiny_inputs(seed=22)
    gate, up = wl.gate_up_views(w13)
    a, _ = oracle.moe_forward(x, gate, up, w2, ids, wts)
    b, _ = oracle.moe_forward(x, up, gate, w2, ids, wts)
    assert torch.max(torch.abs(a - b)).item() > 1e-3


def test_token_permutation_permutes_rows():
    x, w13, w2, ids, wts = _tiny_inputs(T=9, seed=31)
    gate, up = wl.gate_up_views(w13)
    perm = torch.randperm(9, generator=torch.Generator().manual_seed(0))
    a, _ = oracle.moe_forward(x, gate, up, w2, ids, wts)
    b, _ = oracle.moe_forward(x[perm].contiguous(), gate, up, w2, ids[perm].contiguous(),
                              wts[perm].contiguous())
    assert torch.equal(a[perm], b)


def test_linear_in_routing_weights_and_zero_weight_slot():
    x, w13, w2, ids, wts = _tiny_inputs(seed=41)
    gate, up = wl.gate_up_views(w13)
    only0 = wts.clone()
    only0[:, 1] = 0.0
    only1 = wts.clone()
    only1[:, 0] = 0.0
    a, _ = oracle.moe_forward(x, gate, up, w2, ids, wts)
    b0, _ = oracle.moe_forward(x, gate, up, w2, ids, only0)
    b1, _ = oracle.moe_forward(x, gate, up, w2, ids, only1)
    assert torch.max(torch.abs(a - (b0 + b1))).item() <= 1e-12 * torch.max(torch.abs(a)).item()
    # a zero-weight column behaves exactly like dropping that column
    c, _ = oracle.moe_forward(x, gate, up, w2, ids[:, :1].contiguous(), wts[:, :1].contiguous())
    assert torch.equal(b0, c)


def test_out_of_range_ids_are_skipped_and_counted():
    x, w13, w2, ids, wts = _tiny_inputs(seed=51)
    gate, up = wl.gate_up_views(w13)
    bad = ids.clone()
    bad[0, 0] = -1
    bad[3, 1] = 4  # E = 4
    a, nbad = oracle.moe_forward(x, gate, up, w2, bad, wts)
    z = wts.clone()
    z[0, 0] = 0.0
    z[3, 1] = 0.0
    b, _ = oracle.moe_forward(x, gate, up, w2, ids, z)
    assert nbad == 2
    assert torch.max(torch.abs(a - b)).item() <= 1e-12 * torch.max(torch.abs(a)).item()


def test_shared_expert_fused_equals_routed_plus_dense():
    T, H, I, E = 6, 64, 32, 5
    torch.manual_seed(61)
    x = _bf16(torch.randn(T, H))
    w13 = _bf16(torch.randn(E + 1, 2 * I, H) / 8)
    w2 = _bf16(torch.randn(E + 1, H, I) / 6)
    ids, wts = wl.route_shared_expert(T, E, 2, seed=5)
    assert torch.all(ids[:, 2] == E) and torch.all(wts[:, 2] == 1.0)
    gate, up = wl.gate_up_views(w13)
    fused, _ = oracle.moe_forward(x, gate, up, w2, ids, wts)
    routed, _ = oracle.moe_forward(x, gate, up, w2, ids[:, :2].contiguous(), wts[:, :2].contiguous())
    xd = x.double()
    shared = (torch.nn.functional.silu(xd @ gate[E].double().T) * (xd @ up[E].double().T)) @ w2[E].double().T
    assert torch.max(torch.abs(fused - routed - shared)).item() <= 1e-12 * torch.max(torch.abs(fused)).item()


def test_token_subset_rows_match_full_run():
    x, w13, w2, ids, wts = _tiny_inputs(T=10, seed=71)
    gate, up = wl.gate_up_views(w13)
    full, _ = oracle.moe_forward(x, gate, up, w2, ids, wts)
    toks = torch.tensor([9, 0, 4])
    sub, _ = oracle.moe_forward(x, gate, up, w2, ids, wts, tokens=toks)
    assert torch.equal(sub, full[toks])


# --------------------------------------------------------------------------- align

def _brute_align(ids, E, bm):
    flat = ids.reshape(-1).long().tolist()
    S = len(flat)
    valid = [(e, s) for s, e in enumerate(flat) if 0 <= e < E]
    order = sorted(valid)  # by (expert, slot)
    counts = [0] * E
    for e, _ in valid:
        counts[e] += 1
    offsets = [0]
    for e in range(E):
        offsets.append(offsets[-1] + -(-counts[e] // bm) * bm)
    sorted_ = [S] * offsets[-1]
    pos = {e: offsets[e] for e in range(E)}
    for e, s in order:
        sorted_[pos[e]] = s
        pos[e] += 1
    block_expert = []
    for e in range(E):
        block_expert += [e] * ((offsets[e + 1] - offsets[e]) // bm)
    return counts, offsets, sorted_, block_expert, S - len(valid)


@pytest.mark.parametrize("T,E,k,bm", [(1, 8, 2, 16), (17, 8, 2, 16), (64, 8, 2, 128), (33, 513, 11, 32),
                                      (100, 128, 8, 64), (0, 4, 2, 16)])
def test_align_matches_brute_force(T, E, k, bm):
    g = torch.Generator().manual_seed(T * 31 + E)
    ids = torch.randint(-1, E + 1, (T, k), generator=g, dtype=torch.int32)
    got = oracle.moe_align(ids, E, bm)
    counts, offsets, sorted_, be, nbad = _brute_align(ids, E, bm)
    assert got["counts"].tolist() == counts
    assert got["offsets"].tolist() == offsets
    assert got["sorted"].tolist() == sorted_
    assert got["block_expert"].tolist() == be
    assert got["num_blocks"] == offsets[-1] // bm
    assert got["n_bad"] == nbad


def test_align_strided_int64_slice():
    T, L, k, E, bm = 40, 46, 8, 16, 16
    ids_all = torch.randint(0, E, (T, L, k), generator=torch.Generator().manual_seed(1))
    ids = ids_all[:, 23, :]
    assert ids.stride() == (368, 1)  # prime-rl PR #2860: 46 layers x top_k 8
    got = oracle.moe_align(ids, E, bm)
    ref = _brute_align(ids.contiguous(), E, bm)
    assert got["sorted"].tolist() == ref[2] and got["counts"].tolist() == ref[0]
