"""Seeded synthetic workloads for the fused MoE expert forward.

This module only draws inputs: hidden states, expert weights and routing
(ids + weights).  It holds none of the MoE arithmetic.  Both the GPU tests and
the CPU oracle read what it produces, so it imports neither of them.

Shapes follow the pages' workloads:
  * Qwen3-235B-shaped layer: H=4096, I=1536, E=128, top_k=8 (Liger-Kernel
    PR #1377, "Problems": I=1536 worked example; 0.375 GiB per layer of
    retained copies implies 16 local experts x 2*1536*4096 bf16, i.e. H=4096).
  * GLM-4.5-Air-shaped layer: H=4096, I=1408, E=128, top_k=8, routing read as
    the per-layer slice of a [tokens, 46, 8] tensor, token stride 368
    (prime-rl PR #2860, "Problem").
  * Qwen3.5-397B TP2 MXFP4 layer: H=4096, I=512, E=512/top_k=10 and the
    shared-expert-fused E=513/top_k=11 convention (ROCm/aiter PR #3859,
    "Summary" and "Details").

Recipe (fixed seeds): weights seed 0, x seed 1, routing seed 2 (or
1000+T / 2000+T in the token sweep).  Weights are N(0, std=1/sqrt(fan_in))
drawn in fp32 (fan_in = H for w13, I for w2); x is N(0, 1).  Routing draws
N(0, 1) logits, takes softmax, keeps the top-k (lower expert index wins a tie)
and renormalises the kept probabilities to sum to one.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class MoEShape:
    T: int
    H: int
    I: int
    E: int
    k: int


TINY = MoEShape(T=64, H=256, I=128, E=8, k=2)
QWEN3_235B = MoEShape(T=4096, H=4096, I=1536, E=128, k=8)
GLM45_AIR = MoEShape(T=16384, H=4096, I=1408, E=128, k=8)
QWEN35_TP2_MXFP4 = MoEShape(T=4096, H=4096, I=512, E=512, k=10)
QWEN35_TP2_MXFP4_SHARED = MoEShape(T=4096, H=4096, I=512, E=513, k=11)
TOKEN_SWEEP = (1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1023, 1024, 2048, 4096, 4097, 8192, 16384)
MXFP4_TOKEN_SWEEP = (1, 16, 256, 4096, 32768)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_x(T: int, H: int, seed: int = 1, device="cpu") -> torch.Tensor:
    """x ~ N(0, 1) rounded to bf16, [T, H] contiguous."""
    return torch.randn(T, H, generator=_gen(seed, device), device=device).to(torch.bfloat16)


def make_weights_fp32(E: int, I: int, H: int, seed: int = 0, device="cpu"):
    """Packed w13 [E, 2I, H] and w2 [E, H, I] in fp32, std 1/sqrt(fan_in)."""
    g = _gen(seed, device)
    w13 = torch.randn(E, 2 * I, H, generator=g, device=device).mul_(1.0 / math.sqrt(H))
    w2 = torch.randn(E, H, I, generator=g, device=device).mul_(1.0 / math.sqrt(I))
    return w13, w2


def make_weights_bf16(E: int, I: int, H: int, seed: int = 0, device="cpu"):
    """Packed w13 [E, 2I, H] and w2 [E, H, I] bf16, drawn expert by expert in
    fp32 so the full-size tensors never need an fp32 copy at once."""
    g = _gen(seed, device)
    w13 = torch.empty(E, 2 * I, H, dtype=torch.bfloat16, device=device)
    w2 = torch.empty(E, H, I, dtype=torch.bfloat16, device=device)
    for e in range(E):
        w13[e] = torch.randn(2 * I, H, generator=g, device=device).mul_(1.0 / math.sqrt(H))
    for e in range(E):
        w2[e] = torch.randn(H, I, generator=g, device=device).mul_(1.0 / math.sqrt(I))
    return w13, w2


def iter_weights_fp32(E: int, I: int, H: int, seed: int = 0, device="cpu"):
    """Expert by expert: (e, w13_e [2I, H] fp32, w2_e [H, I] fp32), std 1/sqrt(fan_in).
    For MXFP4 layers, whose fp32 weights are quantised once and never held whole."""
    g = _gen(seed, device)
    for e in range(E):
        w13 = torch.randn(2 * I, H, generator=g, device=device).mul_(1.0 / math.sqrt(H))
        w2 = torch.randn(H, I, generator=g, device=device).mul_(1.0 / math.sqrt(I))
        yield e, w13, w2


def gate_up_views(w13: torch.Tensor):
    """gate = w13[:, :I, :], up = w13[:, I:, :]: strided views, no copy
    (Liger-Kernel PR #1377, "Problems")."""
    I = w13.shape[1] // 2
    return w13[:, :I, :], w13[:, I:, :]


def _topk_stable(p: torch.Tensor, k: int):
    # descending by probability, lower index first on ties
    order = torch.sort(-p, dim=1, stable=True).indices[:, :k]
    return order, torch.gather(p, 1, order)


def route_softmax_topk(T: int, E: int, k: int, seed: int = 2, device="cpu"):
    """N(0,1) logits -> softmax -> top-k -> renormalise.  ids int32 [T, k], weights fp32 [T, k]."""
    logits = torch.randn(T, E, generator=_gen(seed, device), device=device, dtype=torch.float32)
    p = torch.softmax(logits.double(), dim=1)
    ids, w = _topk_stable(p, k)
    w = w / w.sum(dim=1, keepdim=True)
    return ids.to(torch.int32).contiguous(), w.to(torch.float32).contiguous()


def route_shared_expert(T: int, E_routed: int, k_routed: int, seed: int = 2, device="cpu"):
    """Shared-expert-fused convention: columns 0..k_routed-1 are the renormalised
    top-k of E_routed experts, column k_routed is expert E_routed with weight 1.0
    (E = E_routed + 1, top_k = k_routed + 1; aiter PR #3859 "Summary")."""
    ids, w = route_softmax_topk(T, E_routed, k_routed, seed, device)
    sid = torch.full((T, 1), E_routed, dtype=torch.int32, device=device)
    sw = torch.ones(T, 1, dtype=torch.float32, device=device)
    return torch.cat([ids, sid], 1).contiguous(), torch.cat([w, sw], 1).contiguous()


def route_zipf_layers(T: int, E: int, k: int, layers: int = 46, alpha: float = 1.2, seed: int = 7,
                      device="cpu"):
    """Skewed routing for every layer of a [T, layers, k] router-replay tensor.

    Expert popularity p_e ~ 1 / rank(e)^alpha with ranks from a seeded
    permutation; per token and layer, k distinct experts by Gumbel-top-k over
    log p (sampling without replacement); weights = softmax of N(0,1) over the
    chosen k.  Returns ids int32 [T, layers, k] and weights fp32 [T, layers, k];
    callers pass the strided slice [:, l, :] (token stride layers*k)."""
    g = _gen(seed, device)
    rank = torch.randperm(E, generator=g, device=device).to(torch.float64) + 1.0
    logp = -alpha * torch.log(rank)
    ids = torch.empty(T, layers, k, dtype=torch.int32, device=device)
    wts = torch.empty(T, layers, k, dtype=torch.float32, device=device)
    for l in range(layers):
        u = torch.rand(T, E, generator=g, device=device, dtype=torch.float64).clamp_(1e-300, 1.0)
        gumbel = -torch.log(-torch.log(u))
        order = torch.sort(-(logp[None, :] + gumbel), dim=1, stable=True).indices[:, :k]
        ids[:, l, :] = order.to(torch.int32)
        z = torch.randn(T, k, generator=g, device=device, dtype=torch.float32)
        wts[:, l, :] = torch.softmax(z, dim=1)
    return ids, wts


def l2_flush_buffer(device, nbytes: int = 512 << 20) -> torch.Tensor:
    """A buffer larger than the B200's 126 MB L2; writing it evicts the cache."""
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def flush_l2(buf: torch.Tensor, i: int) -> None:
    """Evicts the L2 before a timed call: writes the whole buffer (4x the L2),
    then reads back its first three quarters so that the lines just written
    are back in HBM and the cache holds only clean lines.  Without the read,
    the write-back of up to 126 MB of the flush's own dirty lines would fall
    inside the timed call (measured: 12 us of a 74 us decode-size layer)."""
    buf.fill_(i & 0xFF)
    buf[: buf.numel() // 4 * 3].view(torch.int64).sum()
