"""Pins for the oracle's MXFP4 arithmetic (aiter PR #3859, "Details": e2m1
weights and activations with per-1x32 e8m0 scales).

The pages name the format only, so the pins come from the format's public
definition (OCP Microscaling Formats v1.0) and from mathematics:
* the e2m1 value of every code, from its bit fields by a formula written here;
* e8m0 decoding against torch's own float8_e8m0fnu conversion;
* round-to-nearest-even worked examples on the e2m1 grid and scale examples
  (tests/golden/mxfp4_examples.json);
* brute force: every chosen code is the nearest of all 16 codes to v/2^s, ties
  to the even mantissa; idempotence; grid values round-trip exactly;
* the MXFP4 forward against a dense numpy formulation whose quantiser is the
  brute-force one above.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_46_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp4_examples.json")


def _e2m1_formula(code):
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else (2.0 ** (e - 1)) * (1.0 + m / 2.0)
    return -mag if s else mag


def test_e2m1_values_from_bit_fields():
    for c in range(16):
        assert oracle.e2m1_value(c) == _e2m1_formula(c)
    with open(GOLDEN) as f:
        gold = json.load(f)
    assert [oracle.e2m1_value(c) for c in range(8)] == gold["e2m1_positive_values"]


def test_e8m0_decode_matches_torch():
    # the oracle's scale decoding against torch's own float8_e8m0fnu conversion,
    # for every finite code (255 is NaN and never produced)
    codes = torch.arange(0, 255, dtype=torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).to(torch.float64)
    got = torch.tensor([oracle.e8m0_value(int(c)) for c in codes], dtype=torch.float64)
    assert torch.equal(got, ref)


def _brute_quant_block(v):
    """Nearest of the 16 e2m1 codes to v/2^s (ties: even mantissa), with the
    shared exponent s = floor(log2(amax)) - 2 found by search."""
    amax = max(abs(float(a)) for a in v)
    if amax == 0.0:
        return [8 if np.signbit(a) else 0 for a in v], 0
    s = -200
    while 2.0 ** (s + 1) <= amax:  # largest s with 2^s <= amax
        s += 1
    s -= 2
    s = max(-127, min(127, s))
    vals = [_e2m1_formula(c) for c in range(16)]
    codes = []
    for a in v:
        q = float(a) / 2.0 ** s
        q = max(-6.0, min(6.0, q))
        best = None
        for c in range(16):
            if (c >> 3) != (1 if np.signbit(a) else 0):
                continue
            d = abs(q - vals[c])
            key = (d, c & 1)  # distance, then prefer even mantissa
            if best is None or key < best[0]:
                best = (key, c)
        codes.append(best[1])
    return codes, s + 127


def _unpack(codes_row):
    out = []
    for b in codes_row.tolist():
        out += [b & 15, b >> 4]
    return out


def test_worked_rounding_examples():
    with open(GOLDEN) as f:
        gold = json.load(f)
    for v, want in gold["rne_examples"]:
        block = torch.zeros(1, 32)
        block[0, 0] = 6.0  # amax 6 -> shared exponent 0, so elements are rounded as given
        block[0, 1] = v
        block[0, 2] = -v
        codes, scales = oracle.mxfp4_quantize(block)
        c = _unpack(codes[0])
        assert int(scales[0, 0]) == 127
        assert oracle.e2m1_value(c[1]) == want, (v, c[1])
        assert oracle.e2m1_value(c[2]) == -want
    for amax, code in gold["scale_examples"]:
        block = torch.zeros(1, 32)
        block[0, 5] = amax
        _, scales = oracle.mxfp4_quantize(block)
        assert int(scales[0, 0]) == code, (amax, int(scales[0, 0]))


def test_quantiser_matches_brute_force():
    g = torch.Generator().manual_seed(9)
    src = torch.randn(24, 64, generator=g) * torch.logspace(-3, 3, 24)[:, None]
    src[3, :32] = 0.0
    src[5, 7] = 6.0 * 2 ** -3  # exact grid point
    codes, scales = oracle.mxfp4_quantize(src)
    for r in range(src.shape[0]):
        cr = _unpack(codes[r])
        for b in range(2):
            want_c, want_s = _brute_quant_block(src[r, 32 * b:32 * b + 32].tolist())
            assert int(scales[r, b]) == want_s
            assert cr[32 * b:32 * b + 32] == want_c


def test_idempotent_and_grid_roundtrip():
    g = torch.Generator().manual_seed(10)
    src = torch.randn(8, 96, generator=g)
    codes, scales = oracle.mxfp4_quantize(src)
    deq = torch.empty_like(src)
    for r in range(8):
        cr = _unpack(codes[r])
        for i in range(96):
            deq[r, i] = oracle.e2m1_value(cr[i]) * 2.0 ** (int(scales[r, i // 32]) - 127)
    codes2, scales2 = oracle.mxfp4_quantize(deq)
    # a dequantised block whose amax shrank keeps its codes only when the
    # shared exponent is unchanged; blocks containing a +-4 or +-6 keep it.
    same = [r for r in range(8) for b in range(3)
            if int(scales2[r, b]) == int(scales[r, b])]
    assert len(same) > 0
    for r in range(8):
        for b in range(3):
            if int(scales2[r, b]) == int(scales[r, b]):
                assert codes2[r, 16 * b:16 * b + 16].tolist() == codes[r, 16 * b:16 * b + 16].tolist()
    # every e2m1 grid value times 2^s is represented exactly
    grid = torch.tensor([[_e2m1_formula(c) for c in range(16)] * 2], dtype=torch.float32) * 0.25
    c, s = oracle.mxfp4_quantize(grid)
    back = [oracle.e2m1_value(x) * 2.0 ** (int(s[0, 0]) - 127) for x in _unpack(c[0])]
    assert back == grid[0].tolist()


def _np_fake_quant(v):
    out = np.empty_like(v)
    for b in range(0, v.shape[0], 32):
        codes, sc = _brute_quant_block(v[b:b + 32].tolist())
        out[b:b + 32] = [_e2m1_formula(c) * 2.0 ** (sc - 127) for c in codes]
    return out


def test_mxfp4_forward_matches_dense_with_brute_force_quantiser():
    T, H, I, E, k = 3, 64, 32, 3, 2
    torch.manual_seed(77)
    x = torch.randn(T, H).to(torch.bfloat16)
    w13f = torch.randn(E, 2 * I, H) / 8
    w2f = torch.randn(E, H, I) / 6
    ids, wts = wl.route_softmax_topk(T, E, k, seed=78)
    c13, s13 = oracle.mxfp4_quantize(w13f.reshape(-1, H))
    c2, s2 = oracle.mxfp4_quantize(w2f.reshape(-1, I))
    c13 = c13.reshape(E, 2 * I, H // 2)
    s13 = s13.reshape(E, 2 * I, H // 32)
    c2 = c2.reshape(E, H, I // 2)
    s2 = s2.reshape(E, H, I // 32)
    got, _ = oracle.moe_forward(x, c13[:, :I], c13[:, I:], c2, ids, wts,
                                scales=(s13[:, :I], s13[:, I:], s2))

    def deq(c, s, K):
        vals = np.array([_e2m1_formula(v) for v in range(16)])
        lo, hi = (c & 15).numpy(), (c >> 4).numpy()
        codes = np.stack([lo, hi], -1).reshape(*c.shape[:-1], K)
        sc = np.repeat(2.0 ** (s.numpy().astype(np.float64) - 127), 32, axis=-1)
        return vals[codes] * sc

    W13 = deq(c13, s13, H)
    W2 = deq(c2, s2, I)
    X = np.stack([_np_fake_quant(r) for r in x.double().numpy()])
    ref = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            g = W13[e, :I] @ X[t]
            u = W13[e, I:] @ X[t]
            a = _np_fake_quant(g / (1 + np.exp(-g)) * u)
            ref[t] += float(wts[t, j]) * (W2[e] @ a)
    assert np.max(np.abs(got.numpy() - ref)) <= 1e-12 * np.max(np.abs(ref))
