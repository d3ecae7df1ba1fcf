"""GPU parity of the MXFP4 path (aiter PR #3859, "Details": e2m1 weights and
activations with per-1x32 e8m0 scales) against the fp64 oracle.

Bars: the quantiser is bit-exact (codes and scales) against the oracle's; the
forward is within max|y - ref| / max|ref| <= 6e-2 (the oracle quantises the
SwiGLU activation from fp64, the GPU from fp32, so a few codes near rounding
boundaries may differ); strided packed views vs contiguous copies are
bit-identical on the GPU.
"""

import pytest
import torch

import mixture_experts_layer_46_b200 as moe
import oracle
from mixture_experts_layer_46_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MX_TOL = 6e-2


def rel_err(got, ref):
    got = got.double().cpu()
    ref = ref.double().cpu()
    return (got - ref).abs().max().item() / ref.abs().max().item()


def _special_rows(K):
    """Rows exercising ties, saturation, zeros, tiny blocks and negative zeros."""
    rows = []
    base = torch.tensor([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.2, -0.25, -3.5, 0.0, -0.0,
                         4.0, 0.5] * 2)
    rows.append(base)
    rows.append(base * 2.0 ** -20)
    rows.append(torch.zeros(32))
    rows.append(-base * 3.0)
    rows.append(torch.full((32,), 1e-30))
    r = torch.cat(rows)
    reps = (K * 8 + r.numel() - 1) // r.numel()
    return r.repeat(reps)[:K * 8].reshape(8, K)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_bit_exact(dtype):
    g = torch.Generator().manual_seed(3)
    K = 512
    src = torch.randn(64, K, generator=g) * torch.logspace(-6, 6, 64)[:, None]
    src = torch.cat([src, _special_rows(K)]).to(dtype)
    ref_c, ref_s = oracle.mxfp4_quantize(src.float())
    got_c, got_s = moe.quantize_mxfp4(src.cuda())
    torch.cuda.synchronize()
    assert torch.equal(got_s.cpu(), ref_s)
    assert torch.equal(got_c.cpu(), ref_c)


def test_quantize_3d_strided_destination():
    g = torch.Generator().manual_seed(4)
    src = torch.randn(3, 40, 256, generator=g)
    ref_c, ref_s = oracle.mxfp4_quantize(src.reshape(-1, 256))
    codes_big = torch.zeros(3, 48, 128, dtype=torch.uint8, device="cuda")
    scales_big = torch.zeros(3, 48, 16, dtype=torch.uint8, device="cuda")
    codes, scales = codes_big[:, 4:44], scales_big[:, 4:44, :8]  # padded rows and row stride
    d_src = moe.desc(src.cuda())
    d_dst = moe.desc(codes, scales)
    import ctypes
    rc = moe.load().moe_quantize_mxfp4(ctypes.byref(d_src), ctypes.byref(d_dst),
                                       torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(codes.cpu().reshape(-1, 128), ref_c)
    assert torch.equal(scales.cpu().reshape(-1, 8), ref_s)
    assert torch.all(codes_big[:, :4] == 0) and torch.all(scales_big[:, 44:] == 0)
    assert torch.all(scales_big[:, :, 8:] == 0)


def make_mx_case(T, H, I, E, k, seed=0, shared=False):
    x = wl.make_x(T, H, seed=seed + 1)
    c13 = torch.empty(E, 2 * I, H // 2, dtype=torch.uint8)
    s13 = torch.empty(E, 2 * I, H // 32, dtype=torch.uint8)
    c2 = torch.empty(E, H, I // 2, dtype=torch.uint8)
    s2 = torch.empty(E, H, I // 32, dtype=torch.uint8)
    for e, w13e, w2e in wl.iter_weights_fp32(E, I, H, seed=seed):
        c13[e], s13[e] = oracle.mxfp4_quantize(w13e)
        c2[e], s2[e] = oracle.mxfp4_quantize(w2e)
    if shared:
        ids, wts = wl.route_shared_expert(T, E - 1, k - 1, seed=seed + 2)
    else:
        ids, wts = wl.route_softmax_topk(T, E, k, seed=seed + 2)
    return {"x": x, "c13": c13, "s13": s13, "c2": c2, "s2": s2, "ids": ids, "wts": wts}


def mx_oracle(case, tokens=None):
    I = case["c13"].shape[1] // 2
    ref, _ = oracle.moe_forward(case["x"], case["c13"][:, :I], case["c13"][:, I:], case["c2"],
                                case["ids"], case["wts"],
                                scales=(case["s13"][:, :I], case["s13"][:, I:], case["s2"]),
                                tokens=tokens)
    return ref


def mx_gpu(c, contiguous=False):
    I = c["c13"].shape[1] // 2
    if contiguous:
        keep = [c["c13"][:, :I].contiguous(), c["c13"][:, I:].contiguous(),
                c["s13"][:, :I].contiguous(), c["s13"][:, I:].contiguous()]
        v = moe.w13_from_views(keep[0], keep[1], keep[2], keep[3])
    else:
        keep = []
        v = moe.w13_from_packed(c["c13"], c["s13"])
    out = moe.forward(c["x"], v, c["c2"], c["ids"], c["wts"], w2_scale=c["s2"])
    torch.cuda.synchronize()
    del keep
    return out


def cuda_case(case):
    return {k: v.cuda() for k, v in case.items()}


@pytest.mark.parametrize("T,H,I,E,k", [
    (64, 256, 256, 8, 2),
    (200, 512, 512, 16, 4),
    (1, 256, 256, 4, 2),
])
def test_mxfp4_forward_matches_oracle(T, H, I, E, k):
    case = make_mx_case(T, H, I, E, k, seed=T)
    ref = mx_oracle(case)
    got = mx_gpu(cuda_case(case))
    assert rel_err(got, ref) <= MX_TOL


def test_mxfp4_strided_equals_contiguous_and_deterministic():
    c = cuda_case(make_mx_case(150, 512, 256, 8, 4, seed=5))
    a = mx_gpu(c)
    b = mx_gpu(c, contiguous=True)
    d = mx_gpu(c)
    assert torch.equal(a, b)
    assert torch.equal(a, d)


@pytest.mark.parametrize("tile", [32, 96, 128])
def test_mxfp4_scale_load_paths_agree(tile):
    # The GEMMs load e8m0 scale rows by TMA where every scale view is 16-byte
    # aligned and by 4-byte cp.async otherwise: scale views whose rows are 24 bytes
    # apart (8-byte aligned only) take the second path and must give the same bits.
    T, H, I, E, k = 300, 512, 512, 8, 4
    case = make_mx_case(T, H, I, E, k, seed=tile + 5)
    ref = mx_oracle(case)
    c = cuda_case(case)
    s13p = torch.zeros(E, 2 * I, H // 32 + 8, dtype=torch.uint8, device="cuda")
    s13p[:, :, :H // 32] = c["s13"]
    s2p = torch.zeros(E, H, I // 32 + 8, dtype=torch.uint8, device="cuda")
    s2p[:, :, :I // 32] = c["s2"]
    with moe.config_override((T, H, I, E, k), mxfp4=True, tile=tile, fused=0):
        assert moe.get_config(T, H, I, E, k, mxfp4=True)["tile"] == tile
        a = mx_gpu(c)
        v = moe.w13_from_packed(c["c13"], s13p[:, :, :H // 32])
        b = moe.forward(c["x"], v, c["c2"], c["ids"], c["wts"], w2_scale=s2p[:, :, :I // 32])
        torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert rel_err(a, ref) <= MX_TOL


def test_mxfp4_stale_workspace_contents_never_reach_the_output():
    # 0xFF scale bytes are NaN in e8m0: padding rows holding them must not matter
    T, H, I, E, k = 45, 512, 256, 6, 3
    case = make_mx_case(T, H, I, E, k, seed=23)
    ref = mx_oracle(case)
    c = cuda_case(case)
    n = moe.workspace_bytes(T, H, I, E, k, mxfp4=True)
    outs = []
    for fill in (0x00, 0xFF):
        ws = torch.full((n,), fill, dtype=torch.uint8, device="cuda")
        v = moe.w13_from_packed(c["c13"], c["s13"])
        outs.append(moe.forward(c["x"], v, c["c2"], c["ids"], c["wts"], w2_scale=c["s2"], workspace=ws))
        torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    assert rel_err(outs[0], ref) <= MX_TOL


@pytest.mark.parametrize("T,k,strided", [(1, 10, False), (3, 10, True), (4, 8, False), (3, 11, False)])
def test_mxfp4_decode_align_permute_one_launch_matches_two(T, k, strided):
    # at most 32 slots: align and the quantising permute run as one launch
    H, I, E = 512, 256, 24
    case = make_mx_case(T, H, I, E, k, seed=T + 29)
    case["ids"][0, 1] = E                            # skipped slot
    case["ids"][T - 1, 2] = case["ids"][T - 1, 3]    # one expert twice for a token
    ref = mx_oracle(case)
    c = cuda_case(case)
    if strided:
        c["x"] = case["x"].t().contiguous().cuda().t()
    moe.device_errors()
    outs, launches = {}, {}
    for tiny in (1, 0):
        with moe.config_override((T, H, I, E, k), mxfp4=True, tiny=tiny, fused=0):
            outs[tiny] = mx_gpu(c)
            launches[tiny] = moe.last_launch_count()
    nbad, nto = moe.device_errors()
    assert nbad == 2 and nto == 0
    assert torch.equal(outs[1], outs[0])
    assert rel_err(outs[1], ref) <= MX_TOL
    assert launches[0] == 5
    assert launches[1] == (4 if T * k <= 32 else 5)


@pytest.mark.parametrize("T,H,I,E,k,case", [
    (1, 512, 256, 24, 10, "plain"),
    (3, 512, 512, 24, 10, "strided-x"),       # x read through strides by the quantising warp
    (2, 512, 256, 25, 11, "shared"),          # 24 routed + 1 shared expert, top 10 + 1
    (1, 256, 256, 40, 32, "one-expert"),      # all 32 slots to one expert (8 gathers of h rows)
    (2, 256, 256, 8, 4, "no-valid-id"),
])
def test_mxfp4_decode_one_kernel_matches_kernels_and_oracle(T, H, I, E, k, case):
    # at most 32 slots: the MXFP4 forward as one kernel (tokens quantised in the
    # kernel with the permute's rule, h requantised by the GEMM1 epilogue's rule)
    # must give the multi-kernel path's bits with GEMM1 unsplit, and match the
    # oracle with GEMM1 split along K (its fp32 parts summed in part order)
    cs = make_mx_case(T, H, I, E, k, seed=T + k + 307, shared=(case == "shared"))
    if case in ("plain", "strided-x"):
        cs["ids"][0, 1] = E                           # a skipped slot
        cs["ids"][T - 1, 2] = cs["ids"][T - 1, 3]     # one expert twice for a token
    if case == "one-expert":
        cs["ids"][:] = 7
    if case == "no-valid-id":
        cs["ids"][:] = -1
    c = cuda_case(cs)
    if case == "strided-x":
        c["x"] = cs["x"].t().contiguous().cuda().t()
    moe.device_errors()
    outs, launches = {}, {}
    variants = {"unsplit": dict(fused=1, split=1), "kernels": dict(fused=0), "split": dict(fused=1)}
    for name, flags in variants.items():
        with moe.config_override((T, H, I, E, k), mxfp4=True, **flags):
            outs[name] = mx_gpu(c)
            launches[name] = moe.last_launch_count()
            if name == "split":
                assert torch.equal(mx_gpu(c), outs[name])  # fixed part order: deterministic
    nbad, nto = moe.device_errors()
    n_skip = int(((cs["ids"] < 0) | (cs["ids"] >= E)).sum().item())
    assert nbad == 4 * n_skip and nto == 0
    assert launches["unsplit"] == 1 and launches["split"] == 1 and launches["kernels"] == 4
    assert torch.equal(outs["unsplit"], outs["kernels"])
    if case == "no-valid-id":
        assert bool((outs["split"] == 0).all()) and bool((outs["unsplit"] == 0).all())
    else:
        ref = mx_oracle(cs)
        assert rel_err(outs["unsplit"], ref) <= MX_TOL
        assert rel_err(outs["split"], ref) <= MX_TOL


@pytest.mark.parametrize("T,E,k", [(1, 16, 4), (2, 24, 10), (3, 40, 8)])
def test_mxfp4_decode_split_gemm1_each_part_count_matches_oracle(T, E, k):
    # the MXFP4 one-kernel path with GEMM1 split along K into at most 2, 3 and 4
    # parts (H = 4096: 16 k-steps of 256 codes, at least four per part; the
    # cases with few routed experts take the most): each count matches the
    # oracle and repeats its own bits; unsplit equals the multi-kernel path
    H, I = 4096, 256
    cs = make_mx_case(T, H, I, E, k, seed=11 * T + E + k)
    if T > 1:
        cs["ids"][T - 1, 0] = cs["ids"][0, 0]          # an expert shared by two tokens
    c = cuda_case(cs)
    ref = mx_oracle(cs)
    outs = {}
    for split in (1, 2, 3, 4):
        with moe.config_override((T, H, I, E, k), mxfp4=True, fused=1, split=split):
            assert moe.get_config(T, H, I, E, k, mxfp4=True)["split"] == split
            outs[split] = mx_gpu(c)
            assert moe.last_launch_count() == 1
            assert torch.equal(mx_gpu(c), outs[split]), split
        assert rel_err(outs[split], ref) <= MX_TOL, split
    with moe.config_override((T, H, I, E, k), mxfp4=True, fused=0):
        assert torch.equal(mx_gpu(c), outs[1])


@pytest.mark.parametrize("T,H,I,E,k", [
    (300, 512, 512, 8, 4),     # 150 slots per expert: several tiles of each size, ragged last tiles
    (77, 256, 256, 6, 3),
])
def test_mxfp4_token_tile_configs_agree_and_match_oracle(T, H, I, E, k):
    # 32- and 96-row tiles (two accumulator buffers) and 128-row tiles (one) are a
    # performance choice of the block-scaled GEMMs: every one must give the same bits
    case = make_mx_case(T, H, I, E, k, seed=T + 91)
    ref = mx_oracle(case)
    c = cuda_case(case)
    outs = {}
    for tile in (32, 96, 128):
        with moe.config_override((T, H, I, E, k), mxfp4=True, tile=tile):
            assert moe.get_config(T, H, I, E, k, mxfp4=True)["tile"] == tile
            outs[tile] = mx_gpu(c)
        assert rel_err(outs[tile], ref) <= MX_TOL, tile
    assert torch.equal(outs[32], outs[96]) and torch.equal(outs[96], outs[128])


def test_mxfp4_shared_expert_fused_routing():
    # E = 32 routed + 1 shared, top_k = 4 + 1, the 513/11 convention at reduced size
    case = make_mx_case(96, 512, 256, 33, 5, seed=7, shared=True)
    assert torch.all(case["ids"][:, 4] == 32)
    ref = mx_oracle(case)
    got = mx_gpu(cuda_case(case))
    assert rel_err(got, ref) <= MX_TOL


def _tp2_case(tp2_weights, T, shared, seed_x, seed_r):
    s = wl.QWEN35_TP2_MXFP4_SHARED if shared else wl.QWEN35_TP2_MXFP4
    E = s.E
    cw, gw = tp2_weights["cpu"], tp2_weights["gpu"]
    x = wl.make_x(T, s.H, seed=seed_x)
    if shared:
        ids, wts = wl.route_shared_expert(T, E - 1, s.k - 1, seed=seed_r)
    else:
        ids, wts = wl.route_softmax_topk(T, E, s.k, seed=seed_r)
    cpu = {"x": x, "ids": ids, "wts": wts}
    gpu = {"x": x.cuda(), "ids": ids.cuda(), "wts": wts.cuda()}
    for key in ("c13", "s13", "c2", "s2"):
        cpu[key] = cw[key][:E]
        gpu[key] = gw[key][:E]
    return s, cpu, gpu


def _mx_sample(T, ids, E, n, seed):
    g = torch.Generator().manual_seed(seed)
    ids = ids.long()
    counts = torch.bincount(ids.flatten(), minlength=E)
    routed = torch.nonzero(counts > 0).flatten()
    light = routed[torch.argsort(counts[routed], stable=True)[:4]]
    parts = [torch.randperm(T, generator=g)[:n], torch.arange(min(16, T)),
             torch.arange(max(0, T - 16), T)]
    parts += [torch.nonzero((ids == e).any(dim=1)).flatten()[:4] for e in light.tolist()]
    return torch.unique(torch.cat(parts))


@pytest.mark.slow
@pytest.mark.parametrize("shared", [False, True])
def test_qwen35_tp2_mxfp4_full_size_sampled(tp2_weights, shared):
    s, cpu, gpu = _tp2_case(tp2_weights, 4096, shared, seed_x=1, seed_r=2)
    got = mx_gpu(gpu)
    toks = _mx_sample(s.T, cpu["ids"], s.E, 96, 11)
    ref = mx_oracle(cpu, tokens=toks)
    assert rel_err(got.cpu()[toks], ref) <= MX_TOL


@pytest.mark.slow
@pytest.mark.parametrize("T", [1, 16, 32768])
@pytest.mark.parametrize("shared", [False, True])
def test_qwen35_tp2_mxfp4_token_sweep(tp2_weights, T, shared):
    # the MXFP4 token buckets at full width (E = 512 / top-10 and the 513 / 11
    # shared-expert-fused routing): T = 1 and 16 run the decode path (32-row
    # tiles, one-launch align + quantising permute for T = 1), T = 32768 the
    # 96-row tiles; all tokens up to 16, else a sample
    s, cpu, gpu = _tp2_case(tp2_weights, T, shared, seed_x=2000 + T, seed_r=1000 + T)
    got = mx_gpu(gpu)
    toks = None if T <= 16 else _mx_sample(T, cpu["ids"], s.E, 48, T)
    ref = mx_oracle(cpu, tokens=toks)
    g = got.cpu() if toks is None else got.cpu()[toks]
    assert rel_err(g, ref) <= MX_TOL
    assert torch.isfinite(got.float()).all()


def _ws_forward(case, T, H, I, E, k):
    """moe_forward_ws with a caller workspace on the multi-kernel path (whose grouped
    buffers live in the workspace); returns (out, workspace, layout)."""
    c = cuda_case(case)
    n = moe.workspace_bytes(T, H, I, E, k, mxfp4=True)
    ws = torch.full((n,), 0xAB, dtype=torch.uint8, device="cuda")
    v = moe.w13_from_packed(c["c13"], c["s13"])
    with moe.config_override((T, H, I, E, k), mxfp4=True, fused=0):
        out = moe.forward(c["x"], v, c["c2"], c["ids"], c["wts"], w2_scale=c["s2"], workspace=ws)
        torch.cuda.synchronize()
    return out, ws, moe.workspace_layout(T, H, I, E, k, mxfp4=True)


def _region(ws, off, rows, cols, dtype=torch.uint8):
    nbytes = rows * cols * torch.tensor([], dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype).view(rows, cols).cpu()


@pytest.mark.parametrize("T,H,I,E,k", [
    (200, 512, 256, 16, 4),    # single-CTA align, quantising permute kernel
    (3, 512, 256, 24, 10),     # at most 32 slots: align and quantising permute in one launch
    (700, 256, 256, 8, 8),     # multi-CTA align (5600 slots)
])
def test_permute_quant_grouped_codes_bit_exact(T, H, I, E, k):
    # every routed slot's grouped row holds the oracle's 1x32 codes and scales of
    # its token's x row, at the row the oracle's align gives it (inv bit-exact)
    case = make_mx_case(T, H, I, E, k, seed=T + 61)
    case["ids"][0, 1] = E                          # a skipped slot
    _, ws, L = _ws_forward(case, T, H, I, E, k)
    S = T * k
    inv = _region(ws, L["inv"], 1, S, torch.int32).flatten()
    ref_al = oracle.moe_align(case["ids"], E, 32)
    want_inv = torch.full((S,), -1, dtype=torch.int32)
    want_inv[ref_al["sorted"][ref_al["sorted"] < S].long()] = torch.nonzero(
        ref_al["sorted"] < S).flatten().to(torch.int32)
    assert torch.equal(inv, want_inv)
    rows = L["rows"]
    codes = _region(ws, L["a1"], rows, H // 2)
    scales = _region(ws, L["a1_scale"], rows, H // 32)
    ref_c, ref_s = oracle.mxfp4_quantize(case["x"].float())
    valid = inv >= 0
    assert int(valid.sum()) == S - 1
    slot_tok = torch.arange(S)[valid] // k
    assert torch.equal(codes[inv[valid].long()], ref_c[slot_tok])
    assert torch.equal(scales[inv[valid].long()], ref_s[slot_tok])


@pytest.mark.parametrize("T,H,I,E,k", [
    (200, 512, 512, 16, 4),    # 96-row token tiles
    (2, 512, 256, 24, 10),     # decode: 32-row tiles
])
def test_gemm1_h_requantisation_bit_exact(T, H, I, E, k):
    # GEMM1's epilogue quantises its fp32 SwiGLU output per 1x32 block along I; the
    # captured fp32 values quantised by the oracle must give the same codes and scales
    case = make_mx_case(T, H, I, E, k, seed=T + 71)
    L = moe.workspace_layout(T, H, I, E, k, mxfp4=True)
    cap = torch.full((L["rows"], I), float("nan"), dtype=torch.float32, device="cuda")
    moe.debug_capture(moe.MOE_CAPTURE_H_PREQUANT, cap)
    try:
        out, ws, L = _ws_forward(case, T, H, I, E, k)
    finally:
        moe.debug_capture(moe.MOE_CAPTURE_H_PREQUANT, None)
    S = T * k
    inv = _region(ws, L["inv"], 1, S, torch.int32).flatten()
    rows = inv[inv >= 0].long()
    assert rows.numel() == S
    h = cap.cpu()[rows]
    assert torch.isfinite(h).all()
    codes = _region(ws, L["h"], L["rows"], I // 2)[rows]
    scales = _region(ws, L["h_scale"], L["rows"], I // 32)[rows]
    ref_c, ref_s = oracle.mxfp4_quantize(h.contiguous())
    assert torch.equal(scales, ref_s)
    assert torch.equal(codes, ref_c)
    # and the capture did not change the result
    out2, _, _ = _ws_forward(case, T, H, I, E, k)
    assert torch.equal(out, out2)
