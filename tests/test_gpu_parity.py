"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Bars (the precision bounds stated for the method):
  * align: counts, offsets, slot permutation and block map bit-exact;
  * forward (bf16): max|y - ref| / max|ref| <= 1e-2;
  * strided packed w13 views vs .contiguous() copies: bit-identical outputs
    (Liger-Kernel PR #1377, "Testing Done": packed views match contiguous weights);
  * run-to-run bit-identical.
"""

import pytest
import torch

import mixture_experts_layer_46_b200 as moe
import oracle
from mixture_experts_layer_46_b200 import workloads as wl

pytestmark = pytest.mark.gpu

BF16_TOL = 1e-2


def rel_err(got: torch.Tensor, ref: torch.Tensor) -> float:
    got = got.double().cpu()
    ref = ref.double().cpu()
    return (got - ref).abs().max().item() / ref.abs().max().item()


def make_case(T, H, I, E, k, seed=0, device="cuda"):
    x = wl.make_x(T, H, seed=seed + 1)
    w13, w2 = wl.make_weights_bf16(E, I, H, seed=seed)
    ids, wts = wl.route_softmax_topk(T, E, k, seed=seed + 2)
    return {"x": x, "w13": w13, "w2": w2, "ids": ids, "wts": wts}


def to_cuda(case):
    return {k: v.cuda() for k, v in case.items()}


def run_gpu(c, contiguous=False, out=None, ws=None):
    gate, up = wl.gate_up_views(c["w13"])
    if contiguous:
        # descriptors hold raw pointers: keep the copies alive until the forward is done
        gc, uc = gate.contiguous(), up.contiguous()
        v = moe.w13_from_views(gc, uc)
        res = moe.forward(c["x"], v, c["w2"], c["ids"], c["wts"], out=out, workspace=ws)
        torch.cuda.synchronize()
        del gc, uc
        return res
    v = moe.w13_from_packed(c["w13"])
    res = moe.forward(c["x"], v, c["w2"], c["ids"], c["wts"], out=out, workspace=ws)
    torch.cuda.synchronize()
    return res


def run_oracle(case, tokens=None):
    gate, up = wl.gate_up_views(case["w13"])
    ref, _ = oracle.moe_forward(case["x"], gate, up, case["w2"], case["ids"], case["wts"],
                                tokens=tokens)
    return ref


# ----------------------------------------------------------------------------- align

@pytest.mark.parametrize("T,E,k,bm,idt", [
    (64, 8, 2, 128, torch.int32),      # tiny config
    (1, 128, 8, 128, torch.int32),     # decode
    (37, 16, 4, 16, torch.int64),      # int64 ids, small block
    (4096, 128, 8, 128, torch.int32),  # multi-CTA path (32768 slots)
    (3000, 513, 11, 64, torch.int32),  # shared-expert-fused routing width
    (512, 128, 8, 32, torch.int32),    # largest single-CTA size class (4096 slots)
    (2000, 128, 8, 32, torch.int32),   # multi-CTA, ragged last chunk (16000 slots)
    (400, 1024, 8, 32, torch.int32),   # widest expert count, one CTA
    (5000, 1024, 8, 32, torch.int64),  # widest expert count, multi-CTA
])
def test_align_bit_exact(T, E, k, bm, idt):
    if E == 513:
        ids, _ = wl.route_shared_expert(T, 512, 10, seed=5)
    else:
        ids, _ = wl.route_softmax_topk(T, E, k, seed=T)
    ids = ids.to(idt)
    ref = oracle.moe_align(ids, E, bm)
    got = moe.align(ids.cuda(), E, bm)
    torch.cuda.synchronize()
    assert got["counts"].cpu().tolist() == ref["counts"].tolist()
    assert got["offsets"].cpu().tolist() == ref["offsets"].tolist()
    assert got["num_blocks"] == ref["num_blocks"]
    assert torch.equal(got["sorted"].cpu(), ref["sorted"])
    assert torch.equal(got["block_expert"].cpu(), ref["block_expert"])


def test_align_strided_slice_and_bad_ids():
    ids_all, _ = wl.route_zipf_layers(2000, 128, 8, layers=46, seed=7)
    assert ids_all[:, 23, :].stride() == (368, 1)
    ids_all[5, 23, 3] = -1
    ids_all[17, 23, 0] = 128
    ids = ids_all[:, 23, :]
    ref = oracle.moe_align(ids, 128, 128)
    moe.device_errors()  # clear
    got = moe.align(ids_all.cuda()[:, 23, :], 128, 128)
    nbad, nto = moe.device_errors()
    assert torch.equal(got["sorted"].cpu(), ref["sorted"])
    assert got["counts"].cpu().tolist() == ref["counts"].tolist()
    assert nbad == 2 and nto == 0


# ----------------------------------------------------------------------------- forward

def test_forward_tiny_config_full_oracle():
    s = wl.TINY
    case = make_case(s.T, s.H, s.I, s.E, s.k)
    ref = run_oracle(case)
    got = run_gpu(to_cuda(case))
    assert rel_err(got, ref) <= BF16_TOL
    assert moe.last_launch_count() >= 5


@pytest.mark.parametrize("T,H,I,E,k", [
    (300, 512, 384, 16, 4),   # several row blocks, 3 gate/up column tiles, 2 down tiles
    (77, 288, 96, 6, 3),      # ragged K (288 = 4.5 x 64), partial N tiles for both GEMMs
    (1, 256, 128, 8, 2),      # one token
    (513, 256, 128, 4, 1),    # top-1, >4 row blocks per expert
])
def test_forward_ragged_shapes(T, H, I, E, k):
    case = make_case(T, H, I, E, k, seed=T)
    ref = run_oracle(case)
    got = run_gpu(to_cuda(case))
    assert rel_err(got, ref) <= BF16_TOL


def test_strided_equals_contiguous_bit_identical_and_deterministic():
    case = to_cuda(make_case(200, 512, 256, 8, 2, seed=3))
    a = run_gpu(case)
    b = run_gpu(case, contiguous=True)
    c = run_gpu(case)
    assert torch.equal(a, b)
    assert torch.equal(a, c)


def test_expert_addressing_regression_distinct_constants():
    # every expert's gate and up hold different values; addressing experts by
    # e * I / TileN (instead of the real stride) would mix them up
    T, H, I, E, k = 64, 256, 128, 4, 2
    case = make_case(T, H, I, E, k, seed=9)
    w13 = case["w13"]
    for e in range(E):
        w13[e, :I] *= (1.0 + 0.25 * e)
        w13[e, I:] *= (-0.5 - 0.125 * e)
    ref = run_oracle(case)
    got = run_gpu(to_cuda(case))
    assert rel_err(got, ref) <= BF16_TOL


def test_strided_activations_ids_weights_and_out():
    T, H, I, E, k, L = 96, 256, 128, 8, 4, 5
    case = make_case(T, H, I, E, k, seed=13)
    ids_all = torch.randint(0, E, (T, L, k), generator=torch.Generator().manual_seed(1))
    w_all = torch.rand(T, L, k, generator=torch.Generator().manual_seed(2))
    ids_all[:, 2, :] = case["ids"].long()
    w_all[:, 2, :] = case["wts"]
    ref = run_oracle(case)
    c = to_cuda(case)
    x_dev = case["x"].t().contiguous().cuda().t()
    assert x_dev.stride() == (1, T)
    ids_dev = ids_all.cuda()[:, 2, :]
    w_dev = w_all.cuda()[:, 2, :]
    out_big = torch.zeros(T, 2 * H, dtype=torch.bfloat16, device="cuda")
    out = out_big[:, ::2]
    v = moe.w13_from_packed(c["w13"])
    moe.forward(x_dev, v, c["w2"], ids_dev, w_dev, out=out)
    torch.cuda.synchronize()
    assert rel_err(out, ref) <= BF16_TOL
    assert torch.all(out_big[:, 1::2] == 0)


def test_out_of_range_ids_skipped_and_counted():
    T, H, I, E, k = 40, 256, 128, 8, 2
    case = make_case(T, H, I, E, k, seed=21)
    case["ids"][3, 1] = -1
    case["ids"][7, 0] = E
    ref = run_oracle(case)
    moe.device_errors()
    got = run_gpu(to_cuda(case))
    nbad, nto = moe.device_errors()
    assert rel_err(got, ref) <= BF16_TOL
    assert nbad == 2 and nto == 0


def test_forward_ws_allocates_nothing_and_matches_forward():
    case = to_cuda(make_case(128, 512, 256, 8, 4, seed=31))
    nbytes = moe.workspace_bytes(128, 512, 256, 8, 4)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    a = run_gpu(case, ws=ws)
    out = torch.empty_like(a)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    run_gpu(case, ws=ws, out=out)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0
    assert torch.equal(a, out)
    b = run_gpu(case)
    assert torch.equal(a, b)


def test_forward_host_matches_device():
    case = make_case(50, 256, 128, 8, 2, seed=41)
    c = to_cuda(case)
    dev = run_gpu(c)
    out_h = torch.empty(50, 256, dtype=torch.bfloat16).pin_memory()
    x_h = case["x"].pin_memory()
    ids_h = case["ids"].pin_memory()
    w_h = case["wts"].pin_memory()
    moe.forward_host(x_h, moe.w13_from_packed(c["w13"]), c["w2"], ids_h, w_h, out_h)
    assert torch.equal(out_h, dev.cpu())


def test_forward_host_ws_two_calls_in_flight_on_two_streams():
    # the asynchronous host form: two calls with their own workspaces, host inputs and
    # outputs, enqueued on two streams before either is waited for, each equal to the
    # device forward of its own inputs
    T, H, I, E, k = 300, 512, 384, 8, 4
    cases = [make_case(T, H, I, E, k, seed=s) for s in (71, 72)]
    w13, w2 = cases[0]["w13"].cuda(), cases[0]["w2"].cuda()  # shared weights
    v = moe.w13_from_packed(w13)
    devs = [run_gpu(dict(to_cuda(cs), w13=w13, w2=w2)) for cs in cases]
    nbytes = moe.host_workspace_bytes(T, H, I, E, k)
    assert nbytes >= moe.workspace_bytes(T, H, I, E, k) + 2 * T * H * 2
    streams = [torch.cuda.Stream() for _ in cases]
    wss = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in cases]
    hosts = [{n: cs[n].contiguous().pin_memory() for n in ("x", "ids", "wts")} for cs in cases]
    outs = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in cases]
    torch.cuda.synchronize()
    for i in range(2):
        h = hosts[i]
        moe.forward_host(h["x"], v, w2, h["ids"], h["wts"], outs[i], workspace=wss[i], stream=streams[i])
    for st in streams:
        st.synchronize()
    for i in range(2):
        assert torch.equal(outs[i], devs[i].cpu())
    small = torch.empty(nbytes - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as err:
        h = hosts[0]
        moe.forward_host(h["x"], v, w2, h["ids"], h["wts"], outs[0], workspace=small)
    assert err.value.status == 5  # MOE_ERR_WORKSPACE_TOO_SMALL


@pytest.mark.parametrize("T,H,I,E,k", [
    (37, 288, 96, 6, 3),       # one-CTA kernels, padded 32-row granules
    (300, 512, 384, 4, 2),     # CTA pairs
])
def test_stale_workspace_contents_never_reach_the_output(T, H, I, E, k):
    # padding rows of the expert-grouped buffers are never written; a workspace
    # full of NaN bit patterns must give the same bits as a zeroed one
    case = make_case(T, H, I, E, k, seed=T + 17)
    ref = run_oracle(case)
    c = to_cuda(case)
    n = moe.workspace_bytes(T, H, I, E, k)
    ws0 = torch.zeros(n, dtype=torch.uint8, device="cuda")
    wsn = torch.full((n,), 0xFF, dtype=torch.uint8, device="cuda")
    a = run_gpu(c, ws=ws0)
    b = run_gpu(c, ws=wsn)
    assert torch.equal(a, b)
    assert rel_err(a, ref) <= BF16_TOL


def test_zero_tokens():
    case = to_cuda(make_case(0, 256, 128, 8, 2))
    out = run_gpu(case)
    assert out.shape == (0, 256)


# ----------------------------------------------------------------------------- full size

def _sample_tokens(T, n, seed, ids=None, E=None, per_expert=8, n_light=4):
    """Tokens the oracle checks at full size: n spread at random, the first
    and last 16, and (given the routing) up to `per_expert` tokens routed to
    each of the `n_light` least-loaded routed experts, whose short, ragged
    token tiles are the edge cases of the grouped GEMMs."""
    g = torch.Generator().manual_seed(seed)
    parts = [torch.randperm(T, generator=g)[:n], torch.arange(min(16, T)),
             torch.arange(max(0, T - 16), T)]
    if ids is not None:
        ids = ids.long().cpu()
        counts = torch.bincount(ids[(ids >= 0) & (ids < E)], minlength=E)
        routed = torch.nonzero(counts > 0).flatten()
        light = routed[torch.argsort(counts[routed], stable=True)[:n_light]]
        for e in light.tolist():
            parts.append(torch.nonzero((ids == e).any(dim=1)).flatten()[:per_expert])
    return torch.unique(torch.cat(parts))


@pytest.mark.slow
def test_qwen3_235b_shape_full_size_sampled(qwen3_weights):
    s = wl.QWEN3_235B
    w13, w2 = qwen3_weights["w13"], qwen3_weights["w2"]
    x = wl.make_x(s.T, s.H, seed=1, device="cuda")
    ids, wts = wl.route_softmax_topk(s.T, s.E, s.k, seed=2, device="cuda")
    c = {"x": x, "w13": w13, "w2": w2, "ids": ids, "wts": wts}
    a = run_gpu(c)
    b = run_gpu(c, contiguous=True)
    assert torch.equal(a, b)
    toks = _sample_tokens(s.T, 128, 0, ids=ids, E=s.E)
    case_cpu = {"x": x.cpu(), "w13": qwen3_weights["w13_cpu"], "w2": qwen3_weights["w2_cpu"],
                "ids": ids.cpu(), "wts": wts.cpu()}
    ref = run_oracle(case_cpu, tokens=toks)
    assert rel_err(a.cpu()[toks], ref) <= BF16_TOL


@pytest.mark.slow
@pytest.mark.parametrize("T", [1, 4, 64, 1023, 4097, 16384])
def test_qwen3_235b_token_sweep_full_shape(qwen3_weights, T):
    # the decode and prefill sweep on the full expert shapes (H=4096, I=1536,
    # E=128, top-8), strided packed w13, the sweep's per-T seeds: decode sizes
    # stream 32-row tiles on most SMs; 1023 / 4097 leave ragged last tiles and
    # 4097 runs the multi-CTA align; 16384 runs the 256-row CTA-pair tiles.
    # All tokens up to 64, else a sample: first and last 16, spread tokens and
    # the least-loaded experts' tokens (their short tiles are the edge cases).
    s = wl.QWEN3_235B
    w13, w2 = qwen3_weights["w13"], qwen3_weights["w2"]
    x = wl.make_x(T, s.H, seed=2000 + T, device="cuda")
    ids, wts = wl.route_softmax_topk(T, s.E, s.k, seed=1000 + T, device="cuda")
    a = run_gpu({"x": x, "w13": w13, "w2": w2, "ids": ids, "wts": wts})
    toks = None if T <= 64 else _sample_tokens(T, 48, T, ids=ids, E=s.E, per_expert=4)
    case_cpu = {"x": x.cpu(), "w13": qwen3_weights["w13_cpu"], "w2": qwen3_weights["w2_cpu"],
                "ids": ids.cpu(), "wts": wts.cpu()}
    ref = run_oracle(case_cpu, tokens=toks)
    got = a.cpu() if toks is None else a.cpu()[toks]
    assert rel_err(got, ref) <= BF16_TOL
    assert torch.isfinite(a.float()).all()


@pytest.mark.slow
def test_glm45_air_shape_skewed_strided_ids_sampled():
    s = wl.GLM45_AIR
    w13, w2 = wl.make_weights_bf16(s.E, s.I, s.H, seed=0, device="cuda")
    x = wl.make_x(s.T, s.H, seed=1, device="cuda")
    ids_all, w_all = wl.route_zipf_layers(s.T, s.E, s.k, layers=46, seed=7, device="cuda")
    ids, wts = ids_all[:, 23, :], w_all[:, 23, :]
    assert ids.stride() == (368, 1)
    c = {"x": x, "w13": w13, "w2": w2, "ids": ids, "wts": wts}
    a = run_gpu(c)
    toks = _sample_tokens(s.T, 256, 1, ids=ids, E=s.E)
    case_cpu = {"x": x.cpu(), "w13": w13.cpu(), "w2": w2.cpu(), "ids": ids_all.cpu()[:, 23, :],
                "wts": w_all.cpu()[:, 23, :]}
    ref = run_oracle(case_cpu, tokens=toks)
    assert rel_err(a.cpu()[toks], ref) <= BF16_TOL


TILE_VARIANTS = {
    "32": dict(tile=32),
    "128/one-cta": dict(tile=128, pair=0),
    "128/pair-two-slice": dict(tile=128, pair=1, g2_single=0),
    "128/pair-one-slice": dict(tile=128, pair=1, g2_single=1, g1_256=0),
    "128/pair-one-slice-g1-256": dict(tile=128, pair=1, g2_single=1, g1_256=1),
    "256": dict(tile=256),
    "pair-gate-up-interleaved-256": dict(g1_il=256),
    "pair-gate-up-interleaved-512": dict(g1_il=512),
}


@pytest.mark.parametrize("T,H,I,E,k", [
    (300, 512, 384, 4, 2),     # 150 slots per expert: several 32-row granules, partial tiles
    (600, 512, 640, 3, 2),     # 400 slots per expert: >1 token tile of 256 rows, N tail of I
    (77, 288, 96, 6, 3),       # ragged K and output columns
    (700, 256, 256, 2, 2),     # 700 slots per expert: two 352-row tiles of the 512-row list
    (1000, 256, 256, 8, 2),    # ~250 slots per expert: one or two 256-row tiles (paired work items)
])
def test_token_tile_configs_agree_and_match_oracle(T, H, I, E, k):
    # the token-tile size (32 / 128 rows on one CTA, 128 / 256 rows on a CTA pair)
    # and the GEMM variants are a performance choice (moe_set_config_table):
    # every configuration must give the same bits
    case = make_case(T, H, I, E, k, seed=T + 5)
    ref = run_oracle(case)
    c = to_cuda(case)
    outs = {}
    for name, flags in TILE_VARIANTS.items():
        with moe.config_override((T, H, I, E, k), **flags):
            got = moe.get_config(T, H, I, E, k)
            assert all(got[f] == v for f, v in flags.items() if f != "pair" or flags["tile"] == 128), name
            outs[name] = run_gpu(c)
        assert rel_err(outs[name], ref) <= BF16_TOL, name
    for name in TILE_VARIANTS:
        assert torch.equal(outs["32"], outs[name]), name


@pytest.mark.parametrize("T,k,idt", [(1, 8, torch.int32), (4, 8, torch.int64), (3, 10, torch.int32)])
def test_decode_weight_prefetch_matches_oracle_and_unprefetched(T, k, idt):
    # at most 32 slots: GEMM1 finds its experts from the routing ids and requests
    # weights before align has run; results must not depend on it
    H, I, E = 512, 384, 16
    case = make_case(T, H, I, E, k, seed=T + 97)
    case["ids"] = case["ids"].to(idt)
    case["ids"][0, 1] = E            # skipped slot
    case["ids"][T - 1, 2] = case["ids"][T - 1, 3]  # one expert twice for a token
    ref = run_oracle(case)
    c = to_cuda(case)
    moe.device_errors()
    outs = {}
    for pre in (1, 0):
        with moe.config_override((T, H, I, E, k), prefetch=pre, fused=0):
            assert moe.get_config(T, H, I, E, k)["prefetch"] == pre
            outs[pre] = run_gpu(c)
    nbad, nto = moe.device_errors()
    assert nbad == 2 and nto == 0
    assert torch.equal(outs[1], outs[0])
    assert rel_err(outs[1], ref) <= BF16_TOL


@pytest.mark.parametrize("T,k", [(1, 8), (4, 8)])
def test_decode_prefetch_with_ids_from_the_router_just_before(T, k):
    # the router kernel writes the ids and weights on the same stream right before
    # each forward; it releases its dependents at its start, so GEMM1 can issue its
    # early weight requests while the router is still writing: the prefetch must be
    # checked against align's tile list, and every call must match its own routing
    H, I, E = 512, 384, 16
    case = make_case(T, H, I, E, k, seed=T + 151)
    gen = torch.Generator().manual_seed(T + 7)
    logits = [torch.randn(T, E, generator=gen) for _ in range(2)]
    refs = []
    for lg in logits:
        ids, wts = oracle.router_topk(lg, k)
        refs.append(run_oracle(dict(case, ids=ids, wts=wts.float())))
    c = to_cuda(case)
    lg_dev = [lg.cuda() for lg in logits]
    ids_buf = torch.empty(T, k, dtype=torch.int32, device="cuda")
    wts_buf = torch.empty(T, k, dtype=torch.float32, device="cuda")
    v = moe.w13_from_packed(c["w13"])
    ws = torch.empty(moe.workspace_bytes(T, H, I, E, k), dtype=torch.uint8, device="cuda")
    moe.device_errors()
    outs = []
    with moe.config_override((T, H, I, E, k), prefetch=1, fused=0):
        assert moe.get_config(T, H, I, E, k)["prefetch"] == 1
        for it in range(24):
            moe.router_topk(lg_dev[it % 2], k, topk_ids=ids_buf, topk_weights=wts_buf)
            outs.append(moe.forward(c["x"], v, c["w2"], ids_buf, wts_buf, workspace=ws))
        torch.cuda.synchronize()
    nbad, nto = moe.device_errors()
    assert nbad == 0 and nto == 0
    for it, o in enumerate(outs):
        assert rel_err(o, refs[it % 2]) <= BF16_TOL, it
        assert torch.equal(o, outs[it % 2]), it


@pytest.mark.parametrize("T,k,idt,tile,strided", [
    (1, 8, torch.int32, None, False),      # decode
    (4, 8, torch.int64, None, False),      # 32 slots, the largest one-launch batch
    (3, 10, torch.int32, None, True),      # strided x and ids
    (2, 8, torch.int32, 128, False),       # 128-row token tiles
    (3, 11, torch.int32, None, False),     # 33 slots: align + permute kernels either way
])
def test_decode_align_permute_one_launch_matches_two(T, k, idt, tile, strided):
    # at most 32 routing slots: align and permute run as one launch that groups
    # the slots with warp ballots; it must give the general kernels' bits
    H, I, E = 512, 384, 24
    case = make_case(T, H, I, E, k, seed=T + 131)
    case["ids"] = case["ids"].to(idt)
    case["ids"][0, 1] = -1                          # skipped slot
    case["ids"][T - 1, 2] = case["ids"][T - 1, 3]   # one expert twice for a token
    ref = run_oracle(case)
    c = to_cuda(case)
    if strided:
        c["x"] = case["x"].t().contiguous().cuda().t()
        big = torch.zeros(T, 3, k, dtype=idt, device="cuda")
        big[:, 1, :] = c["ids"]
        c["ids"] = big[:, 1, :]
    extra = {"tile": tile} if tile else {}
    moe.device_errors()
    outs, launches = {}, {}
    for tiny in (1, 0):
        with moe.config_override((T, H, I, E, k), tiny=tiny, fused=0, **extra):
            outs[tiny] = run_gpu(c)
            launches[tiny] = moe.last_launch_count()
    nbad, nto = moe.device_errors()
    assert nbad == 2 and nto == 0
    assert torch.equal(outs[1], outs[0])
    assert rel_err(outs[1], ref) <= BF16_TOL
    assert launches[0] == 5
    assert launches[1] == (4 if T * k <= 32 else 5)


@pytest.mark.parametrize("T,H,I,E,k,idt,case", [
    (1, 512, 384, 24, 8, torch.int32, "plain"),
    (4, 512, 384, 24, 8, torch.int64, "plain"),            # 32 slots, int64 ids
    (3, 512, 384, 24, 10, torch.int32, "strided-ids"),     # ids read through a replay slice
    (2, 288, 96, 20, 16, torch.int32, "ragged"),           # H, I off the 256/128 tiles
    (1, 512, 384, 40, 32, torch.int32, "one-expert"),      # all 32 slots to one expert (8 gathers)
    (2, 512, 256, 8, 4, torch.int32, "no-valid-id"),       # every id out of range: out must be zero
])
def test_decode_one_kernel_matches_kernels_and_oracle(T, H, I, E, k, idt, case):
    # at most 32 slots: the whole forward as one kernel (slots grouped in every CTA,
    # token rows gathered from x, combine by the last CTA of each output tile) must
    # give the multi-kernel path's bits with GEMM1 unsplit, and match the oracle
    # with GEMM1 split along K (these shapes take two parts when few experts are routed)
    cs = make_case(T, H, I, E, k, seed=T + k + 211)
    ids = cs["ids"].to(idt)
    if case in ("plain", "strided-ids", "ragged"):
        ids[0, 1] = E                                 # a skipped slot
        ids[T - 1, 2] = ids[T - 1, 3]                 # one expert twice for a token
    if case == "one-expert":
        ids[:] = 5
    if case == "no-valid-id":
        ids[:] = -1
    cs["ids"] = ids
    c = to_cuda(cs)
    if case == "strided-ids":
        big = torch.zeros(T, 3, k, dtype=idt, device="cuda")
        big[:, 1, :] = c["ids"]
        c["ids"] = big[:, 1, :]
    moe.device_errors()
    outs, launches = {}, {}
    variants = {"unsplit": dict(fused=1, split=1), "kernels": dict(fused=0), "split": dict(fused=1)}
    for name, flags in variants.items():
        with moe.config_override((T, H, I, E, k), **flags):
            out = torch.full((T, H), 7.0, dtype=torch.bfloat16, device="cuda")  # stale contents
            outs[name] = run_gpu(c, out=out)
            launches[name] = moe.last_launch_count()
            if name == "split":
                assert torch.equal(run_gpu(c), outs[name])  # fixed part order: deterministic
    nbad, nto = moe.device_errors()
    n_skip = int(((ids < 0) | (ids >= E)).sum().item())
    assert nbad == 4 * n_skip and nto == 0
    assert launches["unsplit"] == 1 and launches["split"] == 1 and launches["kernels"] == 4
    assert torch.equal(outs["unsplit"], outs["kernels"])
    if case == "no-valid-id":
        assert bool((outs["split"] == 0).all()) and bool((outs["unsplit"] == 0).all())
    else:
        ref = run_oracle(cs)
        assert rel_err(outs["unsplit"], ref) <= BF16_TOL
        assert rel_err(outs["split"], ref) <= BF16_TOL


@pytest.mark.parametrize("T,E,k", [(1, 16, 4), (2, 16, 6), (1, 64, 8), (4, 40, 8)])
def test_decode_split_gemm1_each_part_count_matches_oracle(T, E, k):
    # GEMM1 split along K into at most 2, 3 and 4 parts (H = 2048: 32 k-blocks,
    # so every count keeps at least four per part; the cases with few routed
    # experts take the most parts; I = 320 leaves a ragged 64-row last item):
    # each count matches the oracle and repeats its own bits, and the unsplit
    # one-kernel result equals the multi-kernel path's
    H, I = 2048, 320
    cs = make_case(T, H, I, E, k, seed=7 * T + E + k)
    if T > 1:
        cs["ids"][T - 1, 0] = cs["ids"][0, 0]          # an expert shared by two tokens
    c = to_cuda(cs)
    ref = run_oracle(cs)
    outs = {}
    for split in (1, 2, 3, 4):
        with moe.config_override((T, H, I, E, k), fused=1, split=split):
            assert moe.get_config(T, H, I, E, k)["split"] == split
            outs[split] = run_gpu(c)
            assert moe.last_launch_count() == 1
            assert torch.equal(run_gpu(c), outs[split]), split
        assert rel_err(outs[split], ref) <= BF16_TOL, split
    with moe.config_override((T, H, I, E, k), fused=0):
        assert torch.equal(run_gpu(c), outs[1])


def test_decode_one_kernel_repeated_calls_and_fallback_for_strided_x():
    # the kernel's cross-CTA counters are reset by its last CTA: back-to-back calls
    # (more than the counter sets in the library) keep giving the same bits; an x
    # whose rows TMA cannot gather runs the multi-kernel path instead
    T, H, I, E, k = 3, 512, 384, 24, 8
    cs = make_case(T, H, I, E, k, seed=401)
    c = to_cuda(cs)
    first = run_gpu(c)
    assert moe.last_launch_count() == 1
    for _ in range(40):
        assert torch.equal(run_gpu(c), first)
    with moe.config_override((T, H, I, E, k), split=1):
        unsplit = run_gpu(c)
        xs = cs["x"].t().contiguous().cuda().t()
        c2 = dict(c, x=xs)
        got = run_gpu(c2)
        assert moe.last_launch_count() == 4
    assert torch.equal(got, unsplit)
    ref = run_oracle(cs)
    assert rel_err(first, ref) <= BF16_TOL and rel_err(unsplit, ref) <= BF16_TOL
