"""Host-side tests of the C ABI (no GPU needed): the library loads and exports
every entry point include/moe.h declares, status codes, packed-view metadata,
workspace sizing, and the validation errors that must come before anything is
launched or any descriptor is built (Liger-Kernel PR #1377, "Testing Done")."""

import json
import os
import re

import pytest
import torch

import mixture_experts_layer_46_b200 as moe
from mixture_experts_layer_46_b200 import _abi
from mixture_experts_layer_46_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLD = os.path.join(ROOT, "tests", "golden")


def _declared_entry_points():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_entry_point():
    lib = moe.load()
    declared = _declared_entry_points()
    assert declared, "no entry points parsed from include/*.h"
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(_abi.EXPORTS) | (declared - set(_abi.EXPORTS))
    assert set(_abi.EXPORTS) <= declared


def test_status_strings():
    lib = moe.load()
    for code, name in _abi.STATUS.items():
        assert lib.moe_status_string(code).decode() == name


def test_w13_from_packed_locates_up_by_stride():
    # I=1536, TileN=128 worked example (tests/golden/liger_tile_example.json)
    g = json.load(open(os.path.join(GOLD, "liger_tile_example.json")))
    I, tile_n, H, E = g["intermediate"], g["tile_n"], 64, 3
    w13 = torch.empty(E, 2 * I, H, dtype=torch.bfloat16)  # storage only
    v = moe.w13_from_packed(w13)
    assert v.gate.sizes[1] == I and v.up.sizes[1] == I
    assert v.gate.strides[0] == 2 * I * H  # the real expert stride is kept
    row = lambda d, e, n: (d.data - w13.data_ptr()) // 2 // H + e * d.strides[0] // H + n * tile_n
    # tile index (in TileN-row units) of (expert, n-th useful tile) for each view
    tile = lambda d, e, n: row(d, e, n) // tile_n
    assert I // tile_n == g["useful_tiles_per_expert"]
    assert v.gate.strides[0] // H // tile_n == g["packed_physical_stride_tiles"]
    assert tile(v.gate, 0, 0) == g["packed_tile_ranges"]["expert0_gate"][0]
    assert tile(v.gate, 0, 11) == g["packed_tile_ranges"]["expert0_gate"][1]
    assert tile(v.up, 0, 0) == g["packed_tile_ranges"]["expert0_up"][0]
    assert tile(v.gate, 1, 0) == g["packed_tile_ranges"]["expert1_gate"][0]
    # the old addressing, expert * (I / TileN), would put expert 1's gate on expert 0's up
    assert 1 * (I // tile_n) == g["old_offset_expert1_gate_first_tile"] == tile(v.up, 0, 0)
    # contiguous copies: physical stride equals the useful tile count
    c = moe.w13_from_views(w13[:, :I].contiguous(), w13[:, I:].contiguous())
    assert c.gate.strides[0] // H // tile_n == g["useful_tiles_per_expert"]


def test_packed_copy_cost_matches_the_pages():
    # 16 local experts x 2 * 1536 * 4096 bf16 = 0.375 GiB per layer of retained copies
    g = json.load(open(os.path.join(GOLD, "liger_tile_example.json")))
    assert 16 * 2 * g["intermediate"] * 4096 * 2 / 2 ** 30 == g["copy_cost_gib_per_layer"]


def test_workspace_independent_of_weight_size_and_layout():
    base = moe.workspace_bytes(4096, 4096, 1536, 128, 8)
    assert base > 0
    w_bytes = 128 * 3 * 1536 * 4096 * 2
    assert base < w_bytes / 4
    assert moe.workspace_bytes(0, 4096, 1536, 128, 8) > 0
    assert moe.workspace_bytes(4096, 4096, 1536, 128, 8, mxfp4=True) < base
    assert moe.load().moe_workspace_bytes(4, 64, 64, 4, 2, 9) == 0


def test_host_workspace_holds_the_forward_workspace_and_the_staging():
    # the asynchronous host form stages x, the ids (room for int64), the weights and out
    # after the forward's own workspace, each region 256-byte aligned
    T, H, I, E, k = 4096, 4096, 1536, 128, 8
    for mx in (False, True):
        core = moe.workspace_bytes(T, H, I, E, k, mxfp4=mx)
        got = moe.host_workspace_bytes(T, H, I, E, k, mxfp4=mx)
        staging = T * H * 2 + T * k * 8 + T * k * 4 + T * H * 2
        assert core + staging <= got <= core + staging + 5 * 256
        assert got % 256 == 0
    assert moe.load().moe_host_workspace_bytes(4, 64, 64, 4, 2, 9) == 0
    assert moe.load().moe_host_workspace_bytes(4, 0, 64, 4, 2, 0) == 0


def test_host_forward_rejects_a_small_workspace_before_any_copy():
    x, w13, w2, ids, wts, out = _cpu_problem()
    v = moe.w13_from_packed(w13)
    need = moe.host_workspace_bytes(8, 64, 32, 4, 2)
    ws = torch.zeros(need - 256, dtype=torch.uint8)  # never touched: the size is checked first
    with pytest.raises(moe.MoeError) as err:
        moe.forward_host(x, v, w2, ids, wts, out, workspace=ws, stream=0)
    assert err.value.status == 5
    assert moe.last_launch_count() == 0


def _cpu_problem(T=8, H=64, I=32, E=4, k=2):
    x = torch.zeros(T, H, dtype=torch.bfloat16)
    w13 = torch.zeros(E, 2 * I, H, dtype=torch.bfloat16)
    w2 = torch.zeros(E, H, I, dtype=torch.bfloat16)
    ids = torch.zeros(T, k, dtype=torch.int32)
    wts = torch.zeros(T, k, dtype=torch.float32)
    out = torch.empty(T, H, dtype=torch.bfloat16)
    return x, w13, w2, ids, wts, out


def _status(x, w13v, w2, ids, wts, out, ws=None):
    return moe.forward_status(x, w13v, w2, ids, wts, out, workspace=ws)


def test_mismatched_gate_hidden_dim_fails_before_descriptors():
    x, w13, w2, ids, wts, out = _cpu_problem()
    bad_gate = torch.zeros(4, 32, 96, dtype=torch.bfloat16)
    v = moe.w13_from_views(bad_gate, w13[:, 32:])
    # host tensors: validation must reject before touching any device or launching
    assert _status(x, v, w2, ids, wts, out) == 2
    assert moe.last_launch_count() == 0


def test_validation_errors():
    x, w13, w2, ids, wts, out = _cpu_problem()
    v = moe.w13_from_packed(w13)
    assert _status(x, v, w2[:, :, :16], ids, wts, out) == 2             # w2 cols != I
    assert _status(x, v, w2, ids[:3], wts, out) == 2                      # ids rows != T
    assert _status(x.float(), v, w2, ids, wts, out) == 3                  # x must be bf16
    assert _status(x, v, w2, ids.float(), wts, out) == 3                  # ids int32/int64
    assert _status(x, v, w2, ids, wts.double(), out) == 3                 # weights f32
    ids_many = torch.zeros(8, 33, dtype=torch.int32)
    assert _status(x, v, w2, ids_many, torch.zeros(8, 33), out) == 1      # k > 32
    # weight views with a non-unit inner stride cannot be read by the copy engine: loud error
    gt = torch.zeros(4, 64, 32, dtype=torch.bfloat16).transpose(1, 2)
    vt = moe.w13_from_views(gt, gt)
    assert _status(x, vt, w2, ids, wts, out) == 4
    # a weight base that is not 16-byte aligned
    flat = torch.zeros(4 * 64 * 64 + 8, dtype=torch.bfloat16)
    mis = flat[1:1 + 4 * 64 * 64].view(4, 64, 64)
    assert _status(x, moe.w13_from_packed(mis), w2, ids, wts, out) == 4
    # workspace too small is reported before any device work
    ws = torch.zeros(16, dtype=torch.uint8)
    assert _status(x, v, w2, ids, wts, out, ws) == 5


def test_backward_validation_errors():
    # the gradient entry point rejects bad arguments on the host, before any device work
    x, w13, w2, ids, wts, dx = _cpu_problem(T=8, H=64, I=32, E=4, k=2)
    v = moe.w13_from_packed(w13)
    w13t = torch.zeros(4, 64, 64, dtype=torch.bfloat16)
    w2t = torch.zeros(4, 32, 64, dtype=torch.bfloat16)
    dout = torch.zeros(8, 64, dtype=torch.bfloat16)
    dw = torch.zeros(8, 2, dtype=torch.float32)
    ws = torch.zeros(16, dtype=torch.uint8)

    def st(**kw):
        a = dict(x=x, w13=v, w2=w2, w13t=w13t, w2t=w2t, topk_ids=ids, topk_weights=wts, dout=dout, dx=dx,
                 dweights=dw, workspace=ws)
        a.update(kw)
        return moe.backward_status(**a)

    assert st() == 5                                                       # workspace too small
    assert st(w13t=torch.zeros(4, 64, 32, dtype=torch.bfloat16)) == 4     # w13t must be [E, H, 2I]
    assert st(w2t=torch.zeros(4, 64, 32, dtype=torch.bfloat16)) == 4      # w2t must be [E, I, H]
    assert st(w2t=torch.zeros(4, 64, 32, dtype=torch.bfloat16).transpose(1, 2)) == 4  # inner stride
    assert st(dout=torch.zeros(8, 32, dtype=torch.bfloat16)) == 2         # dout [T, H]
    assert st(dout=torch.zeros(8, 64, dtype=torch.float32)) == 3          # dout bf16
    assert st(dweights=torch.zeros(8, 2, dtype=torch.bfloat16)) == 3      # dweights f32
    assert st(dweights=torch.zeros(8, 3, dtype=torch.float32)) == 2       # dweights [T, k]
    assert st(dx=torch.zeros(8, 64, dtype=torch.float32)) == 3            # dx bf16, like out
    g13 = torch.zeros(4, 64, 64, dtype=torch.float32)
    g2 = torch.zeros(4, 64, 32, dtype=torch.float32)
    assert st(dw13=g13, dw2=g2) == 5                                       # valid weight gradients
    assert st(dw13=g13.int(), dw2=g2) == 4                                 # f32 or bf16 only
    assert st(dw13=g13, dw2=g2.to(torch.bfloat16)) == 4                    # bf16 rows: 64-column tiles
    assert st(dw13=torch.zeros(4, 32, 64), dw2=g2) == 4                    # [E, 2I, H]
    assert moe.last_launch_count() == 0


def test_zero_tokens_is_a_noop():
    x, w13, w2, ids, wts, out = _cpu_problem(T=0)
    assert _status(x, moe.w13_from_packed(w13), w2, ids, wts, out) == 0
    assert moe.last_launch_count() == 0


def test_router_replay_slice_stride():
    g = json.load(open(os.path.join(GOLD, "router_replay_stride.json")))
    ids, _ = wl.route_zipf_layers(16, 128, g["top_k"], layers=g["num_layers"], seed=7)
    sl = ids[:, 23, :]
    assert sl.stride(0) == g["token_stride"] and sl.stride(1) == 1
    d = _abi.desc(sl)
    assert d.strides[0] == 368 and d.data == ids.data_ptr() + 23 * 8 * 4
    # every token picks top_k distinct experts
    assert all(len(set(r.tolist())) == g["top_k"] for r in sl)


def test_product_path_has_no_oracle_dependency():
    pkg = os.path.join(ROOT, "mixture_experts_layer_46_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in src and "from oracle" not in src, fn
                assert "moe_oracle" not in src, fn


def test_config_table_lookup_and_fixed_workspace():
    # the per-shape configuration table (moe_set_config_table) decides the kernels
    # only: the workspace a caller sizes with moe_workspace_bytes never depends on it
    shape = (4096, 4096, 1536, 128, 8)
    base = moe.get_config(*shape)
    ws0 = moe.workspace_bytes(*shape)
    assert base["tile"] in (32, 128, 256)
    e = moe.make_config(_abi.MOE_BF16, H=4096, I=1536, E=128, k=8, t_lo=4000, t_hi=5000, tile=32,
                        tiny=1, prefetch=1)
    other_shape = moe.make_config(_abi.MOE_BF16, H=2048, t_lo=0, t_hi=10 ** 9, tile=256)
    try:
        moe.set_config_table([other_shape, e])
        got = moe.get_config(*shape)
        assert got["tile"] == 32 and got["pair"] == 0
        assert got["tiny"] == 0 and got["prefetch"] == 0   # 32768 slots: decode-only flags cleared
        assert moe.get_config(5001, 4096, 1536, 128, 8)["tile"] == 128  # outside the bucket
        assert moe.get_config(64, 2048, 1536, 128, 8)["tile"] == 256
        assert moe.get_config(64, 2048, 1536, 128, 8)["pair"] == 1   # 256-row tiles run on pairs
        assert moe.workspace_bytes(*shape) == ws0
        assert moe.get_config(*shape, mxfp4=True)["tile"] in (32, 96)  # bf16 entries only
    finally:
        moe.set_config_table([])
    assert moe.get_config(*shape) == base


def test_config_normalisation_of_the_split_and_interleaved_flags():
    # flags that only one path reads are normalised to what the kernels run:
    # the interleaved 512-row GEMM1 implies CTA pairs and the 256-row GEMM2 list
    # (bf16 only); the split count is 1 off the one-kernel path and 0 -> 4 on it
    shape = (4096, 4096, 1536, 128, 8)
    try:
        moe.set_config_table([moe.make_config(_abi.MOE_BF16, t_lo=0, t_hi=10 ** 9, tile=32,
                                              g1_il=512, g1_256=1, split=3),
                              moe.make_config(_abi.MOE_E2M1X2, t_lo=0, t_hi=10 ** 9, tile=96,
                                              g1_il=256)])
        got = moe.get_config(*shape)
        assert (got["g1_il"], got["pair"], got["g2_single"], got["g1_256"], got["tile"]) == (512, 1, 1, 0, 128)
        assert got["fused"] == 0 and got["split"] == 1
        assert moe.get_config(*shape, mxfp4=True)["g1_il"] == 0
        assert moe.get_config(2, 4096, 1536, 128, 8)["fused"] == 0  # the entry says fused = 0
        moe.set_config_table([moe.make_config(_abi.MOE_BF16, t_lo=0, t_hi=4, tile=32, fused=1)])
        assert moe.get_config(2, 4096, 1536, 128, 8)["split"] == 4
        moe.set_config_table([moe.make_config(_abi.MOE_BF16, t_lo=0, t_hi=4, tile=32, fused=1, split=2)])
        assert moe.get_config(2, 4096, 1536, 128, 8)["split"] == 2
        for bad in (dict(split=5), dict(g1_il=128), dict(g1_il=1)):
            with pytest.raises(moe.MoeError):
                moe.set_config_table([moe.make_config(_abi.MOE_BF16, tile=32, **bad)])
    finally:
        moe.set_config_table([])


def test_config_table_rejects_malformed_entries():
    bad = [moe.make_config(_abi.MOE_BF16, tile=64),            # no such tile
           moe.make_config(_abi.MOE_E2M1X2, tile=256),         # MXFP4 tiles are 32, 96 or 128
           moe.make_config(_abi.MOE_BF16, tile=32, pair=2),    # flags are 0 or 1
           moe.make_config(_abi.MOE_BF16, t_lo=10, t_hi=5, tile=32),
           moe.make_config(7, tile=32)]
    for b in bad:
        with pytest.raises(moe.MoeError):
            moe.set_config_table([b])
    assert moe.get_config(1, 4096, 1536, 128, 8)["tile"] == 32


def test_builtin_config_table_matches_committed_csv():
    from mixture_experts_layer_46_b200 import build

    rows = build.read_config_csv()
    assert moe.builtin_config_count() == len(rows)
    for r in rows:
        T = r["t_hi"]
        got = moe.get_config(T, r["H"], r["I"], r["E"], r["k"], mxfp4=r["wdtype"] == 4)
        assert got["tile"] == r["tile"], r
        assert got["g1_il"] == r["g1_il"] and got["fused"] == r["fused"], r


def test_router_argument_errors_before_launch():
    # refused on the host, before any device call
    lg = torch.zeros(4, 16)
    ids = torch.zeros(4, 2, dtype=torch.int32)
    w = torch.zeros(4, 2)
    assert moe.router_status(lg, 17, 1, 0, torch.zeros(4, 17, dtype=torch.int32), torch.zeros(4, 17)) == 1
    assert moe.router_status(lg, 2, 1, 1, ids, w) == 2          # shared column missing
    assert moe.router_status(lg, 2, 1, 0, ids.long().double(), w) == 3
    assert moe.router_status(lg.half(), 2, 1, 0, ids, w) == 3
    assert moe.router_status(lg, 2, 1, 0, ids, w.double()) == 3
    assert moe.router_status(lg, 2, 2, 0, ids, w) == 1          # flags are 0 or 1
    big = torch.zeros(2, 40)
    assert moe.router_status(big, 32, 1, 1, torch.zeros(2, 33, dtype=torch.int32),
                             torch.zeros(2, 33)) == 1          # more than 32 columns
    assert moe.router_status(torch.zeros(0, 16), 2, 1, 0, torch.zeros(0, 2, dtype=torch.int32),
                             torch.zeros(0, 2)) == 0           # no tokens: nothing to do
