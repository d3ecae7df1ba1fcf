"""The committed kernel-configuration table (configs/b200_tuned.csv, compiled
into the library) checked against the fp64 oracle, row by row, the way the
pages' tuner refuses tuned kernels above an error ratio (ROCm/aiter PR #3859,
"Details": errRatio=0.05; here the method's own bounds, 1e-2 bf16 and 6e-2
MXFP4, on every checked element).  Each row runs at its bucket's token count on
its full layer shape: the library must select the row's configuration, the
output must equal that of a fixed reference configuration bit for bit, and a
token sample must match the oracle."""

import pytest
import torch

import mixture_experts_layer_46_b200 as moe
import oracle
from mixture_experts_layer_46_b200 import build
from mixture_experts_layer_46_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ROWS = build.read_config_csv()
T_CAP = 16384


def _row_T(r):
    return r["t_hi"] if r["t_hi"] <= T_CAP else max(r["t_lo"], 1)


def _rel(got, ref):
    return (got.double().cpu() - ref).abs().max().item() / ref.abs().max().item()


def _tokens(T):
    g = torch.Generator().manual_seed(T)
    t = torch.cat([torch.arange(min(4, T)), torch.arange(max(0, T - 4), T),
                   torch.randperm(T, generator=g)[:8]])
    return torch.unique(t)


@pytest.mark.skipif(not ROWS, reason="no tuned rows committed")
@pytest.mark.parametrize("row", ROWS, ids=lambda r: f"{'mx' if r['wdtype'] else 'bf16'}-E{r['E']}-T{r['t_lo']}-{r['t_hi']}")
def test_tuned_row_matches_oracle(row, request):
    mx = row["wdtype"] == 4
    H, I, E, k = row["H"], row["I"], row["E"], row["k"]
    T = _row_T(row)
    got_cfg = moe.get_config(T, H, I, E, k, mxfp4=mx)
    for f in ("tile", "pair", "g1_256", "g2_single", "fused"):
        assert got_cfg[f] == row[f] or (f == "pair" and got_cfg["tile"] != 128), (f, got_cfg, row)
    if row["fused"]:
        assert got_cfg["split"] == (row["split"] or 4), (got_cfg, row)
    x = wl.make_x(T, H, seed=2000 + T)
    if mx:
        w = request.getfixturevalue("tp2_weights")
        cw, gw = w["cpu"], w["gpu"]
        if E == 513:
            ids, wts = wl.route_shared_expert(T, E - 1, k - 1, seed=1000 + T)
        else:
            ids, wts = wl.route_softmax_topk(T, E, k, seed=1000 + T)
        v = moe.w13_from_packed(gw["c13"][:E], gw["s13"][:E])
        args = (x.cuda(), v, gw["c2"][:E], ids.cuda(), wts.cuda())
        kw = {"w2_scale": gw["s2"][:E]}
        tol = 6e-2
    else:
        shapes = {(4096, 1536, 128, 8): "qwen3_weights", (4096, 1408, 128, 8): "glm_weights"}
        assert (H, I, E, k) in shapes, "only the Qwen3-235B and GLM-4.5-Air shapes are tuned here"
        w = request.getfixturevalue(shapes[(H, I, E, k)])
        ids, wts = wl.route_softmax_topk(T, E, k, seed=1000 + T)
        args = (x.cuda(), moe.w13_from_packed(w["w13"]), w["w2"], ids.cuda(), wts.cuda())
        kw = {}
        tol = 1e-2
    out = moe.forward(*args, **kw)
    with moe.config_override((T, H, I, E, k), mxfp4=mx, tile=32):
        ref_cfg_out = moe.forward(*args, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_cfg_out)
    toks = _tokens(T)
    if mx:
        I2 = I
        ref, _ = oracle.moe_forward(x, cw["c13"][:E, :I2], cw["c13"][:E, I2:], cw["c2"][:E], ids, wts,
                                    scales=(cw["s13"][:E, :I2], cw["s13"][:E, I2:], cw["s2"][:E]),
                                    tokens=toks)
    else:
        gate, up = wl.gate_up_views(w["w13_cpu"])
        ref, _ = oracle.moe_forward(x, gate, up, w["w2_cpu"], ids, wts, tokens=toks)
    assert _rel(out.cpu()[toks], ref) <= tol
