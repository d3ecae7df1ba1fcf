"""Per-shape tuner of the forward's kernel configuration (token-tile size and
GEMM variant per token bucket), in the spirit of the pages' tuned fused-MoE
tables (ROCm/aiter PR #3859, "Details": a tuner writes the best kernel per
shape into a tuned CSV; "Tuned MoE latency": block_m chosen per token bucket).

    python -m mixture_experts_layer_46_b200.tune --workload qwen3-235b [--tokens 1,2,4,...]
           [--reps 15] [--out mixture_experts_layer_46_b200/configs/b200_tuned.csv]

For every token count T it runs each candidate configuration the kernels
support (moe_set_config_table with one exact entry) and checks its output
against the default configuration run with GEMM1 unsplit: every configuration
with an unsplit GEMM1 computes the same sums in the same order, so it must give
the same bits (anything else is a defect and the candidate is refused); a
one-kernel candidate whose GEMM1 is split along K sums its parts in a fixed
order, so it must repeat its own bits and stay within the method's error bound
of the reference (1e-2 bf16, 6e-2 MXFP4, relative to the largest output).
aiter's tuner refuses candidates above an error ratio in the same way.  The
accepted candidates are timed round-robin (L2 flushed clean before every call,
CUDA events, median of `reps`), so that clock and power drift hit them alike.  The winner covers the token bucket (previous T, T].  Rows are
merged into the CSV (same shape and bucket replaced); rebuild the library to
compile the table in.  The committed rows are checked against the fp64 oracle
by tests/test_gpu_config_table.py.
"""

from __future__ import annotations

import argparse
import csv
import os
import statistics
import sys

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(PKG))

import mixture_experts_layer_46_b200 as moe  # noqa: E402
from mixture_experts_layer_46_b200 import build  # noqa: E402
from mixture_experts_layer_46_b200 import workloads as wl  # noqa: E402

SHAPES = {
    "qwen3-235b": dict(H=4096, I=1536, E=128, k=8, mxfp4=False, routing="softmax",
                       tokens=(1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 16384)),
    "glm45-air": dict(H=4096, I=1408, E=128, k=8, mxfp4=False, routing="softmax",
                      tokens=(1, 4, 16, 64, 256, 1024, 4096, 16384)),
    "qwen35-tp2-mxfp4": dict(H=4096, I=512, E=512, k=10, mxfp4=True, routing="softmax",
                             tokens=(1, 2, 4, 16, 64, 256, 1024, 4096, 32768)),
    "qwen35-tp2-mxfp4-shared": dict(H=4096, I=512, E=513, k=11, mxfp4=True, routing="shared",
                                    tokens=(1, 2, 4, 16, 64, 256, 1024, 4096, 32768)),
}
T_MAX = 1 << 40


def candidates(T: int, k: int, mxfp4: bool):
    """Every configuration the kernels run for T tokens (flags that change nothing removed)."""
    S = T * k
    decode = S <= 32
    tinies = (1, 0) if decode else (0,)
    out = []
    fused = [dict(tile=32, fused=1, split=s) for s in (1, 2, 3, 4)] if decode else []
    if mxfp4:
        if decode:
            out.extend(fused)
        for tile in (32, 96, 128):
            for tiny in tinies:
                out.append(dict(tile=tile, tiny=tiny, fused=0))
        return out
    out.extend(fused)
    for tiny in tinies:
        for pre in ((1, 0) if decode else (0,)):
            out.append(dict(tile=32, tiny=tiny, prefetch=pre, fused=0, g1_il=0))
        out.append(dict(tile=128, pair=0, tiny=tiny, fused=0, g1_il=0))
        out.append(dict(tile=128, pair=1, g2_single=0, tiny=tiny, fused=0, g1_il=0))
        out.append(dict(tile=128, pair=1, g2_single=1, g1_256=0, tiny=tiny, fused=0, g1_il=0))
        out.append(dict(tile=128, pair=1, g2_single=1, g1_256=1, tiny=tiny, fused=0, g1_il=0))
        for il in (256, 512):
            out.append(dict(tile=128, pair=1, g2_single=1, g1_il=il, tiny=tiny, fused=0))
        out.append(dict(tile=256, tiny=tiny, fused=0, g1_il=0))
    return out


def make_weights(sh, dev):
    if not sh["mxfp4"]:
        w13, w2 = wl.make_weights_bf16(sh["E"], sh["I"], sh["H"], seed=0, device=dev)
        return moe.w13_from_packed(w13), w2, None, (w13, w2)
    E, I, H = sh["E"], sh["I"], sh["H"]
    c13 = torch.empty(E, 2 * I, H // 2, dtype=torch.uint8, device=dev)
    s13 = torch.empty(E, 2 * I, H // 32, dtype=torch.uint8, device=dev)
    c2 = torch.empty(E, H, I // 2, dtype=torch.uint8, device=dev)
    s2 = torch.empty(E, H, I // 32, dtype=torch.uint8, device=dev)
    for e, w13e, w2e in wl.iter_weights_fp32(E, I, H, seed=0, device=dev):
        c13[e], s13[e] = moe.quantize_mxfp4(w13e)
        c2[e], s2[e] = moe.quantize_mxfp4(w2e)
    return moe.w13_from_packed(c13, s13), c2, s2, (c13, s13, c2, s2)


def routing(sh, T, dev):
    if sh["routing"] == "shared":
        return wl.route_shared_expert(T, sh["E"] - 1, sh["k"] - 1, seed=1000 + T, device=dev)
    return wl.route_softmax_topk(T, sh["E"], sh["k"], seed=1000 + T, device=dev)


def tune_one(sh, T, v13, w2, s2, flush, reps, dev, log):
    H, I, E, k, mx = sh["H"], sh["I"], sh["E"], sh["k"], sh["mxfp4"]
    x = wl.make_x(T, H, seed=2000 + T, device=dev)
    ids, wts = routing(sh, T, dev)
    ws = torch.empty(moe.workspace_bytes(T, H, I, E, k, mxfp4=mx), dtype=torch.uint8, device=dev)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def run():
        moe.forward(x, v13, w2, ids, wts, out=out, workspace=ws, stream=stream, w2_scale=s2)

    def install(flags):
        entry = dict(default)
        entry.update(flags)
        entry.update(t_lo=T, t_hi=T)
        wd = entry.pop("wdtype")
        cfg = moe.make_config(wd, **entry)
        moe.set_config_table([cfg])
        return cfg

    moe.set_config_table([])
    default = moe.get_config(T, H, I, E, k, mxfp4=mx)
    install(dict(split=1))
    run()
    torch.cuda.synchronize(dev)
    ref = out.clone()
    tol = 6e-2 if mx else 1e-2
    cands = []
    for flags in candidates(T, k, mx):
        cfg = install(flags)
        got = moe.get_config(T, H, I, E, k, mxfp4=mx)
        key = tuple(got[f] for f in moe._abi.CONFIG_FLAGS)
        if any(key == c[0] for c in cands):
            continue  # the kernels normalise it to a configuration already listed
        run()
        torch.cuda.synchronize(dev)
        if got["split"] == 1:
            if not torch.equal(out, ref):
                n_diff = int((out != ref).sum().item())
                log(f"  T={T} {got}: REFUSED, {n_diff} of {out.numel()} outputs differ from the default")
                continue
        else:
            first = out.clone()
            run()
            torch.cuda.synchronize(dev)
            err = ((first.float() - ref.float()).abs().max() / ref.float().abs().max().clamp_min(1e-30)).item()
            if not torch.equal(out, first) or not err <= tol:
                log(f"  T={T} {got}: REFUSED, repeat equal {torch.equal(out, first)}, error {err:.2e}")
                continue
        cands.append((key, cfg, got))
    times = {c[0]: [] for c in cands}
    for c in cands:  # warm-up
        moe.set_config_table([c[1]])
        for _ in range(2):
            run()
    for i in range(reps):
        for key, cfg, _ in cands:
            moe.set_config_table([cfg])
            wl.flush_l2(flush, i)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            run()
            b.record(stream)
            torch.cuda.synchronize(dev)
            times[key].append(a.elapsed_time(b) * 1e3)
    moe.set_config_table([])
    med = {key: statistics.median(v) for key, v in times.items()}
    best_key = min(med, key=med.get)
    best = next(c[2] for c in cands if c[0] == best_key)
    dkey = tuple(default[f] for f in moe._abi.CONFIG_FLAGS)
    for key, cfg, got in cands:
        mark = " <- best" if key == best_key else (" (default)" if key == dkey else "")
        log(f"  T={T} {dict(zip(moe._abi.CONFIG_FLAGS, key))}: {med[key]:.1f} us{mark}")
    return best, med[best_key], med.get(dkey, float("nan")), len(cands)


def merge_rows(path, rows):
    old = []
    if os.path.exists(path):
        with open(path, newline="") as f:
            old = list(csv.DictReader(line for line in f if not line.startswith("#")))
    key = lambda r: tuple(str(r[c]) for c in ("wdtype", "H", "I", "E", "k", "t_lo", "t_hi"))
    new_keys = {key(r) for r in rows}
    shapes = {tuple(str(r[c]) for c in ("wdtype", "H", "I", "E", "k")) for r in rows}
    kept = [r for r in old if key(r) not in new_keys
            and tuple(r[c] for c in ("wdtype", "H", "I", "E", "k")) not in shapes]
    cols = list(build.CONFIG_COLUMNS) + ["us", "us_default", "candidates"]
    os.makedirs(os.path.dirname(path), exist_ok=True)
    with open(path, "w", newline="") as f:
        f.write("# kernel configuration per shape and token bucket [t_lo, t_hi], written by "
                "mixture_experts_layer_46_b200/tune.py on one B200 (us: median forward time of the "
                "chosen configuration at T = t_hi, us_default: the heuristic's)\n")
        wr = csv.DictWriter(f, fieldnames=cols)
        wr.writeheader()
        for r in kept + rows:
            wr.writerow({c: r.get(c, "") for c in cols})


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", action="append", choices=sorted(SHAPES), required=True)
    ap.add_argument("--tokens", default=None, help="comma-separated token counts")
    ap.add_argument("--reps", type=int, default=15)
    ap.add_argument("--out", default=build.CONFIG_CSV)
    args = ap.parse_args()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = wl.l2_flush_buffer(dev)
    rows = []
    for name in args.workload:
        sh = SHAPES[name]
        tokens = ([int(t) for t in args.tokens.split(",")] if args.tokens else list(sh["tokens"]))
        v13, w2, s2, keep = make_weights(sh, dev)
        print(f"{name}: H={sh['H']} I={sh['I']} E={sh['E']} k={sh['k']} "
              f"{'mxfp4' if sh['mxfp4'] else 'bf16'}", flush=True)
        prev = 0
        for i, T in enumerate(sorted(tokens)):
            best, us, us_def, n = tune_one(sh, T, v13, w2, s2, flush, args.reps, dev,
                                           lambda m: print(m, flush=True))
            t_hi = T if i + 1 < len(tokens) else T_MAX
            row = {"wdtype": "mxfp4" if sh["mxfp4"] else "bf16", "H": sh["H"], "I": sh["I"],
                   "E": sh["E"], "k": sh["k"], "t_lo": prev + 1, "t_hi": t_hi,
                   "us": f"{us:.1f}", "us_default": f"{us_def:.1f}", "candidates": n}
            for f in moe._abi.CONFIG_FLAGS:
                row[f] = best[f]
            rows.append(row)
            prev = T
        del keep, v13, w2, s2
        torch.cuda.empty_cache()
    merge_rows(args.out, rows)
    print(f"wrote {len(rows)} rows to {args.out}")


if __name__ == "__main__":
    main()
