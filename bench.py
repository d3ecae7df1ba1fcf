#!/usr/bin/env python
"""Throughput of the fused MoE expert forward on B200.

Default workload: the Qwen3-235B-shaped MoE layer, bf16, H=4096, I=1536,
E=128, top_k=8, T=4096 tokens, packed w13 [E, 2I, H] read through its
expert-strided gate/up views (Liger-Kernel PR #1377).  One step is one full
forward (align -> permute -> GEMM1+SwiGLU -> GEMM2+weight -> combine) over one
batch of T tokens, inputs resident in HBM; the L2 is flushed (512 MB write,
then 384 MB of it read back so no dirty line is left) before every timed step,
outside the timed events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qwen3-235b|glm45-air|tiny] [--T T] [--sweep FILE]

Multi-GPU runs (torchrun, one process per GPU) are independent replicas: each
rank runs the same layer on its own batch, no collective on the data path
(weak scaling); timing is the max over ranks.  The reference arm times the
fp64 CPU oracle on the host cores on a bounded token sample of the same
workload.  Prints one JSON line (rank 0).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "fused-MoE layer tokens/s (us/call) on 1 B200"
UNIT = "tokens/s"

WORKLOADS = {
    "qwen3-235b": dict(H=4096, I=1536, E=128, k=8, T=4096, routing="softmax"),
    "glm45-air": dict(H=4096, I=1408, E=128, k=8, T=16384, routing="zipf-layer-slice"),
    "tiny": dict(H=256, I=128, E=8, k=2, T=64, routing="softmax"),
    "qwen35-tp2-mxfp4": dict(H=4096, I=512, E=512, k=10, T=4096, routing="softmax", mxfp4=True),
    "qwen35-tp2-mxfp4-shared": dict(H=4096, I=512, E=513, k=11, T=4096, routing="shared",
                                    mxfp4=True),
}

# DRAM traffic per launch of the dominant kernel from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed to the hash of the kernel
# source it was taken on; reported as null once the source has changed.
NCU_TRAFFIC = {
    # GEMM1 on the benchmarked workload (T=4096, E=128, the table's configuration for that
    # bucket: gate/up interleaved on 256-row pair tiles), one-pass ncu capture at the full
    # size: 3.805 GB read + 0.107 GB written per launch; reported only while the GEMM
    # sources and the configuration hash to `src` (the hash the capturing run printed)
    "qwen3-235b": {"T": 4096, "E": 128, "bytes_per_launch": 3.8048e9 + 0.10703e9,
                   "src": "dc8721d8a820bb53"},
}


def kernel_src_hash(config: dict) -> str:
    """Hash of the sources of the GEMM kernels the timed forward's weight type runs, and
    of its configuration: a recorded traffic figure is reported only while both are
    unchanged."""
    h = hashlib.sha256()
    mx = config.get("wdtype") == 4
    files = (("moe_gemm_mxfp4.cu", "moe_mx.cuh") if mx else
             ("moe_gemm_ws.cu", "moe_gemm_ws2.cu", "moe_gemm_il.cu", "moe_pair.cuh"))
    for fn in files + ("moe_common.cuh",):
        with open(os.path.join(ROOT, "mixture_experts_layer_46_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    h.update(json.dumps({k: config[k] for k in sorted(config) if k not in ("t_lo", "t_hi")}).encode())
    return h.hexdigest()[:16]


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# Dense FP4 (kind::mxf4) tensor rate measured on this machine's B200s with the
# library's MMA-rate probe (moe_measure_mma_peak: back-to-back M=128 N=128 MMAs
# from shared memory on all 148 SMs, CUDA events, best of five launches of
# 100000 x 4 instructions per SM), beside the same probe's bf16 rate.  The
# MXFP4 roofline takes the measured bf16 GEMM burst peak x their ratio.
FP4_PEAK = {"bf16_tflops": 2231.4, "mxf4_tflops": 8925.7,
            "note": "MMA-rate probe on one B200: bf16 2231 TFLOP/s, mxf4 8926 TFLOP/s"}


def fp4_peak(bf16_burst: float):
    """(peak TFLOP/s, source) for kind::mxf4: the measured probe figure scaled to the
    burst bf16 peak by the probe's own mxf4/bf16 ratio, else the nominal 4x ratio."""
    if FP4_PEAK:
        ratio = FP4_PEAK["mxf4_tflops"] / FP4_PEAK["bf16_tflops"]
        return bf16_burst * ratio, (f"measured bf16 burst peak x the measured mxf4/bf16 MMA-rate "
                                    f"ratio {ratio:.3f} ({FP4_PEAK['note']})")
    return bf16_burst * 4.0, "measured bf16 burst peak x4 nominal FP4/bf16 ratio (FP4 peak not measured)"


def workload_name(w) -> str:
    dt = "mxfp4 (e2m1 + e8m0 per 1x32)" if w.get("mxfp4") else "bf16"
    return (f"moe-layer {dt} T={w['T']} H={w['H']} I={w['I']} E={w['E']} top_k={w['k']} "
            f"packed-strided-w13 routing={w['routing']}")


def make_mx_weights(w, device):
    """MXFP4 weights: fp32 N(0, 1/sqrt(fan_in)) drawn expert by expert and quantised
    with the library's 1x32 quantiser (the bench times the forward, not this)."""
    import mixture_experts_layer_46_b200 as moe
    from mixture_experts_layer_46_b200 import workloads as wl

    E, I, H = w["E"], w["I"], w["H"]
    c13 = torch.empty(E, 2 * I, H // 2, dtype=torch.uint8, device=device)
    s13 = torch.empty(E, 2 * I, H // 32, dtype=torch.uint8, device=device)
    c2 = torch.empty(E, H, I // 2, dtype=torch.uint8, device=device)
    s2 = torch.empty(E, H, I // 32, dtype=torch.uint8, device=device)
    for e, w13e, w2e in wl.iter_weights_fp32(E, I, H, seed=0, device=device):
        c13[e], s13[e] = moe.quantize_mxfp4(w13e)
        c2[e], s2[e] = moe.quantize_mxfp4(w2e)
    return c13, s13, c2, s2


def make_inputs(w, device, seed_offset=0):
    from mixture_experts_layer_46_b200 import workloads as wl

    if w.get("mxfp4"):
        c13, s13, c2, s2 = make_mx_weights(w, device)
        w13, w2 = c13, c2
        scales = (s13, s2)
    else:
        w13, w2 = wl.make_weights_bf16(w["E"], w["I"], w["H"], seed=0, device=device)
        scales = None
    x = wl.make_x(w["T"], w["H"], seed=1 + seed_offset, device=device)
    if w["routing"] == "softmax":
        ids, wts = wl.route_softmax_topk(w["T"], w["E"], w["k"], seed=2 + seed_offset, device=device)
        keep = None
    elif w["routing"] == "shared":
        ids, wts = wl.route_shared_expert(w["T"], w["E"] - 1, w["k"] - 1, seed=2 + seed_offset,
                                          device=device)
        keep = None
    else:
        ids_all, w_all = wl.route_zipf_layers(w["T"], w["E"], w["k"], layers=46, seed=7 + seed_offset,
                                              device=device)
        ids, wts = ids_all[:, 23, :], w_all[:, 23, :]
        keep = (ids_all, w_all)
    return {"x": x, "w13": w13, "w2": w2, "ids": ids, "wts": wts, "keep": keep, "scales": scales}


def algorithmic(w, ids):
    """Algorithmic FLOPs and bytes of one forward and of GEMM1 alone."""
    H, I, E, k, T = w["H"], w["I"], w["E"], w["k"], w["T"]
    idc = ids.reshape(-1).long()
    valid = idc[(idc >= 0) & (idc < E)]
    n_slots = int(valid.numel())
    n_act = int(torch.unique(valid).numel())
    wbytes = (0.5 + 1.0 / 32.0) if w.get("mxfp4") else 2.0   # per weight element
    flops = 6.0 * H * I * n_slots
    bytes_total = 3.0 * I * H * wbytes * n_act + 2.0 * T * H * 2 + 8.0 * T * k
    g1_flops = 4.0 * H * I * n_slots
    abytes = (0.5 + 1.0 / 32.0) if w.get("mxfp4") else 2.0
    g1_bytes = 2.0 * I * H * wbytes * n_act + T * H * abytes
    return dict(flops=flops, bytes=bytes_total, gemm1_flops=g1_flops, gemm1_bytes=g1_bytes,
                slots=n_slots, active_experts=n_act)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.lines = []
        self.dev = device_index

    def start(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def oracle_runner(inp, w):
    """A closure that runs the fp64 oracle on a list of token indices of the workload."""
    import oracle
    from mixture_experts_layer_46_b200 import workloads as wl

    cpu = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()
           if k != "scales"}
    if inp["keep"] is not None:
        ids_all, w_all = (t.cpu() for t in inp["keep"])
        cpu["ids"], cpu["wts"] = ids_all[:, 23, :], w_all[:, 23, :]
    gate, up = wl.gate_up_views(cpu["w13"])
    scales = None
    if w.get("mxfp4"):
        s13, s2 = (t.cpu() for t in inp["scales"])
        sg, su = wl.gate_up_views(s13)
        scales = (sg, su, s2)

    def run(tokens, nthreads):
        oracle.moe_forward(cpu["x"], gate, up, cpu["w2"], cpu["ids"], cpu["wts"], scales=scales,
                           tokens=tokens, nthreads=nthreads)

    return run


def oracle_tokens_per_s(inp, w, budget_s, cores):
    """The fp64 oracle on a bounded sample of the workload's tokens."""
    run = oracle_runner(inp, w)
    g = torch.Generator().manual_seed(123)
    order = torch.randperm(w["T"], generator=g)
    # calibrate with one token per core, then size the sample to the budget
    n = max(1, cores)
    t0 = time.perf_counter()
    run(order[:n], cores)
    dt = time.perf_counter() - t0
    reps = max(1, int(budget_s / max(dt, 1e-6)))
    n2 = min(w["T"], n * reps)
    t0 = time.perf_counter()
    run(order[:n2], cores)
    dt2 = time.perf_counter() - t0
    return n2 / dt2, n2, dt2


def run_reference(args, w, rank):
    if rank != 0:
        return
    cores = os.cpu_count() or 1
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(w, dev)
    run = oracle_runner(inp, w)
    order = torch.randperm(w["T"], generator=torch.Generator().manual_seed(123))
    per_step_budget = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    # tokens per step: one per core, grown while it fits the per-step budget
    t0 = time.perf_counter()
    run(order[:cores], cores)
    dt = time.perf_counter() - t0
    n = max(1, min(w["T"], int(cores * max(1.0, per_step_budget / max(dt, 1e-6)))))
    times = []
    for step in range(args.warmup + args.steps):
        toks = order[(step * n) % w["T"]:][:n]
        if toks.numel() < n:
            toks = order[:n]
        t0 = time.perf_counter()
        run(toks, cores)
        if step >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = n / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) activations, N(0,1/sqrt(fan_in)) weights)",
            "config": {"workload": workload_name(w), "tokens_per_step_sample": n,
                       "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{n} of {w['T']} tokens per step (all their {w['k']} slots), fp64 C++ loop, OpenMP over tokens"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def init_replicas(world: int, local: int, backend: str = "nccl") -> bool:
    """Process group of the N independent replicas (torchrun env: RANK, WORLD_SIZE, MASTER_*):
    NCCL on the GPUs, gloo in the CPU tests.  The short timeout turns a rank that never arrives
    into an error on the others instead of a hang."""
    if world <= 1:
        return False
    import datetime

    import torch.distributed as dist

    kw = {}
    if backend == "nccl":
        torch.cuda.set_device(local)
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return True


def max_over_ranks(x: float, pg: bool, device) -> float:
    """The slowest replica's figure; every rank calls it at the same point of the run."""
    if not pg:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, tokens_per_rank: int, ms: float) -> float:
    """Whole-job tokens/s: each of the `world` replicas runs its own batch of tokens_per_rank
    tokens, and the job takes the slowest replica's ms (weak scaling)."""
    return world * tokens_per_rank / (ms * 1e-3)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen3-235b", choices=sorted(WORKLOADS))
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--E", type=int, default=None, help="override the expert count (profiling)")
    ap.add_argument("--sweep", default=None, help="write a token-sweep JSONL here (extra lines)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--grad", action="store_true",
                    help="time the gradient (dx, the routing-weight and the expert-weight gradients) "
                         "instead of the forward; prints its own JSON line")
    ap.add_argument("--grad-weights", default="bf16", choices=["bf16", "fp32", "none"],
                    help="with --grad: the expert-weight gradients' dtype, or none for dx and the "
                         "routing-weight gradient alone (moe_backward_input_ws)")
    ap.add_argument("--config", default=None,
                    help="override configuration flags of the timed forward, e.g. fused=1,tile=32 "
                         "(installed with moe_set_config_table for this problem only)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    w = dict(WORKLOADS[args.workload])
    if args.T is not None:
        w["T"] = args.T
    if args.E is not None:
        w["E"] = args.E

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = init_replicas(world, local)

    if args.impl == "reference":
        run_reference(args, w, rank)
        if pg:
            import torch.distributed as dist

            dist.destroy_process_group()
        return

    import mixture_experts_layer_46_b200 as moe
    from mixture_experts_layer_46_b200 import workloads as wl

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    inp = make_inputs(w, dev)
    mx = bool(w.get("mxfp4"))
    s13, s2 = inp["scales"] if mx else (None, None)
    v13 = moe.w13_from_packed(inp["w13"], s13)
    ws = torch.empty(moe.workspace_bytes(w["T"], w["H"], w["I"], w["E"], w["k"], mxfp4=mx),
                     dtype=torch.uint8, device=dev)
    out = torch.empty(w["T"], w["H"], dtype=torch.bfloat16, device=dev)
    flush = wl.l2_flush_buffer(dev)

    def step():
        moe.forward(inp["x"], v13, inp["w2"], inp["ids"], inp["wts"], out=out, workspace=ws,
                    stream=stream, w2_scale=s2)

    if args.grad:
        if mx:
            raise SystemExit("--grad: the gradient path takes bf16 weights")
        run_grad(args, w, moe, wl, inp, v13, dev, stream, flush)
        return

    if args.config:
        flags = {kv.split("=")[0]: int(kv.split("=")[1]) for kv in args.config.split(",")}
        moe.config_override((w["T"], w["H"], w["I"], w["E"], w["k"]), mxfp4=mx, **flags).__enter__()

    for _ in range(args.warmup):
        step()
    launches_per_step = moe.last_launch_count()
    torch.cuda.synchronize(dev)

    # ---------------------------------------------------------------- timed region
    sampler = ClockSampler(dev.index)
    sampler.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    if pg:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        wl.flush_l2(flush, i)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if pg:
        torch.distributed.barrier()
    clocks = sampler.stop()
    per = [a.elapsed_time(b) for a, b in evs]
    ms = max_over_ranks(sum(per) / len(per), pg, dev)
    value = replica_throughput(world, w["T"], ms)

    # ---------------------------------------------------------------- per-step breakdown
    moe.profile_enable(True)
    brk = {}
    nb = min(args.steps, 20)
    for i in range(nb):
        wl.flush_l2(flush, i)
        step()
        for kname, kms in moe.profile_read().items():
            brk[kname] = brk.get(kname, 0.0) + kms / nb
    moe.profile_enable(False)

    # ---------------------------------------------------------------- end to end (host buffers)
    x_h = inp["x"].cpu().pin_memory()
    ids_h = inp["ids"].contiguous().cpu().pin_memory()
    w_h = inp["wts"].contiguous().cpu().pin_memory()
    out_h = torch.empty(w["T"], w["H"], dtype=torch.bfloat16).pin_memory()
    for _ in range(2):
        moe.forward_host(x_h, v13, inp["w2"], ids_h, w_h, out_h, stream=stream, w2_scale=s2)
    e2e_ms = []
    for i in range(min(args.steps, 50)):
        wl.flush_l2(flush, i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        moe.forward_host(x_h, v13, inp["w2"], ids_h, w_h, out_h, stream=stream, w2_scale=s2)
        e1.record(stream)
        e1.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    e2e_serial = max_over_ranks(sum(e2e_ms) / len(e2e_ms), pg, dev)
    # the same calls through the asynchronous host form, two in flight on two streams with
    # their own device staging and host outputs: each call's copies overlap the other's
    # kernels.  The weights (GBs) are larger than L2 and x is copied in by every call.
    streams2 = [stream, torch.cuda.Stream(dev)]
    hws = [torch.empty(moe.host_workspace_bytes(w["T"], w["H"], w["I"], w["E"], w["k"], mxfp4=mx),
                       dtype=torch.uint8, device=dev) for _ in streams2]
    outs_h = [out_h, torch.empty_like(out_h).pin_memory()]

    def host_call(i):
        moe.forward_host(x_h, v13, inp["w2"], ids_h, w_h, outs_h[i % 2], stream=streams2[i % 2], w2_scale=s2,
                         workspace=hws[i % 2])

    for i in range(4):
        host_call(i)
    torch.cuda.synchronize(dev)
    n_pipe = min(args.steps, 50)
    wl.flush_l2(flush, 0)
    torch.cuda.synchronize(dev)
    p0, p1, pj = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                  torch.cuda.Event())
    p0.record(streams2[0])
    streams2[1].wait_event(p0)
    for i in range(n_pipe):
        host_call(i)
    pj.record(streams2[1])
    streams2[0].wait_event(pj)
    p1.record(streams2[0])
    p1.synchronize()
    e2e = max_over_ranks(p0.elapsed_time(p1) / n_pipe, pg, dev)
    h2d = x_h.numel() * 2 + ids_h.numel() * ids_h.element_size() + w_h.numel() * 4
    d2h = out_h.numel() * 2

    # ---------------------------------------------------------------- roofline
    hbm, tf_burst, tf_sus, src = peaks()
    fp4_src = None
    if mx:
        tf_burst, fp4_src = fp4_peak(tf_burst)
    alg = algorithmic(w, inp["ids"])
    g1_ms = brk.get("gemm1_swiglu", float("nan"))
    t_tc = alg["gemm1_flops"] / (tf_burst * 1e12)
    t_mem = alg["gemm1_bytes"] / (hbm * 1e9)
    if t_tc >= t_mem:
        roof = {"bound": "tensor", "achieved": alg["gemm1_flops"] / (g1_ms * 1e-3) / 1e12,
                "peak": tf_burst, "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": alg["gemm1_bytes"] / (g1_ms * 1e-3) / 1e9, "peak": hbm,
                "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    tr = NCU_TRAFFIC.get(args.workload)
    cfg_now = moe.get_config(w["T"], w["H"], w["I"], w["E"], w["k"], mxfp4=mx)
    same_case = tr is not None and tr.get("T") == w["T"] and tr.get("E") == w["E"]
    roof["traffic"] = (tr["bytes_per_launch"] if same_case and tr.get("src") == kernel_src_hash(cfg_now)
                       else None)
    roof["traffic_src"] = kernel_src_hash(cfg_now)
    pair = (not mx) and (w["T"] * w["k"] >= 32 * w["E"])
    roof["kernel"] = ("gemm1_swiglu (weight-stationary grouped gate/up GEMM + SwiGLU, tcgen05 "
                      + ("kind::mxf4 block-scaled)" if mx else
                         ("kind::f16 on CTA pairs)" if pair else "kind::f16)")))
    roof["peak_source"] = (f"{src} (MEASURED_PEAKS.json burst)" if src == "measured" else "fallback")
    if mx and roof["bound"] == "tensor":
        roof["peak_source"] = fp4_src
    roof["scope"] = "the gemm1_swiglu kernel alone; layer_roofline covers the whole forward"
    t_roof_layer = max(alg["flops"] / (tf_burst * 1e12), alg["bytes"] / (hbm * 1e9))
    layer_frac = t_roof_layer / (ms * 1e-3)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e2m1/e8m0 (fp32 accumulate)" if mx else "bf16",
            "data": "synthetic (seeded N(0,1) activations, N(0,1/sqrt(fan_in)) random-init weights)",
            "config": {"workload": workload_name(w), "tokens_per_gpu": w["T"],
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "flushed before every timed step, outside the events: 512 MB written, "
                             "then 384 MB of it read back (clean L2, no write-back in the step)",
                       "us_per_call": ms * 1e3,
                       "us_per_call_p10": sorted(per)[len(per) // 10] * 1e3,
                       "us_per_call_p90": sorted(per)[(9 * len(per)) // 10] * 1e3},
            "roofline": roof,
            "layer_roofline": {"t_roof_us": t_roof_layer * 1e6, "frac": layer_frac,
                               "flops": alg["flops"], "bytes": alg["bytes"],
                               "active_experts": alg["active_experts"]},
            "step_breakdown_ms": brk,
            "e2e": {"value": replica_throughput(world, w["T"], e2e), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e,
                    "api": "moe_forward_host_ws (pinned host x/ids/weights in, host out; two calls in "
                           "flight on two streams, each call's copies overlapping the other's kernels)",
                    "serial_ms_per_step": e2e_serial,
                    "serial_api": "moe_forward_host (one call at a time, stream synchronised in the call; "
                                  "L2 flushed before each)"},
            "gpu_launches": launches_per_step * args.steps,
            "kernel_config": moe.get_config(w["T"], w["H"], w["I"], w["E"], w["k"], mxfp4=mx),
            "clocks": clocks}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        tps, n, dt = oracle_tokens_per_s(inp, w, 12.0, cores)
        line["cpu_baseline"] = {"value": tps, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"{n} of {w['T']} tokens (all their slots) in {dt:.1f} s, fp64 C++ loop, OpenMP over tokens"}

    if args.sweep and rank == 0:
        sweep(args, w, moe, wl, dev, stream, flush)

    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_grad(args, w, moe, wl, inp, v13, dev, stream, flush):
    """The full gradient (moe_backward_ws: dx, the routing-weight gradient and the
    expert-weight gradients) on the forward's workload, timed like the forward: L2
    flushed clean before every step, CUDA events, clocks sampled.  Roofline: 16 H I
    FLOPs per slot (dh' = w2^T dout 2, the gate/up recompute 4, da 4, dw2 2, dw13 4;
    10 without the weight gradients) at the bf16 burst peak against the HBM time of the
    activated experts' weights as the path must read them (w2 once, for dh'; w13 twice,
    for the gate/up recompute and for da: 5 I H bf16 values per expert, five thirds of
    the weights), the weight gradients of all E experts written, and x, dout and dx."""
    hbm, tf_burst, _, _ = peaks()
    T, H = w["T"], w["H"]
    w13t = moe.transpose_experts(inp["w13"])
    w2t = moe.transpose_experts(inp["w2"])
    dout = wl.make_x(T, H, seed=3, device=dev)
    dx = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    dwt = torch.empty(T, w["k"], dtype=torch.float32, device=dev)
    gws = torch.empty(moe.backward_workspace_bytes(T, H, w["I"], w["E"], w["k"]), dtype=torch.uint8,
                      device=dev)
    # weight gradients by default in the weights' own dtype (bf16), as an autograd framework
    # keeps them; fp32, or none (dx and the routing-weight gradient alone), on request
    gw = args.grad_weights
    gdt = torch.float32 if gw == "fp32" else torch.bfloat16
    dw13 = torch.empty(w["E"], 2 * w["I"], H, dtype=gdt, device=dev) if gw != "none" else None
    dw2 = torch.empty(w["E"], H, w["I"], dtype=gdt, device=dev) if gw != "none" else None

    def gstep():
        moe.backward(inp["x"], v13, inp["w2"], w13t, w2t, inp["ids"], inp["wts"], dout, dx, dwt, dw13, dw2,
                     weights=gw != "none", workspace=gws, stream=stream)

    for _ in range(args.warmup):
        gstep()
    launches = moe.last_launch_count()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index)
    sampler.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        wl.flush_l2(flush, i)
        evs[i][0].record(stream)
        gstep()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    per = sorted(a.elapsed_time(b) for a, b in evs)
    ms = sum(per) / len(per)
    alg = algorithmic(w, inp["ids"])
    flops = alg["flops"] * 16.0 / 6.0  # the forward's 6 H I per slot
    wread = 5.0 * w["I"] * H * 2.0 * alg["active_experts"]
    if gw == "none":
        flops = alg["flops"] * 10.0 / 6.0
        gbytes = wread + 3.0 * T * H * 2
    else:
        gbytes = wread + 3.0 * w["I"] * H * gdt.itemsize * w["E"] + 3.0 * T * H * 2
    t_roof = max(flops / (tf_burst * 1e12), gbytes / (hbm * 1e9))
    print(json.dumps({
        "metric": "fused-MoE layer gradient (dx, routing weights, expert weights) tokens/s on 1 B200",
        "value": T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16",
        "config": {"workload": workload_name(w) + " gradient", "tokens_per_gpu": T,
                   "weight_gradients": gw,
                   "us_per_call_p10": per[len(per) // 10] * 1e3,
                   "us_per_call_p90": per[(9 * len(per)) // 10] * 1e3},
        "roofline": {"t_roof_us": t_roof * 1e6, "frac": t_roof / (ms * 1e-3), "flops": flops,
                     "bytes": gbytes, "bound": "tensor" if flops / (tf_burst * 1e12) > gbytes / (hbm * 1e9) else "hbm"},
        "gpu_launches": launches * args.steps, "clocks": clocks}), flush=True)


def sweep(args, w, moe, wl, dev, stream, flush):
    """Token sweep on the same weights (fresh routing per T): one JSONL row per T."""
    hbm, tf_burst, _, _ = peaks()
    mx = bool(w.get("mxfp4"))
    fp4_src = None
    if mx:
        tf_burst, fp4_src = fp4_peak(tf_burst)
        c13, s13, w2, s2 = make_mx_weights(w, dev)
        v13 = moe.w13_from_packed(c13, s13)
        tokens = wl.MXFP4_TOKEN_SWEEP
    else:
        w13, w2 = wl.make_weights_bf16(w["E"], w["I"], w["H"], seed=0, device=dev)
        v13 = moe.w13_from_packed(w13)
        s2 = None
        tokens = wl.TOKEN_SWEEP
    with open(args.sweep, "w") as f:
        for T in tokens:
            wt = dict(w, T=T)
            x = wl.make_x(T, w["H"], seed=2000 + T, device=dev)
            if w["routing"] == "shared":
                ids, wts = wl.route_shared_expert(T, w["E"] - 1, w["k"] - 1, seed=1000 + T, device=dev)
            else:
                ids, wts = wl.route_softmax_topk(T, w["E"], w["k"], seed=1000 + T, device=dev)
            ws = torch.empty(moe.workspace_bytes(T, w["H"], w["I"], w["E"], w["k"], mxfp4=mx),
                             dtype=torch.uint8, device=dev)
            out = torch.empty(T, w["H"], dtype=torch.bfloat16, device=dev)
            for _ in range(5):
                moe.forward(x, v13, w2, ids, wts, out=out, workspace=ws, stream=stream, w2_scale=s2)
            reps = 50 if T < 8192 else 20 if T <= 16384 else 10
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(reps)]
            sampler = ClockSampler(dev.index)
            sampler.start()
            torch.cuda.synchronize(dev)
            for i in range(reps):
                wl.flush_l2(flush, i)
                evs[i][0].record(stream)
                moe.forward(x, v13, w2, ids, wts, out=out, workspace=ws, stream=stream, w2_scale=s2)
                evs[i][1].record(stream)
            torch.cuda.synchronize(dev)
            clocks = sampler.stop()
            per = [a.elapsed_time(b) for a, b in evs]
            med = statistics.median(per)
            moe.profile_enable(True)
            brk = {}
            for i in range(5):
                wl.flush_l2(flush, i)
                moe.forward(x, v13, w2, ids, wts, out=out, workspace=ws, stream=stream, w2_scale=s2)
                for kname, kms in moe.profile_read().items():
                    brk[kname] = brk.get(kname, 0.0) + kms * 1e3 / 5
            moe.profile_enable(False)
            alg = algorithmic(wt, ids)
            t_roof = max(alg["flops"] / (tf_burst * 1e12), alg["bytes"] / (hbm * 1e9))
            row = {"T": T, "workload": workload_name(wt), "us_median": med * 1e3,
                   "us_p10": sorted(per)[len(per) // 10] * 1e3,
                   "us_p90": sorted(per)[(9 * len(per)) // 10] * 1e3, "reps": reps,
                   "tokens_per_s": T / (med * 1e-3),
                   "roofline_us": t_roof * 1e6, "frac": t_roof / (med * 1e-3),
                   "bound": "tensor" if alg["flops"] / (tf_burst * 1e12) >= alg["bytes"] / (hbm * 1e9) else "hbm",
                   "fp4_peak": fp4_src if mx else None, "clocks": clocks,
                   "config": moe.get_config(T, w["H"], w["I"], w["E"], w["k"], mxfp4=mx),
                   "hbm_GBs_alg": alg["bytes"] / (med * 1e-3) / 1e9,
                   "tflops_alg": alg["flops"] / (med * 1e-3) / 1e12,
                   "active_experts": alg["active_experts"],
                   "step_us": {k: round(v, 1) for k, v in brk.items()}}
            f.write(json.dumps(row) + "\n")
            f.flush()
            del ws, out


if __name__ == "__main__":
    main()
