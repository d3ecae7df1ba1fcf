import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case")


def pytest_collection_modifyitems(config, items):
    import torch

    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def mx_weights(E, I, H, seed=0):
    """MXFP4 expert weights on the host: fp32 N(0, 1/sqrt(fan_in)) drawn expert by
    expert and quantised with the oracle's 1x32 rule.  (codes13, scales13, codes2, scales2)"""
    import torch

    import oracle
    from mixture_experts_layer_46_b200 import workloads as wl

    c13 = torch.empty(E, 2 * I, H // 2, dtype=torch.uint8)
    s13 = torch.empty(E, 2 * I, H // 32, dtype=torch.uint8)
    c2 = torch.empty(E, H, I // 2, dtype=torch.uint8)
    s2 = torch.empty(E, H, I // 32, dtype=torch.uint8)
    for e, w13e, w2e in wl.iter_weights_fp32(E, I, H, seed=seed):
        c13[e], s13[e] = oracle.mxfp4_quantize(w13e)
        c2[e], s2[e] = oracle.mxfp4_quantize(w2e)
    return c13, s13, c2, s2


@pytest.fixture(scope="session")
def qwen3_weights():
    """Qwen3-235B-shaped expert weights (seed 0) on the GPU and a host copy for the oracle."""
    from mixture_experts_layer_46_b200 import workloads as wl

    s = wl.QWEN3_235B
    w13, w2 = wl.make_weights_bf16(s.E, s.I, s.H, seed=0, device="cuda")
    return {"w13": w13, "w2": w2, "w13_cpu": w13.cpu(), "w2_cpu": w2.cpu()}


@pytest.fixture(scope="session")
def glm_weights():
    """GLM-4.5-Air-shaped expert weights (seed 0) on the GPU and a host copy for the oracle."""
    from mixture_experts_layer_46_b200 import workloads as wl

    s = wl.GLM45_AIR
    w13, w2 = wl.make_weights_bf16(s.E, s.I, s.H, seed=0, device="cuda")
    return {"w13": w13, "w2": w2, "w13_cpu": w13.cpu(), "w2_cpu": w2.cpu()}


@pytest.fixture(scope="session")
def tp2_weights():
    """Qwen3.5-397B TP2 MXFP4 expert weights for E = 513 (seed 0), host and GPU.  The
    weights are drawn expert by expert, so the first 512 are exactly the E = 512 layer's."""
    from mixture_experts_layer_46_b200 import workloads as wl

    s = wl.QWEN35_TP2_MXFP4_SHARED
    c13, s13, c2, s2 = mx_weights(s.E, s.I, s.H, seed=0)
    cpu = {"c13": c13, "s13": s13, "c2": c2, "s2": s2}
    return {"cpu": cpu, "gpu": {k: v.cuda() for k, v in cpu.items()}}
