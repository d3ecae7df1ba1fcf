"""moe_align_noalloc: the align step for callers that cannot allocate device
memory (e.g. a plugin inside an engine whose memory is already split between
its own pools) and so cannot pass a workspace either.  It keeps its scratch
in a fixed array inside the library.

Checked here through the C ABI: on two calls in a row (different routing, so
the second call starts from the first call's leftover scratch) its outputs
equal, bit for bit (align is integer work, so the tolerance is exact
equality), both those of moe_align, which uses a caller-provided workspace, and
those of the CPU oracle's align.  The second routing holds out-of-range ids,
which both skip.  The problem size uses the multi-CTA path, so both scratch
regions are exercised.  Oversized problems are refused.

This file sorts last so a run that stops at the first failure has already run
every other test.
"""

import ctypes

import pytest
import torch

import mixture_experts_layer_46_b200 as moe
import oracle
from mixture_experts_layer_46_b200 import _abi
from mixture_experts_layer_46_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _outputs(ids: torch.Tensor, E: int, bm: int):
    """Output buffers of one call (the caller's own memory, allocated up front)."""
    T, k = ids.shape
    S = T * k
    pmax = S + min(E, S) * (bm - 1) + bm
    dev = ids.device
    return {"counts": torch.full((E,), -1, dtype=torch.int32, device=dev),
            "offsets": torch.full((E + 1,), -1, dtype=torch.int32, device=dev),
            "sorted": torch.full((pmax,), -7, dtype=torch.int32, device=dev),
            "block_expert": torch.full((pmax // bm + 1,), -7, dtype=torch.int32, device=dev),
            "nb": torch.zeros(1, dtype=torch.int32, device=dev)}


def _call(ids: torch.Tensor, E: int, bm: int, o: dict) -> int:
    d = _abi.desc(ids)
    return moe.load().moe_align_noalloc(ctypes.byref(d), E, bm, o["counts"].data_ptr(),
                                        o["offsets"].data_ptr(), o["sorted"].data_ptr(),
                                        o["block_expert"].data_ptr(), o["nb"].data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)


def _result(o: dict, E: int):
    torch.cuda.synchronize()
    P = int(o["offsets"][E].item())
    n = int(o["nb"].item())
    return {"counts": o["counts"], "offsets": o["offsets"], "sorted": o["sorted"][:P],
            "block_expert": o["block_expert"][:n], "num_blocks": n}


def _noalloc(ids: torch.Tensor, E: int, bm: int):
    o = _outputs(ids, E, bm)
    rc = _call(ids, E, bm, o)
    assert rc == 0, _abi.STATUS.get(rc, rc)
    return _result(o, E)


def _same(a, b):
    assert a["num_blocks"] == b["num_blocks"]
    for key in ("counts", "offsets", "sorted", "block_expert"):
        assert torch.equal(a[key].cpu(), b[key].cpu()), key


def test_noalloc_align_matches_workspace_align_twice():
    E, bm = 128, 128
    ids1, _ = wl.route_softmax_topk(4096, E, 8, seed=11, device="cuda")
    ids_all, _ = wl.route_zipf_layers(3000, E, 8, layers=46, seed=12, device="cuda")
    ids_all[5, 23, 3] = -1      # out-of-range ids: skipped by every implementation
    ids_all[77, 23, 0] = E
    ids2 = ids_all[:, 23, :]  # strided slice, token stride 368
    first = _noalloc(ids1, E, bm)
    ref1 = moe.align(ids1, E, bm)
    torch.cuda.synchronize()
    _same(first, ref1)
    _same(first, oracle.moe_align(ids1.cpu(), E, bm))
    out2 = _outputs(ids2, E, bm)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    rc = _call(ids2, E, bm, out2)           # only the call itself sits between the readings
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    alloc1 = torch.cuda.memory_allocated()
    assert rc == 0, _abi.STATUS.get(rc, rc)
    second = _result(out2, E)
    ref2 = moe.align(ids2, E, bm)
    torch.cuda.synchronize()
    _same(second, ref2)
    _same(second, oracle.moe_align(ids_all.cpu()[:, 23, :], E, bm))
    assert int(second["counts"].sum().item()) == 3000 * 8 - 2
    # the call itself allocated nothing: neither through torch's allocator nor on
    # the device (device-wide free memory also moves if another process on the
    # same GPU allocates, so this assumes the GPU is not shared meanwhile)
    assert alloc1 == alloc0
    assert free1 == free0


def test_noalloc_align_refuses_oversized_problem():
    T, k = (1 << 20) // 8 + 1, 8  # one token past the fixed scratch
    ids = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    d = _abi.desc(ids)
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    rc = moe.load().moe_align_noalloc(ctypes.byref(d), 8, 128, p, p, p, p, p,
                                      torch.cuda.current_stream().cuda_stream)
    assert rc == 5  # MOE_ERR_WORKSPACE_TOO_SMALL, nothing launched
    torch.cuda.synchronize()
    assert torch.all(dummy == 0)
