"""The kernels' failure path, exercised without faulting the GPU: every wait in
the forward's kernels gives up after a time limit, counts a timeout and lets the
kernel return.  moe_selftest_bounded_wait runs that same bounded wait on an
mbarrier nothing arrives on (no copy or tensor-core operation in flight), with a
1 ms limit; the timeout must be counted, reported as MOE_ERR_DEVICE_TIMEOUT and
cleared by the read, and the context must stay usable."""

import ctypes

import pytest
import torch

import mixture_experts_layer_46_b200 as moe
from mixture_experts_layer_46_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_is_reported():
    lib = moe.load()
    moe.device_errors()  # clear
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert lib.moe_selftest_bounded_wait(1000, done.data_ptr(), st) == 0
    torch.cuda.synchronize()
    assert int(done.item()) == 2
    nb, to = ctypes.c_uint32(0), ctypes.c_uint32(0)
    rc = lib.moe_get_device_errors(st, ctypes.byref(nb), ctypes.byref(to))
    assert rc == 8 and nb.value == 0 and to.value == 1   # MOE_ERR_DEVICE_TIMEOUT
    assert moe.device_errors() == (0, 0)                  # the read cleared it
    # the context is still usable: a forward runs and reports no timeout
    s = wl.TINY
    w13, w2 = wl.make_weights_bf16(s.E, s.I, s.H, seed=0, device="cuda")
    x = wl.make_x(s.T, s.H, seed=1, device="cuda")
    ids, wts = wl.route_softmax_topk(s.T, s.E, s.k, seed=2, device="cuda")
    out = moe.forward(x, moe.w13_from_packed(w13), w2, ids, wts)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert moe.device_errors() == (0, 0)


def test_bounded_wait_rejects_limits_outside_the_range():
    lib = moe.load()
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert lib.moe_selftest_bounded_wait(0, done.data_ptr(), st) == 1
    assert lib.moe_selftest_bounded_wait(100001, done.data_ptr(), st) == 1
    assert lib.moe_selftest_bounded_wait(10, None, st) == 1
    torch.cuda.synchronize()
    assert int(done.item()) == 0
