"""CPU fp64 oracle for the fused MoE expert forward.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product path
never does: the library fails loudly when its CUDA extension is missing instead
of falling back to anything in here.

The arithmetic lives in ``moe_oracle.cpp`` (plain loops, double precision,
every element read through its strides); this module compiles it with g++ and
marshals torch CPU tensors into its strided-view descriptors.  It shares no code
with ``mixture_experts_layer_46_b200`` and never imports it.

Parity pins: tests/test_oracle_pins.py (brute force against a dense numpy
formulation, the one-expert special case against a textbook SwiGLU MLP, the
invariants), tests/test_oracle_mxfp4_pins.py (the MXFP4 worked examples and
brute-force quantiser), tests/test_oracle_router_pins.py (the router against
torch's softmax and sort, brute force, ties and invariants) and
tests/test_oracle_backward_pins.py (the input and routing-weight gradient against
central finite differences of the oracle forward and against torch autograd of a
dense fp64 formulation).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

OR_BF16, OR_F32, OR_I32, OR_I64, OR_E2M1X2 = 0, 1, 2, 3, 4


class OracleTensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("ndim", ctypes.c_int32),
        ("sizes", ctypes.c_int64 * 4),
        ("strides", ctypes.c_int64 * 4),
        ("scale", ctypes.c_void_p),
        ("scale_strides", ctypes.c_int64 * 4),
    ]


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/libmoe_oracle.so (g++, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c++17", _SRC, "-o", _LIB]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.POINTER
            lib.oracle_e2m1_value.restype = ctypes.c_double
            lib.oracle_e2m1_value.argtypes = [ctypes.c_uint32]
            lib.oracle_mxfp4_quantize.restype = ctypes.c_int
            lib.oracle_mxfp4_quantize.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                  ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
            lib.oracle_moe_align.restype = ctypes.c_int
            lib.oracle_moe_align.argtypes = [P(OracleTensor), ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                             ctypes.c_void_p, ctypes.c_void_p]
            lib.oracle_moe_forward.restype = ctypes.c_int
            lib.oracle_moe_forward.argtypes = [P(OracleTensor)] * 6 + [
                ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                ctypes.c_int]
            lib.oracle_moe_backward_input.restype = ctypes.c_int
            lib.oracle_moe_backward_input.argtypes = [P(OracleTensor)] * 7 + [
                ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
            lib.oracle_moe_backward_weights.restype = ctypes.c_int
            lib.oracle_moe_backward_weights.argtypes = [P(OracleTensor)] * 7 + [ctypes.c_void_p] * 3
            lib.oracle_router_topk.restype = ctypes.c_int
            lib.oracle_router_topk.argtypes = [P(OracleTensor), ctypes.c_int64, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
            lib.oracle_e8m0_value.restype = ctypes.c_double
            lib.oracle_e8m0_value.argtypes = [ctypes.c_uint32]
            lib.oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


_DT = {torch.bfloat16: OR_BF16, torch.float32: OR_F32, torch.int32: OR_I32, torch.int64: OR_I64,
       torch.uint8: OR_E2M1X2}


def _desc(t: torch.Tensor, scale: torch.Tensor | None = None) -> OracleTensor:
    assert t.device.type == "cpu", "the oracle reads host memory only"
    d = OracleTensor()
    d.data = t.data_ptr()
    d.dtype = _DT[t.dtype]
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.sizes[i] = t.shape[i]
        d.strides[i] = t.stride(i)
    if t.dtype == torch.uint8:
        # packed e2m1 pairs: logical innermost size is twice the byte count
        d.sizes[t.dim() - 1] = 2 * t.shape[-1]
        assert scale is not None and scale.dtype == torch.uint8
        d.scale = scale.data_ptr()
        for i in range(scale.dim()):
            d.scale_strides[i] = scale.stride(i)
    return d


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def e2m1_value(code: int) -> float:
    return float(_load().oracle_e2m1_value(code))


def e8m0_value(code: int) -> float:
    return float(_load().oracle_e8m0_value(code))


def moe_backward_input(x, gate, up, w2, ids, weights, dout, *, tokens=None, nthreads=0):
    """fp64 gradient of the bf16 forward with respect to x and topk_weights (experts
    frozen), given dout = dL/dout [T, H].  Returns (dx [n, H], dweights [n, k]) float64
    for the tokens listed (default all)."""
    d = [_desc(v) for v in (x, gate, up, w2, ids, weights, dout)]
    T, H = x.shape
    k = ids.shape[1]
    if tokens is not None:
        tokens = tokens.to(torch.int64).contiguous()
        n_out, tptr = tokens.numel(), tokens.data_ptr()
    else:
        n_out, tptr = T, None
    dx = torch.zeros(n_out, H, dtype=torch.float64)
    dw = torch.zeros(n_out, k, dtype=torch.float64)
    rc = _load().oracle_moe_backward_input(*[ctypes.byref(v) for v in d], tptr, n_out,
                                           dx.data_ptr(), dw.data_ptr(), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_moe_backward_input: shape mismatch")
    return dx, dw


def moe_backward_weights(x, gate, up, w2, ids, weights, dout):
    """fp64 gradient of the bf16 forward with respect to the expert weights given
    dout [T, H]: (dgate [E, I, H], dup [E, I, H], dw2 [E, H, I]) float64."""
    d = [_desc(v) for v in (x, gate, up, w2, ids, weights, dout)]
    E, I, H = gate.shape
    dg = torch.zeros(E, I, H, dtype=torch.float64)
    du = torch.zeros(E, I, H, dtype=torch.float64)
    dw2 = torch.zeros(E, H, I, dtype=torch.float64)
    rc = _load().oracle_moe_backward_weights(*[ctypes.byref(v) for v in d], dg.data_ptr(),
                                             du.data_ptr(), dw2.data_ptr())
    if rc != 0:
        raise ValueError("oracle_moe_backward_weights: shape mismatch")
    return dg, du, dw2


def router_topk(logits: torch.Tensor, k: int, renormalize: bool = True, shared_expert: bool = False):
    """fp64 router: softmax over the experts, the k most probable (lower index on
    ties), optionally renormalised; with shared_expert one more column holding
    expert E with weight 1.0.  Returns (ids int32 [T, kk], weights float64 [T, kk])."""
    T, E = logits.shape
    kk = k + (1 if shared_expert else 0)
    ids = torch.empty(T, kk, dtype=torch.int32)
    w = torch.empty(T, kk, dtype=torch.float64)
    d = _desc(logits)
    rc = _load().oracle_router_topk(ctypes.byref(d), k, 1 if renormalize else 0,
                                    1 if shared_expert else 0, ids.data_ptr(), w.data_ptr())
    if rc != 0:
        raise ValueError("oracle_router_topk: need 1 <= k <= E")
    return ids, w


def mxfp4_quantize(src: torch.Tensor):
    """1x32 MX quantisation of the rows of a 2-D fp32 CPU tensor (unit inner stride).

    Returns (codes uint8 [R, K/2], scales uint8 [R, K/32])."""
    assert src.dim() == 2 and src.dtype == torch.float32 and src.stride(1) == 1
    R, K = src.shape
    codes = torch.empty(R, K // 2, dtype=torch.uint8)
    scales = torch.empty(R, K // 32, dtype=torch.uint8)
    rc = _load().oracle_mxfp4_quantize(src.data_ptr(), R, K, src.stride(0), codes.data_ptr(),
                                       scales.data_ptr())
    if rc != 0:
        raise ValueError("oracle_mxfp4_quantize: K must be a multiple of 32")
    return codes, scales


def moe_align(ids: torch.Tensor, E: int, bm: int):
    """Stable grouping of slots by expert.  Returns a dict of CPU int32 tensors."""
    T, k = ids.shape
    S = T * k
    cap = S + min(E, max(S, 1)) * (bm - 1) + bm
    counts = torch.zeros(E, dtype=torch.int32)
    offsets = torch.zeros(E + 1, dtype=torch.int32)
    sorted_ = torch.empty(cap, dtype=torch.int32)
    block_expert = torch.empty(cap // bm + 1, dtype=torch.int32)
    nb = torch.zeros(1, dtype=torch.int32)
    nbad = torch.zeros(1, dtype=torch.int64)
    d = _desc(ids)
    rc = _load().oracle_moe_align(ctypes.byref(d), E, bm, counts.data_ptr(), offsets.data_ptr(),
                                  sorted_.data_ptr(), cap, block_expert.data_ptr(),
                                  block_expert.numel(), nb.data_ptr(), nbad.data_ptr())
    if rc != 0:
        raise RuntimeError("oracle_moe_align: buffer too small")
    P = int(offsets[E])
    return {"counts": counts, "offsets": offsets, "sorted": sorted_[:P].clone(),
            "block_expert": block_expert[: P // bm].clone(), "num_blocks": int(nb[0]),
            "n_bad": int(nbad[0])}


def moe_forward(x, gate, up, w2, ids, weights, *, scales=None, tokens=None, nthreads=0):
    """fp64 MoE forward.  bf16 mode: gate/up/w2 bf16 or f32 views.  MXFP4 mode:
    pass uint8 code tensors [.., K/2] and scales=(gate_s, up_s, w2_s) e8m0 uint8.

    tokens: optional 1-D int64 tensor of token indices; returns [len(tokens), H]
    (else [T, H]) float64 plus the number of skipped slots."""
    mx = scales is not None
    gs, us, ws = scales if mx else (None, None, None)
    dx, dg, du, dw = _desc(x), _desc(gate, gs), _desc(up, us), _desc(w2, ws)
    di, dwt = _desc(ids), _desc(weights)
    T, H = x.shape
    if tokens is not None:
        tokens = tokens.to(torch.int64).contiguous()
        n_out = tokens.numel()
        tptr = tokens.data_ptr()
    else:
        n_out, tptr = T, None
    out = torch.zeros(n_out, H, dtype=torch.float64)
    nbad = torch.zeros(1, dtype=torch.int64)
    rc = _load().oracle_moe_forward(ctypes.byref(dx), ctypes.byref(dg), ctypes.byref(du),
                                    ctypes.byref(dw), ctypes.byref(di), ctypes.byref(dwt),
                                    1 if mx else 0, tptr, n_out, out.data_ptr(),
                                    nbad.data_ptr(), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_moe_forward: shape mismatch")
    return out, int(nbad[0])
