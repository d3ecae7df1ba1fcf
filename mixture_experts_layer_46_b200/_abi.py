"""ctypes binding of libmoe_b200.so (include/moe.h).

Argument marshalling only: torch tensors become moe_tensor_t descriptors
(base pointer, dtype, sizes, strides) and every step of the forward runs in the
library's CUDA kernels.  There is no fallback: if the shared library is missing
or fails to load, every call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_BF16, MOE_F32, MOE_I32, MOE_I64, MOE_E2M1X2 = 0, 1, 2, 3, 4
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_SHAPE_MISMATCH",
          3: "MOE_ERR_UNSUPPORTED_DTYPE", 4: "MOE_ERR_UNSUPPORTED_LAYOUT",
          5: "MOE_ERR_WORKSPACE_TOO_SMALL", 6: "MOE_ERR_CUDA", 7: "MOE_ERR_NO_DEVICE",
          8: "MOE_ERR_DEVICE_TIMEOUT"}

# Names the header declares; tests check the library exports each of them.
EXPORTS = ("moe_status_string", "moe_last_cuda_error", "moe_w13_from_packed",
           "moe_workspace_bytes", "moe_forward_ws", "moe_forward", "moe_forward_host",
           "moe_align", "moe_quantize_mxfp4", "moe_get_device_errors", "moe_last_launch_count",
           "moe_profile_enable", "moe_profile_read", "moe_version", "moe_align_noalloc",
           "moe_set_config_table", "moe_get_config", "moe_builtin_config_count",
           "moe_router_topk", "moe_selftest_bounded_wait", "moe_workspace_layout",
           "moe_debug_capture", "moe_measure_mma_peak", "moe_backward_workspace_bytes",
           "moe_backward_input_ws", "moe_backward_ws", "moe_transpose_experts",
           "moe_host_workspace_bytes", "moe_forward_host_ws")
STEP_NAMES = ("align", "permute", "gemm1_swiglu", "gemm2_weighted", "combine")


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class MoeTensor(ctypes.Structure):
    _fields_ = [
        ("data", ctypes.c_void_p),
        ("dtype", ctypes.c_int32),
        ("ndim", ctypes.c_int32),
        ("sizes", ctypes.c_int64 * 4),
        ("strides", ctypes.c_int64 * 4),
        ("scale", ctypes.c_void_p),
        ("scale_strides", ctypes.c_int64 * 4),
    ]


class MoeW13(ctypes.Structure):
    _fields_ = [("gate", MoeTensor), ("up", MoeTensor)]


class MoeWorkspaceLayout(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64)] + [(n, ctypes.c_size_t) for n in (
        "inv", "sorted", "a1", "a1_scale", "h", "h_scale", "y", "total")]


class MoeConfig(ctypes.Structure):
    """moe_config_t: the kernel configuration of one shape and token bucket."""
    _fields_ = [("wdtype", ctypes.c_int32), ("H", ctypes.c_int64), ("I", ctypes.c_int64),
                ("E", ctypes.c_int64), ("k", ctypes.c_int64), ("t_lo", ctypes.c_int64),
                ("t_hi", ctypes.c_int64), ("tile", ctypes.c_int32), ("pair", ctypes.c_int32),
                ("g1_256", ctypes.c_int32), ("g2_single", ctypes.c_int32), ("tiny", ctypes.c_int32),
                ("prefetch", ctypes.c_int32), ("fused", ctypes.c_int32), ("split", ctypes.c_int32),
                ("g1_il", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {name: int(getattr(self, name)) for name, _ in self._fields_}


CONFIG_FLAGS = ("tile", "pair", "g1_256", "g2_single", "tiny", "prefetch", "fused", "split", "g1_il")


_lock = threading.Lock()
_lib = None


def load() -> ctypes.CDLL:
    """Load the CUDA library (raises if it is not built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m mixture_experts_layer_46_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            P = ctypes.POINTER
            vp = ctypes.c_void_p
            lib.moe_status_string.restype = ctypes.c_char_p
            lib.moe_status_string.argtypes = [ctypes.c_int]
            lib.moe_last_cuda_error.restype = ctypes.c_char_p
            lib.moe_version.restype = ctypes.c_char_p
            lib.moe_last_launch_count.restype = ctypes.c_int32
            lib.moe_w13_from_packed.restype = ctypes.c_int
            lib.moe_w13_from_packed.argtypes = [P(MoeTensor), P(MoeW13)]
            lib.moe_workspace_bytes.restype = ctypes.c_size_t
            lib.moe_workspace_bytes.argtypes = [ctypes.c_int64] * 5 + [ctypes.c_int32]
            lib.moe_forward_ws.restype = ctypes.c_int
            lib.moe_forward_ws.argtypes = [P(MoeTensor), P(MoeW13), P(MoeTensor), P(MoeTensor),
                                           P(MoeTensor), P(MoeTensor), vp, ctypes.c_size_t, vp]
            lib.moe_forward.restype = ctypes.c_int
            lib.moe_forward.argtypes = [P(MoeTensor), P(MoeW13), P(MoeTensor), P(MoeTensor),
                                        P(MoeTensor), P(MoeTensor), vp]
            lib.moe_forward_host.restype = ctypes.c_int
            lib.moe_forward_host.argtypes = lib.moe_forward.argtypes
            lib.moe_host_workspace_bytes.restype = ctypes.c_size_t
            lib.moe_host_workspace_bytes.argtypes = [ctypes.c_int64] * 5 + [ctypes.c_int32]
            lib.moe_forward_host_ws.restype = ctypes.c_int
            lib.moe_forward_host_ws.argtypes = lib.moe_forward_ws.argtypes
            lib.moe_backward_workspace_bytes.restype = ctypes.c_size_t
            lib.moe_backward_workspace_bytes.argtypes = [ctypes.c_int64] * 5
            lib.moe_backward_input_ws.restype = ctypes.c_int
            lib.moe_backward_input_ws.argtypes = [P(MoeTensor), P(MoeW13)] + [P(MoeTensor)] * 8 + [
                vp, ctypes.c_size_t, vp]
            lib.moe_backward_ws.restype = ctypes.c_int
            lib.moe_backward_ws.argtypes = [P(MoeTensor), P(MoeW13)] + [P(MoeTensor)] * 10 + [
                vp, ctypes.c_size_t, vp]
            lib.moe_transpose_experts.restype = ctypes.c_int
            lib.moe_transpose_experts.argtypes = [P(MoeTensor), P(MoeTensor), vp]
            lib.moe_align.restype = ctypes.c_int
            lib.moe_align.argtypes = [P(MoeTensor), ctypes.c_int64, ctypes.c_int32, vp, vp, vp, vp,
                                      vp, vp, ctypes.c_size_t, vp]
            lib.moe_quantize_mxfp4.restype = ctypes.c_int
            lib.moe_quantize_mxfp4.argtypes = [P(MoeTensor), P(MoeTensor), vp]
            lib.moe_get_device_errors.restype = ctypes.c_int
            lib.moe_get_device_errors.argtypes = [vp, P(ctypes.c_uint32), P(ctypes.c_uint32)]
            lib.moe_align_noalloc.restype = ctypes.c_int
            lib.moe_align_noalloc.argtypes = [P(MoeTensor), ctypes.c_int64, ctypes.c_int32, vp, vp,
                                              vp, vp, vp, vp]
            lib.moe_set_config_table.restype = ctypes.c_int
            lib.moe_set_config_table.argtypes = [P(MoeConfig), ctypes.c_int32]
            lib.moe_get_config.restype = ctypes.c_int
            lib.moe_get_config.argtypes = [ctypes.c_int64] * 5 + [ctypes.c_int32, P(MoeConfig)]
            lib.moe_builtin_config_count.restype = ctypes.c_int32
            lib.moe_router_topk.restype = ctypes.c_int
            lib.moe_router_topk.argtypes = [P(MoeTensor), ctypes.c_int32, ctypes.c_int32,
                                            ctypes.c_int32, P(MoeTensor), P(MoeTensor), vp]
            lib.moe_selftest_bounded_wait.restype = ctypes.c_int
            lib.moe_selftest_bounded_wait.argtypes = [ctypes.c_int32, vp, vp]
            lib.moe_workspace_layout.restype = ctypes.c_int
            lib.moe_workspace_layout.argtypes = [ctypes.c_int64] * 5 + [ctypes.c_int32,
                                                                        P(MoeWorkspaceLayout)]
            lib.moe_debug_capture.restype = ctypes.c_int
            lib.moe_debug_capture.argtypes = [ctypes.c_int32, vp, ctypes.c_size_t]
            lib.moe_measure_mma_peak.restype = ctypes.c_int
            lib.moe_measure_mma_peak.argtypes = [ctypes.c_int32, ctypes.c_int32,
                                                 P(ctypes.c_double)]
            lib.moe_profile_enable.restype = ctypes.c_int
            lib.moe_profile_enable.argtypes = [ctypes.c_int32]
            lib.moe_profile_read.restype = ctypes.c_int
            lib.moe_profile_read.argtypes = [P(ctypes.c_float), ctypes.c_int32, P(ctypes.c_int32)]
            _lib = lib
    return _lib


def _check(rc: int, where: str):
    if rc != 0:
        detail = load().moe_last_cuda_error().decode() if rc == 6 else ""
        raise MoeError(rc, where, detail)


_TORCH_DT = {torch.bfloat16: MOE_BF16, torch.float32: MOE_F32, torch.int32: MOE_I32,
             torch.int64: MOE_I64}


def desc(t: torch.Tensor, scale: torch.Tensor | None = None) -> MoeTensor:
    """moe_tensor_t for a torch tensor.  uint8 (or float4_e2m1fn_x2) tensors are
    packed e2m1 pairs: the logical innermost size is twice the byte count and
    `scale` (uint8 e8m0 codes, one per 32 logical elements) is required."""
    d = MoeTensor()
    d.data = t.data_ptr() if t.numel() > 0 else None
    d.ndim = t.dim()
    if hasattr(torch, "float4_e2m1fn_x2") and t.dtype == torch.float4_e2m1fn_x2:
        t = t.view(torch.uint8)
    if t.dtype == torch.uint8:
        d.dtype = MOE_E2M1X2
        if scale is None:
            raise ValueError("an e2m1 tensor needs its e8m0 scale tensor")
        if scale.dtype != torch.uint8:
            scale = scale.view(torch.uint8)
        d.scale = scale.data_ptr()
        for i in range(scale.dim()):
            d.scale_strides[i] = scale.stride(i)
    else:
        d.dtype = _TORCH_DT.get(t.dtype, 99)  # unknown dtypes are rejected by the library
    for i in range(t.dim()):
        d.sizes[i] = t.shape[i]
        d.strides[i] = t.stride(i)
    if d.dtype == MOE_E2M1X2:
        d.sizes[t.dim() - 1] = 2 * t.shape[-1]
    return d


def _stream_ptr(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def w13_from_packed(w13: torch.Tensor, scale: torch.Tensor | None = None) -> MoeW13:
    out = MoeW13()
    d = desc(w13, scale)
    _check(load().moe_w13_from_packed(ctypes.byref(d), ctypes.byref(out)), "moe_w13_from_packed")
    return out


def w13_from_views(gate: torch.Tensor, up: torch.Tensor, gate_scale=None, up_scale=None) -> MoeW13:
    out = MoeW13()
    out.gate = desc(gate, gate_scale)
    out.up = desc(up, up_scale)
    return out


def workspace_bytes(T: int, H: int, I: int, E: int, k: int, mxfp4: bool = False) -> int:
    return int(load().moe_workspace_bytes(T, H, I, E, k, MOE_E2M1X2 if mxfp4 else MOE_BF16))


def forward(x, w13: MoeW13, w2, topk_ids, topk_weights, out=None, *, w2_scale=None,
            workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[t] = sum_j w[t,j] * SwiGLU-expert_{ids[t,j]}(x[t]) on the GPU.

    w13: MoeW13 from w13_from_packed / w13_from_views.  With `workspace` (a
    uint8 CUDA tensor of at least workspace_bytes(...)) this calls
    moe_forward_ws, else moe_forward (library-owned workspace)."""
    if out is None:
        out = torch.empty(x.shape[0], x.shape[1], dtype=torch.bfloat16, device=x.device)
    dx, dw2, di, dw, do = desc(x), desc(w2, w2_scale), desc(topk_ids), desc(topk_weights), desc(out)
    lib = load()
    st = _stream_ptr(stream)
    if workspace is not None:
        rc = lib.moe_forward_ws(ctypes.byref(dx), ctypes.byref(w13), ctypes.byref(dw2),
                                ctypes.byref(di), ctypes.byref(dw), ctypes.byref(do),
                                workspace.data_ptr(), workspace.numel(), st)
        _check(rc, "moe_forward_ws")
    else:
        rc = lib.moe_forward(ctypes.byref(dx), ctypes.byref(w13), ctypes.byref(dw2),
                             ctypes.byref(di), ctypes.byref(dw), ctypes.byref(do), st)
        _check(rc, "moe_forward")
    return out


def backward_workspace_bytes(T: int, H: int, I: int, E: int, k: int) -> int:
    return int(load().moe_backward_workspace_bytes(T, H, I, E, k))


def transpose_experts(src: torch.Tensor, dst: torch.Tensor | None = None, *, stream=None) -> torch.Tensor:
    """dst[e, c, r] = src[e, r, c] (bf16 [E, R, C] -> [E, C, R]) on the GPU."""
    if dst is None:
        dst = torch.empty(src.shape[0], src.shape[2], src.shape[1], dtype=src.dtype, device=src.device)
    ds, dd = desc(src), desc(dst)
    _check(load().moe_transpose_experts(ctypes.byref(ds), ctypes.byref(dd), _stream_ptr(stream)),
           "moe_transpose_experts")
    return dst


def backward(x, w13: MoeW13, w2, w13t, w2t, topk_ids, topk_weights, dout, dx=None, dweights=None,
             dw13=None, dw2=None, *, weights=True, grad_dtype=torch.float32,
             workspace: torch.Tensor | None = None, stream=None):
    """(dx, dweights, dw13, dw2): the forward's gradients given dout; dw13 [E, 2I, H]
    (packed like w13) and dw2 [E, H, I] in grad_dtype (float32 or bfloat16) are
    computed when `weights` (else None)."""
    T, H = x.shape
    k = topk_ids.shape[1]
    E, _, I = w2.shape
    dev = x.device
    if dx is None:
        dx = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    if dweights is None:
        dweights = torch.empty(T, k, dtype=torch.float32, device=dev)
    if weights and dw13 is None:
        dw13 = torch.empty(E, 2 * I, H, dtype=grad_dtype, device=dev)
    if weights and dw2 is None:
        dw2 = torch.empty(E, H, I, dtype=grad_dtype, device=dev)
    if workspace is None:
        n = backward_workspace_bytes(T, H, I, E, k)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=dev)
    d = [desc(v) for v in (x, w2, w13t, w2t, topk_ids, topk_weights, dout, dx, dweights)]
    g13 = ctypes.byref(desc(dw13)) if dw13 is not None else None
    g2 = ctypes.byref(desc(dw2)) if dw2 is not None else None
    rc = load().moe_backward_ws(ctypes.byref(d[0]), ctypes.byref(w13), *[ctypes.byref(v) for v in d[1:]],
                                g13, g2, workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(rc, "moe_backward_ws")
    return dx, dweights, dw13, dw2


def backward_status(x, w13: MoeW13, w2, w13t, w2t, topk_ids, topk_weights, dout, dx, dweights, dw13=None,
                    dw2=None, *, workspace=None, stream=None) -> int:
    """Like backward() but returns the raw moe_status_t (for error-path tests)."""
    d = [desc(v) for v in (x, w2, w13t, w2t, topk_ids, topk_weights, dout, dx, dweights)]
    g13 = ctypes.byref(desc(dw13)) if dw13 is not None else None
    g2 = ctypes.byref(desc(dw2)) if dw2 is not None else None
    st = _stream_ptr(stream) if torch.cuda.is_available() else None
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_n = workspace.numel() if workspace is not None else 0
    return int(load().moe_backward_ws(ctypes.byref(d[0]), ctypes.byref(w13), *[ctypes.byref(v) for v in d[1:]],
                                      g13, g2, ws_ptr, ws_n, st))


def backward_input(x, w13: MoeW13, w2, w13t, w2t, topk_ids, topk_weights, dout, dx=None, dweights=None,
                   *, workspace: torch.Tensor | None = None, stream=None):
    """(dx, dweights): the forward's gradient with respect to x and the routing
    weights given dout, experts frozen; w13t [E, H, 2I] and w2t [E, I, H] are the
    weights' transposes (transpose_experts)."""
    T, H = x.shape
    k = topk_ids.shape[1]
    if dx is None:
        dx = torch.empty(T, H, dtype=torch.bfloat16, device=x.device)
    if dweights is None:
        dweights = torch.empty(T, k, dtype=torch.float32, device=x.device)
    if workspace is None:
        n = backward_workspace_bytes(T, H, w2.shape[2], w2.shape[0], k)
        workspace = torch.empty(max(n, 1), dtype=torch.uint8, device=x.device)
    d = [desc(v) for v in (x, w2, w13t, w2t, topk_ids, topk_weights, dout, dx, dweights)]
    rc = load().moe_backward_input_ws(ctypes.byref(d[0]), ctypes.byref(w13), *[ctypes.byref(v) for v in d[1:]],
                                      workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(rc, "moe_backward_input_ws")
    return dx, dweights


def forward_status(x, w13: MoeW13, w2, topk_ids, topk_weights, out, *, w2_scale=None,
                   workspace=None, stream=None) -> int:
    """Like forward() but returns the raw moe_status_t (for error-path tests)."""
    dx, dw2, di, dw, do = desc(x), desc(w2, w2_scale), desc(topk_ids), desc(topk_weights), desc(out)
    lib = load()
    st = _stream_ptr(stream) if torch.cuda.is_available() else None
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_n = workspace.numel() if workspace is not None else 0
    return int(lib.moe_forward_ws(ctypes.byref(dx), ctypes.byref(w13), ctypes.byref(dw2),
                                  ctypes.byref(di), ctypes.byref(dw), ctypes.byref(do), ws_ptr,
                                  ws_n, st))


def host_workspace_bytes(T: int, H: int, I: int, E: int, k: int, mxfp4: bool = False) -> int:
    return int(load().moe_host_workspace_bytes(T, H, I, E, k, MOE_E2M1X2 if mxfp4 else MOE_BF16))


def forward_host(x_host, w13: MoeW13, w2, ids_host, weights_host, out_host, *, w2_scale=None,
                 workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Host activations in, host result out.  Without `workspace`: moe_forward_host
    (library staging, the stream synchronised before it returns).  With a device
    `workspace` of host_workspace_bytes(...): moe_forward_host_ws, which only enqueues
    the copies and the forward on `stream`; out_host is ready once the stream is."""
    dx, dw2, di, dw, do = (desc(x_host), desc(w2, w2_scale), desc(ids_host), desc(weights_host),
                           desc(out_host))
    if workspace is None:
        rc = load().moe_forward_host(ctypes.byref(dx), ctypes.byref(w13), ctypes.byref(dw2),
                                     ctypes.byref(di), ctypes.byref(dw), ctypes.byref(do),
                                     _stream_ptr(stream))
        _check(rc, "moe_forward_host")
        return out_host
    rc = load().moe_forward_host_ws(ctypes.byref(dx), ctypes.byref(w13), ctypes.byref(dw2),
                                    ctypes.byref(di), ctypes.byref(dw), ctypes.byref(do),
                                    workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(rc, "moe_forward_host_ws")
    return out_host


def align(topk_ids: torch.Tensor, E: int, block_m: int, *, stream=None):
    """Run the align step alone; returns a dict of device int32 tensors."""
    T, k = topk_ids.shape
    S = T * k
    dev = topk_ids.device
    pmax = S + min(E, max(S, 1)) * (block_m - 1) + block_m
    counts = torch.zeros(E, dtype=torch.int32, device=dev)
    offsets = torch.zeros(E + 1, dtype=torch.int32, device=dev)
    sorted_ = torch.full((pmax,), -7, dtype=torch.int32, device=dev)
    block_expert = torch.full((pmax // block_m + 1,), -7, dtype=torch.int32, device=dev)
    nb = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = torch.empty(workspace_bytes(max(T, 1), 32, 32, E, k), dtype=torch.uint8, device=dev)
    d = desc(topk_ids)
    rc = load().moe_align(ctypes.byref(d), E, block_m, counts.data_ptr(), offsets.data_ptr(),
                          sorted_.data_ptr(), block_expert.data_ptr(), nb.data_ptr(),
                          ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    _check(rc, "moe_align")
    P = int(offsets[E].item())
    n = int(nb.item())
    return {"counts": counts, "offsets": offsets, "sorted": sorted_[:P], "block_expert": block_expert[:n],
            "num_blocks": n}


def router_topk(logits: torch.Tensor, k: int, *, renormalize: bool = True,
                shared_expert: bool = False, topk_ids: torch.Tensor | None = None,
                topk_weights: torch.Tensor | None = None, id_dtype=torch.int32, stream=None):
    """softmax -> top-k -> renormalise on the GPU (moe_router_topk).  Writes into
    the given (possibly strided) outputs or new [T, k + shared] tensors."""
    T = logits.shape[0]
    kk = k + (1 if shared_expert else 0)
    if topk_ids is None:
        topk_ids = torch.empty(T, kk, dtype=id_dtype, device=logits.device)
    if topk_weights is None:
        topk_weights = torch.empty(T, kk, dtype=torch.float32, device=logits.device)
    dl, di, dw = desc(logits), desc(topk_ids), desc(topk_weights)
    rc = load().moe_router_topk(ctypes.byref(dl), k, 1 if renormalize else 0,
                                1 if shared_expert else 0, ctypes.byref(di), ctypes.byref(dw),
                                _stream_ptr(stream))
    _check(rc, "moe_router_topk")
    return topk_ids, topk_weights


def router_status(logits, k, renormalize, shared_expert, topk_ids, topk_weights) -> int:
    """The raw moe_status_t of moe_router_topk (for argument-check tests)."""
    dl, di, dw = desc(logits), desc(topk_ids), desc(topk_weights)
    st = _stream_ptr(None) if torch.cuda.is_available() else None
    return int(load().moe_router_topk(ctypes.byref(dl), k, renormalize, shared_expert,
                                      ctypes.byref(di), ctypes.byref(dw), st))


def quantize_mxfp4(src: torch.Tensor, *, stream=None):
    """1x32 e8m0 / e2m1 quantisation of the last axis of a bf16/f32 CUDA tensor.
    Returns (codes uint8 [..., K/2], scales uint8 [..., K/32])."""
    K = src.shape[-1]
    codes = torch.empty(*src.shape[:-1], K // 2, dtype=torch.uint8, device=src.device)
    scales = torch.empty(*src.shape[:-1], K // 32, dtype=torch.uint8, device=src.device)
    ds = desc(src)
    dd = desc(codes, scales)
    _check(load().moe_quantize_mxfp4(ctypes.byref(ds), ctypes.byref(dd), _stream_ptr(stream)),
           "moe_quantize_mxfp4")
    return codes, scales


def workspace_layout(T: int, H: int, I: int, E: int, k: int, mxfp4: bool = False) -> dict:
    """Byte offsets of the inspectable workspace regions (moe_workspace_layout)."""
    out = MoeWorkspaceLayout()
    _check(load().moe_workspace_layout(T, H, I, E, k, MOE_E2M1X2 if mxfp4 else MOE_BF16,
                                       ctypes.byref(out)), "moe_workspace_layout")
    return {name: int(getattr(out, name)) for name, _ in out._fields_}


def measure_mma_peak(kind: str, iters: int = 100000) -> float:
    """Dense tensor-core rate (TFLOP/s) of back-to-back MMAs: kind 'bf16' or 'mxf4'."""
    out = ctypes.c_double(0.0)
    _check(load().moe_measure_mma_peak({"bf16": 0, "mxf4": 1}[kind], iters, ctypes.byref(out)),
           "moe_measure_mma_peak")
    return float(out.value)


MOE_CAPTURE_H_PREQUANT = 1


def debug_capture(what: int, buf: torch.Tensor | None) -> None:
    """Capture an intermediate of the next forwards into `buf` (None stops it)."""
    ptr = buf.data_ptr() if buf is not None else None
    n = buf.numel() * buf.element_size() if buf is not None else 0
    _check(load().moe_debug_capture(what, ptr, n), "moe_debug_capture")


def device_errors(stream=None):
    """(skipped out-of-range slots, kernel waits that gave up) since the last read;
    reading clears them.  MOE_ERR_DEVICE_TIMEOUT only flags a non-zero second count."""
    nb = ctypes.c_uint32(0)
    to = ctypes.c_uint32(0)
    rc = load().moe_get_device_errors(_stream_ptr(stream), ctypes.byref(nb), ctypes.byref(to))
    if rc not in (0, 8):
        _check(rc, "moe_get_device_errors")
    return int(nb.value), int(to.value)


def make_config(wdtype: int = MOE_BF16, H=0, I=0, E=0, k=0, t_lo=0, t_hi=1 << 40, **flags) -> MoeConfig:
    c = MoeConfig()
    c.wdtype, c.H, c.I, c.E, c.k, c.t_lo, c.t_hi = wdtype, H, I, E, k, t_lo, t_hi
    for name in CONFIG_FLAGS:
        setattr(c, name, int(flags.get(name, 0)))
    return c


def set_config_table(entries) -> None:
    """Install a process-wide configuration table (a list of MoeConfig; [] removes it)."""
    n = len(entries)
    arr = (MoeConfig * max(n, 1))(*entries)
    _check(load().moe_set_config_table(arr, n), "moe_set_config_table")


def get_config(T: int, H: int, I: int, E: int, k: int, mxfp4: bool = False) -> dict:
    """The configuration a forward of this problem uses."""
    c = MoeConfig()
    _check(load().moe_get_config(T, H, I, E, k, MOE_E2M1X2 if mxfp4 else MOE_BF16, ctypes.byref(c)),
           "moe_get_config")
    return c.as_dict()


class config_override:
    """Context manager: forwards of the problem (T, H, I, E, k) run the
    configuration they would use, with the given flags changed, e.g.
    config_override((T, H, I, E, k), tile=32) or (..., mxfp4=True, tiny=0)."""

    def __init__(self, shape, mxfp4: bool = False, **flags):
        self.shape, self.mxfp4, self.flags = tuple(shape), mxfp4, flags

    def __enter__(self):
        set_config_table([])
        T, H, I, E, k = self.shape
        base = get_config(T, H, I, E, k, mxfp4=self.mxfp4)
        base.update(self.flags)
        base.update(H=H, I=I, E=E, k=k, t_lo=T, t_hi=T)
        wd = base.pop("wdtype")
        set_config_table([make_config(wd, **base)])
        return self

    def __exit__(self, *exc):
        set_config_table([])
        return False


def builtin_config_count() -> int:
    return int(load().moe_builtin_config_count())


def profile_enable(on: bool = True):
    _check(load().moe_profile_enable(1 if on else 0), "moe_profile_enable")


def profile_read() -> dict:
    """Step durations (ms) of the last forward run with profiling enabled."""
    buf = (ctypes.c_float * 8)()
    n = ctypes.c_int32(0)
    _check(load().moe_profile_read(buf, 8, ctypes.byref(n)), "moe_profile_read")
    return {STEP_NAMES[i]: float(buf[i]) for i in range(n.value)}


def last_launch_count() -> int:
    return int(load().moe_last_launch_count())


def version() -> str:
    return load().moe_version().decode()
