/*
 * moe.h — C ABI of the B200 (sm_100a) fused mixture-of-experts expert forward.
 *
 * The operation (per token t and routing column j, slot s = t*k + j):
 *     e = topk_ids[t, j]        w = topk_weights[t, j]
 *     g = x[t] . gate[e]^T      u = x[t] . up[e]^T          gate = w13[:, :I, :], up = w13[:, I:, :]
 *     a = silu(g) * u           y = a . w2[e]^T
 *     out[t] = sum_j w * y      (j = 0 .. k-1, in order)
 * The packed w13 [E, 2I, H] layout and its expert-strided gate/up views are the
 * subject of Liger-Kernel PR #1377 ("Problems"): each expert's first weight tile
 * is located from the view's real stride(0), never from expert * I / TileN.
 * The SiLU activation and the MXFP4 format (e2m1 values, one e8m0 scale per 32
 * consecutive elements) follow ROCm/aiter PR #3859 ("Details").
 *
 * Conventions shared by every entry point:
 *   - Every tensor is described by a moe_tensor_t: base pointer, dtype, sizes and
 *     strides in elements of the storage type.  Any stride is honoured as given
 *     (LightLLM issue #1467 and prime-rl PR #2860 show what goes wrong otherwise);
 *     nothing is ever copied to make it contiguous.  Where the tensor-memory
 *     copy engine cannot express a layout (weights with an inner stride other
 *     than 1, or a base / outer stride that is not a multiple of 16 bytes) the
 *     call returns MOE_ERR_UNSUPPORTED_LAYOUT.
 *   - Device pointers unless the entry point says "host".  The caller owns every
 *     buffer; the library keeps no pointer after a call returns, except as keys of
 *     its cache of encoded TMA descriptors (it never dereferences a cached
 *     address; an entry is reused only for the same address, type, sizes,
 *     strides and tile shape, whose encoding is then identical).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and is asynchronous unless stated otherwise.
 *   - Shape, dtype and layout errors are reported before anything is launched or
 *     any descriptor is built (Liger-Kernel PR #1377, "Testing Done": mismatched
 *     gate hidden dimensions fail before descriptor construction).
 *   - No entry point aborts the process; every failure is a moe_status_t.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum {
  MOE_BF16 = 0,   /* bfloat16 */
  MOE_F32 = 1,    /* float32 */
  MOE_I32 = 2,    /* int32 */
  MOE_I64 = 3,    /* int64 */
  MOE_E2M1X2 = 4  /* two FP4 e2m1 codes per byte, even logical element in the low nibble
                     (torch.float4_e2m1fn_x2); sizes are LOGICAL elements, strides count bytes
                     (so the innermost logical size is twice the innermost byte extent) */
} moe_dtype_t;

/* A strided tensor view.  For MOE_E2M1X2 tensors `scale` points at the e8m0
 * scale codes (one byte per 32 logical elements of the innermost axis) and
 * scale_strides gives their strides in bytes; the other dtypes ignore both. */
typedef struct {
  void* data;
  int32_t dtype; /* moe_dtype_t */
  int32_t ndim;
  int64_t sizes[4];
  int64_t strides[4];
  void* scale;
  int64_t scale_strides[4];
} moe_tensor_t;

/* The two input projections, each [E, I, H].  Usually expert-strided views of
 * one packed w13 [E, 2I, H] (see moe_w13_from_packed); contiguous copies work
 * the same way and give bit-identical results. */
typedef struct {
  moe_tensor_t gate;
  moe_tensor_t up;
} moe_w13_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* null pointer, negative size, ndim wrong */
  MOE_ERR_SHAPE_MISMATCH = 2,     /* sizes disagree between tensors */
  MOE_ERR_UNSUPPORTED_DTYPE = 3,  /* dtype not accepted for that argument */
  MOE_ERR_UNSUPPORTED_LAYOUT = 4, /* stride/alignment the copy engine cannot express */
  MOE_ERR_WORKSPACE_TOO_SMALL = 5,
  MOE_ERR_CUDA = 6,               /* a CUDA runtime/driver call failed (see moe_last_cuda_error) */
  MOE_ERR_NO_DEVICE = 7,          /* current device is not an sm_100 GPU */
  MOE_ERR_DEVICE_TIMEOUT = 8      /* a kernel's bounded wait expired (see moe_get_device_errors) */
} moe_status_t;

/* Human-readable name of a status code (static string, never NULL).  Every
 * failure is reported by name rather than silently worked around, the rule the
 * Liger-Kernel PR #1377 discussion sets for layouts the kernel cannot read
 * ("Testing Done": a mismatched gate hidden dimension fails loudly). */
const char* moe_status_string(moe_status_t st);

/* The last CUDA error string seen by the calling thread (static storage). */
const char* moe_last_cuda_error(void);

/* Split a packed w13 [E, 2I, H] view into its gate (rows [0, I)) and up
 * (rows [I, 2I)) halves (Liger-Kernel PR #1377, "Problems").  Pure metadata: the
 * up view's base is w13 + I * stride(1) storage elements (or the matching scale
 * rows for MXFP4); both keep w13's stride(0), the real expert stride.
 * Errors: MOE_ERR_INVALID_ARG (null, ndim != 3), MOE_ERR_SHAPE_MISMATCH (odd 2I). */
moe_status_t moe_w13_from_packed(const moe_tensor_t* w13, moe_w13_t* out);

/* Bytes of device workspace moe_forward_ws needs for T tokens, hidden H,
 * intermediate I, E experts, top_k k and weight dtype wdtype (MOE_BF16 or
 * MOE_E2M1X2).  Depends only on these scalars — never on the weights' strides or
 * addresses — and does not grow with E*I*H (no weight-sized buffer is used;
 * the pages' point is that the strided views replace a 0.375 GiB/layer copy).
 * Returns 0 for invalid arguments. */
size_t moe_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, int32_t wdtype);

/* The fused MoE expert forward (all steps on the GPU, on `stream`).
 *   x            [T, H]  bf16, any strides
 *   w13          gate/up [E, I, H]: bf16, or MOE_E2M1X2 with e8m0 scales [E, I, H/32];
 *                inner stride 1; base and stride(0), stride(1) multiples of 16 bytes
 *   w2           [E, H, I]: same dtype and layout rules as w13
 *   topk_ids     [T, k]  int32 or int64, any strides (e.g. the per-layer slice
 *                [:, l, :] of a [T, layers, k] router-replay tensor, prime-rl PR #2860)
 *   topk_weights [T, k]  float32, any strides; used as given (no renormalisation)
 *   out          [T, H]  bf16, any strides; fully overwritten
 *   workspace    device buffer of at least moe_workspace_bytes(...) bytes,
 *                256-byte aligned; contents are scratch (not preserved)
 * Ids outside [0, E) are skipped (contribute zero) and counted in a device
 * counter read by moe_get_device_errors.  T = 0 is a no-op.  No allocation and
 * no host synchronisation happen inside this call.  The combine over the k
 * columns is in fixed order, so results are run-to-run deterministic and do not
 * depend on the weights' strides.  In MXFP4 mode x and the SwiGLU activation are
 * quantised on the fly with the 1x32 e8m0 rule of moe_quantize_mxfp4. */
moe_status_t moe_forward_ws(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                            const moe_tensor_t* topk_ids, const moe_tensor_t* topk_weights,
                            moe_tensor_t* out, void* workspace, size_t workspace_bytes,
                            moe_stream_t stream);

/* The forward as the pages state the problem: moe_forward(x, w13, w2,
 * topk_ids, topk_weights, out, stream), with w13 the gate/up views of the
 * packed [E, 2I, H] tensor (Liger-Kernel PR #1377, "Problems": the fused MoE
 * kernel reads the packed expert weights through strided views instead of a
 * retained contiguous copy).  Arguments as for moe_forward_ws; the workspace is
 * library-owned: one buffer per device, grown with cudaMalloc when a call needs
 * more (growth synchronises the device, so size it once with a first call
 * outside any stream capture). */
moe_status_t moe_forward(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                         const moe_tensor_t* topk_ids, const moe_tensor_t* topk_weights,
                         moe_tensor_t* out, moe_stream_t stream);

/* End-to-end form for callers whose activations live in host memory: x,
 * topk_ids, topk_weights and out are HOST tensors (pinned memory gives
 * asynchronous copies; inner stride 1 is required for these four), the weights
 * stay on the device.  Copies the inputs to the library workspace, runs the
 * forward, copies `out` back and synchronises `stream` before returning. */
moe_status_t moe_forward_host(const moe_tensor_t* x_host, const moe_w13_t* w13,
                              const moe_tensor_t* w2, const moe_tensor_t* topk_ids_host,
                              const moe_tensor_t* topk_weights_host, moe_tensor_t* out_host,
                              moe_stream_t stream);

/* Device bytes moe_forward_host_ws needs for (T, H, I, E, k, weight dtype): the
 * forward's workspace plus staging for x, the ids (room for int64), the routing
 * weights and out.  Returns 0 for invalid arguments. */
size_t moe_host_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, int32_t wdtype);

/* moe_forward_host without the wait (the operation of moe_forward, Liger-Kernel PR #1377,
 * "Problems", with host activations): enqueues on `stream` the copies of x, topk_ids and
 * topk_weights (HOST tensors, inner stride 1) into `workspace` (device, at least
 * moe_host_workspace_bytes(...), 256-byte aligned), the forward, and the copy of the
 * result into out_host, then returns.  out_host holds the result once `stream` has
 * reached that point (synchronise the stream or an event recorded after the call), and
 * the host inputs must stay unchanged until then.  With pinned host memory the copies
 * are asynchronous, so calls on different streams with different workspaces can be in
 * flight together and one call's copies overlap another call's kernels.  Two calls of
 * at most 32 routing slots each should not overlap: the configuration table may pick
 * the one-kernel decode for them, whose thread blocks wait on one another and need the
 * GPU to themselves.  No allocation, no synchronisation.  Errors as for moe_forward_ws;
 * a workspace below the size is MOE_ERR_WORKSPACE_TOO_SMALL. */
moe_status_t moe_forward_host_ws(const moe_tensor_t* x_host, const moe_w13_t* w13, const moe_tensor_t* w2,
                                 const moe_tensor_t* topk_ids_host, const moe_tensor_t* topk_weights_host,
                                 moe_tensor_t* out_host, void* workspace, size_t workspace_bytes,
                                 moe_stream_t stream);

/* Gradient path (bf16 weights): given dout = dL/dout
 * [T, H] bf16, writes dx = dL/dx [T, H] bf16 and dweights = dL/dtopk_weights
 * [T, k] f32 (any strides), the routing ids held fixed (they are discrete).
 * The fused-MoE training path of Liger-Kernel PR #1377 ("Testing Done":
 * forward and backward CUDA graphs) differentiates this layer; this entry point
 * gives its input and routing-weight gradients (moe_backward_ws adds the expert
 * weights').
 * Per slot (t, j) with e = topk_ids[t, j] in [0, E), w = topk_weights[t, j]:
 *   dweights[t, j] = dout_t . (w2_e h),  h = silu(gate_e x_t) * (up_e x_t)
 *   dh = w w2_e^T dout_t;  dg = dh u s (1 + g (1 - s)),  du = dh g s  (s = sigmoid(g))
 *   dx_t += gate_e^T dg + up_e^T du
 * (computed as dh' = w2_e^T dout_t once: dweights = dh' . h, the routing weight w
 * applied where da = w [gate_e^T | up_e^T] [dg' | du'] leaves its GEMM).
 * Skipped slots (ids outside [0, E)) contribute nothing and get dweights 0.
 * The GEMMs read the weights K-major, so the caller passes their transposes too:
 * w13t [E, H, 2I] (the packed w13 [E, 2I, H] transposed: gate^T in columns
 * [0, I), up^T in [I, 2I)) and w2t [E, I, H]; moe_transpose_experts makes them
 * (they stay valid while the weights are frozen).  Inner stride 1, 16-byte
 * aligned strides.  x, w13, w2, topk_ids, topk_weights as for moe_forward_ws;
 * dx in place of out.  Workspace: moe_backward_workspace_bytes, 256-byte
 * aligned.  Asynchronous on `stream`, no allocation.  MXFP4 weights:
 * MOE_ERR_UNSUPPORTED_DTYPE (the forward's quantisation steps have no gradient). */
size_t moe_backward_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k);

/* The same plus the expert-weight gradients (either may be NULL): dw13 = dL/dw13
 * [E, 2I, H] packed like w13 (dgate rows [0, I), dup rows [I, 2I)) and dw2 = dL/dw2
 * [E, H, I], f32 or bf16 (fp32 sums rounded once), overwritten (zero for an expert no
 * slot routes to); inner stride 1, the other strides multiples of 16 bytes, 16-byte
 * aligned, the last dimension a multiple of 32 (f32) or 64 (bf16) elements.  With the
 * routing fixed:
 *   dw2[e]   = sum over e's slots (t, j) of w (dout_t) a^T,   a = silu(g) * u
 *   dgate[e] = sum of dg x_t^T,  dup[e] = sum of du x_t^T
 * each a GEMM that contracts over the expert's slots (fp32 accumulation). */
moe_status_t moe_backward_ws(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                             const moe_tensor_t* w13t, const moe_tensor_t* w2t,
                             const moe_tensor_t* topk_ids, const moe_tensor_t* topk_weights,
                             const moe_tensor_t* dout, moe_tensor_t* dx, moe_tensor_t* dweights,
                             moe_tensor_t* dw13, moe_tensor_t* dw2, void* workspace, size_t workspace_bytes,
                             moe_stream_t stream);
moe_status_t moe_backward_input_ws(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                                   const moe_tensor_t* w13t, const moe_tensor_t* w2t,
                                   const moe_tensor_t* topk_ids, const moe_tensor_t* topk_weights,
                                   const moe_tensor_t* dout, moe_tensor_t* dx, moe_tensor_t* dweights,
                                   void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* dst[e, c, r] = src[e, r, c] for bf16 [E, R, C] -> [E, C, R] (inner stride 1 on
 * both, other strides free): the K-major weight copies the gradient path reads.
 * Asynchronous on `stream`. */
moe_status_t moe_transpose_experts(const moe_tensor_t* src, moe_tensor_t* dst, moe_stream_t stream);

/* Step "align" alone, for inspection and tests: group the T*k slots by expert
 * into block_m-row blocks, block_m being the per-token-bucket block size the
 * aiter kernels tune (ROCm/aiter PR #3859, "Tuned MoE latency": block_m 32, 64
 * or 128 by token count).
 *   counts[e]        number of valid slots routed to expert e          int32 [E]
 *   offsets[e]       exclusive prefix sum of ceil(counts/block_m)*block_m int32 [E+1]
 *   sorted_slots[p]  slot ids grouped by expert, ascending within an expert;
 *                    padding positions hold the sentinel T*k            int32 [>= max_padded]
 *   block_expert[b]  expert owning block_m-row block b                  int32 [>= max_padded/block_m]
 *   num_blocks       number of blocks                                   int32 [1]
 * max_padded = T*k + min(E, T*k)*(block_m-1); block_m in {16,32,64,128,256}.
 * `workspace` as for moe_forward_ws (moe_workspace_bytes covers it). */
moe_status_t moe_align(const moe_tensor_t* topk_ids, int64_t E, int32_t block_m, int32_t* counts,
                       int32_t* offsets, int32_t* sorted_slots, int32_t* block_expert,
                       int32_t* num_blocks, void* workspace, size_t workspace_bytes,
                       moe_stream_t stream);

/* moe_align without a workspace argument and without any allocation.  The
 * pages have no counterpart to this entry point; it exists for callers that
 * cannot allocate device memory at all — for instance a plugin running inside
 * a serving engine that has already split the GPU's memory between its own
 * pools, or a component whose host framework only hands it the input and
 * output tensors — and so can neither call cudaMalloc nor pass a workspace.
 * Arguments and outputs are those of moe_align.  The scratch lives in a fixed
 * 5 MiB array inside the library (held on every GPU that loads it until the
 * process exits), which limits the problem to T*k <= 1,048,576 slots; larger
 * problems return MOE_ERR_WORKSPACE_TOO_SMALL and nothing is launched.
 * The first call on each device looks up that array's device address (a
 * one-time host-side query); make that first call before any stream capture.
 * The address is kept until the process exits, so do not call this across a
 * cudaDeviceReset of the device.
 * All calls share the array and it keeps the previous call's contents (the
 * kernels rewrite everything they read).  Calls whose GPU work overlaps, e.g.
 * on two unordered streams, race on it.  Out-of-range ids are skipped but not
 * counted in the device error word. */
moe_status_t moe_align_noalloc(const moe_tensor_t* topk_ids, int64_t E, int32_t block_m,
                               int32_t* counts, int32_t* offsets, int32_t* sorted_slots,
                               int32_t* block_expert, int32_t* num_blocks, moe_stream_t stream);

/* The router, the step that produces topk_ids / topk_weights for the forward.
 * For every token t:
 *     p = softmax(logits[t, :]) over the E experts,
 *     topk_ids[t, 0..k-1]     = the k experts of largest p, in descending p,
 *                               a tie going to the lower expert index,
 *     topk_weights[t, 0..k-1] = those p, divided by their sum when renormalize = 1.
 * shared_expert = 1 adds a column k holding expert E with weight 1.0: the
 * fused-shared-expert routing of ROCm/aiter PR #3859 ("Summary": expert=513,
 * topk=11 beside the unfused expert=512, topk=10), so the forward then runs
 * with E + 1 experts and k + 1 columns.  The outputs are written through their
 * strides, e.g. straight into the per-layer slice [:, l, :] of a
 * [T, layers, k] routing replay tensor (prime-rl PR #2860, "Problem").
 *   logits        [T, E] float32 or bf16, any strides; E <= 1024
 *   topk_ids      [T, k + shared_expert] int32 or int64, any strides
 *   topk_weights  [T, k + shared_expert] float32, any strides
 * 1 <= k <= E and k + shared_expert <= 32.  The weights are computed in fp32
 * with expf (within a few 1e-7 relative of the exact values); the choice of
 * experts is exact (softmax is monotonic, so it compares the logits).  NaN
 * logits rank below every number.  T = 0 is a no-op.  Errors:
 * MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_DTYPE, MOE_ERR_SHAPE_MISMATCH, all
 * before anything is launched. */
moe_status_t moe_router_topk(const moe_tensor_t* logits, int32_t k, int32_t renormalize,
                             int32_t shared_expert, moe_tensor_t* topk_ids,
                             moe_tensor_t* topk_weights, moe_stream_t stream);

/* MXFP4 quantisation of the rows of src [.., K] (bf16 or f32, inner stride 1,
 * K % 32 == 0) into dst (MOE_E2M1X2 with dst->scale set): per 32 consecutive
 * elements, scale exponent s = clamp(floor(log2(amax)) - 2, -127, 127) stored as
 * the e8m0 code s + 127 (code 0 for an all-zero block), elements rounded to the
 * nearest e2m1 value of v / 2^s with ties to even, saturating at +-6 (OCP MX
 * v1.0; format named by aiter PR #3859, "Details").  src and dst have the same
 * logical shape (ndim 2 or 3); dst's strides may be anything 1-byte aligned. */
moe_status_t moe_quantize_mxfp4(const moe_tensor_t* src, moe_tensor_t* dst, moe_stream_t stream);

/* Reads and clears the device error counters of the current device:
 * *n_bad_ids = slots skipped because their id was outside [0, E) (a routing
 * replay slice read with the wrong stride produces such ids, prime-rl PR #2860,
 * "Problem"; they are counted instead of being read out of bounds);
 * *timeouts = kernel waits that gave up (every wait in the kernels is bounded,
 * so a missing arrival ends the kernel with this count instead of a hang).
 * Synchronises `stream`.  Returns MOE_ERR_DEVICE_TIMEOUT when *timeouts > 0
 * (both counters are still written), else MOE_OK. */
moe_status_t moe_get_device_errors(moe_stream_t stream, uint32_t* n_bad_ids, uint32_t* timeouts);

/* ---- inspection (tests and debugging) ------------------------------------ */

/* Byte offsets, inside a moe_forward_ws workspace, of the regions a test can
 * read back after a forward of the same problem: rows = the padded row count
 * of the expert-grouped buffers; inv = int32 [T*k], the grouped row of each
 * slot (-1 for a skipped slot); sorted = int32 [rows], the slot of each row;
 * a1 = the gathered x rows (bf16 [rows, H], or MXFP4 codes [rows, H/2] with
 * e8m0 scales at a1_scale [rows, H/32]); h = the SwiGLU activation (bf16
 * [rows, I], or codes [rows, I/2] with scales at h_scale [rows, I/32]);
 * y = the weighted down-projection rows (bf16 [rows, H]).  Only rows named by
 * inv hold results; the others are padding and hold stale data. */
typedef struct {
  int64_t rows;
  size_t inv, sorted, a1, a1_scale, h, h_scale, y, total;
} moe_workspace_layout_t;
moe_status_t moe_workspace_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k,
                                  int32_t wdtype, moe_workspace_layout_t* out);

/* Captures an intermediate of the next forwards on the calling host thread
 * into the device buffer dst (16-byte aligned) until called again with
 * dst = NULL.  MOE_CAPTURE_H_PREQUANT: the MXFP4 forward's SwiGLU activation
 * in fp32 just before it is quantised, [rows, I] row-major (rows as in
 * moe_workspace_layout); skipped when `bytes` is smaller than rows * I * 4.
 * It lets a test apply its own quantiser to the very values the GPU
 * quantised.  Costs one extra store per element while on. */
enum { MOE_CAPTURE_H_PREQUANT = 1 };
moe_status_t moe_debug_capture(int32_t what, void* dst, size_t bytes);

/* Measures the dense tensor-core rate of this GPU in TFLOP/s (*tflops):
 * every SM issues `iters` (1 .. 2^20) x 4 back-to-back tcgen05.mma (M = 128, N = 128)
 * from operand tiles resident in shared memory, no global memory involved;
 * kind 0 = kind::f16 (bf16 inputs, fp32 accumulate, K = 16 per instruction),
 * kind 1 = kind::mxf4 (e2m1 inputs with e8m0 scales per 32, K = 64).  The
 * MXFP4 roofline of the forward uses the ratio of the two rates times the
 * measured bf16 GEMM peak, instead of a nominal ratio.  Blocking: six launches
 * on the legacy default stream timed with CUDA events, the best of the last
 * five.  A measurement tool; not on the forward's path. */
moe_status_t moe_measure_mma_peak(int32_t kind, int32_t iters, double* tflops);

/* Self-test of the failure path that every wait in the kernels shares: one
 * GPU thread waits on an mbarrier that nothing arrives on and gives up after
 * limit_us microseconds (1 .. 100000), exactly as a GEMM's bounded wait gives
 * up on a missing copy, MMA or epilogue arrival instead of hanging the GPU.
 * Giving up counts one timeout in the device error counters (read them with
 * moe_get_device_errors, which then returns MOE_ERR_DEVICE_TIMEOUT) and writes
 * *done = 2 (device int32; 1 would mean the barrier completed).  No copy or
 * tensor-core operation is in flight when the wait gives up.  The pages have
 * no counterpart: they state no failure handling for the kernels. */
moe_status_t moe_selftest_bounded_wait(int32_t limit_us, int32_t* done, moe_stream_t stream);

/* Number of kernels the last moe_forward_ws / moe_forward call on this thread
 * enqueued (for launch accounting): 1 on the one-kernel decode path, 4 with at
 * most 32 routing slots otherwise, else 5, plus 2 when align runs its
 * multi-CTA form (more than 4096 slots). */
int32_t moe_last_launch_count(void);

/* Per-kernel timing for profiling.  While enabled on the calling thread, each
 * moe_forward* call records a CUDA event on its stream before the first kernel
 * and after each step (align, permute, GEMM1, GEMM2, combine); this serialises
 * the steps (no overlap between neighbouring kernels), so time the end-to-end
 * call with profiling off.  moe_profile_read synchronises on the last event and
 * writes up to `capacity` step durations in milliseconds, in that order, for
 * the last profiled call; *n receives the number of steps.  With at most 32
 * routing slots align and permute are one kernel: its time is reported as
 * align's and permute's duration is zero. */
moe_status_t moe_profile_enable(int32_t on);
moe_status_t moe_profile_read(float* ms, int32_t capacity, int32_t* n);

/* ---- kernel configuration (per-shape tuning table) ----------------------
 * Which token-tile size and GEMM variant the forward runs for a problem.  The
 * pages keep tuned kernel choices in a table keyed by shape and token count
 * (ROCm/aiter PR #3859, "Details": tuned configurations per shape; "Tuned MoE
 * latency": block_m per token bucket).  A forward looks its configuration up
 * in the table installed by moe_set_config_table, then in the table compiled
 * into the library from the committed tuning results, then falls back to a
 * heuristic.  Every configuration with split = 1 gives bit-identical results
 * (the GEMMs sum each output in the same k order whatever the tiling); a
 * one-kernel configuration whose GEMM1 is split along K sums the parts' fp32
 * partials in fixed part order, so it is deterministic but may round
 * differently.  The workspace size (moe_workspace_bytes) does not depend on
 * the configuration. */
typedef struct {
  int32_t wdtype;      /* MOE_BF16 or MOE_E2M1X2 */
  int64_t H, I, E, k;  /* shape the entry applies to; 0 matches any value */
  int64_t t_lo, t_hi;  /* token bucket: applies when t_lo <= T <= t_hi */
  int32_t tile;        /* token-tile rows: 32, 128 or 256 (bf16; 256 runs on CTA pairs),
                          32, 96 or 128 (MXFP4; 128 with one accumulator buffer) */
  int32_t pair;        /* bf16 128-row tiles: GEMMs on CTA pairs (tcgen05 cta_group::2) */
  int32_t g1_256;      /* bf16 pairs: GEMM1 on 256-row token tiles (needs g2_single) */
  int32_t g2_single;   /* bf16 pairs: GEMM2 with one 256-row w2 slice per 256-row tile */
  int32_t tiny;        /* at most 32 slots: align and permute in one launch */
  int32_t prefetch;    /* at most 32 slots, 32-row tiles: GEMM1 requests its first weight
                          stages before align has finished (checked against align after) */
  int32_t fused;       /* at most 32 slots: the whole forward as one kernel (slots grouped
                          in every CTA, token rows gathered from x (bf16) or quantised from
                          x in the kernel (MXFP4), GEMM2 weights streamed across the GEMM1
                          hand-off, combine by the last CTA of each output tile); bf16
                          needs x with unit inner stride and 16-byte aligned rows; both
                          need H <= 16384; otherwise the kernels above run */
  int32_t split;       /* one-kernel path: GEMM1 split along K into at most this many parts
                          (0 = the library's default, 4; 1 = not split).  The kernel takes
                          as many as put about two GEMM1 units on every SM, with at least
                          four 64-wide k-blocks per part; the unit that completes a (routed
                          expert, 128-row) item sums all parts' fp32 partials in part order */
  int32_t g1_il;       /* bf16: 0, or GEMM1 on CTA pairs with gate and up rows interleaved in
                          one accumulator, on token tiles of up to g1_il rows: 256 (two
                          accumulator buffers, the epilogue under the next item's MMAs) or
                          512 (an expert's gate/up weights read once per 512 rows; one
                          buffer); implies pair = 1, g2_single = 1, g1_256 = 0 */
} moe_config_t;

/* Installs a process-wide configuration table (copied; n = 0 removes it).
 * Entries are tried in order; flags that do not apply to an entry's tile are
 * ignored.  Errors: MOE_ERR_INVALID_ARG for a malformed entry (nothing is
 * installed then).  Not synchronised with forwards already running on other
 * host threads: install it before them. */
moe_status_t moe_set_config_table(const moe_config_t* entries, int32_t n);

/* The configuration a forward of this problem would use (after the rules
 * above), in *out.  Errors: MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_DTYPE. */
moe_status_t moe_get_config(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, int32_t wdtype,
                            moe_config_t* out);

/* Number of entries of the table compiled into the library. */
int32_t moe_builtin_config_count(void);

/* Library version string. */
const char* moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
