// Internal declarations shared by the host runtime and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"
#include "moe_common.cuh"

namespace moe {

// Strided 2-D view of a small integer/float tensor read by SIMT code.
struct View2 {
  const void* data;
  int64_t s0, s1;  // strides in elements
  int32_t dtype;   // MOE_* code
};

// Byte layout of the forward's workspace.  Every region starts on a 256-byte
// boundary.  Sizes depend only on (T, H, I, E, k, weight dtype).
struct WsLayout {
  int64_t T, H, I, E, k, S;
  int32_t bm;         // block_m: padding granule of each expert's rows
  int32_t tile_max;   // smallest token-tile size the list capacity is sized for
  int64_t t_max;      // upper bound of the token-tile count (any tile size)
  int32_t tile_max2;  // rows of the second token-tile list (bf16 pairs: 256; 0: none)
  int64_t t_max2;     // upper bound of its tile count
  int64_t n_chunks;   // align chunks
  int64_t p_max;      // upper bound of padded slot count
  int64_t nb_max;     // upper bound of the block count
  bool mxfp4;
  size_t counts, offsets, num_blocks, chunk_counts, sorted, inv, block_expert;
  size_t tile_row, tile_rows, tile_expert;
  size_t tile_row2, tile_rows2, tile_expert2;
  size_t a1, a1_scale, h, h_scale, y;
  size_t w_row;       // MXFP4: routing weight per grouped row (written by permute)
  size_t part;        // at most 32 slots: GEMM1 split-K partials of the one-kernel path
  size_t total;
};

constexpr int kMaxTopK = 32;            // routing columns per token
constexpr int kMaxExperts = 1024;       // experts per layer
constexpr int kAlignChunk = 4096;        // slots per CTA in the multi-CTA align
constexpr int kAlignSmallMax = 4096;     // single-CTA align up to this many slots
constexpr int32_t kBm = 32;              // padding granule of each expert's rows (block_m)
constexpr int32_t kMinTile = 32;         // smallest token tile of any configuration

WsLayout make_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, bool mxfp4,
                     int32_t bm);

// The kernel configuration a forward of this problem uses: the caller's table,
// then the built-in tuned table, then the heuristic; flags that do not apply
// to the chosen tile are cleared.
moe_config_t select_config(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, bool mxfp4);

// ---- launchers (return cudaError_t of the launch) ----------------------------

// Token-tile list for the weight-stationary GEMMs: tiles of up to tile_max
// padded rows that never cross an expert boundary.
struct AlignTileList {
  int32_t tile_max;  // 0: not produced
  int32_t* tile_row;
  int32_t* tile_rows;
  int32_t* tile_expert;
  int32_t* num_tiles;
};
struct AlignTiles {
  AlignTileList list[2];  // [0]: the GEMMs' tiles, [1]: 256-row tiles for the pair GEMM2
};

// align and permute in one launch, for 1..32 routing slots (decode).  a1 is
// bf16 rows, or MXFP4 codes when a1_scales is given (then topk_w and w_row as
// in launch_permute_quant)
cudaError_t launch_align_permute_tiny(const View2& ids, int64_t T, int64_t k, int64_t E, int32_t bm,
                                      int32_t* counts, int32_t* offsets, int32_t* sorted,
                                      int32_t* inv, int32_t* block_expert, int32_t* num_blocks,
                                      DeviceErrors* err, const AlignTiles* tiles, const View2& x,
                                      int64_t H, void* a1, uint8_t* a1_scales, const View2* topk_w,
                                      float* w_row, cudaStream_t st, int* launches);

// align: ids -> counts, offsets, sorted, block_expert, num_blocks (+ tile list)
cudaError_t launch_align(const View2& ids, int64_t T, int64_t k, int64_t E, int32_t bm,
                         int32_t* counts, int32_t* offsets, int32_t* sorted, int32_t* inv,
                         int32_t* block_expert, int32_t* num_blocks, int32_t* chunk_counts,
                         int64_t n_chunks, DeviceErrors* err, cudaStream_t st, int* launches,
                         const AlignTiles* tiles = nullptr);

// permute: A1[inv[t*k+j], :] = x[t, :] (x read once per token); padding rows untouched
cudaError_t launch_permute_bf16(const View2& x, int64_t T, int64_t H, int64_t k,
                                const int32_t* inv, __nv_bfloat16* a1, cudaStream_t st,
                                int* launches);

// permute + MXFP4 quantisation of x rows (codes [P, H/2], scales [P, H/32]);
// also w_row[p] = routing weight of the slot at grouped row p (valid rows only)
cudaError_t launch_permute_quant(const View2& x, int64_t T, int64_t H, int64_t k,
                                 const int32_t* inv, uint8_t* codes, uint8_t* scales,
                                 const View2& topk_w, float* w_row, cudaStream_t st,
                                 int* launches);

// routing-weight gradient: dw[t, j] = sum_o a[o] * y[inv[t*k + j], o] (fp32; 0 for a
// skipped slot), a = row t of dout [T, H] (grouped = 0) or row inv[t*k + j] of dout
// (grouped = 1: grouped rows [P, H]); bf16 strided rows, y [P, H] contiguous, dw [T, k] f32 strided
cudaError_t launch_slot_dot(const View2& dout, int grouped, const __nv_bfloat16* y, const int32_t* inv,
                            int64_t T, int64_t H, int64_t k, const View2& dw, cudaStream_t st,
                            int* launches);

constexpr int kKgroupTileM = 128, kKgroupTileN = 256;  // the GEMM's output tile
// Expert-weight gradient GEMM grouped along K: C[e, m, n] = sum over expert e's
// grouped rows p of A[m, p] B[n, p]; a / b map A [M, P] and B [N, P] bf16 ([64 x
// kKgroupTileM] and [64 x kKgroupTileN] boxes, 128-byte swizzle); offsets [E + 1] multiples of 64; c maps C [E, M, N] (dims
// {N, M, E}, 128-byte swizzle): fp32 in [32 x 32 x 1] boxes (N % 32 == 0) or, with
// bf16_out, bf16 in [64 x 32 x 1] boxes (N % 64 == 0)
cudaError_t launch_gemm_kgroup(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c, int bf16_out,
                               int64_t M, int64_t N, int64_t E, const int32_t* offsets, DeviceErrors* err,
                               int num_sms, cudaStream_t st, int* launches);
// dst [C, P] (row-major) = the grouped rows transposed, padding rows as zeros:
// dst[c, p] = scale(p) * src_row(p)[c], src_row(p) = row sorted[p] / k of src
// (gather = 1) or row p of src, scale(p) = routing weight of slot sorted[p] (scale = 1) or 1
cudaError_t launch_gather_transpose(const View2& src, int gather, const int32_t* sorted, int64_t S, int64_t k,
                                    const View2& wts, int scale, void* dst, int64_t P, int64_t C,
                                    cudaStream_t st, int* launches);

// dst[e, c, r] = src[e, r, c] for bf16 [E, R, C] (element strides; inner stride 1 both)
cudaError_t launch_transpose_experts(const void* src, int64_t s0, int64_t s1, void* dst, int64_t d0,
                                     int64_t d1, int64_t E, int64_t R, int64_t C, cudaStream_t st);

// combine: out[t, :] = sum_j y[inv[t*k + j], :] over valid slots (fixed j order)
cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* inv, int64_t T, int64_t H,
                           int64_t k, void* out, int64_t os0, int64_t os1, cudaStream_t st,
                           int* launches);

// Weight-stationary ("swap AB") bf16 GEMMs over the token-tile list of align.
struct WsGemm {
  int64_t K, N, n_wt, max_tiles;
  const int32_t* num_tiles;
  const int32_t* tile_row;
  const int32_t* tile_rows;
  const int32_t* tile_expert;
  const int32_t* sorted;
  int64_t S;
  void* out;
  int64_t out_ld;
  View2 topk_w;
  int64_t k;
  int32_t weights_evict_first;  // L2 policy of the weight loads (tokens: evict-last)
  int32_t tok_box;              // rows per token-tile TMA box of the x map (tile rows per CTA: one box)
  // GEMM1 on 32-row tiles with at most 32 routing slots: the routing ids, from
  // which each CTA finds its first expert before align has finished (pre_S = 0: off)
  View2 pre_ids;
  int32_t pre_E, pre_S;
  DeviceErrors* err;
  // mode 1: every routed slot gets weight 1 instead of its routing weight
  int32_t unit_w;
  // mode 3 (gradient of GEMM1 + SwiGLU): dh [P, N] in, h [P, N] out (row strides in elements)
  const void* dh;
  int64_t dh_ld;
  void* h_out;
  int64_t h_ld;
};
// mode 0: GEMM1 (gate/up + SwiGLU -> h), mode 1: GEMM2 (down + routing weight -> y),
// mode 3: GEMM1 recomputed for the gradient: with g, u the two accumulators and dh
// read from p.dh, out[p, i] = dh s u (1 + g (1 - s)), out[p, N + i] = dh g s
// (s = sigmoid(g)) and h_out[p, i] = g s u, for every row of the token tiles.
// tile_max: 128 (4-stage ring) or 32 (6-stage ring)
cudaError_t launch_gemm_ws_bf16(int mode, int tile_max, const CUtensorMap& w0,
                                const CUtensorMap& w1, const CUtensorMap& x, const WsGemm& p,
                                int num_sms, cudaStream_t st, int* launches);

// The same GEMMs on CTA pairs (cluster of 2, tcgen05 cta_group::2): M = 256
// weight rows split over the pair, token tiles of up to 256 rows (tile_max 256);
// modes 0, 1, 3 as above (mode 3 at tile_max 256 only), mode 2: one 256-row weight
// slice per item (GEMM2).
cudaError_t launch_gemm_ws_pair_bf16(int mode, int tile_max, const CUtensorMap& w0,
                                     const CUtensorMap& w1, const CUtensorMap& x, const WsGemm& p,
                                     int num_sms, cudaStream_t st, int* launches);

// GEMM1 on CTA pairs with gate and up rows interleaved along M (64 of each per
// CTA, one accumulator), token tiles of up to tile_max = 256 or 512 rows:
// gate64 / up64 are the gate and up maps with [64 x 64] boxes, x the
// expert-grouped token rows with boxes of p.tok_box rows (a divisor of 128);
// p.n_wt = ceil(I / 128).
cudaError_t launch_gemm_il_pair_bf16(int tile_max, const CUtensorMap& gate64, const CUtensorMap& up64,
                                    const CUtensorMap& x, const WsGemm& p, int num_sms,
                                    cudaStream_t st, int* launches);

// Weight-stationary block-scaled MXFP4 GEMMs over the token-tile list of align.
// Codes through the TMA maps; scales through their own pointers (byte strides).
struct WsGemmMx {
  int64_t K, N, n_wt, max_tiles;
  const int32_t* num_tiles;
  const int32_t* tile_row;
  const int32_t* tile_rows;
  const int32_t* tile_expert;
  const int32_t* sorted;
  int64_t S;
  void* out;              // GEMM1: h codes; GEMM2: y bf16
  int64_t out_ld;
  uint8_t* out_sf;        // GEMM1: h scales
  int64_t out_sf_ld;
  View2 topk_w;
  int64_t k;
  const uint8_t* x_sf;    // token scales [P, K/32]
  int64_t x_sf_ld;
  const uint8_t* w0_sf;   // GEMM1: gate scales; GEMM2: w2 scales
  int64_t w0_s0, w0_s1;
  const uint8_t* w1_sf;   // GEMM1: up scales; GEMM2: w2 scales
  int64_t w1_s0, w1_s1;
  const float* w_row;     // GEMM2: routing weight per grouped row
  float* h_capture;       // GEMM1: fp32 h before quantisation, [P, I] (inspection; null: off)
  DeviceErrors* err;
};
// tile_max: 128 (3-stage ring), 96 (4-stage ring) or 32 (5-stage ring).  sf: null, or
// three maps of the raw e8m0 scales (W0, W1, token rows; uint8, no swizzle, boxes of
// 16 bytes x 128 weight rows and 16 bytes x tile_max token rows) for the TMA scale path.
cudaError_t launch_gemm_ws_mxfp4(int mode, int tile_max, const CUtensorMap& w0,
                                 const CUtensorMap& w1, const CUtensorMap& x, const CUtensorMap* sf,
                                 const WsGemmMx& p, int num_sms, cudaStream_t st, int* launches);

// MXFP4 quantiser for rows of a [R, K] bf16/f32 matrix (unit inner stride)
cudaError_t launch_quantize_rows(const void* src, int32_t src_dtype, int64_t R, int64_t K,
                                 int64_t src_ld, uint8_t* codes, int64_t codes_ld,
                                 uint8_t* scales, int64_t scales_ld, cudaStream_t st,
                                 int* launches = nullptr);

// the whole bf16 forward as one kernel for at most 32 routing slots
struct DecodeArgs {
  int64_t T, H, I, E, k;
  View2 ids, topk_w;
  __nv_bfloat16* h_ws;  // [32, I] workspace rows (by slot)
  __nv_bfloat16* y_ws;  // [32, H] workspace rows (by slot)
  __nv_bfloat16* out;
  int64_t os0, os1;
  float* part_ws;     // GEMM1 split-K partials (decode_part_bytes(I))
  int32_t max_split;  // at most this many GEMM1 K parts (1: not split)
  DeviceErrors* err;
};
// maps: gate/up/w2 3-D weight maps ([64 x 128] boxes), x1 = x [T, H] and h1 = h_ws [32, I]
// with one-row [64 x 1] boxes (read by four-row gathers); grid = num_sms
cudaError_t launch_decode_fused(const CUtensorMap& gate, const CUtensorMap& up, const CUtensorMap& w2,
                                const CUtensorMap& x1, const CUtensorMap& h1, const DecodeArgs& p,
                                int num_sms, cudaStream_t st, int* launches);

// Cross-CTA counters of the one-kernel decode paths: kDecodeSlots sets in
// library memory, dealt round-robin to calls; each launch's last CTA resets its set.
struct DecodeSync {
  unsigned int g1[32];    // GEMM1 items finished, per routed expert
  unsigned int g2[64];    // GEMM2 items finished, per 256-column output tile
  unsigned int exit_cnt;  // CTAs finished
  unsigned int pad[31];
  unsigned int g1p[1024]; // K parts of a split GEMM1 item finished, per item
};
constexpr int kDecodeMaxSplit = 4;  // GEMM1 K parts of the one-kernel path
// GEMM1 split-K partial buffer of the decode kernels, fp32
// [part][128-row tile of I][slot column][gate, up][128 rows]: the routed
// experts' token columns are packed (at most 32 slots in all), so one column
// range per (part, row tile) holds every expert's partials
inline int64_t decode_part_bytes(int64_t I) {
  return int64_t(kDecodeMaxSplit) * ((I + 127) / 128) * 32 * 2 * 128 * 4;
}
constexpr int kDecodeSlots = 16;
unsigned next_decode_slot();
DecodeSync* decode_sync_sets();  // device address on the current device (null on error)

// the MXFP4 forward as one kernel for at most 32 routing slots
struct DecodeMxArgs {
  int64_t T, H, I, E, k;
  View2 ids, topk_w, x;
  const uint8_t* gate_sf;
  int64_t gate_s0, gate_s1;
  const uint8_t* up_sf;
  int64_t up_s0, up_s1;
  const uint8_t* w2_sf;
  int64_t w2_s0, w2_s1;
  uint8_t* h_codes;  // [32, I/2] workspace rows (by slot)
  uint8_t* h_sf;     // [32, I/32]
  __nv_bfloat16* y_ws;
  __nv_bfloat16* out;
  int64_t os0, os1;
  float* part_ws;    // GEMM1 split-K partials (decode_part_bytes(I))
  int32_t max_split; // at most this many GEMM1 K parts (1: not split)
  DeviceErrors* err;
};
// maps: gate/up/w2 code maps ([128 B x 128] boxes), hc = h codes [32, I/2] bytes with a
// one-row [128 x 1] box (read by four-row gathers); grid = num_sms
cudaError_t launch_decode_fused_mx(const CUtensorMap& gate, const CUtensorMap& up,
                                   const CUtensorMap& w2, const CUtensorMap& hc,
                                   const DecodeMxArgs& p, int num_sms, cudaStream_t st,
                                   int* launches);

// router: softmax -> top-k (lower index on ties) -> optional renormalisation,
// plus the shared-expert column; one warp per token, E <= 1024, k + shared <= 32
cudaError_t launch_router_topk(const View2& logits, int64_t T, int E, int k, int renorm, int shared,
                               const View2& ids, const View2& wts, cudaStream_t st, int* launches);

// one thread waits on an mbarrier nobody arrives on, giving up after limit_ns:
// *done = 2 and one timeout counted (1 would mean the barrier completed)
cudaError_t launch_bounded_wait_probe(unsigned long long limit_ns, DeviceErrors* err,
                                      int32_t* done, cudaStream_t st);

// tensor-pipe rate of back-to-back MMAs on every SM (kind 0: bf16, 1: mxf4), TFLOP/s;
// blocking (times six launches on the legacy stream with CUDA events, best of the last five)
cudaError_t measure_mma_rate(int kind, int iters, int num_sms, DeviceErrors* err, double* tflops);

// launch helper: PDL attribute on every kernel of the forward
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace moe
