// Internal declarations shared by the host runtime and the kernel launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

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
  int32_t bm;         // block_m: rows per expert block (the MMA tile M)
  int64_t n_chunks;   // align chunks
  int64_t p_max;      // upper bound of padded slot count
  int64_t nb_max;     // upper bound of the block count
  bool mxfp4;
  size_t counts, offsets, num_blocks, chunk_counts, sorted, inv, block_expert;
  size_t a1, a1_scale, h, h_scale, y;
  size_t total;
};

constexpr int kMaxTopK = 32;            // routing columns per token
constexpr int kMaxExperts = 1024;       // experts per layer
constexpr int kAlignChunk = 4096;        // slots per CTA in the multi-CTA align
constexpr int kAlignSmallMax = 8192;     // single-CTA align up to this many slots

int32_t choose_block_m(int64_t T, int64_t k, int64_t E);
WsLayout make_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, bool mxfp4, int32_t bm);

// ---- launchers (return cudaError_t of the launch) ----------------------------

// align: ids -> counts, offsets, sorted, block_expert, num_blocks
cudaError_t launch_align(const View2& ids, int64_t T, int64_t k, int64_t E, int32_t bm,
                         int32_t* counts, int32_t* offsets, int32_t* sorted, int32_t* inv,
                         int32_t* block_expert, int32_t* num_blocks, int32_t* chunk_counts,
                         int64_t n_chunks, DeviceErrors* err, cudaStream_t st, int* launches);

// permute: A1[inv[t*k+j], :] = x[t, :] (x read once per token), padding rows zeroed
cudaError_t launch_permute_bf16(const View2& x, int64_t T, int64_t H, int64_t k, int64_t E,
                                const int32_t* inv, const int32_t* offsets, const int32_t* counts,
                                __nv_bfloat16* a1, cudaStream_t st, int* launches);

// permute + MXFP4 quantisation of x rows (codes [P, H/2], scales [P, H/32])
cudaError_t launch_permute_quant(const View2& x, int64_t T, int64_t H, int64_t k, int64_t E,
                                 const int32_t* inv, const int32_t* offsets, const int32_t* counts,
                                 uint8_t* codes, uint8_t* scales, cudaStream_t st, int* launches);

// combine: out[t, :] = sum_j y[t*k + j, :] over valid slots (fixed j order)
cudaError_t launch_combine(const __nv_bfloat16* y, const View2& ids, int64_t E, int64_t T,
                           int64_t H, int64_t k, void* out, int64_t os0, int64_t os1,
                           cudaStream_t st, int* launches);

struct GemmArgs {
  int64_t K;            // contraction length
  int64_t N;            // output columns (I for GEMM1, H for GEMM2)
  int64_t n_tiles;      // output column tiles
  int64_t max_tiles;    // upper bound of (blocks x n_tiles)
  const int32_t* num_blocks;
  const int32_t* block_expert;
  const int32_t* sorted;
  int64_t S;            // sentinel / number of slots
  void* out;            // GEMM1: h [P, I] (bf16 or e2m1 codes); GEMM2: y [S, H] bf16
  uint8_t* out_scale;   // GEMM1 MXFP4: h scales [P, I/32]
  int64_t out_ld;       // row stride of out in elements (bytes for codes)
  View2 topk_w;         // GEMM2: routing weights [T, k] f32
  int64_t k;            // top_k (GEMM2: slot -> (t, j))
  DeviceErrors* err;
};

cudaError_t launch_gemm1_bf16(const CUtensorMap& a, const CUtensorMap& gate, const CUtensorMap& up,
                              const GemmArgs& g, int num_sms, cudaStream_t st, int* launches);
cudaError_t launch_gemm2_bf16(const CUtensorMap& a, const CUtensorMap& w2, const GemmArgs& g,
                              int num_sms, cudaStream_t st, int* launches);

// MXFP4 (e2m1 codes + e8m0 scales): A codes through TMA maps, scales read
// through their own pointers/strides (bytes).  GEMM1 writes h codes to g.out and
// h scales to h_sf; GEMM2 writes y like the bf16 GEMM2.
cudaError_t launch_gemm1_mxfp4(const CUtensorMap& a, const uint8_t* a_sf, int64_t a_sf_ld,
                               const CUtensorMap& gate, const uint8_t* gate_sf, int64_t gs0,
                               int64_t gs1, const CUtensorMap& up, const uint8_t* up_sf,
                               int64_t us0, int64_t us1, uint8_t* h_sf, int64_t h_sf_ld,
                               const GemmArgs& g, int num_sms, cudaStream_t st, int* launches);
cudaError_t launch_gemm2_mxfp4(const CUtensorMap& a, const uint8_t* a_sf, int64_t a_sf_ld,
                               const CUtensorMap& w2, const uint8_t* w2_sf, int64_t ws0,
                               int64_t ws1, const GemmArgs& g, int num_sms, cudaStream_t st,
                               int* launches);

// standalone MXFP4 quantiser for rows of a [R, K] bf16/f32 matrix (unit inner stride)
cudaError_t launch_quantize_rows(const void* src, int32_t src_dtype, int64_t R, int64_t K,
                                 int64_t src_ld, uint8_t* codes, int64_t codes_ld,
                                 uint8_t* scales, int64_t scales_ld, cudaStream_t st);

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
