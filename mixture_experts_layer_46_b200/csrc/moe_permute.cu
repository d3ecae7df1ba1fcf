// Step "permute": gather the token rows of x into expert-grouped order so each
// bm-row block of the grouped GEMM reads one expert's tokens contiguously.
//   A1[inv[t*k + j], :] = x[t, :]     for every valid slot, x read once per token
// Padding rows are left as they are: a token tile's padding rows only feed MMA
// output columns (tokens) that no later step reads, and every output column
// depends on its own B row alone, so their contents cannot reach a result.
// x is read through its strides (LightLLM issue #1467 shows what dropping the
// inner stride does); the fast path needs a unit inner stride and 16-byte rows.
//
// The MXFP4 form quantises each x row with the 1x32 e8m0 rule while gathering
// (aiter PR #3859, "Details": activations are e2m1 with per-1x32 scales):
// codes [P, H/2] (even element in the low nibble) and scales [P, H/32].
#include "../../include/moe.h"
#include "moe_internal.h"
#include "moe_mx.cuh"

namespace moe {

namespace {

__device__ __forceinline__ float bf16_to_f(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

__global__ void __launch_bounds__(256) permute_bf16_kernel(View2 x, int64_t T, int64_t H, int64_t k,
                                                           const int32_t* __restrict__ inv,
                                                           __nv_bfloat16* __restrict__ a1, int vec_ok) {
  // dependents may start before align is done (the GEMM requests weights
  // meanwhile); everything here still waits for align
  pdl_launch_dependents();
  pdl_wait();
  const int64_t H8 = H / 8;
  {
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
      const int32_t* pos = inv + t * k;
      if (vec_ok) {
        // up to four 16-byte chunks of the row loaded before any store
        const uint4* __restrict__ src =
            reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x.data) + t * x.s0);
        for (int64_t c0 = threadIdx.x; c0 < H8; c0 += 4 * blockDim.x) {
          uint4 v[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int64_t c = c0 + i * blockDim.x;
            if (c < H8) v[i] = __ldg(src + c);
          }
          for (int j = 0; j < k; ++j) {
            const int32_t p = __ldg(pos + j);
            if (p < 0) continue;
            uint4* dst = reinterpret_cast<uint4*>(a1 + static_cast<int64_t>(p) * H);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int64_t c = c0 + i * blockDim.x;
              if (c < H8) dst[c] = v[i];
            }
          }
        }
      } else {
        const uint16_t* src = static_cast<const uint16_t*>(x.data) + t * x.s0;
        for (int64_t h = threadIdx.x; h < H; h += blockDim.x) {
          const uint16_t v = src[h * x.s1];
          for (int j = 0; j < k; ++j) {
            const int32_t p = __ldg(pos + j);
            if (p >= 0) reinterpret_cast<uint16_t*>(a1 + static_cast<int64_t>(p) * H)[h] = v;
          }
        }
      }
    }
  }
}

// One thread per 32-element block of a row; a CTA walks tokens.
__global__ void __launch_bounds__(128) permute_quant_kernel(View2 x, int64_t T, int64_t H, int64_t k,
                                                            const int32_t* inv, uint8_t* codes,
                                                            uint8_t* scales, View2 topk_w,
                                                            float* w_row, int vec_ok) {
  // dependents may be scheduled at once; everything here still waits for align
  pdl_launch_dependents();
  pdl_wait();
  const int64_t nb = H / 32;  // blocks per row
  {
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
      const int32_t* pos = inv + t * k;
      // routing weight of each slot at its grouped row, for the down projection's epilogue
      if (threadIdx.x < k && pos[threadIdx.x] >= 0)
        w_row[pos[threadIdx.x]] =
            static_cast<const float*>(topk_w.data)[t * topk_w.s0 + threadIdx.x * topk_w.s1];
      for (int64_t b = threadIdx.x; b < nb; b += blockDim.x) {
        float v[32];
        if (vec_ok) {
          const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x.data) + t * x.s0 + b * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 u = src[q];
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              v[q * 8 + 2 * i] = bf16_to_f(static_cast<uint16_t>(w4[i] & 0xffffu));
              v[q * 8 + 2 * i + 1] = bf16_to_f(static_cast<uint16_t>(w4[i] >> 16));
            }
          }
        } else {
          const uint16_t* src = static_cast<const uint16_t*>(x.data) + t * x.s0;
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = bf16_to_f(src[(b * 32 + i) * x.s1]);
        }
        uint32_t w[4];
        const uint32_t sc = mx_quant32(v, w);
        for (int j = 0; j < k; ++j) {
          const int32_t p = __ldg(pos + j);
          if (p < 0) continue;
          *reinterpret_cast<uint4*>(codes + static_cast<int64_t>(p) * (H / 2) + b * 16) =
              make_uint4(w[0], w[1], w[2], w[3]);
          scales[static_cast<int64_t>(p) * nb + b] = static_cast<uint8_t>(sc);
        }
      }
    }
  }
}

// Row quantiser: one thread per 32-element block (weights, offline); 16-byte
// accesses when the rows allow them.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const void* src, int32_t src_dtype,
                                                            int64_t R, int64_t K, int64_t src_ld,
                                                            uint8_t* codes, int64_t codes_ld,
                                                            uint8_t* scales, int64_t scales_ld,
                                                            int vec_ok) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t nb = K / 32;
  const int64_t total = R * nb;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / nb, b = i - r * nb;
    float v[32];
    if (src_dtype == MOE_BF16) {
      const uint16_t* p = static_cast<const uint16_t*>(src) + r * src_ld + b * 32;
      if (vec_ok) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + q);
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            v[q * 8 + 2 * h] = bf16_to_f(static_cast<uint16_t>(w4[h] & 0xffffu));
            v[q * 8 + 2 * h + 1] = bf16_to_f(static_cast<uint16_t>(w4[h] >> 16));
          }
        }
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q) v[q] = bf16_to_f(p[q]);
      }
    } else {
      const float* p = static_cast<const float*>(src) + r * src_ld + b * 32;
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] = p[q];
    }
    uint32_t w[4];
    const uint32_t sc = mx_quant32(v, w);
    uint8_t* c = codes + r * codes_ld + b * 16;
    if (vec_ok) {
      *reinterpret_cast<uint4*>(c) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        c[4 * q + 0] = w[q] & 0xffu;
        c[4 * q + 1] = (w[q] >> 8) & 0xffu;
        c[4 * q + 2] = (w[q] >> 16) & 0xffu;
        c[4 * q + 3] = w[q] >> 24;
      }
    }
    scales[r * scales_ld + b] = static_cast<uint8_t>(sc);
  }
}

}  // namespace

static int token_blocks(int64_t T) {
  int64_t b = T < 2048 ? T : 2048;
  return static_cast<int>(b < 1 ? 1 : b);
}

cudaError_t launch_permute_bf16(const View2& x, int64_t T, int64_t H, int64_t k,
                                const int32_t* inv, __nv_bfloat16* a1, cudaStream_t st,
                                int* launches) {
  const int vec_ok = (x.s1 == 1) && ((x.s0 * 2) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(x.data) % 16 == 0);
  if (launches) *launches += 1;
  return launch_pdl(permute_bf16_kernel, dim3(static_cast<unsigned>(token_blocks(T))), dim3(256), 0,
                    st, x, T, H, k, inv, a1, vec_ok);
}

cudaError_t launch_permute_quant(const View2& x, int64_t T, int64_t H, int64_t k,
                                 const int32_t* inv, uint8_t* codes, uint8_t* scales,
                                 const View2& topk_w, float* w_row, cudaStream_t st,
                                 int* launches) {
  const int vec_ok = (x.s1 == 1) && ((x.s0 * 2) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(x.data) % 16 == 0);
  if (launches) *launches += 1;
  return launch_pdl(permute_quant_kernel, dim3(static_cast<unsigned>(token_blocks(T))), dim3(128), 0,
                    st, x, T, H, k, inv, codes, scales, topk_w, w_row, vec_ok);
}

cudaError_t launch_quantize_rows(const void* src, int32_t src_dtype, int64_t R, int64_t K,
                                 int64_t src_ld, uint8_t* codes, int64_t codes_ld,
                                 uint8_t* scales, int64_t scales_ld, cudaStream_t st,
                                 int* launches) {
  const int64_t total = R * (K / 32);
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  // 16-byte source and code accesses when every block starts on a 16-byte boundary
  const int vec_ok = src_dtype == MOE_BF16 && (src_ld * 2) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(src) % 16 == 0 && codes_ld % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(codes) % 16 == 0;
  if (launches) *launches += 1;
  return launch_pdl(quantize_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st,
                    src, src_dtype, R, K, src_ld, codes, codes_ld, scales, scales_ld, vec_ok);
}

}  // namespace moe
