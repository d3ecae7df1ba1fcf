// Kernels of the gradient path that the GEMMs do not cover.
//
// The gradient of the forward with respect to x and the routing weights, the
// experts frozen (the routing ids are discrete), is computed by the GEMM kernels
// run on transposed weights plus these two steps:
//   slot_dot:  dweights[t, j] = sum_o a[o] * y[inv[t*k + j], o], a = row t of a
//              token-major tensor or row inv[t*k + j] of a grouped one; the gradient
//              path takes a = dh' = w2_e^T dout_t and y = h (grouped rows, length I),
//              the same value as dout_t . (w2_e h), the expert's output before its
//              routing weight scales it;
//   transpose: the expert weights with the contraction axis swapped, so that the
//              gradient GEMMs read them K-major like the forward does: w2 [E, H, I]
//              -> [E, I, H] (dh' = w2^T dout) and the packed w13 [E, 2I, H] ->
//              [E, H, 2I] (dx = gate^T dg + up^T du in one contraction over 2I).
#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kDotWarps = 8;

// one warp per routing slot: lane l sums elements [8 l + 256 m, 8 l + 256 m + 8) for m =
// 0, 1, ... in order (16-byte loads of both rows where they are aligned), then the
// warp adds its lanes in a fixed tree; `grouped` picks row inv[s] of dout instead of row t
__global__ void __launch_bounds__(kDotWarps * 32) slot_dot_kernel(View2 dout, int grouped,
                                                                 const __nv_bfloat16* y,
                                                                 const int32_t* inv, int64_t T,
                                                                 int64_t H, int64_t k, View2 dw,
                                                                 int vec) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t s = static_cast<int64_t>(blockIdx.x) * kDotWarps + (threadIdx.x >> 5);
  if (s < T * k) {
    const int64_t t = s / k, j = s - t * k;
    const int32_t row = inv[s];
    float acc = 0.0f;
    if (row >= 0) {
      const uint16_t* d = static_cast<const uint16_t*>(dout.data) + (grouped ? row : t) * dout.s0;
      const uint16_t* yr = reinterpret_cast<const uint16_t*>(y) + static_cast<int64_t>(row) * H;
      if (vec) {
        for (int64_t o = lane * 8; o < H; o += 256) {
          const uint4 a = *reinterpret_cast<const uint4*>(d + o);
          const uint4 b = *reinterpret_cast<const uint4*>(yr + o);
          const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc = fmaf(__uint_as_float(av[q] << 16), __uint_as_float(bv[q] << 16), acc);
            acc = fmaf(__uint_as_float(av[q] & 0xffff0000u), __uint_as_float(bv[q] & 0xffff0000u), acc);
          }
        }
      } else {
        // the same elements per lane in the same order as the vector path, so a
        // strided dout gives the same bits as a contiguous one
        for (int64_t o0 = lane * 8; o0 < H; o0 += 256)
          for (int q = 0; q < 8 && o0 + q < H; ++q)
            acc = fmaf(__uint_as_float(static_cast<uint32_t>(d[(o0 + q) * dout.s1]) << 16),
                       __uint_as_float(static_cast<uint32_t>(yr[o0 + q]) << 16), acc);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    }
    if (lane == 0) static_cast<float*>(const_cast<void*>(dw.data))[t * dw.s0 + j * dw.s1] = acc;
  }
  pdl_launch_dependents();
}

// 32 x 32 tiles through shared memory (one padding column against bank conflicts)
__global__ void __launch_bounds__(32 * 8) transpose_kernel(const uint16_t* src, int64_t s0, int64_t s1,
                                                          uint16_t* dst, int64_t d0, int64_t d1,
                                                          int64_t R, int64_t C) {
  __shared__ uint16_t tile[32][33];
  const int64_t e = blockIdx.z;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 32, c0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const int64_t r = r0 + i, c = c0 + tx;
    tile[i][tx] = (r < R && c < C) ? src[e * s0 + r * s1 + c] : uint16_t(0);
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int64_t c = c0 + i, r = r0 + tx;
    if (c < C && r < R) dst[e * d0 + c * d1 + r] = tile[tx][i];
  }
}

}  // namespace

cudaError_t launch_slot_dot(const View2& dout, int grouped, const __nv_bfloat16* y, const int32_t* inv,
                            int64_t T, int64_t H, int64_t k, const View2& dw, cudaStream_t st,
                            int* launches) {
  const int64_t S = T * k;
  if (S == 0) return cudaSuccess;
  const int vec = dout.s1 == 1 && H % 8 == 0 && (dout.s0 * 2) % 16 == 0 &&
                  reinterpret_cast<uintptr_t>(dout.data) % 16 == 0 &&
                  reinterpret_cast<uintptr_t>(y) % 16 == 0;
  if (launches) *launches += 1;
  const dim3 grid(static_cast<unsigned>((S + kDotWarps - 1) / kDotWarps));
  return launch_pdl(slot_dot_kernel, grid, dim3(kDotWarps * 32), 0, st, dout, grouped, y, inv, T, H, k, dw,
                    vec);
}

cudaError_t launch_transpose_experts(const void* src, int64_t s0, int64_t s1, void* dst, int64_t d0,
                                     int64_t d1, int64_t E, int64_t R, int64_t C, cudaStream_t st) {
  if (E == 0 || R == 0 || C == 0) return cudaSuccess;
  if (E > 65535 || (R + 31) / 32 > 65535) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>((C + 31) / 32), static_cast<unsigned>((R + 31) / 32),
                  static_cast<unsigned>(E));
  transpose_kernel<<<grid, 32 * 8, 0, st>>>(static_cast<const uint16_t*>(src), s0, s1,
                                            static_cast<uint16_t*>(dst), d0, d1, R, C);
  return cudaGetLastError();
}

}  // namespace moe
