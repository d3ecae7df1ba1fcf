// Step "combine": out[t, :] = sum_{j = 0..k-1} y[inv[t*k + j], :] over the
// valid slots of token t (inv = the slot's row in expert-grouped order, -1 for
// a skipped slot), accumulated in fp32 in fixed j order and rounded once to
// bf16.  The routing weight is already folded into y by the down-projection
// epilogue.  No atomics, so the result is identical run to run and does not
// depend on how the slots were grouped.  out is written through its strides.
#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i] += __uint_as_float(w[i] << 16);
    a[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
  }
}

// One CTA per token; thread c owns 16-byte column chunks c, c + blockDim, ...
// Every thread reads the token's k row indices itself (the same k words for
// the whole CTA, served by L1), so there is no block barrier, and up to 8 row
// loads of a chunk are issued back to back before they are summed (in j order).
__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ y,
                                                      const int32_t* __restrict__ inv, int64_t T,
                                                      int64_t H, int64_t k,
                                                      __nv_bfloat16* __restrict__ out, int64_t os0,
                                                      int64_t os1, int vec_out) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t H8 = H / 8;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const int32_t* rows = inv + t * k;
    for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
      float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      int j = 0;
      for (; j + 8 <= k; j += 8) {
        int32_t r[8];
        uint4 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) r[q] = __ldg(rows + j + q);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          v[q] = r[q] >= 0 ? __ldg(reinterpret_cast<const uint4*>(y + static_cast<int64_t>(r[q]) * H) + c)
                           : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (r[q] >= 0) acc_bf16x8(a, v[q]);
      }
      for (; j < k; ++j) {
        const int32_t r = __ldg(rows + j);
        if (r >= 0) acc_bf16x8(a, __ldg(reinterpret_cast<const uint4*>(y + static_cast<int64_t>(r) * H) + c));
      }
      if (vec_out) {
        uint4 o;
        o.x = pack_bf16x2(a[0], a[1]);
        o.y = pack_bf16x2(a[2], a[3]);
        o.z = pack_bf16x2(a[4], a[5]);
        o.w = pack_bf16x2(a[6], a[7]);
        reinterpret_cast<uint4*>(out + t * os0)[c] = o;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) out[t * os0 + (c * 8 + i) * os1] = __float2bfloat16_rn(a[i]);
      }
    }
  }
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* inv, int64_t T, int64_t H,
                           int64_t k, void* out, int64_t os0, int64_t os1, cudaStream_t st,
                           int* launches) {
  const int vec_out = (os1 == 1) && ((os0 * 2) % 16 == 0) &&
                      (reinterpret_cast<uintptr_t>(out) % 16 == 0);
  int64_t blocks = T < 65535 ? T : 65535;
  if (blocks < 1) blocks = 1;
  if (launches) *launches += 1;
  return launch_pdl(combine_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, y, inv,
                    T, H, k, static_cast<__nv_bfloat16*>(out), os0, os1, vec_out);
}

}  // namespace moe
