// Tensor-pipe rate probe: the denominator of the roofline fractions for the
// block-scaled MXFP4 GEMMs, measured instead of assumed.
//
// One CTA per SM issues `iters` back-to-back tcgen05.mma instructions of one
// kind (M = 128, N = 128 accumulating into TMEM) from operand tiles that stay
// in shared memory, then waits for them through one commit.  No global memory
// is read, so the time is the tensor pipe's alone.  Run for kind::f16 (bf16)
// and kind::mxf4 (e2m1 with e8m0 block scales), the ratio of the two rates is
// the MXFP4/bf16 peak ratio of this GPU; the absolute bf16 figure can be set
// against a library GEMM's measured bf16 peak.  Operand values are zero (their
// values do not change the rate).
#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kM = 128, kN = 128;
constexpr int kABytes = kM * 128;  // 128-byte K-major rows, 128-byte swizzle
constexpr int kBBytes = kN * 128;
constexpr int kSfAtom = 512;       // 128 rows x 4 scale bytes

template <int kKind>  // 0: kind::f16 (bf16), 1: kind::mxf4
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int iters, DeviceErrors* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a = base;
  uint8_t* b = a + kABytes;
  uint8_t* sf = b + kBBytes;                  // two scale atoms (A, B)
  uint64_t* done = reinterpret_cast<uint64_t*>(sf + 2 * kSfAtom);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (kABytes + kBBytes + 2 * kSfAtom) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(base)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0 && elect_one()) {
    const uint32_t a_addr = smem_u32(a), b_addr = smem_u32(b);
    if (kKind == 1) {
      // scale factors of A and B into TMEM columns [128, 132) and [132, 136)
      tmem_cp_32x128b_x4(tmem + 128, plain_rows16_desc(smem_u32(sf)));
      tmem_cp_32x128b_x4(tmem + 132, plain_rows16_desc(smem_u32(sf) + kSfAtom));
    }
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
        if (kKind == 0) {
          mma_bf16(tmem, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32),
                   idesc_bf16_f32(kM, kN), acc);
        } else {
          mma_mxf4(tmem, sw128_kmajor_desc(a_addr + kk * 32), sw128_kmajor_desc(b_addr + kk * 32),
                   idesc_mxf4(kM, kN, 0, 0), tmem + 128, tmem + 132, acc);
        }
      }
    }
    mma_commit(done);
    // the MMAs must have finished before TMEM is released: a second bounded
    // wait if the first gives up (a few ms of work at the largest iters)
    if (!mbar_wait(done, 0, err)) mbar_wait(done, 0, err);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

template <int kKind>
cudaError_t run_rate(int iters, int num_sms, DeviceErrors* err, float* ms) {
  // more shared memory than the tiles need, so exactly one CTA fits per SM
  const size_t smem = 120 * 1024;
  cudaError_t rc = cudaFuncSetAttribute(mma_rate_kernel<kKind>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (rc != cudaSuccess) return rc;
  cudaEvent_t e0, e1;
  if ((rc = cudaEventCreate(&e0)) != cudaSuccess) return rc;
  if ((rc = cudaEventCreate(&e1)) != cudaSuccess) {
    cudaEventDestroy(e0);
    return rc;
  }
  float best = 0.0f;
  for (int rep = 0; rep < 6 && rc == cudaSuccess; ++rep) {  // first launch is a warm-up
    cudaEventRecord(e0, 0);
    mma_rate_kernel<kKind><<<num_sms, 128, smem, 0>>>(iters, err);
    cudaEventRecord(e1, 0);
    rc = cudaEventSynchronize(e1);
    if (rc == cudaSuccess) rc = cudaGetLastError();
    float t = 0.0f;
    if (rc == cudaSuccess && rep > 0 && cudaEventElapsedTime(&t, e0, e1) == cudaSuccess)
      best = (best == 0.0f || t < best) ? t : best;
  }
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  *ms = best;
  return rc;
}

}  // namespace

cudaError_t measure_mma_rate(int kind, int iters, int num_sms, DeviceErrors* err, double* tflops) {
  float ms = 0.0f;
  const cudaError_t rc = kind == 0 ? run_rate<0>(iters, num_sms, err, &ms)
                                   : run_rate<1>(iters, num_sms, err, &ms);
  if (rc != cudaSuccess) return rc;
  // per instruction 2 * M * N * K flops, K = 16 (bf16) or 64 (e2m1); four per iteration
  const double k = kind == 0 ? 16.0 : 64.0;
  const double flops = double(num_sms) * iters * 4.0 * 2.0 * kM * kN * k;
  *tflops = ms > 0.0f ? flops / (ms * 1e-3) / 1e12 : 0.0;
  return cudaSuccess;
}

}  // namespace moe
