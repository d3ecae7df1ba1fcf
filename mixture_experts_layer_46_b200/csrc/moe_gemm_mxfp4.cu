// Block-scaled MXFP4 grouped expert GEMMs (tcgen05.mma kind::mxf4, sm_100a).
//
// Operands are packed e2m1 codes (two per byte) with one e8m0 scale per 32
// consecutive elements of the contraction axis (aiter PR #3859, "Details":
// float4_e2m1fn_x2 weights and activations, QuantType.per_1x32):
//   GEMM1: A1 codes [P, H/2] x gate/up codes [E, I, H/2] -> G, U (fp32 in TMEM)
//          h = silu(G) * U quantised per 1x32 along I -> codes [P, I/2], scales [P, I/32]
//   GEMM2: h codes x w2 codes [E, H, I/2] -> Y; y[slot] = bf16(w_slot * Y[row])
// Expert addressing is the same as the bf16 kernels: 3-D TMA maps whose expert
// stride is each view's real stride(0) (Liger-Kernel PR #1377, "Problems").
//
// Kernel shape: one persistent CTA per SM, 7 warps.
//   warp 0    TMA producer: A [128 rows x 128 B] + two B boxes [64 rows x 128 B]
//             per k-step (256 elements of K), 6-stage ring, 128-byte swizzle
//   warp 1    TMEM allocator, MMA issuer: per stage copies the stage's scales
//             from shared memory to TMEM (tcgen05.cp 32x128b.warpx4) and issues
//             4 x tcgen05.mma.kind::mxf4.block_scale (M=128, N=128, K=64)
//   warp 2    scale producer: reads the stage's e8m0 scales through their strides
//             and writes them in the 128-row x 4-block atom the tensor core reads:
//             byte (m % 32) * 16 + (m / 32) * 4 + block
//   warps 3-6 epilogue (one accumulator row per thread)
// TMEM: two 128-column accumulators, then 16 scale columns per stage
// (A: 2 atoms x 4 columns, B: 2 atoms x 4 columns).
#include "../../include/moe.h"
#include "moe_internal.h"
#include "moe_mx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;
constexpr int kRowBytes = 128;                 // packed bytes per row per stage (256 elements)
constexpr int kBoxRows = 64;                   // rows per B TMA box
constexpr int kUmmaN = 128;
constexpr int kUmmaKBytes = 32;                // 64 e2m1 elements per instruction
constexpr int kStages = 6;
constexpr int kABytes = kBM * kRowBytes;       // 16 KiB
constexpr int kBBytes = kUmmaN * kRowBytes;    // 16 KiB
constexpr int kAtomBytes = 512;                // 128 rows x 4 scale blocks
constexpr int kSfABytes = 2 * kAtomBytes;      // 8 blocks of 32 per stage
constexpr int kSfBBytes = 2 * kAtomBytes;
constexpr int kStageBytes = kABytes + kBBytes + kSfABytes + kSfBBytes;  // 34 KiB
constexpr int kEpiWarps = 4;
constexpr int kStagingBytes = 32 * 64;
constexpr int kAccCols = 128;
constexpr int kSfColsPerStage = 16;
constexpr int kTmemCols = 512;
constexpr int kThreads = 224;
constexpr size_t kSmemBytes = 1024 + size_t(kStages) * kStageBytes + kEpiWarps * kStagingBytes +
                              (2 * kStages + 5) * 8 + 16;

struct Smem {
  uint8_t* stages;
  uint8_t* staging;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* drain;
  uint32_t* tmem_slot;
};

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.stages = base;
  s.staging = base + kStages * kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.staging + kEpiWarps * kStagingBytes);
  s.full = bars;
  s.empty = bars + kStages;
  s.tfull = bars + 2 * kStages;
  s.tempty = s.tfull + 2;
  s.drain = s.tempty + 2;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.drain + 1);
  return s;
}

__device__ __forceinline__ uint32_t stg_off(int r, int part) {
  return static_cast<uint32_t>(r * 64 + ((part ^ ((r >> 1) & 3)) << 4));
}

struct MxArgs {
  const uint8_t* a_sf;   // [P, K/32] activation scales (row stride a_sf_ld bytes)
  int64_t a_sf_ld;
  const uint8_t* b0_sf;  // GEMM1: gate scales; GEMM2: w2 scales ([E, N, K/32], strides in bytes)
  int64_t b0_s0, b0_s1;
  const uint8_t* b1_sf;  // GEMM1: up scales
  int64_t b1_s0, b1_s1;
  uint8_t* h_sf;         // GEMM1 output scales [P, I/32]
  int64_t h_sf_ld;
};

__device__ __forceinline__ uint2 ld_u2(const uint8_t* p) {
  return *reinterpret_cast<const uint2*>(p);
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_mxfp4_kernel(const __grid_constant__ CUtensorMap tmA,
                              const __grid_constant__ CUtensorMap tmB0,
                              const __grid_constant__ CUtensorMap tmB1, const GemmArgs g,
                              const MxArgs mx) {
  extern __shared__ uint8_t smem_raw[];
  const Smem sm = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (kMode == 0) tma_prefetch_desc(&tmB1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 2);  // TMA producer (with bytes) + scale producer
      mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.tfull[a], 1);
      mbar_init(&sm.tempty[a], kEpiWarps);
    }
    mbar_init(sm.drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(sm.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_slot;

  pdl_wait();
  const int64_t num_blocks = *g.num_blocks;
  const int64_t total = num_blocks * g.n_tiles;
  const int num_k = static_cast<int>(g.K / 256);  // K % 256 == 0 (validated)

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      uint32_t stage = 0, phase = 0;
      int8_t last_phase[kStages];
      for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
      const uint64_t pol = l2_policy_evict_last();
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const int64_t m = tile / g.n_tiles, n = tile - m * g.n_tiles;
        const int32_t e = g.block_expert[m];
        const int32_t row0 = static_cast<int32_t>(kMode == 0 ? n * kBoxRows : n * kUmmaN);
        const int32_t row1 = kMode == 0 ? row0 : row0 + kBoxRows;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
          uint8_t* sa = sm.stages + stage * kStageBytes;
          uint8_t* sb = sa + kABytes;
          mbar_arrive_expect_tx(&sm.full[stage], kABytes + kBBytes);
          tma_load_2d(sa, &tmA, &sm.full[stage], kb * kRowBytes, static_cast<int32_t>(m * kBM), pol);
          tma_load_3d(sb, &tmB0, &sm.full[stage], kb * kRowBytes, row0, e, pol);
          tma_load_3d(sb + kBoxRows * kRowBytes, kMode == 0 ? &tmB1 : &tmB0, &sm.full[stage],
                      kb * kRowBytes, row1, e, pol);
          last_phase[stage] = static_cast<int8_t>(phase);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (last_phase[s] >= 0) mbar_wait(&sm.full[s], static_cast<uint32_t>(last_phase[s]), g.err);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale producer
    uint32_t stage = 0, phase = 0;
    for (int64_t tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const int64_t m = tile / g.n_tiles, n = tile - m * g.n_tiles;
      const int32_t e = g.block_expert[m];
      bool ok = true;
      for (int kb = 0; kb < num_k; ++kb) {
        if (!mbar_wait(&sm.empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
        uint8_t* sfa = sm.stages + stage * kStageBytes + kABytes + kBBytes;
        uint8_t* sfb = sfa + kSfABytes;
        uint32_t alo[4], ahi[4], blo[4], bhi[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = lane + 32 * j;
          const uint2 va = ld_u2(mx.a_sf + (m * kBM + r) * mx.a_sf_ld + kb * 8);
          alo[j] = va.x;
          ahi[j] = va.y;
          const uint8_t* pb;
          if (kMode == 0) {
            pb = (r < kBoxRows)
                     ? mx.b0_sf + e * mx.b0_s0 + (n * kBoxRows + r) * mx.b0_s1
                     : mx.b1_sf + e * mx.b1_s0 + (n * kBoxRows + (r - kBoxRows)) * mx.b1_s1;
          } else {
            pb = mx.b0_sf + e * mx.b0_s0 + (n * kUmmaN + r) * mx.b0_s1;
          }
          const uint2 vb = ld_u2(pb + kb * 8);
          blo[j] = vb.x;
          bhi[j] = vb.y;
        }
        const uint32_t a_s = smem_u32(sfa) + 16 * lane, b_s = smem_u32(sfb) + 16 * lane;
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a_s), "r"(alo[0]), "r"(alo[1]),
                     "r"(alo[2]), "r"(alo[3]) : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a_s + kAtomBytes), "r"(ahi[0]),
                     "r"(ahi[1]), "r"(ahi[2]), "r"(ahi[3]) : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(b_s), "r"(blo[0]), "r"(blo[1]),
                     "r"(blo[2]), "r"(blo[3]) : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(b_s + kAtomBytes), "r"(bhi[0]),
                     "r"(bhi[1]), "r"(bhi[2]), "r"(bhi[3]) : "memory");
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.full[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true, issued = false;
      for (int64_t tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        if (!mbar_wait(&sm.tempty[acc], acc_phase ^ 1u, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + acc * kAccCols;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sm.stages + stage * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
          const uint32_t sfa_smem = b_addr + kBBytes;
          const uint32_t sfb_smem = sfa_smem + kSfABytes;
          const uint32_t sfa_t = tmem_base + 2 * kAccCols + stage * kSfColsPerStage;
          const uint32_t sfb_t = sfa_t + 8;
          tmem_cp_32x128b_x4(sfa_t, plain_rows16_desc(sfa_smem));
          tmem_cp_32x128b_x4(sfa_t + 4, plain_rows16_desc(sfa_smem + kAtomBytes));
          tmem_cp_32x128b_x4(sfb_t, plain_rows16_desc(sfb_smem));
          tmem_cp_32x128b_x4(sfb_t + 4, plain_rows16_desc(sfb_smem + kAtomBytes));
#pragma unroll
          for (int kk = 0; kk < kRowBytes / kUmmaKBytes; ++kk) {
            const uint32_t atom = kk >> 1, sfid = 2u * (kk & 1);
            const uint32_t idesc = idesc_mxf4(kBM, kUmmaN, sfid, sfid);
            mma_mxf4(d, sw128_kmajor_desc(a_addr + kk * kUmmaKBytes),
                     sw128_kmajor_desc(b_addr + kk * kUmmaKBytes), idesc,
                     (sfa_t + 4 * atom) | (sfid << 30), (sfb_t + 4 * atom) | (sfid << 30),
                     (kb > 0 || kk > 0) ? 1u : 0u);
          }
          issued = true;
          mma_commit(&sm.empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&sm.tfull[acc]);
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok && issued) {
        mma_commit(sm.drain);
        mbar_wait(sm.drain, 0, g.err);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    uint8_t* stg = sm.staging + (warp - 3) * kStagingBytes;
    const uint32_t stg_s = smem_u32(stg);
    uint32_t acc = 0, acc_phase = 0;
    for (int64_t tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const int64_t m = tile / g.n_tiles, n = tile - m * g.n_tiles;
      int32_t slot = 0;
      float wgt = 0.0f;
      if (kMode == 1) {
        slot = g.sorted[m * kBM + row_in_tile];
        if (slot < g.S) {
          const int64_t t = slot / g.k, j = slot - t * g.k;
          wgt = static_cast<const float*>(g.topk_w.data)[t * g.topk_w.s0 + j * g.topk_w.s1];
        }
      }
      if (!mbar_wait(&sm.tfull[acc], acc_phase, g.err)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * kAccCols;
      if (kMode == 0) {
        // 64 intermediate columns per tile: two 1x32 blocks, quantised in registers
        const int64_t p = m * kBM + row_in_tile;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t gv[32], uv[32];
          tmem_ld32(tbase + c * 32, gv);
          tmem_ld32(tbase + kBoxRows + c * 32, uv);
          tmem_wait_ld();
          float hv[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) hv[i] = silu_mul(__uint_as_float(gv[i]), __uint_as_float(uv[i]));
          uint32_t w[4];
          const uint32_t sc = mx_quant32(hv, w);
          const int64_t col = n * kBoxRows + c * 32;  // intermediate index of the block start
          *reinterpret_cast<uint4*>(static_cast<uint8_t*>(g.out) + p * g.out_ld + col / 2) =
              make_uint4(w[0], w[1], w[2], w[3]);
          mx.h_sf[p * mx.h_sf_ld + col / 32] = static_cast<uint8_t>(sc);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kUmmaN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tbase + c * 32, v);
          tmem_wait_ld();
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            packed[i] = pack_bf16x2(wgt * __uint_as_float(v[2 * i]), wgt * __uint_as_float(v[2 * i + 1]));
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg_s + stg_off(lane, q)),
                         "r"(packed[4 * q]), "r"(packed[4 * q + 1]), "r"(packed[4 * q + 2]),
                         "r"(packed[4 * q + 3])
                         : "memory");
          }
          __syncwarp();
          const int64_t col0 = n * kUmmaN + c * 32;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int idx = q * 32 + lane;
            const int r = idx >> 2, part = idx & 3;
            uint4 vv;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(vv.x), "=r"(vv.y), "=r"(vv.z), "=r"(vv.w)
                         : "r"(stg_s + stg_off(r, part)));
            const int32_t s_r = __shfl_sync(0xffffffffu, slot, r);
            if (col0 < g.N && s_r < g.S)
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + static_cast<int64_t>(s_r) * g.out_ld + col0 + part * 8) = vv;
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.tempty[acc]);
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  pdl_launch_dependents();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int kMode>
cudaError_t launch_mx(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                      const GemmArgs& g, const MxArgs& mx, int num_sms, cudaStream_t st) {
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    rc = cudaFuncSetAttribute(grouped_gemm_mxfp4_kernel<kMode>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
    if (rc != cudaSuccess) return rc;
    if (dev < 64) configured |= 1ull << dev;
  }
  int64_t grid = g.max_tiles < num_sms ? g.max_tiles : num_sms;
  if (grid < 1) grid = 1;
  return launch_pdl(grouped_gemm_mxfp4_kernel<kMode>, dim3(static_cast<unsigned>(grid)),
                    dim3(kThreads), kSmemBytes, st, a, b0, b1, g, mx);
}

}  // namespace

cudaError_t launch_gemm1_mxfp4(const CUtensorMap& a, const uint8_t* a_sf, int64_t a_sf_ld,
                               const CUtensorMap& gate, const uint8_t* gate_sf, int64_t gs0,
                               int64_t gs1, const CUtensorMap& up, const uint8_t* up_sf,
                               int64_t us0, int64_t us1, uint8_t* h_sf, int64_t h_sf_ld,
                               const GemmArgs& g, int num_sms, cudaStream_t st, int* launches) {
  MxArgs mx;
  mx.a_sf = a_sf;
  mx.a_sf_ld = a_sf_ld;
  mx.b0_sf = gate_sf;
  mx.b0_s0 = gs0;
  mx.b0_s1 = gs1;
  mx.b1_sf = up_sf;
  mx.b1_s0 = us0;
  mx.b1_s1 = us1;
  mx.h_sf = h_sf;
  mx.h_sf_ld = h_sf_ld;
  if (launches) *launches += 1;
  return launch_mx<0>(a, gate, up, g, mx, num_sms, st);
}

cudaError_t launch_gemm2_mxfp4(const CUtensorMap& a, const uint8_t* a_sf, int64_t a_sf_ld,
                               const CUtensorMap& w2, const uint8_t* w2_sf, int64_t ws0,
                               int64_t ws1, const GemmArgs& g, int num_sms, cudaStream_t st,
                               int* launches) {
  MxArgs mx;
  mx.a_sf = a_sf;
  mx.a_sf_ld = a_sf_ld;
  mx.b0_sf = w2_sf;
  mx.b0_s0 = ws0;
  mx.b0_s1 = ws1;
  mx.b1_sf = w2_sf;
  mx.b1_s0 = ws0;
  mx.b1_s1 = ws1;
  mx.h_sf = nullptr;
  mx.h_sf_ld = 0;
  if (launches) *launches += 1;
  return launch_mx<1>(a, w2, w2, g, mx, num_sms, st);
}

}  // namespace moe
