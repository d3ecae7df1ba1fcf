// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a).
//
//   GEMM1 (gate/up + SwiGLU):  for each bm-row block b of expert e = block_expert[b]
//       G = A1_b . gate_e^T,  U = A1_b . up_e^T        (fp32 accumulators in TMEM)
//       h_b = bf16(silu(G) * U)                          (fused epilogue)
//   GEMM2 (down + routing weight):
//       Y = h_b . w2_e^T;  y[slot] = bf16(w_slot * Y[row])  for the valid rows
//
// Expert addressing (Liger-Kernel PR #1377, "Problems"): gate and up are
// [E, I, H] views of one packed w13 [E, 2I, H].  Each is described to the TMA
// unit as a 3-D tensor (H, I, E) whose expert stride is the view's real
// stride(0) in bytes, so tile (n, e) starts at base + e*stride(0) + n*TileN*stride(1)
// and each expert still covers exactly I rows: the expert's first tile is found
// from its stride, never from e * I / TileN.
//
// Kernel shape: one persistent CTA per SM, 6 warps.
//   warp 0  TMA producer (one elected lane): A tile [128 x 64] + two B boxes
//           [128 x 64] per k-step into a 4-stage ring, 128-byte swizzle
//   warp 1  TMEM allocator and MMA issuer (one elected lane):
//           tcgen05.mma.cta_group::1.kind::f16, M=128, N=256, K=16
//   warps 2-5 epilogue: tcgen05.ld of the fp32 accumulator (one row per
//           thread), fused math, staging through shared memory, coalesced stores
// Two 256-column accumulators in TMEM let the epilogue of tile i overlap the
// mainloop of tile i+1.  Tiles are ordered block-major, column-minor, so the
// CTAs working at the same time share A blocks and an expert's weight tiles in L2.
#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kBM = 128;           // tile rows (tokens): MMA M
constexpr int kBK = 64;            // bf16 elements per 128-byte swizzled row
constexpr int kBoxRows = 128;      // rows per B TMA box
constexpr int kUmmaN = 256;        // MMA N: two B boxes
constexpr int kUmmaK = 16;         // K per tcgen05.mma (kind::f16)
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;                // 16 KiB
constexpr int kBBytes = kUmmaN * kBK * 2;             // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;        // 48 KiB
constexpr int kEpiWarps = 4;
constexpr int kStagingBytes = 32 * 64;                // per epilogue warp: 32 rows x 32 bf16
constexpr int kTmemCols = 512;                        // two 256-column fp32 accumulators
constexpr int kThreads = 192;
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

// Position of 16-byte chunk `part` of staging row r (32 rows x 64 bytes), XOR
// swizzled so that both the row-wise writes and the chunk-wise reads are free
// of shared-memory bank conflicts.
__device__ __forceinline__ uint32_t stg_off(int r, int part) {
  return static_cast<uint32_t>(r * 64 + ((part ^ ((r >> 1) & 3)) << 4));
}

template <int kMode>
__device__ __forceinline__ void tile_rows(int64_t n, int32_t& row0, int32_t& row1) {
  if (kMode == 0) {  // gate and up boxes cover the same 128 intermediate rows
    row0 = static_cast<int32_t>(n * kBoxRows);
    row1 = row0;
  } else {           // one 256-row slice of w2's H rows
    row0 = static_cast<int32_t>(n * kUmmaN);
    row1 = row0 + kBoxRows;
  }
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1, const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const Smem sm = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (kMode == 0) tma_prefetch_desc(&tmB1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
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

  // Everything below reads what align/permute (or GEMM1) wrote.
  pdl_wait();
  const int64_t num_blocks = *g.num_blocks;
  const int64_t total = num_blocks * g.n_tiles;
  const int num_k = static_cast<int>((g.K + kBK - 1) / kBK);

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
        int32_t row0, row1;
        tile_rows<kMode>(n, row0, row1);
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
          uint8_t* sa = sm.stages + stage * kStageBytes;
          uint8_t* sb = sa + kABytes;
          mbar_arrive_expect_tx(&sm.full[stage], kStageBytes);
          tma_load_2d(sa, &tmA, &sm.full[stage], kb * kBK, static_cast<int32_t>(m * kBM), pol);
          tma_load_3d(sb, &tmB0, &sm.full[stage], kb * kBK, row0, e, pol);
          tma_load_3d(sb + kBoxRows * kBK * 2, kMode == 0 ? &tmB1 : &tmB0, &sm.full[stage],
                      kb * kBK, row1, e, pol);
          last_phase[stage] = static_cast<int8_t>(phase);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // unwind: let every copy this thread issued land before the CTA exits
        for (int s = 0; s < kStages; ++s)
          if (last_phase[s] >= 0) mbar_wait(&sm.full[s], static_cast<uint32_t>(last_phase[s]), g.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kUmmaN);
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      bool ok = true, issued = false;
      for (int64_t tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        if (!mbar_wait(&sm.tempty[acc], acc_phase ^ 1u, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + acc * kUmmaN;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sm.stages + stage * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            mma_bf16(d, sw128_kmajor_desc(a_addr + kk * kUmmaK * 2),
                     sw128_kmajor_desc(b_addr + kk * kUmmaK * 2), idesc,
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
    const int quad = warp & 3;  // TMEM lanes this warp may read: [32*quad, 32*quad + 32)
    const int row_in_tile = quad * 32 + lane;
    uint8_t* stg = sm.staging + (warp - 2) * kStagingBytes;
    const uint32_t stg_s = smem_u32(stg);
    uint32_t acc = 0, acc_phase = 0;
    for (int64_t tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const int64_t m = tile / g.n_tiles, n = tile - m * g.n_tiles;
      // per-row routing info (GEMM2) is independent of the accumulator: fetch it first
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
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * kUmmaN;
      constexpr int kChunks = (kMode == 0) ? 4 : 8;  // 32-column chunks of the output tile
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        uint32_t packed[16];
        if (kMode == 0) {
          uint32_t gv[32], uv[32];
          tmem_ld32(tbase + c * 32, gv);
          tmem_ld32(tbase + kBoxRows + c * 32, uv);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            packed[i] = pack_bf16x2(silu_mul(__uint_as_float(gv[2 * i]), __uint_as_float(uv[2 * i])),
                                    silu_mul(__uint_as_float(gv[2 * i + 1]), __uint_as_float(uv[2 * i + 1])));
        } else {
          uint32_t v[32];
          tmem_ld32(tbase + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            packed[i] = pack_bf16x2(wgt * __uint_as_float(v[2 * i]), wgt * __uint_as_float(v[2 * i + 1]));
        }
        // stage this thread's 32 values (64 bytes of row `lane`)
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stg_s + stg_off(lane, p)),
                       "r"(packed[4 * p]), "r"(packed[4 * p + 1]), "r"(packed[4 * p + 2]),
                       "r"(packed[4 * p + 3])
                       : "memory");
        }
        __syncwarp();
        const int64_t col0 = (kMode == 0 ? n * kBoxRows : n * kUmmaN) + c * 32;
        const bool col_ok = col0 < g.N;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int idx = q * 32 + lane;
          const int r = idx >> 2, part = idx & 3;
          uint4 v;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(stg_s + stg_off(r, part)));
          if (kMode == 0) {
            const int64_t grow = m * kBM + quad * 32 + r;
            if (col_ok)
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + grow * g.out_ld + col0 + part * 8) = v;
          } else {
            const int32_t s_r = __shfl_sync(0xffffffffu, slot, r);
            if (col_ok && s_r < g.S)
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + static_cast<int64_t>(s_r) * g.out_ld + col0 + part * 8) = v;
          }
        }
        __syncwarp();
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
cudaError_t launch_grouped(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                           const GemmArgs& g, int num_sms, cudaStream_t st) {
  static unsigned long long configured = 0;  // one bit per device
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    rc = cudaFuncSetAttribute(grouped_gemm_bf16_kernel<kMode>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmemBytes));
    if (rc != cudaSuccess) return rc;
    if (dev < 64) configured |= 1ull << dev;
  }
  int64_t grid = g.max_tiles < num_sms ? g.max_tiles : num_sms;
  if (grid < 1) grid = 1;
  return launch_pdl(grouped_gemm_bf16_kernel<kMode>, dim3(static_cast<unsigned>(grid)),
                    dim3(kThreads), kSmemBytes, st, a, b0, b1, g);
}

}  // namespace

cudaError_t launch_gemm1_bf16(const CUtensorMap& a, const CUtensorMap& gate, const CUtensorMap& up,
                              const GemmArgs& g, int num_sms, cudaStream_t st, int* launches) {
  if (launches) *launches += 1;
  return launch_grouped<0>(a, gate, up, g, num_sms, st);
}

cudaError_t launch_gemm2_bf16(const CUtensorMap& a, const CUtensorMap& w2, const GemmArgs& g,
                              int num_sms, cudaStream_t st, int* launches) {
  if (launches) *launches += 1;
  return launch_grouped<1>(a, w2, w2, g, num_sms, st);
}

}  // namespace moe
