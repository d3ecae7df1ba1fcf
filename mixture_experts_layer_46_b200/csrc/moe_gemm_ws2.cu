// Weight-stationary grouped expert GEMMs on CTA pairs (bf16, tcgen05 cta_group::2).
//
// Same work decomposition as moe_gemm_ws.cu — the expert weights are the
// MMA's M side, one expert's token tile the N side — but two CTAs of a
// cluster share every MMA: M = 256 weight rows (128 in each CTA's shared
// memory), N = up to 256 token rows (each CTA loads half).  Each CTA moves
// 48 KiB per 8.4 MFLOP through shared memory, half the bytes per FLOP of the
// single-CTA kernel.  Expert addressing is unchanged: 3-D TMA maps whose
// expert stride is the view's real stride(0) (Liger-Kernel PR #1377, "Problems").
//
//   GEMM1: W0 = gate rows [256 w, 256 w + 256), W1 = the same up rows;
//          CTA r holds rows 256 w + 128 r + [0, 128) of both;
//          h[token, i] = bf16(silu(acc0) * acc1)
//   GEMM2: W0 = w2 rows [512 w, 512 w + 256), W1 = [512 w + 256, 512 w + 512);
//          y[token row, o] = bf16(w_slot * acc)
//   GEMM2, one slice (mode 2): W0 = w2 rows [256 w, 256 w + 256) only, so a
//          256-row token tile still fits two accumulator buffers in TMEM
//
// Pair protocol (cluster of 2, rank 0 leads):
//   * both producers wait on their own `empty` slot, load their halves with
//     cta_group::2 TMA that completes on the LEADER's `full` barrier; only the
//     leader arms that barrier with the bytes of both CTAs;
//   * the leader's MMA thread waits on its `full`, issues
//     tcgen05.mma.cta_group::2 (M=256) into both CTAs' TMEM and commits with
//     multicast to `empty` / `tfull` of both CTAs;
//   * each CTA's epilogue reads its own TMEM lanes (its 128 weight rows x all
//     N tokens) and arrives on the leader's `tempty` through the cluster window.
// No TMA multicast is used: every CTA loads only its own tiles.
#include "../../include/moe.h"
#include "moe_internal.h"
#include "moe_pair.cuh"

namespace moe {
namespace {

constexpr int kWRows = 128;                  // weight rows per CTA per weight tile
constexpr int kBK = 64;
constexpr int kUmmaK = 16;
constexpr int kEpiWarps = 8;                 // two per TMEM lane quadrant
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kTmemCols = 512;
constexpr int kWBytes = kWRows * kBK * 2;    // 16 KiB
constexpr int kStagingBytes = 32 * 64;

// kNmax token rows per tile (per pair, each CTA loads half).  Modes 0 and 1
// stage two weight tiles per k-block and accumulate into acc0 [0, kNmax) +
// acc1 [kNmax, 2 kNmax); mode 2 stages one and accumulates into acc0 only.
// Two accumulator buffers when they fit, so the epilogue overlaps the next
// item's mainloop; as many stages as about 208 KiB of shared memory holds.
template <int kMode, int kNmax>
struct PairCfg {
  static constexpr int kTiles = kMode == 2 ? 1 : 2;
  static constexpr int kXBytes = (kNmax / 2) * kBK * 2;
  static constexpr int kStageBytes = kTiles * kWBytes + kXBytes;
  static constexpr int kStagesFit = (208 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kBufCols = kTiles * kNmax;
  static constexpr int kBufs = kTmemCols / kBufCols >= 2 ? 2 : 1;
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes +
                                  kEpiWarps * kStagingBytes + (2 * kStages + 5) * 8 + 16;
};

struct Args {
  int64_t K, N, n_wt;
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
  int32_t weights_evict_first;
  int32_t tok_box;  // token rows per TMA box (the map's box height)
  int32_t unit_w;   // modes 1/2: weight 1 for every routed slot
  const __nv_bfloat16* dh;  // mode 3: gradient of h [P, N], row stride dh_ld
  int64_t dh_ld;
  __nv_bfloat16* h_out;     // mode 3: recomputed h [P, N], row stride h_ld
  int64_t h_ld;
  DeviceErrors* err;
};

template <int kMode, int kNmax>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_ws_pair_kernel(const __grid_constant__ CUtensorMap tmW0,
                        const __grid_constant__ CUtensorMap tmW1,
                        const __grid_constant__ CUtensorMap tmX, const Args g) {
  using C = PairCfg<kMode, kNmax>;
  constexpr int kStages = C::kStages;
  constexpr int kStageBytes = C::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint8_t* staging = base + kStages * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + kEpiWarps * kStagingBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = (rank == 0);

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW0);
    if (kMode == 0 || kMode == 3) tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmX);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  pdl_wait();
  const int64_t total = static_cast<int64_t>(*g.num_tiles) * g.n_wt;
  const int num_k = static_cast<int>((g.K + kBK - 1) / kBK);
  const int64_t pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (elect_one()) {
      uint32_t stage = 0, phase = 0;
      int8_t last_phase[kStages];
      for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
      const uint64_t pol = l2_policy_evict_last();
      const uint64_t wpol = g.weights_evict_first ? l2_policy_evict_first() : pol;
      bool ok = true;
      for (int64_t item = pair; item < total && ok; item += n_pairs) {
        const int64_t t = item / g.n_wt, wt = item - t * g.n_wt;
        const int32_t e = g.tile_expert[t], row0 = g.tile_row[t], rows = g.tile_rows[t];
        // weight rows of this CTA: GEMM1 gate/up rows 256 wt + 128 rank; GEMM2 w2
        // rows 512 wt + 128 rank (+ 256 for the second slice); single-slice
        // GEMM2 w2 rows 256 wt + 128 rank
        const int32_t w0 = static_cast<int32_t>((kMode == 1 ? wt * 4 * kWRows : wt * 2 * kWRows) + rank * kWRows);
        const int32_t w1 = kMode == 1 ? w0 + 2 * kWRows : w0;
        const int32_t half = rows / 2;
        const int32_t my_row0 = row0 + static_cast<int32_t>(rank) * half;
        // whole boxes: a box may run past this CTA's half (rows the MMA's N excludes)
        const int nbox = (half + g.tok_box - 1) / g.tok_box;
        const uint32_t bytes_pair = 2 * (C::kTiles * kWBytes + nbox * g.tok_box * kBK * 2);
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
          uint8_t* sw0 = stages + stage * kStageBytes;
          uint8_t* sw1 = sw0 + kWBytes;
          uint8_t* sx = sw0 + C::kTiles * kWBytes;
          if (leader) mbar_arrive_expect_tx(&full[stage], bytes_pair);
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          tma_load_3d_pair(sw0, &tmW0, fb, kb * kBK, w0, e, wpol);
          if (C::kTiles == 2)
            tma_load_3d_pair(sw1, (kMode == 0 || kMode == 3) ? &tmW1 : &tmW0, fb, kb * kBK, w1, e, wpol);
          for (int b = 0; b < nbox; ++b)
            tma_load_2d_pair(sx + b * g.tok_box * kBK * 2, &tmX, fb, kb * kBK, my_row0 + b * g.tok_box, pol);
          last_phase[stage] = static_cast<int8_t>(phase);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && leader) {
        for (int s = 0; s < kStages; ++s)
          if (last_phase[s] >= 0) mbar_wait(&full[s], static_cast<uint32_t>(last_phase[s]), g.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (leader && elect_one()) {
      uint32_t stage = 0, phase = 0, buf = 0, acc_phase = 0;
      bool ok = true, issued = false;
      for (int64_t item = pair; item < total && ok; item += n_pairs) {
        const int64_t t = item / g.n_wt;
        const int32_t rows = g.tile_rows[t];
        const uint32_t idesc = idesc_bf16_f32(2 * kWRows, rows);
        if (!mbar_wait(&tempty[buf], acc_phase ^ 1u, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc0 = tmem_base + buf * C::kBufCols, acc1 = acc0 + kNmax;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&full[stage], phase, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t w0_addr = smem_u32(stages + stage * kStageBytes);
          const uint32_t w1_addr = w0_addr + kWBytes;
          const uint32_t x_addr = w0_addr + C::kTiles * kWBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint64_t xd = sw128_kmajor_desc(x_addr + kk * kUmmaK * 2);
            const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
            mma_bf16_pair(acc0, sw128_kmajor_desc(w0_addr + kk * kUmmaK * 2), xd, idesc, acc);
            if (C::kTiles == 2)
              mma_bf16_pair(acc1, sw128_kmajor_desc(w1_addr + kk * kUmmaK * 2), xd, idesc, acc);
          }
          issued = true;
          commit_pair(&empty[stage], 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        commit_pair(&tfull[buf], 0x3);
        if (++buf == C::kBufs) { buf = 0; acc_phase ^= 1u; }
      }
      if (issued) {
        // let every tcgen05 operation of the pair (and its multicast arrivals) finish
        commit_pair(drain, 0x1);
        mbar_wait(drain, 0, g.err);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    uint8_t* stg = staging + (warp - 2) * kStagingBytes;
    const uint32_t stg_s = smem_u32(stg);
    const uint32_t lane_quad = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t buf = 0, acc_phase = 0;
    for (int64_t item = pair; item < total; item += n_pairs) {
      const int64_t t = item / g.n_wt, wt = item - t * g.n_wt;
      const int32_t row0 = g.tile_row[t], rows = g.tile_rows[t];
      // GEMM2: this warp's chunks are c = half, half + 2, ...: fetch their slots
      // and routing weights while the accumulator is being built
      int32_t slot_r[kNmax / 64];
      float w_r[kNmax / 64];
      if (kMode == 1 || kMode == 2) {
#pragma unroll
        for (int i = 0; i < kNmax / 64; ++i) {
          const int c = half + 2 * i;
          slot_r[i] = (c * 32 < rows) ? g.sorted[row0 + c * 32 + lane] : static_cast<int32_t>(g.S);
        }
#pragma unroll
        for (int i = 0; i < kNmax / 64; ++i) {
          w_r[i] = 0.0f;
          if (slot_r[i] < g.S) {
            const int64_t tt = slot_r[i] / g.k, jj = slot_r[i] - tt * g.k;
            w_r[i] = g.unit_w ? 1.0f
                              : static_cast<const float*>(g.topk_w.data)[tt * g.topk_w.s0 + jj * g.topk_w.s1];
          }
        }
      }
      if (!mbar_wait(&tfull[buf], acc_phase, g.err)) break;
      tc_fence_after();
      const uint32_t lane_base = lane_quad + buf * C::kBufCols;
#pragma unroll
      for (int i = 0; i < kNmax / 64; ++i) {
        const int c = half + 2 * i;
        if (c * 32 >= rows) break;
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem_base + lane_base + c * 32, v0);
        if (C::kTiles == 2) tmem_ld32(tmem_base + lane_base + kNmax + c * 32, v1);
        float wj[32];
        if (kMode == 1 || kMode == 2) {
#pragma unroll
          for (int j = 0; j < 32; ++j) wj[j] = __shfl_sync(0xffffffffu, w_r[i], j);
        }
        if (kMode == 3) {
          // gradient of h = silu(g) u for this warp's 32 rows of I and the chunk's 32
          // token rows: dg, du and h go out through the staging tile in turn
          const int64_t col0 = wt * 2 * kWRows + rank * kWRows + quad * 32;
          const bool col_ok = col0 < g.N;
          float dhv[32];
          const __nv_bfloat16* dsrc = g.dh + (row0 + c * 32) * g.dh_ld + col0 + lane;
#pragma unroll
          for (int j = 0; j < 32; ++j) dhv[j] = col_ok ? __bfloat162float(dsrc[j * g.dh_ld]) : 0.0f;
          tmem_wait_ld();
#pragma unroll 1
          for (int o = 0; o < 3; ++o) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float gg = __uint_as_float(v0[j]), uu = __uint_as_float(v1[j]);
              const float sg = __fdividef(1.0f, 1.0f + __expf(-gg));
              const float v = o == 0 ? dhv[j] * uu * sg * (1.0f + gg * (1.0f - sg))
                            : o == 1 ? dhv[j] * gg * sg
                                     : gg * sg * uu;
              const __nv_bfloat16 vb = __float2bfloat16_rn(v);
              asm volatile("st.shared.b16 [%0], %1;" ::"r"(stg_s + j * 64 + lane * 2),
                           "h"(*reinterpret_cast<const uint16_t*>(&vb)) : "memory");
            }
            __syncwarp();
            __nv_bfloat16* dst = o == 2 ? g.h_out : static_cast<__nv_bfloat16*>(g.out);
            const int64_t ld = o == 2 ? g.h_ld : g.out_ld;
            const int64_t cbase = col0 + (o == 1 ? g.N : 0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int idx = q * 32 + lane;
              const int j = idx >> 2, part = idx & 3;
              uint4 v;
              asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                           : "r"(stg_s + j * 64 + part * 16));
              if (col_ok)
                *reinterpret_cast<uint4*>(dst + (row0 + c * 32 + j) * ld + cbase + part * 8) = v;
            }
            __syncwarp();
          }
          continue;
        }
        tmem_wait_ld();
        constexpr int kOuts = (kMode == 1) ? 2 : 1;
#pragma unroll
        for (int a = 0; a < kOuts; ++a) {
          const int64_t col0 = (kMode == 1)
                                   ? wt * 4 * kWRows + a * 2 * kWRows + rank * kWRows + quad * 32
                                   : wt * 2 * kWRows + rank * kWRows + quad * 32;
          const bool col_ok = col0 < g.N;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float y;
            if (kMode == 0)
              y = silu_mul(__uint_as_float(v0[j]), __uint_as_float(v1[j]));
            else
              y = wj[j] * __uint_as_float(a == 0 ? v0[j] : v1[j]);
            const __nv_bfloat16 yb = __float2bfloat16_rn(y);
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(stg_s + j * 64 + lane * 2),
                         "h"(*reinterpret_cast<const uint16_t*>(&yb)) : "memory");
          }
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int idx = q * 32 + lane;
            const int j = idx >> 2, part = idx & 3;
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(stg_s + j * 64 + part * 16));
            const int32_t s_j = (kMode == 1 || kMode == 2) ? __shfl_sync(0xffffffffu, slot_r[i], j) : 0;
            if (!col_ok) continue;
            if ((kMode == 1 || kMode == 2) && s_j >= g.S) continue;
            const int64_t p = row0 + c * 32 + j;
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + p * g.out_ld + col0 + part * 8) = v;
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
      if (++buf == C::kBufs) { buf = 0; acc_phase ^= 1u; }
    }
  }

  pdl_launch_dependents();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while the other may still signal it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

template <int kMode, int kNmax>
cudaError_t launch_pair(const CUtensorMap& w0, const CUtensorMap& w1, const CUtensorMap& x,
                        const Args& g, int64_t max_items, int num_sms, cudaStream_t st) {
  using C = PairCfg<kMode, kNmax>;
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    rc = cudaFuncSetAttribute(gemm_ws_pair_kernel<kMode, kNmax>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::kSmem));
    if (rc != cudaSuccess) return rc;
    if (dev < 64) configured |= 1ull << dev;
  }
  int64_t pairs = max_items < num_sms / 2 ? max_items : num_sms / 2;
  if (pairs < 1) pairs = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_ws_pair_kernel<kMode, kNmax>, w0, w1, x, g);
}

}  // namespace

cudaError_t launch_gemm_ws_pair_bf16(int mode, int tile_max, const CUtensorMap& w0,
                                     const CUtensorMap& w1, const CUtensorMap& x, const WsGemm& p,
                                     int num_sms, cudaStream_t st, int* launches) {
  Args g;
  g.K = p.K;
  g.N = p.N;
  g.n_wt = p.n_wt;
  g.num_tiles = p.num_tiles;
  g.tile_row = p.tile_row;
  g.tile_rows = p.tile_rows;
  g.tile_expert = p.tile_expert;
  g.sorted = p.sorted;
  g.S = p.S;
  g.out = p.out;
  g.out_ld = p.out_ld;
  g.topk_w = p.topk_w;
  g.k = p.k;
  g.err = p.err;
  g.weights_evict_first = p.weights_evict_first;
  g.tok_box = p.tok_box;
  g.unit_w = p.unit_w;
  g.dh = static_cast<const __nv_bfloat16*>(p.dh);
  g.dh_ld = p.dh_ld;
  g.h_out = static_cast<__nv_bfloat16*>(p.h_out);
  g.h_ld = p.h_ld;
  if (mode == 3 && (!p.dh || !p.h_out)) return cudaErrorInvalidValue;
  if (launches) *launches += 1;
  const int64_t max_items = p.max_tiles * p.n_wt;
  if (tile_max == 256) {
    if (mode == 0) return launch_pair<0, 256>(w0, w1, x, g, max_items, num_sms, st);
    if (mode == 2) return launch_pair<2, 256>(w0, w1, x, g, max_items, num_sms, st);
    return launch_pair<1, 256>(w0, w1, x, g, max_items, num_sms, st);
  }
  if (tile_max == 128) {
    if (mode == 0) return launch_pair<0, 128>(w0, w1, x, g, max_items, num_sms, st);
    if (mode == 3) return launch_pair<3, 128>(w0, w1, x, g, max_items, num_sms, st);
    if (mode == 2) return launch_pair<2, 128>(w0, w1, x, g, max_items, num_sms, st);
    return launch_pair<1, 128>(w0, w1, x, g, max_items, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
