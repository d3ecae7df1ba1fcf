// Weight-stationary grouped expert GEMMs (bf16, tcgen05, sm_100a).
//
// The expert weights are the MMA's M side and a tile of one expert's token
// rows is the N side ("swap AB"), so a token tile needs no padding beyond the
// 32-row granule of align and each weight byte loaded into shared memory is
// reused by up to 128 tokens.
// Two weight tiles share every token tile:
//   GEMM1 (gate/up + SwiGLU): W0 = gate rows [128 w, 128 w + 128), W1 = the same
//       up rows of expert e (views of the packed w13, expert found from the real
//       stride(0): Liger-Kernel PR #1377, "Problems");
//       acc0 = W0 . X^T, acc1 = W1 . X^T (fp32, TMEM), h[token, i] = bf16(silu(acc0) * acc1)
//   GEMM2 (down + routing weight): W0, W1 = w2 rows [256 w, 256 w + 128) and
//       [256 w + 128, 256 w + 256); y[slot, o] = bf16(w_slot * acc[o, token])
//
// Kernel shape: one persistent CTA per SM, 6 warps.
//   warp 0    TMA producer: two weight boxes [128 x 64] + the token tile in
//             32-row boxes per k-step (128-byte swizzle, kStages ring)
//   warp 1    TMEM allocator, MMA issuer: per 16-wide k slice two
//             tcgen05.mma.cta_group::1.kind::f16, M=128, N=tile rows (32..128);
//             two accumulator buffers in TMEM, so the epilogue of one work
//             item overlaps the mainloop of the next
//   warps 2-5 epilogue: each thread owns one weight row of both accumulators;
//             32-token chunks are transposed through shared memory so global
//             stores are 16-byte vectors along the output row.
// Work item = (token tile, weight tile), token-tile major, so the CTAs running
// together share one token tile and the weight tiles of one expert in L2.
#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kWRows = 128;                  // rows per weight tile (MMA M)
constexpr int kBK = 64;                      // bf16 elements per 128-byte row
constexpr int kUmmaK = 16;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kStagingBytes = 32 * 64;       // per epilogue warp: 32 tokens x 32 bf16

// An accumulator buffer holds acc0 at [0, kNmax) and acc1 at [kNmax, 2 kNmax)
// columns; with kNmax <= 128 two buffers fit in TMEM, so the epilogue of one
// work item overlaps the mainloop of the next.
template <int kNmax, int kStages>
struct Cfg {
  static constexpr int kWBytes = kWRows * kBK * 2;                  // 16 KiB per weight tile
  static constexpr int kTokBytes = kNmax * kBK * 2;
  static constexpr int kStageBytes = 2 * kWBytes + kTokBytes;
  static constexpr int kBufCols = 2 * kNmax;
  static constexpr int kBufs = kTmemCols / kBufCols >= 2 ? 2 : 1;
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes +
                                  kEpiWarps * kStagingBytes + (3 * kStages + 2 * 2 + 1) * 8 + 16;
};

struct WsArgs {
  int64_t K;              // contraction length
  int64_t N;              // output columns (I for GEMM1, H for GEMM2)
  int64_t n_wt;           // weight tiles per token tile
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
  View2 pre_ids;     // GEMM1, at most 32 slots: routing ids (pre_S = 0: not used)
  int32_t pre_E, pre_S;
  DeviceErrors* err;
  int32_t unit_w;    // GEMM2: weight 1 for every routed slot
  const __nv_bfloat16* dh;  // mode 3: gradient of h [P, N], row stride dh_ld
  int64_t dh_ld;
  __nv_bfloat16* h_out;     // mode 3: recomputed h [P, N], row stride h_ld
  int64_t h_ld;
};

// Decode batches (at most 32 routing slots on 32-row tiles) have one tile per
// routed expert, in ascending expert order, so the expert of work item `item`
// follows from the routing ids alone.  Whole warp; returns -1 past the items.
__device__ __forceinline__ int first_expert_from_ids(const WsArgs& g, int64_t item, int lane) {
  int64_t id = -1;
  if (lane < g.pre_S) {
    const int64_t t = lane / g.k, j = lane - t * g.k;
    const int64_t off = t * g.pre_ids.s0 + j * g.pre_ids.s1;
    id = g.pre_ids.dtype == MOE_I64 ? static_cast<const int64_t*>(g.pre_ids.data)[off]
                                    : static_cast<const int32_t*>(g.pre_ids.data)[off];
  }
  const bool valid = id >= 0 && id < g.pre_E;
  const int key = valid ? static_cast<int>(id) : -1 - lane;  // invalid slots: distinct keys
  const unsigned same = __match_any_sync(0xffffffffu, key);
  const bool first = valid && (__ffs(same) - 1 == lane);
  const unsigned firsts = __ballot_sync(0xffffffffu, first);
  int rank = 0;  // routed experts below this lane's
  for (int j = 0; j < 32; ++j) {
    const int other = __shfl_sync(0xffffffffu, key, j);
    rank += (((firsts >> j) & 1u) != 0u && other < key) ? 1 : 0;
  }
  const int64_t tile = item / g.n_wt;
  if (tile >= __popc(firsts)) return -1;
  const unsigned who = __ballot_sync(0xffffffffu, first && rank == tile);
  return __shfl_sync(0xffffffffu, key, __ffs(who) - 1);
}

template <int kStages>
struct Smem {
  uint8_t* stages;
  uint8_t* staging;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* drain;
  uint64_t* pre;  // decode prefetch: the early weight copies of each stage land here
  uint32_t* tmem_slot;
};

template <int kNmax, int kStages>
__device__ __forceinline__ Smem<kStages> carve(uint8_t* raw) {
  using C = Cfg<kNmax, kStages>;
  Smem<kStages> s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.stages = base;
  s.staging = base + kStages * C::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.staging + kEpiWarps * kStagingBytes);
  s.full = bars;
  s.empty = bars + kStages;
  s.tfull = bars + 2 * kStages;
  s.tempty = s.tfull + 2;
  s.drain = s.tempty + 2;
  s.pre = s.drain + 1;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.pre + kStages);
  return s;
}

template <int kMode, int kNmax, int kStages>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_ws_bf16_kernel(const __grid_constant__ CUtensorMap tmW0,
                        const __grid_constant__ CUtensorMap tmW1,
                        const __grid_constant__ CUtensorMap tmX, const WsArgs g) {
  constexpr bool kG1 = kMode == 0 || kMode == 3;  // gate and up tiles (GEMM1 forms)
  using C = Cfg<kNmax, kStages>;
  extern __shared__ uint8_t smem_raw[];
  const Smem<kStages> sm = carve<kNmax, kStages>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW0);
    if (kG1) tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmX);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
      mbar_init(&sm.pre[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], kEpiWarps);
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

  const int num_k = static_cast<int>((g.K + kBK - 1) / kBK);
  // GEMM1 at decode sizes: request the first weight stages of this CTA's first
  // work item before waiting for align and permute.  The expert comes from the
  // routing ids read before the PDL wait, which may still be in flight from an
  // earlier kernel, so the copies land on their own `pre` barriers and the
  // producer checks the expert against align's tile list after the wait: on a
  // match the stages are used as they are (the token boxes follow on the
  // stages' full barriers), else the early copies are let land and the stages
  // are loaded again from the right expert.
  int npre = 0, pre_e = -1;
  if (kMode == 0 && kNmax == 32 && g.pre_S > 0 && warp == 0) {
    const int e = first_expert_from_ids(g, blockIdx.x, lane);
    if (e >= 0) {
      npre = num_k < kStages ? num_k : kStages;
      pre_e = e;
      if (lane == 0) {
        const int64_t wt = blockIdx.x % g.n_wt;
        const uint64_t wpol = g.weights_evict_first ? l2_policy_evict_first() : l2_policy_evict_last();
        for (int kb = 0; kb < npre; ++kb) {
          uint8_t* sw0 = sm.stages + kb * C::kStageBytes;
          mbar_arrive_expect_tx(&sm.pre[kb], 2 * C::kWBytes);
          tma_load_3d(sw0, &tmW0, &sm.pre[kb], kb * kBK, static_cast<int32_t>(wt * kWRows), e, wpol);
          tma_load_3d(sw0 + C::kWBytes, &tmW1, &sm.pre[kb], kb * kBK, static_cast<int32_t>(wt * kWRows), e, wpol);
        }
      }
    }
  }
  pdl_wait();
  const int64_t total = static_cast<int64_t>(*g.num_tiles) * g.n_wt;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      uint32_t stage = 0, phase = 0;
      int8_t last_phase[kStages];
      for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
      const uint64_t pol = l2_policy_evict_last();
      const uint64_t wpol = g.weights_evict_first ? l2_policy_evict_first() : pol;
      bool ok = true, pre_waited = false;
      for (int64_t item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const int64_t t = item / g.n_wt, wt = item - t * g.n_wt;
        const int32_t e = g.tile_expert[t], row0 = g.tile_row[t], rows = g.tile_rows[t];
        const int32_t w0 = static_cast<int32_t>(kG1 ? wt * kWRows : wt * 2 * kWRows);
        const int32_t w1 = kG1 ? w0 : w0 + kWRows;
        // whole boxes: a box may run past the tile (rows the MMA's N excludes)
        const int nbox = (rows + g.tok_box - 1) / g.tok_box;
        const uint32_t tok_bytes = nbox * g.tok_box * kBK * 2;
        const uint32_t bytes = 2 * C::kWBytes + tok_bytes;
        // the early weight copies are this item's only if align agrees on the expert
        const int use_pre = (item == blockIdx.x && npre > 0 && e == pre_e) ? npre : 0;
        if (item == blockIdx.x && npre > 0 && !use_pre) {
          for (int kb = 0; kb < npre; ++kb) mbar_wait(&sm.pre[kb], 0, g.err);
          pre_waited = true;
        }
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
          uint8_t* sw0 = sm.stages + stage * C::kStageBytes;
          uint8_t* sw1 = sw0 + C::kWBytes;
          uint8_t* sx = sw1 + C::kWBytes;
          if (kb < use_pre) {
            // weights requested before the PDL wait: the token boxes join the
            // stage now; the stage's arrival waits until the weights have landed
            mbar_expect_tx(&sm.full[stage], tok_bytes);
          } else {
            mbar_arrive_expect_tx(&sm.full[stage], bytes);
            tma_load_3d(sw0, &tmW0, &sm.full[stage], kb * kBK, w0, e, wpol);
            tma_load_3d(sw1, kG1 ? &tmW1 : &tmW0, &sm.full[stage], kb * kBK, w1, e, wpol);
          }
          for (int b = 0; b < nbox; ++b)
            tma_load_2d(sx + b * g.tok_box * kBK * 2, &tmX, &sm.full[stage], kb * kBK,
                        row0 + b * g.tok_box, pol);
          if (kb + 1 == use_pre) {
            for (int j = 0; j < use_pre; ++j) {
              mbar_wait(&sm.pre[j], 0, g.err);
              mbar_arrive(&sm.full[j]);
            }
            pre_waited = true;
          }
          last_phase[stage] = static_cast<int8_t>(phase);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (last_phase[s] >= 0) mbar_wait(&sm.full[s], static_cast<uint32_t>(last_phase[s]), g.err);
      }
      if (npre > 0 && !pre_waited) {
        // early copies nobody consumed (no item for this CTA, or a wait gave up
        // first): let them land before the CTA exits
        for (int kb = 0; kb < npre; ++kb) mbar_wait(&sm.pre[kb], 0, g.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      uint32_t stage = 0, phase = 0, buf = 0, acc_phase = 0;
      bool ok = true, issued = false;
      for (int64_t item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const int64_t t = item / g.n_wt;
        const int32_t rows = g.tile_rows[t];
        const uint32_t idesc = idesc_bf16_f32(kWRows, rows);
        if (!mbar_wait(&sm.tempty[buf], acc_phase ^ 1u, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc0 = tmem_base + buf * C::kBufCols, acc1 = acc0 + kNmax;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t w0_addr = smem_u32(sm.stages + stage * C::kStageBytes);
          const uint32_t w1_addr = w0_addr + C::kWBytes;
          const uint32_t x_addr = w1_addr + C::kWBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint64_t xd = sw128_kmajor_desc(x_addr + kk * kUmmaK * 2);
            const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
            mma_bf16(acc0, sw128_kmajor_desc(w0_addr + kk * kUmmaK * 2), xd, idesc, acc);
            mma_bf16(acc1, sw128_kmajor_desc(w1_addr + kk * kUmmaK * 2), xd, idesc, acc);
          }
          issued = true;
          mma_commit(&sm.empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&sm.tfull[buf]);
        if (++buf == C::kBufs) { buf = 0; acc_phase ^= 1u; }
      }
      if (!ok && issued) {
        mma_commit(sm.drain);
        mbar_wait(sm.drain, 0, g.err);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32) = weight rows of this warp
    uint8_t* stg = sm.staging + (warp - 2) * kStagingBytes;
    const uint32_t stg_s = smem_u32(stg);
    uint32_t buf = 0, acc_phase = 0;
    for (int64_t item = blockIdx.x; item < total; item += gridDim.x) {
      const int64_t t = item / g.n_wt, wt = item - t * g.n_wt;
      const int32_t row0 = g.tile_row[t], rows = g.tile_rows[t];
      // GEMM2: slots and routing weights of the tile's tokens (lane j of chunk c
      // holds token c*32 + j), fetched while the accumulator is still being built
      int32_t slot_r[kNmax / 32];
      float w_r[kNmax / 32];
      if (kMode == 1) {
#pragma unroll
        for (int c = 0; c < kNmax / 32; ++c)
          slot_r[c] = (c * 32 < rows) ? g.sorted[row0 + c * 32 + lane] : static_cast<int32_t>(g.S);
#pragma unroll
        for (int c = 0; c < kNmax / 32; ++c) {
          w_r[c] = 0.0f;
          if (slot_r[c] < g.S) {
            const int64_t tt = slot_r[c] / g.k, jj = slot_r[c] - tt * g.k;
            w_r[c] = g.unit_w ? 1.0f
                              : static_cast<const float*>(g.topk_w.data)[tt * g.topk_w.s0 + jj * g.topk_w.s1];
          }
        }
      }
      if (!mbar_wait(&sm.tfull[buf], acc_phase, g.err)) break;
      tc_fence_after();
      const uint32_t lane_base = (static_cast<uint32_t>(quad * 32) << 16) + buf * C::kBufCols;
      constexpr int kAccs = kG1 ? 1 : 2;  // GEMM1 combines both into one output
#pragma unroll 1
      for (int a = 0; a < kAccs; ++a) {
        // output column (weight row) block of this warp
        const int64_t col0 = kG1 ? wt * kWRows + quad * 32 : wt * 2 * kWRows + a * kWRows + quad * 32;
        const bool col_ok = col0 < g.N;
#pragma unroll
        for (int c = 0; c < kNmax / 32; ++c) {
          if (c * 32 >= rows) break;
          const int32_t my_slot = (kMode == 1) ? slot_r[c] : 0;
          const float my_w = (kMode == 1) ? w_r[c] : 0.0f;
          uint32_t v0[32];
          tmem_ld32(tmem_base + lane_base + a * kNmax + c * 32, v0);
          if (kMode == 3) {
            // gradient of h = silu(g) u for this warp's 32 rows of I and the chunk's
            // 32 token rows: dg, du and h go out through the staging tile in turn
            uint32_t v1[32];
            tmem_ld32(tmem_base + lane_base + kNmax + c * 32, v1);
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
          if (kMode == 0) {
            uint32_t v1[32];
            tmem_ld32(tmem_base + lane_base + kNmax + c * 32, v1);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float h = silu_mul(__uint_as_float(v0[j]), __uint_as_float(v1[j]));
              const __nv_bfloat16 hb = __float2bfloat16_rn(h);
              asm volatile("st.shared.b16 [%0], %1;" ::"r"(stg_s + j * 64 + lane * 2),
                           "h"(*reinterpret_cast<const uint16_t*>(&hb)) : "memory");
            }
          } else {
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float y = __shfl_sync(0xffffffffu, my_w, j) * __uint_as_float(v0[j]);
              const __nv_bfloat16 yb = __float2bfloat16_rn(y);
              asm volatile("st.shared.b16 [%0], %1;" ::"r"(stg_s + j * 64 + lane * 2),
                           "h"(*reinterpret_cast<const uint16_t*>(&yb)) : "memory");
            }
          }
          __syncwarp();
          // 32 tokens x 64 bytes: four lanes per token row, 16-byte stores
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int idx = q * 32 + lane;
            const int j = idx >> 2, part = idx & 3;
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(stg_s + j * 64 + part * 16));
            const int32_t s_j = (kMode == 1) ? __shfl_sync(0xffffffffu, my_slot, j) : 0;
            if (!col_ok) continue;
            if (kMode == 0) {
              const int64_t p = row0 + c * 32 + j;
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + p * g.out_ld + col0 + part * 8) = v;
            } else {
              if (s_j < g.S)
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + (row0 + c * 32 + j) * g.out_ld + col0 + part * 8) = v;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.tempty[buf]);
      if (++buf == C::kBufs) { buf = 0; acc_phase ^= 1u; }
    }
  }

  pdl_launch_dependents();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int kMode, int kNmax, int kStages>
cudaError_t launch_ws(const CUtensorMap& w0, const CUtensorMap& w1, const CUtensorMap& x,
                      const WsArgs& g, int64_t max_items, int num_sms, cudaStream_t st) {
  using C = Cfg<kNmax, kStages>;
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    rc = cudaFuncSetAttribute(gemm_ws_bf16_kernel<kMode, kNmax, kStages>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(C::kSmem));
    if (rc != cudaSuccess) return rc;
    if (dev < 64) configured |= 1ull << dev;
  }
  int64_t grid = max_items < num_sms ? max_items : num_sms;
  if (grid < 1) grid = 1;
  return launch_pdl(gemm_ws_bf16_kernel<kMode, kNmax, kStages>, dim3(static_cast<unsigned>(grid)),
                    dim3(kThreads), C::kSmem, st, w0, w1, x, g);
}

}  // namespace

cudaError_t launch_gemm_ws_bf16(int mode, int tile_max, const CUtensorMap& w0,
                                const CUtensorMap& w1, const CUtensorMap& x, const WsGemm& p,
                                int num_sms, cudaStream_t st, int* launches) {
  WsArgs g;
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
  g.pre_ids = p.pre_ids;
  g.pre_E = p.pre_E;
  g.pre_S = (mode == 0 && tile_max == 32 && p.pre_S <= 32) ? p.pre_S : 0;
  g.unit_w = p.unit_w;
  g.dh = static_cast<const __nv_bfloat16*>(p.dh);
  g.dh_ld = p.dh_ld;
  g.h_out = static_cast<__nv_bfloat16*>(p.h_out);
  g.h_ld = p.h_ld;
  if (mode == 3 && (!p.dh || !p.h_out)) return cudaErrorInvalidValue;
  if (launches) *launches += 1;
  const int64_t max_items = p.max_tiles * p.n_wt;
  if (tile_max == 128) {
    if (mode == 0) return launch_ws<0, 128, 4>(w0, w1, x, g, max_items, num_sms, st);
    if (mode == 3) return launch_ws<3, 128, 4>(w0, w1, x, g, max_items, num_sms, st);
    return launch_ws<1, 128, 4>(w0, w1, x, g, max_items, num_sms, st);
  }
  if (tile_max == 32) {
    if (mode == 0) return launch_ws<0, 32, 6>(w0, w1, x, g, max_items, num_sms, st);
    return launch_ws<1, 32, 6>(w0, w1, x, g, max_items, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
