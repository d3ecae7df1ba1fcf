// GEMM1 (gate/up + SwiGLU) on CTA pairs with gate and up rows interleaved
// along M, for token tiles of up to 256 or 512 rows.
//
// The weight-stationary pair GEMM1 (moe_gemm_ws2.cu) keeps gate and up in two
// accumulators of N columns each, so a token tile holds at most 256 rows (the
// 512 TMEM columns) and an expert with more padded rows than that streams its
// gate/up weights once per tile.  Here one weight tile of the pair is 128 rows
// of I: each CTA stages 64 gate rows and the same 64 up rows as one 128-row A
// operand, so gate and up land in one accumulator (TMEM lanes 0-63 gate, 64-127
// up) of N columns.  With 512-row tiles N can reach 512 (two MMAs of up to 256
// columns per k-step; one accumulator buffer): every expert whose padded rows
// fit in 512 is one token tile and its weights are read from HBM once.  With
// 256-row tiles two accumulator buffers fit, so the epilogue of one item runs
// under the next item's MMAs, and each item moves less through shared memory
// per FLOP than the two-accumulator kernel's 128-row tiles (half the weight
// rows, twice the tokens).  The results are those of the
// two-accumulator kernel bit for bit: every output is the same fp32 dot
// product over k in the same k order, then SwiGLU and one bf16 rounding.
//
//   weight tile wt: I rows [128 wt, 128 wt + 128); CTA r stages gate rows
//       128 wt + 64 r + [0, 64) as A rows 0-63 and the same up rows as A rows
//       64-127 (two 64-row TMA boxes, one 16 KiB operand);
//   token tile: rows [row0, row0 + rows), rows <= 512 in 32-row granules, as
//       MMA chunks of up to 256 columns; chunk c holds rows 256 c + [0, n_c),
//       the first n_c / 2 of them in CTA 0's shared memory, the rest in CTA 1's;
//   epilogue: warps of lane quadrants 0/1 (gate) and 2/3 (up) pair up; for
//       every 32 columns each warp hands the partner the half of its values the
//       partner finishes (16 columns, fp32, through shared memory; double
//       buffered, one mbarrier per warp pair, bounded waits), then each writes
//       h = bf16(silu(gate) * up) for its 16 tokens.
//
// Pair protocol as in moe_gemm_ws2.cu: both producers load their halves with
// cta_group::2 TMA completing on the leader's barrier, the leader issues the
// M = 256 MMAs and commits to both CTAs.  No TMA multicast.
#include "../../include/moe.h"
#include "moe_internal.h"
#include "moe_pair.cuh"

namespace moe {
namespace {

constexpr int kBK = 64;
constexpr int kUmmaK = 16;
constexpr int kHalf = 64;                        // gate (and up) rows per CTA per weight tile
constexpr int kTileI = 2 * kHalf;                // rows of I per pair weight tile
constexpr int kPairM = 2 * kTileI;               // MMA M over the pair: 128 A rows per CTA
constexpr int kChunkN = 256;                     // token columns per MMA
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kTmemCols = 512;
constexpr int kWBytes = 2 * kHalf * kBK * 2;     // 16 KiB: 64 gate rows, then 64 up rows
constexpr int kXChunkBytes = (kChunkN / 2) * kBK * 2;  // 16 KiB: 128 token rows of one chunk
constexpr int kXchgFloats = 16 * 32;             // 16 token columns x 32 lanes
constexpr int kXchgBytes = 2 * kXchgFloats * 4;  // double buffered, per epilogue warp

// kNmax token rows per tile: 512 (two MMA chunks, one accumulator buffer, 4
// stages) or 256 (one chunk, two buffers, 6 stages).
template <int kNmax>
struct IlCfg {
  static constexpr int kChunks = kNmax / kChunkN;
  static constexpr int kStageBytes = kWBytes + kChunks * kXChunkBytes;
  static constexpr int kStages = kChunks == 2 ? 4 : 6;
  static constexpr int kBufs = kChunks == 2 ? 1 : 2;
  static constexpr int kNumBars = 2 * kStages + 2 * kBufs + 1 + 4;  // full, empty, tfull, tempty, drain, exchange
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes + size_t(kEpiWarps) * kXchgBytes +
                                  kNumBars * 8 + 16;
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static_assert(kBufs * kNmax <= kTmemCols, "TMEM");
};

struct IlArgs {
  int64_t K, N, n_wt;
  const int32_t* num_tiles;
  const int32_t* tile_row;
  const int32_t* tile_rows;
  const int32_t* tile_expert;
  __nv_bfloat16* out;  // h [P, I]
  int64_t out_ld;
  int32_t weights_evict_first;
  int32_t tok_box;     // token rows per TMA box of the x map (divides 128)
  DeviceErrors* err;
};

template <int kNmax>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_il_pair_kernel(const __grid_constant__ CUtensorMap tmGate,
                        const __grid_constant__ CUtensorMap tmUp,
                        const __grid_constant__ CUtensorMap tmX, const IlArgs g) {
  using C = IlCfg<kNmax>;
  constexpr int kStages = C::kStages;
  constexpr int kStageBytes = C::kStageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  float* xchg = reinterpret_cast<float*>(base + kStages * kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * kStageBytes + kEpiWarps * kXchgBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;      // [kBufs]
  uint64_t* tempty = tfull + C::kBufs;    // [kBufs]
  uint64_t* drain = tempty + C::kBufs;
  uint64_t* xbar = drain + 1;  // [4]: one per gate/up warp pair
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = (rank == 0);

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmGate);
    tma_prefetch_desc(&tmUp);
    tma_prefetch_desc(&tmX);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kBufs; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&xbar[i], 2);
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
        const int32_t wrow = static_cast<int32_t>(wt * kTileI + rank * kHalf);
        int32_t n_c[2], my0[2], nbox[2];
        n_c[0] = rows < kChunkN ? rows : kChunkN;
        n_c[1] = C::kChunks == 2 ? rows - n_c[0] : 0;
        uint32_t x_bytes = 0;
        for (int c = 0; c < 2; ++c) {
          my0[c] = row0 + c * kChunkN + static_cast<int32_t>(rank) * (n_c[c] / 2);
          nbox[c] = n_c[c] > 0 ? (n_c[c] / 2 + g.tok_box - 1) / g.tok_box : 0;
          x_bytes += static_cast<uint32_t>(nbox[c] * g.tok_box * kBK * 2);
        }
        const uint32_t bytes_pair = 2 * (kWBytes + x_bytes);
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
          uint8_t* sw = stages + stage * kStageBytes;
          uint8_t* sx = sw + kWBytes;
          if (leader) mbar_arrive_expect_tx(&full[stage], bytes_pair);
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          tma_load_3d_pair(sw, &tmGate, fb, kb * kBK, wrow, e, wpol);
          tma_load_3d_pair(sw + kWBytes / 2, &tmUp, fb, kb * kBK, wrow, e, wpol);
          for (int c = 0; c < C::kChunks; ++c)
            for (int b = 0; b < nbox[c]; ++b)
              tma_load_2d_pair(sx + c * kXChunkBytes + b * g.tok_box * kBK * 2, &tmX, fb, kb * kBK,
                               my0[c] + b * g.tok_box, pol);
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
        const int32_t n0 = rows < kChunkN ? rows : kChunkN;
        const int32_t n1 = C::kChunks == 2 ? rows - n0 : 0;
        const uint32_t idesc0 = idesc_bf16_f32(kPairM, n0);
        const uint32_t idesc1 = idesc_bf16_f32(kPairM, n1 > 0 ? n1 : 16);
        if (!mbar_wait(&tempty[buf], acc_phase ^ 1u, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc = tmem_base + buf * kChunkN;  // two buffers: columns [0, 256) and [256, 512)
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&full[stage], phase, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t w_addr = smem_u32(stages + stage * kStageBytes);
          const uint32_t x_addr = w_addr + kWBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint64_t wd = sw128_kmajor_desc(w_addr + kk * kUmmaK * 2);
            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
            mma_bf16_pair(acc, wd, sw128_kmajor_desc(x_addr + kk * kUmmaK * 2), idesc0, accum);
            if (n1 > 0)
              mma_bf16_pair(acc + kChunkN, wd,
                            sw128_kmajor_desc(x_addr + kXChunkBytes + kk * kUmmaK * 2), idesc1, accum);
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
    const bool gate_side = quad < 2;
    const int partner = gate_side ? warp - 2 : warp + 2;  // the warp with the other lanes of these rows
    uint64_t* xb = &xbar[(quad & 1) + 2 * half];
    float* mine = xchg + (warp - 2) * (2 * kXchgFloats);
    const float* theirs = xchg + (partner - 2) * (2 * kXchgFloats);
    const uint32_t lane_quad = static_cast<uint32_t>(quad * 32) << 16;
    // the gate warp finishes columns 0-15 of every 32 and hands over 16-31, the
    // up warp the other way round (register indices stay compile-time constants)
    const int keep0 = gate_side ? 0 : 16;
    uint32_t buf = 0, acc_phase = 0, x_count = 0;
    for (int64_t item = pair; item < total; item += n_pairs) {
      const int64_t t = item / g.n_wt, wt = item - t * g.n_wt;
      const int32_t row0 = g.tile_row[t], rows = g.tile_rows[t];
      const int64_t col = wt * kTileI + rank * kHalf + (quad & 1) * 32 + lane;
      const bool col_ok = col < g.N;
      if (!mbar_wait(&tfull[buf], acc_phase, g.err)) break;
      tc_fence_after();
      bool ok = true;
      for (int cc = half * 32; cc < rows; cc += 64) {
        uint32_t v[32];
        tmem_ld32(tmem_base + lane_quad + buf * kChunkN + static_cast<uint32_t>(cc), v);
        tmem_wait_ld();
        float* mb = mine + (x_count & 1u) * kXchgFloats;
        float keep[16];
        if (gate_side) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            mb[j * 32 + lane] = __uint_as_float(v[16 + j]);
            keep[j] = __uint_as_float(v[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            mb[j * 32 + lane] = __uint_as_float(v[j]);
            keep[j] = __uint_as_float(v[16 + j]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(xb);
        if (!mbar_wait(xb, x_count & 1u, g.err)) { ok = false; break; }
        const float* tb = theirs + (x_count & 1u) * kXchgFloats;
        ++x_count;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float other = tb[j * 32 + lane];
          const float hv = gate_side ? silu_mul(keep[j], other) : silu_mul(other, keep[j]);
          const int64_t p = row0 + cc + keep0 + j;
          if (col_ok) g.out[p * g.out_ld + col] = __float2bfloat16_rn(hv);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
      if (++buf == C::kBufs) { buf = 0; acc_phase ^= 1u; }
      if (!ok) break;
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

template <int kNmax>
cudaError_t launch_il(const CUtensorMap& gate64, const CUtensorMap& up64, const CUtensorMap& x,
                      const IlArgs& g, int64_t max_items, int num_sms, cudaStream_t st) {
  using C = IlCfg<kNmax>;
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    rc = cudaFuncSetAttribute(gemm_il_pair_kernel<kNmax>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(C::kSmem));
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
  return cudaLaunchKernelEx(&cfg, gemm_il_pair_kernel<kNmax>, gate64, up64, x, g);
}

}  // namespace

cudaError_t launch_gemm_il_pair_bf16(int tile_max, const CUtensorMap& gate64, const CUtensorMap& up64,
                                    const CUtensorMap& x, const WsGemm& p, int num_sms,
                                    cudaStream_t st, int* launches) {
  if (p.tok_box <= 0 || 128 % p.tok_box != 0) return cudaErrorInvalidValue;
  IlArgs g;
  g.K = p.K;
  g.N = p.N;
  g.n_wt = p.n_wt;
  g.num_tiles = p.num_tiles;
  g.tile_row = p.tile_row;
  g.tile_rows = p.tile_rows;
  g.tile_expert = p.tile_expert;
  g.out = static_cast<__nv_bfloat16*>(p.out);
  g.out_ld = p.out_ld;
  g.weights_evict_first = p.weights_evict_first;
  g.tok_box = p.tok_box;
  g.err = p.err;
  const int64_t max_items = p.max_tiles * p.n_wt;
  if (launches) *launches += 1;
  if (tile_max == 512) return launch_il<512>(gate64, up64, x, g, max_items, num_sms, st);
  if (tile_max == 256) return launch_il<256>(gate64, up64, x, g, max_items, num_sms, st);
  return cudaErrorInvalidValue;
}

}  // namespace moe
