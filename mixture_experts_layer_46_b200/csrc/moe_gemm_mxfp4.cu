// Weight-stationary block-scaled MXFP4 grouped expert GEMMs
// (tcgen05.mma kind::mxf4.block_scale, sm_100a).
//
// Operands are packed e2m1 codes (two per byte) with one e8m0 scale per 32
// consecutive elements of the contraction axis (aiter PR #3859, "Details":
// float4_e2m1fn_x2 weights and activations, QuantType.per_1x32).  As in the
// bf16 kernels the weights are the MMA's M side (two 128-row tiles per work
// item) and one expert's token tile (up to 32 or 96 rows) is the N side:
//   GEMM1: acc0 = gate_tile . X^T, acc1 = up_tile . X^T (fp32 in TMEM);
//          h = silu(acc0) * acc1, requantised per 1x32 along I -> codes [P, I/2], scales [P, I/32]
//   GEMM2: acc0/acc1 = two 128-row w2 slices . H^T; y[slot, o] = bf16(w_slot * acc)
// Expert addressing: 3-D TMA maps whose expert stride is each view's real
// stride(0) (Liger-Kernel PR #1377, "Problems").
//
// Kernel shape: one persistent CTA per SM, 11 warps.
//   warp 0    TMA producer: two weight boxes [128 rows x 128 B] + the token tile
//             in 32-row boxes per k-step (256 elements of K), 128-byte swizzle
//   warp 1    TMEM allocator, MMA issuer: per stage copies the stage's scales
//             from shared memory to TMEM (tcgen05.cp 32x128b.warpx4) and issues
//             2 x 4 x tcgen05.mma.kind::mxf4.block_scale (M=128, N=tile, K=64)
//   warp 2    scale producer: puts the stage's e8m0 scales into the 128-row x
//             4-block atom the tensor core reads: byte (row % 32) * 16 +
//             (row / 32) * 4 + block.  Where the scale views are 16-byte aligned
//             the TMA producer also loads the raw scale rows of every pair of
//             k-blocks ([rows x 16 bytes], in the same stream as the codes) and
//             this warp only moves their words into the atoms; otherwise it
//             copies them through their strides with 4-byte cp.async.
//   warps 3-10 epilogue: two warps per 32-lane TMEM quadrant (one weight row
//             per thread), each taking every other 32-token chunk
// TMEM: kBufs accumulator buffers of 2 x kNmax columns, then 24 scale columns
// per stage (two weight tiles and the token tile, each 2 atoms x 4 columns).
#include "../../include/moe.h"
#include "moe_internal.h"
#include "moe_mx.cuh"

namespace moe {
namespace {

constexpr int kWRows = 128;
constexpr int kRowBytes = 128;                 // packed bytes per row per stage (256 elements)
constexpr int kTokBox = 32;
constexpr int kUmmaKBytes = 32;                // 64 e2m1 elements per instruction
constexpr int kAtomBytes = 512;                // 128 rows x 4 scale blocks
constexpr int kSfBytes = 2 * kAtomBytes;       // 8 blocks of 32 per stage
constexpr int kEpiWarps = 8;                   // two per TMEM lane quadrant, alternating chunks
constexpr int kSfWarps = 1;                    // scale producer warps
constexpr int kFirstEpiWarp = 2 + kSfWarps;
constexpr int kStagingTile = 32 * 64;                 // a 32 x 32 bf16 tile (or 32 x 32 codes)
constexpr int kStagingBytes = kStagingTile + 32 * 4;  // + the chunk's 32 routing weights (GEMM2)
constexpr int kSfColsPerStage = 24;
constexpr int kSfRing = 3;                     // raw scale slots (pairs of k-blocks), TMA path
constexpr int kTmemCols = 512;
constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);

__device__ __forceinline__ void st_shared_v4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

template <int kNmax, int kStages>
struct Cfg {
  static constexpr int kWBytes = kWRows * kRowBytes;                 // 16 KiB
  static constexpr int kTokBytes = kNmax * kRowBytes;
  // [W0][W1][X][SF W0][SF W1][SF X]; 1024-byte aligned stage size
  static constexpr int kRaw = 2 * kWBytes + kTokBytes + 3 * kSfBytes;
  static constexpr int kStageBytes = (kRaw + 1023) / 1024 * 1024;
  static constexpr int kBufCols = 2 * kNmax;
  static constexpr int kBufs = (2 * kBufCols + kStages * kSfColsPerStage <= kTmemCols) ? 2 : 1;
  static constexpr int kSfCol0 = kBufs * kBufCols;
  static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");
  // raw scale slot (TMA path): 16 bytes (two k-blocks) for each row of W0, W1 and the token tile
  static constexpr int kSfRawBytes = (2 * kWRows + kNmax) * 16;
  static constexpr uint32_t kSfRawTx = static_cast<uint32_t>(kSfRawBytes);
  static constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes + kEpiWarps * kStagingBytes +
                                  size_t(kSfRing) * kSfRawBytes + (2 * kStages + 2 * kSfRing + 5) * 8 + 16;
  static_assert(kSmem <= 232448, "shared memory per block");
  static_assert(kSfRawBytes % 128 == 0, "TMA destinations stay 128-byte aligned");
};

struct MxArgs {
  int64_t K, N, n_wt;
  const int32_t* num_tiles;
  const int32_t* tile_row;
  const int32_t* tile_rows;
  const int32_t* tile_expert;
  const int32_t* sorted;
  int64_t S;
  void* out;             // GEMM1: h codes [P, I/2]; GEMM2: y [S, H] bf16
  int64_t out_ld;        // bytes (codes) or elements (y)
  uint8_t* out_sf;       // GEMM1: h scales [P, I/32]
  int64_t out_sf_ld;
  View2 topk_w;
  int64_t k;
  const uint8_t* x_sf;   // token scales [P, K/32]
  int64_t x_sf_ld;
  const uint8_t* w0_sf;  // weight scales [E, rows, K/32] (byte strides)
  int64_t w0_s0, w0_s1;
  const uint8_t* w1_sf;
  int64_t w1_s0, w1_s1;
  const float* w_row;    // GEMM2: routing weight per grouped row (valid rows)
  float* h_capture;      // GEMM1, inspection only: fp32 h before quantisation [P, N] (or null)
  DeviceErrors* err;
};

struct Smem {
  uint8_t* stages;
  uint8_t* staging;
  uint8_t* sf_raw;
  uint64_t* raw_full;
  uint64_t* raw_empty;
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  uint64_t* drain;
  uint32_t* tmem_slot;
};

template <int kNmax, int kStages>
__device__ __forceinline__ Smem carve(uint8_t* raw) {
  using C = Cfg<kNmax, kStages>;
  Smem s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.stages = base;
  s.staging = base + kStages * C::kStageBytes;
  s.sf_raw = s.staging + kEpiWarps * kStagingBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.sf_raw + kSfRing * C::kSfRawBytes);
  s.raw_full = bars;
  s.raw_empty = bars + kSfRing;
  bars += 2 * kSfRing;
  s.full = bars;
  s.empty = bars + kStages;
  s.tfull = bars + 2 * kStages;
  s.tempty = s.tfull + 2;
  s.drain = s.tempty + 2;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.drain + 1);
  return s;
}

template <int kMode, int kNmax, int kStages, bool kTmaSf>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_ws_mxfp4_kernel(const __grid_constant__ CUtensorMap tmW0,
                         const __grid_constant__ CUtensorMap tmW1,
                         const __grid_constant__ CUtensorMap tmX,
                         const __grid_constant__ CUtensorMap tmSf0,
                         const __grid_constant__ CUtensorMap tmSf1,
                         const __grid_constant__ CUtensorMap tmSfX, const MxArgs g) {
  using C = Cfg<kNmax, kStages>;
  extern __shared__ uint8_t smem_raw[];
  const Smem sm = carve<kNmax, kStages>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW0);
    if (kMode == 0) tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmX);
    if (kTmaSf) {
      tma_prefetch_desc(&tmSf0);
      if (kMode == 0) tma_prefetch_desc(&tmSf1);
      tma_prefetch_desc(&tmSfX);
      for (int r = 0; r < kSfRing; ++r) {
        mbar_init(&sm.raw_full[r], 1);    // the TMA producer (with bytes)
        mbar_init(&sm.raw_empty[r], 32);  // every lane of the scale producer
      }
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1 + 32);  // TMA producer (with bytes) + 32 scale-producer lanes
      mbar_init(&sm.empty[s], 1);
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

  pdl_wait();
  const int64_t total = static_cast<int64_t>(*g.num_tiles) * g.n_wt;
  const int num_k = static_cast<int>(g.K / 256);  // K % 256 == 0 (validated)

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      uint32_t stage = 0, phase = 0, rslot = 0, rphase = 0;
      int8_t last_phase[kStages], last_rphase[kSfRing];
      for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
      for (int r = 0; r < kSfRing; ++r) last_rphase[r] = -1;
      const uint64_t pol = l2_policy_evict_last();
      bool ok = true;
      for (int64_t item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const int64_t t = item / g.n_wt, wt = item - t * g.n_wt;
        const int32_t e = g.tile_expert[t], row0 = g.tile_row[t], rows = g.tile_rows[t];
        const int32_t w0 = static_cast<int32_t>(kMode == 0 ? wt * kWRows : wt * 2 * kWRows);
        const int32_t w1 = kMode == 0 ? w0 : w0 + kWRows;
        const int nbox = rows / kTokBox;
        const uint32_t bytes = 2 * C::kWBytes + nbox * kTokBox * kRowBytes;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
          uint8_t* sw0 = sm.stages + stage * C::kStageBytes;
          uint8_t* sw1 = sw0 + C::kWBytes;
          uint8_t* sx = sw1 + C::kWBytes;
          if (kTmaSf && (kb & 1) == 0) {
            // raw scale rows of k-blocks kb and kb + 1: [W0 128 x 16 B][W1 128 x 16 B][X kNmax x 16 B];
            // rows past the weight matrix or the token rows read as zeros
            if (!mbar_wait(&sm.raw_empty[rslot], rphase ^ 1u, g.err)) { ok = false; break; }
            uint8_t* raw = sm.sf_raw + rslot * C::kSfRawBytes;
            mbar_arrive_expect_tx(&sm.raw_full[rslot], C::kSfRawTx);
            tma_load_3d(raw, &tmSf0, &sm.raw_full[rslot], kb * 8, w0, e, pol);
            tma_load_3d(raw + kWRows * 16, kMode == 0 ? &tmSf1 : &tmSf0, &sm.raw_full[rslot], kb * 8, w1, e, pol);
            tma_load_2d(raw + 2 * kWRows * 16, &tmSfX, &sm.raw_full[rslot], kb * 8, row0, pol);
            last_rphase[rslot] = static_cast<int8_t>(rphase);
            if (++rslot == kSfRing) { rslot = 0; rphase ^= 1u; }
          }
          mbar_arrive_expect_tx(&sm.full[stage], bytes);
          tma_load_3d(sw0, &tmW0, &sm.full[stage], kb * kRowBytes, w0, e, pol);
          tma_load_3d(sw1, kMode == 0 ? &tmW1 : &tmW0, &sm.full[stage], kb * kRowBytes, w1, e, pol);
          for (int b = 0; b < nbox; ++b)
            tma_load_2d(sx + b * kTokBox * kRowBytes, &tmX, &sm.full[stage], kb * kRowBytes,
                        row0 + b * kTokBox, pol);
          last_phase[stage] = static_cast<int8_t>(phase);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (last_phase[s] >= 0) mbar_wait(&sm.full[s], static_cast<uint32_t>(last_phase[s]), g.err);
        for (int r = 0; r < kSfRing; ++r)
          if (last_rphase[r] >= 0) mbar_wait(&sm.raw_full[r], static_cast<uint32_t>(last_rphase[r]), g.err);
      }
    }
  } else if (kTmaSf && warp >= 2 && warp < kFirstEpiWarp) {
    // ------------------------------------------------------------ scale producer (TMA path)
    // Lane l moves the words of rows l, l+32, l+64 and l+96: an atom row is the
    // words of four rows 32 apart, so each atom takes one 16-byte shared store
    // per lane.  Token rows past the tile get zero scales.
    uint32_t stage = 0, phase = 0, rslot = 0, rphase = 0;
    bool ok = true;
    for (int64_t item = blockIdx.x; item < total && ok; item += gridDim.x) {
      const int64_t t = item / g.n_wt;
      const int32_t rows = g.tile_rows[t];
      for (int kb = 0; kb < num_k; ++kb) {
        if ((kb & 1) == 0 && !mbar_wait(&sm.raw_full[rslot], rphase, g.err)) { ok = false; break; }
        if (!mbar_wait(&sm.empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
        const uint32_t raw = smem_u32(sm.sf_raw + rslot * C::kSfRawBytes) + (kb & 1) * 8;
        const uint32_t sf = smem_u32(sm.stages + stage * C::kStageBytes + 2 * C::kWBytes + C::kTokBytes);
#pragma unroll
        for (int o = 0; o < 3; ++o) {
          uint32_t lo[4], hi[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int r = lane + 32 * j;
            lo[j] = 0u;
            hi[j] = 0u;
            if (o < 2 || r < rows)
              asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];"
                           : "=r"(lo[j]), "=r"(hi[j]) : "r"(raw + (o * kWRows + r) * 16) : "memory");
          }
          st_shared_v4(sf + o * kSfBytes + 16 * lane, lo[0], lo[1], lo[2], lo[3]);
          st_shared_v4(sf + o * kSfBytes + kAtomBytes + 16 * lane, hi[0], hi[1], hi[2], hi[3]);
        }
        fence_proxy_async_smem();  // the tensor core's tcgen05.cp reads these bytes
        mbar_arrive(&sm.full[stage]);
        if ((kb & 1) == 1 || kb + 1 == num_k) {
          mbar_arrive(&sm.raw_empty[rslot]);  // this lane's reads of the slot are done
          if (++rslot == kSfRing) { rslot = 0; rphase ^= 1u; }
        }
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp >= 2 && warp < kFirstEpiWarp) {
    // ------------------------------------------------------------ scale producer
    // Asynchronous 4-byte copies place every scale word directly at its atom
    // position; the stage's full barrier completes only once they have landed,
    // so this warp never waits for load latency and runs ahead like the TMA warp.
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int64_t item = blockIdx.x; item < total && ok; item += gridDim.x) {
      const int64_t t = item / g.n_wt, wt = item - t * g.n_wt;
      const int32_t e = g.tile_expert[t], row0 = g.tile_row[t], rows = g.tile_rows[t];
      const int64_t w0 = kMode == 0 ? wt * kWRows : wt * 2 * kWRows;
      const int64_t w1 = kMode == 0 ? w0 : w0 + kWRows;
      for (int kb = 0; kb < num_k; ++kb) {
        if (!mbar_wait(&sm.empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
        const uint32_t sf = smem_u32(sm.stages + stage * C::kStageBytes + 2 * C::kWBytes + C::kTokBytes);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int64_t r = lane + 32 * j;  // row inside the tile: atom row = lane, column = j
          const uint32_t dst = sf + 16 * lane + 4 * j;
          // rows outside the weight matrix or the token tile are zero-filled
          const uint8_t* p0 = g.w0_sf + e * g.w0_s0 + (w0 + r) * g.w0_s1 + kb * 8;
          const uint8_t* p1 = g.w1_sf + e * g.w1_s0 + (w1 + r) * g.w1_s1 + kb * 8;
          const uint8_t* px = g.x_sf + (row0 + r) * g.x_sf_ld + kb * 8;
          const uint32_t n0 = (w0 + r < g.N) ? 4u : 0u;
          const uint32_t n1 = (w1 + r < g.N) ? 4u : 0u;
          const uint32_t nx = (r < rows) ? 4u : 0u;
          cp_async_4(dst, n0 ? p0 : g.w0_sf, n0);
          cp_async_4(dst + kAtomBytes, n0 ? p0 + 4 : g.w0_sf, n0);
          cp_async_4(dst + kSfBytes, n1 ? p1 : g.w1_sf, n1);
          cp_async_4(dst + kSfBytes + kAtomBytes, n1 ? p1 + 4 : g.w1_sf, n1);
          cp_async_4(dst + 2 * kSfBytes, nx ? px : g.x_sf, nx);
          cp_async_4(dst + 2 * kSfBytes + kAtomBytes, nx ? px + 4 : g.x_sf, nx);
        }
        cp_async_mbar_arrive(&sm.full[stage]);
        mbar_arrive(&sm.full[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
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
        if (!mbar_wait(&sm.tempty[buf], acc_phase ^ 1u, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc0 = tmem_base + buf * C::kBufCols, acc1 = acc0 + kNmax;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, g.err)) { ok = false; break; }
          tc_fence_after();
          fence_proxy_async_smem();  // scales were written by cp.async, read by tcgen05.cp
          const uint32_t w0_addr = smem_u32(sm.stages + stage * C::kStageBytes);
          const uint32_t w1_addr = w0_addr + C::kWBytes;
          const uint32_t x_addr = w1_addr + C::kWBytes;
          const uint32_t sf_smem = x_addr + C::kTokBytes;
          const uint32_t sf_t = tmem_base + C::kSfCol0 + stage * kSfColsPerStage;
          // scales of W0 -> cols [0, 8), W1 -> [8, 16), X -> [16, 24); 4 columns per atom
#pragma unroll
          for (int q = 0; q < 6; ++q)
            tmem_cp_32x128b_x4(sf_t + 4 * q, plain_rows16_desc(sf_smem + kAtomBytes * q));
#pragma unroll
          for (int kk = 0; kk < kRowBytes / kUmmaKBytes; ++kk) {
            const uint32_t atom = kk >> 1, sfid = 2u * (kk & 1);
            const uint32_t idesc = idesc_mxf4(kWRows, rows, sfid, sfid);
            const uint64_t xd = sw128_kmajor_desc(x_addr + kk * kUmmaKBytes);
            const uint32_t sfx = (sf_t + 16 + 4 * atom) | (sfid << 30);
            const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
            mma_mxf4(acc0, sw128_kmajor_desc(w0_addr + kk * kUmmaKBytes), xd, idesc,
                     (sf_t + 4 * atom) | (sfid << 30), sfx, acc);
            mma_mxf4(acc1, sw128_kmajor_desc(w1_addr + kk * kUmmaKBytes), xd, idesc,
                     (sf_t + 8 + 4 * atom) | (sfid << 30), sfx, acc);
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
    const int quad = warp & 3;
    const int half = (warp - kFirstEpiWarp) >> 2;  // which of the quadrant's two warps
    uint8_t* stg = sm.staging + (warp - kFirstEpiWarp) * kStagingBytes;
    const uint32_t stg_s = smem_u32(stg);
    uint32_t buf = 0, acc_phase = 0;
    // GEMM2: slot ids and routing weights of a tile's tokens (lane j of chunk c
    // holds token c*32 + j), two independent loads per chunk (the weight comes
    // from the grouped-row copy permute wrote), issued one work item ahead so
    // their latency hides behind the previous item's epilogue
    int32_t slot_r[kNmax / 32], slot_n[kNmax / 32];
    float w_r[kNmax / 32], w_n[kNmax / 32];
    auto fetch_rows = [&](int64_t it, int32_t (&sl)[kNmax / 32], float (&wv)[kNmax / 32]) {
      if (kMode != 1 || it >= total) return;
      const int64_t tt = it / g.n_wt;
      const int32_t r0 = g.tile_row[tt], nr = g.tile_rows[tt];
#pragma unroll
      for (int c = 0; c < kNmax / 32; ++c) {
        const bool in = c * 32 < nr;
        sl[c] = in ? g.sorted[r0 + c * 32 + lane] : static_cast<int32_t>(g.S);
        wv[c] = in ? g.w_row[r0 + c * 32 + lane] : 0.0f;
      }
    };
    fetch_rows(blockIdx.x, slot_n, w_n);
    for (int64_t item = blockIdx.x; item < total; item += gridDim.x) {
      const int64_t t = item / g.n_wt, wt = item - t * g.n_wt;
      const int32_t row0 = g.tile_row[t], rows = g.tile_rows[t];
      if (kMode == 1) {
#pragma unroll
        for (int c = 0; c < kNmax / 32; ++c) {
          slot_r[c] = slot_n[c];
          w_r[c] = slot_n[c] < g.S ? w_n[c] : 0.0f;
        }
        fetch_rows(item + gridDim.x, slot_n, w_n);
      }
      if (!mbar_wait(&sm.tfull[buf], acc_phase, g.err)) break;
      tc_fence_after();
      const uint32_t lane_base = (static_cast<uint32_t>(quad * 32) << 16) + buf * C::kBufCols;
      if (kMode == 0) {
        // this warp's 32 weight rows = one 1x32 block of I for every token; the
        // quadrant's two warps each requantise 16 tokens of every 32-token chunk
        const int64_t i0 = wt * kWRows + quad * 32;
#pragma unroll 1
        for (int c = 0; c < rows / 32; ++c) {
          const int j0 = c * 32 + half * 16;
          uint32_t gv[16], uv[16];
          tmem_ld16(tmem_base + lane_base + j0, gv);
          tmem_ld16(tmem_base + lane_base + kNmax + j0, uv);
          tmem_wait_ld();
          uint32_t my_sc = 0;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float h = silu_mul(__uint_as_float(gv[j]), __uint_as_float(uv[j]));
            if (g.h_capture && i0 < g.N)
              g.h_capture[(row0 + j0 + j) * g.N + i0 + lane] = h;
            // |h| as bits orders like its value: one warp reduction gives the block amax
            const float amax = __uint_as_float(
                __reduce_max_sync(0xffffffffu, __float_as_uint(h) & 0x7fffffffu));
            const int sexp = mx_scale_exp(amax);
            const float q = h * exp2i_neg(sexp);
            const float qn = __shfl_xor_sync(0xffffffffu, q, 1);
            if ((lane & 1) == 0) {
              const uint32_t byte = cvt_e2m1x2(q, qn);
              asm volatile("st.shared.b8 [%0], %1;" ::"r"(stg_s + j * 16 + (lane >> 1)), "r"(byte)
                           : "memory");
            }
            if (lane == j) my_sc = static_cast<uint32_t>(sexp + 127);
          }
          __syncwarp();
          // lane j < 16 stores token j's 16 code bytes and its scale
          if (lane < 16 && i0 < g.N) {
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(stg_s + lane * 16));
            const int64_t p = row0 + j0 + lane;
            *reinterpret_cast<uint4*>(static_cast<uint8_t*>(g.out) + p * g.out_ld + i0 / 2) = v;
            g.out_sf[p * g.out_sf_ld + i0 / 32] = static_cast<uint8_t>(my_sc);
          }
          __syncwarp();
        }
      } else {
        // both accumulators of a 32-token chunk are loaded together (one wait)
        // and share the chunk's routing weights (splitting the two w2 slices
        // between the quadrant's warps instead measured slower: every warp then
        // broadcasts every chunk's weights)
#pragma unroll
        for (int c = 0; c < kNmax / 32; ++c) {
          if (c * 32 >= rows) break;
          if ((c & 1) != half) continue;
          const int32_t my_slot = slot_r[c];
          uint32_t v0[32], v1[32];
          tmem_ld32(tmem_base + lane_base + c * 32, v0);
          tmem_ld32(tmem_base + lane_base + kNmax + c * 32, v1);
          // token j's routing weight to every lane: one store per lane, then
          // eight broadcast 16-byte reads (instead of 32 shuffles)
          asm volatile("st.shared.f32 [%0], %1;" ::"r"(stg_s + kStagingTile + lane * 4), "f"(w_r[c])
                       : "memory");
          __syncwarp();
          float wj[32];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(wj[4 * q]), "=f"(wj[4 * q + 1]), "=f"(wj[4 * q + 2]), "=f"(wj[4 * q + 3])
                         : "r"(stg_s + kStagingTile + 16 * q));
          tmem_wait_ld();
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            const int64_t col0 = wt * 2 * kWRows + a * kWRows + quad * 32;
            const bool col_ok = col0 < g.N;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float y = wj[j] * __uint_as_float(a == 0 ? v0[j] : v1[j]);
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
              const int32_t s_j = __shfl_sync(0xffffffffu, my_slot, j);
              if (col_ok && s_j < g.S)
                *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out) + (row0 + c * 32 + j) * g.out_ld + col0 + part * 8) = v;
            }
            __syncwarp();
          }
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

template <int kMode, int kNmax, int kStages, bool kTmaSf>
cudaError_t launch_mx_sf(const CUtensorMap& w0, const CUtensorMap& w1, const CUtensorMap& x,
                         const CUtensorMap& sf0, const CUtensorMap& sf1, const CUtensorMap& sfx,
                         const MxArgs& g, int64_t max_items, int num_sms, cudaStream_t st) {
  using C = Cfg<kNmax, kStages>;
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    rc = cudaFuncSetAttribute(gemm_ws_mxfp4_kernel<kMode, kNmax, kStages, kTmaSf>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(C::kSmem));
    if (rc != cudaSuccess) return rc;
    if (dev < 64) configured |= 1ull << dev;
  }
  int64_t grid = max_items < num_sms ? max_items : num_sms;
  if (grid < 1) grid = 1;
  return launch_pdl(gemm_ws_mxfp4_kernel<kMode, kNmax, kStages, kTmaSf>, dim3(static_cast<unsigned>(grid)),
                    dim3(kThreads), C::kSmem, st, w0, w1, x, sf0, sf1, sfx, g);
}

template <int kMode, int kNmax, int kStages>
cudaError_t launch_mx(const CUtensorMap& w0, const CUtensorMap& w1, const CUtensorMap& x,
                      const CUtensorMap* sf, const MxArgs& g, int64_t max_items, int num_sms,
                      cudaStream_t st) {
  if (sf)
    return launch_mx_sf<kMode, kNmax, kStages, true>(w0, w1, x, sf[0], sf[1], sf[2], g, max_items,
                                                     num_sms, st);
  return launch_mx_sf<kMode, kNmax, kStages, false>(w0, w1, x, w0, w1, x, g, max_items, num_sms, st);
}

}  // namespace

cudaError_t launch_gemm_ws_mxfp4(int mode, int tile_max, const CUtensorMap& w0,
                                 const CUtensorMap& w1, const CUtensorMap& x, const CUtensorMap* sf,
                                 const WsGemmMx& p, int num_sms, cudaStream_t st, int* launches) {
  MxArgs g;
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
  g.out_sf = p.out_sf;
  g.out_sf_ld = p.out_sf_ld;
  g.topk_w = p.topk_w;
  g.k = p.k;
  g.x_sf = p.x_sf;
  g.x_sf_ld = p.x_sf_ld;
  g.w0_sf = p.w0_sf;
  g.w0_s0 = p.w0_s0;
  g.w0_s1 = p.w0_s1;
  g.w1_sf = p.w1_sf;
  g.w1_s0 = p.w1_s0;
  g.w1_s1 = p.w1_s1;
  g.w_row = p.w_row;
  g.h_capture = p.h_capture;
  g.err = p.err;
  if (launches) *launches += 1;
  const int64_t max_items = p.max_tiles * p.n_wt;
  if (tile_max == 128) {  // one accumulator buffer: fewer weight re-reads, epilogue not overlapped
    if (mode == 0) return launch_mx<0, 128, 3>(w0, w1, x, sf, g, max_items, num_sms, st);
    return launch_mx<1, 128, 3>(w0, w1, x, sf, g, max_items, num_sms, st);
  }
  if (tile_max == 96) {
    if (mode == 0) return launch_mx<0, 96, 4>(w0, w1, x, sf, g, max_items, num_sms, st);
    return launch_mx<1, 96, 4>(w0, w1, x, sf, g, max_items, num_sms, st);
  }
  if (tile_max == 32) {
    if (mode == 0) return launch_mx<0, 32, 5>(w0, w1, x, sf, g, max_items, num_sms, st);
    return launch_mx<1, 32, 5>(w0, w1, x, sf, g, max_items, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
