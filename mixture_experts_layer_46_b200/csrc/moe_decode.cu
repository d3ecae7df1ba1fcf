// Single-kernel decode path (at most 32 routing slots): the whole forward in
// one launch, for the token counts where the layer is the latency of streaming
// the routed experts' weights once (the pages' single-token dispatch case,
// Liger-Kernel PR #1377, "Testing Done").
//
// Every CTA groups the slots by expert itself from the routing ids (warp
// match / ballot; no align kernel, no permute kernel), then runs its share of
// two lists of work items on the tensor cores:
//   GEMM1 item (routed expert r, 128 rows wt of I): gate/up weight boxes
//       [64 x 128] from the expert-strided views (3-D TMA maps whose expert
//       stride is each view's real stride(0), Liger-Kernel PR #1377,
//       "Problems"), the expert's token rows gathered straight from x with
//       TMA four-row gathers into a 32-row tile; h = silu(G) * U in bf16, stored
//       per slot in the workspace; then the expert's GEMM1 counter is raised.
//   GEMM2 item (routed expert r, 256 rows ot of H): two w2 slices, the
//       expert's h rows as the token tile; y = w_slot * acc in bf16 per slot.
//       Its weight stages are requested at once: only the h rows wait for the
//       expert's GEMM1 counter to be complete, so weights keep streaming
//       across the GEMM1 -> GEMM2 hand-off.  (Requesting all of GEMM2's w2
//       tiles into L2 at kernel start was measured slower: the extra traffic
//       slowed GEMM1's stream more than it sped up GEMM2.)  Then the output tile's counter is
//       raised; the CTA that completes it (the last of the routed experts for
//       those 256 columns) sums each token's k slot rows in fixed j order in
//       fp32 and writes out[t, ot] (the same order and rounding as the combine
//       kernel, so the result is bit-identical to the multi-kernel path).
// Items are dealt round-robin over the CTAs, GEMM1 items first, so a CTA's
// GEMM2 weights stream in right behind its GEMM1 work.  No CTA ever waits for
// work of a CTA that is waiting itself: GEMM1 items have no dependency.
// Every wait is bounded.  The counters live in library memory, one set per
// call slot (kDecodeSlots sets, dealt round-robin), and the last CTA to exit
// resets them, so each launch finds them zero.
#include <atomic>
#include <mutex>

#include "../../include/moe.h"
#include "moe_decode_units.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kWRows = 128;
constexpr int kBK = 64;
constexpr int kUmmaK = 16;
constexpr int kNtok = 32;                    // token rows per tile (MMA N)
constexpr int kStages = 6;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kTmemCols = 128;               // two buffers of acc0 + acc1 (32 columns each)
constexpr int kWBytes = kWRows * kBK * 2;    // 16 KiB
constexpr int kXBytes = kNtok * kBK * 2;     // 4 KiB
constexpr int kStageBytes = 2 * kWBytes + kXBytes;
constexpr int kStagingBytes = 32 * 64;
constexpr int kMaxOutTiles = 64;             // H <= 16384
constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes + kEpiWarps * kStagingBytes +
                         (2 * kStages + 7) * 8 + 16 + 3 * 32 * 4 + 16;

static_assert(sizeof(DecodeSync::g2) / sizeof(unsigned) == kMaxOutTiles, "counter sets");

}  // namespace

// The counter sets of the decode kernels: library memory, zero at load, left
// zero by every launch (its last CTA resets the set it used).
__device__ DecodeSync g_decode_sync[kDecodeSlots];

namespace {

struct DecArgs {
  int64_t T, H, I, E, k;
  View2 ids, topk_w;
  __nv_bfloat16* h_ws;   // [32, I]: h row of each slot
  __nv_bfloat16* y_ws;   // [32, H]: weighted down-projection row of each slot
  __nv_bfloat16* out;
  int64_t os0, os1;
  int32_t vec_out;
  int32_t slot;          // counter set of this call
  float* part_ws;        // GEMM1 split-K partials (layout of decode_part_bytes)
  int32_t max_split;     // at most this many GEMM1 K parts
  DeviceErrors* err;
};

__device__ __forceinline__ int64_t read_id(const View2& v, int64_t s, int64_t k) {
  const int64_t t = s / k, j = s - t * k;
  const int64_t off = t * v.s0 + j * v.s1;
  if (v.dtype == MOE_I64) return static_cast<const int64_t*>(v.data)[off];
  return static_cast<int64_t>(static_cast<const int32_t*>(v.data)[off]);
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned int* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Spins (bounded) until *p >= want, backing off to one poll a microsecond so
// that many waiting CTAs do not crowd the counter's L2 line; false on timeout (counted).
__device__ __forceinline__ bool wait_count(const unsigned int* p, unsigned want, DeviceErrors* err) {
  if (ld_acquire(p) >= want) return true;
  const unsigned long long t0 = global_ns();
  unsigned ns = 32;
  while (true) {
    __nanosleep(ns);
    if (ns < 1024) ns <<= 1;
    if (ld_acquire(p) >= want) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      if (err) atomicAdd(&err->timeouts, 1u);
      return false;
    }
  }
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Four rows (r0..r3) of a 2-D tensor, 64 bf16 columns from `col`, into four
// consecutive 128-byte rows at dst (the map's box is one row high); the
// 128-byte swizzle follows the destination address, so the rows land where a
// 4-row box would put them.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t col, int32_t r0, int32_t r1, int32_t r2,
                                            int32_t r3, uint64_t hint) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(col), "r"(r0), "r"(r1), "r"(r2),
      "r"(r3), "l"(hint)
      : "memory");
}

// the n-th set bit (0-based) of m
__device__ __forceinline__ int nth_bit(unsigned m, int n) {
  for (int i = 0; i < n; ++i) m &= m - 1;
  return __ffs(m) - 1;
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_decode_fused_kernel(const __grid_constant__ CUtensorMap tmGate,
                            const __grid_constant__ CUtensorMap tmUp,
                            const __grid_constant__ CUtensorMap tmW2,
                            const __grid_constant__ CUtensorMap tmX,
                            const __grid_constant__ CUtensorMap tmH, const DecArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint8_t* staging = base + kStages * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + kEpiWarps * kStagingBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* epi_done = drain + 1;  // the epilogue warps have written an item's rows
  uint64_t* epi_last = drain + 2;  // the counter of an output tile is complete (or not)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 3);
  int* misc = reinterpret_cast<int*>(tmem_slot + 1);  // [0] routed experts, [1] valid slots, [2] last
  int* d_e = misc + 3;                                // routed experts, ascending
  int* d_cnt = d_e + 32;                              // their slot counts
  unsigned* d_mask = reinterpret_cast<unsigned*>(d_cnt + 32);  // their slots (bit s)
  DecodeSync& sync = g_decode_sync[g.slot];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmGate);
    tma_prefetch_desc(&tmUp);
    tma_prefetch_desc(&tmW2);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmH);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    mbar_init(epi_done, kEpiWarps);
    mbar_init(epi_last, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();
  const int S = static_cast<int>(g.T * g.k);
  if (warp == 0) {
    // group the slots by expert: one lane per slot
    int64_t id = -1;
    if (lane < S) id = read_id(g.ids, lane, g.k);
    const bool valid = lane < S && id >= 0 && id < g.E;
    const int key = valid ? static_cast<int>(id) : -1 - lane;  // skipped slots: distinct keys
    const unsigned same = __match_any_sync(0xffffffffu, key);
    const bool first = valid && (__ffs(same) - 1 == lane);
    const unsigned firsts = __ballot_sync(0xffffffffu, first);
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    const unsigned bad = __ballot_sync(0xffffffffu, lane < S && !valid);
    int r = 0;
    for (int j = 0; j < 32; ++j) {
      const int o = __shfl_sync(0xffffffffu, key, j);
      r += (((firsts >> j) & 1u) != 0u && o < key) ? 1 : 0;
    }
    if (first) {
      d_e[r] = key;
      d_cnt[r] = __popc(same);
      d_mask[r] = same;
    }
    if (lane == 0) {
      misc[0] = __popc(firsts);
      misc[1] = static_cast<int>(vmask);
      if (blockIdx.x == 0 && bad && g.err) atomicAdd(&g.err->bad_ids, static_cast<unsigned>(__popc(bad)));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nd = misc[0];
  const int n_wt1 = static_cast<int>((g.I + kWRows - 1) / kWRows);
  const int n_wt2 = static_cast<int>((g.H + 2 * kWRows - 1) / (2 * kWRows));
  const int n1 = nd * n_wt1;
  const int num_k1 = static_cast<int>((g.H + kBK - 1) / kBK);
  const int num_k2 = static_cast<int>((g.I + kBK - 1) / kBK);
  const int ks = split_count(n1, num_k1, static_cast<int>(gridDim.x), g.max_split);
  const int n_items = n1 * ks + nd * n_wt2;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      uint32_t stage = 0, phase = 0;
      int8_t last_phase[kStages];
      for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
      const uint64_t pol = l2_policy_evict_last();
      bool ok = true;
      for (int u = blockIdx.x; u < n_items && ok; u += gridDim.x) {
        const Unit x = unit_of(u, n1, ks, n_wt1, n_wt2, num_k1, num_k2);
        const bool g1 = x.g1;
        const int r = x.r, wt = x.wt;
        const int e = d_e[r], cnt = d_cnt[r];
        const unsigned mask = d_mask[r];
        // token rows go in groups of four (one gather each); a group's unused
        // entries repeat its first row, filling tile rows the MMA results skip
        const int n_groups = (cnt + 3) / 4;
        const uint32_t tok_bytes = static_cast<uint32_t>(n_groups) * 4 * kBK * 2;
        // GEMM2: weights go out at once, the h rows only once the expert's h is complete
        bool ready = g1;
        int pend_stage[kStages], pend_kb[kStages], npend = 0;
        auto load_tokens = [&](int st, int kb) {
          uint8_t* sx = stages + st * kStageBytes + 2 * kWBytes;
          unsigned m = mask;
          for (int gi = 0; gi < n_groups; ++gi) {
            int32_t row[4];
            for (int i = 0; i < 4; ++i) {
              // GEMM1 gathers x rows (token = slot / k), GEMM2 the slots' h rows
              const int s = m ? __ffs(m) - 1 : -1;
              if (m) m &= m - 1;
              row[i] = s < 0 ? row[0] : (g1 ? static_cast<int32_t>(s / g.k) : s);
            }
            tma_gather4(sx + gi * 4 * kBK * 2, g1 ? &tmX : &tmH, &full[st], kb * kBK, row[0], row[1],
                        row[2], row[3], pol);
          }
        };
        auto release_pending = [&]() {
          if (!wait_count(&sync.g1[r], static_cast<unsigned>(n_wt1), g.err)) ok = false;
          fence_proxy_async_global();
          for (int i = 0; i < npend; ++i) {
            mbar_expect_tx(&full[pend_stage[i]], tok_bytes);
            load_tokens(pend_stage[i], pend_kb[i]);
            mbar_arrive(&full[pend_stage[i]]);
          }
          npend = 0;
          ready = true;
        };
        for (int kb = x.kb0; kb < x.kb1 && ok; ++kb) {
          if (!ready && npend == kStages) release_pending();
          if (!mbar_wait(&empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
          uint8_t* sw0 = stages + stage * kStageBytes;
          uint8_t* sw1 = sw0 + kWBytes;
          if (g1) {
            mbar_arrive_expect_tx(&full[stage], 2 * kWBytes + tok_bytes);
            tma_load_3d(sw0, &tmGate, &full[stage], kb * kBK, wt * kWRows, e, pol);
            tma_load_3d(sw1, &tmUp, &full[stage], kb * kBK, wt * kWRows, e, pol);
            load_tokens(stage, kb);
          } else if (!ready) {
            mbar_expect_tx(&full[stage], 2 * kWBytes);
            tma_load_3d(sw0, &tmW2, &full[stage], kb * kBK, wt * 2 * kWRows, e, pol);
            tma_load_3d(sw1, &tmW2, &full[stage], kb * kBK, wt * 2 * kWRows + kWRows, e, pol);
            pend_stage[npend] = stage;
            pend_kb[npend] = kb;
            ++npend;
          } else {
            mbar_arrive_expect_tx(&full[stage], 2 * kWBytes + tok_bytes);
            tma_load_3d(sw0, &tmW2, &full[stage], kb * kBK, wt * 2 * kWRows, e, pol);
            tma_load_3d(sw1, &tmW2, &full[stage], kb * kBK, wt * 2 * kWRows + kWRows, e, pol);
            load_tokens(stage, kb);
          }
          last_phase[stage] = static_cast<int8_t>(phase);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ready && npend > 0) release_pending();
      }
      if (!ok) {
        for (int s = 0; s < kStages; ++s)
          if (last_phase[s] >= 0) mbar_wait(&full[s], static_cast<uint32_t>(last_phase[s]), g.err);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      uint32_t stage = 0, phase = 0, buf = 0, acc_phase = 0;
      bool ok = true, issued = false;
      const uint32_t idesc = idesc_bf16_f32(kWRows, kNtok);
      for (int u = blockIdx.x; u < n_items && ok; u += gridDim.x) {
        const Unit x = unit_of(u, n1, ks, n_wt1, n_wt2, num_k1, num_k2);
        if (!mbar_wait(&tempty[buf], acc_phase ^ 1u, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc0 = tmem_base + buf * 2 * kNtok, acc1 = acc0 + kNtok;
        for (int kb = x.kb0; kb < x.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t w0_addr = smem_u32(stages + stage * kStageBytes);
          const uint32_t w1_addr = w0_addr + kWBytes;
          const uint32_t x_addr = w1_addr + kWBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint64_t xd = sw128_kmajor_desc(x_addr + kk * kUmmaK * 2);
            const uint32_t acc = (kb > x.kb0 || kk > 0) ? 1u : 0u;
            mma_bf16(acc0, sw128_kmajor_desc(w0_addr + kk * kUmmaK * 2), xd, idesc, acc);
            mma_bf16(acc1, sw128_kmajor_desc(w1_addr + kk * kUmmaK * 2), xd, idesc, acc);
          }
          issued = true;
          mma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);
        if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
      }
      if (issued) {
        mma_commit(drain);
        mbar_wait(drain, 0, g.err);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int et = threadIdx.x - 64;  // 0..127 over the epilogue warps
    uint8_t* stg = staging + (warp - 2) * kStagingBytes;
    const uint32_t stg_s = smem_u32(stg);
    uint32_t buf = 0, acc_phase = 0, sync_phase = 0;
    const unsigned vmask = static_cast<unsigned>(misc[1]);
    if (nd == 0 && blockIdx.x == 0) {
      // no slot routed to an expert: every output row is zero
      for (int64_t idx = et; idx < g.T * g.H; idx += 32 * kEpiWarps) {
        const int64_t t = idx / g.H, c = idx - t * g.H;
        g.out[t * g.os0 + c * g.os1] = __float2bfloat16_rn(0.0f);
      }
    }
    for (int u = blockIdx.x; u < n_items; u += gridDim.x) {
      const Unit x = unit_of(u, n1, ks, n_wt1, n_wt2, num_k1, num_k2);
      const bool g1 = x.g1;
      const int r = x.r, wt = x.wt;
      const unsigned mask = d_mask[r];
      const int cnt = d_cnt[r];
      // the token column j of this tile is the slot my_slot (lane j holds it)
      const int my_slot = lane < cnt ? nth_bit(mask, lane) : -1;
      float my_w = 0.0f;
      if (!g1 && my_slot >= 0) {
        const int64_t t = my_slot / g.k, j = my_slot - t * g.k;
        my_w = static_cast<const float*>(g.topk_w.data)[t * g.topk_w.s0 + j * g.topk_w.s1];
      }
      if (!mbar_wait(&tfull[buf], acc_phase, g.err)) break;
      tc_fence_after();
      const uint32_t lane_base = (static_cast<uint32_t>(quad * 32) << 16) + buf * 2 * kNtok;
      if (g1 && ks > 1) {
        // ---- one K part of a GEMM1 item: park the fp32 partials; the unit that
        // completes the item sums all parts in part order and writes h
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem_base + lane_base, v0);
        tmem_ld32(tmem_base + lane_base + kNtok, v1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
        if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
        // this expert's token columns follow those of the routed experts before it
        int colb = 0;
        for (int q = 0; q < r; ++q) colb += d_cnt[q];
        const int row = quad * 32 + lane;
        const size_t tile_stride = static_cast<size_t>(n_wt1) * kNtok * 2 * kWRows;
        float* pb = g.part_ws + x.part * tile_stride + (static_cast<size_t>(wt) * kNtok + colb) * 2 * kWRows + row;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (j >= cnt) break;
          pb[j * 2 * kWRows] = __uint_as_float(v0[j]);
          pb[j * 2 * kWRows + kWRows] = __uint_as_float(v1[j]);
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(epi_done);
        if (et == 0) {
          mbar_wait(epi_done, sync_phase, g.err);
          __threadfence();
          const unsigned old = atomicAdd(&sync.g1p[x.item], 1u);
          misc[2] = (old + 1 == static_cast<unsigned>(ks)) ? 1 : 0;
          __threadfence();
          mbar_arrive(epi_last);
        }
        mbar_wait(epi_last, sync_phase, g.err);
        const bool done_item = misc[2] != 0;
        sync_phase ^= 1u;
        if (!done_item) continue;
        __threadfence();
        float sg[32], su[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) sg[j] = su[j] = 0.0f;
        for (int p = 0; p < ks; ++p) {
          if (p == x.part) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              sg[j] += __uint_as_float(v0[j]);
              su[j] += __uint_as_float(v1[j]);
            }
          } else {
            const float* qb = pb + static_cast<ptrdiff_t>(p - x.part) * static_cast<ptrdiff_t>(tile_stride);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j >= cnt) break;
              sg[j] += __ldcg(qb + j * 2 * kWRows);
              su[j] += __ldcg(qb + j * 2 * kWRows + kWRows);
            }
          }
        }
        const int64_t col0 = static_cast<int64_t>(wt) * kWRows + quad * 32;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const __nv_bfloat16 hb = __float2bfloat16_rn(silu_mul(sg[j], su[j]));
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(stg_s + j * 64 + lane * 2),
                       "h"(*reinterpret_cast<const uint16_t*>(&hb)) : "memory");
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
          const int s_j = __shfl_sync(0xffffffffu, my_slot, j);
          if (s_j >= 0 && col0 < g.I) *reinterpret_cast<uint4*>(g.h_ws + s_j * g.I + col0 + part * 8) = v;
        }
        __syncwarp();
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(epi_done);
        if (et == 0) {
          mbar_wait(epi_done, sync_phase, g.err);
          __threadfence();
          atomicAdd(&sync.g1[r], 1u);
          mbar_arrive(epi_last);
        }
        mbar_wait(epi_last, sync_phase, g.err);
        sync_phase ^= 1u;
        continue;
      }
      const int n_out = g1 ? 1 : 2;
      const int64_t ld = g1 ? g.I : g.H;
      __nv_bfloat16* dst = g1 ? g.h_ws : g.y_ws;
#pragma unroll 1
      for (int a = 0; a < n_out; ++a) {
        const int64_t col0 = g1 ? static_cast<int64_t>(wt) * kWRows + quad * 32
                                : static_cast<int64_t>(wt) * 2 * kWRows + a * kWRows + quad * 32;
        uint32_t v0[32];
        tmem_ld32(tmem_base + lane_base + a * kNtok, v0);
        if (g1) {
          uint32_t v1[32];
          tmem_ld32(tmem_base + lane_base + kNtok, v1);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const __nv_bfloat16 hb = __float2bfloat16_rn(silu_mul(__uint_as_float(v0[j]), __uint_as_float(v1[j])));
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(stg_s + j * 64 + lane * 2),
                         "h"(*reinterpret_cast<const uint16_t*>(&hb)) : "memory");
          }
        } else {
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const __nv_bfloat16 yb = __float2bfloat16_rn(__shfl_sync(0xffffffffu, my_w, j) * __uint_as_float(v0[j]));
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(stg_s + j * 64 + lane * 2),
                         "h"(*reinterpret_cast<const uint16_t*>(&yb)) : "memory");
          }
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
          const int s_j = __shfl_sync(0xffffffffu, my_slot, j);
          if (s_j >= 0 && col0 < (g1 ? g.I : g.H))
            *reinterpret_cast<uint4*>(dst + s_j * ld + col0 + part * 8) = v;
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
      // publish this item's rows, then raise its counter (one thread, once all
      // four epilogue warps have written theirs); bounded mbarrier waits only
      __threadfence();
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_done);
      bool last = false;
      if (et == 0) {
        mbar_wait(epi_done, sync_phase, g.err);
        __threadfence();
        if (g1) {
          atomicAdd(&sync.g1[r], 1u);
        } else {
          const unsigned old = atomicAdd(&sync.g2[wt], 1u);
          misc[2] = (old + 1 == static_cast<unsigned>(nd)) ? 1 : 0;
          __threadfence();
        }
        mbar_arrive(epi_last);
      }
      mbar_wait(epi_last, sync_phase, g.err);
      last = !g1 && misc[2] != 0;
      sync_phase ^= 1u;
      if (!g1) {
        if (last) {
          // every routed expert's rows for these 256 columns are in y: combine them
          __threadfence();
          const int64_t c0 = static_cast<int64_t>(wt) * 2 * kWRows;
          const int64_t ncol = (g.H - c0) < 2 * kWRows ? (g.H - c0) : 2 * kWRows;
          const int64_t n8 = ncol / 8;
          for (int64_t idx = et; idx < g.T * n8; idx += 32 * kEpiWarps) {
            const int64_t t = idx / n8, c = c0 + (idx - t * n8) * 8;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int j = 0; j < g.k; ++j) {
              const int s = static_cast<int>(t * g.k + j);
              if (!((vmask >> s) & 1u)) continue;
              const uint4 v = __ldcg(reinterpret_cast<const uint4*>(g.y_ws + s * g.H + c));
              const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                acc[2 * i] += __uint_as_float(w4[i] << 16);
                acc[2 * i + 1] += __uint_as_float(w4[i] & 0xffff0000u);
              }
            }
            if (g.vec_out) {
              uint4 o;
              o.x = pack_bf16x2(acc[0], acc[1]);
              o.y = pack_bf16x2(acc[2], acc[3]);
              o.z = pack_bf16x2(acc[4], acc[5]);
              o.w = pack_bf16x2(acc[6], acc[7]);
              *reinterpret_cast<uint4*>(g.out + t * g.os0 + c) = o;
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) g.out[t * g.os0 + (c + i) * g.os1] = __float2bfloat16_rn(acc[i]);
            }
          }
        }
      }
    }
  }

  pdl_launch_dependents();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0) {
    // the last CTA out resets this call slot's counters for the next launch
    __threadfence();
    const unsigned old = atomicAdd(&sync.exit_cnt, 1u);
    if (old + 1 == gridDim.x) {
      __threadfence();
      for (int i = 0; i < 32; ++i) sync.g1[i] = 0u;
      for (int i = 0; i < kMaxOutTiles; ++i) sync.g2[i] = 0u;
      if (ks > 1)
        for (int i = 0; i < n1; ++i) sync.g1p[i] = 0u;
      __threadfence();
      sync.exit_cnt = 0u;
    }
  }
}

std::atomic<unsigned> g_next_slot{0};
std::mutex g_sync_mu;
DecodeSync* g_sync_addr[64] = {};

}  // namespace

unsigned next_decode_slot() { return g_next_slot.fetch_add(1u) % kDecodeSlots; }

DecodeSync* decode_sync_sets() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_sync_mu);
  if (!g_sync_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_sync) != cudaSuccess) return nullptr;
    g_sync_addr[dev] = static_cast<DecodeSync*>(p);
  }
  return g_sync_addr[dev];
}

cudaError_t launch_decode_fused(const CUtensorMap& gate, const CUtensorMap& up, const CUtensorMap& w2,
                                const CUtensorMap& x1, const CUtensorMap& h1, const DecodeArgs& p,
                                int num_sms, cudaStream_t st, int* launches) {
  if (p.T * p.k > 32 || p.T * p.k < 1 || p.H > 2 * kWRows * kMaxOutTiles) return cudaErrorInvalidValue;
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    rc = cudaFuncSetAttribute(moe_decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmem));
    if (rc != cudaSuccess) return rc;
    if (dev < 64) configured |= 1ull << dev;
  }
  DecArgs g;
  g.T = p.T;
  g.H = p.H;
  g.I = p.I;
  g.E = p.E;
  g.k = p.k;
  g.ids = p.ids;
  g.topk_w = p.topk_w;
  g.h_ws = p.h_ws;
  g.y_ws = p.y_ws;
  g.out = p.out;
  g.os0 = p.os0;
  g.os1 = p.os1;
  g.vec_out = (p.os1 == 1 && (p.os0 * 2) % 16 == 0 && reinterpret_cast<uintptr_t>(p.out) % 16 == 0) ? 1 : 0;
  g.slot = static_cast<int32_t>(next_decode_slot());
  g.part_ws = p.part_ws;
  g.max_split = p.max_split;
  g.err = p.err;
  if (launches) *launches += 1;
  return launch_pdl(moe_decode_fused_kernel, dim3(static_cast<unsigned>(num_sms)), dim3(kThreads), kSmem,
                    st, gate, up, w2, x1, h1, g);
}

}  // namespace moe
