// Single-kernel decode path of the MXFP4 forward (at most 32 routing slots),
// the block-scaled counterpart of moe_decode.cu: e2m1 weights and activations
// with one e8m0 scale per 32 elements (aiter PR #3859, "Details":
// float4_e2m1fn_x2, QuantType.per_1x32), tcgen05.mma kind::mxf4.block_scale.
//
// Every CTA groups the slots by expert from the routing ids, then runs its
// share of two work lists:
//   GEMM1 item (routed expert r, 128 rows wt of I): gate/up code boxes
//       [128 B x 128 rows] from the expert-strided views, their scales copied
//       into the tensor cores' scale atoms, and the expert's token rows
//       quantised from x (the 1x32 rule of the quantising permute), once per
//       item into a shared buffer when they fit (else per k-step), and copied
//       into each stage at their 128-byte-swizzled positions;
//       h = silu(G) * U requantised per 1x32 along I into per-slot rows of the
//       workspace; then the expert's GEMM1 counter is raised.
//   GEMM2 item (routed expert r, 256 rows ot of H): two w2 slices (codes by
//       TMA, scales by copies), the expert's h rows gathered four at a time;
//       only the h rows and their scales wait for the expert's GEMM1 counter,
//       the weights stream at once.  y = w_slot * acc in bf16 per slot; the CTA
//       that completes an output tile's counter sums each token's slot rows in
//       fixed j order (the combine kernel's order and rounding).
// Warps: 0 TMA producer, 1 MMA issuer (and the scales' copy into TMEM),
// 2 scale copies and token quantisation, 3-6 epilogue.  Every wait is bounded;
// the cross-CTA counters are the decode slots' sets shared with moe_decode.cu.
#include "../../include/moe.h"
#include "moe_decode_units.cuh"
#include "moe_internal.h"
#include "moe_mx.cuh"

namespace moe {

using DecodeSyncMx = DecodeSync;  // the counter sets of the decode kernels (moe_decode.cu)

namespace {

constexpr int kWRows = 128;
constexpr int kRowBytes = 128;        // 256 e2m1 codes per row per k-step
constexpr int kUmmaKBytes = 32;       // 64 codes per instruction
constexpr int kNtok = 32;
constexpr int kStages = 5;
constexpr int kEpiWarps = 4;
constexpr int kFirstEpiWarp = 3;
constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
constexpr int kWBytes = kWRows * kRowBytes;     // 16 KiB
constexpr int kXBytes = kNtok * kRowBytes;      // 4 KiB
constexpr int kAtomBytes = 512;                 // 128 rows x 4 scale bytes
constexpr int kSfBytes = 2 * kAtomBytes;        // 8 scale blocks per row per stage
constexpr int kStageBytes = (2 * kWBytes + kXBytes + 3 * kSfBytes + 1023) / 1024 * 1024;
constexpr int kSfColsPerStage = 24;
constexpr int kAccCols = 2 * kNtok;             // acc0 + acc1 of one buffer
constexpr int kSfCol0 = 2 * kAccCols;
constexpr int kTmemCols = 256;
static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");
constexpr int kStagingBytes = 32 * 64;
constexpr int kMaxOutTiles = 64;
// a GEMM1 item's token rows, quantised once for all its k-steps (codes [cnt, H/2],
// then scales [cnt, H/32]) when they fit; else they are quantised per k-step
constexpr int kXbufBytes = 16 * 1024;
constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes + kEpiWarps * kStagingBytes +
                         kXbufBytes + (2 * kStages + 7) * 8 + 16 + 3 * 32 * 4 + 16;

struct MxDecArgs {
  int64_t T, H, I, E, k;
  View2 ids, topk_w, x;
  const uint8_t* gate_sf;
  int64_t gate_s0, gate_s1;
  const uint8_t* up_sf;
  int64_t up_s0, up_s1;
  const uint8_t* w2_sf;
  int64_t w2_s0, w2_s1;
  uint8_t* h_codes;      // [32, I/2] by slot
  uint8_t* h_sf;         // [32, I/32] by slot
  __nv_bfloat16* y_ws;   // [32, H] by slot
  __nv_bfloat16* out;
  int64_t os0, os1;
  int32_t vec_x, vec_out;
  int32_t slot;
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

// The whole warp waits: lane 0 polls, the others follow through the warp barrier
// (which orders lane 0's acquire before their later loads).
__device__ __forceinline__ bool warp_wait_count(const unsigned int* p, unsigned want,
                                                DeviceErrors* err, int lane) {
  int ok = 1;
  if (lane == 0) ok = wait_count(p, want, err) ? 1 : 0;
  __syncwarp();
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

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

__device__ __forceinline__ int nth_bit(unsigned m, int n) {
  for (int i = 0; i < n; ++i) m &= m - 1;
  return __ffs(m) - 1;
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_decode_mx_kernel(const __grid_constant__ CUtensorMap tmGate,
                         const __grid_constant__ CUtensorMap tmUp,
                         const __grid_constant__ CUtensorMap tmW2,
                         const __grid_constant__ CUtensorMap tmHc, const MxDecArgs g,
                         DecodeSyncMx* sync_sets) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint8_t* staging = base + kStages * kStageBytes;
  uint8_t* xbuf = staging + kEpiWarps * kStagingBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(xbuf + kXbufBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* epi_done = drain + 1;
  uint64_t* epi_last = drain + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 3);
  int* misc = reinterpret_cast<int*>(tmem_slot + 1);  // [0] routed experts, [1] valid slots, [2] last
  int* d_e = misc + 3;
  int* d_cnt = d_e + 32;
  unsigned* d_mask = reinterpret_cast<unsigned*>(d_cnt + 32);
  DecodeSyncMx& sync = sync_sets[g.slot];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmGate);
    tma_prefetch_desc(&tmUp);
    tma_prefetch_desc(&tmW2);
    tma_prefetch_desc(&tmHc);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1 + 32);  // TMA producer (with bytes) + the 32 lanes of warp 2
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
    int64_t id = -1;
    if (lane < S) id = read_id(g.ids, lane, g.k);
    const bool valid = lane < S && id >= 0 && id < g.E;
    const int key = valid ? static_cast<int>(id) : -1 - lane;
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
  const int n_wt1 = static_cast<int>(g.I / kWRows);        // I % 256 == 0 (validated)
  const int n_wt2 = static_cast<int>(g.H / (2 * kWRows));  // H % 256 == 0 (validated)
  const int n1 = nd * n_wt1;
  const int num_k1 = static_cast<int>(g.H / 256);
  const int num_k2 = static_cast<int>(g.I / 256);
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
        const int n_groups = (cnt + 3) / 4;
        const uint32_t tok_bytes = g1 ? 0u : static_cast<uint32_t>(n_groups) * 4 * kRowBytes;
        bool ready = g1;
        int pend_stage[kStages], pend_kb[kStages], npend = 0;
        auto load_h = [&](int st, int kb) {
          uint8_t* sx = stages + st * kStageBytes + 2 * kWBytes;
          unsigned m = mask;
          for (int gi = 0; gi < n_groups; ++gi) {
            int32_t row[4];
            for (int i = 0; i < 4; ++i) {
              const int s = m ? __ffs(m) - 1 : -1;
              if (m) m &= m - 1;
              row[i] = s < 0 ? row[0] : s;
            }
            tma_gather4(sx + gi * 4 * kRowBytes, &tmHc, &full[st], kb * kRowBytes, row[0], row[1],
                        row[2], row[3], pol);
          }
        };
        auto release_pending = [&]() {
          if (!wait_count(&sync.g1[r], static_cast<unsigned>(n_wt1), g.err)) ok = false;
          fence_proxy_async_global();
          for (int i = 0; i < npend; ++i) {
            mbar_expect_tx(&full[pend_stage[i]], tok_bytes);
            load_h(pend_stage[i], pend_kb[i]);
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
          const int32_t w0 = g1 ? wt * kWRows : wt * 2 * kWRows;
          const int32_t w1 = g1 ? w0 : w0 + kWRows;
          if (!ready) {
            mbar_expect_tx(&full[stage], 2 * kWBytes);
          } else {
            mbar_arrive_expect_tx(&full[stage], 2 * kWBytes + tok_bytes);
          }
          tma_load_3d(sw0, g1 ? &tmGate : &tmW2, &full[stage], kb * kRowBytes, w0, e, pol);
          tma_load_3d(sw1, g1 ? &tmUp : &tmW2, &full[stage], kb * kRowBytes, w1, e, pol);
          if (!ready) {
            pend_stage[npend] = stage;
            pend_kb[npend] = kb;
            ++npend;
          } else if (!g1) {
            load_h(stage, kb);
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
  } else if (warp == 2) {
    // ------------------------------------------------ scales and token quantisation
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_items && ok; u += gridDim.x) {
      const Unit x = unit_of(u, n1, ks, n_wt1, n_wt2, num_k1, num_k2);
      const bool g1 = x.g1;
      const int r = x.r, wt = x.wt;
      const int e = d_e[r], cnt = d_cnt[r];
      const unsigned mask = d_mask[r];
      const int64_t w0 = g1 ? wt * kWRows : wt * 2 * kWRows;
      const int64_t w1 = g1 ? w0 : w0 + kWRows;
      const uint8_t* sf0 = g1 ? g.gate_sf : g.w2_sf;
      const uint8_t* sf1 = g1 ? g.up_sf : g.w2_sf;
      const int64_t s00 = g1 ? g.gate_s0 : g.w2_s0, s01 = g1 ? g.gate_s1 : g.w2_s1;
      const int64_t s10 = g1 ? g.up_s0 : g.w2_s0, s11 = g1 ? g.up_s1 : g.w2_s1;
      const int64_t nrows = g1 ? g.I : g.H;
      const int my_slot = lane < cnt ? nth_bit(mask, lane) : -1;  // token row `lane` of the tile
      bool ready = g1;
      int pend_stage[kStages], pend_kb[kStages], npend = 0;
      // 32 bf16 of x: block (idx % 8) of this k-step for the tile's token row idx / 8
      auto load_x_block = [&](int idx, int kb, float (&v)[32]) {
        const int q = idx >> 3, b = idx & 7;
        const int64_t t = nth_bit(mask, q) / g.k;
        const int64_t c0 = static_cast<int64_t>(kb) * 256 + b * 32;
        if (g.vec_x) {
          const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(g.x.data) + t * g.x.s0 + c0);
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const uint4 w4v = __ldg(src + qq);
            const uint32_t w4[4] = {w4v.x, w4v.y, w4v.z, w4v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              v[qq * 8 + 2 * i] = __uint_as_float((w4[i] & 0xffffu) << 16);
              v[qq * 8 + 2 * i + 1] = __uint_as_float(w4[i] & 0xffff0000u);
            }
          }
        } else {
          const uint16_t* src = static_cast<const uint16_t*>(g.x.data) + t * g.x.s0;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            v[i] = __uint_as_float(static_cast<uint32_t>(src[(c0 + i) * g.x.s1]) << 16);
        }
      };
      // the h scale bytes of the tile's token rows, written by other CTAs during
      // this kernel: read from L2 (a line of L1 could hold an older copy of a
      // neighbouring slot's row) and stored into the token scale atoms
      auto h_scales = [&](int st, int kb) {
        const uint32_t sfx = smem_u32(stages + st * kStageBytes + 2 * kWBytes + kXBytes) + 2 * kSfBytes;
        uint32_t a = 0u, b = 0u;
        if (my_slot >= 0) {
          const unsigned int* p =
              reinterpret_cast<const unsigned int*>(g.h_sf + my_slot * (g.I / 32) + kb * 8);
          a = __ldcg(p);
          b = __ldcg(p + 1);
        }
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sfx + 16 * lane), "r"(a) : "memory");
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(sfx + kAtomBytes + 16 * lane), "r"(b) : "memory");
        fence_proxy_async_smem();
      };
      // GEMM1: quantise the unit's token rows once, for all its k-steps
      const int64_t rb = g.H / 2, sbytes = g.H / 32;
      const bool use_buf = g1 && cnt * (rb + sbytes) <= kXbufBytes;
      __syncwarp();  // every lane is done with the previous item's buffer
      if (use_buf) {
        const int nb = 8 * (x.kb1 - x.kb0);  // 1x32 blocks of the unit's k-steps, per row
        for (int idx = lane; idx < cnt * nb; idx += 32) {
          const int q = idx / nb, b = idx - q * nb + 8 * x.kb0;
          float v[32];
          load_x_block(q * 8 + (b & 7), b >> 3, v);  // row q, k-step b / 8, block b % 8
          uint32_t wq[4];
          const uint32_t sc = mx_quant32(v, wq);
          *reinterpret_cast<uint4*>(xbuf + q * rb + b * 16) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
          xbuf[cnt * rb + q * sbytes + b] = static_cast<uint8_t>(sc);
        }
        __syncwarp();
      }
      for (int kb = x.kb0; kb < x.kb1 && ok; ++kb) {
        if (!ready && npend == kStages) {
          if (!warp_wait_count(&sync.g1[r], static_cast<unsigned>(n_wt1), g.err, lane)) ok = false;
          for (int i = 0; i < npend; ++i) {
            h_scales(pend_stage[i], pend_kb[i]);
            cp_async_mbar_arrive(&full[pend_stage[i]]);
            mbar_arrive(&full[pend_stage[i]]);
          }
          npend = 0;
          ready = true;
        }
        // GEMM1: this lane's first x block of the k-step is loaded before the
        // wait for the stage, so its latency overlaps the wait
        float v[32];
        const bool early = g1 && !use_buf && lane < cnt * 8;
        if (early) load_x_block(lane, kb, v);
        if (!mbar_wait(&empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
        uint8_t* st_base = stages + stage * kStageBytes;
        const uint32_t sf = smem_u32(st_base + 2 * kWBytes + kXBytes);
        // weight scales of this k-step straight into the scale atoms (byte
        // (row % 32) * 16 + (row / 32) * 4 + block); rows past the matrix read as zero
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int64_t rr = lane + 32 * j;
          const uint32_t dst = sf + 16 * lane + 4 * j;
          const uint32_t n0 = (w0 + rr < nrows) ? 4u : 0u;
          const uint32_t n1 = (w1 + rr < nrows) ? 4u : 0u;
          const uint8_t* p0 = sf0 + e * s00 + (w0 + rr) * s01 + kb * 8;
          const uint8_t* p1 = sf1 + e * s10 + (w1 + rr) * s11 + kb * 8;
          cp_async_4(dst, n0 ? p0 : sf0, n0);
          cp_async_4(dst + kAtomBytes, n0 ? p0 + 4 : sf0, n0);
          cp_async_4(dst + kSfBytes, n1 ? p1 : sf1, n1);
          cp_async_4(dst + kSfBytes + kAtomBytes, n1 ? p1 + 4 : sf1, n1);
        }
        if (g1) {
          // the expert's token rows, quantised per 1x32 block into the stage:
          // codes of block b of row q at 16-byte chunk b ^ (q % 8) (128-byte swizzle)
          uint8_t* sx = st_base + 2 * kWBytes;
          uint8_t* sfx = st_base + 2 * kWBytes + kXBytes + 2 * kSfBytes;
          if (use_buf) {
            // the k-step's 128 code bytes of each row and its 8 scale bytes, from the item's buffer
            for (int idx = lane; idx < cnt * 8; idx += 32) {
              const int q = idx >> 3, b = idx & 7;
              *reinterpret_cast<uint4*>(sx + (q >> 3) * 1024 + (q & 7) * 128 + ((b ^ (q & 7)) * 16)) =
                  *reinterpret_cast<const uint4*>(xbuf + q * rb + kb * 128 + b * 16);
            }
            if (lane < cnt) {
              const uint32_t* sw = reinterpret_cast<const uint32_t*>(xbuf + cnt * rb + lane * sbytes + kb * 8);
              *reinterpret_cast<uint32_t*>(sfx + lane * 16) = sw[0];
              *reinterpret_cast<uint32_t*>(sfx + kAtomBytes + lane * 16) = sw[1];
            }
          } else {
            for (int idx = lane; idx < cnt * 8; idx += 32) {
              const int q = idx >> 3, b = idx & 7;
              if (idx != lane) load_x_block(idx, kb, v);
              uint32_t wq[4];
              const uint32_t sc = mx_quant32(v, wq);
              *reinterpret_cast<uint4*>(sx + (q >> 3) * 1024 + (q & 7) * 128 + ((b ^ (q & 7)) * 16)) =
                  make_uint4(wq[0], wq[1], wq[2], wq[3]);
              sfx[(b >> 2) * kAtomBytes + q * 16 + (b & 3)] = static_cast<uint8_t>(sc);
            }
          }
          fence_proxy_async_smem();
          cp_async_mbar_arrive(&full[stage]);
          mbar_arrive(&full[stage]);
        } else if (ready) {
          h_scales(stage, kb);
          cp_async_mbar_arrive(&full[stage]);
          mbar_arrive(&full[stage]);
        } else {
          pend_stage[npend] = stage;
          pend_kb[npend] = kb;
          ++npend;
        }
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ready && npend > 0) {
        if (!warp_wait_count(&sync.g1[r], static_cast<unsigned>(n_wt1), g.err, lane)) ok = false;
        for (int i = 0; i < npend; ++i) {
          h_scales(pend_stage[i], pend_kb[i]);
          cp_async_mbar_arrive(&full[pend_stage[i]]);
          mbar_arrive(&full[pend_stage[i]]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      uint32_t stage = 0, phase = 0, buf = 0, acc_phase = 0;
      bool ok = true, issued = false;
      for (int u = blockIdx.x; u < n_items && ok; u += gridDim.x) {
        const Unit x = unit_of(u, n1, ks, n_wt1, n_wt2, num_k1, num_k2);
        if (!mbar_wait(&tempty[buf], acc_phase ^ 1u, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc0 = tmem_base + buf * kAccCols, acc1 = acc0 + kNtok;
        for (int kb = x.kb0; kb < x.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, g.err)) { ok = false; break; }
          tc_fence_after();
          fence_proxy_async_smem();  // scales by cp.async and codes by st.shared, read below
          const uint32_t w0_addr = smem_u32(stages + stage * kStageBytes);
          const uint32_t w1_addr = w0_addr + kWBytes;
          const uint32_t x_addr = w1_addr + kWBytes;
          const uint32_t sf_smem = x_addr + kXBytes;
          const uint32_t sf_t = tmem_base + kSfCol0 + stage * kSfColsPerStage;
#pragma unroll
          for (int q = 0; q < 6; ++q)
            tmem_cp_32x128b_x4(sf_t + 4 * q, plain_rows16_desc(sf_smem + kAtomBytes * q));
#pragma unroll
          for (int kk = 0; kk < kRowBytes / kUmmaKBytes; ++kk) {
            const uint32_t atom = kk >> 1, sfid = 2u * (kk & 1);
            const uint32_t idesc = idesc_mxf4(kWRows, kNtok, sfid, sfid);
            const uint64_t xd = sw128_kmajor_desc(x_addr + kk * kUmmaKBytes);
            const uint32_t sfx = (sf_t + 16 + 4 * atom) | (sfid << 30);
            const uint32_t acc = (kb > x.kb0 || kk > 0) ? 1u : 0u;
            mma_mxf4(acc0, sw128_kmajor_desc(w0_addr + kk * kUmmaKBytes), xd, idesc,
                     (sf_t + 4 * atom) | (sfid << 30), sfx, acc);
            mma_mxf4(acc1, sw128_kmajor_desc(w1_addr + kk * kUmmaKBytes), xd, idesc,
                     (sf_t + 8 + 4 * atom) | (sfid << 30), sfx, acc);
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
    const int et = threadIdx.x - 32 * kFirstEpiWarp;  // 0..127
    uint8_t* stg = staging + (warp - kFirstEpiWarp) * kStagingBytes;
    const uint32_t stg_s = smem_u32(stg);
    uint32_t buf = 0, acc_phase = 0, sync_phase = 0;
    const unsigned vmask = static_cast<unsigned>(misc[1]);
    if (nd == 0 && blockIdx.x == 0) {
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
      const int my_slot = lane < cnt ? nth_bit(mask, lane) : -1;
      float my_w = 0.0f;
      if (!g1 && my_slot >= 0) {
        const int64_t t = my_slot / g.k, j = my_slot - t * g.k;
        my_w = static_cast<const float*>(g.topk_w.data)[t * g.topk_w.s0 + j * g.topk_w.s1];
      }
      if (!mbar_wait(&tfull[buf], acc_phase, g.err)) break;
      tc_fence_after();
      const uint32_t lane_base = (static_cast<uint32_t>(quad * 32) << 16) + buf * kAccCols;
      bool released = false;  // the accumulator buffer was handed back to the MMA warp
      if (g1) {
        // this warp's 32 rows of I = one 1x32 block for every token: requantise
        const int64_t i0 = static_cast<int64_t>(wt) * kWRows + quad * 32;
        uint32_t gv[32], uv[32];
        tmem_ld32(tmem_base + lane_base, gv);
        tmem_ld32(tmem_base + lane_base + kNtok, uv);
        tmem_wait_ld();
        if (ks > 1) {
          // one K part of the item: park the fp32 partials; the unit that
          // completes the item sums all parts in part order and requantises
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[buf]);
          if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
          released = true;
          int colb = 0;  // this expert's token columns follow those of the routed experts before it
          for (int q = 0; q < r; ++q) colb += d_cnt[q];
          const size_t tile_stride = static_cast<size_t>(n_wt1) * kNtok * 2 * kWRows;
          float* pb = g.part_ws + x.part * tile_stride +
                      (static_cast<size_t>(wt) * kNtok + colb) * 2 * kWRows + quad * 32 + lane;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j >= cnt) break;
            pb[j * 2 * kWRows] = __uint_as_float(gv[j]);
            pb[j * 2 * kWRows + kWRows] = __uint_as_float(uv[j]);
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
                sg[j] += __uint_as_float(gv[j]);
                su[j] += __uint_as_float(uv[j]);
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
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            gv[j] = __float_as_uint(sg[j]);
            uv[j] = __float_as_uint(su[j]);
          }
        }
        uint32_t my_sc = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float h = silu_mul(__uint_as_float(gv[j]), __uint_as_float(uv[j]));
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
        uint4 v;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(stg_s + lane * 16));
        if (my_slot >= 0 && i0 < g.I) {
          *reinterpret_cast<uint4*>(g.h_codes + my_slot * (g.I / 2) + i0 / 2) = v;
          g.h_sf[my_slot * (g.I / 32) + i0 / 32] = static_cast<uint8_t>(my_sc);
        }
        __syncwarp();
      } else {
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem_base + lane_base, v0);
        tmem_ld32(tmem_base + lane_base + kNtok, v1);
        float wj[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) wj[j] = __shfl_sync(0xffffffffu, my_w, j);
        tmem_wait_ld();
#pragma unroll 1
        for (int a = 0; a < 2; ++a) {
          const int64_t col0 = static_cast<int64_t>(wt) * 2 * kWRows + a * kWRows + quad * 32;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const __nv_bfloat16 yb = __float2bfloat16_rn(wj[j] * __uint_as_float(a == 0 ? v0[j] : v1[j]));
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
            const int s_j = __shfl_sync(0xffffffffu, my_slot, j);
            if (s_j >= 0 && col0 < g.H)
              *reinterpret_cast<uint4*>(g.y_ws + s_j * g.H + col0 + part * 8) = v;
          }
          __syncwarp();
        }
      }
      if (!released) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
        if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
      }
      __threadfence();
      __syncwarp();
      if (lane == 0) mbar_arrive(epi_done);
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
      const bool last = !g1 && misc[2] != 0;
      sync_phase ^= 1u;
      if (last) {
        __threadfence();
        const int64_t c0 = static_cast<int64_t>(wt) * 2 * kWRows;
        const int64_t n8 = 2 * kWRows / 8;
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

  pdl_launch_dependents();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (threadIdx.x == 0) {
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

}  // namespace

cudaError_t launch_decode_fused_mx(const CUtensorMap& gate, const CUtensorMap& up,
                                   const CUtensorMap& w2, const CUtensorMap& hc,
                                   const DecodeMxArgs& p, int num_sms, cudaStream_t st,
                                   int* launches) {
  if (p.T * p.k > 32 || p.T * p.k < 1 || p.H > 2 * kWRows * kMaxOutTiles) return cudaErrorInvalidValue;
  if (p.H % 256 != 0 || p.I % 256 != 0) return cudaErrorInvalidValue;
  static unsigned long long configured = 0;
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  if (dev >= 64 || !(configured & (1ull << dev))) {
    rc = cudaFuncSetAttribute(moe_decode_mx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(kSmem));
    if (rc != cudaSuccess) return rc;
    if (dev < 64) configured |= 1ull << dev;
  }
  MxDecArgs g;
  g.T = p.T;
  g.H = p.H;
  g.I = p.I;
  g.E = p.E;
  g.k = p.k;
  g.ids = p.ids;
  g.topk_w = p.topk_w;
  g.x = p.x;
  g.gate_sf = p.gate_sf;
  g.gate_s0 = p.gate_s0;
  g.gate_s1 = p.gate_s1;
  g.up_sf = p.up_sf;
  g.up_s0 = p.up_s0;
  g.up_s1 = p.up_s1;
  g.w2_sf = p.w2_sf;
  g.w2_s0 = p.w2_s0;
  g.w2_s1 = p.w2_s1;
  g.h_codes = p.h_codes;
  g.h_sf = p.h_sf;
  g.y_ws = p.y_ws;
  g.out = p.out;
  g.os0 = p.os0;
  g.os1 = p.os1;
  g.vec_x = (p.x.s1 == 1 && (p.x.s0 * 2) % 16 == 0 && reinterpret_cast<uintptr_t>(p.x.data) % 16 == 0) ? 1 : 0;
  g.vec_out = (p.os1 == 1 && (p.os0 * 2) % 16 == 0 && reinterpret_cast<uintptr_t>(p.out) % 16 == 0) ? 1 : 0;
  g.slot = static_cast<int32_t>(next_decode_slot());
  g.part_ws = p.part_ws;
  g.max_split = p.max_split;
  g.err = p.err;
  DecodeSyncMx* sets = decode_sync_sets();
  if (!sets) return cudaErrorInvalidDevicePointer;
  if (launches) *launches += 1;
  return launch_pdl(moe_decode_mx_kernel, dim3(static_cast<unsigned>(num_sms)), dim3(kThreads), kSmem,
                    st, gate, up, w2, hc, g, sets);
}

}  // namespace moe
