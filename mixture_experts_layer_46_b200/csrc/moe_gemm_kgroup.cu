// Expert-weight gradients: GEMMs grouped along K (tcgen05, sm_100a).
//
//   C[e, m, n] = sum over the expert's grouped rows p of A[m, p] * B[n, p]
//
// A [M, P] and B [N, P] are row-major bf16 (the grouped activations transposed,
// so the contraction over an expert's rows is contiguous and both operands are
// K-major like every other GEMM here); expert e owns rows [offsets[e],
// offsets[e + 1]), a multiple of 64 (the align granule of the gradient path), and
// its padding rows hold zeros in A and B.  C is [E, M, N], fp32 or bf16 (fp32 sums):
//   dw2[e]          = (w dout)^T_e h_e        A = (w dout)^T [H, P], B = h^T [I, P]
//   [dgate; dup][e] = [dg | du]^T_e x_e       A = [dg | du]^T [2I, P], B = x^T [H, P]
// (the gradients of out = sum_j w y with respect to w2, gate and up).
//
// Kernel shape: one persistent CTA per SM, 6 warps: warp 0 TMA producer (one
// [64 x 128] box of A and one [64 x 256] box of B per k-block, 128-byte swizzle),
// warp 1 TMEM allocator and MMA issuer (M = 128, N = 256, fp32 accumulators, two
// buffers: all 512 TMEM columns), warps 2-5 epilogue, one per TMEM lane quadrant
// (one row m per thread: the warp's 32-row tile of 32 fp32 or 64 bf16 columns, 128
// bytes a row, goes to shared memory in the 128-byte swizzled layout and out with one
// TMA store, which also clips the M and N tails; two staging tiles per warp, so a
// tile is filled while the previous one's store is still reading).  Work item = (expert,
// 128-row tile of M, 256-column tile of N), expert-major; an expert with no rows
// gets zeros.  The operand tiles come from L2 once per work item (each A tile is read
// N / 256 times, each B tile M / 128 times), so the 256-column tile moves a quarter
// fewer operand bytes per FLOP than a square 128 x 128 one.
#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kTM = kKgroupTileM, kTN = kKgroupTileN, kBK = 64, kUmmaK = 16;
constexpr int kStages = 4;
constexpr int kEpiWarps = 4;  // one per TMEM lane quadrant
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kTmemCols = 2 * kTN;
constexpr int kABytes = kTM * kBK * 2;  // 16 KiB
constexpr int kBBytes = kTN * kBK * 2;  // 32 KiB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kStgBytes = 32 * 128;  // one staging tile: 32 rows x 32 fp32 (two per epilogue warp)
constexpr size_t kSmem = 1024 + size_t(kStages) * kStageBytes + 2 * kEpiWarps * kStgBytes +
                         (2 * kStages + 4 + 1) * 8 + 16;
static_assert(kSmem <= 227 * 1024, "K-grouped GEMM shared memory");
static_assert(kTmemCols <= 512, "two accumulator buffers fit the 512 TMEM columns");

struct KgArgs {
  int64_t M, N, E;
  int64_t n_mt, n_nt;
  const int32_t* offsets;  // [E + 1] grouped-row offsets, multiples of 64
  DeviceErrors* err;
};

// shared -> global tile store (bulk group of the issuing thread)
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int32_t c0, int32_t c1,
                                             int32_t c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

template <bool kBf16Out>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kgroup_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmC, const KgArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint8_t* staging = stages + kStages * kStageBytes;  // 1024-byte aligned: the swizzle atom
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + 2 * kEpiWarps * kStgBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmC);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  pdl_wait();
  const int64_t per_e = g.n_mt * g.n_nt;
  const int64_t total = g.E * per_e;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      uint32_t stage = 0, phase = 0;
      int8_t last_phase[kStages];
      for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
      const uint64_t pol = l2_policy_evict_last();
      bool ok = true;
      for (int64_t item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const int64_t e = item / per_e, r = item - e * per_e;
        const int32_t m0 = static_cast<int32_t>((r / g.n_nt) * kTM);
        const int32_t n0 = static_cast<int32_t>((r % g.n_nt) * kTN);
        const int k0 = g.offsets[e] / kBK, k1 = g.offsets[e + 1] / kBK;
        for (int kb = k0; kb < k1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, g.err)) { ok = false; break; }
          uint8_t* sa = stages + stage * kStageBytes;
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          tma_load_2d(sa, &tmA, &full[stage], kb * kBK, m0, pol);
          tma_load_2d(sa + kABytes, &tmB, &full[stage], kb * kBK, n0, pol);
          last_phase[stage] = static_cast<int8_t>(phase);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
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
      const uint32_t idesc = idesc_bf16_f32(kTM, kTN);
      for (int64_t item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const int64_t e = item / per_e;
        const int k0 = g.offsets[e] / kBK, k1 = g.offsets[e + 1] / kBK;
        if (!mbar_wait(&tempty[buf], acc_phase ^ 1u, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc = tmem_base + buf * kTN;
        for (int kb = k0; kb < k1; ++kb) {
          if (!mbar_wait(&full[stage], phase, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(stages + stage * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk)
            mma_bf16(acc, sw128_kmajor_desc(a_addr + kk * kUmmaK * 2), sw128_kmajor_desc(b_addr + kk * kUmmaK * 2),
                     idesc, (kb > k0 || kk > 0) ? 1u : 0u);
          issued = true;
          mma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);  // with no k-block it completes at once (the epilogue writes zeros)
        if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
      }
      if (!ok && issued) {
        mma_commit(drain);
        mbar_wait(drain, 0, g.err);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32) = rows m of this warp
    const uint32_t stg = smem_u32(staging + (warp - 2) * 2 * kStgBytes);
    uint32_t buf = 0, acc_phase = 0, nstore = 0;
    for (int64_t item = blockIdx.x; item < total; item += gridDim.x) {
      const int64_t e = item / per_e, r = item - e * per_e;
      const int32_t m0 = static_cast<int32_t>((r / g.n_nt) * kTM + quad * 32);
      const int32_t n0 = static_cast<int32_t>((r % g.n_nt) * kTN);
      const bool empty_e = g.offsets[e + 1] == g.offsets[e];
      if (!mbar_wait(&tfull[buf], acc_phase, g.err)) break;
      tc_fence_after();
      const uint32_t lane_base = (static_cast<uint32_t>(quad * 32) << 16) + buf * kTN;
      // one staged tile row is 128 bytes: 32 fp32 or 64 bf16 columns
      constexpr int kCols = kBf16Out ? 64 : 32;
#pragma unroll 1
      for (int c = 0; c < kTN / kCols; ++c) {
        uint32_t v[32];
        if (empty_e) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0u;
        } else if (kBf16Out) {
          uint32_t a[32], b[32];
          tmem_ld32(tmem_base + lane_base + c * 64, a);
          tmem_ld32(tmem_base + lane_base + c * 64 + 32, b);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v[j] = pack_bf16x2(__uint_as_float(a[2 * j]), __uint_as_float(a[2 * j + 1]));
            v[16 + j] = pack_bf16x2(__uint_as_float(b[2 * j]), __uint_as_float(b[2 * j + 1]));
          }
        } else {
          tmem_ld32(tmem_base + lane_base + c * 32, v);
          tmem_wait_ld();
        }
        if (m0 < g.M && n0 + c * kCols < g.N) {
          // two staging tiles in turn: the store issued two tiles ago (the last one to use
          // this tile) has read it, while the previous one may still be in flight
          const uint32_t sb = stg + (nstore & 1u) * kStgBytes;
          ++nstore;
          if (lane == 0) bulk_wait_read_1();
          __syncwarp();
          // row `lane` of the tile: 16-byte chunk q at position q ^ (row % 8) (128-byte swizzle)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sb + lane * 128 + ((q ^ (lane & 7)) * 16)),
                         "r"(v[4 * q]), "r"(v[4 * q + 1]), "r"(v[4 * q + 2]), "r"(v[4 * q + 3])
                         : "memory");
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmC, sb, n0 + c * kCols, m0, static_cast<int32_t>(e));
            bulk_commit();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (++buf == 2) { buf = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait_all();  // C is written before the kernel ends
  }

  pdl_launch_dependents();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// dst[c, p] = 0 for a padding row p (sorted[p] >= S), else scale(p) * src_row(p)[c],
// where src_row(p) is row sorted[p] / k of a token-major tensor (gather) or row p
// of a grouped [P, C] matrix, and scale(p) is the slot's routing weight or 1.
// A block moves 64 rows p by kGtTiles 64-column tiles through unpadded [p][c]
// shared tiles, 256 threads.  Load phase: a thread resolves its two rows once, then
// issues all its source reads (8 consecutive columns, 16 bytes, per row and tile;
// element loads where the rows are not 16-byte aligned) before it stores any, so
// each thread keeps 2 x kGtTiles loads in flight; a warp fills 512 contiguous bytes
// of a tile.  Store phase: a thread owns one column c and 16 rows p of a tile; a
// warp's 32 columns of one tile row are 16 consecutive 4-byte words (no bank
// conflict), and each thread writes 32 contiguous bytes (one sector) of dst row c.
// P is a multiple of 64 (the granule), dst 16-byte aligned.
constexpr int kGtTiles = 4;

__device__ __forceinline__ uint16_t gt_scale(uint16_t raw, float w) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(w * __uint_as_float(static_cast<uint32_t>(raw) << 16)));
}
__device__ __forceinline__ uint32_t gt_scale2(uint32_t pair, float w) {
  return static_cast<uint32_t>(gt_scale(static_cast<uint16_t>(pair & 0xffffu), w)) |
         (static_cast<uint32_t>(gt_scale(static_cast<uint16_t>(pair >> 16), w)) << 16);
}

__global__ void __launch_bounds__(256) gather_transpose_kernel(View2 src, int gather, int vec, const int32_t* sorted,
                                                               int64_t S, int64_t k, View2 wts, int scale,
                                                               uint16_t* dst, int64_t P, int64_t C) {
  __shared__ __align__(16) uint16_t tile[kGtTiles][64][64];  // [column tile][row p][column c]
  pdl_wait();
  const int64_t p0 = static_cast<int64_t>(blockIdx.x) * 64, cb = static_cast<int64_t>(blockIdx.y) * (64 * kGtTiles);
  const int tid = threadIdx.x, q = tid & 7;
  const uint16_t* row[2];
  float wr[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int64_t p = p0 + (tid >> 3) + 32 * h;
    row[h] = nullptr;
    wr[h] = 1.0f;
    const int32_t s = p < P ? sorted[p] : -1;
    if (s >= 0 && s < S) {
      const int64_t t = s / k, j = s - t * k;
      row[h] = static_cast<const uint16_t*>(src.data) + (gather ? t : p) * src.s0;
      if (scale) wr[h] = static_cast<const float*>(wts.data)[t * wts.s0 + j * wts.s1];
    }
  }
  uint4 u[2][kGtTiles];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int ct = 0; ct < kGtTiles; ++ct) {
      const int64_t c = cb + 64 * ct + 8 * q;
      u[h][ct] = make_uint4(0u, 0u, 0u, 0u);
      if (row[h] != nullptr && c < C) {
        if (vec && c + 8 <= C) {
          u[h][ct] = *reinterpret_cast<const uint4*>(row[h] + c);
        } else {
          uint32_t e4[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const uint32_t lo = c + 2 * r < C ? row[h][(c + 2 * r) * src.s1] : 0u;
            const uint32_t hi = c + 2 * r + 1 < C ? row[h][(c + 2 * r + 1) * src.s1] : 0u;
            e4[r] = lo | (hi << 16);
          }
          u[h][ct] = make_uint4(e4[0], e4[1], e4[2], e4[3]);
        }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int ct = 0; ct < kGtTiles; ++ct) {
      uint4 v = u[h][ct];
      if (scale) {
        v.x = gt_scale2(v.x, wr[h]);
        v.y = gt_scale2(v.y, wr[h]);
        v.z = gt_scale2(v.z, wr[h]);
        v.w = gt_scale2(v.w, wr[h]);
      }
      *reinterpret_cast<uint4*>(&tile[ct][(tid >> 3) + 32 * h][8 * q]) = v;
    }
  }
  __syncthreads();
  const int ci = tid & 63, g = tid >> 6;  // destination rows cb + 64 ct + ci, rows p 16g .. 16g + 15
#pragma unroll
  for (int ct = 0; ct < kGtTiles; ++ct) {
    const int64_t c = cb + 64 * ct + ci;
    if (c < C) {
      uint32_t w8[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        w8[r] = static_cast<uint32_t>(tile[ct][16 * g + 2 * r][ci]) |
                (static_cast<uint32_t>(tile[ct][16 * g + 2 * r + 1][ci]) << 16);
      uint4* d = reinterpret_cast<uint4*>(dst + c * P + p0 + 16 * g);
      d[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
      d[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
    }
  }
  pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_gemm_kgroup(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c, int bf16_out,
                               int64_t M, int64_t N, int64_t E, const int32_t* offsets, DeviceErrors* err,
                               int num_sms, cudaStream_t st, int* launches) {
  static unsigned long long configured[2] = {0, 0};
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  const int bi = bf16_out ? 1 : 0;
  if (dev >= 64 || !(configured[bi] & (1ull << dev))) {
    rc = cudaFuncSetAttribute(bf16_out ? gemm_kgroup_kernel<true> : gemm_kgroup_kernel<false>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
    if (rc != cudaSuccess) return rc;
    if (dev < 64) configured[bi] |= 1ull << dev;
  }
  KgArgs g;
  g.M = M;
  g.N = N;
  g.E = E;
  g.n_mt = (M + kTM - 1) / kTM;
  g.n_nt = (N + kTN - 1) / kTN;
  g.offsets = offsets;
  g.err = err;
  const int64_t total = E * g.n_mt * g.n_nt;
  int64_t grid = total < num_sms ? total : num_sms;
  if (grid < 1) grid = 1;
  if (launches) *launches += 1;
  if (bf16_out)
    return launch_pdl(gemm_kgroup_kernel<true>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), kSmem, st, a, b,
                      c, g);
  return launch_pdl(gemm_kgroup_kernel<false>, dim3(static_cast<unsigned>(grid)), dim3(kThreads), kSmem, st, a, b,
                    c, g);
}

cudaError_t launch_gather_transpose(const View2& src, int gather, const int32_t* sorted, int64_t S, int64_t k,
                                    const View2& wts, int scale, void* dst, int64_t P, int64_t C,
                                    cudaStream_t st, int* launches) {
  if (P == 0 || C == 0) return cudaSuccess;
  constexpr int64_t kCols = 64 * kGtTiles;
  if ((C + kCols - 1) / kCols > 65535 || P % 64 != 0 || reinterpret_cast<uintptr_t>(dst) % 16 != 0)
    return cudaErrorInvalidValue;
  const int vec = src.s1 == 1 && (src.s0 * 2) % 16 == 0 && reinterpret_cast<uintptr_t>(src.data) % 16 == 0;
  if (launches) *launches += 1;
  const dim3 grid(static_cast<unsigned>(P / 64), static_cast<unsigned>((C + kCols - 1) / kCols));
  return launch_pdl(gather_transpose_kernel, grid, dim3(256), 0, st, src, gather, vec, sorted, S, k, wts, scale,
                    static_cast<uint16_t*>(dst), P, C);
}

}  // namespace moe
