// Step "align": group the T*k routing slots by expert.
//
// Slot s = t*k + j is routed to expert e = topk_ids[t, j] (ids read through
// their strides: a per-layer routing slice of a [T, layers, k] tensor has token
// stride layers*k, prime-rl PR #2860 "Problem").  Outputs:
//   counts[e]       slots of expert e
//   offsets[e]      exclusive prefix sum of ceil(counts[e] / bm) * bm
//   sorted[p]       slots grouped by expert, ascending slot order inside an
//                   expert, padding rows hold the sentinel S = T*k
//   block_expert[b] the expert of bm-row block b; num_blocks = offsets[E] / bm
// The per-token-bucket block size bm plays the role of aiter PR #3859's
// block_m ("Tuned MoE latency" table).  Ids outside [0, E) are skipped and
// counted.  The order inside an expert is stable so results are reproducible.
//
// Small problems run in one CTA; larger ones in three kernels: per-chunk
// histograms, one scan CTA, per-chunk stable scatter.
#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ int64_t read_id(const View2& v, int64_t s, int64_t k) {
  const int64_t t = s / k, j = s - t * k;
  const int64_t off = t * v.s0 + j * v.s1;
  if (v.dtype == MOE_I64) return static_cast<const int64_t*>(v.data)[off];
  return static_cast<int64_t>(static_cast<const int32_t*>(v.data)[off]);
}

// Histogram of the slots [s0, s1) into hist (shared, zeroed by the caller).
// Returns this thread's count of invalid ids.
__device__ int block_hist(const View2& ids, int64_t k, int64_t E, int64_t s0, int64_t s1,
                          int* hist) {
  int bad = 0;
  for (int64_t s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
    const int64_t e = read_id(ids, s, k);
    if (e >= 0 && e < E)
      atomicAdd(&hist[e], 1);
    else
      ++bad;
  }
  return bad;
}

// Stable scatter of slots [s0, s1): slot s of expert e goes to
// sorted[base[e] + (number of earlier slots of e in [s0, s))].  base[] lives in
// shared memory and is advanced as slots are placed; warp_cnt is a
// [kWarps][E] shared array that must be all zero on entry (and is left zero).
__device__ void block_scatter(const View2& ids, int64_t k, int64_t E, int64_t s0, int64_t s1,
                              int* base, int* warp_cnt, int32_t* sorted, int32_t* inv) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int64_t c0 = s0; c0 < s1; c0 += blockDim.x) {
    const int64_t s = c0 + threadIdx.x;
    int e = -1;
    if (s < s1) {
      const int64_t v = read_id(ids, s, k);
      if (v >= 0 && v < E) e = static_cast<int>(v);
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(peers) - 1;
    const int rank = __popc(peers & lt_mask);
    if (e >= 0 && lane == leader) warp_cnt[warp * E + e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += warp_cnt[w * E + e];
      const int pos = base[e] + before + rank;
      sorted[pos] = static_cast<int32_t>(s);
      inv[s] = pos;
    } else if (s < s1) {
      inv[s] = -1;
    }
    __syncthreads();
    if (e >= 0 && lane == leader) {
      atomicAdd(&base[e], __popc(peers));
      warp_cnt[warp * E + e] = 0;
    }
    __syncthreads();
  }
}

// Block-wide exclusive scan over experts of v(e) (each thread owns a
// contiguous run of experts).  out[e] receives the prefix, out[E] the total;
// every thread gets the total back.
template <class F>
__device__ int block_scan_experts(int64_t E, F v, int* out) {
  __shared__ int warp_sums[32];
  __shared__ int total_sh;
  const int per = static_cast<int>((E + blockDim.x - 1) / blockDim.x);
  const int e0 = threadIdx.x * per;
  int local = 0;
  for (int i = 0; i < per; ++i)
    if (e0 + i < E) local += v(e0 + i);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = local;
  for (int d = 1; d < 32; d <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += u;
  }
  __syncthreads();  // warp_sums may still be read by a previous call
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) / 32;
    int x = lane < nw ? warp_sums[lane] : 0;
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, x, d);
      if (lane >= d) x += u;
    }
    if (lane < nw) warp_sums[lane] = x;
    if (lane == nw - 1) total_sh = x;
  }
  __syncthreads();
  int run = incl - local + (warp > 0 ? warp_sums[warp - 1] : 0);
  for (int i = 0; i < per; ++i) {
    if (e0 + i < E) {
      out[e0 + i] = run;
      run += v(e0 + i);
    }
  }
  if (threadIdx.x == 0) out[E] = total_sh;
  __syncthreads();
  return total_sh;
}

// Outputs of align beyond sorted/offsets: the token-tile list consumed by the
// weight-stationary GEMMs (tiles of at most tile_max rows, balanced within an
// expert, never crossing one), written when tile_max > 0.
struct TileOut {
  int32_t tile_max;
  int32_t* tile_row;     // first padded row of the tile
  int32_t* tile_rows;    // rows in the tile (multiple of bm)
  int32_t* tile_expert;
  int32_t* num_tiles;
};

// From per-expert counts (shared), write counts, offsets, num_blocks,
// block_expert, the sentinel padding of sorted and the tile list.  offs
// (shared, E+1 ints) receives the offsets; tsc (shared, E+1 ints) is scratch.
__device__ void block_finalize(const int* cnt, int64_t E, int32_t bm, int32_t S, int* offs, int* tsc,
                               int32_t* counts, int32_t* offsets, int32_t* sorted,
                               int32_t* block_expert, int32_t* num_blocks, const TileOut& to) {
  const int total = block_scan_experts(E, [&](int e) { return (cnt[e] + bm - 1) / bm * bm; }, offs);
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    offsets[e] = offs[e];
    if (e < E) counts[e] = cnt[e];
  }
  if (threadIdx.x == 0) *num_blocks = total / bm;
  const int nb = total / bm;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) {
    // last expert whose offset is <= b*bm (empty experts share offsets with the next one)
    int lo = 0, hi = static_cast<int>(E);  // answer in [lo, hi)
    const int p = b * bm;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (offs[mid] <= p) lo = mid; else hi = mid;
    }
    block_expert[b] = lo;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    for (int p = offs[e] + cnt[e]; p < offs[e + 1]; ++p) sorted[p] = S;
  if (to.tile_max > 0) {
    const int tm = to.tile_max;
    const int nt = block_scan_experts(
        E, [&](int e) { return (offs[e + 1] - offs[e] + tm - 1) / tm; }, tsc);
    // an expert's rows are split into its n tiles as evenly as the bm granule
    // allows (e.g. 288 rows with tm = 256 -> 160 + 128, not 256 + 32), so no
    // work item streams a whole weight tile for a handful of tokens
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      const int rows = offs[e + 1] - offs[e];
      const int n = (rows + tm - 1) / tm;
      if (n == 0) continue;
      const int units = rows / bm;  // rows is a multiple of bm
      int start = offs[e];
      for (int j = 0; j < n; ++j) {
        const int u = units / n + (j < units % n ? 1 : 0);
        to.tile_row[tsc[e] + j] = start;
        to.tile_rows[tsc[e] + j] = u * bm;
        to.tile_expert[tsc[e] + j] = e;
        start += u * bm;
      }
    }
    if (threadIdx.x == 0) *to.num_tiles = nt;
  }
}

__global__ void __launch_bounds__(kThreads) align_small_kernel(
    View2 ids, int64_t T, int64_t k, int64_t E, int32_t bm, int32_t* counts, int32_t* offsets,
    int32_t* sorted, int32_t* inv, int32_t* block_expert, int32_t* num_blocks, TileOut to,
    DeviceErrors* err) {
  extern __shared__ int sm[];
  int* hist = sm;                       // [E]
  int* offs = hist + E;                 // [E + 1]
  int* base = offs + E + 1;             // [E]
  int* warp_cnt = base + E;             // [kWarps * E]
  int* tsc = warp_cnt + kWarps * E;     // [E + 1]
  __shared__ int bad_sh;
  pdl_wait();
  const int64_t S = T * k;
  for (int i = threadIdx.x; i < E * (kWarps + 1); i += blockDim.x) {
    if (i < E) hist[i] = 0;
    else warp_cnt[i - E] = 0;
  }
  if (threadIdx.x == 0) bad_sh = 0;
  __syncthreads();
  const int bad = block_hist(ids, k, E, 0, S, hist);
  if (bad) atomicAdd(&bad_sh, bad);
  __syncthreads();
  block_finalize(hist, E, bm, static_cast<int32_t>(S), offs, tsc, counts, offsets, sorted,
                 block_expert, num_blocks, to);
  for (int e = threadIdx.x; e < E; e += blockDim.x) base[e] = offs[e];
  __syncthreads();
  block_scatter(ids, k, E, 0, S, base, warp_cnt, sorted, inv);
  if (threadIdx.x == 0 && bad_sh && err) atomicAdd(&err->bad_ids, static_cast<unsigned>(bad_sh));
  pdl_launch_dependents();
}

__global__ void __launch_bounds__(kThreads) align_count_kernel(View2 ids, int64_t T, int64_t k,
                                                               int64_t E, int32_t* chunk_counts,
                                                               DeviceErrors* err) {
  extern __shared__ int hist[];
  __shared__ int bad_sh;
  pdl_wait();
  const int64_t S = T * k;
  for (int i = threadIdx.x; i < E; i += blockDim.x) hist[i] = 0;
  if (threadIdx.x == 0) bad_sh = 0;
  __syncthreads();
  const int64_t s0 = static_cast<int64_t>(blockIdx.x) * kAlignChunk;
  const int64_t s1 = min(S, s0 + kAlignChunk);
  const int bad = block_hist(ids, k, E, s0, s1, hist);
  if (bad) atomicAdd(&bad_sh, bad);
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x) chunk_counts[blockIdx.x * E + i] = hist[i];
  if (threadIdx.x == 0 && bad_sh && err) atomicAdd(&err->bad_ids, static_cast<unsigned>(bad_sh));
  pdl_launch_dependents();
}

__global__ void __launch_bounds__(1024) align_scan_kernel(int64_t T, int64_t k, int64_t E,
                                                          int32_t bm, int64_t n_chunks,
                                                          int32_t* chunk_counts, int32_t* counts,
                                                          int32_t* offsets, int32_t* sorted,
                                                          int32_t* block_expert,
                                                          int32_t* num_blocks, TileOut to) {
  extern __shared__ int sm[];
  int* cnt = sm;              // [E]
  int* offs = cnt + E;        // [E + 1]
  int* tsc = offs + E + 1;    // [E + 1]
  pdl_wait();
  // per expert: exclusive prefix over chunks (in place), total count
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int64_t c = 0; c < n_chunks; ++c) {
      const int v = chunk_counts[c * E + e];
      chunk_counts[c * E + e] = run;
      run += v;
    }
    cnt[e] = run;
  }
  __syncthreads();
  block_finalize(cnt, E, bm, static_cast<int32_t>(T * k), offs, tsc, counts, offsets, sorted,
                 block_expert, num_blocks, to);
  pdl_launch_dependents();
}

__global__ void __launch_bounds__(kThreads) align_scatter_kernel(View2 ids, int64_t T, int64_t k,
                                                                 int64_t E,
                                                                 const int32_t* chunk_counts,
                                                                 const int32_t* offsets,
                                                                 int32_t* sorted, int32_t* inv) {
  extern __shared__ int sm[];
  int* base = sm;            // [E]
  int* warp_cnt = base + E;  // [kWarps * E]
  pdl_wait();
  const int64_t S = T * k;
  for (int i = threadIdx.x; i < E; i += blockDim.x)
    base[i] = offsets[i] + chunk_counts[blockIdx.x * E + i];
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) warp_cnt[i] = 0;
  __syncthreads();
  const int64_t s0 = static_cast<int64_t>(blockIdx.x) * kAlignChunk;
  const int64_t s1 = min(S, s0 + kAlignChunk);
  block_scatter(ids, k, E, s0, s1, base, warp_cnt, sorted, inv);
  pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_align(const View2& ids, int64_t T, int64_t k, int64_t E, int32_t bm,
                         int32_t* counts, int32_t* offsets, int32_t* sorted, int32_t* inv,
                         int32_t* block_expert, int32_t* num_blocks, int32_t* chunk_counts,
                         int64_t n_chunks, DeviceErrors* err, cudaStream_t st, int* launches,
                         const AlignTiles* tiles) {
  TileOut to;
  to.tile_max = tiles ? tiles->tile_max : 0;
  to.tile_row = tiles ? tiles->tile_row : nullptr;
  to.tile_rows = tiles ? tiles->tile_rows : nullptr;
  to.tile_expert = tiles ? tiles->tile_expert : nullptr;
  to.num_tiles = tiles ? tiles->num_tiles : nullptr;
  if (E > kMaxExperts) return cudaErrorInvalidValue;
  const int64_t S = T * k;
  cudaError_t rc;
  if (S <= kAlignSmallMax) {
    const size_t smem = sizeof(int) * (E * (kWarps + 4) + 2);
    if (smem > 48 * 1024) {
      rc = cudaFuncSetAttribute(align_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem);
      if (rc != cudaSuccess) return rc;
    }
    rc = launch_pdl(align_small_kernel, dim3(1), dim3(kThreads), smem, st, ids, T, k, E, bm,
                    counts, offsets, sorted, inv, block_expert, num_blocks, to, err);
    if (launches) *launches += 1;
    return rc;
  }
  const size_t smem_count = sizeof(int) * E;
  rc = launch_pdl(align_count_kernel, dim3((unsigned)n_chunks), dim3(kThreads), smem_count, st,
                  ids, T, k, E, chunk_counts, err);
  if (rc != cudaSuccess) return rc;
  const size_t smem_scan = sizeof(int) * (3 * E + 2);
  rc = launch_pdl(align_scan_kernel, dim3(1), dim3(1024), smem_scan, st, T, k, E, bm, n_chunks,
                  chunk_counts, counts, offsets, sorted, block_expert, num_blocks, to);
  if (rc != cudaSuccess) return rc;
  const size_t smem_sc = sizeof(int) * E * (kWarps + 1);
  if (smem_sc > 48 * 1024) {
    rc = cudaFuncSetAttribute(align_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem_sc);
    if (rc != cudaSuccess) return rc;
  }
  rc = launch_pdl(align_scatter_kernel, dim3((unsigned)n_chunks), dim3(kThreads), smem_sc, st, ids,
                  T, k, E, chunk_counts, offsets, sorted, inv);
  if (launches) *launches += 3;
  return rc;
}

}  // namespace moe
