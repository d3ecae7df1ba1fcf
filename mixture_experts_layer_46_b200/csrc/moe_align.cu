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
// histograms and in-chunk ranks, one scan CTA, an element-wise scatter.  Ranks
// come from warps walking contiguous runs of slots, 32 at a time, with a
// ballot-built mask of the lanes sharing an expert, so a CTA needs only two
// block-wide barriers.
#include "../../include/moe.h"
#include "moe_internal.h"
#include "moe_mx.cuh"

namespace moe {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kSmallGroups = kAlignSmallMax / kThreads;  // 32-slot groups per warp, one CTA
constexpr int kChunkGroups = kAlignChunk / kThreads;     // 32-slot groups per warp, per chunk
static_assert(kAlignSmallMax % kThreads == 0 && kAlignChunk % kThreads == 0, "align tiling");

__device__ __forceinline__ int64_t read_id(const View2& v, int64_t s, int64_t k) {
  // slot counts are far below 2^31 (validated), so 32-bit division suffices
  const int64_t t = static_cast<int32_t>(s) / static_cast<int32_t>(k), j = s - t * k;
  const int64_t off = t * v.s0 + j * v.s1;
  if (v.dtype == MOE_I64) return static_cast<const int64_t*>(v.data)[off];
  return static_cast<int64_t>(static_cast<const int32_t*>(v.data)[off]);
}

// Lanes of the warp holding the same value v in [0, 2^nbits): one ballot per
// bit, each lane keeping the lanes that agree with it on that bit.  The same
// mask match.any returns, at a fraction of its cost for nbits <= 11.
__device__ __forceinline__ unsigned same_value_lanes(unsigned v, int nbits) {
  unsigned peers = 0xffffffffu;
  for (int b = 0; b < nbits; ++b) {
    const unsigned bit = (v >> b) & 1u;
    const unsigned bal = __ballot_sync(0xffffffffu, bit);
    peers &= bit ? bal : ~bal;
  }
  return peers;
}

// Stable ranks of the slots [s_begin, s_end) inside one CTA.  Warp w owns the
// contiguous run of per_warp slots starting at s_begin + w * per_warp (per_warp
// a multiple of 32, at most kG * 32) and walks it in 32-slot groups: lanes of a
// group that share an expert find each other (same_value_lanes), and the warp's
// running count of that expert (wcnt[w * E + e], zero on entry) gives the
// group's base.  On return e_reg[g] is the expert of the lane's slot in group g
// (-1: invalid or past the end), r_reg[g] its rank among the warp's slots of
// that expert, and wcnt holds the per-warp totals.  Returns the lane's count of
// ids outside [0, E).
template <int kG>
__device__ int warp_rank_slots(const View2& ids, int64_t k, int64_t E, int64_t s_begin,
                               int64_t s_end, int per_warp, int* wcnt, int (&e_reg)[kG],
                               int (&r_reg)[kG]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  const int64_t base = s_begin + static_cast<int64_t>(warp) * per_warp;
  int bad = 0;
#pragma unroll
  for (int g = 0; g < kG; ++g) {  // all loads first: one memory round trip
    const int64_t s = base + g * 32 + lane;
    int e = -1;
    if (g * 32 < per_warp && s < s_end) {
      const int64_t v = read_id(ids, s, k);
      if (v >= 0 && v < E)
        e = static_cast<int>(v);
      else
        ++bad;
    }
    e_reg[g] = e;
  }
  int* mine = wcnt + warp * E;
  const int nbits = 32 - __clz(static_cast<int>(E));  // e + 1 lies in [0, E]
#pragma unroll
  for (int g = 0; g < kG; ++g) {
    r_reg[g] = 0;
    if (g * 32 < per_warp) {  // uniform over the warp
      const int e = e_reg[g];
      const unsigned peers = same_value_lanes(static_cast<unsigned>(e + 1), nbits);
      const int c = e >= 0 ? mine[e] : 0;
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) mine[e] = c + __popc(peers);
      __syncwarp();
      r_reg[g] = c + __popc(peers & lt_mask);
    }
  }
  return bad;
}

// Per expert: exclusive prefix of the per-warp counts over warps (in place) and
// the CTA total in hist[e].
__device__ void warp_prefix(int64_t E, int* wcnt, int* hist) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < kWarps; ++w) {
      const int v = wcnt[w * E + e];
      wcnt[w * E + e] = run;
      run += v;
    }
    hist[e] = run;
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

// Outputs of align beyond sorted/offsets: up to two token-tile lists consumed
// by the weight-stationary GEMMs (tiles of at most tile_max rows, balanced
// within an expert, never crossing one), each written when its tile_max > 0.
struct TileList {
  int32_t tile_max;
  int32_t* tile_row;     // first padded row of the tile
  int32_t* tile_rows;    // rows in the tile (multiple of bm)
  int32_t* tile_expert;
  int32_t* num_tiles;
};
struct TileOut {
  TileList list[2];
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
  for (int li = 0; li < 2; ++li) {
    const TileList& tl = to.list[li];
    if (tl.tile_max <= 0) continue;
    const int tm = tl.tile_max;
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
        tl.tile_row[tsc[e] + j] = start;
        tl.tile_rows[tsc[e] + j] = u * bm;
        tl.tile_expert[tsc[e] + j] = e;
        start += u * bm;
      }
    }
    if (threadIdx.x == 0) *tl.num_tiles = nt;
  }
}

__global__ void __launch_bounds__(kThreads) align_small_kernel(
    View2 ids, int64_t T, int64_t k, int64_t E, int32_t bm, int32_t* counts, int32_t* offsets,
    int32_t* sorted, int32_t* inv, int32_t* block_expert, int32_t* num_blocks, TileOut to,
    DeviceErrors* err) {
  extern __shared__ int sm[];
  int* wcnt = sm;                    // [kWarps * E]
  int* hist = wcnt + kWarps * E;     // [E]
  int* offs = hist + E;              // [E + 1]
  int* tsc = offs + E + 1;           // [E + 1]
  __shared__ int bad_sh;
  // permute and, through it, the GEMM may be scheduled at once: both wait for
  // this kernel before reading what it writes
  pdl_launch_dependents();
  pdl_wait();
  const int64_t S = T * k;
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) wcnt[i] = 0;
  if (threadIdx.x == 0) bad_sh = 0;
  __syncthreads();
  const int per_warp = static_cast<int>((S + kThreads - 1) / kThreads) * 32;
  int e_reg[kSmallGroups], r_reg[kSmallGroups];
  const int bad = warp_rank_slots<kSmallGroups>(ids, k, E, 0, S, per_warp, wcnt, e_reg, r_reg);
  if (bad) atomicAdd(&bad_sh, bad);
  __syncthreads();
  warp_prefix(E, wcnt, hist);
  __syncthreads();
  block_finalize(hist, E, bm, static_cast<int32_t>(S), offs, tsc, counts, offsets, sorted,
                 block_expert, num_blocks, to);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t base = static_cast<int64_t>(warp) * per_warp;
#pragma unroll
  for (int g = 0; g < kSmallGroups; ++g) {
    const int64_t s = base + g * 32 + lane;
    if (g * 32 >= per_warp || s >= S) continue;
    const int e = e_reg[g];
    if (e >= 0) {
      const int pos = offs[e] + wcnt[warp * E + e] + r_reg[g];
      sorted[pos] = static_cast<int32_t>(s);
      inv[s] = pos;
    } else {
      inv[s] = -1;
    }
  }
  if (threadIdx.x == 0 && bad_sh && err) atomicAdd(&err->bad_ids, static_cast<unsigned>(bad_sh));
}

// Multi-CTA path, kernel 1: per chunk of kAlignChunk slots, the per-expert
// histogram (chunk_counts[c * E + e]) and each slot's stable rank inside its
// chunk and expert, parked in inv[s] (-1 for a skipped slot).
__global__ void __launch_bounds__(kThreads) align_count_kernel(View2 ids, int64_t T, int64_t k,
                                                               int64_t E, int32_t* chunk_counts,
                                                               int32_t* inv, DeviceErrors* err) {
  extern __shared__ int sm[];
  int* wcnt = sm;                 // [kWarps * E]
  int* hist = wcnt + kWarps * E;  // [E]
  __shared__ int bad_sh;
  pdl_wait();
  pdl_launch_dependents();
  const int64_t S = T * k;
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) wcnt[i] = 0;
  if (threadIdx.x == 0) bad_sh = 0;
  __syncthreads();
  const int64_t s0 = static_cast<int64_t>(blockIdx.x) * kAlignChunk;
  const int64_t s1 = min(S, s0 + kAlignChunk);
  constexpr int per_warp = kChunkGroups * 32;
  int e_reg[kChunkGroups], r_reg[kChunkGroups];
  const int bad = warp_rank_slots<kChunkGroups>(ids, k, E, s0, s1, per_warp, wcnt, e_reg, r_reg);
  if (bad) atomicAdd(&bad_sh, bad);
  __syncthreads();
  warp_prefix(E, wcnt, hist);
  __syncthreads();
  for (int i = threadIdx.x; i < E; i += blockDim.x) chunk_counts[blockIdx.x * E + i] = hist[i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t base = s0 + static_cast<int64_t>(warp) * per_warp;
#pragma unroll
  for (int g = 0; g < kChunkGroups; ++g) {
    const int64_t s = base + g * 32 + lane;
    if (s >= s1) continue;
    const int e = e_reg[g];
    inv[s] = e >= 0 ? wcnt[warp * E + e] + r_reg[g] : -1;
  }
  if (threadIdx.x == 0 && bad_sh && err) atomicAdd(&err->bad_ids, static_cast<unsigned>(bad_sh));
}

// Kernel 2 (one CTA): per expert, exclusive prefix of the chunk histograms
// over chunks (in place), then the counts, offsets, padding and tile list.
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
  pdl_launch_dependents();
  constexpr int kBatch = 8;  // independent loads in flight per thread
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int64_t c0 = 0; c0 < n_chunks; c0 += kBatch) {
      int v[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i)
        v[i] = c0 + i < n_chunks ? chunk_counts[(c0 + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        if (c0 + i < n_chunks) chunk_counts[(c0 + i) * E + e] = run;
        run += v[i];
      }
    }
    cnt[e] = run;
  }
  __syncthreads();
  block_finalize(cnt, E, bm, static_cast<int32_t>(T * k), offs, tsc, counts, offsets, sorted,
                 block_expert, num_blocks, to);
}

// Kernel 3: every slot independently: position = offset of its expert + the
// expert's slots in earlier chunks + its rank inside the chunk.
__global__ void __launch_bounds__(256) align_scatter_kernel(View2 ids, int64_t T, int64_t k,
                                                            int64_t E,
                                                            const int32_t* chunk_counts,
                                                            const int32_t* offsets,
                                                            int32_t* sorted, int32_t* inv) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t S = T * k;
  for (int64_t s = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; s < S;
       s += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int32_t r = inv[s];
    if (r < 0) continue;
    const int e = static_cast<int>(read_id(ids, s, k));
    const int pos = offsets[e] + chunk_counts[(s / kAlignChunk) * E + e] + r;
    sorted[pos] = static_cast<int32_t>(s);
    inv[s] = pos;
  }
}

// Decode batches (at most 32 slots, one CTA per token): align and permute in
// one kernel.  Warp 0 of every CTA groups the slots by expert with
// match/ballot instead of a histogram over all E experts: for a slot routed
// to expert e, its row is the padded rows of the routed experts below e plus
// its rank among the earlier slots of e.  CTA 0 writes align's outputs (the
// same values as the general kernels); every CTA copies its token's x row to
// the token's rows of a1 (kQuant: quantised to MXFP4 once, codes and scales
// written to each row, with the slot's routing weight in w_row, as permute_quant).
constexpr int kTinyThreads = 256;

template <bool kQuant>
__global__ void __launch_bounds__(kTinyThreads) align_permute_tiny_kernel(
    View2 ids, int64_t T, int64_t k, int64_t E, int32_t bm, int32_t* counts, int32_t* offsets,
    int32_t* sorted, int32_t* inv, int32_t* block_expert, int32_t* num_blocks, TileOut to,
    DeviceErrors* err, View2 x, int64_t H, void* a1, uint8_t* a1_scales, View2 topk_w,
    float* w_row, int vec_ok) {
  // routed experts in ascending order: id, slot count, first padded row (d_off[nd] = total rows)
  __shared__ int d_e[32], d_cnt[32], d_off[33], pos_sh[32];
  __shared__ int nd_sh;
  pdl_launch_dependents();
  pdl_wait();
  const int S = static_cast<int>(T * k);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool writer = blockIdx.x == 0;
  if (warp == 0) {
    int64_t id = -1;
    if (lane < S) id = read_id(ids, lane, k);
    const bool valid = lane < S && id >= 0 && id < E;
    const int key = valid ? static_cast<int>(id) : -1 - lane;  // skipped slots: distinct keys
    const unsigned same = __match_any_sync(0xffffffffu, key);
    const bool first = valid && (__ffs(same) - 1 == lane);
    const unsigned firsts = __ballot_sync(0xffffffffu, first);
    const unsigned bad = __ballot_sync(0xffffffffu, lane < S && !valid);
    int r = 0;  // routed experts below this slot's
    for (int j = 0; j < 32; ++j) {
      const int o = __shfl_sync(0xffffffffu, key, j);
      r += (((firsts >> j) & 1u) != 0u && o < key) ? 1 : 0;
    }
    const int nd = __popc(firsts);
    if (first) {
      d_e[r] = key;
      d_cnt[r] = __popc(same);
    }
    __syncwarp();
    // lane r < nd: padded rows of the r-th routed expert, scanned across lanes
    const int pr = lane < nd ? (d_cnt[lane] + bm - 1) / bm * bm : 0;
    int incl = pr;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane < nd) d_off[lane] = incl - pr;
    const int total_rows = __shfl_sync(0xffffffffu, incl, 31);
    if (lane == 0) {
      d_off[nd] = total_rows;
      nd_sh = nd;
    }
    __syncwarp();
    pos_sh[lane] = valid ? d_off[r] + __popc(same & ((1u << lane) - 1u)) : -1;
    __syncwarp();
    if (writer && lane < S) {
      inv[lane] = pos_sh[lane];
      if (valid) sorted[pos_sh[lane]] = lane;
    }
    if (writer && lane == 0 && bad && err) atomicAdd(&err->bad_ids, static_cast<unsigned>(__popc(bad)));
    if (writer) {
      // token-tile lists: lane r < nd holds the r-th routed expert's tiles
      for (int li = 0; li < 2; ++li) {
        const TileList& tl = to.list[li];
        if (tl.tile_max <= 0) continue;
        const int n = pr > 0 ? (pr + tl.tile_max - 1) / tl.tile_max : 0;
        int tincl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, tincl, o);
          if (lane >= o) tincl += v;
        }
        const int units = pr / bm;
        int start = lane < nd ? d_off[lane] : 0;
        for (int j = 0; j < n; ++j) {
          const int u = units / n + (j < units % n ? 1 : 0);
          tl.tile_row[tincl - n + j] = start;
          tl.tile_rows[tincl - n + j] = u * bm;
          tl.tile_expert[tincl - n + j] = d_e[lane];
          start += u * bm;
        }
        const int ntiles = __shfl_sync(0xffffffffu, tincl, 31);
        if (lane == 0) *tl.num_tiles = ntiles;
      }
    }
  }
  __syncthreads();
  const int nd = nd_sh;
  if (writer) {
    const int total = d_off[nd];
    for (int e = threadIdx.x; e <= E; e += blockDim.x) {
      int below = 0, c = 0;
      for (int r = 0; r < nd; ++r) {
        below += d_e[r] < e ? 1 : 0;
        if (d_e[r] == e) c = d_cnt[r];
      }
      offsets[e] = d_off[below];
      if (e < E) counts[e] = c;
    }
    if (threadIdx.x == 0) *num_blocks = total / bm;
    for (int p = threadIdx.x; p < total; p += blockDim.x) {
      int r = 0;
      while (r + 1 < nd && d_off[r + 1] <= p) ++r;
      if (p - d_off[r] >= d_cnt[r]) sorted[p] = S;
      if (p % bm == 0) block_expert[p / bm] = d_e[r];
    }
  }
  // this CTA's token: its x row to the rows of its valid slots
  const int64_t t = blockIdx.x;
  if (kQuant) {
    if (threadIdx.x < k && pos_sh[t * k + threadIdx.x] >= 0)
      w_row[pos_sh[t * k + threadIdx.x]] =
          static_cast<const float*>(topk_w.data)[t * topk_w.s0 + threadIdx.x * topk_w.s1];
    const int64_t nb = H / 32;
    uint8_t* codes = static_cast<uint8_t*>(a1);
    for (int64_t b = threadIdx.x; b < nb; b += blockDim.x) {
      float v[32];
      if (vec_ok) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x.data) + t * x.s0 + b * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 u = __ldg(src + q);
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            v[q * 8 + 2 * i] = __uint_as_float((w4[i] & 0xffffu) << 16);
            v[q * 8 + 2 * i + 1] = __uint_as_float(w4[i] & 0xffff0000u);
          }
        }
      } else {
        const uint16_t* src = static_cast<const uint16_t*>(x.data) + t * x.s0;
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(static_cast<uint32_t>(src[(b * 32 + i) * x.s1]) << 16);
      }
      uint32_t wq[4];
      const uint32_t sc = mx_quant32(v, wq);
      for (int j = 0; j < k; ++j) {
        const int p = pos_sh[t * k + j];
        if (p < 0) continue;
        *reinterpret_cast<uint4*>(codes + static_cast<int64_t>(p) * (H / 2) + b * 16) =
            make_uint4(wq[0], wq[1], wq[2], wq[3]);
        a1_scales[static_cast<int64_t>(p) * nb + b] = static_cast<uint8_t>(sc);
      }
    }
    return;
  }
  __nv_bfloat16* a1b = static_cast<__nv_bfloat16*>(a1);
  const int64_t H8 = H / 8;
  if (vec_ok) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x.data) + t * x.s0);
    for (int64_t c = threadIdx.x; c < H8; c += blockDim.x) {
      const uint4 v = __ldg(src + c);
      for (int j = 0; j < k; ++j) {
        const int p = pos_sh[t * k + j];
        if (p >= 0) reinterpret_cast<uint4*>(a1b + static_cast<int64_t>(p) * H)[c] = v;
      }
    }
  } else {
    const uint16_t* src = static_cast<const uint16_t*>(x.data) + t * x.s0;
    for (int64_t h = threadIdx.x; h < H; h += blockDim.x) {
      const uint16_t v = src[h * x.s1];
      for (int j = 0; j < k; ++j) {
        const int p = pos_sh[t * k + j];
        if (p >= 0) reinterpret_cast<uint16_t*>(a1b + static_cast<int64_t>(p) * H)[h] = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_align(const View2& ids, int64_t T, int64_t k, int64_t E, int32_t bm,
                         int32_t* counts, int32_t* offsets, int32_t* sorted, int32_t* inv,
                         int32_t* block_expert, int32_t* num_blocks, int32_t* chunk_counts,
                         int64_t n_chunks, DeviceErrors* err, cudaStream_t st, int* launches,
                         const AlignTiles* tiles) {
  TileOut to;
  for (int li = 0; li < 2; ++li) {
    TileList& tl = to.list[li];
    tl.tile_max = tiles ? tiles->list[li].tile_max : 0;
    tl.tile_row = tiles ? tiles->list[li].tile_row : nullptr;
    tl.tile_rows = tiles ? tiles->list[li].tile_rows : nullptr;
    tl.tile_expert = tiles ? tiles->list[li].tile_expert : nullptr;
    tl.num_tiles = tiles ? tiles->list[li].num_tiles : nullptr;
  }
  if (E > kMaxExperts) return cudaErrorInvalidValue;
  const int64_t S = T * k;
  cudaError_t rc;
  if (S <= kAlignSmallMax) {
    const size_t smem = sizeof(int) * (E * (kWarps + 3) + 2);
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
  const size_t smem_count = sizeof(int) * E * (kWarps + 1);
  if (smem_count > 48 * 1024) {
    rc = cudaFuncSetAttribute(align_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem_count);
    if (rc != cudaSuccess) return rc;
  }
  rc = launch_pdl(align_count_kernel, dim3((unsigned)n_chunks), dim3(kThreads), smem_count, st,
                  ids, T, k, E, chunk_counts, inv, err);
  if (rc != cudaSuccess) return rc;
  const size_t smem_scan = sizeof(int) * (3 * E + 2);
  rc = launch_pdl(align_scan_kernel, dim3(1), dim3(1024), smem_scan, st, T, k, E, bm, n_chunks,
                  chunk_counts, counts, offsets, sorted, block_expert, num_blocks, to);
  if (rc != cudaSuccess) return rc;
  int64_t sc_blocks = (S + 255) / 256;
  if (sc_blocks > 148 * 8) sc_blocks = 148 * 8;
  rc = launch_pdl(align_scatter_kernel, dim3((unsigned)sc_blocks), dim3(256), 0, st, ids, T, k, E,
                  chunk_counts, offsets, sorted, inv);
  if (launches) *launches += 3;
  return rc;
}

cudaError_t launch_align_permute_tiny(const View2& ids, int64_t T, int64_t k, int64_t E, int32_t bm,
                                      int32_t* counts, int32_t* offsets, int32_t* sorted,
                                      int32_t* inv, int32_t* block_expert, int32_t* num_blocks,
                                      DeviceErrors* err, const AlignTiles* tiles, const View2& x,
                                      int64_t H, void* a1, uint8_t* a1_scales, const View2* topk_w,
                                      float* w_row, cudaStream_t st, int* launches) {
  if (T * k > 32 || T * k < 1) return cudaErrorInvalidValue;
  const bool quant = a1_scales != nullptr;
  if (quant && (topk_w == nullptr || w_row == nullptr || k > kMaxTopK)) return cudaErrorInvalidValue;
  TileOut to;
  for (int li = 0; li < 2; ++li) {
    TileList& tl = to.list[li];
    tl.tile_max = tiles ? tiles->list[li].tile_max : 0;
    tl.tile_row = tiles ? tiles->list[li].tile_row : nullptr;
    tl.tile_rows = tiles ? tiles->list[li].tile_rows : nullptr;
    tl.tile_expert = tiles ? tiles->list[li].tile_expert : nullptr;
    tl.num_tiles = tiles ? tiles->list[li].num_tiles : nullptr;
  }
  const int vec_ok = (x.s1 == 1) && ((x.s0 * 2) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(x.data) % 16 == 0);
  if (launches) *launches += 1;
  const View2 tw = topk_w ? *topk_w : View2{nullptr, 0, 0, 0};
  if (quant)
    return launch_pdl(align_permute_tiny_kernel<true>, dim3(static_cast<unsigned>(T)), dim3(kTinyThreads),
                      0, st, ids, T, k, E, bm, counts, offsets, sorted, inv, block_expert, num_blocks,
                      to, err, x, H, a1, a1_scales, tw, w_row, vec_ok);
  return launch_pdl(align_permute_tiny_kernel<false>, dim3(static_cast<unsigned>(T)), dim3(kTinyThreads),
                    0, st, ids, T, k, E, bm, counts, offsets, sorted, inv, block_expert, num_blocks,
                    to, err, x, H, a1, a1_scales, tw, w_row, vec_ok);
}

}  // namespace moe
