// Router: the step just before the expert forward.  For every token t,
//   p = softmax(logits[t, :]) over the E experts,
//   the k experts of largest p in descending order (a tie goes to the lower index),
//   weights = those p, renormalised to sum to one when asked,
// written straight into the forward's topk_ids / topk_weights through their
// strides (e.g. the per-layer slice [:, l, :] of a [T, layers, k] routing
// replay tensor, prime-rl PR #2860, "Problem").  With the shared expert on, a
// last column holds expert E with weight 1.0: the fused-shared-expert routing
// of aiter PR #3859 ("Summary": expert=513, topk=11 next to the unfused
// expert=512, topk=10).
//
// One warp per token.  Lane l holds the logits of experts l, l + 32, ... in
// registers (coalesced row reads).  The selection never forms p: softmax is
// monotonic, so the k largest probabilities are the k largest logits.  Each of
// the k rounds takes the warp-wide maximum of an order-preserving integer key
// of the remaining logits (redux.sync max), then the lowest expert index
// holding it (redux.sync min), which is exactly the tie rule.  The weights are
// exp(l - l_max) over the chosen experts (or over all experts without
// renormalisation) divided by their sum, in fp32.
#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kRouterWarps = 8;

// Unsigned key ordering floats like their values; NaN ranks below every number
// and -0 is read as +0 (equal probabilities must tie).
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v != v) return 0u;
  const uint32_t b = __float_as_uint(v + 0.0f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

template <int kPer>  // logits per lane: E <= 32 * kPer
__global__ void __launch_bounds__(32 * kRouterWarps) router_topk_kernel(
    View2 logits, int64_t T, int E, int k, int renorm, int shared, View2 ids, View2 wts) {
  // the forward's first kernel waits for this grid to finish before it reads
  // the routing, so it may be scheduled at once
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kRouterWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  float v[kPer];
  uint32_t key[kPer];
  uint32_t taken = 0;  // bit i: expert lane + 32 i is chosen already or does not exist
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    v[i] = 0.0f;
    if (e < E) {
      const int64_t off = t * logits.s0 + static_cast<int64_t>(e) * logits.s1;
      v[i] = logits.dtype == MOE_F32
                 ? static_cast<const float*>(logits.data)[off]
                 : __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(logits.data)[off]) << 16);
    } else {
      taken |= 1u << i;
    }
    key[i] = order_key(v[i]);
  }
  int my_id = -1;
  uint32_t my_key = 0, top_key = 0;
  for (int r = 0; r < k; ++r) {
    uint32_t best = 0;
    int bidx = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      // strict > keeps the lower index among this lane's equal keys
      const bool cand = !((taken >> i) & 1u) && (bidx == 0x7fffffff || key[i] > best);
      if (cand) {
        best = key[i];
        bidx = lane + 32 * i;
      }
    }
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, bidx != 0x7fffffff ? best : 0u);
    const int sel = static_cast<int>(__reduce_min_sync(
        0xffffffffu, static_cast<unsigned>((bidx != 0x7fffffff && best == kmax) ? bidx : 0x7fffffff)));
    if ((sel & 31) == lane) taken |= 1u << (sel >> 5);
    if (lane == r) {
      my_id = sel;
      my_key = kmax;
    }
    if (r == 0) top_key = kmax;
  }
  const float m = key_value(top_key);
  const float ex = lane < k ? expf(key_value(my_key) - m) : 0.0f;
  float part = ex;
  if (!renorm) {
    part = 0.0f;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (lane + 32 * i < E) part += expf(v[i] - m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  const int kk = k + (shared ? 1 : 0);
  if (lane < kk) {
    const bool sh = lane == k;
    const int64_t id = sh ? E : my_id;
    const float w = sh ? 1.0f : ex / part;
    const int64_t io = t * ids.s0 + lane * ids.s1;
    if (ids.dtype == MOE_I64)
      static_cast<int64_t*>(const_cast<void*>(ids.data))[io] = id;
    else
      static_cast<int32_t*>(const_cast<void*>(ids.data))[io] = static_cast<int32_t>(id);
    static_cast<float*>(const_cast<void*>(wts.data))[t * wts.s0 + lane * wts.s1] = w;
  }
}

template <int kPer>
cudaError_t launch_router(const View2& logits, int64_t T, int E, int k, int renorm, int shared,
                          const View2& ids, const View2& wts, cudaStream_t st) {
  const int64_t blocks = (T + kRouterWarps - 1) / kRouterWarps;
  return launch_pdl(router_topk_kernel<kPer>, dim3(static_cast<unsigned>(blocks)),
                    dim3(32 * kRouterWarps), 0, st, logits, T, E, k, renorm, shared, ids, wts);
}

}  // namespace

cudaError_t launch_router_topk(const View2& logits, int64_t T, int E, int k, int renorm, int shared,
                               const View2& ids, const View2& wts, cudaStream_t st, int* launches) {
  if (launches) *launches += 1;
  const int per = (E + 31) / 32;
  if (per <= 1) return launch_router<1>(logits, T, E, k, renorm, shared, ids, wts, st);
  if (per <= 2) return launch_router<2>(logits, T, E, k, renorm, shared, ids, wts, st);
  if (per <= 4) return launch_router<4>(logits, T, E, k, renorm, shared, ids, wts, st);
  if (per <= 8) return launch_router<8>(logits, T, E, k, renorm, shared, ids, wts, st);
  if (per <= 16) return launch_router<16>(logits, T, E, k, renorm, shared, ids, wts, st);
  if (per <= 32) return launch_router<32>(logits, T, E, k, renorm, shared, ids, wts, st);
  return cudaErrorInvalidValue;
}

}  // namespace moe
