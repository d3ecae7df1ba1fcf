// Work units of the single-kernel decode paths (moe_decode.cu, moe_decode_mx.cu):
// how GEMM1 is split along K and which item and k-range a unit index names.
#pragma once

#include "moe_internal.h"

namespace moe {

constexpr int kMaxSplitItems = 1024;  // GEMM1 items that can be split (counter slots)
static_assert(sizeof(DecodeSync::g1p) / sizeof(unsigned) == kMaxSplitItems, "split counters");

// GEMM1 K parts: with few routed experts the (expert, 128-row) items alone
// leave most SMs idle, so each is split along K.  The count minimises the
// longest CTA's GEMM1 time, ceil(units / CTAs) x (k-steps per part + a fixed
// cost per unit of about three k-steps: pipeline fill, the partials' round
// trip and the hand-off), with at least four k-steps per part.
__device__ __forceinline__ int split_count(int n1, int num_k1, int ctas, int max_split) {
  if (n1 <= 0 || n1 > kMaxSplitItems) return 1;
  int best = 1;
  long best_cost = static_cast<long>((n1 + ctas - 1) / ctas) * (num_k1 + 2) * 12;
  for (int ks = 2; ks <= max_split && ks <= kDecodeMaxSplit && num_k1 / ks >= 4; ++ks) {
    const long cost = static_cast<long>((n1 * ks + ctas - 1) / ctas) * (12 * num_k1 / ks + 36);
    if (cost < best_cost) { best = ks; best_cost = cost; }
  }
  return best;
}

// A work unit of the kernel: GEMM1 units (one k-range `part` of the item
// (routed expert r, 128 rows wt of I)) come first, then GEMM2 items.
struct Unit {
  bool g1;
  int r, wt, item, part, kb0, kb1;
};
__device__ __forceinline__ Unit unit_of(int u, int n1, int ks, int n_wt1, int n_wt2, int num_k1,
                                        int num_k2) {
  Unit x;
  if (u < n1 * ks) {
    x.g1 = true;
    x.part = u / n1;
    x.item = u - x.part * n1;
    x.r = x.item / n_wt1;
    x.wt = x.item - x.r * n_wt1;
    x.kb0 = x.part * num_k1 / ks;
    x.kb1 = (x.part + 1) * num_k1 / ks;
  } else {
    const int v = u - n1 * ks;
    x.g1 = false;
    x.r = v / n_wt2;
    x.wt = v - x.r * n_wt2;
    x.item = -1;
    x.part = 0;
    x.kb0 = 0;
    x.kb1 = num_k2;
  }
  return x;
}

}  // namespace moe
