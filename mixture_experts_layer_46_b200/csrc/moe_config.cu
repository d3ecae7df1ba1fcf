// Kernel configuration of the forward: which token-tile size and GEMM variant
// runs for a given problem shape and token count.
//
// The pages tune their fused-MoE kernels per shape and token bucket (aiter PR
// #3859, "Details": tuned configurations kept in a table keyed by the problem
// shape; "Tuned MoE latency": a different block_m per token bucket).  Here the
// choice is looked up, in order, in
//   1. the table a caller installed with moe_set_config_table (process-wide),
//   2. the table compiled into the library from the committed tuning results
//      (configs/b200_tuned.csv, turned into a C array at build time),
//   3. a heuristic on the average number of routing slots per expert.
// The first entry whose shape and token bucket match wins.  Every choice with
// an unsplit GEMM1 gives bit-identical results (the GEMMs sum each output in
// the same k order whatever the tiling); the one-kernel path's split GEMM1
// sums its K parts in fixed order (deterministic, rounded differently).
#include <mutex>
#include <vector>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

#include "moe_config_table.inc"  // kBuiltinConfigs[], kNumBuiltinConfigs (generated)

std::mutex g_cfg_mu;
std::vector<moe_config_t> g_cfg_table;

bool matches(const moe_config_t& c, int64_t T, int64_t H, int64_t I, int64_t E, int64_t k,
             bool mxfp4) {
  if ((c.wdtype == MOE_E2M1X2) != mxfp4) return false;
  if (c.H && c.H != H) return false;
  if (c.I && c.I != I) return false;
  if (c.E && c.E != E) return false;
  if (c.k && c.k != k) return false;
  return T >= c.t_lo && T <= c.t_hi;
}

bool tile_ok(int32_t tile, bool mxfp4) {
  return mxfp4 ? (tile == 32 || tile == 96 || tile == 128) : (tile == 32 || tile == 128 || tile == 256);
}

bool flag_ok(int32_t v) { return v == 0 || v == 1; }

bool entry_ok(const moe_config_t& c) {
  if (c.wdtype != MOE_BF16 && c.wdtype != MOE_E2M1X2) return false;
  if (c.H < 0 || c.I < 0 || c.E < 0 || c.k < 0 || c.t_lo < 0 || c.t_hi < c.t_lo) return false;
  if (!tile_ok(c.tile, c.wdtype == MOE_E2M1X2)) return false;
  return flag_ok(c.pair) && flag_ok(c.g1_256) && flag_ok(c.g2_single) && flag_ok(c.tiny) &&
         flag_ok(c.prefetch) && flag_ok(c.fused) && c.split >= 0 && c.split <= kDecodeMaxSplit &&
         (c.g1_il == 0 || c.g1_il == 256 || c.g1_il == 512);
}

// The measured defaults of the kernels when no table entry matches: 32-row
// token tiles while experts average at most 8 slots (decode: more weight bytes
// in flight per SM), else 128 rows (bf16) or 96 rows (MXFP4, where both
// accumulator buffers and the per-stage scales must fit in TMEM); bf16
// 128-row tiles on CTA pairs once experts average 32 slots, GEMM2 with one
// 256-row w2 slice per 256-row token tile, and GEMM1 on those 256-row tiles
// from 96 slots per expert.
moe_config_t heuristic(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, bool mxfp4) {
  moe_config_t c = {};
  c.wdtype = mxfp4 ? MOE_E2M1X2 : MOE_BF16;
  c.H = H;
  c.I = I;
  c.E = E;
  c.k = k;
  c.t_lo = T;
  c.t_hi = T;
  const int64_t S = T * k;
  const int64_t avg = E > 0 ? S / E : 0;
  c.tiny = S <= 32 ? 1 : 0;
  c.fused = S <= 32 ? 1 : 0;
  if (mxfp4) {
    c.tile = avg <= 8 ? 32 : 96;
    return c;
  }
  c.tile = avg <= 8 ? 32 : 128;
  c.pair = (c.tile == 128 && S >= 32 * E) ? 1 : 0;
  c.g2_single = c.pair;
  c.g1_256 = (c.g2_single && avg >= 96) ? 1 : 0;
  c.prefetch = (c.tile == 32 && S <= 32) ? 1 : 0;
  return c;
}

}  // namespace

moe_config_t select_config(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, bool mxfp4) {
  moe_config_t c = heuristic(T, H, I, E, k, mxfp4);
  bool found = false;
  {
    std::lock_guard<std::mutex> lk(g_cfg_mu);
    for (const moe_config_t& e : g_cfg_table)
      if (matches(e, T, H, I, E, k, mxfp4)) {
        c = e;
        found = true;
        break;
      }
  }
  if (!found) {
    for (int i = 0; i < kNumBuiltinConfigs; ++i)
      if (entry_ok(kBuiltinConfigs[i]) && matches(kBuiltinConfigs[i], T, H, I, E, k, mxfp4)) {
        c = kBuiltinConfigs[i];
        break;
      }
  }
  // what the kernels can run: flags that do not apply to the chosen tile are cleared
  const int64_t S = T * k;
  if (mxfp4) {
    c.pair = c.g1_256 = c.g2_single = c.prefetch = c.g1_il = 0;
  } else {
    if (c.g1_il) {
      // interleaved GEMM1 on the 256-row list (or its own 512-row list), GEMM2 on the 256-row list
      c.tile = 128;
      c.pair = c.g2_single = 1;
      c.g1_256 = 0;
    }
    if (c.tile == 256) c.pair = 1;  // 256-row token tiles exist only on CTA pairs
    if (c.tile == 32) c.pair = 0;
    if (!(c.pair && c.tile == 128)) c.g2_single = 0;
    if (!c.g2_single) c.g1_256 = 0;
    if (!(c.tile == 32 && S <= 32)) c.prefetch = 0;
  }
  if (S > 32) c.tiny = c.fused = 0;
  c.split = !c.fused ? 1 : (c.split == 0 ? kDecodeMaxSplit : c.split);
  return c;
}

}  // namespace moe

using namespace moe;

extern "C" {

moe_status_t moe_set_config_table(const moe_config_t* entries, int32_t n) {
  if (n < 0 || (n > 0 && !entries)) return MOE_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i)
    if (!entry_ok(entries[i])) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_cfg_mu);
  g_cfg_table.assign(entries, entries + n);
  return MOE_OK;
}

moe_status_t moe_get_config(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, int32_t wdtype,
                            moe_config_t* out) {
  if (!out || T < 0 || H < 1 || I < 1 || E < 1 || k < 1) return MOE_ERR_INVALID_ARG;
  if (wdtype != MOE_BF16 && wdtype != MOE_E2M1X2) return MOE_ERR_UNSUPPORTED_DTYPE;
  *out = select_config(T, H, I, E, k, wdtype == MOE_E2M1X2);
  return MOE_OK;
}

int32_t moe_builtin_config_count(void) { return kNumBuiltinConfigs; }

}  // extern "C"
