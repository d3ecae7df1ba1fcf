// Oracle for the fused mixture-of-experts expert forward.
//
// TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
// CPU statement of what the GPU path computes.  Only the test suite, the
// smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
// code, header, table or constant with the CUDA library: it reads the same
// seeded inputs and nothing else.
//
// Everything here is double precision.  Every element is read through its
// tensor's base pointer and strides, the way the pages insist a strided view
// must be read (LightLLM issue #1467, "Summary": a pass that drops a stride
// silently reads the wrong elements; prime-rl PR #2860, "Problem": a per-layer
// routing slice has token stride layers*top_k).
//
// What is computed (for every token t and every routing column j, in order):
//   e = topk_ids[t, j], w = topk_weights[t, j]            (slot skipped if e not in [0, E))
//   g_i = sum_h x[t, h] * gate[e, i, h]                    gate = w13[:, :I, :]
//   u_i = sum_h x[t, h] * up[e, i, h]                      up   = w13[:, I:, :]
//        (Liger-Kernel PR #1377, "Problems": packed w13 [experts, 2*intermediate, hidden])
//   a_i = silu(g_i) * u_i = g_i / (1 + exp(-g_i)) * u_i    (ROCm/aiter PR #3859, "Details": ActivationType.Silu)
//   y_o = sum_i a_i * w2[e, o, i]
//   out[t, o] += w * y_o
// In MXFP4 mode (aiter PR #3859, "Details": float4_e2m1fn_x2 weights and
// activations, QuantType.per_1x32) the weights are e2m1 codes with one e8m0
// scale per 32 consecutive elements along the contraction axis, dequantised by
// definition (value = e2m1(code) * 2^(scale - 127)); x is quantised with the
// same 1x32 rule along H and a is quantised along I before the down projection.
//
// Parity pins for this file live in tests/test_oracle_*.py (brute force,
// a dense formulation, special cases, invariants, worked MXFP4 examples).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// dtype codes understood by the oracle (its own numbering).
enum { OR_BF16 = 0, OR_F32 = 1, OR_I32 = 2, OR_I64 = 3, OR_E2M1X2 = 4 };

// A strided tensor view as the oracle sees it.  Strides are in elements of the
// storage type; for OR_E2M1X2 the storage element is one byte holding two codes
// (even logical element in the low nibble), so the innermost stride counts bytes
// and logical element k lives in byte k/2.  `scale` (MXFP4 only) holds one e8m0
// code per 32 logical elements of the innermost axis, addressed by scale_strides.
typedef struct {
  const void* data;
  int32_t dtype;
  int32_t ndim;
  int64_t sizes[4];
  int64_t strides[4];
  const uint8_t* scale;
  int64_t scale_strides[4];
} oracle_tensor_t;

}  // extern "C"

namespace {

double bf16_bits_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

// e2m1 (OCP MX v1.0 FP4): bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
// Exponent field 0 is subnormal: value = mantissa * 2^-1.
double e2m1_value(unsigned code) {
  unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
  double mag = (e == 0) ? 0.5 * (double)m : std::ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
  return s ? -mag : mag;
}

// e8m0 scale: value = 2^(code - 127); code 255 is NaN and never produced here.
double e8m0_value(unsigned code) { return std::ldexp(1.0, (int)code - 127); }

// Round |q| (already divided by the block scale) to the nearest e2m1 magnitude
// with ties to the even mantissa, saturating at 6.  Returns the 3-bit magnitude
// code; the e2m1 magnitudes in code order are 0, .5, 1, 1.5, 2, 3, 4, 6.
unsigned e2m1_round_magnitude(double m) {
  static const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  if (m >= 6.0) return 7u;
  unsigned i = 0;
  while (i < 7 && grid[i + 1] <= m) ++i;  // grid[i] <= m < grid[i+1]
  double lo = m - grid[i], hi = grid[i + 1] - m;
  if (lo < hi) return i;
  if (hi < lo) return i + 1;
  return (i & 1u) ? i + 1 : i;  // tie: the even mantissa bit wins
}

// One 1x32 block, OCP MX v1.0 rule for an FP4 (E2M1) element type:
//   shared exponent = floor(log2(amax)) - emax_elem, emax_elem = 2, clamped to [-127, 127];
//   element = round_to_nearest_even(v / 2^shared), saturated to the largest normal (6).
// amax == 0 gives scale code 0 and zero elements.
void mx_quantize_block(const double* v, int n, uint8_t* codes /*n nibble codes, one per byte*/,
                       uint8_t* scale_code) {
  double amax = 0.0;
  for (int i = 0; i < n; ++i) amax = std::max(amax, std::fabs(v[i]));
  if (amax == 0.0) {
    *scale_code = 0;
    for (int i = 0; i < n; ++i) codes[i] = std::signbit(v[i]) ? 8u : 0u;
    return;
  }
  int ex;
  std::frexp(amax, &ex);  // amax = f * 2^ex, f in [0.5, 1)  =>  floor(log2(amax)) = ex - 1
  int s = (ex - 1) - 2;
  s = std::min(127, std::max(-127, s));
  *scale_code = (uint8_t)(s + 127);
  for (int i = 0; i < n; ++i) {
    double q = std::ldexp(v[i], -s);
    unsigned mag = e2m1_round_magnitude(std::fabs(q));
    codes[i] = (uint8_t)(mag | (std::signbit(v[i]) ? 8u : 0u));
  }
}

// Element readers through strides.
inline const char* at(const oracle_tensor_t* t, int64_t i0, int64_t i1, int64_t i2, int esz) {
  int64_t off = i0 * t->strides[0] + i1 * t->strides[1] + (t->ndim > 2 ? i2 * t->strides[2] : 0);
  return (const char*)t->data + off * esz;
}

double read_real2(const oracle_tensor_t* t, int64_t i0, int64_t i1) {
  int64_t off = i0 * t->strides[0] + i1 * t->strides[1];
  if (t->dtype == OR_BF16) return bf16_bits_to_double(((const uint16_t*)t->data)[off]);
  return (double)((const float*)t->data)[off];
}

int64_t read_id(const oracle_tensor_t* t, int64_t i0, int64_t i1) {
  int64_t off = i0 * t->strides[0] + i1 * t->strides[1];
  if (t->dtype == OR_I64) return ((const int64_t*)t->data)[off];
  return (int64_t)((const int32_t*)t->data)[off];
}

// Weight element w[e, n, k] of a 3-D view, dequantised by definition in MXFP4 mode.
double read_weight(const oracle_tensor_t* t, int64_t e, int64_t n, int64_t k) {
  if (t->dtype == OR_BF16) {
    int64_t off = e * t->strides[0] + n * t->strides[1] + k * t->strides[2];
    return bf16_bits_to_double(((const uint16_t*)t->data)[off]);
  }
  if (t->dtype == OR_F32) {
    int64_t off = e * t->strides[0] + n * t->strides[1] + k * t->strides[2];
    return (double)((const float*)t->data)[off];
  }
  // OR_E2M1X2
  int64_t off = e * t->strides[0] + n * t->strides[1] + (k >> 1) * t->strides[2];
  uint8_t byte = ((const uint8_t*)t->data)[off];
  unsigned code = (k & 1) ? (byte >> 4) : (byte & 15u);
  int64_t soff = e * t->scale_strides[0] + n * t->scale_strides[1] + (k >> 5) * t->scale_strides[2];
  return e2m1_value(code) * e8m0_value(t->scale[soff]);
}

// Quantise-then-dequantise a vector in place with the 1x32 rule (n % 32 == 0).
void mx_fake_quant(std::vector<double>& v) {
  uint8_t codes[32], sc;
  for (size_t b = 0; b + 32 <= v.size(); b += 32) {
    mx_quantize_block(&v[b], 32, codes, &sc);
    for (int i = 0; i < 32; ++i) v[b + i] = e2m1_value(codes[i]) * e8m0_value(sc);
  }
}

}  // namespace

extern "C" {

// Value of one e2m1 code (low 4 bits), by the format definition.
double oracle_e2m1_value(uint32_t code) { return e2m1_value(code & 15u); }

// Quantise rows of a [R, K] fp32 matrix (row stride `rs` elements, unit inner
// stride) with the 1x32 MX rule.  codes: [R, K/2] bytes, two codes per byte, even
// element in the low nibble.  scales: [R, K/32] e8m0 codes.  K % 32 must be 0.
int oracle_mxfp4_quantize(const float* src, int64_t R, int64_t K, int64_t rs, uint8_t* codes,
                          uint8_t* scales) {
  if (K % 32 != 0) return 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t b = 0; b < K / 32; ++b) {
      double v[32];
      uint8_t c[32];
      for (int i = 0; i < 32; ++i) v[i] = (double)src[r * rs + b * 32 + i];
      mx_quantize_block(v, 32, c, &scales[r * (K / 32) + b]);
      for (int i = 0; i < 32; i += 2)
        codes[r * (K / 2) + b * 16 + i / 2] = (uint8_t)(c[i] | (c[i + 1] << 4));
    }
  }
  return 0;
}

// Stable grouping of token slots by expert (the "align" step).
//   slot s = t*k + j;  counts[e] = #{valid s : ids[s] == e}
//   padded_e = ceil(counts[e] / bm) * bm;  offsets[0] = 0, offsets[e+1] = offsets[e] + padded_e
//   sorted[offsets[e] + r] = the r-th slot of expert e in ascending slot order;
//   the padding positions of expert e hold the sentinel S = T*k;
//   block_expert[b] = e for every bm-row block b inside [offsets[e], offsets[e+1]).
// Block sizes that vary with the token count are what aiter PR #3859 tunes
// ("Tuned MoE latency" table, block_m column).  Ids outside [0, E) are skipped
// and counted in *n_bad.  sorted must hold offsets[E] entries, block_expert
// offsets[E]/bm entries; returns 1 if either is too short.
int oracle_moe_align(const oracle_tensor_t* ids, int64_t E, int64_t bm, int32_t* counts,
                     int32_t* offsets, int32_t* sorted, int64_t sorted_len, int32_t* block_expert,
                     int64_t be_len, int32_t* num_blocks, int64_t* n_bad) {
  const int64_t T = ids->sizes[0], k = ids->sizes[1], S = T * k;
  int64_t bad = 0;
  for (int64_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t s = 0; s < S; ++s) {
    int64_t e = read_id(ids, s / k, s % k);
    if (e < 0 || e >= E) { ++bad; continue; }
    counts[e]++;
  }
  offsets[0] = 0;
  for (int64_t e = 0; e < E; ++e) {
    int64_t padded = (counts[e] + bm - 1) / bm * bm;
    offsets[e + 1] = (int32_t)(offsets[e] + padded);
  }
  const int64_t P = offsets[E];
  if (P > sorted_len || P / bm > be_len) return 1;
  for (int64_t p = 0; p < P; ++p) sorted[p] = (int32_t)S;
  std::vector<int64_t> cursor(E, 0);
  for (int64_t s = 0; s < S; ++s) {
    int64_t e = read_id(ids, s / k, s % k);
    if (e < 0 || e >= E) continue;
    sorted[offsets[e] + cursor[e]++] = (int32_t)s;
  }
  for (int64_t e = 0; e < E; ++e)
    for (int64_t b = offsets[e] / bm; b < offsets[e + 1] / bm; ++b) block_expert[b] = (int32_t)e;
  *num_blocks = (int32_t)(P / bm);
  *n_bad = bad;
  return 0;
}

// The fused MoE expert forward in fp64 (definition in the file header).
//   x [T, H] bf16 or f32; gate, up [E, I, H] and w2 [E, H, I] bf16/f32, or e2m1x2
//   with e8m0 scales when mxfp4 != 0; ids [T, k] i32/i64; weights [T, k] f32.
//   tokens: optional list of n_out token indices (NULL: all T tokens, n_out = T).
//   out: [n_out, H] fp64, row r for token tokens[r].
// Returns 0, or 1 on a shape error.  *n_bad receives the number of skipped slots.
int oracle_moe_forward(const oracle_tensor_t* x, const oracle_tensor_t* gate,
                       const oracle_tensor_t* up, const oracle_tensor_t* w2,
                       const oracle_tensor_t* ids, const oracle_tensor_t* weights, int mxfp4,
                       const int64_t* tokens, int64_t n_out, double* out, int64_t* n_bad,
                       int nthreads) {
  const int64_t T = x->sizes[0], H = x->sizes[1];
  const int64_t E = gate->sizes[0], I = gate->sizes[1];
  const int64_t k = ids->sizes[1];
  if (gate->sizes[2] != H || up->sizes[0] != E || up->sizes[1] != I || up->sizes[2] != H ||
      w2->sizes[0] != E || w2->sizes[1] != H || w2->sizes[2] != I || ids->sizes[0] != T ||
      weights->sizes[0] != T || weights->sizes[1] != k)
    return 1;
  if (mxfp4 && (H % 32 != 0 || I % 32 != 0)) return 1;
  if (!tokens) n_out = T;
  int64_t bad = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
#endif
  for (int64_t r = 0; r < n_out; ++r) {
    const int64_t t = tokens ? tokens[r] : r;
    std::vector<double> xt(H), a(I), acc(H, 0.0);
    for (int64_t h = 0; h < H; ++h) xt[h] = read_real2(x, t, h);
    if (mxfp4) mx_fake_quant(xt);
    for (int64_t j = 0; j < k; ++j) {
      const int64_t e = read_id(ids, t, j);
      if (e < 0 || e >= E) { ++bad; continue; }
      const double w = read_real2(weights, t, j);
      for (int64_t i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int64_t h = 0; h < H; ++h) {
          g += xt[h] * read_weight(gate, e, i, h);
          u += xt[h] * read_weight(up, e, i, h);
        }
        a[i] = g / (1.0 + std::exp(-g)) * u;
      }
      if (mxfp4) mx_fake_quant(a);
      for (int64_t o = 0; o < H; ++o) {
        double y = 0.0;
        for (int64_t i = 0; i < I; ++i) y += a[i] * read_weight(w2, e, o, i);
        acc[o] += w * y;
      }
    }
    for (int64_t o = 0; o < H; ++o) out[r * H + o] = acc[o];
  }
  *n_bad = bad;
  return 0;
}

// Gradient of the forward with respect to x and topk_weights with the experts
// frozen (the routing ids are discrete), given dout = dL/dout, in the forward's
// order: for every token t and column j with e = topk_ids[t, j] in [0, E) and
// w = topk_weights[t, j]:
//   g, u, a, y as in the forward;  s_i = 1 / (1 + exp(-g_i))
//   dweights[t, j] = sum_o dout[t, o] * y_o
//   da_i = w * sum_o dout[t, o] * w2[e, o, i]
//   dg_i = da_i * u_i * s_i * (1 + g_i * (1 - s_i))      (the derivative of silu(g) = g s)
//   du_i = da_i * g_i * s_i
//   dx[t, h] += sum_i dg_i * gate[e, i, h] + du_i * up[e, i, h]
// Slots with e outside [0, E) contribute nothing (their dweights is 0).  bf16
// weights only (the MXFP4 forward's quantisation steps have no gradient).
//   dout [T, H] bf16/f32 (strided); dx [n_out, H] and dw [n_out, k] fp64, contiguous.
int oracle_moe_backward_input(const oracle_tensor_t* x, const oracle_tensor_t* gate,
                              const oracle_tensor_t* up, const oracle_tensor_t* w2,
                              const oracle_tensor_t* ids, const oracle_tensor_t* weights,
                              const oracle_tensor_t* dout, const int64_t* tokens, int64_t n_out,
                              double* dx, double* dw, int nthreads) {
  const int64_t T = x->sizes[0], H = x->sizes[1];
  const int64_t E = gate->sizes[0], I = gate->sizes[1];
  const int64_t k = ids->sizes[1];
  if (gate->sizes[2] != H || up->sizes[0] != E || up->sizes[1] != I || up->sizes[2] != H ||
      w2->sizes[0] != E || w2->sizes[1] != H || w2->sizes[2] != I || ids->sizes[0] != T ||
      weights->sizes[0] != T || weights->sizes[1] != k || dout->sizes[0] != T ||
      dout->sizes[1] != H || gate->dtype == OR_E2M1X2)
    return 1;
  if (!tokens) n_out = T;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t r = 0; r < n_out; ++r) {
    const int64_t t = tokens ? tokens[r] : r;
    std::vector<double> xt(H), dot(H), g(I), u(I), a(I), dgi(I), dui(I), acc(H, 0.0);
    for (int64_t h = 0; h < H; ++h) {
      xt[h] = read_real2(x, t, h);
      dot[h] = read_real2(dout, t, h);
    }
    for (int64_t j = 0; j < k; ++j) {
      dw[r * k + j] = 0.0;
      const int64_t e = read_id(ids, t, j);
      if (e < 0 || e >= E) continue;
      const double w = read_real2(weights, t, j);
      for (int64_t i = 0; i < I; ++i) {
        double gg = 0.0, uu = 0.0;
        for (int64_t h = 0; h < H; ++h) {
          gg += xt[h] * read_weight(gate, e, i, h);
          uu += xt[h] * read_weight(up, e, i, h);
        }
        g[i] = gg;
        u[i] = uu;
        a[i] = gg / (1.0 + std::exp(-gg)) * uu;
      }
      double dwj = 0.0;
      for (int64_t o = 0; o < H; ++o) {
        double y = 0.0;
        for (int64_t i = 0; i < I; ++i) y += a[i] * read_weight(w2, e, o, i);
        dwj += dot[o] * y;
      }
      dw[r * k + j] = dwj;
      for (int64_t i = 0; i < I; ++i) {
        double da = 0.0;
        for (int64_t o = 0; o < H; ++o) da += dot[o] * read_weight(w2, e, o, i);
        da *= w;
        const double sg = 1.0 / (1.0 + std::exp(-g[i]));
        dgi[i] = da * u[i] * sg * (1.0 + g[i] * (1.0 - sg));
        dui[i] = da * g[i] * sg;
      }
      for (int64_t h = 0; h < H; ++h) {
        double v = 0.0;
        for (int64_t i = 0; i < I; ++i)
          v += dgi[i] * read_weight(gate, e, i, h) + dui[i] * read_weight(up, e, i, h);
        acc[h] += v;
      }
    }
    for (int64_t h = 0; h < H; ++h) dx[r * H + h] = acc[h];
  }
  return 0;
}

// Gradient of the forward with respect to the expert weights, given dout, the
// routing fixed: for every token t and column j with e = topk_ids[t, j] in
// [0, E) and w = topk_weights[t, j], with g, u, a = silu(g) u, s, dg, du as in
// oracle_moe_backward_input:
//   dw2[e, o, i]   += w * dout[t, o] * a_i
//   dgate[e, i, h] += dg_i * x[t, h]
//   dup[e, i, h]   += du_i * x[t, h]
// (tokens in ascending order, columns in order).  bf16 weights only.
//   dgate, dup [E, I, H] and dw2 [E, H, I] fp64, contiguous, overwritten.
int oracle_moe_backward_weights(const oracle_tensor_t* x, const oracle_tensor_t* gate,
                                const oracle_tensor_t* up, const oracle_tensor_t* w2,
                                const oracle_tensor_t* ids, const oracle_tensor_t* weights,
                                const oracle_tensor_t* dout, double* dgate, double* dup,
                                double* dw2) {
  const int64_t T = x->sizes[0], H = x->sizes[1];
  const int64_t E = gate->sizes[0], I = gate->sizes[1];
  const int64_t k = ids->sizes[1];
  if (gate->sizes[2] != H || up->sizes[0] != E || up->sizes[1] != I || up->sizes[2] != H ||
      w2->sizes[0] != E || w2->sizes[1] != H || w2->sizes[2] != I || ids->sizes[0] != T ||
      weights->sizes[0] != T || weights->sizes[1] != k || dout->sizes[0] != T ||
      dout->sizes[1] != H || gate->dtype == OR_E2M1X2)
    return 1;
  std::fill(dgate, dgate + E * I * H, 0.0);
  std::fill(dup, dup + E * I * H, 0.0);
  std::fill(dw2, dw2 + E * H * I, 0.0);
  std::vector<double> xt(H), dot(H), g(I), u(I), a(I), dg(I), du(I);
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t h = 0; h < H; ++h) {
      xt[h] = read_real2(x, t, h);
      dot[h] = read_real2(dout, t, h);
    }
    for (int64_t j = 0; j < k; ++j) {
      const int64_t e = read_id(ids, t, j);
      if (e < 0 || e >= E) continue;
      const double w = read_real2(weights, t, j);
      for (int64_t i = 0; i < I; ++i) {
        double gg = 0.0, uu = 0.0;
        for (int64_t h = 0; h < H; ++h) {
          gg += xt[h] * read_weight(gate, e, i, h);
          uu += xt[h] * read_weight(up, e, i, h);
        }
        g[i] = gg;
        u[i] = uu;
        a[i] = gg / (1.0 + std::exp(-gg)) * uu;
      }
      for (int64_t o = 0; o < H; ++o)
        for (int64_t i = 0; i < I; ++i) dw2[(e * H + o) * I + i] += w * dot[o] * a[i];
      for (int64_t i = 0; i < I; ++i) {
        double da = 0.0;
        for (int64_t o = 0; o < H; ++o) da += dot[o] * read_weight(w2, e, o, i);
        da *= w;
        const double sg = 1.0 / (1.0 + std::exp(-g[i]));
        dg[i] = da * u[i] * sg * (1.0 + g[i] * (1.0 - sg));
        du[i] = da * g[i] * sg;
      }
      for (int64_t i = 0; i < I; ++i)
        for (int64_t h = 0; h < H; ++h) {
          dgate[(e * I + i) * H + h] += dg[i] * xt[h];
          dup[(e * I + i) * H + h] += du[i] * xt[h];
        }
    }
  }
  return 0;
}

// The router that produces the forward's routing inputs, in fp64:
//   p = softmax(logits[t, :]) over the E experts,
//   the k experts of largest p, in descending p (a tie goes to the lower expert index),
//   weights = those p, divided by their sum when `renormalize` is set.
// With `shared_expert` set the row gets one more column: expert E (the shared
// expert, which every token uses) with weight 1.0, the fused-shared-expert
// convention of aiter PR #3859 ("Summary": expert=513, topk=11 next to the
// unfused expert=512, topk=10).  The ids and weights are what the forward reads
// as topk_ids / topk_weights (prime-rl PR #2860, "Problem": the per-layer routing
// slice a router replay feeds the MoE forward).
//   logits [T, E] bf16/f32 (strided); ids [T, kk] int32, weights [T, kk] fp64, both
//   contiguous, kk = k + (shared_expert ? 1 : 0).  Returns 1 on bad arguments.
int oracle_router_topk(const oracle_tensor_t* logits, int64_t k, int renormalize,
                       int shared_expert, int32_t* ids, double* weights) {
  const int64_t T = logits->sizes[0], E = logits->sizes[1];
  if (k < 1 || k > E) return 1;
  const int64_t kk = k + (shared_expert ? 1 : 0);
  for (int64_t t = 0; t < T; ++t) {
    std::vector<double> l(E), p(E);
    double mx = -INFINITY;
    for (int64_t e = 0; e < E; ++e) {
      l[e] = read_real2(logits, t, e);
      mx = std::max(mx, l[e]);
    }
    double z = 0.0;
    for (int64_t e = 0; e < E; ++e) {
      p[e] = std::exp(l[e] - mx);
      z += p[e];
    }
    for (int64_t e = 0; e < E; ++e) p[e] /= z;
    std::vector<int64_t> order(E);
    for (int64_t e = 0; e < E; ++e) order[e] = e;
    std::stable_sort(order.begin(), order.end(),
                     [&](int64_t a, int64_t b) { return p[a] > p[b]; });
    double sel = 0.0;
    for (int64_t j = 0; j < k; ++j) sel += p[order[j]];
    for (int64_t j = 0; j < k; ++j) {
      ids[t * kk + j] = (int32_t)order[j];
      weights[t * kk + j] = renormalize ? p[order[j]] / sel : p[order[j]];
    }
    if (shared_expert) {
      ids[t * kk + k] = (int32_t)E;
      weights[t * kk + k] = 1.0;
    }
  }
  return 0;
}

// Value of one e8m0 scale code, by the format definition.
double oracle_e8m0_value(uint32_t code) { return e8m0_value(code & 255u); }

// Threads OpenMP would use (for reporting the CPU baseline's core count).
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
