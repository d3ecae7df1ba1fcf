// Host runtime behind include/moe.h: argument validation, workspace layout,
// TMA tensor-map encoding from each view's real strides, and the launch
// sequence align -> permute -> GEMM1(+SwiGLU) -> GEMM2(+routing weight) -> combine
// on the caller's stream (programmatic dependent launch between kernels).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {

// Device error counters: library memory, one copy per device, no allocation.
__device__ DeviceErrors g_device_errors;

namespace {

thread_local std::string t_last_cuda_error = "";
thread_local int32_t t_last_launches = 0;

// inspection captures requested with moe_debug_capture (per host thread)
struct Capture {
  void* ptr = nullptr;
  size_t bytes = 0;
};
thread_local Capture t_capture_h;

// per-thread step timing (moe_profile_enable / moe_profile_read)
constexpr int kProfSteps = 5;
struct Profiler {
  bool on = false;
  bool have = false;
  cudaEvent_t ev[kProfSteps + 1] = {};
  int n = 0;
};
thread_local Profiler t_prof;

void prof_mark(cudaStream_t st) {
  if (!t_prof.on || t_prof.n > kProfSteps) return;
  cudaEventRecord(t_prof.ev[t_prof.n++], st);
}

moe_status_t cuda_fail(cudaError_t rc, const char* where) {
  t_last_cuda_error = std::string(where) + ": " + cudaGetErrorName(rc) + " (" +
                      cudaGetErrorString(rc) + ")";
  return MOE_ERR_CUDA;
}

#define MOE_CUDA(call)                                   \
  do {                                                   \
    cudaError_t _rc = (call);                            \
    if (_rc != cudaSuccess) return cuda_fail(_rc, #call); \
  } while (0)

// ---------------------------------------------------------------- devices

struct DeviceInfo {
  bool init = false;
  bool ok = false;
  int num_sms = 0;
  DeviceErrors* errors = nullptr;
};

std::mutex g_dev_mu;
DeviceInfo g_dev[64];

moe_status_t device_info(DeviceInfo** out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MOE_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0;
    MOE_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    MOE_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    MOE_CUDA(cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev));
    d.ok = (major == 10 && minor == 0);
    void* p = nullptr;
    MOE_CUDA(cudaGetSymbolAddress(&p, g_device_errors));
    d.errors = static_cast<DeviceErrors*>(p);
    d.init = true;
  }
  if (!d.ok) return MOE_ERR_NO_DEVICE;
  *out = &d;
  return MOE_OK;
}

// ---------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// rank-2/3 K-major tile map: dims[0] is the contiguous (K) axis.
// Encoded maps are cached by everything the encoding depends on (base
// address, type, rank, sizes, strides, box, swizzle), so repeated calls on the
// same weights and workspace skip the host-side encoding.  The cache holds
// only keys and map bytes, never dereferences a cached address, and is cleared
// when it reaches kMapCacheMax entries.
struct MapKey {
  uintptr_t base;
  int32_t dt, rank, swz;
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  bool operator==(const MapKey& o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    // FNV-1a over the key bytes
    const unsigned char* p = reinterpret_cast<const unsigned char*>(&k);
    uint64_t h = 1469598103934665603ull;
    for (size_t i = 0; i < sizeof(MapKey); ++i) h = (h ^ p[i]) * 1099511628211ull;
    return static_cast<size_t>(h);
  }
};
constexpr size_t kMapCacheMax = 256;
std::mutex g_map_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;

moe_status_t make_map(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                      const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                      CUtensorMapSwizzle swz) {
  MapKey key;
  std::memset(&key, 0, sizeof(key));  // padding bytes take part in the comparison
  key.base = reinterpret_cast<uintptr_t>(base);
  key.dt = static_cast<int32_t>(dt);
  key.rank = rank;
  key.swz = static_cast<int32_t>(swz);
  for (int i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) key.strides[i] = strides_bytes[i];
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *map = it->second;
      return MOE_OK;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    t_last_cuda_error = "cuTensorMapEncodeTiled entry point unavailable";
    return MOE_ERR_CUDA;
  }
  cuuint64_t gd[3], gs[2];
  cuuint32_t bx[3], es[3];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(map, dt, rank, const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    snprintf(buf, sizeof(buf), "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    t_last_cuda_error = buf;
    return MOE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_map_mu);
  if (g_maps.size() >= kMapCacheMax) g_maps.clear();
  g_maps.emplace(key, *map);
  return MOE_OK;
}

// ---------------------------------------------------------------- validation

int64_t dtype_size(int32_t dt) {
  switch (dt) {
    case MOE_BF16: return 2;
    case MOE_F32: return 4;
    case MOE_I32: return 4;
    case MOE_I64: return 8;
    case MOE_E2M1X2: return 1;
    default: return 0;
  }
}

bool sizes_ok(const moe_tensor_t* t, int ndim) {
  if (!t || t->ndim != ndim) return false;
  for (int i = 0; i < ndim; ++i)
    if (t->sizes[i] < 0) return false;
  return true;
}

// Weight view [E, N, K] for TMA: unit inner stride, 16-byte aligned base and outer strides.
bool weight_layout_ok(const moe_tensor_t* w) {
  const int64_t es = dtype_size(w->dtype);
  if (w->strides[2] != 1) return false;
  if (reinterpret_cast<uintptr_t>(w->data) % 16 != 0) return false;
  if ((w->strides[1] * es) % 16 != 0 || (w->strides[0] * es) % 16 != 0) return false;
  if (w->strides[1] <= 0 || w->strides[0] < 0) return false;
  return true;
}

View2 view2(const moe_tensor_t* t) {
  View2 v;
  v.data = t->data;
  v.s0 = t->strides[0];
  v.s1 = t->strides[1];
  v.dtype = t->dtype;
  return v;
}

struct Problem {
  int64_t T, H, I, E, k;
  bool mxfp4;
};

moe_status_t validate(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                      const moe_tensor_t* ids, const moe_tensor_t* wts, const moe_tensor_t* out,
                      bool host_io, Problem* pr) {
  if (!x || !w13 || !w2 || !ids || !wts || !out) return MOE_ERR_INVALID_ARG;
  const moe_tensor_t* gate = &w13->gate;
  const moe_tensor_t* up = &w13->up;
  if (!sizes_ok(x, 2) || !sizes_ok(gate, 3) || !sizes_ok(up, 3) || !sizes_ok(w2, 3) ||
      !sizes_ok(ids, 2) || !sizes_ok(wts, 2) || !sizes_ok(out, 2))
    return MOE_ERR_INVALID_ARG;
  // dtypes
  if (x->dtype != MOE_BF16 || out->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (ids->dtype != MOE_I32 && ids->dtype != MOE_I64) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (wts->dtype != MOE_F32) return MOE_ERR_UNSUPPORTED_DTYPE;
  const int32_t wd = gate->dtype;
  if (wd != MOE_BF16 && wd != MOE_E2M1X2) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (up->dtype != wd || w2->dtype != wd) return MOE_ERR_UNSUPPORTED_DTYPE;
  // shapes (mismatched hidden dims fail here, before any descriptor is built)
  const int64_t T = x->sizes[0], H = x->sizes[1];
  const int64_t E = gate->sizes[0], I = gate->sizes[1];
  if (gate->sizes[2] != H || up->sizes[2] != H) return MOE_ERR_SHAPE_MISMATCH;
  if (up->sizes[0] != E || up->sizes[1] != I) return MOE_ERR_SHAPE_MISMATCH;
  if (w2->sizes[0] != E || w2->sizes[1] != H || w2->sizes[2] != I) return MOE_ERR_SHAPE_MISMATCH;
  if (ids->sizes[0] != T || wts->sizes[0] != T || wts->sizes[1] != ids->sizes[1])
    return MOE_ERR_SHAPE_MISMATCH;
  if (out->sizes[0] != T || out->sizes[1] != H) return MOE_ERR_SHAPE_MISMATCH;
  const int64_t k = ids->sizes[1];
  if (k < 1 || k > kMaxTopK) return MOE_ERR_INVALID_ARG;
  if (E < 1 || E > kMaxExperts || H < 1 || I < 1) return MOE_ERR_INVALID_ARG;
  if (H % 32 != 0 || I % 32 != 0) return MOE_ERR_SHAPE_MISMATCH;
  if (T * k >= (int64_t(1) << 30)) return MOE_ERR_INVALID_ARG;
  // pointers
  if ((T > 0 && (!x->data || !ids->data || !wts->data || !out->data)) || !gate->data ||
      !up->data || !w2->data)
    return MOE_ERR_INVALID_ARG;
  // layouts the copy engine must express
  if (!weight_layout_ok(gate) || !weight_layout_ok(up) || !weight_layout_ok(w2))
    return MOE_ERR_UNSUPPORTED_LAYOUT;
  if (wd == MOE_E2M1X2) {
    if (!gate->scale || !up->scale || !w2->scale) return MOE_ERR_INVALID_ARG;
    // scales are read 8 blocks (8 bytes) at a time per row and k-step
    for (const moe_tensor_t* t : {gate, up, w2}) {
      if (t->scale_strides[2] != 1 || t->scale_strides[1] % 8 != 0 ||
          t->scale_strides[0] % 8 != 0 || reinterpret_cast<uintptr_t>(t->scale) % 8 != 0)
        return MOE_ERR_UNSUPPORTED_LAYOUT;
    }
    // k-steps of 256 elements; GEMM1 column tiles of 64, GEMM2 column tiles of 128
    if (H % 256 != 0 || I % 256 != 0) return MOE_ERR_SHAPE_MISMATCH;
  }
  if (host_io) {
    if (x->strides[1] != 1 || ids->strides[1] != 1 || wts->strides[1] != 1 ||
        out->strides[1] != 1)
      return MOE_ERR_UNSUPPORTED_LAYOUT;
  }
  pr->T = T;
  pr->H = H;
  pr->I = I;
  pr->E = E;
  pr->k = k;
  pr->mxfp4 = (wd == MOE_E2M1X2);
  return MOE_OK;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

std::mutex g_ws_mu;
struct CachedWs {
  void* ptr = nullptr;
  size_t bytes = 0;
} g_ws[64];

moe_status_t cached_workspace(size_t need, void** ptr) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MOE_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_ws_mu);
  CachedWs& w = g_ws[dev];
  if (w.bytes < need) {
    if (w.ptr) {
      MOE_CUDA(cudaDeviceSynchronize());
      MOE_CUDA(cudaFree(w.ptr));
      w.ptr = nullptr;
      w.bytes = 0;
    }
    MOE_CUDA(cudaMalloc(&w.ptr, need));
    w.bytes = need;
  }
  *ptr = w.ptr;
  return MOE_OK;
}

}  // namespace

// ---------------------------------------------------------------- layout

// The workspace holds the token-tile lists of every configuration the forward
// can choose (32-row tiles give the longest list; the second list is the
// 256-row one of the bf16 CTA-pair GEMMs), so its size depends on the problem
// alone and never on the configuration table.
WsLayout make_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, bool mxfp4,
                     int32_t bm) {
  const int32_t tile_max = kMinTile;
  WsLayout L;
  std::memset(&L, 0, sizeof(L));
  L.T = T;
  L.H = H;
  L.I = I;
  L.E = E;
  L.k = k;
  L.S = T * k;
  L.bm = bm;
  L.tile_max = tile_max;
  L.mxfp4 = mxfp4;
  const int64_t S = L.S;
  const int64_t nonempty = S < E ? S : E;
  int64_t p = S + nonempty * (bm - 1);
  p = (p + bm - 1) / bm * bm;
  if (p < bm) p = bm;
  L.p_max = p;
  L.nb_max = p / bm;
  L.t_max = tile_max > 0 ? p / tile_max + nonempty + 1 : 0;
  // second token-tile list: 256-row tiles for the single-slice GEMM2 on CTA
  // pairs (bf16 with 128-row tiles)
  L.tile_max2 = !mxfp4 ? 256 : 0;
  L.t_max2 = L.tile_max2 > 0 ? p / L.tile_max2 + nonempty + 1 : 0;
  L.n_chunks = (S + kAlignChunk - 1) / kAlignChunk;
  if (L.n_chunks < 1) L.n_chunks = 1;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.counts = take(sizeof(int32_t) * E);
  L.offsets = take(sizeof(int32_t) * (E + 1));
  L.num_blocks = take(sizeof(int32_t) * 4);
  L.chunk_counts = take(S > kAlignSmallMax ? sizeof(int32_t) * L.n_chunks * E : 0);
  L.sorted = take(sizeof(int32_t) * p);
  L.inv = take(sizeof(int32_t) * (S > 0 ? S : 1));
  L.block_expert = take(sizeof(int32_t) * L.nb_max);
  L.tile_row = take(sizeof(int32_t) * L.t_max);
  L.tile_rows = take(sizeof(int32_t) * L.t_max);
  L.tile_expert = take(sizeof(int32_t) * L.t_max);
  L.tile_row2 = take(sizeof(int32_t) * L.t_max2);
  L.tile_rows2 = take(sizeof(int32_t) * L.t_max2);
  L.tile_expert2 = take(sizeof(int32_t) * L.t_max2);
  if (!mxfp4) {
    L.a1 = take(size_t(p) * H * 2);
    L.a1_scale = off;
    L.h = take(size_t(p) * I * 2);
    L.h_scale = off;
  } else {
    L.a1 = take(size_t(p) * H / 2);
    L.a1_scale = take(size_t(p) * H / 32);
    L.h = take(size_t(p) * I / 2);
    L.h_scale = take(size_t(p) * I / 32);
  }
  L.y = take(size_t(p) * H * 2);
  L.w_row = take(mxfp4 ? sizeof(float) * size_t(p) : 0);
  L.part = take(S <= 32 ? size_t(decode_part_bytes(I)) : 0);
  L.total = off;
  return L;
}

namespace {

// MXFP4: align -> permute+quantise -> block-scaled GEMM1 (+SwiGLU, requantise)
// -> block-scaled GEMM2 (+routing weight) -> combine.
moe_status_t forward_mxfp4(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                           const moe_tensor_t* ids, const moe_tensor_t* wts, moe_tensor_t* out,
                           const Problem& pr, const WsLayout& L, const moe_config_t& cfg,
                           uint8_t* w, DeviceInfo* dev, cudaStream_t st) {
  int launches = 0;
  int32_t* counts = reinterpret_cast<int32_t*>(w + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(w + L.offsets);
  int32_t* num_blocks = reinterpret_cast<int32_t*>(w + L.num_blocks);
  int32_t* chunk_counts = reinterpret_cast<int32_t*>(w + L.chunk_counts);
  int32_t* sorted = reinterpret_cast<int32_t*>(w + L.sorted);
  int32_t* inv = reinterpret_cast<int32_t*>(w + L.inv);
  int32_t* block_expert = reinterpret_cast<int32_t*>(w + L.block_expert);
  const moe_tensor_t* gate = &w13->gate;
  const moe_tensor_t* up = &w13->up;
  moe_status_t s;
  CUtensorMap mA1, mGate, mUp, mH, mW2;
  const uint32_t boxt[2] = {128, 32};
  const uint32_t boxw[3] = {128, 128, 1};
  {
    const uint64_t d[2] = {uint64_t(pr.H / 2), uint64_t(L.p_max)};
    const uint64_t sb[1] = {uint64_t(pr.H / 2)};
    s = make_map(&mA1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w + L.a1, d, sb, boxt,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
    // packed e2m1 views: strides are bytes; the expert stride is the view's real stride(0)
    const uint64_t d3[3] = {uint64_t(pr.H / 2), uint64_t(pr.I), uint64_t(pr.E)};
    const uint64_t sg[2] = {uint64_t(gate->strides[1]), uint64_t(gate->strides[0])};
    s = make_map(&mGate, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, gate->data, d3, sg, boxw,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
    const uint64_t su[2] = {uint64_t(up->strides[1]), uint64_t(up->strides[0])};
    s = make_map(&mUp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, up->data, d3, su, boxw,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
    const uint64_t dh[2] = {uint64_t(pr.I / 2), uint64_t(L.p_max)};
    const uint64_t sh[1] = {uint64_t(pr.I / 2)};
    s = make_map(&mH, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w + L.h, dh, sh, boxt,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
    const uint64_t dw[3] = {uint64_t(pr.I / 2), uint64_t(pr.H), uint64_t(pr.E)};
    const uint64_t sw[2] = {uint64_t(w2->strides[1]), uint64_t(w2->strides[0])};
    s = make_map(&mW2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w2->data, dw, sw, boxw,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
  }
  if (cfg.fused && L.S <= 32 && pr.H <= 16384) {
    // one kernel for decode sizes: h codes of each slot are gathered by TMA
    CUtensorMap mHc;
    const uint32_t box1[2] = {128, 1};
    const uint64_t dh[2] = {uint64_t(pr.I / 2), 32};
    const uint64_t sh[1] = {uint64_t(pr.I / 2)};
    s = make_map(&mHc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w + L.h, dh, sh, box1,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
    DecodeMxArgs dp;
    dp.T = pr.T;
    dp.H = pr.H;
    dp.I = pr.I;
    dp.E = pr.E;
    dp.k = pr.k;
    dp.ids = view2(ids);
    dp.topk_w = view2(wts);
    dp.x = view2(x);
    dp.gate_sf = static_cast<const uint8_t*>(gate->scale);
    dp.gate_s0 = gate->scale_strides[0];
    dp.gate_s1 = gate->scale_strides[1];
    dp.up_sf = static_cast<const uint8_t*>(up->scale);
    dp.up_s0 = up->scale_strides[0];
    dp.up_s1 = up->scale_strides[1];
    dp.w2_sf = static_cast<const uint8_t*>(w2->scale);
    dp.w2_s0 = w2->scale_strides[0];
    dp.w2_s1 = w2->scale_strides[1];
    dp.h_codes = w + L.h;
    dp.h_sf = w + L.h_scale;
    dp.y_ws = reinterpret_cast<__nv_bfloat16*>(w + L.y);
    dp.out = static_cast<__nv_bfloat16*>(out->data);
    dp.os0 = out->strides[0];
    dp.os1 = out->strides[1];
    dp.part_ws = reinterpret_cast<float*>(w + L.part);
    dp.max_split = cfg.split;
    dp.err = dev->errors;
    t_prof.n = 0;
    t_prof.have = false;
    prof_mark(st);
    const cudaError_t rc = launch_decode_fused_mx(mGate, mUp, mW2, mHc, dp, dev->num_sms, st, &launches);
    if (rc != cudaSuccess) return cuda_fail(rc, "decode_fused_mxfp4");
    for (int i = 0; i < kProfSteps; ++i) prof_mark(st);
    t_prof.have = t_prof.on && t_prof.n == kProfSteps + 1;
    t_last_launches = launches;
    return MOE_OK;
  }
  AlignTiles tiles;
  std::memset(&tiles, 0, sizeof(tiles));
  tiles.list[0].tile_max = cfg.tile;
  tiles.list[0].tile_row = reinterpret_cast<int32_t*>(w + L.tile_row);
  tiles.list[0].tile_rows = reinterpret_cast<int32_t*>(w + L.tile_rows);
  tiles.list[0].tile_expert = reinterpret_cast<int32_t*>(w + L.tile_expert);
  tiles.list[0].num_tiles = num_blocks + 1;
  t_prof.n = 0;
  t_prof.have = false;
  prof_mark(st);
  cudaError_t rc;
  // decode sizes (at most 32 slots): align and the quantising permute in one launch
  if (cfg.tiny) {
    const View2 tw = view2(wts);
    rc = launch_align_permute_tiny(view2(ids), pr.T, pr.k, pr.E, L.bm, counts, offsets, sorted, inv,
                                   block_expert, num_blocks, dev->errors, &tiles, view2(x), pr.H,
                                   w + L.a1, w + L.a1_scale, &tw,
                                   reinterpret_cast<float*>(w + L.w_row), st, &launches);
    if (rc != cudaSuccess) return cuda_fail(rc, "align_permute_quant");
    prof_mark(st);
  } else {
    rc = launch_align(view2(ids), pr.T, pr.k, pr.E, L.bm, counts, offsets, sorted, inv,
                      block_expert, num_blocks, chunk_counts, L.n_chunks, dev->errors,
                      st, &launches, &tiles);
    if (rc != cudaSuccess) return cuda_fail(rc, "align");
    prof_mark(st);
    rc = launch_permute_quant(view2(x), pr.T, pr.H, pr.k, inv, w + L.a1, w + L.a1_scale, view2(wts),
                              reinterpret_cast<float*>(w + L.w_row), st, &launches);
    if (rc != cudaSuccess) return cuda_fail(rc, "permute_quant");
  }
  prof_mark(st);
  WsGemmMx g1;
  std::memset(&g1, 0, sizeof(g1));
  g1.K = pr.H;
  g1.N = pr.I;
  g1.n_wt = pr.I / 128;
  g1.max_tiles = L.t_max;
  g1.num_tiles = tiles.list[0].num_tiles;
  g1.tile_row = tiles.list[0].tile_row;
  g1.tile_rows = tiles.list[0].tile_rows;
  g1.tile_expert = tiles.list[0].tile_expert;
  g1.sorted = sorted;
  g1.S = L.S;
  g1.out = w + L.h;
  g1.out_ld = pr.I / 2;
  g1.out_sf = w + L.h_scale;
  g1.out_sf_ld = pr.I / 32;
  g1.k = pr.k;
  g1.x_sf = w + L.a1_scale;
  g1.x_sf_ld = pr.H / 32;
  g1.w0_sf = static_cast<const uint8_t*>(gate->scale);
  g1.w0_s0 = gate->scale_strides[0];
  g1.w0_s1 = gate->scale_strides[1];
  g1.w1_sf = static_cast<const uint8_t*>(up->scale);
  g1.w1_s0 = up->scale_strides[0];
  g1.w1_s1 = up->scale_strides[1];
  g1.err = dev->errors;
  if (t_capture_h.ptr && t_capture_h.bytes >= sizeof(float) * size_t(L.p_max) * size_t(pr.I))
    g1.h_capture = static_cast<float*>(t_capture_h.ptr);
  // raw e8m0 scale maps for the GEMMs' TMA scale path, where every view it reads is
  // 16-byte aligned (base and strides); otherwise the GEMM copies scales with cp.async
  auto a16 = [](const void* ptr, int64_t s0, int64_t s1) {
    return reinterpret_cast<uintptr_t>(ptr) % 16 == 0 && s0 % 16 == 0 && s1 % 16 == 0;
  };
  CUtensorMap sf1[3], sf2[3];
  bool sf1_ok = a16(gate->scale, gate->scale_strides[0], gate->scale_strides[1]) &&
                a16(up->scale, up->scale_strides[0], up->scale_strides[1]) &&
                a16(w + L.a1_scale, pr.H / 32, 0);
  bool sf2_ok = a16(w2->scale, w2->scale_strides[0], w2->scale_strides[1]) &&
                a16(w + L.h_scale, pr.I / 32, 0);
  {
    const uint32_t boxw[3] = {16, 128, 1};
    const uint32_t boxt[2] = {16, static_cast<uint32_t>(cfg.tile)};
    if (sf1_ok) {
      const uint64_t d3[3] = {uint64_t(pr.H / 32), uint64_t(pr.I), uint64_t(pr.E)};
      const uint64_t sg[2] = {uint64_t(gate->scale_strides[1]), uint64_t(gate->scale_strides[0])};
      const uint64_t su[2] = {uint64_t(up->scale_strides[1]), uint64_t(up->scale_strides[0])};
      const uint64_t dx[2] = {uint64_t(pr.H / 32), uint64_t(L.p_max)};
      const uint64_t sx[1] = {uint64_t(pr.H / 32)};
      s = make_map(&sf1[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, gate->scale, d3, sg, boxw, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (s == MOE_OK)
        s = make_map(&sf1[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, up->scale, d3, su, boxw, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (s == MOE_OK)
        s = make_map(&sf1[2], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w + L.a1_scale, dx, sx, boxt, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (s != MOE_OK) return s;
    }
    if (sf2_ok) {
      const uint64_t d3[3] = {uint64_t(pr.I / 32), uint64_t(pr.H), uint64_t(pr.E)};
      const uint64_t sw[2] = {uint64_t(w2->scale_strides[1]), uint64_t(w2->scale_strides[0])};
      const uint64_t dh[2] = {uint64_t(pr.I / 32), uint64_t(L.p_max)};
      const uint64_t sh[1] = {uint64_t(pr.I / 32)};
      s = make_map(&sf2[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, w2->scale, d3, sw, boxw, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (s == MOE_OK)
        s = make_map(&sf2[2], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w + L.h_scale, dh, sh, boxt, CU_TENSOR_MAP_SWIZZLE_NONE);
      if (s != MOE_OK) return s;
      sf2[1] = sf2[0];
    }
  }
  rc = launch_gemm_ws_mxfp4(0, cfg.tile, mGate, mUp, mA1, sf1_ok ? sf1 : nullptr, g1, dev->num_sms, st,
                            &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "gemm1_mxfp4");
  prof_mark(st);
  WsGemmMx g2 = g1;
  g2.K = pr.I;
  g2.N = pr.H;
  g2.n_wt = pr.H / 256;
  g2.out = w + L.y;
  g2.out_ld = pr.H;
  g2.out_sf = nullptr;
  g2.out_sf_ld = 0;
  g2.topk_w = view2(wts);
  g2.x_sf = w + L.h_scale;
  g2.x_sf_ld = pr.I / 32;
  g2.w0_sf = static_cast<const uint8_t*>(w2->scale);
  g2.w0_s0 = w2->scale_strides[0];
  g2.w0_s1 = w2->scale_strides[1];
  g2.w1_sf = g2.w0_sf;
  g2.w1_s0 = g2.w0_s0;
  g2.w1_s1 = g2.w0_s1;
  g2.w_row = reinterpret_cast<const float*>(w + L.w_row);
  g2.h_capture = nullptr;
  rc = launch_gemm_ws_mxfp4(1, cfg.tile, mW2, mW2, mH, sf2_ok ? sf2 : nullptr, g2, dev->num_sms, st,
                            &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "gemm2_mxfp4");
  prof_mark(st);
  rc = launch_combine(reinterpret_cast<const __nv_bfloat16*>(w + L.y), inv, pr.T, pr.H, pr.k,
                      out->data, out->strides[0], out->strides[1], st, &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "combine");
  prof_mark(st);
  t_prof.have = t_prof.on && t_prof.n == kProfSteps + 1;
  t_last_launches = launches;
  return MOE_OK;
}

moe_status_t forward_impl(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                          const moe_tensor_t* ids, const moe_tensor_t* wts, moe_tensor_t* out,
                          const Problem& pr, void* ws, size_t ws_bytes, cudaStream_t st) {
  int launches = 0;
  t_last_launches = 0;
  if (pr.T == 0) return MOE_OK;
  const int32_t bm = kBm;
  const moe_config_t cfg = select_config(pr.T, pr.H, pr.I, pr.E, pr.k, pr.mxfp4);
  const WsLayout L = make_layout(pr.T, pr.H, pr.I, pr.E, pr.k, pr.mxfp4, bm);
  if (!ws || ws_bytes < L.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  moe_status_t s = device_info(&dev);
  if (s != MOE_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* counts = reinterpret_cast<int32_t*>(w + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(w + L.offsets);
  int32_t* num_blocks = reinterpret_cast<int32_t*>(w + L.num_blocks);
  int32_t* chunk_counts = reinterpret_cast<int32_t*>(w + L.chunk_counts);
  int32_t* sorted = reinterpret_cast<int32_t*>(w + L.sorted);
  int32_t* inv = reinterpret_cast<int32_t*>(w + L.inv);
  int32_t* block_expert = reinterpret_cast<int32_t*>(w + L.block_expert);

  const moe_tensor_t* gate = &w13->gate;
  const moe_tensor_t* up = &w13->up;

  if (pr.mxfp4) return forward_mxfp4(x, w13, w2, ids, wts, out, pr, L, cfg, w, dev, st);

  // ---- tensor maps (bf16, 128-byte swizzle): weights in [64 x 128] boxes,
  // expert-grouped token rows in one box per CTA and token tile
  CUtensorMap mA1, mGate, mUp, mH, mW2, mGate64, mUp64;
  // the configuration: token-tile rows (32 / 128 on one CTA, 128 / 256 on CTA
  // pairs, which move a sixth fewer shared-memory bytes per FLOP); GEMM2 on
  // pairs with one 256-row w2 slice per 256-row token tile (align's second
  // list: two accumulator buffers still fit in TMEM); GEMM1 on those 256-row
  // tiles (halved weight re-reads against an epilogue that is not overlapped)
  const int32_t tile = cfg.tile;
  const bool pair = cfg.pair != 0;
  const bool g2_single = cfg.g2_single != 0;
  const bool g1_256 = cfg.g1_256 != 0;
  // GEMM1 with gate and up interleaved in one accumulator: 256-row token tiles
  // (align's second list, as GEMM2's) or 512-row tiles (their own list); 32-row
  // token boxes (a tile's last MMA chunk is often short)
  const int32_t g1_il = cfg.g1_il;
  const int32_t wpolicy = 0;
  const uint32_t boxw[3] = {64, 128, 1};
  // one TMA box covers a CTA's share of a token tile
  const uint32_t tok_box = pair ? static_cast<uint32_t>(tile / 2) : static_cast<uint32_t>(tile);
  const uint32_t boxt2[2] = {64, g2_single ? 128u : tok_box};
  const uint32_t boxt1[2] = {64, g1_il ? 32u : (g1_256 ? 128u : tok_box)};
  {
    const uint64_t d[2] = {uint64_t(pr.H), uint64_t(L.p_max)};
    const uint64_t sb[1] = {uint64_t(pr.H) * 2};
    s = make_map(&mA1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w + L.a1, d, sb, boxt1,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
  }
  {
    // expert stride = the view's real stride(0): the first tile of expert e is
    // base + e * stride(0), whatever lies between experts (e.g. the up half).
    const uint64_t d[3] = {uint64_t(pr.H), uint64_t(pr.I), uint64_t(pr.E)};
    const uint64_t sg[2] = {uint64_t(gate->strides[1]) * 2, uint64_t(gate->strides[0]) * 2};
    s = make_map(&mGate, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, gate->data, d, sg, boxw,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
    const uint64_t su[2] = {uint64_t(up->strides[1]) * 2, uint64_t(up->strides[0]) * 2};
    s = make_map(&mUp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, up->data, d, su, boxw,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
    if (g1_il) {
      const uint32_t box64[3] = {64, 64, 1};
      s = make_map(&mGate64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, gate->data, d, sg, box64,
                   CU_TENSOR_MAP_SWIZZLE_128B);
      if (s != MOE_OK) return s;
      s = make_map(&mUp64, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, up->data, d, su, box64,
                   CU_TENSOR_MAP_SWIZZLE_128B);
      if (s != MOE_OK) return s;
    }
  }
  {
    const uint64_t d[2] = {uint64_t(pr.I), uint64_t(L.p_max)};
    const uint64_t sb[1] = {uint64_t(pr.I) * 2};
    s = make_map(&mH, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w + L.h, d, sb, boxt2,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
    const uint64_t d3[3] = {uint64_t(pr.I), uint64_t(pr.H), uint64_t(pr.E)};
    const uint64_t s3[2] = {uint64_t(w2->strides[1]) * 2, uint64_t(w2->strides[0]) * 2};
    s = make_map(&mW2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, w2->data, d3, s3, boxw,
                 CU_TENSOR_MAP_SWIZZLE_128B);
    if (s != MOE_OK) return s;
  }

  // ---- one kernel for decode sizes, when x can be gathered row by row with TMA
  const bool x_rows_ok = x->strides[1] == 1 && (x->strides[0] * 2) % 16 == 0 &&
                         reinterpret_cast<uintptr_t>(x->data) % 16 == 0 && x->strides[0] > 0;
  if (cfg.fused && L.S <= 32 && x_rows_ok && pr.H <= 16384) {
    CUtensorMap mX1, mH1;
    const uint32_t box1[2] = {64, 1};
    {
      const uint64_t d[2] = {uint64_t(pr.H), uint64_t(pr.T)};
      const uint64_t sb[1] = {uint64_t(x->strides[0]) * 2};
      s = make_map(&mX1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x->data, d, sb, box1,
                   CU_TENSOR_MAP_SWIZZLE_128B);
      if (s != MOE_OK) return s;
      const uint64_t dh[2] = {uint64_t(pr.I), 32};
      const uint64_t sh[1] = {uint64_t(pr.I) * 2};
      s = make_map(&mH1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w + L.h, dh, sh, box1,
                   CU_TENSOR_MAP_SWIZZLE_128B);
      if (s != MOE_OK) return s;
    }
    DecodeArgs dp;
    dp.T = pr.T;
    dp.H = pr.H;
    dp.I = pr.I;
    dp.E = pr.E;
    dp.k = pr.k;
    dp.ids = view2(ids);
    dp.topk_w = view2(wts);
    dp.h_ws = reinterpret_cast<__nv_bfloat16*>(w + L.h);
    dp.y_ws = reinterpret_cast<__nv_bfloat16*>(w + L.y);
    dp.out = static_cast<__nv_bfloat16*>(out->data);
    dp.os0 = out->strides[0];
    dp.os1 = out->strides[1];
    dp.part_ws = reinterpret_cast<float*>(w + L.part);
    dp.max_split = cfg.split;
    dp.err = dev->errors;
    t_prof.n = 0;
    t_prof.have = false;
    prof_mark(st);
    cudaError_t rc = launch_decode_fused(mGate, mUp, mW2, mX1, mH1, dp, dev->num_sms, st, &launches);
    if (rc != cudaSuccess) return cuda_fail(rc, "decode_fused");
    // one kernel: its time is reported as the first step's, the others as zero
    for (int i = 0; i < kProfSteps; ++i) prof_mark(st);
    t_prof.have = t_prof.on && t_prof.n == kProfSteps + 1;
    t_last_launches = launches;
    return MOE_OK;
  }

  // ---- launches
  AlignTiles tiles;
  std::memset(&tiles, 0, sizeof(tiles));
  tiles.list[0].tile_max = g1_il == 512 ? 512 : tile;
  tiles.list[0].tile_row = reinterpret_cast<int32_t*>(w + L.tile_row);
  tiles.list[0].tile_rows = reinterpret_cast<int32_t*>(w + L.tile_rows);
  tiles.list[0].tile_expert = reinterpret_cast<int32_t*>(w + L.tile_expert);
  tiles.list[0].num_tiles = num_blocks + 1;
  if (g2_single) {
    tiles.list[1].tile_max = 256;
    tiles.list[1].tile_row = reinterpret_cast<int32_t*>(w + L.tile_row2);
    tiles.list[1].tile_rows = reinterpret_cast<int32_t*>(w + L.tile_rows2);
    tiles.list[1].tile_expert = reinterpret_cast<int32_t*>(w + L.tile_expert2);
    tiles.list[1].num_tiles = num_blocks + 2;
  }
  t_prof.n = 0;
  t_prof.have = false;
  prof_mark(st);
  cudaError_t rc;
  // decode sizes (at most 32 slots): align and permute in one launch
  if (cfg.tiny) {
    rc = launch_align_permute_tiny(view2(ids), pr.T, pr.k, pr.E, bm, counts, offsets, sorted, inv,
                                   block_expert, num_blocks, dev->errors, &tiles, view2(x), pr.H,
                                   w + L.a1, nullptr, nullptr, nullptr, st, &launches);
    if (rc != cudaSuccess) return cuda_fail(rc, "align_permute");
    prof_mark(st);
  } else {
    rc = launch_align(view2(ids), pr.T, pr.k, pr.E, bm, counts, offsets, sorted, inv, block_expert,
                      num_blocks, chunk_counts, L.n_chunks, dev->errors, st, &launches, &tiles);
    if (rc != cudaSuccess) return cuda_fail(rc, "align");
    prof_mark(st);
    rc = launch_permute_bf16(view2(x), pr.T, pr.H, pr.k, inv,
                             reinterpret_cast<__nv_bfloat16*>(w + L.a1), st, &launches);
    if (rc != cudaSuccess) return cuda_fail(rc, "permute");
  }
  prof_mark(st);

  WsGemm g1;
  std::memset(&g1, 0, sizeof(g1));
  g1.K = pr.H;
  g1.N = pr.I;
  g1.n_wt = pair ? (pr.I + 255) / 256 : (pr.I + 127) / 128;
  g1.max_tiles = L.t_max;
  g1.num_tiles = tiles.list[0].num_tiles;
  g1.tile_row = tiles.list[0].tile_row;
  g1.tile_rows = tiles.list[0].tile_rows;
  g1.tile_expert = tiles.list[0].tile_expert;
  g1.sorted = sorted;
  g1.S = L.S;
  g1.out = w + L.h;
  g1.out_ld = pr.I;
  g1.k = pr.k;
  g1.err = dev->errors;
  g1.weights_evict_first = wpolicy;
  g1.tok_box = static_cast<int32_t>(tok_box);
  // decode sizes: GEMM1 finds its experts from the routing ids and requests
  // weights while align and permute run
  if (cfg.prefetch) {
    g1.pre_ids = view2(ids);
    g1.pre_E = static_cast<int32_t>(pr.E);
    g1.pre_S = static_cast<int32_t>(L.S);
  }
  if (g1_256) {
    g1.max_tiles = L.t_max2;
    g1.num_tiles = tiles.list[1].num_tiles;
    g1.tile_row = tiles.list[1].tile_row;
    g1.tile_rows = tiles.list[1].tile_rows;
    g1.tile_expert = tiles.list[1].tile_expert;
    g1.tok_box = 128;
  }
  if (g1_il) {
    if (g1_il == 256) {
      g1.max_tiles = L.t_max2;
      g1.num_tiles = tiles.list[1].num_tiles;
      g1.tile_row = tiles.list[1].tile_row;
      g1.tile_rows = tiles.list[1].tile_rows;
      g1.tile_expert = tiles.list[1].tile_expert;
    }
    g1.n_wt = (pr.I + 127) / 128;
    g1.tok_box = 32;
    rc = launch_gemm_il_pair_bf16(g1_il, mGate64, mUp64, mA1, g1, dev->num_sms, st, &launches);
  } else {
    rc = pair ? launch_gemm_ws_pair_bf16(0, g1_256 ? 256 : tile, mGate, mUp, mA1, g1, dev->num_sms, st, &launches)
              : launch_gemm_ws_bf16(0, tile, mGate, mUp, mA1, g1, dev->num_sms, st, &launches);
  }
  if (rc != cudaSuccess) return cuda_fail(rc, "gemm1");
  prof_mark(st);

  WsGemm g2 = g1;
  g2.pre_S = 0;
  g2.K = pr.I;
  g2.N = pr.H;
  g2.n_wt = pair ? (pr.H + 511) / 512 : (pr.H + 255) / 256;
  if (g2_single) {
    g2.n_wt = (pr.H + 255) / 256;
    g2.max_tiles = L.t_max2;
    g2.num_tiles = tiles.list[1].num_tiles;
    g2.tile_row = tiles.list[1].tile_row;
    g2.tile_rows = tiles.list[1].tile_rows;
    g2.tile_expert = tiles.list[1].tile_expert;
    g2.tok_box = 128;
  }
  g2.out = w + L.y;
  g2.out_ld = pr.H;
  g2.topk_w = view2(wts);
  rc = g2_single ? launch_gemm_ws_pair_bf16(2, 256, mW2, mW2, mH, g2, dev->num_sms, st, &launches)
     : pair      ? launch_gemm_ws_pair_bf16(1, tile, mW2, mW2, mH, g2, dev->num_sms, st, &launches)
            : launch_gemm_ws_bf16(1, tile, mW2, mW2, mH, g2, dev->num_sms, st, &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "gemm2");
  prof_mark(st);

  rc = launch_combine(reinterpret_cast<const __nv_bfloat16*>(w + L.y), inv, pr.T, pr.H, pr.k,
                      out->data, out->strides[0], out->strides[1], st, &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "combine");
  prof_mark(st);
  t_prof.have = t_prof.on && t_prof.n == kProfSteps + 1;
  t_last_launches = launches;
  return MOE_OK;
}

// ---------------------------------------------------------------- gradient (experts frozen)

// The forward's workspace plus the gradient's own rows: dout gathered into
// expert-grouped order, dh = dL/dh and [dg | du], each [P_max, .] bf16.
// The weight-gradient GEMMs contract over each expert's grouped rows in 64-row
// k-blocks, so the gradient path groups slots in 64-row granules.
constexpr int32_t kBwdBm = 64;

struct BwdLayout {
  WsLayout L;
  size_t d1, dh, dgu, dyT, hT, dguT, a1T, total;
};

// The forward's workspace plus the gradient's own rows: dout gathered into
// expert-grouped order, dh and [dg | du] ([P, .] bf16), and the four transposed
// grouped matrices of the weight gradients ([., P] bf16).
BwdLayout make_bwd_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k) {
  BwdLayout B;
  B.L = make_layout(T, H, I, E, k, false, kBwdBm);
  const size_t P = size_t(B.L.p_max);
  size_t off = align256(B.L.total);
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  B.d1 = take(P * H * 2);
  B.dh = take(P * I * 2);
  B.dgu = take(P * 2 * I * 2);
  B.dyT = take(P * H * 2);
  B.hT = take(P * I * 2);
  B.dguT = take(P * 2 * I * 2);
  B.a1T = take(P * H * 2);
  B.total = off;
  return B;
}

bool kmajor_bf16(const moe_tensor_t* t, int64_t d0, int64_t d1, int64_t d2) {
  return t && t->data && t->dtype == MOE_BF16 && t->ndim == 3 && t->sizes[0] == d0 &&
         t->sizes[1] == d1 && t->sizes[2] == d2 && t->strides[2] == 1 &&
         (t->strides[1] * 2) % 16 == 0 && (t->strides[0] * 2) % 16 == 0 &&
         reinterpret_cast<uintptr_t>(t->data) % 16 == 0;
}

// dx = d out / d x and dweights = d out / d topk_weights contracted with dout,
// with the routing ids fixed and the experts frozen (see moe.h):
//   align; x and dout gathered into expert-grouped rows (A1, D1);
//   dh'[p] = w2_e^T dout_t                  (GEMM2 kernel on w2^T [E, I, H], K = H, weights 1)
//   g, u recomputed from A1 (GEMM1 kernel, mode 3) with dh': dg', du' -> [dg' | du'], h
//   dweights[t, j] = dh'[p] . h[p], p = inv(t, j)   (slot_dot on grouped rows)
//   da[p]  = w_slot [gate_e^T | up_e^T] [dg' | du'] (GEMM2 kernel on w13^T [E, H, 2I], K = 2I)
//   dx[t]  = sum_j da[inv(t, j)]            (combine)
// The routing weight w_slot scales dh = w_slot dh', and dg, du are linear in dh, so it is
// applied once, in da's epilogue (and to [dg' | du'] where the weight gradients transpose
// them); the routing-weight gradient dout_t . (w2_e h) is the same bilinear form as
// (w2_e^T dout_t) . h, so no separate y = w2_e h GEMM is run.
moe_status_t backward_impl(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                           const moe_tensor_t* w13t, const moe_tensor_t* w2t,
                           const moe_tensor_t* ids, const moe_tensor_t* wts,
                           const moe_tensor_t* dout, moe_tensor_t* dx, moe_tensor_t* dw,
                           moe_tensor_t* dw13, moe_tensor_t* dw2, const Problem& pr, void* ws,
                           size_t ws_bytes, cudaStream_t st) {
  int launches = 0;
  t_last_launches = 0;
  if (pr.T == 0) {
    // no tokens: the weight gradients are zero
    if (dw13) MOE_CUDA(cudaMemsetAsync(dw13->data, 0, size_t(pr.E) * dw13->strides[0] * dtype_size(dw13->dtype), st));
    if (dw2) MOE_CUDA(cudaMemsetAsync(dw2->data, 0, size_t(pr.E) * dw2->strides[0] * dtype_size(dw2->dtype), st));
    return MOE_OK;
  }
  const int32_t bm = kBwdBm;
  const BwdLayout B = make_bwd_layout(pr.T, pr.H, pr.I, pr.E, pr.k);
  const WsLayout& L = B.L;
  if (!ws || ws_bytes < B.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  moe_status_t s = device_info(&dev);
  if (s != MOE_OK) return s;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* counts = reinterpret_cast<int32_t*>(w + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(w + L.offsets);
  int32_t* num_blocks = reinterpret_cast<int32_t*>(w + L.num_blocks);
  int32_t* chunk_counts = reinterpret_cast<int32_t*>(w + L.chunk_counts);
  int32_t* sorted = reinterpret_cast<int32_t*>(w + L.sorted);
  int32_t* inv = reinterpret_cast<int32_t*>(w + L.inv);
  int32_t* block_expert = reinterpret_cast<int32_t*>(w + L.block_expert);
  const moe_tensor_t* gate = &w13->gate;
  const moe_tensor_t* up = &w13->up;

  // every GEMM on 128-row token tiles, one CTA each (tensor maps: 128-byte swizzle)
  constexpr int32_t kTile = 128;
  const uint32_t boxw[3] = {64, 128, 1};
  const uint32_t boxt[2] = {64, static_cast<uint32_t>(kTile)};
  const uint32_t boxt64[2] = {64, 64};  // half of a 128-row tile: one CTA of a pair
  CUtensorMap mA1, mA1h, mD1, mDGU, mGate, mUp, mW2T, mW13T;
  auto rows_map = [&](CUtensorMap* m, uint8_t* base, int64_t K, const uint32_t* box) {
    const uint64_t d[2] = {uint64_t(K), uint64_t(L.p_max)};
    const uint64_t sb[1] = {uint64_t(K) * 2};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, d, sb, box, CU_TENSOR_MAP_SWIZZLE_128B);
  };
  auto weight_map = [&](CUtensorMap* m, const moe_tensor_t* t, int64_t K, int64_t N) {
    const uint64_t d[3] = {uint64_t(K), uint64_t(N), uint64_t(pr.E)};
    const uint64_t sb[2] = {uint64_t(t->strides[1]) * 2, uint64_t(t->strides[0]) * 2};
    return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, t->data, d, sb, boxw, CU_TENSOR_MAP_SWIZZLE_128B);
  };
  if ((s = rows_map(&mA1, w + L.a1, pr.H, boxt)) != MOE_OK) return s;
  if ((s = rows_map(&mA1h, w + L.a1, pr.H, boxt64)) != MOE_OK) return s;
  if ((s = rows_map(&mD1, w + B.d1, pr.H, boxt)) != MOE_OK) return s;
  if ((s = rows_map(&mDGU, w + B.dgu, 2 * pr.I, boxt)) != MOE_OK) return s;
  if ((s = weight_map(&mGate, gate, pr.H, pr.I)) != MOE_OK) return s;
  if ((s = weight_map(&mUp, up, pr.H, pr.I)) != MOE_OK) return s;
  if ((s = weight_map(&mW2T, w2t, pr.H, pr.I)) != MOE_OK) return s;
  if ((s = weight_map(&mW13T, w13t, 2 * pr.I, pr.H)) != MOE_OK) return s;

  AlignTiles tiles;
  std::memset(&tiles, 0, sizeof(tiles));
  tiles.list[0].tile_max = kTile;
  tiles.list[0].tile_row = reinterpret_cast<int32_t*>(w + L.tile_row);
  tiles.list[0].tile_rows = reinterpret_cast<int32_t*>(w + L.tile_rows);
  tiles.list[0].tile_expert = reinterpret_cast<int32_t*>(w + L.tile_expert);
  tiles.list[0].num_tiles = num_blocks + 1;
  // the GEMMs on CTA pairs over 256-row token tiles wherever the forward's table picks
  // that form for GEMM2: dh, y and da with one 256-row weight slice per item, the gate/up
  // recompute with 256 rows of I per item
  const bool pair2 = select_config(pr.T, pr.H, pr.I, pr.E, pr.k, false).g2_single != 0;
  if (pair2) {
    tiles.list[1].tile_max = 256;
    tiles.list[1].tile_row = reinterpret_cast<int32_t*>(w + L.tile_row2);
    tiles.list[1].tile_rows = reinterpret_cast<int32_t*>(w + L.tile_rows2);
    tiles.list[1].tile_expert = reinterpret_cast<int32_t*>(w + L.tile_expert2);
    tiles.list[1].num_tiles = num_blocks + 2;
  }
  cudaError_t rc = launch_align(view2(ids), pr.T, pr.k, pr.E, bm, counts, offsets, sorted, inv,
                                block_expert, num_blocks, chunk_counts, L.n_chunks, dev->errors, st,
                                &launches, &tiles);
  if (rc != cudaSuccess) return cuda_fail(rc, "align");
  rc = launch_permute_bf16(view2(x), pr.T, pr.H, pr.k, inv, reinterpret_cast<__nv_bfloat16*>(w + L.a1),
                           st, &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "permute x");
  rc = launch_permute_bf16(view2(dout), pr.T, pr.H, pr.k, inv,
                           reinterpret_cast<__nv_bfloat16*>(w + B.d1), st, &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "permute dout");

  WsGemm gb;
  std::memset(&gb, 0, sizeof(gb));
  gb.max_tiles = L.t_max;
  gb.num_tiles = tiles.list[0].num_tiles;
  gb.tile_row = tiles.list[0].tile_row;
  gb.tile_rows = tiles.list[0].tile_rows;
  gb.tile_expert = tiles.list[0].tile_expert;
  gb.sorted = sorted;
  gb.S = L.S;
  gb.k = pr.k;
  gb.err = dev->errors;
  gb.tok_box = kTile;
  gb.topk_w = view2(wts);
  WsGemm gp = gb;  // the same on align's 256-row tiles (CTA pairs: 128 token rows per CTA)
  if (pair2) {
    gp.max_tiles = L.t_max2;
    gp.num_tiles = tiles.list[1].num_tiles;
    gp.tile_row = tiles.list[1].tile_row;
    gp.tile_rows = tiles.list[1].tile_rows;
    gp.tile_expert = tiles.list[1].tile_expert;
  }
  auto down_form = [&](const WsGemm& p, const CUtensorMap& wm, const CUtensorMap& xm) {
    return pair2 ? launch_gemm_ws_pair_bf16(2, 256, wm, wm, xm, p, dev->num_sms, st, &launches)
                 : launch_gemm_ws_bf16(1, kTile, wm, wm, xm, p, dev->num_sms, st, &launches);
  };

  WsGemm g = gp;  // dh' = w2^T dout, unweighted
  g.K = pr.H;
  g.N = pr.I;
  g.n_wt = (pr.I + 255) / 256;
  g.out = w + B.dh;
  g.out_ld = pr.I;
  g.unit_w = 1;
  rc = down_form(g, mW2T, mD1);
  if (rc != cudaSuccess) return cuda_fail(rc, "gemm dh");

  // g, u recomputed: [dg' | du'] and h.  CTA pairs take align's 128-row tiles (64 token rows
  // per CTA) and 256 rows of I per item: gate and up accumulators of 128 columns each leave
  // room for a second TMEM buffer, so the SwiGLU-gradient epilogue overlaps the next item
  g = gb;
  if (pair2) g.tok_box = 64;
  g.K = pr.H;
  g.N = pr.I;
  g.n_wt = pair2 ? (pr.I + 255) / 256 : (pr.I + 127) / 128;
  g.out = w + B.dgu;
  g.out_ld = 2 * pr.I;
  g.dh = w + B.dh;
  g.dh_ld = pr.I;
  g.h_out = w + L.h;
  g.h_ld = pr.I;
  rc = pair2 ? launch_gemm_ws_pair_bf16(3, 128, mGate, mUp, mA1h, g, dev->num_sms, st, &launches)
             : launch_gemm_ws_bf16(3, kTile, mGate, mUp, mA1, g, dev->num_sms, st, &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "gemm dg du");

  View2 dh_rows;  // dh' in grouped rows [P, I]
  dh_rows.data = w + B.dh;
  dh_rows.s0 = pr.I;
  dh_rows.s1 = 1;
  dh_rows.dtype = MOE_BF16;
  rc = launch_slot_dot(dh_rows, 1, reinterpret_cast<const __nv_bfloat16*>(w + L.h), inv, pr.T, pr.I, pr.k,
                       view2(dw), st, &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "slot_dot");

  g = gp;  // da = w [gate^T | up^T] [dg' | du']
  g.K = 2 * pr.I;
  g.N = pr.H;
  g.n_wt = (pr.H + 255) / 256;
  g.out = w + L.y;
  g.out_ld = pr.H;
  g.unit_w = 0;
  rc = down_form(g, mW13T, mDGU);
  if (rc != cudaSuccess) return cuda_fail(rc, "gemm da");
  rc = launch_combine(reinterpret_cast<const __nv_bfloat16*>(w + L.y), inv, pr.T, pr.H, pr.k,
                      dx->data, dx->strides[0], dx->strides[1], st, &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "combine dx");

  if (dw13 || dw2) {
    // expert-weight gradients: the grouped rows transposed (padding rows zero), then
    // GEMMs contracting over each expert's rows
    const int64_t P = L.p_max;
    View2 none;
    std::memset(&none, 0, sizeof(none));
    View2 dgu_rows;
    dgu_rows.data = w + B.dgu;
    dgu_rows.s0 = 2 * pr.I;
    dgu_rows.s1 = 1;
    dgu_rows.dtype = MOE_BF16;
    CUtensorMap mA, mB, mC;
    // gradient [E, M, N] stored by TMA in 32-row tiles of 128-byte rows (fp32 or bf16)
    auto cmap = [&](CUtensorMap* m, const moe_tensor_t* t, int64_t M, int64_t N) {
      const bool b16 = t->dtype == MOE_BF16;
      const uint64_t es = b16 ? 2 : 4;
      const uint64_t d[3] = {uint64_t(N), uint64_t(M), uint64_t(pr.E)};
      const uint64_t sb[2] = {uint64_t(t->strides[1]) * es, uint64_t(t->strides[0]) * es};
      const uint32_t cbox[3] = {b16 ? 64u : 32u, 32, 1};
      return make_map(m, b16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, t->data, d,
                      sb, cbox, CU_TENSOR_MAP_SWIZZLE_128B);
    };
    auto tmap = [&](CUtensorMap* m, uint8_t* base, int64_t rows, uint32_t box_rows) {
      const uint64_t d[2] = {uint64_t(P), uint64_t(rows)};
      const uint64_t sb[1] = {uint64_t(P) * 2};
      const uint32_t box[2] = {64, box_rows};
      return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, d, sb, box, CU_TENSOR_MAP_SWIZZLE_128B);
    };
    if (dw2) {
      View2 h_rows;
      h_rows.data = w + L.h;
      h_rows.s0 = pr.I;
      h_rows.s1 = 1;
      h_rows.dtype = MOE_BF16;
      rc = launch_gather_transpose(view2(dout), 1, sorted, L.S, pr.k, view2(wts), 1, w + B.dyT, P, pr.H, st,
                                   &launches);
      if (rc == cudaSuccess)
        rc = launch_gather_transpose(h_rows, 0, sorted, L.S, pr.k, none, 0, w + B.hT, P, pr.I, st, &launches);
      if (rc != cudaSuccess) return cuda_fail(rc, "transpose dy h");
      if ((s = tmap(&mA, w + B.dyT, pr.H, kKgroupTileM)) != MOE_OK) return s;
      if ((s = tmap(&mB, w + B.hT, pr.I, kKgroupTileN)) != MOE_OK) return s;
      if ((s = cmap(&mC, dw2, pr.H, pr.I)) != MOE_OK) return s;
      rc = launch_gemm_kgroup(mA, mB, mC, dw2->dtype == MOE_BF16, pr.H, pr.I, pr.E, offsets, dev->errors,
                              dev->num_sms, st, &launches);
      if (rc != cudaSuccess) return cuda_fail(rc, "gemm dw2");
    }
    if (dw13) {
      rc = launch_gather_transpose(dgu_rows, 0, sorted, L.S, pr.k, view2(wts), 1, w + B.dguT, P, 2 * pr.I, st,
                                   &launches);
      if (rc == cudaSuccess)
        rc = launch_gather_transpose(view2(x), 1, sorted, L.S, pr.k, none, 0, w + B.a1T, P, pr.H, st, &launches);
      if (rc != cudaSuccess) return cuda_fail(rc, "transpose dgu x");
      if ((s = tmap(&mA, w + B.dguT, 2 * pr.I, kKgroupTileM)) != MOE_OK) return s;
      if ((s = tmap(&mB, w + B.a1T, pr.H, kKgroupTileN)) != MOE_OK) return s;
      if ((s = cmap(&mC, dw13, 2 * pr.I, pr.H)) != MOE_OK) return s;
      rc = launch_gemm_kgroup(mA, mB, mC, dw13->dtype == MOE_BF16, 2 * pr.I, pr.H, pr.E, offsets, dev->errors,
                              dev->num_sms, st, &launches);
      if (rc != cudaSuccess) return cuda_fail(rc, "gemm dw13");
    }
  }
  t_last_launches = launches;
  return MOE_OK;
}

// device staging of the host-buffer forms: the forward's own workspace, then x, the ids
// (8 bytes per id, so int32 and int64 ids share one layout), the routing weights and out
struct HostLayout {
  size_t core, x_off, ids_off, w_off, o_off, total;
};
HostLayout host_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, int32_t wdtype) {
  HostLayout hl;
  hl.core = moe_workspace_bytes(T, H, I, E, k, wdtype);
  hl.x_off = align256(hl.core);
  hl.ids_off = align256(hl.x_off + size_t(T) * H * 2);
  hl.w_off = align256(hl.ids_off + size_t(T) * k * 8);
  hl.o_off = align256(hl.w_off + size_t(T) * k * 4);
  hl.total = align256(hl.o_off + size_t(T) * H * 2);
  return hl;
}

// H2D copies of x, ids and weights, the forward on the staged copies, D2H of out: all
// enqueued on `st`, nothing waited for
moe_status_t forward_host_enqueue(const moe_tensor_t* x_host, const moe_w13_t* w13, const moe_tensor_t* w2,
                                  const moe_tensor_t* topk_ids_host, const moe_tensor_t* topk_weights_host,
                                  moe_tensor_t* out_host, const Problem& pr, const HostLayout& hl, uint8_t* w,
                                  cudaStream_t st) {
  const int64_t idsz = dtype_size(topk_ids_host->dtype);
  MOE_CUDA(cudaMemcpy2DAsync(w + hl.x_off, pr.H * 2, x_host->data, x_host->strides[0] * 2, pr.H * 2,
                             pr.T, cudaMemcpyHostToDevice, st));
  MOE_CUDA(cudaMemcpy2DAsync(w + hl.ids_off, pr.k * idsz, topk_ids_host->data,
                             topk_ids_host->strides[0] * idsz, pr.k * idsz, pr.T,
                             cudaMemcpyHostToDevice, st));
  MOE_CUDA(cudaMemcpy2DAsync(w + hl.w_off, pr.k * 4, topk_weights_host->data,
                             topk_weights_host->strides[0] * 4, pr.k * 4, pr.T,
                             cudaMemcpyHostToDevice, st));
  moe_tensor_t xd = *x_host, idd = *topk_ids_host, wd = *topk_weights_host, od = *out_host;
  xd.data = w + hl.x_off;
  xd.strides[0] = pr.H;
  xd.strides[1] = 1;
  idd.data = w + hl.ids_off;
  idd.strides[0] = pr.k;
  idd.strides[1] = 1;
  wd.data = w + hl.w_off;
  wd.strides[0] = pr.k;
  wd.strides[1] = 1;
  od.data = w + hl.o_off;
  od.strides[0] = pr.H;
  od.strides[1] = 1;
  moe_status_t s = forward_impl(&xd, w13, w2, &idd, &wd, &od, pr, w, hl.core, st);
  if (s != MOE_OK) return s;
  MOE_CUDA(cudaMemcpy2DAsync(out_host->data, out_host->strides[0] * 2, w + hl.o_off, pr.H * 2,
                             pr.H * 2, pr.T, cudaMemcpyDeviceToHost, st));
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status_t st) {
  switch (st) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_SHAPE_MISMATCH: return "MOE_ERR_SHAPE_MISMATCH";
    case MOE_ERR_UNSUPPORTED_DTYPE: return "MOE_ERR_UNSUPPORTED_DTYPE";
    case MOE_ERR_UNSUPPORTED_LAYOUT: return "MOE_ERR_UNSUPPORTED_LAYOUT";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_NO_DEVICE: return "MOE_ERR_NO_DEVICE";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
  }
  return "MOE_ERR_UNKNOWN";
}

const char* moe_last_cuda_error(void) { return t_last_cuda_error.c_str(); }

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

int32_t moe_last_launch_count(void) { return t_last_launches; }

moe_status_t moe_profile_enable(int32_t on) {
  if (on && !t_prof.ev[0]) {
    for (int i = 0; i <= kProfSteps; ++i) MOE_CUDA(cudaEventCreate(&t_prof.ev[i]));
  }
  t_prof.on = on != 0;
  t_prof.have = false;
  return MOE_OK;
}

moe_status_t moe_profile_read(float* ms, int32_t capacity, int32_t* n) {
  if (!ms || !n) return MOE_ERR_INVALID_ARG;
  *n = 0;
  if (!t_prof.have) return MOE_OK;
  MOE_CUDA(cudaEventSynchronize(t_prof.ev[kProfSteps]));
  int32_t m = 0;
  for (int i = 0; i < kProfSteps && m < capacity; ++i, ++m)
    MOE_CUDA(cudaEventElapsedTime(&ms[m], t_prof.ev[i], t_prof.ev[i + 1]));
  *n = m;
  return MOE_OK;
}

moe_status_t moe_w13_from_packed(const moe_tensor_t* w13, moe_w13_t* out) {
  if (!w13 || !out || w13->ndim != 3) return MOE_ERR_INVALID_ARG;
  if (w13->sizes[1] % 2 != 0) return MOE_ERR_SHAPE_MISMATCH;
  const int64_t I = w13->sizes[1] / 2;
  const int64_t es = dtype_size(w13->dtype);
  if (es == 0) return MOE_ERR_UNSUPPORTED_DTYPE;
  out->gate = *w13;
  out->gate.sizes[1] = I;
  out->up = out->gate;
  // up = rows [I, 2I): same strides, base advanced by I rows (Liger-Kernel PR #1377, "Problems")
  out->up.data = static_cast<uint8_t*>(w13->data) + I * w13->strides[1] * es;
  if (w13->dtype == MOE_E2M1X2 && w13->scale)
    out->up.scale = static_cast<uint8_t*>(w13->scale) + I * w13->scale_strides[1];
  return MOE_OK;
}

size_t moe_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, int32_t wdtype) {
  if (T < 0 || H < 1 || I < 1 || E < 1 || k < 1) return 0;
  if (wdtype != MOE_BF16 && wdtype != MOE_E2M1X2) return 0;
  return make_layout(T, H, I, E, k, wdtype == MOE_E2M1X2, kBm).total;
}

moe_status_t moe_forward_ws(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                            const moe_tensor_t* topk_ids, const moe_tensor_t* topk_weights,
                            moe_tensor_t* out, void* workspace, size_t workspace_bytes,
                            moe_stream_t stream) {
  t_last_launches = 0;
  Problem pr;
  moe_status_t s = validate(x, w13, w2, topk_ids, topk_weights, out, false, &pr);
  if (s != MOE_OK) return s;
  return forward_impl(x, w13, w2, topk_ids, topk_weights, out, pr, workspace, workspace_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_forward(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                         const moe_tensor_t* topk_ids, const moe_tensor_t* topk_weights,
                         moe_tensor_t* out, moe_stream_t stream) {
  t_last_launches = 0;
  Problem pr;
  moe_status_t s = validate(x, w13, w2, topk_ids, topk_weights, out, false, &pr);
  if (s != MOE_OK) return s;
  if (pr.T == 0) return MOE_OK;
  const size_t need = moe_workspace_bytes(pr.T, pr.H, pr.I, pr.E, pr.k, w13->gate.dtype);
  void* ws = nullptr;
  s = cached_workspace(need, &ws);
  if (s != MOE_OK) return s;
  return forward_impl(x, w13, w2, topk_ids, topk_weights, out, pr, ws, need,
                      reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_backward_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k) {
  if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0) return 0;
  return make_bwd_layout(T, H, I, E, k).total;
}

moe_status_t moe_backward_ws(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                             const moe_tensor_t* w13t, const moe_tensor_t* w2t,
                             const moe_tensor_t* topk_ids, const moe_tensor_t* topk_weights,
                             const moe_tensor_t* dout, moe_tensor_t* dx, moe_tensor_t* dweights,
                             moe_tensor_t* dw13, moe_tensor_t* dw2, void* workspace, size_t workspace_bytes,
                             moe_stream_t stream) {
  t_last_launches = 0;
  Problem pr;
  moe_status_t s = validate(x, w13, w2, topk_ids, topk_weights, dx, false, &pr);
  if (s != MOE_OK) return s;
  if (pr.mxfp4) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (!w13t || !w2t || !dout || !dweights) return MOE_ERR_INVALID_ARG;
  if (!kmajor_bf16(w13t, pr.E, pr.H, 2 * pr.I) || !kmajor_bf16(w2t, pr.E, pr.I, pr.H))
    return MOE_ERR_UNSUPPORTED_LAYOUT;
  if (!sizes_ok(dout, 2) || dout->sizes[0] != pr.T || dout->sizes[1] != pr.H) return MOE_ERR_SHAPE_MISMATCH;
  if (dout->dtype != MOE_BF16 || dweights->dtype != MOE_F32) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (!sizes_ok(dweights, 2) || dweights->sizes[0] != pr.T || dweights->sizes[1] != pr.k)
    return MOE_ERR_SHAPE_MISMATCH;
  if (!dout->data || !dweights->data) return MOE_ERR_INVALID_ARG;
  // weight gradients [E, 2I, H] (packed like w13) and [E, H, I], fp32 or bf16: 16-byte
  // aligned rows; the columns a multiple of one 128-byte tile row (32 fp32, 64 bf16)
  auto grad_ok = [&](const moe_tensor_t* t, int64_t R, int64_t C) {
    if (t->dtype != MOE_F32 && t->dtype != MOE_BF16) return false;
    const int64_t v = 16 / dtype_size(t->dtype), cols = 128 / dtype_size(t->dtype);
    return t->data && t->ndim == 3 && t->sizes[0] == pr.E && t->sizes[1] == R && t->sizes[2] == C &&
           t->strides[2] == 1 && t->strides[1] % v == 0 && t->strides[0] % v == 0 && C % cols == 0 &&
           t->strides[0] >= R * t->strides[1] && reinterpret_cast<uintptr_t>(t->data) % 16 == 0;
  };
  if ((dw13 && !grad_ok(dw13, 2 * pr.I, pr.H)) || (dw2 && !grad_ok(dw2, pr.H, pr.I)))
    return MOE_ERR_UNSUPPORTED_LAYOUT;
  return backward_impl(x, w13, w2, w13t, w2t, topk_ids, topk_weights, dout, dx, dweights, dw13, dw2, pr,
                       workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_backward_input_ws(const moe_tensor_t* x, const moe_w13_t* w13, const moe_tensor_t* w2,
                                   const moe_tensor_t* w13t, const moe_tensor_t* w2t,
                                   const moe_tensor_t* topk_ids, const moe_tensor_t* topk_weights,
                                   const moe_tensor_t* dout, moe_tensor_t* dx, moe_tensor_t* dweights,
                                   void* workspace, size_t workspace_bytes, moe_stream_t stream) {
  return moe_backward_ws(x, w13, w2, w13t, w2t, topk_ids, topk_weights, dout, dx, dweights, nullptr, nullptr,
                         workspace, workspace_bytes, stream);
}

moe_status_t moe_transpose_experts(const moe_tensor_t* src, moe_tensor_t* dst, moe_stream_t stream) {
  if (!src || !dst || !src->data || !dst->data) return MOE_ERR_INVALID_ARG;
  if (src->dtype != MOE_BF16 || dst->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (src->ndim != 3 || dst->ndim != 3) return MOE_ERR_SHAPE_MISMATCH;
  const int64_t E = src->sizes[0], R = src->sizes[1], C = src->sizes[2];
  if (E < 0 || R < 0 || C < 0 || dst->sizes[0] != E || dst->sizes[1] != C || dst->sizes[2] != R)
    return MOE_ERR_SHAPE_MISMATCH;
  if (src->strides[2] != 1 || dst->strides[2] != 1) return MOE_ERR_UNSUPPORTED_LAYOUT;
  const cudaError_t rc = launch_transpose_experts(src->data, src->strides[0], src->strides[1], dst->data,
                                                  dst->strides[0], dst->strides[1], E, R, C,
                                                  reinterpret_cast<cudaStream_t>(stream));
  return rc == cudaSuccess ? MOE_OK : cuda_fail(rc, "transpose");
}

moe_status_t moe_forward_host(const moe_tensor_t* x_host, const moe_w13_t* w13,
                              const moe_tensor_t* w2, const moe_tensor_t* topk_ids_host,
                              const moe_tensor_t* topk_weights_host, moe_tensor_t* out_host,
                              moe_stream_t stream) {
  t_last_launches = 0;
  Problem pr;
  moe_status_t s =
      validate(x_host, w13, w2, topk_ids_host, topk_weights_host, out_host, true, &pr);
  if (s != MOE_OK) return s;
  if (pr.T == 0) return MOE_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const HostLayout hl = host_layout(pr.T, pr.H, pr.I, pr.E, pr.k, w13->gate.dtype);
  void* ws = nullptr;
  s = cached_workspace(hl.total, &ws);
  if (s != MOE_OK) return s;
  s = forward_host_enqueue(x_host, w13, w2, topk_ids_host, topk_weights_host, out_host, pr, hl,
                           static_cast<uint8_t*>(ws), st);
  if (s != MOE_OK) return s;
  const int32_t fwd_launches = t_last_launches;
  MOE_CUDA(cudaStreamSynchronize(st));
  t_last_launches = fwd_launches;
  return MOE_OK;
}

size_t moe_host_workspace_bytes(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k, int32_t wdtype) {
  if (moe_workspace_bytes(T, H, I, E, k, wdtype) == 0) return 0;
  return host_layout(T, H, I, E, k, wdtype).total;
}

moe_status_t moe_forward_host_ws(const moe_tensor_t* x_host, const moe_w13_t* w13, const moe_tensor_t* w2,
                                 const moe_tensor_t* topk_ids_host, const moe_tensor_t* topk_weights_host,
                                 moe_tensor_t* out_host, void* workspace, size_t workspace_bytes,
                                 moe_stream_t stream) {
  t_last_launches = 0;
  Problem pr;
  moe_status_t s =
      validate(x_host, w13, w2, topk_ids_host, topk_weights_host, out_host, true, &pr);
  if (s != MOE_OK) return s;
  if (pr.T == 0) return MOE_OK;
  const HostLayout hl = host_layout(pr.T, pr.H, pr.I, pr.E, pr.k, w13->gate.dtype);
  if (!workspace || workspace_bytes < hl.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return MOE_ERR_INVALID_ARG;
  return forward_host_enqueue(x_host, w13, w2, topk_ids_host, topk_weights_host, out_host, pr, hl,
                              static_cast<uint8_t*>(workspace), reinterpret_cast<cudaStream_t>(stream));
}

moe_status_t moe_align(const moe_tensor_t* topk_ids, int64_t E, int32_t block_m, int32_t* counts,
                       int32_t* offsets, int32_t* sorted_slots, int32_t* block_expert,
                       int32_t* num_blocks, void* workspace, size_t workspace_bytes,
                       moe_stream_t stream) {
  if (!topk_ids || !sizes_ok(topk_ids, 2) || !counts || !offsets || !sorted_slots ||
      !block_expert || !num_blocks)
    return MOE_ERR_INVALID_ARG;
  if (topk_ids->dtype != MOE_I32 && topk_ids->dtype != MOE_I64) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (E < 1 || E > kMaxExperts) return MOE_ERR_INVALID_ARG;
  if (block_m != 16 && block_m != 32 && block_m != 64 && block_m != 128 && block_m != 256)
    return MOE_ERR_INVALID_ARG;
  const int64_t T = topk_ids->sizes[0], k = topk_ids->sizes[1];
  if (k < 1 || k > kMaxTopK || T * k >= (int64_t(1) << 30)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!topk_ids->data) return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  moe_status_t s = device_info(&dev);
  if (s != MOE_OK) return s;
  const WsLayout L = make_layout(T, 32, 32, E, k, false, block_m);
  // inv and chunk counts live in the caller's workspace
  const size_t need = align256(L.inv + sizeof(int32_t) * T * k);
  if (!workspace || workspace_bytes < need) return MOE_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  int launches = 0;
  cudaError_t rc = launch_align(view2(topk_ids), T, k, E, block_m, counts, offsets, sorted_slots,
                                reinterpret_cast<int32_t*>(w + L.inv), block_expert, num_blocks,
                                reinterpret_cast<int32_t*>(w + L.chunk_counts), L.n_chunks,
                                dev->errors, reinterpret_cast<cudaStream_t>(stream), &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "align");
  return MOE_OK;
}

moe_status_t moe_router_topk(const moe_tensor_t* logits, int32_t k, int32_t renormalize,
                             int32_t shared_expert, moe_tensor_t* topk_ids,
                             moe_tensor_t* topk_weights, moe_stream_t stream) {
  if (!sizes_ok(logits, 2) || !sizes_ok(topk_ids, 2) || !sizes_ok(topk_weights, 2))
    return MOE_ERR_INVALID_ARG;
  if (logits->dtype != MOE_F32 && logits->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (topk_ids->dtype != MOE_I32 && topk_ids->dtype != MOE_I64) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (topk_weights->dtype != MOE_F32) return MOE_ERR_UNSUPPORTED_DTYPE;
  if ((renormalize != 0 && renormalize != 1) || (shared_expert != 0 && shared_expert != 1))
    return MOE_ERR_INVALID_ARG;
  const int64_t T = logits->sizes[0], E = logits->sizes[1];
  const int64_t kk = int64_t(k) + shared_expert;
  if (E < 1 || E > kMaxExperts || k < 1 || k > E || kk > kMaxTopK) return MOE_ERR_INVALID_ARG;
  if (topk_ids->sizes[0] != T || topk_weights->sizes[0] != T || topk_ids->sizes[1] != kk ||
      topk_weights->sizes[1] != kk)
    return MOE_ERR_SHAPE_MISMATCH;
  if (T == 0) return MOE_OK;
  if (!logits->data || !topk_ids->data || !topk_weights->data) return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  moe_status_t s = device_info(&dev);
  if (s != MOE_OK) return s;
  int launches = 0;
  const cudaError_t rc =
      launch_router_topk(view2(logits), T, static_cast<int>(E), k, renormalize, shared_expert,
                         view2(topk_ids), view2(topk_weights),
                         reinterpret_cast<cudaStream_t>(stream), &launches);
  if (rc != cudaSuccess) return cuda_fail(rc, "router_topk");
  return MOE_OK;
}

moe_status_t moe_quantize_mxfp4(const moe_tensor_t* src, moe_tensor_t* dst, moe_stream_t stream) {
  if (!src || !dst || !src->data || !dst->data || !dst->scale) return MOE_ERR_INVALID_ARG;
  if (src->ndim != dst->ndim || (src->ndim != 2 && src->ndim != 3)) return MOE_ERR_INVALID_ARG;
  if (src->dtype != MOE_BF16 && src->dtype != MOE_F32) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (dst->dtype != MOE_E2M1X2) return MOE_ERR_UNSUPPORTED_DTYPE;
  for (int i = 0; i < src->ndim; ++i)
    if (src->sizes[i] != dst->sizes[i] || src->sizes[i] < 0) return MOE_ERR_SHAPE_MISMATCH;
  const int nd = src->ndim;
  const int64_t K = src->sizes[nd - 1];
  if (K % 32 != 0) return MOE_ERR_SHAPE_MISMATCH;
  if (src->strides[nd - 1] != 1 || dst->strides[nd - 1] != 1 || dst->scale_strides[nd - 1] != 1)
    return MOE_ERR_UNSUPPORTED_LAYOUT;
  DeviceInfo* dev = nullptr;
  moe_status_t s = device_info(&dev);
  if (s != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t es = dtype_size(src->dtype);
  // rank 3 is walked one leading index at a time; each slice is a row-strided matrix
  const int64_t outer = (nd == 3) ? src->sizes[0] : 1;
  const int64_t R = src->sizes[nd - 2];
  for (int64_t o = 0; o < outer; ++o) {
    const uint8_t* sp = static_cast<const uint8_t*>(src->data) + (nd == 3 ? o * src->strides[0] * es : 0);
    uint8_t* dp = static_cast<uint8_t*>(dst->data) + (nd == 3 ? o * dst->strides[0] : 0);
    uint8_t* sc = static_cast<uint8_t*>(dst->scale) + (nd == 3 ? o * dst->scale_strides[0] : 0);
    cudaError_t rc = launch_quantize_rows(sp, src->dtype, R, K, src->strides[nd - 2], dp,
                                          dst->strides[nd - 2], sc, dst->scale_strides[nd - 2], st);
    if (rc != cudaSuccess) return cuda_fail(rc, "quantize");
  }
  return MOE_OK;
}

moe_status_t moe_workspace_layout(int64_t T, int64_t H, int64_t I, int64_t E, int64_t k,
                                  int32_t wdtype, moe_workspace_layout_t* out) {
  if (!out || T < 0 || H < 1 || I < 1 || E < 1 || k < 1) return MOE_ERR_INVALID_ARG;
  if (wdtype != MOE_BF16 && wdtype != MOE_E2M1X2) return MOE_ERR_UNSUPPORTED_DTYPE;
  const bool mx = wdtype == MOE_E2M1X2;
  const WsLayout L = make_layout(T, H, I, E, k, mx, kBm);
  out->rows = L.p_max;
  out->inv = L.inv;
  out->sorted = L.sorted;
  out->a1 = L.a1;
  out->a1_scale = mx ? L.a1_scale : 0;
  out->h = L.h;
  out->h_scale = mx ? L.h_scale : 0;
  out->y = L.y;
  out->total = L.total;
  return MOE_OK;
}

moe_status_t moe_debug_capture(int32_t what, void* dst, size_t bytes) {
  if (what != MOE_CAPTURE_H_PREQUANT) return MOE_ERR_INVALID_ARG;
  if (dst && reinterpret_cast<uintptr_t>(dst) % 16 != 0) return MOE_ERR_INVALID_ARG;
  t_capture_h.ptr = dst;
  t_capture_h.bytes = dst ? bytes : 0;
  return MOE_OK;
}

moe_status_t moe_measure_mma_peak(int32_t kind, int32_t iters, double* tflops) {
  if ((kind != 0 && kind != 1) || iters < 1 || iters > (1 << 20) || !tflops)
    return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  moe_status_t s = device_info(&dev);
  if (s != MOE_OK) return s;
  const cudaError_t rc = measure_mma_rate(kind, iters, dev->num_sms, dev->errors, tflops);
  if (rc != cudaSuccess) return cuda_fail(rc, "mma_rate");
  return MOE_OK;
}

moe_status_t moe_selftest_bounded_wait(int32_t limit_us, int32_t* done, moe_stream_t stream) {
  if (limit_us < 1 || limit_us > 100000 || !done) return MOE_ERR_INVALID_ARG;
  DeviceInfo* dev = nullptr;
  moe_status_t s = device_info(&dev);
  if (s != MOE_OK) return s;
  const cudaError_t rc = launch_bounded_wait_probe(static_cast<unsigned long long>(limit_us) * 1000ull,
                                                   dev->errors, done,
                                                   reinterpret_cast<cudaStream_t>(stream));
  if (rc != cudaSuccess) return cuda_fail(rc, "bounded_wait_probe");
  return MOE_OK;
}

moe_status_t moe_get_device_errors(moe_stream_t stream, uint32_t* n_bad_ids, uint32_t* timeouts) {
  DeviceInfo* dev = nullptr;
  moe_status_t s = device_info(&dev);
  if (s != MOE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  DeviceErrors h;
  MOE_CUDA(cudaMemcpyAsync(&h, dev->errors, sizeof(h), cudaMemcpyDeviceToHost, st));
  MOE_CUDA(cudaMemsetAsync(dev->errors, 0, sizeof(h), st));
  MOE_CUDA(cudaStreamSynchronize(st));
  if (n_bad_ids) *n_bad_ids = h.bad_ids;
  if (timeouts) *timeouts = h.timeouts;
  return h.timeouts ? MOE_ERR_DEVICE_TIMEOUT : MOE_OK;
}

}  // extern "C"
