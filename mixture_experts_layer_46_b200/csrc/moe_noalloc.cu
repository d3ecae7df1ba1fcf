// moe_align_noalloc: the align step with its scratch in library-owned device
// memory, for callers that can neither allocate device memory nor hand the
// library a workspace buffer.
//
// Who needs this: code that runs under someone else's memory plan.  Examples
// are a plugin loaded into a serving engine that has already divided the
// device memory between its own pools and forbids further allocation, or a
// component whose only device memory is the input and output tensors its host
// framework gives it.  Such a caller cannot call cudaMalloc (or any allocating
// library routine) and has no spare buffer to pass as `workspace`.
//
// The scratch (per-slot positions and per-chunk expert histograms) lives in a
// fixed array below.  Every GPU that loads the library holds it until the
// process exits, so it is kept small: kNoAllocScratchBytes.  All calls share
// it and it keeps the last call's contents; the kernels overwrite every entry
// they later read, so nothing has to start at zero.  Two calls whose work
// overlaps on the GPU (different streams, no ordering between them) race on
// this array and may produce wrong results.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

// Largest routing problem the fixed scratch serves: T * top_k slots.
constexpr int64_t kNoAllocMaxSlots = int64_t(1) << 20;
constexpr int64_t kNoAllocMaxChunks = (kNoAllocMaxSlots + kAlignChunk - 1) / kAlignChunk;
// inv[slots] then chunk histograms [chunks][experts], 256-byte aligned regions
constexpr size_t kInvBytes = size_t(kNoAllocMaxSlots) * sizeof(int32_t);
constexpr size_t kChunkBytes = size_t(kNoAllocMaxChunks) * kMaxExperts * sizeof(int32_t);
constexpr size_t kNoAllocScratchBytes = kInvBytes + kChunkBytes;  // 5 MiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchAddr {
  bool ready = false;
  unsigned char* ptr = nullptr;
};
std::mutex g_mu;
ScratchAddr g_addr[64];

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the real address is looked
// up once per device (with that device current) and cached for the life of the
// process: do not use this entry point across a cudaDeviceReset of that device
// (the cached address would belong to the destroyed context).
cudaError_t scratch_on_current_device(unsigned char** out) {
  int dev = 0;
  cudaError_t rc = cudaGetDevice(&dev);
  if (rc != cudaSuccess) return rc;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev].ready) {
    unsigned char* p = nullptr;
    rc = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_noalloc_scratch);
    if (rc != cudaSuccess) return rc;
    g_addr[dev].ptr = p;
    g_addr[dev].ready = true;
  }
  *out = g_addr[dev].ptr;
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status_t moe_align_noalloc(const moe_tensor_t* topk_ids, int64_t E, int32_t block_m,
                                          int32_t* counts, int32_t* offsets, int32_t* sorted_slots,
                                          int32_t* block_expert, int32_t* num_blocks,
                                          moe_stream_t stream) {
  if (!topk_ids || topk_ids->ndim != 2 || !counts || !offsets || !sorted_slots || !block_expert ||
      !num_blocks)
    return MOE_ERR_INVALID_ARG;
  if (topk_ids->dtype != MOE_I32 && topk_ids->dtype != MOE_I64) return MOE_ERR_UNSUPPORTED_DTYPE;
  if (E < 1 || E > kMaxExperts) return MOE_ERR_INVALID_ARG;
  if (block_m != 16 && block_m != 32 && block_m != 64 && block_m != 128 && block_m != 256)
    return MOE_ERR_INVALID_ARG;
  const int64_t T = topk_ids->sizes[0], k = topk_ids->sizes[1];
  if (T < 0 || k < 1 || k > kMaxTopK) return MOE_ERR_INVALID_ARG;
  // the fixed scratch holds at most kNoAllocMaxSlots slots: larger problems are refused
  if (T * k > kNoAllocMaxSlots) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if (T == 0) return MOE_OK;
  if (!topk_ids->data) return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10) return MOE_ERR_NO_DEVICE;
  unsigned char* scratch = nullptr;
  if (scratch_on_current_device(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t* inv = reinterpret_cast<int32_t*>(scratch);
  int32_t* chunk_counts = reinterpret_cast<int32_t*>(scratch + kInvBytes);
  const int64_t n_chunks = (T * k + kAlignChunk - 1) / kAlignChunk;
  View2 ids;
  ids.data = topk_ids->data;
  ids.s0 = topk_ids->strides[0];
  ids.s1 = topk_ids->strides[1];
  ids.dtype = topk_ids->dtype;
  int launches = 0;
  // slots outside [0, E) are still skipped; they are not counted here (no
  // device error word is touched by this entry point)
  const cudaError_t rc = launch_align(ids, T, k, E, block_m, counts, offsets, sorted_slots, inv,
                                      block_expert, num_blocks, chunk_counts, n_chunks, nullptr,
                                      reinterpret_cast<cudaStream_t>(stream), &launches);
  return rc == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
