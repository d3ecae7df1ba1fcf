// Self-test of the kernels' failure path: every wait in the forward's kernels
// is bounded (mbar_wait gives up after a time limit, counts a timeout in the
// device error counters and lets the kernel unwind) so that a missing arrival
// ends in an error status instead of a hung GPU.  This kernel exercises that
// path on purpose and safely: one thread initialises an mbarrier that nothing
// ever arrives on and waits on it with a short limit.  No copy, no tensor-core
// operation and no other thread is involved, so giving up leaves nothing in
// flight.
#include "../../include/moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

__global__ void bounded_wait_probe_kernel(unsigned long long limit_ns, DeviceErrors* err,
                                          int32_t* done) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const bool ok = mbar_wait(&bar, 0, err, limit_ns);  // nobody arrives: gives up
  *done = ok ? 1 : 2;
}

}  // namespace

cudaError_t launch_bounded_wait_probe(unsigned long long limit_ns, DeviceErrors* err,
                                      int32_t* done, cudaStream_t st) {
  bounded_wait_probe_kernel<<<1, 32, 0, st>>>(limit_ns, err, done);
  return cudaGetLastError();
}

}  // namespace moe
