// Self-test of the bounded-wait failure path shared by the tensor-core kernels.
//
// Every wait of the chunked kernels on an mbarrier is bounded: the waiting thread gives up after a
// number of SM clocks, the group learns of it through a barrier that ORs a predicate, the status word
// gets KDN_ERR_TIMEOUT, the CTA frees its tensor memory and returns.  In a correct run no wait comes
// near its limit, so that path would otherwise never run.  This kernel takes it on purpose, safely: it
// allocates tensor memory like the scan kernels, waits on an mbarrier that nothing arrives at (no TMA
// copy and no MMA is in flight, so nothing can land after the CTA is gone), and takes the same abort
// steps with the caller's limit.
#include <cuda_runtime.h>

#include <string>

#include "../../include/kdn.h"
#include "api_internal.h"
#include "chunk_common.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace kdn {
namespace {

constexpr int kSelfTestThreads = 64;  // two warps: one waits, both take part in the abort barrier
constexpr uint32_t kSelfTestCols = 32;

__global__ void __launch_bounds__(kSelfTestThreads, 1) wait_timeout_selftest_kernel(unsigned* status,
                                                                                     long long wait_cycles) {
  __shared__ uint64_t never;  // nothing arrives here
  __shared__ uint32_t tmem_base;
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) {
    sm100::mbar_init(&never, 1);
    sm100::fence_mbar_init();
  }
  if (warp == 0) {
    sm100::tmem_alloc(&tmem_base, kSelfTestCols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  bool bad = false;
  if (tid == 0) bad = !sm100::mbar_wait_bounded(&never, 0, wait_cycles);
  bad = chunk::named_sync_or(1, kSelfTestThreads, bad);
  if (bad && tid == 0) raise_status(status, kStatusTimeout);
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 0) sm100::tmem_dealloc(tmem_base, kSelfTestCols);
}

}  // namespace
}  // namespace kdn

using namespace kdn::api;

extern "C" kdn_status kdn_selftest_wait_timeout(void* workspace, long long wait_cycles, void* stream) {
  if (!(wait_cycles >= 1 && wait_cycles <= kdn::chunk::kWaitCycles))
    return fail(KDN_ERR_INVALID_ARG, "wait_cycles must be in 1 .. " + std::to_string(kdn::chunk::kWaitCycles));
  DeviceGuard guard;
  void* word = workspace;
  if (workspace == nullptr) {
    kdn_status st = noalloc_scratch_on_current_device(&word);
    if (st != KDN_OK) return st;
  } else {
    kdn_status st = check_ptr(workspace, "workspace", 256, false);
    if (st != KDN_OK) return st;
    st = use_device_of(workspace, guard);
    if (st != KDN_OK) return st;
  }
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(word, 0, kStatusBytes, s);
  if (e != cudaSuccess) return cuda_status(e, "clearing the status word");
  kdn::wait_timeout_selftest_kernel<<<1, kdn::kSelfTestThreads, 0, s>>>(reinterpret_cast<unsigned*>(word),
                                                                        wait_cycles);
  return cuda_status(cudaGetLastError(), "wait self-test launch");
}
