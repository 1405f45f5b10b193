// Full-Kalman scan that allocates nothing: its scratch is a static device array.
//
// kdn_scan_kalman_full asks the caller for a workspace (a 256-byte status word
// plus one fp32 gain per token and key coordinate).  Some callers cannot hand
// one over: code that must not call cudaMalloc once it is running (a server
// that reserves all device memory at start-up and hands out fixed pools, a
// plugin whose host framework owns the device allocator, a real-time loop that
// forbids allocation) and that has no spare buffer of the right size.  This
// entry point runs the same kernels with the scratch in the file-scope array
// below instead.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "../../include/kdn.h"
#include "api_internal.h"

namespace {

// 256-byte status word, then up to 16 MiB of fp32 gains (B*H*L*d_k <= 4,194,304).
constexpr size_t kNoAllocScratchBytes = kdn::api::kStatusBytes + (size_t(16) << 20);

// Every GPU that loads this library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device, looked up once per device.
kdn_status scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return kdn::api::cuda_status(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return kdn::api::fail(KDN_ERR_UNSUPPORTED, "device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return kdn::api::fail(KDN_ERR_CUDA, std::string("cudaGetSymbolAddress of the static scratch: ") +
                                              cudaGetErrorString(e));
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KDN_OK;
}

}  // namespace

extern "C" kdn_status kdn_scan_kalman_full_noalloc(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                                   const float* a, const float* r, const float* qn, float qn_scalar,
                                                   float* S, float* P, void* o, float* m, void* stream) {
  kdn_status st = kdn::api::check_dims(dims);
  if (st != KDN_OK) return st;
  // the static array holds the gains of the serial scan: the library's segment choice is turned off
  kdn_dims d = *dims;
  if (d.segments == 0) d.segments = 1;
  dims = &d;
  const size_t need = kdn_workspace_bytes(KDN_KALMAN_FULL, dims);
  if (need > kNoAllocScratchBytes)
    return kdn::api::fail(KDN_ERR_UNSUPPORTED,
                          "kdn_scan_kalman_full_noalloc: this scan needs " + std::to_string(need) +
                              " bytes of scratch but the static array holds " + std::to_string(kNoAllocScratchBytes) +
                              " (B*H*L*d_k must be <= 4194304); use kdn_scan_kalman_full with a workspace");
  st = kdn::api::check_ptr(S, "S", 16, false);
  if (st != KDN_OK) return st;
  st = kdn::api::use_device_of(S);  // the scratch address is per device: look it up on the state's device
  if (st != KDN_OK) return st;
  void* scratch = nullptr;
  st = scratch_on_current_device(&scratch);
  if (st != KDN_OK) return st;
  return kdn::api::kalman_scan(KDN_KALMAN_FULL, dims, q, k, v, a, r, qn, qn_scalar, S, P, o, m, scratch,
                               kNoAllocScratchBytes, stream);
}
