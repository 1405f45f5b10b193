// Shared device helpers of the kdn library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kdn {

// Device status word bits (first 32-bit word of the workspace).
enum : unsigned { kStatusNumeric = 1u, kStatusTimeout = 2u };

// Runtime dtype codes, equal to the kdn_dtype values of the public header.
enum : int { kF32 = 0, kBF16 = 1 };

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Load element i of a bf16 or fp32 array chosen at run time.
__device__ __forceinline__ float load_elem(const void* p, size_t i, int dtype) {
  if (dtype == kBF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}

__device__ __forceinline__ void store_elem(void* p, size_t i, float x, int dtype) {
  if (dtype == kBF16)
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
  else
    reinterpret_cast<float*>(p)[i] = x;
}

// Asynchronous global -> shared copies (Ampere-style cp.async) for input rings.
__device__ __forceinline__ void async_copy16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void async_copy4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
// ``bytes`` (a multiple of 16, both addresses 16-byte aligned) by the threads t = 0, stride, 2 stride, ...
__device__ __forceinline__ void async_copy_rows(void* dst, const void* src, int bytes, int t, int stride) {
  for (int c = t; c < bytes / 16; c += stride)
    async_copy16(static_cast<uint8_t*>(dst) + 16 * c, static_cast<const uint8_t*>(src) + 16 * c);
}

__device__ __forceinline__ void raise_status(unsigned* status, unsigned bits) {
  if (status != nullptr) atomicOr(status, bits);
}

// Thread layout used by the per-token kernels for a (R x C) fp32 matrix held in
// registers: C/4 column groups of 4 (one float4 per row), R rows strided over
// the row groups, so that one warp reads whole rows with 16-byte accesses.
template <int R, int C>
struct RowBlockLayout {
  static constexpr int kColGroups = C / 4;
  static constexpr int kThreads = (kColGroups * R < 256) ? kColGroups * R : 256;
  static constexpr int kRowGroups = kThreads / kColGroups;
  static constexpr int kRowsPerThread = R / kRowGroups;
  static_assert(kRowsPerThread >= 1 && kRowsPerThread * kRowGroups == R, "layout");
};

}  // namespace kdn
