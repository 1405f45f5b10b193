// Device helpers shared by the chunked tensor-core kernels (state side and covariance side).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "sm100.cuh"

namespace kdn {
namespace chunk {

constexpr int kC = 64;                            // tokens per chunk
constexpr long long kWaitCycles = 2000000000LL;   // bounded waits: about one second
constexpr int kLD = 68;                           // row stride of the fp32 [64][68] scratch matrices

// fp32 -> bf16 hi + lo for 8 consecutive values, stored as two 16-byte chunks.
__device__ __forceinline__ void store8_split(uint8_t* hi, uint8_t* lo, uint32_t off, const float (&x)[8]) {
  __align__(16) __nv_bfloat16 h[8], l[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) sm100::split_bf16(x[e], h[e], l[e]);
  *reinterpret_cast<uint4*>(hi + off) = *reinterpret_cast<const uint4*>(h);
  *reinterpret_cast<uint4*>(lo + off) = *reinterpret_cast<const uint4*>(l);
}

// 8 consecutive bf16 of a swizzled panel (one 16-byte chunk) as floats.
__device__ __forceinline__ void load8_bf16(const uint8_t* base, uint32_t off, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(base + off);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    x[2 * e] = f.x, x[2 * e + 1] = f.y;
  }
}

__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Sum over the 8 consecutive lanes that share a token.
__device__ __forceinline__ float oct_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}

// T = (I + N)^-1 for a 64 x 64 strictly lower N (fp32, row stride kLD, only the strict lower part is
// read).  T's lower part (the unit diagonal excluded) is written to Tf; its upper blocks are used as
// scratch.  Run by the 256 threads gt = 0..255 of a group that synchronises with ``sync()``.
// Blocked by 16: diagonal blocks right-looking (one thread per column), then the off-diagonal blocks by
// distance d = 1..3, T_ab = -T_aa sum_{k=b}^{a-1} N_ak T_kb.
template <class Sync>
__device__ __forceinline__ void invert_unit_lower_64(const float* Nf, float* Tf, int gt, Sync sync) {
  constexpr int LD = kLD;
  if (gt < 64) {
    const int b = gt >> 4, cc = gt & 15;
    const float* Nb = Nf + (16 * b) * LD + 16 * b;
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = (i == cc) ? 1.f : 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float tj = acc[j];
#pragma unroll
      for (int i = 1; i < 16; ++i)  // fixed bounds: every register index is a constant
        if (i > j) acc[i] = fmaf(-Nb[i * LD + j], tj, acc[i]);
    }
    float* Tb = Tf + (16 * b) * LD + 16 * b;
#pragma unroll
    for (int i = 0; i < 16; ++i) Tb[i * LD + cc] = acc[i];
  }
  sync();
#pragma unroll
  for (int d = 1; d < 4; ++d) {
    const bool act = gt < (4 - d) * 64;
    const int b = gt >> 6, a = b + d, ii = (gt >> 2) & 15, jq = gt & 3;
    if (act) {
      float nv[16 * 3];
#pragma unroll
      for (int k = 0; k < d; ++k)
#pragma unroll
        for (int l = 0; l < 16; l += 4) {
          const float4 n4 = *reinterpret_cast<const float4*>(Nf + (16 * a + ii) * LD + 16 * (b + k) + l);
          nv[16 * k + l] = n4.x, nv[16 * k + l + 1] = n4.y, nv[16 * k + l + 2] = n4.z, nv[16 * k + l + 3] = n4.w;
        }
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < d; ++k)
#pragma unroll
        for (int l = 0; l < 16; ++l) {
          const float n = nv[16 * k + l];
          const float4 t4 = *reinterpret_cast<const float4*>(Tf + (16 * (b + k) + l) * LD + 16 * b + 4 * jq);
          acc.x = fmaf(n, t4.x, acc.x), acc.y = fmaf(n, t4.y, acc.y);
          acc.z = fmaf(n, t4.z, acc.z), acc.w = fmaf(n, t4.w, acc.w);
        }
      // M_ab parked in the unused upper block (b, a)
      *reinterpret_cast<float4*>(Tf + (16 * b + ii) * LD + 16 * a + 4 * jq) = acc;
    }
    sync();
    if (act) {
      float tv[16];
#pragma unroll
      for (int l = 0; l < 16; l += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(Tf + (16 * a + ii) * LD + 16 * a + l);
        tv[l] = t4.x, tv[l + 1] = t4.y, tv[l + 2] = t4.z, tv[l + 3] = t4.w;
      }
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int l = 0; l < 16; ++l) {
        const float4 m4 = *reinterpret_cast<const float4*>(Tf + (16 * b + l) * LD + 16 * a + 4 * jq);
        acc.x = fmaf(tv[l], m4.x, acc.x), acc.y = fmaf(tv[l], m4.y, acc.y);
        acc.z = fmaf(tv[l], m4.z, acc.z), acc.w = fmaf(tv[l], m4.w, acc.w);
      }
      *reinterpret_cast<float4*>(Tf + (16 * a + ii) * LD + 16 * b + 4 * jq) =
          make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    sync();
  }
}

}  // namespace chunk
}  // namespace kdn
