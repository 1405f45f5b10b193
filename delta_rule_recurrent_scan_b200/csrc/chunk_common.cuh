// Device helpers shared by the chunked tensor-core kernels (state side and covariance side).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100.cuh"

namespace kdn {
namespace chunk {

constexpr int kC = 64;                            // tokens per chunk
constexpr long long kWaitCycles = 2000000000LL;   // bounded waits: about one second
constexpr int kLD = 68;                           // row stride of the fp32 [64][68] scratch matrices

// fp32 -> bf16 hi + lo for 8 consecutive values, stored as two 16-byte chunks.
__device__ __forceinline__ void store8_split(uint8_t* hi, uint8_t* lo, uint32_t off, const float (&x)[8]) {
  uint4 h, l;
  sm100::split2_bf16(x[0], x[1], h.x, l.x);
  sm100::split2_bf16(x[2], x[3], h.y, l.y);
  sm100::split2_bf16(x[4], x[5], h.z, l.z);
  sm100::split2_bf16(x[6], x[7], h.w, l.w);
  *reinterpret_cast<uint4*>(hi + off) = h;
  *reinterpret_cast<uint4*>(lo + off) = l;
}

// 8 consecutive fp32 values -> fp16, stored as one 16-byte chunk.
__device__ __forceinline__ void store8_f16(uint8_t* dst, uint32_t off, const float (&x)[8]) {
  uint4 h;
  h.x = sm100::pack2_f16(x[0], x[1]);
  h.y = sm100::pack2_f16(x[2], x[3]);
  h.z = sm100::pack2_f16(x[4], x[5]);
  h.w = sm100::pack2_f16(x[6], x[7]);
  *reinterpret_cast<uint4*>(dst + off) = h;
}

// 8 consecutive fp16 of a swizzled panel (one 16-byte chunk) as floats.
__device__ __forceinline__ void load8_f16(const uint8_t* base, uint32_t off, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(base + off);
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(h[e]);
    x[2 * e] = f.x, x[2 * e + 1] = f.y;
  }
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

// Named barrier over ``count`` threads that also ORs a predicate across them.
__device__ __forceinline__ bool named_sync_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// TMEM column of the fp16 pairs of the 16-token block ks (K step of 16) when thread half h holds tokens
// 32 h .. 32 h + 31 of a 64-token operand as 16 pair columns at 32 h.
__device__ __forceinline__ uint32_t tok_pair_col(int ks) { return 32u * (ks >> 1) + 8u * (ks & 1); }

// Sum over the 8 consecutive lanes that share a token.
__device__ __forceinline__ float oct_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}

// T = (I + N)^-1 for a 64 x 64 strictly lower N (fp32, row stride kLD; only the strict lower part of N
// is read).  T's lower part is written to Tf (its unit diagonal and the zeros above it inside the 16 x 16
// diagonal blocks too); the other upper blocks of Tf are scratch.  Run by the 256 threads gt = 0..255 of
// a group that synchronises with ``sync()``.
//   (1) diagonal blocks T_bb = (I + N_bb)^-1 by forward substitution, one thread per column;
//   (2) 16 -> 32: T_{b+1,b} = -T_{b+1,b+1} (N_{b+1,b} T_bb) for b = 0, 2;
//   (3) 32 -> 64: T_{[23],[01]} = -T_{[23],[23]} (N_{[23],[01]} T_{[01],[01]}),
// the block form of the inverse of [[X, 0], [Y, Z]] at each doubling.
template <class Sync>
__device__ __forceinline__ void invert_unit_lower_64(const float* Nf, float* Tf, int gt, Sync sync) {
  constexpr int LD = kLD;
  if (gt < 64) {
    const int b = gt >> 4, cc = gt & 15;
    const float* Nb = Nf + (16 * b) * LD + 16 * b;
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) t[i] = (i == cc) ? 1.f : 0.f;
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int q = 0; q < (i + 3) / 4; ++q) {
        const float4 n4 = *reinterpret_cast<const float4*>(Nb + i * LD + 4 * q);
        const float nv[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (4 * q + e < i) acc = fmaf(nv[e], t[4 * q + e], acc);  // compile-time bounds: strict lower only
      }
      if (i > cc) t[i] = -acc;
    }
    float* Tb = Tf + (16 * b) * LD + 16 * b;
#pragma unroll
    for (int i = 0; i < 16; ++i) Tb[i * LD + cc] = t[i];
  }
  sync();
  // (2) pairs (a, b) = (1, 0), (3, 2): M = N_ab T_bb parked in the upper block (b, a), then T_ab = -T_aa M
  {
    const int pr = gt >> 6, i = (gt >> 2) & 15, jq = gt & 3;
    const int a = 2 * pr + 1, b = 2 * pr;
    if (gt < 128) {
      float nv[16];
#pragma unroll
      for (int l = 0; l < 16; l += 4) {
        const float4 n4 = *reinterpret_cast<const float4*>(Nf + (16 * a + i) * LD + 16 * b + l);
        nv[l] = n4.x, nv[l + 1] = n4.y, nv[l + 2] = n4.z, nv[l + 3] = n4.w;
      }
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float4 t4 = *reinterpret_cast<const float4*>(Tf + (16 * b + k) * LD + 16 * b + 4 * jq);
        acc.x = fmaf(nv[k], t4.x, acc.x), acc.y = fmaf(nv[k], t4.y, acc.y);
        acc.z = fmaf(nv[k], t4.z, acc.z), acc.w = fmaf(nv[k], t4.w, acc.w);
      }
      *reinterpret_cast<float4*>(Tf + (16 * b + i) * LD + 16 * a + 4 * jq) = acc;
    }
    sync();
    if (gt < 128) {
      float tv[16];
#pragma unroll
      for (int l = 0; l < 16; l += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(Tf + (16 * a + i) * LD + 16 * a + l);
        tv[l] = t4.x, tv[l + 1] = t4.y, tv[l + 2] = t4.z, tv[l + 3] = t4.w;
      }
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float4 m4 = *reinterpret_cast<const float4*>(Tf + (16 * b + k) * LD + 16 * a + 4 * jq);
        acc.x = fmaf(tv[k], m4.x, acc.x), acc.y = fmaf(tv[k], m4.y, acc.y);
        acc.z = fmaf(tv[k], m4.z, acc.z), acc.w = fmaf(tv[k], m4.w, acc.w);
      }
      *reinterpret_cast<float4*>(Tf + (16 * a + i) * LD + 16 * b + 4 * jq) =
          make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
    }
    sync();
  }
  // (3) X = N_{[23],[01]} T_{[01],[01]} parked in rows 0..31, columns 32..63; then the lower-left 32 x 32
  // block of T = -T_{[23],[23]} X.  Threads 0..127 each take rows {r, r + 16} x four columns (register
  // tiles halve the shared-memory reads of the broadcast operand); warps take uniform column ranges.
  {
    const int u = gt & 127;
    if (gt < 128) {
      const int jh = u >> 6, r = (u >> 2) & 15, j0 = 16 * jh + 4 * (u & 3);
      float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
#pragma unroll
      for (int kb = 0; kb < 32; kb += 4) {
        if (kb < 16 * jh) continue;  // T_{[01],[01]}[k][j] = 0 for k < 16 <= j
        const float4 na = *reinterpret_cast<const float4*>(Nf + (32 + r) * LD + kb);
        const float4 nb = *reinterpret_cast<const float4*>(Nf + (48 + r) * LD + kb);
        const float n0[4] = {na.x, na.y, na.z, na.w}, n1[4] = {nb.x, nb.y, nb.z, nb.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 t4 = *reinterpret_cast<const float4*>(Tf + (kb + e) * LD + j0);
          acc0.x = fmaf(n0[e], t4.x, acc0.x), acc0.y = fmaf(n0[e], t4.y, acc0.y);
          acc0.z = fmaf(n0[e], t4.z, acc0.z), acc0.w = fmaf(n0[e], t4.w, acc0.w);
          acc1.x = fmaf(n1[e], t4.x, acc1.x), acc1.y = fmaf(n1[e], t4.y, acc1.y);
          acc1.z = fmaf(n1[e], t4.z, acc1.z), acc1.w = fmaf(n1[e], t4.w, acc1.w);
        }
      }
      *reinterpret_cast<float4*>(Tf + r * LD + 32 + j0) = acc0;
      *reinterpret_cast<float4*>(Tf + (16 + r) * LD + 32 + j0) = acc1;
    }
    sync();
    if (gt < 128) {
      const int r = u >> 3, j0 = 4 * (u & 7);
      float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
#pragma unroll
      for (int kb = 0; kb < 32; kb += 4) {
        // row r of T_{[23],[23]} is zero past column 15; row 16 + r runs to column 31
        float t0v[4] = {0.f, 0.f, 0.f, 0.f};
        if (kb < 16) {
          const float4 ta = *reinterpret_cast<const float4*>(Tf + (32 + r) * LD + 32 + kb);
          t0v[0] = ta.x, t0v[1] = ta.y, t0v[2] = ta.z, t0v[3] = ta.w;
        }
        const float4 tb = *reinterpret_cast<const float4*>(Tf + (48 + r) * LD + 32 + kb);
        const float t1v[4] = {tb.x, tb.y, tb.z, tb.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 x4 = *reinterpret_cast<const float4*>(Tf + (kb + e) * LD + 32 + j0);
          if (kb < 16) {
            acc0.x = fmaf(t0v[e], x4.x, acc0.x), acc0.y = fmaf(t0v[e], x4.y, acc0.y);
            acc0.z = fmaf(t0v[e], x4.z, acc0.z), acc0.w = fmaf(t0v[e], x4.w, acc0.w);
          }
          acc1.x = fmaf(t1v[e], x4.x, acc1.x), acc1.y = fmaf(t1v[e], x4.y, acc1.y);
          acc1.z = fmaf(t1v[e], x4.z, acc1.z), acc1.w = fmaf(t1v[e], x4.w, acc1.w);
        }
      }
      *reinterpret_cast<float4*>(Tf + (32 + r) * LD + j0) = make_float4(-acc0.x, -acc0.y, -acc0.z, -acc0.w);
      *reinterpret_cast<float4*>(Tf + (48 + r) * LD + j0) = make_float4(-acc1.x, -acc1.y, -acc1.z, -acc1.w);
    }
    sync();
  }
}

}  // namespace chunk
}  // namespace kdn
