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

// One m16n8k8 warp-level tensor-core product with tf32 operands and fp32 accumulation: d += a b.  The
// operands are fp32 bit patterns, of which the unit reads the sign, exponent and 10 leading mantissa bits.
// Fragments, with g = lane / 4 and t = lane % 4: a = A[g][t], A[g + 8][t], A[g][t + 4], A[g + 8][t + 4];
// b = B[t][g], B[t + 4][g]; d = D[g][2 t], D[g][2 t + 1], D[g + 8][2 t], D[g + 8][2 t + 1].
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// x = hi + lo with hi the leading 19 bits (sign, exponent, 10 mantissa bits) and lo = x - hi exactly.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = __float_as_uint(x) & 0xffffe000u;
  lo = __float_as_uint(x - __uint_as_float(hi));
}

// acc = A B for one 16 x 8 tile over KS steps of 8 along k (from k0): A points at the tile's row 0, B at
// its column 0, both fp32 row-major with row stride kLD in shared memory.  Every operand is split as
// hi + lo and the product taken as hi hi + (hi lo + lo hi): the dropped lo lo term and the tf32 reading of
// lo leave about 2^-20 of |A| |B|, against 2^-11 for a single tf32 product.  Run by a whole warp.
template <int KS>
__device__ __forceinline__ void tile_mma_x3(const float* A, const float* B, int k0, float (&acc)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  float hh[4] = {0.f, 0.f, 0.f, 0.f}, cr[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int s = 0; s < KS; ++s) {
    const int k = k0 + 8 * s;
    const float av[4] = {A[g * kLD + k + t], A[(g + 8) * kLD + k + t], A[g * kLD + k + t + 4],
                         A[(g + 8) * kLD + k + t + 4]};
    const float bv[2] = {B[(k + t) * kLD + g], B[(k + t + 4) * kLD + g]};
    uint32_t ah[4], al[4], bh[2], bl[2];
#pragma unroll
    for (int e = 0; e < 4; ++e) split_tf32(av[e], ah[e], al[e]);
#pragma unroll
    for (int e = 0; e < 2; ++e) split_tf32(bv[e], bh[e], bl[e]);
    mma_tf32_16x8x8(hh, ah, bh);
    mma_tf32_16x8x8(cr, ah, bl);
    mma_tf32_16x8x8(cr, al, bh);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] = hh[e] + cr[e];
}

// scale * acc into the 16 x 8 tile at D (row stride kLD), in the fragment layout of mma_tf32_16x8x8.
__device__ __forceinline__ void store_tile(float* D, const float (&acc)[4], float scale) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  *reinterpret_cast<float2*>(D + g * kLD + 2 * t) = make_float2(scale * acc[0], scale * acc[1]);
  *reinterpret_cast<float2*>(D + (g + 8) * kLD + 2 * t) = make_float2(scale * acc[2], scale * acc[3]);
}

// T = (I + N)^-1 for a 64 x 64 strictly lower N (fp32, row stride kLD; only the strict lower part of N
// is read).  T's lower part is written to Tf (its unit diagonal and the zeros above it inside the 16 x 16
// diagonal blocks too); the other upper blocks of Tf are scratch.  Run by the 256 threads gt = 0..255 of
// a group that synchronises with ``sync()``.
//   (1) diagonal blocks T_bb = (I + N_bb)^-1 by forward substitution, one thread per column;
//   (2) 16 -> 32: T_{b+1,b} = -T_{b+1,b+1} (N_{b+1,b} T_bb) for b = 0, 2;
//   (3) 32 -> 64: T_{[23],[01]} = -T_{[23],[23]} (N_{[23],[01]} T_{[01],[01]}),
// the block form of the inverse of [[X, 0], [Y, Z]] at each doubling.  The products of (2) and (3) run as
// warp-level tf32 tensor-core products split three ways (tile_mma_x3), one 16 x 8 output tile per warp: the
// tiles are too small for a tcgen05 round trip through shared and tensor memory, and on the fp32 pipe half the
// group waited on the other half's 32-term dot products.
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
  // (2) pairs (a, b) = (1, 0), (3, 2): M = N_ab T_bb parked in the upper block (b, a), then T_ab = -T_aa M;
  // warps 0..3 take pair w / 2, columns 8 (w % 2) ..
  const int w = gt >> 5;
  {
    const int pr = w >> 1, n0 = 8 * (w & 1);
    const int a = 2 * pr + 1, b = 2 * pr;
    if (w < 4) {
      float acc[4];
      tile_mma_x3<2>(Nf + (16 * a) * LD + 16 * b, Tf + (16 * b) * LD + 16 * b + n0, 0, acc);
      store_tile(Tf + (16 * b) * LD + 16 * a + n0, acc, 1.f);
    }
    sync();
    if (w < 4) {
      float acc[4];
      tile_mma_x3<2>(Tf + (16 * a) * LD + 16 * a, Tf + (16 * b) * LD + 16 * a + n0, 0, acc);
      store_tile(Tf + (16 * a) * LD + 16 * b + n0, acc, -1.f);
    }
    sync();
  }
  // (3) X = N_{[23],[01]} T_{[01],[01]} parked in rows 0..31, columns 32..63; then the lower-left 32 x 32
  // block of T = -T_{[23],[23]} X.  Warp w < 8 takes rows 16 (w / 4) .., columns 8 (w % 4) .. of each product.
  // Blocks that hold parked products instead of zeros are skipped: T_{[01],[01]} rows 0..15 past column 15
  // (M of the pair (1, 0)), and T_{[23],[23]} rows 32..47 past column 47 (M of the pair (3, 2)).
  {
    const int mt = (w >> 2) & 1, n0 = 8 * (w & 3);
    if (w < 8) {
      float acc[4];
      if (n0 >= 16) {
        tile_mma_x3<2>(Nf + (32 + 16 * mt) * LD + 16, Tf + 16 * LD + n0, 0, acc);
      } else {
        tile_mma_x3<4>(Nf + (32 + 16 * mt) * LD, Tf + n0, 0, acc);
      }
      store_tile(Tf + (16 * mt) * LD + 32 + n0, acc, 1.f);
    }
    sync();
    if (w < 8) {
      float acc[4];
      if (mt == 0) {
        tile_mma_x3<2>(Tf + 32 * LD + 32, Tf + 32 + n0, 0, acc);
      } else {
        tile_mma_x3<4>(Tf + 48 * LD + 32, Tf + 32 + n0, 0, acc);
      }
      store_tile(Tf + (32 + 16 * mt) * LD + n0, acc, -1.f);
    }
    sync();
  }
}

}  // namespace chunk
}  // namespace kdn
