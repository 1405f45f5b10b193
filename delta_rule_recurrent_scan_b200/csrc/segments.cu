// Segment-parallel scans: more than one CTA per head when there are too few heads to fill the GPU.
//
// Kalman Delta Networks, Abstract: the diagonal and isotropic uncertainty recurrences are Moebius maps,
// so they compose associatively and a sequence can be cut into segments whose maps are built
// independently and then chained.  The memory side is linear once the write strengths are known: for
// fixed gains the scan over one segment sends its start state S0 to M S0 + B (every step
// S <- a S + g (v - a S^T k)^T is affine in S).  So each head's sequence is cut into P equal segments
// and
//
//   1. (diagonal Kalman) every segment composes its per-coordinate uncertainty maps, and one thread
//      per coordinate chains them to get p at each segment start;
//   2. the chunk kernel runs every segment twice in parallel, from S0 = 0 (giving B) and from S0 = I
//      (giving M + B); at d = 64 once instead, on the d x 2d state [S | M] from [0 | I] whose extra
//      columns see zero values (the columns of the state evolve independently for fixed gains, so
//      the first block ends at B and the second at M; 2d = 128 fills the chunk kernel's d_v lanes);
//   3. one pass per head chains S_{s+1} = M_s S_s + B_s across segments, in fp32;
//   4. the chunk kernel runs every segment once more from its true start state, writing o and m.
//
// This file holds the kernels of steps 1 and 3 and the initialisation of step 2.  Segment s of head h
// is tokens [s L/P, (s+1) L/P), so the [BH, L, d] inputs viewed as [BH P, L/P, d] are the segments as
// heads of their own, and the chunk kernels run on that view unchanged.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "mobius.cuh"

namespace kdn {

namespace {

using mobius::Mob;

constexpr int kMapThreads = 512;

// 16-byte asynchronous global -> shared copy (Ampere-style cp.async, cached in L2 only)
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ float load_key(const void* k, size_t i, int dtype) {
  if (dtype == kBF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(k)[i]);
  return reinterpret_cast<const float*>(k)[i];
}

// Step 1a: the composed uncertainty map of every (head, segment < P - 1) and key coordinate.  Per
// coordinate i the diagonal-Kalman token map is  p -> p^- / (1 + w p^-),  p^- = a^2 p + Qn,
// w = k_i^2 / r  (the mean-field projection p^- r / (r + p^- k_i^2)), which is the matrix
// [[a^2, Qn], [w a^2, w Qn + 1]].  kMapThreads / DK token groups compose contiguous parts of the
// segment; group 0 then chains the parts in token order.
template <int DK>
__global__ void __launch_bounds__(kMapThreads) seg_maps_kernel(SegArgs p) {
  constexpr int G = kMapThreads / DK;
  __shared__ float4 part[G][DK];
  const int s = blockIdx.x, h = blockIdx.y;
  const int i = threadIdx.x % DK, g = threadIdx.x / DK;
  const int Ls = p.L / p.P;
  const int per = (Ls + G - 1) / G;
  const int t_lo = s * Ls + g * per;
  const int t_hi = min(s * Ls + Ls, t_lo + per);
  const size_t row0 = (size_t)h * p.L;
  Mob acc = mobius::identity();
  for (int t = t_lo; t < t_hi; ++t) {
    const size_t ti = row0 + t;
    const float av = p.a ? p.a[ti] : 1.f;
    const float qv = p.qn ? p.qn[ti] : p.qn_scalar;
    const float kv = load_key(p.k, ti * DK + i, p.in_dtype);
    const float w = kv * kv / p.r[ti];
    acc = mobius::compose(mobius::iso_token(av * av, qv, w), acc);
  }
  part[g][i] = make_float4(acc.a, acc.b, acc.c, acc.d);
  __syncthreads();
  if (g == 0) {
    Mob m = mobius::identity();
#pragma unroll
    for (int q = 0; q < G; ++q) {
      const float4 f = part[q][i];
      m = mobius::compose(Mob{f.x, f.y, f.z, f.w}, m);
    }
    if (!(isfinite(m.a) && isfinite(m.b) && isfinite(m.c))) raise_status(p.status, kStatusNumeric);
    p.maps[((size_t)h * p.P + s) * DK + i] = make_float4(m.a, m.b, m.c, m.d);
  }
}

// Step 1b: p at every segment start, p_{s+1} = map_s(p_s), written to each of the ncopy buffers (each
// later chunk-kernel run updates its own copy in place).
template <int DK>
__global__ void __launch_bounds__(DK) seg_prefix_kernel(SegArgs p) {
  const int h = blockIdx.x, i = threadIdx.x;
  float x = p.p0[(size_t)h * DK + i];
  bool bad = false;
  for (int s = 0; s < p.P; ++s) {
    const size_t j = ((size_t)h * p.P + s) * DK + i;
    for (int c = 0; c < p.ncopy; ++c) p.pcopy[c][j] = x;
    if (s + 1 < p.P) {
      const float4 f = p.maps[j];
      x = mobius::apply(Mob{f.x, f.y, f.z, f.w}, x);
      bad |= !(x >= 0.f && isfinite(x));
    }
  }
  if (bad) raise_status(p.status, kStatusNumeric);
}

// Step 2's start state at d = 64 on [S | M]: [0 | I] ([d][2 d]) for every segment.
__global__ void __launch_bounds__(256) seg_init_aug_kernel(float* SA, int d) {
  float* base = SA + (size_t)blockIdx.x * d * 2 * d;
  for (int u = threadIdx.x; u < 2 * d * d; u += blockDim.x) {
    const int r = u / (2 * d), c = u % (2 * d);
    base[u] = (c == d + r) ? 1.f : 0.f;
  }
}

// Step 2's start states: S0 = 0 in Sz and S0 = I in SI for every segment (d_k = d_v).
__global__ void __launch_bounds__(256) seg_init_kernel(float* Sz, float* SI, int d) {
  const size_t base = (size_t)blockIdx.x * d * d;
  float4* z = reinterpret_cast<float4*>(Sz + base);
  float4* e = reinterpret_cast<float4*>(SI + base);
  for (int u = threadIdx.x; u < d * d / 4; u += blockDim.x) {
    const int r = (4 * u) / d, c = (4 * u) % d;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    z[u] = v;
    if (r >= c && r < c + 4) (&v.x)[r - c] = 1.f;
    e[u] = v;
  }
}

// Step 3 (d = 64 or 128): S_{s+1} = (SI_s - Sz_s) S_s + Sz_s (at d = 64: M_s S_s + B_s from the run on [S | M])
// for one head and a slab of kSlab columns; every
// S_s (s = 0 .. P-1, S_0 the caller's state) is written to Sc.  Per segment the CTA stages SI_s and Sz_s in
// shared memory with asynchronous 16-byte copies (rows padded by 4 floats; every slab of the head reads the
// same L2-resident rows), then each thread forms one row r of the slab (kCombThreads / D threads per row,
// kSlab / that many columns each) from its row of M_s and 16-byte broadcast loads of the slab of S_s.
constexpr int kSlab = 16;
constexpr int kCombThreads = 256;

template <int D>
struct CombLayout {
  static constexpr int RS = D + 4;                               // padded row of the staged SI_s, Sz_s
  static constexpr size_t SMEM = sizeof(float) * (2 * (size_t)D * RS + (size_t)D * kSlab);
};

template <int D>
__global__ void __launch_bounds__(kCombThreads) seg_combine_kernel(SegArgs p) {
  constexpr int TPR = kCombThreads / D;          // threads per row: 2 at D = 128, 4 at D = 64
  constexpr int CPT = kSlab / TPR;               // columns per thread: 8 or 4
  constexpr int RS = CombLayout<D>::RS;
  static_assert(CPT % 4 == 0, "whole 16-byte column groups per thread");
  extern __shared__ __align__(16) float sm[];
  float* SIs = sm;                               // [D][RS]
  float* Szs = sm + D * RS;                      // [D][RS]
  float* X = sm + 2 * D * RS;                    // [D][kSlab]: the slab of S_s
  const int h = blockIdx.y, c0 = blockIdx.x * kSlab;
  const int tid = threadIdx.x;
  const int r = tid / TPR, cg = (tid % TPR) * CPT;
  const size_t DD = (size_t)D * D;

  for (int e = tid; e < D * kSlab; e += kCombThreads) {
    const int rr = e / kSlab, cc = e % kSlab;
    X[e] = p.S[(size_t)h * DD + (size_t)rr * D + c0 + cc];
  }
  __syncthreads();
  for (int s = 0; s < p.P; ++s) {
    const size_t j = (size_t)h * p.P + s;
    if (s + 1 < p.P) {
      // rows of SI_s (or M_s) and Sz_s (B_s): [d][d] each, or side by side in rows of 2 d
      const int ld = p.aug ? 2 * D : D;
      const float* Szg = p.Sz + j * D * ld;
      const float* SIg = p.aug ? Szg + D : p.SI + j * DD;
      for (int q = tid; q < D * D / 4; q += kCombThreads) {
        const int rr = (4 * q) / D, cc = (4 * q) % D;
        cp_async16(SIs + rr * RS + cc, SIg + (size_t)rr * ld + cc);
        cp_async16(Szs + rr * RS + cc, Szg + (size_t)rr * ld + cc);
      }
    }
    for (int e = tid; e < D * kSlab; e += kCombThreads) {
      const int rr = e / kSlab, cc = e % kSlab;
      p.Sc[j * DD + (size_t)rr * D + c0 + cc] = X[e];
    }
    if (s + 1 == p.P) break;
    cp_async_wait_all();
    __syncthreads();                              // SI_s, Sz_s staged
    float acc[CPT];
#pragma unroll
    for (int u = 0; u < CPT; ++u) acc[u] = Szs[r * RS + c0 + cg + u];
#pragma unroll 4
    for (int kq = 0; kq < D / 4; ++kq) {
      const float4 a4 = *reinterpret_cast<const float4*>(SIs + r * RS + 4 * kq);
      const float4 b4 = *reinterpret_cast<const float4*>(Szs + r * RS + 4 * kq);
      const float4 m4 = p.aug ? a4 : make_float4(a4.x - b4.x, a4.y - b4.y, a4.z - b4.z, a4.w - b4.w);
      const float m[4] = {m4.x, m4.y, m4.z, m4.w};  // M_s[r][4 kq ..]
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4* xr = reinterpret_cast<const float4*>(X + (4 * kq + e) * kSlab + cg);
#pragma unroll
        for (int u4 = 0; u4 < CPT / 4; ++u4) {
          const float4 x4 = xr[u4];
          acc[4 * u4 + 0] = fmaf(m[e], x4.x, acc[4 * u4 + 0]);
          acc[4 * u4 + 1] = fmaf(m[e], x4.y, acc[4 * u4 + 1]);
          acc[4 * u4 + 2] = fmaf(m[e], x4.z, acc[4 * u4 + 2]);
          acc[4 * u4 + 3] = fmaf(m[e], x4.w, acc[4 * u4 + 3]);
        }
      }
    }
    __syncthreads();                              // every thread is done with X, SI_s and Sz_s
    bool bad = false;
#pragma unroll
    for (int u4 = 0; u4 < CPT / 4; ++u4) {
      *reinterpret_cast<float4*>(X + r * kSlab + cg + 4 * u4) =
          make_float4(acc[4 * u4], acc[4 * u4 + 1], acc[4 * u4 + 2], acc[4 * u4 + 3]);
      bad |= !(isfinite(acc[4 * u4]) && isfinite(acc[4 * u4 + 1]) && isfinite(acc[4 * u4 + 2]) &&
               isfinite(acc[4 * u4 + 3]));
    }
    if (bad) raise_status(p.status, kStatusNumeric);
    __syncthreads();
  }
}

template <int D>
cudaError_t launch_combine(const SegArgs& p, int BH, cudaStream_t stream) {
  constexpr size_t smem = CombLayout<D>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(seg_combine_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  seg_combine_kernel<D><<<dim3(D / kSlab, BH), kCombThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_seg_uncertainty(int dk, const SegArgs& p, int BH, cudaStream_t stream) {
  if (p.P > 1) {
    const dim3 grid(p.P - 1, BH);
    switch (dk) {
      case 16: seg_maps_kernel<16><<<grid, kMapThreads, 0, stream>>>(p); break;
      case 32: seg_maps_kernel<32><<<grid, kMapThreads, 0, stream>>>(p); break;
      case 64: seg_maps_kernel<64><<<grid, kMapThreads, 0, stream>>>(p); break;
      case 128: seg_maps_kernel<128><<<grid, kMapThreads, 0, stream>>>(p); break;
      default: return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  switch (dk) {
    case 16: seg_prefix_kernel<16><<<BH, 16, 0, stream>>>(p); break;
    case 32: seg_prefix_kernel<32><<<BH, 32, 0, stream>>>(p); break;
    case 64: seg_prefix_kernel<64><<<BH, 64, 0, stream>>>(p); break;
    case 128: seg_prefix_kernel<128><<<BH, 128, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_seg_init(int d, const SegArgs& p, int BH, cudaStream_t stream) {
  if (d % 4 != 0) return cudaErrorInvalidValue;
  if (p.aug)
    seg_init_aug_kernel<<<BH * p.P, 256, 0, stream>>>(p.Sz, d);
  else
    seg_init_kernel<<<BH * p.P, 256, 0, stream>>>(p.Sz, p.SI, d);
  return cudaGetLastError();
}

cudaError_t launch_seg_combine(int d, const SegArgs& p, int BH, cudaStream_t stream) {
  switch (d) {
    case 64: return launch_combine<64>(p, BH, stream);
    case 128: return launch_combine<128>(p, BH, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kdn
