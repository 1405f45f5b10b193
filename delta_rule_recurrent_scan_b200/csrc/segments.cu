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
//      (giving M + B);
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

// Step 3 (d = 64 or 128): S_{s+1} = (SI_s - Sz_s) S_s + Sz_s for one head and a slab of kSlab columns; every
// S_s (s = 0 .. P-1, S_0 the caller's state) is written to Sc.  M_s = SI_s - Sz_s is staged
// transposed in shared memory (rows padded by 4 floats) so that each thread reads the 8 rows of its
// outputs with two 16-byte loads per k.
constexpr int kSlab = 16;
constexpr int kCombThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCombThreads) seg_combine_kernel(SegArgs p) {
  constexpr int MT = D + 4;                       // padded row of the transposed M
  constexpr int RPT = D * kSlab / kCombThreads;   // output rows per thread (8 at D = 128)
  static_assert(RPT % 4 == 0, "two or more 16-byte row groups per thread");
  extern __shared__ __align__(16) float sm[];
  float* Mt = sm;                                 // [D][MT]: Mt[k][r] = M[r][k]
  float* X = sm + D * MT;                         // [D][kSlab]
  const int h = blockIdx.y, c0 = blockIdx.x * kSlab;
  const int tid = threadIdx.x;
  const int c = tid % kSlab, r0 = (tid / kSlab) * RPT;
  const size_t DD = (size_t)D * D;

  for (int e = tid; e < D * kSlab; e += kCombThreads) {
    const int r = e / kSlab, cc = e % kSlab;
    X[e] = p.S[(size_t)h * DD + (size_t)r * D + c0 + cc];
  }
  __syncthreads();
  for (int s = 0; s < p.P; ++s) {
    const size_t j = (size_t)h * p.P + s;
    for (int e = tid; e < D * kSlab; e += kCombThreads) {
      const int r = e / kSlab, cc = e % kSlab;
      p.Sc[j * DD + (size_t)r * D + c0 + cc] = X[e];
    }
    if (s + 1 == p.P) break;
    const float* Sz = p.Sz + j * DD;
    const float* SI = p.SI + j * DD;
    for (int e = tid; e < D * D; e += kCombThreads) {
      const int r = e / D, k = e % D;
      Mt[k * MT + r] = SI[e] - Sz[e];
    }
    __syncthreads();
    float acc[RPT];
#pragma unroll
    for (int u = 0; u < RPT; ++u) acc[u] = Sz[(size_t)(r0 + u) * D + c0 + c];
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      const float x = X[k * kSlab + c];
      const float4* mr = reinterpret_cast<const float4*>(Mt + k * MT + r0);
#pragma unroll
      for (int u4 = 0; u4 < RPT / 4; ++u4) {
        const float4 m4 = mr[u4];
        acc[4 * u4 + 0] = fmaf(m4.x, x, acc[4 * u4 + 0]);
        acc[4 * u4 + 1] = fmaf(m4.y, x, acc[4 * u4 + 1]);
        acc[4 * u4 + 2] = fmaf(m4.z, x, acc[4 * u4 + 2]);
        acc[4 * u4 + 3] = fmaf(m4.w, x, acc[4 * u4 + 3]);
      }
    }
    __syncthreads();                              // every thread is done with X and Mt
    bool bad = false;
#pragma unroll
    for (int u = 0; u < RPT; ++u) {
      X[(r0 + u) * kSlab + c] = acc[u];
      bad |= !isfinite(acc[u]);
    }
    if (bad) raise_status(p.status, kStatusNumeric);
    __syncthreads();
  }
}

template <int D>
cudaError_t launch_combine(const SegArgs& p, int BH, cudaStream_t stream) {
  constexpr size_t smem = sizeof(float) * ((size_t)D * (D + 4) + (size_t)D * kSlab);
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
