// Isotropic-covariance Kalman prologue: per-token write strengths from one uncertainty scalar per head.
//
// Kalman Delta Networks, Abstract: Isotropic KDN keeps a single uncertainty scalar per head, and its
// uncertainty recurrence is a Moebius map, which admits an associative scan of logarithmic depth.  With
// one scalar c per head (reading: propagate c^- = a_t^2 c + Qn_t; the mean is the exact posterior mean
// under the prior c^- I; the variance is the isotropic mean-field optimum d_k / tr(posterior precision)):
//
//   beta_t = c^-_t / (c^-_t ||k_t||^2 + r_t),    c_t = d_k c^-_t r_t / (d_k r_t + c^-_t ||k_t||^2),
//
// and the memory write is the delta rule's with these beta_t.  In homogeneous coordinates c = x / y one
// token is the matrix (divided through by d_k r_t)
//
//   M_t = [[a^2, Qn], [w a^2, w Qn + 1]],   w = ||k_t||^2 / (d_k r_t),
//
// and c after tokens 1..t is M_t ... M_1 applied to c_0.  One CTA per head: each tile of 2048 tokens gets
// its key norms (coalesced, shared by the lanes of a token), each thread composes the maps of its four
// tokens, a block-wide exclusive scan of those 2x2 products (warp shuffles, then one warp over the warp
// totals) gives every thread the map from the tile's start to its first token, and each thread then steps
// its four tokens exactly, writing beta_t.  Products are renormalised so that the lower-right entry is 1
// (the map is projective).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"
#include "mobius.cuh"

namespace kdn {

namespace {

constexpr int kIsoThreads = 512;
constexpr int kIsoPer = 4;                           // tokens per thread per tile
constexpr int kIsoTile = kIsoThreads * kIsoPer;      // 2048 tokens

using mobius::Mob;
using mobius::compose;
using mobius::identity;
using mobius::shfl_up;

template <int DK, bool BF16>
__global__ void __launch_bounds__(kIsoThreads) iso_beta_kernel(IsoArgs p) {
  constexpr int ES = BF16 ? 2 : 4;
  constexpr int ROW = DK * ES;                        // bytes per key row
  constexpr int LPT = ROW / 16;                       // lanes per token (16-byte loads)
  constexpr int TPL = 32 / LPT;                       // tokens per warp load

  __shared__ float knorm[kIsoTile];
  __shared__ Mob wtot[kIsoThreads / 32];
  __shared__ float c_carry;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x;
  const int L = p.L;
  const size_t base = (size_t)bh * L;
  const uint8_t* krow = reinterpret_cast<const uint8_t*>(p.k) + base * ROW;
  if (tid == 0) c_carry = p.c[bh];

  for (int t0 = 0; t0 < L; t0 += kIsoTile) {
    // ---- ||k_t||^2 for the tile: LPT lanes per token, 16-byte loads, several tokens in flight per warp
#pragma unroll 8
    for (int tb = warp * TPL; tb < kIsoTile; tb += (kIsoThreads / 32) * TPL) {
      const int t = tb + lane / LPT;
      float s = 0.f;
      if (t0 + t < L) {
        const uint4 u = *reinterpret_cast<const uint4*>(krow + (size_t)(t0 + t) * ROW + 16 * (lane % LPT));
        if (BF16) {
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h[e]);
            s = fmaf(f.x, f.x, fmaf(f.y, f.y, s));
          }
        } else {
          const float f[4] = {__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w)};
#pragma unroll
          for (int e = 0; e < 4; ++e) s = fmaf(f[e], f[e], s);
        }
      }
#pragma unroll
      for (int o = LPT / 2; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane % LPT == 0) knorm[t] = s;
    }
    __syncthreads();

    // ---- this thread's four tokens: scalars and the composed map
    float a2[kIsoPer], qv[kIsoPer], rv[kIsoPer], kk[kIsoPer];
    Mob mine = identity();
#pragma unroll
    for (int u = 0; u < kIsoPer; ++u) {
      const int t = kIsoPer * tid + u;
      const bool valid = t0 + t < L;
      const size_t ti = base + t0 + t;
      const float av = valid ? (p.a ? p.a[ti] : 1.f) : 1.f;
      a2[u] = av * av;
      qv[u] = valid ? (p.qn ? p.qn[ti] : p.qn_scalar) : 0.f;
      rv[u] = valid ? p.r[ti] : 1.f;
      kk[u] = valid ? knorm[t] : 0.f;
      const float w = kk[u] / (DK * rv[u]);
      const Mob mt = mobius::iso_token(a2[u], qv[u], w);
      mine = compose(mt, mine);
    }

    // ---- exclusive scan of the thread maps in token order
    Mob incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const Mob left = shfl_up(incl, o);
      if (lane >= o) incl = compose(incl, left);
    }
    Mob excl = shfl_up(incl, 1);
    if (lane == 0) excl = identity();
    if (lane == 31) wtot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      Mob x = lane < kIsoThreads / 32 ? wtot[lane] : identity();
#pragma unroll
      for (int o = 1; o < kIsoThreads / 32; o <<= 1) {
        const Mob left = shfl_up(x, o);
        if (lane >= o) x = compose(x, left);
      }
      Mob ex = shfl_up(x, 1);
      if (lane == 0) ex = identity();
      if (lane < kIsoThreads / 32) wtot[lane] = ex;  // exclusive prefix of the warps
    }
    __syncthreads();
    const Mob pre = compose(excl, wtot[warp]);       // tile start -> this thread's first token
    const float cin = c_carry;

    // ---- step the four tokens exactly from the value at the first one
    float c = (pre.a * cin + pre.b) / (pre.c * cin + pre.d);
    bool bad = false;
#pragma unroll
    for (int u = 0; u < kIsoPer; ++u) {
      const int t = kIsoPer * tid + u;
      const float cm = fmaf(a2[u], c, qv[u]);
      const float s = fmaf(cm, kk[u], rv[u]);
      if (t0 + t < L) {
        bad |= !(s > 0.f && isfinite(s) && cm >= 0.f);
        p.beta[base + t0 + t] = cm / s;
      }
      c = DK * cm * rv[u] / fmaf((float)DK, rv[u], cm * kk[u]);
    }
    if (bad) raise_status(p.status, kStatusNumeric);
    __syncthreads();                                 // every thread has read c_carry and knorm
    if (tid == kIsoThreads - 1) c_carry = c;         // the tile's last token
    __syncthreads();
  }
  if (tid == 0) p.c[bh] = c_carry;
}

template <int DK>
cudaError_t launch_dk(const IsoArgs& p, int BH, cudaStream_t stream) {
  if (p.in_dtype == kBF16)
    iso_beta_kernel<DK, true><<<BH, kIsoThreads, 0, stream>>>(p);
  else
    iso_beta_kernel<DK, false><<<BH, kIsoThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_iso_beta(int dk, const IsoArgs& p, int BH, cudaStream_t stream) {
  switch (dk) {
    case 16: return launch_dk<16>(p, BH, stream);
    case 32: return launch_dk<32>(p, BH, stream);
    case 64: return launch_dk<64>(p, BH, stream);
    case 128: return launch_dk<128>(p, BH, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kdn
