// One-token decode step: a bandwidth-bound read-modify-write of the resident state.
//
// Kalman Delta Networks, Abstract: constant-memory decoding with a fixed-size
// recurrent memory.  Per head the d_k x d_v fp32 state is read once from HBM
// (16-byte streaming loads, a warp covers whole rows), updated in registers and
// written once; the token's q, k, v and the gain are staged in shared memory.
//
//   delta  g = beta k
//   diag   p^- = a^2 p + Qn, s = sum p^- k^2 + r, g = p^- k / s,
//          p <- p^- r / (r + p^- k^2)
//   iso    c^- = a^2 c + Qn, g = c^- k / (c^- ||k||^2 + r), c <- d_k c^- r / (d_k r + c^- ||k||^2)
//   e = v - a S^T k,  o = a S^T q + (g . q) e,  S <- a S + g e^T,  m = ||g|| ||e||
#include "common.cuh"
#include "kernels.h"

namespace kdn {

enum DecodeMode : int { kDecDelta = 0, kDecDiag = 1, kDecIso = 2 };

template <int DK, int DV, int MODE>
__global__ void __launch_bounds__(RowBlockLayout<DK, DV>::kThreads) decode_kernel(DecodeArgs args) {
  constexpr bool kDiag = MODE == kDecDiag;
  using Lay = RowBlockLayout<DK, DV>;
  constexpr int NT = Lay::kThreads, CG = Lay::kColGroups, RG = Lay::kRowGroups, RPT = Lay::kRowsPerThread;
  constexpr int DVW = (DV + 31) / 32 * 32;
  constexpr int PER = (DK + 31) / 32;
  static_assert(NT >= DVW, "phase B needs whole warps over d_v");

  __shared__ float k_s[DK], q_s[DK], g_s[DK], v_s[DV];
  __shared__ __align__(16) float red[RG][2][DV];
  __shared__ float e_s[DV];
  __shared__ float ered[DVW / 32];
  __shared__ float gq_s, gn_s;

  const int bh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = tid % CG, rg = tid / CG;

  float* Sg = args.S + (size_t)bh * DK * DV;
  float4 S4[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) S4[i] = __ldcs(reinterpret_cast<const float4*>(Sg + (size_t)(rg + i * RG) * DV + cg * 4));

  for (int i = tid; i < DK; i += NT) {
    k_s[i] = load_elem(args.k, (size_t)bh * DK + i, args.in_dtype);
    q_s[i] = load_elem(args.q, (size_t)bh * DK + i, args.in_dtype);
  }
  for (int i = tid; i < DV; i += NT) v_s[i] = load_elem(args.v, (size_t)bh * DV + i, args.in_dtype);
  const float a = args.a ? args.a[bh] : 1.f;
  __syncthreads();

  if (warp == 0) {
    float g[PER], sq = 0.f, sn = 0.f;
    if constexpr (kDiag) {
      const float r = args.r[bh];
      float pp[PER], kk[PER], part = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        kk[i] = c < DK ? k_s[c] : 0.f;
        pp[i] = c < DK ? fmaf(a * a, args.p[(size_t)bh * DK + c], args.qn_scalar) : 0.f;
        part = fmaf(pp[i] * kk[i], kk[i], part);
      }
      const float inv_s = 1.f / (warp_sum(part) + r);
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        g[i] = pp[i] * kk[i] * inv_s;
        if (c < DK) args.p[(size_t)bh * DK + c] = pp[i] * r / fmaf(pp[i] * kk[i], kk[i], r);
      }
    } else if constexpr (MODE == kDecIso) {
      // one uncertainty scalar per head, kept in the p slot
      const float r = args.r[bh];
      float kk = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        const float kv = c < DK ? k_s[c] : 0.f;
        kk = fmaf(kv, kv, kk);
      }
      kk = warp_sum(kk);
      const float cm = fmaf(a * a, args.p[bh], args.qn_scalar);
      const float beta = cm / fmaf(cm, kk, r);
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        g[i] = c < DK ? beta * k_s[c] : 0.f;
      }
      __syncwarp();
      if (lane == 0) args.p[bh] = DK * cm * r / fmaf((float)DK, r, cm * kk);
    } else {
      const float beta = args.beta[bh];
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        g[i] = c < DK ? beta * k_s[c] : 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int c = lane + 32 * i;
      if (c < DK) {
        g_s[c] = g[i];
        sq = fmaf(g[i], q_s[c], sq);
        sn = fmaf(g[i], g[i], sn);
      }
    }
    sq = warp_sum(sq);
    sn = warp_sum(sn);
    if (lane == 0) gq_s = sq, gn_s = sn;
  }

  float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int row = rg + i * RG;
    const float kr = k_s[row], qr = q_s[row];
    const float s4[4] = {S4[i].x, S4[i].y, S4[i].z, S4[i].w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      pk[c] = fmaf(s4[c], kr, pk[c]);
      pq[c] = fmaf(s4[c], qr, pq[c]);
    }
  }
  *reinterpret_cast<float4*>(&red[rg][0][cg * 4]) = make_float4(pk[0], pk[1], pk[2], pk[3]);
  *reinterpret_cast<float4*>(&red[rg][1][cg * 4]) = make_float4(pq[0], pq[1], pq[2], pq[3]);
  __syncthreads();
  if (tid < DVW) {
    float e = 0.f;
    if (tid < DV) {
      float yk = 0.f, yq = 0.f;
#pragma unroll
      for (int r = 0; r < RG; ++r) yk += red[r][0][tid], yq += red[r][1][tid];
      e = v_s[tid] - a * yk;
      store_elem(args.o, (size_t)bh * DV + tid, fmaf(a, yq, gq_s * e), args.out_dtype);
      e_s[tid] = e;
    }
    const float es = warp_sum(e * e);
    if (lane == 0) ered[warp] = es;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int row = rg + i * RG;
    const float gr = g_s[row];
    float4 x = S4[i];
    x.x = fmaf(a, x.x, gr * e_s[cg * 4 + 0]);
    x.y = fmaf(a, x.y, gr * e_s[cg * 4 + 1]);
    x.z = fmaf(a, x.z, gr * e_s[cg * 4 + 2]);
    x.w = fmaf(a, x.w, gr * e_s[cg * 4 + 3]);
    __stcs(reinterpret_cast<float4*>(Sg + (size_t)row * DV + cg * 4), x);
  }
  if (tid == 0 && args.m != nullptr) {
    float es = 0.f;
#pragma unroll
    for (int w = 0; w < DVW / 32; ++w) es += ered[w];
    args.m[bh] = sqrtf(gn_s) * sqrtf(es);
  }
}

#define KDN_DEC_SWITCH(D, NAME, ...)          \
  switch (D) {                                \
    case 16: { constexpr int NAME = 16; __VA_ARGS__; } break;   \
    case 32: { constexpr int NAME = 32; __VA_ARGS__; } break;   \
    case 64: { constexpr int NAME = 64; __VA_ARGS__; } break;   \
    case 128: { constexpr int NAME = 128; __VA_ARGS__; } break; \
    default: return cudaErrorInvalidValue;    \
  }

cudaError_t launch_decode(int dk, int dv, int mode, const DecodeArgs& args, cudaStream_t stream) {
  if (args.BH <= 0) return cudaSuccess;
  KDN_DEC_SWITCH(dk, DK, KDN_DEC_SWITCH(dv, DV, {
    constexpr int NT = RowBlockLayout<DK, DV>::kThreads;
    if (mode == kDecDiag)
      decode_kernel<DK, DV, kDecDiag><<<args.BH, NT, 0, stream>>>(args);
    else if (mode == kDecIso)
      decode_kernel<DK, DV, kDecIso><<<args.BH, NT, 0, stream>>>(args);
    else
      decode_kernel<DK, DV, kDecDelta><<<args.BH, NT, 0, stream>>>(args);
  }));
  return cudaGetLastError();
}

}  // namespace kdn
