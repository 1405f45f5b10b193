// Backward of the Kalman scans' uncertainty sides (the training-time adjoints), around the memory backward.
//
// Isotropic (Kalman Delta Networks, Abstract: Isotropic KDN keeps one uncertainty scalar per head).  Per
// token (the reading the forward kernels take): c^- = a^2 c + Qn, s = c^- ||k||^2 + r, beta = c^- / s, the
// memory write of the gated delta rule with that beta, and the mean-field update
// c = d_k c^- r / (d_k r + c^- ||k||^2).  Given dbeta_t from the memory backward (the delta rule's
// adjoint with beta as an input), the scalar chain is walked backwards with the adjoint cb of c:
//   dc^- = dbeta / s - dbeta c^- ||k||^2 / s^2 + cb (d_k r)^2 / den^2,   den = d_k r + c^- ||k||^2,
//   dr  = -dbeta c^- / s^2 + cb d_k c^-^2 ||k||^2 / den^2,
//   d||k||^2 = -dbeta c^-^2 / s^2 - cb d_k c^-^2 r / den^2   (dk_t += 2 d||k||^2 k_t),
//   da += 2 a c dc^-,  dQn = dc^-,  cb <- a^2 dc^-   (dc0 = cb after token 0).
//
// Diagonal (the same page: mean-field variational Kalman with a diagonal covariance).  Per token and
// coordinate: p^- = a^2 p + Qn, s = sum_i p^-_i k_i^2 + r, g = p^- o k / s, p = p^- r / (r + p^- k^2).  Given
// dG_t from the memory backward with the gains as inputs, with the adjoint pb of p:
//   dp^- = dG o k / s + pb r^2 / den^2 + ds k^2,   ds = -(dG . g) / s,   den = r + p^- k^2,
//   dk += dG o p^- / s - 2 pb p^-^2 r k / den^2 + 2 ds p^- k,
//   dr  = sum_i pb_i (p^-_i k_i)^2 / den_i^2 + ds,   da += 2 a (dp^- . p),   dQn = sum_i dp^-_i,
//   pb <- a^2 dp^-   (dp0 = pb after token 0).
// Each side has a forward kernel (storing what the reverse chain needs) and a backward kernel, one warp per
// head walking the tokens in order (the chains are serial in t; the lanes share each token's key).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace kdn {

namespace {

// The chains are serial in t and bound by load latency, so each warp loads a batch of kTB tokens at once
// (lane u < kTB the scalars of token t0 + u, every lane its coordinates of all kTB keys) and then steps
// through the batch in registers.
constexpr int kTB = 8;

template <int NPL>
__global__ void __launch_bounds__(32) iso_forward_kernel(IsoBwdArgs p) {
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const size_t tok0 = (size_t)bh * L;
  float c = p.c0 != nullptr ? p.c0[bh] : 1.f;
  for (int t0 = 0; t0 < L; t0 += kTB) {
    const int nb = min(kTB, L - t0);
    float sa = 1.f, sr = 1.f, sq = 0.f;
    if (lane < nb) {
      const size_t ti = tok0 + t0 + lane;
      sa = p.a != nullptr ? p.a[ti] : 1.f, sr = p.r[ti], sq = p.qn != nullptr ? p.qn[ti] : p.qn_scalar;
    }
    float kk[kTB];
#pragma unroll
    for (int u = 0; u < kTB; ++u) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        const float x = u < nb && i < D ? load_elem(p.k, (tok0 + t0 + u) * D + i, p.in_dtype) : 0.f;
        acc = fmaf(x, x, acc);
      }
      kk[u] = acc;
    }
#pragma unroll
    for (int u = 0; u < kTB; ++u) kk[u] = warp_sum(kk[u]);
    float beta_mine = 0.f, c_mine = 0.f, kk_mine = 0.f;
#pragma unroll
    for (int u = 0; u < kTB; ++u) {
      const float at = __shfl_sync(0xffffffffu, sa, u), rt = __shfl_sync(0xffffffffu, sr, u);
      const float qt = __shfl_sync(0xffffffffu, sq, u);
      const float cm = fmaf(at * at, c, qt);
      if (lane == u) beta_mine = cm / fmaf(cm, kk[u], rt), c_mine = c, kk_mine = kk[u];
      if (u < nb) c = (float)D * cm * rt / fmaf((float)D, rt, cm * kk[u]);
    }
    if (lane < nb) {
      const size_t ti = tok0 + t0 + lane;
      p.beta[ti] = beta_mine, p.cprev[ti] = c_mine, p.knorm2[ti] = kk_mine;
    }
  }
}

template <int NPL>
__global__ void __launch_bounds__(32) iso_backward_kernel(IsoBwdArgs p) {
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const size_t tok0 = (size_t)bh * L;
  float cb = p.dc_L != nullptr ? p.dc_L[bh] : 0.f;
  const float fd = (float)D;
  const int nbatch = (L + kTB - 1) / kTB;
  for (int bi = nbatch - 1; bi >= 0; --bi) {
    const int t0 = bi * kTB, nb = min(kTB, L - t0);
    float sa = 1.f, sr = 1.f, sq = 0.f, sc = 0.f, skk = 0.f, sdb = 0.f, sda = 0.f;
    if (lane < nb) {
      const size_t ti = tok0 + t0 + lane;
      sa = p.a != nullptr ? p.a[ti] : 1.f, sr = p.r[ti], sq = p.qn != nullptr ? p.qn[ti] : p.qn_scalar;
      sc = p.cprev[ti], skk = p.knorm2[ti], sdb = p.dbeta[ti];
      if (p.da != nullptr) sda = p.da[ti];
    }
    float kv[kTB][NPL], dko[kTB][NPL];  // the batch's keys and key gradients, loaded at once
#pragma unroll
    for (int u = 0; u < kTB; ++u)
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        const bool ok = u < nb && i < D;
        const size_t off = (tok0 + t0 + u) * D + i;
        kv[u][e] = ok ? load_elem(p.k, off, p.in_dtype) : 0.f;
        dko[u][e] = ok ? p.dk[off] : 0.f;
      }
    float dr_mine = 0.f, dqn_mine = 0.f, da_mine = sda, dkk_b[kTB];
#pragma unroll
    for (int u = kTB - 1; u >= 0; --u) {
      const float at = __shfl_sync(0xffffffffu, sa, u), rt = __shfl_sync(0xffffffffu, sr, u);
      const float qt = __shfl_sync(0xffffffffu, sq, u), c = __shfl_sync(0xffffffffu, sc, u);
      const float kk = __shfl_sync(0xffffffffu, skk, u), db = __shfl_sync(0xffffffffu, sdb, u);
      dkk_b[u] = 0.f;
      if (u < nb) {
        const float cm = fmaf(at * at, c, qt);
        const float st = fmaf(cm, kk, rt), den = fmaf(fd, rt, cm * kk);
        const float is2 = 1.f / (st * st), id2 = 1.f / (den * den);
        const float dcm = db / st - db * cm * kk * is2 + cb * (fd * rt) * (fd * rt) * id2;
        const float dr = -db * cm * is2 + cb * fd * cm * cm * kk * id2;
        dkk_b[u] = -db * cm * cm * is2 - cb * fd * cm * cm * rt * id2;
        if (lane == u) dr_mine = dr, dqn_mine = dcm, da_mine += 2.f * at * c * dcm;
        cb = at * at * dcm;
      }
    }
#pragma unroll
    for (int u = 0; u < kTB; ++u)
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        if (u < nb && i < D) p.dk[(tok0 + t0 + u) * D + i] = fmaf(2.f * dkk_b[u], kv[u][e], dko[u][e]);
      }
    if (lane < nb) {
      const size_t ti = tok0 + t0 + lane;
      p.dr[ti] = dr_mine, p.dqn[ti] = dqn_mine;
      if (p.da != nullptr) p.da[ti] = da_mine;
    }
  }
  if (lane == 0) p.dc0[bh] = cb;
}

template <int NPL>
__global__ void __launch_bounds__(32) diag_forward_kernel(DiagBwdArgs p) {
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const size_t tok0 = (size_t)bh * L;
  float pv[NPL];
#pragma unroll
  for (int e = 0; e < NPL; ++e) {
    const int i = lane + 32 * e;
    pv[e] = i < D ? (p.p0 != nullptr ? p.p0[(size_t)bh * D + i] : 1.f) : 0.f;
  }
  for (int t0 = 0; t0 < L; t0 += kTB) {
    const int nb = min(kTB, L - t0);
    float sa = 1.f, sr = 1.f, sq = 0.f;
    if (lane < nb) {
      const size_t ti = tok0 + t0 + lane;
      sa = p.a != nullptr ? p.a[ti] : 1.f, sr = p.r[ti], sq = p.qn != nullptr ? p.qn[ti] : p.qn_scalar;
    }
    float kv[kTB][NPL];
#pragma unroll
    for (int u = 0; u < kTB; ++u)
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        kv[u][e] = u < nb && i < D ? load_elem(p.k, (tok0 + t0 + u) * D + i, p.in_dtype) : 0.f;
      }
#pragma unroll
    for (int u = 0; u < kTB; ++u) {
      if (u >= nb) break;
      const float at = __shfl_sync(0xffffffffu, sa, u), rt = __shfl_sync(0xffffffffu, sr, u);
      const float qt = __shfl_sync(0xffffffffu, sq, u);
      float pm[NPL], sum = 0.f;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        pm[e] = fmaf(at * at, pv[e], qt);
        sum = fmaf(pm[e] * kv[u][e], kv[u][e], sum);
      }
      const float is = 1.f / (warp_sum(sum) + rt);
      const size_t ti = tok0 + t0 + u;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        if (i < D) {
          p.gains[ti * D + i] = pm[e] * kv[u][e] * is;
          p.pprev[ti * D + i] = pv[e];
        }
        pv[e] = pm[e] * rt / fmaf(pm[e] * kv[u][e], kv[u][e], rt);
      }
    }
  }
}

template <int NPL>
__global__ void __launch_bounds__(32) diag_backward_kernel(DiagBwdArgs p) {
  constexpr int TB = 4;  // tokens per batch (four d_k vectors per token stay in registers)
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const size_t tok0 = (size_t)bh * L;
  float pb[NPL];
#pragma unroll
  for (int e = 0; e < NPL; ++e) {
    const int i = lane + 32 * e;
    pb[e] = i < D && p.dp_L != nullptr ? p.dp_L[(size_t)bh * D + i] : 0.f;
  }
  const int nbatch = (L + TB - 1) / TB;
  for (int bi = nbatch - 1; bi >= 0; --bi) {
    const int t0 = bi * TB, nb = min(TB, L - t0);
    float sa = 1.f, sr = 1.f, sq = 0.f, sda = 0.f;
    if (lane < nb) {
      const size_t ti = tok0 + t0 + lane;
      sa = p.a != nullptr ? p.a[ti] : 1.f, sr = p.r[ti], sq = p.qn != nullptr ? p.qn[ti] : p.qn_scalar;
      if (p.da != nullptr) sda = p.da[ti];
    }
    float kv[TB][NPL], pp[TB][NPL], dg[TB][NPL], dko[TB][NPL];
#pragma unroll
    for (int u = 0; u < TB; ++u)
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        const bool ok = u < nb && i < D;
        const size_t off = (tok0 + t0 + u) * D + i;
        kv[u][e] = ok ? load_elem(p.k, off, p.in_dtype) : 0.f;
        pp[u][e] = ok ? p.pprev[off] : 0.f;
        dg[u][e] = ok ? p.dgain[off] : 0.f;
        dko[u][e] = ok ? p.dk[off] : 0.f;
      }
    float dr_mine = 0.f, dqn_mine = 0.f, da_mine = sda;
#pragma unroll
    for (int u = TB - 1; u >= 0; --u) {
      const float at = __shfl_sync(0xffffffffu, sa, u), rt = __shfl_sync(0xffffffffu, sr, u);
      const float qt = __shfl_sync(0xffffffffu, sq, u);
      if (u >= nb) continue;  // uniform over the warp
      float pm[NPL], sum = 0.f;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        pm[e] = i < D ? fmaf(at * at, pp[u][e], qt) : 0.f;
        sum = fmaf(pm[e] * kv[u][e], kv[u][e], sum);
      }
      const float is = 1.f / (warp_sum(sum) + rt);
      float dgg = 0.f;  // dG . g
#pragma unroll
      for (int e = 0; e < NPL; ++e) dgg = fmaf(dg[u][e], pm[e] * kv[u][e] * is, dgg);
      const float ds = -warp_sum(dgg) * is;
      float drp = 0.f, dap = 0.f, dqp = 0.f;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        const float k1 = kv[u][e], m1 = pm[e];
        const float den = fmaf(m1 * k1, k1, rt), id2 = 1.f / (den * den);
        float dpm = dg[u][e] * k1 * is + pb[e] * rt * rt * id2 + ds * k1 * k1;
        dko[u][e] += dg[u][e] * m1 * is - 2.f * pb[e] * m1 * m1 * rt * k1 * id2 + 2.f * ds * m1 * k1;
        drp = fmaf(pb[e] * (m1 * k1) * (m1 * k1), id2, drp);
        if (i >= D) dpm = 0.f;
        dap = fmaf(dpm, pp[u][e], dap);
        dqp += dpm;
        pb[e] = at * at * dpm;
      }
      const float dr = warp_sum(drp) + ds, dav = warp_sum(dap), dqv = warp_sum(dqp);
      if (lane == u) dr_mine = dr, dqn_mine = dqv, da_mine += 2.f * at * dav;
    }
#pragma unroll
    for (int u = 0; u < TB; ++u)
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        if (u < nb && i < D) p.dk[(tok0 + t0 + u) * D + i] = dko[u][e];
      }
    if (lane < nb) {
      const size_t ti = tok0 + t0 + lane;
      p.dr[ti] = dr_mine, p.dqn[ti] = dqn_mine;
      if (p.da != nullptr) p.da[ti] = da_mine;
    }
  }
#pragma unroll
  for (int e = 0; e < NPL; ++e) {
    const int i = lane + 32 * e;
    if (i < D) p.dp0[(size_t)bh * D + i] = pb[e];
  }
}

}  // namespace

cudaError_t launch_iso_forward(const IsoBwdArgs& args, int BH, cudaStream_t stream) {
  if (BH <= 0 || args.L <= 0) return cudaSuccess;
  if (args.dk_dim <= 32) iso_forward_kernel<1><<<BH, 32, 0, stream>>>(args);
  else if (args.dk_dim <= 64) iso_forward_kernel<2><<<BH, 32, 0, stream>>>(args);
  else if (args.dk_dim <= 128) iso_forward_kernel<4><<<BH, 32, 0, stream>>>(args);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_iso_backward(const IsoBwdArgs& args, int BH, cudaStream_t stream) {
  if (BH <= 0) return cudaSuccess;
  if (args.dk_dim <= 32) iso_backward_kernel<1><<<BH, 32, 0, stream>>>(args);
  else if (args.dk_dim <= 64) iso_backward_kernel<2><<<BH, 32, 0, stream>>>(args);
  else if (args.dk_dim <= 128) iso_backward_kernel<4><<<BH, 32, 0, stream>>>(args);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace kdn

namespace kdn {

cudaError_t launch_diag_forward(const DiagBwdArgs& args, int BH, cudaStream_t stream) {
  if (BH <= 0 || args.L <= 0) return cudaSuccess;
  if (args.dk_dim <= 32) diag_forward_kernel<1><<<BH, 32, 0, stream>>>(args);
  else if (args.dk_dim <= 64) diag_forward_kernel<2><<<BH, 32, 0, stream>>>(args);
  else if (args.dk_dim <= 128) diag_forward_kernel<4><<<BH, 32, 0, stream>>>(args);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_diag_backward(const DiagBwdArgs& args, int BH, cudaStream_t stream) {
  if (BH <= 0) return cudaSuccess;
  if (args.dk_dim <= 32) diag_backward_kernel<1><<<BH, 32, 0, stream>>>(args);
  else if (args.dk_dim <= 64) diag_backward_kernel<2><<<BH, 32, 0, stream>>>(args);
  else if (args.dk_dim <= 128) diag_backward_kernel<4><<<BH, 32, 0, stream>>>(args);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace kdn
