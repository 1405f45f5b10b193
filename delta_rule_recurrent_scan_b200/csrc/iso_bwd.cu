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
// head walking the tokens in order (the chains are serial in t; the warp shares each token's key).
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace kdn {

namespace {

__global__ void __launch_bounds__(32) iso_forward_kernel(IsoBwdArgs p) {
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const size_t tok0 = (size_t)bh * L;
  float c = p.c0 != nullptr ? p.c0[bh] : 1.f;
  for (int t = 0; t < L; ++t) {
    const size_t ti = tok0 + t;
    float kk = 0.f;
    for (int i = lane; i < D; i += 32) {
      const float x = load_elem(p.k, ti * D + i, p.in_dtype);
      kk = fmaf(x, x, kk);
    }
    kk = warp_sum(kk);
    const float at = p.a != nullptr ? p.a[ti] : 1.f, rt = p.r[ti];
    const float qt = p.qn != nullptr ? p.qn[ti] : p.qn_scalar;
    const float cm = fmaf(at * at, c, qt);
    if (lane == 0) {
      p.beta[ti] = cm / fmaf(cm, kk, rt);
      p.cprev[ti] = c;
      p.knorm2[ti] = kk;
    }
    c = (float)D * cm * rt / fmaf((float)D, rt, cm * kk);
  }
}

__global__ void __launch_bounds__(32) iso_backward_kernel(IsoBwdArgs p) {
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const size_t tok0 = (size_t)bh * L;
  float cb = p.dc_L != nullptr ? p.dc_L[bh] : 0.f;
  const float fd = (float)D;
  for (int t = L - 1; t >= 0; --t) {
    const size_t ti = tok0 + t;
    const float at = p.a != nullptr ? p.a[ti] : 1.f, rt = p.r[ti];
    const float qt = p.qn != nullptr ? p.qn[ti] : p.qn_scalar;
    const float c = p.cprev[ti], kk = p.knorm2[ti], db = p.dbeta[ti];
    const float cm = fmaf(at * at, c, qt);
    const float st = fmaf(cm, kk, rt), den = fmaf(fd, rt, cm * kk);
    const float is2 = 1.f / (st * st), id2 = 1.f / (den * den);
    float dcm = db / st - db * cm * kk * is2 + cb * (fd * rt) * (fd * rt) * id2;
    const float dr = -db * cm * is2 + cb * fd * cm * cm * kk * id2;
    const float dkk = -db * cm * cm * is2 - cb * fd * cm * cm * rt * id2;
    for (int i = lane; i < D; i += 32) {
      const size_t off = ti * D + i;
      p.dk[off] = fmaf(2.f * dkk, load_elem(p.k, off, p.in_dtype), p.dk[off]);
    }
    if (lane == 0) {
      p.dr[ti] = dr;
      p.dqn[ti] = dcm;
      if (p.da != nullptr) p.da[ti] += 2.f * at * c * dcm;
    }
    cb = at * at * dcm;
  }
  if (lane == 0) p.dc0[bh] = cb;
}

template <int NPL>
__global__ void __launch_bounds__(32) diag_forward_kernel(DiagBwdArgs p) {
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const size_t tok0 = (size_t)bh * L;
  float pv[NPL];
#pragma unroll
  for (int u = 0; u < NPL; ++u) {
    const int i = lane + 32 * u;
    pv[u] = i < D ? (p.p0 != nullptr ? p.p0[(size_t)bh * D + i] : 1.f) : 0.f;
  }
  for (int t = 0; t < L; ++t) {
    const size_t ti = tok0 + t;
    const float at = p.a != nullptr ? p.a[ti] : 1.f, rt = p.r[ti];
    const float qt = p.qn != nullptr ? p.qn[ti] : p.qn_scalar;
    float kv[NPL], pm[NPL], sum = 0.f;
#pragma unroll
    for (int u = 0; u < NPL; ++u) {
      const int i = lane + 32 * u;
      kv[u] = i < D ? load_elem(p.k, ti * D + i, p.in_dtype) : 0.f;
      pm[u] = fmaf(at * at, pv[u], qt);
      sum = fmaf(pm[u] * kv[u], kv[u], sum);
    }
    const float st = warp_sum(sum) + rt;
#pragma unroll
    for (int u = 0; u < NPL; ++u) {
      const int i = lane + 32 * u;
      if (i < D) {
        p.gains[ti * D + i] = pm[u] * kv[u] / st;
        p.pprev[ti * D + i] = pv[u];
      }
      pv[u] = pm[u] * rt / fmaf(pm[u] * kv[u], kv[u], rt);
    }
  }
}

template <int NPL>
__global__ void __launch_bounds__(32) diag_backward_kernel(DiagBwdArgs p) {
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const size_t tok0 = (size_t)bh * L;
  float pb[NPL];
#pragma unroll
  for (int u = 0; u < NPL; ++u) {
    const int i = lane + 32 * u;
    pb[u] = i < D && p.dp_L != nullptr ? p.dp_L[(size_t)bh * D + i] : 0.f;
  }
  for (int t = L - 1; t >= 0; --t) {
    const size_t ti = tok0 + t;
    const float at = p.a != nullptr ? p.a[ti] : 1.f, rt = p.r[ti];
    const float qt = p.qn != nullptr ? p.qn[ti] : p.qn_scalar;
    float kv[NPL], pm[NPL], pp[NPL], dg[NPL], sum = 0.f;
#pragma unroll
    for (int u = 0; u < NPL; ++u) {
      const int i = lane + 32 * u;
      const bool ok = i < D;
      kv[u] = ok ? load_elem(p.k, ti * D + i, p.in_dtype) : 0.f;
      pp[u] = ok ? p.pprev[ti * D + i] : 0.f;
      dg[u] = ok ? p.dgain[ti * D + i] : 0.f;
      pm[u] = ok ? fmaf(at * at, pp[u], qt) : 0.f;
      sum = fmaf(pm[u] * kv[u], kv[u], sum);
    }
    const float st = warp_sum(sum) + rt, is = 1.f / st;
    float dgg = 0.f;  // dG . g
#pragma unroll
    for (int u = 0; u < NPL; ++u) dgg = fmaf(dg[u], pm[u] * kv[u] * is, dgg);
    const float ds = -warp_sum(dgg) * is;
    float drp = 0.f, dap = 0.f, dqp = 0.f;
#pragma unroll
    for (int u = 0; u < NPL; ++u) {
      const int i = lane + 32 * u;
      const float den = fmaf(pm[u] * kv[u], kv[u], rt), id2 = 1.f / (den * den);
      float dpm = dg[u] * kv[u] * is + pb[u] * rt * rt * id2 + ds * kv[u] * kv[u];
      const float dkv = dg[u] * pm[u] * is - 2.f * pb[u] * pm[u] * pm[u] * rt * kv[u] * id2 + 2.f * ds * pm[u] * kv[u];
      drp = fmaf(pb[u] * (pm[u] * kv[u]) * (pm[u] * kv[u]), id2, drp);
      if (i >= D) dpm = 0.f;
      dap = fmaf(dpm, pp[u], dap);
      dqp += dpm;
      if (i < D) p.dk[ti * D + i] += dkv;
      pb[u] = at * at * dpm;
    }
    const float dr = warp_sum(drp) + ds, dav = warp_sum(dap), dqv = warp_sum(dqp);
    if (lane == 0) {
      p.dr[ti] = dr;
      p.dqn[ti] = dqv;
      if (p.da != nullptr) p.da[ti] += 2.f * at * dav;
    }
  }
#pragma unroll
  for (int u = 0; u < NPL; ++u) {
    const int i = lane + 32 * u;
    if (i < D) p.dp0[(size_t)bh * D + i] = pb[u];
  }
}

}  // namespace

cudaError_t launch_iso_forward(const IsoBwdArgs& args, int BH, cudaStream_t stream) {
  if (BH <= 0 || args.L <= 0) return cudaSuccess;
  iso_forward_kernel<<<BH, 32, 0, stream>>>(args);
  return cudaGetLastError();
}

cudaError_t launch_iso_backward(const IsoBwdArgs& args, int BH, cudaStream_t stream) {
  if (BH <= 0) return cudaSuccess;
  iso_backward_kernel<<<BH, 32, 0, stream>>>(args);
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
