// Backward of the isotropic Kalman scan's uncertainty side (the training-time adjoint).
//
// Kalman Delta Networks, Abstract: Isotropic KDN keeps one uncertainty scalar per head.  Per token
// (the reading the forward kernels take): c^- = a^2 c + Qn, s = c^- ||k||^2 + r, beta = c^- / s, the
// memory write of the gated delta rule with that beta, and the mean-field update
// c = d_k c^- r / (d_k r + c^- ||k||^2).  Given dbeta_t from the memory backward (the delta rule's
// adjoint with beta as an input), the scalar chain is walked backwards with the adjoint cb of c:
//   dc^- = dbeta / s - dbeta c^- ||k||^2 / s^2 + cb (d_k r)^2 / den^2,   den = d_k r + c^- ||k||^2,
//   dr  = -dbeta c^- / s^2 + cb d_k c^-^2 ||k||^2 / den^2,
//   d||k||^2 = -dbeta c^-^2 / s^2 - cb d_k c^-^2 r / den^2   (dk_t += 2 d||k||^2 k_t),
//   da += 2 a c dc^-,  dQn = dc^-,  cb <- a^2 dc^-   (dc0 = cb after token 0).
// Two kernels, one warp per head (the chain is serial in t; the warp shares each token's key):
//   iso_forward_kernel   the forward chain, storing beta_t, c before the token and ||k_t||^2;
//   iso_backward_kernel  the reverse chain above, adding the key and gate terms into dk and da.
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
