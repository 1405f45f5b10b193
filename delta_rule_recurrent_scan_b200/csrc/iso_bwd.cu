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

// The chains are serial in t and one warp per head has nothing else to hide load latency with: each kernel
// takes its inputs in batches of tokens through a ring of kStages batches in shared memory, copied
// asynchronously kStages - 1 batches ahead of the walk, and steps through a batch in registers.
constexpr int kTB = 8;
constexpr int kStages = 4;

__device__ __forceinline__ float smem_elem(const uint8_t* base, int idx, int dtype) {
  return dtype == kBF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx])
                        : reinterpret_cast<const float*>(base)[idx];
}

// N sums across the warp at once: the shuffle stages of the N values interleave.
template <int N>
__device__ __forceinline__ void warp_sum_n(float (&x)[N]) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int i = 0; i < N; ++i) x[i] += __shfl_xor_sync(0xffffffffu, x[i], o);
}

template <int NPL>
__global__ void __launch_bounds__(32) iso_forward_kernel(IsoBwdArgs p) {
  constexpr int KB = kTB * 128 * 4;
  __shared__ __align__(16) uint8_t ks[kStages][KB];
  __shared__ float sa[kStages][kTB], sr[kStages][kTB], sq[kStages][kTB];
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const int es = p.in_dtype == kBF16 ? 2 : 4;
  const size_t tok0 = (size_t)bh * L;
  const int nbt = (L + kTB - 1) / kTB;
  auto issue = [&](int bt) {
    if (bt < nbt) {
      const int t0 = bt * kTB, nb = min(kTB, L - t0), st = bt % kStages;
      async_copy_rows(ks[st], static_cast<const uint8_t*>(p.k) + (tok0 + t0) * D * es, nb * D * es, lane, 32);
      if (lane < nb) {
        const size_t ti = tok0 + t0 + lane;
        if (p.a != nullptr) async_copy4(&sa[st][lane], p.a + ti); else sa[st][lane] = 1.f;
        async_copy4(&sr[st][lane], p.r + ti);
        if (p.qn != nullptr) async_copy4(&sq[st][lane], p.qn + ti); else sq[st][lane] = p.qn_scalar;
      }
    }
    async_commit();
  };
  for (int bt = 0; bt < kStages - 1; ++bt) issue(bt);
  float c = p.c0 != nullptr ? p.c0[bh] : 1.f;
  for (int bt = 0; bt < nbt; ++bt) {
    issue(bt + kStages - 1);
    async_wait<kStages - 1>();
    __syncwarp();
    const int st = bt % kStages, t0 = bt * kTB, nb = min(kTB, L - t0);
    float kk[kTB];
#pragma unroll
    for (int u = 0; u < kTB; ++u) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        const float x = u < nb && i < D ? smem_elem(ks[st], u * D + i, p.in_dtype) : 0.f;
        acc = fmaf(x, x, acc);
      }
      kk[u] = acc;
    }
    warp_sum_n(kk);
    float beta_mine = 0.f, c_mine = 0.f, kk_mine = 0.f;
#pragma unroll
    for (int u = 0; u < kTB; ++u) {
      if (u >= nb) break;
      const float at = sa[st][u], rt = sr[st][u], qt = sq[st][u];
      const float cm = fmaf(at * at, c, qt);
      if (lane == u) beta_mine = cm / fmaf(cm, kk[u], rt), c_mine = c, kk_mine = kk[u];
      c = (float)D * cm * rt / fmaf((float)D, rt, cm * kk[u]);
    }
    if (lane < nb) {
      const size_t ti = tok0 + t0 + lane;
      p.beta[ti] = beta_mine, p.cprev[ti] = c_mine, p.knorm2[ti] = kk_mine;
    }
    __syncwarp();
  }
  async_wait<0>();
}

template <int NPL>
__global__ void __launch_bounds__(32) iso_backward_kernel(IsoBwdArgs p) {
  constexpr int KB = kTB * 128 * 4;
  __shared__ __align__(16) uint8_t ks[kStages][KB];
  __shared__ __align__(16) float sdk[kStages][kTB * 128];
  __shared__ float sa[kStages][kTB], sr[kStages][kTB], sq[kStages][kTB], sc[kStages][kTB], skk[kStages][kTB],
      sdb[kStages][kTB], sda[kStages][kTB];
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const int es = p.in_dtype == kBF16 ? 2 : 4;
  const size_t tok0 = (size_t)bh * L;
  const float fd = (float)D;
  const int nbatch = (L + kTB - 1) / kTB;
  auto issue = [&](int k) {  // the k-th batch of the backward walk
    if (k < nbatch) {
      const int bi = nbatch - 1 - k, t0 = bi * kTB, nb = min(kTB, L - t0), st = k % kStages;
      const size_t row0 = (tok0 + t0) * D;
      async_copy_rows(ks[st], static_cast<const uint8_t*>(p.k) + row0 * es, nb * D * es, lane, 32);
      async_copy_rows(sdk[st], p.dk + row0, nb * D * 4, lane, 32);
      if (lane < nb) {
        const size_t ti = tok0 + t0 + lane;
        if (p.a != nullptr) async_copy4(&sa[st][lane], p.a + ti); else sa[st][lane] = 1.f;
        async_copy4(&sr[st][lane], p.r + ti);
        if (p.qn != nullptr) async_copy4(&sq[st][lane], p.qn + ti); else sq[st][lane] = p.qn_scalar;
        async_copy4(&sc[st][lane], p.cprev + ti);
        async_copy4(&skk[st][lane], p.knorm2 + ti);
        async_copy4(&sdb[st][lane], p.dbeta + ti);
        if (p.da != nullptr) async_copy4(&sda[st][lane], p.da + ti); else sda[st][lane] = 0.f;
      }
    }
    async_commit();
  };
  for (int k = 0; k < kStages - 1; ++k) issue(k);
  float cb = p.dc_L != nullptr ? p.dc_L[bh] : 0.f;
  for (int k = 0; k < nbatch; ++k) {
    issue(k + kStages - 1);
    async_wait<kStages - 1>();
    __syncwarp();
    const int st = k % kStages, bi = nbatch - 1 - k, t0 = bi * kTB, nb = min(kTB, L - t0);
    float dr_mine = 0.f, dqn_mine = 0.f, da_mine = lane < nb ? sda[st][lane] : 0.f, dkk_b[kTB];
#pragma unroll
    for (int u = kTB - 1; u >= 0; --u) {
      dkk_b[u] = 0.f;
      if (u < nb) {
        const float at = sa[st][u], rt = sr[st][u], qt = sq[st][u], c = sc[st][u], kk = skk[st][u], db = sdb[st][u];
        const float cm = fmaf(at * at, c, qt);
        const float stv = fmaf(cm, kk, rt), den = fmaf(fd, rt, cm * kk);
        const float is2 = 1.f / (stv * stv), id2 = 1.f / (den * den);
        const float dcm = db / stv - db * cm * kk * is2 + cb * (fd * rt) * (fd * rt) * id2;
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
        if (u < nb && i < D)
          p.dk[(tok0 + t0 + u) * D + i] =
              fmaf(2.f * dkk_b[u], smem_elem(ks[st], u * D + i, p.in_dtype), sdk[st][u * D + i]);
      }
    if (lane < nb) {
      const size_t ti = tok0 + t0 + lane;
      p.dr[ti] = dr_mine, p.dqn[ti] = dqn_mine;
      if (p.da != nullptr) p.da[ti] = da_mine;
    }
    __syncwarp();
  }
  async_wait<0>();
  if (lane == 0) p.dc0[bh] = cb;
}

// Only p is serial in t (p_{t+1} = p^-_t r_t / (r_t + p^-_t k_t^2) per coordinate); the coupled sum s_t of each
// token depends on p^-_t but nothing serial depends on s_t.  So each batch steps the per-coordinate chain over
// its kTB tokens first, then reduces the kTB sums at once, then writes the gains.  The inputs arrive through
// the ring of kStages batches.

template <int NPL>
__global__ void __launch_bounds__(32) diag_forward_kernel(DiagBwdArgs p) {
  constexpr int KB = kTB * 128 * 4;  // key bytes of a stage (at most fp32 keys of d_k = 128)
  __shared__ __align__(16) uint8_t ks[kStages][KB];
  __shared__ float sa[kStages][kTB], sr[kStages][kTB], sq[kStages][kTB];
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const int es = p.in_dtype == kBF16 ? 2 : 4;
  const size_t tok0 = (size_t)bh * L;
  const int nbt = (L + kTB - 1) / kTB;
  auto issue = [&](int bt) {
    if (bt < nbt) {
      const int t0 = bt * kTB, nb = min(kTB, L - t0), st = bt % kStages;
      async_copy_rows(ks[st], static_cast<const uint8_t*>(p.k) + (tok0 + t0) * D * es, nb * D * es, lane, 32);
      if (lane < nb) {
        const size_t ti = tok0 + t0 + lane;
        if (p.a != nullptr) async_copy4(&sa[st][lane], p.a + ti); else sa[st][lane] = 1.f;
        async_copy4(&sr[st][lane], p.r + ti);
        if (p.qn != nullptr) async_copy4(&sq[st][lane], p.qn + ti); else sq[st][lane] = p.qn_scalar;
      }
    }
    async_commit();  // (an empty group past the end keeps the wait count uniform)
  };
  for (int bt = 0; bt < kStages - 1; ++bt) issue(bt);
  float pv[NPL];
#pragma unroll
  for (int e = 0; e < NPL; ++e) {
    const int i = lane + 32 * e;
    pv[e] = i < D ? (p.p0 != nullptr ? p.p0[(size_t)bh * D + i] : 1.f) : 0.f;
  }
  for (int bt = 0; bt < nbt; ++bt) {
    issue(bt + kStages - 1);
    async_wait<kStages - 1>();  // this batch has landed
    __syncwarp();
    const int st = bt % kStages, t0 = bt * kTB, nb = min(kTB, L - t0);
    float pm[kTB][NPL], kv[kTB][NPL], sum[kTB];
#pragma unroll
    for (int u = 0; u < kTB; ++u) {  // the serial chain (tokens past the end: a = 1, Qn = 0, k = 0 keep p)
      const bool ok = u < nb;
      const float at = ok ? sa[st][u] : 1.f, rt = ok ? sr[st][u] : 1.f, qt = ok ? sq[st][u] : 0.f;
      sum[u] = 0.f;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        kv[u][e] = ok && i < D ? smem_elem(ks[st], u * D + i, p.in_dtype) : 0.f;
        if (ok && i < D) p.pprev[(tok0 + t0 + u) * D + i] = pv[e];
        pm[u][e] = fmaf(at * at, pv[e], qt);
        const float pk = pm[u][e] * kv[u][e];
        sum[u] = fmaf(pk, kv[u][e], sum[u]);
        pv[e] = __fdividef(pm[u][e] * rt, fmaf(pk, kv[u][e], rt));
      }
    }
    warp_sum_n(sum);
#pragma unroll
    for (int u = 0; u < kTB; ++u) {
      if (u >= nb) break;
      const float is = __fdividef(1.f, sum[u] + sr[st][u]);
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        if (i < D) p.gains[(tok0 + t0 + u) * D + i] = pm[u][e] * kv[u][e] * is;
      }
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  async_wait<0>();
}

// The adjoint pb of p is the only serial quantity backwards: pb_{t-1} = a_t^2 (c1 + pb_t c2) per coordinate,
// with c1 = dG k / s + ds k^2 and c2 = r^2 / den^2 fixed by the token's own inputs.  Each batch first forms
// p^- and reduces its TB sums s and dG . g at once (ds = -(dG . g) / s), then steps pb through the batch,
// collecting the per-token parts of dr, da and dQn, and reduces those at once.  The inputs arrive through a
// ring of kStages batches in shared memory, copied kStages - 1 batches ahead of the (backward) walk.
template <int NPL>
__global__ void __launch_bounds__(32) diag_backward_kernel(DiagBwdArgs p) {
  constexpr int TB = 4;                    // tokens per batch
  constexpr int RB = TB * 128 * 4;         // bytes of one array's rows in a stage
  __shared__ __align__(16) uint8_t ks[kStages][RB];
  __shared__ __align__(16) float spp[kStages][TB * 128], sdg[kStages][TB * 128], sdk[kStages][TB * 128];
  __shared__ float sa[kStages][TB], sr[kStages][TB], sq[kStages][TB], sda[kStages][TB];
  const int bh = blockIdx.x, lane = threadIdx.x, L = p.L, D = p.dk_dim;
  const int es = p.in_dtype == kBF16 ? 2 : 4;
  const size_t tok0 = (size_t)bh * L;
  const int nbatch = (L + TB - 1) / TB;
  // batches in walk order: k-th is batch nbatch - 1 - k
  auto issue = [&](int k) {
    if (k < nbatch) {
      const int bi = nbatch - 1 - k, t0 = bi * TB, nb = min(TB, L - t0), st = k % kStages;
      const size_t row0 = (tok0 + t0) * D;
      async_copy_rows(ks[st], static_cast<const uint8_t*>(p.k) + row0 * es, nb * D * es, lane, 32);
      async_copy_rows(spp[st], p.pprev + row0, nb * D * 4, lane, 32);
      async_copy_rows(sdg[st], p.dgain + row0, nb * D * 4, lane, 32);
      async_copy_rows(sdk[st], p.dk + row0, nb * D * 4, lane, 32);
      if (lane < nb) {
        const size_t ti = tok0 + t0 + lane;
        if (p.a != nullptr) async_copy4(&sa[st][lane], p.a + ti); else sa[st][lane] = 1.f;
        async_copy4(&sr[st][lane], p.r + ti);
        if (p.qn != nullptr) async_copy4(&sq[st][lane], p.qn + ti); else sq[st][lane] = p.qn_scalar;
        if (p.da != nullptr) async_copy4(&sda[st][lane], p.da + ti); else sda[st][lane] = 0.f;
      }
    }
    async_commit();
  };
  for (int k = 0; k < kStages - 1; ++k) issue(k);
  float pb[NPL];
#pragma unroll
  for (int e = 0; e < NPL; ++e) {
    const int i = lane + 32 * e;
    pb[e] = i < D && p.dp_L != nullptr ? p.dp_L[(size_t)bh * D + i] : 0.f;
  }
  for (int k = 0; k < nbatch; ++k) {
    issue(k + kStages - 1);
    async_wait<kStages - 1>();
    __syncwarp();
    const int st = k % kStages, bi = nbatch - 1 - k, t0 = bi * TB, nb = min(TB, L - t0);
    float kv[TB][NPL], pp[TB][NPL], dg[TB][NPL], dko[TB][NPL];
#pragma unroll
    for (int u = 0; u < TB; ++u)
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        const bool ok = u < nb && i < D;
        kv[u][e] = ok ? smem_elem(ks[st], u * D + i, p.in_dtype) : 0.f;
        pp[u][e] = ok ? spp[st][u * D + i] : 0.f;
        dg[u][e] = ok ? sdg[st][u * D + i] : 0.f;
        dko[u][e] = ok ? sdk[st][u * D + i] : 0.f;
      }
    // ---- p^-, s and ds of every token of the batch (nothing serial in them)
    float at[TB], rt[TB], pm[TB][NPL], red[2 * TB];
#pragma unroll
    for (int u = 0; u < TB; ++u) {
      const bool ok = u < nb;
      at[u] = ok ? sa[st][u] : 1.f, rt[u] = ok ? sr[st][u] : 1.f;
      const float qt = ok ? sq[st][u] : 0.f;
      red[u] = 0.f;
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        pm[u][e] = i < D ? fmaf(at[u] * at[u], pp[u][e], qt) : 0.f;
        red[u] = fmaf(pm[u][e] * kv[u][e], kv[u][e], red[u]);
      }
    }
    {
      float s4[TB];
#pragma unroll
      for (int u = 0; u < TB; ++u) s4[u] = red[u];
      warp_sum_n(s4);
#pragma unroll
      for (int u = 0; u < TB; ++u) red[u] = __fdividef(1.f, s4[u] + rt[u]);  // 1 / s
    }
    {
      float g4[TB];
#pragma unroll
      for (int u = 0; u < TB; ++u) {
        g4[u] = 0.f;
#pragma unroll
        for (int e = 0; e < NPL; ++e) g4[u] = fmaf(dg[u][e], pm[u][e] * kv[u][e] * red[u], g4[u]);
      }
      warp_sum_n(g4);
#pragma unroll
      for (int u = 0; u < TB; ++u) red[TB + u] = -g4[u] * red[u];  // ds
    }
    // ---- the serial adjoint through the batch, newest token first
    float drp[TB], dap[TB], dqp[TB];
#pragma unroll
    for (int u = TB - 1; u >= 0; --u) {
      drp[u] = dap[u] = dqp[u] = 0.f;
      if (u >= nb) continue;  // uniform over the warp
      const float is = red[u], ds = red[TB + u], r = rt[u];
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        const float k1 = kv[u][e], m1 = pm[u][e];
        const float den = fmaf(m1 * k1, k1, r), id2 = __fdividef(1.f, den * den);
        float dpm = fmaf(pb[e], r * r * id2, fmaf(dg[u][e] * k1, is, ds * k1 * k1));
        dko[u][e] += dg[u][e] * m1 * is - 2.f * pb[e] * m1 * m1 * r * k1 * id2 + 2.f * ds * m1 * k1;
        drp[u] = fmaf(pb[e] * (m1 * k1) * (m1 * k1), id2, drp[u]);
        if (i >= D) dpm = 0.f;
        dap[u] = fmaf(dpm, pp[u][e], dap[u]);
        dqp[u] += dpm;
        pb[e] = at[u] * at[u] * dpm;
      }
    }
    warp_sum_n(drp);
    warp_sum_n(dap);
    warp_sum_n(dqp);
#pragma unroll
    for (int u = 0; u < TB; ++u)
#pragma unroll
      for (int e = 0; e < NPL; ++e) {
        const int i = lane + 32 * e;
        if (u < nb && i < D) p.dk[(tok0 + t0 + u) * D + i] = dko[u][e];
      }
    float dr_mine = 0.f, dqn_mine = 0.f, da_mine = lane < nb ? sda[st][lane] : 0.f;
#pragma unroll
    for (int u = 0; u < TB; ++u)
      if (lane == u) dr_mine = drp[u] + red[TB + u], dqn_mine = dqp[u], da_mine += 2.f * at[u] * dap[u];
    if (lane < nb) {
      const size_t ti = tok0 + t0 + lane;
      p.dr[ti] = dr_mine, p.dqn[ti] = dqn_mine;
      if (p.da != nullptr) p.da[ti] = da_mine;
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  async_wait<0>();
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
