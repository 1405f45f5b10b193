// Surprise-cache read on the sm_100a tensor cores: bf16 q, k, v with d_k = d_v = 128, blocks of 64.
//
// The read of A Hippocampus for Linear Attention, section 3.4, Eq. (7): token t of block b takes a
// softmax, temperature 1, over the top-w cache of blocks 0..b-1 (by surprise m, section 3.3), the causal
// tokens of its own block and a null sink.  With q~ = q / rms(q) * gamma_q and k~ = k / rms(k) * gamma_k,
//
//   q~_t . k~_j = rq_t rk_j sum_d (q_td gamma_q,d gamma_k,d) k_jd,
//
// so the keys enter the product raw (exact bf16) and only the queries, scaled by gamma_q gamma_k, are
// split into bf16 hi + lo.  Per block, with the 128 keys (64 cache rows, then 64 block rows) on the TMEM
// lanes:
//
//   S^T = K [q o gamma]^T        M = 128 keys, N = 64 queries, K = 128      (2 MMAs per K step)
//   softmax over the keys of each query column (warp butterflies, then the four lane quarters), sink
//   O^T = V^T P                  M = 128 (d_v), N = 64 queries, K = 128 keys (P as bf16 hi + lo)
//
// The cache lives in two ping-pong buffers of 128 key / value rows: block b reads buffer b & 1 (cache in
// rows 0..63, its own tokens in rows 64..127) and merges the best w candidates into rows 0..63 of the
// other buffer (rank = number of candidates with a larger m, ties towards the earlier token).
#include <cuda.h>
#include <cuda_bf16.h>

#include <climits>

#include "chunk.h"
#include "chunk_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace kdn {

namespace {

using chunk::kWaitCycles;
using chunk::store8_split;

constexpr int kTThreads = 256;
constexpr int kD = 128;
constexpr int kNP = kD / 64;                // 64-wide panels across d
constexpr int kRows = 128;                  // key / value rows of a buffer: 64 cache + 64 block
constexpr int kPanel = kRows * 128;         // 16 KB: 128 rows x 64 bf16, 128-byte swizzle
constexpr int kBuf = kNP * kPanel;          // 32 KB
constexpr int kQPanel = 64 * 128;           // 8 KB: 64 query rows x 64 bf16
constexpr int OFF_K = 0;                    // 2 x kBuf raw keys
constexpr int OFF_V = OFF_K + 2 * kBuf;     // 2 x kBuf values
constexpr int OFF_H = OFF_V + 2 * kBuf;     // scaled queries hi (kNP x kQPanel), then P hi (one kPanel)
constexpr int OFF_L = OFF_H + kPanel;       // scaled queries lo, then P lo
constexpr int OFF_QS = OFF_L + kPanel;      // raw queries of the next block (TMA staging), kNP x kQPanel
constexpr int kTotal = OFF_QS + kNP * kQPanel;
constexpr int kSmem = kTotal + 1024;
constexpr uint32_t T_S = 0, T_O = 64, kTmemCols = 128;
static_assert(kNP * kQPanel == kPanel, "query panels and the P panel share a region");

// Max (kind 0) or sum (kind 1) over the warp's 32 lanes for each of 32 values: afterwards lane l holds
// the result for value index l.
template <int KIND>
__device__ __forceinline__ float butterfly(float (&x)[32], int lane) {
#pragma unroll
  for (int k = 16; k >= 1; k >>= 1) {
    const bool up = (lane & k) != 0;
#pragma unroll
    for (int i = 0; i < k; ++i) {
      const float send = up ? x[i] : x[i + k];
      const float keep = up ? x[i + k] : x[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, k);
      x[i] = KIND == 0 ? fmaxf(keep, got) : keep + got;
    }
  }
  return x[0];
}

__device__ __forceinline__ bool before(float mc, int ic, float md, int id) { return mc > md || (mc == md && ic < id); }

__global__ void __launch_bounds__(kTThreads, 1)
    hola_read_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, HolaArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ float rk[2][kRows];     // 1 / rms(k) per buffer row
  __shared__ float mcs[2][kRows];    // m per buffer row (-inf = empty)
  __shared__ int ics[2][kRows];      // token index per buffer row (-1 = empty)
  __shared__ float rq[64];
  __shared__ float gqk[kD];          // gamma_q * gamma_k
  __shared__ float red[4][64];
  __shared__ float mxs[64], inv_den[64];
  __shared__ int newpos[kRows];
  __shared__ int rank_part[2][kRows];
  __shared__ int ncache;
  __shared__ uint64_t bar_mma, bar_load;
  __shared__ uint32_t tmem_base;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qw = warp & 3, half = warp >> 2;
  const int bh = blockIdx.x, h = bh % p.H;
  const int L = p.L, w = p.w;
  const size_t tok0 = (size_t)bh * L;
  const float sink = p.sink[h];
  const float inv_sqrt_d = rsqrtf((float)kD);
  const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;

  for (int e = tid; e < 2 * kRows; e += kTThreads) {
    mcs[e / kRows][e % kRows] = -INFINITY, ics[e / kRows][e % kRows] = -1, rk[e / kRows][e % kRows] = 0.f;
  }
  if (tid < kD) gqk[tid] = p.gamma_q[tid] * p.gamma_k[tid];
  // both buffers start as zeros: empty cache rows meet probability 0 and must stay finite
  for (int e = tid; e < (4 * kBuf) / 16; e += kTThreads) reinterpret_cast<uint4*>(sm + OFF_K)[e] = make_uint4(0, 0, 0, 0);
  // TMA of one block's raw k, v (rows 64..127 of a buffer) and q (staging): six 64 x 64 boxes
  auto issue_block = [&](int bb, int buf) {
    sm100::mbar_arrive_expect_tx(&bar_load, 3 * kNP * 64 * 128);
#pragma unroll
    for (int pn = 0; pn < kNP; ++pn) {
      sm100::tma_load_3d(sm + OFF_K + buf * kBuf + pn * kPanel + 64 * 128, &tm_k, &bar_load, 64 * pn, bb, bh);
      sm100::tma_load_3d(sm + OFF_V + buf * kBuf + pn * kPanel + 64 * 128, &tm_v, &bar_load, 64 * pn, bb, bh);
      sm100::tma_load_3d(sm + OFF_QS + pn * kQPanel, &tm_q, &bar_load, 64 * pn, bb, bh);
    }
  };
  if (tid == 0) {
    ncache = 0;
    sm100::prefetch_tmap(&tm_q);
    sm100::prefetch_tmap(&tm_k);
    sm100::prefetch_tmap(&tm_v);
    sm100::mbar_init(&bar_mma, 1);
    sm100::mbar_init(&bar_load, 1);
    sm100::fence_mbar_init();
  }
  if (warp == 0) {
    sm100::tmem_alloc(&tmem_base, kTmemCols);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = tmem_base;
  uint32_t phase = 0, lphase = 0;
  bool aborted = false;
  if (tid == 0 && L > 0) {
    sm100::fence_async_smem();  // the zeroed buffers precede the first copy in
    issue_block(0, 0);
  }
  const uint32_t qh = sm100::smem_u32(sm + OFF_H), ql = sm100::smem_u32(sm + OFF_L);

  int nblocks = 0;
  for (int b0 = 0; b0 < L; b0 += 64, ++nblocks) {
    const int X = nblocks & 1, Y = X ^ 1;
    const int nb = min(64, L - b0);
    uint8_t* KB = sm + OFF_K + X * kBuf;
    uint8_t* VB = sm + OFF_V + X * kBuf;

    // ---------------------------------------------------------------- block tokens: scales of k, scaled q hi/lo
    {
      int bad = 0;
      if (tid == 0) bad = !sm100::mbar_wait_bounded(&bar_load, lphase, kWaitCycles);
      bad = __syncthreads_or(bad);
      if (bad) {
        if (tid == 0) raise_status(p.status, kStatusTimeout);
        aborted = true;
        break;
      }
      lphase ^= 1;
    }
    {
      const int i = tid >> 2, part = tid & 3;   // token, quarter of its 16 chunks
      const bool valid = i < nb;
      float kss = 0.f, qss = 0.f;
      const float mt = valid ? p.m[tok0 + b0 + i] : -INFINITY;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = 4 * part + u;             // chunk: elements 8 c .. 8 c + 7
        const uint4 kc = *reinterpret_cast<const uint4*>(KB + (c / 8) * kPanel + sm100::sw128_chunk(64 + i, c % 8));
        const uint4 qc = *reinterpret_cast<const uint4*>(sm + OFF_QS + (c / 8) * kQPanel + sm100::sw128_chunk(i, c % 8));
        const __nv_bfloat162* kh = reinterpret_cast<const __nv_bfloat162*>(&kc);
        const __nv_bfloat162* qh2 = reinterpret_cast<const __nv_bfloat162*>(&qc);
        float qs[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 kf = __bfloat1622float2(kh[e]), qf = __bfloat1622float2(qh2[e]);
          kss = fmaf(kf.x, kf.x, fmaf(kf.y, kf.y, kss));
          qss = fmaf(qf.x, qf.x, fmaf(qf.y, qf.y, qss));
          qs[2 * e] = qf.x * gqk[8 * c + 2 * e];
          qs[2 * e + 1] = qf.y * gqk[8 * c + 2 * e + 1];
        }
        store8_split(sm + OFF_H, sm + OFF_L, (c / 8) * kQPanel + sm100::sw128_chunk(i, c % 8), qs);
      }
      kss += __shfl_xor_sync(0xffffffffu, kss, 1);
      kss += __shfl_xor_sync(0xffffffffu, kss, 2);
      qss += __shfl_xor_sync(0xffffffffu, qss, 1);
      qss += __shfl_xor_sync(0xffffffffu, qss, 2);
      if (part == 0) {
        rk[X][64 + i] = valid ? rsqrtf(kss / kD + 1e-6f) : 0.f;
        rq[i] = rsqrtf(qss / kD + 1e-6f);
        mcs[X][64 + i] = mt;
        ics[X][64 + i] = valid ? b0 + i : -1;
      }
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();

    // ---------------------------------------------------------------- S^T = K [q o gamma]^T
    if (tid == 0 && b0 + 64 < L) issue_block(b0 + 64, Y);  // rows 64.. of the other buffer and the staging are free
    if (tid == 0) {
      constexpr uint32_t id = sm100::idesc_bf16(128, 64, false, false);
      const uint32_t kb = sm100::smem_u32(KB);
#pragma unroll
      for (int ks = 0; ks < kD / 16; ++ks) {
        const uint64_t a = sm100::smem_desc(kb + (ks / 4) * kPanel + (ks % 4) * 32, 16, 1024);
        const uint32_t boff = (ks / 4) * kQPanel + (ks % 4) * 32;
        sm100::mma_bf16(tmem + T_S, a, sm100::smem_desc(qh + boff, 16, 1024), id, ks > 0);
        sm100::mma_bf16(tmem + T_S, a, sm100::smem_desc(ql + boff, 16, 1024), id, true);
      }
      sm100::mma_commit(&bar_mma);
    }
    {
      int bad = 0;
      if (tid == 0) bad = !sm100::mbar_wait_bounded(&bar_mma, phase, kWaitCycles);
      bad = __syncthreads_or(bad);
      if (bad) {
        if (tid == 0) raise_status(p.status, kStatusTimeout);
        aborted = true;
        break;
      }
      sm100::tc_fence_after();
      phase ^= 1;
    }

    // ---------------------------------------------------------------- softmax over the keys (lanes) of each query
    const int j = 32 * qw + lane;             // key row
    float x[32];
    {
      float s[32];
      sm100::tmem_ld32(tmem + t_lane + T_S + 32 * half, s);
      sm100::tmem_wait_ld();
      const float kscale = rk[X][j] * inv_sqrt_d;
      const int nc = ncache;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int t = 32 * half + u;
        const bool vis = j < 64 ? j < nc : (j - 64 <= t && j - 64 < nb);
        x[u] = vis ? s[u] * kscale * rq[t] : -INFINITY;
        s[u] = x[u];
      }
      red[qw][32 * half + lane] = butterfly<0>(s, lane);
    }
    __syncthreads();
    if (tid < 64) mxs[tid] = fmaxf(fmaxf(fmaxf(red[0][tid], red[1][tid]), fmaxf(red[2][tid], red[3][tid])), sink);
    __syncthreads();
    {
      float s[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        x[u] = __expf(x[u] - mxs[32 * half + u]);  // exp(-inf) = 0 for hidden keys
        s[u] = x[u];
      }
      red[qw][32 * half + lane] = butterfly<1>(s, lane);
    }
    __syncthreads();
    if (tid < 64) inv_den[tid] = 1.f / (red[0][tid] + red[1][tid] + red[2][tid] + red[3][tid] + __expf(sink - mxs[tid]));
    __syncthreads();
    // P (key rows, query columns) as bf16 hi / lo over the query panels, which the S product no longer reads
#pragma unroll
    for (int q8 = 0; q8 < 4; ++q8) {
      float pv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pv[e] = x[8 * q8 + e] * inv_den[32 * half + 8 * q8 + e];
      store8_split(sm + OFF_H, sm + OFF_L, sm100::sw128_chunk(j, 4 * half + q8), pv);
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();

    // ---------------------------------------------------------------- O^T = V^T P
    if (tid == 0) {
      constexpr uint32_t id = sm100::idesc_bf16(128, 64, true, true);
      const uint32_t vb = sm100::smem_u32(VB);
#pragma unroll
      for (int ks = 0; ks < kRows / 16; ++ks) {
        const uint64_t a = sm100::smem_desc(vb + ks * 2048, kPanel, 1024);
        sm100::mma_bf16(tmem + T_O, a, sm100::smem_desc(qh + ks * 2048, kPanel, 1024), id, ks > 0);
        sm100::mma_bf16(tmem + T_O, a, sm100::smem_desc(ql + ks * 2048, kPanel, 1024), id, true);
      }
      sm100::mma_commit(&bar_mma);
    }
    // meanwhile: rank every candidate for the merged cache (two threads per candidate, half the others each)
    {
      const int cand = tid & (kRows - 1), hf = tid >> 7;
      const float m0 = mcs[X][cand];
      const int i0 = ics[X][cand];
      int rank = 0;
      for (int c = 64 * hf; c < 64 * hf + 64; ++c)
        rank += (ics[X][c] >= 0 && c != cand && before(mcs[X][c], ics[X][c], m0, i0)) ? 1 : 0;
      rank_part[hf][cand] = rank;
    }
    {
      int bad = 0;
      if (tid == 0) bad = !sm100::mbar_wait_bounded(&bar_mma, phase, kWaitCycles);
      bad = __syncthreads_or(bad);
      if (bad) {
        if (tid == 0) raise_status(p.status, kStatusTimeout);
        aborted = true;
        break;
      }
      sm100::tc_fence_after();
      phase ^= 1;
    }
    int kept = 0;
    if (tid < kRows) {
      const int rank = rank_part[0][tid] + rank_part[1][tid];
      kept = (ics[X][tid] >= 0 && rank < w) ? 1 : 0;
      newpos[tid] = kept ? rank : -1;
    }
    {
      float o[32];
      sm100::tmem_ld32(tmem + t_lane + T_O + 32 * half, o);
      sm100::tmem_wait_ld();
      const int dv = j;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int t = 32 * half + u;
        if (t < nb) p.o[(tok0 + b0 + t) * kD + dv] = o[u];
      }
    }

    // ---------------------------------------------------------------- merge into rows 0..63 of the other buffer
    const int n_kept = __syncthreads_count(kept);  // also: newpos complete; the kept rows are 0 .. n_kept - 1
    {
      uint8_t* KY = sm + OFF_K + Y * kBuf;
      uint8_t* VY = sm + OFF_V + Y * kBuf;
      for (int e = tid; e < kRows * 2 * 2 * kNP * 8 / 2; e += kTThreads) {   // rows x (key, value) x 16 chunks
        const int c = e >> 5, q = e & 31;
        const int np = newpos[c];
        if (np < 0) continue;
        const int which = q >> 4, cc = q & 15;
        const uint8_t* src = (which ? VB : KB) + (cc / 8) * kPanel + sm100::sw128_chunk(c, cc % 8);
        uint8_t* dst = (which ? VY : KY) + (cc / 8) * kPanel + sm100::sw128_chunk(np, cc % 8);
        *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
      }
    }
    if (tid < kRows && newpos[tid] >= 0) {
      const int np = newpos[tid];
      mcs[Y][np] = mcs[X][tid], ics[Y][np] = ics[X][tid], rk[Y][np] = rk[X][tid];
    }
    if (tid < 64 && tid >= n_kept) mcs[Y][tid] = -INFINITY, ics[Y][tid] = -1;
    if (tid == 0) ncache = n_kept;
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
  }

  // ---------------------------------------------------------------- the final cache's token indices, ascending
  if (!aborted && p.cache != nullptr && tid < w) {
    const int F = nblocks & 1;
    const int mine = tid < 64 ? ics[F][tid] : -1;
    if (mine >= 0) {
      int pos = 0;
      for (int c = 0; c < 64; ++c) pos += (ics[F][c] >= 0 && ics[F][c] < mine) ? 1 : 0;
      p.cache[(size_t)bh * w + pos] = mine;
    }
    if (tid >= ncache) p.cache[(size_t)bh * w + tid] = -1;
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 0) sm100::tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------------------- parallel form
// The cache a block reads depends only on m (section 3.3: the top-w tokens by surprise), not on any read, so
// it can be fixed for every block first.  hola_cache_select_kernel walks one head's blocks with one CTA,
// keeping the cache as a list in rank order (larger m first, ties to the earlier token: a strict total
// order).  Per block: the block's 64 candidates are put in rank order among themselves (eight lanes per
// candidate count the others before it), then the two ordered lists are merged: an element's place in the
// union is its index in its own list plus the number of elements of the other list before it (a binary
// search), and the first w places form the next cache.  The cache read by block b goes to cidx[head][b] in
// rank order (-1 past its size); the final cache's indices are also written, ascending.
constexpr int kSelThreads = 512;

__global__ void __launch_bounds__(kSelThreads) hola_cache_select_kernel(HolaArgs p) {
  __shared__ float cm[2][64];  // the cache in rank order, two buffers
  __shared__ int ci[2][64];
  __shared__ float rm[64];     // the block's candidates as they come
  __shared__ int ri[64];
  __shared__ float bm[64];     // ... and in rank order
  __shared__ int bi[64];
  const int tid = threadIdx.x, bh = blockIdx.x, L = p.L, w = p.w;
  const int nblocks = (L + 63) / 64;
  const size_t tok0 = (size_t)bh * L;
  int ncache = 0, cur = 0;
  float mnext = tid < 64 && tid < L ? p.m[tok0 + tid] : -INFINITY;  // the next block's m, in flight
  for (int b = 0; b < nblocks; ++b) {
    const int nv = min(64, L - 64 * b);  // valid tokens of the block (the others sort last)
    if (tid < 64) {
      rm[tid] = tid < nv ? mnext : -INFINITY;
      ri[tid] = tid < nv ? 64 * b + tid : INT_MAX;
      const int tn = 64 * (b + 1) + tid;
      mnext = tn < L ? p.m[tok0 + tn] : -INFINITY;
    } else if (tid < 128) {  // the cache block b reads
      const int r = tid - 64;
      p.cidx[((size_t)bh * nblocks + b) * 64 + r] = r < ncache ? ci[cur][r] : -1;
    }
    __syncthreads();
    {
      const int cand = tid >> 3, part = tid & 7;
      const float m0 = rm[cand];
      const int i0 = ri[cand];
      int rank = 0;
#pragma unroll
      for (int c = part; c < 64; c += 8) rank += before(rm[c], ri[c], m0, i0) ? 1 : 0;
      rank += __shfl_xor_sync(0xffffffffu, rank, 1);
      rank += __shfl_xor_sync(0xffffffffu, rank, 2);
      rank += __shfl_xor_sync(0xffffffffu, rank, 4);
      if (part == 0) bm[rank] = m0, bi[rank] = i0;
    }
    __syncthreads();
    if (tid < 128) {  // warps 0..1: the cache's elements, warps 2..3: the block's
      const bool from_cache = tid < 64;
      const int k = tid & 63;
      if (k < (from_cache ? ncache : nv)) {
        const float mx = from_cache ? cm[cur][k] : bm[k];
        const int ix = from_cache ? ci[cur][k] : bi[k];
        const float* om = from_cache ? bm : cm[cur];
        const int* oi = from_cache ? bi : ci[cur];
        int lo = 0, hi = from_cache ? nv : ncache;  // the other list's elements before this one: a prefix
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (before(om[mid], oi[mid], mx, ix)) lo = mid + 1;
          else hi = mid;
        }
        const int pos = k + lo;
        if (pos < w) cm[cur ^ 1][pos] = mx, ci[cur ^ 1][pos] = ix;
      }
    }
    ncache = min(w, ncache + nv);
    cur ^= 1;
    __syncthreads();
  }
  if (p.cache != nullptr && tid < w) {  // the final cache, ascending token indices, -1 past its size
    const int mine = tid < ncache ? ci[cur][tid] : -1;
    if (mine >= 0) {
      int pos = 0;
      for (int c = 0; c < ncache; ++c) pos += ci[cur][c] < mine ? 1 : 0;
      p.cache[(size_t)bh * w + pos] = mine;
    } else {
      p.cache[(size_t)bh * w + tid] = -1;
    }
  }
}

// hola_cache_scan_kernel: the same caches by a log-depth scan instead of the walk.  The cache block b reads is
// the top w of blocks 0 .. b - 1, and the top w of a union of disjoint sets is the top w of the union of their
// top w, so the lists combine associatively: an inclusive scan over the blocks (Hillis-Steele: at distance
// d = 1, 2, 4, .. each block's list is merged with that of the block d before it) gives at block b the top w of
// blocks 0 .. b, i.e. the cache of block b + 1.  An entry is one 64-bit key, larger first in rank order: m
// mapped to an order-preserving unsigned word above INT_MAX - token (the rank order of `before`: larger m
// first, ties to the earlier token; -0 is taken as +0), and the padding past a list's size is key 0 below every
// token.  Every list is 64 keys in rank order, held by one warp as two keys per lane (positions lane and
// lane + 32) and ordered by bitonic networks over the lanes: a block's own candidates by a full sort, a merge
// of lists A and B as the bitonic sequence C_i = max(A_i, B_63-i) (exactly the 64 first of A u B) followed by
// six half-cleaner stages.  Positions from w on are cleared to the padding.  One CTA of kScanThreads per head;
// the lists are double-buffered in shared memory (2 x blocks x 64 keys), hence at most kScanMaxBlocks blocks.
constexpr int kScanThreads = 1024;
constexpr int kScanMaxBlocks = 192;

__host__ __device__ constexpr size_t scan_smem_bytes(int nblocks) { return (size_t)nblocks * 2 * 64 * 8; }

__device__ __forceinline__ unsigned long long rank_key(float m, int token) {
  uint32_t u = __float_as_uint(m + 0.f);  // (-0 + 0 = +0)
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<unsigned long long>(u) << 32) | static_cast<uint32_t>(0x7fffffff - token);
}
__device__ __forceinline__ int key_token(unsigned long long key) {
  return key == 0ull ? -1 : 0x7fffffff - static_cast<int>(static_cast<uint32_t>(key));
}

// Bitonic stages j = jstart, jstart / 2, .., 1 of sub-sequence size k over the two keys at positions lane (x0)
// and lane + 32 (x1): the lower position of each pair (pos, pos ^ j) keeps the larger key where the
// sub-sequence runs in rank order (pos & k clear, or k = 64), the smaller one elsewhere.
__device__ __forceinline__ void bitonic_stages(unsigned long long& x0, unsigned long long& x1, int k, int jstart,
                                               int lane) {
  for (int j = jstart; j >= 1; j >>= 1) {
    unsigned long long y0, y1;
    if (j == 32) {
      y0 = x1, y1 = x0;
    } else {
      y0 = __shfl_xor_sync(0xffffffffu, x0, j);
      y1 = __shfl_xor_sync(0xffffffffu, x1, j);
    }
    const int p0 = lane, p1 = lane + 32;
    const bool w0 = ((p0 & j) == 0) == ((p0 & k) == 0 || k == 64);  // this position keeps the larger key
    const bool w1 = ((p1 & j) == 0) == ((p1 & k) == 0 || k == 64);
    x0 = (w0 == (y0 > x0)) ? y0 : x0;
    x1 = (w1 == (y1 > x1)) ? y1 : x1;
  }
}

__global__ void __launch_bounds__(kScanThreads, 1) hola_cache_scan_kernel(HolaArgs p) {
  extern __shared__ __align__(16) uint8_t scan_raw[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, bh = blockIdx.x, L = p.L, w = p.w;
  constexpr int kWarps = kScanThreads / 32;
  const int nblocks = (L + 63) / 64;
  const size_t tok0 = (size_t)bh * L;
  unsigned long long* lk = reinterpret_cast<unsigned long long*>(scan_raw);  // [2][nblocks][64] keys
  auto at = [&](int buf, int b, int pos) -> unsigned long long& { return lk[(buf * nblocks + b) * 64 + pos]; };
  auto put = [&](int buf, int b, unsigned long long x0, unsigned long long x1) {  // positions from w on: padding
    at(buf, b, lane) = lane < w ? x0 : 0ull;
    at(buf, b, lane + 32) = lane + 32 < w ? x1 : 0ull;
  };
  // each block's own candidates, sorted into rank order
  for (int b = warp; b < nblocks; b += kWarps) {
    const int t0 = 64 * b + lane, t1 = t0 + 32;
    unsigned long long x0 = t0 < L ? rank_key(p.m[tok0 + t0], t0) : 0ull;
    unsigned long long x1 = t1 < L ? rank_key(p.m[tok0 + t1], t1) : 0ull;
    for (int k = 2; k <= 64; k <<= 1) bitonic_stages(x0, x1, k, k / 2, lane);
    put(0, b, x0, x1);
  }
  __syncthreads();
  int cur = 0;
  for (int d = 1; d < nblocks; d <<= 1) {
    for (int b = warp; b < nblocks; b += kWarps) {
      unsigned long long x0 = at(cur, b, lane), x1 = at(cur, b, lane + 32);
      if (b >= d) {  // C_i = max(A_i, B_63-i): A block b's list, B the list d blocks before
        x0 = max(x0, at(cur, b - d, 63 - lane));
        x1 = max(x1, at(cur, b - d, 31 - lane));
        bitonic_stages(x0, x1, 64, 32, lane);
      }
      put(cur ^ 1, b, x0, x1);
    }
    cur ^= 1;
    __syncthreads();
  }
  // block b reads the top w of blocks 0 .. b - 1, in rank order, -1 past its size
  for (int e = tid; e < nblocks * 64; e += kScanThreads) {
    const int b = e >> 6, r = e & 63;
    p.cidx[((size_t)bh * nblocks + b) * 64 + r] = b > 0 ? key_token(at(cur, b - 1, r)) : -1;
  }
  if (p.cache != nullptr && tid < w) {  // the final cache, ascending token indices, -1 past its size
    const int last = nblocks - 1;
    const int mine = key_token(at(cur, last, tid));
    if (mine >= 0) {
      int pos = 0;
      for (int c = 0; c < w; ++c) {
        const int o = key_token(at(cur, last, c));
        pos += (o >= 0 && o < mine) ? 1 : 0;
      }
      p.cache[(size_t)bh * w + pos] = mine;
    } else {
      p.cache[(size_t)bh * w + tid] = -1;
    }
  }
}

// hola_read_block_kernel: one CTA per head and run of kBlocksPerCta consecutive blocks, two CTAs per SM.  Each
// block's q, k, v arrive by TMA, its cache rows by 16-byte cp.async gathers of the token indices chosen above
// (rows 0..63; empty rows zero), then the same S product, softmax with the sink and P V product as the serial
// kernel.  (An L2 prefetch of the next block's tiles and cache rows while a block was read cost 6 %: the
// cache rows repeat from block to block and are mostly in L2 already.)
// The raw queries land in the lo panel: each thread reads its 16-byte chunk there before it writes the lo
// half of the scaled query to the same address, so the CTA fits twice in an SM's shared memory.
constexpr int kBlocksPerCta = 4;
constexpr int PB_K = 0, PB_V = kBuf, PB_H = 2 * kBuf, PB_L = PB_H + kPanel, PB_QS = PB_L;
constexpr int kPSmem = PB_L + kPanel + 1024;

__device__ __forceinline__ void cp_async16_cg(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}

__global__ void __launch_bounds__(kTThreads, 2)
    hola_read_block_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, HolaArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ float rk[kRows];        // 1 / rms(k) per row (0 for empty rows)
  __shared__ int crow[64];           // token index of cache row r (-1 = empty)
  __shared__ float rq[64];
  __shared__ float gqk[kD];          // gamma_q * gamma_k
  __shared__ float red[4][64];
  __shared__ float mxs[64], inv_den[64];
  __shared__ int ncache;
  __shared__ uint64_t bar_mma, bar_load;
  __shared__ uint32_t tmem_base;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qw = warp & 3, half = warp >> 2;
  const int bh = blockIdx.y, h = bh % p.H;
  const int L = p.L, nblocks = (L + 63) / 64;
  const int blk_begin = blockIdx.x * kBlocksPerCta, blk_end = min(nblocks, blk_begin + kBlocksPerCta);
  const size_t tok0 = (size_t)bh * L;
  const float sink = p.sink[h];
  const float inv_sqrt_d = rsqrtf((float)kD);
  const uint32_t t_lane = static_cast<uint32_t>(32 * qw) << 16;
  uint8_t* KB = sm + PB_K;
  uint8_t* VB = sm + PB_V;
  const uint8_t* kbytes = reinterpret_cast<const uint8_t*>(p.k);
  const uint8_t* vbytes = reinterpret_cast<const uint8_t*>(p.v);

  if (tid == 0) {
    sm100::prefetch_tmap(&tm_q);
    sm100::prefetch_tmap(&tm_k);
    sm100::prefetch_tmap(&tm_v);
    sm100::mbar_init(&bar_mma, 1);
    sm100::mbar_init(&bar_load, 1);
    sm100::fence_mbar_init();
  }
  if (warp == 0) {
    sm100::tmem_alloc(&tmem_base, kTmemCols);
    sm100::tmem_relinquish();
  }
  if (tid < kD) gqk[tid] = p.gamma_q[tid] * p.gamma_k[tid];
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t qh = sm100::smem_u32(sm + PB_H), ql = sm100::smem_u32(sm + PB_L);
  uint32_t lphase = 0;
  bool bad = false;

  for (int blk = blk_begin; blk < blk_end && !bad; ++blk) {
    const int b0 = 64 * blk, nb = min(64, L - b0);
    if (tid == 0) {  // the block's raw k, v (rows 64..127) and q (the lo panel): six 64 x 64 boxes
      sm100::mbar_arrive_expect_tx(&bar_load, 3 * kNP * 64 * 128);
#pragma unroll
      for (int pn = 0; pn < kNP; ++pn) {
        sm100::tma_load_3d(KB + pn * kPanel + 64 * 128, &tm_k, &bar_load, 64 * pn, b0, bh);
        sm100::tma_load_3d(VB + pn * kPanel + 64 * 128, &tm_v, &bar_load, 64 * pn, b0, bh);
        sm100::tma_load_3d(sm + PB_QS + pn * kQPanel, &tm_q, &bar_load, 64 * pn, b0, bh);
      }
    }
    if (tid < 64) crow[tid] = p.cidx[((size_t)bh * nblocks + blk) * 64 + tid];
    __syncthreads();
    // cache rows: 64 rows x (key, value) x 16 chunks of 16 bytes, gathered by token index; empty rows zero
    for (int e = tid; e < 64 * 2 * 2 * kNP * 8 / 2; e += kTThreads) {
      const int r = e >> 5, q = e & 31, which = q >> 4, cc = q & 15;
      uint8_t* dst = (which ? VB : KB) + (cc / 8) * kPanel + sm100::sw128_chunk(r, cc % 8);
      const int t = crow[r];
      if (t >= 0) cp_async16_cg(dst, (which ? vbytes : kbytes) + ((tok0 + t) * kD + 8 * cc) * 2);
      else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    {
      int fail = 0;
      if (tid == 0) {
        int n = 0;
        for (int r = 0; r < 64; ++r) n += crow[r] >= 0 ? 1 : 0;
        ncache = n;
        fail = !sm100::mbar_wait_bounded(&bar_load, lphase, kWaitCycles);
      }
      bad = __syncthreads_or(fail);
      lphase ^= 1;
      if (bad) break;
    }

    // ---------------------------------------------------------------- scales of k (cache and block rows), scaled q hi/lo
    {
      const int i = tid >> 2, part = tid & 3;   // row of each half, quarter of its 16 chunks
      float kss_c = 0.f, kss = 0.f, qss = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = 4 * part + u;             // chunk: elements 8 c .. 8 c + 7
        const uint4 kc0 = *reinterpret_cast<const uint4*>(KB + (c / 8) * kPanel + sm100::sw128_chunk(i, c % 8));
        const uint4 kc = *reinterpret_cast<const uint4*>(KB + (c / 8) * kPanel + sm100::sw128_chunk(64 + i, c % 8));
        const uint4 qc = *reinterpret_cast<const uint4*>(sm + PB_QS + (c / 8) * kQPanel + sm100::sw128_chunk(i, c % 8));
        const __nv_bfloat162* k0 = reinterpret_cast<const __nv_bfloat162*>(&kc0);
        const __nv_bfloat162* kh = reinterpret_cast<const __nv_bfloat162*>(&kc);
        const __nv_bfloat162* qh2 = reinterpret_cast<const __nv_bfloat162*>(&qc);
        float qs[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 c0 = __bfloat1622float2(k0[e]), kf = __bfloat1622float2(kh[e]), qf = __bfloat1622float2(qh2[e]);
          kss_c = fmaf(c0.x, c0.x, fmaf(c0.y, c0.y, kss_c));
          kss = fmaf(kf.x, kf.x, fmaf(kf.y, kf.y, kss));
          qss = fmaf(qf.x, qf.x, fmaf(qf.y, qf.y, qss));
          qs[2 * e] = qf.x * gqk[8 * c + 2 * e];
          qs[2 * e + 1] = qf.y * gqk[8 * c + 2 * e + 1];
        }
        store8_split(sm + PB_H, sm + PB_L, (c / 8) * kQPanel + sm100::sw128_chunk(i, c % 8), qs);
      }
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        kss_c += __shfl_xor_sync(0xffffffffu, kss_c, o);
        kss += __shfl_xor_sync(0xffffffffu, kss, o);
        qss += __shfl_xor_sync(0xffffffffu, qss, o);
      }
      if (part == 0) {
        rk[i] = crow[i] >= 0 ? rsqrtf(kss_c / kD + 1e-6f) : 0.f;
        rk[64 + i] = i < nb ? rsqrtf(kss / kD + 1e-6f) : 0.f;
        rq[i] = rsqrtf(qss / kD + 1e-6f);
      }
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();

    // ---------------------------------------------------------------- S^T = K [q o gamma]^T
    {
      int fail = 0;
      if (tid == 0) {
        constexpr uint32_t id = sm100::idesc_bf16(128, 64, false, false);
        const uint32_t kb = sm100::smem_u32(KB);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint64_t a = sm100::smem_desc(kb + (ks / 4) * kPanel + (ks % 4) * 32, 16, 1024);
          const uint32_t boff = (ks / 4) * kQPanel + (ks % 4) * 32;
          sm100::mma_bf16(tmem + T_S, a, sm100::smem_desc(qh + boff, 16, 1024), id, ks > 0);
          sm100::mma_bf16(tmem + T_S, a, sm100::smem_desc(ql + boff, 16, 1024), id, true);
        }
        sm100::mma_commit(&bar_mma);
        fail = !sm100::mbar_wait_bounded(&bar_mma, 0, kWaitCycles);
      }
      bad = __syncthreads_or(fail);
      sm100::tc_fence_after();
      if (bad) break;
    }

    // ---------------------------------------------------------------- softmax over the keys (lanes) of each query
    const int j = 32 * qw + lane;             // key row
    float x[32];
    {
      float s2[32];
      sm100::tmem_ld32(tmem + t_lane + T_S + 32 * half, s2);
      sm100::tmem_wait_ld();
      const float kscale = rk[j] * inv_sqrt_d;
      const int nc = ncache;
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int t = 32 * half + u;
        const bool vis = j < 64 ? j < nc : (j - 64 <= t && j - 64 < nb);
        x[u] = vis ? s2[u] * kscale * rq[t] : -INFINITY;
        s2[u] = x[u];
      }
      red[qw][32 * half + lane] = butterfly<0>(s2, lane);
    }
    __syncthreads();
    if (tid < 64) mxs[tid] = fmaxf(fmaxf(fmaxf(red[0][tid], red[1][tid]), fmaxf(red[2][tid], red[3][tid])), sink);
    __syncthreads();
    {
      float s2[32];
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        x[u] = __expf(x[u] - mxs[32 * half + u]);  // exp(-inf) = 0 for hidden keys
        s2[u] = x[u];
      }
      red[qw][32 * half + lane] = butterfly<1>(s2, lane);
    }
    __syncthreads();
    if (tid < 64) inv_den[tid] = 1.f / (red[0][tid] + red[1][tid] + red[2][tid] + red[3][tid] + __expf(sink - mxs[tid]));
    __syncthreads();
    // P (key rows, query columns) as bf16 hi / lo over the query panels, which the S product no longer reads
#pragma unroll
    for (int q8 = 0; q8 < 4; ++q8) {
      float pv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) pv[e] = x[8 * q8 + e] * inv_den[32 * half + 8 * q8 + e];
      store8_split(sm + PB_H, sm + PB_L, sm100::sw128_chunk(j, 4 * half + q8), pv);
    }
    sm100::fence_async_smem();
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();

    // ---------------------------------------------------------------- O^T = V^T P
    {
      int fail = 0;
      if (tid == 0) {
        constexpr uint32_t id = sm100::idesc_bf16(128, 64, true, true);
        const uint32_t vb = sm100::smem_u32(VB);
#pragma unroll
        for (int ks = 0; ks < kRows / 16; ++ks) {
          const uint64_t a = sm100::smem_desc(vb + ks * 2048, kPanel, 1024);
          sm100::mma_bf16(tmem + T_O, a, sm100::smem_desc(qh + ks * 2048, kPanel, 1024), id, ks > 0);
          sm100::mma_bf16(tmem + T_O, a, sm100::smem_desc(ql + ks * 2048, kPanel, 1024), id, true);
        }
        sm100::mma_commit(&bar_mma);
        fail = !sm100::mbar_wait_bounded(&bar_mma, 1, kWaitCycles);
      }
      bad = __syncthreads_or(fail);
      sm100::tc_fence_after();
      if (bad) break;
    }
    {
      float o[32];
      sm100::tmem_ld32(tmem + t_lane + T_O + 32 * half, o);
      sm100::tmem_wait_ld();
#pragma unroll
      for (int u = 0; u < 32; ++u) {
        const int t = 32 * half + u;
        if (t < nb) p.o[(tok0 + b0 + t) * kD + j] = o[u];
      }
    }
    // the next block's copies overwrite every buffer this one read: all reads done, also by the async proxy
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
  }
  if (bad && tid == 0) raise_status(p.status, kStatusTimeout);
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 0) sm100::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

bool hola_tc_supported(int dk, int dv, int in_dtype, int block) {
  return dk == kD && dv == kD && in_dtype == kBF16 && block == 64;
}

cudaError_t launch_hola_read_tc(const HolaArgs& p, int BH, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (!make_bf16_tmap(&tq, p.q, BH, p.L, kD) || !make_bf16_tmap(&tk, p.k, BH, p.L, kD) ||
      !make_bf16_tmap(&tv, p.v, BH, p.L, kD))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (p.cidx != nullptr) {  // every block's cache first, then all blocks at once
    if (p.w < 1 || p.w > 64) return cudaErrorInvalidValue;
    const int nb = (p.L + 63) / 64;
    if (nb <= kScanMaxBlocks) {
      const size_t sb = scan_smem_bytes(nb);
      e = cudaFuncSetAttribute(hola_cache_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
      if (e != cudaSuccess) return e;
      hola_cache_scan_kernel<<<BH, kScanThreads, sb, stream>>>(p);
    } else {
      hola_cache_select_kernel<<<BH, kSelThreads, 0, stream>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(hola_read_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmem);
    if (e != cudaSuccess) return e;
    const int nblocks = (p.L + 63) / 64;
    hola_read_block_kernel<<<dim3((nblocks + kBlocksPerCta - 1) / kBlocksPerCta, BH), kTThreads, kPSmem, stream>>>(
        tq, tk, tv, p);
    return cudaGetLastError();
  }
  e = cudaFuncSetAttribute(hola_read_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  hola_read_tc_kernel<<<BH, kTThreads, kSmem, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace kdn
