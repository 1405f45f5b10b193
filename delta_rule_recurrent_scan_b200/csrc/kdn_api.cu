// C-ABI layer of libkdn: argument validation, workspace layout, dispatch.
//
// Declared in include/kdn.h.  Every entry point validates its arguments on the
// host (enqueuing nothing on failure), clears the device status word in the
// caller's workspace, and enqueues its kernels on the caller's stream.
#include <cuda_runtime.h>

#include <cstdio>
#include <string>
#include <utility>

#include "../../include/kdn.h"
#include "api_internal.h"
#include "chunk.h"
#include "common.cuh"
#include "kernels.h"

namespace kdn {
namespace api {

thread_local std::string g_last_error;

kdn_status fail(kdn_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

kdn_status ok() {
  g_last_error.clear();
  return KDN_OK;
}

bool supported_dim(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

// A device-accessible pointer: device or managed memory.
kdn_status check_ptr(const void* p, const char* name, size_t align, bool allow_null) {
  if (p == nullptr) {
    if (allow_null) return KDN_OK;
    return fail(KDN_ERR_INVALID_ARG, std::string(name) + " is NULL");
  }
  if (reinterpret_cast<uintptr_t>(p) % align != 0)
    return fail(KDN_ERR_INVALID_ARG, std::string(name) + " is not " + std::to_string(align) + "-byte aligned");
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(KDN_ERR_INVALID_ARG, std::string(name) + ": cudaPointerGetAttributes failed (" +
                                         cudaGetErrorString(e) + ")");
  }
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail(KDN_ERR_INVALID_ARG, std::string(name) + " is not a device pointer");
  return KDN_OK;
}

// Launch on the device that owns the state buffer (the library links its own CUDA runtime, whose
// current device need not be the caller's); ``guard`` puts the caller's device back on return.
kdn_status use_device_of(const void* p, DeviceGuard& guard) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return fail(KDN_ERR_INVALID_ARG, "cannot query the device of the state buffer");
  }
  const cudaError_t e = static_cast<cudaError_t>(guard.switch_to(attr.device));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(KDN_ERR_CUDA, std::string("cudaSetDevice: ") + cudaGetErrorString(e));
  }
  return KDN_OK;
}

#define KDN_TRY(expr)                 \
  do {                                \
    kdn_status _s = (expr);           \
    if (_s != KDN_OK) return _s;      \
  } while (0)

kdn_status check_dims(const kdn_dims* d) {
  if (d == nullptr) return fail(KDN_ERR_INVALID_ARG, "dims is NULL");
  if (d->B < 1 || d->H < 1 || d->L < 0)
    return fail(KDN_ERR_INVALID_ARG, "B and H must be >= 1 and L >= 0");
  if ((long long)d->B * d->H * (long long)(d->L > 0 ? d->L : 1) > (1LL << 40))
    return fail(KDN_ERR_INVALID_ARG, "B*H*L too large");
  if (d->in_dtype != KDN_F32 && d->in_dtype != KDN_BF16) return fail(KDN_ERR_INVALID_ARG, "bad in_dtype");
  if (d->out_dtype != KDN_F32 && d->out_dtype != KDN_BF16) return fail(KDN_ERR_INVALID_ARG, "bad out_dtype");
  if (!supported_dim(d->dk) || !supported_dim(d->dv))
    return fail(KDN_ERR_UNSUPPORTED, "dk and dv must be 16, 32, 64 or 128");
  if (d->chunk != 0 && d->chunk != 16 && d->chunk != 32 && d->chunk != 64)
    return fail(KDN_ERR_UNSUPPORTED, "chunk must be 0, 16, 32 or 64");
  return KDN_OK;
}



size_t gains_bytes(const kdn_dims* d) { return (size_t)d->B * d->H * (size_t)d->L * d->dk * sizeof(float); }

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

// ---------------------------------------------------------------- segment-parallel scans
constexpr int kSegTargetCtas = 148;  // one chunk-kernel CTA per SM of a B200

kdn_variant body_of(kdn_variant var) { return var == KDN_KALMAN_ISO ? KDN_DELTA : var; }

// Segments per head for this request (1 = the serial scan).  An explicit request that cannot be served
// fails; the library choice never does.
kdn_status resolve_segments(kdn_variant var, const kdn_dims* d, int* P_out) {
  *P_out = 1;
  if (d->segments < 0) return fail(KDN_ERR_INVALID_ARG, "segments must be >= 0");
  if (d->segments == 1 || d->L == 0) return KDN_OK;
  const bool chunked = kdn::chunk_supported(body_of(var), *d);
  if (d->segments >= 2) {
    if (!chunked) return fail(KDN_ERR_UNSUPPORTED, "segments > 1 needs the chunked path (bf16, dk = dv in {64, 128})");
    if (d->L % d->segments != 0) return fail(KDN_ERR_INVALID_ARG, "segments must divide L");
    *P_out = d->segments;
    return KDN_OK;
  }
  if (!chunked) return KDN_OK;
  const long long BH = (long long)d->B * d->H;
  for (int P = 16; P >= 4; P /= 2)
    if (BH * P <= kSegTargetCtas && d->L % (64 * P) == 0 && d->L / (64 * P) >= 2) {
      *P_out = P;
      return KDN_OK;
    }
  return KDN_OK;
}

// Full Kalman with P segments: the covariance side runs as P runs of chunks (the last one possibly shorter),
// each from its own start covariance.
int riccati_run_chunks(const kdn_dims* d, int P) {
  const int nch = (d->L + 63) / 64;
  return (nch + P - 1) / P;
}

// Byte offsets inside the segment area of the workspace.
struct SegLayout {
  size_t sz, si, sc, maps, p[3], end;
};

SegLayout seg_layout(kdn_variant body, const kdn_dims* d, int P) {
  SegLayout l{};
  const size_t V = (size_t)d->B * d->H * P;
  const size_t states = round256(V * d->dk * d->dv * sizeof(float));
  l.sz = 0, l.si = states, l.sc = 2 * states, l.end = 3 * states;
  if (body == KDN_KALMAN_DIAG) {
    l.maps = l.end, l.end += round256(V * d->dk * 4 * sizeof(float));
    for (int i = 0; i < 3; ++i) l.p[i] = l.end, l.end += round256(V * d->dk * sizeof(float));
  }
  return l;
}

// Start of the segment area: after the status word and the variant's own scratch.
size_t seg_area_offset(kdn_variant var, const kdn_dims* d) {
  size_t n = kStatusBytes;
  if (var == KDN_KALMAN_DIAG || var == KDN_KALMAN_FULL) n += gains_bytes(d);
  if (var == KDN_KALMAN_ISO) n += (size_t)d->B * d->H * (size_t)d->L * sizeof(float);
  return round256(n);
}

kdn_status common_checks(kdn_variant var, const kdn_dims* d, const void* q, const void* k, const void* v,
                         const float* S, const void* o, const float* m, const void* ws, size_t ws_bytes,
                         DeviceGuard& guard) {
  KDN_TRY(check_dims(d));
  int P = 1;
  KDN_TRY(resolve_segments(var, d, &P));
  const bool any = d->L > 0;
  KDN_TRY(check_ptr(S, "S", 16, false));
  KDN_TRY(check_ptr(q, "q", 16, !any));
  KDN_TRY(check_ptr(k, "k", 16, !any));
  KDN_TRY(check_ptr(v, "v", 16, !any));
  KDN_TRY(check_ptr(o, "o", 16, !any));
  KDN_TRY(check_ptr(m, "m", 4, true));
  KDN_TRY(check_ptr(ws, "workspace", 256, false));
  const size_t need = kdn_workspace_bytes(var, d);
  if (ws_bytes < need)
    return fail(KDN_ERR_INVALID_ARG, "workspace_bytes " + std::to_string(ws_bytes) + " < required " +
                                         std::to_string(need));
  return use_device_of(S, guard);
}

kdn_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(KDN_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// The memory side over P segments per head (the steps are listed with kdn_dims.segments in kdn.h).
// ``c`` carries the caller's buffers (c.P: diagonal p); ``gains``: full-Kalman per-token gains.
kdn_status seg_scan(kdn_variant body, const kdn_dims* d, int P, const kdn::ChunkArgs& c, const float* gains,
                    char* area, cudaStream_t st) {
  const int BH = c.BH, D = d->dk;
  const size_t DD = (size_t)D * d->dv;
  const SegLayout lay = seg_layout(body, d, P);
  kdn::SegArgs sa{};
  sa.P = P, sa.L = c.L, sa.k = c.k, sa.in_dtype = d->in_dtype, sa.a = c.a, sa.r = c.r, sa.qn = c.qn;
  sa.qn_scalar = c.qn_scalar, sa.p0 = c.P, sa.status = c.status;
  sa.S = c.S;
  sa.Sz = reinterpret_cast<float*>(area + lay.sz);
  sa.SI = reinterpret_cast<float*>(area + lay.si);
  sa.Sc = reinterpret_cast<float*>(area + lay.sc);
  const bool diag = body == KDN_KALMAN_DIAG;
  // d = 64: B and M from one run on the d x 2d state [S | M] (Sz and SI hold it side by side)
  sa.aug = D == 64 && d->dv == 64 ? 1 : 0;
  if (diag) {
    sa.maps = reinterpret_cast<float4*>(area + lay.maps);
    for (int i = 0; i < 3; ++i) sa.pcopy[i] = reinterpret_cast<float*>(area + lay.p[i]);
    sa.ncopy = 3;
    KDN_TRY(cuda_status(kdn::launch_seg_uncertainty(D, sa, BH, st), "segment uncertainty launch"));
  }
  KDN_TRY(cuda_status(kdn::launch_seg_init(D, sa, BH, st), "segment start-state launch"));
  // every segment as a head of its own: [BH, L, d] viewed as [BH P, L / P, d]
  kdn_dims dv = *d;
  dv.B = BH * P, dv.H = 1, dv.L = c.L / P, dv.segments = 1;
  kdn::ChunkArgs v = c;
  v.BH = BH * P, v.L = c.L / P;
  // each segment's map S0 -> M S0 + B: runs from S0 = 0 and S0 = I, or one run from [0 | I] (no read-out
  // or surprise: o and m are written by the true run below)
  v.o = nullptr, v.m = nullptr;
  v.S = sa.Sz, v.P = diag ? sa.pcopy[0] : c.P;
  if (sa.aug) v.state_cols = 2 * d->dv;
  KDN_TRY(cuda_status(kdn::launch_chunk_sside(body, dv, v, gains, st), "segment scan launch"));
  if (!sa.aug) {
    v.S = sa.SI, v.P = diag ? sa.pcopy[1] : c.P;
    KDN_TRY(cuda_status(kdn::launch_chunk_sside(body, dv, v, gains, st), "segment scan launch"));
  }
  v.state_cols = 0;
  KDN_TRY(cuda_status(kdn::launch_seg_combine(D, sa, BH, st), "segment chaining launch"));
  // the true scan of every segment from its start state
  v.o = c.o, v.m = c.m;
  v.S = sa.Sc, v.P = diag ? sa.pcopy[2] : c.P;
  KDN_TRY(cuda_status(kdn::launch_chunk_sside(body, dv, v, gains, st), "segment scan launch"));
  // the last segment's end state (and p) is the head's
  cudaError_t e = cudaMemcpy2DAsync(c.S, DD * sizeof(float), sa.Sc + (size_t)(P - 1) * DD, P * DD * sizeof(float),
                                    DD * sizeof(float), BH, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess && diag)
    e = cudaMemcpy2DAsync(c.P, D * sizeof(float), sa.pcopy[2] + (size_t)(P - 1) * D, P * D * sizeof(float),
                          D * sizeof(float), BH, cudaMemcpyDeviceToDevice, st);
  return cuda_status(e, "copying the final state");
}

}  // namespace api
}  // namespace kdn

using namespace kdn::api;

extern "C" {

int kdn_api_version(void) { return KDN_API_VERSION; }

const char* kdn_status_string(kdn_status s) {
  switch (s) {
    case KDN_OK: return "KDN_OK";
    case KDN_ERR_INVALID_ARG: return "KDN_ERR_INVALID_ARG";
    case KDN_ERR_UNSUPPORTED: return "KDN_ERR_UNSUPPORTED";
    case KDN_ERR_CUDA: return "KDN_ERR_CUDA";
    case KDN_ERR_NUMERIC: return "KDN_ERR_NUMERIC";
    case KDN_ERR_TIMEOUT: return "KDN_ERR_TIMEOUT";
  }
  return "KDN_UNKNOWN_STATUS";
}

const char* kdn_last_error(void) { return g_last_error.c_str(); }

size_t kdn_workspace_bytes(kdn_variant variant, const kdn_dims* dims) {
  if (dims == nullptr || dims->B < 1 || dims->H < 1 || dims->L < 0) return 0;
  if (!supported_dim(dims->dk) || !supported_dim(dims->dv)) return 0;
  if (variant != KDN_DELTA && variant != KDN_KALMAN_DIAG && variant != KDN_KALMAN_FULL && variant != KDN_KALMAN_ISO)
    return 0;
  int P = 1;
  if (resolve_segments(variant, dims, &P) != KDN_OK) return 0;
  size_t n = seg_area_offset(variant, dims);
  if (P > 1) n += seg_layout(body_of(variant), dims, P).end;
  // few heads, full Kalman: the covariance side runs chunk-parallel from every chunk's start covariance
  if (P > 1 && variant == KDN_KALMAN_FULL)
    n = round256(n) + kdn::riccati_scratch_bytes(dims->dk, dims->B * dims->H, dims->L, riccati_run_chunks(dims, P));
  return round256(n);
}

kdn_status kdn_plan(kdn_variant variant, const kdn_dims* dims, int* launches, const char** kernel,
                    const char** arith) {
  KDN_TRY(check_dims(dims));
  if (variant != KDN_DELTA && variant != KDN_KALMAN_DIAG && variant != KDN_KALMAN_FULL && variant != KDN_KALMAN_ISO)
    return fail(KDN_ERR_INVALID_ARG, "bad variant");
  // the isotropic scan is the delta scan after its beta prologue (one more launch)
  const kdn_variant body = variant == KDN_KALMAN_ISO ? KDN_DELTA : variant;
  int n = 0;
  const char* name = "";
  const char* ar = "f32";
  if (dims->L == 0) {
    n = 0, name = "none";
  } else if (kdn::chunk_supported(body, *dims)) {
    kdn::chunk_plan(body, *dims, &n, &name, &ar);
  } else if (body == KDN_DELTA) {
    n = 1, name = "seq_scan_kernel";
  } else {
    n = 2, name = "seq_scan_kernel";
  }
  int nseg = 1;
  KDN_TRY(resolve_segments(variant, dims, &nseg));
  if (nseg > 1) {
    // start states, two map runs (one on [S | M] at d = 64), chaining, the true run (+ the diagonal
    // uncertainty maps and starts; for full Kalman the chunk maps, their chain, the run-start covariances
    // and the covariance side)
    n = (dims->dk == 64 ? 4 : 5) + (body == KDN_KALMAN_DIAG ? 2 : 0) + (body == KDN_KALMAN_FULL ? 4 : 0);
    if (body == KDN_KALMAN_FULL)  // the longest of those launches (d = 128: on the tensor cores)
      name = dims->dk == 128 ? "riccati_chain_tc_kernel" : "riccati_chain_kernel", ar = dims->dk == 128 ? "bf16-tc" : "f32";
  }
  if (variant == KDN_KALMAN_ISO && n > 0 && !(kdn::chunk_supported(KDN_DELTA, *dims) && nseg == 1))
    n += 1;  // the beta prologue (the one-segment chunk kernel runs it itself on the serial path)
  if (launches) *launches = n;
  if (kernel) *kernel = name;
  if (arith) *arith = ar;
  return ok();
}

kdn_status kdn_read_device_status(const void* workspace, int* status_out, void* stream) {
  if (status_out == nullptr) return fail(KDN_ERR_INVALID_ARG, "status_out is NULL");
  DeviceGuard guard;
  const void* word_ptr = workspace;
  if (workspace == nullptr) {
    // the no-alloc entry point's status word, in its static array on the current device
    void* p = nullptr;
    KDN_TRY(noalloc_scratch_on_current_device(&p));
    word_ptr = p;
  } else {
    KDN_TRY(check_ptr(workspace, "workspace", 256, false));
    KDN_TRY(use_device_of(workspace, guard));
  }
  unsigned word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, word_ptr, sizeof(word), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "reading the device status");
  *status_out = (word & kdn::kStatusNumeric) ? KDN_ERR_NUMERIC : (word & kdn::kStatusTimeout) ? KDN_ERR_TIMEOUT : KDN_OK;
  return ok();
}

kdn_status kdn_scan_delta(const kdn_dims* dims, const void* q, const void* k, const void* v, const float* beta,
                          const float* a, float* S, void* o, float* m, void* workspace, size_t workspace_bytes,
                          void* stream) {
  DeviceGuard guard;
  KDN_TRY(common_checks(KDN_DELTA, dims, q, k, v, S, o, m, workspace, workspace_bytes, guard));
  const bool any = dims->L > 0;
  KDN_TRY(check_ptr(beta, "beta", 4, !any));
  KDN_TRY(check_ptr(a, "a", 4, true));
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_status(e, "clearing the status word");
  if (!any) return ok();
  const int BH = dims->B * dims->H;
  if (kdn::chunk_supported(KDN_DELTA, *dims)) {
    kdn::ChunkArgs c{};
    c.q = q, c.k = k, c.v = v, c.beta = beta, c.a = a, c.S = S, c.o = o, c.m = m;
    c.out_dtype = dims->out_dtype, c.BH = BH, c.L = dims->L;
    c.status = reinterpret_cast<unsigned*>(workspace);
    int P = 1;
    KDN_TRY(resolve_segments(KDN_DELTA, dims, &P));
    if (P > 1)
      return seg_scan(KDN_DELTA, dims, P, c, nullptr,
                      reinterpret_cast<char*>(workspace) + seg_area_offset(KDN_DELTA, dims), st);
    return cuda_status(kdn::launch_chunk(KDN_DELTA, *dims, c, st), "chunked delta scan launch");
  }
  kdn::SeqScanArgs s{q, k, v, dims->in_dtype, dims->out_dtype, beta, a, nullptr, S, o, m, BH, dims->L};
  return cuda_status(kdn::launch_seq_scan(dims->dk, dims->dv, s, st), "delta scan launch");
}

}  // extern "C"

kdn_status kdn::api::kalman_scan(kdn_variant var, const kdn_dims* dims, const void* q, const void* k, const void* v,
                              const float* a, const float* r, const float* qn, float qn_scalar, float* S, float* P,
                              void* o, float* m, void* workspace, size_t workspace_bytes, void* stream) {
  DeviceGuard guard;
  KDN_TRY(common_checks(var, dims, q, k, v, S, o, m, workspace, workspace_bytes, guard));
  const bool any = dims->L > 0;
  KDN_TRY(check_ptr(P, var == KDN_KALMAN_FULL ? "P" : "p", var == KDN_KALMAN_FULL ? 16 : 4, false));
  KDN_TRY(check_ptr(r, "r", 4, !any));
  KDN_TRY(check_ptr(a, "a", 4, true));
  KDN_TRY(check_ptr(qn, "qn", 4, true));
  if (!(qn_scalar >= 0.f)) return fail(KDN_ERR_INVALID_ARG, "qn_scalar must be >= 0");
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_status(e, "clearing the status word");
  if (!any) return ok();
  const int BH = dims->B * dims->H;
  unsigned* status = reinterpret_cast<unsigned*>(workspace);
  if (kdn::chunk_supported(var, *dims)) {
    kdn::ChunkArgs c{};
    c.q = q, c.k = k, c.v = v, c.a = a, c.r = r, c.qn = qn, c.qn_scalar = qn_scalar, c.S = S, c.o = o, c.m = m;
    c.P = P, c.out_dtype = dims->out_dtype, c.BH = BH, c.L = dims->L, c.status = status;
    c.workspace = reinterpret_cast<char*>(workspace) + kStatusBytes;
    int nseg = 1;
    KDN_TRY(resolve_segments(var, dims, &nseg));
    if (nseg > 1) {
      float* gains = nullptr;
      if (var == KDN_KALMAN_FULL) {
        // the covariance at every chunk start through the chunks' Riccati transfer matrices, then every
        // chunk's gains at once; the gains fix every segment's memory map
        gains = reinterpret_cast<float*>(c.workspace);
        char* area = reinterpret_cast<char*>(workspace) + seg_area_offset(var, dims);
        char* rs = area + round256(seg_layout(KDN_KALMAN_FULL, dims, nseg).end);
        const int cps = riccati_run_chunks(dims, nseg), nch = (dims->L + 63) / 64;
        const size_t chunks = (size_t)BH * nch, runs = (size_t)BH * ((nch + cps - 1) / cps), dk = dims->dk;
        kdn::RiccatiArgs ra{};
        ra.k = k, ra.a = a, ra.r = r, ra.qn = qn, ra.qn_scalar = qn_scalar, ra.P0 = P, ra.cps = cps;
        ra.map_g = reinterpret_cast<float*>(rs);
        rs += round256(chunks * 64 * 64 * 4);
        ra.map_u = reinterpret_cast<float*>(rs);
        rs += round256(chunks * 64 * 4);
        ra.map_ab = reinterpret_cast<float*>(rs);
        rs += round256(chunks * 2 * 64 * 4);
        ra.xy = reinterpret_cast<float*>(rs);
        rs += round256(runs * 2 * dk * dk * 4);
        ra.P_starts = reinterpret_cast<float*>(rs);
        ra.status = status, ra.BH = BH, ra.L = dims->L;
        KDN_TRY(cuda_status(kdn::launch_riccati_starts(dims->dk, ra, st), "Kalman run-start covariance launch"));
        KDN_TRY(cuda_status(kdn::launch_kalman_pside(dims->dk, k, a, r, qn, qn_scalar, P, gains, status, BH, dims->L, st,
                                                     ra.P_starts, cps),
                            "Kalman covariance launch"));
      }
      return seg_scan(var, dims, nseg, c, gains, reinterpret_cast<char*>(workspace) + seg_area_offset(var, dims), st);
    }
    return cuda_status(kdn::launch_chunk(var, *dims, c, st), "chunked Kalman scan launch");
  }
  float* gains = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + kStatusBytes);
  kdn::GainArgs g{k, dims->in_dtype, a, r, qn, qn_scalar, var == KDN_KALMAN_FULL ? P : nullptr,
                  var == KDN_KALMAN_DIAG ? P : nullptr, gains, status, BH, dims->L};
  e = var == KDN_KALMAN_FULL ? kdn::launch_kalman_full_gains(dims->dk, g, st)
                             : kdn::launch_kalman_diag_gains(dims->dk, g, st);
  if (e != cudaSuccess) return cuda_status(e, "Kalman gain launch");
  kdn::SeqScanArgs s{q, k, v, dims->in_dtype, dims->out_dtype, nullptr, a, gains, S, o, m, BH, dims->L};
  return cuda_status(kdn::launch_seq_scan(dims->dk, dims->dv, s, st), "Kalman scan launch");
}

extern "C" {

kdn_status kdn_scan_kalman_full(const kdn_dims* dims, const void* q, const void* k, const void* v, const float* a,
                                const float* r, const float* qn, float qn_scalar, float* S, float* P, void* o,
                                float* m, void* workspace, size_t workspace_bytes, void* stream) {
  return kalman_scan(KDN_KALMAN_FULL, dims, q, k, v, a, r, qn, qn_scalar, S, P, o, m, workspace, workspace_bytes,
                     stream);
}

kdn_status kdn_scan_kalman_diag(const kdn_dims* dims, const void* q, const void* k, const void* v, const float* a,
                                const float* r, const float* qn, float qn_scalar, float* S, float* p, void* o,
                                float* m, void* workspace, size_t workspace_bytes, void* stream) {
  return kalman_scan(KDN_KALMAN_DIAG, dims, q, k, v, a, r, qn, qn_scalar, S, p, o, m, workspace, workspace_bytes,
                     stream);
}

kdn_status kdn_scan_kalman_iso(const kdn_dims* dims, const void* q, const void* k, const void* v, const float* a,
                               const float* r, const float* qn, float qn_scalar, float* S, float* c, void* o,
                               float* m, void* workspace, size_t workspace_bytes, void* stream) {
  DeviceGuard guard;
  KDN_TRY(common_checks(KDN_KALMAN_ISO, dims, q, k, v, S, o, m, workspace, workspace_bytes, guard));
  const bool any = dims->L > 0;
  KDN_TRY(check_ptr(c, "c", 4, false));
  KDN_TRY(check_ptr(r, "r", 4, !any));
  KDN_TRY(check_ptr(a, "a", 4, true));
  KDN_TRY(check_ptr(qn, "qn", 4, true));
  if (!(qn_scalar >= 0.f)) return fail(KDN_ERR_INVALID_ARG, "qn_scalar must be >= 0");
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_status(e, "clearing the status word");
  if (!any) return ok();
  const int BH = dims->B * dims->H;
  unsigned* status = reinterpret_cast<unsigned*>(workspace);
  int nseg = 1;
  KDN_TRY(resolve_segments(KDN_KALMAN_ISO, dims, &nseg));
  if (kdn::chunk_supported(KDN_DELTA, *dims) && nseg == 1) {
    // the chunk kernel runs the uncertainty scan in its own preparation: one launch
    kdn::ChunkArgs ch{};
    ch.q = q, ch.k = k, ch.v = v, ch.a = a, ch.r = r, ch.qn = qn, ch.qn_scalar = qn_scalar, ch.P = c;
    ch.S = S, ch.o = o, ch.m = m, ch.out_dtype = dims->out_dtype, ch.BH = BH, ch.L = dims->L, ch.status = status;
    return cuda_status(kdn::launch_chunk(KDN_KALMAN_ISO, *dims, ch, st), "chunked isotropic scan launch");
  }
  float* beta = reinterpret_cast<float*>(reinterpret_cast<char*>(workspace) + kStatusBytes);
  kdn::IsoArgs ia{k, dims->in_dtype, a, r, qn, qn_scalar, c, beta, status, dims->L};
  e = kdn::launch_iso_beta(dims->dk, ia, BH, st);
  if (e != cudaSuccess) return cuda_status(e, "isotropic beta launch");
  if (kdn::chunk_supported(KDN_DELTA, *dims)) {
    kdn::ChunkArgs ch{};
    ch.q = q, ch.k = k, ch.v = v, ch.beta = beta, ch.a = a, ch.S = S, ch.o = o, ch.m = m;
    ch.out_dtype = dims->out_dtype, ch.BH = BH, ch.L = dims->L, ch.status = status;
    if (nseg > 1)
      return seg_scan(KDN_DELTA, dims, nseg, ch, nullptr,
                      reinterpret_cast<char*>(workspace) + seg_area_offset(KDN_KALMAN_ISO, dims), st);
    return cuda_status(kdn::launch_chunk(KDN_DELTA, *dims, ch, st), "chunked isotropic scan launch");
  }
  kdn::SeqScanArgs sa{q, k, v, dims->in_dtype, dims->out_dtype, beta, a, nullptr, S, o, m, BH, dims->L};
  return cuda_status(kdn::launch_seq_scan(dims->dk, dims->dv, sa, st), "isotropic scan launch");
}

size_t kdn_backward_workspace_bytes(kdn_variant variant, const kdn_dims* dims) {
  if (variant != KDN_DELTA && variant != KDN_KALMAN_ISO && variant != KDN_KALMAN_DIAG && variant != KDN_KALMAN_FULL)
    return 0;
  if (dims == nullptr || dims->B < 1 || dims->H < 1 || dims->L < 0) return 0;
  if (!supported_dim(dims->dk) || !supported_dim(dims->dv)) return 0;
  const size_t BH = (size_t)dims->B * dims->H, DD = (size_t)dims->dk * dims->dv, tok = BH * (size_t)dims->L;
  const size_t nck = ((size_t)dims->L + kdn::kDeltaBwdChunk - 1) / kdn::kDeltaBwdChunk;
  size_t n = kStatusBytes + round256(BH * DD * 4) + round256(BH * nck * DD * 4) + round256(tok * 4);
  // isotropic: beta, the uncertainty before every token, ||k||^2 and dbeta
  if (variant == KDN_KALMAN_ISO) n += 4 * round256(tok * 4);
  // diagonal: the gains, p before every token and dG (d_k values per token each)
  if (variant == KDN_KALMAN_DIAG) n += 3 * round256(tok * dims->dk * 4);
  // full: the gains and dG, then P at every 32-token block start and one block's P before every token per head
  if (variant == KDN_KALMAN_FULL)
    n += 2 * round256(tok * dims->dk * 4) + kdn::full_backward_scratch_bytes((int)BH, dims->L, dims->dk);
  return n;
}

// The gated-delta backward after validation, on the current device: ``ws`` holds the status word, then
// the working state, the chunk-start checkpoints and the residual norms (kdn_backward_workspace_bytes).
kdn_status delta_backward_run(const kdn_dims* dims, const void* q, const void* k, const void* v, const float* beta,
                              const float* a, const float* S0, const float* dO, const float* dm, const float* dS_L,
                              float* dq, float* dk, float* dv, float* dbeta, float* da, float* dS0, void* workspace,
                              cudaStream_t st, const float* gains = nullptr, float* dgain = nullptr) {
  // gains != nullptr: the per-token gains are given (diagonal Kalman) and dG goes to dgain; beta, dbeta unused
  const bool any = dims->L > 0;
  const size_t BH = (size_t)dims->B * dims->H, L = dims->L, DD = (size_t)dims->dk * dims->dv;
  const size_t nck = (L + kdn::kDeltaBwdChunk - 1) / kdn::kDeltaBwdChunk;
  char* ws = reinterpret_cast<char*>(workspace);
  float* S_work = reinterpret_cast<float*>(ws + kStatusBytes);
  float* ckpt = reinterpret_cast<float*>(ws + kStatusBytes + round256(BH * DD * 4));
  float* enorm = reinterpret_cast<float*>(ws + kStatusBytes + round256(BH * DD * 4) + round256(BH * nck * DD * 4));
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_status(e, "clearing the status word");
  if (!any) {  // nothing to go back through: dS0 = dS_L
    e = dS_L != nullptr ? cudaMemcpyAsync(dS0, dS_L, BH * DD * 4, cudaMemcpyDeviceToDevice, st)
                        : cudaMemsetAsync(dS0, 0, BH * DD * 4, st);
    return cuda_status(e, "dS0 of an empty sequence");
  }
  // the sums over value-column blocks accumulate into zeroed outputs
  e = cudaMemsetAsync(dq, 0, BH * L * dims->dk * 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dk, 0, BH * L * dims->dk * 4, st);
  if (e == cudaSuccess)
    e = gains != nullptr ? cudaMemsetAsync(dgain, 0, BH * L * dims->dk * 4, st) : cudaMemsetAsync(dbeta, 0, BH * L * 4, st);
  if (e == cudaSuccess && da != nullptr) e = cudaMemsetAsync(da, 0, BH * L * 4, st);
  if (e == cudaSuccess)
    e = S0 != nullptr ? cudaMemcpyAsync(S_work, S0, BH * DD * 4, cudaMemcpyDeviceToDevice, st)
                      : cudaMemsetAsync(S_work, 0, BH * DD * 4, st);
  if (e != cudaSuccess) return cuda_status(e, "preparing the backward buffers");
  // forward again, keeping the state at every chunk start and the residual norms
  kdn::SeqScanArgs fw{q, k, v, dims->in_dtype, KDN_F32, gains != nullptr ? nullptr : beta, a, gains, S_work, nullptr,
                      nullptr, (int)BH, (int)L};
  fw.S_ckpt = ckpt, fw.enorm = enorm, fw.ckpt_every = kdn::kDeltaBwdChunk;
  KDN_TRY(cuda_status(kdn::launch_seq_scan(dims->dk, dims->dv, fw, st), "backward: forward checkpoints launch"));
  kdn::DeltaBwdArgs bw{q, k, v, dims->in_dtype, beta, a, dO, dm, dS_L, ckpt, enorm, dq, dk, dv, dbeta, da, dS0,
                       (int)BH, (int)L};
  bw.gains = gains, bw.dgain = dgain;
  return cuda_status(kdn::launch_delta_bwd(dims->dk, dims->dv, bw, st), "backward launch");
}

kdn_status kdn_scan_delta_backward(const kdn_dims* dims, const void* q, const void* k, const void* v, const float* beta,
                                   const float* a, const float* S0, const float* dO, const float* dm, const float* dS_L,
                                   float* dq, float* dk, float* dv, float* dbeta, float* da, float* dS0,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  KDN_TRY(check_dims(dims));
  const bool any = dims->L > 0;
  KDN_TRY(check_ptr(dS0, "dS0", 16, false));
  for (const auto& pr : {std::make_pair((const void*)q, "q"), std::make_pair((const void*)k, "k"),
                         std::make_pair((const void*)v, "v"), std::make_pair((const void*)dO, "dO"),
                         std::make_pair((const void*)dq, "dq"), std::make_pair((const void*)dk, "dk"),
                         std::make_pair((const void*)dv, "dv")})
    KDN_TRY(check_ptr(pr.first, pr.second, 16, !any));
  KDN_TRY(check_ptr(beta, "beta", 4, !any));
  KDN_TRY(check_ptr(dbeta, "dbeta", 4, !any));
  KDN_TRY(check_ptr(a, "a", 4, true));
  KDN_TRY(check_ptr(da, "da", 4, true));
  KDN_TRY(check_ptr(dm, "dm", 4, true));
  KDN_TRY(check_ptr(S0, "S0", 16, true));
  KDN_TRY(check_ptr(dS_L, "dS_L", 16, true));
  KDN_TRY(check_ptr(workspace, "workspace", 256, false));
  const size_t need = kdn_backward_workspace_bytes(KDN_DELTA, dims);
  if (workspace_bytes < need)
    return fail(KDN_ERR_INVALID_ARG, "workspace_bytes " + std::to_string(workspace_bytes) + " < required " +
                                         std::to_string(need));
  DeviceGuard guard;
  KDN_TRY(use_device_of(dS0, guard));
  cudaStream_t st = (cudaStream_t)stream;
  return delta_backward_run(dims, q, k, v, beta, a, S0, dO, dm, dS_L, dq, dk, dv, dbeta, da, dS0, workspace, st);
}

kdn_status kdn_scan_kalman_iso_backward(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                       const float* r, const float* a, const float* qn, float qn_scalar,
                                       const float* S0, const float* c0, const float* dO, const float* dm,
                                       const float* dS_L, const float* dc_L, float* dq, float* dk, float* dv,
                                       float* dr, float* da, float* dqn, float* dS0, float* dc0, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  KDN_TRY(check_dims(dims));
  const bool any = dims->L > 0;
  KDN_TRY(check_ptr(dS0, "dS0", 16, false));
  KDN_TRY(check_ptr(dc0, "dc0", 4, false));
  for (const auto& pr : {std::make_pair((const void*)q, "q"), std::make_pair((const void*)k, "k"),
                         std::make_pair((const void*)v, "v"), std::make_pair((const void*)dO, "dO"),
                         std::make_pair((const void*)dq, "dq"), std::make_pair((const void*)dk, "dk"),
                         std::make_pair((const void*)dv, "dv")})
    KDN_TRY(check_ptr(pr.first, pr.second, 16, !any));
  KDN_TRY(check_ptr(r, "r", 4, !any));
  KDN_TRY(check_ptr(dr, "dr", 4, !any));
  KDN_TRY(check_ptr(dqn, "dqn", 4, !any));
  KDN_TRY(check_ptr(a, "a", 4, true));
  KDN_TRY(check_ptr(da, "da", 4, true));
  KDN_TRY(check_ptr(qn, "qn", 4, true));
  KDN_TRY(check_ptr(dm, "dm", 4, true));
  KDN_TRY(check_ptr(S0, "S0", 16, true));
  KDN_TRY(check_ptr(c0, "c0", 4, true));
  KDN_TRY(check_ptr(dS_L, "dS_L", 16, true));
  KDN_TRY(check_ptr(dc_L, "dc_L", 4, true));
  KDN_TRY(check_ptr(workspace, "workspace", 256, false));
  if (!(qn_scalar >= 0.f)) return fail(KDN_ERR_INVALID_ARG, "qn_scalar must be >= 0");
  const size_t need = kdn_backward_workspace_bytes(KDN_KALMAN_ISO, dims);
  if (workspace_bytes < need)
    return fail(KDN_ERR_INVALID_ARG, "workspace_bytes " + std::to_string(workspace_bytes) + " < required " +
                                         std::to_string(need));
  DeviceGuard guard;
  KDN_TRY(use_device_of(dS0, guard));
  cudaStream_t st = (cudaStream_t)stream;
  const size_t BH = (size_t)dims->B * dims->H, tok = BH * (size_t)dims->L;
  // the scalar side's arrays sit after the memory backward's part of the workspace
  kdn_dims dd = *dims;
  char* iso = reinterpret_cast<char*>(workspace) + kdn_backward_workspace_bytes(KDN_DELTA, &dd);
  kdn::IsoBwdArgs ia{};
  ia.k = k, ia.in_dtype = dims->in_dtype, ia.a = a, ia.r = r, ia.qn = qn, ia.qn_scalar = qn_scalar, ia.c0 = c0;
  ia.beta = reinterpret_cast<float*>(iso);
  ia.cprev = reinterpret_cast<float*>(iso + round256(tok * 4));
  ia.knorm2 = reinterpret_cast<float*>(iso + 2 * round256(tok * 4));
  float* dbeta = reinterpret_cast<float*>(iso + 3 * round256(tok * 4));
  ia.dbeta = dbeta, ia.dc_L = dc_L, ia.dk = dk, ia.da = da, ia.dr = dr, ia.dqn = dqn, ia.dc0 = dc0;
  ia.L = dims->L, ia.dk_dim = dims->dk;
  if (any) KDN_TRY(cuda_status(kdn::launch_iso_forward(ia, (int)BH, st), "isotropic backward: forward chain launch"));
  // the memory backward with beta_t as an input gives dq, dv, dS0, the key's memory terms, dbeta and the
  // decay terms of da; the uncertainty chain then adds its key and gate terms
  KDN_TRY(delta_backward_run(dims, q, k, v, ia.beta, a, S0, dO, dm, dS_L, dq, dk, dv, dbeta, da, dS0, workspace, st));
  if (!any) {
    if (dc_L != nullptr)
      return cuda_status(cudaMemcpyAsync(dc0, dc_L, BH * 4, cudaMemcpyDeviceToDevice, st), "dc0 of an empty sequence");
    return cuda_status(cudaMemsetAsync(dc0, 0, BH * 4, st), "dc0 of an empty sequence");
  }
  return cuda_status(kdn::launch_iso_backward(ia, (int)BH, st), "isotropic backward: uncertainty chain launch");
}

kdn_status kdn_scan_kalman_diag_backward(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                        const float* r, const float* a, const float* qn, float qn_scalar,
                                        const float* S0, const float* p0, const float* dO, const float* dm,
                                        const float* dS_L, const float* dp_L, float* dq, float* dk, float* dv,
                                        float* dr, float* da, float* dqn, float* dS0, float* dp0, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  KDN_TRY(check_dims(dims));
  const bool any = dims->L > 0;
  KDN_TRY(check_ptr(dS0, "dS0", 16, false));
  KDN_TRY(check_ptr(dp0, "dp0", 4, false));
  for (const auto& pr : {std::make_pair((const void*)q, "q"), std::make_pair((const void*)k, "k"),
                         std::make_pair((const void*)v, "v"), std::make_pair((const void*)dO, "dO"),
                         std::make_pair((const void*)dq, "dq"), std::make_pair((const void*)dk, "dk"),
                         std::make_pair((const void*)dv, "dv")})
    KDN_TRY(check_ptr(pr.first, pr.second, 16, !any));
  KDN_TRY(check_ptr(r, "r", 4, !any));
  KDN_TRY(check_ptr(dr, "dr", 4, !any));
  KDN_TRY(check_ptr(dqn, "dqn", 4, !any));
  KDN_TRY(check_ptr(a, "a", 4, true));
  KDN_TRY(check_ptr(da, "da", 4, true));
  KDN_TRY(check_ptr(qn, "qn", 4, true));
  KDN_TRY(check_ptr(dm, "dm", 4, true));
  KDN_TRY(check_ptr(S0, "S0", 16, true));
  KDN_TRY(check_ptr(p0, "p0", 4, true));
  KDN_TRY(check_ptr(dS_L, "dS_L", 16, true));
  KDN_TRY(check_ptr(dp_L, "dp_L", 4, true));
  KDN_TRY(check_ptr(workspace, "workspace", 256, false));
  if (!(qn_scalar >= 0.f)) return fail(KDN_ERR_INVALID_ARG, "qn_scalar must be >= 0");
  const size_t need = kdn_backward_workspace_bytes(KDN_KALMAN_DIAG, dims);
  if (workspace_bytes < need)
    return fail(KDN_ERR_INVALID_ARG, "workspace_bytes " + std::to_string(workspace_bytes) + " < required " +
                                         std::to_string(need));
  DeviceGuard guard;
  KDN_TRY(use_device_of(dS0, guard));
  cudaStream_t st = (cudaStream_t)stream;
  const size_t BH = (size_t)dims->B * dims->H, tok = BH * (size_t)dims->L;
  kdn_dims dd = *dims;
  char* side = reinterpret_cast<char*>(workspace) + kdn_backward_workspace_bytes(KDN_DELTA, &dd);
  kdn::DiagBwdArgs da_args{};
  da_args.k = k, da_args.in_dtype = dims->in_dtype, da_args.a = a, da_args.r = r, da_args.qn = qn;
  da_args.qn_scalar = qn_scalar, da_args.p0 = p0;
  da_args.gains = reinterpret_cast<float*>(side);
  da_args.pprev = reinterpret_cast<float*>(side + round256(tok * dims->dk * 4));
  float* dgain = reinterpret_cast<float*>(side + 2 * round256(tok * dims->dk * 4));
  da_args.dgain = dgain, da_args.dp_L = dp_L, da_args.dk = dk, da_args.da = da, da_args.dr = dr;
  da_args.dqn = dqn, da_args.dp0 = dp0, da_args.L = dims->L, da_args.dk_dim = dims->dk;
  if (any) KDN_TRY(cuda_status(kdn::launch_diag_forward(da_args, (int)BH, st), "diagonal backward: forward chain launch"));
  // the memory backward with the gains as inputs gives dq, dv, dS0, the key's memory terms, dG and the decay
  // terms of da; the uncertainty chain then adds its key and gate terms
  KDN_TRY(delta_backward_run(dims, q, k, v, nullptr, a, S0, dO, dm, dS_L, dq, dk, dv, nullptr, da, dS0, workspace, st,
                             da_args.gains, dgain));
  if (!any) {
    if (dp_L != nullptr)
      return cuda_status(cudaMemcpyAsync(dp0, dp_L, BH * dims->dk * 4, cudaMemcpyDeviceToDevice, st),
                         "dp0 of an empty sequence");
    return cuda_status(cudaMemsetAsync(dp0, 0, BH * dims->dk * 4, st), "dp0 of an empty sequence");
  }
  return cuda_status(kdn::launch_diag_backward(da_args, (int)BH, st), "diagonal backward: uncertainty chain launch");
}

kdn_status kdn_scan_kalman_full_backward(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                        const float* r, const float* a, const float* qn, float qn_scalar,
                                        const float* S0, const float* P0, const float* dO, const float* dm,
                                        const float* dS_L, const float* dP_L, float* dq, float* dk, float* dv,
                                        float* dr, float* da, float* dqn, float* dS0, float* dP0, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  KDN_TRY(check_dims(dims));
  const bool any = dims->L > 0;
  KDN_TRY(check_ptr(dS0, "dS0", 16, false));
  KDN_TRY(check_ptr(dP0, "dP0", 16, false));
  for (const auto& pr : {std::make_pair((const void*)q, "q"), std::make_pair((const void*)k, "k"),
                         std::make_pair((const void*)v, "v"), std::make_pair((const void*)dO, "dO"),
                         std::make_pair((const void*)dq, "dq"), std::make_pair((const void*)dk, "dk"),
                         std::make_pair((const void*)dv, "dv")})
    KDN_TRY(check_ptr(pr.first, pr.second, 16, !any));
  KDN_TRY(check_ptr(r, "r", 4, !any));
  KDN_TRY(check_ptr(dr, "dr", 4, !any));
  KDN_TRY(check_ptr(dqn, "dqn", 4, !any));
  KDN_TRY(check_ptr(a, "a", 4, true));
  KDN_TRY(check_ptr(da, "da", 4, true));
  KDN_TRY(check_ptr(qn, "qn", 4, true));
  KDN_TRY(check_ptr(dm, "dm", 4, true));
  KDN_TRY(check_ptr(S0, "S0", 16, true));
  KDN_TRY(check_ptr(P0, "P0", 16, true));
  KDN_TRY(check_ptr(dS_L, "dS_L", 16, true));
  KDN_TRY(check_ptr(dP_L, "dP_L", 16, true));
  KDN_TRY(check_ptr(workspace, "workspace", 256, false));
  if (!(qn_scalar >= 0.f)) return fail(KDN_ERR_INVALID_ARG, "qn_scalar must be >= 0");
  const size_t need = kdn_backward_workspace_bytes(KDN_KALMAN_FULL, dims);
  if (workspace_bytes < need)
    return fail(KDN_ERR_INVALID_ARG, "workspace_bytes " + std::to_string(workspace_bytes) + " < required " +
                                         std::to_string(need));
  DeviceGuard guard;
  KDN_TRY(use_device_of(dS0, guard));
  cudaStream_t st = (cudaStream_t)stream;
  const size_t BH = (size_t)dims->B * dims->H, tok = BH * (size_t)dims->L;
  kdn_dims dd = *dims;
  char* side = reinterpret_cast<char*>(workspace) + kdn_backward_workspace_bytes(KDN_DELTA, &dd);
  kdn::FullBwdArgs fa{};
  fa.k = k, fa.in_dtype = dims->in_dtype, fa.a = a, fa.r = r, fa.qn = qn, fa.qn_scalar = qn_scalar, fa.P0 = P0;
  fa.gains = reinterpret_cast<float*>(side);
  float* dgain = reinterpret_cast<float*>(side + round256(tok * dims->dk * 4));
  fa.dgain = dgain, fa.dP_L = dP_L, fa.dk = dk, fa.da = da, fa.dr = dr, fa.dqn = dqn, fa.dP0 = dP0;
  fa.status = reinterpret_cast<unsigned*>(workspace), fa.L = dims->L, fa.d = dims->dk;
  kdn::full_backward_bind_scratch(fa, side + 2 * round256(tok * dims->dk * 4), (int)BH);
  if (any)
    KDN_TRY(cuda_status(kdn::launch_full_cov_forward(fa, (int)BH, st), "full-Kalman backward: covariance forward launch"));
  // the memory backward with the gains as inputs (it clears the status word first) gives dq, dv, dS0, the key's
  // memory terms, dG and the decay terms of da; the covariance side then adds its key and gate terms and
  // writes dr, dQn and dP0 (for an empty sequence: dP0 = the symmetric part of dP_L)
  KDN_TRY(delta_backward_run(dims, q, k, v, nullptr, a, S0, dO, dm, dS_L, dq, dk, dv, nullptr, da, dS0, workspace, st,
                             fa.gains, dgain));
  return cuda_status(kdn::launch_full_cov_backward(fa, (int)BH, st), "full-Kalman backward: covariance chain launch");
}

size_t kdn_hola_workspace_bytes(const kdn_dims* dims) {
  if (dims == nullptr || dims->B < 1 || dims->H < 1 || dims->L < 0) return 0;
  const int block = dims->chunk == 0 ? 64 : dims->chunk;
  size_t n = kStatusBytes;
  if (kdn::hola_tc_supported(dims->dk, dims->dv, dims->in_dtype, block))  // every block's cache indices
    n += round256((size_t)dims->B * dims->H * ((dims->L + 63) / 64) * 64 * sizeof(int));
  return n;
}

kdn_status kdn_hola_cache_read(const kdn_dims* dims, const void* q, const void* k, const void* v, const float* m,
                               const float* gamma_q, const float* gamma_k, const float* sink, int w, float* o_cache,
                               int* cache_idx, void* workspace, size_t workspace_bytes, void* stream) {
  KDN_TRY(check_dims(dims));
  if (w < 1 || w > 64) return fail(KDN_ERR_UNSUPPORTED, "w must be in 1..64");
  const int block = dims->chunk == 0 ? 64 : dims->chunk;
  const bool any = dims->L > 0;
  KDN_TRY(check_ptr(q, "q", 16, !any));
  KDN_TRY(check_ptr(k, "k", 16, !any));
  KDN_TRY(check_ptr(v, "v", 16, !any));
  KDN_TRY(check_ptr(m, "m", 4, !any));
  KDN_TRY(check_ptr(o_cache, "o_cache", 16, !any));
  KDN_TRY(check_ptr(gamma_q, "gamma_q", 4, false));
  KDN_TRY(check_ptr(gamma_k, "gamma_k", 4, false));
  KDN_TRY(check_ptr(sink, "sink", 4, false));
  KDN_TRY(check_ptr(cache_idx, "cache_idx", 4, true));
  KDN_TRY(check_ptr(workspace, "workspace", 256, false));
  if (workspace_bytes < kStatusBytes) return fail(KDN_ERR_INVALID_ARG, "workspace_bytes < 256");
  DeviceGuard guard;
  KDN_TRY(use_device_of(gamma_q, guard));
  const int BH = dims->B * dims->H;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, st);
  if (e != cudaSuccess) return cuda_status(e, "clearing the status word");
  if (!any) {
    if (cache_idx == nullptr) return ok();
    return cuda_status(cudaMemsetAsync(cache_idx, 0xff, (size_t)BH * w * sizeof(int), st), "clearing cache_idx");
  }
  kdn::HolaArgs ha{q, k, v, dims->in_dtype, m, gamma_q, gamma_k, sink, o_cache, cache_idx, dims->H, dims->L, block, w,
                   reinterpret_cast<unsigned*>(workspace)};
  // with room for every block's cache indices, the tensor-core path reads all blocks at once
  if (kdn::hola_tc_supported(dims->dk, dims->dv, dims->in_dtype, block) &&
      workspace_bytes >= kdn_hola_workspace_bytes(dims))
    ha.cidx = reinterpret_cast<int*>(reinterpret_cast<char*>(workspace) + kStatusBytes);
  return cuda_status(kdn::launch_hola_read(dims->dk, dims->dv, ha, BH, st), "surprise-cache read launch");
}

kdn_status kdn_decode_step(kdn_variant variant, int B, int H, int dk, int dv, kdn_dtype in_dtype, kdn_dtype out_dtype,
                           const void* q, const void* k, const void* v, const float* beta, const float* a,
                           const float* r, float qn_scalar, float* S, float* p, void* o, float* m, void* stream) {
  if (variant != KDN_DELTA && variant != KDN_KALMAN_DIAG && variant != KDN_KALMAN_ISO)
    return fail(KDN_ERR_UNSUPPORTED, "decode supports KDN_DELTA, KDN_KALMAN_DIAG and KDN_KALMAN_ISO");
  kdn_dims d{B, H, 1, dk, dv, 0, in_dtype, out_dtype};
  KDN_TRY(check_dims(&d));
  KDN_TRY(check_ptr(q, "q", 16, false));
  KDN_TRY(check_ptr(k, "k", 16, false));
  KDN_TRY(check_ptr(v, "v", 16, false));
  KDN_TRY(check_ptr(S, "S", 16, false));
  KDN_TRY(check_ptr(o, "o", 16, false));
  KDN_TRY(check_ptr(m, "m", 4, true));
  KDN_TRY(check_ptr(a, "a", 4, true));
  if (variant == KDN_DELTA) {
    KDN_TRY(check_ptr(beta, "beta", 4, false));
  } else {
    KDN_TRY(check_ptr(r, "r", 4, false));
    KDN_TRY(check_ptr(p, "p", 4, false));
    if (!(qn_scalar >= 0.f)) return fail(KDN_ERR_INVALID_ARG, "qn_scalar must be >= 0");
  }
  DeviceGuard guard;
  KDN_TRY(use_device_of(S, guard));
  kdn::DecodeArgs args{q, k, v, in_dtype, out_dtype, beta, a, r, qn_scalar, S, p, o, m, B * H};
  const int mode = variant == KDN_KALMAN_DIAG ? 1 : variant == KDN_KALMAN_ISO ? 2 : 0;
  return cuda_status(kdn::launch_decode(dk, dv, mode, args, (cudaStream_t)stream), "decode launch");
}

}  // extern "C"
