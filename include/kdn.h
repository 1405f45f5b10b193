/*
 * kdn.h - C ABI of the B200 (sm_100a) forward scan of a recurrent
 * associative memory written by a gain-weighted residual.
 *
 * Per head (b, h) the memory is a matrix S (d_k x d_v, fp32) read as
 * o_t = S_t^T q_t.  Every entry point writes it token by token with
 *
 *     S_t = a_t S_{t-1} + g_t e_t^T,     e_t = v_t - (a_t S_{t-1})^T k_t,
 *
 * and emits the surprise score m_t = ||g_t|| ||e_t||, the Frobenius norm of
 * the write (A Hippocampus for Linear Attention, section 3.3, Eq. (5)-(6);
 * the decay gate and the residual against the decayed state: same page,
 * section 3.5 "Instantiation (GDN)").  The entry points differ in the gain:
 *
 *   kdn_scan_delta        g_t = beta_t k_t                    (gated delta rule)
 *   kdn_scan_kalman_full  g_t = P^- k_t / (k_t^T P^- k_t + r_t), with
 *                         P^- = a_t^2 P + Qn_t I and P <- P^- - s_t g_t g_t^T
 *                         (Kalman Delta Networks, Abstract; Memory by Design,
 *                         Abstract; DeltaNet-PC, "How it works", Eq. (5)-(7))
 *   kdn_scan_kalman_diag  the same with P = diag(p), p_i <- p^-_i r /
 *                         (r + p^-_i k_i^2): the one-step posterior projected on
 *                         diagonal Gaussians by mean-field VI (Kalman Delta
 *                         Networks, Abstract)
 *   kdn_decode_step       one token against a resident state (delta or diag)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.  Every array argument is a DEVICE pointer (cudaMalloc, a CUDA
 *   caching allocator, or managed memory) to a dense row-major array.  q, k,
 *   v, o, S and P must be 16-byte aligned, the workspace 256-byte aligned, and
 *   the fp32 per-token arrays (beta, a, r, qn, m) and p 4-byte aligned.  Host
 *   pointers are rejected with KDN_ERR_INVALID_ARG.
 * Ownership.  The caller owns every buffer; the library allocates nothing and
 *   keeps no pointer after the call returns.  Scratch space is the caller's
 *   workspace, sized by kdn_workspace_bytes().
 * Layouts (B batch, H heads, L tokens):
 *   q, k      [B, H, L, d_k]   in_dtype (bf16 or fp32); keys are expected
 *                               unit-L2 (HOLA section 3.4) but not required
 *   v         [B, H, L, d_v]   in_dtype
 *   o         [B, H, L, d_v]   out_dtype
 *   m         [B, H, L]        fp32, may be NULL (not written)
 *   beta, a, r, qn [B, H, L]   fp32; a == NULL means a_t = 1; qn == NULL means
 *                               Qn_t = qn_scalar for every token
 *   S         [B, H, d_k, d_v] fp32, in: initial state, out: state after token L
 *   P         [B, H, d_k, d_k] fp32 symmetric PD, in: P_0, out: P_L
 *   p         [B, H, d_k]      fp32 positive, in: p_0, out: p_L
 *   States are updated in place, so consecutive calls continue one scan.
 * Streams.  ``stream`` is a cudaStream_t (NULL = legacy default stream).
 *   Every call only enqueues work on it and returns; nothing synchronises.
 * Devices.  A call launches on the device that owns its state buffer and
 *   restores the calling thread's current device before it returns.
 * Errors.  Argument errors return synchronously and enqueue nothing.  A failed
 *   launch returns KDN_ERR_CUDA.  Numeric failures found on the device (a
 *   non-positive or non-finite innovation variance) set the status word in
 *   the workspace, read back with kdn_read_device_status().  Nothing in the
 *   library aborts, exits or traps.  kdn_last_error() gives a message for the
 *   last failing call on the calling thread.
 * Supported sizes.  d_k, d_v in {16, 32, 64, 128}; any L >= 0 (L = 0 is a
 *   no-op); chunk 0 (library choice) or 16/32/64.
 * Precision.  State, gains and accumulation are fp32.  Where a product runs
 *   on the tensor cores, bf16 inputs enter it exactly and every fp32 operand
 *   (the state, the gains, the chunk solves) is split into two bf16 terms
 *   (hi + lo), keeping about 16 mantissa bits.
 */
#ifndef KDN_H_
#define KDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDN_API_VERSION 2

#if defined(__GNUC__)
#define KDN_EXPORT __attribute__((visibility("default")))
#else
#define KDN_EXPORT
#endif

typedef enum kdn_status {
  KDN_OK = 0,
  KDN_ERR_INVALID_ARG = 1,  /* null / host / misaligned pointer, bad size or dtype */
  KDN_ERR_UNSUPPORTED = 2,  /* valid request outside the supported sizes */
  KDN_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  KDN_ERR_NUMERIC = 4,      /* device status: non-positive / non-finite innovation variance */
  KDN_ERR_TIMEOUT = 5       /* device status: a bounded wait gave up */
} kdn_status;

typedef enum kdn_dtype { KDN_F32 = 0, KDN_BF16 = 1 } kdn_dtype;

typedef enum kdn_variant { KDN_DELTA = 0, KDN_KALMAN_DIAG = 1, KDN_KALMAN_FULL = 2, KDN_KALMAN_ISO = 3 } kdn_variant;

typedef struct kdn_dims {
  int B, H, L;          /* batch, heads, tokens */
  int dk, dv;           /* key and value head dimensions */
  int chunk;            /* 0 = library choice; else 16, 32 or 64 tokens per chunk */
  kdn_dtype in_dtype;   /* dtype of q, k, v */
  kdn_dtype out_dtype;  /* dtype of o */
  int segments;         /* sequence segments per head scanned in parallel:
                         * 0 = library choice, 1 = one serial pass per head, P >= 2 = P segments
                         * (L % P == 0; chunked path only, else KDN_ERR_UNSUPPORTED).  See below. */
} kdn_dims;

/* Segment-parallel scans.  With few heads (B*H well below the GPU's 148 SMs) one CTA per head leaves
 * most of the GPU idle, and the chunk loop is serial.  The scan functions then cut each head's sequence
 * into P equal segments (Kalman Delta Networks, Abstract: the uncertainty recurrences of the diagonal
 * and isotropic variants are Moebius maps and compose associatively; for fixed gains the memory scan is
 * affine in its start state):
 *   - diagonal Kalman: each segment composes its per-coordinate uncertainty maps, and the maps are
 *     chained to get p at every segment start; isotropic: the one-scalar beta prologue runs first;
 *     full Kalman: the covariance side runs over the whole sequence first (it is not a per-coordinate
 *     map), giving every token's gain;
 *   - the chunk kernel runs all segments from S0 = 0 and from S0 = I (giving each segment's map
 *     S0 -> M S0 + B; at d = 64 one run on the d x 2d state [S | M] from [0 | I] gives both), one fp32
 *     pass per head chains the segment start states, and a last chunk-kernel run from the true start
 *     states writes o, m and the final state.
 * Results equal the serial scan's up to rounding.  The library choice (segments = 0) is P in {16, 8, 4}
 * (the largest with B*H*P <= 148, L % (64 P) == 0 and at least two chunks per segment), else 1.  The
 * workspace grows by 3 B*H*P*dk*dv floats (plus 7 B*H*P*dk for the diagonal variant) when P > 1. */

/* Gated delta rule scan (A Hippocampus for Linear Attention, section 3.3
 * Eq. (5)-(6), section 3.5).  beta: write strengths, required.  a: decay gates
 * in (0, 1] or NULL.  S: state in/out.  o, m: outputs. */
KDN_EXPORT kdn_status kdn_scan_delta(const kdn_dims* dims, const void* q, const void* k, const void* v,
                          const float* beta, const float* a, float* S, void* o, float* m,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Full-covariance Kalman / RLS scan (Kalman Delta Networks, Abstract; Memory
 * by Design, Abstract; DeltaNet-PC, Eq. (5)-(7)).  Per token: propagate
 * S^- = a S, P^- = a^2 P + Qn I, then update with the Kalman gain.  r: observation
 * noise variances (> 0), required.  P: covariance in/out, symmetric PD. */
KDN_EXPORT kdn_status kdn_scan_kalman_full(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                const float* a, const float* r, const float* qn, float qn_scalar,
                                float* S, float* P, void* o, float* m,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Diagonal-covariance Kalman scan (Kalman Delta Networks, Abstract: mean-field
 * projection on diagonal Gaussians).  p: diagonal of P in/out, positive. */
KDN_EXPORT kdn_status kdn_scan_kalman_diag(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                const float* a, const float* r, const float* qn, float qn_scalar,
                                float* S, float* p, void* o, float* m,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Isotropic-covariance Kalman scan (Kalman Delta Networks, Abstract: Isotropic
 * KDN keeps a single uncertainty scalar per head; its recurrence is a Moebius
 * map, scanned associatively).  Per token: c^- = a^2 c + Qn, gain
 * c^- k / (c^- ||k||^2 + r) (the delta rule's write with that beta), and the
 * isotropic mean-field variance c = d_k c^- r / (d_k r + c^- ||k||^2).
 * c: [B,H] uncertainty in/out, positive.  Other arguments as for
 * kdn_scan_kalman_diag.  The workspace also holds the per-token beta
 * ([B,H,L] fp32 after the status word). */
KDN_EXPORT kdn_status kdn_scan_kalman_iso(const kdn_dims* dims, const void* q, const void* k, const void* v,
                               const float* a, const float* r, const float* qn, float qn_scalar,
                               float* S, float* c, void* o, float* m,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Backward pass of the gated delta rule scan (the adjoint of kdn_scan_delta for
 * training; A Hippocampus for Linear Attention, section 4, and Kalman Delta
 * Networks, Abstract, train these layers end to end; the pages print no
 * backward).  Given the forward inputs and the upstream gradients of a scalar
 * loss, returns its gradients with respect to every input of the scan:
 *   in   q, k [B,H,L,d_k], v [B,H,L,d_v] (dims->in_dtype); beta, a [B,H,L]
 *        fp32 (a NULL = 1); S0 [B,H,d_k,d_v] fp32, the state the forward started
 *        from (NULL = 0; not modified);
 *        dO [B,H,L,d_v] fp32 = dLoss/do; dm [B,H,L] fp32 = dLoss/dm or NULL;
 *        dS_L [B,H,d_k,d_v] fp32 = dLoss/dS_L or NULL
 *   out  dq, dk [B,H,L,d_k], dv [B,H,L,d_v], dbeta [B,H,L], da [B,H,L] (or
 *        NULL; with a NULL it is the gradient at a = 1), dS0 [B,H,d_k,d_v]:
 *        all fp32, overwritten.
 * The surprise m_t = beta_t ||k_t|| ||e_t|| has no gradient where e_t = 0 or
 * k_t = 0 (the one-sided value 0 is taken).  A gate a_t = 0 is allowed.
 * Method: the forward is run again, keeping the state at every 32-token
 * chunk start and ||e_t||, in the workspace; then the chunks are walked
 * backwards with the state adjoint, every step a product of 32 x 32, 32 x d
 * or d x d blocks on the fp32 CUDA cores (one CTA per head and block of 32
 * value columns).  workspace: kdn_backward_workspace_bytes(KDN_DELTA, dims)
 * bytes (256-byte status word, the states, the norms).  dims->chunk and
 * dims->out_dtype are ignored.  Asynchronous on ``stream``. */
KDN_EXPORT kdn_status kdn_scan_delta_backward(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                              const float* beta, const float* a, const float* S0, const float* dO,
                                              const float* dm, const float* dS_L, float* dq, float* dk, float* dv,
                                              float* dbeta, float* da, float* dS0, void* workspace,
                                              size_t workspace_bytes, void* stream);

/* Backward of the isotropic Kalman scan (Kalman Delta Networks, Abstract:
 * Isotropic KDN, one uncertainty scalar per head; the layers are trained end to
 * end).  The forward is kdn_scan_kalman_iso's: c^- = a^2 c + Qn, the delta-rule
 * write with beta_t = c^- / (c^- ||k_t||^2 + r_t), c = d_k c^- r / (d_k r +
 * c^- ||k_t||^2).  For upstream dO (and optional dm, dS_L, dc_L [B,H]) it gives
 * dq, dk, dv [B,H,L,d] fp32, dr, dqn [B,H,L] (dqn per token: its sum is the
 * gradient of a scalar Qn), da [B,H,L] (optional), dS0 [B,H,d_k,d_v] and dc0
 * [B,H].  r [B,H,L]; a, qn (else qn_scalar), S0 (else 0), c0 (else 1)
 * optional.  Runs the uncertainty chain forward (one warp per head), the
 * gated-delta backward with that beta (kdn_scan_delta_backward's kernels), and
 * the uncertainty chain backwards, which adds its key and gate terms.
 * workspace: kdn_backward_workspace_bytes(KDN_KALMAN_ISO, dims) bytes.
 * Asynchronous on ``stream``. */
KDN_EXPORT kdn_status kdn_scan_kalman_iso_backward(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                                   const float* r, const float* a, const float* qn, float qn_scalar,
                                                   const float* S0, const float* c0, const float* dO, const float* dm,
                                                   const float* dS_L, const float* dc_L, float* dq, float* dk,
                                                   float* dv, float* dr, float* da, float* dqn, float* dS0,
                                                   float* dc0, void* workspace, size_t workspace_bytes, void* stream);

/* Backward of the diagonal-Kalman scan (Kalman Delta Networks, Abstract:
 * mean-field variational Kalman with a diagonal covariance; the layers are
 * trained end to end).  The forward is kdn_scan_kalman_diag's: p^- = a^2 p + Qn,
 * s = sum_i p^-_i k_i^2 + r, gain g = p^- o k / s, p = p^- r / (r + p^- o k^2)
 * per coordinate, the delta-rule memory write with that gain.  Same inputs and
 * outputs as kdn_scan_kalman_iso_backward with p0, dp_L, dp0 [B,H,d_k] in place
 * of c0, dc_L, dc0.  Runs the variance chain forward (one warp per head,
 * storing the gains and the variances), the memory backward with the gains as
 * inputs (its kernels write dG), and the variance chain backwards, which adds
 * its key and gate terms.  workspace: kdn_backward_workspace_bytes(
 * KDN_KALMAN_DIAG, dims) bytes.  Asynchronous on ``stream``. */
KDN_EXPORT kdn_status kdn_scan_kalman_diag_backward(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                                    const float* r, const float* a, const float* qn, float qn_scalar,
                                                    const float* S0, const float* p0, const float* dO, const float* dm,
                                                    const float* dS_L, const float* dp_L, float* dq, float* dk,
                                                    float* dv, float* dr, float* da, float* dqn, float* dS0,
                                                    float* dp0, void* workspace, size_t workspace_bytes, void* stream);

/* Backward of the full-covariance Kalman scan (Kalman Delta Networks, Abstract:
 * the dense Riccati recursion of the memory's uncertainty; the layers are
 * trained end to end).  The forward is kdn_scan_kalman_full's: P^- = a^2 P +
 * Qn I, u = P^- k, s = k^T u + r, gain g = u / s, P = P^- - u u^T / s, the
 * delta-rule memory write with that gain.  Same inputs and outputs as
 * kdn_scan_kalman_diag_backward with P0 (NULL = I), dP_L (NULL = 0) and dP0
 * [B,H,d_k,d_k] fp32 in place of p0, dp_L, dp0.  P0 must be symmetric, as the
 * forward requires; dP0 is the gradient with respect to a symmetric P0, i.e.
 * the symmetric part of the entrywise derivative (for an empty sequence the
 * symmetric part of dP_L).  Runs the covariance chain forward (one CTA of 4 d_k
 * threads per head, storing the gains and P at every 32-token block start),
 * the memory backward with the gains as inputs (its kernels write dG), and the
 * covariance chain backwards (each block's P recomputed from its checkpoint,
 * the adjoint carried as its symmetric sum), which adds its key and gate terms.
 * A non-positive or non-finite s raises KDN_ERR_NUMERIC in the status word.
 * workspace: kdn_backward_workspace_bytes(KDN_KALMAN_FULL, dims) bytes.
 * Asynchronous on ``stream``. */
KDN_EXPORT kdn_status kdn_scan_kalman_full_backward(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                                    const float* r, const float* a, const float* qn, float qn_scalar,
                                                    const float* S0, const float* P0, const float* dO, const float* dm,
                                                    const float* dS_L, const float* dP_L, float* dq, float* dk,
                                                    float* dv, float* dr, float* da, float* dqn, float* dS0,
                                                    float* dP0, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace the backward entry points need (KDN_DELTA,
 * KDN_KALMAN_ISO, KDN_KALMAN_DIAG or KDN_KALMAN_FULL; 0 for invalid dims). */
KDN_EXPORT size_t kdn_backward_workspace_bytes(kdn_variant variant, const kdn_dims* dims);

/* Surprise-cache read (A Hippocampus for Linear Attention, sections 3.3-3.4,
 * Eq. (6)-(7)).  Each head keeps the exact (k, v) of the w tokens with the
 * largest surprise m seen so far (ties: the earlier token); token t of block b
 * (dims->chunk tokens per block: 16, 32 or 64; 0 = 64) reads with a softmax,
 * temperature 1, over the cache of blocks 0..b-1, the tokens of its own block
 * up to t, and a null sink (logit sink[h], no value):
 *   o_t = sum_j softmax_j(q~_t . k~_j / sqrt(d_k)) v_j,
 *   q~ = RMSNorm(q) * gamma_q, k~ = RMSNorm(k) * gamma_k (eps 1e-6).
 * q, k [B,H,L,d_k], v [B,H,L,d_v] (dims->in_dtype); m [B,H,L] fp32 (finite;
 * the m of a scan); gamma_q, gamma_k [d_k] shared by the heads; sink [H];
 * 1 <= w <= 64.  Out: o_cache [B,H,L,d_v] fp32; cache_idx [B,H,w] int32 token
 * indices of the final cache, ascending, -1 for empty slots, or NULL.  The
 * state-read gate that mixes o_cache into the layer output is the caller's.
 * workspace: >= 256 bytes (the device status word, read with
 * kdn_read_device_status).  For bf16 q, k, v with d_k = d_v = 128 and blocks of
 * 64, a workspace of kdn_hola_workspace_bytes(dims) also holds the cache
 * indices of every block: the cache each block reads is chosen first (from m
 * alone: up to 192 blocks by a log-depth scan of the blocks' ranked top-w
 * lists, beyond that by one pass over the blocks per head), then all blocks
 * are read at once; with 256 bytes one CTA per head walks the blocks in order.
 * All give the same caches; m must not hold NaN. */
KDN_EXPORT kdn_status kdn_hola_cache_read(const kdn_dims* dims, const void* q, const void* k, const void* v,
                               const float* m, const float* gamma_q, const float* gamma_k, const float* sink,
                               int w, float* o_cache, int* cache_idx, void* workspace, size_t workspace_bytes,
                               void* stream);

/* Bytes of device workspace for kdn_hola_cache_read's parallel form (256 for
 * the status word, plus B*H*ceil(L/64)*64 int32 cache indices where the
 * tensor-core path applies); 0 for invalid dims.  Pure host call. */
KDN_EXPORT size_t kdn_hola_workspace_bytes(const kdn_dims* dims);

/* kdn_scan_kalman_full for callers that cannot allocate device memory.  The
 * pages have no counterpart: this is a deployment variant.  Callers that must
 * not call cudaMalloc while running (a server that reserves all device memory
 * at start-up, a plugin whose host framework owns the device allocator, a
 * real-time loop that forbids allocation) and have no buffer to spare for
 * the workspace use this instead.  Same arguments, layouts and results as
 * kdn_scan_kalman_full, minus the workspace; the library allocates nothing.
 *   Scratch: a static device array inside the library (256-byte status word
 *   plus 16 MiB of per-token gains), which every GPU that loads the library
 *   holds until the process exits.  Limit: B*H*L*d_k <= 4,194,304; larger
 *   requests return KDN_ERR_UNSUPPORTED (kdn_last_error() says why) and
 *   enqueue nothing.
 *   Set-up: on each device the array is reserved when the library's module
 *   that holds it is loaded, which under CUDA's lazy module loading (the
 *   default) is the first no-alloc call there, not library load.  A caller
 *   that reserves device memory at start-up should make that first call
 *   before it does (an L = 0 call with valid S and P is enough: it enqueues
 *   only the status-word clear), and before any stream capture.  Each call
 *   looks the array's device address up again (cudaGetSymbolAddress, with
 *   the state's device current), so a device reset leaves no stale address.
 *   Sharing: every call, on every stream, uses the same array and leaves its
 *   last contents behind (the status word is cleared at the start of each
 *   call).  Calls whose GPU work overlaps race on it: serialise them.
 *   Status: kdn_read_device_status(NULL, ...) reads this entry point's
 *   device status word (timeouts, non-positive innovation variances) on the
 *   calling thread's current device. */
KDN_EXPORT kdn_status kdn_scan_kalman_full_noalloc(const kdn_dims* dims, const void* q, const void* k, const void* v,
                                                   const float* a, const float* r, const float* qn, float qn_scalar,
                                                   float* S, float* P, void* o, float* m, void* stream);

/* One recurrent token per head against a resident state (constant-memory
 * decoding: Kalman Delta Networks, Abstract).  variant: KDN_DELTA (beta
 * required, p ignored), KDN_KALMAN_DIAG (r and p [B,H,d_k] required) or
 * KDN_KALMAN_ISO (r required; p is the uncertainty scalar c, [B,H]).  q, k
 * [B,H,d_k], v [B,H,d_v], scalars [B,H], o [B,H,d_v], m [B,H] or NULL;
 * S [B,H,d_k,d_v] and p in/out.  Needs no workspace. */
KDN_EXPORT kdn_status kdn_decode_step(kdn_variant variant, int B, int H, int dk, int dv, kdn_dtype in_dtype,
                           kdn_dtype out_dtype, const void* q, const void* k, const void* v,
                           const float* beta, const float* a, const float* r, float qn_scalar,
                           float* S, float* p, void* o, float* m, void* stream);

/* Bytes of device workspace a scan with these dims needs (always >= 256: the
 * first 256 bytes hold the device status word).  Returns 0 for invalid dims. */
KDN_EXPORT size_t kdn_workspace_bytes(kdn_variant variant, const kdn_dims* dims);

/* Synchronises ``stream``, then reads the device status word of ``workspace``
 * into *status_out (a kdn_status value: KDN_OK, KDN_ERR_NUMERIC or
 * KDN_ERR_TIMEOUT).  Each scan clears the word when it is enqueued.
 * workspace == NULL reads the word of kdn_scan_kalman_full_noalloc, kept in
 * its static array on the calling thread's current device. */
KDN_EXPORT kdn_status kdn_read_device_status(const void* workspace, int* status_out, void* stream);

/* Failure-path self-test (no counterpart on the pages: it checks the
 * library's own failure detection).  Every wait of the tensor-core kernels
 * is bounded: on expiry the kernel sets KDN_ERR_TIMEOUT in the status word,
 * frees its tensor memory and returns.  This launches one small kernel that
 * takes that path on purpose: it waits on an mbarrier nothing arrives at
 * (no copy or MMA in flight) for ``wait_cycles`` SM clocks (1 .. 2e9, about
 * one second at most), then aborts exactly as the scans do.  Afterwards
 * kdn_read_device_status(workspace, ...) reports KDN_ERR_TIMEOUT.
 * workspace: >= 256 bytes, 256-byte aligned, or NULL for the no-alloc entry
 * point's status word on the current device.  Asynchronous on ``stream``. */
KDN_EXPORT kdn_status kdn_selftest_wait_timeout(void* workspace, long long wait_cycles, void* stream);

/* Which kernels a scan with these dims runs: *launches = kernel launches per
 * call (the status-word clear, a 256-byte memset, not counted), *kernel = name
 * of the kernel that takes most of the time, *arith = arithmetic of that
 * kernel ("bf16-tc" for tensor-core products with fp32 accumulation, "f32"
 * for fp32 CUDA-core arithmetic).  Strings are static.  Pure host call. */
KDN_EXPORT kdn_status kdn_plan(kdn_variant variant, const kdn_dims* dims, int* launches, const char** kernel,
                               const char** arith);

/* Static string for a status code. */
KDN_EXPORT const char* kdn_status_string(kdn_status status);

/* Message for the last failing call on the calling thread ("" if none). */
KDN_EXPORT const char* kdn_last_error(void);

/* KDN_API_VERSION of the loaded library. */
KDN_EXPORT int kdn_api_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDN_H_ */
