/*
 * kdn.h -- C ABI of libkdn, the B200 (sm_100a) Kalman Delta Network layer.
 *
 * The model (from "Kalman Delta Networks: Uncertainty-aware Associative
 * Memory", abstract, and "Kalman Delta Networks: 不确定性感知的联想记忆",
 * 方法): per batch element b and head h the memory S (d_v x d_k) is the
 * latent state of a linear-Gaussian model, S_t = a_t S_{t-1} + noise(w_t)
 * and v_t = S_t k_t + noise(r_t).  Each token predicts, then writes the
 * residual v_t - a_t S_{t-1} k_t with the Kalman gain g_t, then reads
 * o_t = S_t q_t.  The uncertainty is one variance per head (Isotropic KDN)
 * or per key dimension (Diagonal KDN); both follow the Mobius map
 *     p_t = (r a^2 p_{t-1} + r w) / (c a^2 p_{t-1} + r + c w)
 * with c = info_scale * ||k_t||^2 (iso) or c = k_{t,i}^2 (diag).
 *
 * Conventions for every call:
 *   - Pointers are caller-owned.  Device pointers unless stated otherwise
 *     (CUDA device memory of the current device, e.g. PyTorch tensors).  The
 *     library never allocates device memory; calls that need scratch take a
 *     caller-provided workspace whose size the matching *_workspace_size()
 *     returns.
 *   - All arrays are dense, row-major, with the last index fastest.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call only enqueues work on it and never synchronises the host,
 *     except kdn_read_workspace_status().
 *   - Arguments are checked before anything is enqueued.  A call that returns
 *     anything but KDN_OK has enqueued nothing.  No C++ exception crosses
 *     this interface.
 *   - Floating-point state (a, w, r, S, p, o) is always fp32.  q, k, v are
 *     fp32 or bf16 (in_dtype).  The output o is fp32: the bf16 rounding of an
 *     exact output alone exceeds the layer's error bound (max-abs / RMS
 *     <= 2e-2) for outputs whose max is ~10x their RMS.
 */
#ifndef KDN_H_
#define KDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kdn_status {
  KDN_OK = 0,
  KDN_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, bad size or enum  */
  KDN_ERR_UNSUPPORTED = 2,  /* valid but not implemented (shape, path)      */
  KDN_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required   */
  KDN_ERR_TIMEOUT = 4,      /* a bounded on-device wait gave up             */
  KDN_ERR_CUDA = 5          /* the CUDA runtime reported an error           */
} kdn_status;

typedef enum kdn_dtype { KDN_F32 = 0, KDN_BF16 = 1 } kdn_dtype;
typedef enum kdn_variant { KDN_ISO = 0, KDN_DIAG = 1 } kdn_variant;

/* Forward-path selector (the `chunk` argument of the forward calls). */
enum {
  KDN_CHUNK_AUTO = 0,       /* chunked engine when supported, else recurrent */
  KDN_CHUNK_RECURRENT = 1,  /* token-by-token kernel, any supported shape    */
  KDN_CHUNK_64 = 64         /* chunkwise tensor-core engine, 64-token chunks */
};

/* Human-readable name of a status code (static storage, never NULL). */
const char* kdn_status_string(kdn_status status);

/* Library version, major*10000 + minor*100 + patch (0.2.0: adds the packed,
 * host-buffer, backward, dense-filter and KLA entry points). */
int kdn_version(void);

/* ------------------------------------------------------------------------
 * kdn_mobius_scan -- the uncertainty recursion alone, over N independent
 * lanes of length T ("Kalman Delta Networks: Uncertainty-aware Associative
 * Memory", abstract: the variance recursions are Mobius maps composed by an
 * associative scan; "Kalman Linear Attention ...", 方法论 §2 prints the
 * fractional-linear form).  For every lane i and step t:
 *     c          = info_scale * n[i,t]
 *     prior[i,t] = a^2 lambda[i,t-1] + w
 *     lambda[i,t]= (r a^2 lambda[i,t-1] + r w) / (c a^2 lambda[i,t-1] + r + c w)
 *     gain[i,t]  = prior / (prior * n + r)     (the isotropic write strength)
 * with lambda[i,-1] = lambda0[i] (or 1 when lambda0 is NULL).
 *
 * a, w, r, n     [N, T] fp32 device; n is the squared key norm (or k_i^2)
 * lambda0        [N] fp32 device, or NULL for all ones
 * info_scale     c = info_scale * n; must be finite and >= 0
 * lambda_out     [N, T] fp32 device, posterior variances (required)
 * prior_out      [N, T] fp32 device or NULL
 * gain_out       [N, T] fp32 device or NULL
 * workspace      device scratch of >= kdn_mobius_scan_workspace_size(N, T)
 *                bytes, 256-byte aligned; its contents are overwritten
 *                (the call clears what it needs on the stream first)
 * Requires a, w, r, n, lambda_out (and prior_out / gain_out when given) to be
 * 16-byte aligned; any T >= 1 and N >= 1 with N*T < 2^40.
 * Errors: KDN_ERR_INVALID_ARG, KDN_ERR_WORKSPACE, KDN_ERR_CUDA.  A look-back
 * wait that gives up (it cannot in correct use) is recorded in the workspace
 * and reported by kdn_read_workspace_status().
 * ---------------------------------------------------------------------- */
size_t kdn_mobius_scan_workspace_size(int64_t N, int64_t T);
kdn_status kdn_mobius_scan(const float* a, const float* w, const float* r,
                           const float* n, const float* lambda0,
                           float info_scale, float* lambda_out,
                           float* prior_out, float* gain_out, int64_t N,
                           int64_t T, void* workspace, size_t workspace_bytes,
                           void* stream);

/* ------------------------------------------------------------------------
 * kdn_mobius_scan_noalloc -- kdn_mobius_scan without a workspace argument,
 * for callers that cannot allocate device memory where they call the scan
 * (for example a host program that gives all device memory to its own pool
 * at start-up and permits no cudaMalloc afterwards, or a plug-in that such a
 * host hands only its input and output buffers).  The pages have no
 * counterpart of this entry point; it only changes where scratch lives.
 *
 * The scratch is a fixed array of about 7.9 MiB inside the library's device
 * code.  Every GPU that loads the library holds it until the process exits.
 * Limit: N * ceil(T / 2048) <= KDN_SCAN_NOALLOC_MAX_TILES (e.g. 4096 lanes
 * up to T = 114688); larger calls return KDN_ERR_WORKSPACE without enqueuing
 * anything.  The call allocates nothing.  Every call looks up the array's
 * device address in the caller's current device and context (the lookup
 * allocates nothing), so the address stays right across context switches
 * and device resets.  The first call in a context also loads the library's
 * device code there: make that first call before any stream capture.  Every
 * call clears the part of the array that must start at zero on `stream`
 * before its kernel.  All calls share the one array: calls whose work
 * overlaps on the GPU (for example on two streams without ordering between
 * them) race and give wrong results, so order them.  A look-back wait that
 * gives up (after 1 s, which only a stalled GPU reaches) is recorded only in
 * that internal array and is not reported by this entry point; callers that
 * must detect it use kdn_mobius_scan with a workspace and
 * kdn_read_workspace_status.  Otherwise the arguments, results and errors
 * are those of kdn_mobius_scan.
 * ---------------------------------------------------------------------- */
#define KDN_SCAN_NOALLOC_MAX_TILES 229376
kdn_status kdn_mobius_scan_noalloc(const float* a, const float* w,
                                   const float* r, const float* n,
                                   const float* lambda0, float info_scale,
                                   float* lambda_out, float* prior_out,
                                   float* gain_out, int64_t N, int64_t T,
                                   void* stream);

/* ------------------------------------------------------------------------
 * kdn_iso_forward -- Isotropic KDN layer forward ("Kalman Delta Networks:
 * Uncertainty-aware Associative Memory", abstract: one uncertainty scalar
 * per head; "Kalman Delta Networks: 不确定性感知的联想记忆", 方法 — 关键模块
 * steps 1-3 and 输出与差异点).  Per (b, h) and token t:
 *     n = ||k_t||^2;  p- = a^2 p + w;  beta = p- / (p- n + r)
 *     p = 1 / (1/p- + info_scale * n / r)
 *     S = a S + (v_t - a S k_t) (beta k_t)';   o_t = S q_t
 *
 * q, k     [B, T, H, dk] in_dtype device
 * v        [B, T, H, dv] in_dtype device
 * a, w, r  [B, T, H] fp32 device (decay in (0,1], process-noise variance
 *          >= 0, observation-noise variance > 0)
 * S0       [B, H, dv, dk] fp32 device initial memory, or NULL for zeros
 * p0       [B, H] fp32 device initial variance, or NULL for ones
 * o        [B, T, H, dv] fp32 device output
 * S_out    [B, H, dv, dk] fp32 device final memory (may alias S0)
 * p_out    [B, H] fp32 device final variance (may alias p0)
 * info_scale  kappa; <= 0 selects 1/dk
 * chunk    KDN_CHUNK_AUTO, KDN_CHUNK_RECURRENT or KDN_CHUNK_64
 * workspace   device scratch of >= kdn_forward_workspace_size(...) bytes,
 *             256-byte aligned (NULL allowed when that size is 0).  The
 *             chunked path keeps its device error word and a copy of p0
 *             there; kdn_read_workspace_status() reads the error word.
 *             The size depends on B, T, H and the current device: few heads
 *             over a long sequence take the segmented forward below, whose
 *             scratch (per segment: a state transition, a state and the
 *             start variances) is much larger, so query the size with the
 *             device that will run the call current.
 * Segmented forward: with dk = dv = 128 on the chunked path, when B H is at
 * most a quarter of the SM count and T is a multiple of 2048 (the segment
 * count S, a power of two >= 4 with B H S <= SMs and 512 S dividing T, is
 * chosen by the library), the sequence is cut into S segments run as extra
 * heads of the engine: the variance at each segment start from the composed
 * Mobius maps, each segment's state transition from a run with V = 0 and
 * S0 = I and its zero-start state and outputs from a run with S0 = 0, the
 * segment starts chained, and the outputs corrected by the segment start
 * state times the transition run's outputs (a tf32 tensor-core product).
 * The memory recursion is affine in the state, so the result is the same up
 * to rounding; it takes two engine passes over T / S tokens each instead of
 * one over T, and a workspace the size of o.
 * Supported: T >= 1; dk in {32, 64, 128}; 1 <= dv <= 128.  KDN_CHUNK_64
 * additionally needs in_dtype == KDN_BF16, dk == 128 and dv in {64, 128}.
 * All pointers 16-byte aligned.  o must not alias the inputs.
 * Errors: KDN_ERR_INVALID_ARG, KDN_ERR_UNSUPPORTED, KDN_ERR_WORKSPACE,
 * KDN_ERR_CUDA.
 * ---------------------------------------------------------------------- */
size_t kdn_forward_workspace_size(kdn_variant variant, int B, int T, int H,
                                  int dk, int dv, int chunk);
kdn_status kdn_iso_forward(const void* q, const void* k, const void* v,
                           kdn_dtype in_dtype, const float* a, const float* w,
                           const float* r, const float* S0, const float* p0,
                           float* o, float* S_out, float* p_out, int B, int T,
                           int H, int dk, int dv, float info_scale, int chunk,
                           void* workspace, size_t workspace_bytes,
                           void* stream);

/* ------------------------------------------------------------------------
 * kdn_diag_forward -- Diagonal KDN layer forward ("Kalman Delta Networks:
 * Uncertainty-aware Associative Memory", abstract: online mean-field
 * variational projection onto diagonal Gaussians).  Per (b, h), token t and
 * key dimension i:
 *     p-_i = a^2 p_i + w_i;   s = sum_i p-_i k_i^2 + r;   g = p- * k / s
 *     p_i  = 1 / (1/p-_i + k_i^2 / r)
 *     S = a S + (v_t - a S k_t) g';   o_t = S q_t
 * Arguments as kdn_iso_forward except:
 * w        [B, T, H, dk] fp32 device (per-dimension process noise)
 * p0, p_out  [B, H, dk] fp32 device (NULL p0 = ones)
 * (no info_scale: the diagonal projection has none)
 * ---------------------------------------------------------------------- */
kdn_status kdn_diag_forward(const void* q, const void* k, const void* v,
                            kdn_dtype in_dtype, const float* a, const float* w,
                            const float* r, const float* S0, const float* p0,
                            float* o, float* S_out, float* p_out, int B, int T,
                            int H, int dk, int dv, int chunk, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * kdn_forward_varlen -- kdn_iso_forward / kdn_diag_forward (variant) over N
 * packed sequences of different lengths: sequence s is tokens
 * [cu_seqlens[s], cu_seqlens[s+1]) of tensors laid out [total, H, ...]
 * (that is [1, total, H, ...]), and it starts from its own S0[s], p0[s] and
 * ends in its own S_out[s], p_out[s] (the prefill -> decode handoff:
 * kdn_decode_step continues from them; "Kalman Delta Networks: ..."
 * abstract, constant-memory decoding).  A sequence may be empty; it then
 * hands S0, p0 (or zeros, ones) through.  On the chunked engine, when the
 * N x H (sequence, head) problems outnumber the SMs, a one-block kernel first
 * orders the sequences longest first (by chunk count) into the workspace and
 * the engine starts them in that order; results do not depend on the order.
 *
 * q, k     [total, H, dk] in_dtype device;  v [total, H, dv]
 * a, r     [total, H] fp32 device;  w [total, H] (iso) or [total, H, dk]
 * cu_seqlens  [N + 1] int32 device, cu_seqlens[0] = 0, non-decreasing,
 *          cu_seqlens[N] = total.  Offsets out of order or out of range are
 *          clamped and reported through the workspace (KDN_ERR_INVALID_ARG
 *          from kdn_read_workspace_status).
 * S0, S_out  [N, H, dv, dk];  p0, p_out  [N, H] (iso) or [N, H, dk] (diag)
 * o        [total, H, dv] fp32 device
 * info_scale  iso only, as kdn_iso_forward
 * chunk    as kdn_iso_forward; the chunked engine serves d_v = 128 here (at
 *          d_v = 64, KDN_CHUNK_AUTO takes the token-recurrent kernel and
 *          KDN_CHUNK_64 returns KDN_ERR_UNSUPPORTED)
 * workspace   device scratch of >= kdn_forward_varlen_workspace_size(...)
 *             bytes (at least 256), 256-byte aligned: the error word, then
 *             (chunked engine) the sequence order
 * total >= 0, N >= 1.  Other arguments and errors as kdn_iso_forward.
 * ---------------------------------------------------------------------- */
size_t kdn_forward_varlen_workspace_size(kdn_variant variant, int N, int H,
                                         int dk, int dv, int chunk);
kdn_status kdn_forward_varlen(kdn_variant variant, const void* q,
                              const void* k, const void* v, kdn_dtype in_dtype,
                              const float* a, const float* w, const float* r,
                              const int32_t* cu_seqlens, const float* S0,
                              const float* p0, float* o, float* S_out,
                              float* p_out, int N, int total, int H, int dk,
                              int dv, float info_scale, int chunk,
                              void* workspace, size_t workspace_bytes,
                              void* stream);

/* ------------------------------------------------------------------------
 * kdn_forward_host -- kdn_iso_forward / kdn_diag_forward (variant) with every
 * tensor in host memory, for callers whose data is not on the device yet.
 * The batch goes through the device in slices of slice_b entries (<= 0
 * selects 1): a slice's inputs are copied in, the forward runs on them and
 * its o, S_out and p_out are copied back, on two internal streams that
 * alternate between slices, so that the copies of one slice overlap the
 * copies of the next and the kernels.  Results equal those of the device
 * calls on the same data.  The pages have no counterpart of this entry point.
 *
 * q, k, v, a, w, r, S0, p0, o, S_out, p_out  as in kdn_iso_forward /
 *          kdn_diag_forward, but host pointers; pinned (page-locked) memory
 *          is needed for the copies to overlap.  S0, p0 may be NULL.
 * info_scale  iso only (as kdn_iso_forward); ignored for KDN_DIAG
 * workspace   device scratch of >= kdn_forward_host_workspace_size(...)
 *             bytes, 256-byte aligned: an error word, then two slots of
 *             one slice's device buffers.  kdn_read_workspace_status() on it
 *             reports a bounded wait that gave up in any slice.
 * stream   the work is ordered after earlier work on `stream`, and later
 *          work on `stream` waits for all of it; synchronise `stream` before
 *          reading the outputs.  Calls on one device are enqueued one at a
 *          time (an internal lock); the host buffers must stay valid until
 *          `stream` has passed the call.
 * Errors: as kdn_iso_forward.  All checks run before anything is enqueued;
 * a KDN_ERR_CUDA from a runtime call part-way still leaves `stream` waiting
 * for what was enqueued.
 * ---------------------------------------------------------------------- */
size_t kdn_forward_host_workspace_size(kdn_variant variant, int B, int T,
                                       int H, int dk, int dv,
                                       kdn_dtype in_dtype, int chunk,
                                       int slice_b);
kdn_status kdn_forward_host(kdn_variant variant, const void* q, const void* k,
                            const void* v, kdn_dtype in_dtype, const float* a,
                            const float* w, const float* r, const float* S0,
                            const float* p0, float* o, float* S_out,
                            float* p_out, int B, int T, int H, int dk, int dv,
                            float info_scale, int chunk, int slice_b,
                            void* workspace, size_t workspace_bytes,
                            void* stream);

/* ------------------------------------------------------------------------
 * kdn_decode_step -- one recurrent decoding step for B x H heads, updating
 * the state in place (the constant-memory decoding of "Kalman Delta
 * Networks: Uncertainty-aware Associative Memory", abstract).  The same
 * update as one token of kdn_iso_forward / kdn_diag_forward.
 *
 * variant  KDN_ISO or KDN_DIAG
 * q, k     [B, H, dk] in_dtype device;  v [B, H, dv] in_dtype device
 * a, r     [B, H] fp32 device
 * w        [B, H] (iso) or [B, H, dk] (diag) fp32 device
 * S        [B, H, dv, dk] fp32 device, read and overwritten
 * p        [B, H] (iso) or [B, H, dk] (diag) fp32 device, read and overwritten
 * o        [B, H, dv] fp32 device output
 * info_scale  iso only; <= 0 selects 1/dk
 * Supported: dk in {32, 64, 128}; 1 <= dv <= 128; pointers 16-byte aligned.
 * ---------------------------------------------------------------------- */
kdn_status kdn_decode_step(kdn_variant variant, const void* q, const void* k,
                           const void* v, kdn_dtype in_dtype, const float* a,
                           const float* w, const float* r, float* S, float* p,
                           float* o, int B, int H, int dk, int dv,
                           float info_scale, void* stream);

/* ------------------------------------------------------------------------
 * kdn_exact_forward -- the dense (full-covariance) Kalman filter of the same
 * memory model, for small d_k: every row of S shares one d_k x d_k covariance
 * P, carried exactly by the Riccati recursion instead of being projected to a
 * scalar or a diagonal.  The pages name this exact filter as what the KDN
 * projection approximates ("Kalman Delta Networks: Uncertainty-aware
 * Associative Memory", abstract; "Kalman Delta Networks: 不确定性感知的联想
 * 记忆", 局限), so this call measures the projection's error.  Per token:
 *   P- = a^2 P + W,  u = P- k,  s = k.u + r,  g = u / s,
 *   S <- a S + (v - a S k) g^T,  o = S q,  P = P- - u u^T / s
 * with W = w I (variant KDN_ISO) or diag(w) (KDN_DIAG).  There is no
 * information scale: nothing is projected.
 *
 * q, k     [B, T, H, dk] in_dtype device;  v [B, T, H, dv] in_dtype device
 * a, r     [B, T, H] fp32 device
 * w        [B, T, H] (iso) or [B, T, H, dk] (diag) fp32 device
 * S0       [B, H, dv, dk] fp32 device, or NULL for zeros
 * P0       [B, H, dk, dk] fp32 device, or NULL for the identity; only its
 *          symmetric part (P0 + P0^T) / 2 is used
 * o        [B, T, H, dv] fp32 device output
 * S_out    [B, H, dv, dk];  P_out [B, H, dk, dk] fp32 device outputs; they
 *          may alias S0 and P0 (each head reads its state before writing)
 * Supported: dk in {32, 64}; 8 <= dv <= 128 with dv a multiple of 8; every
 * pointer 16-byte aligned.  KDN_ERR_UNSUPPORTED for other sizes.  One CTA
 * per (b, h) runs the T tokens in order; no workspace, no on-device waits.
 * Errors: KDN_ERR_INVALID_ARG (NULL, shape, alignment, variant or dtype),
 * KDN_ERR_CUDA (launch).
 * ---------------------------------------------------------------------- */
kdn_status kdn_exact_forward(kdn_variant variant, const void* q, const void* k,
                             const void* v, kdn_dtype in_dtype, const float* a,
                             const float* w, const float* r, const float* S0,
                             const float* P0, float* o, float* S_out,
                             float* P_out, int B, int T, int H, int dk, int dv,
                             void* stream);

/* ------------------------------------------------------------------------
 * kdn_backward -- the backward pass of kdn_iso_forward / kdn_diag_forward
 * (variant): the gradients of a loss L with respect to every input, given
 * dL/do, dL/dS_T and dL/dp_T ("Kalman Delta Networks: 不确定性感知的联想记忆",
 * 实验: the layers are trained in language models).  It runs the forward
 * again on the token-recurrent kernel, saving the variance before every
 * token and the state before every 16th token in the workspace, then the
 * adjoint recursion from the last token to the first (dS, dp carried
 * backwards), block by block of 16 tokens: each block's states are rebuilt
 * from its checkpoint, with the forward's arithmetic, before its adjoint.
 *
 * q, k, v, a, w, r, S0, p0, info_scale, in_dtype: as the forward call
 * dO       [B, T, H, dv] fp32 device: dL/do
 * dS_T     [B, H, dv, dk], dp_T [B, H] (iso) or [B, H, dk] (diag) fp32
 *          device, or NULL for zero
 * dq, dk   [B, T, H, dk];  dv [B, T, H, dv];  da, dr [B, T, H];
 * dw       [B, T, H] (iso) or [B, T, H, dk] (diag);  dS0 [B, H, dv, dk];
 * dp0      [B, H] (iso) or [B, H, dk] (diag): fp32 device outputs
 * workspace   device scratch of >= kdn_backward_workspace_size(...) bytes,
 *          256-byte aligned: B H ceil(T / 16) dv dk floats of checkpoints,
 *          B H T (1 or dk) floats of variances, B H 16 dv dk floats of
 *          rebuilt states, plus the forward's outputs
 * Supported: dk in {32, 64, 128}; 1 <= dv <= 128; every pointer 16-byte
 * aligned.
 * Errors: KDN_ERR_INVALID_ARG, KDN_ERR_UNSUPPORTED, KDN_ERR_WORKSPACE,
 * KDN_ERR_CUDA, all before anything is enqueued except KDN_ERR_CUDA.
 * ---------------------------------------------------------------------- */
size_t kdn_backward_workspace_size(kdn_variant variant, int B, int T, int H,
                                   int dk, int dv);
kdn_status kdn_backward(kdn_variant variant, const void* q, const void* k,
                        const void* v, kdn_dtype in_dtype, const float* a,
                        const float* w, const float* r, const float* S0,
                        const float* p0, const float* dO, const float* dS_T,
                        const float* dp_T, float* dq, float* dk, float* dv,
                        float* da, float* dw, float* dr, float* dS0,
                        float* dp0, int B, int T, int H, int dk_dim,
                        int dv_dim, float info_scale, void* workspace,
                        size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * kdn_kla_forward -- the diagonal Kalman filter in information form ("Kalman
 * Linear Attention: Parallel Bayesian Filtering ...", 方法论 §1-§3): a
 * precision per key dimension, updated by a Mobius map of the previous one,
 * and an information mean that is an affine recursion given the precisions,
 * read out with the query.  It runs on the Diagonal KDN's inputs (decay a,
 * process noise w per key dimension, value precision 1 / r) with every
 * element of the memory filtered on its own, so per token and dimension i:
 *   lambda-_i = 1 / (a^2 / lambda_i + w_i),  lambda_i = lambda-_i + k_i^2 / r
 *   S <- S diag(f) + v u^T,  f = a lambda- / lambda,  u = (k / r) / lambda
 *   o = S q
 * (forget gate f and write gate u: ratios of precisions).
 *
 * q, k     [B, T, H, dk] in_dtype device;  v [B, T, H, dv] in_dtype device
 * a, r     [B, T, H] fp32 device;  w [B, T, H, dk] fp32 device
 * S0       [B, H, dv, dk] fp32 device posterior mean, or NULL for zeros
 * lam0     [B, H, dk] fp32 device precision, or NULL for ones
 * o        [B, T, H, dv] fp32 device output
 * S_out    [B, H, dv, dk];  lam_out [B, H, dk] fp32 device outputs; they may
 *          alias S0 and lam0
 * Supported: dk in {32, 64, 128}; 8 <= dv <= 128 with dv a multiple of 8;
 * every pointer 16-byte aligned.  One CTA per (b, h); no workspace and no
 * on-device waits.  Errors: KDN_ERR_INVALID_ARG (NULL, shape, alignment,
 * dtype), KDN_ERR_UNSUPPORTED (sizes), KDN_ERR_CUDA (launch).
 * ---------------------------------------------------------------------- */
kdn_status kdn_kla_forward(const void* q, const void* k, const void* v,
                           kdn_dtype in_dtype, const float* a, const float* w,
                           const float* r, const float* S0, const float* lam0,
                           float* o, float* S_out, float* lam_out, int B, int T,
                           int H, int dk, int dv, void* stream);

/* ------------------------------------------------------------------------
 * kdn_kla_forward_ws -- the same filter and arguments as kdn_kla_forward, plus
 * a workspace.  For dk = dv = 128 with bf16 q, k, v it runs the chunked
 * tensor-core engine ("Kalman Linear Attention: ...", 方法论 §2: given the
 * precisions the mean recursion is affine, so a stretch of tokens is a few
 * dense products).  Per 64-token chunk, with G the running product of the
 * forget gates and Q~ = Q . G, U~ = U / G:
 *   A = (Q~ U~^T) masked causal,  O = S0 Q~^T + A V,
 *   S_C = (S0 + V^T U~) diag(G_C),
 * on tcgen05 tensor cores with every fp32 operand split into bf16 hi + lo
 * and fp32 accumulation; the precision recursion runs in fp32 per key
 * dimension.  A chunk whose gates would drive G below 2^-100 is cut into
 * shorter pieces (down to single tokens), so every input is served.  Other
 * shapes and fp32 inputs run kdn_kla_forward's token-recurrent kernel.
 * workspace   device memory of kdn_kla_workspace_size bytes (16-byte
 *             aligned): the call's error word; kdn_read_workspace_status
 *             reports KDN_ERR_TIMEOUT if a bounded on-device wait gave up
 * Results match kdn_kla_forward's to the engine's operand precision (the
 * bf16 hi/lo split keeps 16 significant bits of each fp32 operand).
 * Errors: as kdn_kla_forward, plus KDN_ERR_WORKSPACE (NULL, misaligned or
 * too small).
 * ---------------------------------------------------------------------- */
size_t kdn_kla_workspace_size(int B, int T, int H, int dk, int dv);
kdn_status kdn_kla_forward_ws(const void* q, const void* k, const void* v,
                              kdn_dtype in_dtype, const float* a,
                              const float* w, const float* r, const float* S0,
                              const float* lam0, float* o, float* S_out,
                              float* lam_out, int B, int T, int H, int dk,
                              int dv, void* workspace, size_t workspace_bytes,
                              void* stream);

/* ------------------------------------------------------------------------
 * kdn_read_workspace_status -- synchronise `stream`, then report the device
 * error word a previous call left in `workspace`: KDN_OK, KDN_ERR_TIMEOUT
 * if a bounded on-device wait gave up, or KDN_ERR_INVALID_ARG if packed-
 * sequence offsets were out of order or out of range.  Also returns
 * KDN_ERR_CUDA if the stream reports an error.  This is the only call that
 * blocks the host.
 * ---------------------------------------------------------------------- */
kdn_status kdn_read_workspace_status(const void* workspace,
                                     size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KDN_H_ */
