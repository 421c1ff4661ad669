/*
 * kla.h -- C ABI of the B200 (sm_100a) Kalman Linear Attention filter scan.
 *
 * The library computes, for every channel (b, h, n) independently, the scalar
 * information-form Kalman filter of Kalman Linear Attention (KLA):
 *
 *   precision   lambda_t = ((1 + p_t phi_t) lambda_{t-1} + a_t^2 phi_t)
 *                          / (p_t lambda_{t-1} + a_t^2)
 *               i.e. the Moebius map of M_t = [[1 + p_t phi_t, a_t^2 phi_t],
 *                                              [p_t,           a_t^2      ]]
 *               (Pith review of "Kalman Linear Attention: Parallel Bayesian
 *                Filtering For Efficient Language Modelling and State
 *                Tracking", section "What carries the argument"; its
 *                derivation from the information-form predict / update is
 *                the review's "Circularity Check", Theorem 1)
 *   gate        f_t = a_t / (a_t^2 + p_t lambda_{t-1})
 *   info mean   eta_t = f_t eta_{t-1} + b_t
 *               (the affine information-mean recursion with the
 *                precision-ratio forget gate, review "Core claim" and
 *                Theorem 2)
 *   outputs     lambda_t, eta_t, mu_t = eta_t / lambda_t, var_t = 1 / lambda_t
 *               (explicit belief-state uncertainty, review "Core claim" and
 *                the ICML 2026 poster abstract)
 *
 * a_t is the state decay, p_t the process-noise variance, phi_t the
 * token-evidence precision (k_t^2 Lambda^v_t) and b_t the token information
 * (k_t Lambda^v_t v_t).  (lambda_0, eta_0) is the prior before token 1; output
 * row t-1 holds the posterior after token t.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Layout: per-token tensors are [B, T, H, N] row-major (N fastest), dense.
 *   Per-channel tensors (prior, decode state, one decode token) are
 *   [B, H, N] row-major, dense.  A "channel" is one (b, h, n).
 * - Memory: every pointer is DEVICE memory owned by the caller (allocate it
 *   with cudaMalloc, torch, ...).  The library allocates nothing and keeps no
 *   pointer after a call returns.
 * - Streams: `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *   default stream).  Calls enqueue work and return without synchronising;
 *   results are valid once the stream reaches that point.
 * - Errors: argument errors are detected on the host before anything is
 *   enqueued and return a kla_status_t != KLA_OK; nothing is written then.
 *   A launch failure returns KLA_ERR_CUDA.  Device-side failures (a bounded
 *   wait that ran out) are recorded on the device and reported by
 *   kla_get_error(); the affected outputs are NaN.
 * - Preconditions, not checked per element: p_t >= 0, phi_t >= 0,
 *   lambda_0 > 0, and a_t^2 + p_t lambda_{t-1} > 0 (e.g. a_t != 0 or p_t > 0);
 *   the row sums of M_t stay below 2^63 per token (1 + p phi + a^2 phi + p +
 *   a^2; 2^31 for kla_layer_forward), which keeps the chunk aggregates finite.
 *   Any real a_t is allowed (only a_t^2 enters the precision; the sign of a_t
 *   enters the gate).  The state must stay within fp32 range: with p_t = 0
 *   and |a_t| < 1 the precision grows like a^(-2t) and overflows after about
 *   44 / -ln|a| tokens (the fp64 oracle goes further).
 * - Arithmetic: inputs are fp32 or bf16 (converted exactly to fp32 on load);
 *   state, arithmetic and outputs are fp32 (the gradients of an input are
 *   written in that input's dtype); reciprocals use the hardware instruction
 *   (PTX rcp.approx.ftz.f32, within 1 ulp); nothing else is approximated.
 * - Outputs must not overlap inputs or each other.
 */
#ifndef KLA_H
#define KLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KLA_ABI_VERSION 1

typedef enum {
    KLA_F32 = 0,  /* IEEE binary32 */
    KLA_BF16 = 1  /* bfloat16 (8-bit exponent, 7-bit mantissa) */
} kla_dtype_t;

typedef enum {
    KLA_OK = 0,
    KLA_ERR_INVALID_ARG = 1,         /* null pointer, negative size, overlap, size overflow */
    KLA_ERR_UNSUPPORTED_DTYPE = 2,   /* dtype is not KLA_F32 / KLA_BF16 */
    KLA_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes below the required size */
    KLA_ERR_CUDA = 4,                /* a CUDA runtime / driver call failed */
    KLA_ERR_TIMEOUT = 5,             /* a device-side bounded wait ran out */
    KLA_ERR_MISALIGNED = 6,          /* workspace not 256-byte aligned */
    KLA_ERR_TOO_LARGE = 7            /* problem exceeds the static scratch of kla_scan_forward_static */
} kla_status_t;

/* ABI version of the loaded library (KLA_ABI_VERSION it was built with). */
int kla_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *kla_strerror(kla_status_t status);

/*
 * Size in bytes of the device workspace that kla_scan_forward needs for a
 * problem of this shape and input dtype, written to *bytes.  The workspace
 * holds the cross-chunk carries of the scan (per chunk and channel: a 3x3
 * homogeneous aggregate and the inclusive state) and their ready flags.
 * Returns KLA_ERR_INVALID_ARG for negative sizes or a null `bytes`.
 */
kla_status_t kla_scan_forward_workspace_size(int64_t B, int64_t T, int64_t H, int64_t N,
                                             kla_dtype_t in_dtype, size_t *bytes);

/*
 * Forward filter over whole sequences (the parallel scan; review "Core claim":
 * both recursions compose associatively, O(T) work).
 *
 *   a, p, phi, b   [B, T, H, N] inputs of dtype in_dtype (device, read only)
 *   lambda0, eta0  [B, H, N] fp32 prior (device, read only)
 *   lambda_out     [B, T, H, N] fp32 posterior precision (device, written)
 *   eta_out        [B, T, H, N] fp32 information mean (device, written)
 *   mu_out         [B, T, H, N] fp32 posterior mean, or NULL to skip
 *   var_out        [B, T, H, N] fp32 posterior variance, or NULL to skip
 *   workspace      device scratch of at least
 *                  kla_scan_forward_workspace_size(...) bytes, 256-byte
 *                  aligned; its contents on entry do not matter and are
 *                  undefined on return.  Two calls in flight at the same time
 *                  (e.g. on two streams) need two workspaces.
 *
 * T == 0 or B*H*N == 0 is a valid empty problem (nothing is enqueued).
 * The last row of lambda_out / eta_out is the state to continue decoding from
 * with kla_scan_step.
 */
kla_status_t kla_scan_forward(const void *a, const void *p, const void *phi, const void *b,
                              kla_dtype_t in_dtype,
                              const float *lambda0, const float *eta0,
                              float *lambda_out, float *eta_out, float *mu_out, float *var_out,
                              int64_t B, int64_t T, int64_t H, int64_t N,
                              void *workspace, size_t workspace_bytes, void *stream);

/*
 * Which forward kernel kla_scan_forward would launch for a problem of this
 * shape and dtype with these input pointers (only their alignment matters;
 * they are not dereferenced), written to *kernel: 1 = the chunked kernel whose
 * chunks exchange carries through the workspace, 2 = the channel-owning
 * streaming kernel; *launches = the kernel launches one call enqueues (2 for
 * the chunked kernel, preceded by a workspace clear; 1 or 2 for the
 * streaming kernel, 2 when it takes its work units by ticket from the
 * workspace: tiles split into runs, or more tiles than SMs, each at least 8
 * chunks long).  0 and 0 for an empty problem.  Honours
 * kla_debug_force_forward_kernel.
 */
kla_status_t kla_scan_forward_plan(int64_t B, int64_t T, int64_t H, int64_t N, kla_dtype_t in_dtype,
                                   const void *a, const void *p, const void *phi, const void *b,
                                   int *kernel, int *launches);

/*
 * Test hook: which forward kernel kla_scan_forward calls enqueued afterwards
 * use.  0 (default): chosen by shape; 1: the chunked kernel whose chunks
 * exchange carries through the workspace (any shape); 2: the channel-owning
 * streaming kernel (used only when its geometry holds: 16-byte aligned
 * inputs, H*N*elem a multiple of 16 bytes, H*N >= 32, T >= 32; otherwise the
 * chunked kernel runs).  Both compute the same filter; their chunkings
 * differ, so results agree to rounding, not bit for bit.  KLA_ERR_INVALID_ARG
 * for other values.
 */
kla_status_t kla_debug_force_forward_kernel(int which);

/* Size of the static device scratch array used by kla_scan_forward_static. */
#define KLA_STATIC_SCRATCH_BYTES (32u << 20) /* 32 MiB */

/*
 * kla_scan_forward for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this entry point: it exists for callers
 * that cannot call cudaMalloc (or torch's allocator) at the point where they
 * run the filter -- for example code running inside a CUDA stream capture,
 * code under a fixed memory budget, or a host runtime without an allocator of
 * its own -- and so cannot provide the workspace kla_scan_forward needs.
 *
 * Same arguments, results and errors as kla_scan_forward, minus the
 * workspace: the carry scratch is a static device array of
 * KLA_STATIC_SCRATCH_BYTES inside this library (one per device that loads
 * the library, held until the process exits).  The call allocates and frees
 * nothing.  The caller still provides the inputs and outputs.
 *
 * - Size limit: a problem is accepted when kla_scan_forward_workspace_size()
 *   reports at most KLA_STATIC_SCRATCH_BYTES (about 59 million
 *   token-channels with full 64-channel tiles, e.g. B=8, T=2048, H=16,
 *   N=128); larger problems return KLA_ERR_TOO_LARGE before anything is
 *   enqueued.
 * - First call on a device: it looks up the device address of the static
 *   array (cudaGetSymbolAddress) with that device current, and caches it for
 *   the life of the process.  Make that first call before any stream capture
 *   begins.  cudaDeviceReset unloads the library's device code with the
 *   context, and the array may sit elsewhere afterwards while the cached
 *   address does not change: a process that resets a device must not call
 *   this entry point on that device again.
 * - Sharing: every call on a device uses the same array, which keeps what the
 *   last call left in it; each call re-zeroes, on its stream, the part that
 *   must start at zero.  Calls whose work overlaps on the GPU (two streams,
 *   two host threads) race on the array and give wrong results: serialise
 *   them, or use kla_scan_forward with one workspace each.
 */
kla_status_t kla_scan_forward_static(const void *a, const void *p, const void *phi, const void *b,
                                     kla_dtype_t in_dtype,
                                     const float *lambda0, const float *eta0,
                                     float *lambda_out, float *eta_out, float *mu_out, float *var_out,
                                     int64_t B, int64_t T, int64_t H, int64_t N, void *stream);

/*
 * Device workspace that kla_scan_forward_host needs (two device slots of one
 * block each, plus the scan workspace of one block), written to *bytes.
 * t_block = tokens per block, or 0 to let the library pick (about T / 64,
 * whole 64-token chunks, at least 64 tokens).
 */
kla_status_t kla_scan_forward_host_workspace_size(int64_t B, int64_t T, int64_t H, int64_t N,
                                                  kla_dtype_t in_dtype, int64_t t_block, size_t *bytes);

/*
 * The forward filter on HOST buffers (same arguments and results as
 * kla_scan_forward, but a, p, phi, b, lambda0, eta0 and the outputs are host
 * memory, ideally page-locked).  The sequence is processed in blocks of
 * t_block tokens: the copy of block k+1 to the device, the scan of block k
 * (entering with the state that left block k-1, i.e. its last lambda / eta
 * row) and the copy of block k-1 back overlap on two internal copy streams and
 * `stream`.  Sequences longer than device memory can thus be filtered.
 *
 *   workspace   device memory of at least
 *               kla_scan_forward_host_workspace_size(...) bytes, 256-byte
 *               aligned, owned by the caller.
 *   stream      the caller's stream; when it reaches the end of the call every
 *               output has been written to host memory.
 *
 * The internal copy streams and events are created once per device; calls on
 * one device must not overlap (serialise them on one stream).  Results agree
 * with kla_scan_forward to rounding (block boundaries are extra carry points).
 */
kla_status_t kla_scan_forward_host(const void *a, const void *p, const void *phi, const void *b,
                                   kla_dtype_t in_dtype,
                                   const float *lambda0, const float *eta0,
                                   float *lambda_out, float *eta_out, float *mu_out, float *var_out,
                                   int64_t B, int64_t T, int64_t H, int64_t N, int64_t t_block,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * One recurrent decode token for every channel (constant work per token;
 * the running posterior is a sufficient summary: "Kalman filter" primer
 * section 6.2, and the review's O(1)-per-step recurrent form).
 *
 *   a, p, phi, b   [B, H, N] inputs of this token, dtype in_dtype (read only)
 *   lambda_state   [B, H, N] fp32 precision, read and overwritten in place
 *   eta_state      [B, H, N] fp32 information mean, read and overwritten
 *   mu_out         [B, H, N] fp32 posterior mean of this token, or NULL
 *   var_out        [B, H, N] fp32 posterior variance of this token, or NULL
 *
 * B*H*N == 0 is valid (nothing is enqueued).  The state pointers may not
 * overlap the inputs or the other outputs.
 */
kla_status_t kla_scan_step(const void *a, const void *p, const void *phi, const void *b,
                           kla_dtype_t in_dtype,
                           float *lambda_state, float *eta_state,
                           float *mu_out, float *var_out,
                           int64_t B, int64_t H, int64_t N, void *stream);

/*
 * Size in bytes of the device workspace kla_scan_backward needs for a problem
 * of this shape (the run-boundary carries and flags used when the sequence
 * of a channel tile is split into runs across SMs), written to *bytes.  0 for
 * an empty problem.  KLA_ERR_INVALID_ARG for negative sizes or a null `bytes`.
 */
kla_status_t kla_scan_backward_workspace_size(int64_t B, int64_t T, int64_t H, int64_t N,
                                              kla_dtype_t in_dtype, size_t *bytes);

/*
 * Gradients of a scalar loss through kla_scan_forward (reverse mode).  The
 * review claims end-to-end parallel training of the layer but gives no
 * backward pass; this one differentiates the information-form recursion
 * above.  With D_t = a_t^2 + p_t lambda_{t-1}, r_t = 1/D_t, f_t = a_t r_t:
 *
 *   fold        gl_t = g_lambda_t - v_t (g_mu_t mu_t + g_var_t v_t),
 *               ge_t = g_eta_t + g_mu_t v_t      (v_t = 1/lambda_t, mu_t = eta_t v_t)
 *   adjoint     E_t = dL/d eta_t    = ge_t + f_{t+1} E_{t+1},
 *               L_t = dL/d lambda_t = gl_t + f_{t+1}^2 L_{t+1} + c_{t+1} E_{t+1},
 *               c_t = -p_t f_t r_t eta_{t-1}      (a reverse-time scan)
 *   inputs      d/d phi_t = L_t,  d/d b_t = E_t,
 *               d/d a_t = r_t^2 (-2 a_t lambda_{t-1} L_t + (p_t lambda_{t-1} - a_t^2) eta_{t-1} E_t),
 *               d/d p_t = -r_t^2 lambda_{t-1} (lambda_{t-1} L_t + a_t eta_{t-1} E_t),
 *               d/d eta_0 = f_1 E_1,  d/d lambda_0 = f_1^2 L_1 + c_1 E_1.
 *
 *   a, p           [B, T, H, N] forward inputs, dtype in_dtype (read only);
 *                  phi and b are not needed (they enter through lambda, eta)
 *   lambda0, eta0  [B, H, N] fp32 prior of the forward call (read only)
 *   lambda_out, eta_out
 *                  [B, T, H, N] fp32 outputs of that forward call (read only)
 *   g_lambda, g_eta, g_mu, g_var
 *                  [B, T, H, N] fp32 gradients of the loss with respect to the
 *                  four forward outputs; NULL = zero (that array is not read)
 *   grad_a, grad_p, grad_phi, grad_b
 *                  [B, T, H, N] gradients with respect to the inputs, written
 *                  in in_dtype (fp32 arithmetic, rounded once on store); NULL =
 *                  not wanted
 *   grad_lambda0, grad_eta0
 *                  [B, H, N] fp32 gradients with respect to the prior, or NULL
 *   workspace      device scratch of at least
 *                  kla_scan_backward_workspace_size(...) bytes, 256-byte
 *                  aligned (may be NULL when that size is 0); contents on
 *                  entry do not matter.  Concurrent calls need their own.
 *
 * B*H*N == 0 is valid (nothing is enqueued).  T == 0 writes zero prior
 * gradients.  Outputs must not overlap the inputs, the workspace or each
 * other (KLA_ERR_INVALID_ARG).  Same preconditions as the forward call; the
 * forward outputs are trusted as given.
 */
kla_status_t kla_scan_backward(const void *a, const void *p, kla_dtype_t in_dtype,
                               const float *lambda0, const float *eta0,
                               const float *lambda_out, const float *eta_out,
                               const float *g_lambda, const float *g_eta,
                               const float *g_mu, const float *g_var,
                               void *grad_a, void *grad_p, void *grad_phi, void *grad_b,
                               float *grad_lambda0, float *grad_eta0,
                               int64_t B, int64_t T, int64_t H, int64_t N,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * Which backward kernel kla_scan_backward would launch (only the alignment of
 * a and p is looked at; outputs are assumed 16-byte aligned), written to
 * *kernel: 1 = one thread per channel walking the sequence backwards (any
 * shape), 2 = the channel-owning streaming kernel (16-byte aligned arrays,
 * H*N*elem a multiple of 16 bytes, H*N >= 32); *launches = kernel launches
 * per call (2 when a workspace clear precedes the streaming kernel).  0 and
 * 0 for B*H*N == 0.  Honours kla_debug_force_backward_kernel.
 */
kla_status_t kla_scan_backward_plan(int64_t B, int64_t T, int64_t H, int64_t N, kla_dtype_t in_dtype,
                                    const void *a, const void *p, int *kernel, int *launches);

/*
 * Test hook: which backward kernel later kla_scan_backward calls use.
 * 0 (default): by shape; 1: one thread per channel; 2: the streaming kernel
 * where its geometry holds.  Results agree to rounding.  KLA_ERR_INVALID_ARG
 * for other values.
 */
kla_status_t kla_debug_force_backward_kernel(int which);

/*
 * Device workspace that kla_layer_forward needs (run-boundary carries and
 * flags, as for kla_scan_backward), written to *bytes; 0 when there is no
 * token or no channel.  KLA_ERR_INVALID_ARG for negative sizes, a null
 * `bytes`, Ns other than 8 or 16, or D not a multiple of 32 / Ns.
 */
kla_status_t kla_layer_forward_workspace_size(int64_t B, int64_t T, int64_t H, int64_t D, int64_t Ns,
                                              kla_dtype_t in_dtype, size_t *bytes);

/*
 * The KLA layer's filter with its input formation and readout fused: for H
 * heads of value dimension D and state expansion Ns, the H x D x Ns state
 * channels (h, d, n) are independent scalar filters (the review's diagonal
 * model) that observe value coordinate d through the observation operator
 * k_n with the value precision w_d = Lambda^v_d:
 *
 *   phi_t = k_{t,n}^2 w_{t,d},  b_t = k_{t,n} w_{t,d} v_{t,d}   (the update adds
 *          k^2 Lambda^v: review "Circularity Check", Theorem 1)
 *   the filter above with the channel's time-invariant decay a and process
 *          noise p (the review lists the OU decay as time-invariant; a and p
 *          are taken already discretised)
 *   y_{t,d} = sum_n q_{t,n} mu_{t,d,n},   s_{t,d} = sum_n q_{t,n}^2 var_{t,d,n}
 *          (the readout operator q on the posterior mean, and the variance of
 *          that readout under the diagonal posterior)
 *
 *   k, q          [B, T, H, Ns] observation / readout operators, in_dtype
 *   v, w          [B, T, H, D] values and value precisions (w > 0), in_dtype
 *   a, p          [H, D, Ns] fp32 per-channel decay and process noise (p >= 0)
 *   lambda0, eta0 [B, H, D, Ns] fp32 prior
 *   y             [B, T, H, D] fp32 readout (written)
 *   s             [B, T, H, D] fp32 variance readout, or NULL
 *   lambda_T, eta_T
 *                 [B, H, D, Ns] fp32 state after the last token (for decoding
 *                 on with kla_scan_step), or both NULL
 *   workspace     at least kla_layer_forward_workspace_size(...) bytes,
 *                 256-byte aligned (NULL when that is 0)
 *
 * Precondition (besides the scan's): per token and state channel,
 * 1 + p phi + a^2 phi + p + a^2 < 2^31 with phi = k^2 w (the kernel
 * renormalises its chunk aggregates every fourth token).
 *
 * Supported shapes: Ns = 8 or 16 (the state expansions the review lists),
 * D a multiple of 32 / Ns; k, q, v, w 16-byte aligned.  Anything else returns
 * KLA_ERR_INVALID_ARG before anything is enqueued (there is no fallback
 * kernel).  T == 0 copies the prior into lambda_T / eta_T.  Outputs must not
 * overlap inputs, the workspace or each other.  Results agree with
 * kla_scan_forward on the formed phi, b followed by the readout, to rounding.
 */
kla_status_t kla_layer_forward(const void *k, const void *q, const void *v, const void *w,
                               kla_dtype_t in_dtype, const float *a, const float *p,
                               const float *lambda0, const float *eta0,
                               float *y, float *s, float *lambda_T, float *eta_T,
                               int64_t B, int64_t T, int64_t H, int64_t D, int64_t Ns,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * One decode token of the fused layer, from the resident state: the
 * recurrent counterpart of kla_layer_forward (continue from its lambda_T /
 * eta_T).  Same channels, evidence, filter and readout, for one token.
 *
 *   k, q          [B, H, Ns] this token's operators, in_dtype
 *   v, w          [B, H, D] this token's values and value precisions, in_dtype
 *   a, p          [H, D, Ns] fp32
 *   lambda_state, eta_state
 *                 [B, H, D, Ns] fp32 state, read and overwritten in place
 *   y             [B, H, D] fp32 readout of this token (written)
 *   s             [B, H, D] fp32 variance readout, or NULL
 *
 * Ns = 8 or 16 and D a multiple of 32 / Ns (KLA_ERR_INVALID_ARG otherwise);
 * any alignment.  B*H*D == 0 is valid (nothing is enqueued).  Outputs must
 * not overlap the inputs or each other.
 */
kla_status_t kla_layer_step(const void *k, const void *q, const void *v, const void *w, kla_dtype_t in_dtype,
                            const float *a, const float *p, float *lambda_state, float *eta_state,
                            float *y, float *s, int64_t B, int64_t H, int64_t D, int64_t Ns, void *stream);

/* Largest window (tokens) of kla_attention_weights. */
#define KLA_ATTENTION_MAX_WINDOW 64

/*
 * The Kalman attention weights: how the information mean of a later token
 * responds to an earlier one (the review's "Kalman Attention Matrix", its
 * minor comment on App. E.3/E.4).  The affine recursion eta_k = f_k eta_{k-1}
 * + b_k (review "Core claim") unrolls into
 *
 *   eta_t = F(t, s) eta_s + sum_{r = s+1..t} F(t, r) b_r,
 *   F(t, s) = prod_{k = s+1..t} f_k,   f_k = a_k / (a_k^2 + p_k lambda_{k-1}),
 *
 * (rows 0-based; F(t, t) = 1), which also equals prod(a) / (C lambda_s + D)
 * for [[A, B], [C, D]] = M_t ... M_{s+1}.  The tokens [t0, t0 + span) are cut
 * into windows of W tokens and F is written for every pair inside a window:
 *
 *   a, p        [B, T, H, N] forward inputs, dtype in_dtype (read only)
 *   lambda_out  [B, T, H, N] fp32 posterior precision written by
 *               kla_scan_forward on the same inputs (read only; the gate of
 *               token k uses row k-1)
 *   F           [B, nwin, W, W, H, N] fp32, nwin = ceil(span / W) (written):
 *               F[b, w, i, j, h, n] = F(t, s) with t = t0 + w W + i,
 *               s = t0 + w W + j, for j <= i < (tokens of window w inside the
 *               span); every other entry (above the diagonal, past the span)
 *               is written as 0.
 *
 * 1 <= W <= KLA_ATTENTION_MAX_WINDOW and 0 <= t0 <= t0 + span <= T, else
 * KLA_ERR_INVALID_ARG.  span == 0 or B*H*N == 0 is a valid empty call.  F may
 * not overlap the inputs.  The gates use the hardware reciprocal, as the
 * scan does; the products are plain fp32 multiplies (an entry below the fp32
 * normal range flushes to 0).  Bound by the bytes of F: W^2 * 4 per channel
 * and window.
 */
kla_status_t kla_attention_weights(const void *a, const void *p, kla_dtype_t in_dtype,
                                   const float *lambda_out, float *F,
                                   int64_t B, int64_t T, int64_t H, int64_t N,
                                   int64_t t0, int64_t span, int64_t W, void *stream);

/*
 * Device workspace that kla_scan_forward_lti needs (run-boundary carries and
 * flags), written to *bytes; 0 for an empty problem.
 */
kla_status_t kla_scan_forward_lti_workspace_size(int64_t B, int64_t T, int64_t H, int64_t N,
                                                 kla_dtype_t in_dtype, size_t *bytes);

/*
 * The filter of deterministic time-invariant channels in its convolutional
 * form (the review's Theorem 3: for a deterministic LTI system the filter is
 * a convolution).  With no process noise (p_t = 0) and a decay a constant in
 * time, the precision map is affine and the gate is 1/a, so (rows 0-based)
 *
 *   lambda_t = a^(-2(t+1)) lambda_0 + sum_{s<=t} a^(-2(t-s)) phi_s,
 *   eta_t    = a^(-(t+1))  eta_0    + sum_{s<=t} a^(-(t-s))  b_s,
 *
 * mu_t = eta_t / lambda_t, var_t = 1 / lambda_t: the same results as
 * kla_scan_forward with a_t = a and p_t = 0, computed as blocked causal
 * convolutions with the geometric kernels and reading only phi and b per
 * token.  The carry between chunks is kept in fp64, so a constant decay does
 * not accumulate a drift over long sequences.
 *
 *   a              [B, H, N] fp32 decay of each channel, nonzero (read only)
 *   phi, b         [B, T, H, N] dtype in_dtype (read only)
 *   lambda0, eta0  [B, H, N] fp32 prior (read only)
 *   lambda_out, eta_out, mu_out, var_out
 *                  [B, T, H, N] fp32 outputs, as for kla_scan_forward (mu_out
 *                  and var_out may be NULL)
 *   workspace      at least kla_scan_forward_lti_workspace_size(...) bytes,
 *                  256-byte aligned; contents on entry do not matter
 *
 * Preconditions as for kla_scan_forward; the state must stay in fp32 range
 * (with |a| < 1 the precision grows like a^(-2t)).  Empty problems are valid.
 */
kla_status_t kla_scan_forward_lti(const float *a, const void *phi, const void *b, kla_dtype_t in_dtype,
                                  const float *lambda0, const float *eta0,
                                  float *lambda_out, float *eta_out, float *mu_out, float *var_out,
                                  int64_t B, int64_t T, int64_t H, int64_t N,
                                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * Which kernel kla_scan_forward_lti would launch (only the alignment of phi
 * and b is looked at), written to *kernel: 1 = one thread per channel (any
 * shape), 2 = the channel-owning streaming kernel (16-byte aligned phi and
 * b, H*N*elem a multiple of 16 bytes, H*N >= 32, T >= 32); *launches = kernel
 * launches per call (2 when a workspace clear precedes the streaming
 * kernel).  0 and 0 for an empty problem.
 */
kla_status_t kla_scan_forward_lti_plan(int64_t B, int64_t T, int64_t H, int64_t N, kla_dtype_t in_dtype,
                                       const void *phi, const void *b, int *kernel, int *launches);

/*
 * Synchronise `stream`, then report the first failure since the previous
 * call on the current device: KLA_ERR_CUDA for a CUDA error (sticky or not),
 * KLA_ERR_TIMEOUT if a kernel's bounded wait ran out (the outputs that
 * depended on it are NaN), KLA_OK otherwise.  Clears the device-side record.
 */
kla_status_t kla_get_error(void *stream);

/*
 * Upper bound, in nanoseconds, of every device-side wait (a chunk waiting for
 * the carry of its predecessor; a CTA waiting for its own tile load).  The
 * default is 1e9 (one second).  A wait that runs out records KLA_ERR_TIMEOUT
 * and writes NaN instead of blocking.  Applies to calls enqueued afterwards.
 * Returns KLA_ERR_INVALID_ARG for 0.
 */
kla_status_t kla_set_wait_limit_ns(uint64_t ns);

/*
 * Test hook for the failure path: enqueue one kernel on `stream` that waits,
 * through the same bounded wait the scan uses, on a device flag that nothing
 * ever sets, with the current wait limit.  The wait runs out, records
 * KLA_ERR_TIMEOUT, and the kernel returns; kla_get_error() then reports it.
 */
kla_status_t kla_debug_unset_flag_wait(void *stream);

/*
 * Number of tokens in one chunk of the forward scan (the unit of the
 * cross-chunk carry).  Informational; results do not depend on it.
 */
int kla_forward_chunk_tokens(void);

/*
 * Test hook for the forward scan's failure path: in kla_scan_forward calls
 * enqueued afterwards, the carry into the chunk that starts at token
 * chunk * kla_forward_chunk_tokens() first waits on a device flag that
 * nothing sets.  The wait runs out after the wait limit, records
 * KLA_ERR_TIMEOUT and poisons that chunk's entering state: its outputs are
 * NaN and earlier tokens are unaffected.  In the chunked kernel a later chunk
 * is either exact (its look-back composed the stalled chunk's aggregate) or
 * NaN; in the streaming kernel every later token of the same channels is NaN
 * (the state is handed from chunk to chunk).  The streaming backward kernel
 * of kla_scan_backward honours it too: the carry into the backward chunk
 * holding that token is poisoned, so the gradients of that chunk and of every
 * earlier token of the same channels are NaN, later tokens are exact.  -1
 * (the default) turns the hook off.
 */
kla_status_t kla_debug_stall_chunk(int64_t chunk);

#ifdef __cplusplus
}
#endif

#endif /* KLA_H */
