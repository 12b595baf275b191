/*
 * rope_attn.h -- C ABI of librope_attn.so: exact RoPE / LeRoPE softmax attention,
 * forward, loss and backward, on one NVIDIA B200 (sm_100a).
 *
 * What is computed (per batch b, head h; positions p = 0..n-1; M = d/2 bands):
 *
 *   theta_m     = base^(-2m/d),  theta_hat_m = exp(alpha_m) * theta_m
 *       "LeRoPE: learnable RoPE frequencies", Mecanismo Central (effective
 *       frequency = learned exponential rescaling of the standard RoPE
 *       frequency) and Declaracao do Problema (geometric sequence in base b).
 *   q~_p, k~_p  = band m of q_p, k_p (coordinates 2m, 2m+1) rotated by p*theta_hat_m
 *       same page, Declaracao do Problema (rotation in 2-D frequency bands).
 *   O = softmax(Q~ K~^T / sqrt(d)) V, lse = log-sum-exp of each score row
 *       "RoPE attention can be trained in almost-linear time", Metodologia 1
 *       (normalised softmax s(x)).
 *   L = 1/2 ||O - E||_F^2, dO = O - E
 *       same page, Metodologia 1 (error term l(x): output minus target).
 *   dV = P^T dO; dP = dO V^T (beta); dS = P o (dP - rowsum(dO o O)) (gamma =
 *   diag(s) beta - s s^T beta); dQ = R(-p theta_hat) dS K~ / sqrt(d);
 *   dK = R(-p theta_hat) dS^T Q~ / sqrt(d)
 *       same page, Metodologia 1-2 (beta, gamma_1, gamma_2).
 *   dalpha_m = theta_hat_m * sum_{b,h,p} p * (<dQ~_pm, J q~_pm> + <dK~_pm, J k~_pm>)
 *       "LeRoPE", Escolhas de Design Principais (log-space parameters shared by
 *       every head) and Analise Teorica (frequency gradient).
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  Q, K, V, O,
 *     E, dO, dQ, dK, dV are dense row-major [B, H, n, d] in the problem dtype
 *     (fp32 or bf16); lse is fp32 [B, H, n]; alpha and dalpha are fp32 [d/2];
 *     L is one fp32 in device memory.  Pointers must be 16-byte aligned.
 *   - ws / ws_bytes: caller-owned device workspace of at least
 *     rope_attn_workspace_bytes(p) bytes, 256-byte aligned.  The library
 *     allocates no device memory of its own and keeps nothing between calls
 *     in it; two calls that run concurrently need two workspaces.
 *   - stream: a cudaStream_t (0 = legacy default stream).  All calls are
 *     asynchronous on that stream; outputs are valid once it has synchronised.
 *   - Arguments are validated before anything is launched; a rejected call
 *     launches nothing and returns RA_ERR_INVALID_ARG / RA_ERR_UNSUPPORTED /
 *     RA_ERR_WORKSPACE.  A failed launch returns RA_ERR_CUDA.  Device-side
 *     waits are bounded: a wait that expires makes the kernel record
 *     RA_ERR_TIMEOUT in the workspace error word and return; read it with
 *     rope_attn_device_status().  No entry point aborts or traps.
 *   - Supported: fp32 with even d, 2 <= d <= 128 (CUDA-core path); bf16 with
 *     d in {64, 128} (tcgen05 tensor-core path); n >= 1; B, H >= 1.
 *   - Precision of the bf16 path: the rotated Q~, K~ feed the score products
 *     S = Q~ K~^T as fp16 (11-bit significand, 8x finer than bf16: sharp softmaxes
 *     amplify score rounding), P, V and dO stay bf16, dS is fp16 with a power-of-two
 *     scale derived on the device from max_i |dO_i| * max_j |v_j|; every product
 *     accumulates in fp32.  Rotated entries must stay within fp16 range
 *     (|q|, |k| below about 46000); a larger one is clamped and reported as
 *     RA_ERR_RANGE by rope_attn_device_status.
 */
#ifndef ROPE_ATTN_H
#define ROPE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RA_OK = 0,
    RA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad shape or flag        */
    RA_ERR_UNSUPPORTED = 2,   /* valid request this build does not implement       */
    RA_ERR_WORKSPACE = 3,     /* ws null, misaligned or smaller than required      */
    RA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed       */
    RA_ERR_TIMEOUT = 5,       /* a device-side wait expired (see device_status)    */
    RA_ERR_RANGE = 6          /* an input exceeds the fp16 range of the bf16 path's
                                 score operands (see device_status)                */
} ra_status;

typedef enum { RA_F32 = 0, RA_BF16 = 1 } ra_dtype;

/* Problem description, passed by pointer to every call.  Limits (RA_ERR_UNSUPPORTED
 * beyond them): B, H, n <= 2^30; B*H <= 2^30 (fp32: <= 65535); B*H*n*d <= 2^38. */
typedef struct {
    int64_t B, H, n, d;  /* batch, heads, sequence length, head dimension      */
    int32_t dtype;       /* ra_dtype of Q, K, V, O, E, dO, dQ, dK, dV          */
    int32_t causal;      /* 1: key j is visible to query i only when j <= i     */
    double base;         /* RoPE base b > 0 (theta_m = b^(-2m/d))               */
    int32_t fixed_bands; /* 0..d/2: the slowest bands m >= d/2 - fixed_bands are not
                            rotated (theta_hat_m = 0, dalpha_m = 0): partial RoPE, the
                            p-RoPE baseline of "LeRoPE" (Configuracao Experimental) with
                            p = 1 - fixed_bands / (d/2); 0 = every band rotates        */
    int32_t reserved;    /* must be 0                                             */
} ra_problem;

/* Bytes of workspace the calls below need for problem *p (0 if *p is invalid).
 * Holds: the fp32 cos/sin table [n, d/2, 2], the rotated Q~ and K~ in the
 * problem dtype, rowsum(dO o O) [B, H, n] fp32, per-tile dalpha partials,
 * loss partials and the device error word. */
size_t rope_attn_workspace_bytes(const ra_problem* p);

/* Bytes of workspace rope_attn_fwd alone needs (a prefix of the full layout: error word,
 * loss partials, table, Q~, K~); 0 if *p is invalid. */
size_t rope_attn_fwd_workspace_bytes(const ra_problem* p);

/* Forward: o = softmax(Q~ K~^T / sqrt(d)) V and lse (natural log) from q, k, v
 * and alpha.  ws needs at least rope_attn_fwd_workspace_bytes(p) bytes (a workspace of
 * rope_attn_workspace_bytes(p) bytes serves every call).  Overwrites the table, Q~ and K~
 * regions of ws. */
ra_status rope_attn_fwd(const ra_problem* p, const void* q, const void* k, const void* v,
                        const float* alpha, void* o, float* lse,
                        void* ws, size_t ws_bytes, void* stream);

/* Loss: *L = 1/2 sum (o - e)^2 over all B*H*n*d elements (fixed-order, deterministic
 * fp64 reduction, stored as fp32) and dO = o - e rounded to the dtype. */
ra_status rope_attn_loss(const ra_problem* p, const void* o, const void* e,
                         float* L, void* dO, void* ws, size_t ws_bytes, void* stream);

/* Backward: dq, dk, dv ([B,H,n,d], dtype) and dalpha ([d/2], fp32, summed over
 * every batch and head) from q, k, v, the forward's o and lse, the upstream
 * gradient dO and alpha.  Deterministic: no atomics, fixed-order reductions (every output
 * bitwise reproducible).
 * Recomputes the table, Q~ and K~ in ws (it does not rely on a previous fwd). */
ra_status rope_attn_bwd(const ra_problem* p, const void* q, const void* k, const void* v,
                        const void* o, const float* lse, const void* dO, const float* alpha,
                        void* dq, void* dk, void* dv, float* dalpha,
                        void* ws, size_t ws_bytes, void* stream);

/* Backward from the forward's saved operands: the same dq, dk, dv, dalpha as
 * rope_attn_bwd, but the table, Q~ and K~ are taken from ws as the most recent
 * rope_attn_fwd on this ws left them (the saved-for-backward tensors of a training
 * step), so q and k are not passed and the rotation is not redone.
 * Caller contract: that forward ran on the same problem, q, k and alpha (their
 * contents unchanged since), on a stream ordered before this call, and nothing wrote
 * ws in between except rope_attn_loss.  Nothing checks the contract: other contents of
 * those regions give wrong gradients, not an error.  alpha is still read (dalpha is
 * theta_hat times the summed torques).  Leaves the device error word as the forward
 * set it (an RA_ERR_RANGE from the forward's rotation stays visible). */
ra_status rope_attn_bwd_saved(const ra_problem* p, const void* v, const void* o,
                              const float* lse, const void* dO, const float* alpha,
                              void* dq, void* dk, void* dv, float* dalpha,
                              void* ws, size_t ws_bytes, void* stream);

/* ---- the projections around the path --------------------------------------------
 * "RoPE attention can be trained in almost-linear time" (Lemma 4.1) states the loss
 * gradient with respect to the weights; these two calls carry the path's dQ, dK, dV back
 * to the projection weights and the layer input.  Row-major layouts: x [B, n, d_model]
 * (dtype of p); each W [d_model, H*d] (dtype of p) with head h in columns h*d..h*d+d-1;
 * q, k, v, dq, dk, dv [B, H, n, d] (dtype of p); dW [d_model, H*d] fp32; dx [B, n, d_model]
 * fp32.  The library's own GEMMs: bf16 on the tcgen05 tensor cores (d in {64, 128},
 * d_model a multiple of 8, else RA_ERR_UNSUPPORTED), fp32 on CUDA cores (exact fp32
 * products); fp32 accumulation in a fixed order (deterministic).  Pointers 16-byte
 * aligned; d_model in 1..2^20.  Only p's B, H, n, d and dtype are used; B, H, n, d <= 2^30,
 * B*n and 3*H*d <= 2^30, B*H*n*d <= 2^38 (RA_ERR_UNSUPPORTED beyond).
 * ws / ws_bytes (both calls): caller workspace, 256-byte aligned, of at least
 * rope_attn_proj_workspace_bytes(p) bytes for rope_attn_proj_bwd and at least 1024 bytes
 * for rope_attn_proj_fwd (RA_ERR_WORKSPACE otherwise).  Its first 64 bytes are the device
 * error word, read with rope_attn_device_status (a GEMM wait that expires records
 * RA_ERR_TIMEOUT there). */

/* [q | k | v][b, h] = x[b] [W_Q | W_K | W_V][:, h] (one GEMM). */
ra_status rope_attn_proj_fwd(const ra_problem* p, int64_t d_model, const void* x,
                             const void* wq, const void* wk, const void* wv,
                             void* q, void* k, void* v, void* ws, size_t ws_bytes,
                             void* stream);

/* Bytes of caller workspace rope_attn_proj_bwd needs: the error word and the three
 * gradients, each merged to [B*n, H*d] rows in the dtype (0 if *p is invalid). */
size_t rope_attn_proj_workspace_bytes(const ra_problem* p);

/* dW_Q = sum_b x[b]^T dq[b] (dq[b] read as [n, H*d]), likewise dW_K, dW_V (one GEMM), and
 * dx[b] = sum_h dq[b,h] W_Q[:,h]^T + dk[b,h] W_K[:,h]^T + dv[b,h] W_V[:,h]^T (one GEMM over
 * the three gradients side by side). */
ra_status rope_attn_proj_bwd(const ra_problem* p, int64_t d_model, const void* x,
                             const void* wq, const void* wk, const void* wv,
                             const void* dq, const void* dk, const void* dv,
                             float* dwq, float* dwk, float* dwv, float* dx,
                             void* ws, size_t ws_bytes, void* stream);

/* ---- the frequency-spectrum diagnostic ----------------------------------------
 * "LeRoPE" (Analise Teorica): the offset-aggregated gradient signal
 *   g_m(D) = sum_{b,h} sum_{i-j=D} dS_ij z_q,i conj(z_k,j) / sqrt(d),  D = -(n-1)..n-1,
 * with band m of a row read as z = x_2m + i x_2m+1 of the unrotated q, k, and the frequency
 * gradient from the derivative of its DTFT surrogate P_m(theta) = Re sum_D g_m(D) e^{iD theta}:
 * dalpha_m = theta_hat_m P_m'(theta_hat_m) (the backward's dalpha by a second route).
 * Inputs as for rope_attn_bwd (o, lse from the forward, dO the upstream gradient).
 * Outputs: g [d/2][2n-1][2] fp32 (re, im; offset D at index D + n - 1; causal: D < 0 is 0)
 * and dalpha [d/2] fp32.  A diagnostic: one (batch, head) and one block of 64 query rows at
 * a time, with 64 x n fp32 scratch for the block's score matrices (fp32 CUDA-core GEMMs;
 * workspace from rope_attn_spectrum_workspace_bytes, O(n d); n <= 32768; B, H <= 2^30,
 * B*H <= 2^30, B*H*n*d <= 2^38); sums in a fixed order (deterministic). */
size_t rope_attn_spectrum_workspace_bytes(const ra_problem* p);
ra_status rope_attn_spectrum(const ra_problem* p, const void* q, const void* k, const void* v,
                             const void* o, const float* lse, const void* dO,
                             const float* alpha, float* g, float* dalpha,
                             void* ws, size_t ws_bytes, void* stream);

/* ---- the optimiser step for the learned frequencies ---------------------------
 * "LeRoPE" (Escolhas de Design Principais: Otimizacao) trains alpha without weight decay
 * and clips its gradient separately from the model's.  The page names neither the
 * optimiser nor the clipping rule; this is Adam with weight decay 0 after scaling dalpha
 * to L2 norm clip_norm when its norm exceeds it (clip_norm <= 0: no clipping). */
typedef struct {
    float lr, beta1, beta2, eps;
    float clip_norm;     /* L2 norm bound for dalpha; <= 0 disables the clipping        */
    int32_t step;        /* 1-based step t (bias corrections 1 - beta^t)                 */
} ra_adam;

/* alpha, m1 (first moment), m2 (second moment): count fp32 each, updated in place from
 * dalpha (count fp32), on `stream`.  All four device pointers 16-byte aligned; count in
 * 1..2^20; m1 = m2 = 0 before the first step.  RA_ERR_INVALID_ARG on a bad argument
 * (nothing launched). */
ra_status rope_attn_alpha_adam(const ra_adam* opt, int64_t count, float* alpha,
                               const float* dalpha, float* m1, float* m2, void* stream);

/* Synchronises `stream`, reads and clears the device error word in ws.
 * Returns RA_OK; RA_ERR_TIMEOUT if a kernel gave up on a wait during the most recent
 * call on ws (kernel id / wait site / block id are written to info[0..2] when info is
 * non-null); or RA_ERR_RANGE if a rotated query or key entry exceeded the fp16 range
 * of the bf16 path's score operands. */
ra_status rope_attn_device_status(void* ws, size_t ws_bytes, void* stream, int32_t info[3]);

/* Static text for a status code. */
const char* rope_attn_status_string(ra_status s);

/* ---- forward without a caller workspace --------------------------------------
 * The papers have no counterpart to this entry point; it exists for callers that
 * cannot allocate device memory at all -- a memory plan fixed before start-up, a
 * runtime that forbids allocation after initialisation, or a host framework that owns
 * every device byte -- and so have no workspace to hand over.
 *
 * Same arguments and results as rope_attn_fwd, minus ws / ws_bytes.  Its scratch (the
 * error word, cos/sin table, Q~ and K~) lives in one static device array of
 * RA_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU that loads the
 * library holds until the process exits.  The call itself allocates nothing: no
 * cudaMalloc, no cudaFree, no allocating library routine.
 *   - Limit: a problem with rope_attn_fwd_workspace_bytes(p) > RA_NOALLOC_SCRATCH_BYTES
 *     (e.g. more than about 1.9M elements per [B,H,n,d] tensor in bf16) is rejected
 *     with RA_ERR_UNSUPPORTED before anything is launched.
 *   - Set-up: the first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before
 *     any stream capture begins.  Later calls reuse the cached address.
 *   - Sharing: every call on a device uses the same array, which keeps the last call's
 *     contents.  Each call clears the error word and rewrites every region it reads,
 *     but calls that overlap on the GPU (other streams, other host threads) race on
 *     the array: issue them on one stream.
 *   - Device: the tensors must live on the current device (the array used is that
 *     device's copy).
 *   - Device-side errors (a wait timeout, RA_ERR_TIMEOUT, or a rotated entry beyond the
 *     fp16 range, RA_ERR_RANGE) are recorded in the array's own error word; the call's
 *     return value cannot show them (it returns before the kernels run).  Read them with
 *     rope_attn_noalloc_status. */
#define RA_NOALLOC_SCRATCH_BYTES (8u << 20)
ra_status rope_attn_fwd_noalloc(const ra_problem* p, const void* q, const void* k, const void* v,
                                const float* alpha, void* o, float* lse, void* stream);

/* Synchronises `stream`, then reads and clears the error word of the current device's
 * static array: RA_OK, RA_ERR_TIMEOUT (info as for rope_attn_device_status) or RA_ERR_RANGE
 * from the most recent rope_attn_fwd_noalloc on this device.  Allocates nothing. */
ra_status rope_attn_noalloc_status(void* stream, int32_t info[3]);

/* ---- optional per-kernel timing (instrumentation, off by default) --------
 * While enabled, every kernel launch made by the calls above is bracketed by
 * CUDA events on the caller's stream (rope_attn_spectrum: its whole sequence
 * of launches as one).  rope_attn_timing_read synchronises
 * those events and writes, per kernel id, the number of launches and the sum
 * of their durations in milliseconds; it returns the number of kernel ids
 * (at most max_ids) and clears the record. */
void rope_attn_timing_enable(int on);
int rope_attn_timing_read(int32_t* launches, double* total_ms, int max_ids);
const char* rope_attn_kernel_name(int id);

#ifdef __cplusplus
}
#endif

#endif /* ROPE_ATTN_H */
