/*
 * saf.h — C ABI of the B200 (sm_100a) mixed-head causal attention library
 * (libsaf.so).
 *
 * The layer is the one described in "When Can Attention Heads Be Statically
 * Defined?" (Selective Attention Freezing).  In one layer:
 *   - an ORDINARY head computes causal softmax attention
 *       A = softmax_causal(Q K^T / sqrt(d_h)),  O = A V
 *     (reading notes, section 一, the first displayed equation);
 *   - a REPLACED head mixes the current V with a frozen causal pattern rebuilt
 *     from two length-T vectors, the absolute-position preference a and the
 *     relative-distance preference r:
 *       P(i,j) = exp(a[j] + r[i-j]) / Z(i)  for j <= i, 0 for j > i,
 *       Z(i)   = sum_{k<=i} exp(a[k] + r[i-k]),        O = P V
 *     (Eq. (3), section 二.3; indices are 0-based here, so the distance i-j
 *     runs over 0..T-1 and both vectors have length T);
 *   - the backward gives dQ, dK, dV for ordinary heads, and only dV = P^T dO
 *     for replaced heads (section 二.4: the pattern is a frozen buffer; the
 *     head's query/key path is gone, so dQ = dK = 0 there).
 *
 * Conventions shared by every entry point
 *   Layout     Q, K, V, O, dO, dQ, dK, dV: contiguous row-major [B, H, T, d_h]
 *              (d_h fastest), bf16 (IEEE bfloat16 bit patterns) unless stated.
 *              lse: [B, H, T] fp32.  a, r, logz: [H, T] fp32; rows of ordinary
 *              heads are never read (they may hold anything, NaN included).
 *              d_h must be 64 (SAF_ERR_UNSUPPORTED otherwise).  Any T >= 1.
 *   Memory     Every tensor pointer is a DEVICE pointer on the current CUDA
 *              device, 16-byte aligned.  replaced_mask is a HOST array of H
 *              bytes (nonzero = replaced head), read only during the call.
 *              The caller owns all buffers, including the workspace; the
 *              library allocates no device memory in these calls.
 *   Streams    `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *              default stream).  Calls enqueue work and return; results are
 *              ready when the stream reaches that point.
 *   Errors     Argument errors are detected on the host before anything is
 *              enqueued and return SAF_ERR_INVALID_ARG / SAF_ERR_UNSUPPORTED /
 *              SAF_ERR_WORKSPACE.  A failed launch returns SAF_ERR_CUDA.
 *              Device-side waits are bounded; one that gives up records an
 *              error word in the workspace, which saf_device_status reports
 *              as SAF_ERR_TIMEOUT.
 *   Workspace  Its first 256 bytes hold the device error word and the work
 *              counters of the persistent kernels; they must be zero before
 *              the workspace is first used (e.g. one cudaMemset), and every
 *              call leaves the counters zero again.  The rest needs no
 *              clearing.
 *   Outputs    Always overwritten, never accumulated into.  Inputs and outputs
 *              must not alias.  Calls that share a workspace must not overlap
 *              on the GPU.
 *   Empty      B == 0, H == 0 or T == 0 is valid and enqueues nothing.
 */
#ifndef SAF_H_
#define SAF_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SAF_API __attribute__((visibility("default")))
#else
#define SAF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum saf_status {
    SAF_OK = 0,
    SAF_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, overflow */
    SAF_ERR_UNSUPPORTED = 2, /* d_h != 64, or grad_dtype not 0/1           */
    SAF_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required  */
    SAF_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed        */
    SAF_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up          */
} saf_status;

/* Human-readable name of a status code (static string; never NULL). */
SAF_API const char *saf_status_string(saf_status status);

/* Library version, as major*10000 + minor*100 + patch. */
SAF_API int saf_version(void);

/*
 * Bytes of device workspace that saf_mixed_attn_fwd (is_bwd = 0) or
 * saf_mixed_attn_bwd (is_bwd = 1) needs for this shape, whatever the mask.
 * 0 for an empty problem.  Returns (size_t)-1 for an invalid shape.
 */
SAF_API size_t saf_workspace_size(int B, int H, int T, int d_h, int is_bwd);

/*
 * Row log-normalisers of the replaced heads' patterns (Eq. (3)):
 *   logz[h, i] = log sum_{k<=i} exp(a[h,k] + r[h,i-k])     (natural log)
 * for every h with replaced_mask[h] != 0; other rows of logz are untouched.
 * a, r: [H, T] fp32 device; logz: [H, T] fp32 device output.
 * The values depend only on a and r, never on the batch, so a caller may
 * compute them once and pass them to the forward and backward calls.
 */
SAF_API saf_status saf_replaced_lognorm(const float *a, const float *r,
                                const uint8_t *replaced_mask, int H, int T,
                                float *logz, void *stream);

/*
 * Forward pass (causal prefill) of one mixed-head layer.
 *   q, k, v  [B,H,T,d_h] bf16 in.  q and k rows of replaced heads are not read.
 *   o        [B,H,T,d_h] bf16 out.
 *   lse      [B,H,T] fp32 out: ordinary heads, log sum_{j<=i} exp(q_i.k_j/sqrt(d_h));
 *            replaced heads, log Z(i).  The backward needs it.
 *   a, r     [H,T] fp32 pattern vectors (read for replaced heads only).
 *   logz     [H,T] fp32 from saf_replaced_lognorm, or NULL to compute it
 *            inside the call (into the workspace).
 *   workspace, workspace_bytes: device scratch of at least
 *            saf_workspace_size(B,H,T,d_h,0) bytes, 256-byte aligned.
 */
SAF_API saf_status saf_mixed_attn_fwd(const void *q, const void *k, const void *v,
                              void *o, float *lse,
                              const float *a, const float *r, const float *logz,
                              const uint8_t *replaced_mask,
                              int B, int H, int T, int d_h,
                              void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * Backward pass of one mixed-head layer.
 *   q, k, v, o, dout  [B,H,T,d_h] bf16 in (o and lse as written by the forward).
 *   lse      [B,H,T] fp32 in.
 *   a, r     as in the forward.
 *   logz     [H,T] fp32, or NULL: the replaced heads' log Z is then read from
 *            lse (the forward writes log Z(i) into every batch's lse row of a
 *            replaced head; batch 0's rows are used).
 *   dq, dk, dv  [B,H,T,d_h] out, bf16 (grad_dtype = 0) or fp32 (grad_dtype = 1).
 *            Replaced heads: dq and dk are written as zeros, dv = P^T dout.
 *   workspace: at least saf_workspace_size(B,H,T,d_h,1) bytes, 256-byte aligned.
 * No gradient flows to a, r or logz (they are frozen buffers).
 */
SAF_API saf_status saf_mixed_attn_bwd(const void *q, const void *k, const void *v,
                              const void *o, const void *dout, const float *lse,
                              const float *a, const float *r, const float *logz,
                              const uint8_t *replaced_mask,
                              int B, int H, int T, int d_h,
                              void *dq, void *dk, void *dv, int grad_dtype,
                              void *workspace, size_t workspace_bytes,
                              void *stream);

/*
 * Shared K/V (grouped-query attention): the same layer with k and v holding
 * H_kv heads ([B,H_kv,T,d_h]) shared by groups of H / H_kv consecutive query
 * heads: query head h reads K/V head h / (H / H_kv).  H_kv must divide H
 * (SAF_ERR_INVALID_ARG otherwise); H_kv == H is the plain layer.  Replaced
 * heads read the V head of their group.  In the backward, dk and dv are
 * [B,H_kv,T,d_h]: the gradient of a shared K/V head is the sum over the query
 * heads of its group (computed per query head in fp32 in the workspace, then
 * summed).  The pages measure their attention speed-ups on this variant
 * ("When Can Attention Heads Be Statically Defined?", Table 26); its math is
 * the plain layer with K and V repeated over each group.  Workspace sizes come
 * from saf_workspace_size_gqa.  Not available on the SAF_FORCE_MMA path
 * (SAF_ERR_UNSUPPORTED).
 */
SAF_API size_t saf_workspace_size_gqa(int B, int H, int H_kv, int T, int d_h, int is_bwd);
SAF_API saf_status saf_mixed_attn_fwd_gqa(const void *q, const void *k, const void *v,
                                          void *o, float *lse,
                                          const float *a, const float *r, const float *logz,
                                          const uint8_t *replaced_mask,
                                          int B, int H, int H_kv, int T, int d_h,
                                          void *workspace, size_t workspace_bytes,
                                          void *stream);
SAF_API saf_status saf_mixed_attn_bwd_gqa(const void *q, const void *k, const void *v,
                                          const void *o, const void *dout, const float *lse,
                                          const float *a, const float *r, const float *logz,
                                          const uint8_t *replaced_mask,
                                          int B, int H, int H_kv, int T, int d_h,
                                          void *dq, void *dk, void *dv, int grad_dtype,
                                          void *workspace, size_t workspace_bytes,
                                          void *stream);

/*
 * Allocation-free backward, for callers that cannot pass a workspace: code
 * that may not call cudaMalloc (custom allocators' own callbacks, frameworks
 * that own all device memory), or that has no allocator to draw one from.
 * (The paper has no counterpart: this is an integration aid.)
 *
 * Same arguments and results as saf_mixed_attn_bwd minus the workspace, but
 * a slower path: it runs the warp-level (mma.sync) backward kernels, which
 * need only per-row scratch, not the tensor-core (tcgen05) backward, whose
 * fp32 dQ accumulator of B*H*T*64 floats no fixed array of modest size can
 * hold.  Measured on one B200 at B=8, H=12, T=4096 (3 heads replaced, bf16
 * gradients): 2.81 ms against 0.60 ms for saf_mixed_attn_bwd.  Its
 * scratch (the per-row terms rowsum(dO o O), and the replaced heads' log Z
 * when logz is NULL) lives in one 8 MiB array of device memory inside the
 * library, one per GPU, held from load until process exit.  Limit:
 *     round_up(B*H*T, 64) + (logz == NULL && any head replaced ? H*T : 0)
 *         <= 2,097,152 fp32 values,
 * otherwise SAF_ERR_WORKSPACE is returned and nothing is enqueued.
 * The first call on a device looks up that array's device address (once per
 * device, with the device current); make that first call before any stream
 * capture.  Every call shares the array: calls that overlap on the GPU race
 * and give wrong results.  Nothing in it needs clearing between calls.  It
 * allocates no device memory.
 */
SAF_API saf_status saf_mixed_attn_bwd_noalloc(const void *q, const void *k, const void *v,
                                              const void *o, const void *dout, const float *lse,
                                              const float *a, const float *r, const float *logz,
                                              const uint8_t *replaced_mask,
                                              int B, int H, int T, int d_h,
                                              void *dq, void *dk, void *dv, int grad_dtype,
                                              void *stream);

/*
 * Trainable pattern (the variant of Table 14 of "When Can Attention Heads Be
 * Statically Defined?", where the pattern vectors are trained): the gradients
 * of a loss with output gradient `dout` with respect to a and r, through
 * Eq. (3).  With P the pattern, dP = dout V^T and D(i) = sum_j P(i,j) dP(i,j):
 *   dS(i,j) = P(i,j) (dP(i,j) - D(i)),
 *   da[h,j] = sum over b, i of dS(i,j),   dr[h,d] = sum over b, i - j = d of dS(i,j).
 *   v, dout  [B,H,T,d_h] bf16 in (rows of ordinary heads are not read).
 *   a, r     [H,T] fp32; logz [H,T] from saf_replaced_lognorm, or NULL to
 *            compute it into `workspace` (saf_workspace_size(B,H,T,d_h,0)
 *            bytes, 256-byte aligned; unused when logz is given).
 *   da, dr   [H,T] fp32 out, overwritten; rows of ordinary heads are zero.
 * Sums are accumulated with fp32 atomics (the summation order, and so the
 * last bits, vary from run to run).
 */
SAF_API saf_status saf_replaced_pattern_grad(const void *v, const void *dout,
                                             const float *a, const float *r, const float *logz,
                                             const uint8_t *replaced_mask,
                                             int B, int H, int T, int d_h,
                                             float *da, float *dr,
                                             void *workspace, size_t workspace_bytes,
                                             void *stream);

/*
 * Pattern fitting (section 二.3 of the reading notes for "When Can Attention
 * Heads Be Statically Defined?", with Appendix A.2 as summarised there): for
 * each of n_heads target patterns (e.g. a_hat rows of saf_attn_calibration),
 * the a, r of Eq. (3) minimising the row-wise cross-entropy
 *   L = -(1/T) sum_i sum_{j<=i} A(i,j) log P(i,j),
 * which sees the target only through its column sums and distance sums
 * (Eq. (4)), by `steps` bias-corrected Adam steps (beta1 0.9, beta2 0.999,
 * eps 1e-8, learning rate lr) from a = r = 0; the pages use 400 steps and
 * accept a head at a mean row KL of at most 0.2 nat.
 *   target  [n_heads,T,T] fp32 in: causal, rows summing to 1.
 *   a, r    [n_heads,T] fp32 out;  kl [n_heads] fp32 out: mean row KL(A || P).
 *   workspace: at least saf_fit_workspace_size(n_heads,T) bytes, 256-byte aligned.
 * n_heads <= 256 and T <= 16384 (SAF_ERR_UNSUPPORTED otherwise).  One Adam
 * step is three kernel launches.
 */
SAF_API size_t saf_fit_workspace_size(int n_heads, int T);
SAF_API saf_status saf_fit_pattern(const float *target, int n_heads, int T, int steps, float lr,
                                   float *a, float *r, float *kl,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Calibration statistics (section 二.1 of the reading notes for "When Can
 * Attention Heads Be Statically Defined?"): over N >= 2 calibration sequences
 * run through plain causal softmax attention (every head ordinary), the
 * sample mean of each head's attention matrix and its reconstruction error,
 *   a_hat[h] = (1/N) sum_n A_h^(n)                       [H,T,T] fp32 out
 *   svar[h]  = sum_n ||A_h^(n) - a_hat[h]||_F^2 / ((N-1) T^2)   (Eq. (1)) [H] fp32 out
 * with A^(n) = softmax_causal(q_n k_n^T / sqrt(d_h)); no per-sample T x T
 * matrix is stored.
 *   q, k   [N,H,T,d_h] bf16 in (the N samples as the batch dimension).
 *   lse    [N,H,T] fp32: the row log-sum-exp the forward pass returns for
 *          these inputs (saf_mixed_attn_fwd with no replaced head).
 *   workspace: at least saf_calibration_workspace_size(H,T,d_h) bytes.
 * N < 2 returns SAF_ERR_INVALID_ARG.  Deterministic (fixed-order sums).
 */
SAF_API size_t saf_calibration_workspace_size(int H, int T, int d_h);
SAF_API saf_status saf_attn_calibration(const void *q, const void *k, const float *lse,
                                        int N, int H, int T, int d_h,
                                        float *a_hat, float *svar,
                                        void *workspace, size_t workspace_bytes,
                                        void *stream);

/*
 * Reads (synchronously: waits for `stream`) and clears the device error word
 * that the kernels keep in the first 256 bytes of `workspace` (zero before
 * first use, see Workspace above); the kernels only ever set the word, and
 * this call clears it again.
 * Returns SAF_OK, SAF_ERR_TIMEOUT if a bounded device wait gave up since the
 * last check, SAF_ERR_WORKSPACE for a missing/short workspace, or SAF_ERR_CUDA.
 */
SAF_API saf_status saf_device_status(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Failure-path self-test (the pages have no counterpart): enqueues a kernel
 * whose single wait, on an mbarrier that nothing completes, gives up after
 * limit_cycles SM cycles (1 .. 2^31) and records the time-out in the
 * workspace's error word, exactly as a kernel wait that timed out would; no
 * copy or MMA is in flight, so the device stays usable.  A following
 * saf_device_status returns SAF_ERR_TIMEOUT (and clears the word).
 */
SAF_API saf_status saf_selftest_wait_timeout(void *workspace, size_t workspace_bytes, long long limit_cycles,
                                             void *stream);

/* ------------------------------------------------------------------------
 * Launch accounting and per-kernel timing (for benchmarks and tracing).
 * ------------------------------------------------------------------------ */

/* Kernels enqueued by this library since it was loaded (all threads). */
SAF_API uint64_t saf_launch_count(void);

/*
 * Starts (max_launches > 0) or stops (0) per-kernel timing.  While on, every
 * kernel the library enqueues, up to max_launches, is bracketed by two CUDA
 * events recorded on its stream (host-side event objects created here; no
 * device memory).  Restarting discards earlier records.
 */
SAF_API saf_status saf_profile_enable(int max_launches);

/*
 * Copies up to n timing records (kernel id and milliseconds between the
 * bracketing events) of the current profiling session; waits for those
 * events.  Returns the number of records available, or -1 on a CUDA error.
 */
SAF_API int saf_profile_read(int *kernel_ids, float *ms, int n);

/* Name of a kernel id from saf_profile_read ("?" if unknown). */
SAF_API const char *saf_kernel_name(int kernel_id);

#ifdef __cplusplus
}
#endif

#endif /* SAF_H_ */
