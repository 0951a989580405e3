/*
 * efla.h -- C ABI of the B200 (sm_100a) Exact Flow Linear Attention forward.
 *
 * Method: "Exact Flow Linear Attention: Exact Solution from Continuous-Time
 * Dynamics" (technical summary).  Per head, for t = 1..L:
 *
 *   lambda_t = ||k_t||^2                                     (Methodology 2)
 *   alpha_t  = (1 - exp(-beta_t lambda_t)) / lambda_t        (Methodology 3)
 *   S_t      = (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T
 *                                                            (Methodology 3)
 *   o_t      = S_t^T q_t          (delta-rule readout, after the update)
 *
 * The summary states that this update keeps the delta rule's rank-1 algebra
 * and therefore its WY/UT chunkwise parallel form (Methodology 3, last
 * paragraph); efla_chunk_fwd evaluates that form.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees or retains them past the call.  The library allocates no
 *    device memory: scratch space comes from the caller's workspace.
 *  - Layouts are dense row-major (C order):
 *        q, k : [B, H, L, dk]      v, o : [B, H, L, dv]      beta : [B, H, L]
 *        S0, S_final, S : [B, H, dk, dv]  (fp32; row i is key dimension i)
 *        alpha : [B, H, L]  (fp32)
 *    q, k, v and beta share the element type `dt`; o has the element type
 *    `o_dt` (fp32 keeps the fp32 accumulator; bf16 rounds it).
 *  - Alignment: fp32 state pointers (S, S0, S_final) and, for
 *    efla_chunk_fwd, q, k, v and o must be 16-byte aligned (they are read
 *    with 16-byte vector or bulk-tensor copies); every other pointer must be
 *    aligned to its element size.  Violations return EFLA_ERR_ALIGN.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *    call is asynchronous with respect to the host: it checks its arguments on
 *    the host, enqueues kernels on `stream` and returns.  Nothing here
 *    synchronises the device.
 *  - Errors are returned as efla_status; no call aborts or throws.  Argument
 *    errors are detected before anything is enqueued.  EFLA_ERR_CUDA reports a
 *    failed launch (cudaGetLastError after the launch).  Faults that happen
 *    later on the device surface through the CUDA runtime as usual.
 *  - Input values are not inspected: NaN/Inf propagate, negative beta is
 *    evaluated by the same formula.
 *  - No scaling or normalisation is applied to q or k (lambda is the raw
 *    squared norm).
 */
#ifndef EFLA_H_
#define EFLA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EFLA_OK = 0,
    EFLA_ERR_NULL = 1,        /* a required pointer is NULL */
    EFLA_ERR_SHAPE = 2,       /* a size is negative, zero where not allowed, or too large */
    EFLA_ERR_DTYPE = 3,       /* unknown efla_dtype */
    EFLA_ERR_UNSUPPORTED = 4, /* valid but not implemented (e.g. dk > 256) */
    EFLA_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
    EFLA_ERR_TIMEOUT = 6,     /* a bounded device-side wait gave up */
    EFLA_ERR_WORKSPACE = 7,   /* workspace missing or smaller than the query said */
    EFLA_ERR_ALIGN = 8,       /* a pointer is not aligned as required */
    EFLA_ERR_TOO_LARGE = 9,   /* sizes need more than the fixed scratch of efla_chunk_fwd_noalloc */
    EFLA_ERR_RULE = 10        /* unknown efla_rule */
} efla_status;

typedef enum {
    EFLA_F32 = 0,  /* float32 inputs/outputs; all arithmetic in fp32 */
    EFLA_BF16 = 1  /* bfloat16 inputs/outputs; fp32 state and accumulation */
} efla_dtype;

/*
 * Update rule.  Both integrate the same per-token ODE, dS/dtau = -k k^T S + k v^T
 * over an interval of length beta_t (Methodology 1), and share every kernel,
 * layout and error; they differ in the coefficient alpha_t of the rank-1 update
 * S_t = (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T:
 *   EFLA_RULE_EXACT -- the exact flow, alpha_t = (1 - e^{-beta_t lambda_t}) /
 *                      lambda_t (Methodology 3).  The method; the default of
 *                      every entry point without a rule argument.
 *   EFLA_RULE_EULER -- one explicit Euler step of the ODE, alpha_t = beta_t: the
 *                      delta rule (DeltaNet), which the summary identifies as
 *                      that Euler step (Key Contributions) and compares against.
 */
typedef enum {
    EFLA_RULE_EXACT = 0,
    EFLA_RULE_EULER = 1
} efla_rule;

/* Human-readable name of a status code (static string, never NULL). */
const char *efla_status_str(int status);

/* ABI version: major*10000 + minor*100 + patch. */
int efla_version(void);

/*
 * efla_alpha -- per-token effective coefficient (Methodology 2 and 3).
 *
 *   alpha[b,h,t] = -expm1(-beta*lambda)/lambda,  lambda = sum_i k[b,h,t,i]^2,
 *   and alpha = beta when beta*lambda is 0 (the lambda -> 0 limit).
 *
 * k: [B,H,L,dk] of type dt; beta: [B,H,L] of type dt; alpha: [B,H,L] fp32.
 * Sizes: B,H,L >= 0 (0 tokens is a no-op), 1 <= dk <= 256.
 */
efla_status efla_alpha(const void *k, const void *beta, float *alpha,
                       int B, int H, int L, int dk, efla_dtype dt, void *stream);

/* efla_alpha under a chosen update rule (alpha = beta for EFLA_RULE_EULER).
 * EFLA_ERR_RULE for an unknown rule; otherwise as efla_alpha. */
efla_status efla_alpha_rule(const void *k, const void *beta, float *alpha,
                            int B, int H, int L, int dk, efla_dtype dt, efla_rule rule,
                            void *stream);

/*
 * Bytes of device workspace efla_chunk_fwd needs for these sizes (0 when the
 * selected kernels need none).  The same arguments must be passed to
 * efla_chunk_fwd.  Returns 0 for invalid sizes as well (efla_chunk_fwd then
 * reports the error).
 */
size_t efla_chunk_fwd_workspace_size(int B, int H, int L, int dk, int dv, int chunk,
                                     efla_dtype dt, efla_dtype o_dt);

/*
 * efla_chunk_fwd -- the whole forward pass in the WY/UT chunkwise form
 * (Methodology 3: rank-1 updates keep the delta rule's chunkwise
 * parallelism).  For every head (b, h), chunks of `chunk` tokens are folded
 * into the carried state; the last chunk may be partial (L need not be a
 * multiple of chunk).
 *
 *   q, k  : [B,H,L,dk]  (dt)          v : [B,H,L,dv] (dt)     beta : [B,H,L] (dt)
 *   S0    : [B,H,dk,dv] fp32 initial state, or NULL for zeros
 *   o     : [B,H,L,dv]  (o_dt) output, o_t = S_t^T q_t
 *   S_final : [B,H,dk,dv] fp32 state after token L, or NULL to skip
 *   chunk : 16, 32 or 64 (tokens per WY/UT block)
 *   workspace, workspace_bytes : caller-owned device scratch of at least
 *       efla_chunk_fwd_workspace_size(...) bytes (may be NULL when that is 0);
 *       its contents on entry are ignored and on exit unspecified.
 * S0 and S_final may alias (in-place state carry).  o must not alias inputs.
 * Sizes: B,H >= 1, L >= 0, 1 <= dk,dv <= 128.  L == 0 copies S0 to S_final.
 * Calls on the same workspace must be ordered on one stream.
 * Range: with bf16 inputs, dk and dv in {64, 128} and chunk 64, the products
 * run on the tensor cores with fp16 operands and fp32 accumulation: q, k and v
 * are converted to fp16 (exact for bf16 values of magnitude 2^-14 .. 65504),
 * and so are the intermediates u_t = alpha_t (v_t - S_{t-1}^T k_t) and the
 * state's operand copy.  A value beyond fp16's largest finite magnitude,
 * 65504, in the inputs or in those intermediates becomes inf and the outputs
 * inf or NaN, with status EFLA_OK (input values are not inspected).  fp32
 * inputs take the SIMT path, which has no such limit.
 */
efla_status efla_chunk_fwd(const void *q, const void *k, const void *v, const void *beta,
                           const float *S0, void *o, float *S_final,
                           int B, int H, int L, int dk, int dv, int chunk, efla_dtype dt,
                           efla_dtype o_dt, void *workspace, size_t workspace_bytes,
                           void *stream);

/* efla_chunk_fwd under a chosen update rule: the same kernels, workspace and
 * paths, with alpha = beta for EFLA_RULE_EULER.  EFLA_ERR_RULE for an unknown
 * rule; otherwise as efla_chunk_fwd. */
efla_status efla_chunk_fwd_rule(const void *q, const void *k, const void *v, const void *beta,
                                const float *S0, void *o, float *S_final,
                                int B, int H, int L, int dk, int dv, int chunk, efla_dtype dt,
                                efla_dtype o_dt, efla_rule rule, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * efla_chunk_fwd_gated -- the gated form: a per-token decay g_t on the carried
 * state,
 *
 *   S_t = g_t (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T,  o_t = S_t^T q_t.
 *
 * The summary names Gated DeltaNet among its baselines (Experimental Results)
 * without printing its equations; this is Gated DeltaNet's placement of the
 * gate, on the previous state's transition, with EFLA's coefficient (or beta
 * under EFLA_RULE_EULER, which is then Gated DeltaNet's own update).  g_t = 1
 * is efla_chunk_fwd_rule; k_t = 0 is a pure decay S_t = g_t S_{t-1}.
 *
 *   g : [B,H,L] (dt), the decay of each token, expected in (0, 1] (not
 *       checked: the chunkwise form takes its logarithm, so g <= 0 gives NaN).
 * The chunkwise form carries the decays as cumulative logarithms within each
 * chunk, so every factor it applies is a decay of at most 1.  Everything else
 * (arguments, layouts, workspace, sizes, errors) is as efla_chunk_fwd_rule;
 * the workspace query is efla_chunk_fwd_workspace_size.  EFLA_ERR_NULL when g
 * is NULL and L > 0.
 */
efla_status efla_chunk_fwd_gated(const void *q, const void *k, const void *v, const void *beta,
                                 const void *g, const float *S0, void *o, float *S_final,
                                 int B, int H, int L, int dk, int dv, int chunk, efla_dtype dt,
                                 efla_dtype o_dt, efla_rule rule, void *workspace,
                                 size_t workspace_bytes, void *stream);

/*
 * efla_chunk_fwd_noalloc -- the same forward pass as efla_chunk_fwd for callers
 * that cannot allocate device memory.  The paper has no counterpart: this is
 * an interface for embedding, not part of the method.
 *
 * Who cannot allocate: code that is handed only its input and output buffers,
 * with no allocator and no workspace (for example an operator plugin inside a
 * runtime whose memory pool owns all device memory), and latency-critical
 * loops that must not call cudaMalloc, which can synchronise the device and
 * can fail at run time when memory is short.  Such callers cannot provide the
 * workspace efla_chunk_fwd asks for.
 *
 * Scratch: instead of a caller workspace, the tensor-core path keeps its
 * per-chunk T*diag(alpha) tiles (8 KiB per 64-token chunk of each head) in one
 * fixed array of EFLA_NOALLOC_SCRATCH_BYTES inside the library's device code.
 * Every GPU on which the library's kernels are loaded holds that memory until
 * the process exits.  Where efla_chunk_fwd would cut the sequence into
 * segments (few heads, long sequences) it also keeps their states there; when
 * those do not fit beside the tiles, this call runs the one-pass form instead
 * (same results, fewer SMs busy).  Sizes whose tiles alone need more --
 * B*H*ceil(L/64) > 4096 chunks on the tensor-core path -- return
 * EFLA_ERR_TOO_LARGE before anything is enqueued.  Sizes served by the SIMT
 * path need no scratch at all.
 *
 * Set-up: the first call on a device looks up the array's device address once
 * for that device (it must be the current device); make that first call before
 * any stream capture.
 *
 * Sharing: every call uses the same array, which keeps the last call's
 * contents.  Nothing in it has to start at zero: each call writes every byte it
 * later reads.  Calls whose GPU work overlaps (different streams with no
 * ordering between them, on the same device) race on the array and give wrong
 * results; order them.
 *
 * Arguments, layouts, sizes and the remaining errors are those of
 * efla_chunk_fwd.  Allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library call.
 */
#define EFLA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
efla_status efla_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *beta,
                                   const float *S0, void *o, float *S_final,
                                   int B, int H, int L, int dk, int dv, int chunk, efla_dtype dt,
                                   efla_dtype o_dt, void *stream);

/*
 * efla_recurrent_step -- one decode token per head: the update rule of
 * Methodology 3 applied once, S updated in place, then o = S^T q.
 *
 *   q, k : [B,H,dk] (dt)   v : [B,H,dv] (dt)   beta : [B,H] (dt)
 *   S    : [B,H,dk,dv] fp32, read and overwritten with the new state
 *   o    : [B,H,dv] (o_dt)
 * Sizes: B,H >= 1, 1 <= dk <= 256, 1 <= dv <= 256.
 */
efla_status efla_recurrent_step(const void *q, const void *k, const void *v, const void *beta,
                                float *S, void *o, int B, int H, int dk, int dv,
                                efla_dtype dt, efla_dtype o_dt, void *stream);

/* efla_recurrent_step under a chosen update rule (alpha = beta for
 * EFLA_RULE_EULER).  EFLA_ERR_RULE for an unknown rule; otherwise as
 * efla_recurrent_step. */
efla_status efla_recurrent_step_rule(const void *q, const void *k, const void *v,
                                     const void *beta, float *S, void *o, int B, int H, int dk,
                                     int dv, efla_dtype dt, efla_dtype o_dt, efla_rule rule,
                                     void *stream);

/*
 * efla_recurrent_step_gated -- one decode token of the gated form (see
 * efla_chunk_fwd_gated): S <- g (I - alpha k k^T) S + alpha k v^T in place,
 * then o = S^T q.  g : [B,H] (dt).  EFLA_ERR_NULL when g is NULL; otherwise as
 * efla_recurrent_step_rule.
 */
efla_status efla_recurrent_step_gated(const void *q, const void *k, const void *v,
                                      const void *beta, const void *g, float *S, void *o, int B,
                                      int H, int dk, int dv, efla_dtype dt, efla_dtype o_dt,
                                      efla_rule rule, void *stream);

/*
 * efla_state_affine -- S_out = P S_in + H for every head, in fp32.  No counterpart
 * on the pages as a call: it chains the affine state maps of sequence stretches
 * (a stretch of tokens maps the state as S_out = P S_in + H, where P is the
 * product of the stretch's transitions I - alpha k k^T and H its state from zero,
 * by the update rule of Methodology 3), so that stretches held by different GPUs
 * can be run side by side and then given their true starting states.
 *
 *   P     : [B,H,dk,dk] fp32     S_in, H, S_out : [B,H,dk,dv] fp32
 * S_in or H may be NULL (zero).  S_out may alias S_in (not P or H).
 * Sizes: B,H >= 1, 1 <= dk,dv <= 256.  Pointers aligned to 4 bytes.
 * P for a stretch is the S_final of efla_chunk_fwd run over it from S0 = I with
 * v = 0 (dv = dk); H is its S_final from S0 = NULL.
 */
efla_status efla_state_affine(const float *P, const float *S_in, const float *H, float *S_out,
                              int B, int Hh, int dk, int dv, void *stream);

/*
 * efla_bwd -- gradients of efla_chunk_fwd_rule (the same function of the inputs:
 * the chunkwise form equals the token recurrence): given dO = dL/do and dS_final
 * = dL/dS_final (NULL = 0), writes dq, dkey, dval (the gradients with respect to
 * q, k, v), dbeta and dS0 (NULL to skip).  Reverse mode through the update of
 * Methodology 3 (or the Euler step under EFLA_RULE_EULER), including the
 * dependence of alpha on ||k||^2 and beta.  The pages give no backward pass; its
 * arithmetic is derived from the forward.
 *
 *   q, k : [B,H,L,dk] (dt)   v : [B,H,L,dv] (dt)   beta : [B,H,L] (dt)
 *   S0 : [B,H,dk,dv] fp32 or NULL        dO : [B,H,L,dv] fp32
 *   dq, dkey : [B,H,L,dk] fp32   dval : [B,H,L,dv] fp32   dbeta : [B,H,L] fp32
 *   dS0 : [B,H,dk,dv] fp32 or NULL
 *   workspace : efla_bwd_workspace_size(B,H,L,dk,dv) bytes, caller-owned scratch,
 *               16-byte aligned
 * Sizes: B,H >= 1, L >= 0, 1 <= dk,dv <= 128.  Other pointers aligned to their
 * element.  Two paths, chosen per head on the device:
 *   - tensor cores: with bf16 inputs at the sizes efla_chunk_fwd runs on tensor
 *     cores (chunk 64; dk, dv in {64, 128}) and q, k, v, dO and S0 16-byte
 *     aligned, heads whose largest ||k||^2 is at most 16 and whose alpha are all
 *     positive and span at most a factor of 1024.  The tensor-core forward runs
 *     first and saves every token's alpha r and the state after every 64 tokens
 *     (fp16); a reverse chain over the chunks then gives every token's dU' and the
 *     state gradient after every chunk, and every chunk's dq, dkey, dval and dbeta
 *     follow in parallel, with fp16 operands and fp32 accumulation (the products'
 *     precision of the forward; dO is rounded to fp16 for them, so |dO| must stay
 *     below 65504).
 *   - CUDA cores (every other head, and fp32 inputs): fp32 throughout; one CTA
 *     takes one head and 16 of its state columns and walks the sequence twice
 *     (forward, then reverse); dq, dkey and dbeta are sums over the columns, and
 *     a second kernel adds the column blocks' shares in a fixed order.
 * Both give results that do not depend on scheduling.  The workspace size covers
 * the tensor-core path whenever the sizes allow it.
 * EFLA_ERR_ALIGN: a misaligned pointer.  EFLA_ERR_WORKSPACE: the workspace is
 * missing or too small.
 */
size_t efla_bwd_workspace_size(int B, int H, int L, int dk, int dv);
efla_status efla_bwd(const void *q, const void *k, const void *v, const void *beta,
                     const float *S0, const float *dO, const float *dS_final, float *dq,
                     float *dkey, float *dval, float *dbeta, float *dS0, int B, int H, int L,
                     int dk, int dv, efla_dtype dt, efla_rule rule, void *workspace,
                     size_t workspace_bytes, void *stream);

/*
 * A training step without the backward's second forward (the forward's own values,
 * kept from the step's forward to its backward):
 *
 * efla_bwd_kept_size -- bytes of the kept buffer for these sizes: the tensor-core
 * forward's T diag(alpha) tiles (with the sequence segments' states where it cuts the
 * sequence), every token's alpha r and the state after every 64 tokens (fp16); 0 where
 * the backward does not run on tensor cores (dk or dv not in {64, 128}, L = 0).
 *
 * efla_chunk_fwd_keep -- efla_chunk_fwd_rule at chunk 64 (same arguments; o and
 * S_final bit for bit the same) that also fills `kept` (efla_bwd_kept_size bytes,
 * 16-byte aligned, caller-owned until the matching efla_bwd_kept).  bf16 inputs only,
 * q, k, v, o, S0 and S_final 16-byte aligned; EFLA_ERR_UNSUPPORTED for sizes or dtypes
 * without a kept buffer (use efla_chunk_fwd_rule and efla_bwd); EFLA_ERR_WORKSPACE for
 * a missing or short `kept`.
 *
 * efla_bwd_kept -- efla_bwd (same arguments and results, its own workspace as
 * efla_bwd's) for a `kept` buffer that efla_chunk_fwd_keep filled for the same q, k,
 * v, beta, S0, sizes and rule, unchanged since: the tensor-core heads read it instead
 * of running the forward again (heads that walk on CUDA cores ignore it).  A buffer not
 * filled that way gives wrong gradients; the library cannot tell.
 */
size_t efla_bwd_kept_size(int B, int H, int L, int dk, int dv);
efla_status efla_chunk_fwd_keep(const void *q, const void *k, const void *v, const void *beta,
                                const float *S0, void *o, float *S_final, int B, int H, int L,
                                int dk, int dv, efla_dtype dt, efla_dtype o_dt, efla_rule rule,
                                void *kept, size_t kept_bytes, void *stream);
efla_status efla_bwd_kept(const void *q, const void *k, const void *v, const void *beta,
                          const float *S0, const float *dO, const float *dS_final, float *dq,
                          float *dkey, float *dval, float *dbeta, float *dS0, int B, int H, int L,
                          int dk, int dv, efla_dtype dt, efla_rule rule, const void *kept,
                          size_t kept_bytes, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Reads and clears the library's device error word after synchronising
 * `stream`.  Kernels that wait on barriers do so with bounded spins; when a
 * wait gives up the kernel records it here and exits, leaving the context
 * usable.  Returns EFLA_OK, EFLA_ERR_TIMEOUT, or EFLA_ERR_CUDA if the
 * synchronisation itself failed.
 */
efla_status efla_last_device_error(void *stream);

/*
 * efla_selftest_bounded_wait -- a test hook for the failure path (no counterpart
 * on the pages): launches one small kernel whose single wait is on an mbarrier
 * that nothing arrives on, bounded by budget_cycles (1 .. 2e9 SM cycles, about
 * a second at most).  When the bound runs out the kernel records a timeout in
 * the device error word, exactly as the forward kernels do when a wait gives up,
 * and returns; nothing faults or hangs and the context stays usable.  A later
 * efla_last_device_error then reports EFLA_ERR_TIMEOUT (and clears the word).
 * EFLA_ERR_SHAPE for a budget outside its range.
 */
efla_status efla_selftest_bounded_wait(long long budget_cycles, void *stream);

/*
 * Which chunk-forward kernels the library selects for these sizes on the current
 * device: 0 = SIMT fp32 path, 1 = tensor-core (tcgen05) path, 2 = tensor-core path
 * with the sequence cut into segments that run in parallel (few heads, long
 * sequences: each segment maps the state affinely, S_out = P S_in + H, so the
 * segments' maps are computed side by side, chained, and the segments rerun from
 * their true starting states).  Without a usable device, 2 is never reported.
 * For tests and tools.
 */
int efla_chunk_fwd_path(int B, int H, int L, int dk, int dv, int chunk, efla_dtype dt,
                        efla_dtype o_dt);

/*
 * Number of kernels this library has enqueued since it was loaded (a
 * host-side counter, incremented per launch; thread-safe).  Lets a caller
 * count the library's launches inside a timed region.
 */
unsigned long long efla_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* EFLA_H_ */
