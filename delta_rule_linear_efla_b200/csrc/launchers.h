// launchers.h -- host-side launch functions of the EFLA kernels (internal to
// the library; the public ABI is include/efla.h).  Each returns a
// cudaError_t from cudaGetLastError() after its launches.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>

namespace efla {

// Host-side count of kernels enqueued by the library (efla_kernel_launches).
void count_launches(unsigned n);

// Per-token alpha (fused norm + closed-form coefficient).  is_bf16 selects the
// element type of k and beta.
// euler: the coefficient is beta (the delta rule's explicit Euler step) instead of the exact flow's.
cudaError_t launch_alpha(const void *k, const void *beta, float *alpha, long long ntok, int dk,
                         bool is_bf16, bool euler, cudaStream_t s);

// SIMT fp32 chunkwise forward: WY/UT per chunk, state carried in fp32.
// Any dk, dv <= 128 and chunk <= 64.
// o_bf16 selects the output element type (fp32 or bf16).  g: the gated form's per-token decay
// ([B,H,L], the input type) or NULL for none.
cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const void *beta,
                              const void *g, const float *S0, void *o, float *S_final, int B,
                              int H, int L, int dk, int dv, int chunk, bool is_bf16, bool o_bf16,
                              bool euler, cudaStream_t s);

// Recurrent single-token step per head (decode), S updated in place.  g: the gated form's
// per-head decay of this token ([BH], the input type), or NULL for none.
cudaError_t launch_decode(const void *q, const void *k, const void *v, const void *beta,
                          const void *g, float *S, void *o, int BH, int dk, int dv, bool is_bf16,
                          bool o_bf16, bool euler, cudaStream_t s);

// S_out = P S_in + H per head (fp32); S_in and H may be NULL (zero); S_out may alias S_in.
cudaError_t launch_state_affine(const float *P, const float *S_in, const float *H, float *S_out,
                                int BH, int dk, int dv, cudaStream_t s);

// Backward pass (SIMT, one CTA per head): gradients of the forward given dO and dS_final.
size_t bwd_workspace_bytes(int B, int H, int L, int dk, int dv);
cudaError_t launch_bwd(const void *q, const void *k, const void *v, const void *beta,
                       const float *S0, const float *dO, const float *dSL, float *dq, float *dkey,
                       float *dval, float *dbeta, float *dS0, int B, int H, int L, int dk, int dv,
                       bool is_bf16, bool euler, void *ws, cudaStream_t s, const void *kept = nullptr);
// A kept buffer (bwd_kept_bytes, 0 where the tensor-core backward does not run) holds the
// tensor-core forward's workspace (its Ta tiles), every token's u and the state after every
// chunk; bwd_kept_regions gives the three (false for sizes and dtypes the tensor-core backward
// does not take).  launch_bwd with `kept` reads them from there instead of running that forward
// again: launch_chunk_tc_keep must have filled them for the same inputs.
size_t bwd_kept_bytes(int B, int H, int L, int dk, int dv);
bool bwd_kept_regions(int B, int H, int L, int dk, int dv, bool is_bf16, void *kept, void **tc_ws, __half **u,
                      __half **ck);

// Tensor-core (tcgen05) chunkwise forward, bf16 only.
bool tc_supported(int B, int H, int L, int dk, int dv, int chunk, bool is_bf16);
// allow_segments = false keeps the one-pass form (no sequence segments, whose state buffers
// the workspace would otherwise have to hold).
size_t tc_workspace_bytes(int B, int H, int L, int dk, int dv, int chunk, bool allow_segments = true);
int tc_segments(int B, int H, int L, int dk, int dv);  // sequence segments the launch uses (1: none)
// g: the gated form's per-token decay ([B,H,L], bf16) or NULL.
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const void *beta,
                            const float *S0, void *o, float *S_final, int B, int H, int L,
                            int dk, int dv, int chunk, bool o_bf16, bool euler, void *ws,
                            cudaStream_t s, bool allow_segments = true, const void *g = nullptr);

// efla_chunk_fwd_rule with the choice of allowing sequence segments (the public entry points
// allow them); returns an efla_status.
// g: the gated form's per-token decay ([B,H,L], input type) or NULL.
int chunk_fwd_entry(const void *q, const void *k, const void *v, const void *beta, const float *S0,
                    void *o, float *S_final, int B, int H, int L, int dk, int dv, int chunk, int dt,
                    int o_dt, int rule, void *workspace, size_t workspace_bytes, void *stream,
                    bool allow_segments, const void *g);
// The tensor-core forward without outputs, saving what the backward needs instead: every
// token's u_t = a_t (v_t - S_{t-1}^T k_t) into u_out [B*H][L][dv] and the state after every
// 64-token chunk into ck_out [B*H][ceil(L/64)][dk][dv], rounded to fp16 (the backward's products
// take them as fp16 operands).  Same sizes as launch_chunk_tc, chunk 64, and the same workspace.
cudaError_t launch_chunk_tc_save(const void *q, const void *k, const void *v, const void *beta,
                                 const float *S0, int B, int H, int L, int dk, int dv, bool euler,
                                 void *ws, __half *u_out, __half *ck_out, cudaStream_t s);
// The tensor-core forward writing o and S_final as launch_chunk_tc (chunk 64, ungated) and also
// keeping u_out and ck_out as launch_chunk_tc_save does (ws: the workspace of that call).
cudaError_t launch_chunk_tc_keep(const void *q, const void *k, const void *v, const void *beta,
                                 const float *S0, void *o, float *S_final, int B, int H, int L, int dk,
                                 int dv, bool o_bf16, bool euler, void *ws, __half *u_out, __half *ck_out,
                                 cudaStream_t s);
// The backward on tensor cores for the heads the saved-forward gate lets through (bf16, chunk
// 64, dk and dv in {64, 128}, q, k, dO and S0 16-byte aligned): dO to fp16, the reverse chain
// over the chunks (dU' of every token and the state gradient after every chunk), then every
// chunk's dq, dk, dv and dbeta in parallel; dS0 from the chain.  coef: the coefficient
// kernel's per-token float4 pairs; hs: its per-head gate statistics; u_saved, ck_saved, ta: the
// saving forward's outputs and Ta tiles.  Workspace: bwd_tc_workspace_bytes; dO16_ready: its
// head already holds dO rounded to fp16 ([BH][L][dv]), so the conversion kernel is skipped.
size_t bwd_tc_workspace_bytes(int B, int H, int L, int dk, int dv);
cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const float *S0, const float *dO,
                          const float *dSL, const void *coef, const int *hs, const __half *u_saved,
                          const __half *ck_saved, const void *ta, float *dq, float *dkey, float *dval,
                          float *dbeta, float *dS0, int B, int H, int L, int dk, int dv, void *ws,
                          cudaStream_t s, bool dO16_ready);
cudaError_t bwd_tc_read_and_clear_error(unsigned int *out);
// A kernel whose one bounded wait runs out (nothing arrives): records a timeout, then returns.
cudaError_t launch_selftest_wait(long long budget_cycles, cudaStream_t s);
// Device error word of the tensor-core kernels (bounded waits): read and clear.
cudaError_t tc_read_and_clear_error(unsigned int *out, cudaStream_t s);

}  // namespace efla
