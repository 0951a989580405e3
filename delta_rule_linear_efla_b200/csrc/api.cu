// api.cu -- extern "C" entry points declared in include/efla.h.
//
// Each entry point validates its arguments on the host, selects kernels and
// enqueues them on the caller's stream.  No device memory is allocated here.
#include <stdint.h>

#include <atomic>

#include "../../include/efla.h"
#include "launchers.h"

namespace efla {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace efla

namespace {

bool aligned16(const void *p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_elem(const void *p, efla_dtype dt) {
    const uintptr_t m = dt == EFLA_BF16 ? 1u : 3u;
    return p == nullptr || (reinterpret_cast<uintptr_t>(p) & m) == 0;
}

efla_status from_cuda(cudaError_t e) { return e == cudaSuccess ? EFLA_OK : EFLA_ERR_CUDA; }

bool chunk_ok(int c) { return c == 16 || c == 32 || c == 64; }

bool dtype_ok(efla_dtype d) { return d == EFLA_F32 || d == EFLA_BF16; }

bool rule_ok(efla_rule r) { return r == EFLA_RULE_EXACT || r == EFLA_RULE_EULER; }

}  // namespace

extern "C" {

const char *efla_status_str(int status) {
    switch (status) {
        case EFLA_OK: return "ok";
        case EFLA_ERR_NULL: return "null pointer";
        case EFLA_ERR_SHAPE: return "invalid size";
        case EFLA_ERR_DTYPE: return "invalid dtype";
        case EFLA_ERR_UNSUPPORTED: return "unsupported size or chunk";
        case EFLA_ERR_CUDA: return "CUDA error";
        case EFLA_ERR_TIMEOUT: return "device wait timed out";
        case EFLA_ERR_WORKSPACE: return "workspace missing or too small";
        case EFLA_ERR_ALIGN: return "pointer not aligned as required";
        case EFLA_ERR_TOO_LARGE: return "sizes exceed the fixed scratch of efla_chunk_fwd_noalloc";
        case EFLA_ERR_RULE: return "unknown update rule";
        default: return "unknown status";
    }
}

int efla_version(void) { return 100; /* 0.1.0 */ }

efla_status efla_alpha_rule(const void *k, const void *beta, float *alpha, int B, int H, int L,
                            int dk, efla_dtype dt, efla_rule rule, void *stream) {
    if (!rule_ok(rule)) return EFLA_ERR_RULE;
    if (dt != EFLA_F32 && dt != EFLA_BF16) return EFLA_ERR_DTYPE;
    if (B < 0 || H < 0 || L < 0 || dk < 1) return EFLA_ERR_SHAPE;
    if (dk > 256) return EFLA_ERR_UNSUPPORTED;
    const long long ntok = (long long)B * H * L;
    if (ntok == 0) return EFLA_OK;
    if (!k || !beta || !alpha) return EFLA_ERR_NULL;
    if (!aligned_elem(k, dt) || !aligned_elem(beta, dt) || !aligned_elem(alpha, EFLA_F32))
        return EFLA_ERR_ALIGN;
    return from_cuda(efla::launch_alpha(k, beta, alpha, ntok, dk, dt == EFLA_BF16,
                                        rule == EFLA_RULE_EULER, (cudaStream_t)stream));
}

efla_status efla_alpha(const void *k, const void *beta, float *alpha, int B, int H, int L, int dk,
                       efla_dtype dt, void *stream) {
    return efla_alpha_rule(k, beta, alpha, B, H, L, dk, dt, EFLA_RULE_EXACT, stream);
}

int efla_chunk_fwd_path(int B, int H, int L, int dk, int dv, int chunk, efla_dtype dt,
                        efla_dtype o_dt) {
    (void)o_dt;
    if (!efla::tc_supported(B, H, L, dk, dv, chunk, dt == EFLA_BF16)) return 0;
    return efla::tc_segments(B, H, L, dk, dv) >= 3 ? 2 : 1;
}

size_t efla_chunk_fwd_workspace_size(int B, int H, int L, int dk, int dv, int chunk,
                                     efla_dtype dt, efla_dtype o_dt) {
    if (B < 1 || H < 1 || L < 0 || dk < 1 || dv < 1 || !chunk_ok(chunk)) return 0;
    if (!dtype_ok(dt) || !dtype_ok(o_dt)) return 0;
    if (efla::tc_supported(B, H, L, dk, dv, chunk, dt == EFLA_BF16))
        return efla::tc_workspace_bytes(B, H, L, dk, dv, chunk);
    return 0;
}

}  // extern "C"

namespace efla {
int chunk_fwd_entry(const void *q, const void *k, const void *v, const void *beta, const float *S0,
                    void *o, float *S_final, int B, int H, int L, int dk, int dv, int chunk, int dt_i,
                    int o_dt_i, int rule_i, void *workspace, size_t workspace_bytes, void *stream,
                    bool allow_segments, const void *g) {
    const efla_dtype dt = (efla_dtype)dt_i, o_dt = (efla_dtype)o_dt_i;
    const efla_rule rule = (efla_rule)rule_i;
    if (!rule_ok(rule)) return EFLA_ERR_RULE;
    const bool euler = rule == EFLA_RULE_EULER;
    if (!dtype_ok(dt) || !dtype_ok(o_dt)) return EFLA_ERR_DTYPE;
    if (B < 1 || H < 1 || L < 0 || dk < 1 || dv < 1) return EFLA_ERR_SHAPE;
    if ((long long)B * H > 0x7fffffffLL || (long long)B * H * L > (1LL << 40)) return EFLA_ERR_SHAPE;
    if (dk > 128 || dv > 128 || !chunk_ok(chunk)) return EFLA_ERR_UNSUPPORTED;
    if (L > 0 && (!q || !k || !v || !beta || !o)) return EFLA_ERR_NULL;
    if (!aligned_elem(g, dt)) return EFLA_ERR_ALIGN;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned_elem(beta, dt) ||
        !aligned16(S0) || !aligned16(o) || !aligned16(S_final))
        return EFLA_ERR_ALIGN;
    const bool bf16 = dt == EFLA_BF16, o_bf16 = o_dt == EFLA_BF16;
    cudaStream_t s = (cudaStream_t)stream;
    if (L == 0) {
        if (!S_final) return EFLA_OK;
        const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
        if (S0 == S_final) return EFLA_OK;
        return from_cuda(S0 ? cudaMemcpyAsync(S_final, S0, bytes, cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(S_final, 0, bytes, s));
    }
    if (efla::tc_supported(B, H, L, dk, dv, chunk, bf16)) {
        const size_t need = efla::tc_workspace_bytes(B, H, L, dk, dv, chunk, allow_segments);
        if (need > 0 && (!workspace || workspace_bytes < need)) return EFLA_ERR_WORKSPACE;
        if (!aligned16(workspace)) return EFLA_ERR_ALIGN;
        return from_cuda(efla::launch_chunk_tc(q, k, v, beta, S0, o, S_final, B, H, L, dk, dv,
                                               chunk, o_bf16, euler, workspace, s, allow_segments, g));
    }
    return from_cuda(efla::launch_chunk_simt(q, k, v, beta, g, S0, o, S_final, B, H, L, dk, dv,
                                             chunk, bf16, o_bf16, euler, s));
}
}  // namespace efla

extern "C" {

efla_status efla_chunk_fwd_rule(const void *q, const void *k, const void *v, const void *beta,
                                const float *S0, void *o, float *S_final, int B, int H, int L,
                                int dk, int dv, int chunk, efla_dtype dt, efla_dtype o_dt,
                                efla_rule rule, void *workspace, size_t workspace_bytes,
                                void *stream) {
    return (efla_status)efla::chunk_fwd_entry(q, k, v, beta, S0, o, S_final, B, H, L, dk, dv, chunk, dt,
                                              o_dt, rule, workspace, workspace_bytes, stream, true,
                                              nullptr);
}

efla_status efla_chunk_fwd_gated(const void *q, const void *k, const void *v, const void *beta,
                                 const void *g, const float *S0, void *o, float *S_final, int B,
                                 int H, int L, int dk, int dv, int chunk, efla_dtype dt,
                                 efla_dtype o_dt, efla_rule rule, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    if (L > 0 && !g) return EFLA_ERR_NULL;
    return (efla_status)efla::chunk_fwd_entry(q, k, v, beta, S0, o, S_final, B, H, L, dk, dv, chunk, dt,
                                              o_dt, rule, workspace, workspace_bytes, stream, true, g);
}

efla_status efla_chunk_fwd(const void *q, const void *k, const void *v, const void *beta,
                           const float *S0, void *o, float *S_final, int B, int H, int L, int dk,
                           int dv, int chunk, efla_dtype dt, efla_dtype o_dt, void *workspace,
                           size_t workspace_bytes, void *stream) {
    return efla_chunk_fwd_rule(q, k, v, beta, S0, o, S_final, B, H, L, dk, dv, chunk, dt, o_dt,
                               EFLA_RULE_EXACT, workspace, workspace_bytes, stream);
}

static efla_status recurrent_step_entry(const void *q, const void *k, const void *v, const void *beta,
                                       const void *g, float *S, void *o, int B, int H, int dk, int dv,
                                       efla_dtype dt, efla_dtype o_dt, efla_rule rule, void *stream) {
    if (!rule_ok(rule)) return EFLA_ERR_RULE;
    if (!dtype_ok(dt) || !dtype_ok(o_dt)) return EFLA_ERR_DTYPE;
    if (B < 1 || H < 1 || dk < 1 || dv < 1) return EFLA_ERR_SHAPE;
    if ((long long)B * H > 0x7fffffffLL) return EFLA_ERR_SHAPE;
    if (dk > 256 || dv > 256) return EFLA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !beta || !S || !o) return EFLA_ERR_NULL;
    if (!aligned_elem(q, dt) || !aligned_elem(k, dt) || !aligned_elem(v, dt) ||
        !aligned_elem(beta, dt) || !aligned_elem(g, dt) || !aligned16(S) || !aligned_elem(o, o_dt))
        return EFLA_ERR_ALIGN;
    return from_cuda(efla::launch_decode(q, k, v, beta, g, S, o, B * H, dk, dv, dt == EFLA_BF16,
                                         o_dt == EFLA_BF16, rule == EFLA_RULE_EULER,
                                         (cudaStream_t)stream));
}

efla_status efla_recurrent_step_rule(const void *q, const void *k, const void *v, const void *beta,
                                     float *S, void *o, int B, int H, int dk, int dv, efla_dtype dt,
                                     efla_dtype o_dt, efla_rule rule, void *stream) {
    return recurrent_step_entry(q, k, v, beta, nullptr, S, o, B, H, dk, dv, dt, o_dt, rule, stream);
}

efla_status efla_recurrent_step_gated(const void *q, const void *k, const void *v, const void *beta,
                                      const void *g, float *S, void *o, int B, int H, int dk, int dv,
                                      efla_dtype dt, efla_dtype o_dt, efla_rule rule, void *stream) {
    if (!g) return EFLA_ERR_NULL;
    return recurrent_step_entry(q, k, v, beta, g, S, o, B, H, dk, dv, dt, o_dt, rule, stream);
}

efla_status efla_recurrent_step(const void *q, const void *k, const void *v, const void *beta,
                                float *S, void *o, int B, int H, int dk, int dv, efla_dtype dt,
                                efla_dtype o_dt, void *stream) {
    return efla_recurrent_step_rule(q, k, v, beta, S, o, B, H, dk, dv, dt, o_dt, EFLA_RULE_EXACT,
                                    stream);
}

efla_status efla_state_affine(const float *P, const float *S_in, const float *Hm, float *S_out,
                              int B, int H, int dk, int dv, void *stream) {
    if (B < 1 || H < 1 || dk < 1 || dv < 1) return EFLA_ERR_SHAPE;
    if ((long long)B * H * ((dv + 15) / 16) > 0x7fffffffLL) return EFLA_ERR_SHAPE;
    if (dk > 256 || dv > 256) return EFLA_ERR_UNSUPPORTED;
    if (!P || !S_out) return EFLA_ERR_NULL;
    if (!aligned_elem(P, EFLA_F32) || !aligned_elem(S_in, EFLA_F32) || !aligned_elem(Hm, EFLA_F32) ||
        !aligned_elem(S_out, EFLA_F32))
        return EFLA_ERR_ALIGN;
    return from_cuda(efla::launch_state_affine(P, S_in, Hm, S_out, B * H, dk, dv,
                                               (cudaStream_t)stream));
}

size_t efla_bwd_workspace_size(int B, int H, int L, int dk, int dv) {
    if (B < 1 || H < 1 || L < 0 || dk < 1 || dv < 1 || dk > 128 || dv > 128) return 0;
    return efla::bwd_workspace_bytes(B, H, L, dk, dv);
}

static efla_status bwd_entry(const void *q, const void *k, const void *v, const void *beta,
                             const float *S0, const float *dO, const float *dS_final, float *dq,
                             float *dkey, float *dval, float *dbeta, float *dS0, int B, int H, int L,
                             int dk, int dv, efla_dtype dt, efla_rule rule, void *workspace,
                             size_t workspace_bytes, void *stream, const void *kept) {
    if (!rule_ok(rule)) return EFLA_ERR_RULE;
    if (!dtype_ok(dt)) return EFLA_ERR_DTYPE;
    if (B < 1 || H < 1 || L < 0 || dk < 1 || dv < 1) return EFLA_ERR_SHAPE;
    if ((long long)B * H > 0x7fffffffLL || (long long)B * H * L > (1LL << 40)) return EFLA_ERR_SHAPE;
    if (dk > 128 || dv > 128) return EFLA_ERR_UNSUPPORTED;
    if (L > 0 && (!q || !k || !v || !beta || !dO || !dq || !dkey || !dval || !dbeta))
        return EFLA_ERR_NULL;
    if (!aligned_elem(q, dt) || !aligned_elem(k, dt) || !aligned_elem(v, dt) ||
        !aligned_elem(beta, dt))
        return EFLA_ERR_ALIGN;
    const void *fp[] = {S0, dO, dS_final, dq, dkey, dval, dbeta, dS0, workspace};
    for (const void *p : fp)
        if (!aligned_elem(p, EFLA_F32)) return EFLA_ERR_ALIGN;
    if (!aligned16(workspace)) return EFLA_ERR_ALIGN;  // float4 rows of the saved states
    const size_t need = efla::bwd_workspace_bytes(B, H, L, dk, dv);
    if (need > 0 && (!workspace || workspace_bytes < need)) return EFLA_ERR_WORKSPACE;
    return from_cuda(efla::launch_bwd(q, k, v, beta, S0, dO, dS_final, dq, dkey, dval, dbeta, dS0,
                                      B, H, L, dk, dv, dt == EFLA_BF16, rule == EFLA_RULE_EULER,
                                      workspace, (cudaStream_t)stream, kept));
}

efla_status efla_bwd(const void *q, const void *k, const void *v, const void *beta,
                     const float *S0, const float *dO, const float *dS_final, float *dq,
                     float *dkey, float *dval, float *dbeta, float *dS0, int B, int H, int L,
                     int dk, int dv, efla_dtype dt, efla_rule rule, void *workspace,
                     size_t workspace_bytes, void *stream) {
    return bwd_entry(q, k, v, beta, S0, dO, dS_final, dq, dkey, dval, dbeta, dS0, B, H, L, dk, dv, dt, rule,
                     workspace, workspace_bytes, stream, nullptr);
}

size_t efla_bwd_kept_size(int B, int H, int L, int dk, int dv) {
    if (B < 1 || H < 1 || L < 1 || dk < 1 || dv < 1 || dk > 128 || dv > 128) return 0;
    return efla::bwd_kept_bytes(B, H, L, dk, dv);
}

efla_status efla_bwd_kept(const void *q, const void *k, const void *v, const void *beta,
                          const float *S0, const float *dO, const float *dS_final, float *dq,
                          float *dkey, float *dval, float *dbeta, float *dS0, int B, int H, int L,
                          int dk, int dv, efla_dtype dt, efla_rule rule, const void *kept,
                          size_t kept_bytes, void *workspace, size_t workspace_bytes, void *stream) {
    const size_t need = efla_bwd_kept_size(B, H, L, dk, dv);
    if (dt != EFLA_BF16 || need == 0) return EFLA_ERR_UNSUPPORTED;
    if (!kept || kept_bytes < need) return EFLA_ERR_WORKSPACE;
    if (!aligned16(kept)) return EFLA_ERR_ALIGN;
    return bwd_entry(q, k, v, beta, S0, dO, dS_final, dq, dkey, dval, dbeta, dS0, B, H, L, dk, dv, dt, rule,
                     workspace, workspace_bytes, stream, kept);
}

efla_status efla_chunk_fwd_keep(const void *q, const void *k, const void *v, const void *beta,
                                const float *S0, void *o, float *S_final, int B, int H, int L,
                                int dk, int dv, efla_dtype dt, efla_dtype o_dt, efla_rule rule,
                                void *kept, size_t kept_bytes, void *stream) {
    if (!rule_ok(rule)) return EFLA_ERR_RULE;
    if (!dtype_ok(dt) || !dtype_ok(o_dt)) return EFLA_ERR_DTYPE;
    if (B < 1 || H < 1 || L < 0 || dk < 1 || dv < 1) return EFLA_ERR_SHAPE;
    if ((long long)B * H > 0x7fffffffLL || (long long)B * H * L > (1LL << 40)) return EFLA_ERR_SHAPE;
    void *tc_ws = nullptr;
    __half *u = nullptr, *ck = nullptr;
    if (L < 1 || !efla::bwd_kept_regions(B, H, L, dk, dv, dt == EFLA_BF16, kept, &tc_ws, &u, &ck))
        return EFLA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !beta || !o) return EFLA_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned_elem(beta, dt) || !aligned16(S0) ||
        !aligned16(o) || !aligned16(S_final))
        return EFLA_ERR_ALIGN;
    const size_t need = efla::bwd_kept_bytes(B, H, L, dk, dv);
    if (!kept || kept_bytes < need) return EFLA_ERR_WORKSPACE;
    if (!aligned16(kept)) return EFLA_ERR_ALIGN;
    return from_cuda(efla::launch_chunk_tc_keep(q, k, v, beta, S0, o, S_final, B, H, L, dk, dv, o_dt == EFLA_BF16,
                                                rule == EFLA_RULE_EULER, tc_ws, u, ck, (cudaStream_t)stream));
}

efla_status efla_selftest_bounded_wait(long long budget_cycles, void *stream) {
    if (budget_cycles < 1 || budget_cycles > 2000000000LL) return EFLA_ERR_SHAPE;
    return from_cuda(efla::launch_selftest_wait(budget_cycles, (cudaStream_t)stream));
}

unsigned long long efla_kernel_launches(void) {
    return efla::g_launches.load(std::memory_order_relaxed);
}

efla_status efla_last_device_error(void *stream) {
    unsigned int word = 0, bwd_word = 0;
    if (efla::tc_read_and_clear_error(&word, (cudaStream_t)stream) != cudaSuccess ||
        efla::bwd_tc_read_and_clear_error(&bwd_word) != cudaSuccess)
        return EFLA_ERR_CUDA;
    return (word | bwd_word) ? EFLA_ERR_TIMEOUT : EFLA_OK;
}

}  // extern "C"
