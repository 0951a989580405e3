// backward.cu -- gradients of the EFLA forward (and of the delta rule's Euler step), fp32.
//
// Reverse mode through the token recurrence of "Exact Flow Linear Attention", technical summary,
// Methodology 3.  Per token, with S the state before it:
//   lambda = k.k, a = f(lambda, beta), x = S^T k, r = v - x, u = a r, S' = S + k u^T, o = S'^T q.
// Given G = dL/dS' gathered from the later tokens, the reverse step is
//   G += q do^T;  dq = S' do;  du = G^T k;  dk = G u;  da = du.r;  dv = a du;  dx = -a du;
//   dk += S dx;  dbeta = da df/dbeta;  dk += 2 da df/dlambda k;  G += k dx^T  (-> dL/dS).
//
// One CTA per head, 256 threads, S and G in shared memory (d <= 128).  A forward sweep stores
// every token's r and the state at every 64-token boundary in the workspace; the reverse sweep
// starts each 64-token block from the stored state at its end and steps back exactly with
// S = S' - a k r^T, so rounding never accumulates over more than 64 tokens.  This is the first
// correct path for the backward: it is bound by the per-token barrier chain, not by HBM.
#include "common.cuh"
#include "launchers.h"

namespace efla {

constexpr int BWD_THREADS = 256;
constexpr int BWD_BLOCK = 64;  // tokens between stored states

// df/dbeta and df/dlambda of the coefficient under the rule.
__device__ __forceinline__ void coeff_grads(float lambda, float beta, bool euler, float a,
                                            float &dfdb, float &dfdl) {
    if (euler) {
        dfdb = 1.f;
        dfdl = 0.f;
        return;
    }
    const float x = beta * lambda;
    dfdb = expf(-x);
    if (fabsf(x) < 0.1f) {  // beta^2 (-1/2 + x/3 - x^2/8 + x^3/30 - x^4/144): rel. error < 3e-8
        dfdl = beta * beta * (-0.5f + x * (1.f / 3.f + x * (-0.125f + x * (1.f / 30.f - x * (1.f / 144.f)))));
    } else {
        dfdl = (beta * dfdb - a) / lambda;
    }
}

// Sum over the CTA of one value per thread (all threads call it; the result is returned to all).
__device__ __forceinline__ float block_sum(float v, float *red) {
    v = warp_sum(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < BWD_THREADS / 32; ++i) s += red[i];
    return s;
}

// sum_j M[row][j] w[j] over this thread's half of the columns (two threads per row).  With an
// even dv the walk starts at column 2*row + half and wraps, so the 16 rows of a warp read 32
// different banks instead of two.
__device__ __forceinline__ float row_dot_half(const float *M, const float *w, int row, int half,
                                              int dv) {
    float s = 0.f;
    if (dv % 2 == 0) {
        int j = (2 * row + half) % dv;
        for (int m = 0; m < dv / 2; ++m) {
            s = fmaf(M[row * dv + j], w[j], s);
            j += 2;
            if (j >= dv) j -= dv;
        }
    } else {
        for (int j = half; j < dv; j += 2) s = fmaf(M[row * dv + j], w[j], s);
    }
    return s;
}

template <typename T>
__global__ void __launch_bounds__(BWD_THREADS)
    bwd_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
               const T *__restrict__ beta, const float *__restrict__ S0, const float *__restrict__ dO,
               const float *__restrict__ dSL, float *__restrict__ dq, float *__restrict__ dkey,
               float *__restrict__ dval, float *__restrict__ dbeta, float *__restrict__ dS0, int L,
               int dk, int dv, bool euler, float *__restrict__ ws) {
    extern __shared__ float sm[];
    const int DD = dk * dv, NB = (L + BWD_BLOCK - 1) / BWD_BLOCK;
    float *S = sm, *G = sm + DD;
    float *qs = G + DD, *ks = qs + 128, *dos = ks + 128, *rs = dos + 128, *dxs = rs + 128;
    float *red = dxs + 128;
    const int tid = threadIdx.x, bh = blockIdx.x;
    const size_t tk = (size_t)bh * L * dk, tv = (size_t)bh * L * dv, tb = (size_t)bh * L;
    float *R = ws + (size_t)bh * ((size_t)L * dv + (size_t)(NB + 1) * DD);  // r of every token
    float *CK = R + (size_t)L * dv;                                         // states S_{64 b}, S_L

    // ---- forward sweep: r_t and the block-boundary states
    for (int e = tid; e < DD; e += BWD_THREADS) S[e] = S0 ? S0[(size_t)bh * DD + e] : 0.f;
    __syncthreads();
    for (int t = 0; t < L; ++t) {
        if (t % BWD_BLOCK == 0)
            for (int e = tid; e < DD; e += BWD_THREADS) CK[(size_t)(t / BWD_BLOCK) * DD + e] = S[e];
        float kk = 0.f;
        if (tid < dk) {
            const float kv = to_f32(k[tk + (size_t)t * dk + tid]);
            ks[tid] = kv;
            kk = kv * kv;
        }
        const float lambda = block_sum(kk, red);  // (syncs: ks is visible)
        const float a = alpha_rule(lambda, to_f32(beta[tb + t]), euler);
        if (tid < dv) {  // r = v - S^T k
            float x = 0.f;
            for (int i = 0; i < dk; ++i) x = fmaf(S[i * dv + tid], ks[i], x);
            const float r = to_f32(v[tv + (size_t)t * dv + tid]) - x;
            rs[tid] = r;
            R[(size_t)t * dv + tid] = r;
        }
        __syncthreads();
        if (BWD_THREADS % dv == 0) {  // fixed column per thread: no division per element
            const int j = tid % dv;
            for (int i = tid / dv; i < dk; i += BWD_THREADS / dv)
                S[i * dv + j] = fmaf(a * ks[i], rs[j], S[i * dv + j]);
        } else {
            for (int e = tid; e < DD; e += BWD_THREADS) S[e] = fmaf(a * ks[e / dv], rs[e % dv], S[e]);
        }
        __syncthreads();
    }
    for (int e = tid; e < DD; e += BWD_THREADS) CK[(size_t)NB * DD + e] = S[e];

    // ---- reverse sweep
    for (int e = tid; e < DD; e += BWD_THREADS) G[e] = dSL ? dSL[(size_t)bh * DD + e] : 0.f;
    const int row = tid >> 1, half = tid & 1;  // two threads per state row for row reductions
    for (int b = NB - 1; b >= 0; --b) {
        __syncthreads();
        for (int e = tid; e < DD; e += BWD_THREADS) S[e] = CK[(size_t)(b + 1) * DD + e];
        const int t_end = min(L, (b + 1) * BWD_BLOCK);
        for (int t = t_end - 1; t >= b * BWD_BLOCK; --t) {
            float kk = 0.f;
            if (tid < dk) {
                const float kv = to_f32(k[tk + (size_t)t * dk + tid]);
                ks[tid] = kv;
                kk = kv * kv;
                qs[tid] = to_f32(q[tk + (size_t)t * dk + tid]);
            }
            if (tid < dv) {
                dos[tid] = dO[tv + (size_t)t * dv + tid];
                rs[tid] = R[(size_t)t * dv + tid];
            }
            const float lambda = block_sum(kk, red);  // syncs: the vectors and S are visible
            const float bt = to_f32(beta[tb + t]);
            const float a = alpha_rule(lambda, bt, euler);
            // G += q do^T; dq = S' do (S holds S' = the state after token t)
            if (BWD_THREADS % dv == 0) {
                const int j = tid % dv;
                for (int i = tid / dv; i < dk; i += BWD_THREADS / dv)
                    G[i * dv + j] = fmaf(qs[i], dos[j], G[i * dv + j]);
            } else {
                for (int e = tid; e < DD; e += BWD_THREADS) G[e] = fmaf(qs[e / dv], dos[e % dv], G[e]);
            }
            {
                float s = row < dk ? row_dot_half(S, dos, row, half, dv) : 0.f;
                s += __shfl_xor_sync(0xffffffffu, s, 1);
                if (row < dk && half == 0) dq[tk + (size_t)t * dk + row] = s;
            }
            __syncthreads();
            // du = G^T k, dv = a du, da = du . r
            float dap = 0.f;
            if (tid < dv) {
                float s = 0.f;
                for (int i = 0; i < dk; ++i) s = fmaf(G[i * dv + tid], ks[i], s);
                dxs[tid] = -a * s;
                dval[tv + (size_t)t * dv + tid] = a * s;
                dap = s * rs[tid];
            }
            const float da = block_sum(dap, red);  // syncs: dxs visible
            // dk = G u + (added below) S dx + 2 da df/dlambda k, with u = a r
            float dka = row < dk ? a * row_dot_half(G, rs, row, half, dv) : 0.f;  // G u, u = a r
            dka += __shfl_xor_sync(0xffffffffu, dka, 1);
            const float krow = row < dk ? ks[row] : 0.f;  // ks is rewritten by the next token
            __syncthreads();  // every read of G and S' for this token is done
            // S = S' - a k r^T (the state before token t); G += k dx^T (dL/dS)
            if (BWD_THREADS % dv == 0) {
                const int j = tid % dv;
                for (int i = tid / dv; i < dk; i += BWD_THREADS / dv) {
                    S[i * dv + j] = fmaf(-a * ks[i], rs[j], S[i * dv + j]);
                    G[i * dv + j] = fmaf(ks[i], dxs[j], G[i * dv + j]);
                }
            } else {
                for (int e = tid; e < DD; e += BWD_THREADS) {
                    const int i = e / dv, j = e % dv;
                    S[e] = fmaf(-a * ks[i], rs[j], S[e]);
                    G[e] = fmaf(ks[i], dxs[j], G[e]);
                }
            }
            __syncthreads();
            float dkb = row < dk ? row_dot_half(S, dxs, row, half, dv) : 0.f;
            dkb += __shfl_xor_sync(0xffffffffu, dkb, 1);
            float dfdb, dfdl;
            coeff_grads(lambda, bt, euler, a, dfdb, dfdl);
            if (row < dk && half == 0)
                dkey[tk + (size_t)t * dk + row] = dka + dkb + 2.f * da * dfdl * krow;
            if (tid == 0) dbeta[tb + t] = da * dfdb;
        }
    }
    __syncthreads();
    if (dS0)
        for (int e = tid; e < DD; e += BWD_THREADS) dS0[(size_t)bh * DD + e] = G[e];
}

size_t bwd_workspace_bytes(int B, int H, int L, int dk, int dv) {
    const size_t NB = (size_t)(L + BWD_BLOCK - 1) / BWD_BLOCK;
    return (size_t)B * H * ((size_t)L * dv + (NB + 1) * (size_t)dk * dv) * sizeof(float);
}

cudaError_t launch_bwd(const void *q, const void *k, const void *v, const void *beta,
                       const float *S0, const float *dO, const float *dSL, float *dq, float *dkey,
                       float *dval, float *dbeta, float *dS0, int B, int H, int L, int dk, int dv,
                       bool is_bf16, bool euler, void *ws, cudaStream_t s) {
    const int BH = B * H;
    const size_t smem = (size_t)(2 * dk * dv + 5 * 128 + 32) * sizeof(float);
    cudaError_t e;
    if (is_bf16) {
        e = cudaFuncSetAttribute(bwd_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return e;
        bwd_kernel<__nv_bfloat16><<<BH, BWD_THREADS, smem, s>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,
            (const __nv_bfloat16 *)beta, S0, dO, dSL, dq, dkey, dval, dbeta, dS0, L, dk, dv, euler,
            (float *)ws);
    } else {
        e = cudaFuncSetAttribute(bwd_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        bwd_kernel<float><<<BH, BWD_THREADS, smem, s>>>((const float *)q, (const float *)k, (const float *)v,
                                                       (const float *)beta, S0, dO, dSL, dq, dkey, dval,
                                                       dbeta, dS0, L, dk, dv, euler, (float *)ws);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace efla
