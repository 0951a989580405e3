// chunk_simt.cu -- SIMT fp32 evaluation of the EFLA chunkwise (WY/UT) form.
//
// "Exact Flow Linear Attention" technical summary, Methodology 3: the update
// S_t = (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T keeps the delta
// rule's rank-1 algebra, so chunks of C tokens can be folded in at once.
// Writing S_t = S_{t-1} + k_t u_t^T with u_t = alpha_t (v_t - S_{t-1}^T k_t) and
// unrolling a chunk that starts from state S gives, in matrix form,
//
//   A  = strictly-lower(diag(alpha) K K^T),   T = (I + A)^{-1}
//   W  = T diag(alpha) K,                     U = T diag(alpha) V
//   U' = U - W S                              (the chunk's u_t rows)
//   O  = Q S + lower-incl-diagonal(Q K^T) U'  (o_t = S_t^T q_t)
//   S <- S + K^T U'
//
// The gated form (a per-token decay g_t on the carried state, S_t = g_t (I - alpha_t k_t
// k_t^T) S_{t-1} + alpha_t k_t v_t^T; Gated DeltaNet's gate placement, the pages name it as a
// baseline) unrolls the same way with the cumulative log-decay l_t of the chunk (l = 0 at its
// start) and Gam_ts = e^{l_t - l_s} <= 1 for s <= t:
//
//   A  = strictly-lower(diag(alpha) (Gam o K K^T)),   W = T diag(alpha e^{l}) K
//   O  = diag(e^{l}) Q S + (lower-incl(Gam) o Q K^T) U'
//   S <- e^{l_C} S + K^T diag(e^{l_C - l}) U'
//
// Every factor is a decay of at most 1, so nothing grows; without a gate the kernel runs the
// ungated arithmetic unchanged.
//
// Everything here is fp32 on CUDA cores, which keeps fp32 inputs within
// 1e-4 of the fp64 oracle.  One CTA owns one head and a slice of NV state
// columns (columns of S evolve independently given K, W and U); chunks run in
// order.  This kernel is the general path (any dk, dv <= 128, chunk <= 64) and
// the path for fp32 inputs; bf16 inputs at the large sizes take the
// tensor-core kernels.
#include "common.cuh"
#include "launchers.h"

namespace efla {

static constexpr int SIMT_THREADS = 256;
static constexpr int SIMT_NV = 32;

struct SimtSmem {
    int dkp, Cp, NVp;
    size_t off_K, off_Q, off_W, off_A, off_T, off_P, off_V, off_S, off_al, off_lg, total;
    __host__ __device__ SimtSmem(int dk, int C, int NV) {
        dkp = dk + 1;
        Cp = C + 1;
        NVp = NV + 1;
        size_t o = 0;
        off_K = o; o += (size_t)C * dkp;
        off_Q = o; o += (size_t)C * dkp;
        off_W = o; o += (size_t)C * dkp;
        off_A = o; o += (size_t)C * Cp;
        off_T = o; o += (size_t)C * Cp;
        off_P = o; o += (size_t)C * Cp;
        off_V = o; o += (size_t)C * NVp;  // V slice, then U, then U'
        off_S = o; o += (size_t)dk * NVp;
        off_al = o; o += (size_t)C;
        off_lg = o; o += (size_t)3 * C;  // gated form: l_t, alpha_t e^{l_t}, e^{l_C - l_t}
        total = o * sizeof(float);
    }
};

template <typename T, typename TO>
__global__ void __launch_bounds__(SIMT_THREADS)
    chunk_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                      const T *__restrict__ beta, const T *__restrict__ gate,
                      const float *__restrict__ S0, TO *__restrict__ o,
                      float *__restrict__ S_final, int L, int dk, int dv, int C, int NV,
                      bool euler) {
    extern __shared__ float sm[];
    const SimtSmem lay(dk, C, NV);
    float *Ks = sm + lay.off_K, *Qs = sm + lay.off_Q, *Ws = sm + lay.off_W;
    float *As = sm + lay.off_A, *Ts = sm + lay.off_T, *Ps = sm + lay.off_P;
    float *Vs = sm + lay.off_V, *Ss = sm + lay.off_S, *al = sm + lay.off_al;
    float *lg = sm + lay.off_lg, *alg = lg + C, *gl = lg + 2 * C;
    const bool gated = gate != nullptr;
    const int dkp = lay.dkp, Cp = lay.Cp, NVp = lay.NVp;

    const int bh = blockIdx.x;
    const int v0 = blockIdx.y * NV;
    const int nv = min(NV, dv - v0);
    const int tid = threadIdx.x, nth = blockDim.x;
    const int warp = tid >> 5, lane = tid & 31, nwarps = nth >> 5;

    // initial state slice
    for (int idx = tid; idx < dk * nv; idx += nth) {
        const int d = idx / nv, n = idx % nv;
        Ss[d * NVp + n] = S0 ? S0[((size_t)bh * dk + d) * dv + v0 + n] : 0.f;
    }

    for (int c0 = 0; c0 < L; c0 += C) {
        const int cl = min(C, L - c0);
        const size_t row0 = (size_t)bh * L + c0;
        __syncthreads();  // previous chunk finished with every buffer
        for (int idx = tid; idx < cl * dk; idx += nth) {
            const int i = idx / dk, d = idx % dk;
            Ks[i * dkp + d] = to_f32(k[(row0 + i) * dk + d]);
            Qs[i * dkp + d] = to_f32(q[(row0 + i) * dk + d]);
        }
        for (int idx = tid; idx < cl * nv; idx += nth) {
            const int i = idx / nv, n = idx % nv;
            Vs[i * NVp + n] = to_f32(v[(row0 + i) * dv + v0 + n]);
        }
        __syncthreads();
        // alpha per token (fused squared norm)
        for (int i = warp; i < cl; i += nwarps) {
            float s = 0.f;
            for (int d = lane; d < dk; d += 32) s = fmaf(Ks[i * dkp + d], Ks[i * dkp + d], s);
            s = warp_sum(s);
            if (lane == 0) al[i] = alpha_rule(s, to_f32(beta[row0 + i]), euler);
        }
        if (gated && tid == 0) {  // cumulative log-decay of the chunk
            float l = 0.f;
            for (int i = 0; i < cl; ++i) {
                l += logf(to_f32(gate[row0 + i]));
                lg[i] = l;
            }
        }
        __syncthreads();
        if (gated) {
            for (int i = tid; i < cl; i += nth) {
                alg[i] = al[i] * expf(lg[i]);
                gl[i] = expf(lg[cl - 1] - lg[i]);
            }
        }
        // A = strictly-lower(diag(alpha) K K^T) and P = lower-incl-diag(Q K^T)
        for (int idx = tid; idx < cl * cl; idx += nth) {
            const int i = idx / cl, j = idx % cl;
            float a = 0.f, p = 0.f;
            if (j <= i) {
                for (int d = 0; d < dk; ++d) {
                    const float kj = Ks[j * dkp + d];
                    a = fmaf(Ks[i * dkp + d], kj, a);
                    p = fmaf(Qs[i * dkp + d], kj, p);
                }
            }
            if (gated && j <= i) {
                const float gm = expf(lg[i] - lg[j]);
                a *= gm;
                p *= gm;
            }
            As[i * Cp + j] = (j < i) ? al[i] * a : 0.f;
            Ps[i * Cp + j] = p;
        }
        __syncthreads();
        // T = (I + A)^{-1} by forward substitution, one column per thread:
        // T[i][j] = delta_ij - sum_{m=j}^{i-1} A[i][m] T[m][j]
        for (int j = tid; j < cl; j += nth) {
            for (int i = 0; i < cl; ++i) {
                float t;
                if (i < j) {
                    t = 0.f;
                } else if (i == j) {
                    t = 1.f;
                } else {
                    float s = 0.f;
                    for (int m = j; m < i; ++m) s = fmaf(As[i * Cp + m], Ts[m * Cp + j], s);
                    t = -s;
                }
                Ts[i * Cp + j] = t;
            }
        }
        __syncthreads();
        // W = T diag(alpha) K  (gated: T diag(alpha e^{l}) K)
        const float *alw = gated ? alg : al;
        for (int idx = tid; idx < cl * dk; idx += nth) {
            const int i = idx / dk, d = idx % dk;
            float s = 0.f;
            for (int j = 0; j <= i; ++j) s = fmaf(Ts[i * Cp + j] * alw[j], Ks[j * dkp + d], s);
            Ws[i * dkp + d] = s;
        }
        // U = T diag(alpha) V, staged in registers until every thread has read V
        float ureg[(SIMT_NV * 64 + SIMT_THREADS - 1) / SIMT_THREADS];
        int nr = 0;
        for (int idx = tid; idx < cl * nv; idx += nth, ++nr) {
            const int i = idx / nv, n = idx % nv;
            float s = 0.f;
            for (int j = 0; j <= i; ++j) s = fmaf(Ts[i * Cp + j] * al[j], Vs[j * NVp + n], s);
            ureg[nr] = s;
        }
        __syncthreads();
        // U' = U - W S  (stored in Vs)
        nr = 0;
        for (int idx = tid; idx < cl * nv; idx += nth, ++nr) {
            const int i = idx / nv, n = idx % nv;
            float s = 0.f;
            for (int d = 0; d < dk; ++d) s = fmaf(Ws[i * dkp + d], Ss[d * NVp + n], s);
            Vs[i * NVp + n] = ureg[nr] - s;
        }
        __syncthreads();
        // O = Q S + P U'  (gated: diag(e^{l}) Q S + P U')
        for (int idx = tid; idx < cl * nv; idx += nth) {
            const int i = idx / nv, n = idx % nv;
            float s = 0.f;
            for (int d = 0; d < dk; ++d) s = fmaf(Qs[i * dkp + d], Ss[d * NVp + n], s);
            if (gated) s *= expf(lg[i]);
            for (int j = 0; j <= i; ++j) s = fmaf(Ps[i * Cp + j], Vs[j * NVp + n], s);
            o[(row0 + i) * dv + v0 + n] = from_f32<TO>(s);
        }
        __syncthreads();
        // S <- S + K^T U'  (gated: e^{l_C} S + K^T diag(e^{l_C - l}) U')
        if (gated) {
            const float gC = expf(lg[cl - 1]);
            for (int idx = tid; idx < dk * nv; idx += nth) {
                const int d = idx / nv, n = idx % nv;
                float s = 0.f;
                for (int i = 0; i < cl; ++i) s = fmaf(Ks[i * dkp + d] * gl[i], Vs[i * NVp + n], s);
                Ss[d * NVp + n] = fmaf(gC, Ss[d * NVp + n], s);
            }
        } else {
            for (int idx = tid; idx < dk * nv; idx += nth) {
                const int d = idx / nv, n = idx % nv;
                float s = 0.f;
                for (int i = 0; i < cl; ++i) s = fmaf(Ks[i * dkp + d], Vs[i * NVp + n], s);
                Ss[d * NVp + n] += s;
            }
        }
    }
    __syncthreads();
    if (S_final) {
        for (int idx = tid; idx < dk * nv; idx += nth) {
            const int d = idx / nv, n = idx % nv;
            S_final[((size_t)bh * dk + d) * dv + v0 + n] = Ss[d * NVp + n];
        }
    }
}

template <typename T, typename TO>
static cudaError_t launch_simt_t(const void *q, const void *k, const void *v, const void *beta,
                                 const void *g, const float *S0, void *o, float *S_final, int B,
                                 int H, int L, int dk, int dv, int chunk, bool euler, cudaStream_t s) {
    const int NV = dv < SIMT_NV ? dv : SIMT_NV;
    const SimtSmem lay(dk, chunk, NV);
    dim3 grid(B * H, (dv + NV - 1) / NV);
    cudaError_t e = cudaFuncSetAttribute(chunk_simt_kernel<T, TO>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)lay.total);
    if (e != cudaSuccess) return e;
    chunk_simt_kernel<T, TO><<<grid, SIMT_THREADS, lay.total, s>>>(
        (const T *)q, (const T *)k, (const T *)v, (const T *)beta, (const T *)g, S0, (TO *)o, S_final,
        L, dk, dv, chunk, NV, euler);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const void *beta,
                              const void *g, const float *S0, void *o, float *S_final, int B,
                              int H, int L, int dk, int dv, int chunk, bool is_bf16, bool o_bf16,
                              bool euler, cudaStream_t s) {
    using bf = __nv_bfloat16;
    if (is_bf16)
        return o_bf16 ? launch_simt_t<bf, bf>(q, k, v, beta, g, S0, o, S_final, B, H, L, dk, dv, chunk, euler, s)
                      : launch_simt_t<bf, float>(q, k, v, beta, g, S0, o, S_final, B, H, L, dk, dv, chunk, euler, s);
    return o_bf16 ? launch_simt_t<float, bf>(q, k, v, beta, g, S0, o, S_final, B, H, L, dk, dv, chunk, euler, s)
                  : launch_simt_t<float, float>(q, k, v, beta, g, S0, o, S_final, B, H, L, dk, dv, chunk, euler, s);
}

}  // namespace efla
