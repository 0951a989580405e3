// alpha.cu -- fused per-token squared key norm and EFLA coefficient.
//
// "Exact Flow Linear Attention" technical summary, Methodology 2
// (lambda_t = ||k_t||^2) and Methodology 3 (alpha_t = (1 - e^{-beta_t lambda_t}) / lambda_t).
//
// One warp per token; lanes stride over the key dimension so that each warp
// load instruction covers consecutive elements of one key row.  The kernel is
// HBM-bound: it reads dk + 1 elements and writes one fp32 per token.
#include "common.cuh"
#include "launchers.h"

namespace efla {

template <typename T>
__global__ void __launch_bounds__(256) alpha_kernel(const T *__restrict__ k,
                                                    const T *__restrict__ beta,
                                                    float *__restrict__ alpha, long long ntok,
                                                    int dk, bool euler) {
    const int lane = threadIdx.x & 31;
    const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
    for (long long t = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < ntok;
         t += warps) {
        const T *kr = k + t * dk;
        float s = 0.f;
        for (int i = lane; i < dk; i += 32) {
            const float x = to_f32(kr[i]);
            s = fmaf(x, x, s);
        }
        s = warp_sum(s);
        if (lane == 0) alpha[t] = alpha_rule(s, to_f32(beta[t]), euler);
    }
}

cudaError_t launch_alpha(const void *k, const void *beta, float *alpha, long long ntok, int dk,
                         bool is_bf16, bool euler, cudaStream_t s) {
    if (ntok <= 0) return cudaSuccess;
    long long blocks = (ntok + 7) / 8;
    if (blocks > 148LL * 16) blocks = 148LL * 16;
    if (is_bf16)
        alpha_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
            (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)beta, alpha, ntok, dk, euler);
    else
        alpha_kernel<float><<<(unsigned)blocks, 256, 0, s>>>((const float *)k,
                                                             (const float *)beta, alpha, ntok, dk,
                                                             euler);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace efla
