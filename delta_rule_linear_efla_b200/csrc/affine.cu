// affine.cu -- S_out = P S_in + H per head, in fp32.
//
// A stretch of the sequence maps the state affinely: S_out = P S_in + H, with P the product of
// the stretch's transitions (I - alpha k k^T) and H the stretch's state from zero (the chunk
// update S <- (I - K^T W) S + K^T U of "Exact Flow Linear Attention", technical summary,
// Methodology 3, applied over the stretch).  Chaining such maps gives a later stretch its
// starting state without rerunning the earlier ones -- the step that lets sequence shards on
// different GPUs (or segments on one) run side by side.
//
// One CTA per (head, 16 state columns), one state row per thread: the CTA stages its 16-column
// block of S_in in shared memory before any thread writes, so S_out may alias S_in.
#include "common.cuh"
#include "launchers.h"

namespace efla {

__global__ void __launch_bounds__(256) state_affine_kernel(const float *__restrict__ P,
                                                           const float *S_in,
                                                           const float *__restrict__ H,
                                                           float *S_out, int dk, int dv) {
    __shared__ float X[256][17];  // the S_in block (padded against bank conflicts)
    const int nb = (dv + 15) / 16, bh = blockIdx.x / nb, c0 = (blockIdx.x % nb) * 16;
    const int t = threadIdx.x, nc = dv - c0 < 16 ? dv - c0 : 16;
    const size_t off = (size_t)bh * dk * dv;
    if (t < dk) {
        for (int c = 0; c < 16; ++c)
            X[t][c] = (S_in && c < nc) ? S_in[off + (size_t)t * dv + c0 + c] : 0.f;
    }
    __syncthreads();
    if (t >= dk) return;
    float y[16];
    for (int c = 0; c < 16; ++c) y[c] = (H && c < nc) ? H[off + (size_t)t * dv + c0 + c] : 0.f;
    const float *prow = P + (size_t)bh * dk * dk + (size_t)t * dk;
    for (int m = 0; m < dk; ++m) {
        const float p = prow[m];
#pragma unroll
        for (int c = 0; c < 16; ++c) y[c] = fmaf(p, X[m][c], y[c]);
    }
    for (int c = 0; c < nc; ++c) S_out[off + (size_t)t * dv + c0 + c] = y[c];
}

cudaError_t launch_state_affine(const float *P, const float *S_in, const float *H, float *S_out,
                                int BH, int dk, int dv, cudaStream_t s) {
    if (BH <= 0) return cudaSuccess;
    const int nb = (dv + 15) / 16;
    state_affine_kernel<<<BH * nb, 256, 0, s>>>(P, S_in, H, S_out, dk, dv);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace efla
