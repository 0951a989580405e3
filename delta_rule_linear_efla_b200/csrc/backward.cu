// backward.cu -- gradients of the EFLA forward (and of the delta rule's Euler step), fp32.
//
// Reverse mode through the token recurrence of "Exact Flow Linear Attention", technical summary,
// Methodology 3.  Per token, with S the state before it:
//   lambda = k.k, a = f(lambda, beta), x = S^T k, r = v - x, u = a r, S' = S + k u^T, o = S'^T q.
// Given G = dL/dS' gathered from the later tokens, the reverse step is
//   G += q do^T;  dq = S' do;  du = G^T k;  dk = G u;  da = du.r;  dv = a du;  dx = -a du;
//   dk += S dx;  dbeta = da df/dbeta;  dk += 2 da df/dlambda k;  G += k dx^T  (-> dL/dS).
//
// The state's columns evolve independently (column j: s <- (I - a k k^T) s + a k v_j), so the
// work is split by columns: one CTA per (head, block of 16 state columns), one state row per
// thread (128 threads, dk <= 128), that row of S and of G in registers.  What couples the column
// blocks is linear -- dq, dk and dbeta are sums over the columns (dk and dbeta through da, itself
// a sum over the columns) -- so each CTA writes its share of them to the workspace and a second
// kernel adds the shares up in a fixed order: the result does not depend on scheduling.
//
// A forward sweep stores each column block's r and its state every 64 tokens; the reverse sweep
// starts each 64-token block from the stored state at its end and steps back with
// S = S' - a k r^T, so rounding never accumulates over more than 64 tokens.  Each token takes
// one CTA-wide sum (the 16 column dot products over the rows, and lambda = |k|^2): a
// reduce-scatter across each warp's lanes, then one barrier to add the four warps' shares
// through shared memory, double-buffered by token parity so that one barrier per token suffices.
#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "launchers.h"

namespace efla {

#ifndef EFLA_BWD_ROWS_PER_THREAD
#define EFLA_BWD_ROWS_PER_THREAD 1
#endif
constexpr int BW_RPT = EFLA_BWD_ROWS_PER_THREAD;  // state rows per thread
constexpr int BW_THREADS = 128 / BW_RPT;           // 128 rows per CTA (dk <= 128)
constexpr int BW_MINB = BW_RPT == 1 ? 4 : 6;       // CTAs per SM the register budget allows
constexpr int BW_CB = 16;                          // state columns per CTA
constexpr int BWD_BLOCK = 64;    // tokens between stored states

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

struct BwdRed {  // the four warps' shares of one CTA-wide sum, double-buffered by token parity
    float col[2][BW_THREADS / 32][BW_CB];
};

// Two fp32 lanes at once (packed f32x2 arithmetic of sm_100; each lane rounds as the scalar op).
__device__ __forceinline__ void fma2(float &d0, float &d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rd, {%0, %1};\n\tfma.rn.f32x2 rd, ra, rb, rd;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void mul2(float &d0, float &d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void add2(float &d0, float &d1, float a0, float a1) {
    asm("{\n\t.reg .b64 ra, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rd, {%0, %1};\n\t"
        "add.rn.f32x2 rd, rd, ra;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1));
}

// Sum over the warp of 16 values per lane, scattered: every lane returns the sum of value
// (lane >> 1).  Each step halves the values a lane keeps and trades the other half with the
// lane whose index differs in one bit: 8 + 4 + 2 + 1 + 1 shuffles in place of 16 x 5.
__device__ __forceinline__ float warp_reduce_scatter16(float (&p)[BW_CB], int lane) {
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const bool up = lane & 16;
        const float send = up ? p[m] : p[m + 8], keep = up ? p[m + 8] : p[m];
        p[m] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const bool up = lane & 8;
        const float send = up ? p[m] : p[m + 4], keep = up ? p[m + 4] : p[m];
        p[m] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const bool up = lane & 4;
        const float send = up ? p[m] : p[m + 2], keep = up ? p[m + 2] : p[m];
        p[m] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    {
        const bool up = lane & 2;
        const float send = up ? p[0] : p[1], keep = up ? p[1] : p[0];
        p[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    return p[0] + __shfl_xor_sync(0xffffffffu, p[0], 1);
}

// Column c of a CTA-wide sum: the four warps' shares added in the order 0, 1, 2, 3.
__device__ __forceinline__ float col_sum(const BwdRed &red, int par, int c) {
    float a = red.col[par][0][c];
#pragma unroll
    for (int ww = 1; ww < BW_THREADS / 32; ++ww) a += red.col[par][ww][c];
    return a;
}

// CTA-wide sums of p[0..16) into out (every thread calls it; one barrier).  Each lane adds up
// one column's four warp shares (lanes 2c and 2c + 1 take column c) and the totals reach every
// lane by shuffles: shared memory sees one conflict-free load per warp share, not a broadcast
// read of all 64 shares by every thread.
__device__ __forceinline__ void cta_sum16(float (&p)[BW_CB], BwdRed &red, int par, float (&out)[BW_CB]) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const float c = warp_reduce_scatter16(p, lane);
    if ((lane & 1) == 0) red.col[par][w][lane >> 1] = c;
    __syncthreads();
    const float t = col_sum(red, par, lane >> 1);
#pragma unroll
    for (int j = 0; j < BW_CB; ++j) out[j] = __shfl_sync(0xffffffffu, t, 2 * j);
}

__device__ __forceinline__ void load_row16(const float *p, float (&x)[BW_CB]) {
#pragma unroll
    for (int j4 = 0; j4 < BW_CB / 4; ++j4) {
        const float4 a = reinterpret_cast<const float4 *>(p)[j4];
        x[4 * j4] = a.x; x[4 * j4 + 1] = a.y; x[4 * j4 + 2] = a.z; x[4 * j4 + 3] = a.w;
    }
}

__device__ __forceinline__ void store_row16(float *p, const float (&x)[BW_CB]) {
#pragma unroll
    for (int j4 = 0; j4 < BW_CB / 4; ++j4)
        reinterpret_cast<float4 *>(p)[j4] = make_float4(x[4 * j4], x[4 * j4 + 1], x[4 * j4 + 2], x[4 * j4 + 3]);
}

// Per token: (lambda = |k|^2, a = f(lambda, beta), df/dbeta, df/dlambda), one warp per token.
// Every column block of a head reads them, so they are computed once, ahead of the sweeps.
template <typename T>
__global__ void __launch_bounds__(256) bwd_coeff_kernel(const T *__restrict__ k, const T *__restrict__ beta,
                                                       size_t ntok, int dk, bool euler,
                                                       float4 *__restrict__ coef) {
    const int lane = threadIdx.x & 31;
    for (size_t tok = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5); tok < ntok; tok += (size_t)gridDim.x * 8) {
        float s = 0.f;
        for (int i = lane; i < dk; i += 32) {
            const float x = to_f32(k[tok * dk + i]);
            s = fmaf(x, x, s);
        }
        s = warp_sum(s);
        if (lane == 0) {
            const float bt = to_f32(beta[tok]);
            const float a = alpha_rule(s, bt, euler);
            float dfdb, dfdl;
            coeff_grads(s, bt, euler, a, dfdb, dfdl);
            coef[tok] = make_float4(s, a, dfdb, dfdl);
        }
    }
}

// Workspace: the per-token coefficients [B*H][L] (float4); per (head, column block) r of every
// token [L][16], then the block's state at every 64-token boundary and at the end
// [NB + 1][dk][16]; after all of those the column blocks' shares of dq and dk
// ([NS][B*H][L][dk] each) and of dbeta ([NS][B*H][L]).
template <typename T>
__global__ void __launch_bounds__(BW_THREADS, BW_MINB)
    bwd_cols_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                    const float4 *__restrict__ coef, const float *__restrict__ S0,
                    const float *__restrict__ dO, const float *__restrict__ dSL,
                    float *__restrict__ dval, float *__restrict__ dS0, int L, int dk, int dv, int NS,
                    float *__restrict__ ws, float *__restrict__ part) {
    __shared__ __align__(16) BwdRed red;
    __shared__ __align__(16) float xb[BWD_BLOCK][BW_CB];  // v (forward sweep) or dO (reverse)
    __shared__ __align__(16) float rb[BWD_BLOCK][BW_CB];  // r (reverse sweep)
    __shared__ __align__(16) float4 cb[BWD_BLOCK];        // the block's token coefficients
    const int tid = threadIdx.x;
    const int bh = blockIdx.x / NS, s = blockIdx.x % NS, c0 = s * BW_CB;
    const int BH = gridDim.x / NS, nc = min(BW_CB, dv - c0);
    const int NB = (L + BWD_BLOCK - 1) / BWD_BLOCK;
    int row[BW_RPT];  // this thread's state rows: tid, tid + BW_THREADS, ...
    bool act[BW_RPT];
#pragma unroll
    for (int u = 0; u < BW_RPT; ++u) {
        row[u] = tid + u * BW_THREADS;
        act[u] = row[u] < dk;
    }
    const size_t tk = (size_t)bh * L * dk, tv = (size_t)bh * L * dv, tb = (size_t)bh * L;
    const size_t DD = (size_t)dk * dv;
    float *R = ws + ((size_t)bh * NS + s) * ((size_t)L * BW_CB + (size_t)(NB + 1) * dk * BW_CB);
    float *CK = R + (size_t)L * BW_CB;
    const size_t nq = (size_t)BH * L * dk;
    float *pdq = part + (size_t)s * nq + tk;
    float *pdk = part + (size_t)NS * nq + (size_t)s * nq + tk;
    float *pdb = part + 2 * (size_t)NS * nq + (size_t)s * BH * L + tb;
    auto ld = [&](const T *x, int t, int u) {  // element row[u] of token t's q or k (0 off the edge)
        return (act[u] && t >= 0 && t < L) ? to_f32(x[tk + (size_t)t * dk + row[u]]) : 0.f;
    };

    float S[BW_RPT][BW_CB], G[BW_RPT][BW_CB];
#pragma unroll
    for (int u = 0; u < BW_RPT; ++u)
#pragma unroll
        for (int j = 0; j < BW_CB; ++j)
            S[u][j] = (S0 && act[u] && j < nc) ? S0[(size_t)bh * DD + (size_t)row[u] * dv + c0 + j] : 0.f;

    // ---- forward sweep: r of every token and the block-boundary states
    int par = 0;
    float kr1[BW_RPT], kr2[BW_RPT], qr1[BW_RPT], qr2[BW_RPT];
#pragma unroll
    for (int u = 0; u < BW_RPT; ++u) {
        kr1[u] = ld(k, 0, u);
        kr2[u] = ld(k, 1, u);
    }
    for (int b = 0; b < NB; ++b) {
        const int t0 = b * BWD_BLOCK, cnt = min(BWD_BLOCK, L - t0);
        __syncthreads();  // the previous block's reads of xb and cb are done
        for (int e = tid; e < cnt * BW_CB; e += BW_THREADS) {
            const int tt = e / BW_CB, j = e % BW_CB;
            xb[tt][j] = j < nc ? to_f32(v[tv + (size_t)(t0 + tt) * dv + c0 + j]) : 0.f;
        }
        for (int e = tid; e < cnt; e += BW_THREADS) cb[e] = coef[tb + t0 + e];
#pragma unroll
        for (int u = 0; u < BW_RPT; ++u)
            if (act[u]) store_row16(CK + ((size_t)b * dk + row[u]) * BW_CB, S[u]);
        __syncthreads();
        for (int tt = 0; tt < cnt; ++tt) {
            const int t = t0 + tt;
            float ki[BW_RPT];
#pragma unroll
            for (int u = 0; u < BW_RPT; ++u) {
                ki[u] = kr1[u];
                kr1[u] = kr2[u];
                kr2[u] = ld(k, t + 2, u);
            }
            float p[BW_CB], x[BW_CB], r[BW_CB];
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) {
                mul2(p[j], p[j + 1], S[0][j], S[0][j + 1], ki[0], ki[0]);
#pragma unroll
                for (int u = 1; u < BW_RPT; ++u) fma2(p[j], p[j + 1], S[u][j], S[u][j + 1], ki[u], ki[u]);
            }
            cta_sum16(p, red, par, x);  // x = S^T k
            const float a = cb[tt].y;
            load_row16(xb[tt], r);
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) add2(r[j], r[j + 1], -x[j], -x[j + 1]);  // r = v - S^T k
            if (tid < BW_CB) R[(size_t)t * BW_CB + tid] = xb[tt][tid] + -col_sum(red, par, tid);
#pragma unroll
            for (int u = 0; u < BW_RPT; ++u) {
                const float ak = a * ki[u];
#pragma unroll
                for (int j = 0; j < BW_CB; j += 2) fma2(S[u][j], S[u][j + 1], ak, ak, r[j], r[j + 1]);
            }
            par ^= 1;
        }
    }
#pragma unroll
    for (int u = 0; u < BW_RPT; ++u)
        if (act[u]) store_row16(CK + ((size_t)NB * dk + row[u]) * BW_CB, S[u]);

    // ---- reverse sweep
#pragma unroll
    for (int u = 0; u < BW_RPT; ++u) {
#pragma unroll
        for (int j = 0; j < BW_CB; ++j)
            G[u][j] = (dSL && act[u] && j < nc) ? dSL[(size_t)bh * DD + (size_t)row[u] * dv + c0 + j] : 0.f;
        kr1[u] = ld(k, L - 1, u);
        kr2[u] = ld(k, L - 2, u);
        qr1[u] = ld(q, L - 1, u);
        qr2[u] = ld(q, L - 2, u);
    }
    for (int b = NB - 1; b >= 0; --b) {
        const int t0 = b * BWD_BLOCK, cnt = min(BWD_BLOCK, L - t0);
        __syncthreads();  // the previous block's reads of xb, rb and cb are done
        for (int e = tid; e < cnt * BW_CB; e += BW_THREADS) {
            const int tt = e / BW_CB, j = e % BW_CB;
            xb[tt][j] = j < nc ? dO[tv + (size_t)(t0 + tt) * dv + c0 + j] : 0.f;
            rb[tt][j] = R[(size_t)(t0 + tt) * BW_CB + j];
        }
        for (int e = tid; e < cnt; e += BW_THREADS) cb[e] = coef[tb + t0 + e];
#pragma unroll
        for (int u = 0; u < BW_RPT; ++u)  // S' after the block
            if (act[u]) load_row16(CK + ((size_t)(b + 1) * dk + row[u]) * BW_CB, S[u]);
        __syncthreads();
        for (int tt = cnt - 1; tt >= 0; --tt) {
            const int t = t0 + tt;
            float ki[BW_RPT], qi[BW_RPT];
#pragma unroll
            for (int u = 0; u < BW_RPT; ++u) {
                ki[u] = kr1[u];
                qi[u] = qr1[u];
                kr1[u] = kr2[u];
                qr1[u] = qr2[u];
                kr2[u] = ld(k, t - 2, u);
                qr2[u] = ld(q, t - 2, u);
            }
            float d[BW_CB], r[BW_CB], p[BW_CB], du[BW_CB];
            load_row16(xb[tt], d);
            load_row16(rb[tt], r);
            // G += q do^T;  dq = S' do
            float dq0[BW_RPT], dq1[BW_RPT];
#pragma unroll
            for (int u = 0; u < BW_RPT; ++u) {
                dq0[u] = 0.f;
                dq1[u] = 0.f;
#pragma unroll
                for (int j = 0; j < BW_CB; j += 2) {
                    fma2(G[u][j], G[u][j + 1], qi[u], qi[u], d[j], d[j + 1]);
                    fma2(dq0[u], dq1[u], S[u][j], S[u][j + 1], d[j], d[j + 1]);
                }
            }
            // du = G^T k
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) {
                mul2(p[j], p[j + 1], G[0][j], G[0][j + 1], ki[0], ki[0]);
#pragma unroll
                for (int u = 1; u < BW_RPT; ++u) fma2(p[j], p[j + 1], G[u][j], G[u][j + 1], ki[u], ki[u]);
            }
            cta_sum16(p, red, par, du);
            const float4 cf = cb[tt];  // (lambda, a, df/dbeta, df/dlambda)
            const float a = cf.y;
            float da0 = 0.f, da1 = 0.f;  // this column block's share of da = du . r
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) fma2(da0, da1, du[j], du[j + 1], r[j], r[j + 1]);
            const float da = da0 + da1;
            // S = S' - a k r^T;  dk = a G r - a S du + 2 da df/dlambda k;  G -= a k du^T
#pragma unroll
            for (int u = 0; u < BW_RPT; ++u) {
                const float nak = -a * ki[u];
                float gr0 = 0.f, gr1 = 0.f, sd0 = 0.f, sd1 = 0.f;
#pragma unroll
                for (int j = 0; j < BW_CB; j += 2) {
                    fma2(S[u][j], S[u][j + 1], nak, nak, r[j], r[j + 1]);
                    fma2(gr0, gr1, G[u][j], G[u][j + 1], r[j], r[j + 1]);
                    fma2(sd0, sd1, S[u][j], S[u][j + 1], du[j], du[j + 1]);
                    fma2(G[u][j], G[u][j + 1], nak, nak, du[j], du[j + 1]);
                }
                if (act[u]) {
                    pdq[(size_t)t * dk + row[u]] = dq0[u] + dq1[u];
                    pdk[(size_t)t * dk + row[u]] = a * ((gr0 + gr1) - (sd0 + sd1)) + 2.f * da * cf.w * ki[u];
                }
            }
            if (tid < nc) dval[tv + (size_t)t * dv + c0 + tid] = a * col_sum(red, par, tid);
            if (tid == 0) pdb[t] = da * cf.z;
            par ^= 1;
        }
    }
    if (dS0) {
#pragma unroll
        for (int u = 0; u < BW_RPT; ++u)
#pragma unroll
            for (int j = 0; j < BW_CB; ++j)
                if (act[u] && j < nc) dS0[(size_t)bh * DD + (size_t)row[u] * dv + c0 + j] = G[u][j];
    }
}

// out[e] = sum over s = 0..NS-1 of part[s n + e], in that order (blockIdx.y picks dq, dk, dbeta).
struct SumSeg {
    const float *part;
    float *out;
    size_t n;
    int vec;  // 1: n % 4 == 0 and both arrays 16-byte aligned
};
struct SumSegs {
    SumSeg seg[3];
};

__global__ void __launch_bounds__(256) bwd_sum_kernel(SumSegs segs, int NS) {
    const SumSeg g = blockIdx.y == 0 ? segs.seg[0] : (blockIdx.y == 1 ? segs.seg[1] : segs.seg[2]);
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g.vec) {
        const size_t n4 = g.n / 4;
        const float4 *p4 = reinterpret_cast<const float4 *>(g.part);
        float4 *o4 = reinterpret_cast<float4 *>(g.out);
        for (size_t e = i0; e < n4; e += stride) {
            float4 a = p4[e];
            for (int s = 1; s < NS; ++s) {
                const float4 b = p4[(size_t)s * n4 + e];
                a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
            }
            o4[e] = a;
        }
    } else {
        for (size_t e = i0; e < g.n; e += stride) {
            float a = g.part[e];
            for (int s = 1; s < NS; ++s) a += g.part[(size_t)s * g.n + e];
            g.out[e] = a;
        }
    }
}

static size_t bwd_state_floats(size_t BH, int L, int dk, int dv) {
    const size_t NB = (size_t)(L + BWD_BLOCK - 1) / BWD_BLOCK;
    const size_t NS = (size_t)(dv + BW_CB - 1) / BW_CB;
    return BH * NS * ((size_t)L * BW_CB + (NB + 1) * (size_t)dk * BW_CB);
}

size_t bwd_workspace_bytes(int B, int H, int L, int dk, int dv) {
    const size_t BH = (size_t)B * H, NS = (size_t)(dv + BW_CB - 1) / BW_CB;
    const size_t coef = 4 * BH * (size_t)L;
    const size_t shares = NS * BH * (size_t)L * (2 * (size_t)dk + 1);
    return (coef + bwd_state_floats(BH, L, dk, dv) + shares) * sizeof(float);
}

cudaError_t launch_bwd(const void *q, const void *k, const void *v, const void *beta,
                       const float *S0, const float *dO, const float *dSL, float *dq, float *dkey,
                       float *dval, float *dbeta, float *dS0, int B, int H, int L, int dk, int dv,
                       bool is_bf16, bool euler, void *ws, cudaStream_t s) {
    const long long BH = (long long)B * H;
    const int NS = (dv + BW_CB - 1) / BW_CB;
    if (BH * NS > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const size_t ntok = (size_t)BH * L;
    float4 *coef = (float4 *)ws;
    float *state = (float *)ws + 4 * ntok;
    float *part = state + bwd_state_floats((size_t)BH, L, dk, dv);
    if (ntok > 0) {
        const int gc = (int)std::min<size_t>((ntok + 7) / 8, (size_t)nsm * 64);
        if (is_bf16)
            bwd_coeff_kernel<__nv_bfloat16><<<gc, 256, 0, s>>>((const __nv_bfloat16 *)k,
                                                               (const __nv_bfloat16 *)beta, ntok, dk,
                                                               euler, coef);
        else
            bwd_coeff_kernel<float><<<gc, 256, 0, s>>>((const float *)k, (const float *)beta, ntok, dk,
                                                       euler, coef);
        count_launches(1);
    }
    const int grid = (int)(BH * NS);
    if (is_bf16)
        bwd_cols_kernel<__nv_bfloat16><<<grid, BW_THREADS, 0, s>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, coef, S0, dO,
            dSL, dval, dS0, L, dk, dv, NS, state, part);
    else
        bwd_cols_kernel<float><<<grid, BW_THREADS, 0, s>>>((const float *)q, (const float *)k,
                                                          (const float *)v, coef, S0, dO, dSL, dval,
                                                          dS0, L, dk, dv, NS, state, part);
    count_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || L == 0) return e;
    // add the column blocks' shares of dq, dk and dbeta
    const size_t nq = (size_t)BH * L * dk, nb = (size_t)BH * L;
    auto seg = [&](const float *pp, float *out, size_t n) {
        SumSeg g;
        g.part = pp;
        g.out = out;
        g.n = n;
        g.vec = (n % 4 == 0 && ((uintptr_t)pp % 16) == 0 && ((uintptr_t)out % 16) == 0) ? 1 : 0;
        return g;
    };
    SumSegs segs;
    segs.seg[0] = seg(part, dq, nq);
    segs.seg[1] = seg(part + (size_t)NS * nq, dkey, nq);
    segs.seg[2] = seg(part + 2 * (size_t)NS * nq, dbeta, nb);
    const size_t want = (nq / 4 + 255) / 256;
    const int gx = (int)std::min<size_t>(std::max<size_t>(want, 1), (size_t)nsm * 8);
    bwd_sum_kernel<<<dim3(gx, 3), 256, 0, s>>>(segs, NS);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace efla
