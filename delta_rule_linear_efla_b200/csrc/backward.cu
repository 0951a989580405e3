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
// S = S' - a k r^T, so rounding never accumulates over more than 64 tokens.  Tokens go in
// pairs, with one CTA-wide sum per pair (32 column dot products over the rows): a
// reduce-scatter across each warp's lanes, then one barrier to add the four warps' shares
// through shared memory, double-buffered by parity so that one barrier per pair suffices.
// The per-token coefficients and the two dot products that link a pair's tokens come from a
// prologue kernel.
//
// With bf16 inputs at the tensor-core sizes (16-byte aligned), the heads that pass an accuracy
// gate (bwd_gate.cuh: moderate key norms) take the tensor-core backward instead (bwd_tc.cu: the
// tensor-core forward saves every token's u and the state after every 64-token chunk, then a
// reverse chain over the chunks and per-chunk products); this walk takes the other heads.
#include <algorithm>
#include <cstdint>

#include "bwd_gate.cuh"
#include "common.cuh"
#include "launchers.h"

namespace efla {

constexpr int BW_THREADS = 128;  // one state row per thread (dk <= 128)
constexpr int BW_CB = 16;        // state columns per CTA
constexpr int BWD_BLOCK = 64;    // tokens between stored states (even: tokens go in pairs)

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

struct BwdRed {  // the four warps' shares of one CTA-wide sum, double-buffered by parity
    float col[2][BW_THREADS / 32][2 * BW_CB];
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

// Sum over the warp of 32 values per lane, scattered: lane l returns the sum of value l.  Each
// step halves the values a lane keeps and trades the other half with the lane whose index
// differs in one bit: 16 + 8 + 4 + 2 + 1 shuffles in place of 32 x 5.
__device__ __forceinline__ float warp_reduce_scatter32(float (&p)[2 * BW_CB], int lane) {
#pragma unroll
    for (int h = 16; h >= 1; h >>= 1) {
        const bool up = lane & h;
#pragma unroll
        for (int m = 0; m < h; ++m) {
            const float send = up ? p[m] : p[m + h], keep = up ? p[m + h] : p[m];
            p[m] = keep + __shfl_xor_sync(0xffffffffu, send, h);
        }
    }
    return p[0];
}

// CTA-wide sums of p[0..32) into out (every thread calls it; one barrier).  Lane l adds up the
// four warps' shares of value l and the totals reach every lane by shuffles: shared memory sees
// one conflict-free load per warp share, not a broadcast read of all of them by every thread.
__device__ __forceinline__ void cta_sum32(float (&p)[2 * BW_CB], BwdRed &red, int par,
                                          float (&out)[2 * BW_CB]) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    red.col[par][w][lane] = warp_reduce_scatter32(p, lane);
    __syncthreads();
    float t = red.col[par][0][lane];
#pragma unroll
    for (int ww = 1; ww < BW_THREADS / 32; ++ww) t += red.col[par][ww][lane];
#pragma unroll
    for (int j = 0; j < 2 * BW_CB; ++j) out[j] = __shfl_sync(0xffffffffu, t, j);
}

// Value i of a register array without dynamic indexing (which would go through local memory).
__device__ __forceinline__ float pick(const float *x, int i) {
    float m = 0.f;
#pragma unroll
    for (int j = 0; j < BW_CB; ++j) m = (i == j) ? x[j] : m;
    return m;
}

__device__ __forceinline__ void load_row16(const float *p, float *x) {
#pragma unroll
    for (int j4 = 0; j4 < BW_CB / 4; ++j4) {
        const float4 a = reinterpret_cast<const float4 *>(p)[j4];
        x[4 * j4] = a.x; x[4 * j4 + 1] = a.y; x[4 * j4 + 2] = a.z; x[4 * j4 + 3] = a.w;
    }
}

__device__ __forceinline__ void store_row16(float *p, const float *x) {
#pragma unroll
    for (int j4 = 0; j4 < BW_CB / 4; ++j4)
        reinterpret_cast<float4 *>(p)[j4] = make_float4(x[4 * j4], x[4 * j4 + 1], x[4 * j4 + 2], x[4 * j4 + 3]);
}

// Per token t, two float4: (lambda = |k_t|^2, a_t, df/dbeta, df/dlambda) and
// (q_t . k_t, k_t . k_{t-1}, 0, 0) (k_{-1} = 0); one warp per token.  Every column block of a
// head reads them, so they are computed once, ahead of the sweeps.  It also gathers, per head,
// what decides whether the head takes the tensor-core forward's saved values (bwd_gate.cuh):
// hs[head] = {a token has a <= 0 (or NaN); max lambda (float bits); INT_MAX - min a (float bits);
// max a (float bits)}, every field zero-initialised (a >= 0, lambda >= 0, so the bit patterns
// order as the values do).
template <typename T>
__global__ void __launch_bounds__(256) bwd_coeff_kernel(const T *__restrict__ q, const T *__restrict__ k,
                                                       const T *__restrict__ beta, size_t ntok, int L,
                                                       int dk, bool euler, float4 *__restrict__ coef,
                                                       int *__restrict__ hs) {
    // Work units of up to 64 tokens within one head, one warp each.  The warp computes the dot
    // products of 32 tokens at a time (8 tokens' rows loaded at once, lane i holding elements
    // i, i + 32, ... of a row) and hands token j's sums to lane j, so the coefficients of the
    // 32 tokens are computed by the 32 lanes side by side; the head's gate statistics are
    // reduced over the warp and added to hs once per unit.
    constexpr int UNIT = 64, RJ = 4;  // dk <= 128
    const int lane = threadIdx.x & 31;
    const long long BH = (long long)(ntok / (size_t)L), upH = (L + UNIT - 1) / UNIT;
    const long long nw = (long long)gridDim.x * 8, w0 = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    for (long long u = w0; u < BH * upH; u += nw) {
        const long long head = u / upH;
        const int r0 = (int)(u % upH) * UNIT, r1 = min(L, r0 + UNIT);
        const size_t hb = (size_t)head * L;
        int bad = 0, m_lam = 0, m_ia = 0, m_a = 0;
        float kprev[RJ];  // k of the token before the current one (0 before the head's first)
#pragma unroll
        for (int e = 0; e < RJ; ++e) {
            const int i = lane + 32 * e;
            kprev[e] = (r0 > 0 && i < dk) ? to_f32(k[(hb + r0 - 1) * dk + i]) : 0.f;
        }
        for (int g0 = r0; g0 < r1; g0 += 32) {
            float mylam = 0.f, myqk = 0.f, mykk = 0.f;
            for (int b0 = 0; b0 < 32 && g0 + b0 < r1; b0 += 8) {
                float kx[8][RJ], qx[8][RJ];
#pragma unroll
                for (int j = 0; j < 8; ++j)
#pragma unroll
                    for (int e = 0; e < RJ; ++e) {
                        const int t = g0 + b0 + j, i = lane + 32 * e;
                        const bool in = t < r1 && i < dk;
                        kx[j][e] = in ? to_f32(k[(hb + t) * dk + i]) : 0.f;
                        qx[j][e] = in ? to_f32(q[(hb + t) * dk + i]) : 0.f;
                    }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float lam = 0.f, qk = 0.f, kk = 0.f;
#pragma unroll
                    for (int e = 0; e < RJ; ++e) {
                        const float kp = j == 0 ? kprev[e] : kx[j - 1][e];
                        lam = fmaf(kx[j][e], kx[j][e], lam);
                        qk = fmaf(qx[j][e], kx[j][e], qk);
                        kk = fmaf(kp, kx[j][e], kk);
                    }
                    lam = warp_sum(lam);
                    qk = warp_sum(qk);
                    kk = warp_sum(kk);
                    if (lane == b0 + j) {
                        mylam = lam;
                        myqk = qk;
                        mykk = g0 + b0 + j == 0 ? 0.f : kk;  // k_{-1} = 0
                    }
                }
#pragma unroll
                for (int e = 0; e < RJ; ++e) kprev[e] = kx[7][e];
            }
            const int t = g0 + lane;
            if (t < r1) {
                const size_t tok = hb + t;
                const float bt = to_f32(beta[tok]);
                const float a = alpha_rule(mylam, bt, euler);
                float dfdb, dfdl;
                coeff_grads(mylam, bt, euler, a, dfdb, dfdl);
                coef[2 * tok] = make_float4(mylam, a, dfdb, dfdl);
                coef[2 * tok + 1] = make_float4(myqk, mykk, 0.f, 0.f);
                // a zero a (u / a cannot give r), a negative one (from a negative beta) or NaN
                // would also escape the min/max statistics, whose integer order holds for
                // positive floats only: all of them send the head to the fp32 walk
                if (!(a > 0.f)) bad = 1;
                m_lam = max(m_lam, __float_as_int(mylam));
                m_ia = max(m_ia, 0x7fffffff - __float_as_int(a));
                m_a = max(m_a, __float_as_int(a));
            }
        }
        bad = __any_sync(0xffffffffu, bad);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            m_lam = max(m_lam, __shfl_xor_sync(0xffffffffu, m_lam, o));
            m_ia = max(m_ia, __shfl_xor_sync(0xffffffffu, m_ia, o));
            m_a = max(m_a, __shfl_xor_sync(0xffffffffu, m_a, o));
        }
        if (lane == 0) {
            int *h = hs + 4 * head;
            if (bad) atomicOr(h, 1);
            atomicMax(h + 1, m_lam);
            atomicMax(h + 2, m_ia);
            atomicMax(h + 3, m_a);
        }
    }
}

// The same for bf16 rows of 64 or 128 elements, 16-byte aligned: eight lanes per token (16-byte
// loads, a row's dot products summed over the eight), four tokens per warp at a time, and the
// coefficients of a token computed by the first lane of its eight.  Without PAIRS (the form that
// runs before the tensor-core backward) it writes only the first record (lambda, a and the two
// derivatives) and reads no q: the second record (q_t . k_t, k_{t-1} . k_t) is for the heads that
// walk on CUDA cores, which bwd_pairs_vec_kernel fills once the gate has been decided.  That form
// also rounds its unit's rows of dO (fp32, dv per token) to the fp16 copy dO16 that the
// tensor-core products read.
template <int DKV, bool PAIRS = true>
__global__ void __launch_bounds__(256) bwd_coeff_vec_kernel(const __nv_bfloat16 *__restrict__ q,
                                                           const __nv_bfloat16 *__restrict__ k,
                                                           const __nv_bfloat16 *__restrict__ beta, size_t ntok,
                                                           int L, bool euler, float4 *__restrict__ coef,
                                                           int *__restrict__ hs, const float *__restrict__ dO,
                                                           __half *__restrict__ dO16, int dv) {
    constexpr int UNIT = 64, EPL = DKV / 8, NV = EPL / 8;  // elements and 16-byte words per lane
    const int lane = threadIdx.x & 31, g = lane >> 3, sl = lane & 7;
    const long long BH = (long long)(ntok / (size_t)L), upH = (L + UNIT - 1) / UNIT;
    const long long nw = (long long)gridDim.x * 8, w0 = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    auto dot = [](const uint4 &a, const uint4 &b) {
        const __nv_bfloat162 *x = reinterpret_cast<const __nv_bfloat162 *>(&a);
        const __nv_bfloat162 *y = reinterpret_cast<const __nv_bfloat162 *>(&b);
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 u = __bfloat1622float2(x[e]), v = __bfloat1622float2(y[e]);
            s = fmaf(u.x, v.x, fmaf(u.y, v.y, s));
        }
        return s;
    };
    for (long long u = w0; u < BH * upH; u += nw) {
        const long long head = u / upH;
        const int r0 = (int)(u % upH) * UNIT, r1 = min(L, r0 + UNIT);
        const size_t hb = (size_t)head * L;
        int bad = 0, m_lam = 0, m_ia = 0, m_a = 0;
        for (int t = r0 + g; t - g < r1; t += 4) {
            const bool in = t < r1;
            const size_t tok = hb + (in ? t : r0);
            uint4 kx[NV], qx[NV], kp[NV];
#pragma unroll
            for (int w = 0; w < NV; ++w) {
                const size_t o = tok * DKV + (size_t)sl * EPL + 8 * w;
                kx[w] = *reinterpret_cast<const uint4 *>(k + o);
                if constexpr (PAIRS) {
                    qx[w] = *reinterpret_cast<const uint4 *>(q + o);
                    kp[w] = (in && t > 0) ? *reinterpret_cast<const uint4 *>(k + o - DKV) : make_uint4(0u, 0u, 0u, 0u);
                }
            }
            float lam = 0.f, qk = 0.f, kk = 0.f;
#pragma unroll
            for (int w = 0; w < NV; ++w) {
                lam += dot(kx[w], kx[w]);
                if constexpr (PAIRS) {
                    qk += dot(qx[w], kx[w]);
                    kk += dot(kp[w], kx[w]);
                }
            }
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) {
                lam += __shfl_xor_sync(0xffffffffu, lam, o);
                if constexpr (PAIRS) {
                    qk += __shfl_xor_sync(0xffffffffu, qk, o);
                    kk += __shfl_xor_sync(0xffffffffu, kk, o);
                }
            }
            if (in && sl == 0) {
                const float bt = __bfloat162float(beta[tok]);
                const float a = alpha_rule(lam, bt, euler);
                float dfdb, dfdl;
                coeff_grads(lam, bt, euler, a, dfdb, dfdl);
                coef[2 * tok] = make_float4(lam, a, dfdb, dfdl);
                if constexpr (PAIRS) coef[2 * tok + 1] = make_float4(qk, kk, 0.f, 0.f);
                // see bwd_coeff_kernel: any a that is not positive fails the gate
                if (!(a > 0.f)) bad = 1;
                m_lam = max(m_lam, __float_as_int(lam));
                m_ia = max(m_ia, 0x7fffffff - __float_as_int(a));
                m_a = max(m_a, __float_as_int(a));
            }
        }
        if constexpr (!PAIRS) {  // the unit's rows of dO, 16 bytes in and 8 out per lane at a time
            const size_t e0 = (hb + r0) * (size_t)dv / 4, n4 = (size_t)(r1 - r0) * dv / 4;
            const float4 *src = reinterpret_cast<const float4 *>(dO) + e0;
            uint2 *dst = reinterpret_cast<uint2 *>(dO16) + e0;
#pragma unroll 4
            for (size_t e = lane; e < n4; e += 32) {
                const float4 x = src[e];
                const __half2 lo = __floats2half2_rn(x.x, x.y), hi = __floats2half2_rn(x.z, x.w);
                dst[e] = make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
            }
        }
        bad = __any_sync(0xffffffffu, bad);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            m_lam = max(m_lam, __shfl_xor_sync(0xffffffffu, m_lam, o));
            m_ia = max(m_ia, __shfl_xor_sync(0xffffffffu, m_ia, o));
            m_a = max(m_a, __shfl_xor_sync(0xffffffffu, m_a, o));
        }
        if (lane == 0) {
            int *h = hs + 4 * head;
            if (bad) atomicOr(h, 1);
            atomicMax(h + 1, m_lam);
            atomicMax(h + 2, m_ia);
            atomicMax(h + 3, m_a);
        }
    }
}

// The second coefficient record (q_t . k_t, k_{t-1} . k_t) of the heads that the gate sends to the
// CUDA-core walk, after bwd_coeff_vec_kernel<DKV, false> has decided it; the same lanes and dot
// products as that kernel's PAIRS form.  Warps whose unit belongs to a tensor-core head skip it.
template <int DKV>
__global__ void __launch_bounds__(256) bwd_pairs_vec_kernel(const __nv_bfloat16 *__restrict__ q,
                                                           const __nv_bfloat16 *__restrict__ k, size_t ntok,
                                                           int L, float4 *__restrict__ coef,
                                                           const int *__restrict__ hs) {
    constexpr int UNIT = 64, EPL = DKV / 8, NV = EPL / 8;
    const int lane = threadIdx.x & 31, g = lane >> 3, sl = lane & 7;
    const long long BH = (long long)(ntok / (size_t)L), upH = (L + UNIT - 1) / UNIT;
    const long long nw = (long long)gridDim.x * 8, w0 = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    auto dot = [](const uint4 &a, const uint4 &b) {
        const __nv_bfloat162 *x = reinterpret_cast<const __nv_bfloat162 *>(&a);
        const __nv_bfloat162 *y = reinterpret_cast<const __nv_bfloat162 *>(&b);
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 u = __bfloat1622float2(x[e]), v = __bfloat1622float2(y[e]);
            s = fmaf(u.x, v.x, fmaf(u.y, v.y, s));
        }
        return s;
    };
    for (long long u = w0; u < BH * upH; u += nw) {
        const long long head = u / upH;
        if (head_takes_saved(hs, head)) continue;  // uniform over the warp
        const int r0 = (int)(u % upH) * UNIT, r1 = min(L, r0 + UNIT);
        const size_t hb = (size_t)head * L;
        for (int t = r0 + g; t - g < r1; t += 4) {
            const bool in = t < r1;
            const size_t tok = hb + (in ? t : r0);
            uint4 kx[NV], qx[NV], kp[NV];
#pragma unroll
            for (int w = 0; w < NV; ++w) {
                const size_t o = tok * DKV + (size_t)sl * EPL + 8 * w;
                kx[w] = *reinterpret_cast<const uint4 *>(k + o);
                qx[w] = *reinterpret_cast<const uint4 *>(q + o);
                kp[w] = (in && t > 0) ? *reinterpret_cast<const uint4 *>(k + o - DKV) : make_uint4(0u, 0u, 0u, 0u);
            }
            float qk = 0.f, kk = 0.f;
#pragma unroll
            for (int w = 0; w < NV; ++w) {
                qk += dot(qx[w], kx[w]);
                kk += dot(kp[w], kx[w]);
            }
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) {
                qk += __shfl_xor_sync(0xffffffffu, qk, o);
                kk += __shfl_xor_sync(0xffffffffu, kk, o);
            }
            if (in && sl == 0) coef[2 * tok + 1] = make_float4(qk, kk, 0.f, 0.f);
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(BW_THREADS, 4)
    bwd_cols_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                    const float4 *__restrict__ coef, const float *__restrict__ S0,
                    const float *__restrict__ dO, const float *__restrict__ dSL,
                    float *__restrict__ dval, float *__restrict__ dS0, int L, int dk, int dv, int NS,
                    float *__restrict__ ws, float *__restrict__ part, const int *__restrict__ hs,
                    bool tc_heads) {
    __shared__ __align__(16) BwdRed red;
    __shared__ __align__(16) float xb[BWD_BLOCK][BW_CB];  // v (forward sweep) or dO (reverse)
    __shared__ __align__(16) float rb[BWD_BLOCK][BW_CB];  // r (reverse sweep)
    __shared__ __align__(16) float4 cb[BWD_BLOCK][2];     // the block's token coefficients
    const int tid = threadIdx.x, row = tid;
    const int bh = blockIdx.x / NS, s = blockIdx.x % NS, c0 = s * BW_CB;
    const int BH = gridDim.x / NS, nc = min(BW_CB, dv - c0);
    const int NB = (L + BWD_BLOCK - 1) / BWD_BLOCK;
    const bool act = row < dk;
    const size_t tk = (size_t)bh * L * dk, tv = (size_t)bh * L * dv, tb = (size_t)bh * L;
    const size_t DD = (size_t)dk * dv;
    float *R = ws + ((size_t)bh * NS + s) * ((size_t)L * BW_CB + (size_t)(NB + 1) * dk * BW_CB);
    float *CK = R + (size_t)L * BW_CB;
    const size_t nq = (size_t)BH * L * dk;
    float *pdq = part + (size_t)s * nq + tk;
    float *pdk = part + (size_t)NS * nq + (size_t)s * nq + tk;
    float *pdb = part + 2 * (size_t)NS * nq + (size_t)s * BH * L + tb;
    // With tc_heads, the heads the gate admits (bwd_gate.cuh) take the tensor-core backward; this
    // kernel walks the others (uniform over the CTA: one head per CTA).
    if (tc_heads && head_takes_saved(hs, bh)) return;
    auto ld = [&](const T *x, int t) {  // row `row` of token t's q or k (0 off the sequence)
        return (act && t >= 0 && t < L) ? to_f32(x[tk + (size_t)t * dk + row]) : 0.f;
    };
    // the block's per-token rows and coefficients, zero at the absent partner of an odd count
    auto stage = [&](int t0, int cnt, bool reverse) {
        const int n = cnt + (cnt & 1);
        for (int e = tid; e < n * BW_CB; e += BW_THREADS) {
            const int tt = e / BW_CB, j = e % BW_CB;
            const bool in = tt < cnt && j < nc;
            const size_t g = tv + (size_t)(t0 + tt) * dv + c0 + j;
            if (reverse) {
                xb[tt][j] = in ? dO[g] : 0.f;
                rb[tt][j] = tt < cnt ? R[(size_t)(t0 + tt) * BW_CB + j] : 0.f;
            } else {
                xb[tt][j] = in ? to_f32(v[g]) : 0.f;
            }
        }
        for (int e = tid; e < 2 * n; e += BW_THREADS)
            cb[e >> 1][e & 1] = (e >> 1) < cnt ? coef[2 * (tb + t0) + e] : make_float4(0.f, 0.f, 0.f, 0.f);
    };

    float S[BW_CB], G[BW_CB];
#pragma unroll
    for (int j = 0; j < BW_CB; ++j)
        S[j] = (S0 && act && j < nc) ? S0[(size_t)bh * DD + (size_t)row * dv + c0 + j] : 0.f;

    // ---- forward sweep: r of every token and the block-boundary states
    int par = 0;
    float kn0 = ld(k, 0), kn1 = ld(k, 1);  // k rows of the next pair
    for (int b = 0; b < NB; ++b) {
        const int t0 = b * BWD_BLOCK, cnt = min(BWD_BLOCK, L - t0);
        __syncthreads();  // the previous block's reads of xb and cb are done
        stage(t0, cnt, false);
        if (act) store_row16(CK + ((size_t)b * dk + row) * BW_CB, S);
        __syncthreads();
        for (int tt = 0; tt < cnt; tt += 2) {
            const int t = t0 + tt;
            const float k0 = kn0, k1 = kn1;
            kn0 = ld(k, t + 2);
            kn1 = ld(k, t + 3);
            float p[2 * BW_CB], y[2 * BW_CB];
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) {
                mul2(p[j], p[j + 1], S[j], S[j + 1], k0, k0);
                mul2(p[BW_CB + j], p[BW_CB + j + 1], S[j], S[j + 1], k1, k1);
            }
            cta_sum32(p, red, par, y);  // y = [S^T k_t | S^T k_{t+1}]
            const float a0 = cb[tt][0].y, a1 = cb[tt + 1][0].y, kap = cb[tt + 1][1].y;
            float r0[BW_CB], r1[BW_CB];
            load_row16(xb[tt], r0);
            load_row16(xb[tt + 1], r1);
            const float c = a0 * kap;
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) {
                add2(r0[j], r0[j + 1], -y[j], -y[j + 1]);  // r_t = v_t - S^T k_t
                float x0 = y[BW_CB + j], x1 = y[BW_CB + j + 1];
                fma2(x0, x1, c, c, r0[j], r0[j + 1]);      // S_t^T k_{t+1}
                add2(r1[j], r1[j + 1], -x0, -x1);
            }
            if (tid < BW_CB) {
                R[(size_t)t * BW_CB + tid] = pick(r0, tid);
                if (tt + 1 < cnt) R[(size_t)(t + 1) * BW_CB + tid] = pick(r1, tid);
            }
            const float ak0 = a0 * k0, ak1 = a1 * k1;
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) {
                fma2(S[j], S[j + 1], ak0, ak0, r0[j], r0[j + 1]);
                fma2(S[j], S[j + 1], ak1, ak1, r1[j], r1[j + 1]);
            }
            par ^= 1;
        }
    }
    if (act) store_row16(CK + ((size_t)NB * dk + row) * BW_CB, S);

    // ---- reverse sweep
#pragma unroll
    for (int j = 0; j < BW_CB; ++j)
        G[j] = (dSL && act && j < nc) ? dSL[(size_t)bh * DD + (size_t)row * dv + c0 + j] : 0.f;
    // the top pair of the last block: (L, L-1) when L is odd (token L absent), else (L-1, L-2)
    const int top = L - 1 + (L & 1);
    kn0 = ld(k, top);
    kn1 = ld(k, top - 1);
    float qn0 = ld(q, top), qn1 = ld(q, top - 1);
    for (int b = NB - 1; b >= 0; --b) {
        const int t0 = b * BWD_BLOCK, cnt = min(BWD_BLOCK, L - t0);
        __syncthreads();  // the previous block's reads of xb, rb and cb are done
        stage(t0, cnt, true);
        if (act) load_row16(CK + ((size_t)(b + 1) * dk + row) * BW_CB, S);  // S' after the block
        __syncthreads();
        for (int tt = cnt - 1 + (cnt & 1); tt > 0; tt -= 2) {  // pair (t, t-1), t = t0 + tt
            const int t = t0 + tt;
            const float k0 = kn0, k1 = kn1, q0 = qn0, q1 = qn1;
            kn0 = ld(k, t - 2);
            kn1 = ld(k, t - 3);
            qn0 = ld(q, t - 2);
            qn1 = ld(q, t - 3);
            float d0[BW_CB], r0[BW_CB];
            load_row16(xb[tt], d0);
            load_row16(rb[tt], r0);
            // token t: G1 = G + q_t do_t^T;  dq_t = S_t do_t
            float dqa = 0.f, dqb = 0.f;
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) {
                fma2(G[j], G[j + 1], q0, q0, d0[j], d0[j + 1]);
                fma2(dqa, dqb, S[j], S[j + 1], d0[j], d0[j + 1]);
            }
            float p[2 * BW_CB], du[2 * BW_CB];  // du = [G1^T k_t | G1^T k_{t-1}]
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) {
                mul2(p[j], p[j + 1], G[j], G[j + 1], k0, k0);
                mul2(p[BW_CB + j], p[BW_CB + j + 1], G[j], G[j + 1], k1, k1);
            }
            cta_sum32(p, red, par, du);
            const float4 cA0 = cb[tt][0], cB0 = cb[tt][1], cA1 = cb[tt - 1][0], cB1 = cb[tt - 1][1];
            const float a0 = cA0.y, a1 = cA1.y;
            // token t: da, S_{t-1} = S_t - a k r^T, dk, G2 = G1 - a k du^T
            float daa = 0.f, dab = 0.f;
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) fma2(daa, dab, du[j], du[j + 1], r0[j], r0[j + 1]);
            const float da0 = daa + dab;
            {
                const float nak = -a0 * k0;
                float gr0 = 0.f, gr1 = 0.f, sd0 = 0.f, sd1 = 0.f;
#pragma unroll
                for (int j = 0; j < BW_CB; j += 2) {
                    fma2(S[j], S[j + 1], nak, nak, r0[j], r0[j + 1]);
                    fma2(gr0, gr1, G[j], G[j + 1], r0[j], r0[j + 1]);
                    fma2(sd0, sd1, S[j], S[j + 1], du[j], du[j + 1]);
                    fma2(G[j], G[j + 1], nak, nak, du[j], du[j + 1]);
                }
                if (tt < cnt) {
                    if (act) {
                        pdq[(size_t)t * dk + row] = dqa + dqb;
                        pdk[(size_t)t * dk + row] = a0 * ((gr0 + gr1) - (sd0 + sd1)) + 2.f * da0 * cA0.w * k0;
                    }
                    if (tid < nc) dval[tv + (size_t)t * dv + c0 + tid] = a0 * pick(du, tid);
                    if (tid == 0) pdb[t] = da0 * cA0.z;
                }
            }
            // token t-1: du_{t-1} = z - a_t (k_t . k_{t-1}) du_t + (q_{t-1} . k_{t-1}) do_{t-1}
            float d1[BW_CB], r1[BW_CB];
            load_row16(xb[tt - 1], d1);
            load_row16(rb[tt - 1], r1);
            {
                const float c = -a0 * cB0.y, e = cB1.x;
#pragma unroll
                for (int j = 0; j < BW_CB; j += 2) {
                    fma2(du[BW_CB + j], du[BW_CB + j + 1], c, c, du[j], du[j + 1]);
                    fma2(du[BW_CB + j], du[BW_CB + j + 1], e, e, d1[j], d1[j + 1]);
                }
            }
            float *du1 = du + BW_CB;
            // G3 = G2 + q_{t-1} do_{t-1}^T;  dq_{t-1} = S_{t-1} do_{t-1}
            dqa = 0.f;
            dqb = 0.f;
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) {
                fma2(G[j], G[j + 1], q1, q1, d1[j], d1[j + 1]);
                fma2(dqa, dqb, S[j], S[j + 1], d1[j], d1[j + 1]);
            }
            daa = 0.f;
            dab = 0.f;
#pragma unroll
            for (int j = 0; j < BW_CB; j += 2) fma2(daa, dab, du1[j], du1[j + 1], r1[j], r1[j + 1]);
            const float da1 = daa + dab;
            {
                const float nak = -a1 * k1;
                float gr0 = 0.f, gr1 = 0.f, sd0 = 0.f, sd1 = 0.f;
#pragma unroll
                for (int j = 0; j < BW_CB; j += 2) {
                    fma2(S[j], S[j + 1], nak, nak, r1[j], r1[j + 1]);
                    fma2(gr0, gr1, G[j], G[j + 1], r1[j], r1[j + 1]);
                    fma2(sd0, sd1, S[j], S[j + 1], du1[j], du1[j + 1]);
                    fma2(G[j], G[j + 1], nak, nak, du1[j], du1[j + 1]);
                }
                if (act) {
                    pdq[(size_t)(t - 1) * dk + row] = dqa + dqb;
                    pdk[(size_t)(t - 1) * dk + row] = a1 * ((gr0 + gr1) - (sd0 + sd1)) + 2.f * da1 * cA1.w * k1;
                }
                if (tid < nc) dval[tv + (size_t)(t - 1) * dv + c0 + tid] = a1 * pick(du1, tid);
                if (tid == 0) pdb[t - 1] = da1 * cA1.z;
            }
            par ^= 1;
        }
    }
    if (dS0 && act) {
#pragma unroll
        for (int j = 0; j < BW_CB; ++j)
            if (j < nc) dS0[(size_t)bh * DD + (size_t)row * dv + c0 + j] = G[j];
    }
}

// out[e] = sum over s = 0..NS-1 of part[s n + e], in that order; with tc_hs, the heads that the
// tensor-core backward takes are left alone.
struct SumSeg {
    const float *part;
    float *out;
    size_t n;
    size_t per_head;  // elements per head
    int vec;          // 1: n and per_head multiples of 4, both arrays 16-byte aligned
};
struct SumSegs {
    SumSeg seg[3];
};

// Grid: (BH x SL, 3): block x takes head x / SL and, within it, every SL-th piece of 256
// elements (float4 groups when vec); blockIdx.y picks dq, dk or dbeta.
__global__ void __launch_bounds__(256) bwd_sum_kernel(SumSegs segs, int NS, int SL, const int *__restrict__ tc_hs) {
    const SumSeg g = blockIdx.y == 0 ? segs.seg[0] : (blockIdx.y == 1 ? segs.seg[1] : segs.seg[2]);
    const long long head = blockIdx.x / SL;
    const int sl = blockIdx.x % SL;
    if (tc_hs && head_takes_saved(tc_hs, head)) return;
    if (g.vec) {
        const size_t n4 = g.n / 4, ph4 = g.per_head / 4, h0 = (size_t)head * ph4;
        const float4 *p4 = reinterpret_cast<const float4 *>(g.part);
        float4 *o4 = reinterpret_cast<float4 *>(g.out);
        for (size_t e = h0 + (size_t)sl * blockDim.x + threadIdx.x; e < h0 + ph4; e += (size_t)SL * blockDim.x) {
            float4 a = p4[e];
            for (int s = 1; s < NS; ++s) {
                const float4 b = p4[(size_t)s * n4 + e];
                a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
            }
            o4[e] = a;
        }
    } else {
        const size_t h0 = (size_t)head * g.per_head;
        for (size_t e = h0 + (size_t)sl * blockDim.x + threadIdx.x; e < h0 + g.per_head; e += (size_t)SL * blockDim.x) {
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

// Sizes for which the tensor-core forward (bf16 inputs) saves u and the block states for the
// reverse sweep.  The workspace is sized for it whenever the sizes allow it (the input dtype is
// not an argument of the size query).
static bool bwd_tc_saves(int B, int H, int L, int dk, int dv) {
    return L > 0 && tc_supported(B, H, L, dk, dv, BWD_BLOCK, true);
}

struct BwdLayout {  // float offsets into the workspace
    size_t coef, zero, state, part, tc, u, ck, tcb, total;
};

static BwdLayout bwd_layout(int B, int H, int L, int dk, int dv) {
    const size_t BH = (size_t)B * H, NS = (size_t)(dv + BW_CB - 1) / BW_CB, ntok = BH * (size_t)L;
    const size_t NB = (size_t)(L + BWD_BLOCK - 1) / BWD_BLOCK;
    auto up = [](size_t f) { return (f + 63) / 64 * 64; };  // every region 256-byte aligned
    BwdLayout a;
    a.coef = 0;
    a.zero = up(8 * ntok);
    a.state = a.zero + up(4 * BH);
    a.part = a.state + up(bwd_state_floats(BH, L, dk, dv));
    a.tc = a.part + up(NS * ntok * (2 * (size_t)dk + 1));
    a.u = a.ck = a.tcb = a.total = a.tc;
    if (bwd_tc_saves(B, H, L, dk, dv)) {
        a.u = a.tc + up((tc_workspace_bytes(B, H, L, dk, dv, BWD_BLOCK) + 3) / 4);
        a.ck = a.u + up((ntok * (size_t)dv + 1) / 2);  // fp16
        a.tcb = a.ck + up((BH * NB * (size_t)dk * dv + 1) / 2);
        a.total = a.tcb + (bwd_tc_workspace_bytes(B, H, L, dk, dv) + 3) / 4;
    }
    return a;
}

size_t bwd_workspace_bytes(int B, int H, int L, int dk, int dv) {
    return bwd_layout(B, H, L, dk, dv).total * sizeof(float);
}

// The kept buffer: the forward's workspace (Ta tiles, segment states), every token's u and the
// state after every chunk, in the order and with the sizes of the workspace's own regions.
size_t bwd_kept_bytes(int B, int H, int L, int dk, int dv) {
    if (!bwd_tc_saves(B, H, L, dk, dv)) return 0;
    const BwdLayout lay = bwd_layout(B, H, L, dk, dv);
    return (lay.tcb - lay.tc) * sizeof(float);
}

bool bwd_kept_regions(int B, int H, int L, int dk, int dv, bool is_bf16, void *kept, void **tc_ws, __half **u,
                      __half **ck) {
    if (!is_bf16 || !bwd_tc_saves(B, H, L, dk, dv)) return false;
    const BwdLayout lay = bwd_layout(B, H, L, dk, dv);
    float *kf = (float *)kept;
    *tc_ws = kf;
    *u = (__half *)(kf + (lay.u - lay.tc));
    *ck = (__half *)(kf + (lay.ck - lay.tc));
    return true;
}

cudaError_t launch_bwd(const void *q, const void *k, const void *v, const void *beta,
                       const float *S0, const float *dO, const float *dSL, float *dq, float *dkey,
                       float *dval, float *dbeta, float *dS0, int B, int H, int L, int dk, int dv,
                       bool is_bf16, bool euler, void *ws, cudaStream_t s, const void *kept) {
    const long long BH = (long long)B * H;
    const int NS = (dv + BW_CB - 1) / BW_CB;
    if (BH * NS > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const size_t ntok = (size_t)BH * L;
    const BwdLayout lay = bwd_layout(B, H, L, dk, dv);
    float *wsf = (float *)ws;
    float4 *coef = (float4 *)(wsf + lay.coef);
    int *hs = (int *)(wsf + lay.zero);  // per-head statistics for the saved-forward gate
    float *state = wsf + lay.state;
    float *part = wsf + lay.part;
    __half *u_saved = nullptr, *ck_saved = nullptr;
    void *ta_ws = wsf + lay.tc;  // the tensor-core forward's workspace (its Ta tiles)
    cudaError_t e;
    // the tensor-core forward (TMA) and backward load q, k, v, S0 and dO 16 bytes at a time and
    // store dq, dk, dv 8 bytes at a time; arrays that are only element-aligned send every head to
    // the CUDA-core path
    auto al16 = [](const void *p) { return ((uintptr_t)p & 15) == 0; };
    auto al8 = [](const void *p) { return ((uintptr_t)p & 7) == 0; };
    const bool tc_bwd = is_bf16 && bwd_tc_saves(B, H, L, dk, dv) && al16(q) && al16(k) && al16(v) &&
                        al16(dO) && (S0 == nullptr || al16(S0)) && al8(dq) && al8(dkey) && al8(dval);
    if (tc_bwd) {
        // the tensor-core forward, saving u and the block states (fp16) instead of writing outputs
        if (kept) {  // the forward of this step kept them
            bwd_kept_regions(B, H, L, dk, dv, true, const_cast<void *>(kept), &ta_ws, &u_saved, &ck_saved);
        } else {
            u_saved = (__half *)(wsf + lay.u);
            ck_saved = (__half *)(wsf + lay.ck);
            e = launch_chunk_tc_save(q, k, v, beta, S0, B, H, L, dk, dv, euler, ta_ws, u_saved, ck_saved, s);
            if (e != cudaSuccess) return e;
        }
    }
    bool dO16_done = false;  // the coefficient pass has written dO's fp16 copy
    if (ntok > 0) {
        e = cudaMemsetAsync(hs, 0, 4 * (size_t)BH * sizeof(int), s);
        if (e != cudaSuccess) return e;
        // one warp per unit of up to 64 tokens within a head
        const long long units = (long long)BH * ((L + 63) / 64);
        const int gc = (int)std::max<long long>(1, std::min<long long>((units + 7) / 8, (long long)nsm * 64));
        const bool vec_rows = is_bf16 && (dk == 64 || dk == 128) && ((uintptr_t)q & 15) == 0 &&
                              ((uintptr_t)k & 15) == 0;
        const __nv_bfloat16 *qb = (const __nv_bfloat16 *)q, *kb = (const __nv_bfloat16 *)k;
        if (vec_rows && tc_bwd) {
            // the first records and the gate; then the second records of the heads the gate
            // sends to the CUDA-core walk only (the tensor-core heads never read them)
            const __nv_bfloat16 *bb = (const __nv_bfloat16 *)beta;
            // and dO's fp16 copy for the tensor-core products, at the head of their workspace
            __half *dO16 = (__half *)(wsf + lay.tcb);
            const int gp = std::min(gc, nsm);  // its warps mostly only check the gate
            if (dk == 128) {
                bwd_coeff_vec_kernel<128, false><<<gc, 256, 0, s>>>(qb, kb, bb, ntok, L, euler, coef, hs, dO,
                                                                    dO16, dv);
                bwd_pairs_vec_kernel<128><<<gp, 256, 0, s>>>(qb, kb, ntok, L, coef, hs);
            } else {
                bwd_coeff_vec_kernel<64, false><<<gc, 256, 0, s>>>(qb, kb, bb, ntok, L, euler, coef, hs, dO,
                                                                   dO16, dv);
                bwd_pairs_vec_kernel<64><<<gp, 256, 0, s>>>(qb, kb, ntok, L, coef, hs);
            }
            dO16_done = true;
            count_launches(1);
        } else if (vec_rows && dk == 128)
            bwd_coeff_vec_kernel<128><<<gc, 256, 0, s>>>((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                                         (const __nv_bfloat16 *)beta, ntok, L, euler, coef, hs,
                                                         nullptr, nullptr, 0);
        else if (vec_rows)
            bwd_coeff_vec_kernel<64><<<gc, 256, 0, s>>>((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                                        (const __nv_bfloat16 *)beta, ntok, L, euler, coef, hs,
                                                        nullptr, nullptr, 0);
        else if (is_bf16)
            bwd_coeff_kernel<__nv_bfloat16><<<gc, 256, 0, s>>>(
                (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)beta, ntok, L,
                dk, euler, coef, hs);
        else
            bwd_coeff_kernel<float><<<gc, 256, 0, s>>>((const float *)q, (const float *)k,
                                                       (const float *)beta, ntok, L, dk, euler, coef,
                                                       hs);
        count_launches(1);
    }
    if (tc_bwd && L > 0) {
        e = launch_bwd_tc(q, k, v, S0, dO, dSL, coef, hs, u_saved, ck_saved, ta_ws, dq, dkey, dval, dbeta,
                          dS0, B, H, L, dk, dv, wsf + lay.tcb, s, dO16_done);
        if (e != cudaSuccess) return e;
    }
    const int grid = (int)(BH * NS);
    if (is_bf16)
        bwd_cols_kernel<__nv_bfloat16><<<grid, BW_THREADS, 0, s>>>(
            (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, coef, S0, dO,
            dSL, dval, dS0, L, dk, dv, NS, state, part, hs, tc_bwd);
    else
        bwd_cols_kernel<float><<<grid, BW_THREADS, 0, s>>>((const float *)q, (const float *)k,
                                                          (const float *)v, coef, S0, dO, dSL, dval,
                                                          dS0, L, dk, dv, NS, state, part, hs, false);
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess || L == 0) return e;
    // add the column blocks' shares of dq, dk and dbeta
    const size_t nq = (size_t)BH * L * dk, nb = (size_t)BH * L;
    auto seg = [&](const float *pp, float *out, size_t n, size_t per_head) {
        SumSeg g;
        g.part = pp;
        g.out = out;
        g.n = n;
        g.per_head = per_head;
        g.vec = (n % 4 == 0 && per_head % 4 == 0 && ((uintptr_t)pp % 16) == 0 && ((uintptr_t)out % 16) == 0)
                    ? 1 : 0;
        return g;
    };
    SumSegs segs;
    segs.seg[0] = seg(part, dq, nq, (size_t)L * dk);
    segs.seg[1] = seg(part + (size_t)NS * nq, dkey, nq, (size_t)L * dk);
    segs.seg[2] = seg(part + 2 * (size_t)NS * nq, dbeta, nb, (size_t)L);
    // slices per head: enough blocks to fill the GPU when every head walks; with the tensor-core
    // heads returning at once, about one block per SM (most blocks would only check the gate)
    const long long fill = tc_bwd ? std::max<long long>(1, nsm / BH) : ((long long)nsm * 8 + BH - 1) / BH;
    const int SL = (int)std::max<long long>(1, std::min<long long>(fill, ((long long)L * dk / 4 + 255) / 256));
    if (BH * SL > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    bwd_sum_kernel<<<dim3((unsigned)(BH * SL), 3), 256, 0, s>>>(segs, NS, SL, tc_bwd ? hs : nullptr);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace efla
