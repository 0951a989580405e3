// decode.cu -- recurrent single-token EFLA step per head (decode).
//
// "Exact Flow Linear Attention" technical summary, Methodology 3:
//   S_t = (I - alpha k k^T) S_{t-1} + alpha k v^T = S_{t-1} + k u^T,
//   u = alpha (v - S_{t-1}^T k),
// and the delta-rule readout o = S_t^T q = S_{t-1}^T q + (k.q) u.
// The gated form (a per-token decay g on the carried state, the gate placement of Gated
// DeltaNet, which the summary names as a baseline) is S_t = g (I - alpha k k^T) S_{t-1} +
// alpha k v^T = g S_{t-1} + k u^T with u = alpha (v - g S_{t-1}^T k), o = g S_{t-1}^T q +
// (k.q) u; without a gate g = 1, and every product with it is exact.
//
// The step is HBM-bound: per head the fp32 state (dk*dv*4 bytes) is read once
// and written once; q, k, v and o are negligible.  One CTA per head.  In the
// register kernel each thread owns float4 column groups of several rows, so
// the state is read with 16-byte coalesced loads, kept in registers while the
// two column reductions (S^T k and S^T q) finish, and written back from the
// same registers.
#include "common.cuh"
#include "launchers.h"

namespace efla {

template <typename T, int DK, int DV>
struct DecodeCfg {
    static constexpr int TPR = DV / 4;                                // threads per row
    static constexpr int NT = (TPR * DK < 256) ? TPR * DK : 256;      // threads per CTA
    static constexpr int RPP = NT / TPR;                              // rows per pass
    static constexpr int PASSES = DK / RPP;
};

template <typename T, typename TO, int DK, int DV>
__global__ void __launch_bounds__(DecodeCfg<T, DK, DV>::NT)
    decode_reg_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                      const T *__restrict__ beta, const T *__restrict__ gate, float *__restrict__ S,
                      TO *__restrict__ o, bool euler) {
    using Cfg = DecodeCfg<T, DK, DV>;
    constexpr int TPR = Cfg::TPR, RPP = Cfg::RPP, PASSES = Cfg::PASSES, NT = Cfg::NT;
    __shared__ float ks[DK], qs[DK], vs[DV];
    __shared__ __align__(16) float us[DV];
    __shared__ __align__(16) float red_x[RPP][DV + 4];
    __shared__ __align__(16) float red_y[RPP][DV + 4];
    __shared__ float sc[2];  // alpha, k.q
    const int bh = blockIdx.x;
    const int tid = threadIdx.x;
    const float gt = gate ? to_f32(gate[bh]) : 1.f;
    for (int i = tid; i < DK; i += NT) {
        ks[i] = to_f32(k[(size_t)bh * DK + i]);
        qs[i] = to_f32(q[(size_t)bh * DK + i]);
    }
    for (int i = tid; i < DV; i += NT) vs[i] = to_f32(v[(size_t)bh * DV + i]);
    __syncthreads();
    if (tid < 32) {
        float l = 0.f, kq = 0.f;
        for (int i = tid; i < DK; i += 32) {
            l = fmaf(ks[i], ks[i], l);
            kq = fmaf(ks[i], qs[i], kq);
        }
        l = warp_sum(l);
        kq = warp_sum(kq);
        if (tid == 0) {
            sc[0] = alpha_rule(l, to_f32(beta[bh]), euler);
            sc[1] = kq;
        }
    }
    const int cg = tid % TPR, rg = tid / TPR;
    float4 *Sh = reinterpret_cast<float4 *>(S + (size_t)bh * DK * DV);
    float4 st[PASSES];
    float4 px = make_float4(0.f, 0.f, 0.f, 0.f), py = px;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int r = rg + p * RPP;
        st[p] = Sh[r * TPR + cg];
        const float kr = ks[r], qr = qs[r];
        px.x = fmaf(st[p].x, kr, px.x); px.y = fmaf(st[p].y, kr, px.y);
        px.z = fmaf(st[p].z, kr, px.z); px.w = fmaf(st[p].w, kr, px.w);
        py.x = fmaf(st[p].x, qr, py.x); py.y = fmaf(st[p].y, qr, py.y);
        py.z = fmaf(st[p].z, qr, py.z); py.w = fmaf(st[p].w, qr, py.w);
    }
    *reinterpret_cast<float4 *>(&red_x[rg][4 * cg]) = px;
    *reinterpret_cast<float4 *>(&red_y[rg][4 * cg]) = py;
    __syncthreads();
    for (int c = tid; c < DV; c += NT) {
        float x = 0.f, y = 0.f;
#pragma unroll 8
        for (int g = 0; g < RPP; ++g) {
            x += red_x[g][c];
            y += red_y[g][c];
        }
        const float u = sc[0] * (vs[c] - gt * x);
        us[c] = u;
        o[(size_t)bh * DV + c] = from_f32<TO>(fmaf(sc[1], u, gt * y));
    }
    __syncthreads();
    const float4 u4 = *reinterpret_cast<const float4 *>(&us[4 * cg]);
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
        const int r = rg + p * RPP;
        const float kr = ks[r];
        float4 s4 = st[p];
        s4.x = fmaf(kr, u4.x, gt * s4.x); s4.y = fmaf(kr, u4.y, gt * s4.y);
        s4.z = fmaf(kr, u4.z, gt * s4.z); s4.w = fmaf(kr, u4.w, gt * s4.w);
        Sh[r * TPR + cg] = s4;
    }
}

// Any dk, dv <= 256: one thread per state column, two passes over the state.
template <typename T, typename TO>
__global__ void __launch_bounds__(256)
    decode_generic_kernel(const T *__restrict__ q, const T *__restrict__ k,
                          const T *__restrict__ v, const T *__restrict__ beta,
                          const T *__restrict__ gate, float *__restrict__ S, TO *__restrict__ o,
                          int dk, int dv, bool euler) {
    __shared__ float ks[256], qs[256];
    __shared__ float sc[2];
    const int bh = blockIdx.x, tid = threadIdx.x;
    const float gt = gate ? to_f32(gate[bh]) : 1.f;
    for (int i = tid; i < dk; i += blockDim.x) {
        ks[i] = to_f32(k[(size_t)bh * dk + i]);
        qs[i] = to_f32(q[(size_t)bh * dk + i]);
    }
    __syncthreads();
    if (tid < 32) {
        float l = 0.f, kq = 0.f;
        for (int i = tid; i < dk; i += 32) {
            l = fmaf(ks[i], ks[i], l);
            kq = fmaf(ks[i], qs[i], kq);
        }
        l = warp_sum(l);
        kq = warp_sum(kq);
        if (tid == 0) {
            sc[0] = alpha_rule(l, to_f32(beta[bh]), euler);
            sc[1] = kq;
        }
    }
    __syncthreads();
    float *Sh = S + (size_t)bh * dk * dv;
    for (int c = tid; c < dv; c += blockDim.x) {
        float x = 0.f, y = 0.f;
        for (int r = 0; r < dk; ++r) {
            const float s = Sh[(size_t)r * dv + c];
            x = fmaf(s, ks[r], x);
            y = fmaf(s, qs[r], y);
        }
        const float u = sc[0] * (to_f32(v[(size_t)bh * dv + c]) - gt * x);
        o[(size_t)bh * dv + c] = from_f32<TO>(fmaf(sc[1], u, gt * y));
        for (int r = 0; r < dk; ++r) Sh[(size_t)r * dv + c] = fmaf(ks[r], u, gt * Sh[(size_t)r * dv + c]);
    }
}

template <typename T, typename TO, int DK, int DV>
static void launch_reg(const void *q, const void *k, const void *v, const void *beta, const void *g,
                       float *S, void *o, int BH, bool euler, cudaStream_t s) {
    decode_reg_kernel<T, TO, DK, DV><<<BH, DecodeCfg<T, DK, DV>::NT, 0, s>>>(
        (const T *)q, (const T *)k, (const T *)v, (const T *)beta, (const T *)g, S, (TO *)o, euler);
}

template <typename T, typename TO, int DK>
static bool dispatch_dv(const void *q, const void *k, const void *v, const void *beta, const void *g,
                        float *S, void *o, int BH, int dv, bool euler, cudaStream_t s) {
    switch (dv) {
        case 16: launch_reg<T, TO, DK, 16>(q, k, v, beta, g, S, o, BH, euler, s); return true;
        case 32: launch_reg<T, TO, DK, 32>(q, k, v, beta, g, S, o, BH, euler, s); return true;
        case 64: launch_reg<T, TO, DK, 64>(q, k, v, beta, g, S, o, BH, euler, s); return true;
        case 128: launch_reg<T, TO, DK, 128>(q, k, v, beta, g, S, o, BH, euler, s); return true;
        default: return false;
    }
}

template <typename T, typename TO>
static void dispatch(const void *q, const void *k, const void *v, const void *beta, const void *g,
                     float *S, void *o, int BH, int dk, int dv, bool euler, cudaStream_t s) {
    bool done = false;
    switch (dk) {
        case 16: done = dispatch_dv<T, TO, 16>(q, k, v, beta, g, S, o, BH, dv, euler, s); break;
        case 32: done = dispatch_dv<T, TO, 32>(q, k, v, beta, g, S, o, BH, dv, euler, s); break;
        case 64: done = dispatch_dv<T, TO, 64>(q, k, v, beta, g, S, o, BH, dv, euler, s); break;
        case 128: done = dispatch_dv<T, TO, 128>(q, k, v, beta, g, S, o, BH, dv, euler, s); break;
        default: break;
    }
    if (!done)
        decode_generic_kernel<T, TO><<<BH, 256, 0, s>>>((const T *)q, (const T *)k, (const T *)v,
                                                        (const T *)beta, (const T *)g, S, (TO *)o, dk,
                                                        dv, euler);
}

cudaError_t launch_decode(const void *q, const void *k, const void *v, const void *beta,
                          const void *g, float *S, void *o, int BH, int dk, int dv, bool is_bf16,
                          bool o_bf16, bool euler, cudaStream_t s) {
    using bf = __nv_bfloat16;
    if (BH <= 0) return cudaSuccess;
    if (is_bf16) {
        if (o_bf16) dispatch<bf, bf>(q, k, v, beta, g, S, o, BH, dk, dv, euler, s);
        else dispatch<bf, float>(q, k, v, beta, g, S, o, BH, dk, dv, euler, s);
    } else {
        if (o_bf16) dispatch<float, bf>(q, k, v, beta, g, S, o, BH, dk, dv, euler, s);
        else dispatch<float, float>(q, k, v, beta, g, S, o, BH, dk, dv, euler, s);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace efla
