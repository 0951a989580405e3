// chunk_tc.cu -- tensor-core (tcgen05 + TMEM + TMA) EFLA chunkwise forward, sm_100a.
//
// "Exact Flow Linear Attention: Exact Solution from Continuous-Time Dynamics",
// technical summary, Methodology 3: the update S_t = (I - a_t k_t k_t^T) S_{t-1}
// + a_t k_t v_t^T keeps the delta rule's rank-1 algebra and with it the WY/UT
// chunkwise form.  Per chunk of C = 64 tokens entering with state S:
//
//   A  = strictly-lower(diag(a) K K^T)        T = (I + A)^{-1}
//   Ta = T diag(a)                            (so W = Ta K, U = Ta V)
//   U' = U - W S
//   O  = Q S + lower-incl-diagonal(Q K^T) U'   (o_t = S_t^T q_t)
//   S <- S + K^T U'
//
// Two kernels:
//  prep  -- one chunk at a time, all chunks in parallel: the fused squared norm
//           and a, the Gram matrix K K^T on the tensor cores (TMEM accumulator),
//           the unit-lower-triangular inverse T by blocked forward substitution
//           on CUDA cores in fp32, and Ta = T diag(a) written as bf16 to the
//           workspace (64x64 per chunk).
//  state -- one CTA per (head, 64-column slice of the state), chunks in order.
//           W = Ta K, U = Ta V, P = Q K^T, X = W S, dS = K^T U' and
//           O = Q S + mask(P) U' are tcgen05 MMAs with fp32 accumulators in
//           TMEM; the carried state S is fp32 in registers (one row per
//           thread) with a bf16 copy in shared memory as the MMA operand.
//           Q, K, V and Ta arrive by TMA (128-byte swizzle), double buffered.
//
// Every mbarrier wait is bounded; a wait that gives up sets the device error
// word, drains the copies this CTA has in flight (again bounded), releases
// its tensor memory and exits.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "launchers.h"
#include "tc_ptx.cuh"

namespace efla {

static __device__ unsigned int g_tc_error = 0;

namespace {

constexpr int C = 64;         // chunk (tokens)
constexpr int THREADS = 128;  // 4 warps = the 4 TMEM lane quarters
constexpr long long WAIT_BUDGET = 2000000000LL;  // ~1 s of SM cycles

__device__ __forceinline__ void record_error(unsigned code) { atomicOr(&g_tc_error, code); }

// ------------------------------------------------------------------ prep
struct PrepSmem {
    static constexpr int A_STRIDE = C + 1;
    template <int DK>
    static constexpr int k_bytes() { return DK * C * 2; }
};

// T = (I + A)^{-1} for the 64x64 strictly lower A (row stride 65), result in Ts.
// Diagonal 16x16 blocks by forward substitution (one column per thread, in
// registers), then the off-diagonal blocks level by level:
//   T_IJ = -T_II * sum_{K=J}^{I-1} A_IK T_KJ.
__device__ __forceinline__ void unit_lower_inverse(const float *As, float *Ts, float *Rs, int tid) {
    constexpr int S = PrepSmem::A_STRIDE;
    for (int idx = tid; idx < C * C; idx += THREADS) Ts[(idx >> 6) * S + (idx & 63)] = 0.f;
    __syncthreads();
    if (tid < 64) {
        const int b = tid >> 4, c = tid & 15;
        const float *Ab = As + (16 * b) * S + 16 * b;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float s = (i == c) ? 1.f : 0.f;
#pragma unroll
            for (int m = 0; m < i; ++m) s = fmaf(-Ab[i * S + m], x[m], s);
            x[i] = s;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Ts[(16 * b + i) * S + 16 * b + c] = x[i];
    }
    __syncthreads();
    for (int lvl = 1; lvl < 4; ++lvl) {
        const int nblk = 4 - lvl;
        for (int e = tid; e < nblk * 256; e += THREADS) {
            const int J = e >> 8, I = J + lvl, r = (e >> 4) & 15, cc = e & 15;
            float s = 0.f;
            for (int K = J; K < I; ++K) {
                const float *Ar = As + (16 * I + r) * S + 16 * K;
                const float *Tc = Ts + (16 * K) * S + 16 * J + cc;
#pragma unroll
                for (int m = 0; m < 16; ++m) s = fmaf(Ar[m], Tc[m * S], s);
            }
            Rs[J * 256 + r * 16 + cc] = s;
        }
        __syncthreads();
        for (int e = tid; e < nblk * 256; e += THREADS) {
            const int J = e >> 8, I = J + lvl, r = (e >> 4) & 15, cc = e & 15;
            const float *Tr = Ts + (16 * I + r) * S + 16 * I;
            float s = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) s = fmaf(Tr[m], Rs[J * 256 + m * 16 + cc], s);
            Ts[(16 * I + r) * S + 16 * J + cc] = -s;
        }
        __syncthreads();
    }
}

template <int DK>
__global__ void __launch_bounds__(THREADS)
    tc_prep_kernel(const __grid_constant__ CUtensorMap tmap_k, const __nv_bfloat16 *__restrict__ beta,
                   __half *__restrict__ ta_out, int L, int NC, int total) {
    constexpr int KB = PrepSmem::k_bytes<DK>();
    constexpr int S = PrepSmem::A_STRIDE;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    uint8_t *base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    uint8_t *Kt[2] = {base, base + KB};
    float *As = reinterpret_cast<float *>(base + 2 * KB);
    float *Ts = As + C * S;
    float *Rs = Ts + C * S;
    float *al = Rs + 3 * 256;
    __shared__ uint64_t full[2], mma_bar;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        tc::mbar_init(&full[0], 1);
        tc::mbar_init(&full[1], 1);
        tc::mbar_init(&mma_bar, 1);
        tc::fence_mbar_init();
        abort_flag = 0;
        tc::tma_prefetch_desc(&tmap_k);
    }
    if (warp == 0) {
        tc::tmem_alloc(&tmem_base, 64);
        tc::tmem_relinquish();
    }
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_base;
    bool issued[2] = {false, false};

    auto issue = [&](int stage, int g) {
        const int bh = g / NC, n = g - bh * NC;
        tc::mbar_expect_tx(&full[stage], KB);
#pragma unroll
        for (int s = 0; s < DK / 64; ++s)
            tc::tma_load_3d(Kt[stage] + s * 8192, &tmap_k, &full[stage], s * 64, n * C, bh);
    };
    if (tid == 0) {
        for (int st = 0; st < 2; ++st) {
            const int g = blockIdx.x + st * gridDim.x;
            if (g < total) {
                issue(st, g);
                issued[st] = true;
            }
        }
    }
    uint32_t mma_phase = 0;
    int it = 0;
    bool aborted = false;
    bool mma_pending = false;
    for (int g = blockIdx.x; g < total; g += gridDim.x, ++it) {
        const int st = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        const int bh = g / NC, n = g - bh * NC, c0 = n * C;
        bool ok = tc::mbar_wait(&full[st], ph, WAIT_BUDGET);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        if (tid == 0) {
            issued[st] = false;
            tc::tc_fence_after();
            const uint32_t kb = tc::smem_u32(Kt[st]);
            constexpr uint32_t id = tc::idesc_bf16(64, 64, false, false);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint64_t d = tc::sdesc(kb + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                tc::mma_bf16(tmem, d, d, id, kk > 0 ? 1u : 0u);
            }
            tc::mma_commit(&mma_bar);
        }
        mma_pending = true;
        // a per row: squared norm from the swizzled K tile, beta with a bounds check
        if (tid < C) {
            const int r = tid;
            float s = 0.f;
#pragma unroll
            for (int sl = 0; sl < DK / 64; ++sl) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(Kt[st] + sl * 8192 + tc::sw128_off(r, ch));
                    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h[e]);
                        s = fmaf(f.x, f.x, fmaf(f.y, f.y, s));
                    }
                }
            }
            const float b = (c0 + r < L) ? __bfloat162float(beta[(size_t)bh * L + c0 + r]) : 0.f;
            al[r] = alpha_from(s, b);
        }
        ok = tc::mbar_wait(&mma_bar, mma_phase, WAIT_BUDGET);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        mma_phase ^= 1;
        mma_pending = false;
        tc::tc_fence_after();
        {
            const int r = 16 * warp + lane;  // valid for lane < 16 (M = 64 layout)
            const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float v[16];
                tc::tmem_ld16(ta + cb * 16, v);
                if (lane < 16) {
                    const float ar = al[r];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int col = cb * 16 + j;
                        As[r * S + col] = (col < r) ? ar * v[j] : 0.f;
                    }
                }
            }
        }
        tc::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            const int g2 = g + 2 * gridDim.x;
            if (g2 < total) {
                issue(st, g2);
                issued[st] = true;
            }
        }
        unit_lower_inverse(As, Ts, Rs, tid);
        {
            const int i = tid >> 1, h = tid & 1;
            uint4 *dst = reinterpret_cast<uint4 *>(ta_out + ((size_t)g * C + i) * C + h * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint4 u;
                const int j0 = h * 32 + q4 * 8;
                u.x = tc::pack_f16(Ts[i * S + j0 + 0] * al[j0 + 0], Ts[i * S + j0 + 1] * al[j0 + 1]);
                u.y = tc::pack_f16(Ts[i * S + j0 + 2] * al[j0 + 2], Ts[i * S + j0 + 3] * al[j0 + 3]);
                u.z = tc::pack_f16(Ts[i * S + j0 + 4] * al[j0 + 4], Ts[i * S + j0 + 5] * al[j0 + 5]);
                u.w = tc::pack_f16(Ts[i * S + j0 + 6] * al[j0 + 6], Ts[i * S + j0 + 7] * al[j0 + 7]);
                dst[q4] = u;
            }
        }
        __syncthreads();
    }
    if (aborted) {
        if (tid == 0) {
            record_error(1u);
            for (int st = 0; st < 2; ++st)  // drain copies still in flight (bounded)
                if (issued[st]) tc::mbar_wait(&full[st], ((it + (st != (it & 1))) >> 1) & 1, WAIT_BUDGET / 4);
            if (mma_pending) tc::mbar_wait(&mma_bar, mma_phase, WAIT_BUDGET / 4);
        }
        __syncthreads();
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

// ------------------------------------------------------------------ state
// Transposed products so that the state and value dimensions are the MMA M
// dimension (M = 128 runs the tensor core at its full rate):
//   W^T  = K^T Ta^T              [DK x C]
//   U^T  = V^T Ta^T              [DV x C]
//   P    = Q K^T                 [C x C]   (masked to the lower triangle incl. diagonal)
//   X^T  = S^T W^T               [DV x C]
//   U'^T = U^T - X^T
//   S^T += U'^T K                [DV x DK] (fp32 accumulator resident in TMEM)
//   O^T  = S^T Q^T + U'^T P^T    [DV x C]
// MMA operands are fp16 (the bf16 Q, K, V tiles are converted in place; fp16
// holds every bf16 value of magnitude >= 2^-14 exactly and rounds the
// intermediates 8x finer than bf16); accumulation is fp32.
template <int DK, int DV>
struct StateLayout {
    static constexpr int QB = DK * C * 2;            // Q or K tile, DK/64 slabs of 8 KB
    static constexpr int VB = DV * C * 2;            // V tile, DV/64 slabs
    static constexpr int TB = C * C * 2;             // Ta tile
    static constexpr int STAGE = 2 * QB + VB + TB;
    static constexpr int OFF_WT = 2 * STAGE;         // W^T, MN-major B operand [DK x C]
    static constexpr int OFF_P = OFF_WT + DK * 128;  // P, K-major B operand [C x C]
    static constexpr int OFF_UP = OFF_P + TB;        // U'^T, K-major A operand [DV x C]
    static constexpr int OFF_S = OFF_UP + DV * 128;  // S^T, K-major A operand [DV x DK], 2 slots
    static constexpr int S_SLAB = DV * 128;          // bytes per 64-column slab of S^T
    static constexpr int BYTES = OFF_S + 2 * DV * DK * 2;
    static constexpr int SMEM = BYTES + 1024;        // alignment slack
};

// TMEM columns (fp32): S^T [0, DK), W^T, U^T, X^T, P, O^T 64 each.
constexpr uint32_t TM_S = 0, TM_W = 128, TM_U = 192, TM_X = 256, TM_P = 320, TM_O = 384;

// Row of an M-row accumulator held by this thread, or -1: M = 128 puts row r in
// lane r; M = 64 puts row r in lane (r % 16) + 32 (r / 16).
template <int M>
__device__ __forceinline__ int acc_row(int warp, int lane) {
    if constexpr (M == 128) return 32 * warp + lane;
    else return lane < 16 ? 16 * warp + lane : -1;
}

__device__ __forceinline__ void store_row_f16(uint8_t *tile, int row, int ch0, const float (&v)[16]) {
    uint4 u0, u1;
    u0.x = tc::pack_f16(v[0], v[1]);   u0.y = tc::pack_f16(v[2], v[3]);
    u0.z = tc::pack_f16(v[4], v[5]);   u0.w = tc::pack_f16(v[6], v[7]);
    u1.x = tc::pack_f16(v[8], v[9]);   u1.y = tc::pack_f16(v[10], v[11]);
    u1.z = tc::pack_f16(v[12], v[13]); u1.w = tc::pack_f16(v[14], v[15]);
    *reinterpret_cast<uint4 *>(tile + tc::sw128_off(row, ch0)) = u0;
    *reinterpret_cast<uint4 *>(tile + tc::sw128_off(row, ch0 + 1)) = u1;
}

// Warp roles of the state kernel.  Three warpgroups (one warp per TMEM lane
// quarter each) plus two single-thread roles:
//   warps 0-3   converter: bf16 -> fp16 in place for the Q, K, V tiles of a stage
//   warps 4-7   side:      W^T and P from TMEM to fp16 operand tiles; O^T to global
//   warps 8-11  chain:     U'^T = U^T - X^T and the fp16 copy of the new state
//   warp 12     MMA issuer (one thread)
//   warp 13     TMA producer (one thread)
// Hand-offs are mbarriers (arrive count 1; a warpgroup arrives through one thread
// after a named barrier).  Every wait is bounded and also ends when any role has
// flagged an abort.
constexpr int ST_WARPS = 14;
constexpr int ST_THREADS = ST_WARPS * 32;
constexpr int W_ISSUE = 12, W_PROD = 13;

struct StateBars {
    uint64_t full[2], conv[2], freeb[2];
    uint64_t wdone, pdone, xdone, sdone, odone, drain;
    uint64_t wt_ready, p_ready, o_free, up_ready, s_ready;
};

template <int DK, int DV, typename TO>
__global__ void __launch_bounds__(ST_THREADS, 1)
    tc_state_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_t, const float *__restrict__ S0,
                    TO *__restrict__ o, float *__restrict__ S_final, int L, int NC) {
    using Lay = StateLayout<DK, DV>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    uint8_t *base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    __shared__ StateBars bars;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2, gtid = tid & 127;  // warpgroup and thread within it
    const int bh = blockIdx.x;
    if (tid == 0) {
        uint64_t *b = reinterpret_cast<uint64_t *>(&bars);
        for (int i = 0; i < (int)(sizeof(StateBars) / sizeof(uint64_t)); ++i) tc::mbar_init(b + i, 1);
        tc::fence_mbar_init();
        abort_flag = 0;
        tc::tma_prefetch_desc(&tmap_q);
        tc::tma_prefetch_desc(&tmap_k);
        tc::tma_prefetch_desc(&tmap_v);
        tc::tma_prefetch_desc(&tmap_t);
    }
    if (warp == 0) {
        tc::tmem_alloc(&tmem_base, 512);
        tc::tmem_relinquish();
    }
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t sb = tc::smem_u32(base);
    const uint32_t wt_s = sb + Lay::OFF_WT, p_s = sb + Lay::OFF_P, up_s = sb + Lay::OFF_UP;
    auto s16 = [&](int slot) { return sb + Lay::OFF_S + slot * (DV * DK * 2); };
    uint8_t *s16p[2] = {base + Lay::OFF_S, base + Lay::OFF_S + DV * DK * 2};
    const int vrow = acc_row<DV>(warp & 3, lane);  // state column v of this thread's TMEM lane

    // ---- initial state (chain warpgroup): S^T into TMEM and its fp16 copy (slot 0)
    if (wg == 2) {
#pragma unroll
        for (int cb = 0; cb < DK / 16; ++cb) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
                v[j] = (S0 && vrow >= 0) ? S0[((size_t)bh * DK + cb * 16 + j) * DV + vrow] : 0.f;
            if (S0) tc::tmem_st16(tmem + lane_base + TM_S + cb * 16, v);
            if (vrow >= 0) store_row_f16(s16p[0] + (cb >> 2) * Lay::S_SLAB, vrow, (cb & 3) * 2, v);
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
    }
    __syncthreads();
    tc::tc_fence_after();

    const long long budget = WAIT_BUDGET;
    if (warp == W_PROD) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            int last[2] = {-1, -1};
            for (int n = 0; n < NC; ++n) {
                const int st = n & 1;
                if (n >= 2 && !tc::mbar_wait_or_abort(&bars.freeb[st], ((n - 2) >> 1) & 1, &abort_flag, budget))
                    break;
                uint64_t *bar = &bars.full[st];
                tc::mbar_expect_tx(bar, Lay::STAGE);
                uint8_t *q = base + st * Lay::STAGE;
#pragma unroll
                for (int s = 0; s < DK / 64; ++s) {
                    tc::tma_load_3d(q + s * 8192, &tmap_q, bar, s * 64, n * C, bh);
                    tc::tma_load_3d(q + Lay::QB + s * 8192, &tmap_k, bar, s * 64, n * C, bh);
                }
#pragma unroll
                for (int s = 0; s < DV / 64; ++s)
                    tc::tma_load_3d(q + 2 * Lay::QB + s * 8192, &tmap_v, bar, s * 64, n * C, bh);
                tc::tma_load_2d(q + 2 * Lay::QB + Lay::VB, &tmap_t, bar, 0, (bh * NC + n) * C);
                last[st] = n;
            }
            if (abort_flag) {  // let this CTA's own copies land before it exits (bounded)
                for (int st = 0; st < 2; ++st)
                    if (last[st] >= 0) tc::mbar_wait(&bars.full[st], (last[st] >> 1) & 1, budget / 4);
            }
        }
    } else if (warp == W_ISSUE) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_w = tc::idesc_f16(DK, 64, true, false);
            constexpr uint32_t id_u = tc::idesc_f16(DV, 64, true, false);
            constexpr uint32_t id_p = tc::idesc_f16(64, 64, false, false);
            constexpr uint32_t id_x = tc::idesc_f16(DV, 64, false, true);
            constexpr uint32_t id_s = tc::idesc_f16(DV, DK, false, true);
            constexpr uint32_t id_o = tc::idesc_f16(DV, 64, false, false);
            bool issued_any = false;
            for (int n = 0; n < NC; ++n) {
                const int st = n & 1;
                const uint32_t sq = sb + st * Lay::STAGE, sk = sq + Lay::QB, sv = sq + 2 * Lay::QB,
                               stt = sv + Lay::VB;
                const uint32_t cur = s16(n & 1);
                if (!tc::mbar_wait_or_abort(&bars.conv[st], (n >> 1) & 1, &abort_flag, budget)) break;
                tc::tc_fence_after();
                issued_any = true;
                // W^T = K^T Ta^T ; U^T = V^T Ta^T ; P = Q K^T
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_W, tc::sdesc(sk + kk * 2048, 8192, 1024),
                                 tc::sdesc(stt + kk * 32, 16, 1024), id_w, kk > 0);
                tc::mma_commit(&bars.wdone);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_U, tc::sdesc(sv + kk * 2048, 8192, 1024),
                                 tc::sdesc(stt + kk * 32, 16, 1024), id_u, kk > 0);
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 8192 + (kk & 3) * 32;
                    tc::mma_bf16(tmem + TM_P, tc::sdesc(sq + off, 16, 1024),
                                 tc::sdesc(sk + off, 16, 1024), id_p, kk > 0);
                }
                tc::mma_commit(&bars.pdone);
                // X^T = S^T W^T  (needs W^T(n) in smem and S_n in smem)
                if (!tc::mbar_wait_or_abort(&bars.wt_ready, n & 1, &abort_flag, budget)) break;
                if (n > 0 && !tc::mbar_wait_or_abort(&bars.s_ready, (n - 1) & 1, &abort_flag, budget)) break;
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    tc::mma_bf16(tmem + TM_X,
                                 tc::sdesc(cur + (kk >> 2) * Lay::S_SLAB + (kk & 3) * 32, 16, 1024),
                                 tc::sdesc(wt_s + kk * 2048, 8192, 1024), id_x, kk > 0);
                tc::mma_commit(&bars.xdone);
                // O^T = S^T Q^T (first part; TMEM O must have been read out)
                if (n > 0 && !tc::mbar_wait_or_abort(&bars.o_free, (n - 1) & 1, &abort_flag, budget)) break;
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    tc::mma_bf16(tmem + TM_O,
                                 tc::sdesc(cur + (kk >> 2) * Lay::S_SLAB + (kk & 3) * 32, 16, 1024),
                                 tc::sdesc(sq + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_o,
                                 kk > 0);
                // S^T += U'^T K
                if (!tc::mbar_wait_or_abort(&bars.up_ready, n & 1, &abort_flag, budget)) break;
                tc::tc_fence_after();
                const uint32_t acc0 = (n > 0 || S0) ? 1u : 0u;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_S, tc::sdesc(up_s + kk * 32, 16, 1024),
                                 tc::sdesc(sk + kk * 2048, 8192, 1024), id_s, kk > 0 ? 1u : acc0);
                tc::mma_commit(&bars.sdone);
                // O^T += U'^T P^T
                if (!tc::mbar_wait_or_abort(&bars.p_ready, n & 1, &abort_flag, budget)) break;
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_O, tc::sdesc(up_s + kk * 32, 16, 1024),
                                 tc::sdesc(p_s + kk * 32, 16, 1024), id_o, 1u);
                tc::mma_commit(&bars.odone);
                tc::mma_commit(&bars.freeb[st]);
            }
            if (abort_flag && issued_any) {  // wait (bounded) for every issued MMA to finish
                tc::mma_commit(&bars.drain);
                tc::mbar_wait(&bars.drain, 0, budget / 4);
            }
        }
    } else if (wg == 0) {
        // ---------------------------------------------------------- converter
        for (int n = 0; n < NC; ++n) {
            const int st = n & 1;
            const bool ok = tc::mbar_wait_or_abort(&bars.full[st], (n >> 1) & 1, &abort_flag, budget);
            if (tc::named_bar_or(1, 128, !ok)) break;
            uint4 *t = reinterpret_cast<uint4 *>(base + st * Lay::STAGE);
            constexpr int N16 = (2 * Lay::QB + Lay::VB) / 16;
#pragma unroll 4
            for (int i = gtid; i < N16; i += 128) {
                uint4 u = t[i];
                u.x = tc::bf16x2_to_f16x2(u.x); u.y = tc::bf16x2_to_f16x2(u.y);
                u.z = tc::bf16x2_to_f16x2(u.z); u.w = tc::bf16x2_to_f16x2(u.w);
                t[i] = u;
            }
            tc::fence_async_smem();
            tc::named_bar_sync(1, 128);
            if (gtid == 0) tc::mbar_arrive(&bars.conv[st]);
        }
    } else if (wg == 1) {
        // ---------------------------------------------------------- side epilogue
        const int drow = acc_row<DK>(warp & 3, lane);
        const int prow = acc_row<64>(warp & 3, lane);
        for (int n = 0; n < NC; ++n) {
            const int c0 = n * C;
            bool ok = tc::mbar_wait_or_abort(&bars.wdone, n & 1, &abort_flag, budget);
            if (tc::named_bar_or(2, 128, !ok)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float v[16];
                tc::tmem_ld16(tmem + lane_base + TM_W + cb * 16, v);
                if (drow >= 0) store_row_f16(base + Lay::OFF_WT, drow, 2 * cb, v);
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::named_bar_sync(2, 128);
            if (gtid == 0) tc::mbar_arrive(&bars.wt_ready);

            ok = tc::mbar_wait_or_abort(&bars.pdone, n & 1, &abort_flag, budget);
            if (tc::named_bar_or(2, 128, !ok)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float v[16];
                tc::tmem_ld16(tmem + lane_base + TM_P + cb * 16, v);
                if (prow >= 0) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (cb * 16 + j > prow) v[j] = 0.f;
                    store_row_f16(base + Lay::OFF_P, prow, 2 * cb, v);
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::named_bar_sync(2, 128);
            if (gtid == 0) tc::mbar_arrive(&bars.p_ready);

            ok = tc::mbar_wait_or_abort(&bars.odone, n & 1, &abort_flag, budget);
            if (tc::named_bar_or(2, 128, !ok)) break;
            tc::tc_fence_after();
            const int cl = min(C, L - c0);
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float v[16];
                tc::tmem_ld16(tmem + lane_base + TM_O + cb * 16, v);
                if (vrow >= 0) {
                    TO *dst = o + ((size_t)bh * L + c0 + cb * 16) * DV + vrow;
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (cb * 16 + j < cl) dst[(size_t)j * DV] = from_f32<TO>(v[j]);
                }
            }
            tc::tc_fence_before();
            tc::named_bar_sync(2, 128);
            if (gtid == 0) tc::mbar_arrive(&bars.o_free);
        }
    } else if (wg == 2) {
        // ---------------------------------------------------------- chain epilogue
        bool done_all = true;
        for (int n = 0; n < NC; ++n) {
            bool ok = tc::mbar_wait_or_abort(&bars.xdone, n & 1, &abort_flag, budget);
            if (tc::named_bar_or(3, 128, !ok)) { done_all = false; break; }
            tc::tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float u[16], x[16];
                tc::tmem_ld16(tmem + lane_base + TM_U + cb * 16, u);
                tc::tmem_ld16(tmem + lane_base + TM_X + cb * 16, x);
                if (vrow >= 0) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) u[j] -= x[j];
                    store_row_f16(base + Lay::OFF_UP, vrow, 2 * cb, u);
                }
            }
            tc::fence_async_smem();
            tc::tc_fence_before();
            tc::named_bar_sync(3, 128);
            if (gtid == 0) tc::mbar_arrive(&bars.up_ready);

            ok = tc::mbar_wait_or_abort(&bars.sdone, n & 1, &abort_flag, budget);
            if (tc::named_bar_or(3, 128, !ok)) { done_all = false; break; }
            tc::tc_fence_after();
            if (n + 1 < NC) {
                uint8_t *stile = s16p[(n + 1) & 1];
#pragma unroll
                for (int cb = 0; cb < DK / 16; ++cb) {
                    float v[16];
                    tc::tmem_ld16(tmem + lane_base + TM_S + cb * 16, v);
                    if (vrow >= 0) store_row_f16(stile + (cb >> 2) * Lay::S_SLAB, vrow, (cb & 3) * 2, v);
                }
                tc::fence_async_smem();
            }
            tc::tc_fence_before();
            tc::named_bar_sync(3, 128);
            if (gtid == 0) tc::mbar_arrive(&bars.s_ready);
        }
        if (done_all && S_final) {
#pragma unroll
            for (int cb = 0; cb < DK / 16; ++cb) {
                float v[16];
                tc::tmem_ld16(tmem + lane_base + TM_S + cb * 16, v);
                if (vrow >= 0) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        S_final[((size_t)bh * DK + cb * 16 + j) * DV + vrow] = v[j];
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (tid == 0 && abort_flag) record_error(2u);
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// bf16 tensor [d2][d1][d0] (d0 innermost) with a (b0, b1, 1) box, 128-byte swizzle;
// out-of-range elements read as zero.
bool make_map_3d(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint32_t b0, uint32_t b1) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    const cuuint32_t box[3] = {b0, b1, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_2d(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint32_t b0,
                 uint32_t b1, CUtensorMapDataType dt) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {d0, d1};
    const cuuint64_t strides[1] = {d0 * 2};
    const cuuint32_t box[2] = {b0, b1};
    const cuuint32_t es[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DK>
int prep_smem_bytes() {
    return 2 * PrepSmem::k_bytes<DK>() + (2 * C * PrepSmem::A_STRIDE + 3 * 256 + C) * 4 + 1024;
}

template <int DK, int DV, typename TO>
cudaError_t launch_tc_t(const void *q, const void *k, const void *v, const void *beta,
                        const float *S0, void *o, float *S_final, int B, int H, int L, void *ws,
                        cudaStream_t s) {
    const int BH = B * H, NC = (L + C - 1) / C, total = BH * NC;
    CUtensorMap mq, mk, mv, mt;
    if (!make_map_3d(&mq, q, DK, L, BH, 64, C) || !make_map_3d(&mk, k, DK, L, BH, 64, C) ||
        !make_map_3d(&mv, v, DV, L, BH, 64, C) ||
        !make_map_2d(&mt, ws, C, (uint64_t)total * C, 64, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return cudaErrorInvalidValue;
    const int psm = prep_smem_bytes<DK>();
    cudaError_t e = cudaFuncSetAttribute(tc_prep_kernel<DK>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, psm);
    if (e != cudaSuccess) return e;
    const int pgrid = total < 148 * 3 ? total : 148 * 3;
    tc_prep_kernel<DK><<<pgrid, THREADS, psm, s>>>(mk, (const __nv_bfloat16 *)beta, (__half *)ws,
                                                    L, NC, total);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int ssm = StateLayout<DK, DV>::SMEM;
    e = cudaFuncSetAttribute(tc_state_kernel<DK, DV, TO>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, ssm);
    if (e != cudaSuccess) return e;
    tc_state_kernel<DK, DV, TO><<<BH, ST_THREADS, ssm, s>>>(mq, mk, mv, mt, S0, (TO *)o, S_final, L, NC);
    count_launches(2);
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_tc_o(const void *q, const void *k, const void *v, const void *beta,
                        const float *S0, void *o, float *S_final, int B, int H, int L, bool o_bf16,
                        void *ws, cudaStream_t s) {
    return o_bf16 ? launch_tc_t<DK, DV, __nv_bfloat16>(q, k, v, beta, S0, o, S_final, B, H, L, ws, s)
                  : launch_tc_t<DK, DV, float>(q, k, v, beta, S0, o, S_final, B, H, L, ws, s);
}

}  // namespace

bool tc_supported(int B, int H, int L, int dk, int dv, int chunk, bool is_bf16) {
    if (!is_bf16 || chunk != C || L < 1) return false;
    if (dk != 64 && dk != 128) return false;
    if (dv != 64 && dv != 128) return false;
    const long long total = (long long)B * H * ((L + C - 1) / C);
    if (total * C >= (1LL << 31)) return false;
    return true;  // cuTensorMapEncodeTiled is resolved at launch (an error there is reported)
}

size_t tc_workspace_bytes(int B, int H, int L, int dk, int dv, int chunk) {
    (void)dk; (void)dv; (void)chunk;
    const size_t total = (size_t)B * H * ((L + C - 1) / C);
    return total * C * C * sizeof(__half);
}

cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const void *beta,
                            const float *S0, void *o, float *S_final, int B, int H, int L,
                            int dk, int dv, int chunk, bool o_bf16, void *ws, cudaStream_t s) {
    (void)chunk;
    if (dk == 128 && dv == 128)
        return launch_tc_o<128, 128>(q, k, v, beta, S0, o, S_final, B, H, L, o_bf16, ws, s);
    if (dk == 128 && dv == 64)
        return launch_tc_o<128, 64>(q, k, v, beta, S0, o, S_final, B, H, L, o_bf16, ws, s);
    if (dk == 64 && dv == 128)
        return launch_tc_o<64, 128>(q, k, v, beta, S0, o, S_final, B, H, L, o_bf16, ws, s);
    return launch_tc_o<64, 64>(q, k, v, beta, S0, o, S_final, B, H, L, o_bf16, ws, s);
}

cudaError_t tc_read_and_clear_error(unsigned int *out, cudaStream_t s) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(out, g_tc_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(unsigned int));
}

}  // namespace efla
