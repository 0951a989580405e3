// bwd_tc.cu -- tensor-core backward of the EFLA chunkwise forward, sm_100a (bf16 inputs,
// chunk 64, dk and dv in {64, 128}).
//
// "Exact Flow Linear Attention: Exact Solution from Continuous-Time Dynamics", technical
// summary, Methodology 3: the forward per chunk of C = 64 tokens entering with state S is
//
//   A = strictly-lower(diag(a) K K^T),  T = (I + A)^{-1},  R = V - K S,  U' = T diag(a) R,
//   O = Q S + P U'  (P = lower-incl(Q K^T)),  S' = S + K^T U'.
//
// Reverse mode through those lines, given dO and dS' (the gradient of the state after the
// chunk), splits into a chain over the chunks and work that is independent per chunk:
//
//   chain (bwd_state_kernel, one CTA per head, chunks last to first):
//     dU' = K dS' + P^T dO,           dS = dS' + Q^T dO - W^T dU'   (W = Ta K, Ta = T diag(a))
//   per chunk (bwd_chunk_kernel, every chunk in parallel):
//     dR = Ta^T dU',  B = -strictly-lower(dR U'^T),  G = K K^T,
//     da_t = (dR_t . R_t + sum_s B_ts G_ts) / a_t,   dP = lower-incl(dO U'^T),
//     dQ = dO S^T + dP K,
//     dK = U' dS'^T + dP^T Q - dR S^T + B K + B^T K + 2 da (df/dlambda) K,
//     dV = dR,  dbeta = da (df/dbeta).
//
// (dR = diag(a) T^T dU' and B = diag(a) dA with dA = strictly-lower(-T^T dT T^T), dT =
// dU' (diag(a) R)^T, which is -(T^T dU') U'^T since T diag(a) R = U'.)  The chain carries
// dS^T in TMEM the way the forward carries S^T; both kernels take fp16 operands with fp32
// accumulation, the precision of the forward's products.  The per-head gate of the backward
// (keys of squared norm at most 16, a spanning at most a factor of 1024, every a positive)
// decides which heads take this path; the others walk the forward in fp32 on CUDA cores.
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <type_traits>

#include "bwd_gate.cuh"
#include "common.cuh"
#include "launchers.h"
#include "tc_ptx.cuh"
#include "tmap.h"

namespace efla {

namespace {

constexpr int C = 64;
constexpr long long WAIT_BUDGET = 2000000000LL;  // ~1 s of SM cycles
__device__ unsigned int g_bwd_error = 0;

// ------------------------------------------------------------------ the chain over chunks
// Shared memory per stage (double buffered): Q, K (bf16 by TMA, fp16 after the converter),
// dO (fp16), Ta (fp16), -W and P (fp16, written by the side group); 64-token tiles of 128-byte
// rows, 128-byte swizzle, one 8 KB slab per 64 columns.
template <int DK, int DV>
struct RevLayout {
    static constexpr int QB = (DK / 64) * 8192, KB = QB, OB = (DV / 64) * 8192;
    static constexpr int TB = C * C * 2, WB = QB, PB = C * C * 2;
    static constexpr int OFF_Q = 0, OFF_K = QB, OFF_O = OFF_K + KB, OFF_T = OFF_O + OB;
    static constexpr int OFF_W = OFF_T + TB, OFF_P = OFF_W + WB;
    static constexpr int STAGE = OFF_P + PB;
    // the chain group's outputs on their way to global memory by TMA: dU' [64][DV], dS [DK][DV]
    static constexpr int OFF_SU = 2 * STAGE, OFF_SS = OFF_SU + 128 * DV;
    static constexpr int SMEM = OFF_SS + 2 * DK * DV + 1024;  // + alignment slack
};

// Single-arrival barriers first, then those a warpgroup arrives on once per warp.
struct RevBars {
    uint64_t full[2], freeS[2], wdone, pdone, d1done, d2done, drain, su_free, ss_free;
    uint64_t conv[2], w_ready, p_ready, up_ready, s_ready, su_full, ss_full;
};
constexpr int REV_ONE = 11;
constexpr int REV_WARPS = 14;  // converter, side, chain warpgroups; MMA issuer; TMA producer
constexpr int REV_THREADS = REV_WARPS * 32;
constexpr int RW_ISSUE = 12, RW_PROD = 13;
constexpr uint32_t RT_W = 256, RT_P = 384, RT_S16 = 448;

__device__ __forceinline__ void rev_arrive(uint64_t *bar, int lane) {
    tc::tc_fence_before();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(bar);
}

__device__ __forceinline__ void store_row16x32(uint8_t *tile, int row, int ch0, const float (&v)[32]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 u;
        u.x = tc::pack_f16(v[8 * c + 0], v[8 * c + 1]); u.y = tc::pack_f16(v[8 * c + 2], v[8 * c + 3]);
        u.z = tc::pack_f16(v[8 * c + 4], v[8 * c + 5]); u.w = tc::pack_f16(v[8 * c + 6], v[8 * c + 7]);
        *reinterpret_cast<uint4 *>(tile + tc::sw128_off(row, ch0 + c)) = u;
    }
}

__device__ __forceinline__ bool head_ok(const int *hs, int bh) { return head_takes_saved(hs, bh); }
// every bulk store group of this thread has read its shared-memory source
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }


// One CTA per head, chunks from last to first.  TMEM (fp32 columns): dS^T [0, DK), dU'^T
// [DK, DK + 64) (fp16 dU'^T packed over its first 32 after the epilogue), W [256, 256 + DK),
// P [384, 448), dS^T fp16 [448, 448 + DK/2).  Per chunk, in tensor-pipe order:
//   D1a  dU'^T  = dO^T P            (off the chain)
//   D1b  dU'^T += dS16^T K^T        (A = the fp16 copy of dS^T in TMEM)
//   D2a  dS^T  += dO^T Q            (off the chain)
//   W, P of the next chunk
//   D2b  dS^T  += dU'16^T (-W)      (A = fp16 dU'^T in TMEM)
// Outputs (fp16): dU' of every token [BH][L][dv] and the gradient of the state after every
// chunk, dSp [BH][NC][dk][dv] (dSp[NC-1] is dS_final), each written column by column into a
// shared-memory tile (a warp's lanes write consecutive columns) and stored by TMA; dS0 (fp32).
template <int DK, int DV>
__global__ void __launch_bounds__(REV_THREADS, 1)
    bwd_state_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_o, const __grid_constant__ CUtensorMap tmap_t,
                     const __grid_constant__ CUtensorMap tmap_du, const __grid_constant__ CUtensorMap tmap_ds,
                     const float *__restrict__ dSL, __half *__restrict__ dSp,
                     float *__restrict__ dS0, const int *__restrict__ hs, int L, int NC) {
    using Lay = RevLayout<DK, DV>;
    constexpr uint32_t TM_S = 0, TM_U = DK;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    uint8_t *base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    __shared__ RevBars bars;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;

    const int bh = blockIdx.x;
    if (!head_ok(hs, bh)) return;  // this head walks on CUDA cores (uniform over the CTA)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2, gtid = tid & 127;
    const size_t DD = (size_t)DK * DV;
    if (tid == 0) {
        uint64_t *b = reinterpret_cast<uint64_t *>(&bars);
        for (int i = 0; i < (int)(sizeof(RevBars) / sizeof(uint64_t)); ++i)
            tc::mbar_init(b + i, i < REV_ONE ? 1 : 4);
        tc::fence_mbar_init();
        abort_flag = 0;
        tc::tma_prefetch_desc(&tmap_q);
        tc::tma_prefetch_desc(&tmap_k);
        tc::tma_prefetch_desc(&tmap_o);
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
    // state column v of this thread's TMEM lane (M = DV accumulators), or -1
    const int vrow = DV == 128 ? 32 * (warp & 3) + lane : (lane < 16 ? 16 * (warp & 3) + lane : -1);

    // ---- the initial state gradient dS_final (chain warpgroup): fp32 and fp16 copies in TMEM
    if (wg == 2) {
#pragma unroll
        for (int cb = 0; cb < DK / 32; ++cb) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                v[j] = (dSL && vrow >= 0) ? dSL[(size_t)bh * DD + (size_t)(cb * 32 + j) * DV + vrow] : 0.f;
            float lo[16], hi[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) { lo[j] = v[j]; hi[j] = v[16 + j]; }
            tc::tmem_st16(tmem + lane_base + TM_S + cb * 32, lo);
            tc::tmem_st16(tmem + lane_base + TM_S + cb * 32 + 16, hi);
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) w[j] = tc::pack_f16(v[2 * j], v[2 * j + 1]);
            tc::tmem_st16u(tmem + lane_base + RT_S16 + cb * 16, w);
            if (vrow >= 0) {  // dSp[NC - 1]: the gradient of the last chunk's final state
                __half *dst = dSp + ((size_t)bh * NC + (NC - 1)) * DD + vrow;
#pragma unroll
                for (int j = 0; j < 32; ++j) dst[(size_t)(cb * 32 + j) * DV] = __float2half_rn(v[j]);
            }
        }
        tc::tc_fence_before();
    }
    __syncthreads();
    tc::tc_fence_after();

    const long long budget = WAIT_BUDGET;
    if (warp == RW_PROD) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            int last[2] = {-1, -1};
            for (int i = 0; i < NC; ++i) {
                const int n = NC - 1 - i, st = i & 1;
                uint8_t *stg = base + st * Lay::STAGE;
                if (i >= 2 && !tc::mbar_wait_or_abort(&bars.freeS[st], ((i - 2) >> 1) & 1, &abort_flag, budget))
                    break;
                tc::mbar_expect_tx(&bars.full[st], Lay::QB + Lay::KB + Lay::OB + Lay::TB);
#pragma unroll
                for (int j = 0; j < DK / 64; ++j) {
                    tc::tma_load_3d(stg + Lay::OFF_Q + j * 8192, &tmap_q, &bars.full[st], j * 64, n * C, bh);
                    tc::tma_load_3d(stg + Lay::OFF_K + j * 8192, &tmap_k, &bars.full[st], j * 64, n * C, bh);
                }
#pragma unroll
                for (int j = 0; j < DV / 64; ++j)
                    tc::tma_load_3d(stg + Lay::OFF_O + j * 8192, &tmap_o, &bars.full[st], j * 64, n * C, bh);
                tc::tma_load_2d(stg + Lay::OFF_T, &tmap_t, &bars.full[st], 0, (bh * NC + n) * C);
                last[st] = i;
            }
            if (abort_flag) {  // let this CTA's own copies land before it exits (bounded)
                for (int st = 0; st < 2; ++st)
                    if (last[st] >= 0) tc::mbar_wait(&bars.full[st], (last[st] >> 1) & 1, budget / 8);
            }
        }
    } else if (warp == RW_ISSUE) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_w = tc::idesc_f16(64, DK, false, true);   // W = Ta K
            constexpr uint32_t id_p = tc::idesc_f16(64, 64, false, false);  // P = Q K^T
            constexpr uint32_t id_1a = tc::idesc_f16(DV, 64, true, true);   // dO^T P
            constexpr uint32_t id_1b = tc::idesc_f16(DV, 64, false, false); // dS16^T K^T
            constexpr uint32_t id_2a = tc::idesc_f16(DV, DK, true, true);   // dO^T Q
            constexpr uint32_t id_2b = tc::idesc_f16(DV, DK, false, true);  // dU'16^T (-W)
            auto stage_addr = [&](int i) { return sb + (i & 1) * Lay::STAGE; };
            auto issue_w = [&](int i) {  // W of local chunk i (into its TMEM columns)
                const uint32_t stg = stage_addr(i);
                const uint32_t k = stg + Lay::OFF_K, t = stg + Lay::OFF_T;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + RT_W, tc::sdesc(t + kk * 32, 16, 1024), tc::sdesc(k + kk * 2048, 8192, 1024),
                                 id_w, kk > 0);
                tc::mma_commit(&bars.wdone);
            };
            auto issue_p = [&](int i) {  // P of local chunk i (into its TMEM columns)
                const uint32_t stg = stage_addr(i);
                const uint32_t q = stg + Lay::OFF_Q, k = stg + Lay::OFF_K;
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    tc::mma_bf16(tmem + RT_P, tc::sdesc(q + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                                 tc::sdesc(k + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_p, kk > 0);
                tc::mma_commit(&bars.pdone);
            };
            auto wait = [&](uint64_t *bar, uint32_t par) {
                return tc::mbar_wait_or_abort(bar, par, &abort_flag, budget);
            };
            bool issued_any = false;
            bool ok = wait(&bars.conv[0], 0);
            if (ok) {
                tc::tc_fence_after();
                issued_any = true;
                issue_w(0);
                issue_p(0);
            }
            for (int i = 0; ok && i < NC; ++i) {
                const int st = i & 1;
                const uint32_t stg = stage_addr(i);
                const uint32_t q = stg + Lay::OFF_Q, k = stg + Lay::OFF_K, o = stg + Lay::OFF_O;
                const uint32_t w = stg + Lay::OFF_W, p = stg + Lay::OFF_P;
                // D1a: dU'^T = dO^T P  (P read out of TMEM and stored masked by the side group)
                if (!wait(&bars.p_ready, i & 1)) break;
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_U, tc::sdesc(o + kk * 2048, 8192, 1024), tc::sdesc(p + kk * 2048, 8192, 1024),
                                 id_1a, kk > 0);
                // D1b: dU'^T += dS16^T K^T  (the fp16 copy of the state gradient)
                if (i > 0 && !wait(&bars.s_ready, (i - 1) & 1)) break;
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    tc::mma_tmem_a(tmem + TM_U, tmem + RT_S16 + kk * 8,
                                   tc::sdesc(k + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_1b, 1u);
                tc::mma_commit(&bars.d1done);
                // D2a: dS^T += dO^T Q  (the chain has read dS^T for this chunk: s_ready above)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_S, tc::sdesc(o + kk * 2048, 8192, 1024), tc::sdesc(q + kk * 2048, 8192, 1024),
                                 id_2a, 1u);
                // D2b: dS^T += dU'16^T (-W)  (-W of this chunk is in shared memory: w_ready)
                if (!wait(&bars.w_ready, i & 1)) break;
                if (!wait(&bars.up_ready, i & 1)) break;
                tc::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_tmem_a(tmem + TM_S, tmem + TM_U + kk * 8, tc::sdesc(w + kk * 2048, 8192, 1024), id_2b, 1u);
                tc::mma_commit(&bars.d2done);
                tc::mma_commit(&bars.freeS[st]);
                // W and P of the next chunk after D2b, off the chain's path between D1b and D2b
                // (this chunk's W and P were read out of TMEM before: w_ready, and before D1a)
                if (i + 1 < NC) {
                    if (!wait(&bars.conv[(i + 1) & 1], ((i + 1) >> 1) & 1)) break;
                    tc::tc_fence_after();
                    issue_w(i + 1);
                    issue_p(i + 1);
                }
            }
            if (abort_flag && issued_any) {  // wait (bounded) for every issued MMA to finish
                tc::mma_commit(&bars.drain);
                tc::mbar_wait(&bars.drain, 0, budget / 4);
            }
        }
    } else if (wg == 0) {
        // ---------------------------------------------------------- converter: q, k bf16 -> fp16
        auto cvt = [](uint4 *t) {
            uint4 u = *t;
            u.x = tc::bf16x2_to_f16x2(u.x); u.y = tc::bf16x2_to_f16x2(u.y);
            u.z = tc::bf16x2_to_f16x2(u.z); u.w = tc::bf16x2_to_f16x2(u.w);
            *t = u;
        };
        for (int i = 0; i < NC; ++i) {
            const int st = i & 1;
            uint8_t *stg = base + st * Lay::STAGE;
            if (!tc::mbar_wait_or_abort(&bars.full[st], (i >> 1) & 1, &abort_flag, budget)) break;
            uint4 *tq = reinterpret_cast<uint4 *>(stg + Lay::OFF_Q);  // Q then K: contiguous
#pragma unroll 4
            for (int e = gtid; e < (Lay::QB + Lay::KB) / 16; e += 128) cvt(tq + e);
            tc::fence_async_smem();
            rev_arrive(&bars.conv[st], lane);
        }
    } else if (wg == 1) {
        // ---------------------------------------------------------- side: -W and the masked P
        const int crow = lane < 16 ? 16 * (warp & 3) + lane : -1;  // token row of M = 64 accumulators
        for (int i = 0; i < NC; ++i) {
            const int st = i & 1;
            uint8_t *stg = base + st * Lay::STAGE;
            if (!tc::mbar_wait_or_abort(&bars.wdone, i & 1, &abort_flag, budget)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < DK / 32; ++cb) {  // -W, rows s
                float v[32];
                tc::tmem_ld32(tmem + lane_base + RT_W + cb * 32, v);
                if (crow >= 0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = -v[j];
                    store_row16x32(stg + Lay::OFF_W + (cb >> 1) * 8192, crow, (cb & 1) * 4, v);
                }
            }
            tc::fence_async_smem();
            rev_arrive(&bars.w_ready, lane);
            if (!tc::mbar_wait_or_abort(&bars.pdone, i & 1, &abort_flag, budget)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {  // P, row t, column s <= t
                float v[32];
                tc::tmem_ld32(tmem + lane_base + RT_P + cb * 32, v);
                if (crow >= 0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (cb * 32 + j > crow) v[j] = 0.f;
                    store_row16x32(stg + Lay::OFF_P, crow, cb * 4, v);
                }
            }
            tc::fence_async_smem();
            rev_arrive(&bars.p_ready, lane);
        }
    } else if (wg == 2) {
        // ---------------------------------------------------------- chain epilogue
        bool done_all = true;
        for (int i = 0; i < NC; ++i) {
            const int n = NC - 1 - i;
            if (!tc::mbar_wait_or_abort(&bars.d1done, i & 1, &abort_flag, budget)) { done_all = false; break; }
            tc::tc_fence_after();
            uint32_t wu[2][16];
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // dU'^T to fp16 in place, 32 tokens at a time
                float u[32];
                tc::tmem_ld32(tmem + lane_base + TM_U + h * 32, u);
#pragma unroll
                for (int j = 0; j < 16; ++j) wu[h][j] = tc::pack_f16(u[2 * j], u[2 * j + 1]);
                tc::tmem_st16u(tmem + lane_base + TM_U + h * 16, wu[h]);  // over columns already read
            }
            rev_arrive(&bars.up_ready, lane);
            // dU' of the chunk's tokens to its staging tile ([64][dv], rows past L are not
            // stored), once the tile's previous store has read it
            if (gtid == 0 && i > 0) {
                tc::bulk_wait_read1();
                tc::mbar_arrive(&bars.su_free);
            }
            if (i > 0 && !tc::mbar_wait_or_abort(&bars.su_free, (i - 1) & 1, &abort_flag, budget)) { done_all = false; break; }
            if (vrow >= 0) {
                uint8_t *tile = base + Lay::OFF_SU + (vrow >> 6) * 8192 + 2 * (vrow & 7);
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int t = 32 * h + 2 * j;
                        const __half2 pr = *reinterpret_cast<const __half2 *>(&wu[h][j]);
                        *reinterpret_cast<__half *>(tile + tc::sw128_off(t, (vrow & 63) >> 3)) = __low2half(pr);
                        *reinterpret_cast<__half *>(tile + tc::sw128_off(t + 1, (vrow & 63) >> 3)) = __high2half(pr);
                    }
            }
            tc::fence_async_smem();
            rev_arrive(&bars.su_full, lane);
            if (gtid == 0) {
                if (!tc::mbar_wait_or_abort(&bars.su_full, i & 1, &abort_flag, budget)) { done_all = false; break; }
                for (int j = 0; j < DV / 64; ++j)
                    tc::tma_store_3d(&tmap_du, base + Lay::OFF_SU + j * 8192, j * 64, n * C, bh);
                tc::bulk_commit();
            }
            if (!tc::mbar_wait_or_abort(&bars.d2done, i & 1, &abort_flag, budget)) { done_all = false; break; }
            tc::tc_fence_after();
            if (i + 1 < NC) {
                // the state gradient after chunk n - 1: its fp16 copy for D1b, and to dSp
                // the fp16 copy first (D1b of the next chunk waits for it), the global copy after
                uint32_t w[DK / 2];
#pragma unroll
                for (int cb = 0; cb < DK / 32; ++cb) {
                    float v[32];
                    tc::tmem_ld32(tmem + lane_base + TM_S + cb * 32, v);
#pragma unroll
                    for (int j = 0; j < 16; ++j) w[cb * 16 + j] = tc::pack_f16(v[2 * j], v[2 * j + 1]);
                    tc::tmem_st16u(tmem + lane_base + RT_S16 + cb * 16, *reinterpret_cast<uint32_t(*)[16]>(w + cb * 16));
                }
                rev_arrive(&bars.s_ready, lane);
                if (gtid == 0 && i > 0) {
                    tc::bulk_wait_read1();
                    tc::mbar_arrive(&bars.ss_free);
                }
                if (i > 0 && !tc::mbar_wait_or_abort(&bars.ss_free, (i - 1) & 1, &abort_flag, budget)) { done_all = false; break; }
                if (vrow >= 0) {
                    uint8_t *tile = base + Lay::OFF_SS + (vrow >> 6) * (DK * 128) + 2 * (vrow & 7);
#pragma unroll
                    for (int j = 0; j < DK / 2; ++j) {
                        const __half2 pr = *reinterpret_cast<const __half2 *>(&w[j]);
                        *reinterpret_cast<__half *>(tile + tc::sw128_off(2 * j, (vrow & 63) >> 3)) = __low2half(pr);
                        *reinterpret_cast<__half *>(tile + tc::sw128_off(2 * j + 1, (vrow & 63) >> 3)) = __high2half(pr);
                    }
                }
                tc::fence_async_smem();
                rev_arrive(&bars.ss_full, lane);
                if (gtid == 0) {
                    if (!tc::mbar_wait_or_abort(&bars.ss_full, i & 1, &abort_flag, budget)) { done_all = false; break; }
                    for (int j = 0; j < DV / 64; ++j)
                        tc::tma_store_2d(&tmap_ds, base + Lay::OFF_SS + j * (DK * 128), j * 64, ((int)bh * NC + n - 1) * DK);
                    tc::bulk_commit();
                }
            }
        }
        if (gtid == 0) tc::bulk_wait_all();  // the stores have read their tiles and written dU', dSp
        if (done_all && dS0) {  // the gradient of the initial state
#pragma unroll
            for (int cb = 0; cb < DK / 16; ++cb) {
                float v[16];
                tc::tmem_ld16(tmem + lane_base + TM_S + cb * 16, v);
                if (vrow >= 0) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) dS0[(size_t)bh * DD + (size_t)(cb * 16 + j) * DV + vrow] = v[j];
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (tid == 0 && abort_flag) atomicOr(&g_bwd_error, 2u);
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ per chunk, in parallel
// One CTA (8 warps) per chunk; every product on mma.sync (fp16 operands, fp32 accumulation)
// out of 128-byte-swizzled fp16 tiles (64-column slabs of 128-byte rows, as the TMA lays them
// out, so that ldmatrix reads are free of bank conflicts).
namespace cw {
constexpr int THREADS = 256;

// Byte offset of element (r, c) (c a multiple of 8) in a tile of `rows` rows.
__device__ __forceinline__ uint32_t off(int rows, int r, int c) {
    return (uint32_t)((c >> 6) * rows * 128) + tc::sw128_off(r, (c & 63) >> 3);
}
// Not volatile, so that the compiler may schedule the fragment loads of an unrolled k-loop ahead
// of the MMAs that consume them; the loads keep a memory clobber, which orders them after the
// shared-memory writes and barriers that precede each block of products.
__device__ __forceinline__ void ldsm4(uint32_t (&d)[4], uint32_t addr) {
    asm("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm4t(uint32_t (&d)[4], uint32_t addr) {
    asm("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// An operand tile in shared memory: `rows` rows of 16-bit elements, row index first.
struct Tile {
    uint32_t base;  // shared address, 1024-aligned
    int rows;
};

// acc[mt][nt] += A[m0 + 16 mt .., k] B[k, n0 + 8 nt ..] over k in [0, K), for one warp.
// A_T = false: A's tile is [M][K] (row m); true: its tile is [K][M].  B_T = false: B's tile
// is [N][K] (row n); true: [K][N].
template <bool A_T, bool B_T, int MT, int NT>
__device__ __forceinline__ void gemm(float (&acc)[MT][NT][4], Tile A, Tile B, int m0, int n0, int K, int lane) {
    const int i = lane >> 3, r8 = lane & 7;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t a[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int mm = m0 + 16 * mt;
            if (!A_T) ldsm4(a[mt], A.base + off(A.rows, mm + r8 + 8 * (i & 1), k0 + 8 * (i >> 1)));
            else ldsm4t(a[mt], A.base + off(A.rows, k0 + 8 * (i >> 1) + r8, mm + 8 * (i & 1)));
        }
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
            const int nn = n0 + 16 * np;
            uint32_t b[4];  // {b0, b1} of n-tile 2 np, then of n-tile 2 np + 1
            if (!B_T) ldsm4(b, B.base + off(B.rows, nn + 8 * (i >> 1) + r8, k0 + 8 * (i & 1)));
            else ldsm4t(b, B.base + off(B.rows, k0 + 8 * (i & 1) + r8, nn + 8 * (i >> 1)));
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                mma(acc[mt][2 * np], a[mt], b[0], b[1]);
                mma(acc[mt][2 * np + 1], a[mt], b[2], b[3]);
            }
        }
    }
}
template <int MT, int NT>
__device__ __forceinline__ void zero(float (&acc)[MT][NT][4]) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
}
// Row and column of accumulator element e of tile (mt, nt) for this lane.
__device__ __forceinline__ int acc_r(int m0, int mt, int e, int lane) { return m0 + 16 * mt + (lane >> 2) + 8 * (e >> 1); }
__device__ __forceinline__ int acc_c(int n0, int nt, int e, int lane) { return n0 + 8 * nt + 2 * (lane & 3) + (e & 1); }

// Store a warp's accumulators as fp16 into a tile ([rows][cols], row = accumulator row).
template <int MT, int NT>
__device__ __forceinline__ void store16(uint8_t *tile, int rows, const float (&acc)[MT][NT][4], int m0, int n0,
                                        int lane) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int r = acc_r(m0, mt, 2 * h, lane), c = acc_c(n0, nt, 0, lane);
                *reinterpret_cast<uint32_t *>(tile + off(rows, r, c & ~7) + 2 * (c & 7)) =
                    tc::pack_f16(acc[mt][nt][2 * h], acc[mt][nt][2 * h + 1]);
            }
}

// Tiles of fp16 in shared memory filled from global memory 16 bytes (8 elements) per thread
// and step: every step's loads of a tile are issued before any of its stores (global memory
// latency is paid once per tile, not once per step).  [rows][cols] with row stride ld
// elements in global memory; rows at or past `valid` read as zero.
template <typename T, int ROWS, int COLS>
struct TileIn {
    static constexpr int PER = ROWS * COLS / 8 / THREADS;  // steps per thread
    static constexpr int W = sizeof(T) == 4 ? 2 : 1;       // 16-byte words per 8 elements
    uint4 x[PER][W];
    __device__ __forceinline__ void load(const T *src, size_t ld, int valid) {
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int e = threadIdx.x + j * THREADS, r = e / (COLS / 8), c = (e % (COLS / 8)) * 8;
#pragma unroll
            for (int w = 0; w < W; ++w)
                x[j][w] = r < valid ? *reinterpret_cast<const uint4 *>(src + (size_t)r * ld + c + 4 * w)
                                    : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    __device__ __forceinline__ void store(uint8_t *tile) const {
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int e = threadIdx.x + j * THREADS, r = e / (COLS / 8), c = (e % (COLS / 8)) * 8;
            uint4 u;
            if constexpr (std::is_same<T, __half>::value) {
                u = x[j][0];
            } else if constexpr (std::is_same<T, __nv_bfloat16>::value) {
                u = make_uint4(tc::bf16x2_to_f16x2(x[j][0].x), tc::bf16x2_to_f16x2(x[j][0].y),
                               tc::bf16x2_to_f16x2(x[j][0].z), tc::bf16x2_to_f16x2(x[j][0].w));
            } else {
                const uint4 a = x[j][0], b = x[j][W - 1];
                u = make_uint4(tc::pack_f16(__uint_as_float(a.x), __uint_as_float(a.y)),
                               tc::pack_f16(__uint_as_float(a.z), __uint_as_float(a.w)),
                               tc::pack_f16(__uint_as_float(b.x), __uint_as_float(b.y)),
                               tc::pack_f16(__uint_as_float(b.z), __uint_as_float(b.w)));
            }
            *reinterpret_cast<uint4 *>(tile + off(ROWS, r, c)) = u;
        }
    }
};
}  // namespace cw

// Shared memory of the per-chunk kernel: fp16 tiles Q, K, dO, U', dU', -dR [64][d]; S, dS'
// [dk][dv]; Ta, B, dP [64][64]; V [64][dv] (bf16, for R = V - K S); per-token a, df/dbeta,
// df/dlambda and the partial sums of da.
template <int DK, int DV>
struct ChunkLayout {
    static constexpr int TQ = 0, TK = TQ + 128 * DK, TO = TK + 128 * DK, TU = TO + 128 * DV,
                         TDU = TU + 128 * DV, TNR = TDU + 128 * DV, TS = TNR + 128 * DV,
                         TDS = TS + 2 * DK * DV, TT = TDS + 2 * DK * DV, TB = TT + 8192, TP = TB + 8192,
                         TV = TP + 8192, TEND = TV + 128 * DV;
    static constexpr int SMEM = TEND + 1024;  // + alignment slack
};

// One CTA per SM walks the chunks blockIdx.x, blockIdx.x + gridDim.x, ... (skipping heads that
// walk on CUDA cores) and loads its next chunk's tiles by TMA into the buffers the current
// chunk is done with, in three groups:
//   group 0 (Ta, dU', V), read only by R and dR: refilled after them;
//   group 1 (K, S, dO), last read by dQ and by the K- and S-terms of dK: refilled after those;
//   group 2 (Q, U', dS'), last read by the rest of dK: refilled at the end of the chunk;
// so the next chunk's first products find their operands in place.  S of a head's first chunk
// is its initial state (fp32), rounded here.
template <int DK, int DV>
__global__ void __launch_bounds__(cw::THREADS, 1)
    bwd_chunk_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_o, const __grid_constant__ CUtensorMap tmap_u,
                     const __grid_constant__ CUtensorMap tmap_du, const __grid_constant__ CUtensorMap tmap_s,
                     const __grid_constant__ CUtensorMap tmap_ds, const __grid_constant__ CUtensorMap tmap_t,
                     const __grid_constant__ CUtensorMap tmap_v,
                     const float4 *__restrict__ coef, const float *__restrict__ S0, const int *__restrict__ hs,
                     float *__restrict__ dq, float *__restrict__ dkey, float *__restrict__ dval,
                     float *__restrict__ dbeta, int L, int NC, int NCH) {
    using Lay = ChunkLayout<DK, DV>;
    using namespace cw;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    uint8_t *base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    const uint32_t sb = tc::smem_u32(base);
    __shared__ float sa[C], sfb[C], sfl[C], sda[2][4][C];  // sda: partials of da (2 kinds x 4 column groups)
    __shared__ uint64_t full[3];  // the three tile groups (TMA)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t DD = (size_t)DK * DV;
    auto next_chunk = [&](int ch) {  // this CTA's next chunk whose head takes this path
        for (ch += gridDim.x; ch < NCH; ch += gridDim.x)
            if (head_ok(hs, ch / NC)) break;
        return ch;
    };
    int ch = blockIdx.x;
    if (ch < NCH && !head_ok(hs, ch / NC)) ch = next_chunk(ch);
    if (ch >= NCH) return;  // uniform over the CTA

    // thread 0's bookkeeping of the copies in flight: group g is pending with parity pph[g]
    bool pend[3] = {false, false, false};
    uint32_t pph[3] = {0u, 0u, 0u};
    auto issue = [&](int g, int c, uint32_t parity) {
        const int bh = c / NC, n = c - bh * NC, t0 = n * C;
        if (g == 0) {
            tc::mbar_expect_tx(&full[0], C * C * 2 + 2 * 128 * DV);
            for (int j = 0; j < DV / 64; ++j) {
                tc::tma_load_3d(base + Lay::TDU + j * 8192, &tmap_du, &full[0], j * 64, t0, bh);
                tc::tma_load_3d(base + Lay::TV + j * 8192, &tmap_v, &full[0], j * 64, t0, bh);
            }
            tc::tma_load_2d(base + Lay::TT, &tmap_t, &full[0], 0, c * C);
        } else if (g == 1) {
            tc::mbar_expect_tx(&full[1], 128 * DK + (n > 0 ? 2 * DK * DV : 0) + 128 * DV);
            for (int j = 0; j < DK / 64; ++j) tc::tma_load_3d(base + Lay::TK + j * 8192, &tmap_k, &full[1], j * 64, t0, bh);
            for (int j = 0; j < DV / 64; ++j) {
                if (n > 0) tc::tma_load_2d(base + Lay::TS + j * 128 * DK, &tmap_s, &full[1], j * 64, (c - 1) * DK);
                tc::tma_load_3d(base + Lay::TO + j * 8192, &tmap_o, &full[1], j * 64, t0, bh);
            }
        } else {
            tc::mbar_expect_tx(&full[2], 128 * DK + 128 * DV + 2 * DK * DV);
            for (int j = 0; j < DK / 64; ++j) tc::tma_load_3d(base + Lay::TQ + j * 8192, &tmap_q, &full[2], j * 64, t0, bh);
            for (int j = 0; j < DV / 64; ++j) {
                tc::tma_load_3d(base + Lay::TU + j * 8192, &tmap_u, &full[2], j * 64, t0, bh);
                tc::tma_load_2d(base + Lay::TDS + j * 128 * DK, &tmap_ds, &full[2], j * 64, c * DK);
            }
        }
        pend[g] = true;
        pph[g] = parity;
    };
    if (tid == 0) {
        for (int g = 0; g < 3; ++g) tc::mbar_init(&full[g], 1);
        tc::fence_mbar_init();
        for (int g = 0; g < 3; ++g) issue(g, ch, 0u);
    }
    __syncthreads();  // the barriers' initialisation

    const Tile tQ{sb + Lay::TQ, C}, tK{sb + Lay::TK, C}, tO{sb + Lay::TO, C}, tU{sb + Lay::TU, C};
    const Tile tDU{sb + Lay::TDU, C}, tNR{sb + Lay::TNR, C}, tS{sb + Lay::TS, DK}, tDS{sb + Lay::TDS, DK};
    const Tile tT{sb + Lay::TT, C}, tB{sb + Lay::TB, C}, tP{sb + Lay::TP, C};
    // warp tile: rows m0 .. m0 + 31; columns n0 .. of a 64 x N output (N / 4 columns per warp)
    const int m0 = 32 * (warp & 1), wc = warp >> 1;
    constexpr int NV = DV / 32, NKK = DK / 32;  // n-tiles of 8 per warp for N = dv, N = dk
    const int n0k = wc * (DK / 4);
    uint32_t ph = 0;
    bool ok = true, aborted = false;
    auto wait_group = [&](int g) {
        const bool w = tc::mbar_wait(&full[g], ph, WAIT_BUDGET);
        if (w && tid == 0) pend[g] = false;
        ok = ok && w;
    };
    // the end of a step: every thread's accesses to the buffers about to be refilled are ordered
    // before the copies (proxy fence, then the barrier); false if some copy did not land in time
    auto step_end = [&]() {
        tc::fence_async_smem();
        aborted = __syncthreads_or(!ok);  // uniform over the CTA
        return !aborted;
    };

    while (true) {
        const int bh = ch / NC, n = ch - bh * NC;
        const int t0 = n * C, valid = min(C, L - t0);
        const size_t tokq = (size_t)bh * L + t0;
        const int nx = next_chunk(ch);
        if (n == 0) {  // the initial state (fp32 [dk][dv]), or zero; S's buffer is free since the last dQ
            for (int e = tid; e < DK * DV; e += THREADS) {
                const int kr = e / DV, vc = e - kr * DV;
                const float x = S0 ? S0[(size_t)bh * DD + e] : 0.f;
                *reinterpret_cast<__half *>(base + Lay::TS + off(DK, kr, vc & ~7) + 2 * (vc & 7)) = __float2half_rn(x);
            }
        }
        if (tid < C) {
            const float4 c = tid < valid ? coef[2 * (tokq + tid)] : make_float4(0.f, 1.f, 0.f, 0.f);
            sa[tid] = c.y;
            sfb[tid] = c.z;
            sfl[tid] = c.w;
        }
        wait_group(1);
        // K to fp16 in place (bf16 values are exact in fp16 from 2^-14 up)
        for (int e = tid; e < 128 * DK / 16; e += THREADS) {
            uint4 *p = reinterpret_cast<uint4 *>(base + Lay::TK) + e;
            uint4 u = *p;
            u.x = tc::bf16x2_to_f16x2(u.x); u.y = tc::bf16x2_to_f16x2(u.y);
            u.z = tc::bf16x2_to_f16x2(u.z); u.w = tc::bf16x2_to_f16x2(u.w);
            *p = u;
        }
        wait_group(0);
        __syncthreads();

        // ---- R = V - K S and dR = Ta^T dU' ([64][dv]); da's first part dR_t . R_t; dV = dR
        {
            float accR[2][NV][4], accD[2][NV][4];
            zero(accR);
            zero(accD);
            const int n0 = wc * (DV / 4);
            gemm<false, true>(accR, tK, tS, m0, n0, DK, lane);
            gemm<true, true>(accD, tT, tDU, m0, n0, C, lane);
            float part[2][2] = {{0.f, 0.f}, {0.f, 0.f}};  // [mt][row half]
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < NV; ++nt)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int r = acc_r(m0, mt, 2 * h, lane), c = acc_c(n0, nt, 0, lane);
                        const __nv_bfloat162 vv = *reinterpret_cast<const __nv_bfloat162 *>(  // 0 past the end
                            base + Lay::TV + off(C, r, c & ~7) + 2 * (c & 7));
                        float *a = &accD[mt][nt][2 * h];
                        part[mt][h] += a[0] * (__low2float(vv) - accR[mt][nt][2 * h]) +
                                       a[1] * (__high2float(vv) - accR[mt][nt][2 * h + 1]);
                        if (r < valid) *reinterpret_cast<float2 *>(dval + (tokq + r) * DV + c) = make_float2(a[0], a[1]);
                        a[0] = -a[0];
                        a[1] = -a[1];
                    }
            store16(base + Lay::TNR, C, accD, m0, n0, lane);  // -dR
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float x = part[mt][h];
                    x += __shfl_xor_sync(0xffffffffu, x, 1);
                    x += __shfl_xor_sync(0xffffffffu, x, 2);
                    if ((lane & 3) == 0) sda[0][wc][acc_r(m0, mt, 2 * h, lane)] = x;
                }
        }
        if (!step_end()) break;
        if (tid == 0 && nx < NCH) issue(0, nx, ph ^ 1u);  // Ta, dU', V are done with
        wait_group(2);
        for (int e = tid; e < 128 * DK / 16; e += THREADS) {  // Q to fp16 in place
            uint4 *p = reinterpret_cast<uint4 *>(base + Lay::TQ) + e;
            uint4 u = *p;
            u.x = tc::bf16x2_to_f16x2(u.x); u.y = tc::bf16x2_to_f16x2(u.y);
            u.z = tc::bf16x2_to_f16x2(u.z); u.w = tc::bf16x2_to_f16x2(u.w);
            *p = u;
        }
        if ((aborted = __syncthreads_or(!ok))) break;
        // ---- G = K K^T, B = strictly-lower(-dR U'^T), dP = lower-incl(dO U'^T) ([64][64]);
        // da's second part sum_s B_ts G_ts
        {
            float accG[2][2][4], accB[2][2][4];
            zero(accG);
            zero(accB);
            const int n0 = wc * 16;
            gemm<false, false>(accG, tK, tK, m0, n0, DK, lane);
            gemm<false, false>(accB, tNR, tU, m0, n0, DV, lane);
            float part[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = acc_r(m0, mt, e, lane), c = acc_c(n0, nt, e, lane);
                        if (c >= r) accB[mt][nt][e] = 0.f;
                        part[mt][e >> 1] += accB[mt][nt][e] * accG[mt][nt][e];
                    }
            store16(base + Lay::TB, C, accB, m0, n0, lane);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float x = part[mt][h];
                    x += __shfl_xor_sync(0xffffffffu, x, 1);
                    x += __shfl_xor_sync(0xffffffffu, x, 2);
                    if ((lane & 3) == 0) sda[1][wc][acc_r(m0, mt, 2 * h, lane)] = x;
                }
            float accP[2][2][4];
            zero(accP);
            gemm<false, false>(accP, tO, tU, m0, n0, DV, lane);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (acc_c(n0, nt, e, lane) > acc_r(m0, mt, e, lane)) accP[mt][nt][e] = 0.f;
            store16(base + Lay::TP, C, accP, m0, n0, lane);
        }
        __syncthreads();
        // ---- da_t = (dR_t . R_t + sum_s B_ts G_ts) / a_t;  dbeta = da df/dbeta
        if (tid < C) {
            const float s1 = sda[0][0][tid] + sda[0][1][tid] + sda[0][2][tid] + sda[0][3][tid];
            const float s2 = sda[1][0][tid] + sda[1][1][tid] + sda[1][2][tid] + sda[1][3][tid];
            const float da = tid < valid ? (s1 + s2) / sa[tid] : 0.f;
            sa[tid] = da;  // from here on: da
            if (tid < valid) dbeta[tokq + tid] = da * sfb[tid];
        }
        __syncthreads();
        // ---- dQ = dO S^T + dP K ([64][dk])
        {
            float acc[2][NKK][4];
            zero(acc);
            gemm<false, false>(acc, tO, tS, m0, n0k, DV, lane);
            gemm<false, true>(acc, tP, tK, m0, n0k, C, lane);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < NKK; ++nt)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int r = acc_r(m0, mt, 2 * h, lane), c = acc_c(n0k, nt, 0, lane);
                        if (r < valid)
                            *reinterpret_cast<float2 *>(dq + (tokq + r) * DK + c) =
                                make_float2(acc[mt][nt][2 * h], acc[mt][nt][2 * h + 1]);
                    }
        }
        // ---- dK = U' dS'^T + dP^T Q - dR S^T + B K + B^T K + 2 da (df/dlambda) K ([64][dk]):
        // the terms in S and K first, so that K, S and dO can be refilled while the rest runs
        float acc[2][NKK][4];
        __half2 kreg[2][NKK][2];  // K at this thread's accumulator positions (exact bf16 values)
        zero(acc);
        gemm<false, false>(acc, tNR, tS, m0, n0k, DV, lane);
        gemm<false, true>(acc, tB, tK, m0, n0k, C, lane);
        gemm<true, true>(acc, tB, tK, m0, n0k, C, lane);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NKK; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = acc_r(m0, mt, 2 * h, lane), c = acc_c(n0k, nt, 0, lane);
                    kreg[mt][nt][h] = *reinterpret_cast<const __half2 *>(base + Lay::TK + off(C, r, c & ~7) + 2 * (c & 7));
                }
        if (!step_end()) break;
        if (tid == 0 && nx < NCH) issue(1, nx, ph ^ 1u);  // K, S, dO are done with
        gemm<false, false>(acc, tU, tDS, m0, n0k, DV, lane);
        gemm<true, true>(acc, tP, tQ, m0, n0k, C, lane);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NKK; ++nt)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = acc_r(m0, mt, 2 * h, lane), c = acc_c(n0k, nt, 0, lane);
                    if (r < valid) {
                        const float2 kk = __half22float2(kreg[mt][nt][h]);
                        const float f = 2.f * sa[r] * sfl[r];
                        *reinterpret_cast<float2 *>(dkey + (tokq + r) * DK + c) =
                            make_float2(acc[mt][nt][2 * h] + f * kk.x, acc[mt][nt][2 * h + 1] + f * kk.y);
                    }
                }
        if (!step_end()) break;
        if (tid == 0 && nx < NCH) issue(2, nx, ph ^ 1u);  // Q, U', dS' are done with
        if (nx >= NCH) break;
        ch = nx;
        ph ^= 1u;
    }
    if (aborted && tid == 0) {  // a copy did not land in time: let this CTA's copies land (bounded)
        atomicOr(&g_bwd_error, 4u);
        for (int g = 0; g < 3; ++g)
            if (pend[g]) tc::mbar_wait(&full[g], pph[g], WAIT_BUDGET / 4);
    }
}

// ------------------------------------------------------------------ per-chunk products on tcgen05 (d = 128)
// The same products transposed so that d_k or d_v (128) is the MMA M dimension and the chunk's
// 64 tokens are N, with fp32 accumulators in tensor memory:
//   (K S)^T = S^T K^T,  dR^T = dU'^T Ta,  G = K K^T,  dP = dO U'^T,  B = (-dR) U'^T   (the last
//   three 64 x 64, M = 64, both operands K-major),  dQ^T = S dO^T + K^T dP^T,
//   dK^T = dS' U'^T + Q^T dP + S (-dR)^T + K^T B^T + K^T B.
// One CTA of 8 warps per SM walks the chunks as the mma.sync kernel does; thread 0 issues the
// MMAs in five groups, each started as soon as the tiles it reads are written (the -dR tile is
// [64][128], written from dR^T column by column), so that every epilogue but the first runs
// beside the next group; and the TMA copies of the next chunk, in four groups, each as soon as
// the buffers it refills are done with.  Each warp reads one TMEM lane quarter and half of the 64 token columns.
struct TcChunkLayout {
    // 1024-aligned byte offsets: K twice (the next chunk's is loaded while this one's is read),
    // Q, dO, U', dU', V, -dR [64][128]; S, dS' [128][128]; Ta, B, dP [64][64]
    static constexpr int K0 = 0, Q = 32768, O = 49152, U = 65536, DU = 81920, V = 98304, S = 114688,
                         DS = 147456, T = 180224, NR = 188416, BM = 204800, DP = 212992, END = 221184;
    static constexpr int SMEM = END + 1024;  // + alignment slack
};
// TMEM columns of the accumulators (fp32, 64 columns each)
constexpr uint32_t TM_R = 0, TM_DR = 64, TM_G = 128, TM_DP = 192, TM_B = 256, TM_DQ = 320, TM_DK = 384;

__global__ void __launch_bounds__(cw::THREADS, 1)
    bwd_chunk_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_o, const __grid_constant__ CUtensorMap tmap_u,
                        const __grid_constant__ CUtensorMap tmap_du, const __grid_constant__ CUtensorMap tmap_s,
                        const __grid_constant__ CUtensorMap tmap_ds, const __grid_constant__ CUtensorMap tmap_t,
                        const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_dk,
                        int dk_tma, const float4 *__restrict__ coef, const float *__restrict__ S0,
                        const int *__restrict__ hs, float *__restrict__ dq, float *__restrict__ dkey,
                        float *__restrict__ dval, float *__restrict__ dbeta, int L, int NC, int NCH) {
    using Lay = TcChunkLayout;
    using cw::off;
    constexpr int DK = 128, DV = 128, THREADS = cw::THREADS;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    uint8_t *base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    const uint32_t sb = tc::smem_u32(base);
    __shared__ float sa[C], sfb[C], sfl[C], sda[2][4][C];  // sda[0][quarter][t], sda[1][half][t]
    __shared__ uint64_t full[4], mbar[6];  // TMA groups; MMA groups (see below) and the final drain
    __shared__ uint32_t tmem_base;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qw = warp & 3, hh = warp >> 2;  // TMEM lane quarter, token-column half
    const size_t DD = (size_t)DK * DV;
    // The walk takes the chunks in the order chunk 0 of every head, then chunk 1, ...: the reverse
    // chain has just written the low chunks' dU' and dS' last, so the first chunks walked find
    // them (and the chain's q, k, dO and Ta tiles) still in L2.  Walk index w is chunk n = w / BH
    // of head w % BH; NCH (as returned) means past the end.
    const int BH = NCH / NC;
    auto chunk_at = [&](int w) { return w < NCH ? (w % BH) * NC + w / BH : NCH; };
    auto next_walk = [&](int w) {  // this CTA's next walk index whose head takes this path
        for (w += gridDim.x; w < NCH; w += gridDim.x)
            if (head_ok(hs, w % BH)) break;
        return w;
    };
    int wk = blockIdx.x;
    if (wk < NCH && !head_ok(hs, wk % BH)) wk = next_walk(wk);
    if (wk >= NCH) return;  // uniform over the CTA
    int ch = chunk_at(wk);

    // thread 0's bookkeeping of the copies in flight: group g is pending with parity pph[g]
    bool pend[4] = {false, false, false, false};
    uint32_t pph[4] = {0u, 0u, 0u, 0u};
    // group 0: Ta, dU' and K (into buffer kbuf); group 1: dO, dS', V; group 2: S (past a head's
    // first chunk), U'; group 3: Q
    // every tile is read once here (the last reader of each), so it comes in under evict-first:
    // the lines the reverse chain left in L2 outlive this kernel's own reads
    const uint64_t pol = tc::l2_evict_first_policy();
    auto issue = [&](int g, int c, uint32_t parity, int kbuf) {
        const int bh = c / NC, n = c - bh * NC, t0 = n * C;
        if (g == 0) {
            tc::mbar_expect_tx(&full[0], C * C * 2 + 2 * 128 * DV);
            for (int j = 0; j < 2; ++j) {
                tc::tma_load_3d_hint(base + Lay::DU + j * 8192, &tmap_du, &full[0], j * 64, t0, bh, pol);
                tc::tma_load_3d_hint(base + Lay::K0 + kbuf * 16384 + j * 8192, &tmap_k, &full[0], j * 64, t0, bh, pol);
            }
            tc::tma_load_2d_hint(base + Lay::T, &tmap_t, &full[0], 0, c * C, pol);
        } else if (g == 1) {
            tc::mbar_expect_tx(&full[1], 2 * 128 * DV + 2 * DK * DV);
            for (int j = 0; j < 2; ++j) {
                tc::tma_load_3d_hint(base + Lay::O + j * 8192, &tmap_o, &full[1], j * 64, t0, bh, pol);
                tc::tma_load_3d_hint(base + Lay::V + j * 8192, &tmap_v, &full[1], j * 64, t0, bh, pol);
                tc::tma_load_2d_hint(base + Lay::DS + j * 128 * DK, &tmap_ds, &full[1], j * 64, c * DK, pol);
            }
        } else if (g == 2) {
            tc::mbar_expect_tx(&full[2], (n > 0 ? 2 * DK * DV : 0) + 128 * DV);
            for (int j = 0; j < 2; ++j) {
                if (n > 0) tc::tma_load_2d_hint(base + Lay::S + j * 128 * DK, &tmap_s, &full[2], j * 64, (c - 1) * DK, pol);
                tc::tma_load_3d_hint(base + Lay::U + j * 8192, &tmap_u, &full[2], j * 64, t0, bh, pol);
            }
        } else {
            tc::mbar_expect_tx(&full[3], 128 * DK);
            for (int j = 0; j < 2; ++j) tc::tma_load_3d_hint(base + Lay::Q + j * 8192, &tmap_q, &full[3], j * 64, t0, bh, pol);
        }
        pend[g] = true;
        pph[g] = parity;
    };
    if (tid == 0) {
        for (int g = 0; g < 4; ++g) tc::mbar_init(&full[g], 1);
        for (int g = 0; g < 6; ++g) tc::mbar_init(&mbar[g], 1);
        tc::fence_mbar_init();
        for (int g = 0; g < 4; ++g) issue(g, ch, 0u, 0);
    }
    if (warp == 0) {
        tc::tmem_alloc(&tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t tq = tmem + ((uint32_t)(32 * qw) << 16);  // this warp's lane quarter

    // instruction descriptors (fp16 operands, fp32 accumulators): M, N, A MN-major, B MN-major
    constexpr uint32_t ID_R = tc::idesc_f16(128, 64, true, false);     // S^T K^T
    constexpr uint32_t ID_DR = tc::idesc_f16(128, 64, true, true);     // dU'^T Ta
    constexpr uint32_t ID_G = tc::idesc_f16(64, 64, false, false);     // K K^T, dO U'^T, (-dR) U'^T
    constexpr uint32_t ID_KM = tc::idesc_f16(128, 64, false, false);   // S dO^T, dS' U'^T, S (-dR)^T
    constexpr uint32_t ID_KT = tc::idesc_f16(128, 64, true, false);    // K^T dP^T, K^T B^T
    constexpr uint32_t ID_KTM = tc::idesc_f16(128, 64, true, true);    // Q^T dP, K^T B
    // shared-memory descriptors: K-major [rows][64-column slabs] tiles step 32 bytes per 16
    // columns and `slab` bytes per 64; MN-major tiles step 2048 bytes per 16 rows, their
    // 64-element blocks `slab` bytes apart
    auto kmaj = [&](int off0, int slab, int kk) {
        return tc::sdesc(sb + off0 + (kk >> 2) * slab + (kk & 3) * 32, 16, 1024);
    };
    auto mnmaj = [&](int off0, int slab, int kk) { return tc::sdesc(sb + off0 + kk * 2048, slab, 1024); };

    uint32_t ph = 0;
    int kb = 0;  // K buffer of the current chunk
    bool ok = true, aborted = false;
    // token tid's coefficients {lambda, a, df/dbeta, df/dlambda} of chunk c (tid < 64), loaded a
    // chunk ahead so that the global-load latency is off the chunk's path
    auto load_coef = [&](int c) {
        if (tid >= C || c >= NCH) return make_float4(0.f, 1.f, 0.f, 0.f);
        const int b2 = c / NC, t2 = (c - b2 * NC) * C + tid;
        return t2 < L ? coef[2 * ((size_t)b2 * L + t2)] : make_float4(0.f, 1.f, 0.f, 0.f);
    };
    float4 coef_next = load_coef(ch);
    auto wait_group = [&](int g) {
        const bool w = tc::mbar_wait(&full[g], ph, WAIT_BUDGET);
        if (w && tid == 0) pend[g] = false;
        ok = ok && w;
    };
    auto wait_mma = [&](int i) {
        ok = tc::mbar_wait(&mbar[i], ph, WAIT_BUDGET) && ok;
        tc::tc_fence_after();
    };
    // the end of a step: shared-memory writes and reads and TMEM reads of every thread are
    // ordered before the MMAs and copies issued next; false if some wait ran out
    auto step_end = [&]() {
        tc::fence_async_smem();
        tc::tc_fence_before();
        aborted = __syncthreads_or(!ok);
        tc::tc_fence_after();
        return !aborted;
    };
    auto to_f16_in_place = [&](int off0) {  // a [64][128] bf16 tile to fp16
        for (int e = tid; e < 1024; e += THREADS) {
            uint4 *p = reinterpret_cast<uint4 *>(base + off0) + e;
            uint4 u = *p;
            u.x = tc::bf16x2_to_f16x2(u.x); u.y = tc::bf16x2_to_f16x2(u.y);
            u.z = tc::bf16x2_to_f16x2(u.z); u.w = tc::bf16x2_to_f16x2(u.w);
            *p = u;
        }
    };

    // MMA groups and their commit barriers (thread 0 issues them in this order):
    //   mbar[0]: (K S)^T, dR^T                      -> E1
    //   mbar[1]: G, S dO^T, dP, dS' U'^T            -> E2a (dP tile)
    //   mbar[2]: B, S (-dR)^T (after E1's tile)     -> E2b (B tile, da)
    //   mbar[3]: K^T dP^T, Q^T dP (after E2a)       -> E3a (dq)
    //   mbar[4]: K^T B^T, K^T B (after E2b)         -> E3b (dk)
    while (true) {
        const int bh = ch / NC, n = ch - bh * NC;
        const int t0 = n * C, valid = min(C, L - t0);
        const size_t tokq = (size_t)bh * L + t0;
        const int nwk = next_walk(wk), nx = chunk_at(nwk);
        const int KB = Lay::K0 + kb * 16384;
        if (n == 0) {  // the initial state (fp32 [dk][dv]), or zero; S's buffer is free since mbar[2]
            for (int e = tid; e < DK * DV; e += THREADS) {
                const int kr = e / DV, vc = e - kr * DV;
                const float x = S0 ? S0[(size_t)bh * DD + e] : 0.f;
                *reinterpret_cast<__half *>(base + Lay::S + off(DK, kr, vc & ~7) + 2 * (vc & 7)) = __float2half_rn(x);
            }
        }
        if (tid < C) {
            sa[tid] = coef_next.y;
            sfb[tid] = coef_next.z;
            sfl[tid] = coef_next.w;
        }
        coef_next = load_coef(nx);
        wait_group(0);
        wait_group(1);
        wait_group(2);
        to_f16_in_place(KB);  // bf16 values are exact in fp16 from 2^-14 up
        if (tid == 0 && dk_tma) bulk_wait_read0();  // the last dk store has read -dR, B and dP's tiles
        if (!step_end()) break;
        if (tid == 0) {
            for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + TM_R, mnmaj(Lay::S, 16384, kk), kmaj(KB, 8192, kk), ID_R, kk > 0);
            for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(tmem + TM_DR, mnmaj(Lay::DU, 8192, kk), mnmaj(Lay::T, 8192, kk), ID_DR, kk > 0);
            tc::mma_commit(&mbar[0]);
            for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + TM_G, kmaj(KB, 8192, kk), kmaj(KB, 8192, kk), ID_G, kk > 0);
            for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + TM_DQ, kmaj(Lay::S, 16384, kk), kmaj(Lay::O, 8192, kk), ID_KM, kk > 0);
            for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + TM_DP, kmaj(Lay::O, 8192, kk), kmaj(Lay::U, 8192, kk), ID_G, kk > 0);
            for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + TM_DK, kmaj(Lay::DS, 16384, kk), kmaj(Lay::U, 8192, kk), ID_KM, kk > 0);
            tc::mma_commit(&mbar[1]);
        }
        __syncwarp();
        // ---- E1: R = V - K S and dR (lane = value column v, 32 token columns per warp): dV = dR;
        // -dR as an fp16 tile; da's first part sum_v dR_tv R_tv
        wait_mma(0);
        if (tid == 0 && nx < NCH) issue(0, nx, ph ^ 1u, kb ^ 1);  // Ta and dU' are done with
        __syncwarp();
        {
            const int v = 32 * qw + lane;
            float R[32], D[32];
            tc::tmem_ld32(tq + TM_R + 32 * hh, R);
            tc::tmem_ld32(tq + TM_DR + 32 * hh, D);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int t = 32 * hh + j;
                const uint32_t o = off(C, t, v & ~7) + 2 * (v & 7);
                const float vv = __bfloat162float(  // 0 past the sequence end (TMA fill)
                    *reinterpret_cast<const __nv_bfloat16 *>(base + Lay::V + o));
                if (t < valid) dval[(tokq + t) * DV + v] = D[j];
                *reinterpret_cast<__half *>(base + Lay::NR + o) = __float2half_rn(-D[j]);
                R[j] = D[j] * (vv - R[j]);
            }
            // sum over the warp's 32 values of v for each of its 32 tokens (lane j ends with token j)
#pragma unroll
            for (int s = 16; s >= 1; s >>= 1) {
                const bool up = (lane & s) != 0;
#pragma unroll
                for (int j = 0; j < s; ++j) {
                    const float keep = up ? R[j + s] : R[j], send = up ? R[j] : R[j + s];
                    R[j] = keep + __shfl_xor_sync(0xffffffffu, send, s);
                }
            }
            sda[0][qw][32 * hh + lane] = R[0];
        }
        // ---- E2a: dP (M = 64: row t = 16 quarter + lane at lanes 0-15 of the quarter; 32
        // columns s per warp), masked to s <= t, as an fp16 tile; Q to fp16
        wait_mma(1);
        {
            float P[32];
            tc::tmem_ld32(tq + TM_DP + 32 * hh, P);
            if (lane < 16) {
                const int t = 16 * qw + lane;
                uint32_t pp[16];
#pragma unroll
                for (int j = 0; j < 32; j += 2)
                    pp[j >> 1] = tc::pack_f16(32 * hh + j <= t ? P[j] : 0.f, 32 * hh + j + 1 <= t ? P[j + 1] : 0.f);
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    *reinterpret_cast<uint4 *>(base + Lay::DP + t * 128 + (((4 * hh + m) ^ (t & 7)) << 4)) =
                        make_uint4(pp[4 * m], pp[4 * m + 1], pp[4 * m + 2], pp[4 * m + 3]);
            }
        }
        wait_group(3);
        to_f16_in_place(Lay::Q);
        if (!step_end()) break;  // -dR, dP and Q visible to the MMAs; V, dO, dS' are done with
        if (tid == 0) {
            for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + TM_B, kmaj(Lay::NR, 8192, kk), kmaj(Lay::U, 8192, kk), ID_G, kk > 0);
            for (int kk = 0; kk < 8; ++kk) tc::mma_bf16(tmem + TM_DK, kmaj(Lay::S, 16384, kk), kmaj(Lay::NR, 8192, kk), ID_KM, 1u);
            tc::mma_commit(&mbar[2]);
            for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(tmem + TM_DQ, mnmaj(KB, 8192, kk), kmaj(Lay::DP, 8192, kk), ID_KT, 1u);
            for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(tmem + TM_DK, mnmaj(Lay::Q, 8192, kk), mnmaj(Lay::DP, 8192, kk), ID_KTM, 1u);
            tc::mma_commit(&mbar[3]);
            if (nx < NCH) issue(1, nx, ph ^ 1u, 0);
        }
        __syncwarp();
        // ---- E2b: G and B (M = 64 as dP): B masked to s < t as an fp16 tile; da's second part
        // sum_s B_ts G_ts
        wait_mma(2);
        {
            float G[32], Bv[32];
            tc::tmem_ld32(tq + TM_G + 32 * hh, G);
            tc::tmem_ld32(tq + TM_B + 32 * hh, Bv);
            if (lane < 16) {
                const int t = 16 * qw + lane;
                float part = 0.f;
                uint32_t pb[16];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    Bv[j] = 32 * hh + j < t ? Bv[j] : 0.f;
                    part += Bv[j] * G[j];
                    if (j & 1) pb[j >> 1] = tc::pack_f16(Bv[j - 1], Bv[j]);
                }
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    *reinterpret_cast<uint4 *>(base + Lay::BM + t * 128 + (((4 * hh + m) ^ (t & 7)) << 4)) =
                        make_uint4(pb[4 * m], pb[4 * m + 1], pb[4 * m + 2], pb[4 * m + 3]);
                sda[1][hh][t] = part;
            }
        }
        if (!step_end()) break;  // the B tile visible to the MMAs; S and U' are done with
        if (tid == 0) {
            for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(tmem + TM_DK, mnmaj(KB, 8192, kk), kmaj(Lay::BM, 8192, kk), ID_KT, 1u);
            for (int kk = 0; kk < 4; ++kk) tc::mma_bf16(tmem + TM_DK, mnmaj(KB, 8192, kk), mnmaj(Lay::BM, 8192, kk), ID_KTM, 1u);
            tc::mma_commit(&mbar[4]);
            if (nx < NCH) issue(2, nx, ph ^ 1u, 0);
        }
        __syncwarp();
        // ---- da_t = (dR_t . R_t + sum_s B_ts G_ts) / a_t;  dbeta = da df/dbeta
        if (tid < C) {
            const float s1 = sda[0][0][tid] + sda[0][1][tid] + sda[0][2][tid] + sda[0][3][tid];
            const float da = tid < valid ? (s1 + sda[1][0][tid] + sda[1][1][tid]) / sa[tid] : 0.f;
            sa[tid] = da;  // from here on: da
            if (tid < valid) dbeta[tokq + tid] = da * sfb[tid];
        }
        // ---- E3a: dQ^T (lane = key column c, 32 token columns per warp)
        const int c = 32 * qw + lane;
        float A[32];
        wait_mma(3);
        tc::tmem_ld32(tq + TM_DQ + 32 * hh, A);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int t = 32 * hh + j;
            if (t < valid) dq[(tokq + t) * DK + c] = A[j];
        }
        __syncthreads();  // da
        // ---- E3b: dK^T, plus 2 da (df/dlambda) k; into the [64][128] fp32 tile over -dR, B and
        // dP (their products are done), stored by TMA (rows past L are not stored), or straight
        // to global memory where dk is not 16-byte aligned
        wait_mma(4);
        tc::tmem_ld32(tq + TM_DK + 32 * hh, A);
        float *dk_tile = reinterpret_cast<float *>(base + Lay::NR);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int t = 32 * hh + j;
            // K's fp16 tile holds the bf16 values exactly (zero past the sequence end)
            const float kk = __half2float(
                *reinterpret_cast<const __half *>(base + KB + off(C, t, c & ~7) + 2 * (c & 7)));
            const float x = A[j] + 2.f * sa[t] * sfl[t] * kk;
            if (dk_tma) dk_tile[t * DK + c] = x;
            else if (t < valid) dkey[(tokq + t) * DK + c] = x;
        }
        if (!step_end()) break;  // Q and this K are done with; the dk tile written
        if (tid == 0 && dk_tma) {
            tc::tma_store_3d(&tmap_dk, dk_tile, 0, t0, bh);
            tc::bulk_commit();
        }
        if (tid == 0 && nx < NCH) issue(3, nx, ph ^ 1u, 0);
        if (nx >= NCH) break;
        ch = nx;
        wk = nwk;
        ph ^= 1u;
        kb ^= 1;
    }
    if (tid == 0) {
        if (aborted) {  // a wait ran out: let this CTA's copies land (bounded)
            atomicOr(&g_bwd_error, 4u);
            for (int g = 0; g < 4; ++g)
                if (pend[g]) tc::mbar_wait(&full[g], pph[g], WAIT_BUDGET / 4);
        }
        tc::bulk_wait_all();       // the dk stores are done
        tc::mma_commit(&mbar[5]);  // arrives once every MMA issued so far has completed
        if (!tc::mbar_wait(&mbar[5], 0, WAIT_BUDGET)) atomicOr(&g_bwd_error, 4u);
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

// dO (fp32) to fp16 for the products; and which heads take the tensor-core path.
__global__ void __launch_bounds__(256) bwd_prepare_kernel(const float *__restrict__ dO, __half *__restrict__ dO16,
                                                         size_t n4) {
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4; e += (size_t)gridDim.x * blockDim.x) {
        const float4 x = reinterpret_cast<const float4 *>(dO)[e];
        reinterpret_cast<uint2 *>(dO16)[e] = make_uint2(tc::pack_f16(x.x, x.y), tc::pack_f16(x.z, x.w));
    }
}

template <int DK, int DV>
cudaError_t launch_bwd_tc_t(const void *q, const void *k, const void *v, const float *S0, const float *dO,
                            const float *dSL, const float4 *coef, const int *hs, const __half *u_saved,
                            const __half *ck_saved, const void *ta, float *dq, float *dkey, float *dval,
                            float *dbeta, float *dS0, int B, int H, int L, void *ws, cudaStream_t s,
                            bool dO16_ready) {
    const int BH = B * H, NC = (L + C - 1) / C;
    const size_t ntok = (size_t)BH * L;
    __half *dO16 = (__half *)ws;
    __half *dU = dO16 + ntok * DV;  // 16-byte aligned: dv is 64 or 128
    __half *dSp = dU + ntok * DV;
    // the per-chunk products on tcgen05 at d = 128 (transposed, d the MMA M), on mma.sync otherwise
    constexpr bool TC_CHUNK = DK == 128 && DV == 128;
    static bool attr_done[64] = {};
    int dev = 0, nsm = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
        e = cudaFuncSetAttribute(bwd_state_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 RevLayout<DK, DV>::SMEM);
        if (e == cudaSuccess) {
            if constexpr (TC_CHUNK)
                e = cudaFuncSetAttribute(bwd_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         TcChunkLayout::SMEM);
            else
                e = cudaFuncSetAttribute(bwd_chunk_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         ChunkLayout<DK, DV>::SMEM);
        }
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    CUtensorMap mq, mk, mo, mt;
    if (!tmap::make_3d(&mq, q, DK, L, BH, 64, C) || !tmap::make_3d(&mk, k, DK, L, BH, 64, C) ||
        !tmap::make_3d(&mo, dO16, DV, L, BH, 64, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !tmap::make_2d(&mt, ta, C, (uint64_t)BH * NC * C, 64, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return cudaErrorInvalidValue;
    const size_t n4 = ntok * DV / 4;
    const int g = (int)std::min<size_t>((n4 + 255) / 256, (size_t)nsm * 16);
    CUtensorMap mu, mdu, ms, mds, mv;
    const uint64_t rows = (uint64_t)BH * NC * DK;  // [BH][NC][dk] rows of dv columns
    if (!tmap::make_3d(&mu, u_saved, DV, L, BH, 64, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !tmap::make_3d(&mdu, dU, DV, L, BH, 64, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !tmap::make_2d(&ms, ck_saved, DV, rows, 64, DK, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !tmap::make_2d(&mds, dSp, DV, rows, 64, DK, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
        !tmap::make_3d(&mv, v, DV, L, BH, 64, C))
        return cudaErrorInvalidValue;
    if (!dO16_ready) bwd_prepare_kernel<<<g, 256, 0, s>>>(dO, dO16, n4);
    bwd_state_kernel<DK, DV><<<BH, REV_THREADS, RevLayout<DK, DV>::SMEM, s>>>(mq, mk, mo, mt, mdu, mds, dSL, dSp,
                                                                              dS0, hs, L, NC);
    const int nch = BH * NC;  // as many CTAs as fit on the SMs at once, each walking every grid-th chunk
    if constexpr (TC_CHUNK) {  // one CTA per SM
        // dk by TMA stores of [64][dk] fp32 row-major tiles where dk is 16-byte aligned
        CUtensorMap mdk;
        memset(&mdk, 0, sizeof(mdk));
        int dk_tma = 0;
        if (((uintptr_t)dkey & 15) == 0) {
            auto fn = tmap::encode_fn();
            const cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)L, (cuuint64_t)BH};
            const cuuint64_t strides[2] = {(cuuint64_t)DK * 4, (cuuint64_t)L * DK * 4};
            const cuuint32_t box[3] = {(cuuint32_t)DK, (cuuint32_t)C, 1}, es[3] = {1, 1, 1};
            dk_tma = fn && fn(&mdk, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, dkey, dims, strides, box, es,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
        }
        bwd_chunk_tc_kernel<<<std::min(nch, nsm), cw::THREADS, TcChunkLayout::SMEM, s>>>(
            mq, mk, mo, mu, mdu, ms, mds, mt, mv, mdk, dk_tma, coef, S0, hs, dq, dkey, dval, dbeta, L, NC, nch);
    } else {
        int per_sm = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bwd_chunk_kernel<DK, DV>, cw::THREADS,
                                                          ChunkLayout<DK, DV>::SMEM) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
        bwd_chunk_kernel<DK, DV><<<std::min(nch, nsm * per_sm), cw::THREADS, ChunkLayout<DK, DV>::SMEM, s>>>(
            mq, mk, mo, mu, mdu, ms, mds, mt, mv, coef, S0, hs, dq, dkey, dval, dbeta, L, NC, nch);
    }
    count_launches(dO16_ready ? 2 : 3);
    return cudaGetLastError();
}

}  // namespace

size_t bwd_tc_workspace_bytes(int B, int H, int L, int dk, int dv) {
    const size_t BH = (size_t)B * H, NC = (size_t)(L + C - 1) / C;
    // fp16 dO and dU' [BH][L][dv], dSp [BH][NC][dk][dv]
    return (2 * BH * (size_t)L * dv + BH * NC * (size_t)dk * dv) * sizeof(__half);
}

cudaError_t launch_bwd_tc(const void *q, const void *k, const void *v, const float *S0, const float *dO,
                          const float *dSL, const void *coef, const int *hs, const __half *u_saved,
                          const __half *ck_saved, const void *ta, float *dq, float *dkey, float *dval,
                          float *dbeta, float *dS0, int B, int H, int L, int dk, int dv, void *ws,
                          cudaStream_t s, bool dO16_ready) {
    const float4 *cf = (const float4 *)coef;
    if (dk == 128 && dv == 128)
        return launch_bwd_tc_t<128, 128>(q, k, v, S0, dO, dSL, cf, hs, u_saved, ck_saved, ta, dq, dkey, dval, dbeta,
                                         dS0, B, H, L, ws, s, dO16_ready);
    if (dk == 128 && dv == 64)
        return launch_bwd_tc_t<128, 64>(q, k, v, S0, dO, dSL, cf, hs, u_saved, ck_saved, ta, dq, dkey, dval, dbeta,
                                        dS0, B, H, L, ws, s, dO16_ready);
    if (dk == 64 && dv == 128)
        return launch_bwd_tc_t<64, 128>(q, k, v, S0, dO, dSL, cf, hs, u_saved, ck_saved, ta, dq, dkey, dval, dbeta,
                                        dS0, B, H, L, ws, s, dO16_ready);
    return launch_bwd_tc_t<64, 64>(q, k, v, S0, dO, dSL, cf, hs, u_saved, ck_saved, ta, dq, dkey, dval, dbeta,
                                   dS0, B, H, L, ws, s, dO16_ready);
}

cudaError_t bwd_tc_read_and_clear_error(unsigned int *out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_bwd_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_bwd_error, &zero, sizeof(unsigned int));
}

}  // namespace efla
