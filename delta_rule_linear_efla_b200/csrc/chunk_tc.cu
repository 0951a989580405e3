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
// Kernels:
//  prep  -- one chunk per 128-thread pipeline, every chunk in parallel: the squared
//           norms and a, the Gram matrix K K^T on the tensor cores (TMEM accumulator),
//           the unit-lower-triangular inverse T (16x16 diagonal blocks by fp32
//           substitution, the off-diagonal blocks by mma.sync block merges), and
//           Ta = T diag(a) written as fp16 to the workspace (64x64 per chunk).
//  state -- one CTA per head (or per segment run of a head), chunks in order, warp-
//           specialised: TMA loads q, k, v, Ta (128-byte swizzle, double buffered), an
//           in-place bf16 -> fp16 conversion, one thread issuing every tcgen05.mma
//           (W, P^T, the U' prefill and the fused D1/D2 products), and epilogue
//           warpgroups that move results between TMEM and the operand tiles; the
//           fp32 state S^T stays in TMEM across chunks, with an fp16 copy as D1's A.
//  seg_combine -- for sequence segments: chains the segments' affine state maps.
//
// The gated form (a per-token decay g_t on the carried state, S_t = g_t (I - a_t k_t
// k_t^T) S_{t-1} + a_t k_t v_t^T) runs on the same two kernels.  With l_t the cumulative
// log-decay from the chunk start to token t (l_C at the chunk's last token) and
// Gam_ts = e^{l_t - l_s}, the chunk algebra becomes
//
//   A  = strictly-lower(diag(a) (Gam o K K^T))    Ta = T diag(a) as before
//   W  = Ta diag(e^{l}) K,  U = Ta V,  U' = U - W S
//   O  = diag(e^{l}) Q S + (lower-incl(Gam) o Q K^T) U'
//   S <- e^{l_C} S + K^T diag(e^{l_C - l}) U'
//
// and every factor it applies is a decay of at most 1 (a split of Gam into e^{l_t - l_C}
// e^{l_C - l_s} would over- and underflow): the prep kernel weights the Gram by Gam; the
// state kernel's converter writes q and k both as they are and with their rows scaled by
// e^{l_t} (the scaled q for D1, the scaled k for W), the side group weights P^T by Gam, the chain group hands D2 U' twice
// (as it is for the output, with its rows scaled by e^{l_C - l_t} for the state update),
// and scales the fp32 state by the next chunk's e^{l_C} when it copies it for D1.
//
// Every mbarrier wait is bounded; a wait that gives up sets the device error
// word, drains the copies this CTA has in flight (again bounded), releases
// its tensor memory and exits.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstring>
#include <mutex>

#include <type_traits>

#include "common.cuh"
#include "launchers.h"
#include "tc_ptx.cuh"
#include "tmap.h"

namespace efla {

static __device__ unsigned int g_tc_error = 0;

namespace {

constexpr int C = 64;         // chunk (tokens)
constexpr int THREADS = 128;  // 4 warps = the 4 TMEM lane quarters
constexpr long long WAIT_BUDGET = 2000000000LL;  // ~1 s of SM cycles

__device__ __forceinline__ void record_error(unsigned code) { atomicOr(&g_tc_error, code); }

// ------------------------------------------------------------------ gated form: per-token log-decays
// l_t of a chunk's tokens 2 lane and 2 lane + 1, for every lane of a warp (0 past the sequence
// end, where the decay is taken as 1): a warp-wide inclusive scan of the pairs' logarithms.
__device__ __forceinline__ float2 chunk_logdecay(const __nv_bfloat16 *gate_row, int t0, int L, int lane) {
    const int t = t0 + 2 * lane;
    const float x0 = t < L ? logf(__bfloat162float(gate_row[t])) : 0.f;
    const float x1 = t + 1 < L ? logf(__bfloat162float(gate_row[t + 1])) : 0.f;
    float s = x0 + x1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
    }
    return make_float2(s - x1, s);
}
// Element t of a per-token quantity held as pairs (lane t / 2 holds tokens 2 lane, 2 lane + 1),
// e.g. l_t itself or a factor made from it (every lane of the warp takes part; t need not be
// uniform).
__device__ __forceinline__ float logdecay_at(float2 p, int t) {
    const float a = __shfl_sync(0xffffffffu, p.x, t >> 1), b = __shfl_sync(0xffffffffu, p.y, t >> 1);
    return (t & 1) ? b : a;
}

// ------------------------------------------------------------------ prep
// One chunk at a time (all chunks in parallel across the grid):
//   1. K arrives by TMA; a per row from the squared norm (fp32).
//   2. Gram G = K K^T on the tensor cores (tcgen05, TMEM accumulator).
//   3. A = strictly-lower(diag(a) G); T = (I + A)^{-1} by blocked forward
//      substitution on 16x16 blocks: the diagonal blocks by fp32 substitution
//      on CUDA cores, the off-diagonal blocks level by level as
//        T_IJ = -T_II * sum_{K=J}^{I-1} A_IK T_KJ
//      with warp-level mma.sync (fp16 operands, fp32 accumulation).
//   4. Ta = T diag(a), rounded to fp16, written to the workspace (64x64 per chunk).
// Gated form: the Gram's entry (t, s) is weighted by e^{l_t - l_s} (at most 1 below the
// diagonal), with l the chunk's cumulative log-decays.
namespace prep {
constexpr int LD16 = 72;   // fp16 row stride (halves) of the 64x64 operand tiles

struct Smem {
    template <int DK>
    static constexpr int k_bytes() { return DK * C * 2; }
    static constexpr int A16 = C * LD16 * 2;      // A, fp16, row-major
    static constexpr int TD16 = 4 * 16 * 24 * 2;  // T's diagonal blocks, fp16, row-major (A operands)
    static constexpr int T16T = C * LD16 * 2;     // T, fp16, transposed (B operands)
    // A's fp32 diagonal blocks (read by the diagonal solve) share their space with the
    // per-warp transposed-R scratch of the block merges, which run after the solve.
    static constexpr int ADIAG = C * 16 * 4;      // diagonal 16x16 blocks of A, fp32
    static constexpr int RT = 4 * 16 * 24 * 2;    // per-warp 16x16 scratch (transposed R), fp16
    static constexpr int AD_RT = ADIAG > RT ? ADIAG : RT;
    template <int DK>
    static constexpr int bytes() { return region0<DK>() + T16T + 2 * C * 4; }  // + a, l per row
    // The K tile is dead once the Gram MMA and the norms have read it; the solve's A, T
    // diagonal blocks and scratch then take its place (the next K is loaded after the solve).
    static constexpr int SCRATCH = A16 + TD16 + AD_RT;
    template <int DK>
    static constexpr int region0() { return k_bytes<DK>() > SCRATCH ? k_bytes<DK>() : SCRATCH; }
};

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// A fragment (16x16, row-major source with row stride ld halves) at (r0, k0).
__device__ __forceinline__ void load_a(uint32_t (&a)[4], const __half *M, int ld, int r0, int k0, int lane) {
    const int g = lane >> 2, t = lane & 3;
    a[0] = *reinterpret_cast<const uint32_t *>(M + (r0 + g) * ld + k0 + 2 * t);
    a[1] = *reinterpret_cast<const uint32_t *>(M + (r0 + g + 8) * ld + k0 + 2 * t);
    a[2] = *reinterpret_cast<const uint32_t *>(M + (r0 + g) * ld + k0 + 2 * t + 8);
    a[3] = *reinterpret_cast<const uint32_t *>(M + (r0 + g + 8) * ld + k0 + 2 * t + 8);
}
// B fragment (16 x 8) of B[k][n], read from its transpose Bt[n][k] (row stride ld).
__device__ __forceinline__ void load_b(uint32_t &b0, uint32_t &b1, const __half *Bt, int ld, int k0, int n0, int lane) {
    const int g = lane >> 2, t = lane & 3;
    b0 = *reinterpret_cast<const uint32_t *>(Bt + (n0 + g) * ld + k0 + 2 * t);
    b1 = *reinterpret_cast<const uint32_t *>(Bt + (n0 + g) * ld + k0 + 2 * t + 8);
}
}  // namespace prep

template <int DK, bool GATED = false>
__global__ void __launch_bounds__(THREADS)
    tc_prep_kernel(const __grid_constant__ CUtensorMap tmap_k, const __nv_bfloat16 *__restrict__ beta,
                   const __nv_bfloat16 *__restrict__ gate, __half *__restrict__ ta_out, int L, int NC,
                   int total, bool euler) {
    using namespace prep;
    constexpr int KB = Smem::k_bytes<DK>();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    uint8_t *base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    uint8_t *Kt = base;  // the K tile; after the Gram and the norms, the solve's scratch below
    __half *A16 = reinterpret_cast<__half *>(base);
    __half *TD16 = A16 + C * LD16;                   // [4][16][24]
    float *Ad = reinterpret_cast<float *>(TD16 + 4 * 16 * 24);  // [64 rows][16]: A's diagonal blocks
    __half *Rt = reinterpret_cast<__half *>(Ad);                // after the solve: merge scratch
    __half *T16t = reinterpret_cast<__half *>(base + Smem::region0<DK>());
    float *al = reinterpret_cast<float *>(T16t + C * LD16);
    float *lg = al + C;  // gated: l_t of the chunk's rows
    __shared__ uint64_t full, mma_bar;
    __shared__ uint32_t tmem_base;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        tc::mbar_init(&full, 1);
        tc::mbar_init(&mma_bar, 1);
        tc::fence_mbar_init();
        tc::tma_prefetch_desc(&tmap_k);
    }
    if (warp == 0) {
        tc::tmem_alloc(&tmem_base, 64);
        tc::tmem_relinquish();
    }
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_base;
    bool issued = false;

    auto issue = [&](int g) {
        const int bh = g / NC, n = g - bh * NC;
        tc::mbar_expect_tx(&full, KB);
#pragma unroll
        for (int s = 0; s < DK / 64; ++s)
            tc::tma_load_3d(Kt + s * 8192, &tmap_k, &full, s * 64, n * C, bh);
    };
    if (tid == 0 && blockIdx.x < total) {
        issue(blockIdx.x);
        issued = true;
    }
    // beta of row `tid` of chunk g (0 past the sequence end), loaded one chunk ahead so
    // the global-load latency is not on the chunk's critical path
    auto load_beta = [&](int gg) {
        if (tid >= C || gg >= total) return 0.f;
        const int bh = gg / NC, n = gg - bh * NC;
        return n * C + tid < L ? __bfloat162float(beta[(size_t)bh * L + n * C + tid]) : 0.f;
    };
    float beta_next = load_beta(blockIdx.x);
    // gated: warp 0's lane holds log g of rows 2 lane and 2 lane + 1 of chunk gg (0 past the
    // sequence end), also loaded a chunk ahead
    auto load_gate = [&](int gg) {
        float2 x = make_float2(0.f, 0.f);
        if (!GATED || warp != 0 || gg >= total) return x;
        const int bh = gg / NC, t = (gg - bh * NC) * C + 2 * lane;
        const __nv_bfloat16 *row = gate + (size_t)bh * L;
        if (t < L) x.x = logf(__bfloat162float(row[t]));
        if (t + 1 < L) x.y = logf(__bfloat162float(row[t + 1]));
        return x;
    };
    float2 gate_next = load_gate(blockIdx.x);
    uint32_t mma_phase = 0;
    int it = 0;
    bool aborted = false;
    bool mma_pending = false;
    for (int g = blockIdx.x; g < total; g += gridDim.x, ++it) {
        const uint32_t ph = it & 1;
        const int bh = g / NC, n = g - bh * NC, c0 = n * C;
        __half *gta = ta_out + (size_t)g * C * C;  // this chunk's Ta tile (row-major 64x64)
        const float beta_row = beta_next;
        beta_next = load_beta(g + gridDim.x);
        const float2 gate_pair = gate_next;
        gate_next = load_gate(g + gridDim.x);
        (void)bh;
        (void)c0;
        bool ok = tc::mbar_wait(&full, ph, WAIT_BUDGET);
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        if (tid == 0) issued = false;
        if (tid == 96) {  // warp 3 issues: warps 0-1 compute the norms meanwhile
            tc::tc_fence_after();
            const uint32_t kb = tc::smem_u32(Kt);
            constexpr uint32_t id = tc::idesc_bf16(64, 64, false, false);
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                const uint64_t d = tc::sdesc(kb + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                tc::mma_bf16(tmem, d, d, id, kk > 0 ? 1u : 0u);
            }
            tc::mma_commit(&mma_bar);
        }
        mma_pending = true;
        // a per row: squared norm from the swizzled K tile
        if (tid < C) {
            const int r = tid;
            float sq = 0.f;
#pragma unroll
            for (int sl = 0; sl < DK / 64; ++sl) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(Kt + sl * 8192 + tc::sw128_off(r, ch));
                    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h[e]);
                        sq = fmaf(f.x, f.x, fmaf(f.y, f.y, sq));
                    }
                }
            }
            al[r] = alpha_rule(sq, beta_row, euler);
        }
        if (GATED && warp == 0) {  // l_t: inclusive scan of the row pairs' log-decays
            float sc = gate_pair.x + gate_pair.y;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, sc, o);
                if (lane >= o) sc += y;
            }
            lg[2 * lane] = sc - gate_pair.y;
            lg[2 * lane + 1] = sc;
        }
        ok = tc::mbar_wait(&mma_bar, mma_phase, WAIT_BUDGET);
        if (__syncthreads_or(!ok)) { aborted = true; break; }  // also: every norm has been read
        mma_phase ^= 1;
        mma_pending = false;
        tc::tc_fence_after();
        // ---- A = strictly-lower(diag(a) G): fp16 copy (all blocks), fp32 diagonal blocks
        {
            const int r = 16 * warp + lane;  // valid for lane < 16 (M = 64 accumulator layout)
            const uint32_t ta = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float v[16];
                tc::tmem_ld16(ta + cb * 16, v);
                if (lane < 16) {
                    const float ar = al[r];
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = (cb * 16 + j < r) ? ar * v[j] : 0.f;
                    if constexpr (GATED) {  // Gam o G below the diagonal: e^{l_r - l_c} <= 1
                        // (the fast exponential: CUDA bounds its error by 2 + 1.17 |x| ulp, under
                        // 5e-5 relative for arguments down to -300, far below A's fp16 rounding)
                        const float lr = lg[r];
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (cb * 16 + j < r) v[j] *= __expf(fminf(lr - lg[cb * 16 + j], 0.f));
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(A16 + r * LD16 + cb * 16);
                    dst[0] = make_uint4(tc::pack_f16(v[0], v[1]), tc::pack_f16(v[2], v[3]),
                                        tc::pack_f16(v[4], v[5]), tc::pack_f16(v[6], v[7]));
                    dst[1] = make_uint4(tc::pack_f16(v[8], v[9]), tc::pack_f16(v[10], v[11]),
                                        tc::pack_f16(v[12], v[13]), tc::pack_f16(v[14], v[15]));
                    if (cb == (r >> 4)) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) Ad[r * 16 + j] = v[j];
                    }
                }
            }
        }
        tc::tc_fence_before();
        __syncthreads();
        // ---- diagonal blocks: column c of (I + A_bb)^{-1}, one column per thread
        if (tid < 64) {
            const int b = tid >> 4, c = tid & 15;
            const float ac = al[16 * b + c];
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float *arow = Ad + (16 * b + i) * 16;
                float s0 = (i == c) ? 1.f : 0.f, s1 = 0.f;  // two chains: half the dependent latency
#pragma unroll
                for (int m = 0; m + 1 < i; m += 2) {
                    s0 = fmaf(-arow[m], x[m], s0);
                    s1 = fmaf(-arow[m + 1], x[m + 1], s1);
                }
                if (i & 1) s0 = fmaf(-arow[i - 1], x[i - 1], s0);
                x[i] = s0 + s1;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int row = 16 * b + i, col = 16 * b + c;
                TD16[(b * 16 + i) * 24 + c] = __float2half_rn(x[i]);
                T16t[col * LD16 + row] = __float2half_rn(x[i]);
                gta[row * C + col] = __float2half_rn(x[i] * ac);
            }
        } else {
            // zero the strictly-upper 16x16 blocks of the output tile
            for (int e = tid - 64; e < 6 * 128; e += 64) {
                const int blk = e >> 7, w = e & 127;
                const int I = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
                const int J = blk < 3 ? 1 + blk : (blk < 5 ? blk - 1 : 3);
                *reinterpret_cast<uint32_t *>(gta + (16 * I + (w >> 3)) * C + 16 * J + 2 * (w & 7)) = 0u;
            }
        }
        __syncthreads();
        // ---- off-diagonal blocks, one 16x16 block per warp, level by level
        for (int lvl = 1; lvl < 4; ++lvl) {
            const int J = warp, I = J + lvl;
            if (I < 4) {
                float r[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                for (int K = J; K < I; ++K) {
                    uint32_t a[4];
                    load_a(a, A16, LD16, 16 * I, 16 * K, lane);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        uint32_t b0, b1;
                        load_b(b0, b1, T16t, LD16, 16 * K, 16 * J + 8 * nt, lane);
                        mma16816(r[nt], a, b0, b1);
                    }
                }
                // R -> fp16, transposed, into this warp's scratch
                __half *rt = Rt + warp * 16 * 24;
                const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int n0 = 8 * nt + 2 * tq;
                    rt[(n0) * 24 + gq] = __float2half_rn(r[nt][0]);
                    rt[(n0 + 1) * 24 + gq] = __float2half_rn(r[nt][1]);
                    rt[(n0) * 24 + gq + 8] = __float2half_rn(r[nt][2]);
                    rt[(n0 + 1) * 24 + gq + 8] = __float2half_rn(r[nt][3]);
                }
                __syncwarp();
                uint32_t a[4];
                load_a(a, TD16 + I * 16 * 24, 24, 0, 0, lane);
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
                    uint32_t b0, b1;
                    load_b(b0, b1, rt, 24, 0, 8 * nt, lane);
                    mma16816(d, a, b0, b1);
                    const int row = 16 * I + gq, col = 16 * J + 8 * nt + 2 * tq;
                    const float a0 = al[col], a1 = al[col + 1];
                    *reinterpret_cast<uint32_t *>(gta + row * C + col) = tc::pack_f16(-d[0] * a0, -d[1] * a1);
                    *reinterpret_cast<uint32_t *>(gta + (row + 8) * C + col) = tc::pack_f16(-d[2] * a0, -d[3] * a1);
                    T16t[col * LD16 + row] = __float2half_rn(-d[0]);
                    T16t[(col + 1) * LD16 + row] = __float2half_rn(-d[1]);
                    T16t[col * LD16 + row + 8] = __float2half_rn(-d[2]);
                    T16t[(col + 1) * LD16 + row + 8] = __float2half_rn(-d[3]);
                }
            }
            __syncthreads();
        }
        if (tid == 0 && g + (int)gridDim.x < total) {  // the solve's scratch is dead: next K tile
            tc::fence_async_smem();
            issue(g + gridDim.x);
            issued = true;
        }
    }
    if (aborted) {
        if (tid == 0) {
            record_error(1u);
            if (issued) tc::mbar_wait(&full, it & 1, WAIT_BUDGET / 4);  // drain the copy in flight
            if (mma_pending) tc::mbar_wait(&mma_bar, mma_phase, WAIT_BUDGET / 4);
        }
        __syncthreads();
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

// ------------------------------------------------------------------ state
// Products are arranged so that the state and value dimensions are the MMA M
// dimension and so that every MMA is as wide (N) as the algebra allows; a
// tcgen05.mma instruction costs about the same for every N up to 128, so
// products that share an operand are fused into one wide instruction stream:
//
//   U'^T  = V^T Ta^T                   [DV x C]   prefill of the U' accumulator
//   W     = Ta K                       [C x DK]
//   P^T   = K Q^T                      [C x C]    masked to c_in <= c_out
//   D1:  [O^T | U'^T] += S^T [Q | -W]^T           O^T from zero, U'^T = U^T - X^T
//   D2:  [S^T | O^T]  += U'^T [K | P^T]           state update and intra-chunk output
//
// TMEM columns (fp32): S^T [0, DK), O^T [DK, DK+64), U'^T [DK+64, DK+128),
// W [256, 256+DK), P^T [384, 448); [O^T | U'^T] and [S^T | O^T] are contiguous.
// The A operands of D1 and D2 -- the fp16 copy of S^T and fp16 U'^T -- also live
// in tensor memory (packed two per column: S^T at [448, 448+DK/2), U'^T over the
// first 32 columns of its own fp32 accumulator), which keeps them out of shared
// memory: with small N an MMA is bound by shared-memory bandwidth.
// MMA operands are fp16 (the bf16 Q, K, V tiles are converted in place; fp16
// holds every bf16 value of magnitude >= 2^-14 exactly and rounds the
// intermediates 8x finer than bf16); accumulation is fp32.
//
// Gated form: two more fp16 tiles per stage -- q as it is (P^T's B; the QW slabs then hold q
// with its rows scaled by e^{l_t}) and k with its rows scaled by e^{l_t} (W's B) -- and the
// masked P^T leaves the stage for two single tiles, its fp16 value and the fp16 remainder
// (P^T = hi + lo to 22 bits; the side group writes a chunk's only after the previous D2 has
// run, which the P^T product of the chunk waits for in the tensor pipe).
template <int DK, int DV, bool GATED = false>
struct StateLayout {
    static constexpr int QW_SLAB = 16384;                // per 64-column K slab: 64 Q rows, 64 -W rows
    static constexpr int QW = (DK / 64) * QW_SLAB;
    static constexpr int KP = (DK / 64 + (GATED ? 0 : 1)) * 8192;  // K slabs then the P^T block (MN-major)
    static constexpr int VB = (DV / 64) * 8192;
    static constexpr int TB = C * C * 2;
    static constexpr int XB = GATED ? (DK / 64) * 8192 : 0;  // gated: q, and k scaled by e^{l}
    static constexpr int OFF_QW = 0, OFF_KP = QW, OFF_V = QW + KP, OFF_T = QW + KP + VB;
    static constexpr int OFF_QP = OFF_T + TB, OFF_KH = OFF_QP + XB;
    static constexpr int STAGE = OFF_KH + XB;
    static constexpr int OFF_PH = 2 * STAGE, OFF_PL = OFF_PH + 8192;  // gated: P^T hi and lo
    static constexpr int BYTES = 2 * STAGE + (GATED ? 2 * 8192 : 0);
    static constexpr int SMEM = BYTES + 1024;             // alignment slack
    // the forward that keeps u and the chunk states (ungated): u [64][DV] and the state
    // [DK][DV] (fp16) on their way out by TMA, after the stages
    static constexpr int OFF_KU = BYTES, OFF_KS = OFF_KU + 128 * DV;
    static_assert(!GATED || OFF_PL + 8192 == BYTES, "gated shared-memory layout");
};

// Shared memory the keeping and saving forwards add after the stages (StateLayout::OFF_KU, OFF_KS).
template <int DK, int DV>
constexpr int keep_stage_bytes() { return 128 * DV + 2 * DK * DV; }

// Row of an M-row accumulator held by this thread, or -1: M = 128 puts row r in
// lane r; M = 64 puts row r in lane (r % 16) + 32 (r / 16).
template <int M>
__device__ __forceinline__ int acc_row(int warp, int lane) {
    if constexpr (M == 128) return 32 * warp + lane;
    else return lane < 16 ? 16 * warp + lane : -1;
}

__device__ __forceinline__ void store_row_f16x32(uint8_t *tile, int row, int ch0, const float (&v)[32]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint4 u;
        u.x = tc::pack_f16(v[8 * c + 0], v[8 * c + 1]); u.y = tc::pack_f16(v[8 * c + 2], v[8 * c + 3]);
        u.z = tc::pack_f16(v[8 * c + 4], v[8 * c + 5]); u.w = tc::pack_f16(v[8 * c + 6], v[8 * c + 7]);
        *reinterpret_cast<uint4 *>(tile + tc::sw128_off(row, ch0 + c)) = u;
    }
}

// Warp roles.  Four warpgroups (one warp per TMEM lane quarter each) plus two
// single-thread roles; hand-offs are mbarriers (arrive count 1; a warpgroup
// arrives through one thread after a named barrier).  Every wait is bounded and
// also ends as soon as any role has flagged an abort.
//   warps 0-3   converter: bf16 -> fp16 in place for the Q, K, V tiles of a stage
//   warps 4-7   side:      -W and the masked P^T from TMEM into the B operand tiles
//   warps 8-11  chain:     U'^T and the new state from TMEM into the A operand tiles
//   warps 12-15 output:    O^T from TMEM to global memory, then zero it for the next chunk
//   warp 16     MMA issuer (one thread)
//   warp 17     TMA producer (one thread)
constexpr int ST_WARPS = 18;
constexpr int ST_THREADS = ST_WARPS * 32;
constexpr int W_ISSUE = 16, W_PROD = 17;
constexpr uint32_t TM_W = 256, TM_P = 384, TM_S16 = 448;

// Pack 32 fp32 values into 16 words of fp16 pairs (element 2j in the low half).
__device__ __forceinline__ void pack32_f16(const float (&v)[32], uint32_t (&w)[16]) {
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = tc::pack_f16(v[2 * j], v[2 * j + 1]);
}

// Each stage is three buffer groups with their own load and release barriers, so
// every group is refilled as soon as its last reader is done:
//   V and Ta  -- read by U'^T(n) and W(n)            released after U'^T(n)
//   Q (+ -W)  -- read by P^T(n) and D1(n)            released after D1(n)
//   K (+ P^T) -- read by W(n), P^T(n) and D2(n)      released after D2(n)
// The barriers an epilogue warpgroup signals take one arrival per warp, so no warp
// waits for the other three before the issuer can go on.
struct StateBars {
    uint64_t fullV[2], fullQ[2], fullK[2];
    uint64_t freeV[2], freeQ[2], freeK[2];
    uint64_t wdone, pdone, d1done, d2done, drain, ku_free, ks_free;
    // per-warp arrivals (4 each) from here on
    uint64_t conv[2], w_ready, p_ready, up_ready_a, up_ready, s_ready_a, s_ready, o_free, ku_full, ks_full;
};
constexpr int BARS_ONE = 19;  // barriers before `conv` take a single arrival

// Signal `bar` once this warp's TMEM and shared-memory writes are done (a shared-memory
// writer issues fence.proxy.async first, so the tensor core sees its stores).
__device__ __forceinline__ void warp_arrive(uint64_t *bar, int lane) {
    tc::tc_fence_before();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(bar);
}

// SEG = false compiles the one-pass form only (pass 0); SEG = true also takes the segment runs.
// SAVE: the forward of the backward pass (every token's u and the state after every chunk
// instead of o).  GATED: the gated form, with the decays in `gate` ([B,H,L]).
template <int DK, int DV, typename TO, bool SEG, bool SAVE = false, bool GATED = false, bool KEEP = false>
__global__ void __launch_bounds__(ST_THREADS, 1)
    tc_state_kernel(const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_t, const __grid_constant__ CUtensorMap tmap_ku,
                    const __grid_constant__ CUtensorMap tmap_ks, const float *__restrict__ S0,
                    TO *__restrict__ o, float *__restrict__ S_final, int L, int NC,
                    float *__restrict__ segbuf, int G, int seg_chunks, int pass,
                    __half *__restrict__ u_out, __half *__restrict__ ck_out,
                    const __nv_bfloat16 *__restrict__ gate, uint8_t *ta_drop) {
    static_assert(!((SAVE || KEEP) && GATED), "the saving and keeping forwards are for the ungated form");
    using Lay = StateLayout<DK, DV, GATED>;
    constexpr uint32_t TM_S = 0, TM_O = DK, TM_U = DK + 64;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = tc::smem_u32(smem_raw);
    uint8_t *base = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
    __shared__ StateBars bars;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int abort_flag;
    // gated: per stage, l_t and e^{l_C - l_t} of the chunk's tokens and e^{l_C} (written by the
    // converter with the stage's tiles; readers wait for the stage's conversion first)
    __shared__ float gfac[GATED ? 2 * 3 * C : 1];
    auto gf = [&](int st, int which) { return gfac + (st * 3 + which) * C; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wg = warp >> 2, gtid = tid & 127;
    // ---- the run this CTA makes: head bh, chunks [n0, n1), and what it starts from and keeps.
    // pass 0: the whole sequence.  With the sequence cut into G segments of seg_chunks chunks
    // (each segment maps the state affinely, S_out = P S_in + H), pass 1 runs segment 0 from
    // S0 and, for every middle segment g, H_g (from zero) and P_g (the transition: from the
    // identity with v = 0), with no output; pass 2 runs segments 1..G-1 from their true
    // starting states, which the combine kernel chains together in between.
    int bh = blockIdx.x, n0 = 0, n1 = NC, mode = 0;  // mode 0: outputs, 1: H run, 2: P run
    const size_t DD = (size_t)DK * DV;
    const float *s0p = S0 ? S0 + (size_t)bh * DD : nullptr;
    float *sfp = S_final ? S_final + (size_t)bh * DD : nullptr;
    if (!SEG) pass = 0;
    if (pass == 1) {
        const int R = 2 * G - 3, r = blockIdx.x % R, g = (r + 1) / 2;
        bh = blockIdx.x / R;
        n0 = g * seg_chunks;
        n1 = min(NC, n0 + seg_chunks);
        float *seg = segbuf + ((size_t)bh * G + g) * 3 * DD;  // [S_in | H | P] of segment g
        if (r == 0) {
            s0p = S0 ? S0 + (size_t)bh * DD : nullptr;
            sfp = segbuf + ((size_t)bh * G + 1) * 3 * DD;  // S_in of segment 1
        } else {
            mode = (r & 1) ? 1 : 2;
            s0p = nullptr;
            sfp = seg + (size_t)mode * DD;
        }
    } else if (pass == 2) {
        const int R = G - 1, g = 1 + (int)blockIdx.x % R;
        bh = blockIdx.x / R;
        n0 = g * seg_chunks;
        n1 = min(NC, n0 + seg_chunks);
        s0p = segbuf + ((size_t)bh * G + g) * 3 * DD;
        sfp = (g == G - 1 && S_final) ? S_final + (size_t)bh * DD : nullptr;
    }
    if (!SEG) mode = 0;
    const int cnt = n1 - n0;  // chunks of this run; stage and barrier phases follow the local index
    if (tid == 0) {
        uint64_t *b = reinterpret_cast<uint64_t *>(&bars);
        for (int i = 0; i < (int)(sizeof(StateBars) / sizeof(uint64_t)); ++i)
            tc::mbar_init(b + i, i < BARS_ONE ? 1 : 4);
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
    const int vrow = acc_row<DV>(warp & 3, lane);  // state column v of this thread's TMEM lane

    // ---- a P run reads no values: its V tiles stay zero
    if (mode == 2) {
        for (int i = tid; i < 2 * Lay::VB / 16; i += ST_THREADS) {
            const int stg = i / (Lay::VB / 16), w = i - stg * (Lay::VB / 16);
            reinterpret_cast<uint4 *>(base + stg * Lay::STAGE + Lay::OFF_V)[w] = make_uint4(0u, 0u, 0u, 0u);
        }
        tc::fence_async_smem();
    }
    // ---- initial state (chain warpgroup): S^T, its fp16 copy and a zero O^T in TMEM (gated:
    // the fp32 S^T already scaled by the first chunk's e^{l_C}, which D2 adds to)
    const __nv_bfloat16 *grow = GATED ? gate + (size_t)bh * L : nullptr;  // this head's decays
    if (wg == 2) {
        float gC0 = 1.f;
        if constexpr (GATED) gC0 = expf(__shfl_sync(0xffffffffu, chunk_logdecay(grow, n0 * C, L, lane).y, 31));
#pragma unroll
        for (int cb = 0; cb < DK / 32; ++cb) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                v[j] = mode == 2 ? (cb * 32 + j == vrow ? 1.f : 0.f)
                                 : ((s0p && vrow >= 0) ? s0p[(size_t)(cb * 32 + j) * DV + vrow] : 0.f);
            float lo[16], hi[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) { lo[j] = v[j] * gC0; hi[j] = v[16 + j] * gC0; }
            tc::tmem_st16(tmem + lane_base + TM_S + cb * 32, lo);
            tc::tmem_st16(tmem + lane_base + TM_S + cb * 32 + 16, hi);
            uint32_t w[16];
            pack32_f16(v, w);
            tc::tmem_st16u(tmem + lane_base + TM_S16 + cb * 16, w);
        }
        float z[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) z[j] = 0.f;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) tc::tmem_st16(tmem + lane_base + TM_O + cb * 16, z);
        tc::tc_fence_before();
    }
    __syncthreads();
    tc::tc_fence_after();

    const long long budget = WAIT_BUDGET;
    if (warp == W_PROD) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            // The plain forward reads its tiles once, so they come in under evict-first: the
            // k and Ta tiles that the prep kernel has just read or written then stay in L2 for
            // this kernel.  The saving and keeping forwards load normally (the backward that
            // follows them reads the same tiles again).
            constexpr bool ONCE = !SAVE && !KEEP;
            const uint64_t pol = ONCE ? tc::l2_evict_first_policy() : 0ull;
            auto load3 = [&](void *dst, const CUtensorMap *m, uint64_t *b, int c0, int c1, int c2) {
                if constexpr (ONCE) tc::tma_load_3d_hint(dst, m, b, c0, c1, c2, pol);
                else tc::tma_load_3d(dst, m, b, c0, c1, c2);
            };
            // A run over the whole sequence that only outputs is the last reader of its Ta tiles:
            // with ta_drop set (the tiles' base, 128-byte aligned), each tile's lines leave L2
            // unwritten once its stage is released, which saves their write-back to HBM.
            auto drop_ta = [&](int n) {
                if constexpr (ONCE && !SEG) {
                    if (ta_drop) {
                        const uint8_t *t = ta_drop + (size_t)(bh * NC + n) * (C * C * 2);
                        for (int l = 0; l < C * C * 2 / 128; ++l) tc::l2_discard_line(t + 128 * l);
                    }
                }
            };
            int last[2] = {-1, -1};
            for (int i = 0; i < cnt; ++i) {
                const int n = n0 + i, st = i & 1;
                const uint32_t par = ((i - 2) >> 1) & 1;
                uint8_t *stg = base + st * Lay::STAGE;
                if (i >= 2 && !tc::mbar_wait_or_abort(&bars.freeV[st], par, &abort_flag, budget)) break;
                tc::mbar_expect_tx(&bars.fullV[st], (mode == 2 ? 0 : Lay::VB) + Lay::TB);
                if (mode != 2) {
#pragma unroll
                    for (int j = 0; j < DV / 64; ++j)
                        load3(stg + Lay::OFF_V + j * 8192, &tmap_v, &bars.fullV[st], j * 64, n * C, bh);
                }
                if constexpr (ONCE) tc::tma_load_2d_hint(stg + Lay::OFF_T, &tmap_t, &bars.fullV[st], 0, (bh * NC + n) * C, pol);
                else tc::tma_load_2d(stg + Lay::OFF_T, &tmap_t, &bars.fullV[st], 0, (bh * NC + n) * C);
                if (i >= 2 && !tc::mbar_wait_or_abort(&bars.freeQ[st], par, &abort_flag, budget)) break;
                tc::mbar_expect_tx(&bars.fullQ[st], SAVE ? 0 : DK * 128);  // the saving forward reads no q
                if constexpr (!SAVE) {
#pragma unroll
                    for (int j = 0; j < DK / 64; ++j)
                        load3(stg + Lay::OFF_QW + j * Lay::QW_SLAB, &tmap_q, &bars.fullQ[st], j * 64, n * C, bh);
                }
                if (i >= 2 && !tc::mbar_wait_or_abort(&bars.freeK[st], par, &abort_flag, budget)) break;
                tc::mbar_expect_tx(&bars.fullK[st], DK * 128);
#pragma unroll
                for (int j = 0; j < DK / 64; ++j)
                    load3(stg + Lay::OFF_KP + j * 8192, &tmap_k, &bars.fullK[st], j * 64, n * C, bh);
                last[st] = i;
                if (i >= 2) drop_ta(n - 2);  // its stage was released above
            }
            if (!abort_flag) {  // the last two chunks' tiles, once their stages are released
                for (int j = cnt < 2 ? 0 : cnt - 2; j < cnt; ++j) {
                    if (!(ONCE && !SEG) || !ta_drop) break;
                    if (!tc::mbar_wait_or_abort(&bars.freeV[j & 1], (j >> 1) & 1, &abort_flag, budget)) break;
                    drop_ta(n0 + j);
                }
            }
            if (abort_flag) {  // let this CTA's own copies land before it exits (bounded)
                for (int st = 0; st < 2; ++st) {
                    if (last[st] < 0) continue;
                    const uint32_t par = (last[st] >> 1) & 1;
                    tc::mbar_wait(&bars.fullV[st], par, budget / 8);
                    tc::mbar_wait(&bars.fullQ[st], par, budget / 8);
                    tc::mbar_wait(&bars.fullK[st], par, budget / 8);
                }
            }
        }
    } else if (warp == W_ISSUE) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id_u = tc::idesc_f16(DV, 64, true, false);
            constexpr uint32_t id_w = tc::idesc_f16(64, DK, false, true);
            constexpr uint32_t id_p = tc::idesc_f16(64, 64, false, false);
            constexpr uint32_t id_d1 = tc::idesc_f16(DV, 128, false, false);
            constexpr uint32_t id_d2 = tc::idesc_f16(DV, DK + 64, false, true);
            constexpr uint32_t id_d2s = tc::idesc_f16(DV, DK, false, true);  // gated: S^T += U''^T K
            constexpr uint32_t id_d2o = tc::idesc_f16(DV, 64, false, true);  // gated: O^T += U'^T P^T
            constexpr uint32_t id_d1s = tc::idesc_f16(DV, 64, false, false);  // saving: U'^T += S^T (-W)^T
            auto stage_addr = [&](int n) { return sb + (n & 1) * Lay::STAGE; };
            // U'^T := V^T Ta^T (prefill of the U' accumulator)
            auto issue_u = [&](int n) {
                const uint32_t stg = stage_addr(n);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_U, tc::sdesc(stg + Lay::OFF_V + kk * 2048, 8192, 1024),
                                 tc::sdesc(stg + Lay::OFF_T + kk * 32, 16, 1024), id_u, kk > 0);
                tc::mma_commit(&bars.freeV[n & 1]);  // V and Ta of this stage are no longer read
            };
            // W = Ta K (its own TMEM columns; the side group stores -W as a B operand); gated:
            // W = Ta diag(e^{l}) K, from the converter's scaled copy of K
            auto issue_w = [&](int n) {
                const uint32_t stg = stage_addr(n);
                const uint32_t kw = stg + (GATED ? Lay::OFF_KH : Lay::OFF_KP);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tmem + TM_W, tc::sdesc(stg + Lay::OFF_T + kk * 32, 16, 1024),
                                 tc::sdesc(kw + kk * 2048, 8192, 1024), id_w, kk > 0);
                tc::mma_commit(&bars.wdone);
            };
            // P^T = K Q^T (its own TMEM columns; the side group stores the masked P^T); gated:
            // Q from the converter's unscaled copy (the QW slabs hold the scaled one)
            auto issue_p = [&](int n) {
                const uint32_t stg = stage_addr(n);
                const uint32_t qb = stg + (GATED ? Lay::OFF_QP : Lay::OFF_QW), kp = stg + Lay::OFF_KP;
                constexpr int QSTRIDE = GATED ? 8192 : Lay::QW_SLAB;
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk)
                    tc::mma_bf16(tmem + TM_P, tc::sdesc(kp + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                                 tc::sdesc(qb + (kk >> 2) * QSTRIDE + (kk & 3) * 32, 16, 1024),
                                 id_p, kk > 0);
                tc::mma_commit(&bars.pdone);
            };
            // Tensor-pipe order per chunk: D1(n), W(n+1), D2(n), P^T(n+1), U'^T(n+1), so the
            // next chunk's products run while this chunk's epilogues do.
            bool issued_any = false;
            bool ok = tc::mbar_wait_or_abort(&bars.conv[0], 0, &abort_flag, budget);
            if (ok) {
                tc::tc_fence_after();
                issued_any = true;
                issue_w(0);
                if constexpr (!SAVE) issue_p(0);  // the saving forward computes no output
                issue_u(0);
            }
            for (int n = 0; ok && n < cnt; ++n) {  // n: local chunk index
                const int st = n & 1;
                const uint32_t stg = stage_addr(n);
                const uint32_t qw = stg + Lay::OFF_QW, kp = stg + Lay::OFF_KP;
                // D1: [O^T | U'^T] += S^T [Q | -W]^T   (A = fp16 S^T in TMEM)
                // the first 64 rows of S^T are packed before the rest: start on them
                if (!tc::mbar_wait_or_abort(&bars.w_ready, n & 1, &abort_flag, budget)) break;
                if (!SAVE && n > 0 && !tc::mbar_wait_or_abort(&bars.o_free, (n - 1) & 1, &abort_flag, budget)) break;
                if (n > 0 && !tc::mbar_wait_or_abort(&bars.s_ready_a, (n - 1) & 1, &abort_flag, budget)) break;
                tc::tc_fence_after();
                bool ok2 = true;
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    if (kk == 4 && n > 0) {
                        ok2 = tc::mbar_wait_or_abort(&bars.s_ready, (n - 1) & 1, &abort_flag, budget);
                        if (!ok2) break;
                        tc::tc_fence_after();
                    }
                    if constexpr (SAVE)  // U'^T only: the -W rows of the QW slabs
                        tc::mma_tmem_a(tmem + TM_U, tmem + TM_S16 + kk * 8,
                                       tc::sdesc(qw + 8192 + (kk >> 2) * Lay::QW_SLAB + (kk & 3) * 32, 16, 1024),
                                       id_d1s, 1u);
                    else
                        tc::mma_tmem_a(tmem + TM_O, tmem + TM_S16 + kk * 8,
                                       tc::sdesc(qw + (kk >> 2) * Lay::QW_SLAB + (kk & 3) * 32, 16, 1024),
                                       id_d1, 1u);
                }
                if (!ok2) break;
                tc::mma_commit(&bars.d1done);
                tc::mma_commit(&bars.freeQ[st]);
                if (n + 1 < cnt) {  // W of the next chunk (its TMEM was read out before D1(n))
                    // shared-memory handshake only: the fence before D1(n) already orders
                    // this MMA after the side group's TMEM reads of W(n)
                    if (!tc::mbar_wait_or_abort(&bars.conv[(n + 1) & 1], ((n + 1) >> 1) & 1, &abort_flag, budget)) break;
                    issue_w(n + 1);
                }
                // D2: [S^T | O^T] += U'^T [K | P^T]   (A = fp16 U'^T in TMEM)
                // U' is packed in two halves of 32 tokens: start on the first
                if (!SAVE && !tc::mbar_wait_or_abort(&bars.p_ready, n & 1, &abort_flag, budget)) break;
                if (!tc::mbar_wait_or_abort(&bars.up_ready_a, n & 1, &abort_flag, budget)) break;
                tc::tc_fence_after();
                if constexpr (!GATED) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        if (kk == 2) {
                            ok2 = tc::mbar_wait_or_abort(&bars.up_ready, n & 1, &abort_flag, budget);
                            if (!ok2) break;
                            tc::tc_fence_after();
                        }
                        // the saving forward: the state update alone (N = dk), no output
                        tc::mma_tmem_a(tmem + TM_S, tmem + TM_U + kk * 8, tc::sdesc(kp + kk * 2048, 8192, 1024),
                                       SAVE ? id_d2s : id_d2, 1u);
                    }
                } else {
                    // gated: O^T += U'^T P^T with both factors as fp16 hi + lo (the lo x lo term
                    // dropped): U' hi over TM_U's first 32 columns, U' lo where P^T's accumulator
                    // was; then S^T += U''^T K with U'' = diag(e^{l_C - l}) U' (TM_U's next 32)
                    const uint32_t ph = sb + Lay::OFF_PH, pl = sb + Lay::OFF_PL;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        if (kk == 2) {
                            ok2 = tc::mbar_wait_or_abort(&bars.up_ready, n & 1, &abort_flag, budget);
                            if (!ok2) break;
                            tc::tc_fence_after();
                        }
                        tc::mma_tmem_a(tmem + TM_O, tmem + TM_U + kk * 8, tc::sdesc(ph + kk * 2048, 8192, 1024),
                                       id_d2o, 1u);
                    }
                    if (ok2) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma_tmem_a(tmem + TM_O, tmem + TM_U + kk * 8, tc::sdesc(pl + kk * 2048, 8192, 1024),
                                           id_d2o, 1u);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma_tmem_a(tmem + TM_O, tmem + TM_P + kk * 8, tc::sdesc(ph + kk * 2048, 8192, 1024),
                                           id_d2o, 1u);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma_tmem_a(tmem + TM_S, tmem + TM_U + 32 + kk * 8,
                                           tc::sdesc(kp + kk * 2048, 8192, 1024), id_d2s, 1u);
                    }
                }
                if (!ok2) break;
                tc::mma_commit(&bars.d2done);
                tc::mma_commit(&bars.freeK[st]);
                if (n + 1 < cnt) {  // P^T and the U' prefill of the next chunk
                    if constexpr (!SAVE) issue_p(n + 1);
                    issue_u(n + 1);
                }
            }
            if (abort_flag && issued_any) {  // wait (bounded) for every issued MMA to finish
                tc::mma_commit(&bars.drain);
                tc::mbar_wait(&bars.drain, 0, budget / 4);
            }
        }
    } else if (wg == 0) {
        // ---------------------------------------------------------- converter
        auto cvt = [](uint4 *t) {
            uint4 u = *t;
            u.x = tc::bf16x2_to_f16x2(u.x); u.y = tc::bf16x2_to_f16x2(u.y);
            u.z = tc::bf16x2_to_f16x2(u.z); u.w = tc::bf16x2_to_f16x2(u.w);
            *t = u;
        };
        // gated: also the unscaled fp16 q (P^T's B) and k scaled by e^{l_t} (W's B); the QW
        // slabs get q scaled by e^{l_t} (D1's B), K's tile stays unscaled.  Row r of a tile's
        // 64-column slab is its 16-byte pieces 8 r .. 8 r + 7 (the swizzle stays within a row).
        auto cvt2 = [](const uint4 *src, uint4 *plain, uint4 *scaled, float f) {
            const uint4 u = *src;
            *plain = make_uint4(tc::bf16x2_to_f16x2(u.x), tc::bf16x2_to_f16x2(u.y),
                                tc::bf16x2_to_f16x2(u.z), tc::bf16x2_to_f16x2(u.w));
            *scaled = make_uint4(tc::bf16x2_to_f16x2_scaled(u.x, f), tc::bf16x2_to_f16x2_scaled(u.y, f),
                                 tc::bf16x2_to_f16x2_scaled(u.z, f), tc::bf16x2_to_f16x2_scaled(u.w, f));
        };
        for (int n = 0; n < cnt; ++n) {  // n: local chunk index
            const int st = n & 1;
            const uint32_t par = (n >> 1) & 1;
            uint8_t *stg = base + st * Lay::STAGE;
            float2 lp = make_float2(0.f, 0.f);  // gated: l_t of this chunk's token pairs
            if constexpr (GATED) lp = chunk_logdecay(grow, (n0 + n) * C, L, lane);
            if (!tc::mbar_wait_or_abort(&bars.fullV[st], par, &abort_flag, budget)) break;
            if (mode != 2) {
                uint4 *tv = reinterpret_cast<uint4 *>(stg + Lay::OFF_V);
#pragma unroll
                for (int i = gtid; i < Lay::VB / 16; i += 128) cvt(tv + i);
            }
            if (!tc::mbar_wait_or_abort(&bars.fullQ[st], par, &abort_flag, budget)) break;
#pragma unroll
            for (int j = 0; j < (SAVE ? 0 : DK / 64); ++j) {  // Q: the first 8 KB of each QW slab
                uint4 *tq = reinterpret_cast<uint4 *>(stg + Lay::OFF_QW + j * Lay::QW_SLAB);
                if constexpr (GATED) {
                    uint4 *tqp = reinterpret_cast<uint4 *>(stg + Lay::OFF_QP + j * 8192);
#pragma unroll
                    for (int i = gtid; i < 512; i += 128)
                        cvt2(tq + i, tqp + i, tq + i, expf(logdecay_at(lp, i >> 3)));
                } else {
#pragma unroll
                    for (int i = gtid; i < 512; i += 128) cvt(tq + i);
                }
            }
            if (!tc::mbar_wait_or_abort(&bars.fullK[st], par, &abort_flag, budget)) break;
            {
                uint4 *tk = reinterpret_cast<uint4 *>(stg + Lay::OFF_KP);
                if constexpr (GATED) {
                    uint4 *tkh = reinterpret_cast<uint4 *>(stg + Lay::OFF_KH);
#pragma unroll
                    for (int i = gtid; i < (DK / 64) * 512; i += 128)
                        cvt2(tk + i, tk + i, tkh + i, expf(logdecay_at(lp, (i >> 3) & 63)));
                    // the stage's decay factors: its previous chunk's readers finished before
                    // D2 of that chunk, which the K tile's reload waited for
                    if (gtid < 32) {
                        const float lC = __shfl_sync(0xffffffffu, lp.y, 31);
                        gf(st, 0)[2 * lane] = lp.x;
                        gf(st, 0)[2 * lane + 1] = lp.y;
                        gf(st, 1)[2 * lane] = expf(lC - lp.x);
                        gf(st, 1)[2 * lane + 1] = expf(lC - lp.y);
                        if (lane == 0) gf(st, 2)[0] = expf(lC);
                    }
                } else {
#pragma unroll
                    for (int i = gtid; i < (DK / 64) * 512; i += 128) cvt(tk + i);
                }
            }
            tc::fence_async_smem();
            warp_arrive(&bars.conv[st], lane);
        }
    } else if (wg == 1) {
        // ---------------------------------------------------------- side epilogue
        const int crow = acc_row<64>(warp & 3, lane);  // token row of the M = 64 accumulators
        for (int n = 0; n < cnt; ++n) {  // n: local chunk index
            const int st = n & 1;
            uint8_t *stg = base + st * Lay::STAGE;
            if (!tc::mbar_wait_or_abort(&bars.wdone, n & 1, &abort_flag, budget)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < DK / 32; ++cb) {  // -W rows into rows 64.. of the QW slabs
                float v[32];
                tc::tmem_ld32(tmem + lane_base + TM_W + cb * 32, v);
                if (crow >= 0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = -v[j];
                    store_row_f16x32(stg + Lay::OFF_QW + (cb >> 1) * Lay::QW_SLAB, 64 + crow, (cb & 1) * 4, v);
                }
            }
            tc::fence_async_smem();
            warp_arrive(&bars.w_ready, lane);

            if constexpr (SAVE) continue;  // the saving forward computes no output: no P^T
            if (!tc::mbar_wait_or_abort(&bars.pdone, n & 1, &abort_flag, budget)) break;
            // gated: the chunk's l_t (the converter wrote them with the stage's tiles)
            if (GATED && !tc::mbar_wait_or_abort(&bars.conv[st], (n >> 1) & 1, &abort_flag, budget)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {  // masked P^T (row c_in, column c_out >= c_in)
                float v[32];
                tc::tmem_ld32(tmem + lane_base + TM_P + cb * 32, v);
                if (crow >= 0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (cb * 32 + j < crow) v[j] = 0.f;
                    if constexpr (GATED) {  // entry (c_in, c_out) weighted by e^{l_out - l_in} <= 1
                        const float *lt = gf(st, 0);
                        const float lin = lt[crow];
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] *= __expf(fminf(lt[cb * 32 + j] - lin, 0.f));  // as in prep
                        store_row_f16x32(base + Lay::OFF_PH, crow, cb * 4, v);
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] -= __half2float(__float2half_rn(v[j]));
                        store_row_f16x32(base + Lay::OFF_PL, crow, cb * 4, v);
                    } else {
                        store_row_f16x32(stg + Lay::OFF_KP + (DK / 64) * 8192, crow, cb * 4, v);
                    }
                }
            }
            tc::fence_async_smem();
            warp_arrive(&bars.p_ready, lane);
        }
    } else if (wg == 2) {
        // ---------------------------------------------------------- chain epilogue
        bool done_all = true;
        for (int n = 0; n < cnt; ++n) {  // n: local chunk index
            // gated: the chunk's e^{l_C - l_t} (the converter wrote them with the stage's tiles)
            if (GATED && !tc::mbar_wait_or_abort(&bars.conv[n & 1], (n >> 1) & 1, &abort_flag, budget)) {
                done_all = false;
                break;
            }
            if (!tc::mbar_wait_or_abort(&bars.d1done, n & 1, &abort_flag, budget)) { done_all = false; break; }
            // gated: U'^T's fp16 remainder goes where P^T's accumulator was, once the side group
            // has read it out
            if (GATED && !tc::mbar_wait_or_abort(&bars.p_ready, n & 1, &abort_flag, budget)) {
                done_all = false;
                break;
            }
            tc::tc_fence_after();
            uint32_t wsc[16];  // gated: the first half's U'' = e^{l_C - l_t} U', until its columns are read
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // U'^T to fp16 in place, 32 tokens at a time
                float u[32];
                tc::tmem_ld32(tmem + lane_base + TM_U + h * 32, u);
                uint32_t w[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) w[j] = tc::pack_f16(u[2 * j], u[2 * j + 1]);
                tc::tmem_st16u(tmem + lane_base + TM_U + h * 16, w);  // over fp32 columns already read
                if constexpr (GATED) {
                    // the output's U' as hi + lo (the remainder after fp16 rounding, to 22 bits)
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        w[j] = tc::pack_f16(u[2 * j] - __half2float(__float2half_rn(u[2 * j])),
                                            u[2 * j + 1] - __half2float(__float2half_rn(u[2 * j + 1])));
                    tc::tmem_st16u(tmem + lane_base + TM_P + h * 16, w);
                    // U''^T after both halves' fp32 columns [32, 64) are read
                    const float *e = gf(n & 1, 1) + h * 32;
#pragma unroll
                    for (int j = 0; j < 16; ++j) w[j] = tc::pack_f16(u[2 * j] * e[2 * j], u[2 * j + 1] * e[2 * j + 1]);
                    if (h == 0) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) wsc[j] = w[j];
                    } else {
                        tc::tmem_st16u(tmem + lane_base + TM_U + 32, wsc);
                        tc::tmem_st16u(tmem + lane_base + TM_U + 48, w);
                    }
                }
                warp_arrive(h == 0 ? &bars.up_ready_a : &bars.up_ready, lane);
                if constexpr (SAVE || KEEP) {
                    if (u_out && mode == 0) {
                        // u_t = a_t r_t of every token, for the backward (also by the forward that
                        // writes o, when asked to keep it): fp16 into the [64][dv] tile, column
                        // vrow, once the tile's previous store has read it; stored by TMA
                        if (h == 0 && n > 0) {
                            if (gtid == 0) {
                                tc::bulk_wait_read1();
                                tc::mbar_arrive(&bars.ku_free);
                            }
                            if (!tc::mbar_wait_or_abort(&bars.ku_free, (n - 1) & 1, &abort_flag, budget)) {
                                done_all = false;
                                break;
                            }
                        }
                        if (vrow >= 0) {
                            uint8_t *tile = base + Lay::OFF_KU + (vrow >> 6) * 8192 + 2 * (vrow & 7);
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                *reinterpret_cast<__half *>(tile + tc::sw128_off(h * 32 + j, (vrow & 63) >> 3)) =
                                    __float2half_rn(u[j]);
                        }
                    }
                }
            }
            if constexpr (SAVE || KEEP) {
                if (!done_all) break;
                if (u_out && mode == 0) {  // rows past L are not stored
                    tc::fence_async_smem();
                    warp_arrive(&bars.ku_full, lane);
                    if (gtid == 0) {
                        if (!tc::mbar_wait_or_abort(&bars.ku_full, n & 1, &abort_flag, budget)) {
                            done_all = false;
                            break;
                        }
                        for (int j = 0; j < DV / 64; ++j)
                            tc::tma_store_3d(&tmap_ku, base + Lay::OFF_KU + j * 8192, j * 64, (n0 + n) * C, bh);
                        tc::bulk_commit();
                    }
                }
            }

            if (!tc::mbar_wait_or_abort(&bars.d2done, n & 1, &abort_flag, budget)) { done_all = false; break; }
            tc::tc_fence_after();
            float gCn = 1.f;  // gated: the next chunk's e^{l_C}, applied to the fp32 state for its D2
            if (GATED && n + 1 < cnt) {
                if (!tc::mbar_wait_or_abort(&bars.conv[(n + 1) & 1], ((n + 1) >> 1) & 1, &abort_flag, budget)) {
                    done_all = false;
                    break;
                }
                gCn = gf((n + 1) & 1, 2)[0];
            }
            if constexpr (!GATED) {
#pragma unroll
                for (int cb = 0; cb < DK / 64; ++cb) {  // S^T to fp16, 64 rows of S at a time
                    if (n + 1 < cnt) {
                        float v[64];
                        tc::tmem_ld64(tmem + lane_base + TM_S + cb * 64, v);
                        uint32_t w[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) w[j] = tc::pack_f16(v[2 * j], v[2 * j + 1]);
                        tc::tmem_st32u(tmem + lane_base + TM_S16 + cb * 32, w);
                    }
                    if (cb == 0) warp_arrive(&bars.s_ready_a, lane);
                }
            } else {
                // 32 rows of S at a time: the fp16 copy of S for D1, then the fp32 S scaled by
                // the next chunk's decay for its D2
#pragma unroll
                for (int p = 0; p < DK / 32; ++p) {
                    if (n + 1 < cnt) {
                        float v[32];
                        tc::tmem_ld32(tmem + lane_base + TM_S + p * 32, v);
                        uint32_t w[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) w[j] = tc::pack_f16(v[2 * j], v[2 * j + 1]);
                        tc::tmem_st16u(tmem + lane_base + TM_S16 + p * 16, w);
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            float x[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j) x[j] = v[16 * h2 + j] * gCn;
                            tc::tmem_st16(tmem + lane_base + TM_S + p * 32 + 16 * h2, x);
                        }
                    }
                    if (p == 1) warp_arrive(&bars.s_ready_a, lane);
                }
            }
            warp_arrive(&bars.s_ready, lane);
            if ((SAVE || KEEP) && ck_out && mode == 0) {
                // the state after this chunk, for the backward: S^T stays in TMEM until D2 of the
                // next chunk, which waits for this warpgroup's next U' hand-over.  The TMEM load is
                // warp-collective: every lane takes it, the lanes that hold a state column write
                // it, fp16, into the [dk][dv] tile (column vrow) once the tile's previous store has
                // read it; stored by TMA into [B*H][NC][dk][dv]
                if (n > 0) {
                    if (gtid == 0) {
                        tc::bulk_wait_read1();
                        tc::mbar_arrive(&bars.ks_free);
                    }
                    if (!tc::mbar_wait_or_abort(&bars.ks_free, (n - 1) & 1, &abort_flag, budget)) {
                        done_all = false;
                        break;
                    }
                }
                uint8_t *tile = base + Lay::OFF_KS + (vrow >= 0 ? (vrow >> 6) * (DK * 128) + 2 * (vrow & 7) : 0);
#pragma unroll 1
                for (int cb = 0; cb < DK / 16; ++cb) {
                    float v[16];
                    tc::tmem_ld16(tmem + lane_base + TM_S + cb * 16, v);
                    if (vrow >= 0) {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            *reinterpret_cast<__half *>(tile + tc::sw128_off(cb * 16 + j, (vrow & 63) >> 3)) =
                                __float2half_rn(v[j]);
                    }
                }
                tc::fence_async_smem();
                warp_arrive(&bars.ks_full, lane);
                if (gtid == 0) {
                    if (!tc::mbar_wait_or_abort(&bars.ks_full, n & 1, &abort_flag, budget)) {
                        done_all = false;
                        break;
                    }
                    for (int j = 0; j < DV / 64; ++j)
                        tc::tma_store_2d(&tmap_ks, base + Lay::OFF_KS + j * (DK * 128), j * 64,
                                         ((int)bh * NC + n0 + n) * DK);
                    tc::bulk_commit();
                }
            }
        }
        if constexpr (SAVE || KEEP)
            if (gtid == 0) tc::bulk_wait_all();  // the kept tiles' stores are done
        if (done_all && sfp) {
#pragma unroll
            for (int cb = 0; cb < DK / 16; ++cb) {
                float v[16];
                tc::tmem_ld16(tmem + lane_base + TM_S + cb * 16, v);
                if (vrow >= 0) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        sfp[(size_t)(cb * 16 + j) * DV + vrow] = v[j];
                }
            }
        }
    } else if (wg == 3) {
        // ---------------------------------------------------------- output
        float z[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) z[j] = 0.f;
        for (int n = 0; n < (SAVE ? 0 : cnt); ++n) {  // n: local chunk index (the saving forward writes no o)
            const int c0 = (n0 + n) * C;
            if (!tc::mbar_wait_or_abort(&bars.d2done, n & 1, &abort_flag, budget)) break;
            tc::tc_fence_after();
            const int cl = min(C, L - c0);
            float v[64];
            tc::tmem_ld64(tmem + lane_base + TM_O, v);
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) tc::tmem_st16(tmem + lane_base + TM_O + cb * 16, z);
            warp_arrive(&bars.o_free, lane);  // TMEM O is zero again: D1(n+1) may run
            if (mode == 0 && vrow >= 0 && (!SAVE || o)) {  // the saving forward writes no o
                TO *dst = o + ((size_t)bh * L + c0) * DV + vrow;
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (j < cl) dst[(size_t)j * DV] = from_f32<TO>(v[j]);
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (tid == 0 && abort_flag) record_error(2u);
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}


// ------------------------------------------------------------------ bounded-wait self-test
// One thread waits on an mbarrier that nothing arrives on, for at most `budget` cycles, then
// records a timeout in the device error word the way the kernels above do and returns: the
// test of that path, without a fault or a hang (nothing else is in flight in this CTA).
__global__ void selftest_wait_kernel(long long budget) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
        if (!tc::mbar_wait(&bar, 0, budget)) record_error(4u);
    }
}

// ------------------------------------------------------------------ segment chaining
// Each sequence segment maps the state affinely, S_out = P S_in + H (P is the product of
// the segment's transitions I - K^T W, H the segment's state from zero).  This chains
// S_in(g+1) = P_g S_in(g) + H_g for g = 1..G-2 in fp32, one 16-column block of the state
// per CTA (the state's columns evolve independently), one state row per thread: the
// thread's row of P_g comes straight from global memory with all its loads in flight.
template <int D>
__global__ void __launch_bounds__(D) seg_combine_kernel(float *__restrict__ segbuf, int G) {
    __shared__ __align__(16) float X[D][16];  // the running S_in block
    constexpr int NB = D / 16;
    const int cbk = blockIdx.x % NB, bh = blockIdx.x / NB, t = threadIdx.x;
    const size_t DD = (size_t)D * D;
    float *seg = segbuf + (size_t)bh * G * 3 * DD;  // per segment: [S_in | H | P]
    {
        const float4 *src = reinterpret_cast<const float4 *>(seg + 3 * DD + (size_t)t * D + cbk * 16);
#pragma unroll
        for (int c = 0; c < 4; ++c) reinterpret_cast<float4 *>(X[t])[c] = src[c];
    }
    for (int g = 1; g + 1 < G; ++g) {
        const float4 *prow = reinterpret_cast<const float4 *>(seg + ((size_t)g * 3 + 2) * DD + (size_t)t * D);
        const float4 *hrow = reinterpret_cast<const float4 *>(seg + ((size_t)g * 3 + 1) * DD + (size_t)t * D + cbk * 16);
        float4 p[D / 4];
#pragma unroll
        for (int m = 0; m < D / 4; ++m) p[m] = prow[m];
        float y[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float4 h = hrow[c];
            y[4 * c] = h.x; y[4 * c + 1] = h.y; y[4 * c + 2] = h.z; y[4 * c + 3] = h.w;
        }
        __syncthreads();  // X holds S_in(g)
#pragma unroll
        for (int m4 = 0; m4 < D / 4; ++m4) {
            const float pm[4] = {p[m4].x, p[m4].y, p[m4].z, p[m4].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float4 *xr = reinterpret_cast<const float4 *>(X[4 * m4 + e]);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 xv = xr[c];
                    y[4 * c] = fmaf(pm[e], xv.x, y[4 * c]);
                    y[4 * c + 1] = fmaf(pm[e], xv.y, y[4 * c + 1]);
                    y[4 * c + 2] = fmaf(pm[e], xv.z, y[4 * c + 2]);
                    y[4 * c + 3] = fmaf(pm[e], xv.w, y[4 * c + 3]);
                }
            }
        }
        __syncthreads();  // every row has read X
        float4 *dst = reinterpret_cast<float4 *>(seg + (size_t)(g + 1) * 3 * DD + (size_t)t * D + cbk * 16);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float4 v = make_float4(y[4 * c], y[4 * c + 1], y[4 * c + 2], y[4 * c + 3]);
            reinterpret_cast<float4 *>(X[t])[c] = v;
            dst[c] = v;
        }
    }
}

// ------------------------------------------------------------------ host side
bool make_map_3d(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint32_t b0, uint32_t b1) {
    return tmap::make_3d(m, ptr, d0, d1, d2, b0, b1);
}
bool make_map_2d(CUtensorMap *m, const void *ptr, uint64_t d0, uint64_t d1, uint32_t b0,
                 uint32_t b1, CUtensorMapDataType dt) {
    return tmap::make_2d(m, ptr, d0, d1, b0, b1, dt);
}

template <int DK>
int prep_smem_bytes() {
    return prep::Smem::bytes<DK>() + 1024;
}

// Sequence segments: with few heads and a long sequence, the sequence is cut into G
// segments that run in parallel (pass 1: segment 0 plus each middle segment's H and P;
// pass 2: segments 1..G-1 from their chained starting states).  Pass 1 takes BH (2G - 3)
// CTAs, so G grows while that fits the SMs, up to SEG_MAX, and every segment keeps at
// least 16 chunks.  The workspace reserves SEG_MAX segments' state whenever the sizes
// allow segments (dk == dv, at least 48 chunks, at most 48 heads).
constexpr int SEG_MAX = 8;
bool seg_sizes_ok(long long BH, int NC, int dk, int dv) { return dk == dv && NC >= 48 && BH <= 48; }
int seg_count(long long BH, int NC, int dk, int dv, int nsm) {
    if (!seg_sizes_ok(BH, NC, dk, dv)) return 1;
    long long G = ((long long)nsm + 3 * BH) / (2 * BH);
    G = G < SEG_MAX ? G : SEG_MAX;
    G = G < NC / 16 ? G : NC / 16;
    return G >= 3 ? (int)G : 1;
}
size_t ta_bytes(size_t total) { return (total * C * C * sizeof(__half) + 255) / 256 * 256; }
// What a launch needs to know about the current device, worked out once per device
// and kernel instantiation (the kernels' shared-memory attributes are set then too),
// so that a call costs the tensor-map encodings and the two launches and nothing more.
struct TcDevInfo {
    int nsm = 0;
    int prep_grid = 0;  // CTAs of the prep kernel: every SM, as many as fit by shared memory
    cudaError_t err = cudaSuccess;
};

template <int DK, int DV, typename TO>
TcDevInfo tc_dev_info() {
    constexpr int MAXDEV = 64;
    static TcDevInfo info[MAXDEV];
    static std::atomic<bool> done[MAXDEV];
    static std::mutex mu;
    int dev = 0;
    TcDevInfo d;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAXDEV) {
        d.err = cudaErrorInvalidDevice;
        return d;
    }
    if (done[dev].load(std::memory_order_acquire)) return info[dev];
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev].load(std::memory_order_relaxed)) return info[dev];
    int nsm = 0, smem_sm = 0;
    const int psm = prep_smem_bytes<DK>();
    d.err = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (d.err == cudaSuccess)
        d.err = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (d.err == cudaSuccess)
        d.err = cudaFuncSetAttribute(tc_prep_kernel<DK, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, psm);
    if (d.err == cudaSuccess)
        d.err = cudaFuncSetAttribute(tc_prep_kernel<DK, false>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (d.err == cudaSuccess)
        d.err = cudaFuncSetAttribute(tc_state_kernel<DK, DV, TO, false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, StateLayout<DK, DV>::SMEM);
    if (d.err == cudaSuccess && DK == DV)
        d.err = cudaFuncSetAttribute(tc_state_kernel<DK, DV, TO, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, StateLayout<DK, DV>::SMEM);
    constexpr int KSMEM = StateLayout<DK, DV>::SMEM + keep_stage_bytes<DK, DV>();
    if constexpr (std::is_same<TO, float>::value) {  // the saving forward of the backward
        if (d.err == cudaSuccess)
            d.err = cudaFuncSetAttribute(tc_state_kernel<DK, DV, TO, false, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, KSMEM);
        if (d.err == cudaSuccess && DK == DV)
            d.err = cudaFuncSetAttribute(tc_state_kernel<DK, DV, TO, true, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, KSMEM);
    }
    // the forward that writes o and keeps u and the chunk states
    if (d.err == cudaSuccess)
        d.err = cudaFuncSetAttribute(tc_state_kernel<DK, DV, TO, false, false, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, KSMEM);
    if (d.err == cudaSuccess && DK == DV)
        d.err = cudaFuncSetAttribute(tc_state_kernel<DK, DV, TO, true, false, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, KSMEM);
    constexpr int GSMEM = StateLayout<DK, DV, true>::SMEM;  // the gated form
    if (d.err == cudaSuccess)
        d.err = cudaFuncSetAttribute(tc_prep_kernel<DK, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, psm);
    if (d.err == cudaSuccess)
        d.err = cudaFuncSetAttribute(tc_prep_kernel<DK, true>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (d.err == cudaSuccess)
        d.err = cudaFuncSetAttribute(tc_state_kernel<DK, DV, TO, false, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, GSMEM);
    if (d.err == cudaSuccess && DK == DV)
        d.err = cudaFuncSetAttribute(tc_state_kernel<DK, DV, TO, true, false, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, GSMEM);
    if (d.err != cudaSuccess) return d;
    d.nsm = nsm;
    int per_sm = smem_sm / (psm + 1024);  // 1 KiB per CTA is reserved by the system
    per_sm = per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm);
    d.prep_grid = nsm * per_sm;
    info[dev] = d;
    done[dev].store(true, std::memory_order_release);
    return d;
}

// The prep kernel, then the state kernel: one CTA per head, or the segment passes.  GATED:
// the gated form, with the decays in g.
template <int DK, int DV, typename TO, bool SAVE, bool GATED, bool KEEP = false>
cudaError_t launch_tc_t(const void *q, const void *k, const void *v, const void *beta,
                        const float *S0, void *o, float *S_final, int B, int H, int L, bool euler,
                        void *ws, cudaStream_t s, __half *u_out, __half *ck_out, bool allow_seg,
                        const void *g) {
    const int BH = B * H, NC = (L + C - 1) / C, total = BH * NC;
    const TcDevInfo di = tc_dev_info<DK, DV, TO>();
    if (di.err != cudaSuccess) return di.err;
    CUtensorMap mq, mk, mv, mt;
    if (!make_map_3d(&mq, q, DK, L, BH, 64, C) || !make_map_3d(&mk, k, DK, L, BH, 64, C) ||
        !make_map_3d(&mv, v, DV, L, BH, 64, C) ||
        !make_map_2d(&mt, ws, C, (uint64_t)total * C, 64, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return cudaErrorInvalidValue;
    const __nv_bfloat16 *gt = (const __nv_bfloat16 *)g;
    // the kept u and chunk states go out by TMA stores from shared-memory tiles
    CUtensorMap mku, mks;
    memset(&mku, 0, sizeof(mku));
    memset(&mks, 0, sizeof(mks));
    if (u_out && !tmap::make_3d(&mku, u_out, DV, L, BH, 64, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return cudaErrorInvalidValue;
    if (ck_out && !make_map_2d(&mks, ck_out, DV, (uint64_t)total * DK, 64, DK, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return cudaErrorInvalidValue;
    const int pgrid = total < di.prep_grid ? total : di.prep_grid;
    tc_prep_kernel<DK, GATED><<<pgrid, THREADS, prep_smem_bytes<DK>(), s>>>(
        mk, (const __nv_bfloat16 *)beta, gt, (__half *)ws, L, NC, total, euler);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    constexpr int SSM = StateLayout<DK, DV, GATED>::SMEM + ((SAVE || KEEP) ? keep_stage_bytes<DK, DV>() : 0);
    const int G = allow_seg ? seg_count(BH, NC, DK, DV, di.nsm) : 1;
    if (G < 3) {
        // One CTA per head.  A grid of at most half the SM count lands one CTA per TPC;
        // two heads' chunk loops on the two SMs of one TPC each run 15-25% slower
        // (measured), so nothing else is scheduled beside this kernel.
        // the plain forward drops its Ta tiles from L2 as it goes (nothing reads them again)
        uint8_t *drop = (!SAVE && !KEEP && ((uintptr_t)ws & 127u) == 0) ? (uint8_t *)ws : nullptr;
        tc_state_kernel<DK, DV, TO, false, SAVE, GATED, KEEP><<<BH, ST_THREADS, SSM, s>>>(
            mq, mk, mv, mt, mku, mks, S0, (TO *)o, S_final, L, NC, nullptr, 1, NC, 0, u_out, ck_out, gt, drop);
        count_launches(2);
        return cudaGetLastError();
    }
    if constexpr (DK == DV) {
        const int seg_chunks = (NC + G - 1) / G;
        float *segbuf = (float *)((uint8_t *)ws + ta_bytes(total));
        tc_state_kernel<DK, DV, TO, true, SAVE, GATED, KEEP><<<BH * (2 * G - 3), ST_THREADS, SSM, s>>>(
            mq, mk, mv, mt, mku, mks, S0, (TO *)o, S_final, L, NC, segbuf, G, seg_chunks, 1, u_out, ck_out, gt, nullptr);
        seg_combine_kernel<DK><<<BH * (DV / 16), DK, 0, s>>>(segbuf, G);
        tc_state_kernel<DK, DV, TO, true, SAVE, GATED, KEEP><<<BH * (G - 1), ST_THREADS, SSM, s>>>(
            mq, mk, mv, mt, mku, mks, S0, (TO *)o, S_final, L, NC, segbuf, G, seg_chunks, 2, u_out, ck_out, gt, nullptr);
        count_launches(4);
    }
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_tc_o(const void *q, const void *k, const void *v, const void *beta,
                        const float *S0, void *o, float *S_final, int B, int H, int L, bool o_bf16,
                        bool euler, void *ws, cudaStream_t s, bool allow_seg, const void *g) {
    using bf = __nv_bfloat16;
    if (g)
        return o_bf16 ? launch_tc_t<DK, DV, bf, false, true>(q, k, v, beta, S0, o, S_final, B, H, L, euler, ws, s,
                                                             nullptr, nullptr, allow_seg, g)
                      : launch_tc_t<DK, DV, float, false, true>(q, k, v, beta, S0, o, S_final, B, H, L, euler, ws,
                                                                s, nullptr, nullptr, allow_seg, g);
    return o_bf16 ? launch_tc_t<DK, DV, bf, false, false>(q, k, v, beta, S0, o, S_final, B, H, L, euler, ws, s,
                                                          nullptr, nullptr, allow_seg, nullptr)
                  : launch_tc_t<DK, DV, float, false, false>(q, k, v, beta, S0, o, S_final, B, H, L, euler, ws, s,
                                                             nullptr, nullptr, allow_seg, nullptr);
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

size_t tc_workspace_bytes(int B, int H, int L, int dk, int dv, int chunk, bool allow_segments) {
    (void)chunk;
    const long long BH = (long long)B * H;
    const int NC = (L + C - 1) / C;
    const size_t total = (size_t)BH * NC;
    if (!allow_segments || !seg_sizes_ok(BH, NC, dk, dv)) return total * C * C * sizeof(__half);
    return ta_bytes(total) + (size_t)BH * SEG_MAX * 3 * dk * dv * sizeof(float);
}

int tc_segments(int B, int H, int L, int dk, int dv) {
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return 1;
    }
    return seg_count((long long)B * H, (L + C - 1) / C, dk, dv, nsm);
}

cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const void *beta,
                            const float *S0, void *o, float *S_final, int B, int H, int L,
                            int dk, int dv, int chunk, bool o_bf16, bool euler, void *ws,
                            cudaStream_t s, bool allow_segments, const void *g) {
    (void)chunk;
    if (dk == 128 && dv == 128)
        return launch_tc_o<128, 128>(q, k, v, beta, S0, o, S_final, B, H, L, o_bf16, euler, ws, s, allow_segments, g);
    if (dk == 128 && dv == 64)
        return launch_tc_o<128, 64>(q, k, v, beta, S0, o, S_final, B, H, L, o_bf16, euler, ws, s, allow_segments, g);
    if (dk == 64 && dv == 128)
        return launch_tc_o<64, 128>(q, k, v, beta, S0, o, S_final, B, H, L, o_bf16, euler, ws, s, allow_segments, g);
    return launch_tc_o<64, 64>(q, k, v, beta, S0, o, S_final, B, H, L, o_bf16, euler, ws, s, allow_segments, g);
}

cudaError_t launch_chunk_tc_save(const void *q, const void *k, const void *v, const void *beta,
                                 const float *S0, int B, int H, int L, int dk, int dv, bool euler,
                                 void *ws, __half *u_out, __half *ck_out, cudaStream_t s) {
    if (dk == 128 && dv == 128)
        return launch_tc_t<128, 128, float, true, false>(q, k, v, beta, S0, nullptr, nullptr, B, H, L, euler, ws,
                                                         s, u_out, ck_out, true, nullptr);
    if (dk == 128 && dv == 64)
        return launch_tc_t<128, 64, float, true, false>(q, k, v, beta, S0, nullptr, nullptr, B, H, L, euler, ws,
                                                        s, u_out, ck_out, true, nullptr);
    if (dk == 64 && dv == 128)
        return launch_tc_t<64, 128, float, true, false>(q, k, v, beta, S0, nullptr, nullptr, B, H, L, euler, ws,
                                                        s, u_out, ck_out, true, nullptr);
    return launch_tc_t<64, 64, float, true, false>(q, k, v, beta, S0, nullptr, nullptr, B, H, L, euler, ws, s,
                                                   u_out, ck_out, true, nullptr);
}

cudaError_t launch_chunk_tc_keep(const void *q, const void *k, const void *v, const void *beta,
                                 const float *S0, void *o, float *S_final, int B, int H, int L, int dk,
                                 int dv, bool o_bf16, bool euler, void *ws, __half *u_out, __half *ck_out,
                                 cudaStream_t s) {
    using bf = __nv_bfloat16;
#define EFLA_KEEP(DK_, DV_)                                                                                \
    return o_bf16 ? launch_tc_t<DK_, DV_, bf, false, false, true>(q, k, v, beta, S0, o, S_final, B, H, L, euler, \
                                                                  ws, s, u_out, ck_out, true, nullptr)            \
                  : launch_tc_t<DK_, DV_, float, false, false, true>(q, k, v, beta, S0, o, S_final, B, H, L,     \
                                                                     euler, ws, s, u_out, ck_out, true, nullptr)
    if (dk == 128 && dv == 128) EFLA_KEEP(128, 128);
    if (dk == 128 && dv == 64) EFLA_KEEP(128, 64);
    if (dk == 64 && dv == 128) EFLA_KEEP(64, 128);
    EFLA_KEEP(64, 64);
#undef EFLA_KEEP
}

cudaError_t launch_selftest_wait(long long budget_cycles, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(budget_cycles);
    count_launches(1);
    return cudaGetLastError();
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
