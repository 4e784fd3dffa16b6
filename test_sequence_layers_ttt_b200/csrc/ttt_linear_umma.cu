// TTT-Linear forward scan on the 5th-generation tensor cores (tcgen05, TMEM)
// for sm_100a.  Scope: bf16 Q/K/V, d = 64, f(x) = x + LN(x W + b), mini-batch
// b = 16, T a multiple of 16.  One CTA per (batch, head) runs the whole sequence.
//
// Method ("Learning to (Learn at Test Time)", literature record, Key takeaways
// bullets 1, 2 and 5).  W~ = [W; b] (65 x 64), x~ = [x, 1]; for chunk c (one
// mini-batch of 16 tokens, X = K_c) with W~_c the state at its start:
//   Y_c = X~_c W~_c,   G_c = dl/dY_c (LayerNorm backward of ||X + LN(Y) - V||^2)
//   E_c = -diag(eta_c) G_c,   W~_{c+1} = W~_c + X~_c^T E_c
//   zbar_c = Q~_c W~_c + L_c E_c,  L_c[t][s] = (q_t . x_s + 1) for s <= t, else 0
//   z_c = q + LN(zbar_c)
// Substituting the update twice (lag 2):
//   Y_c = R_c + S1_c E_{c-1},  S1_c = X~_c X~_{c-1}^T              (16 x 16)
//   R_c = X~_c W~_{c-2} + S2_c E_{c-2},  S2_c = X~_c X~_{c-2}^T
// so the sequential chain per chunk is the 16x16x64 product S1_c E_{c-1}, the
// LayerNorm statistics and E_c; R_c has two chunk periods of slack.
//
// Work placement:
//   tcgen05 (one issuing thread, operands in shared memory, fp32 accumulators in
//   TMEM, every product transposed so that M = 64 output features):
//     U_c   dW~^T = E_c^T X~_c            (the state increment)
//     P_c   R_c^T = W~_{c-2}^T X~_c^T     (+ the bias row), then += E_{c-2}^T S2_c^T
//     QW_c  zbar_c^T = W~_c^T Q~_c^T      (+ bias), then += E_c^T L_c^T
//   mma.sync (registers): the chain product S1_c E_{c-1}, and the W-free 16x16
//     products S1, S2, L.
// Warp roles (512 threads):
//   CH  0-3   the chain: warp w owns accumulator rows [16w, 16w+16) (TMEM lane
//             quarter w).  Loads R_c from TMEM in the mma C-fragment layout, adds
//             S1_c E_{c-1}, forms the five LayerNorm sums per token (shuffles +
//             one named barrier), writes E_c as bf16 hi/lo operand tiles and
//             keeps it as A fragments for the next chunk.
//   ST  4-7   the state: fp32 W~^T in registers (mma C-fragment layout of the
//             increment), adds U_c from TMEM, writes W~^T as bf16 hi/lo K-major
//             operand tiles.
//   OW  8-11  the output: zbar from TMEM, LayerNorm, residual, fp32 stores.
//   MMA 12    TMEM allocation and every tcgen05.mma / commit.
//   PR  13    TMA loads of K, V, Q tiles (128-byte swizzle) and eta.
//   PA  14    gamma * (x + beta - v) per (feature, token) and its row sums.
//   PB  15    S1 (as mma B fragments), S2 and L (as hi/lo operand tiles).
// Precision: every product with an fp32 operand splits it into bf16 hi + lo
// (both halves rounded to nearest: |x - hi - lo| at most 2^-16 |x|) and drops only lo*lo; bf16 inputs are exact; the state update is formed in TMEM
// and added to the fp32 registers with fp32 adds (tensor-core accumulation of
// thousands of increments would not round to nearest).
// Feature order: accumulator row r = 16 j + i holds output feature
// 16 j + 2 (i % 8) + i / 8, so each thread's two rows are adjacent features.
// Row centring: the state is kept as W~ minus its per-input-row mean over the
// output features (and b minus its mean).  The update preserves these means
// (every row of G sums to zero), LayerNorm ignores a per-token shift of its
// input, and the means are added back to W_T, b_T at the end; y then has mean
// near zero, so the one-pass variance of the statistics does not cancel.
// Hand-offs are mbarriers with bounded waits: after about a second without
// progress the kernel records an error word, stops waiting (every role still
// runs its loop to the end, so named barriers stay balanced), drains its TMA
// loads and tensor-core work, and frees its TMEM (outputs undefined;
// TTT_ERR_TIMEOUT with TTT_CHECK=1).
#include <cstdlib>

#include "common.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"
#include "tma_host.h"
#include "ttt_internal.h"

namespace ttt {

__device__ unsigned int g_umma_error_word = 0;

namespace {

constexpr int D = 64;
constexpr int NS = 8;    // TMA ring stages
constexpr int NPRE = 8;  // ring of W-free per-chunk inputs
constexpr int NE = 4;    // E_c operand tiles
constexpr int NR = 4;    // R_c accumulators in TMEM
constexpr int NZ = 4;    // zbar_c accumulators in TMEM
constexpr int kWarpST0 = 4, kWarpOW0 = 8, kWarpMMA = 12, kWarpPR = 13, kWarpPA = 14, kWarpPB = 15;
constexpr int kWarps = 16, kThreads = kWarps * 32;
constexpr int TILE = kChunk * D * 2;  // one [16][64] bf16 tile
constexpr uint32_t kStageTx = 3 * TILE + kChunk * 4;
constexpr long long kTimeoutCycles = 2000000000LL;
// TMEM columns
constexpr uint32_t kColDW = 0, kColDB = 64, kColR = 128, kColZ = 192, kTmemCols = 512;
// A operands in TMEM (the kAInTmem variant): W~^T hi (32 columns of bf16 pairs), lo (32), the bias
// K step (8: column 0 holds b hi, b lo), and E_c hi (8), lo (8) per buffer
constexpr uint32_t kColWA = 256, kColWB = 320, kColEA = 384;

struct alignas(1024) Stage {
    unsigned char K[TILE], V[TILE], Q[TILE];
};

struct PreSlot {
    float4 gc[4][32][2];     // gamma*(x+beta-v) in the chain's fragment order [warp][lane]
    uint4 s1[2][32];         // [hi, lo][lane]: S1 as mma B fragments (nt0 b0, nt0 b1, nt1 b0, nt1 b1)
    unsigned char s2[2][512];  // [hi, lo] S2 as [t][s] K-major no-swizzle
    unsigned char l[2][512];   // [hi, lo] L as [t][s]
    float c0[kChunk];        // row sums of gamma*(x+beta-v)
    float eta[kChunk];
};

struct UmmaSmem {
    Stage st[NS];                          // 1024-aligned tiles
    unsigned char Whi[D * 128];            // W~^T hi, K-major 128B swizzle (rows = accumulator rows)
    unsigned char Wlo[D * 128];
    unsigned char Abias[D * 32];           // [row][k] K-major none: k = 0 b hi, k = 1 b lo
    unsigned char E[NE][2][D * 32];        // [buf][hi, lo] E^T as [row][token] K-major none
    unsigned char ones16[16 * 32];         // [t][k]: k = 0, 1 are 1
    unsigned char ones8[8 * 32 + 128];     // [n][k]: row 0 is 1 for every k < 16
    PreSlot pre[NPRE];
    alignas(128) float eta[NS][32];         // TMA destinations: 128-byte aligned rows (16 used)
    float red_ch[2][kChunk][5][4];         // [buf][token][sum][warp]
    float coef_ch[4][kChunk][8];           // [warp][token][mu, a, b2, c2, d2]
    float red_ow[2][kChunk][2][4];
    float coef_ow[4][kChunk][2];
    float gam[D], bet[D], gam2[D];
    float u[D + 1];                        // per-row means removed from the state (row D: bias)
    uint64_t in_full[NS], in_empty[NS];
    uint64_t pre_full[NPRE], pre_empty[NPRE];
    uint64_t e_full[NE], e_empty[NE];
    uint64_t r_full[NR], r_empty[NR];
    uint64_t z_full[NZ], z_empty[NZ];
    uint64_t w_full, dw_full, dw_empty, drain;
    uint32_t tmem_base;
    int abort_flag;
};

__host__ __device__ constexpr int row_feature(int r) { return (r & ~15) + 2 * (r & 7) + ((r >> 3) & 1); }

__device__ __forceinline__ uint32_t swz(int row, int col) {
    return row * 128 + ((((col >> 3) ^ (row & 7))) << 4) + (col & 7) * 2;
}
__device__ __forceinline__ uint32_t swz_chunk(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (int spins = 1;; spins++) {
        if (*abort_flag) return false;
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((spins & 63) == 0 && clock64() - t0 > kTimeoutCycles) {
            *abort_flag = 1;
            atomicOr(&g_umma_error_word, 1u);
            return false;
        }
    }
}
// wait for completion number k (0-based) of a barrier that completes once per use
__device__ __forceinline__ bool wait_k(uint64_t* bar, int k, volatile int* abort_flag) {
    return wait_bounded(bar, (uint32_t)(k & 1), abort_flag);
}
__device__ __forceinline__ void arrive1(uint64_t* bar, int lane) {
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar);
}

template <bool kAInTmem>
__global__ void __launch_bounds__(kThreads, 1)
ttt_linear_umma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmEta,
                       int T, int H, float eps, const float* W0, const float* b0,
                       const float* __restrict__ gamma, const float* __restrict__ beta,
                       float* __restrict__ Z, float* W_T, float* b_T, int drop_chunk) {
    extern __shared__ unsigned char smem_raw[];
    UmmaSmem& s = *reinterpret_cast<UmmaSmem*>(smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int bh = blockIdx.x, h = bh % H;
    const int n = T / kChunk;
    volatile int* abort_flag = &s.abort_flag;

    // ---------------------------------------------------------------- set-up
    if (tid < D) {
        const float gm = gamma[h * D + tid];
        s.gam[tid] = gm;
        s.gam2[tid] = gm * gm;
        s.bet[tid] = beta[h * D + tid];
    }
    // constant operand tiles
    for (int i = tid; i < 16 * 16; i += kThreads) {
        const int r = i >> 4, k = i & 15;
        const __nv_bfloat16 one = __float2bfloat16(1.f), zero = __float2bfloat16(0.f);
        *reinterpret_cast<__nv_bfloat16*>(s.ones16 + tc05::kmajor16_offset(r, k)) = (k < 2) ? one : zero;
        if (r < 8)
            *reinterpret_cast<__nv_bfloat16*>(s.ones8 + tc05::kmajor16_offset(r, k)) = (r == 0) ? one : zero;
    }
    for (int i = tid; i < D * 16; i += kThreads)  // bias tile: zero K columns 2..15
        *reinterpret_cast<__nv_bfloat16*>(s.Abias + tc05::kmajor16_offset(i >> 4, i & 15)) = __float2bfloat16(0.f);
    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < NS; i++) {
            ptx::mbar_init(&s.in_full[i], 1);
            ptx::mbar_init(&s.in_empty[i], 1 + 1 + 1 + 4);  // MMA commit, PA, PB, OW warps
        }
        for (int i = 0; i < NPRE; i++) {
            ptx::mbar_init(&s.pre_full[i], 2);      // PA, PB
            ptx::mbar_init(&s.pre_empty[i], 4 + 1);  // CH warps, MMA commit
        }
        for (int i = 0; i < NE; i++) {
            ptx::mbar_init(&s.e_full[i], 4);
            ptx::mbar_init(&s.e_empty[i], 1);
        }
        for (int i = 0; i < NR; i++) {
            ptx::mbar_init(&s.r_full[i], 1);
            ptx::mbar_init(&s.r_empty[i], 4);
        }
        for (int i = 0; i < NZ; i++) {
            ptx::mbar_init(&s.z_full[i], 1);
            ptx::mbar_init(&s.z_empty[i], 4);
        }
        ptx::mbar_init(&s.w_full, 4);
        ptx::mbar_init(&s.dw_full, 1);
        ptx::mbar_init(&s.dw_empty, 4);
        ptx::mbar_init(&s.drain, 1);
        ptx::fence_mbar_init();
    }
    if (warp == kWarpMMA) tc05::tmem_alloc(ptx::smem_addr(&s.tmem_base), kTmemCols);
    ptx::fence_proxy_async_smem();
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = s.tmem_base;

    // ================================================================ PR: TMA producer
    if (warp == kWarpPR) {
        if (lane == 0) {
            ptx::prefetch_tmap(&tmK);
            ptx::prefetch_tmap(&tmV);
            ptx::prefetch_tmap(&tmQ);
            ptx::prefetch_tmap(&tmEta);
            int issued = 0;
            for (int c = 0; c < n; c++) {
                const int slot = c % NS;
                if (c >= NS && !wait_k(&s.in_empty[slot], c / NS - 1, abort_flag)) break;
                if (c == drop_chunk) continue;  // fault-injection hook: this chunk is never loaded
                ptx::mbar_arrive_expect_tx(&s.in_full[slot], kStageTx);
                ptx::tma_load_3d(s.st[slot].K, &tmK, &s.in_full[slot], 0, c * kChunk, bh);
                ptx::tma_load_3d(s.st[slot].V, &tmV, &s.in_full[slot], 0, c * kChunk, bh);
                ptx::tma_load_3d(s.st[slot].Q, &tmQ, &s.in_full[slot], 0, c * kChunk, bh);
                ptx::tma_load_2d(s.eta[slot], &tmEta, &s.in_full[slot], c * kChunk, bh);
                issued = c + 1;
            }
            for (int c = issued - 1; c >= 0 && c >= issued - NS; c--) {  // drain own loads
                if (c == drop_chunk) continue;
                const long long t0 = clock64();
                while (!ptx::mbar_try_wait(&s.in_full[c % NS], (c / NS) & 1)) {
                    if (clock64() - t0 > 4 * kTimeoutCycles) {
                        atomicOr(&g_umma_error_word, 2u);
                        break;
                    }
                }
            }
        }
    }

    // ================================================================ PA: gamma*(x+beta-v), row sums, eta
    else if (warp == kWarpPA) {
        for (int c = 0; c < n; c++) {
            const int slot = c % NS, p = c % NPRE;
            wait_k(&s.in_full[slot], c / NS, abort_flag);
            if (c >= NPRE) wait_k(&s.pre_empty[p], c / NPRE - 1, abort_flag);
            PreSlot& ps = s.pre[p];
            float rs[4] = {0.f, 0.f, 0.f, 0.f};  // row sums for tokens 8nt + 2t4 + e, index 2nt + e
#pragma unroll
            for (int w = 0; w < 4; w++) {
                const int f0 = 16 * w + 2 * g;
                const float g0 = s.gam[f0], g1 = s.gam[f0 + 1], gb0 = g0 * s.bet[f0], gb1 = g1 * s.bet[f0 + 1];
                float v8[8];
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const int tok = 8 * nt + 2 * t4 + e;
                        const uint32_t xv = *reinterpret_cast<const uint32_t*>(s.st[slot].K + swz(tok, f0));
                        const uint32_t vv = *reinterpret_cast<const uint32_t*>(s.st[slot].V + swz(tok, f0));
                        const float e0 = fmaf(g0, ptx::bf16_lo_f32(xv) - ptx::bf16_lo_f32(vv), gb0);
                        const float e1 = fmaf(g1, ptx::bf16_hi_f32(xv) - ptx::bf16_hi_f32(vv), gb1);
                        v8[4 * nt + e] = e0;
                        v8[4 * nt + 2 + e] = e1;
                        rs[2 * nt + e] += e0 + e1;
                    }
                ps.gc[w][lane][0] = make_float4(v8[0], v8[1], v8[2], v8[3]);
                ps.gc[w][lane][1] = make_float4(v8[4], v8[5], v8[6], v8[7]);
            }
#pragma unroll
            for (int i = 0; i < 4; i++) {
                rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 4);
                rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 8);
                rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 16);
            }
            if (g == 0) {
#pragma unroll
                for (int i = 0; i < 4; i++) ps.c0[8 * (i >> 1) + 2 * t4 + (i & 1)] = rs[i];
            }
            if (lane < kChunk) ps.eta[lane] = s.eta[slot][lane];
            arrive1(&s.pre_full[p], lane);
            arrive1(&s.in_empty[slot], lane);
        }
    }

    // ================================================================ PB: S1, S2, L
    else if (warp == kWarpPB) {
        for (int c = 0; c < n; c++) {
            const int slot = c % NS, p = c % NPRE;
            wait_k(&s.in_full[slot], c / NS, abort_flag);
            if (c >= NPRE) wait_k(&s.pre_empty[p], c / NPRE - 1, abort_flag);
            PreSlot& ps = s.pre[p];
            const uint32_t xs = ptx::smem_addr(s.st[slot].K), qs = ptx::smem_addr(s.st[slot].Q);
            const uint32_t x1s = ptx::smem_addr(s.st[(c + NS - 1) % NS].K);
            const uint32_t x2s = ptx::smem_addr(s.st[(c + NS - 2) % NS].K);
            const int mi = lane >> 3;
            float p1[2][4], p2[2][4], pl[2][4];  // X_c X_{c-1}^T, X_c X_{c-2}^T, Q_c X_c^T (C layout)
#pragma unroll
            for (int nt = 0; nt < 2; nt++)
#pragma unroll
                for (int r = 0; r < 4; r++) p1[nt][r] = p2[nt][r] = pl[nt][r] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                uint32_t xa[4], qa[4], bx[4], b1[4], b2[4];
                {
                    const int row = (mi & 1) * 8 + (lane & 7), chunk = 2 * ks + (mi >> 1);
                    ptx::ldsm_x4(xs + swz_chunk(row, chunk), xa[0], xa[1], xa[2], xa[3]);
                    ptx::ldsm_x4(qs + swz_chunk(row, chunk), qa[0], qa[1], qa[2], qa[3]);
                }
                {
                    const int row = (mi >> 1) * 8 + (lane & 7), chunk = 2 * ks + (mi & 1);
                    ptx::ldsm_x4(xs + swz_chunk(row, chunk), bx[0], bx[1], bx[2], bx[3]);
                    if (c >= 1) ptx::ldsm_x4(x1s + swz_chunk(row, chunk), b1[0], b1[1], b1[2], b1[3]);
                    if (c >= 2) ptx::ldsm_x4(x2s + swz_chunk(row, chunk), b2[0], b2[1], b2[2], b2[3]);
                }
#pragma unroll
                for (int nt = 0; nt < 2; nt++) {
                    ptx::mma_bf16(pl[nt], qa[0], qa[1], qa[2], qa[3], bx[2 * nt], bx[2 * nt + 1]);
                    if (c >= 1) ptx::mma_bf16(p1[nt], xa[0], xa[1], xa[2], xa[3], b1[2 * nt], b1[2 * nt + 1]);
                    if (c >= 2) ptx::mma_bf16(p2[nt], xa[0], xa[1], xa[2], xa[3], b2[2 * nt], b2[2 * nt + 1]);
                }
            }
            // S1 = X~_c X~_{c-1}^T as the chain's B fragments, hi and lo
            {
                uint32_t hi[4], lo[4];
                // b0(nt) = S1[8nt+g][2t4, 2t4+1], b1(nt) = S1[8nt+g][2t4+8, 2t4+9]
                ptx::split_pair_rn(p1[0][0] + 1.f, p1[0][1] + 1.f, hi[0], lo[0]);
                ptx::split_pair_rn(p1[1][0] + 1.f, p1[1][1] + 1.f, hi[1], lo[1]);
                ptx::split_pair_rn(p1[0][2] + 1.f, p1[0][3] + 1.f, hi[2], lo[2]);
                ptx::split_pair_rn(p1[1][2] + 1.f, p1[1][3] + 1.f, hi[3], lo[3]);
                ps.s1[0][lane] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                ps.s1[1][lane] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            // S2 = X~_c X~_{c-2}^T and L = tril(Q~_c X~_c^T) as [t][s] operand tiles, hi and lo
#pragma unroll
            for (int nt = 0; nt < 2; nt++)
#pragma unroll
                for (int rh = 0; rh < 2; rh++) {
                    const int t = g + 8 * rh, s0 = 8 * nt + 2 * t4;
                    const uint32_t off = tc05::kmajor16_offset(t, s0);
                    uint32_t hi, lo;
                    ptx::split_pair_rn(p2[nt][2 * rh] + 1.f, p2[nt][2 * rh + 1] + 1.f, hi, lo);
                    *reinterpret_cast<uint32_t*>(ps.s2[0] + off) = hi;
                    *reinterpret_cast<uint32_t*>(ps.s2[1] + off) = lo;
                    const float l0 = s0 <= t ? pl[nt][2 * rh] + 1.f : 0.f;
                    const float l1 = s0 + 1 <= t ? pl[nt][2 * rh + 1] + 1.f : 0.f;
                    ptx::split_pair_rn(l0, l1, hi, lo);
                    *reinterpret_cast<uint32_t*>(ps.l[0] + off) = hi;
                    *reinterpret_cast<uint32_t*>(ps.l[1] + off) = lo;
                }
            ptx::fence_proxy_async_smem();  // S2 / L are read by the tensor cores
            arrive1(&s.pre_full[p], lane);
            if (c >= 2) arrive1(&s.in_empty[(c - 2) % NS], lane);  // last use of X_{c-2}
        }
        for (int c = n - 2; c < n; c++)
            if (c >= 0) arrive1(&s.in_empty[c % NS], lane);
    }

    // ================================================================ MMA issuer
    else if (warp == kWarpMMA) {
        if (lane == 0) {
            constexpr uint32_t I16 = tc05::idesc_bf16(64, 16, 0, 0);
            constexpr uint32_t I64 = tc05::idesc_bf16(64, 64, 0, 1);
            constexpr uint32_t I8 = tc05::idesc_bf16(64, 8, 0, 0);
            const uint32_t whi = ptx::smem_addr(s.Whi), wlo = ptx::smem_addr(s.Wlo);
            const uint64_t d_bias = tc05::desc_k16(ptx::smem_addr(s.Abias));
            const uint64_t d_one16 = tc05::desc_k16(ptx::smem_addr(s.ones16));
            const uint64_t d_one8 = tc05::desc_k16(ptx::smem_addr(s.ones8));
            bool ok = true;
            // D += W~^T [tile]^T for a [16][64] token tile: 4 K steps x (hi, lo), then the bias row
            auto issue_xw = [&](uint32_t dcol, uint32_t tile) {
#pragma unroll
                for (int ks = 0; ks < 4; ks++) {
                    const uint64_t b = tc05::desc_k128(tile, ks);
                    if constexpr (kAInTmem) {
                        tc05::mma_bf16_ts(tmem + dcol, tmem + kColWA + 8 * ks, b, I16, ks > 0);
                        tc05::mma_bf16_ts(tmem + dcol, tmem + kColWA + 32 + 8 * ks, b, I16, 1);
                    } else {
                        tc05::mma_bf16_ss(tmem + dcol, tc05::desc_k128(whi, ks), b, I16, ks > 0);
                        tc05::mma_bf16_ss(tmem + dcol, tc05::desc_k128(wlo, ks), b, I16, 1);
                    }
                }
                if constexpr (kAInTmem)
                    tc05::mma_bf16_ts(tmem + dcol, tmem + kColWB, d_one16, I16, 1);
                else
                    tc05::mma_bf16_ss(tmem + dcol, d_bias, d_one16, I16, 1);
            };
            // D += E^T M^T for a [16][16] hi/lo operand pair (hi*hi + hi*lo + lo*hi); E buffer e
            auto issue_corr = [&](uint32_t dcol, int e, uint32_t mhi, uint32_t mlo) {
                const uint64_t mh = tc05::desc_k16(mhi), ml = tc05::desc_k16(mlo);
                if constexpr (kAInTmem) {
                    const uint32_t ea = tmem + kColEA + 16 * e;
                    tc05::mma_bf16_ts(tmem + dcol, ea, mh, I16, 1);
                    tc05::mma_bf16_ts(tmem + dcol, ea, ml, I16, 1);
                    tc05::mma_bf16_ts(tmem + dcol, ea + 8, mh, I16, 1);
                } else {
                    const uint64_t eh = tc05::desc_k16(ptx::smem_addr(s.E[e][0]));
                    const uint64_t el = tc05::desc_k16(ptx::smem_addr(s.E[e][1]));
                    tc05::mma_bf16_ss(tmem + dcol, eh, mh, I16, 1);
                    tc05::mma_bf16_ss(tmem + dcol, eh, ml, I16, 1);
                    tc05::mma_bf16_ss(tmem + dcol, el, mh, I16, 1);
                }
            };
            // prologue: W~_0 ready; R_0, R_1, R_2 = X~_j W~_0 (R_0, R_1 final), zbar_0 = Q~_0 W~_0
            ok = wait_k(&s.w_full, 0, abort_flag);
            for (int j = 0; j < 3 && j < n && ok; j++) {
                ok = wait_k(&s.in_full[j % NS], j / NS, abort_flag);
                if (!ok) break;
                tc05::fence_after_sync();
                issue_xw(kColR + 16 * (j % NR), ptx::smem_addr(s.st[j % NS].K));
                if (j < 2) tc05::commit(ptx::smem_addr(&s.r_full[j % NR]));
            }
            if (ok && n > 0) issue_xw(kColZ + 0, ptx::smem_addr(s.st[0].Q));
            for (int c = 1; c <= n && ok; c++) {
                const int e = (c - 1) % NE, pc = (c - 1) % NPRE;
                // ---- E_{c-1} ready: state increment U_{c-1}
                ok = wait_k(&s.e_full[e], (c - 1) / NE, abort_flag);
                if (ok && c >= 2) ok = wait_k(&s.dw_empty, c - 2, abort_flag);
                if (!ok) break;
                tc05::fence_after_sync();
                {
                    const uint64_t xmn = tc05::desc_mn128(ptx::smem_addr(s.st[(c - 1) % NS].K));
                    if constexpr (kAInTmem) {
                        const uint32_t ea = tmem + kColEA + 16 * e;
                        tc05::mma_bf16_ts(tmem + kColDW, ea, xmn, I64, 0);
                        tc05::mma_bf16_ts(tmem + kColDW, ea + 8, xmn, I64, 1);
                        tc05::mma_bf16_ts(tmem + kColDB, ea, d_one8, I8, 0);
                        tc05::mma_bf16_ts(tmem + kColDB, ea + 8, d_one8, I8, 1);
                    } else {
                        const uint64_t eh = tc05::desc_k16(ptx::smem_addr(s.E[e][0]));
                        const uint64_t el = tc05::desc_k16(ptx::smem_addr(s.E[e][1]));
                        tc05::mma_bf16_ss(tmem + kColDW, eh, xmn, I64, 0);
                        tc05::mma_bf16_ss(tmem + kColDW, el, xmn, I64, 1);
                        tc05::mma_bf16_ss(tmem + kColDB, eh, d_one8, I8, 0);
                        tc05::mma_bf16_ss(tmem + kColDB, el, d_one8, I8, 1);
                    }
                }
                tc05::commit(ptx::smem_addr(&s.dw_full));
                tc05::commit(ptx::smem_addr(&s.in_empty[(c - 1) % NS]));
                // ---- R_{c+1} += E_{c-1}^T S2_{c+1}^T
                if (c + 1 < n && c + 1 >= 2) {
                    const int p1 = (c + 1) % NPRE;
                    ok = wait_k(&s.pre_full[p1], (c + 1) / NPRE, abort_flag);
                    if (!ok) break;
                    issue_corr(kColR + 16 * ((c + 1) % NR), e, ptx::smem_addr(s.pre[p1].s2[0]),
                               ptx::smem_addr(s.pre[p1].s2[1]));
                    tc05::commit(ptx::smem_addr(&s.r_full[(c + 1) % NR]));
                }
                // ---- zbar_{c-1} += E_{c-1}^T L_{c-1}^T
                ok = wait_k(&s.pre_full[pc], (c - 1) / NPRE, abort_flag);
                if (!ok) break;
                issue_corr(kColZ + 16 * ((c - 1) % NZ), e, ptx::smem_addr(s.pre[pc].l[0]),
                           ptx::smem_addr(s.pre[pc].l[1]));
                tc05::commit(ptx::smem_addr(&s.z_full[(c - 1) % NZ]));
                tc05::commit(ptx::smem_addr(&s.e_empty[e]));
                tc05::commit(ptx::smem_addr(&s.pre_empty[pc]));
                if (c == n) break;
                // ---- W~_c ready: R_{c+2} = X~_{c+2} W~_c and zbar_c = Q~_c W~_c
                ok = wait_k(&s.w_full, c, abort_flag);
                if (!ok) break;
                if (c + 2 < n) {
                    const int j = c + 2;
                    if (j >= NR) ok = wait_k(&s.r_empty[j % NR], j / NR - 1, abort_flag);
                    if (ok) ok = wait_k(&s.in_full[j % NS], j / NS, abort_flag);
                    if (!ok) break;
                    tc05::fence_after_sync();
                    issue_xw(kColR + 16 * (j % NR), ptx::smem_addr(s.st[j % NS].K));
                }
                if (c >= NZ) ok = wait_k(&s.z_empty[c % NZ], c / NZ - 1, abort_flag);
                if (!ok) break;
                tc05::fence_after_sync();
                issue_xw(kColZ + 16 * (c % NZ), ptx::smem_addr(s.st[c % NS].Q));
            }
            // drain: wait (bounded) for every MMA issued so far before TMEM is freed
            tc05::commit(ptx::smem_addr(&s.drain));
            const long long t0 = clock64();
            while (!ptx::mbar_try_wait(&s.drain, 0)) {
                if (clock64() - t0 > 4 * kTimeoutCycles) {
                    atomicOr(&g_umma_error_word, 4u);
                    break;
                }
            }
        }
        __syncwarp();
    }

    // ================================================================ ST: the state
    else if (warp >= kWarpST0 && warp < kWarpOW0) {
        const int q = warp - kWarpST0;
        const int r0 = 16 * q + g, r1 = r0 + 8;
        const int f0 = row_feature(r0), f1 = row_feature(r1);
        const float* W0b = W0 + (size_t)bh * D * D;
        // row means over the output features, removed from the state during the scan
        {
            const int st = tid - kWarpST0 * 32;
            if (st < D) {
                float acc = 0.f;
                for (int j = 0; j < D; j++) acc += W0b[st * D + j];
                s.u[st] = acc * (1.f / D);
            } else if (st == D) {
                float acc = 0.f;
                for (int j = 0; j < D; j++) acc += b0[(size_t)bh * D + j];
                s.u[D] = acc * (1.f / D);
            }
            ptx::named_bar_sync(3, 128);
        }
        float Wt[32];  // [4 j + 0..3]: (r0, k), (r0, k+1), (r1, k), (r1, k+1) with k = 8 j + 2 t4
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int k = 8 * j + 2 * t4;
            const float u0 = s.u[k], u1 = s.u[k + 1];
            Wt[4 * j + 0] = W0b[k * D + f0] - u0;
            Wt[4 * j + 1] = W0b[(k + 1) * D + f0] - u1;
            Wt[4 * j + 2] = W0b[k * D + f1] - u0;
            Wt[4 * j + 3] = W0b[(k + 1) * D + f1] - u1;
        }
        float bt0 = 0.f, bt1 = 0.f;  // bias rows r0, r1 (held by t4 == 0)
        if (t4 == 0) {
            bt0 = b0[(size_t)bh * D + f0] - s.u[D];
            bt1 = b0[(size_t)bh * D + f1] - s.u[D];
        }
        const uint32_t tq = tmem + tc05::taddr_lane(32 * q);
        if constexpr (kAInTmem) tc05::st_16x128b_x2(tq + kColWB, 0u, 0u, 0u, 0u);  // bias K step: zeros
        auto write_tiles = [&]() {
            if constexpr (kAInTmem) {
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    ptx::split_pair_rn(Wt[4 * j + 0], Wt[4 * j + 1], hi[2 * j], lo[2 * j]);
                    ptx::split_pair_rn(Wt[4 * j + 2], Wt[4 * j + 3], hi[2 * j + 1], lo[2 * j + 1]);
                }
                tc05::st_16x128b_x8(tq + kColWA, hi);
                tc05::st_16x128b_x8(tq + kColWA + 32, lo);
                uint32_t bb0 = 0u, bb1 = 0u;  // bias row: k = 0 holds b hi, k = 1 holds b lo
                if (t4 == 0) {
                    uint32_t h, l;
                    ptx::split_pair_rn(bt0, 0.f, h, l);
                    bb0 = (h & 0xffffu) | (l << 16);
                    ptx::split_pair_rn(bt1, 0.f, h, l);
                    bb1 = (h & 0xffffu) | (l << 16);
                }
                tc05::st_16x128b_x1(tq + kColWB, bb0, bb1);
                tc05::wait_st();
                tc05::fence_before_sync();
            } else {
#pragma unroll
            for (int j = 0; j < 8; j++) {
                uint32_t h0, l0, h1, l1;
                ptx::split_pair_rn(Wt[4 * j + 0], Wt[4 * j + 1], h0, l0);
                ptx::split_pair_rn(Wt[4 * j + 2], Wt[4 * j + 3], h1, l1);
                const int k = 8 * j + 2 * t4;
                *reinterpret_cast<uint32_t*>(s.Whi + swz(r0, k)) = h0;
                *reinterpret_cast<uint32_t*>(s.Wlo + swz(r0, k)) = l0;
                *reinterpret_cast<uint32_t*>(s.Whi + swz(r1, k)) = h1;
                *reinterpret_cast<uint32_t*>(s.Wlo + swz(r1, k)) = l1;
            }
            if (t4 == 0) {  // bias row: k = 0 holds b hi, k = 1 holds b lo
                uint32_t h, l;
                ptx::split_pair_rn(bt0, 0.f, h, l);
                *reinterpret_cast<uint32_t*>(s.Abias + tc05::kmajor16_offset(r0, 0)) = (h & 0xffffu) | (l << 16);
                ptx::split_pair_rn(bt1, 0.f, h, l);
                *reinterpret_cast<uint32_t*>(s.Abias + tc05::kmajor16_offset(r1, 0)) = (h & 0xffffu) | (l << 16);
            }
            ptx::fence_proxy_async_smem();
            }
            arrive1(&s.w_full, lane);
        };
        write_tiles();  // W~_0
        for (int c = 0; c < n; c++) {
            wait_k(&s.dw_full, c, abort_flag);
            tc05::fence_after_sync();
            float dv[32], db[4];
            tc05::ld_16x256b_x8(tq + kColDW, dv);
            tc05::ld_16x256b_x1(tq + kColDB, db);
            tc05::wait_ld();
            tc05::fence_before_sync();
            arrive1(&s.dw_empty, lane);
#pragma unroll
            for (int i = 0; i < 32; i += 2) ptx::add2(Wt[i], Wt[i + 1], dv[i], dv[i + 1]);
            if (t4 == 0) {
                bt0 += db[0];
                bt1 += db[2];
            }
            if (c + 1 < n) write_tiles();  // W~_{c+1}
        }
        // final state, row means added back
        float* WTb = W_T + (size_t)bh * D * D;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int k = 8 * j + 2 * t4;
            const float u0 = s.u[k], u1 = s.u[k + 1];
            WTb[k * D + f0] = Wt[4 * j + 0] + u0;
            WTb[(k + 1) * D + f0] = Wt[4 * j + 1] + u1;
            WTb[k * D + f1] = Wt[4 * j + 2] + u0;
            WTb[(k + 1) * D + f1] = Wt[4 * j + 3] + u1;
        }
        if (t4 == 0) {
            b_T[(size_t)bh * D + f0] = bt0 + s.u[D];
            b_T[(size_t)bh * D + f1] = bt1 + s.u[D];
        }
    }

    // ================================================================ CH: the chain
    else if (warp < 4) {
        const int w = warp;
        const int r0 = 16 * w + g;
        const int f0 = row_feature(r0), f1 = f0 + 1;
        const float ga0 = s.gam2[f0], ga1 = s.gam2[f1];
        float Gamma = 0.f;
        for (int j = 0; j < D; j++) Gamma += s.gam2[j];
        const float inv_d = 1.f / D;
        const uint32_t tq = tmem + tc05::taddr_lane(32 * w);
        const int bit4 = (lane >> 4) & 1, bit3 = (lane >> 3) & 1;
        const int my_tok = 8 * bit4 + 2 * t4 + bit3;  // the token whose sums this lane ends up with

        float y[2][4];                 // R_c, then Y_c (C fragments: rows r0/r1, tokens 8nt + 2t4 + e)
        float gc[8];                   // gamma*(x+beta-v) for the same elements
        uint4 s1h, s1l;                // S1_c B fragments
        float c0_my = 0.f, eta_my = 0.f;
        uint32_t ah[4] = {0u, 0u, 0u, 0u}, al[4] = {0u, 0u, 0u, 0u};  // E_{c-1} A fragments
        auto load_inputs = [&](int c) {
            const int p = c % NPRE, rb = c % NR;
            wait_k(&s.r_full[rb], c / NR, abort_flag);
            tc05::fence_after_sync();
            float v[8];
            tc05::ld_16x256b_x2(tq + kColR + 16 * rb, v);
            wait_k(&s.pre_full[p], c / NPRE, abort_flag);
            const PreSlot& ps = s.pre[p];
            const float4 ga = ps.gc[w][lane][0], gb = ps.gc[w][lane][1];
            gc[0] = ga.x; gc[1] = ga.y; gc[2] = ga.z; gc[3] = ga.w;
            gc[4] = gb.x; gc[5] = gb.y; gc[6] = gb.z; gc[7] = gb.w;
            s1h = ps.s1[0][lane];
            s1l = ps.s1[1][lane];
            c0_my = ps.c0[my_tok];
            eta_my = ps.eta[my_tok];
            tc05::wait_ld();
            tc05::fence_before_sync();
#pragma unroll
            for (int i = 0; i < 8; i++) y[i >> 2][i & 3] = v[i];
            arrive1(&s.r_empty[rb], lane);
            arrive1(&s.pre_empty[p], lane);
        };
        if (n > 0) load_inputs(0);
        for (int c = 0; c < n; c++) {
            const int b = c & 1;
            if (c > 0) {
                float t1[2][4], t2[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int r = 0; r < 4; r++) t1[nt][r] = t2[nt][r] = 0.f;
                const uint32_t bh0[2] = {s1h.x, s1h.z}, bh1[2] = {s1h.y, s1h.w};
                const uint32_t bl0[2] = {s1l.x, s1l.z}, bl1[2] = {s1l.y, s1l.w};
#pragma unroll
                for (int nt = 0; nt < 2; nt++) {
                    ptx::mma_bf16(y[nt], ah[0], ah[1], ah[2], ah[3], bh0[nt], bh1[nt]);
                    ptx::mma_bf16(t1[nt], ah[0], ah[1], ah[2], ah[3], bl0[nt], bl1[nt]);
                    ptx::mma_bf16(t2[nt], al[0], al[1], al[2], al[3], bh0[nt], bh1[nt]);
                }
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int r = 0; r < 4; r++) y[nt][r] += t1[nt][r] + t2[nt][r];
            }
            // per-token partial sums over this thread's two features:
            // [slot = 2 nt + e][y, y^2, g^2 y, g^2 y^2, gc y]
            float v[20];
#pragma unroll
            for (int nt = 0; nt < 2; nt++)
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const float y0 = y[nt][e], y1 = y[nt][2 + e];
                    const float a0 = ga0 * y0, a1 = ga1 * y1;
                    float* o = v + 5 * (2 * nt + e);
                    o[0] = y0 + y1;
                    o[1] = fmaf(y0, y0, y1 * y1);
                    o[2] = a0 + a1;
                    o[3] = fmaf(a0, y0, a1 * y1);
                    o[4] = fmaf(gc[4 * nt + e], y0, gc[4 * nt + 2 + e] * y1);
                }
            // reduce over the 8 lanes that share t4, scattering tokens: lane bit 4 picks the n-tile,
            // bit 3 the token of the pair, bit 2 duplicates
            float w10[10];
#pragma unroll
            for (int i = 0; i < 10; i++) {
                const float keep = bit4 ? v[10 + i] : v[i];
                const float send = bit4 ? v[i] : v[10 + i];
                w10[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
            }
            float w5[5];
#pragma unroll
            for (int i = 0; i < 5; i++) {
                const float keep = bit3 ? w10[5 + i] : w10[i];
                const float send = bit3 ? w10[i] : w10[5 + i];
                w5[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
            }
#pragma unroll
            for (int i = 0; i < 5; i++) w5[i] += __shfl_xor_sync(0xffffffffu, w5[i], 4);
            if ((lane & 4) == 0) {
#pragma unroll
                for (int i = 0; i < 5; i++) s.red_ch[b][my_tok][i][w] = w5[i];
            }
            ptx::named_bar_sync(1, 4 * 32);
            float S[5];
#pragma unroll
            for (int i = 0; i < 5; i++) {
                const float4 a = *reinterpret_cast<const float4*>(s.red_ch[b][my_tok][i]);
                S[i] = (a.x + a.y) + (a.z + a.w);
            }
            {
                const float mu = S[0] * inv_d;
                const float var = fmaxf(S[1] * inv_d - mu * mu, 0.f);
                const float rs = rsqrtf(var + eps);
                const float C0 = c0_my;
                const float sgx = 2.f * C0 + 2.f * rs * (S[2] - mu * Gamma);
                const float sgxx =
                    2.f * rs * (S[4] - mu * C0) + 2.f * rs * rs * (S[3] - 2.f * mu * S[2] + mu * mu * Gamma);
                const float k1 = -rs * inv_d * sgx, k2 = -rs * inv_d * sgxx;
                // E = -eta * (rs gx + xh k2 + k1), gx = 2 gc + 2 g^2 xh, xh = (y - mu) rs
                //   = a gc + (b2 g^2 + c2)(y - mu) + d2
                const float ne = -eta_my;
                if ((lane & 4) == 0) {
                    *reinterpret_cast<float4*>(&s.coef_ch[w][my_tok][0]) =
                        make_float4(mu, 2.f * ne * rs, 2.f * ne * rs * rs, ne * rs * k2);
                    s.coef_ch[w][my_tok][4] = ne * k1;
                }
            }
            __syncwarp();
            float E[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; nt++)
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const int tok = 8 * nt + 2 * t4 + e;
                    const float4 cf = *reinterpret_cast<const float4*>(&s.coef_ch[w][tok][0]);
                    const float d2 = s.coef_ch[w][tok][4];
                    const float m0 = y[nt][e] - cf.x, m1 = y[nt][2 + e] - cf.x;
                    E[nt][e] = fmaf(cf.y, gc[4 * nt + e], fmaf(fmaf(cf.z, ga0, cf.w), m0, d2));
                    E[nt][2 + e] = fmaf(cf.y, gc[4 * nt + 2 + e], fmaf(fmaf(cf.z, ga1, cf.w), m1, d2));
                }
            // E_c as A fragments (rows r0/r1, k = tokens) and as hi/lo operand tiles
            ptx::split_pair_rn(E[0][0], E[0][1], ah[0], al[0]);
            ptx::split_pair_rn(E[0][2], E[0][3], ah[1], al[1]);
            ptx::split_pair_rn(E[1][0], E[1][1], ah[2], al[2]);
            ptx::split_pair_rn(E[1][2], E[1][3], ah[3], al[3]);
            const int eb = c % NE;
            if (c >= NE) wait_k(&s.e_empty[eb], c / NE - 1, abort_flag);
            if constexpr (kAInTmem) {
                tc05::fence_after_sync();
                const uint32_t ea = tq + kColEA + 16 * eb;
                tc05::st_16x128b_x2(ea, ah[0], ah[1], ah[2], ah[3]);
                tc05::st_16x128b_x2(ea + 8, al[0], al[1], al[2], al[3]);
                tc05::wait_st();
                tc05::fence_before_sync();
            } else {
                unsigned char* th = s.E[eb][0];
                unsigned char* tl = s.E[eb][1];
                const uint32_t o00 = tc05::kmajor16_offset(r0, 2 * t4), o10 = tc05::kmajor16_offset(r0 + 8, 2 * t4);
                const uint32_t o01 = tc05::kmajor16_offset(r0, 8 + 2 * t4), o11 = tc05::kmajor16_offset(r0 + 8, 8 + 2 * t4);
                *reinterpret_cast<uint32_t*>(th + o00) = ah[0];
                *reinterpret_cast<uint32_t*>(th + o10) = ah[1];
                *reinterpret_cast<uint32_t*>(th + o01) = ah[2];
                *reinterpret_cast<uint32_t*>(th + o11) = ah[3];
                *reinterpret_cast<uint32_t*>(tl + o00) = al[0];
                *reinterpret_cast<uint32_t*>(tl + o10) = al[1];
                *reinterpret_cast<uint32_t*>(tl + o01) = al[2];
                *reinterpret_cast<uint32_t*>(tl + o11) = al[3];
            }
            if constexpr (!kAInTmem) ptx::fence_proxy_async_smem();
            arrive1(&s.e_full[eb], lane);
            if (c + 1 < n) load_inputs(c + 1);
        }
    }

    // ================================================================ OW: outputs
    else {
        const int q = warp - kWarpOW0;
        const int r0 = 16 * q + g;
        const int f0 = row_feature(r0);
        const float gm0 = s.gam[f0], gm1 = s.gam[f0 + 1], bt0 = s.bet[f0], bt1 = s.bet[f0 + 1];
        const uint32_t tq = tmem + tc05::taddr_lane(32 * q);
        const int bit4 = (lane >> 4) & 1, bit3 = (lane >> 3) & 1;
        const int my_tok = 8 * bit4 + 2 * t4 + bit3;
        float* Zbh = Z + (size_t)bh * T * D;
        for (int c = 0; c < n; c++) {
            const int b = c & 1, zb = c % NZ, slot = c % NS;
            wait_k(&s.z_full[zb], c / NZ, abort_flag);
            tc05::fence_after_sync();
            float z[8];
            tc05::ld_16x256b_x2(tq + kColZ + 16 * zb, z);
            tc05::wait_ld();
            tc05::fence_before_sync();
            arrive1(&s.z_empty[zb], lane);
            // [slot = 2 nt + e][sum, sum of squares] over this thread's two features
            float v[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float a = z[4 * (i >> 1) + (i & 1)], bb = z[4 * (i >> 1) + 2 + (i & 1)];
                v[2 * i] = a + bb;
                v[2 * i + 1] = fmaf(a, a, bb * bb);
            }
            float w4[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float keep = bit4 ? v[4 + i] : v[i];
                const float send = bit4 ? v[i] : v[4 + i];
                w4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
            }
            float w2[2];
#pragma unroll
            for (int i = 0; i < 2; i++) {
                const float keep = bit3 ? w4[2 + i] : w4[i];
                const float send = bit3 ? w4[i] : w4[2 + i];
                w2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
            }
            w2[0] += __shfl_xor_sync(0xffffffffu, w2[0], 4);
            w2[1] += __shfl_xor_sync(0xffffffffu, w2[1], 4);
            if ((lane & 4) == 0) {
                s.red_ow[b][my_tok][0][q] = w2[0];
                s.red_ow[b][my_tok][1][q] = w2[1];
            }
            ptx::named_bar_sync(2, 4 * 32);
            {
                const float4 a = *reinterpret_cast<const float4*>(s.red_ow[b][my_tok][0]);
                const float4 bb = *reinterpret_cast<const float4*>(s.red_ow[b][my_tok][1]);
                const float mu = ((a.x + a.y) + (a.z + a.w)) * (1.f / D);
                const float sq = ((bb.x + bb.y) + (bb.z + bb.w)) * (1.f / D);
                const float rs = rsqrtf(fmaxf(sq - mu * mu, 0.f) + eps);
                if ((lane & 4) == 0) *reinterpret_cast<float2*>(&s.coef_ow[q][my_tok][0]) = make_float2(mu, rs);
            }
            __syncwarp();
            wait_k(&s.in_full[slot], c / NS, abort_flag);
#pragma unroll
            for (int nt = 0; nt < 2; nt++)
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const int tok = 8 * nt + 2 * t4 + e;
                    const float2 cf = *reinterpret_cast<const float2*>(&s.coef_ow[q][tok][0]);
                    const uint32_t qv = *reinterpret_cast<const uint32_t*>(s.st[slot].Q + swz(tok, f0));
                    float2 o;
                    o.x = ptx::bf16_lo_f32(qv) + fmaf(gm0 * (z[4 * nt + e] - cf.x), cf.y, bt0);
                    o.y = ptx::bf16_hi_f32(qv) + fmaf(gm1 * (z[4 * nt + 2 + e] - cf.x), cf.y, bt1);
                    *reinterpret_cast<float2*>(Zbh + (size_t)(c * kChunk + tok) * D + f0) = o;
                }
            arrive1(&s.in_empty[slot], lane);
        }
    }

    // ---------------------------------------------------------------- tear-down
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    if (warp == kWarpMMA) tc05::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

// Where the MMAs read their A operands (the state and E_c): tensor memory, written by the warps that
// hold them with tcgen05.st, or shared-memory tiles.
#ifndef TTT_UMMA_A_IN_SMEM
constexpr bool kUmmaAInTmem = true;
#else
constexpr bool kUmmaAInTmem = false;
#endif

bool linear_umma_supports(const LinearArgs& a) {
    return a.d == D && a.dtype == TTT_BF16 && a.mode == TTT_LN_RESIDUAL && a.mini_batch == kChunk && a.T > 0 &&
           a.T % kChunk == 0;
}

cudaError_t launch_linear_umma(const LinearArgs& a, cudaStream_t stream) {
    if (!linear_umma_supports(a)) return cudaErrorInvalidValue;
    const int BH = a.B * a.H;
    CUtensorMap mk, mv, mq, me;
    if (!make_token_tile_map(&mk, a.K, a.T, BH) || !make_token_tile_map(&mv, a.V, a.T, BH) ||
        !make_token_tile_map(&mq, a.Q, a.T, BH) || !make_eta_row_map(&me, a.eta, a.T, BH))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(UmmaSmem) + 1024;
    auto kernel = kUmmaAInTmem ? ttt_linear_umma_kernel<true> : ttt_linear_umma_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<BH, kThreads, smem, stream>>>(mk, mv, mq, me, a.T, a.H, a.ln_eps, a.W0, a.b0, a.gamma, a.beta, a.Z,
                                           a.W_T, a.b_T, drop_chunk_hook());
    return cudaPeekAtLastError();
}

cudaError_t read_and_clear_umma_error(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_umma_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_umma_error_word, &zero, sizeof(unsigned int));
}

}  // namespace ttt
