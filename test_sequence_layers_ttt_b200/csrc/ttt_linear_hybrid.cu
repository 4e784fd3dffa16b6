// TTT-Linear forward scan for sm_100a, lag-2 form: the state increment on the
// 5th-generation tensor cores (tcgen05, TMEM accumulator), the products with
// the state and the sequential chain on warp-level mma.sync.
// Scope: bf16 Q/K/V, d = 64, f(x) = x + LN(x W + b), mini-batch b = 16, T a
// multiple of 16.  One CTA per (batch, head) runs the whole sequence.
//
// Method ("Learning to (Learn at Test Time)", literature record, Key takeaways
// bullets 1, 2 and 5).  W~ = [W; b], x~ = [x, 1]; for chunk c (one mini-batch of
// 16 tokens, X = K_c) with W~_c the state at its start:
//   Y_c = X~_c W~_c,   G_c = dl/dY_c (LayerNorm backward of ||X + LN(Y) - V||^2)
//   E_c = -diag(eta_c) G_c,   W~_{c+1} = W~_c + X~_c^T E_c
//   zbar_c = Q~_c W~_c + L_c E_c,  L_c[t][s] = (q_t . x_s + 1) for s <= t, else 0
//   z_c = q + LN(zbar_c)
// Substituting the update twice:
//   Y_c = R_c + S1_c E_{c-1},   S1_c = X~_c X~_{c-1}^T                   (16 x 16)
//   R_c = X~_c W~_{c-2} + S2_c E_{c-2},   S2_c = X~_c X~_{c-2}^T
// The chain adds only S1_c E_{c-1}; R_c has two chunk periods of slack.
//
// Why this split: a tcgen05 MMA costs 50-65 cycles at the 64 x 16 x 16 shapes
// of these products, whatever its operands, and the products with the state
// take about 26 of them per chunk; the state increment U_c = E_c^T X~_c takes
// 4 (2 of N = 64, 2 of N = 8 for the bias), issued by one thread with the fp32
// increment in TMEM.  The W products run on mma.sync from registers: the state
// warps hold W~^T in the mma C-fragment layout, which is already the A-fragment
// layout of a product with W~^T on the left, so the hi/lo split feeds the
// tensor cores with no data movement.
//
// Every product is transposed so that its 64 rows are the output features: the
// TMEM accumulator rows, the mma fragment rows and the E_c operand rows agree.
// Warp roles (512 threads):
//   CH  0-3   the chain: warp w owns output-feature rows [16w, 16w+16).  Adds
//             S1_c E_{c-1} to R_c, forms the five LayerNorm sums per token
//             (shuffles + one named barrier), writes E_c into TMEM (the A operand
//             of U_c and of the state and output warps' corrections) and keeps
//             it as A fragments for the next chunk.
//   ST  4-7   the state, same rows: fp32 W~^T in registers; per chunk the
//             products P_{c+2} = X~_{c+2} W~_c and Q~_c W~_c (mma.sync), the
//             correction S2_{c+2} E_c into R_{c+2}, then W~_{c+1} = W~_c + U_c
//             (U_c read from TMEM), split into bf16 hi/lo A fragments.
//   OW  8-11  the output, same rows: zbar_c = Q~_c W~_c + L_c E_c, LayerNorm,
//             residual, fp32 stores.
//   MMA 12    TMEM allocation and the tcgen05 MMAs of U_c.
//   PR  13    TMA loads of K, V, Q tiles (128-byte swizzle) and eta.
//   PA  14    gamma * (x + beta - v) per (feature, token) and its row sums.
//   PB  15    S1, S2 and L as mma B fragments (hi/lo).
// Precision: every product with an fp32 operand splits it into bf16 hi + lo
// (truncated top half, remainder rounded to nearest: |x - hi - lo| <= 2^-15 |x|) and
// drops only lo*lo; bf16 inputs are exact; the state update is formed in TMEM
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
#include "timeline.cuh"
#include "tma_host.h"
#include "ttt_internal.h"

namespace ttt {

__device__ unsigned int g_hybrid_error_word = 0;
TTT_TIMELINE_BUFFER(g_hybrid_timeline);  // roles: 0 CH, 1 ST, 2 OW, 3 PR, 4 PA, 5 PB, 6 MMA

namespace {

constexpr int D = 64;
constexpr int NS = 8;    // TMA ring stages
constexpr int NPRE = 8;  // ring of W-free per-chunk inputs
constexpr int NE = 4;    // E_c operands in TMEM
constexpr int NR = 4;    // R_c hand-offs (state -> chain)
constexpr int NQ = 4;    // Q~_c W~_c hand-offs (state -> output)
constexpr int kWarpST0 = 4, kWarpOW0 = 8, kWarpMMA = 12, kWarpPR = 13, kWarpPA = 14, kWarpPB = 15;
constexpr int kWarps = 16, kThreads = kWarps * 32;
constexpr int TILE = kChunk * D * 2;  // one [16][64] bf16 tile
constexpr uint32_t kStageTx = 3 * TILE + kChunk * 4;
constexpr long long kTimeoutCycles = 2000000000LL;
// TMEM columns: the increment U_c (64 + the bias block of 8), E_c hi (8) / lo (8) per buffer
constexpr uint32_t kColDW = 0, kColDB = 64, kColE = 128, kTmemCols = 256;

struct alignas(1024) Stage {
    unsigned char K[TILE], V[TILE], Q[TILE];
};

struct PreSlot {
    float4 gc[4][32][2];  // gamma*(x+beta-v) in the chain's fragment order [warp][lane]
    uint4 s1[2][32];      // [hi, lo][lane]: S1 as mma B fragments (nt0 b0, nt0 b1, nt1 b0, nt1 b1)
    uint4 s2[2][32];      // S2, same layout
    uint4 l[2][32];       // L, same layout
    float c0[kChunk];     // row sums of gamma*(x+beta-v)
    float eta[kChunk];
};

struct HybSmem {
    Stage st[NS];                       // 1024-aligned TMA tiles
    unsigned char ones8[8 * 32 + 128];  // [n][k] K-major core matrices: row 0 is 1 for every k < 16
    PreSlot pre[NPRE];
    float4 rbuf[NR][4][32][2];          // R_c in the chain's fragment order [warp][lane]
    float4 qwbuf[NQ][4][32][2];         // Q~_c W~_c in the output's fragment order
    alignas(128) float eta[NS][32];     // TMA destinations: 128-byte aligned rows (16 used)
    float red_ch[2][kChunk][5][4];      // [buf][token][sum][warp]
    float coef_ch[4][kChunk][8];        // [warp][token][mu, a, b2, c2, d2]
    float red_ow[2][kChunk][2][4];
    float coef_ow[4][kChunk][2];
    float gam[D], bet[D], gam2[D];
    float u[D + 1];                     // per-row means removed from the state (row D: bias)
    uint64_t in_full[NS], in_empty[NS];
    uint64_t pre_full[NPRE], pre_empty[NPRE];
    uint64_t e_full[NE], e_empty[NE];
    uint64_t r_full[NR], r_empty[NR];
    uint64_t q_full[NQ], q_empty[NQ];
    uint64_t dw_full, dw_empty, drain;
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
            atomicOr(&g_hybrid_error_word, 1u);
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

// TMEM -> registers: E_c hi / lo as mma A fragments (rows of this warp's quarter)
__device__ __forceinline__ void ld_e_frags(uint32_t taddr, uint32_t (&a)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.16x128b.x2.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]) : "r"(taddr));
}

// C (16 rows x 16 tokens, two n-tiles) += A (16 rows x 16 tokens, hi/lo) * B^T (16 x 16, hi/lo fragments):
// hi*hi, hi*lo, lo*hi in three independent accumulators
__device__ __forceinline__ void mma_16x16(float (&c)[2][4], const uint32_t (&ah)[4], const uint32_t (&al)[4],
                                          const uint4& bh, const uint4& bl) {
    float t1[2][4], t2[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; nt++)
#pragma unroll
        for (int r = 0; r < 4; r++) t1[nt][r] = t2[nt][r] = 0.f;
    const uint32_t bh0[2] = {bh.x, bh.z}, bh1[2] = {bh.y, bh.w};
    const uint32_t bl0[2] = {bl.x, bl.z}, bl1[2] = {bl.y, bl.w};
#pragma unroll
    for (int nt = 0; nt < 2; nt++) {
        ptx::mma_bf16(c[nt], ah[0], ah[1], ah[2], ah[3], bh0[nt], bh1[nt]);
        ptx::mma_bf16(t1[nt], ah[0], ah[1], ah[2], ah[3], bl0[nt], bl1[nt]);
        ptx::mma_bf16(t2[nt], al[0], al[1], al[2], al[3], bh0[nt], bh1[nt]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; nt++)
#pragma unroll
        for (int r = 0; r < 4; r++) c[nt][r] += t1[nt][r] + t2[nt][r];
}

__global__ void __launch_bounds__(kThreads, 1)
ttt_linear_hybrid_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                         const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmEta,
                         int T, int H, float eps, const float* W0, const float* b0,
                         const float* __restrict__ gamma, const float* __restrict__ beta,
                         float* __restrict__ Z, float* W_T, float* b_T, int drop_chunk) {
    extern __shared__ unsigned char smem_raw[];
    HybSmem& s = *reinterpret_cast<HybSmem*>(smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int bh = blockIdx.x, h = bh % H;
    const int n = T / kChunk;
    volatile int* abort_flag = &s.abort_flag;
    const bool tl_lead = lane == 0 && (warp == 0 || warp == kWarpST0 || warp == kWarpOW0 || warp >= kWarpMMA);
    (void)tl_lead;

    // ---------------------------------------------------------------- set-up
    if (tid < D) {
        const float gm = gamma[h * D + tid];
        s.gam[tid] = gm;
        s.gam2[tid] = gm * gm;
        s.bet[tid] = beta[h * D + tid];
    }
    for (int i = tid; i < 8 * 16; i += kThreads) {
        const int r = i >> 4, k = i & 15;
        *reinterpret_cast<__nv_bfloat16*>(s.ones8 + tc05::kmajor16_offset(r, k)) =
            __float2bfloat16(r == 0 ? 1.f : 0.f);
    }
    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < NS; i++) {
            ptx::mbar_init(&s.in_full[i], 1);
            ptx::mbar_init(&s.in_empty[i], 1 + 1 + 1 + 4 + 4);  // MMA commit, PA, PB, ST warps, OW warps
        }
        for (int i = 0; i < NPRE; i++) {
            ptx::mbar_init(&s.pre_full[i], 2);              // PA, PB
            ptx::mbar_init(&s.pre_empty[i], 4 + 4 + 4);     // CH, ST, OW warps
        }
        for (int i = 0; i < NE; i++) {
            ptx::mbar_init(&s.e_full[i], 4);
            ptx::mbar_init(&s.e_empty[i], 1 + 4 + 4);       // MMA commit, ST, OW warps
        }
        for (int i = 0; i < NR; i++) {
            ptx::mbar_init(&s.r_full[i], 4);
            ptx::mbar_init(&s.r_empty[i], 4);
        }
        for (int i = 0; i < NQ; i++) {
            ptx::mbar_init(&s.q_full[i], 4);
            ptx::mbar_init(&s.q_empty[i], 4);
        }
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
                TTT_STAMP(g_hybrid_timeline, tl_lead, 3, c, 0);
                if (c >= NS && !wait_k(&s.in_empty[slot], c / NS - 1, abort_flag)) break;
                TTT_STAMP(g_hybrid_timeline, tl_lead, 3, c, 1);
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
                        atomicOr(&g_hybrid_error_word, 2u);
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
            TTT_STAMP(g_hybrid_timeline, tl_lead, 4, c, 0);
            wait_k(&s.in_full[slot], c / NS, abort_flag);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 4, c, 1);
            if (c >= NPRE) wait_k(&s.pre_empty[p], c / NPRE - 1, abort_flag);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 4, c, 2);
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
            TTT_STAMP(g_hybrid_timeline, tl_lead, 4, c, 3);
        }
    }

    // ================================================================ PB: S1, S2, L as B fragments
    else if (warp == kWarpPB) {
        for (int c = 0; c < n; c++) {
            const int slot = c % NS, p = c % NPRE;
            TTT_STAMP(g_hybrid_timeline, tl_lead, 5, c, 0);
            wait_k(&s.in_full[slot], c / NS, abort_flag);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 5, c, 1);
            if (c >= NPRE) wait_k(&s.pre_empty[p], c / NPRE - 1, abort_flag);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 5, c, 2);
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
            // The C layout of a 16x16 product M[t][s] (rows t = g, g + 8; columns s = 2t4.., 8 + 2t4..) is
            // the B-fragment layout of M^T for a product whose k is s and n is t:
            // b0(nt) = M[8nt+g][2t4, 2t4+1], b1(nt) = M[8nt+g][2t4+8, 2t4+9]
            auto frags = [&](const float (&m)[2][4], bool causal, uint4& hi4, uint4& lo4) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int nt_src = i & 1, row_hi = i >> 1;  // i = 2 nt_chain + (b0 | b1)
                    const int t = g + 8 * row_hi, s0 = 8 * nt_src + 2 * t4;
                    float v0 = m[nt_src][2 * row_hi] + 1.f, v1 = m[nt_src][2 * row_hi + 1] + 1.f;
                    if (causal) {
                        v0 = s0 <= t ? v0 : 0.f;
                        v1 = s0 + 1 <= t ? v1 : 0.f;
                    }
                    ptx::split_pair(v0, v1, hi[i], lo[i]);
                }
                hi4 = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                lo4 = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            };
            frags(p1, false, ps.s1[0][lane], ps.s1[1][lane]);
            frags(p2, false, ps.s2[0][lane], ps.s2[1][lane]);
            frags(pl, true, ps.l[0][lane], ps.l[1][lane]);
            arrive1(&s.pre_full[p], lane);
            if (c >= 2) arrive1(&s.in_empty[(c - 2) % NS], lane);  // last use of X_{c-2}
            TTT_STAMP(g_hybrid_timeline, tl_lead, 5, c, 3);
        }
        for (int c = n - 2; c < n; c++)
            if (c >= 0) arrive1(&s.in_empty[c % NS], lane);
    }

    // ================================================================ MMA: the state increment U_c
    else if (warp == kWarpMMA) {
        if (lane == 0) {
            constexpr uint32_t I64 = tc05::idesc_bf16(64, 64, 0, 1);
            constexpr uint32_t I8 = tc05::idesc_bf16(64, 8, 0, 0);
            const uint64_t d_one8 = tc05::desc_k16(ptx::smem_addr(s.ones8));
            bool ok = true;
            for (int c = 0; c < n && ok; c++) {
                const int e = c % NE;
                TTT_STAMP(g_hybrid_timeline, tl_lead, 6, c, 0);
                ok = wait_k(&s.in_full[c % NS], c / NS, abort_flag);  // X_c (complete long before)
                if (ok) ok = wait_k(&s.e_full[e], c / NE, abort_flag);
                TTT_STAMP(g_hybrid_timeline, tl_lead, 6, c, 1);
                if (ok && c >= 1) ok = wait_k(&s.dw_empty, c - 1, abort_flag);
                TTT_STAMP(g_hybrid_timeline, tl_lead, 6, c, 2);
                if (!ok) break;
                tc05::fence_after_sync();
                const uint64_t xmn = tc05::desc_mn128(ptx::smem_addr(s.st[c % NS].K));
                const uint32_t ea = tmem + kColE + 16 * e;
                tc05::mma_bf16_ts(tmem + kColDW, ea, xmn, I64, 0);
                tc05::mma_bf16_ts(tmem + kColDW, ea + 8, xmn, I64, 1);
                tc05::mma_bf16_ts(tmem + kColDB, ea, d_one8, I8, 0);
                tc05::mma_bf16_ts(tmem + kColDB, ea + 8, d_one8, I8, 1);
                tc05::commit(ptx::smem_addr(&s.dw_full));
                tc05::commit(ptx::smem_addr(&s.e_empty[e]));
                tc05::commit(ptx::smem_addr(&s.in_empty[c % NS]));
                TTT_STAMP(g_hybrid_timeline, tl_lead, 6, c, 3);
            }
            // drain: wait (bounded) for every MMA issued so far before TMEM is freed
            tc05::commit(ptx::smem_addr(&s.drain));
            const long long t0 = clock64();
            while (!ptx::mbar_try_wait(&s.drain, 0)) {
                if (clock64() - t0 > 4 * kTimeoutCycles) {
                    atomicOr(&g_hybrid_error_word, 4u);
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
        {   // row means over the output features, removed from the state during the scan
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
        // W~^T rows r0, r1 in the C-fragment layout of a [16 x 64] tile: [4 j + 0..3] =
        // (r0, k), (r0, k+1), (r1, k), (r1, k+1) with k = 8 j + 2 t4
        float Wt[32];
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int k = 8 * j + 2 * t4;
            const float u0 = s.u[k], u1 = s.u[k + 1];
            Wt[4 * j + 0] = W0b[k * D + f0] - u0;
            Wt[4 * j + 1] = W0b[(k + 1) * D + f0] - u1;
            Wt[4 * j + 2] = W0b[k * D + f1] - u0;
            Wt[4 * j + 3] = W0b[(k + 1) * D + f1] - u1;
        }
        float bias0 = b0[(size_t)bh * D + f0] - s.u[D], bias1 = b0[(size_t)bh * D + f1] - s.u[D];
        // The same registers as A fragments of W~^T (rows r0/r1, k = input features) for k step ks:
        // a0 = (r0, 16ks + 2t4..) = Wt[8ks + 0, 1], a1 = (r1, ..) = Wt[8ks + 2, 3],
        // a2 = (r0, 16ks + 8 + 2t4..) = Wt[8ks + 4, 5], a3 = (r1, ..) = Wt[8ks + 6, 7]
        uint32_t wh[16], wl[16];
        auto split_state = [&]() {
#pragma unroll
            for (int i = 0; i < 16; i++) ptx::split_pair_trunc(Wt[2 * i], Wt[2 * i + 1], wh[i], wl[i]);
        };
        // acc (rows r0/r1 x 16 tokens) = W~^T [tile]^T + bias for a [16][64] token tile
        auto product = [&](uint32_t tile, float (&acc)[2][4]) {
            float lo[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; nt++) {
                acc[nt][0] = acc[nt][1] = bias0;
                acc[nt][2] = acc[nt][3] = bias1;
#pragma unroll
                for (int r = 0; r < 4; r++) lo[nt][r] = 0.f;
            }
            const int mi = lane >> 3;
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                uint32_t b[4];  // tokens as n, input features as k
                const int row = (mi >> 1) * 8 + (lane & 7), chunk = 2 * ks + (mi & 1);
                ptx::ldsm_x4(tile + swz_chunk(row, chunk), b[0], b[1], b[2], b[3]);
#pragma unroll
                for (int nt = 0; nt < 2; nt++) {
                    ptx::mma_bf16(acc[nt], wh[4 * ks], wh[4 * ks + 1], wh[4 * ks + 2], wh[4 * ks + 3], b[2 * nt],
                                  b[2 * nt + 1]);
                    ptx::mma_bf16(lo[nt], wl[4 * ks], wl[4 * ks + 1], wl[4 * ks + 2], wl[4 * ks + 3], b[2 * nt],
                                  b[2 * nt + 1]);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 2; nt++)
#pragma unroll
                for (int r = 0; r < 4; r++) acc[nt][r] += lo[nt][r];
        };
        auto store_frag = [&](float4 (&dst)[2], const float (&acc)[2][4]) {
            dst[0] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
            dst[1] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
        };
        const uint32_t tq = tmem + tc05::taddr_lane(32 * q);
        split_state();
        // R_0 = X~_0 W~_0 and R_1 = X~_1 W~_0 (no corrections); the pre slots of chunks 0 and 1 are
        // never read by this role
        for (int j = 0; j < 2 && j < n; j++) {
            wait_k(&s.in_full[j % NS], j / NS, abort_flag);
            float acc[2][4];
            product(ptx::smem_addr(s.st[j % NS].K), acc);
            store_frag(s.rbuf[j % NR][q][lane], acc);
            arrive1(&s.r_full[j % NR], lane);
        }
        for (int j = 0; j < 2 && j < n; j++) arrive1(&s.pre_empty[j % NPRE], lane);
        for (int c = 0; c < n; c++) {
            // ---- P_{c+2} = X~_{c+2} W~_c, before E_c is known
            TTT_STAMP(g_hybrid_timeline, tl_lead, 1, c, 0);
            float racc[2][4];
            const bool has_r = c + 2 < n;
            if (has_r) {
                wait_k(&s.in_full[(c + 2) % NS], (c + 2) / NS, abort_flag);
                product(ptx::smem_addr(s.st[(c + 2) % NS].K), racc);
            }
            // ---- Q~_c W~_c for the output warps
            TTT_STAMP(g_hybrid_timeline, tl_lead, 1, c, 1);
            {
                float qacc[2][4];
                product(ptx::smem_addr(s.st[c % NS].Q), qacc);
                if (c >= NQ) wait_k(&s.q_empty[c % NQ], c / NQ - 1, abort_flag);
                store_frag(s.qwbuf[c % NQ][q][lane], qacc);
                arrive1(&s.q_full[c % NQ], lane);
                arrive1(&s.in_empty[c % NS], lane);  // last use of stage c (K_c was read two chunks ago)
            }
            // ---- E_c: R_{c+2} += E_c^T S2_{c+2}^T
            TTT_STAMP(g_hybrid_timeline, tl_lead, 1, c, 2);
            wait_k(&s.e_full[c % NE], c / NE, abort_flag);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 1, c, 3);
            if (has_r) {
                const int p = (c + 2) % NPRE;
                tc05::fence_after_sync();
                uint32_t eh[4], el[4];
                ld_e_frags(tq + kColE + 16 * (c % NE), eh);
                ld_e_frags(tq + kColE + 16 * (c % NE) + 8, el);
                wait_k(&s.pre_full[p], (c + 2) / NPRE, abort_flag);
                const uint4 sh = s.pre[p].s2[0][lane], sl = s.pre[p].s2[1][lane];
                tc05::wait_ld();
                tc05::fence_before_sync();
                arrive1(&s.e_empty[c % NE], lane);
                arrive1(&s.pre_empty[p], lane);
                mma_16x16(racc, eh, el, sh, sl);
                if (c + 2 >= NR) wait_k(&s.r_empty[(c + 2) % NR], (c + 2) / NR - 1, abort_flag);
                store_frag(s.rbuf[(c + 2) % NR][q][lane], racc);
                arrive1(&s.r_full[(c + 2) % NR], lane);
            } else {
                arrive1(&s.e_empty[c % NE], lane);
            }
            // ---- W~_{c+1} = W~_c + U_c
            TTT_STAMP(g_hybrid_timeline, tl_lead, 1, c, 4);
            wait_k(&s.dw_full, c, abort_flag);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 1, c, 5);
            tc05::fence_after_sync();
            float dv[32], db[4];
            tc05::ld_16x256b_x8(tq + kColDW, dv);
            tc05::ld_16x256b_x1(tq + kColDB, db);
            tc05::wait_ld();
            tc05::fence_before_sync();
            arrive1(&s.dw_empty, lane);
#pragma unroll
            for (int i = 0; i < 32; i += 2) ptx::add2(Wt[i], Wt[i + 1], dv[i], dv[i + 1]);
            // the bias column (64) of the increment sits in the t4 == 0 lanes of each row
            bias0 += __shfl_sync(0xffffffffu, db[0], lane & ~3);
            bias1 += __shfl_sync(0xffffffffu, db[2], lane & ~3);
            if (c + 1 < n) split_state();
            TTT_STAMP(g_hybrid_timeline, tl_lead, 1, c, 6);
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
            b_T[(size_t)bh * D + f0] = bias0 + s.u[D];
            b_T[(size_t)bh * D + f1] = bias1 + s.u[D];
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
            const float4 ra = s.rbuf[rb][w][lane][0], rb4 = s.rbuf[rb][w][lane][1];
            y[0][0] = ra.x; y[0][1] = ra.y; y[0][2] = ra.z; y[0][3] = ra.w;
            y[1][0] = rb4.x; y[1][1] = rb4.y; y[1][2] = rb4.z; y[1][3] = rb4.w;
            arrive1(&s.r_empty[rb], lane);
            wait_k(&s.pre_full[p], c / NPRE, abort_flag);
            const PreSlot& ps = s.pre[p];
            const float4 ga = ps.gc[w][lane][0], gb = ps.gc[w][lane][1];
            gc[0] = ga.x; gc[1] = ga.y; gc[2] = ga.z; gc[3] = ga.w;
            gc[4] = gb.x; gc[5] = gb.y; gc[6] = gb.z; gc[7] = gb.w;
            s1h = ps.s1[0][lane];
            s1l = ps.s1[1][lane];
            c0_my = ps.c0[my_tok];
            eta_my = ps.eta[my_tok];
            arrive1(&s.pre_empty[p], lane);
        };
        if (n > 0) load_inputs(0);
        for (int c = 0; c < n; c++) {
            const int b = c & 1;
            TTT_STAMP(g_hybrid_timeline, tl_lead, 0, c, 0);
            if (c > 0) mma_16x16(y, ah, al, s1h, s1l);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 0, c, 1);
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
            TTT_STAMP(g_hybrid_timeline, tl_lead, 0, c, 2);
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
            // E_c as A fragments (rows r0/r1, k = tokens), kept for the next chunk and written into TMEM
            ptx::split_pair_trunc(E[0][0], E[0][1], ah[0], al[0]);
            ptx::split_pair_trunc(E[0][2], E[0][3], ah[1], al[1]);
            ptx::split_pair_trunc(E[1][0], E[1][1], ah[2], al[2]);
            ptx::split_pair_trunc(E[1][2], E[1][3], ah[3], al[3]);
            const int eb = c % NE;
            TTT_STAMP(g_hybrid_timeline, tl_lead, 0, c, 3);
            if (c >= NE) wait_k(&s.e_empty[eb], c / NE - 1, abort_flag);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 0, c, 4);
            tc05::fence_after_sync();
            const uint32_t ea = tq + kColE + 16 * eb;
            tc05::st_16x128b_x2(ea, ah[0], ah[1], ah[2], ah[3]);
            tc05::st_16x128b_x2(ea + 8, al[0], al[1], al[2], al[3]);
            tc05::wait_st();
            tc05::fence_before_sync();
            arrive1(&s.e_full[eb], lane);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 0, c, 5);
            if (c + 1 < n) load_inputs(c + 1);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 0, c, 6);
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
            const int b = c & 1, slot = c % NS, p = c % NPRE;
            float z[2][4];
            TTT_STAMP(g_hybrid_timeline, tl_lead, 2, c, 0);
            wait_k(&s.q_full[c % NQ], c / NQ, abort_flag);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 2, c, 1);
            {
                const float4 za = s.qwbuf[c % NQ][q][lane][0], zb = s.qwbuf[c % NQ][q][lane][1];
                z[0][0] = za.x; z[0][1] = za.y; z[0][2] = za.z; z[0][3] = za.w;
                z[1][0] = zb.x; z[1][1] = zb.y; z[1][2] = zb.z; z[1][3] = zb.w;
            }
            arrive1(&s.q_empty[c % NQ], lane);
            // zbar_c += E_c^T L_c^T
            wait_k(&s.e_full[c % NE], c / NE, abort_flag);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 2, c, 2);
            tc05::fence_after_sync();
            uint32_t eh[4], el[4];
            ld_e_frags(tq + kColE + 16 * (c % NE), eh);
            ld_e_frags(tq + kColE + 16 * (c % NE) + 8, el);
            wait_k(&s.pre_full[p], c / NPRE, abort_flag);
            const uint4 lh = s.pre[p].l[0][lane], ll = s.pre[p].l[1][lane];
            tc05::wait_ld();
            tc05::fence_before_sync();
            arrive1(&s.e_empty[c % NE], lane);
            arrive1(&s.pre_empty[p], lane);
            mma_16x16(z, eh, el, lh, ll);
            // [slot = 2 nt + e][sum, sum of squares] over this thread's two features
            float v[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const float a = z[i >> 1][i & 1], bb = z[i >> 1][2 + (i & 1)];
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
            TTT_STAMP(g_hybrid_timeline, tl_lead, 2, c, 3);
            ptx::named_bar_sync(2, 4 * 32);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 2, c, 4);
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
                    o.x = ptx::bf16_lo_f32(qv) + fmaf(gm0 * (z[nt][e] - cf.x), cf.y, bt0);
                    o.y = ptx::bf16_hi_f32(qv) + fmaf(gm1 * (z[nt][2 + e] - cf.x), cf.y, bt1);
                    *reinterpret_cast<float2*>(Zbh + (size_t)(c * kChunk + tok) * D + f0) = o;
                }
            arrive1(&s.in_empty[slot], lane);
            TTT_STAMP(g_hybrid_timeline, tl_lead, 2, c, 5);
        }
    }

    // ---------------------------------------------------------------- tear-down
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    if (warp == kWarpMMA) tc05::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

bool linear_hybrid_supports(const LinearArgs& a) {
    return a.d == D && a.dtype == TTT_BF16 && a.mode == TTT_LN_RESIDUAL && a.mini_batch == kChunk && a.T > 0 &&
           a.T % kChunk == 0;
}

cudaError_t launch_linear_hybrid(const LinearArgs& a, cudaStream_t stream) {
    if (!linear_hybrid_supports(a)) return cudaErrorInvalidValue;
    const int BH = a.B * a.H;
    CUtensorMap mk, mv, mq, me;
    if (!make_token_tile_map(&mk, a.K, a.T, BH) || !make_token_tile_map(&mv, a.V, a.T, BH) ||
        !make_token_tile_map(&mq, a.Q, a.T, BH) || !make_eta_row_map(&me, a.eta, a.T, BH))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(HybSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(ttt_linear_hybrid_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    ttt_linear_hybrid_kernel<<<BH, kThreads, smem, stream>>>(mk, mv, mq, me, a.T, a.H, a.ln_eps, a.W0, a.b0,
                                                              a.gamma, a.beta, a.Z, a.W_T, a.b_T, drop_chunk_hook());
    return cudaPeekAtLastError();
}

#ifdef TTT_TIMELINE
cudaError_t read_hybrid_timeline(long long* out) {
    return cudaMemcpyFromSymbol(out, g_hybrid_timeline, sizeof(g_hybrid_timeline));
}
#endif

cudaError_t read_and_clear_hybrid_error(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_hybrid_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_hybrid_error_word, &zero, sizeof(unsigned int));
}

}  // namespace ttt
