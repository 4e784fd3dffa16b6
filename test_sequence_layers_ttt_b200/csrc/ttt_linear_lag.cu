// Tensor-core TTT-Linear forward scan for sm_100a, lag-1 dual form.
//
// Scope: bf16 Q/K/V, d = 64, f(x) = x + LN(x W + b), mini-batch b = 16, T a
// multiple of 16.  One CTA per (batch, head) runs the whole sequence.
//
// Method ("Learning to (Learn at Test Time)", literature record, Key
// takeaways bullets 1, 2 and 5).  Write W~ = [W; b] (65 x 64) and x~ = [x, 1],
// so f's pre-activation is x~ W~.  With W~_c the state at the start of chunk c
// (16 tokens, one mini-batch), X = K_c:
//   Y_c      = X~_c W~_c
//   G_c      = dl/dY_c (LayerNorm backward of ||X + LN(Y) - V||^2, per token)
//   W~_{c+1} = W~_c - X~_c^T diag(eta_c) G_c
//   zbar_c   = Q~_c W~_c + L_c E_c,  E_c = -diag(eta_c) G_c,  L_c[t,s] = q_t . x_s + 1, s <= t
//   z_c      = q + LN(zbar_c)
// Substituting the update once gives the lag-1 form used here:
//   Y_c = P_c + M_c G_{c-1},  P_c = X~_c W~_{c-1},
//   M_c = -(X_c X_{c-1}^T + 1) diag(eta_{c-1})                       (16 x 16)
// so the sequential chain per chunk is only the 16x16x64 product M_c G_{c-1},
// the LayerNorm statistics and G_c; the 16x64x64 products with W~ run one
// chunk ahead on other warps.
//
// Warp roles (480 threads):
//   CH  warps 0-3   the chain: warp w owns output features [16w, 16w+16);
//                   keeps G_c as bf16 hi/lo B fragments in registers (8x8
//                   transposes, movmatrix) and hands E_c = -eta G_c on as fp32
//                   through a ring of four buffers; the consumers split it
//                   themselves, so no tile packing sits on the chain
//   WP  warps 4-7   the state: warp w keeps rows [16w, 16w+16) of W~^T (all
//                   65 input columns, the last one the bias) as fp32 mma
//                   accumulators; applies the update with E_{c-1}, splits the
//                   state into bf16 hi/lo B fragments, forms P_{c+1} and hands
//                   the fragments to the output warps
//   OW  warps 8-11  the output: zbar = Q~W~ (from the state warps' fragments)
//                   + L E, LayerNorm, residual, store
//   PR  warp 12     TMA loads of K, V, Q (128-byte swizzled tiles) and eta
//   PA  warp 13     per-chunk inputs of the chain: g.c', its row sums, eta
//   PB  warp 14     M_c (eta folded in) and L_c (16 x 16 tensor-core products)
// Every product with an fp32 operand splits it into bf16 hi + lo terms
// (both rounded to nearest: relative error at most 2^-16); bf16 inputs are
// exact; accumulation is fp32.
// The state is kept centred on its per-input-row means over the output
// features (added back to W_T, b_T at the end), so y = x W + b has a mean near
// zero and the one-pass LayerNorm variance does not cancel.
// The W-free inputs run up to NPRE chunks ahead in a ring, and Q~W~ is handed
// to the output warps through four buffers, so the slower output path does
// not hold back the chain's inputs.
// Hand-offs between roles are mbarriers with bounded waits: after about a
// second without progress the kernel records an error word, stops waiting and
// drains its TMA loads (outputs undefined; TTT_ERR_TIMEOUT with TTT_CHECK=1).
#include <cstdlib>

#include "common.cuh"
#include "ptx.cuh"
#include "timeline.cuh"
#include "tma_host.h"
#include "ttt_internal.h"

namespace ttt {

// set by kernels that abandon a bounded wait; read (and cleared) by the host with TTT_CHECK=1
__device__ unsigned int g_ttt_error_word = 0;

TTT_TIMELINE_BUFFER(g_lag_timeline);  // roles: 0 CH, 1 WP, 2 OW, 3 PR, 4 PA, 5 PB

namespace {

constexpr int D = 64;
constexpr int NS = 8;            // TMA ring stages
constexpr int NPRE = 8;          // ring of the chain's and output's W-free inputs
constexpr int NGB = 4;           // ring of E_c hand-offs (chain -> state and output warps)
constexpr int kEStride = D + 8;  // fp32 row stride of an E_c buffer (spreads the rows over the banks)
constexpr int kCH = 4, kWP = 4, kOW = 4;
constexpr int kWarpWP0 = kCH, kWarpOW0 = kCH + kWP, kWarpPR = kCH + kWP + kOW;
constexpr int kWarpPA = kWarpPR + 1, kWarpPB = kWarpPR + 2;
constexpr int kWarps = kWarpPB + 1;
constexpr int kThreads = kWarps * 32;
constexpr int TILE = kChunk * D * 2;
constexpr uint32_t kStageTx = 3 * TILE + kChunk * 4;
constexpr long long kTimeoutCycles = 2000000000LL;
constexpr uint32_t kOnesBf16x2 = 0x3f803f80u;  // (1.0, 1.0) in bf16

struct LagSmem {
    unsigned char K[NS][TILE];
    unsigned char V[NS][TILE];
    unsigned char Q[NS][TILE];
    float Ef[NGB][kChunk][kEStride];        // [buf][tok][out] E_c = -eta G_c, fp32
    float4 pbuf[2][kCH][32][2];             // [buf][w][lane]: P_c fragments (8 floats)
    uint4 wsplit[2][kWP][9][32];            // [j % 2][warp][group][lane]: W~_j hi (0-3), lo (4-7) B fragments
                                            // and the bias row of the accumulator (8), for the output warps
    float4 gcbuf[NPRE][kCH][32][2];         // g * (x + beta - v) in chain fragment order
    uint4 mfrag[NPRE][2][32];               // [c % NPRE][hi, lo] -M_c as A fragments
    uint4 afrag[NPRE][2][32];               // [c % NPRE][hi, lo] L_c as A fragments
    float c0[NPRE][kChunk];                 // row sums of g * c'
    float etac[NPRE][kChunk];               // eta of the chunk, for the chain
    alignas(128) float eta[NS][32];
    float red_ch[2][kChunk][5][4];          // [buf][tok][sum][warp]
    float red_ow[2][kChunk][12];            // [buf][tok][2 sums x 4 warps + pad]
    float gam[D], bet[D];
    float u[D + 1];                         // per-input-row means removed from the state (row D: bias)
    uint64_t in_full[NS], in_empty[NS];
    uint64_t pre_full[NPRE], pre_empty[NPRE], p_full[2], p_empty[2];
    uint64_t g_full[NGB], g_empty[NGB], qw_full[4], qw_empty[4];
    int abort_flag;
};

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
            atomicOr(&g_ttt_error_word, 1u);
            return false;
        }
    }
}
// wait for use number `k` (0-based) of a double-buffered barrier pair
__device__ __forceinline__ void wait_use(uint64_t* bar, int k, volatile int* abort_flag) {
    wait_bounded(bar, (uint32_t)(k & 1), abort_flag);
}
__device__ __forceinline__ void arrive1(uint64_t* bar, int lane) {
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar);
}
// acc (16 tokens x 16 output features) = [16][64] token tile x W~ B fragments (hi + lo), starting
// from the bias row br = (col 2t, col 2t+1 of n-tile 0, the same of n-tile 1)
__device__ __forceinline__ void tile_product(uint32_t tile_addr, int lane, const uint32_t (&wh)[8][2],
                                             const uint32_t (&wl)[8][2], float4 br, float (&acc)[2][4]) {
    acc[0][0] = acc[0][2] = br.x;
    acc[0][1] = acc[0][3] = br.y;
    acc[1][0] = acc[1][2] = br.z;
    acc[1][1] = acc[1][3] = br.w;
    const int mi = lane >> 3;
#pragma unroll
    for (int ks = 0; ks < 4; ks++) {
        const int row = (mi & 1) * 8 + (lane & 7), chunk = 2 * ks + (mi >> 1);
        uint32_t a0, a1, a2, a3;
        ptx::ldsm_x4(tile_addr + swz_chunk(row, chunk), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < 2; nt++) {
            ptx::mma_bf16(acc[nt], a0, a1, a2, a3, wh[2 * ks][nt], wh[2 * ks + 1][nt]);
            ptx::mma_bf16(acc[nt], a0, a1, a2, a3, wl[2 * ks][nt], wl[2 * ks + 1][nt]);
        }
    }
}
// E_c (fp32 [tok][out]) at output features f0 = 16w + g and f0 + 8, as bf16 hi/lo pairs of tokens:
// [0] (f0, tokens 2t, 2t+1), [1] (f0 + 8, 2t, 2t+1), [2] (f0, 2t+8, 2t+9), [3] (f0 + 8, 2t+8, 2t+9).
// These are the A fragments of E^T (rows = features, k = tokens) and, reordered, the B fragments of
// E (k = tokens, n = features) for the n-tiles at f0 and f0 + 8.
__device__ __forceinline__ void load_e_pairs(const float (*E)[kEStride], int f0, int t, uint32_t (&hi)[4],
                                             uint32_t (&lo)[4]) {
    const int k0 = 2 * t;
    ptx::split_pair_rn(E[k0][f0], E[k0 + 1][f0], hi[0], lo[0]);
    ptx::split_pair_rn(E[k0][f0 + 8], E[k0 + 1][f0 + 8], hi[1], lo[1]);
    ptx::split_pair_rn(E[k0 + 8][f0], E[k0 + 9][f0], hi[2], lo[2]);
    ptx::split_pair_rn(E[k0 + 8][f0 + 8], E[k0 + 9][f0 + 8], hi[3], lo[3]);
}


// kCkpt: the checkpoint pass of the layer backward.  The state warps store the state at the
// start of every chunk (W_j [in][out], then b_j, row means added back) at ckpt + (bh n + j) (d^2 + d);
// no Z and no final state are written, and the output warps only keep the hand-off protocol.
template <bool kCkpt>
__global__ void __launch_bounds__(kThreads, 1)
ttt_linear_lag_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmEta,
                      int T, int H, float eps, const float* W0, const float* b0,
                      const float* __restrict__ gamma, const float* __restrict__ beta,
                      float* __restrict__ Z, float* W_T, float* b_T, int drop_chunk, float* __restrict__ ckpt) {
    extern __shared__ unsigned char smem_raw[];
    // 1024-byte alignment (128-byte TMA swizzle) by offsetting the shared array itself, so every
    // access through `s` stays a shared-memory access (an integer round trip would make them generic)
    LagSmem& s = *reinterpret_cast<LagSmem*>(smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int bh = blockIdx.x, h = bh % H;
    const int n = T / kChunk;
    volatile int* abort_flag = &s.abort_flag;
    const bool tl_lead = (tid & 31) == 0 && (warp == 0 || warp == kWarpWP0 || warp == kWarpOW0 || warp >= kWarpPR);
    (void)tl_lead;
    TTT_TIMELINE_SMEM();

    if (tid < D) {
        s.gam[tid] = gamma[h * D + tid];
        s.bet[tid] = beta[h * D + tid];
    }
    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < NS; i++) {
            ptx::mbar_init(&s.in_full[i], 1);
            ptx::mbar_init(&s.in_empty[i], 2 + kWP + kOW);  // PA, PB, WP, OW
        }
        for (int i = 0; i < NPRE; i++) {
            ptx::mbar_init(&s.pre_full[i], 2);            // PA, PB
            ptx::mbar_init(&s.pre_empty[i], kCH + kOW);
        }
        for (int i = 0; i < 2; i++) {
            ptx::mbar_init(&s.p_full[i], kWP);
            ptx::mbar_init(&s.p_empty[i], kCH);
            ptx::mbar_init(&s.qw_full[i], kWP);
            ptx::mbar_init(&s.qw_empty[i], kOW);
            ptx::mbar_init(&s.qw_full[i + 2], kWP);
            ptx::mbar_init(&s.qw_empty[i + 2], kOW);
        }
        for (int i = 0; i < NGB; i++) {
            ptx::mbar_init(&s.g_full[i], kCH);
            ptx::mbar_init(&s.g_empty[i], kWP + kOW);
        }
        ptx::fence_mbar_init();
    }
    __syncthreads();

    // ================================================================ producer
    if (warp == kWarpPR) {
        if (lane == 0) {
            ptx::prefetch_tmap(&tmK);
            ptx::prefetch_tmap(&tmV);
            ptx::prefetch_tmap(&tmQ);
            ptx::prefetch_tmap(&tmEta);
            int issued = 0;
            for (int c = 0; c < n; c++) {
                const int slot = c % NS;
                TTT_STAMP(g_lag_timeline, tl_lead, 3, c, 0);
                if (c >= NS && !wait_bounded(&s.in_empty[slot], ((c / NS) - 1) & 1, abort_flag)) break;
                TTT_STAMP(g_lag_timeline, tl_lead, 3, c, 1);
                if (c == drop_chunk) continue;  // fault-injection hook: this chunk is never loaded
                ptx::mbar_arrive_expect_tx(&s.in_full[slot], kStageTx);
                ptx::tma_load_3d(s.K[slot], &tmK, &s.in_full[slot], 0, c * kChunk, bh);
                ptx::tma_load_3d(s.V[slot], &tmV, &s.in_full[slot], 0, c * kChunk, bh);
                ptx::tma_load_3d(s.Q[slot], &tmQ, &s.in_full[slot], 0, c * kChunk, bh);
                ptx::tma_load_2d(s.eta[slot], &tmEta, &s.in_full[slot], c * kChunk, bh);
                issued = c + 1;
            }
            for (int c = issued - 1; c >= 0 && c >= issued - NS; c--) {  // drain own loads
                if (c == drop_chunk) continue;
                const long long t0 = clock64();
                while (!ptx::mbar_try_wait(&s.in_full[c % NS], (c / NS) & 1)) {
                    if (clock64() - t0 > 4 * kTimeoutCycles) {
                        atomicOr(&g_ttt_error_word, 2u);
                        break;
                    }
                }
            }
        }
        TTT_TIMELINE_FLUSH(g_lag_timeline, tl_lead, 3);
        return;
    }

    // ================================================================ PA: g * (x + beta - v), row sums
    if (warp == kWarpPA) {
        for (int c = 0; c < n; c++) {
            const int slot = c % NS, b = c % NPRE;
            TTT_STAMP(g_lag_timeline, tl_lead, 4, c, 0);
            wait_bounded(&s.in_full[slot], (c / NS) & 1, abort_flag);
            TTT_STAMP(g_lag_timeline, tl_lead, 4, c, 1);
            if (c >= NPRE) wait_use(&s.pre_empty[b], c / NPRE - 1, abort_flag);
            TTT_STAMP(g_lag_timeline, tl_lead, 4, c, 2);
            float rs0 = 0.f, rs1 = 0.f;  // row g, row g + 8
#pragma unroll
            for (int w = 0; w < kCH; w++) {
                float v8[8];
#pragma unroll
                for (int rh = 0; rh < 2; rh++)
#pragma unroll
                    for (int nt = 0; nt < 2; nt++) {
                        const int row = 8 * rh + g, col = 16 * w + 8 * nt + 2 * t;
                        const uint32_t xv = *reinterpret_cast<const uint32_t*>(s.K[slot] + swz(row, col));
                        const uint32_t vv = *reinterpret_cast<const uint32_t*>(s.V[slot] + swz(row, col));
                        const float e0 = s.gam[col] * (ptx::bf16_lo_f32(xv) + s.bet[col] - ptx::bf16_lo_f32(vv));
                        const float e1 = s.gam[col + 1] * (ptx::bf16_hi_f32(xv) + s.bet[col + 1] - ptx::bf16_hi_f32(vv));
                        v8[rh * 4 + nt * 2] = e0;
                        v8[rh * 4 + nt * 2 + 1] = e1;
                        if (rh == 0) rs0 += e0 + e1; else rs1 += e0 + e1;
                    }
                s.gcbuf[b][w][lane][0] = make_float4(v8[0], v8[1], v8[2], v8[3]);
                s.gcbuf[b][w][lane][1] = make_float4(v8[4], v8[5], v8[6], v8[7]);
            }
            rs0 += __shfl_xor_sync(0xffffffffu, rs0, 1);
            rs0 += __shfl_xor_sync(0xffffffffu, rs0, 2);
            rs1 += __shfl_xor_sync(0xffffffffu, rs1, 1);
            rs1 += __shfl_xor_sync(0xffffffffu, rs1, 2);
            if (t == 0) {
                s.c0[b][g] = rs0;
                s.c0[b][g + 8] = rs1;
            }
            if (lane < kChunk) s.etac[b][lane] = s.eta[slot][lane];
            arrive1(&s.pre_full[b], lane);
            arrive1(&s.in_empty[slot], lane);
            TTT_STAMP(g_lag_timeline, tl_lead, 4, c, 3);
        }
        TTT_TIMELINE_FLUSH(g_lag_timeline, tl_lead, 4);
        return;
    }

    // ================================================================ PB: M_c and A_c
    if (warp == kWarpPB) {
        for (int c = 0; c < n; c++) {
            const int slot = c % NS, b = c % NPRE;
            TTT_STAMP(g_lag_timeline, tl_lead, 5, c, 0);
            wait_bounded(&s.in_full[slot], (c / NS) & 1, abort_flag);
            TTT_STAMP(g_lag_timeline, tl_lead, 5, c, 1);
            if (c >= NPRE) wait_use(&s.pre_empty[b], c / NPRE - 1, abort_flag);
            TTT_STAMP(g_lag_timeline, tl_lead, 5, c, 2);
            const uint32_t xs = ptx::smem_addr(s.K[slot]);
            const uint32_t qs = ptx::smem_addr(s.Q[slot]);
            const int mi = lane >> 3;
            // 16x16 products: pm = X_c X_{c-1}^T, pa = Q_c X_c^T
            float pm[2][4], pa[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; nt++)
#pragma unroll
                for (int r = 0; r < 4; r++) pm[nt][r] = pa[nt][r] = 0.f;
            const int pslot = (c + NS - 1) % NS;
            const uint32_t xps = ptx::smem_addr(s.K[pslot]);
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                uint32_t xa0, xa1, xa2, xa3, qa0, qa1, qa2, qa3, b0, b1, b2, b3, p0, p1, p2, p3;
                {
                    const int row = (mi & 1) * 8 + (lane & 7), chunk = 2 * ks + (mi >> 1);
                    ptx::ldsm_x4(xs + swz_chunk(row, chunk), xa0, xa1, xa2, xa3);
                    ptx::ldsm_x4(qs + swz_chunk(row, chunk), qa0, qa1, qa2, qa3);
                }
                {
                    const int row = (mi >> 1) * 8 + (lane & 7), chunk = 2 * ks + (mi & 1);
                    ptx::ldsm_x4(xs + swz_chunk(row, chunk), b0, b1, b2, b3);    // X_c as B (k = d, n = s)
                    ptx::ldsm_x4(xps + swz_chunk(row, chunk), p0, p1, p2, p3);   // X_{c-1} as B
                }
                ptx::mma_bf16(pa[0], qa0, qa1, qa2, qa3, b0, b1);
                ptx::mma_bf16(pa[1], qa0, qa1, qa2, qa3, b2, b3);
                if (c > 0) {
                    ptx::mma_bf16(pm[0], xa0, xa1, xa2, xa3, p0, p1);
                    ptx::mma_bf16(pm[1], xa0, xa1, xa2, xa3, p2, p3);
                }
            }
            const float* eta_p = s.eta[pslot];
            float nm[2][4], na[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; nt++)
#pragma unroll
                for (int r = 0; r < 4; r++) {
                    const int row = g + 8 * (r >> 1), col = 8 * nt + 2 * t + (r & 1);
                    nm[nt][r] = c > 0 ? -eta_p[col] * (pm[nt][r] + 1.f) : 0.f;
                    na[nt][r] = col <= row ? pa[nt][r] + 1.f : 0.f;
                }
            uint32_t mh[4], ml[4], ah[4], al[4];
            ptx::split_pair_rn(nm[0][0], nm[0][1], mh[0], ml[0]);
            ptx::split_pair_rn(nm[0][2], nm[0][3], mh[1], ml[1]);
            ptx::split_pair_rn(nm[1][0], nm[1][1], mh[2], ml[2]);
            ptx::split_pair_rn(nm[1][2], nm[1][3], mh[3], ml[3]);
            ptx::split_pair_rn(na[0][0], na[0][1], ah[0], al[0]);
            ptx::split_pair_rn(na[0][2], na[0][3], ah[1], al[1]);
            ptx::split_pair_rn(na[1][0], na[1][1], ah[2], al[2]);
            ptx::split_pair_rn(na[1][2], na[1][3], ah[3], al[3]);
            s.mfrag[b][0][lane] = make_uint4(mh[0], mh[1], mh[2], mh[3]);
            s.mfrag[b][1][lane] = make_uint4(ml[0], ml[1], ml[2], ml[3]);
            s.afrag[b][0][lane] = make_uint4(ah[0], ah[1], ah[2], ah[3]);
            s.afrag[b][1][lane] = make_uint4(al[0], al[1], al[2], al[3]);
            arrive1(&s.pre_full[b], lane);
            if (c > 0) arrive1(&s.in_empty[pslot], lane);  // last use of X_{c-1}, eta_{c-1}
            TTT_STAMP(g_lag_timeline, tl_lead, 5, c, 3);
        }
        if (n > 0) arrive1(&s.in_empty[(n - 1) % NS], lane);
        TTT_TIMELINE_FLUSH(g_lag_timeline, tl_lead, 5);
        return;
    }

    // ================================================================ WP: the state
    if (warp >= kWarpWP0 && warp < kWarpOW0) {
        const int w = warp - kWarpWP0;
        const float* W0b = W0 + (size_t)bh * D * D;
        // The state is kept centred on its per-input-row means over the output
        // features (and b on its mean): every row of G sums to zero, so the update
        // leaves these means unchanged, and LayerNorm ignores the per-token shift
        // they add to x W + b.  With y centred, the one-pass variance of the chain
        // and output statistics does not cancel.  The means are added back at the end.
        {
            const int st = tid - kWarpWP0 * 32;
            if (st < D) {
                float acc = 0.f;
                for (int j = 0; j < D; j++) acc += W0b[st * D + j];
                s.u[st] = acc * (1.f / D);
            } else if (st == D) {
                float acc = 0.f;
                for (int j = 0; j < D; j++) acc += b0[(size_t)bh * D + j];
                s.u[D] = acc * (1.f / D);
            }
            ptx::named_bar_sync(3, kWP * 32);
        }
        float Wt[8][4];  // W^T rows 16w+g (+8), input columns 8j + 2t (+1)
#pragma unroll
        for (int jj = 0; jj < 8; jj++) {
            const int in0 = 8 * jj + 2 * t;
            const float u0 = s.u[in0], u1 = s.u[in0 + 1];
            Wt[jj][0] = W0b[in0 * D + 16 * w + g] - u0;
            Wt[jj][1] = W0b[(in0 + 1) * D + 16 * w + g] - u1;
            Wt[jj][2] = W0b[in0 * D + 16 * w + 8 + g] - u0;
            Wt[jj][3] = W0b[(in0 + 1) * D + 16 * w + 8 + g] - u1;
        }
        // bias column (x~ has a trailing 1): accumulator tile whose column 0 is b
        float Bt[4] = {0.f, 0.f, 0.f, 0.f};
        if (t == 0) {
            Bt[0] = b0[(size_t)bh * D + 16 * w + g] - s.u[D];
            Bt[2] = b0[(size_t)bh * D + 16 * w + 8 + g] - s.u[D];
        }
        const uint32_t ones = g == 0 ? kOnesBf16x2 : 0u;

        uint32_t wh[8][2], wl[8][2];  // W~ as bf16 hi/lo B fragments [n-tile of the input dim][nt]
        auto split_w = [&]() {
#pragma unroll
            for (int jj = 0; jj < 8; jj++)
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
                    ptx::split_pair_rn(Wt[jj][2 * nt], Wt[jj][2 * nt + 1], wh[jj][nt], wl[jj][nt]);
        };
        // the accumulator's starting value: the bias of this lane's output columns
        auto bias_row = [&]() {
            return make_float4(__shfl_sync(0xffffffffu, Bt[0], 4 * (2 * t)), __shfl_sync(0xffffffffu, Bt[0], 4 * (2 * t + 1)),
                               __shfl_sync(0xffffffffu, Bt[2], 4 * (2 * t)), __shfl_sync(0xffffffffu, Bt[2], 4 * (2 * t + 1)));
        };
        // rows16 x W~[:, 16w..16w+16) for a [16][64] token tile, bias included
        auto product = [&](uint32_t tile_addr, float4 (&dst)[2]) {
            float acc[2][4];
            tile_product(tile_addr, lane, wh, wl, bias_row(), acc);
            dst[0] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
            dst[1] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
        };
        // W~_j's fragments and bias row for the output warps (same lanes, same 16 output features)
        auto publish = [&](uint4 (*dst)[32]) {
#pragma unroll
            for (int q = 0; q < 4; q++) {
                dst[q][lane] = make_uint4(wh[2 * q][0], wh[2 * q][1], wh[2 * q + 1][0], wh[2 * q + 1][1]);
                dst[4 + q][lane] = make_uint4(wl[2 * q][0], wl[2 * q][1], wl[2 * q + 1][0], wl[2 * q + 1][1]);
            }
            const float4 br = bias_row();
            dst[8][lane] = make_uint4(__float_as_uint(br.x), __float_as_uint(br.y), __float_as_uint(br.z),
                                      __float_as_uint(br.w));
        };

        // the state with its row means added back, as W [in][out] and b
        auto store_state = [&](float* Wd, float* bd) {
#pragma unroll
            for (int jj = 0; jj < 8; jj++) {
                const int in0 = 8 * jj + 2 * t;
                const float u0 = s.u[in0], u1 = s.u[in0 + 1];
                Wd[in0 * D + 16 * w + g] = Wt[jj][0] + u0;
                Wd[(in0 + 1) * D + 16 * w + g] = Wt[jj][1] + u1;
                Wd[in0 * D + 16 * w + 8 + g] = Wt[jj][2] + u0;
                Wd[(in0 + 1) * D + 16 * w + 8 + g] = Wt[jj][3] + u1;
            }
            if (t == 0) {
                bd[16 * w + g] = Bt[0] + s.u[D];
                bd[16 * w + 8 + g] = Bt[2] + s.u[D];
            }
        };
        constexpr size_t kCkptStride = (size_t)D * D + D;
        float* ck = kCkpt ? ckpt + (size_t)bh * n * kCkptStride : nullptr;
        if (kCkpt && n > 0) store_state(ck, ck + D * D);

        split_w();
        // P_0 = X~_0 W~_0 and P_1 = X~_1 W~_0; Q~_0 W~_0
        for (int c = 0; c < 2 && c < n; c++) {
            wait_bounded(&s.in_full[c % NS], (c / NS) & 1, abort_flag);
            product(ptx::smem_addr(s.K[c % NS]), s.pbuf[c][w][lane]);
            arrive1(&s.p_full[c], lane);
        }
        if (n > 0) {
            if (!kCkpt) publish(s.wsplit[0][w]);
            arrive1(&s.qw_full[0], lane);
        }

        for (int j = 1; j <= n; j++) {
            // ---- update with E_{j-1}: W~_j = W~_{j-1} + X~_{j-1}^T E_{j-1}
            const int pb = (j - 1) % NGB, pslot = (j - 1) % NS;
            TTT_STAMP(g_lag_timeline, tl_lead, 1, j, 0);
            wait_use(&s.g_full[pb], (j - 1) / NGB, abort_flag);
            TTT_STAMP(g_lag_timeline, tl_lead, 1, j, 1);
            uint32_t ah[4], al[4];  // E^T: rows = features 16w.., k = tokens
            load_e_pairs(s.Ef[pb], 16 * w + g, t, ah, al);
            // The increment is formed in fresh accumulators and added to the state with fp32
            // adds (round to nearest): the tensor-core accumulation does not round to nearest,
            // and the state takes thousands of increments.
            {
                const uint32_t xs = ptx::smem_addr(s.K[pslot]);
                const int mi = lane >> 3;
#pragma unroll
                for (int jp = 0; jp < 4; jp++) {
                    const int row = (mi & 1) * 8 + (lane & 7), chunk = 2 * jp + (mi >> 1);
                    uint32_t b0, b1, b2, b3;
                    ptx::ldsm_x4_t(xs + swz_chunk(row, chunk), b0, b1, b2, b3);
                    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
                    ptx::mma_bf16(d0, ah[0], ah[1], ah[2], ah[3], b0, b1);
                    ptx::mma_bf16(d0, al[0], al[1], al[2], al[3], b0, b1);
                    ptx::mma_bf16(d1, ah[0], ah[1], ah[2], ah[3], b2, b3);
                    ptx::mma_bf16(d1, al[0], al[1], al[2], al[3], b2, b3);
                    ptx::add2(Wt[2 * jp][0], Wt[2 * jp][1], d0[0], d0[1]);
                    ptx::add2(Wt[2 * jp][2], Wt[2 * jp][3], d0[2], d0[3]);
                    ptx::add2(Wt[2 * jp + 1][0], Wt[2 * jp + 1][1], d1[0], d1[1]);
                    ptx::add2(Wt[2 * jp + 1][2], Wt[2 * jp + 1][3], d1[2], d1[3]);
                }
                // bias column: x~ has a 1 in it for every token
                float db[4] = {0.f, 0.f, 0.f, 0.f};
                ptx::mma_bf16(db, ah[0], ah[1], ah[2], ah[3], ones, ones);
                ptx::mma_bf16(db, al[0], al[1], al[2], al[3], ones, ones);
#pragma unroll
                for (int r = 0; r < 4; r++) Bt[r] += db[r];
            }
            arrive1(&s.g_empty[pb], lane);
            arrive1(&s.in_empty[pslot], lane);
            TTT_STAMP(g_lag_timeline, tl_lead, 1, j, 2);
            if (j == n) break;
            if (kCkpt) store_state(ck + j * kCkptStride, ck + j * kCkptStride + D * D);

            split_w();
            TTT_STAMP(g_lag_timeline, tl_lead, 1, j, 3);
            // ---- P_{j+1} = X~_{j+1} W~_j
            if (j + 1 < n) {
                const int nb = (j + 1) & 1, nslot = (j + 1) % NS;
                wait_bounded(&s.in_full[nslot], ((j + 1) / NS) & 1, abort_flag);
                if (j + 1 >= 2) wait_use(&s.p_empty[nb], ((j + 1) >> 1) - 1, abort_flag);
                TTT_STAMP(g_lag_timeline, tl_lead, 1, j, 4);
                product(ptx::smem_addr(s.K[nslot]), s.pbuf[nb][w][lane]);
                arrive1(&s.p_full[nb], lane);
                TTT_STAMP(g_lag_timeline, tl_lead, 1, j, 5);
            }
            // ---- W~_j for the output warps, which form Q~_j W~_j
            {
                const int qb = j & 1;
                if (j >= 2) wait_use(&s.qw_empty[qb], (j >> 1) - 1, abort_flag);
                TTT_STAMP(g_lag_timeline, tl_lead, 1, j, 6);
                if (!kCkpt) publish(s.wsplit[qb][w]);
                arrive1(&s.qw_full[qb], lane);
                TTT_STAMP(g_lag_timeline, tl_lead, 1, j, 7);
            }
        }

        // final state W~_n
        if (!kCkpt) store_state(W_T + (size_t)bh * D * D, b_T + (size_t)bh * D);
        TTT_TIMELINE_FLUSH(g_lag_timeline, tl_lead, 1);
        return;
    }

    // ================================================================ CH: the chain
    if (warp < kCH) {
        const int w = warp;
        float gam2[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; nt++)
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const float gm = s.gam[16 * w + 8 * nt + 2 * t + e];
                gam2[nt][e] = gm * gm;
            }
        float Gamma = 0.f;
        for (int j = 0; j < D; j++) Gamma += s.gam[j] * s.gam[j];
        const float inv_d = 1.f / D;

        // per-chunk inputs, loaded one chunk ahead
        float R[2][4], gcv[8], c0v[2], etv[2];
        float ngcv[8], nc0v[2], netv[2];
        uint4 mh, ml, nmh, nml;
        auto load_pre = [&](int c) {
            const int b = c % NPRE;
            wait_use(&s.pre_full[b], c / NPRE, abort_flag);
            const float4 g0 = s.gcbuf[b][w][lane][0], g1 = s.gcbuf[b][w][lane][1];
            ngcv[0] = g0.x; ngcv[1] = g0.y; ngcv[2] = g0.z; ngcv[3] = g0.w;
            ngcv[4] = g1.x; ngcv[5] = g1.y; ngcv[6] = g1.z; ngcv[7] = g1.w;
            nc0v[0] = s.c0[b][g];
            nc0v[1] = s.c0[b][g + 8];
            netv[0] = s.etac[b][g];
            netv[1] = s.etac[b][g + 8];
            nmh = s.mfrag[b][0][lane];
            nml = s.mfrag[b][1][lane];
            arrive1(&s.pre_empty[b], lane);
        };
        auto load_inputs = [&](int c) {
            const int b = c & 1;
#pragma unroll
            for (int i = 0; i < 8; i++) gcv[i] = ngcv[i];
            c0v[0] = nc0v[0]; c0v[1] = nc0v[1];
            etv[0] = netv[0]; etv[1] = netv[1];
            mh = nmh; ml = nml;
            wait_use(&s.p_full[b], c >> 1, abort_flag);
            const float4 p0 = s.pbuf[b][w][lane][0], p1 = s.pbuf[b][w][lane][1];
            R[0][0] = p0.x; R[0][1] = p0.y; R[0][2] = p0.z; R[0][3] = p0.w;
            R[1][0] = p1.x; R[1][1] = p1.y; R[1][2] = p1.z; R[1][3] = p1.w;
            arrive1(&s.p_empty[b], lane);
        };

        uint32_t gbh[4] = {0u, 0u, 0u, 0u}, gbl[4] = {0u, 0u, 0u, 0u};  // G_{c-1} as B fragments
        if (n > 0) {
            load_pre(0);
            load_inputs(0);
        }
        for (int c = 0; c < n; c++) {
            const int b = c & 1;
            TTT_STAMP(g_lag_timeline, tl_lead, 0, c, 0);
            float y[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; nt++)
#pragma unroll
                for (int r = 0; r < 4; r++) y[nt][r] = R[nt][r];
            if (c > 0) {
                ptx::mma_bf16(y[0], mh.x, mh.y, mh.z, mh.w, gbh[0], gbh[1]);
                ptx::mma_bf16(y[1], mh.x, mh.y, mh.z, mh.w, gbh[2], gbh[3]);
                ptx::mma_bf16(y[0], mh.x, mh.y, mh.z, mh.w, gbl[0], gbl[1]);
                ptx::mma_bf16(y[1], mh.x, mh.y, mh.z, mh.w, gbl[2], gbl[3]);
                ptx::mma_bf16(y[0], ml.x, ml.y, ml.z, ml.w, gbh[0], gbh[1]);
                ptx::mma_bf16(y[1], ml.x, ml.y, ml.z, ml.w, gbh[2], gbh[3]);
            }
            TTT_STAMP(g_lag_timeline, tl_lead, 0, c, 1);
            const float* gcc = gcv;
            const float* c0c = c0v;

            // fused LayerNorm statistics: sums of y, y^2, g^2 y, g^2 y^2, g c' y per token
            float sm[2][5];
#pragma unroll
            for (int rh = 0; rh < 2; rh++) {
#pragma unroll
                for (int q = 0; q < 5; q++) sm[rh][q] = 0.f;
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const float yy = y[nt][2 * rh + e];
                        const float a = gam2[nt][e] * yy;
                        sm[rh][0] += yy;
                        sm[rh][1] = fmaf(yy, yy, sm[rh][1]);
                        sm[rh][2] += a;
                        sm[rh][3] = fmaf(a, yy, sm[rh][3]);
                        sm[rh][4] = fmaf(gcc[rh * 4 + nt * 2 + e], yy, sm[rh][4]);
                    }
#pragma unroll
                for (int q = 0; q < 5; q++) {
                    sm[rh][q] += __shfl_xor_sync(0xffffffffu, sm[rh][q], 1);
                    sm[rh][q] += __shfl_xor_sync(0xffffffffu, sm[rh][q], 2);
                }
            }
            if (t == 0) {
#pragma unroll
                for (int rh = 0; rh < 2; rh++)
#pragma unroll
                    for (int q = 0; q < 5; q++) s.red_ch[b][8 * rh + g][q][w] = sm[rh][q];
            }
            ptx::named_bar_sync(1, kCH * 32);
            TTT_STAMP(g_lag_timeline, tl_lead, 0, c, 2);

            float G[2][2][2];  // [rh][nt][e]
#pragma unroll
            for (int rh = 0; rh < 2; rh++) {
                float S[5];
#pragma unroll
                for (int q = 0; q < 5; q++) {
                    const float4 v = *reinterpret_cast<const float4*>(s.red_ch[b][8 * rh + g][q]);
                    S[q] = (v.x + v.y) + (v.z + v.w);
                }
                const float mu = S[0] * inv_d;
                const float var = fmaxf(S[1] * inv_d - mu * mu, 0.f);
                const float rs = rsqrtf(var + eps);
                const float C0 = c0c[rh];
                const float sgx = 2.f * C0 + 2.f * rs * (S[2] - mu * Gamma);
                const float sgxx = 2.f * rs * (S[4] - mu * C0) + 2.f * rs * rs * (S[3] - 2.f * mu * S[2] + mu * mu * Gamma);
                const float k1 = -rs * inv_d * sgx, k2 = -rs * inv_d * sgxx;
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const float xh = (y[nt][2 * rh + e] - mu) * rs;
                        const float gx = 2.f * gcc[rh * 4 + nt * 2 + e] + 2.f * gam2[nt][e] * xh;
                        G[rh][nt][e] = fmaf(gx, rs, fmaf(xh, k2, k1));
                    }
            }
            // G_c back as B fragments for the next chunk (8x8 transposes in registers)
#pragma unroll
            for (int rh = 0; rh < 2; rh++)
#pragma unroll
                for (int nt = 0; nt < 2; nt++) {
                    uint32_t hi, lo;
                    ptx::split_pair_rn(G[rh][nt][0], G[rh][nt][1], hi, lo);
                    gbh[2 * nt + rh] = ptx::movmatrix_t(hi);
                    gbl[2 * nt + rh] = ptx::movmatrix_t(lo);
                }
            // E_c = -eta G_c in fp32 -> the state and output warps, which split it themselves
            TTT_STAMP(g_lag_timeline, tl_lead, 0, c, 3);
            const int gb = c % NGB;
            if (c >= NGB) wait_use(&s.g_empty[gb], c / NGB - 1, abort_flag);
            TTT_STAMP(g_lag_timeline, tl_lead, 0, c, 4);
#pragma unroll
            for (int rh = 0; rh < 2; rh++)
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
                    *reinterpret_cast<float2*>(&s.Ef[gb][8 * rh + g][16 * w + 8 * nt + 2 * t]) =
                        make_float2(-etv[rh] * G[rh][nt][0], -etv[rh] * G[rh][nt][1]);
            __syncwarp();  // every lane's stores before the hand-off
            if (lane == 0) ptx::mbar_arrive(&s.g_full[gb]);
            TTT_STAMP(g_lag_timeline, tl_lead, 0, c, 5);
            // the next chunk's W-free inputs and P, off the chain's path
            if (c + 1 < n) load_pre(c + 1);
            TTT_STAMP(g_lag_timeline, tl_lead, 0, c, 6);
            if (c + 1 < n) load_inputs(c + 1);
            TTT_STAMP(g_lag_timeline, tl_lead, 0, c, 7);
        }
        TTT_TIMELINE_FLUSH(g_lag_timeline, tl_lead, 0);
        return;
    }

    // ================================================================ OW: outputs
    {
        const int w = warp - kWarpOW0;
        float gamv[2][2], betv[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; nt++)
#pragma unroll
            for (int e = 0; e < 2; e++) {
                gamv[nt][e] = s.gam[16 * w + 8 * nt + 2 * t + e];
                betv[nt][e] = s.bet[16 * w + 8 * nt + 2 * t + e];
            }
        if (kCkpt) {
            // no outputs: every hand-off is still waited for and released in order
            for (int c = 0; c < n; c++) {
                const int slot = c % NS, gb = c % NGB;
                wait_use(&s.qw_full[c & 1], c >> 1, abort_flag);
                arrive1(&s.qw_empty[c & 1], lane);
                wait_bounded(&s.in_full[slot], (c / NS) & 1, abort_flag);
                wait_use(&s.pre_full[c % NPRE], c / NPRE, abort_flag);
                arrive1(&s.pre_empty[c % NPRE], lane);
                wait_use(&s.g_full[gb], c / NGB, abort_flag);
                arrive1(&s.g_empty[gb], lane);
                arrive1(&s.in_empty[slot], lane);
            }
            return;
        }
        float* Zbh = Z + (size_t)bh * T * D;
        for (int c = 0; c < n; c++) {
            const int b = c & 1, slot = c % NS;
            float z[2][4];
            TTT_STAMP(g_lag_timeline, tl_lead, 2, c, 0);
            wait_use(&s.qw_full[c & 1], c >> 1, abort_flag);
            TTT_STAMP(g_lag_timeline, tl_lead, 2, c, 1);
            {
                // Q~_c W~_c from the state warps' fragments of W~_c
                uint32_t wh[8][2], wl[8][2];
                const uint4 (*src)[32] = s.wsplit[c & 1][w];
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    const uint4 h = src[q][lane], l = src[4 + q][lane];
                    wh[2 * q][0] = h.x; wh[2 * q][1] = h.y; wh[2 * q + 1][0] = h.z; wh[2 * q + 1][1] = h.w;
                    wl[2 * q][0] = l.x; wl[2 * q][1] = l.y; wl[2 * q + 1][0] = l.z; wl[2 * q + 1][1] = l.w;
                }
                const uint4 bb = src[8][lane];
                arrive1(&s.qw_empty[c & 1], lane);
                wait_bounded(&s.in_full[slot], (c / NS) & 1, abort_flag);
                tile_product(ptx::smem_addr(s.Q[slot]), lane, wh, wl,
                             make_float4(__uint_as_float(bb.x), __uint_as_float(bb.y), __uint_as_float(bb.z),
                                         __uint_as_float(bb.w)), z);
            }
            wait_use(&s.pre_full[c % NPRE], c / NPRE, abort_flag);
            const uint4 ah = s.afrag[c % NPRE][0][lane], al = s.afrag[c % NPRE][1][lane];
            arrive1(&s.pre_empty[c % NPRE], lane);
            TTT_STAMP(g_lag_timeline, tl_lead, 2, c, 2);
            const int gb = c % NGB;
            wait_use(&s.g_full[gb], c / NGB, abort_flag);
            TTT_STAMP(g_lag_timeline, tl_lead, 2, c, 3);
            {
                // zbar += L E: B fragments of E (k = tokens, n = features 16w + 8 nt + g)
                uint32_t eh[4], el[4];
                load_e_pairs(s.Ef[gb], 16 * w + g, t, eh, el);
                ptx::mma_bf16(z[0], ah.x, ah.y, ah.z, ah.w, eh[0], eh[2]);
                ptx::mma_bf16(z[1], ah.x, ah.y, ah.z, ah.w, eh[1], eh[3]);
                ptx::mma_bf16(z[0], ah.x, ah.y, ah.z, ah.w, el[0], el[2]);
                ptx::mma_bf16(z[1], ah.x, ah.y, ah.z, ah.w, el[1], el[3]);
                ptx::mma_bf16(z[0], al.x, al.y, al.z, al.w, eh[0], eh[2]);
                ptx::mma_bf16(z[1], al.x, al.y, al.z, al.w, eh[1], eh[3]);
            }
            arrive1(&s.g_empty[gb], lane);

            float ps[2][2];
#pragma unroll
            for (int rh = 0; rh < 2; rh++) {
                ps[rh][0] = ps[rh][1] = 0.f;
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const float v = z[nt][2 * rh + e];
                        ps[rh][0] += v;
                        ps[rh][1] = fmaf(v, v, ps[rh][1]);
                    }
#pragma unroll
                for (int q = 0; q < 2; q++) {
                    ps[rh][q] += __shfl_xor_sync(0xffffffffu, ps[rh][q], 1);
                    ps[rh][q] += __shfl_xor_sync(0xffffffffu, ps[rh][q], 2);
                }
            }
            if (t == 0) {
#pragma unroll
                for (int rh = 0; rh < 2; rh++)
                    *reinterpret_cast<float2*>(&s.red_ow[b][8 * rh + g][2 * w]) = make_float2(ps[rh][0], ps[rh][1]);
            }
            TTT_STAMP(g_lag_timeline, tl_lead, 2, c, 4);
            ptx::named_bar_sync(2, kOW * 32);
            TTT_STAMP(g_lag_timeline, tl_lead, 2, c, 5);
            TTT_STAMP(g_lag_timeline, tl_lead, 2, c, 6);
#pragma unroll
            for (int rh = 0; rh < 2; rh++) {
                const int row = 8 * rh + g;
                const float4 a = *reinterpret_cast<const float4*>(&s.red_ow[b][row][0]);
                const float4 bb = *reinterpret_cast<const float4*>(&s.red_ow[b][row][4]);
                const float sum = (a.x + a.z) + (bb.x + bb.z);
                const float sq = (a.y + a.w) + (bb.y + bb.w);
                const float mu = sum * (1.f / D);
                const float rs = rsqrtf(fmaxf(sq * (1.f / D) - mu * mu, 0.f) + eps);
                float* zrow = Zbh + (size_t)(c * kChunk + row) * D;
#pragma unroll
                for (int nt = 0; nt < 2; nt++) {
                    const int col = 16 * w + 8 * nt + 2 * t;
                    const uint32_t qv = *reinterpret_cast<const uint32_t*>(s.Q[slot] + swz(row, col));
                    float2 o;
                    o.x = ptx::bf16_lo_f32(qv) + gamv[nt][0] * (z[nt][2 * rh] - mu) * rs + betv[nt][0];
                    o.y = ptx::bf16_hi_f32(qv) + gamv[nt][1] * (z[nt][2 * rh + 1] - mu) * rs + betv[nt][1];
                    *reinterpret_cast<float2*>(zrow + col) = o;
                }
            }
            arrive1(&s.in_empty[slot], lane);
            TTT_STAMP(g_lag_timeline, tl_lead, 2, c, 7);
        }
        TTT_TIMELINE_FLUSH(g_lag_timeline, tl_lead, 2);
    }
}

}  // namespace

int drop_chunk_hook() {
    static const int c = [] {
        const char* v = std::getenv("TTT_DEBUG_DROP_CHUNK");
        return (v && v[0]) ? std::atoi(v) : -1;
    }();
    return c;
}

bool linear_tc_supports(const LinearArgs& a) {
    return a.d == D && a.dtype == TTT_BF16 && a.mode == TTT_LN_RESIDUAL && a.mini_batch == kChunk && a.T > 0 &&
           a.T % kChunk == 0;
}

namespace {

template <bool kCkpt>
cudaError_t launch_lag(const LinearArgs& a, float* ckpt, cudaStream_t stream) {
    if (!linear_tc_supports(a)) return cudaErrorInvalidValue;
    const int BH = a.B * a.H;
    CUtensorMap mk, mv, mq, me;
    if (!make_token_tile_map(&mk, a.K, a.T, BH) || !make_token_tile_map(&mv, a.V, a.T, BH) ||
        !make_token_tile_map(&mq, a.Q, a.T, BH) || !make_eta_row_map(&me, a.eta, a.T, BH))
        return cudaErrorInvalidValue;
    const size_t smem = sizeof(LagSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(ttt_linear_lag_kernel<kCkpt>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    ttt_linear_lag_kernel<kCkpt><<<BH, kThreads, smem, stream>>>(mk, mv, mq, me, a.T, a.H, a.ln_eps, a.W0, a.b0,
                                                                  a.gamma, a.beta, a.Z, a.W_T, a.b_T,
                                                                  kCkpt ? -1 : drop_chunk_hook(), ckpt);
    return cudaPeekAtLastError();
}

}  // namespace

cudaError_t launch_linear_tc(const LinearArgs& a, cudaStream_t stream) { return launch_lag<false>(a, nullptr, stream); }

cudaError_t launch_linear_tc_checkpoints(const LinearArgs& a, float* states, cudaStream_t stream) {
    return launch_lag<true>(a, states, stream);
}

#ifdef TTT_TIMELINE
cudaError_t read_lag_timeline(long long* out) {
    return cudaMemcpyFromSymbol(out, g_lag_timeline, sizeof(g_lag_timeline));
}
#endif

cudaError_t read_and_clear_device_error(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_ttt_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_ttt_error_word, &zero, sizeof(unsigned int));
}

}  // namespace ttt
