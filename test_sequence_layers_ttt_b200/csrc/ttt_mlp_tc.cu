// Tensor-core TTT-MLP forward scan for sm_100a.
//
// Scope: bf16 Q/K/V, d = 64, hidden = 256, mini-batch b = 16, T a multiple of
// 16.  f(x) = x + LN(GELU(x W1 + b1) W2 + b2).  One CTA of 16 warps per
// (batch, head) runs the whole sequence.
//
// Method ("Learning to (Learn at Test Time)", literature record, Key
// takeaways bullets 1, 2 and 5; the codewithpapers.app record's abstract names
// the two-layer MLP state).  Per chunk of 16 tokens (one mini-batch), with the
// state (W1, b1, W2, b2) at the chunk start and X = K_c:
//   Z1 = X W1 + b1, H = GELU(Z1), Y = H W2 + b2
//   G2 = dl/dY (LayerNorm backward), G1 = (G2 W2^T) * GELU'(Z1)
//   Z1q = Q W1 + b1 - A G1,    A[t,s]  = eta_s (q_t . x_s + 1),    s <= t
//   Hq  = GELU(Z1q)
//   Z2q = Hq W2 + b2 - A2 G2,  A2[t,s] = eta_s (hq_t . h_s + 1),  s <= t
//   z   = q + LN(Z2q)
//   W1 -= X^T diag(eta) G1, b1 -= eta^T G1, W2 -= H^T diag(eta) G2, b2 -= eta^T G2
// (token t's output uses the state after the updates of tokens s <= t of the
// mini-batch; the dual form applies them without forming per-token weights).
//
// Layout: the fp32 state lives in shared memory as W1^T [256][64] and W2^T
// [64][256], rows XOR-swizzled in 8-float groups; the increments of a chunk are
// formed by tensor-core products and added with fp32 adds.  Every product runs
// as mma.sync m16n8k16 (bf16 in, fp32 accumulate); an fp32 operand is split into
// bf16 hi + lo (relative error below 2^-15) and the lo*lo term dropped.  The
// chunk's activations sit in shared memory as bf16 hi/lo tiles [16][64] with the
// 128-byte swizzle, read with ldmatrix.  Eight phases per chunk, separated by
// block barriers; the next chunk's Q/K/V/eta are loaded into registers while
// the current one computes.  No waits other than block barriers.
#include "common.cuh"
#include "ptx.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int D = 64;
constexpr int HID = 256;
constexpr int NP = HID / 64;  // 64-column panels of a [16][256] activation
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int PANEL = kChunk * 64 * 2;  // bytes of one bf16 [16][64] tile
constexpr int YLD = 72;                 // row stride (floats) of the fp32 [16][64] tiles

struct MlpTcSmem {
    float w1t[HID * D];                // W1^T [hid][in], swizzled
    float w2t[D * HID];                // W2^T [out][hid], swizzled
    float b1[HID], b2[D];
    float gam[D], bet[D];
    unsigned char K[PANEL], V[PANEL], Q[PANEL];
    unsigned char Hh[NP][PANEL], Hl[NP][PANEL];      // H = GELU(Z1), hi / lo
    unsigned char Hqh[NP][PANEL], Hql[NP][PANEL];    // Hq = GELU(Z1q)
    unsigned char G1h[NP][PANEL], G1l[NP][PANEL];    // G1
    unsigned char G2h[PANEL], G2l[PANEL];            // G2
    unsigned char E2h[PANEL], E2l[PANEL];            // -eta G2
    unsigned char EXh[PANEL], EXl[PANEL];            // -eta X
    float Y[kChunk * YLD];                           // Y, later Z2q
    uint4 afrag[2][32];                              // -A as A fragments [hi, lo][lane]
    float4 a2part[4][2][32];                         // partial Hq H^T over hidden quarters
    alignas(16) float eta[kChunk];
};

// GELU (tanh form) through the logistic identity 0.5 (1 + tanh(u)) = 1 / (1 + e^(-2u)),
// u = sqrt(2/pi) (x + 0.044715 x^3); returns gelu(x) and keeps sig for the derivative
__device__ __forceinline__ float gelu_sig(float x, float& sig) {
    const float c = 0.7978845608028654f;
    const float u = c * fmaf(0.044715f * x, x * x, x);
    sig = __fdividef(1.f, 1.f + __expf(-2.f * u));
    return x * sig;
}
// d/dx [x sig(2u)] = sig + 2 x u' sig (1 - sig)
__device__ __forceinline__ float gelu_prime_sig(float x, float sig) {
    const float c = 0.7978845608028654f;
    const float du = c * fmaf(3.f * 0.044715f * x, x, 1.f);
    return fmaf(2.f * x * du * sig, 1.f - sig, sig);
}

// fp32 state indexing: 8-float groups of a row XOR-swizzled by the row's low bits
__device__ __forceinline__ int w1i(int hid, int in) { return hid * D + ((((in >> 3) ^ (hid & 7))) << 3) + (in & 7); }
__device__ __forceinline__ int w2i(int out, int hid) { return out * HID + ((((hid >> 3) ^ (out & 7))) << 3) + (hid & 7); }
// bf16 [16][64] tile with the 128-byte swizzle
__device__ __forceinline__ uint32_t swz(int row, int col) {
    return row * 128 + ((((col >> 3) ^ (row & 7))) << 4) + (col & 7) * 2;
}
__device__ __forceinline__ uint32_t swz_chunk(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

// ldmatrix address patterns on one [16][64] tile (k-step or 16-column block kb in 0..3)
// A operand, rows = tokens, k = columns
__device__ __forceinline__ void ld_a(uint32_t tile, int kb, int lane, uint32_t (&a)[4]) {
    const int mi = lane >> 3, row = (mi & 1) * 8 + (lane & 7), chunk = 2 * kb + (mi >> 1);
    ptx::ldsm_x4(tile + swz_chunk(row, chunk), a[0], a[1], a[2], a[3]);
}
// B operand with k = tokens, n = columns 16kb..16kb+15: b[0..1] n-tile 0, b[2..3] n-tile 1
__device__ __forceinline__ void ld_b_tok(uint32_t tile, int kb, int lane, uint32_t (&b)[4]) {
    const int mi = lane >> 3, row = (mi & 1) * 8 + (lane & 7), chunk = 2 * kb + (mi >> 1);
    ptx::ldsm_x4_t(tile + swz_chunk(row, chunk), b[0], b[1], b[2], b[3]);
}
// A operand = transpose of columns 16kb..16kb+15: rows = columns, k = tokens
__device__ __forceinline__ void ld_a_t(uint32_t tile, int kb, int lane, uint32_t (&a)[4]) {
    const int mi = lane >> 3, row = (mi >> 1) * 8 + (lane & 7), chunk = 2 * kb + (mi & 1);
    ptx::ldsm_x4_t(tile + swz_chunk(row, chunk), a[0], a[1], a[2], a[3]);
}
// B operand with k = columns 16kb.., n = tokens: b[0..1] tokens 0-7, b[2..3] tokens 8-15
__device__ __forceinline__ void ld_b_col(uint32_t tile, int kb, int lane, uint32_t (&b)[4]) {
    const int mi = lane >> 3, row = (mi >> 1) * 8 + (lane & 7), chunk = 2 * kb + (mi & 1);
    ptx::ldsm_x4(tile + swz_chunk(row, chunk), b[0], b[1], b[2], b[3]);
}

__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    ptx::mma_bf16(d, a[0], a[1], a[2], a[3], b0, b1);
}
// d += (ah + al)(bh + bl) without the lo*lo term
__device__ __forceinline__ void mma3(float (&d)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4], uint32_t bh0,
                                     uint32_t bh1, uint32_t bl0, uint32_t bl1) {
    mma(d, ah, bh0, bh1);
    mma(d, ah, bl0, bl1);
    mma(d, al, bh0, bh1);
}
__device__ __forceinline__ void zero(float (&d)[4]) { d[0] = d[1] = d[2] = d[3] = 0.f; }

// write a C fragment (rows g, g+8; columns col, col+1 of a panel) as bf16 hi/lo pairs
__device__ __forceinline__ void store_pairs(unsigned char* hi, unsigned char* lo, int g, int col, const float (&v)[4]) {
    uint32_t h, l;
    ptx::split_pair(v[0], v[1], h, l);
    *reinterpret_cast<uint32_t*>(hi + swz(g, col)) = h;
    *reinterpret_cast<uint32_t*>(lo + swz(g, col)) = l;
    ptx::split_pair(v[2], v[3], h, l);
    *reinterpret_cast<uint32_t*>(hi + swz(g + 8, col)) = h;
    *reinterpret_cast<uint32_t*>(lo + swz(g + 8, col)) = l;
}

// -eta_s (p + 1) for s <= t (else 0), from a 16x16 C fragment pair, as hi/lo A fragments
__device__ __forceinline__ void causal_frag(const float (&p)[2][4], const float* eta_s, int g, int t, uint4& hi,
                                            uint4& lo) {
    float v[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; nt++)
#pragma unroll
        for (int r = 0; r < 4; r++) {
            const int row = g + 8 * (r >> 1), col = 8 * nt + 2 * t + (r & 1);
            v[nt][r] = col <= row ? -eta_s[col] * (p[nt][r] + 1.f) : 0.f;
        }
    ptx::split_pair(v[0][0], v[0][1], hi.x, lo.x);
    ptx::split_pair(v[0][2], v[0][3], hi.y, lo.y);
    ptx::split_pair(v[1][0], v[1][1], hi.z, lo.z);
    ptx::split_pair(v[1][2], v[1][3], hi.w, lo.w);
}

__global__ void __launch_bounds__(kThreads, 1)
ttt_mlp_tc_kernel(int T, int H, float eps, const __nv_bfloat16* __restrict__ Qg, const __nv_bfloat16* __restrict__ Kg,
                  const __nv_bfloat16* __restrict__ Vg, const float* __restrict__ etag, const float* W1_0,
                  const float* b1_0, const float* W2_0, const float* b2_0, const float* __restrict__ gamma,
                  const float* __restrict__ beta, float* __restrict__ Z, float* W1_T, float* b1_T, float* W2_T,
                  float* b2_T) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    MlpTcSmem& s = *reinterpret_cast<MlpTcSmem*>(smem_raw + ((128u - (ptx::smem_addr(smem_raw) & 127u)) & 127u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const long bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int n = T / kChunk;

    // ---- initial state
    for (int i = tid; i < D * HID; i += kThreads) {
        const int in = i / HID, hid = i % HID;  // W1_0 [in][hid]
        s.w1t[w1i(hid, in)] = W1_0[bh * D * HID + i];
    }
    for (int i = tid; i < HID * D; i += kThreads) {
        const int hid = i / D, out = i % D;  // W2_0 [hid][out]
        s.w2t[w2i(out, hid)] = W2_0[bh * HID * D + i];
    }
    for (int i = tid; i < HID; i += kThreads) s.b1[i] = b1_0[bh * HID + i];
    if (tid < D) {
        s.b2[tid] = b2_0[bh * D + tid];
        s.gam[tid] = gamma[(long)h * D + tid];
        s.bet[tid] = beta[(long)h * D + tid];
    }

    // ---- token loads: thread i < 384 moves one 16-byte piece of K, V or Q; 384..387 eta
    const long tok0 = bh * (long)T;
    const int lt = tid >> 7, lidx = tid & 127, lrow = lidx >> 3, lchunk = lidx & 7;
    const __nv_bfloat16* lsrc = lt == 0 ? Kg : (lt == 1 ? Vg : Qg);
    uint4 pf = make_uint4(0u, 0u, 0u, 0u);
    float4 pfe = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fetch = [&](int c) {
        if (tid < 384) pf = *reinterpret_cast<const uint4*>(lsrc + (tok0 + c * kChunk + lrow) * D + lchunk * 8);
        else if (tid < 388) pfe = *reinterpret_cast<const float4*>(etag + tok0 + c * kChunk + (tid - 384) * 4);
    };
    if (n > 0) fetch(0);

    const uint32_t sK = ptx::smem_addr(s.K), sQ = ptx::smem_addr(s.Q);
    float* Zbh = Z + tok0 * D;

    for (int c = 0; c < n; c++) {
        // ================================================= phase 0: this chunk's tokens in, next chunk's requested
        __syncthreads();  // the previous chunk no longer reads the token tiles
        if (tid < 384) {
            unsigned char* dst = lt == 0 ? s.K : (lt == 1 ? s.V : s.Q);
            *reinterpret_cast<uint4*>(dst + swz_chunk(lrow, lchunk)) = pf;
        } else if (tid < 388) {
            *reinterpret_cast<float4*>(&s.eta[(tid - 384) * 4]) = pfe;
        }
        if (c + 1 < n) fetch(c + 1);
        __syncthreads();

        // ================================================= phase 1: [X; Q] W1 + b1, H = GELU(Z1); A; -eta X
        // warp w: hidden units [16w, 16w + 16)
        float z1[2][4], zq[2][4], sg1[2][4];
        {
#pragma unroll
            for (int nt = 0; nt < 2; nt++) {
                const int col = 16 * warp + 8 * nt + 2 * t;
                z1[nt][0] = z1[nt][2] = zq[nt][0] = zq[nt][2] = s.b1[col];
                z1[nt][1] = z1[nt][3] = zq[nt][1] = zq[nt][3] = s.b1[col + 1];
            }
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                uint32_t ax[4], aq[4];
                ld_a(sK, ks, lane, ax);
                ld_a(sQ, ks, lane, aq);
#pragma unroll
                for (int nt = 0; nt < 2; nt++) {
                    const int hid = 16 * warp + 8 * nt + g, in = 16 * ks + 2 * t;
                    const float2 w0 = *reinterpret_cast<const float2*>(&s.w1t[w1i(hid, in)]);
                    const float2 w1 = *reinterpret_cast<const float2*>(&s.w1t[w1i(hid, in + 8)]);
                    uint32_t bh0, bl0, bh1, bl1;
                    ptx::split_pair(w0.x, w0.y, bh0, bl0);
                    ptx::split_pair(w1.x, w1.y, bh1, bl1);
                    mma(z1[nt], ax, bh0, bh1);
                    mma(z1[nt], ax, bl0, bl1);
                    mma(zq[nt], aq, bh0, bh1);
                    mma(zq[nt], aq, bl0, bl1);
                }
            }
            const int p = warp >> 2;
#pragma unroll
            for (int nt = 0; nt < 2; nt++) {
                float hv[4];
#pragma unroll
                for (int r = 0; r < 4; r++) hv[r] = gelu_sig(z1[nt][r], sg1[nt][r]);
                store_pairs(s.Hh[p], s.Hl[p], g, 16 * (warp & 3) + 8 * nt + 2 * t, hv);
            }
        }
        if (warp == 0) {
            // A = tril(eta_s (q_t . x_s + 1)) as -A hi/lo A fragments
            float pa[2][4];
            zero(pa[0]);
            zero(pa[1]);
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                uint32_t aq[4], bx[4];
                ld_a(sQ, ks, lane, aq);
                ld_b_col(sK, ks, lane, bx);
                mma(pa[0], aq, bx[0], bx[1]);
                mma(pa[1], aq, bx[2], bx[3]);
            }
            uint4 hi, lo;
            causal_frag(pa, s.eta, g, t, hi, lo);
            s.afrag[0][lane] = hi;
            s.afrag[1][lane] = lo;
        }
        {
            // -eta_t X[t][:] for the W1 update (k = tokens)
            const int row = tid >> 5, col = 2 * (tid & 31);
            const uint32_t xv = *reinterpret_cast<const uint32_t*>(s.K + swz(row, col));
            const float e = -s.eta[row];
            uint32_t hi, lo;
            ptx::split_pair(e * ptx::bf16_lo_f32(xv), e * ptx::bf16_hi_f32(xv), hi, lo);
            *reinterpret_cast<uint32_t*>(s.EXh + swz(row, col)) = hi;
            *reinterpret_cast<uint32_t*>(s.EXl + swz(row, col)) = lo;
        }
        __syncthreads();

        // ================================================= phase 2: Y = H W2 + b2 (warps 0-7: output columns [8w, 8w+8))
        auto h_times_w2 = [&](unsigned char (*Ah)[PANEL], unsigned char (*Al)[PANEL], int ot, float (&acc)[4]) {
            float acc2[4];
            zero(acc2);
            acc[0] = acc[2] = s.b2[8 * ot + 2 * t];
            acc[1] = acc[3] = s.b2[8 * ot + 2 * t + 1];
#pragma unroll 4
            for (int ks = 0; ks < 16; ks++) {
                uint32_t ah[4], al[4];
                ld_a(ptx::smem_addr(Ah[ks >> 2]), ks & 3, lane, ah);
                ld_a(ptx::smem_addr(Al[ks >> 2]), ks & 3, lane, al);
                const int out = 8 * ot + g, hid = 16 * ks + 2 * t;
                const float2 w0 = *reinterpret_cast<const float2*>(&s.w2t[w2i(out, hid)]);
                const float2 w1 = *reinterpret_cast<const float2*>(&s.w2t[w2i(out, hid + 8)]);
                uint32_t bh0, bl0, bh1, bl1;
                ptx::split_pair(w0.x, w0.y, bh0, bl0);
                ptx::split_pair(w1.x, w1.y, bh1, bl1);
                if (ks & 1) mma3(acc2, ah, al, bh0, bh1, bl0, bl1);
                else mma3(acc, ah, al, bh0, bh1, bl0, bl1);
            }
#pragma unroll
            for (int r = 0; r < 4; r++) acc[r] += acc2[r];
        };
        if (warp < 8) {
            float y[4];
            h_times_w2(s.Hh, s.Hl, warp, y);
            const int col = 8 * warp + 2 * t;
            *reinterpret_cast<float2*>(&s.Y[g * YLD + col]) = make_float2(y[0], y[1]);
            *reinterpret_cast<float2*>(&s.Y[(g + 8) * YLD + col]) = make_float2(y[2], y[3]);
        }
        __syncthreads();

        // ================================================= phase 3: G2 = dl/dY, E2 = -eta G2 (warp w: token w)
        {
            const int row = warp, col = 2 * lane;
            const float2 y = *reinterpret_cast<const float2*>(&s.Y[row * YLD + col]);
            const uint32_t xv = *reinterpret_cast<const uint32_t*>(s.K + swz(row, col));
            const uint32_t vv = *reinterpret_cast<const uint32_t*>(s.V + swz(row, col));
            const float mu = warp_sum(y.x + y.y) * (1.f / D);
            const float d0 = y.x - mu, d1 = y.y - mu;
            const float rs = rsqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.f / D) + eps);
            const float xh0 = d0 * rs, xh1 = d1 * rs;
            const float g0 = s.gam[col], g1 = s.gam[col + 1];
            const float gx0 = 2.f * g0 * (ptx::bf16_lo_f32(xv) + g0 * xh0 + s.bet[col] - ptx::bf16_lo_f32(vv));
            const float gx1 = 2.f * g1 * (ptx::bf16_hi_f32(xv) + g1 * xh1 + s.bet[col + 1] - ptx::bf16_hi_f32(vv));
            const float mgx = warp_sum(gx0 + gx1) * (1.f / D);
            const float mgxx = warp_sum(gx0 * xh0 + gx1 * xh1) * (1.f / D);
            const float G0 = rs * (gx0 - mgx - xh0 * mgxx), G1 = rs * (gx1 - mgx - xh1 * mgxx);
            const float e = -s.eta[row];
            uint32_t hi, lo;
            ptx::split_pair(G0, G1, hi, lo);
            *reinterpret_cast<uint32_t*>(s.G2h + swz(row, col)) = hi;
            *reinterpret_cast<uint32_t*>(s.G2l + swz(row, col)) = lo;
            ptx::split_pair(e * G0, e * G1, hi, lo);
            *reinterpret_cast<uint32_t*>(s.E2h + swz(row, col)) = hi;
            *reinterpret_cast<uint32_t*>(s.E2l + swz(row, col)) = lo;
        }
        __syncthreads();

        // ================================================= phase 4: G1 = (G2 W2^T) * GELU'(Z1) (warp w: hidden [16w, 16w+16))
        {
            float acc[2][4];
            zero(acc[0]);
            zero(acc[1]);
            const uint32_t g2h = ptx::smem_addr(s.G2h), g2l = ptx::smem_addr(s.G2l);
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                uint32_t ah[4], al[4];
                ld_a(g2h, ks, lane, ah);
                ld_a(g2l, ks, lane, al);
#pragma unroll
                for (int nt = 0; nt < 2; nt++) {
                    const int hid = 16 * warp + 8 * nt + g, out = 16 * ks + 2 * t;
                    uint32_t bh0, bl0, bh1, bl1;
                    ptx::split_pair(s.w2t[w2i(out, hid)], s.w2t[w2i(out + 1, hid)], bh0, bl0);
                    ptx::split_pair(s.w2t[w2i(out + 8, hid)], s.w2t[w2i(out + 9, hid)], bh1, bl1);
                    mma3(acc[nt], ah, al, bh0, bh1, bl0, bl1);
                }
            }
            const int p = warp >> 2;
#pragma unroll
            for (int nt = 0; nt < 2; nt++) {
#pragma unroll
                for (int r = 0; r < 4; r++) acc[nt][r] *= gelu_prime_sig(z1[nt][r], sg1[nt][r]);
                store_pairs(s.G1h[p], s.G1l[p], g, 16 * (warp & 3) + 8 * nt + 2 * t, acc[nt]);
            }
        }
        __syncthreads();

        // ================================================= phase 5: Z1q = Q W1 + b1 - A G1, Hq = GELU(Z1q)
        {
            const uint4 fh = s.afrag[0][lane], fl = s.afrag[1][lane];
            const uint32_t ah[4] = {fh.x, fh.y, fh.z, fh.w}, al[4] = {fl.x, fl.y, fl.z, fl.w};
            const int p = warp >> 2;
            uint32_t bh[4], bl[4];
            ld_b_tok(ptx::smem_addr(s.G1h[p]), warp & 3, lane, bh);
            ld_b_tok(ptx::smem_addr(s.G1l[p]), warp & 3, lane, bl);
            mma3(zq[0], ah, al, bh[0], bh[1], bl[0], bl[1]);
            mma3(zq[1], ah, al, bh[2], bh[3], bl[2], bl[3]);
#pragma unroll
            for (int nt = 0; nt < 2; nt++) {
                float hv[4], sq;
#pragma unroll
                for (int r = 0; r < 4; r++) hv[r] = gelu_sig(zq[nt][r], sq);
                store_pairs(s.Hqh[p], s.Hql[p], g, 16 * (warp & 3) + 8 * nt + 2 * t, hv);
            }
        }
        __syncthreads();

        // ================================================= phase 6: Hq H^T by hidden quarters (warps 0-3); Hq W2 + b2 (warps 8-15)
        float z2[4];
        if (warp < 4) {
            const int p = warp;
            float acc[2][4];
            zero(acc[0]);
            zero(acc[1]);
#pragma unroll
            for (int kb = 0; kb < 4; kb++) {
                uint32_t ah[4], al[4], bh[4], bl[4];
                ld_a(ptx::smem_addr(s.Hqh[p]), kb, lane, ah);
                ld_a(ptx::smem_addr(s.Hql[p]), kb, lane, al);
                ld_b_col(ptx::smem_addr(s.Hh[p]), kb, lane, bh);
                ld_b_col(ptx::smem_addr(s.Hl[p]), kb, lane, bl);
                mma3(acc[0], ah, al, bh[0], bh[1], bl[0], bl[1]);
                mma3(acc[1], ah, al, bh[2], bh[3], bl[2], bl[3]);
            }
            s.a2part[p][0][lane] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
            s.a2part[p][1][lane] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
        } else if (warp >= 8) {
            h_times_w2(s.Hqh, s.Hql, warp - 8, z2);
        }
        __syncthreads();

        // ================================================= phase 7: state update; Z2q = Hq W2 + b2 - A2 G2
        if (warp < 8) {
            // W1^T[hid][in] += G1^T (-eta X), b1 += G1^T (-eta), hidden rows [32w, 32w + 32)
            uint32_t eh[2], el[2];  // -eta as a B column (n = 0): k = tokens 2t..2t+1 and 2t+8..2t+9
            ptx::split_pair(g == 0 ? -s.eta[2 * t] : 0.f, g == 0 ? -s.eta[2 * t + 1] : 0.f, eh[0], el[0]);
            ptx::split_pair(g == 0 ? -s.eta[2 * t + 8] : 0.f, g == 0 ? -s.eta[2 * t + 9] : 0.f, eh[1], el[1]);
#pragma unroll 1
            for (int m = 0; m < 2; m++) {
                const int mt = 2 * warp + m, p = mt >> 2;  // 16 hidden rows [16mt, 16mt + 16)
                uint32_t ah[4], al[4];
                ld_a_t(ptx::smem_addr(s.G1h[p]), mt & 3, lane, ah);
                ld_a_t(ptx::smem_addr(s.G1l[p]), mt & 3, lane, al);
#pragma unroll
                for (int jp = 0; jp < 4; jp++) {
                    uint32_t bh[4], bl[4];
                    ld_b_tok(ptx::smem_addr(s.EXh), jp, lane, bh);
                    ld_b_tok(ptx::smem_addr(s.EXl), jp, lane, bl);
                    float d[2][4];
                    zero(d[0]);
                    zero(d[1]);
                    mma3(d[0], ah, al, bh[0], bh[1], bl[0], bl[1]);
                    mma3(d[1], ah, al, bh[2], bh[3], bl[2], bl[3]);
#pragma unroll
                    for (int nt = 0; nt < 2; nt++)
#pragma unroll
                        for (int rh = 0; rh < 2; rh++) {
                            float2* wp = reinterpret_cast<float2*>(&s.w1t[w1i(16 * mt + g + 8 * rh, 16 * jp + 8 * nt + 2 * t)]);
                            float2 wv = *wp;
                            wv.x += d[nt][2 * rh];
                            wv.y += d[nt][2 * rh + 1];
                            *wp = wv;
                        }
                }
                float db[4];
                zero(db);
                mma3(db, ah, al, eh[0], eh[1], el[0], el[1]);
                if (t == 0) {
                    s.b1[16 * mt + g] += db[0];
                    s.b1[16 * mt + 8 + g] += db[2];
                }
            }
        } else {
            const int v = warp - 8;  // output columns [8v, 8v + 8)
            {
                // A2 = tril(eta_s (hq_t . h_s + 1)) from the four partial products
                float pa[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; nt++) {
                    float4 a = s.a2part[0][nt][lane];
#pragma unroll
                    for (int q = 1; q < 4; q++) {
                        const float4 b = s.a2part[q][nt][lane];
                        a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
                    }
                    pa[nt][0] = a.x; pa[nt][1] = a.y; pa[nt][2] = a.z; pa[nt][3] = a.w;
                }
                uint4 fh, fl;
                causal_frag(pa, s.eta, g, t, fh, fl);
                const uint32_t ah[4] = {fh.x, fh.y, fh.z, fh.w}, al[4] = {fl.x, fl.y, fl.z, fl.w};
                uint32_t bh[4], bl[4];
                ld_b_tok(ptx::smem_addr(s.G2h), v >> 1, lane, bh);
                ld_b_tok(ptx::smem_addr(s.G2l), v >> 1, lane, bl);
                const int o = (v & 1) * 2;
                mma3(z2, ah, al, bh[o], bh[o + 1], bl[o], bl[o + 1]);
                const int col = 8 * v + 2 * t;
                *reinterpret_cast<float2*>(&s.Y[g * YLD + col]) = make_float2(z2[0], z2[1]);
                *reinterpret_cast<float2*>(&s.Y[(g + 8) * YLD + col]) = make_float2(z2[2], z2[3]);
            }
            // W2^T[out][hid] += E2^T H, b2 += E2^T 1; output rows [16mo, 16mo + 16), hidden [128(v>>2), +128)
            const int mo = v & 3;
            uint32_t ah[4], al[4];
            ld_a_t(ptx::smem_addr(s.E2h), mo, lane, ah);
            ld_a_t(ptx::smem_addr(s.E2l), mo, lane, al);
#pragma unroll 1
            for (int pp = 0; pp < 2; pp++) {
                const int p = 2 * (v >> 2) + pp;
#pragma unroll
                for (int jp = 0; jp < 4; jp++) {
                    uint32_t bh[4], bl[4];
                    ld_b_tok(ptx::smem_addr(s.Hh[p]), jp, lane, bh);
                    ld_b_tok(ptx::smem_addr(s.Hl[p]), jp, lane, bl);
                    float d[2][4];
                    zero(d[0]);
                    zero(d[1]);
                    mma3(d[0], ah, al, bh[0], bh[1], bl[0], bl[1]);
                    mma3(d[1], ah, al, bh[2], bh[3], bl[2], bl[3]);
#pragma unroll
                    for (int nt = 0; nt < 2; nt++)
#pragma unroll
                        for (int rh = 0; rh < 2; rh++) {
                            float2* wp = reinterpret_cast<float2*>(
                                &s.w2t[w2i(16 * mo + g + 8 * rh, 64 * p + 16 * jp + 8 * nt + 2 * t)]);
                            float2 wv = *wp;
                            wv.x += d[nt][2 * rh];
                            wv.y += d[nt][2 * rh + 1];
                            *wp = wv;
                        }
                }
            }
            if (v < 4) {
                const uint32_t ones = g == 0 ? 0x3f803f80u : 0u;  // (1, 1) in bf16 on column 0
                float db[4];
                zero(db);
                mma(db, ah, ones, ones);
                mma(db, al, ones, ones);
                if (t == 0) {
                    s.b2[16 * mo + g] += db[0];
                    s.b2[16 * mo + 8 + g] += db[2];
                }
            }
        }
        __syncthreads();

        // ================================================= phase 8: z = q + LN(Z2q) (warp w: token w)
        {
            const int row = warp, col = 2 * lane;
            const float2 zz = *reinterpret_cast<const float2*>(&s.Y[row * YLD + col]);
            const float mu = warp_sum(zz.x + zz.y) * (1.f / D);
            const float d0 = zz.x - mu, d1 = zz.y - mu;
            const float rs = rsqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.f / D) + eps);
            const uint32_t qv = *reinterpret_cast<const uint32_t*>(s.Q + swz(row, col));
            float2 o;
            o.x = ptx::bf16_lo_f32(qv) + s.gam[col] * d0 * rs + s.bet[col];
            o.y = ptx::bf16_hi_f32(qv) + s.gam[col + 1] * d1 * rs + s.bet[col + 1];
            *reinterpret_cast<float2*>(Zbh + (size_t)(c * kChunk + row) * D + col) = o;
        }
    }
    __syncthreads();
    // ---- final state
    for (int i = tid; i < D * HID; i += kThreads) {
        const int in = i / HID, hid = i % HID;
        W1_T[bh * D * HID + i] = s.w1t[w1i(hid, in)];
    }
    for (int i = tid; i < HID * D; i += kThreads) {
        const int hid = i / D, out = i % D;
        W2_T[bh * HID * D + i] = s.w2t[w2i(out, hid)];
    }
    for (int i = tid; i < HID; i += kThreads) b1_T[bh * HID + i] = s.b1[i];
    if (tid < D) b2_T[bh * D + tid] = s.b2[tid];
}

// ============================================================================
// Split variant: the hidden units of one scan are divided between the two CTAs
// of a cluster (CTA r owns units [128r, 128r + 128) of W1's columns, b1, and
// W2's rows); both hold the full b2, gamma, beta and the chunk's tokens.  Every
// product over the hidden units is formed as two partial sums that the CTAs
// swap through distributed shared memory; the rest is either local to a
// hidden slice or repeated bit for bit in both CTAs:
//   Z1, H, G1, Z1q, Hq, the W1 / b1 / W2 updates   local to the slice
//   Y  = b2 + H_0 W2_0 + H_1 W2_1                   partial sums swapped
//   G2, E2 = -eta G2, A, the b2 update              repeated in both CTAs
//   Hq H^T and Hq W2                                partial sums swapped
// Both CTAs add the partials in rank order, so their copies of Y, G2, b2 and
// Z2q agree exactly.  CTA r writes the outputs of tokens [8r, 8r + 8) of each
// chunk.
//
// The fp32 state of the slice stays in registers, one 16 x 64 tile per warp in
// the mma accumulator layout, so an update is a register add; after each
// update the warp writes the tile's bf16 hi / lo split to shared memory, where
// the products read it with ldmatrix.  The Y partials travel by st.async,
// counted in bytes on the receiver's mbarrier (bounded wait, no fence on the
// sender); the Hq partials by plain remote stores ordered by a hardware cluster
// barrier, with the W1 and W2 updates between its arrive and its wait.
namespace split {

constexpr int kSplit = 2;
constexpr int HL = HID / kSplit;  // hidden units per CTA
constexpr int NPL = HL / 64;      // 64-column panels of a [16][HL] activation

// byte offset in a bf16 W2^T slice tile [out][HL] (256-byte rows, 16-byte groups XOR-swizzled)
__device__ __forceinline__ uint32_t w2b(int out, int hid) {
    return out * (HL * 2) + ((((hid >> 3) ^ (out & 7))) << 4) + (hid & 7) * 2;
}
// W1 as the B operand of [16 x in] x W1 (k = inputs 16ks.., n = hidden 8hb..), from the
// bf16 W1^T slice tiles [hid][in] (128-byte rows, swizzled like the activation tiles)
__device__ __forceinline__ void ld_w1(uint32_t wh, uint32_t wl, int ks, int hb, int lane, uint32_t (&b)[4]) {
    const int mi = lane >> 3, r = lane & 7;
    ptx::ldsm_x4((mi >> 1 ? wl : wh) + swz(8 * hb + r, 16 * ks + 8 * (mi & 1)), b[0], b[1], b[2], b[3]);
}
// W2 as the B operand of [16 x hid] x W2 (k = hidden 16ks.., n = outputs 8ot..): hi k-halves, lo k-halves
__device__ __forceinline__ void ld_w2_kh(uint32_t wh, uint32_t wl, int ks, int ot, int lane, uint32_t (&b)[4]) {
    const int mi = lane >> 3, r = lane & 7;
    ptx::ldsm_x4((mi >> 1 ? wl : wh) + w2b(8 * ot + r, 16 * ks + 8 * (mi & 1)), b[0], b[1], b[2], b[3]);
}
// W2^T as the B operand of [16 x out] x W2^T (k = outputs 16ks.., n = hidden 8hb..)
__device__ __forceinline__ void ld_w2_ko(uint32_t wh, uint32_t wl, int ks, int hb, int lane, uint32_t (&b)[4]) {
    const int mi = lane >> 3, r = lane & 7;
    ptx::ldsm_x4_t((mi >> 1 ? wl : wh) + w2b(16 * ks + 8 * (mi & 1) + r, 8 * hb), b[0], b[1], b[2], b[3]);
}

struct Smem {
    unsigned char w1h[HL * D * 2], w1l[HL * D * 2];  // W1^T slice [hid][in] as bf16 hi / lo, swizzled with swz
    unsigned char w2h[D * HL * 2], w2l[D * HL * 2];  // W2^T slice [out][hid] as bf16 hi / lo, swizzled with w2b
    float b1[HL], b2[D];
    float gam[D], bet[D];
    unsigned char K[PANEL], V[PANEL], Q[PANEL];
    unsigned char Hh[NPL][PANEL], Hl[NPL][PANEL];
    unsigned char Hqh[NPL][PANEL], Hql[NPL][PANEL];
    unsigned char G1h[NPL][PANEL], G1l[NPL][PANEL];
    unsigned char G2h[PANEL], G2l[PANEL];
    unsigned char E2h[PANEL], E2l[PANEL];
    unsigned char EXh[PANEL], EXl[PANEL];
    float yp[kSplit][kChunk * YLD];  // H W2 partial of CTA r (written by CTA r in both CTAs)
    float zp[kSplit][kChunk * YLD];  // Hq W2 partial of CTA r
    float Y[kChunk * YLD];           // Z2q
    uint4 afrag[2][32];
    float4 a2p[kSplit * NPL][2][32];  // Hq H^T partial of CTA r, panel p at [NPL r + p]
    alignas(16) float eta[kChunk];
    uint64_t ybar;   // completes when the other CTA's Y partial of the chunk has landed in yp
    int abort_flag;  // set after a wait gave up (in both CTAs)
};

constexpr uint32_t kYBytes = kChunk * D * 4;   // one CTA's Y partial
constexpr long long kTimeoutCycles = 2000000000LL;
__device__ unsigned int g_mlp_error_word = 0;

// bounded wait on a barrier completed by the other CTA's stores; false once the
// wait has given up here or in the other CTA (then both run on without waiting)
__device__ __forceinline__ bool wait_peer(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t peer_abort_flag) {
    if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
    const long long t0 = clock64();
    for (int spins = 1;; spins++) {
        if (*abort_flag) return false;
        if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
        if ((spins & 63) == 0 && clock64() - t0 > kTimeoutCycles) {
            *abort_flag = 1;
            asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort_flag), "r"(1u) : "memory");
            atomicOr(&g_mlp_error_word, 1u);
            return false;
        }
    }
}

// d_h += ah bh, d_l += ah bl + al bh: the split product in two accumulators
__device__ __forceinline__ void mma3s(float (&dh)[4], float (&dl)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4],
                                      uint32_t bh0, uint32_t bh1, uint32_t bl0, uint32_t bl1) {
    mma(dh, ah, bh0, bh1);
    mma(dl, ah, bl0, bl1);
    mma(dl, al, bh0, bh1);
}

}  // namespace split

__global__ void __cluster_dims__(split::kSplit, 1, 1) __launch_bounds__(kThreads, 1)
ttt_mlp_split_kernel(int T, int H, float eps, const __nv_bfloat16* __restrict__ Qg, const __nv_bfloat16* __restrict__ Kg,
                     const __nv_bfloat16* __restrict__ Vg, const float* __restrict__ etag, const float* W1_0,
                     const float* b1_0, const float* W2_0, const float* b2_0, const float* __restrict__ gamma,
                     const float* __restrict__ beta, float* __restrict__ Z, float* W1_T, float* b1_T, float* W2_T,
                     float* b2_T) {
    using split::HL;
    using split::NPL;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    split::Smem& s = *reinterpret_cast<split::Smem*>(smem_raw + ((128u - (ptx::smem_addr(smem_raw) & 127u)) & 127u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t rank = ptx::cluster_ctarank(), peer = rank ^ 1u;
    const long bh = blockIdx.x / split::kSplit;
    const int h = (int)(bh % H);
    const int n = T / kChunk;
    const int hid0 = HL * (int)rank;  // first hidden unit of this CTA's slice
    auto remote = [&](const void* p) { return ptx::mapa_shared(ptx::smem_addr(p), peer); };

    // ---- initial state.  The fp32 state lives in registers, one 16 x 64 tile per warp in
    // the mma accumulator layout: warp w < 8 holds W1^T rows (hidden) [16w, 16w + 16),
    // warp 8 + v holds W2^T rows (outputs) [16 (v & 3), +16) x hidden [64 (v >> 2), +64).
    // Element sr[jp][nt][2 rh + e] sits at row 16 m + g + 8 rh, column 16 jp + 8 nt + 2 t + e.
    // Shared memory holds the bf16 hi / lo copies the products read.
    float sr[4][2][4];
    const bool w1_warp = warp < 8;
    const int vw = warp & 7, mo = vw & 3, pp = vw >> 2;
    auto state_index = [&](int jp, int nt, int rh, int e) -> long {
        if (w1_warp) {  // W1_0 [in][hid]
            const int hid = 16 * vw + g + 8 * rh, in = 16 * jp + 8 * nt + 2 * t + e;
            return bh * D * HID + (long)in * HID + hid0 + hid;
        }
        const int out = 16 * mo + g + 8 * rh, hid = 64 * pp + 16 * jp + 8 * nt + 2 * t + e;  // W2_0 [hid][out]
        return bh * HID * D + (long)(hid0 + hid) * D + out;
    };
    // bf16 hi / lo copy of the pair sr[jp][nt][2 rh], sr[jp][nt][2 rh + 1]
    auto store_split = [&](int jp, int nt, int rh, float x0, float x1) {
        uint32_t hi, lo;
        ptx::split_pair(x0, x1, hi, lo);
        const uint32_t off = w1_warp ? swz(16 * vw + g + 8 * rh, 16 * jp + 8 * nt + 2 * t)
                                     : split::w2b(16 * mo + g + 8 * rh, 64 * pp + 16 * jp + 8 * nt + 2 * t);
        unsigned char* th = w1_warp ? s.w1h : s.w2h;
        unsigned char* tl = w1_warp ? s.w1l : s.w2l;
        *reinterpret_cast<uint32_t*>(th + off) = hi;
        *reinterpret_cast<uint32_t*>(tl + off) = lo;
    };
#pragma unroll
    for (int jp = 0; jp < 4; jp++)
#pragma unroll
        for (int nt = 0; nt < 2; nt++)
#pragma unroll
            for (int rh = 0; rh < 2; rh++) {
                const float* W0 = w1_warp ? W1_0 : W2_0;
                sr[jp][nt][2 * rh] = W0[state_index(jp, nt, rh, 0)];
                sr[jp][nt][2 * rh + 1] = W0[state_index(jp, nt, rh, 1)];
                store_split(jp, nt, rh, sr[jp][nt][2 * rh], sr[jp][nt][2 * rh + 1]);
            }
    for (int i = tid; i < HL; i += kThreads) s.b1[i] = b1_0[bh * HID + hid0 + i];
    if (tid < D) {
        s.b2[tid] = b2_0[bh * D + tid];
        s.gam[tid] = gamma[(long)h * D + tid];
        s.bet[tid] = beta[(long)h * D + tid];
    }
    if (tid == 0) {
        ptx::mbar_init(&s.ybar, 1);
        s.abort_flag = 0;
        ptx::fence_mbar_init();
    }

    // ---- token loads (both CTAs read the whole chunk): as in the one-CTA kernel
    const long tok0 = bh * (long)T;
    const int lt = tid >> 7, lidx = tid & 127, lrow = lidx >> 3, lchunk = lidx & 7;
    const __nv_bfloat16* lsrc = lt == 0 ? Kg : (lt == 1 ? Vg : Qg);
    uint4 pf = make_uint4(0u, 0u, 0u, 0u);
    float4 pfe = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fetch = [&](int c) {
        if (tid < 384) pf = *reinterpret_cast<const uint4*>(lsrc + (tok0 + c * kChunk + lrow) * D + lchunk * 8);
        else if (tid < 388) pfe = *reinterpret_cast<const float4*>(etag + tok0 + c * kChunk + (tid - 384) * 4);
    };
    if (n > 0) fetch(0);

    const uint32_t sK = ptx::smem_addr(s.K), sQ = ptx::smem_addr(s.Q);
    const uint32_t sW2h = ptx::smem_addr(s.w2h), sW2l = ptx::smem_addr(s.w2l);
    const uint32_t sW1h = ptx::smem_addr(s.w1h), sW1l = ptx::smem_addr(s.w1l);
    float* Zbh = Z + tok0 * D;
    // this warp's hidden units [8 warp, 8 warp + 8): panel and column inside it
    const int p = warp >> 3, pc = 8 * (warp & 7) + 2 * t;

    // the peer CTA is running, its barrier initialised, before any store reaches its shared memory
    ptx::cluster_arrive();
    ptx::cluster_wait();
    const uint32_t ybar_peer = remote(&s.ybar), abort_peer = remote(&s.abort_flag);

    for (int c = 0; c < n; c++) {
        // ================================================= phase 0: this chunk's tokens in, next chunk's requested
        __syncthreads();
        // after an abort neither CTA arms its barrier or sends, so no byte count runs away
        const bool live = !*reinterpret_cast<volatile int*>(&s.abort_flag);
        if (tid == 0 && live) ptx::mbar_arrive_expect_tx(&s.ybar, split::kYBytes);
        if (tid < 384) {
            unsigned char* dst = lt == 0 ? s.K : (lt == 1 ? s.V : s.Q);
            *reinterpret_cast<uint4*>(dst + swz_chunk(lrow, lchunk)) = pf;
        } else if (tid < 388) {
            *reinterpret_cast<float4*>(&s.eta[(tid - 384) * 4]) = pfe;
        }
        if (c + 1 < n) fetch(c + 1);
        __syncthreads();

        // ================================================= phase 1: [X; Q] W1 + b1 on this warp's 8 hidden units, H = GELU(Z1)
        float z1[4], zq[4], sg1[4];
        {
            float z1l[4], zql[4];
            zero(z1l);
            zero(zql);
            const int col = 8 * warp + 2 * t;
            z1[0] = z1[2] = zq[0] = zq[2] = s.b1[col];
            z1[1] = z1[3] = zq[1] = zq[3] = s.b1[col + 1];
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                uint32_t ax[4], aq[4];
                ld_a(sK, ks, lane, ax);
                ld_a(sQ, ks, lane, aq);
                uint32_t b[4];
                split::ld_w1(sW1h, sW1l, ks, warp, lane, b);
                mma(z1, ax, b[0], b[1]);
                mma(z1l, ax, b[2], b[3]);
                mma(zq, aq, b[0], b[1]);
                mma(zql, aq, b[2], b[3]);
            }
            float hv[4];
#pragma unroll
            for (int r = 0; r < 4; r++) {
                z1[r] += z1l[r];
                zq[r] += zql[r];
                hv[r] = gelu_sig(z1[r], sg1[r]);
            }
            store_pairs(s.Hh[p], s.Hl[p], g, pc, hv);
        }
        __syncthreads();

        // ================================================= phase 2: partial Y = H W2 (warps 0-7), A and -eta X (warps 8-15)
        if (warp < 8) {
            float acc[4], accl[4], acc2[4], acc2l[4];
            zero(acc);
            zero(accl);
            zero(acc2);
            zero(acc2l);
#pragma unroll 4
            for (int ks = 0; ks < 4 * NPL; ks++) {
                uint32_t ah[4], al[4];
                ld_a(ptx::smem_addr(s.Hh[ks >> 2]), ks & 3, lane, ah);
                ld_a(ptx::smem_addr(s.Hl[ks >> 2]), ks & 3, lane, al);
                uint32_t b[4];
                split::ld_w2_kh(sW2h, sW2l, ks, warp, lane, b);
                if (ks & 1) split::mma3s(acc2, acc2l, ah, al, b[0], b[1], b[2], b[3]);
                else split::mma3s(acc, accl, ah, al, b[0], b[1], b[2], b[3]);
            }
#pragma unroll
            for (int r = 0; r < 4; r++) acc[r] = (acc[r] + accl[r]) + (acc2[r] + acc2l[r]);
            const int col = 8 * warp + 2 * t;
            float* y0 = &s.yp[rank][g * YLD + col];
            float* y1 = &s.yp[rank][(g + 8) * YLD + col];
            *reinterpret_cast<float2*>(y0) = make_float2(acc[0], acc[1]);
            *reinterpret_cast<float2*>(y1) = make_float2(acc[2], acc[3]);
            if (live) {
                ptx::st_async_f32x2(remote(y0), acc[0], acc[1], ybar_peer);
                ptx::st_async_f32x2(remote(y1), acc[2], acc[3], ybar_peer);
            }
        } else {
            if (warp == 8) {
                // A = tril(eta_s (q_t . x_s + 1)) as -A hi/lo A fragments
                float pa[2][4];
                zero(pa[0]);
                zero(pa[1]);
#pragma unroll
                for (int ks = 0; ks < 4; ks++) {
                    uint32_t aq[4], bx[4];
                    ld_a(sQ, ks, lane, aq);
                    ld_b_col(sK, ks, lane, bx);
                    mma(pa[0], aq, bx[0], bx[1]);
                    mma(pa[1], aq, bx[2], bx[3]);
                }
                uint4 hi, lo;
                causal_frag(pa, s.eta, g, t, hi, lo);
                s.afrag[0][lane] = hi;
                s.afrag[1][lane] = lo;
            }
            // -eta_t X[t][:] for the W1 update (k = tokens): 256 threads, two pairs each
#pragma unroll
            for (int k = 0; k < 2; k++) {
                const int i = tid - 256 + 256 * k, row = i >> 5, col = 2 * (i & 31);
                const uint32_t xv = *reinterpret_cast<const uint32_t*>(s.K + swz(row, col));
                const float e = -s.eta[row];
                uint32_t hi, lo;
                ptx::split_pair(e * ptx::bf16_lo_f32(xv), e * ptx::bf16_hi_f32(xv), hi, lo);
                *reinterpret_cast<uint32_t*>(s.EXh + swz(row, col)) = hi;
                *reinterpret_cast<uint32_t*>(s.EXl + swz(row, col)) = lo;
            }
        }
        __syncthreads();
        split::wait_peer(&s.ybar, (uint32_t)(c & 1), &s.abort_flag, abort_peer);

        // ================================================= phase 3: Y = b2 + partials, G2 = dl/dY, E2 = -eta G2 (warp w: token w)
        {
            const int row = warp, col = 2 * lane;
            const float2 p0 = *reinterpret_cast<const float2*>(&s.yp[0][row * YLD + col]);
            const float2 p1 = *reinterpret_cast<const float2*>(&s.yp[1][row * YLD + col]);
            const float y0 = s.b2[col] + p0.x + p1.x, y1 = s.b2[col + 1] + p0.y + p1.y;
            const uint32_t xv = *reinterpret_cast<const uint32_t*>(s.K + swz(row, col));
            const uint32_t vv = *reinterpret_cast<const uint32_t*>(s.V + swz(row, col));
            const float mu = warp_sum(y0 + y1) * (1.f / D);
            const float d0 = y0 - mu, d1 = y1 - mu;
            const float rs = rsqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.f / D) + eps);
            const float xh0 = d0 * rs, xh1 = d1 * rs;
            const float g0 = s.gam[col], g1 = s.gam[col + 1];
            const float gx0 = 2.f * g0 * (ptx::bf16_lo_f32(xv) + g0 * xh0 + s.bet[col] - ptx::bf16_lo_f32(vv));
            const float gx1 = 2.f * g1 * (ptx::bf16_hi_f32(xv) + g1 * xh1 + s.bet[col + 1] - ptx::bf16_hi_f32(vv));
            const float mgx = warp_sum(gx0 + gx1) * (1.f / D);
            const float mgxx = warp_sum(gx0 * xh0 + gx1 * xh1) * (1.f / D);
            const float G0 = rs * (gx0 - mgx - xh0 * mgxx), G1 = rs * (gx1 - mgx - xh1 * mgxx);
            const float e = -s.eta[row];
            uint32_t hi, lo;
            ptx::split_pair(G0, G1, hi, lo);
            *reinterpret_cast<uint32_t*>(s.G2h + swz(row, col)) = hi;
            *reinterpret_cast<uint32_t*>(s.G2l + swz(row, col)) = lo;
            ptx::split_pair(e * G0, e * G1, hi, lo);
            *reinterpret_cast<uint32_t*>(s.E2h + swz(row, col)) = hi;
            *reinterpret_cast<uint32_t*>(s.E2l + swz(row, col)) = lo;
        }
        __syncthreads();

        // ================================================= phase 4: G1 = (G2 W2^T) * GELU'(Z1) on this warp's hidden units
        {
            float acc[4], accl[4];
            zero(acc);
            zero(accl);
            const uint32_t g2h = ptx::smem_addr(s.G2h), g2l = ptx::smem_addr(s.G2l);
#pragma unroll
            for (int ks = 0; ks < 4; ks++) {
                uint32_t ah[4], al[4];
                ld_a(g2h, ks, lane, ah);
                ld_a(g2l, ks, lane, al);
                uint32_t b[4];
                split::ld_w2_ko(sW2h, sW2l, ks, warp, lane, b);
                split::mma3s(acc, accl, ah, al, b[0], b[1], b[2], b[3]);
            }
#pragma unroll
            for (int r = 0; r < 4; r++) acc[r] = (acc[r] + accl[r]) * gelu_prime_sig(z1[r], sg1[r]);
            store_pairs(s.G1h[p], s.G1l[p], g, pc, acc);
        }
        __syncthreads();

        // ================================================= phase 5: Z1q = Q W1 + b1 - A G1, Hq = GELU(Z1q)
        {
            const uint4 fh = s.afrag[0][lane], fl = s.afrag[1][lane];
            const uint32_t ah[4] = {fh.x, fh.y, fh.z, fh.w}, al[4] = {fl.x, fl.y, fl.z, fl.w};
            uint32_t bh[4], bl[4];
            ld_b_tok(ptx::smem_addr(s.G1h[p]), (warp & 7) >> 1, lane, bh);
            ld_b_tok(ptx::smem_addr(s.G1l[p]), (warp & 7) >> 1, lane, bl);
            const int o = 2 * (warp & 1);
            mma3(zq, ah, al, bh[o], bh[o + 1], bl[o], bl[o + 1]);
            float hv[4], sq;
#pragma unroll
            for (int r = 0; r < 4; r++) hv[r] = gelu_sig(zq[r], sq);
            store_pairs(s.Hqh[p], s.Hql[p], g, pc, hv);
        }
        __syncthreads();

        // ================================================= phase 6: partial Hq H^T (warps 0-1), partial Hq W2 (warps 8-15);
        // then, between the arrive and the wait, the W1 / b1 (warps 0-7) and W2 (warps 8-15) updates
        if (warp < NPL) {
            const int pp = warp;
            float acc[2][4];
            zero(acc[0]);
            zero(acc[1]);
#pragma unroll
            for (int kb = 0; kb < 4; kb++) {
                uint32_t ah[4], al[4], bh[4], bl[4];
                ld_a(ptx::smem_addr(s.Hqh[pp]), kb, lane, ah);
                ld_a(ptx::smem_addr(s.Hql[pp]), kb, lane, al);
                ld_b_col(ptx::smem_addr(s.Hh[pp]), kb, lane, bh);
                ld_b_col(ptx::smem_addr(s.Hl[pp]), kb, lane, bl);
                mma3(acc[0], ah, al, bh[0], bh[1], bl[0], bl[1]);
                mma3(acc[1], ah, al, bh[2], bh[3], bl[2], bl[3]);
            }
#pragma unroll
            for (int nt = 0; nt < 2; nt++) {
                float4* dst = &s.a2p[NPL * rank + pp][nt][lane];
                const float4 v = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
                *dst = v;
                ptx::st_cluster_f32x4(remote(dst), v);
            }
        } else if (warp >= 8) {
            const int ot = warp - 8;  // output columns [8 ot, 8 ot + 8)
            float acc[4], accl[4], acc2[4], acc2l[4];
            zero(acc);
            zero(accl);
            zero(acc2);
            zero(acc2l);
#pragma unroll 4
            for (int ks = 0; ks < 4 * NPL; ks++) {
                uint32_t ah[4], al[4];
                ld_a(ptx::smem_addr(s.Hqh[ks >> 2]), ks & 3, lane, ah);
                ld_a(ptx::smem_addr(s.Hql[ks >> 2]), ks & 3, lane, al);
                uint32_t b[4];
                split::ld_w2_kh(sW2h, sW2l, ks, ot, lane, b);
                if (ks & 1) split::mma3s(acc2, acc2l, ah, al, b[0], b[1], b[2], b[3]);
                else split::mma3s(acc, accl, ah, al, b[0], b[1], b[2], b[3]);
            }
#pragma unroll
            for (int r = 0; r < 4; r++) acc[r] = (acc[r] + accl[r]) + (acc2[r] + acc2l[r]);
            const int col = 8 * ot + 2 * t;
            float* z0 = &s.zp[rank][g * YLD + col];
            float* z1p = &s.zp[rank][(g + 8) * YLD + col];
            *reinterpret_cast<float2*>(z0) = make_float2(acc[0], acc[1]);
            *reinterpret_cast<float2*>(z1p) = make_float2(acc[2], acc[3]);
            ptx::st_cluster_f32x2(remote(z0), acc[0], acc[1]);
            ptx::st_cluster_f32x2(remote(z1p), acc[2], acc[3]);
            // every read of W2 in this chunk is done before any warp updates it
            ptx::named_bar_sync(2, 256);
        }
        ptx::cluster_arrive();
        if (warp < 8) {
            // W1^T[hid][in] += G1^T (-eta X), b1 += G1^T (-eta); hidden rows [16 warp, 16 warp + 16)
            uint32_t eh[2], el[2];  // -eta as a B column (n = 0): k = tokens 2t..2t+1 and 2t+8..2t+9
            ptx::split_pair(g == 0 ? -s.eta[2 * t] : 0.f, g == 0 ? -s.eta[2 * t + 1] : 0.f, eh[0], el[0]);
            ptx::split_pair(g == 0 ? -s.eta[2 * t + 8] : 0.f, g == 0 ? -s.eta[2 * t + 9] : 0.f, eh[1], el[1]);
            const int mt = warp, p1 = mt >> 2;
            uint32_t ah[4], al[4];
            ld_a_t(ptx::smem_addr(s.G1h[p1]), mt & 3, lane, ah);
            ld_a_t(ptx::smem_addr(s.G1l[p1]), mt & 3, lane, al);
#pragma unroll
            for (int jp = 0; jp < 4; jp++) {
                uint32_t bh[4], bl[4];
                ld_b_tok(ptx::smem_addr(s.EXh), jp, lane, bh);
                ld_b_tok(ptx::smem_addr(s.EXl), jp, lane, bl);
                float d[2][4];
                zero(d[0]);
                zero(d[1]);
                mma3(d[0], ah, al, bh[0], bh[1], bl[0], bl[1]);
                mma3(d[1], ah, al, bh[2], bh[3], bl[2], bl[3]);
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int rh = 0; rh < 2; rh++) {
                        sr[jp][nt][2 * rh] += d[nt][2 * rh];
                        sr[jp][nt][2 * rh + 1] += d[nt][2 * rh + 1];
                        store_split(jp, nt, rh, sr[jp][nt][2 * rh], sr[jp][nt][2 * rh + 1]);
                    }
            }
            float db[4];
            zero(db);
            mma3(db, ah, al, eh[0], eh[1], el[0], el[1]);
            if (t == 0) {
                s.b1[16 * mt + g] += db[0];
                s.b1[16 * mt + 8 + g] += db[2];
            }
        } else {
            // W2^T[out][hid] += E2^T H; output rows [16 mo, 16 mo + 16), hidden panel pp
            uint32_t ah[4], al[4];
            ld_a_t(ptx::smem_addr(s.E2h), mo, lane, ah);
            ld_a_t(ptx::smem_addr(s.E2l), mo, lane, al);
#pragma unroll
            for (int jp = 0; jp < 4; jp++) {
                uint32_t bh[4], bl[4];
                ld_b_tok(ptx::smem_addr(s.Hh[pp]), jp, lane, bh);
                ld_b_tok(ptx::smem_addr(s.Hl[pp]), jp, lane, bl);
                float d[2][4];
                zero(d[0]);
                zero(d[1]);
                mma3(d[0], ah, al, bh[0], bh[1], bl[0], bl[1]);
                mma3(d[1], ah, al, bh[2], bh[3], bl[2], bl[3]);
#pragma unroll
                for (int nt = 0; nt < 2; nt++)
#pragma unroll
                    for (int rh = 0; rh < 2; rh++) {
                        sr[jp][nt][2 * rh] += d[nt][2 * rh];
                        sr[jp][nt][2 * rh + 1] += d[nt][2 * rh + 1];
                        store_split(jp, nt, rh, sr[jp][nt][2 * rh], sr[jp][nt][2 * rh + 1]);
                    }
            }
        }
        ptx::cluster_wait();

        // ================================================= phase 7 (warps 0-7): Z2q = b2 + partials - A2 G2, b2 update,
        // z = q + LN(Z2q) for this CTA's 8 tokens
        if (warp < 8) {
            const int v = warp;  // output columns [8v, 8v + 8)
            float pa[2][4];
#pragma unroll
            for (int nt = 0; nt < 2; nt++) {
                float4 a = s.a2p[0][nt][lane];
#pragma unroll
                for (int q = 1; q < split::kSplit * NPL; q++) {
                    const float4 b = s.a2p[q][nt][lane];
                    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
                }
                pa[nt][0] = a.x; pa[nt][1] = a.y; pa[nt][2] = a.z; pa[nt][3] = a.w;
            }
            uint4 fh, fl;
            causal_frag(pa, s.eta, g, t, fh, fl);
            const uint32_t ah[4] = {fh.x, fh.y, fh.z, fh.w}, al[4] = {fl.x, fl.y, fl.z, fl.w};
            const int col = 8 * v + 2 * t;
            const float2 p00 = *reinterpret_cast<const float2*>(&s.zp[0][g * YLD + col]);
            const float2 p10 = *reinterpret_cast<const float2*>(&s.zp[1][g * YLD + col]);
            const float2 p01 = *reinterpret_cast<const float2*>(&s.zp[0][(g + 8) * YLD + col]);
            const float2 p11 = *reinterpret_cast<const float2*>(&s.zp[1][(g + 8) * YLD + col]);
            const float bb0 = s.b2[col], bb1 = s.b2[col + 1];
            float z2[4] = {bb0 + p00.x + p10.x, bb1 + p00.y + p10.y, bb0 + p01.x + p11.x, bb1 + p01.y + p11.y};
            uint32_t bh[4], bl[4];
            ld_b_tok(ptx::smem_addr(s.G2h), v >> 1, lane, bh);
            ld_b_tok(ptx::smem_addr(s.G2l), v >> 1, lane, bl);
            const int o = (v & 1) * 2;
            mma3(z2, ah, al, bh[o], bh[o + 1], bl[o], bl[o + 1]);
            *reinterpret_cast<float2*>(&s.Y[g * YLD + col]) = make_float2(z2[0], z2[1]);
            *reinterpret_cast<float2*>(&s.Y[(g + 8) * YLD + col]) = make_float2(z2[2], z2[3]);
            // every read of b2 and of Z2q's producers in this chunk is done
            ptx::named_bar_sync(1, 256);
            if (v < 4) {
                // b2 += E2^T 1 for output rows [16v, 16v + 16)
                uint32_t eh4[4], el4[4];
                ld_a_t(ptx::smem_addr(s.E2h), v, lane, eh4);
                ld_a_t(ptx::smem_addr(s.E2l), v, lane, el4);
                const uint32_t ones = g == 0 ? 0x3f803f80u : 0u;  // (1, 1) in bf16 on column 0
                float db[4];
                zero(db);
                mma(db, eh4, ones, ones);
                mma(db, el4, ones, ones);
                if (t == 0) {
                    s.b2[16 * v + g] += db[0];
                    s.b2[16 * v + 8 + g] += db[2];
                }
            }
            {
                const int row = 8 * (int)rank + v, cc = 2 * lane;
                const float2 zz = *reinterpret_cast<const float2*>(&s.Y[row * YLD + cc]);
                const float mu = warp_sum(zz.x + zz.y) * (1.f / D);
                const float d0 = zz.x - mu, d1 = zz.y - mu;
                const float rs = rsqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.f / D) + eps);
                const uint32_t qv = *reinterpret_cast<const uint32_t*>(s.Q + swz(row, cc));
                float2 o2;
                o2.x = ptx::bf16_lo_f32(qv) + s.gam[cc] * d0 * rs + s.bet[cc];
                o2.y = ptx::bf16_hi_f32(qv) + s.gam[cc + 1] * d1 * rs + s.bet[cc + 1];
                *reinterpret_cast<float2*>(Zbh + (size_t)(c * kChunk + row) * D + cc) = o2;
            }
        }
    }
    // no CTA leaves while the other may still store into its shared memory; after an
    // abort, stores already sent get time to land first
    if (*reinterpret_cast<volatile int*>(&s.abort_flag)) {
        const long long t0 = clock64();
        while (clock64() - t0 < 200000) {
        }
    }
    ptx::cluster_arrive();
    ptx::cluster_wait();
    // ---- final state: this CTA's slice from the registers; CTA 0 writes b2
#pragma unroll
    for (int jp = 0; jp < 4; jp++)
#pragma unroll
        for (int nt = 0; nt < 2; nt++)
#pragma unroll
            for (int rh = 0; rh < 2; rh++) {
                float* WT = w1_warp ? W1_T : W2_T;
                WT[state_index(jp, nt, rh, 0)] = sr[jp][nt][2 * rh];
                WT[state_index(jp, nt, rh, 1)] = sr[jp][nt][2 * rh + 1];
            }
    for (int i = tid; i < HL; i += kThreads) b1_T[bh * HID + hid0 + i] = s.b1[i];
    if (rank == 0 && tid < D) b2_T[bh * D + tid] = s.b2[tid];
}

}  // namespace

bool mlp_tc_supports(const MlpArgs& a) {
    return a.d == D && a.hidden == HID && a.dtype == TTT_BF16 && a.mini_batch == kChunk && a.T > 0 &&
           a.T % kChunk == 0;
}

cudaError_t launch_mlp_tc(const MlpArgs& a, cudaStream_t stream) {
    if (!mlp_tc_supports(a)) return cudaErrorInvalidValue;
    const size_t smem = sizeof(MlpTcSmem) + 128;
    cudaError_t e = cudaFuncSetAttribute(ttt_mlp_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ttt_mlp_tc_kernel<<<a.B * a.H, kThreads, smem, stream>>>(
        a.T, a.H, a.ln_eps, static_cast<const __nv_bfloat16*>(a.Q), static_cast<const __nv_bfloat16*>(a.K),
        static_cast<const __nv_bfloat16*>(a.V), a.eta, a.W1_0, a.b1_0, a.W2_0, a.b2_0, a.gamma, a.beta, a.Z,
        a.W1_T, a.b1_T, a.W2_T, a.b2_T);
    return cudaPeekAtLastError();
}

bool mlp_split_supports(const MlpArgs& a) { return mlp_tc_supports(a); }

cudaError_t read_and_clear_mlp_error(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, split::g_mlp_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(split::g_mlp_error_word, &zero, sizeof(unsigned int));
}

cudaError_t launch_mlp_split(const MlpArgs& a, cudaStream_t stream) {
    if (!mlp_split_supports(a)) return cudaErrorInvalidValue;
    const size_t smem = sizeof(split::Smem) + 128;
    cudaError_t e = cudaFuncSetAttribute(ttt_mlp_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ttt_mlp_split_kernel<<<a.B * a.H * split::kSplit, kThreads, smem, stream>>>(
        a.T, a.H, a.ln_eps, static_cast<const __nv_bfloat16*>(a.Q), static_cast<const __nv_bfloat16*>(a.K),
        static_cast<const __nv_bfloat16*>(a.V), a.eta, a.W1_0, a.b1_0, a.W2_0, a.b2_0, a.gamma, a.beta, a.Z,
        a.W1_T, a.b1_T, a.W2_T, a.b2_T);
    return cudaPeekAtLastError();
}

}  // namespace ttt
