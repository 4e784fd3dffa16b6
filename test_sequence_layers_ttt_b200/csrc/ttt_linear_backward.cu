// TTT-Linear layer backward: the gradients an outer training loop needs
// ("Learning to (Learn at Test Time)", literature record, Key takeaways
// bullet 2: the outer loop trains the views theta_K, theta_V, theta_Q, the
// initial weights and the learning rate), for the scan of bullets 1 and 5
// with f(x) = x + LN(x W + b).
//
// Given upstream gradients dZ (and optionally dW_T, db_T of the final state),
// computes the gradients of  sum(Z dZ) + sum(W_T dW_T) + sum(b_T db_T)  with
// respect to Q, K, V, eta, W0, b0, gamma and beta.
//
// Two passes, one CTA per (batch, head), the mini-batch's arrays in fp32 in shared memory (for d = 64
// the block products run on the tensor cores: mma.sync with bf16 hi/lo operands, fp32 accumulation):
//   1. the forward scan records the state each mini-batch starts from, W_j
//      (d x d) and b_j, in the caller's workspace (d^2 + d floats per
//      mini-batch and head): the tensor-core scan kernel's checkpoint variant
//      for bf16, d = 64, mini-batch 16 and T a multiple of 16, otherwise
//      ttt_linear_states_kernel, mini-batch by mini-batch in fp32.
//   2. ttt_linear_backward_kernel walks the mini-batches in reverse.  For each
//      it reloads W_j, b_j, recomputes the mini-batch's intermediates
//        Y = X W + b,  x^ = LN0(Y),  R = X + gamma x^ + beta - V,
//        Gx = 2 gamma R,  G = s (Gx - mean Gx - x^ mean(Gx x^))   (= dl/dY)
//        P = Q X^T,  A = tril(eta_s (P + 1)),  Zb = Q W + b - A G,  z^ = LN0(Zb)
//      and applies the adjoint of each step, carrying dW, db (the gradient of
//      the state after the mini-batch) backwards.  The LayerNorm backward that
//      forms G is differentiated through, including the explicit dependence of
//      G on s = (var Y + eps)^(-1/2).
//   3. ttt_linear_dgamma_kernel sums the per-(batch, head) gamma / beta
//      partials over the batch in a fixed order (deterministic).
// One mini-batch is processed at a time (mini_batch <= 16 tokens).
#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"
#include "timeline.cuh"
#include "ttt_internal.h"

namespace ttt {

// clock64 stamps of the reverse sweep (TTT_TIMELINE builds only): 16 points per mini-batch
TTT_TIMELINE_BUFFER(g_bwd_timeline);

// Workspace of ttt_linear_backward_static: a fixed array that every device
// loading the library holds until the process exits, for callers that cannot
// allocate device memory.  Shared by every call on a device.
static __device__ __align__(256) unsigned char g_backward_static_workspace[kBackwardStaticWorkspaceBytes];

namespace {

constexpr int kBwdThreads = 512;
constexpr int kMaxD = 64, kMaxN = 16;
constexpr int LD = kMaxD + 1;  // padded row length of every [rows][d] array
constexpr int LDN = kMaxN + 1;  // padded row length of the [n][n] token-pair arrays

// C (=|+=) alpha * op(A) op(B), op(A)(i,k) = TA ? A[k][i] : A[i][k], op(B)(k,j) = TB ? B[j][k] : B[k][j].
// Each thread owns a TM x TN block of C in registers, so every element it loads from shared memory
// feeds TN (or TM) multiply-adds; M % TM == 0 and N % TN == 0.
// KC > 0 fixes K at compile time (the k loop unrolls and its addressing folds into offsets).
template <bool TA, bool TB, int TM, int TN, int KC>
__device__ __forceinline__ void bmm_tiled(float* C, int ldc, const float* A, int lda, const float* B, int ldb, int M, int N, int K_,
                          float alpha, bool accumulate) {
    const int K = KC > 0 ? KC : K_;
    // a thread's block is strided: rows i0 + ii * (M / TM), columns j0 + jj * (N / TN), so that the
    // lanes of a warp read consecutive columns (and one or two rows) of shared memory
    const int tm = M / TM, tn = N / TN, tiles = tm * tn;
    for (int tix = threadIdx.x; tix < tiles; tix += blockDim.x) {
        const int i0 = tix / tn, j0 = tix % tn;
        float acc[TM][TN];
#pragma unroll
        for (int ii = 0; ii < TM; ii++)
#pragma unroll
            for (int jj = 0; jj < TN; jj++) acc[ii][jj] = 0.f;
#pragma unroll(KC > 0 ? 8 : 1)
        for (int k = 0; k < K; k++) {
            float a[TM], b[TN];
#pragma unroll
            for (int ii = 0; ii < TM; ii++) a[ii] = TA ? A[k * lda + i0 + ii * tm] : A[(i0 + ii * tm) * lda + k];
#pragma unroll
            for (int jj = 0; jj < TN; jj++) b[jj] = TB ? B[(j0 + jj * tn) * ldb + k] : B[k * ldb + j0 + jj * tn];
#pragma unroll
            for (int ii = 0; ii < TM; ii++)
#pragma unroll
                for (int jj = 0; jj < TN; jj++) acc[ii][jj] = fmaf(a[ii], b[jj], acc[ii][jj]);
        }
#pragma unroll
        for (int ii = 0; ii < TM; ii++)
#pragma unroll
            for (int jj = 0; jj < TN; jj++) {
                float* c = C + (i0 + ii * tm) * ldc + j0 + jj * tn;
                *c = accumulate ? fmaf(alpha, acc[ii][jj], *c) : alpha * acc[ii][jj];
            }
    }
}
// the register block: the largest that leaves no thread without one (4 x 4 down to 1 x 2), for any
// n up to 16 and d a multiple of 16
template <bool TA, bool TB, int KC>
__device__ __forceinline__ void bmm_k(float* C, int ldc, const float* A, int lda, const float* B, int ldb, int M, int N, int K,
                      float alpha, bool accumulate) {
    // the largest block that still gives every thread one
    const int nt = (int)blockDim.x;
    if (M % 4 == 0 && N % 4 == 0 && M * N >= 16 * nt)
        bmm_tiled<TA, TB, 4, 4, KC>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate);
    else if (M % 2 == 0 && N % 4 == 0 && M * N >= 8 * nt)
        bmm_tiled<TA, TB, 2, 4, KC>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate);
    else if (M % 2 == 0 && N % 2 == 0 && M * N >= 4 * nt)
        bmm_tiled<TA, TB, 2, 2, KC>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate);
    else if (N % 2 == 0)
        bmm_tiled<TA, TB, 1, 2, KC>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate);
    else
        bmm_tiled<TA, TB, 1, 1, KC>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate);
}
// The same product on the tensor cores, for M % 16 == 0, N % 8 == 0, K % 16 == 0: warps take
// the 16 x 8 tiles of C in turn; each fp32 operand element is split into bf16 hi + lo (both rounded
// to nearest, |x - hi - lo| <= 2^-16 |x|) and a tile accumulates hi.hi + hi.lo + lo.hi over k in fp32
// (mma.sync m16n8k16).  Fragments are read element by element from the fp32 arrays.
template <bool TA, bool TB, int KC>
__device__ __forceinline__ void bmm_mma(float* C, int ldc, const float* A, int lda, const float* B, int ldb, int M, int N,
                                        int K_, float alpha, bool accumulate, int w0, int wn) {
    const int K = KC > 0 ? KC : K_;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int wr = warp - w0;  // this warp's place in the range of warps the product runs on
    if (wr < 0 || wr >= wn) return;
    const int tn = N / 8, tiles = (M / 16) * tn;
    auto a_at = [&](int i, int k) { return TA ? A[k * lda + i] : A[i * lda + k]; };
    auto b_at = [&](int k, int j) { return TB ? B[j * ldb + k] : B[k * ldb + j]; };
    // The sum over k may visit k in any order that A and B share.  Position m (0..15) of k-step s
    // takes k = s + 4 m when K = 64 and k = 4 (m % 4) + m / 4 when K = 16, so that the eight row
    // lanes g and four pair lanes t of a fragment load fall in distinct banks of the 65-float rows
    // (bank g + 8 t + s for K = 64; at most two lanes per bank for K = 16).
    auto kk = [&](int s, int m) { return KC == 64 ? s + 4 * m : (KC == 16 ? 4 * (m & 3) + (m >> 2) : 16 * s + m); };
    for (int tix = wr; tix < tiles; tix += wn) {
        const int i0 = (tix / tn) * 16, j0 = (tix % tn) * 8;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll(KC > 0 ? 4 : 1)
        for (int s = 0; s < K / 16; s++) {
            const int k0 = kk(s, 2 * t), k1 = kk(s, 2 * t + 1), k8 = kk(s, 2 * t + 8), k9 = kk(s, 2 * t + 9);
            uint32_t ah[4], al[4], bh[2], bl[2];
            ptx::split_pair_rn(a_at(i0 + g, k0), a_at(i0 + g, k1), ah[0], al[0]);
            ptx::split_pair_rn(a_at(i0 + g + 8, k0), a_at(i0 + g + 8, k1), ah[1], al[1]);
            ptx::split_pair_rn(a_at(i0 + g, k8), a_at(i0 + g, k9), ah[2], al[2]);
            ptx::split_pair_rn(a_at(i0 + g + 8, k8), a_at(i0 + g + 8, k9), ah[3], al[3]);
            ptx::split_pair_rn(b_at(k0, j0 + g), b_at(k1, j0 + g), bh[0], bl[0]);
            ptx::split_pair_rn(b_at(k8, j0 + g), b_at(k9, j0 + g), bh[1], bl[1]);
            ptx::mma_bf16(acc, ah[0], ah[1], ah[2], ah[3], bh[0], bh[1]);
            ptx::mma_bf16(acc, ah[0], ah[1], ah[2], ah[3], bl[0], bl[1]);
            ptx::mma_bf16(acc, al[0], al[1], al[2], al[3], bh[0], bh[1]);
        }
#pragma unroll
        for (int r = 0; r < 4; r++) {
            float* c = C + (i0 + g + 8 * (r >> 1)) * ldc + j0 + 2 * t + (r & 1);
            *c = accumulate ? fmaf(alpha, acc[r], *c) : alpha * acc[r];
        }
    }
}
// K = 64 (the head dimension of the hot shapes) and K = 16 (a full mini-batch) unrolled; with kTC
// (the d = 64 kernels) the shapes the tensor cores take go there, on warps [w0, w0 + wn) only, so
// that products of one phase can share the warps out (the FFMA path always uses every thread)
template <bool TA, bool TB, bool kTC>
__device__ __forceinline__ void bmm(float* C, int ldc, const float* A, int lda, const float* B, int ldb, int M, int N, int K,
                    float alpha, bool accumulate, int w0 = 0, int wn = kBwdThreads / 32) {
    if (kTC && M % 16 == 0 && N % 8 == 0 && K % 16 == 0) {
        if (K == 64)
            bmm_mma<TA, TB, 64>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate, w0, wn);
        else if (K == 16)
            bmm_mma<TA, TB, 16>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate, w0, wn);
        else
            bmm_mma<TA, TB, 0>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate, w0, wn);
    } else if (K == 64)
        bmm_k<TA, TB, 64>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate);
    else if (K == 16)
        bmm_k<TA, TB, 16>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate);
    else
        bmm_k<TA, TB, 0>(C, ldc, A, lda, B, ldb, M, N, K, alpha, accumulate);
}

struct BwdSmem {
    float W[kMaxD * LD], b[kMaxD];         // state at the start of the mini-batch
    float dW[kMaxD * LD], db[kMaxD];       // gradient of the state after it
    float dWp[kMaxD * LD], dbp[kMaxD];     // gradient of the state before it
    float X[kMaxN * LD], Qm[kMaxN * LD], Vm[kMaxN * LD], dZ[kMaxN * LD];
    float xh[kMaxN * LD], R[kMaxN * LD], Gx[kMaxN * LD], G[kMaxN * LD], zh[kMaxN * LD];
    float dZb[kMaxN * LD], dG[kMaxN * LD], dQc[kMaxN * LD], dXc[kMaxN * LD], tmp[kMaxN * LD];
    float P[kMaxN * LDN], A[kMaxN * LDN], dA[kMaxN * LDN];
    float s[kMaxN], s2[kMaxN], m1[kMaxN], m2[kMaxN], mdg[kMaxN], ds[kMaxN], e[kMaxN], de[kMaxN];
    float gam[kMaxD], bet[kMaxD], dgam[kMaxD], dbet[kMaxD];
};

// x^ = (y - mean y) s, s = (var y + eps)^(-1/2), per row of y + bias [n][d] (y updated in place to
// y + bias); one warp per row
__device__ __forceinline__ void ln_rows_bias(float* y, const float* bias, float* xh, float* s, int n, int d,
                                             float eps) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int t = warp; t < n; t += nw) {
        float a = 0.f;
        for (int j = lane; j < d; j += 32) {
            y[t * LD + j] += bias[j];
            a += y[t * LD + j];
        }
        const float mu = warp_sum(a) / d;
        float v = 0.f;
        for (int j = lane; j < d; j += 32) {
            const float c = y[t * LD + j] - mu;
            v = fmaf(c, c, v);
        }
        const float rs = rsqrtf(warp_sum(v) / d + eps);
        for (int j = lane; j < d; j += 32) xh[t * LD + j] = (y[t * LD + j] - mu) * rs;
        if (lane == 0) s[t] = rs;
    }
}

// Y = X W + b into tmp; x^, s; R, Gx, m1, m2, G (the forward of one mini-batch up to G); with kWithA
// also P = Q X^T and A = tril(e_s (P + 1)).  After the products every step is local to a token row,
// so one warp per row runs them all with no block barrier in between.
template <bool kTC, bool kWithA>
__device__ __forceinline__ void chunk_inner_grad(BwdSmem& m, int n, int d, float eps) {
    bmm<false, false, kTC>(m.tmp, LD, m.X, LD, m.W, LD, n, d, d, 1.f, false);  // 8 tiles: warps 0-7
    if (kWithA) bmm<false, true, kTC>(m.P, LDN, m.Qm, LD, m.X, LD, n, n, d, 1.f, false, 8, 8);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int t = warp; t < n; t += nw) {
        float* y = m.tmp + t * LD;
        float a = 0.f;
        for (int j = lane; j < d; j += 32) {
            y[j] += m.b[j];
            a += y[j];
        }
        const float mu = warp_sum(a) / d;
        float v = 0.f;
        for (int j = lane; j < d; j += 32) {
            const float c = y[j] - mu;
            v = fmaf(c, c, v);
        }
        const float rs = rsqrtf(warp_sum(v) / d + eps);
        float s1 = 0.f, s2 = 0.f;
        for (int j = lane; j < d; j += 32) {
            const int o = t * LD + j;
            const float xh = (y[j] - mu) * rs;
            const float r = m.X[o] + m.gam[j] * xh + m.bet[j] - m.Vm[o];
            const float gx = 2.f * m.gam[j] * r;
            m.xh[o] = xh;
            m.R[o] = r;
            m.Gx[o] = gx;
            s1 += gx;
            s2 = fmaf(gx, xh, s2);
        }
        const float m1 = warp_sum(s1) / d, m2 = warp_sum(s2) / d;
        for (int j = lane; j < d; j += 32) {
            const int o = t * LD + j;
            m.G[o] = rs * (m.Gx[o] - m1 - m.xh[o] * m2);
        }
        if (lane == 0) {
            m.s[t] = rs;
            m.m1[t] = m1;
            m.m2[t] = m2;
        }
        if (kWithA && lane < n) m.A[t * LDN + lane] = lane <= t ? m.e[lane] * (m.P[t * LDN + lane] + 1.f) : 0.f;
    }
    __syncthreads();
}

// The next mini-batch's inputs, held in registers while the current one computes, so that their
// global loads overlap the math instead of each waiting out a memory round trip.  Thread tid holds
// elements tid + k * kBwdThreads of each array (n <= 16 tokens, d <= 64).
template <typename T, bool kTokens, bool kBackward>
struct Prefetch {
    static constexpr int kTok = kMaxN * kMaxD / kBwdThreads;  // 2
    static constexpr int kSt = kMaxD * kMaxD / kBwdThreads;   // 8
    // the token rows are held as loaded (bf16 or fp32) and converted in commit(): a conversion
    // here would make every warp wait for its loads before going on
    T x[kTok], q[kTok], v[kTok];
    float dz[kTok], e, w[kSt], bb;
    int n = 0;

    __device__ void issue(const T* Q, const T* K, const T* V, const float* eta, const float* dZ, const float* st,
                          size_t base, int n_, int d) {
        n = n_;
        const int tid = threadIdx.x;
#pragma unroll
        for (int k = 0; k < kTok; k++) {
            const int i = tid + k * kBwdThreads;
            if (i < n * d) {
                const size_t gi = base * d + i;
                x[k] = K[gi];
                q[k] = Q[gi];
                v[k] = V[gi];
                if (kBackward) dz[k] = dZ[gi];
            }
        }
        if (tid < n) e = eta[base + tid];
        if (kBackward) {
#pragma unroll
            for (int k = 0; k < kSt; k++) {
                const int i = tid + k * kBwdThreads;
                if (i < d * d) w[k] = st[i];
            }
            if (tid < d) bb = st[d * d + tid];
        }
    }
    __device__ void commit(BwdSmem& m, int d) const {
        const int tid = threadIdx.x;
#pragma unroll
        for (int k = 0; k < kTok; k++) {
            const int i = tid + k * kBwdThreads;
            if (i < n * d) {
                const int o = (i / d) * LD + i % d;
                m.X[o] = to_f32(x[k]);
                m.Qm[o] = to_f32(q[k]);
                m.Vm[o] = to_f32(v[k]);
                if (kBackward) m.dZ[o] = dz[k];
            }
        }
        if (tid < n) m.e[tid] = e;
        if (kBackward) {
#pragma unroll
            for (int k = 0; k < kSt; k++) {
                const int i = tid + k * kBwdThreads;
                if (i < d * d) m.W[(i / d) * LD + i % d] = w[k];
            }
            if (tid < d) m.b[tid] = bb;
        }
    }
};

// ------------------------------------------------------------------ pass 1: states
// DT: the head dimension, fixed at compile time so that every index computation folds
template <typename T, int DT>
__global__ void __launch_bounds__(kBwdThreads, 1)
ttt_linear_states_kernel(int T_, int d_arg, int mb, float eps, const T* Q, const T* K, const T* V, const float* eta,
                         const float* W0, const float* b0, const float* gamma, const float* beta, int H,
                         float* states) {
    extern __shared__ float smem_f[];
    BwdSmem& m = *reinterpret_cast<BwdSmem*>(smem_f);
    constexpr int d = DT;
    constexpr bool kTC = DT == 64;  // products on the tensor cores
    (void)d_arg;
    const int bh = blockIdx.x, h = bh % H;
    const int nmb = (T_ + mb - 1) / mb;
    const size_t sz = (size_t)d * d + d;
    for (int i = threadIdx.x; i < d * d; i += blockDim.x) m.W[(i / d) * LD + i % d] = W0[(size_t)bh * d * d + i];
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
        m.b[j] = b0[(size_t)bh * d + j];
        m.gam[j] = gamma[h * d + j];
        m.bet[j] = beta[h * d + j];
    }
    __syncthreads();
    Prefetch<T, true, false> pf;
    if (nmb > 0) pf.issue(Q, K, V, eta, nullptr, nullptr, (size_t)bh * T_, min(mb, T_), d);
    for (int jb = 0; jb < nmb; jb++) {
        const int t0 = jb * mb, n_rt = min(mb, T_ - t0);
        float* st = states + ((size_t)bh * nmb + jb) * sz;
        for (int i = threadIdx.x; i < d * d; i += blockDim.x) st[i] = m.W[(i / d) * LD + i % d];
        for (int j = threadIdx.x; j < d; j += blockDim.x) st[d * d + j] = m.b[j];
        pf.commit(m, d);
        if (jb + 1 < nmb)
            pf.issue(Q, K, V, eta, nullptr, nullptr, (size_t)bh * T_ + t0 + mb, min(mb, T_ - t0 - mb), d);
        __syncthreads();
        // full mini-batches take a copy of the body with n fixed at compile time
        auto chunk = [&](auto nc) {
            constexpr int NC = decltype(nc)::value;
            const int n = NC > 0 ? NC : n_rt;
            chunk_inner_grad<kTC, false>(m, n, d, eps);
            // W -= X^T diag(e) G, b -= G^T e
            for (int i = threadIdx.x; i < n * d; i += blockDim.x) {
                const int t = i / d, o = t * LD + i % d;
                m.tmp[o] = m.e[t] * m.G[o];
            }
            __syncthreads();
            bmm<true, false, kTC>(m.W, LD, m.X, LD, m.tmp, LD, d, d, n, -1.f, true);
            for (int j = threadIdx.x; j < d; j += blockDim.x) {
                float a = 0.f;
                for (int t = 0; t < n; t++) a += m.tmp[t * LD + j];
                m.b[j] -= a;
            }
            __syncthreads();
        };
        if (n_rt == kMaxN)
            chunk(std::integral_constant<int, kMaxN>{});
        else
            chunk(std::integral_constant<int, 0>{});
    }
}

// ------------------------------------------------------------------ pass 2: the reverse sweep
template <typename T, int DT>
__global__ void __launch_bounds__(kBwdThreads, 1)
ttt_linear_backward_kernel(int T_, int d_arg, int mb, float eps, const T* Q, const T* K, const T* V, const float* eta,
                           const float* gamma, const float* beta, int H, const float* states, const float* dZ,
                           const float* dW_T, const float* db_T, float* dQ, float* dK, float* dV, float* deta,
                           float* dW0, float* db0, float* gb_partial) {
    extern __shared__ float smem_f[];
    BwdSmem& m = *reinterpret_cast<BwdSmem*>(smem_f);
    TTT_TIMELINE_SMEM();
    constexpr int d = DT;
    constexpr bool kTC = DT == 64;  // products on the tensor cores
    (void)d_arg;
    const int bh = blockIdx.x, h = bh % H;
    const int nmb = (T_ + mb - 1) / mb;
    const size_t sz = (size_t)d * d + d;
    const float inv_d = 1.f / d;
    for (int i = threadIdx.x; i < d * d; i += blockDim.x)
        m.dW[(i / d) * LD + i % d] = dW_T ? dW_T[(size_t)bh * d * d + i] : 0.f;
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
        m.db[j] = db_T ? db_T[(size_t)bh * d + j] : 0.f;
        m.gam[j] = gamma[h * d + j];
        m.bet[j] = beta[h * d + j];
        m.dgam[j] = 0.f;
        m.dbet[j] = 0.f;
    }
    __syncthreads();
    Prefetch<T, true, true> pf;
    auto issue = [&](int jb) {
        const int t0 = jb * mb;
        pf.issue(Q, K, V, eta, dZ, states + ((size_t)bh * nmb + jb) * sz, (size_t)bh * T_ + t0, min(mb, T_ - t0),
                 d);
    };
    // the carried gradient of the state (dW, db) and the one being formed for the state before the
    // current mini-batch (dW_prev, db_prev)
    float* cW = m.dW;
    float* cWp = m.dWp;
    float* cb = m.db;
    float* cbp = m.dbp;
    // point k of mini-batch jb's step (CTA 0, TTT_TIMELINE builds; nothing otherwise)
    auto stamp = [&](int jb_, int k) {
        TTT_STAMP(g_bwd_timeline, threadIdx.x == 0, k >> 3, nmb - 1 - jb_, k & 7);
        (void)jb_;
        (void)k;
    };
    if (nmb > 0) issue(nmb - 1);
    for (int jb = nmb - 1; jb >= 0; jb--) {
        const int t0 = jb * mb, n_rt = min(mb, T_ - t0);
        const size_t base = (size_t)bh * T_ + t0;
        pf.commit(m, d);
        stamp(jb, 14);
        if (jb > 0) issue(jb - 1);
        stamp(jb, 15);
        __syncthreads();
        // full mini-batches take a copy of the body with n fixed at compile time
        auto chunk = [&](auto nc) {
            constexpr int NC = decltype(nc)::value;
            const int n = NC > 0 ? NC : n_rt;
            stamp(jb, 0);
            // ---- recompute the mini-batch's forward
            chunk_inner_grad<kTC, true>(m, n, d, eps);  // also P = Q X^T and A
            // Zb = Q W + b - A G (into tmp), z^ = LN0(Zb).  The two products give each 16 x 8 tile of C to
            // the same warp (off the tensor cores, each element to the same thread), so the second
            // follows the first without a barrier.
            bmm<false, false, kTC>(m.tmp, LD, m.Qm, LD, m.W, LD, n, d, d, 1.f, false, 0, 8);
            bmm<false, false, kTC>(m.tmp, LD, m.A, LDN, m.G, LD, n, d, n, -1.f, true, 0, 8);
            __syncthreads();
            stamp(jb, 1);
            ln_rows_bias(m.tmp, m.b, m.zh, m.s2, n, d, eps);
            __syncthreads();
            stamp(jb, 2);
            // ---- z = q + gamma z^ + beta
            for (int j = threadIdx.x; j < d; j += blockDim.x) {
                float a = 0.f, c = 0.f;
                for (int t = 0; t < n; t++) {
                    a = fmaf(m.dZ[t * LD + j], m.zh[t * LD + j], a);
                    c += m.dZ[t * LD + j];
                }
                m.dgam[j] += a;
                m.dbet[j] += c;
            }
            // dQ = dZ (the residual); dZb = LNback(gamma dZ), one warp per row
            {
                const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
                for (int t = warp; t < n; t += nw) {
                    float a = 0.f, c = 0.f;
                    for (int j = lane; j < d; j += 32) {
                        const int o = t * LD + j;
                        const float g_ = m.dZ[o] * m.gam[j];
                        m.dQc[o] = m.dZ[o];
                        m.dZb[o] = g_;
                        a += g_;
                        c = fmaf(g_, m.zh[o], c);
                    }
                    const float ma = warp_sum(a) / d, mc = warp_sum(c) / d;
                    for (int j = lane; j < d; j += 32) {
                        const int o = t * LD + j;
                        m.dZb[o] = m.s2[t] * (m.dZb[o] - ma - m.zh[o] * mc);
                    }
                }
            }
            __syncthreads();
            stamp(jb, 3);
            // ---- Zb = Q W + b - A G
            bmm<false, true, kTC>(m.dQc, LD, m.dZb, LD, m.W, LD, n, d, d, 1.f, true, 0, 8);  // dQ += dZb W^T
            bmm<true, false, kTC>(cWp, LD, m.Qm, LD, m.dZb, LD, d, d, n, 1.f, false);       // dW_prev = Q^T dZb
            bmm<true, false, kTC>(m.dG, LD, m.A, LDN, m.dZb, LD, n, d, n, -1.f, false, 8, 8);  // dG = -A^T dZb
            // ---- W' = W - X^T diag(e) G, b' = b - G^T e:  dEG = -(X dW) - db (into tmp; -X dW here)
            bmm<false, false, kTC>(m.tmp, LD, m.X, LD, cW, LD, n, d, d, -1.f, false, 8, 8);
            for (int j = threadIdx.x; j < d; j += blockDim.x) {
                float a = 0.f;
                for (int t = 0; t < n; t++) a += m.dZb[t * LD + j];
                cbp[j] = a + cb[j];
            }
            __syncthreads();
            stamp(jb, 4);
            bmm<false, true, kTC>(m.dA, LDN, m.dZb, LD, m.G, LD, n, n, d, -1.f, false);  // dA = -(dZb G^T)
            __syncthreads();
            stamp(jb, 5);
            for (int i = threadIdx.x; i < n * n; i += blockDim.x) {
                const int t = i / n, s_ = i % n;
                if (s_ > t) m.dA[t * LDN + s_] = 0.f;
            }
            for (int i = threadIdx.x; i < n * d; i += blockDim.x) {
                const int t = i / d, j = i % d, o = t * LD + j;
                m.tmp[o] -= cb[j];
                m.dG[o] = fmaf(m.e[t], m.tmp[o], m.dG[o]);
            }
            __syncthreads();
            stamp(jb, 6);
            {
                const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
                for (int t = warp; t < n; t += nw) {  // de = sum_j dEG G + sum_t dA (P + 1)
                    float a = 0.f;
                    for (int j = lane; j < d; j += 32) a = fmaf(m.tmp[t * LD + j], m.G[t * LD + j], a);
                    a = warp_sum(a);
                    float c = 0.f;
                    for (int r = lane; r < n; r += 32) c = fmaf(m.dA[r * LDN + t], m.P[r * LDN + t] + 1.f, c);
                    c = warp_sum(c);
                    if (lane == 0) m.de[t] = a + c;
                }
            }
            __syncthreads();  // tmp and dA are read above and overwritten below
            stamp(jb, 7);
            // dX = -(e G) dW^T  (tmp <- e G)
            for (int i = threadIdx.x; i < n * d; i += blockDim.x) {
                const int t = i / d, o = t * LD + i % d;
                m.tmp[o] = m.e[t] * m.G[o];
            }
            for (int t = threadIdx.x; t < n; t += blockDim.x) deta[base + t] = m.de[t];  // final
            // ---- A = tril(e_s (P + 1)), P = Q X^T:  dP = dA e_s (into dA)
            for (int i = threadIdx.x; i < n * n; i += blockDim.x) m.dA[(i / n) * LDN + i % n] *= m.e[i % n];
            __syncthreads();
            stamp(jb, 8);
            // dX = -(e G) dW^T + dP^T Q (the same tiles on the same warps, so no barrier between them)
            bmm<false, true, kTC>(m.dXc, LD, m.tmp, LD, cW, LD, n, d, d, -1.f, false, 0, 8);
            bmm<true, false, kTC>(m.dXc, LD, m.dA, LDN, m.Qm, LD, n, d, n, 1.f, true, 0, 8);
            bmm<false, false, kTC>(m.dQc, LD, m.dA, LDN, m.X, LD, n, d, n, 1.f, true, 8, 8);   // dQ += dP X
            // dW_prev += dW (the state passes through)
            for (int i = threadIdx.x; i < d * d; i += blockDim.x) {
                const int o = (i / d) * LD + i % d;
                cWp[o] += cW[o];
            }
            // ---- G = s (Gx - m1 - x^ m2), Gx = 2 gamma R, R = X + gamma x^ + beta - V
            {
                const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
                for (int t = warp; t < n; t += nw) {
                    float a = 0.f, c = 0.f, e2 = 0.f;
                    for (int j = lane; j < d; j += 32) {
                        const int o = t * LD + j;
                        a = fmaf(m.dG[o], m.xh[o], a);
                        c += m.dG[o];
                        e2 = fmaf(m.dG[o], m.Gx[o] - m.m1[t] - m.xh[o] * m.m2[t], e2);
                    }
                    a = warp_sum(a) * inv_d;
                    c = warp_sum(c) * inv_d;
                    e2 = warp_sum(e2);
                    if (lane == 0) {
                        m.mdg[t] = a;
                        m.m1[t] = c;  // m1 is no longer needed: reuse it for mean(dG)
                        m.ds[t] = e2;
                    }
                }
            }
            __syncthreads();
            stamp(jb, 9);
            // dGx (into dZb), dR (into dG), and dY = LNback(dxh) - ds s^2 x^ / d (into tmp): x^ = LN0(Y),
            // and s appears explicitly in G; one warp per row
            {
                const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
                for (int t = warp; t < n; t += nw) {
                    for (int j = lane; j < d; j += 32) dQ[(base + t) * d + j] = m.dQc[t * LD + j];  // final
                    const float s_ = m.s[t];
                    float a = 0.f, c = 0.f;
                    for (int j = lane; j < d; j += 32) {
                        const int o = t * LD + j;
                        const float dgx = s_ * (m.dG[o] - m.m1[t]) - s_ * m.mdg[t] * m.xh[o];
                        const float dxh = -s_ * m.m2[t] * m.dG[o] - s_ * m.mdg[t] * m.Gx[o];
                        const float dr = 2.f * m.gam[j] * dgx;
                        const float dx = dxh + m.gam[j] * dr;
                        m.dZb[o] = dgx;
                        m.tmp[o] = dx;
                        m.dG[o] = dr;
                        a += dx;
                        c = fmaf(dx, m.xh[o], c);
                    }
                    const float ma = warp_sum(a) / d, mc = warp_sum(c) / d;
                    for (int j = lane; j < d; j += 32) {
                        const int o = t * LD + j;
                        m.tmp[o] = s_ * (m.tmp[o] - ma - m.xh[o] * mc);
                        m.tmp[o] -= m.ds[t] * s_ * s_ * m.xh[o] * inv_d;
                    }
                }
            }
            __syncthreads();
            stamp(jb, 10);
            for (int j = threadIdx.x; j < d; j += blockDim.x) {
                float a = 0.f, c = 0.f;
                for (int t = 0; t < n; t++) {
                    const int o = t * LD + j;
                    a += 2.f * m.R[o] * m.dZb[o] + m.dG[o] * m.xh[o];
                    c += m.dG[o];
                }
                m.dgam[j] += a;
                m.dbet[j] += c;
            }
            for (int i = threadIdx.x; i < n * d; i += blockDim.x) {
                const int t = i / d, j = i % d, o = t * LD + j;
                m.dXc[o] += m.dG[o];
                dV[(base + t) * d + j] = -m.dG[o];
            }
            __syncthreads();
            stamp(jb, 11);
            // ---- Y = X W + b
            bmm<false, true, kTC>(m.dXc, LD, m.tmp, LD, m.W, LD, n, d, d, 1.f, true, 0, 8);  // dX += dY W^T
            bmm<true, false, kTC>(cWp, LD, m.X, LD, m.tmp, LD, d, d, n, 1.f, true, 8, 8);  // dW_prev += X^T dY
            for (int j = threadIdx.x; j < d; j += blockDim.x) {
                float a = 0.f;
                for (int t = 0; t < n; t++) a += m.tmp[t * LD + j];
                cbp[j] += a;
            }
            __syncthreads();
            stamp(jb, 12);
            for (int i = threadIdx.x; i < n * d; i += blockDim.x) {
                const int t = i / d, j = i % d, o = t * LD + j;
                dK[(base + t) * d + j] = m.dXc[o];
            }
            // the gradient of the state before this mini-batch becomes the carried one: the two
            // buffers swap roles (the next mini-batch overwrites cWp, cbp before reading them)
            float* const sw = cW;
            cW = cWp;
            cWp = sw;
            float* const sb = cb;
            cb = cbp;
            cbp = sb;
            stamp(jb, 13);
        };
        if (n_rt == kMaxN)
            chunk(std::integral_constant<int, kMaxN>{});
        else
            chunk(std::integral_constant<int, 0>{});
    }
    __syncthreads();
    for (int r = 0; r < 2; r++) TTT_TIMELINE_FLUSH(g_bwd_timeline, threadIdx.x == 0, r);
    for (int i = threadIdx.x; i < d * d; i += blockDim.x) dW0[(size_t)bh * d * d + i] = cW[(i / d) * LD + i % d];
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
        db0[(size_t)bh * d + j] = cb[j];
        gb_partial[((size_t)bh * 2 + 0) * d + j] = m.dgam[j];
        gb_partial[((size_t)bh * 2 + 1) * d + j] = m.dbet[j];
    }
}

// ------------------------------------------------------------------ pass 3: gamma / beta over the batch
__global__ void ttt_linear_dgamma_kernel(int B, int H, int d, const float* gb_partial, float* dgamma, float* dbeta) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= H * d) return;
    const int h = i / d, j = i % d;
    float a = 0.f, c = 0.f;
    for (int b = 0; b < B; b++) {
        const size_t bh = (size_t)b * H + h;
        a += gb_partial[(bh * 2 + 0) * d + j];
        c += gb_partial[(bh * 2 + 1) * d + j];
    }
    dgamma[i] = a;
    dbeta[i] = c;
}

}  // namespace

bool linear_backward_supports(const LinearBwdArgs& a) {
    return a.f.mode == TTT_LN_RESIDUAL && (a.f.d == 16 || a.f.d == 32 || a.f.d == 64) && a.f.mini_batch >= 1 &&
           a.f.mini_batch <= kMaxN;
}

size_t linear_backward_workspace_bytes(int B, int H, int T, int d, int mini_batch) {
    if (B < 1 || H < 1 || T < 0 || d < 1 || mini_batch < 1) return 0;
    const size_t nmb = ((size_t)T + mini_batch - 1) / mini_batch;
    const size_t bh = (size_t)B * H;
    return (bh * nmb * ((size_t)d * d + d) + bh * 2 * d) * sizeof(float);
}

namespace {

template <typename T, int DT>
cudaError_t launch_dt(const LinearBwdArgs& a, float* states, float* gb, cudaStream_t stream) {
    const LinearArgs& f = a.f;
    const int BH = f.B * f.H;
    const size_t smem = sizeof(BwdSmem);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(ttt_linear_states_kernel<T, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(ttt_linear_backward_kernel<T, DT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess)
        return e;
    auto* Q = static_cast<const T*>(f.Q);
    auto* K = static_cast<const T*>(f.K);
    auto* V = static_cast<const T*>(f.V);
    if (f.T > 0) {
        // The tensor-core forward scan writes the checkpoints where it takes the shape (bf16, d = 64,
        // mini-batch 16, T a multiple of 16); the fp32 states pass covers every other shape.
        if (std::is_same<T, __nv_bfloat16>::value && DT == 64 && linear_tc_supports(f)) {
            if ((e = launch_linear_tc_checkpoints(f, states, stream)) != cudaSuccess) return e;
        } else {
            ttt_linear_states_kernel<T, DT><<<BH, kBwdThreads, smem, stream>>>(
                f.T, f.d, f.mini_batch, f.ln_eps, Q, K, V, f.eta, f.W0, f.b0, f.gamma, f.beta, f.H, states);
        }
    }
    ttt_linear_backward_kernel<T, DT><<<BH, kBwdThreads, smem, stream>>>(
        f.T, f.d, f.mini_batch, f.ln_eps, Q, K, V, f.eta, f.gamma, f.beta, f.H, states, a.dZ, a.dW_T, a.db_T, a.dQ,
        a.dK, a.dV, a.deta, a.dW0, a.db0, gb);
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_typed(const LinearBwdArgs& a, float* states, float* gb, cudaStream_t stream) {
    switch (a.f.d) {
        case 16: return launch_dt<T, 16>(a, states, gb, stream);
        case 32: return launch_dt<T, 32>(a, states, gb, stream);
        case 64: return launch_dt<T, 64>(a, states, gb, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_linear_backward(const LinearBwdArgs& a, float* workspace, cudaStream_t stream) {
    if (!linear_backward_supports(a)) return cudaErrorInvalidValue;
    const LinearArgs& f = a.f;
    const int BH = f.B * f.H;
    const size_t nmb = ((size_t)f.T + f.mini_batch - 1) / f.mini_batch;
    float* states = workspace;
    float* gb = workspace + (size_t)BH * nmb * ((size_t)f.d * f.d + f.d);
    cudaError_t e = f.dtype == TTT_BF16 ? launch_typed<__nv_bfloat16>(a, states, gb, stream)
                                        : launch_typed<float>(a, states, gb, stream);
    if (e != cudaSuccess) return e;
    const int hd = f.H * f.d;
    ttt_linear_dgamma_kernel<<<(hd + 255) / 256, 256, 0, stream>>>(f.B, f.H, f.d, gb, a.dgamma, a.dbeta);
    return cudaPeekAtLastError();
}

}  // namespace ttt

namespace ttt {

// Device address of the static workspace on the current device.  Host code
// cannot use the array's name as a device pointer; cudaGetSymbolAddress gives
// the address, once per device (with that device current), cached for later
// calls.  Returns nullptr if the runtime reports an error.
float* backward_static_workspace() {
    constexpr int kMaxDevices = 64;
    static std::atomic<void*> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    void* p = cache[dev].load(std::memory_order_acquire);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_backward_static_workspace) != cudaSuccess) return nullptr;
        cache[dev].store(p, std::memory_order_release);
    }
    return static_cast<float*>(p);
}

}  // namespace ttt

#ifdef TTT_TIMELINE
namespace ttt {
cudaError_t read_bwd_timeline(long long* out) {
    return cudaMemcpyFromSymbol(out, g_bwd_timeline, sizeof(g_bwd_timeline));
}
}  // namespace ttt
#endif
