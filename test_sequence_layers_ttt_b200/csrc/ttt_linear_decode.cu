// TTT-Linear decode for d = 64: the scan continued token by token, with the
// state in registers for the whole call.
//
// Method ("Learning to (Learn at Test Time)", literature record, Key
// takeaways bullets 1, 2 and 5).  Per token t at position p of its mini-batch,
// with W_s, b_s the state the mini-batch started from (W_s := W at p = 0):
//   y  = k W_s + b_s,  g = dl/dy (LayerNorm backward of the reconstruction loss)
//   W -= eta_t k^T g,  b -= eta_t g
//   z  = q + LN(q W + b)
// (plain mode: y = k W_s, g = 2 (y - v), z = q W).
//
// One CTA of 256 threads per (batch, head).  Thread (ig, j) = (tid / 64,
// tid % 64) holds column j, rows [16 ig, 16 ig + 16) of W and of W_s in
// registers; a warp's 32 threads cover 32 consecutive columns of a row, so
// every load and store of the state is a 128-byte line.  Per token: the four
// row groups' partial sums of k W_s meet in shared memory, warp 0 runs the
// LayerNorm backward, every thread applies the rank-1 update to its 16
// elements and accumulates its part of q W in the same pass, and warp 0 runs
// the output LayerNorm.  The state is read once and written once per call.
#include "common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int D = 64;
constexpr int kThreads = 256;
constexpr int kRows = D / (kThreads / D);  // rows of W per thread: 16

struct DecodeSmem {
    float k[2][D], q[2][D], v[2][D];  // token vectors, double-buffered by token parity
    float eta[2];
    float part[kThreads / D][D];      // row-group partial sums (k W_s, then q W)
    float g[D];                       // dl/dy of the token
    float gam[D], bet[D];
};

template <typename Tin, bool kPlain>
__global__ void __launch_bounds__(kThreads)
ttt_linear_decode_kernel(int H, int T, int mb, int pos0, float eps, const Tin* __restrict__ Q,
                         const Tin* __restrict__ K, const Tin* __restrict__ V, const float* __restrict__ eta,
                         float* W, float* bvec, float* W_mb, float* b_mb, const float* __restrict__ gamma,
                         const float* __restrict__ beta, float* __restrict__ Z) {
    __shared__ DecodeSmem s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int j = tid & (D - 1), ig = tid / D;
    const long bh = blockIdx.x;
    const int h = (int)(bh % H);
    float* Wbh = W + bh * D * D;
    float* Wmbh = W_mb + bh * D * D;

    float wc[kRows], ws[kRows];
#pragma unroll
    for (int r = 0; r < kRows; r++) wc[r] = Wbh[(ig * kRows + r) * D + j];
    if (pos0 > 0)
#pragma unroll
        for (int r = 0; r < kRows; r++) ws[r] = Wmbh[(ig * kRows + r) * D + j];
    // warp 0 holds b and b_s for columns lane and lane + 32
    float bc[2] = {0.f, 0.f}, bs[2] = {0.f, 0.f};
    if (!kPlain && warp == 0)
#pragma unroll
        for (int e = 0; e < 2; e++) {
            bc[e] = bvec[bh * D + lane + 32 * e];
            if (pos0 > 0) bs[e] = b_mb[bh * D + lane + 32 * e];
        }
    if (tid < D) {
        s.gam[tid] = kPlain ? 1.f : gamma[(long)h * D + tid];
        s.bet[tid] = kPlain ? 0.f : beta[(long)h * D + tid];
    }

    const long tok0 = bh * (long)T;
    for (int t = 0; t < T; t++) {
        const int buf = t & 1;
        if (tid < D) {
            const long gi = (tok0 + t) * D + tid;
            s.k[buf][tid] = to_f32(K[gi]);
            s.q[buf][tid] = to_f32(Q[gi]);
            s.v[buf][tid] = to_f32(V[gi]);
        } else if (tid == D) {
            s.eta[buf] = eta[tok0 + t];
        }
        if ((pos0 + t) % mb == 0) {  // a mini-batch starts at this token: W_s := W
#pragma unroll
            for (int r = 0; r < kRows; r++) ws[r] = wc[r];
            bs[0] = bc[0];
            bs[1] = bc[1];
        }
        __syncthreads();  // token in; the previous token's q W partials consumed

        // partial y over this thread's rows
        float p = 0.f;
#pragma unroll
        for (int r = 0; r < kRows; r++) p = fmaf(s.k[buf][ig * kRows + r], ws[r], p);
        s.part[ig][j] = p;
        __syncthreads();

        if (warp == 0) {
            // y, then g = dl/dy; b -= eta g
            float y[2], gv[2];
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int c = lane + 32 * e;
                y[e] = bs[e] + ((s.part[0][c] + s.part[1][c]) + (s.part[2][c] + s.part[3][c]));
            }
            if (kPlain) {
#pragma unroll
                for (int e = 0; e < 2; e++) gv[e] = 2.f * (y[e] - s.v[buf][lane + 32 * e]);
            } else {
                const float mu = warp_sum(y[0] + y[1]) * (1.f / D);
                const float d0 = y[0] - mu, d1 = y[1] - mu;
                const float rs = rsqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.f / D) + eps);
                const float xh[2] = {d0 * rs, d1 * rs};
                float gx[2];
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    const int c = lane + 32 * e;
                    gx[e] = 2.f * s.gam[c] * (s.k[buf][c] + s.gam[c] * xh[e] + s.bet[c] - s.v[buf][c]);
                }
                const float mgx = warp_sum(gx[0] + gx[1]) * (1.f / D);
                const float mgxx = warp_sum(gx[0] * xh[0] + gx[1] * xh[1]) * (1.f / D);
#pragma unroll
                for (int e = 0; e < 2; e++) gv[e] = rs * (gx[e] - mgx - xh[e] * mgxx);
            }
            const float et = s.eta[buf];
#pragma unroll
            for (int e = 0; e < 2; e++) {
                s.g[lane + 32 * e] = gv[e];
                if (!kPlain) bc[e] -= et * gv[e];
            }
        }
        __syncthreads();

        // W -= eta k^T g on this thread's rows, and the partial q W with the new W
        {
            const float eg = s.eta[buf] * s.g[j];
            float zp = 0.f;
#pragma unroll
            for (int r = 0; r < kRows; r++) {
                wc[r] = fmaf(-s.k[buf][ig * kRows + r], eg, wc[r]);
                zp = fmaf(s.q[buf][ig * kRows + r], wc[r], zp);
            }
            s.part[ig][j] = zp;
        }
        __syncthreads();

        if (warp == 0) {
            float zb[2];
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int c = lane + 32 * e;
                zb[e] = bc[e] + ((s.part[0][c] + s.part[1][c]) + (s.part[2][c] + s.part[3][c]));
            }
            float* out = Z + (tok0 + t) * D;
            if (kPlain) {
                out[lane] = zb[0];
                out[lane + 32] = zb[1];
            } else {
                const float mu = warp_sum(zb[0] + zb[1]) * (1.f / D);
                const float d0 = zb[0] - mu, d1 = zb[1] - mu;
                const float rs = rsqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.f / D) + eps);
                out[lane] = s.q[buf][lane] + s.gam[lane] * d0 * rs + s.bet[lane];
                out[lane + 32] = s.q[buf][lane + 32] + s.gam[lane + 32] * d1 * rs + s.bet[lane + 32];
            }
        }
        // the next token's first barrier orders warp 0's reads of part / q against
        // the next writes to them
    }

    // ---- state out: W, b; W_mb, b_mb when the mini-batch start state changed
#pragma unroll
    for (int r = 0; r < kRows; r++) Wbh[(ig * kRows + r) * D + j] = wc[r];
    const bool boundary = (pos0 + T) % mb == 0;          // the next token starts a mini-batch
    const bool restarted = pos0 == 0 || T > mb - pos0;   // W_s was reset inside this call
    if (boundary || restarted)
#pragma unroll
        for (int r = 0; r < kRows; r++) Wmbh[(ig * kRows + r) * D + j] = boundary ? wc[r] : ws[r];
    if (!kPlain && warp == 0)
#pragma unroll
        for (int e = 0; e < 2; e++) {
            bvec[bh * D + lane + 32 * e] = bc[e];
            if (boundary || restarted) b_mb[bh * D + lane + 32 * e] = boundary ? bc[e] : bs[e];
        }
}

template <typename Tin, bool kPlain>
cudaError_t launch_one(const LinearArgs& a, cudaStream_t stream) {
    ttt_linear_decode_kernel<Tin, kPlain><<<a.B * a.H, kThreads, 0, stream>>>(
        a.H, a.T, a.mini_batch, a.pos0, a.ln_eps, static_cast<const Tin*>(a.Q), static_cast<const Tin*>(a.K),
        static_cast<const Tin*>(a.V), a.eta, a.W_T, a.b_T, a.Wm_T, a.bm_T, a.gamma, a.beta, a.Z);
    return cudaPeekAtLastError();
}

}  // namespace

bool linear_decode_supports(const LinearArgs& a) { return a.d == D; }

// In place: a.W_T / a.b_T hold W, b and a.Wm_T / a.bm_T hold W_s, b_s on entry.
cudaError_t launch_linear_decode(const LinearArgs& a, cudaStream_t stream) {
    if (!linear_decode_supports(a)) return cudaErrorInvalidValue;
    const bool plain = a.mode == TTT_PLAIN;
    if (a.dtype == TTT_BF16)
        return plain ? launch_one<__nv_bfloat16, true>(a, stream) : launch_one<__nv_bfloat16, false>(a, stream);
    return plain ? launch_one<float, true>(a, stream) : launch_one<float, false>(a, stream);
}

}  // namespace ttt
