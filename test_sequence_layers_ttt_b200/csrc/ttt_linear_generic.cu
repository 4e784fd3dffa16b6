// Generic TTT-Linear forward scan: fp32 SIMT, one CTA per (batch, head).
//
// Covers every shape the ABI accepts (d = 16/32/64, bf16 or fp32 Q/K/V, LN or
// plain mode, any mini-batch size, ragged T).  It is the reference CUDA path
// for the fp32 workloads and the fallback for shapes the tensor-core kernel
// does not take.
//
// Algorithm ("Learning to (Learn at Test Time)", literature record, Key
// takeaways bullets 1, 2 and 5), per chunk of C = min(b, 16) tokens, C inside
// one mini-batch:
//   G      = dl/dy of every token of the chunk at the mini-batch start state
//            (W_s, b_s): y = k W_s + b_s, LayerNorm backward.
//   A[t,s] = eta_s (q_t . k_s + 1) for s <= t (plain mode: eta_s q_t . k_s)
//   zbar   = Q W_c + b_c - A G      (W_c: running state at the chunk start;
//            this is q_t W_t + b_t with W_t = W_c - sum_{s<=t} eta_s k_s^T g_s)
//   z      = q + LN(zbar)           (plain mode: z = zbar)
//   W_c   -= K^T diag(eta) G,  b_c -= eta^T G
// and W_s := W_c at every mini-batch boundary.
//
// Decode (the scan continued by T tokens from position pos0 of a mini-batch)
// runs the same loop with the chunks aligned to the stream's mini-batches
// rather than to the call's first token: a chunk never crosses a mini-batch
// boundary, W_s comes in with the call when pos0 > 0, and goes out as the
// start state of the mini-batch the next token falls in.
#include <atomic>

#include "common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kThreads = 256;

template <int D>
struct LinearSmem {
    float Ws[D * D];          // mini-batch start state W_s [in][out]
    float Wc[D * D];          // running state W_c
    float bs[D], bc[D];
    float X[kChunk * D];      // keys of the chunk
    float Vt[kChunk * D];     // values
    float Qt[kChunk * D];     // queries
    float Y[kChunk * D];      // y = X W_s + b_s, then G in place
    float ZQ[kChunk * D];     // Q W_c + b_c, then zbar in place
    float A[kChunk * kChunk];
    float eta[kChunk];
    float gam[D], bet[D];
};

template <int D, typename Tin, bool kPlain>
__global__ void __launch_bounds__(kThreads)
ttt_linear_generic_kernel(int H, int T, int mb, float eps, const Tin* __restrict__ Q,
                          const Tin* __restrict__ K, const Tin* __restrict__ V,
                          const float* __restrict__ eta, const float* W0, const float* b0,
                          const float* __restrict__ gamma, const float* __restrict__ beta,
                          float* __restrict__ Z, float* W_T, float* b_T, int pos0, const float* Ws0,
                          const float* bs0, float* Ws_T, float* bs_T) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    LinearSmem<D>& s = *reinterpret_cast<LinearSmem<D>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int C = mb < kChunk ? mb : kChunk;

    for (int i = tid; i < D * D; i += kThreads) s.Wc[i] = W0[bh * D * D + i];
    if (Ws0 != nullptr)  // decode from inside a mini-batch: its start state comes with the call
        for (int i = tid; i < D * D; i += kThreads) s.Ws[i] = Ws0[bh * D * D + i];
    for (int j = tid; j < D; j += kThreads) {
        s.bs[j] = (kPlain || bs0 == nullptr) ? 0.f : bs0[bh * D + j];
        s.bc[j] = (kPlain || b0 == nullptr) ? 0.f : b0[bh * D + j];
        s.gam[j] = kPlain ? 1.f : gamma[(long)h * D + j];
        s.bet[j] = kPlain ? 0.f : beta[(long)h * D + j];
    }

    const long tok0 = bh * (long)T;
    for (int t0 = 0, n = 0; t0 < T; t0 += n) {
        const int ph = (pos0 + t0) % mb;  // position of the chunk's first token in its mini-batch
        n = min(min(C, T - t0), mb - ph);
        __syncthreads();  // previous chunk fully consumed
        if (ph == 0) {  // mini-batch boundary: W_s := W_c
            for (int i = tid; i < D * D; i += kThreads) s.Ws[i] = s.Wc[i];
            for (int j = tid; j < D; j += kThreads) s.bs[j] = s.bc[j];
        }
        for (int i = tid; i < C * D; i += kThreads) {
            int t = i / D;
            long g = (tok0 + t0 + t) * D + (i % D);
            bool ok = t < n;
            s.X[i] = ok ? to_f32(K[g]) : 0.f;
            s.Vt[i] = ok ? to_f32(V[g]) : 0.f;
            s.Qt[i] = ok ? to_f32(Q[g]) : 0.f;
        }
        for (int t = tid; t < C; t += kThreads) s.eta[t] = t < n ? eta[tok0 + t0 + t] : 0.f;
        __syncthreads();

        // y = X W_s (+ b_s), ZQ = Q W_c (+ b_c), A; only the chunk's n tokens
        for (int o = tid; o < n * D; o += kThreads) {
            int t = o / D, j = o % D;
            float y = kPlain ? 0.f : s.bs[j];
            float zq = kPlain ? 0.f : s.bc[j];
            const float* x = s.X + t * D;
            const float* q = s.Qt + t * D;
#pragma unroll 8
            for (int i = 0; i < D; i++) {
                y = fmaf(x[i], s.Ws[i * D + j], y);
                zq = fmaf(q[i], s.Wc[i * D + j], zq);
            }
            s.Y[o] = y;
            s.ZQ[o] = zq;
        }
        for (int o = tid; o < C * C; o += kThreads) {
            int t = o / C, u = o % C;
            float a = 0.f;
            if (u <= t && t < n) {
                float dot = 0.f;
                for (int i = 0; i < D; i++) dot = fmaf(s.Qt[t * D + i], s.X[u * D + i], dot);
                a = s.eta[u] * (kPlain ? dot : dot + 1.f);
            }
            s.A[o] = a;
        }
        __syncthreads();

        // G = dl/dy, one warp per token
        for (int t = warp; t < n; t += kThreads / 32) {
            float* y = s.Y + t * D;
            if (kPlain) {
                for (int j = lane; j < D; j += 32) y[j] = 2.f * (y[j] - s.Vt[t * D + j]);
                continue;
            }
            float sum = 0.f;
            for (int j = lane; j < D; j += 32) sum += y[j];
            const float mu = warp_sum(sum) / D;
            float sq = 0.f;
            for (int j = lane; j < D; j += 32) sq += (y[j] - mu) * (y[j] - mu);
            const float rs = rsqrtf(warp_sum(sq) / D + eps);
            float sgx = 0.f, sgxx = 0.f;
            constexpr int PER = (D + 31) / 32;
            float gx[PER], xh[PER];
#pragma unroll
            for (int k = 0; k < PER; k++) {
                int j = lane + 32 * k;
                if (j < D) {
                    xh[k] = (y[j] - mu) * rs;
                    float r = s.X[t * D + j] + s.gam[j] * xh[k] + s.bet[j] - s.Vt[t * D + j];
                    gx[k] = 2.f * s.gam[j] * r;
                    sgx += gx[k];
                    sgxx += gx[k] * xh[k];
                }
            }
            const float mgx = warp_sum(sgx) / D, mgxx = warp_sum(sgxx) / D;
#pragma unroll
            for (int k = 0; k < PER; k++) {
                int j = lane + 32 * k;
                if (j < D) y[j] = rs * (gx[k] - mgx - xh[k] * mgxx);
            }
        }
        __syncthreads();

        // zbar = ZQ - A G ; state update W_c -= X^T diag(eta) G, b_c -= eta^T G
        for (int o = tid; o < n * D; o += kThreads) {
            int t = o / D, j = o % D;
            float z = s.ZQ[o];
            for (int u = 0; u <= t; u++) z = fmaf(-s.A[t * C + u], s.Y[u * D + j], z);
            s.ZQ[o] = z;
        }
        for (int o = tid; o < D * D; o += kThreads) {
            int i = o / D, j = o % D;
            float acc = 0.f;
            for (int u = 0; u < n; u++) acc = fmaf(s.X[u * D + i] * s.eta[u], s.Y[u * D + j], acc);
            s.Wc[o] -= acc;
        }
        if (!kPlain)
            for (int j = tid; j < D; j += kThreads) {
                float acc = 0.f;
                for (int u = 0; u < n; u++) acc = fmaf(s.eta[u], s.Y[u * D + j], acc);
                s.bc[j] -= acc;
            }
        __syncthreads();

        // z = q + LN(zbar), one warp per token
        for (int t = warp; t < n; t += kThreads / 32) {
            const float* zb = s.ZQ + t * D;
            float* out = Z + (tok0 + t0 + t) * D;
            if (kPlain) {
                for (int j = lane; j < D; j += 32) out[j] = zb[j];
                continue;
            }
            float sum = 0.f;
            for (int j = lane; j < D; j += 32) sum += zb[j];
            const float mu = warp_sum(sum) / D;
            float sq = 0.f;
            for (int j = lane; j < D; j += 32) sq += (zb[j] - mu) * (zb[j] - mu);
            const float rs = rsqrtf(warp_sum(sq) / D + eps);
            for (int j = lane; j < D; j += 32)
                out[j] = s.Qt[t * D + j] + s.gam[j] * (zb[j] - mu) * rs + s.bet[j];
        }
    }
    __syncthreads();
    for (int i = tid; i < D * D; i += kThreads) W_T[bh * D * D + i] = s.Wc[i];
    if (!kPlain && b_T != nullptr)
        for (int j = tid; j < D; j += kThreads) b_T[bh * D + j] = s.bc[j];
    if (Ws_T != nullptr) {
        // start state of the mini-batch the next token falls in
        const bool boundary = (pos0 + T) % mb == 0;
        for (int i = tid; i < D * D; i += kThreads) Ws_T[bh * D * D + i] = boundary ? s.Wc[i] : s.Ws[i];
        if (!kPlain && bs_T != nullptr)
            for (int j = tid; j < D; j += kThreads) bs_T[bh * D + j] = boundary ? s.bc[j] : s.bs[j];
    }
}

template <int D, typename Tin, bool kPlain>
cudaError_t launch_one(const LinearArgs& a, cudaStream_t stream) {
    auto kern = ttt_linear_generic_kernel<D, Tin, kPlain>;
    const size_t smem = sizeof(LinearSmem<D>);
    // the shared-memory limit is set once per device, so that a launch (a
    // decode step, say, captured in a CUDA graph) makes no other runtime call
    static std::atomic<unsigned long long> attr_set{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(attr_set.load() & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set.fetch_or(bit);
    }
    kern<<<a.B * a.H, kThreads, smem, stream>>>(
        a.H, a.T, a.mini_batch, a.ln_eps, static_cast<const Tin*>(a.Q), static_cast<const Tin*>(a.K),
        static_cast<const Tin*>(a.V), a.eta, a.W0, a.b0, a.gamma, a.beta, a.Z, a.W_T, a.b_T, a.pos0, a.Wm0,
        a.bm0, a.Wm_T, a.bm_T);
    return cudaPeekAtLastError();
}

template <int D>
cudaError_t launch_d(const LinearArgs& a, cudaStream_t stream) {
    const bool plain = a.mode == TTT_PLAIN;
    if (a.dtype == TTT_BF16)
        return plain ? launch_one<D, __nv_bfloat16, true>(a, stream)
                     : launch_one<D, __nv_bfloat16, false>(a, stream);
    return plain ? launch_one<D, float, true>(a, stream) : launch_one<D, float, false>(a, stream);
}

}  // namespace

bool linear_generic_supports(const LinearArgs& a) { return a.d == 16 || a.d == 32 || a.d == 64; }

cudaError_t launch_linear_generic(const LinearArgs& a, cudaStream_t stream) {
    switch (a.d) {
        case 16: return launch_d<16>(a, stream);
        case 32: return launch_d<32>(a, stream);
        case 64: return launch_d<64>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ttt
