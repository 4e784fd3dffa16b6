// Generic TTT-MLP forward scan: fp32 SIMT, one CTA per (batch, head), d = 64,
// hidden = 256.  f(x) = x + LN(GELU(x W1 + b1) W2 + b2).
//
// Per chunk of C = min(b, 16) tokens inside one mini-batch
// ("Learning to (Learn at Test Time)", literature record, Key takeaways
// bullets 1, 2 and 5; the abstract names the two-layer MLP state):
//   at the mini-batch start state (W1_s, b1_s, W2_s, b2_s), for every token:
//     z1 = k W1_s + b1_s, h = GELU(z1), y = h W2_s + b2_s
//     G2 = dl/dy (LayerNorm backward), G1 = (G2 W2_s^T) * GELU'(z1)
//   outputs with the running state (W1_c ...) at the chunk start:
//     z1q = Q W1_c + b1_c - A G1,        A[t,s]  = eta_s (q_t . k_s + 1),   s <= t
//     hq  = GELU(z1q)
//     z2q = hq W2_c + b2_c - A2 G2,      A2[t,s] = eta_s (hq_t . h_s + 1),  s <= t
//     z   = q + LN(z2q)
//   (q_t W1_t with W1_t = W1_c - sum_{s<=t} eta_s k_s^T G1_s, and the same for
//   the second layer, so no per-token state is formed)
//   update: W1_c -= K^T diag(eta) G1, b1_c -= eta^T G1, W2_c -= H^T diag(eta) G2,
//           b2_c -= eta^T G2.
// When b > 16 the start state lives in W1_T/b1_T/W2_T/b2_T (the caller's
// final-state buffers) while the running state stays in shared memory.
//
// Decode (the scan continued by T tokens from position pos0 of a mini-batch):
// the start state lives in the caller's W*_mb buffers (read when pos0 > 0),
// the chunks are aligned to the stream's mini-batches, and W*_mb is left as
// the start state of the mini-batch the next token falls in.
#include "common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kThreads = 256;
constexpr int D = 64;
constexpr int HID = 256;
constexpr int LDW2 = D + 1;  // padded row stride of W2 in shared memory

struct MlpSmem {
    float W1c[D * HID];      // [in][hid]
    float W2c[HID * LDW2];   // [hid][out], padded rows
    float b1c[HID], b2c[D];
    float X[kChunk * D], Vt[kChunk * D], Qt[kChunk * D];
    float Z1[kChunk * HID];  // z1 at the start state; later hq
    float Hs[kChunk * HID];  // h = GELU(z1)
    float G1[kChunk * HID];
    float Y2[kChunk * D];    // y, then G2
    float Zq2[kChunk * D];
    float A[kChunk * kChunk], A2[kChunk * kChunk];
    float eta[kChunk];
    float gam[D], bet[D];
};

template <typename Tin>
__global__ void __launch_bounds__(kThreads)
ttt_mlp_generic_kernel(int H, int T, int mb, float eps, const Tin* __restrict__ Q,
                       const Tin* __restrict__ K, const Tin* __restrict__ V,
                       const float* __restrict__ eta, const float* W1_0, const float* b1_0,
                       const float* W2_0, const float* b2_0, const float* __restrict__ gamma,
                       const float* __restrict__ beta, float* __restrict__ Z, float* W1_T,
                       float* b1_T, float* W2_T, float* b2_T, int pos0, float* W1_mb, float* b1_mb,
                       float* W2_mb, float* b2_mb) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    MlpSmem& s = *reinterpret_cast<MlpSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long bh = blockIdx.x;
    const int h = (int)(bh % H);
    const int C = mb < kChunk ? mb : kChunk;
    const bool decode = W1_mb != nullptr;
    const bool start_in_global = decode || mb > kChunk;

    // global start-state buffers: the caller's W*_mb (decode) or W*_T (b > 16)
    float* gW1 = (decode ? W1_mb : W1_T) + bh * D * HID;
    float* gW2 = (decode ? W2_mb : W2_T) + bh * HID * D;
    float* gb1 = (decode ? b1_mb : b1_T) + bh * HID;
    float* gb2 = (decode ? b2_mb : b2_T) + bh * D;
    for (int i = tid; i < D * HID; i += kThreads) s.W1c[i] = W1_0[bh * D * HID + i];
    for (int i = tid; i < HID * D; i += kThreads) s.W2c[(i / D) * LDW2 + i % D] = W2_0[bh * HID * D + i];
    for (int k = tid; k < HID; k += kThreads) s.b1c[k] = b1_0[bh * HID + k];
    for (int j = tid; j < D; j += kThreads) {
        s.b2c[j] = b2_0[bh * D + j];
        s.gam[j] = gamma[(long)h * D + j];
        s.bet[j] = beta[(long)h * D + j];
    }
    // start-state views: shared (b <= 16, start == running at chunk start) or global
    const float* W1s = start_in_global ? gW1 : s.W1c;
    const float* W2s = start_in_global ? gW2 : s.W2c;
    const int ldw2s = start_in_global ? D : LDW2;
    const float* b1s = start_in_global ? gb1 : s.b1c;
    const float* b2s = start_in_global ? gb2 : s.b2c;

    const long tok0 = bh * (long)T;
    for (int t0 = 0, n = 0; t0 < T; t0 += n) {
        const int ph = (pos0 + t0) % mb;  // position of the chunk's first token in its mini-batch
        n = min(min(C, T - t0), mb - ph);
        __syncthreads();
        if (start_in_global && ph == 0) {
            for (int i = tid; i < D * HID; i += kThreads) gW1[i] = s.W1c[i];
            for (int i = tid; i < HID * D; i += kThreads) gW2[i] = s.W2c[(i / D) * LDW2 + i % D];
            for (int k = tid; k < HID; k += kThreads) gb1[k] = s.b1c[k];
            for (int j = tid; j < D; j += kThreads) gb2[j] = s.b2c[j];
        }
        // the full 16-token tiles are written; tokens past the chunk are zero
        for (int i = tid; i < kChunk * D; i += kThreads) {
            int t = i / D;
            long g = (tok0 + t0 + t) * D + (i % D);
            bool ok = t < n;
            s.X[i] = ok ? to_f32(K[g]) : 0.f;
            s.Vt[i] = ok ? to_f32(V[g]) : 0.f;
            s.Qt[i] = ok ? to_f32(Q[g]) : 0.f;
        }
        for (int t = tid; t < kChunk; t += kThreads) s.eta[t] = t < n ? eta[tok0 + t0 + t] : 0.f;
        __syncthreads();

        // z1 = X W1_s + b1_s, h = GELU(z1): thread k owns hidden unit k
        {
            const int k = tid;
            float acc[kChunk];
#pragma unroll
            for (int t = 0; t < kChunk; t++) acc[t] = b1s[k];
            for (int i = 0; i < D; i++) {
                float w = W1s[i * HID + k];
#pragma unroll
                for (int t = 0; t < kChunk; t++) acc[t] = fmaf(s.X[t * D + i], w, acc[t]);
            }
#pragma unroll
            for (int t = 0; t < kChunk; t++) {
                s.Z1[t * HID + k] = acc[t];
                s.Hs[t * HID + k] = gelu_tanh(acc[t]);
            }
        }
        // A[t,s] = eta_s (q_t . k_s + 1), s <= t
        {
            const int t = tid / kChunk, u = tid % kChunk;
            float a = 0.f;
            if (u <= t) {
                float dot = 0.f;
                for (int i = 0; i < D; i++) dot = fmaf(s.Qt[t * D + i], s.X[u * D + i], dot);
                a = s.eta[u] * (dot + 1.f);
            }
            s.A[tid] = a;
        }
        __syncthreads();

        // y = h W2_s + b2_s: thread -> (out j, 4 tokens)
        {
            const int j = tid % D, tg = tid / D;
            float acc[4];
#pragma unroll
            for (int q = 0; q < 4; q++) acc[q] = b2s[j];
            for (int k = 0; k < HID; k++) {
                float w = W2s[k * ldw2s + j];
#pragma unroll
                for (int q = 0; q < 4; q++) acc[q] = fmaf(s.Hs[(tg * 4 + q) * HID + k], w, acc[q]);
            }
#pragma unroll
            for (int q = 0; q < 4; q++) s.Y2[(tg * 4 + q) * D + j] = acc[q];
        }
        __syncthreads();

        // G2 = dl/dy (LayerNorm backward), one warp per token
        for (int t = warp; t < kChunk; t += kThreads / 32) {
            float* y = s.Y2 + t * D;
            float y0 = y[lane], y1 = y[lane + 32];
            const float mu = warp_sum(y0 + y1) / D;
            const float rs = rsqrtf(warp_sum((y0 - mu) * (y0 - mu) + (y1 - mu) * (y1 - mu)) / D + eps);
            float xh0 = (y0 - mu) * rs, xh1 = (y1 - mu) * rs;
            int j0 = lane, j1 = lane + 32;
            float gx0 = 2.f * s.gam[j0] * (s.X[t * D + j0] + s.gam[j0] * xh0 + s.bet[j0] - s.Vt[t * D + j0]);
            float gx1 = 2.f * s.gam[j1] * (s.X[t * D + j1] + s.gam[j1] * xh1 + s.bet[j1] - s.Vt[t * D + j1]);
            const float mgx = warp_sum(gx0 + gx1) / D;
            const float mgxx = warp_sum(gx0 * xh0 + gx1 * xh1) / D;
            y[j0] = rs * (gx0 - mgx - xh0 * mgxx);
            y[j1] = rs * (gx1 - mgx - xh1 * mgxx);
        }
        __syncthreads();

        // G1 = (G2 W2_s^T) * GELU'(z1): thread k
        {
            const int k = tid;
            float acc[kChunk];
#pragma unroll
            for (int t = 0; t < kChunk; t++) acc[t] = 0.f;
            for (int j = 0; j < D; j++) {
                float w = W2s[k * ldw2s + j];
#pragma unroll
                for (int t = 0; t < kChunk; t++) acc[t] = fmaf(s.Y2[t * D + j], w, acc[t]);
            }
#pragma unroll
            for (int t = 0; t < kChunk; t++) s.G1[t * HID + k] = acc[t] * gelu_tanh_prime(s.Z1[t * HID + k]);
        }
        __syncthreads();

        // z1q = Q W1_c + b1_c - A G1, hq = GELU(z1q) (into Z1)
        {
            const int k = tid;
            float acc[kChunk];
#pragma unroll
            for (int t = 0; t < kChunk; t++) acc[t] = s.b1c[k];
            for (int i = 0; i < D; i++) {
                float w = s.W1c[i * HID + k];
#pragma unroll
                for (int t = 0; t < kChunk; t++) acc[t] = fmaf(s.Qt[t * D + i], w, acc[t]);
            }
#pragma unroll
            for (int u = 0; u < kChunk; u++) {
                float g = s.G1[u * HID + k];
#pragma unroll
                for (int t = 0; t < kChunk; t++) acc[t] = fmaf(-s.A[t * kChunk + u], g, acc[t]);
            }
#pragma unroll
            for (int t = 0; t < kChunk; t++) s.Z1[t * HID + k] = gelu_tanh(acc[t]);
        }
        __syncthreads();

        // A2[t,s] = eta_s (hq_t . h_s + 1), s <= t
        {
            const int t = tid / kChunk, u = tid % kChunk;
            float a = 0.f;
            if (u <= t) {
                float dot = 0.f;
                for (int k = 0; k < HID; k++) dot = fmaf(s.Z1[t * HID + k], s.Hs[u * HID + k], dot);
                a = s.eta[u] * (dot + 1.f);
            }
            s.A2[tid] = a;
        }
        __syncthreads();

        // z2q = hq W2_c + b2_c - A2 G2
        {
            const int j = tid % D, tg = tid / D;
            float acc[4];
#pragma unroll
            for (int q = 0; q < 4; q++) acc[q] = s.b2c[j];
            for (int k = 0; k < HID; k++) {
                float w = s.W2c[k * LDW2 + j];
#pragma unroll
                for (int q = 0; q < 4; q++) acc[q] = fmaf(s.Z1[(tg * 4 + q) * HID + k], w, acc[q]);
            }
#pragma unroll
            for (int q = 0; q < 4; q++) {
                int t = tg * 4 + q;
                for (int u = 0; u <= t; u++) acc[q] = fmaf(-s.A2[t * kChunk + u], s.Y2[u * D + j], acc[q]);
                s.Zq2[t * D + j] = acc[q];
            }
        }
        __syncthreads();

        // state update
        {
            const int k = tid;
            float eg[kChunk], sum = 0.f;
#pragma unroll
            for (int u = 0; u < kChunk; u++) {
                eg[u] = s.eta[u] * s.G1[u * HID + k];
                sum += eg[u];
            }
            for (int i = 0; i < D; i++) {
                float acc = 0.f;
#pragma unroll
                for (int u = 0; u < kChunk; u++) acc = fmaf(s.X[u * D + i], eg[u], acc);
                s.W1c[i * HID + k] -= acc;
            }
            s.b1c[k] -= sum;
            const int j = tid % D, kg = tid / D;
            float eg2[kChunk], sum2 = 0.f;
#pragma unroll
            for (int u = 0; u < kChunk; u++) {
                eg2[u] = s.eta[u] * s.Y2[u * D + j];
                sum2 += eg2[u];
            }
            for (int kk = kg * (HID / 4); kk < (kg + 1) * (HID / 4); kk++) {
                float acc = 0.f;
#pragma unroll
                for (int u = 0; u < kChunk; u++) acc = fmaf(s.Hs[u * HID + kk], eg2[u], acc);
                s.W2c[kk * LDW2 + j] -= acc;
            }
            if (kg == 0) s.b2c[j] -= sum2;
        }
        // z = q + LN(z2q)
        for (int t = warp; t < n; t += kThreads / 32) {
            const float* zb = s.Zq2 + t * D;
            float z0 = zb[lane], z1 = zb[lane + 32];
            const float mu = warp_sum(z0 + z1) / D;
            const float rs = rsqrtf(warp_sum((z0 - mu) * (z0 - mu) + (z1 - mu) * (z1 - mu)) / D + eps);
            float* out = Z + (tok0 + t0 + t) * D;
            out[lane] = s.Qt[t * D + lane] + s.gam[lane] * (z0 - mu) * rs + s.bet[lane];
            out[lane + 32] = s.Qt[t * D + lane + 32] + s.gam[lane + 32] * (z1 - mu) * rs + s.bet[lane + 32];
        }
    }
    __syncthreads();
    float* oW1 = W1_T + bh * D * HID;
    float* oW2 = W2_T + bh * HID * D;
    float* ob1 = b1_T + bh * HID;
    float* ob2 = b2_T + bh * D;
    for (int i = tid; i < D * HID; i += kThreads) oW1[i] = s.W1c[i];
    for (int i = tid; i < HID * D; i += kThreads) oW2[i] = s.W2c[(i / D) * LDW2 + i % D];
    for (int k = tid; k < HID; k += kThreads) ob1[k] = s.b1c[k];
    for (int j = tid; j < D; j += kThreads) ob2[j] = s.b2c[j];
    if (decode && (pos0 + T) % mb == 0) {  // the next token starts a mini-batch from the final state
        for (int i = tid; i < D * HID; i += kThreads) gW1[i] = s.W1c[i];
        for (int i = tid; i < HID * D; i += kThreads) gW2[i] = s.W2c[(i / D) * LDW2 + i % D];
        for (int k = tid; k < HID; k += kThreads) gb1[k] = s.b1c[k];
        for (int j = tid; j < D; j += kThreads) gb2[j] = s.b2c[j];
    }
}

template <typename Tin>
cudaError_t launch_t(const MlpArgs& a, cudaStream_t stream) {
    auto kern = ttt_mlp_generic_kernel<Tin>;
    const size_t smem = sizeof(MlpSmem);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<a.B * a.H, kThreads, smem, stream>>>(
        a.H, a.T, a.mini_batch, a.ln_eps, static_cast<const Tin*>(a.Q), static_cast<const Tin*>(a.K),
        static_cast<const Tin*>(a.V), a.eta, a.W1_0, a.b1_0, a.W2_0, a.b2_0, a.gamma, a.beta, a.Z,
        a.W1_T, a.b1_T, a.W2_T, a.b2_T, a.pos0, a.W1_mb, a.b1_mb, a.W2_mb, a.b2_mb);
    return cudaPeekAtLastError();
}

}  // namespace

bool mlp_generic_supports(const MlpArgs& a) { return a.d == D && a.hidden == HID; }

cudaError_t launch_mlp_generic(const MlpArgs& a, cudaStream_t stream) {
    if (!mlp_generic_supports(a)) return cudaErrorInvalidValue;
    return a.dtype == TTT_BF16 ? launch_t<__nv_bfloat16>(a, stream) : launch_t<float>(a, stream);
}

}  // namespace ttt
