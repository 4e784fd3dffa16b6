// TTT-MLP decode for d = 64, hidden = 256: the MLP scan continued token by
// token, with the running state in registers for the whole call.
//
// Method ("Learning to (Learn at Test Time)", literature record, Key
// takeaways bullets 1, 2 and 5; the abstract names the two-layer MLP state).
// Per token t at position p of its mini-batch, with (W1_s, b1_s, W2_s, b2_s)
// the state the mini-batch started from (:= the running state at p = 0):
//   z1 = k W1_s + b1_s, h = GELU(z1), y = h W2_s + b2_s
//   g2 = dl/dy (LayerNorm backward), g1 = (W2_s g2) * GELU'(z1)
//   W1 -= eta k^T g1, b1 -= eta g1, W2 -= eta h^T g2, b2 -= eta g2
//   z  = q + LN(GELU(q W1 + b1) W2 + b2)
//
// One CTA of 512 threads per (batch, head).  Registers: thread tid holds
// W1[32 (tid / 256) + r][tid % 256] and W2[32 (tid / 64) + r][tid % 64] for
// r < 32, so a warp's loads and stores of the state are whole lines.  Shared
// memory: the mini-batch start state (W2 rows padded to 65 floats, so that
// both its row and its column reads are conflict-free) and the per-token
// vectors.  Each product's row-group partial sums meet in shared memory;
// nine block barriers per token.
#include <atomic>

#include "common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int D = 64;
constexpr int HID = 256;
constexpr int kThreads = 512;
constexpr int R1 = D / (kThreads / HID);   // W1 rows per thread: 32
constexpr int R2 = HID / (kThreads / D);   // W2 rows per thread: 32
constexpr int LDW2 = D + 1;

struct MlpDecodeSmem {
    float W1s[D * HID];                  // start state W1_s [in][hid]
    float W2s[HID * LDW2];               // start state W2_s [hid][out], padded rows
    float b1s[HID], b2s[D];
    float k[2][D], q[2][D], v[2][D];     // token vectors, double-buffered by token parity
    float eta[2];
    float part1[kThreads / HID][HID];    // row-group partial sums over W1 rows
    float part2[kThreads / D][D];        // row-group partial sums over W2 rows
    float z1[HID], h[HID], g1[HID], hq[HID];
    float g2[D];
    float gam[D], bet[D];
};

template <typename Tin>
__global__ void __launch_bounds__(kThreads, 1)
ttt_mlp_decode_kernel(int H, int T, int mb, int pos0, float eps, const Tin* __restrict__ Q,
                      const Tin* __restrict__ K, const Tin* __restrict__ V, const float* __restrict__ eta,
                      float* W1, float* b1, float* W2, float* b2, float* W1_mb, float* b1_mb, float* W2_mb,
                      float* b2_mb, const float* __restrict__ gamma, const float* __restrict__ beta,
                      float* __restrict__ Z) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    MlpDecodeSmem& s = *reinterpret_cast<MlpDecodeSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k1 = tid & (HID - 1), r1 = tid / HID;  // W1 column and row group
    const int j2 = tid & (D - 1), r2 = tid / D;      // W2 column and row group
    const long bh = blockIdx.x;
    const int h = (int)(bh % H);
    float* W1bh = W1 + bh * D * HID;
    float* W2bh = W2 + bh * HID * D;
    float* W1mbh = W1_mb + bh * D * HID;
    float* W2mbh = W2_mb + bh * HID * D;

    // ---- start state into shared memory when the call begins inside a mini-batch (first,
    // while the registers that will hold the running state are still free); running state
    // into registers
    if (pos0 > 0) {
        // 128 KB of start state from L2: 16-byte loads, kBatch per matrix in flight per thread before
        // the stores that consume them (a load-then-store loop would wait out one L2 round trip per
        // element)
        const float4* w1g = reinterpret_cast<const float4*>(W1mbh);
        const float4* w2g = reinterpret_cast<const float4*>(W2mbh);
        float4* w1s = reinterpret_cast<float4*>(s.W1s);
        constexpr int kVec = D * HID / 4 / kThreads;  // 8 float4 per thread and matrix
        constexpr int kBatch = 8;
#pragma unroll
        for (int u0 = 0; u0 < kVec; u0 += kBatch) {
            float4 a[kBatch], c[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; u++) {
                a[u] = w1g[tid + (u0 + u) * kThreads];
                c[u] = w2g[tid + (u0 + u) * kThreads];
            }
#pragma unroll
            for (int u = 0; u < kBatch; u++) {
                w1s[tid + (u0 + u) * kThreads] = a[u];
                const int i = 4 * (tid + (u0 + u) * kThreads);  // element of W2 [hid][out]; i % D <= D - 4
                float* dst = s.W2s + (i / D) * LDW2 + i % D;
                dst[0] = c[u].x;
                dst[1] = c[u].y;
                dst[2] = c[u].z;
                dst[3] = c[u].w;
            }
        }
        if (tid < HID) s.b1s[tid] = b1_mb[bh * HID + tid];
        if (tid < D) s.b2s[tid] = b2_mb[bh * D + tid];
    }
    float w1[R1], w2[R2];
#pragma unroll
    for (int r = 0; r < R1; r++) w1[r] = W1bh[(R1 * r1 + r) * HID + k1];
#pragma unroll
    for (int r = 0; r < R2; r++) w2[r] = W2bh[(R2 * r2 + r) * D + j2];
    float b1r = tid < HID ? b1[bh * HID + tid] : 0.f;                 // b1[k1], threads < 256
    float b2r[2] = {0.f, 0.f};                                         // b2[lane + 32 e], warp 0
    if (warp == 0) {
        b2r[0] = b2[bh * D + lane];
        b2r[1] = b2[bh * D + lane + 32];
    }
    if (tid < D) {
        s.gam[tid] = gamma[(long)h * D + tid];
        s.bet[tid] = beta[(long)h * D + tid];
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
        if ((pos0 + t) % mb == 0) {  // a mini-batch starts at this token: start := running
#pragma unroll
            for (int r = 0; r < R1; r++) s.W1s[(R1 * r1 + r) * HID + k1] = w1[r];
#pragma unroll
            for (int r = 0; r < R2; r++) s.W2s[(R2 * r2 + r) * LDW2 + j2] = w2[r];
            if (tid < HID) s.b1s[tid] = b1r;
            if (warp == 0) {
                s.b2s[lane] = b2r[0];
                s.b2s[lane + 32] = b2r[1];
            }
        }
        __syncthreads();  // 1: token and start state in; the previous token's readers done

        {  // z1 partials: k W1_s over this thread's rows
            float p = 0.f;
#pragma unroll 8
            for (int r = 0; r < R1; r++) p = fmaf(s.k[buf][R1 * r1 + r], s.W1s[(R1 * r1 + r) * HID + k1], p);
            s.part1[r1][k1] = p;
        }
        __syncthreads();  // 2
        if (tid < HID) {
            const float z = s.b1s[tid] + (s.part1[0][tid] + s.part1[1][tid]);
            s.z1[tid] = z;
            s.h[tid] = gelu_tanh(z);
        }
        __syncthreads();  // 3
        {  // y partials: h W2_s over this thread's rows
            float p = 0.f;
#pragma unroll 8
            for (int r = 0; r < R2; r++) p = fmaf(s.h[R2 * r2 + r], s.W2s[(R2 * r2 + r) * LDW2 + j2], p);
            s.part2[r2][j2] = p;
        }
        __syncthreads();  // 4
        if (warp == 0) {  // y, g2 = dl/dy, b2 -= eta g2
            float y[2];
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int c = lane + 32 * e;
                float acc = s.b2s[c];
#pragma unroll
                for (int g = 0; g < kThreads / D; g++) acc += s.part2[g][c];
                y[e] = acc;
            }
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
            const float et = s.eta[buf];
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const float g = rs * (gx[e] - mgx - xh[e] * mgxx);
                s.g2[lane + 32 * e] = g;
                b2r[e] -= et * g;
            }
        }
        __syncthreads();  // 5
        if (tid < HID) {  // g1 = (W2_s g2) * GELU'(z1), b1 -= eta g1
            float acc = 0.f;
#pragma unroll 8
            for (int j = 0; j < D; j++) acc = fmaf(s.W2s[tid * LDW2 + j], s.g2[j], acc);
            const float g = acc * gelu_tanh_prime(s.z1[tid]);
            s.g1[tid] = g;
            b1r -= s.eta[buf] * g;
        }
        __syncthreads();  // 6
        {  // W1 -= eta k^T g1 (with the q W1 partials of the new W1); W2 -= eta h^T g2
            const float et = s.eta[buf];
            const float eg1 = et * s.g1[k1];
            float p = 0.f;
#pragma unroll
            for (int r = 0; r < R1; r++) {
                w1[r] = fmaf(-s.k[buf][R1 * r1 + r], eg1, w1[r]);
                p = fmaf(s.q[buf][R1 * r1 + r], w1[r], p);
            }
            s.part1[r1][k1] = p;
            const float eg2 = et * s.g2[j2];
#pragma unroll
            for (int r = 0; r < R2; r++) w2[r] = fmaf(-s.h[R2 * r2 + r], eg2, w2[r]);
        }
        __syncthreads();  // 7
        if (tid < HID) s.hq[tid] = gelu_tanh(b1r + (s.part1[0][tid] + s.part1[1][tid]));
        __syncthreads();  // 8
        {  // z2 partials: hq W2 with the new W2
            float p = 0.f;
#pragma unroll
            for (int r = 0; r < R2; r++) p = fmaf(s.hq[R2 * r2 + r], w2[r], p);
            s.part2[r2][j2] = p;
        }
        __syncthreads();  // 9
        if (warp == 0) {  // z = q + LN(z2)
            float zz[2];
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int c = lane + 32 * e;
                float acc = b2r[e];
#pragma unroll
                for (int g = 0; g < kThreads / D; g++) acc += s.part2[g][c];
                zz[e] = acc;
            }
            const float mu = warp_sum(zz[0] + zz[1]) * (1.f / D);
            const float d0 = zz[0] - mu, d1 = zz[1] - mu;
            const float rs = rsqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.f / D) + eps);
            float* out = Z + (tok0 + t) * D;
            out[lane] = s.q[buf][lane] + s.gam[lane] * d0 * rs + s.bet[lane];
            out[lane + 32] = s.q[buf][lane + 32] + s.gam[lane + 32] * d1 * rs + s.bet[lane + 32];
        }
        // the next token's barrier 1 orders warp 0's reads of part2 / q against the next writes
    }

    // ---- state out: running state; the start state when it changed in this call
#pragma unroll
    for (int r = 0; r < R1; r++) W1bh[(R1 * r1 + r) * HID + k1] = w1[r];
#pragma unroll
    for (int r = 0; r < R2; r++) W2bh[(R2 * r2 + r) * D + j2] = w2[r];
    if (tid < HID) b1[bh * HID + tid] = b1r;
    if (warp == 0) {
        b2[bh * D + lane] = b2r[0];
        b2[bh * D + lane + 32] = b2r[1];
    }
    const bool boundary = (pos0 + T) % mb == 0;         // the next token starts a mini-batch
    const bool restarted = pos0 == 0 || T > mb - pos0;  // the start state was reset inside this call
    if (boundary) {
#pragma unroll
        for (int r = 0; r < R1; r++) W1mbh[(R1 * r1 + r) * HID + k1] = w1[r];
#pragma unroll
        for (int r = 0; r < R2; r++) W2mbh[(R2 * r2 + r) * D + j2] = w2[r];
        if (tid < HID) b1_mb[bh * HID + tid] = b1r;
        if (warp == 0) {
            b2_mb[bh * D + lane] = b2r[0];
            b2_mb[bh * D + lane + 32] = b2r[1];
        }
    } else if (restarted) {
        __syncthreads();
        float4* w1g = reinterpret_cast<float4*>(W1mbh);
        float4* w2g = reinterpret_cast<float4*>(W2mbh);
        const float4* w1s = reinterpret_cast<const float4*>(s.W1s);
        constexpr int kVec = D * HID / 4 / kThreads;
#pragma unroll
        for (int u = 0; u < kVec; u++) {
            w1g[tid + u * kThreads] = w1s[tid + u * kThreads];
            const int i = 4 * (tid + u * kThreads);
            const float* src = s.W2s + (i / D) * LDW2 + i % D;
            w2g[tid + u * kThreads] = make_float4(src[0], src[1], src[2], src[3]);
        }
        if (tid < HID) b1_mb[bh * HID + tid] = s.b1s[tid];
        if (tid < D) b2_mb[bh * D + tid] = s.b2s[tid];
    }
}

template <typename Tin>
cudaError_t launch_t(const MlpArgs& a, cudaStream_t stream) {
    auto kern = ttt_mlp_decode_kernel<Tin>;
    const size_t smem = sizeof(MlpDecodeSmem);
    // set once per device, so that a launch captured in a CUDA graph makes no other runtime call
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
        a.H, a.T, a.mini_batch, a.pos0, a.ln_eps, static_cast<const Tin*>(a.Q), static_cast<const Tin*>(a.K),
        static_cast<const Tin*>(a.V), a.eta, a.W1_T, a.b1_T, a.W2_T, a.b2_T, a.W1_mb, a.b1_mb, a.W2_mb, a.b2_mb,
        a.gamma, a.beta, a.Z);
    return cudaPeekAtLastError();
}

}  // namespace

bool mlp_decode_supports(const MlpArgs& a) { return a.d == D && a.hidden == HID; }

// In place: a.W*_T / a.b*_T hold the running state and a.W*_mb / a.b*_mb the
// mini-batch start state on entry.
cudaError_t launch_mlp_decode(const MlpArgs& a, cudaStream_t stream) {
    if (!mlp_decode_supports(a)) return cudaErrorInvalidValue;
    return a.dtype == TTT_BF16 ? launch_t<__nv_bfloat16>(a, stream) : launch_t<float>(a, stream);
}

}  // namespace ttt
