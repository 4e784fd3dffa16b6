// The TTT layer's prologue on the 5th-generation tensor cores: the per-head
// projections of the layer input into the scan's Q, K, V, the token-dependent
// learning rate eta, and rotary position embedding of Q and K, fused in one
// kernel ("Learning to (Learn at Test Time)", literature record, Key takeaways
// bullets 1 and 2: the scan sees the views theta_K x_t, theta_V x_t, theta_Q x_t
// of each token, with a learning rate that depends on the token; the
// codewithpapers.app record names the official code's rotate_half helper).
//
// Readings where the pages are silent: per head h, Q = x theta_Q[h],
// K = x theta_K[h], V = x theta_V[h] without bias;
// eta_t = eta_base * sigmoid(x_t . theta_lr[h] + b_lr[h]) / d; rotary embedding
// in the rotate-half convention on Q and K: features i and i + d/2 rotate
// together by p * base^(-2i/d), with p the token's absolute position pos0 + t.
//
// One GEMM with the tokens as rows: [B*T, d_model] x [d_model, 3 H d + H].
// Column tiles of 256 hold four heads of one of Q, K, V (the weights [H][d_model]
// [d] are read MN-major, four heads side by side); one more tile of round16(H)
// columns holds the H learning-rate logits.  Persistent CTAs of 8 warps walk the
// tiles (column tiles fastest, so the CTAs in flight share each row tile in L2):
//   warp 0     TMA loads of x (128 x 64) and weight (64 x 256) tiles, 4-stage ring
//   warp 1     TMEM allocation and the tcgen05 MMAs (M = 128, N = 256, K = 16),
//              fp32 accumulators in two TMEM buffers of 256 columns
//   warps 4-7  the epilogue (warp 4 + i reads TMEM lanes 32 i..32 i + 31, one token
//              row per thread): rotary embedding, bf16 rounding and stores to
//              Q, K, V [B][H][T][d]; the sigmoid gate and stores to eta [B][H][T].
// While the epilogue drains one accumulator the MMA warp fills the other.
// Every wait is bounded: after about a second without progress the kernel
// records an error word and stops waiting (outputs undefined; TTT_ERR_TIMEOUT
// with TTT_CHECK=1).
#include <cstdlib>

#include "common.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"
#include "tma_host.h"
#include "ttt_internal.h"

namespace ttt {

__device__ unsigned int g_prologue_error_word = 0;

namespace {

constexpr int kD = 64;             // head dimension
constexpr int kBM = 128, kBK = 64;  // tile rows (tokens), K step per stage
constexpr int kBN = 256;            // four heads of 64
constexpr int kStages = 4;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;  // two accumulators of 256 columns
constexpr long long kTimeoutCycles = 2000000000LL;

struct alignas(1024) PStage {
    unsigned char A[kBM * kBK * 2];  // x tile [128 tokens][64 k], 128-byte swizzle (K-major)
    unsigned char B[kBN * kBK * 2];  // weights [4 heads][64 k][64 n] (MN-major), or theta_lr [Hp][64 k] (K-major)
};

struct ProSmem {
    PStage st[kStages];
    double inv_freq[kD / 2];  // base^(-2i/d)
    uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (int spins = 1;; spins++) {
        if (*abort_flag) return false;
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((spins & 63) == 0 && clock64() - t0 > kTimeoutCycles) {
            *abort_flag = 1;
            atomicOr(&g_prologue_error_word, 1u);
            return false;
        }
    }
}

__device__ __forceinline__ void ld_32x32b_x32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void ld_32x32b_x16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t pack_rn(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

struct PrologueParams {
    int B, T, H, d_model, pos0, rotary, n_col_tiles, n_tiles, hp;  // hp: H rounded up to 16
    float eta_base, rope_base;
    const float* b_lr;
    __nv_bfloat16 *Q, *K, *V;
    float* eta;
};

__global__ void __launch_bounds__(kThreads, 1)
ttt_prologue_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWq,
                    const __grid_constant__ CUtensorMap tmWk, const __grid_constant__ CUtensorMap tmWv,
                    const __grid_constant__ CUtensorMap tmWl, const PrologueParams p) {
    extern __shared__ unsigned char smem_raw[];
    ProSmem& s = *reinterpret_cast<ProSmem*>(smem_raw + ((1024u - (ptx::smem_addr(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort_flag = &s.abort_flag;
    const int nk = p.d_model / kBK;
    const int M = p.B * p.T;
    const int groups = p.H / 4;  // column tiles per projection
    if (tid == 0) {
        s.abort_flag = 0;
        for (int i = 0; i < kStages; i++) {
            ptx::mbar_init(&s.full[i], 1);
            ptx::mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; i++) {
            ptx::mbar_init(&s.acc_full[i], 1);
            ptx::mbar_init(&s.acc_empty[i], 4);
        }
        ptx::mbar_init(&s.drain, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 1) tc05::tmem_alloc(ptx::smem_addr(&s.tmem_base), kTmemCols);
    if (tid < kD / 2) s.inv_freq[tid] = exp2(-(2.0 * tid / kD) * log2((double)p.rope_base));
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tmem = s.tmem_base;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            ptx::prefetch_tmap(&tmX);
            ptx::prefetch_tmap(&tmWq);
            ptx::prefetch_tmap(&tmWk);
            ptx::prefetch_tmap(&tmWv);
            ptx::prefetch_tmap(&tmWl);
            long long it = 0;
            int inflight = 0;
            for (int tile = blockIdx.x; tile < p.n_tiles && !*abort_flag; tile += gridDim.x) {
                const int mt = tile / p.n_col_tiles, ct = tile % p.n_col_tiles;
                const int proj = ct / groups, grp = ct % groups;  // proj 3: the learning-rate tile
                const void* tmW = proj == 0 ? &tmWq : proj == 1 ? &tmWk : proj == 2 ? &tmWv : &tmWl;
                const uint32_t bytes = kBM * kBK * 2 + (proj == 3 ? p.hp * kBK * 2 : kBN * kBK * 2);
                for (int kb = 0; kb < nk; kb++, it++) {
                    const int st = (int)(it % kStages);
                    if (it >= kStages && !wait_bounded(&s.empty[st], (uint32_t)(((it / kStages) - 1) & 1),
                                                       abort_flag))
                        break;
                    ptx::mbar_arrive_expect_tx(&s.full[st], bytes);
                    ptx::tma_load_2d(s.st[st].A, &tmX, &s.full[st], kb * kBK, mt * kBM);
                    if (proj == 3)
                        ptx::tma_load_2d(s.st[st].B, tmW, &s.full[st], kb * kBK, 0);
                    else
                        ptx::tma_load_3d(s.st[st].B, tmW, &s.full[st], 0, kb * kBK, 4 * grp);
                    inflight = it + 1 < kStages ? (int)(it + 1) : kStages;
                }
            }
            // drain own loads: the last `inflight` stages
            for (long long j = it - 1; j >= 0 && j >= it - inflight; j--) {
                const long long t0 = clock64();
                while (!ptx::mbar_try_wait(&s.full[j % kStages], (uint32_t)((j / kStages) & 1))) {
                    if (clock64() - t0 > 4 * kTimeoutCycles) {
                        atomicOr(&g_prologue_error_word, 2u);
                        break;
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t i_qkv = tc05::idesc_bf16(kBM, kBN, 0, 1);
            const uint32_t i_lr = tc05::idesc_bf16(kBM, p.hp, 0, 0);
            long long it = 0;
            int local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x, local++) {
                const int ct = tile % p.n_col_tiles;
                const bool lr = ct / groups == 3;
                const int buf = local & 1;
                if (local >= 2) ok = wait_bounded(&s.acc_empty[buf], (uint32_t)(((local >> 1) - 1) & 1), abort_flag);
                if (!ok) break;
                tc05::fence_after_sync();
                const uint32_t d = tmem + (uint32_t)(buf * kBN);
                for (int kb = 0; kb < nk; kb++, it++) {
                    const int st = (int)(it % kStages);
                    ok = wait_bounded(&s.full[st], (uint32_t)((it / kStages) & 1), abort_flag);
                    if (!ok) break;
                    tc05::fence_after_sync();
                    const uint32_t a = ptx::smem_addr(s.st[st].A), b = ptx::smem_addr(s.st[st].B);
#pragma unroll
                    for (int ks = 0; ks < kBK / 16; ks++) {
                        const uint64_t ad = tc05::desc_k128(a, ks);
                        // MN-major weights: 16 K rows are two 8-row groups (2048 bytes) further; the four heads
                        // are 64 x 64 atoms 8192 bytes apart.  theta_lr: K-major rows of 128 bytes.
                        const uint64_t bd = lr ? tc05::desc_k128(b, ks)
                                               : tc05::smem_desc(b + 2048u * (uint32_t)ks, 8192, 1024,
                                                                 tc05::kSwizzle128);
                        tc05::mma_bf16_ss(d, ad, bd, lr ? i_lr : i_qkv, (kb > 0 || ks > 0) ? 1u : 0u);
                    }
                    tc05::commit(ptx::smem_addr(&s.empty[st]));
                }
                if (!ok) break;
                tc05::commit(ptx::smem_addr(&s.acc_full[buf]));
            }
            tc05::commit(ptx::smem_addr(&s.drain));
            const long long t0 = clock64();
            while (!ptx::mbar_try_wait(&s.drain, 0)) {
                if (clock64() - t0 > 4 * kTimeoutCycles) {
                    atomicOr(&g_prologue_error_word, 4u);
                    break;
                }
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- epilogue
        const int q = warp - 4;
        const uint32_t tq = tmem + tc05::taddr_lane(32 * q);
        const float inv_d = 1.f / kD;
        int local = 0;
        for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, local++) {
            const int mt = tile / p.n_col_tiles, ct = tile % p.n_col_tiles;
            const int proj = ct / groups, grp = ct % groups;
            const int buf = local & 1;
            wait_bounded(&s.acc_full[buf], (uint32_t)((local >> 1) & 1), abort_flag);
            tc05::fence_after_sync();
            const int m = mt * kBM + 32 * q + lane;  // this thread's token row
            const bool valid = m < M;
            const int bb = valid ? m / p.T : 0, t = valid ? m % p.T : 0;
            const uint32_t tacc = tq + (uint32_t)(buf * kBN);
            if (proj == 3) {
                // learning-rate logits: columns 0..H-1
                for (int c0 = 0; c0 < p.hp; c0 += 16) {  // hp is a multiple of 16, at most 256
                    float v[16];
                    ld_32x32b_x16(tacc + (uint32_t)c0, v);
                    tc05::wait_ld();
                    for (int j = 0; j < 16 && c0 + j < p.H; j++) {
                        const int hh = c0 + j;
                        const float logit = v[j] + p.b_lr[hh];
                        if (valid)
                            p.eta[((size_t)bb * p.H + hh) * p.T + t] = p.eta_base * inv_d / (1.f + __expf(-logit));
                    }
                }
            } else {
                __nv_bfloat16* out = proj == 0 ? p.Q : proj == 1 ? p.K : p.V;
                const bool rope = p.rotary && proj < 2;
                // the rotation of this token row, shared by the tile's four heads: angle
                // pos * base^(-2i/d), reduced modulo 2 pi in double, then sin / cos in fp32
                float cs[32], sn[32];
                if (rope) {
                    const double pos = (double)(p.pos0 + t);
#pragma unroll
                    for (int i = 0; i < 32; i++) {
                        const double turns = pos * s.inv_freq[i] * 0.15915494309189535;  // 1 / (2 pi)
                        const float r = (float)((turns - rint(turns)) * 6.283185307179586);
                        sincosf(r, &sn[i], &cs[i]);
                    }
                }
                for (int hh4 = 0; hh4 < 4; hh4++) {
                    float x1[32], x2[32];  // features 0..31 and 32..63 of the head
                    ld_32x32b_x32(tacc + (uint32_t)(64 * hh4), x1);
                    ld_32x32b_x32(tacc + (uint32_t)(64 * hh4 + 32), x2);
                    tc05::wait_ld();
                    if (rope) {
#pragma unroll
                        for (int i = 0; i < 32; i++) {
                            const float a = x1[i], b2 = x2[i];
                            x1[i] = a * cs[i] - b2 * sn[i];
                            x2[i] = b2 * cs[i] + a * sn[i];
                        }
                    }
                    if (valid) {
                        uint4* dst = reinterpret_cast<uint4*>(
                            out + (((size_t)bb * p.H + (4 * grp + hh4)) * p.T + t) * kD);
#pragma unroll
                        for (int c = 0; c < 4; c++) {
                            dst[c] = make_uint4(pack_rn(x1[8 * c + 0], x1[8 * c + 1]), pack_rn(x1[8 * c + 2], x1[8 * c + 3]),
                                                pack_rn(x1[8 * c + 4], x1[8 * c + 5]), pack_rn(x1[8 * c + 6], x1[8 * c + 7]));
                            dst[4 + c] = make_uint4(pack_rn(x2[8 * c + 0], x2[8 * c + 1]), pack_rn(x2[8 * c + 2], x2[8 * c + 3]),
                                                    pack_rn(x2[8 * c + 4], x2[8 * c + 5]), pack_rn(x2[8 * c + 6], x2[8 * c + 7]));
                        }
                    }
                }
            }
            tc05::fence_before_sync();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&s.acc_empty[buf]);
        }
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    if (warp == 1) tc05::tmem_dealloc(tmem, kTmemCols);
}

bool make_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                 uint32_t box_outer) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [H][d_model][64] bf16 in boxes of [4 heads][64 k][64 n]
bool make_weight_map(CUtensorMap* m, const void* base, int H, int d_model) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)d_model, (cuuint64_t)H};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)d_model * kD * 2};
    cuuint32_t box[3] = {kD, kBK, 4};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prologue_supports(int B, int T, int H, int d, int d_model) {
    return B >= 1 && T >= 1 && d == kD && d_model >= kBK && d_model % kBK == 0 && H >= 4 && H % 4 == 0 &&
           H <= 256 && (long long)B * T < (1LL << 31);
}

cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t stream) {
    if (!prologue_supports(a.B, a.T, a.H, a.d, a.d_model)) return cudaErrorInvalidValue;
    const int M = a.B * a.T, hp = (a.H + 15) / 16 * 16;
    CUtensorMap mx, mq, mk, mv, ml;
    if (!make_map_2d(&mx, a.x, (uint64_t)a.d_model, (uint64_t)M, kBK, kBM) ||
        !make_weight_map(&mq, a.theta_q, a.H, a.d_model) || !make_weight_map(&mk, a.theta_k, a.H, a.d_model) ||
        !make_weight_map(&mv, a.theta_v, a.H, a.d_model) ||
        !make_map_2d(&ml, a.theta_lr, (uint64_t)a.d_model, (uint64_t)a.H, kBK, (uint32_t)hp))
        return cudaErrorInvalidValue;
    PrologueParams p{};
    p.B = a.B;
    p.T = a.T;
    p.H = a.H;
    p.d_model = a.d_model;
    p.pos0 = a.pos0;
    p.rotary = a.rotary;
    p.n_col_tiles = 3 * (a.H / 4) + 1;
    p.n_tiles = ((M + kBM - 1) / kBM) * p.n_col_tiles;
    p.hp = hp;
    p.eta_base = a.eta_base;
    p.rope_base = a.rope_base;
    p.b_lr = a.b_lr;
    p.Q = static_cast<__nv_bfloat16*>(a.Q);
    p.K = static_cast<__nv_bfloat16*>(a.K);
    p.V = static_cast<__nv_bfloat16*>(a.V);
    p.eta = a.eta;
    const size_t smem = sizeof(ProSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(ttt_prologue_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = p.n_tiles < sms ? p.n_tiles : sms;
    ttt_prologue_kernel<<<grid, kThreads, smem, stream>>>(mx, mq, mk, mv, ml, p);
    return cudaPeekAtLastError();
}

cudaError_t read_and_clear_prologue_error(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_prologue_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_prologue_error_word, &zero, sizeof(unsigned int));
}

}  // namespace ttt
