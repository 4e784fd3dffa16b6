// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA (bulk tensor) loads,
// ldmatrix / movmatrix, mma.sync (bf16 -> fp32), named barriers, cluster
// barriers and stores into a peer CTA's shared memory.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace ttt {
namespace ptx {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// ---------------------------------------------------------------- TMA loads
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(smem_addr(dst)), "l"(tmap), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "r"(c2) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_addr(dst)), "l"(tmap), "r"(smem_addr(bar)), "r"(c0), "r"(c1) : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---------------------------------------------------------------- ldmatrix
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}
// transpose of one 8x8 b16 matrix held in the standard fragment layout
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

// ---------------------------------------------------------------- mma.sync
// D = A * B + D, m16n8k16, bf16 operands, fp32 accumulate.  A pure function of
// its register operands (not volatile), so the compiler may interleave
// independent products; back-to-back products on one accumulator wait for the
// previous result.
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- packed bf16 helpers
__device__ __forceinline__ float bf16_lo_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi_f32(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// ---------------------------------------------------------------- named barriers
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- thread-block clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of the same shared-memory byte in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t local_addr, uint32_t rank) {
    uint32_t d;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(local_addr), "r"(rank));
    return d;
}
// Hardware cluster barrier, split in its two halves.  Every thread of every CTA
// of the cluster arrives once per phase; arrive releases this thread's earlier
// shared-memory writes (local and remote) at cluster scope, wait acquires them.
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
// wait with cluster-scope acquire, for a barrier completed by another CTA's st.async
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}
// store into another CTA's shared memory that counts its bytes on that CTA's mbarrier
// (both addresses from mapa_shared)
__device__ __forceinline__ void st_async_f32x2(uint32_t addr, float x, float y, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];"
                 ::"r"(addr), "f"(x), "f"(y), "r"(remote_bar) : "memory");
}
// plain stores into another CTA's shared memory (address from mapa_shared)
__device__ __forceinline__ void st_cluster_f32x2(uint32_t addr, float x, float y) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(x), "f"(y) : "memory");
}
__device__ __forceinline__ void st_cluster_f32x4(uint32_t addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};"
                 ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}

// ---------------------------------------------------------------- bf16 hi/lo split
// x ~= hi + lo: hi = x rounded to bf16 (round half away from zero, done on the
// bit pattern), lo = x - hi (exact in fp32) truncated to bf16.  Relative error
// below 2^-15.  Integer and byte-permute operations only: the packed
// float->bf16 conversion instructions run on a narrow pipe, and these splits
// are on the hot path of every chunk.  Pairs are packed low column first (the
// mma fragment convention).
__device__ __forceinline__ uint32_t bf16_round_bits(float x) {
    return (__float_as_uint(x) + 0x8000u) & 0xffff0000u;
}
__device__ __forceinline__ uint32_t pack_hi_halves(uint32_t lo_col, uint32_t hi_col) {
    return __byte_perm(lo_col, hi_col, 0x7632);
}
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const uint32_t h0 = bf16_round_bits(x0), h1 = bf16_round_bits(x1);
    hi = pack_hi_halves(h0, h1);
    lo = pack_hi_halves(__float_as_uint(x0 - __uint_as_float(h0)), __float_as_uint(x1 - __uint_as_float(h1)));
}

// The most precise split, also five instructions: hi = x rounded to the
// nearest bf16 (one packed conversion for the pair), lo = (x - hi) rounded to
// the nearest bf16.  |x - hi| <= 2^-8 |x| is exact in fp32, so
// |x - hi - lo| <= 2^-16 |x|, unbiased.
__device__ __forceinline__ void split_pair_rn(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(x1), "f"(x0));
    const uint32_t h0 = hi << 16, h1 = hi & 0xffff0000u;
    uint64_t d;
    asm("{\n .reg .b64 a, b;\n mov.b64 a, {%1, %2};\n mov.b64 b, {%3, %4};\n sub.rn.f32x2 %0, a, b;\n}\n"
        : "=l"(d) : "f"(x0), "f"(x1), "r"(h0), "r"(h1));
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(__uint_as_float((uint32_t)(d >> 32))),
        "f"(__uint_as_float((uint32_t)d)));
}
// (x0, x1) += (y0, y1) as one packed fp32 add
__device__ __forceinline__ void add2(float& x0, float& x1, float y0, float y1) {
    uint64_t d;
    asm("{\n .reg .b64 a, b;\n mov.b64 a, {%1, %2};\n mov.b64 b, {%3, %4};\n add.rn.f32x2 %0, a, b;\n}\n"
        : "=l"(d) : "f"(x0), "f"(x1), "f"(y0), "f"(y1));
    x0 = __uint_as_float((uint32_t)d);
    x1 = __uint_as_float((uint32_t)(d >> 32));
}

}  // namespace ptx
}  // namespace ttt
