// Optional clock64 timeline of one CTA's warp roles (build flag TTT_TIMELINE).
//
// In a TTT_TIMELINE build, the leader lane of each role's first warp in CTA 0
// records the SM clock at fixed points of every chunk step in [kTlFirst,
// kTlFirst + kTlChunks) into shared memory, and copies its row to a
// per-kernel __device__ array when the role ends; the host reads that back
// through ttt_debug_timeline (exported by that build only).  Shared memory
// keeps the stamps cheap: an mbarrier arrive has release semantics, so a
// global store just before it would hold the arrive until the store had left
// the SM.  In the normal build the stamps compile to nothing.
#pragma once

namespace ttt {
constexpr int kTlRoles = 8, kTlEvents = 8, kTlChunks = 32, kTlFirst = 1024;
}

#ifdef TTT_TIMELINE
#define TTT_TIMELINE_BUFFER(name) __device__ long long name[ttt::kTlRoles][ttt::kTlChunks][ttt::kTlEvents]
// inside the kernel, before its first block-wide barrier
#define TTT_TIMELINE_SMEM()                                                                   \
    __shared__ long long tl_smem_[ttt::kTlRoles][ttt::kTlChunks][ttt::kTlEvents];             \
    for (int tl_i_ = threadIdx.x; tl_i_ < ttt::kTlRoles * ttt::kTlChunks * ttt::kTlEvents;    \
         tl_i_ += blockDim.x)                                                                 \
        (&tl_smem_[0][0][0])[tl_i_] = 0
#define TTT_STAMP(buf, leader, role, c, ev)                                                   \
    do {                                                                                      \
        const int tl_c_ = (c) - ttt::kTlFirst;                                                \
        if ((leader) && blockIdx.x == 0 && tl_c_ >= 0 && tl_c_ < ttt::kTlChunks)              \
            tl_smem_[role][tl_c_][ev] = clock64();                                            \
    } while (0)
#define TTT_TIMELINE_FLUSH(buf, leader, role)                                                 \
    do {                                                                                      \
        if ((leader) && blockIdx.x == 0)                                                      \
            for (int tl_i_ = 0; tl_i_ < ttt::kTlChunks * ttt::kTlEvents; tl_i_++)             \
                (&buf[role][0][0])[tl_i_] = (&tl_smem_[role][0][0])[tl_i_];                   \
    } while (0)
#else
#define TTT_TIMELINE_BUFFER(name) static_assert(true, "timeline off")
#define TTT_TIMELINE_SMEM() ((void)0)
#define TTT_STAMP(buf, leader, role, c, ev) ((void)0)
#define TTT_TIMELINE_FLUSH(buf, leader, role) ((void)0)
#endif
