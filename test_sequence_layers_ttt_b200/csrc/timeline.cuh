// Optional clock64 timeline of one CTA's warp roles (build flag TTT_TIMELINE).
//
// In a TTT_TIMELINE build, the leader lane of each role's first warp in CTA 0
// stores the SM clock at fixed points of every chunk step in [kTlFirst,
// kTlFirst + kTlChunks) into a per-kernel __device__ array; the host reads it
// back through ttt_debug_timeline (exported by that build only).  The stamps
// show how long each role spends between hand-offs and where the sequential
// chain waits.  In the normal build the stamps compile to nothing.
#pragma once

namespace ttt {
constexpr int kTlRoles = 8, kTlEvents = 8, kTlChunks = 32, kTlFirst = 1024;
}

#ifdef TTT_TIMELINE
#define TTT_TIMELINE_BUFFER(name) __device__ long long name[ttt::kTlRoles][ttt::kTlChunks][ttt::kTlEvents]
#define TTT_STAMP(buf, leader, role, c, ev)                                                   \
    do {                                                                                      \
        const int tl_c_ = (c) - ttt::kTlFirst;                                                \
        if ((leader) && blockIdx.x == 0 && tl_c_ >= 0 && tl_c_ < ttt::kTlChunks)              \
            buf[role][tl_c_][ev] = clock64();                                                 \
    } while (0)
#else
#define TTT_TIMELINE_BUFFER(name) static_assert(true, "timeline off")
#define TTT_STAMP(buf, leader, role, c, ev) ((void)0)
#endif
