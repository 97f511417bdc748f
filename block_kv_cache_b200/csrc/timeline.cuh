// Per-CTA event clocks of instrumented builds (built with -DFDL_TIMELINE by
// `python -m block_kv_cache_b200.build --timeline`, into libfdllm_timeline.so;
// the product library is built without it and these macros expand to
// nothing). An instrumented kernel records %globaltimer (ns) at fixed events
// of its timeline into a per-file device array, slot [kind][cta][event], the
// last launch of a kind overwriting the previous one; a per-file entry point
// (fdl_timeline_<file>) copies the array to the host and clears it.
#pragma once
#include <stdint.h>

namespace fdl {
namespace tl {
constexpr int kKinds = 8, kCtas = 512, kEvents = 8;
constexpr size_t kSlots = (size_t)kKinds * kCtas * kEvents;
}  // namespace tl
}  // namespace fdl

#ifdef FDL_TIMELINE
// One array per translation unit (no relocatable device code): the file that
// includes this header with FDL_TIMELINE_FILE defined owns the reader.
static __device__ unsigned long long g_fdl_stamps[fdl::tl::kSlots];

__device__ __forceinline__ void fdl_stamp(int kind, int ev) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    const int cta = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    if (cta < fdl::tl::kCtas)
        g_fdl_stamps[((size_t)kind * fdl::tl::kCtas + cta) * fdl::tl::kEvents + ev] = t;
}
#define FDL_TL(kind, ev) fdl_stamp((kind), (ev))
// extern "C" reader of this file's array: copies kSlots u64 to host, clears.
#define FDL_TL_READER(name)                                                              \
    extern "C" __attribute__((visibility("default"))) int name(unsigned long long* host) { \
        if (cudaMemcpyFromSymbol(host, g_fdl_stamps, sizeof(g_fdl_stamps)) != cudaSuccess)  \
            return -3;                                                                   \
        static unsigned long long zeros[fdl::tl::kSlots];                                \
        return cudaMemcpyToSymbol(g_fdl_stamps, zeros, sizeof(zeros)) == cudaSuccess ? 0 : -3; \
    }
#else
#define FDL_TL(kind, ev) ((void)0)
#define FDL_TL_READER(name)
#endif
