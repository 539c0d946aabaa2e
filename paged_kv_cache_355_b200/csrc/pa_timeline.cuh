// pa_timeline.cuh -- optional per-CTA timelines of the decode kernels:
// globaltimer stamps at fixed points of each CTA's life, compiled in only
// when PA_TIMELINE is defined (the libpa_timeline.so build).  Without it
// every stamp is an empty statement and the kernels are unchanged.
//
// Layout (read back with pa_timeline_read, include/pa_timeline.h):
//  * events: [kernel][cta][kTlSlots] u64, kernel 0 = the shared-prefix set-up
//    kernel, 1 = the tensor-core prefix pass, 2 = bf16 pass 1; cta = the
//    CTA's linear index x + gridDim.x * (y + gridDim.y * z); slot
//    kTlSlots - 1 holds the SM id, the others nanoseconds of %globaltimer
//    (0 = not reached);
//  * tiles: [cta][kTtTiles][kTtEvents] u64, per-tile events of the prefix
//    pass's first kTtCtas CTAs and first kTtTiles tiles.
// Only the last launch of each kernel since pa_timeline_clear is meaningful
// (later launches overwrite earlier ones).
#pragma once

#include <stdint.h>

#include "pa_device.cuh"

#ifdef PA_TIMELINE
namespace pa {

constexpr int kTlKernels = 3;
constexpr int kTlCtas = 65536;
constexpr int kTlSlots = 16;
constexpr int kTtCtas = 512;
constexpr int kTtTiles = 16;
constexpr int kTtEvents = 8;

__device__ unsigned long long g_pa_tl[(size_t)kTlKernels * kTlCtas * kTlSlots];
__device__ unsigned long long g_pa_tt[(size_t)kTtCtas * kTtTiles * kTtEvents];

__device__ __forceinline__ unsigned tl_cta() { return blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); }

// event `slot` of this CTA of kernel `kernel` (one thread per CTA calls it)
__device__ __forceinline__ void tl_stamp(int kernel, int slot) {
    const unsigned cta = tl_cta();
    if (cta >= (unsigned)kTlCtas) return;
    unsigned smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    unsigned long long* row = g_pa_tl + ((size_t)kernel * kTlCtas + cta) * kTlSlots;
    row[slot] = global_timer_ns();
    row[kTlSlots - 1] = smid;
}

// event `event` of tile `tile` of this CTA of the prefix pass
__device__ __forceinline__ void tt_stamp(int tile, int event) {
    const unsigned cta = tl_cta();
    if (cta >= (unsigned)kTtCtas || tile >= kTtTiles) return;
    g_pa_tt[((size_t)cta * kTtTiles + tile) * kTtEvents + event] = global_timer_ns();
}

}  // namespace pa
#define PA_TL(kernel, slot) ::pa::tl_stamp(kernel, slot)
#define PA_TT(tile, event) ::pa::tt_stamp(tile, event)
#else
#define PA_TL(kernel, slot) ((void)0)
#define PA_TT(tile, event) ((void)0)
#endif
