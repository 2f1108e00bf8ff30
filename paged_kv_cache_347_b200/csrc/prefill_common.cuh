// Helpers shared by the two chunked-prefill kernels.
#pragma once

#include <cstdint>

namespace pa {

// L2 priority for a prefill's K/V loads: every token tile of a (sequence, KV
// head) reads the same blocks at different times, so they keep the default
// priority (the decode kernels, which read each block once, mark theirs
// evict-first).
__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

}  // namespace pa
