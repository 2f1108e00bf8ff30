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

// One 32-byte store of 8 floats (sm_100): a whole L2 sector per lane, half
// the transactions of two 16-byte stores.  ptr must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(float *ptr, const float (&v)[8]) {
    asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr),
                 "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
                 "f"(v[7])
                 : "memory");
}

}  // namespace pa
