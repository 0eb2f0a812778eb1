// yr_status.cuh -- the device status word shared by every kernel of the library.
// Kernels never trap.  A kernel that gives up on a wait, or meets an input it
// cannot process, sets a bit here and returns; yr_device_status() reads it.
#pragma once

namespace yr {
enum StatusBits : unsigned {
    kStatusTimeoutLoad = 1u << 0,     // prefill TMA producer gave up waiting
    kStatusTimeoutMma = 1u << 1,      // prefill MMA issuer gave up waiting
    kStatusTimeoutSoftmax = 1u << 2,  // prefill softmax warps gave up waiting
    kStatusTimeoutDrain = 1u << 3,    // prefill teardown gave up draining copies/MMAs
    kStatusBadCacheLen = 1u << 8,     // decode: a cache length outside [0, T_max-1]
};
}  // namespace yr

// One word per device; only this translation unit defines kernels.
__device__ unsigned int g_yr_status = 0u;

namespace yr {
__device__ __forceinline__ void raise_status(unsigned bits) { atomicOr(&g_yr_status, bits); }
__device__ __forceinline__ bool global_abort() {
    return (*reinterpret_cast<volatile unsigned *>(&g_yr_status) & 0xFFu) != 0u;
}
}  // namespace yr
