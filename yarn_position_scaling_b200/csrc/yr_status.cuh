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
    kStatusRange = 1u << 9,           // prefill: an operand outside the fp16 range (|x| >= 65520,
                                      // or not a number) after rotation or conversion
};
// Largest magnitude that rounds to a finite fp16 (65504 is the largest finite value;
// round-to-nearest sends [65504, 65520) to it and anything from 65520 on to infinity).
constexpr float kF16RoundsFinite = 65520.0f;
}  // namespace yr

// One word per device; only this translation unit defines kernels.
__device__ unsigned int g_yr_status = 0u;

namespace yr {
__device__ __forceinline__ void raise_status(unsigned bits) { atomicOr(&g_yr_status, bits); }
// True when x would not survive conversion to fp16 (overflow to infinity, or NaN).
__device__ __forceinline__ bool f16_out_of_range(float x) { return !(fabsf(x) < kF16RoundsFinite); }
__device__ __forceinline__ bool global_abort() {
    return (*reinterpret_cast<volatile unsigned *>(&g_yr_status) & 0xFFu) != 0u;
}
}  // namespace yr
