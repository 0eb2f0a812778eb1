// kvprep_sm100.cuh -- the pass before the prefill attention: rotate every key
// once and lay keys and values out as fp16 for the tensor cores.
//
// Rotation ("Arch_03_Long_Context", RoPE slide): pair (2i, 2i+1) of the key at
// position n (= pos0 + its index) turns by n * theta'_i; the angle is reduced in
// fp64 (turns minus the nearest integer) before fp32 sin/cos.  Each key is rotated
// once here instead of once per query tile that reads it.
//
// One thread handles 8 consecutive elements (16 bytes) of one key row and the
// same 8 elements of the value row: coalesced 16-byte loads and stores, a
// grid-stride loop sized to the SM count.  A rotated key or a value that does not
// fit fp16 (|x| >= 65520, or not a number) sets the range bit of the device status
// word instead of passing silently into the attention as infinity.
#pragma once
#include "sm100_ptx.cuh"

namespace yr {

struct KvPrepParams {
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;
    long long ksb, ksh, kst, vsb, vsh, vst;
    __half *k16;  // [B*Hkv][T][d]
    __half *v16;  // [B*Hkv][T][d]
    __nv_bfloat16 *kc;  // optional rotated-key output (bf16), caller strides
    long long csb, csh, cst;
    float *k_dbg;  // optional [B*Hkv][T][d] fp32
    int Hkv, T, d;
    int pos0;           // key t is rotated at position pos0 + t
    long long n_items;  // B*Hkv*T*(d/8)
    double turns[64];
};

__device__ __forceinline__ void unpack_bf16x8(const uint4 &raw, float (&x)[8]) {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__global__ void __launch_bounds__(256) kv_prep_kernel(const __grid_constant__ KvPrepParams p) {
    __shared__ double turns[64];
    if (threadIdx.x < p.d / 2) turns[threadIdx.x] = p.turns[threadIdx.x];
    __syncthreads();
    bool bad = false;  // some rotated key or value of this thread does not fit fp16
    const int cpr = p.d >> 3;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
         g < p.n_items; g += stride) {
        const int c = static_cast<int>(g % cpr);
        const long long row = g / cpr;  // (b*Hkv + h)*T + t
        const int t = static_cast<int>(row % p.T);
        const long long bh = row / p.T;
        const int b = static_cast<int>(bh / p.Hkv);
        const int h = static_cast<int>(bh % p.Hkv);
        const uint4 kr = __ldg(reinterpret_cast<const uint4 *>(p.k + b * p.ksb + h * p.ksh +
                                                               t * p.kst + c * 8));
        const uint4 vr = __ldg(reinterpret_cast<const uint4 *>(p.v + b * p.vsb + h * p.vsh +
                                                               t * p.vst + c * 8));
        float x[8], y[8];
        unpack_bf16x8(kr, x);
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            const double tr = static_cast<double>(p.pos0 + t) * turns[c * 4 + pp];
            const double frac = tr - rint(tr);
            float sn, cs;
            __sincosf(static_cast<float>(frac * 6.283185307179586), &sn, &cs);
            y[2 * pp] = x[2 * pp] * cs - x[2 * pp + 1] * sn;
            y[2 * pp + 1] = x[2 * pp] * sn + x[2 * pp + 1] * cs;
        }
        const long long off = row * p.d + c * 8;
        *reinterpret_cast<uint4 *>(p.k16 + off) =
            make_uint4(pack_half2(y[0], y[1]), pack_half2(y[2], y[3]), pack_half2(y[4], y[5]),
                       pack_half2(y[6], y[7]));
        float vf[8];
        unpack_bf16x8(vr, vf);
#pragma unroll
        for (int i = 0; i < 8; ++i) bad |= f16_out_of_range(y[i]) | f16_out_of_range(vf[i]);
        *reinterpret_cast<uint4 *>(p.v16 + off) =
            make_uint4(pack_half2(vf[0], vf[1]), pack_half2(vf[2], vf[3]),
                       pack_half2(vf[4], vf[5]), pack_half2(vf[6], vf[7]));
        if (p.kc != nullptr) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
                w[i] = *reinterpret_cast<uint32_t *>(&b2);
            }
            *reinterpret_cast<uint4 *>(p.kc + b * p.csb + h * p.csh + t * p.cst + c * 8) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (p.k_dbg != nullptr) {
            float4 *d4 = reinterpret_cast<float4 *>(p.k_dbg + off);
            d4[0] = make_float4(y[0], y[1], y[2], y[3]);
            d4[1] = make_float4(y[4], y[5], y[6], y[7]);
        }
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) raise_status(kStatusRange);
}

// Chunked prefill: the Tq new tokens of each sequence sit at positions P0 ..
// P0+Tq-1 after a cached prefix.  Keys [0, P0) come from the rotated bf16 cache
// as they were written; keys [P0, P0+Tq) are the chunk's, rotated at their
// positions and appended to the cache (bf16) at those slots, with their values.
// All Tk = P0 + Tq keys and values land as fp16 in the workspace for the
// attention kernel.  Same thread shape as kv_prep_kernel.
struct ChunkPrepParams {
    const __nv_bfloat16 *k_new;  // [B*Hkv][Tq][d]
    const __nv_bfloat16 *v_new;  // [B*Hkv][Tq][d]
    __nv_bfloat16 *kc;           // [B*Hkv][T_max][d]
    __nv_bfloat16 *vc;           // [B*Hkv][T_max][d]
    __half *k16;                 // [B*Hkv][Tk][d]
    __half *v16;                 // [B*Hkv][Tk][d]
    int Tq, P0, Tk, T_max, d;
    long long n_items;           // B*Hkv*Tk*(d/8)
    double turns[64];
};

// bf16 -> fp16, eight at a time; `bad` is set if one of them does not fit fp16.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4 &raw, bool &bad) {
    float x[8];
    unpack_bf16x8(raw, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) bad |= f16_out_of_range(x[i]);
    return make_uint4(pack_half2(x[0], x[1]), pack_half2(x[2], x[3]), pack_half2(x[4], x[5]),
                      pack_half2(x[6], x[7]));
}

__global__ void __launch_bounds__(256) chunk_prep_kernel(const __grid_constant__ ChunkPrepParams p) {
    __shared__ double turns[64];
    if (threadIdx.x < p.d / 2) turns[threadIdx.x] = p.turns[threadIdx.x];
    __syncthreads();
    bool bad = false;  // some key or value of this thread does not fit fp16
    const int cpr = p.d >> 3;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
         g < p.n_items; g += stride) {
        const int c = static_cast<int>(g % cpr);
        const long long row = g / cpr;  // bh * Tk + t
        const int t = static_cast<int>(row % p.Tk);
        const long long bh = row / p.Tk;
        const long long off = row * p.d + c * 8;
        const long long slot = (bh * p.T_max + t) * p.d + c * 8;
        if (t < p.P0) {
            const uint4 kr = __ldg(reinterpret_cast<const uint4 *>(p.kc + slot));
            const uint4 vr = __ldg(reinterpret_cast<const uint4 *>(p.vc + slot));
            *reinterpret_cast<uint4 *>(p.k16 + off) = bf16x8_to_f16x8(kr, bad);
            *reinterpret_cast<uint4 *>(p.v16 + off) = bf16x8_to_f16x8(vr, bad);
            continue;
        }
        const long long src = (bh * p.Tq + (t - p.P0)) * p.d + c * 8;
        const uint4 kr = __ldg(reinterpret_cast<const uint4 *>(p.k_new + src));
        const uint4 vr = __ldg(reinterpret_cast<const uint4 *>(p.v_new + src));
        float x[8], y[8];
        unpack_bf16x8(kr, x);
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
            const double tr = static_cast<double>(t) * turns[c * 4 + pp];
            const double frac = tr - rint(tr);
            float sn, cs;
            __sincosf(static_cast<float>(frac * 6.283185307179586), &sn, &cs);
            y[2 * pp] = x[2 * pp] * cs - x[2 * pp + 1] * sn;
            y[2 * pp + 1] = x[2 * pp] * sn + x[2 * pp + 1] * cs;
        }
        *reinterpret_cast<uint4 *>(p.k16 + off) =
            make_uint4(pack_half2(y[0], y[1]), pack_half2(y[2], y[3]), pack_half2(y[4], y[5]),
                       pack_half2(y[6], y[7]));
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&b2);
        }
        *reinterpret_cast<uint4 *>(p.kc + slot) = make_uint4(w[0], w[1], w[2], w[3]);
#pragma unroll
        for (int i = 0; i < 8; ++i) bad |= f16_out_of_range(y[i]);
        *reinterpret_cast<uint4 *>(p.v16 + off) = bf16x8_to_f16x8(vr, bad);
        *reinterpret_cast<uint4 *>(p.vc + slot) = vr;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) raise_status(kStatusRange);
}

}  // namespace yr
