// kvprep_sm100.cuh -- the pass before the prefill attention: rotate every key
// once and lay keys and values out as fp16 for the tensor cores.
//
// Rotation ("Arch_03_Long_Context", RoPE slide): pair (2i, 2i+1) of the key at
// position n (= pos0 + its index) turns by n * theta'_i; the angle is reduced in
// fp64 (turns minus the nearest integer) before fp32 sin/cos.  Each key is rotated
// once here instead of once per query tile that reads it.
//
// One thread handles 8 consecutive elements (16 bytes) of one key row and the
// same 8 elements of the value row (for the half-split pair layout, those and the
// 8 elements d/2 further on, which complete their pairs): coalesced 16-byte loads
// and stores, a grid-stride loop sized to the SM count.  A rotated key or a value that does not
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
    long long n_items;  // B*Hkv*T*(d/8), or B*Hkv*T*(d/16) for the half-split layout
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

// Rotates the eight pairs whose elements sit in x_a[e], x_b[e] (e = 0..7) at
// position `pos`; pair index i0 + e.  Interleaved pairs pass one chunk split into
// its even and odd elements; the half-split layout passes two chunks.
__device__ __forceinline__ void rotate8(const double *turns, int i0, long long pos,
                                        const float (&x_a)[8], const float (&x_b)[8],
                                        float (&y_a)[8], float (&y_b)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const double tr = static_cast<double>(pos) * turns[i0 + e];
        const double frac = tr - rint(tr);
        float sn, cs;
        __sincosf(static_cast<float>(frac * 6.283185307179586), &sn, &cs);
        y_a[e] = x_a[e] * cs - x_b[e] * sn;
        y_b[e] = x_a[e] * sn + x_b[e] * cs;
    }
}

__device__ __forceinline__ uint4 pack_half8(const float (&y)[8]) {
    return make_uint4(pack_half2(y[0], y[1]), pack_half2(y[2], y[3]), pack_half2(y[4], y[5]),
                      pack_half2(y[6], y[7]));
}
__device__ __forceinline__ uint4 pack_bf16x8(const float (&y)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&b2);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Rotates pair (2i, 2i+1) = (x[2e], x[2e+1]) of one interleaved chunk, i = i0 + e,
// e = 0..3, at position `pos`.
__device__ __forceinline__ void rotate4_interleaved(const double *turns, int i0, long long pos,
                                                    const float (&x)[8], float (&y)[8]) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const double tr = static_cast<double>(pos) * turns[i0 + e];
        const double frac = tr - rint(tr);
        float sn, cs;
        __sincosf(static_cast<float>(frac * 6.283185307179586), &sn, &cs);
        y[2 * e] = x[2 * e] * cs - x[2 * e + 1] * sn;
        y[2 * e + 1] = x[2 * e] * sn + x[2 * e + 1] * cs;
    }
}

// One key row's share of a thread.  kHalf = false: the 16 bytes at element 8c
// (pairs 4c .. 4c+3, interleaved).  kHalf = true: the 16 bytes at 8c and those at
// 8c + d/2 (pairs 8c .. 8c+7 of the half-split layout).  Writes the rotated keys
// (fp16 workspace, optional bf16 cache and fp32 debug copy) and the values (fp16);
// returns true if one of them does not fit fp16.
template <bool kHalf>
__device__ __forceinline__ bool kv_prep_item(const KvPrepParams &p, const double *turns,
                                             long long g) {
    const int cpr = kHalf ? (p.d >> 4) : (p.d >> 3);
    const int c = static_cast<int>(g % cpr);
    const long long row = g / cpr;  // (b*Hkv + h)*T + t
    const int t = static_cast<int>(row % p.T);
    const long long bh = row / p.T;
    const int b = static_cast<int>(bh / p.Hkv);
    const int h = static_cast<int>(bh % p.Hkv);
    const __nv_bfloat16 *krow = p.k + b * p.ksb + h * p.ksh + t * p.kst;
    const __nv_bfloat16 *vrow = p.v + b * p.vsb + h * p.vsh + t * p.vst;
    __nv_bfloat16 *kcrow = p.kc != nullptr ? p.kc + b * p.csb + h * p.csh + t * p.cst : nullptr;
    const long long off = row * p.d;
    const long long pos = static_cast<long long>(p.pos0) + t;
    constexpr int kChunks = kHalf ? 2 : 1;
    const int e_at[2] = {c * 8, c * 8 + p.d / 2};  // element offsets of the chunks
    float y[kChunks][8];
    if constexpr (kHalf) {
        float xa[8], xb[8];
        unpack_bf16x8(__ldg(reinterpret_cast<const uint4 *>(krow + e_at[0])), xa);
        unpack_bf16x8(__ldg(reinterpret_cast<const uint4 *>(krow + e_at[1])), xb);
        rotate8(turns, c * 8, pos, xa, xb, y[0], y[1]);
    } else {
        float x[8];
        unpack_bf16x8(__ldg(reinterpret_cast<const uint4 *>(krow + e_at[0])), x);
        rotate4_interleaved(turns, c * 4, pos, x, y[0]);
    }
    bool bad = false;
#pragma unroll
    for (int k = 0; k < kChunks; ++k) {
        const int e0 = e_at[k];
        float vf[8];
        unpack_bf16x8(__ldg(reinterpret_cast<const uint4 *>(vrow + e0)), vf);
#pragma unroll
        for (int i = 0; i < 8; ++i) bad |= f16_out_of_range(y[k][i]) | f16_out_of_range(vf[i]);
        *reinterpret_cast<uint4 *>(p.k16 + off + e0) = pack_half8(y[k]);
        *reinterpret_cast<uint4 *>(p.v16 + off + e0) = pack_half8(vf);
        if (kcrow != nullptr) *reinterpret_cast<uint4 *>(kcrow + e0) = pack_bf16x8(y[k]);
        if (p.k_dbg != nullptr) {
            float4 *d4 = reinterpret_cast<float4 *>(p.k_dbg + off + e0);
            d4[0] = make_float4(y[k][0], y[k][1], y[k][2], y[k][3]);
            d4[1] = make_float4(y[k][4], y[k][5], y[k][6], y[k][7]);
        }
    }
    return bad;
}

template <bool kHalf>
__global__ void __launch_bounds__(256) kv_prep_kernel(const __grid_constant__ KvPrepParams p) {
    __shared__ double turns[64];
    if (threadIdx.x < p.d / 2) turns[threadIdx.x] = p.turns[threadIdx.x];
    __syncthreads();
    bool bad = false;  // some rotated key or value of this thread does not fit fp16
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
         g < p.n_items; g += stride)
        bad |= kv_prep_item<kHalf>(p, turns, g);
    if (__syncthreads_or(bad) && threadIdx.x == 0) raise_status(kStatusRange);
}

// Chunked prefill: the Tq new tokens of each sequence sit at positions P0 ..
// P0+Tq-1 after a cached prefix.  Keys [0, P0) come from the rotated bf16 cache
// as they were written; keys [P0, P0+Tq) are the chunk's, rotated at their
// positions and appended to the cache (bf16) at those slots, with their values.
// The attention reads fp16 copies of keys and values [0, P0+Tq) from k16/v16:
// either a workspace that receives all of them on every call (ld16 = P0+Tq,
// first = 0), or a caller-kept fp16 copy of the cache (ld16 = T_max) whose slots
// [0, first) are already valid, so that a call converts only the slots after
// them and appends its own.  Same thread shape as kv_prep_kernel.
struct ChunkPrepParams {
    const __nv_bfloat16 *k_new;  // [B*Hkv][Tq][d]
    const __nv_bfloat16 *v_new;  // [B*Hkv][Tq][d]
    __nv_bfloat16 *kc;           // [B*Hkv][T_max][d]
    __nv_bfloat16 *vc;           // [B*Hkv][T_max][d]
    __half *k16;                 // [B*Hkv][ld16][d]
    __half *v16;                 // [B*Hkv][ld16][d]
    int Tq, P0, Tk, T_max, d;
    int first;                   // first slot to write into k16/v16 (0 .. P0)
    long long ld16;              // slots per (b, KV head) plane of k16/v16
    long long n_items;           // B*Hkv*(Tk-first)*(d/8), or *(d/16) for half-split pairs
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

template <bool kHalf>
__global__ void __launch_bounds__(256) chunk_prep_kernel(const __grid_constant__ ChunkPrepParams p) {
    __shared__ double turns[64];
    if (threadIdx.x < p.d / 2) turns[threadIdx.x] = p.turns[threadIdx.x];
    __syncthreads();
    bool bad = false;  // some key or value of this thread does not fit fp16
    const int cpr = kHalf ? (p.d >> 4) : (p.d >> 3);
    constexpr int kChunks = kHalf ? 2 : 1;
    const int rows = p.Tk - p.first;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
         g < p.n_items; g += stride) {
        const int c = static_cast<int>(g % cpr);
        const long long rr = g / cpr;
        const int t = p.first + static_cast<int>(rr % rows);
        const long long bh = rr / rows;
        const int e_at[2] = {c * 8, c * 8 + p.d / 2};
        const long long off = (bh * p.ld16 + t) * p.d;
        const long long slot = (bh * p.T_max + t) * p.d;
        if (t < p.P0) {
#pragma unroll
            for (int k = 0; k < kChunks; ++k) {
                const int e0 = e_at[k];
                const uint4 kr = __ldg(reinterpret_cast<const uint4 *>(p.kc + slot + e0));
                const uint4 vr = __ldg(reinterpret_cast<const uint4 *>(p.vc + slot + e0));
                *reinterpret_cast<uint4 *>(p.k16 + off + e0) = bf16x8_to_f16x8(kr, bad);
                *reinterpret_cast<uint4 *>(p.v16 + off + e0) = bf16x8_to_f16x8(vr, bad);
            }
            continue;
        }
        const long long src = (bh * p.Tq + (t - p.P0)) * p.d;
        float y[kChunks][8];
        if constexpr (kHalf) {
            float xa[8], xb[8];
            unpack_bf16x8(__ldg(reinterpret_cast<const uint4 *>(p.k_new + src + e_at[0])), xa);
            unpack_bf16x8(__ldg(reinterpret_cast<const uint4 *>(p.k_new + src + e_at[1])), xb);
            rotate8(turns, c * 8, t, xa, xb, y[0], y[1]);
        } else {
            float x[8];
            unpack_bf16x8(__ldg(reinterpret_cast<const uint4 *>(p.k_new + src + e_at[0])), x);
            rotate4_interleaved(turns, c * 4, t, x, y[0]);
        }
#pragma unroll
        for (int k = 0; k < kChunks; ++k) {
            const int e0 = e_at[k];
#pragma unroll
            for (int i = 0; i < 8; ++i) bad |= f16_out_of_range(y[k][i]);
            *reinterpret_cast<uint4 *>(p.k16 + off + e0) = pack_half8(y[k]);
            *reinterpret_cast<uint4 *>(p.kc + slot + e0) = pack_bf16x8(y[k]);
            const uint4 vr = __ldg(reinterpret_cast<const uint4 *>(p.v_new + src + e0));
            *reinterpret_cast<uint4 *>(p.v16 + off + e0) = bf16x8_to_f16x8(vr, bad);
            *reinterpret_cast<uint4 *>(p.vc + slot + e0) = vr;
        }
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) raise_status(kStatusRange);
}

}  // namespace yr
