// merge_sm100.cuh -- combine attention partials computed over disjoint key blocks.
//
// Ring attention ("long-context-models", section "Context parallelism distributes
// exact attention"; "Long context (engineering 100k+ tokens)", sec. 3): each
// worker attends its query block to one key/value block at a time and folds the
// partial result into a running one with the online-softmax weights.  With lse in
// natural-log units and L = log(e^lse_acc + e^lse_part):
//     o_acc <- e^(lse_acc - L) o_acc + e^(lse_part - L) o_part,   lse_acc <- L.
// A row with no visible key in a block has lse_part = -inf and weight 0; a row
// that has seen no key at all keeps lse_acc = -inf (its o_acc is never read).
// With init set, the accumulator is taken as empty without reading it: the first
// block's call needs no pre-filled buffers.
//
// HBM-bound: per row, 4d bytes of o_part and 4d of o_acc read, 4d written (+2d for
// the optional bf16 copy).  One warp covers 32 / (d/8) whole rows, one lane 8
// elements (32-byte loads), so each row's lanes share a warp and the lse update
// waits for all of them with a __syncwarp.  Partials stay fp32 until the last
// merge: one bf16 rounding of the result, as in a single-pass prefill.
#pragma once
#include "sm100_ptx.cuh"

namespace yr {

struct MergeParams {
    const float *o_part;          // [rows][d]
    const float *lse_part;        // [rows]
    float *o_acc;                 // [rows][d], updated in place
    float *lse_acc;               // [rows], updated in place
    __nv_bfloat16 *o_out;         // optional [rows][d]: bf16 of the merged rows
    long long rows;
    int d;
    int init;  // 1: o_acc and lse_acc are empty (not read)
};

__global__ void __launch_bounds__(256) attn_merge_kernel(const __grid_constant__ MergeParams p) {
    const int cpr = p.d >> 3;  // lanes per row (8 or 16)
    const int rows_per_warp = 32 / cpr;
    const int lane = threadIdx.x & 31;
    const int sub = lane / cpr, c = lane % cpr;
    const long long warp0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long n_warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    for (long long rg = warp0; rg * rows_per_warp < p.rows; rg += n_warps) {
        const long long row = rg * rows_per_warp + sub;
        const bool live = row < p.rows;
        float l_new = -INFINITY;
        if (live) {
            const float la = p.init ? -INFINITY : p.lse_acc[row], lp = p.lse_part[row];
            const float m = fmaxf(la, lp);
            if (m > -INFINITY) {
                const float wa = expf(la - m), wp = expf(lp - m);
                const float sum = wa + wp;
                l_new = m + logf(sum);
                const float ca = wa / sum, cp = wp / sum;
                const long long off = row * p.d + c * 8;
                // Rows that are empty on either side are not read: they may be garbage.
                const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
                const float4 *part = reinterpret_cast<const float4 *>(p.o_part + off);
                const float4 p0 = lp > -INFINITY ? part[0] : z, p1 = lp > -INFINITY ? part[1] : z;
                float4 *acc = reinterpret_cast<float4 *>(p.o_acc + off);
                const float4 a0 = la > -INFINITY ? acc[0] : z, a1 = la > -INFINITY ? acc[1] : z;
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                float r[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) r[i] = fmaf(ca, av[i], cp * pv[i]);
                acc[0] = make_float4(r[0], r[1], r[2], r[3]);
                acc[1] = make_float4(r[4], r[5], r[6], r[7]);
                if (p.o_out != nullptr) {
                    uint32_t pk[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(r[2 * i], r[2 * i + 1]);
                        pk[i] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    *reinterpret_cast<uint4 *>(p.o_out + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            } else if (p.o_out != nullptr) {
                *reinterpret_cast<uint4 *>(p.o_out + row * p.d + c * 8) = make_uint4(0, 0, 0, 0);
            }
        }
        __syncwarp();  // every lane of the row has read lse_acc
        if (live && c == 0) p.lse_acc[row] = l_new;
    }
}

// Split-KV prefill: n_split partials per row, each normalised over its share of the
// keys with its log-sum-exp, combined into the bf16 output (and the lse):
//     M = max_s lse_s,  o = sum_s e^(lse_s - M) o_s / sum_s e^(lse_s - M),
//     lse = M + log sum_s e^(lse_s - M).
// A share with no visible key for the row has lse_s = -inf and is not read.  One
// lane per 8 elements of a row; HBM-bound (4d bytes per row and share read, 2d written).
struct SplitMergeParams {
    const float *o_part;    // [n_split][rows][d]
    const float *lse_part;  // [n_split][rows]
    __nv_bfloat16 *o;       // [rows][d]
    float *lse;             // [rows] or null
    long long rows;
    int d, n_split;
};

__global__ void __launch_bounds__(256) split_merge_kernel(const __grid_constant__ SplitMergeParams p) {
    const int cpr = p.d >> 3;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
         g < p.rows * cpr; g += stride) {
        const long long row = g / cpr;
        const int c = static_cast<int>(g % cpr);
        float M = -INFINITY;
        for (int s = 0; s < p.n_split; ++s) M = fmaxf(M, p.lse_part[s * p.rows + row]);
        float r[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float sum = 0.f;
        if (M > -INFINITY) {
            for (int s = 0; s < p.n_split; ++s) {
                const float ls = p.lse_part[s * p.rows + row];
                if (ls == -INFINITY) continue;
                const float w = expf(ls - M);
                sum += w;
                const float4 *src =
                    reinterpret_cast<const float4 *>(p.o_part + (s * p.rows + row) * p.d + c * 8);
                const float4 a = src[0], bq = src[1];
                r[0] = fmaf(w, a.x, r[0]); r[1] = fmaf(w, a.y, r[1]);
                r[2] = fmaf(w, a.z, r[2]); r[3] = fmaf(w, a.w, r[3]);
                r[4] = fmaf(w, bq.x, r[4]); r[5] = fmaf(w, bq.y, r[5]);
                r[6] = fmaf(w, bq.z, r[6]); r[7] = fmaf(w, bq.w, r[7]);
            }
            const float inv = 1.0f / sum;
#pragma unroll
            for (int i = 0; i < 8; ++i) r[i] *= inv;
        }
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(r[2 * i], r[2 * i + 1]);
            pk[i] = *reinterpret_cast<uint32_t *>(&b2);
        }
        *reinterpret_cast<uint4 *>(p.o + row * p.d + c * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        if (p.lse != nullptr && c == 0) p.lse[row] = M > -INFINITY ? M + logf(sum) : -INFINITY;
    }
}

}  // namespace yr
