// decode_sm100.cuh -- single-token decode over a bf16 KV cache, split-KV with
// a log-sum-exp merge ("Long Context" concept page: decode is memory-bound on
// the cache, which is read every step).
//
// Kernel 1 (decode_split_kernel): a balanced split.  The keys the new tokens see
// in all (sequence b, KV head) segments are laid end to end and cut into one equal
// share per block (at least kDecChunk keys), so every block streams the same number
// of bytes whatever the mix of cache lengths, and all finish together.  For each
// segment piece it holds, a block
//   * rotates the new query of each of the g = Hq/Hkv heads of the group at
//     position L_b (pairs (2i, 2i+1), or (i, i + d/2) in the half-split layout;
//     fp64 angle reduction, fp32 sin/cos) and splits it into a
//     bf16 high part and a bf16 remainder, so the product with the bf16 cache
//     keeps ~16 significant bits of the rotated query;
//   * if its piece ends at position L_b, rotates the new key and writes it, with
//     the new value, into cache slot L_b first;
//   * streams its K and V rows with 16-byte cp.async through a 3-stage ring
//     (rows past the piece arrive as zeros), every byte read once for all g heads;
//   * computes S^T = K q~^T (keys on the MMA's M side, heads on N) and
//     O^T += V^T P^T with mma.sync.m16n8k16, online softmax per head;
//   * leaves (max, sum, unnormalised output) per head in the workspace.
// Kernel 2 (decode_merge_kernel): per (b, query head), the log-sum-exp merge of the
// segment's pieces
//   M = max_c m_c;  O = sum_c 2^(m_c-M) o_c / sum_c 2^(m_c-M) l_c
// ("long-context-models", context parallelism: online softmax combines partial
// results).
#pragma once
#include "sm100_ptx.cuh"

namespace yr {

constexpr int kDecChunk = 2048;  // least keys per block of the balanced split
constexpr int kDecTile = 64;     // keys per pipeline stage
constexpr int kDecStages = 3;
constexpr int kDecWarps = 4;     // 16 keys of each stage per warp
constexpr int kDecThreads = kDecWarps * 32;

struct DecodeParams {
    const __nv_bfloat16 *q_new;  // [B][Hq][d]
    const __nv_bfloat16 *k_new;  // [B][Hkv][d]
    const __nv_bfloat16 *v_new;  // [B][Hkv][d]
    __nv_bfloat16 *k_cache;      // [B][Hkv][T_max][d]
    __nv_bfloat16 *v_cache;
    const int *cache_len;        // [B]
    float *ws_o;                 // [B][Hkv][NC][g][d]
    float *ws_ml;                // [B][Hkv][NC][g][2]
    __nv_bfloat16 *o;            // [B][Hq][d]
    float *lse;                  // [B][Hq] or null
    float *q_dbg;                // [B][Hq][d] or null
    int B, Hq, Hkv, T_max, group;
    int n_parts;      // partial-result slots per (b, KV head) in the workspace
    int grid_blocks;  // blocks of the split launch (the partition depends on it)
    int window, n_sink;
    float sl2;
    int alibi;  // 1: add the ALiBi bias -m_h (L - n) to the logits
    int half_pairs;  // 1: rotated pairs are (i, i + d/2); 0: (2i, 2i+1)
    double turns[64];
};

__device__ __forceinline__ bool dec_len_ok(const DecodeParams &p, int L) {
    return L >= 0 && L <= p.T_max - 1;
}
// Keys the new token at position L sees, as the ranges [0, len1) and [lo2, lo2 + len2):
// the sinks and the window, or one range [0, L] without a window or when they meet.
// A sequence with an out-of-range length has none.
struct DecRanges {
    int len1, lo2, len2;
};
__device__ __forceinline__ DecRanges dec_ranges(const DecodeParams &p, int L) {
    DecRanges r{0, 0, 0};
    if (!dec_len_ok(p, L)) return r;
    const int s1 = min(p.n_sink, L + 1);
    const int w0 = max(L - p.window + 1, 0);
    if (p.window <= 0 || w0 <= s1) {
        r.len1 = L + 1;
        r.lo2 = L + 1;
    } else {
        r.len1 = s1;
        r.lo2 = w0;
        r.len2 = L + 1 - w0;
    }
    return r;
}
// Balanced split: the visible keys of all (b, KV head) segments, in that order, are
// units; each block of the split launch takes U consecutive units, U at least
// kDecChunk so that per-block work dwarfs per-block set-up.  Every block and the
// merge derive the same partition from cache_len.
__device__ __forceinline__ long long dec_total_units(const DecodeParams &p) {
    long long t = 0;
    for (int b = 0; b < p.B; ++b) {
        const DecRanges r = dec_ranges(p, p.cache_len[b]);
        t += static_cast<long long>(p.Hkv) * (r.len1 + r.len2);
    }
    return t;
}
__device__ __forceinline__ long long dec_units_per_block(long long total, int grid_blocks) {
    const long long even = (total + grid_blocks - 1) / grid_blocks;
    return even > kDecChunk ? even : kDecChunk;
}
__device__ __forceinline__ bool dec_key_visible(int n, int L, int window, int n_sink) {
    if (n > L) return false;
    return window <= 0 || (L - n) < window || n < n_sink;
}

template <int HD>
struct DecodeSmem {
    static constexpr int kRowBytes = HD * 2;
    static constexpr int kStageBytes = kDecTile * kRowBytes;
    uint8_t k[kDecStages][kStageBytes];
    uint8_t v[kDecStages][kStageBytes];
    __nv_bfloat16 q_hi[16][HD];
    __nv_bfloat16 q_lo[16][HD];
    float red_m[kDecWarps][16];
    float red_l[kDecWarps][16];
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return static_cast<uint32_t>(((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                          uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&b);
}
__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <int HD, int NT>
__global__ void __launch_bounds__(kDecThreads, 2)
    decode_split_kernel(const __grid_constant__ DecodeParams p) {
    using Smem = DecodeSmem<HD>;
    constexpr int kCpr = HD / 8;  // 16-byte chunks per row
    extern __shared__ uint8_t smem_raw[];
    Smem *sm = reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                        ~static_cast<uintptr_t>(127));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = p.group;
    if (blockIdx.x == 0 && tid == 0)
        for (int bb = 0; bb < p.B; ++bb)
            if (!dec_len_ok(p, p.cache_len[bb])) raise_status(kStatusBadCacheLen);
    // This block's units [u_lo, u_hi) of the balanced split, walked segment by segment.
    const long long total = dec_total_units(p);
    const long long U = dec_units_per_block(total, p.grid_blocks);
    const long long u_lo = static_cast<long long>(blockIdx.x) * U;
    const long long u_hi = min(u_lo + U, total);
    long long seg0 = 0;  // first unit of segment (b, kvh)
    for (int b = 0; b < p.B && seg0 < u_hi; ++b) {
    const int L = p.cache_len[b];
    const DecRanges rg = dec_ranges(p, L);
    const long long V = rg.len1 + rg.len2;
    for (int kvh = 0; kvh < p.Hkv && seg0 < u_hi; ++kvh, seg0 += V) {
    if (V == 0 || seg0 + V <= u_lo) continue;
    // Units [a, e) of this segment map to keys [a, min(e, len1)) and the window
    // range from lo2; the key at L (the last unit) is this block's if e == V.
    const int a = static_cast<int>(max(u_lo, seg0) - seg0);
    const int e = static_cast<int>(min(u_hi, seg0 + V) - seg0);
    const int part = static_cast<int>(blockIdx.x - seg0 / U);
    const int r1_lo = a < rg.len1 ? a : 0, r1_hi = a < rg.len1 ? min(e, rg.len1) : 0;
    const int r2_lo = e > rg.len1 ? rg.lo2 + max(a, rg.len1) - rg.len1 : 0;
    const int r2_hi = e > rg.len1 ? rg.lo2 + e - rg.len1 : 0;
    const int n_t1 = (r1_hi - r1_lo + kDecTile - 1) / kDecTile;
    const int n_tiles = n_t1 + (r2_hi - r2_lo + kDecTile - 1) / kDecTile;
    const int n_begin = r1_hi > r1_lo ? r1_lo : r2_lo;   // span of this block's keys
    const int n_end = r2_hi > r2_lo ? r2_hi : r1_hi;
    const bool has_L = e == V;
    auto tile_start = [&](int i) { return i < n_t1 ? r1_lo + i * kDecTile : r2_lo + (i - n_t1) * kDecTile; };
    const long long plane = (static_cast<long long>(b) * p.Hkv + kvh) * p.T_max;
    const __nv_bfloat16 *kbase = p.k_cache + plane * HD;
    const __nv_bfloat16 *vbase = p.v_cache + plane * HD;

    // ---- prologue: rotated queries (hi/lo split), the new key into slot L
    // Elements (ia, ib) of pair i: (2i, 2i+1) interleaved, (i, i + d/2) half-split.
    auto pair_elems = [&](int i, int &ia, int &ib) {
        ia = p.half_pairs ? i : 2 * i;
        ib = p.half_pairs ? i + HD / 2 : 2 * i + 1;
    };
    for (int e = tid; e < 16 * (HD / 2); e += kDecThreads) {
        const int hh = e / (HD / 2), i = e % (HD / 2);
        int ia, ib;
        pair_elems(i, ia, ib);
        float y0 = 0.f, y1 = 0.f;
        if (hh < g && hh < 8 * NT) {
            const int hq = kvh * g + hh;
            const __nv_bfloat16 *qrow = p.q_new + (static_cast<long long>(b) * p.Hq + hq) * HD;
            const float a = __bfloat162float(qrow[ia]), c = __bfloat162float(qrow[ib]);
            const double tr = static_cast<double>(L) * p.turns[i];
            const double frac = tr - rint(tr);
            float sn, cs;
            __sincosf(static_cast<float>(frac * 6.283185307179586), &sn, &cs);
            y0 = a * cs - c * sn;
            y1 = a * sn + c * cs;
            if (p.q_dbg != nullptr && has_L) {
                float *d = p.q_dbg + (static_cast<long long>(b) * p.Hq + hq) * HD;
                d[ia] = y0;
                d[ib] = y1;
            }
        }
        const __nv_bfloat16 hi0 = __float2bfloat16_rn(y0), hi1 = __float2bfloat16_rn(y1);
        sm->q_hi[hh][ia] = hi0;
        sm->q_hi[hh][ib] = hi1;
        sm->q_lo[hh][ia] = __float2bfloat16_rn(y0 - __bfloat162float(hi0));
        sm->q_lo[hh][ib] = __float2bfloat16_rn(y1 - __bfloat162float(hi1));
    }
    if (has_L) {
        for (int i = tid; i < HD / 2; i += kDecThreads) {
            int ia, ib;
            pair_elems(i, ia, ib);
            const long long src = (static_cast<long long>(b) * p.Hkv + kvh) * HD;
            const float a = __bfloat162float(p.k_new[src + ia]);
            const float c = __bfloat162float(p.k_new[src + ib]);
            const double tr = static_cast<double>(L) * p.turns[i];
            const double frac = tr - rint(tr);
            float sn, cs;
            __sincosf(static_cast<float>(frac * 6.283185307179586), &sn, &cs);
            __nv_bfloat16 *kd = p.k_cache + (plane + L) * HD;
            kd[ia] = __float2bfloat16_rn(a * cs - c * sn);
            kd[ib] = __float2bfloat16_rn(a * sn + c * cs);
            __nv_bfloat16 *vd = p.v_cache + (plane + L) * HD;
            vd[ia] = p.v_new[src + ia];
            vd[ib] = p.v_new[src + ib];
        }
    }
    __syncthreads();  // orders the slot-L writes before the copies below

    // B fragments of q~^T (k = dims, n = heads), hi and lo parts, for every k-step.
    uint32_t qb_hi[HD / 16][NT][2], qb_lo[HD / 16][NT][2];
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int hh = nt * 8 + (lane >> 2);
            const int d0 = kk * 16 + 2 * (lane & 3);
            qb_hi[kk][nt][0] = *reinterpret_cast<const uint32_t *>(&sm->q_hi[hh][d0]);
            qb_hi[kk][nt][1] = *reinterpret_cast<const uint32_t *>(&sm->q_hi[hh][d0 + 8]);
            qb_lo[kk][nt][0] = *reinterpret_cast<const uint32_t *>(&sm->q_lo[hh][d0]);
            qb_lo[kk][nt][1] = *reinterpret_cast<const uint32_t *>(&sm->q_lo[hh][d0 + 8]);
        }

    auto load_tile = [&](int t0, int stage) {
        const uint32_t kdst = smem_u32(sm->k[stage]), vdst = smem_u32(sm->v[stage]);
#pragma unroll
        for (int u = 0; u < (kDecTile * kCpr) / kDecThreads; ++u) {
            const int e = tid + u * kDecThreads;
            const int r = e / kCpr, c = e % kCpr;
            const int n = t0 + r;
            const bool valid = n < n_end;
            const long long row = valid ? n : n_begin;
            const uint32_t so = static_cast<uint32_t>(r * Smem::kRowBytes) + swz(r, c);
            cp_async16(kdst + so, kbase + row * HD + c * 8, valid ? 16u : 0u);
            cp_async16(vdst + so, vbase + row * HD + c * 8, valid ? 16u : 0u);
        }
    };

#pragma unroll
    for (int s = 0; s < kDecStages - 1; ++s) {
        if (s < n_tiles) load_tile(tile_start(s), s);
        cp_async_commit();
    }

    float o[HD / 16][NT][4];
#pragma unroll
    for (int mt = 0; mt < HD / 16; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[mt][nt][e] = 0.f;
    float m_run[NT][2], l_run[NT][2];
    // ALiBi slope (log2 units) of this thread's two head columns per n-tile; 0 without ALiBi.
    float slope2[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int col = nt * 8 + 2 * (lane & 3) + jj;
            slope2[nt][jj] = (p.alibi && col < g)
                                 ? exp2f(-8.0f * static_cast<float>(kvh * g + col + 1) /
                                         static_cast<float>(p.Hq)) * 1.4426950408889634f
                                 : 0.0f;
        }
    }

    for (int i = 0; i < n_tiles; ++i) {
        cp_async_wait<kDecStages - 2>();
        __syncthreads();
        {
            const int nxt = i + kDecStages - 1;
            if (nxt < n_tiles) load_tile(tile_start(nxt), nxt % kDecStages);
            cp_async_commit();
        }
        const int stage = i % kDecStages;
        const int t0 = tile_start(i);
        // Keys of this tile's own range only: the last tile of the sink range can reach
        // into the window range, whose tiles count those keys.
        const int k_lo = i < n_t1 ? r1_lo : r2_lo, k_hi = i < n_t1 ? r1_hi : r2_hi;
        const uint32_t kst = smem_u32(sm->k[stage]), vst = smem_u32(sm->v[stage]);
        const int krow0 = warp * 16;  // this warp's 16 keys within the tile

        // S^T[16 keys x 8 heads] per n-tile, hi + lo query parts.
        float sc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
            const int mi = lane >> 3;
            const int r = krow0 + (lane & 7) + 8 * (mi & 1);
            const int c = kk * 2 + (mi >> 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(kst + r * Smem::kRowBytes + swz(r, c), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(sc[nt], a0, a1, a2, a3, qb_hi[kk][nt][0], qb_hi[kk][nt][1]);
                mma_bf16_16816(sc[nt], a0, a1, a2, a3, qb_lo[kk][nt][0], qb_lo[kk][nt][1]);
            }
        }
        // Mask and online softmax per head (columns).
        const int n_a = t0 + krow0 + (lane >> 2);
        const int n_b = n_a + 8;
        const bool vis_a = n_a >= k_lo && n_a < k_hi && dec_key_visible(n_a, L, p.window, p.n_sink);
        const bool vis_b = n_b >= k_lo && n_b < k_hi && dec_key_visible(n_b, L, p.window, p.n_sink);
        const float dist_a = static_cast<float>(L - n_a), dist_b = static_cast<float>(L - n_b);
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float x[4];
            x[0] = vis_a ? fmaf(sc[nt][0], p.sl2, -slope2[nt][0] * dist_a) : -INFINITY;
            x[1] = vis_a ? fmaf(sc[nt][1], p.sl2, -slope2[nt][1] * dist_a) : -INFINITY;
            x[2] = vis_b ? fmaf(sc[nt][2], p.sl2, -slope2[nt][0] * dist_b) : -INFINITY;
            x[3] = vis_b ? fmaf(sc[nt][3], p.sl2, -slope2[nt][1] * dist_b) : -INFINITY;
            float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
            }
            const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
            const float al0 = (m_run[nt][0] == -INFINITY) ? 0.f : ex2f(m_run[nt][0] - mn0);
            const float al1 = (m_run[nt][1] == -INFINITY) ? 0.f : ex2f(m_run[nt][1] - mn1);
            const float r0 = (mn0 == -INFINITY) ? 0.f : mn0;
            const float r1 = (mn1 == -INFINITY) ? 0.f : mn1;
            const float p0 = ex2f(x[0] - r0), p1 = ex2f(x[1] - r1);
            const float p2 = ex2f(x[2] - r0), p3 = ex2f(x[3] - r1);
            l_run[nt][0] = l_run[nt][0] * al0 + p0 + p2;
            l_run[nt][1] = l_run[nt][1] * al1 + p1 + p3;
            m_run[nt][0] = mn0;
            m_run[nt][1] = mn1;
#pragma unroll
            for (int mt = 0; mt < HD / 16; ++mt) {
                o[mt][nt][0] *= al0;
                o[mt][nt][1] *= al1;
                o[mt][nt][2] *= al0;
                o[mt][nt][3] *= al1;
            }
            pb[nt][0] = movm_t(pack_bf16x2(p0, p1));  // keys 0-7 of this warp
            pb[nt][1] = movm_t(pack_bf16x2(p2, p3));  // keys 8-15
        }
        // O^T[dims x heads] += V^T[dims x 16 keys] P^T[16 keys x heads]
#pragma unroll
        for (int mt = 0; mt < HD / 16; ++mt) {
            const int mi = lane >> 3;
            const int r = krow0 + (lane & 7) + 8 * (mi >> 1);
            const int c = mt * 2 + (mi & 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(vst + r * Smem::kRowBytes + swz(r, c), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                mma_bf16_16816(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- combine the 4 warps' states, then write this chunk's partial result
    float *red_o = reinterpret_cast<float *>(sm->k[0]);  // [warps][HD][16], reuses stage memory
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float l0 = l_run[nt][0], l1 = l_run[nt][1];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, off);
            l1 += __shfl_xor_sync(0xffffffffu, l1, off);
        }
        const int h0 = nt * 8 + 2 * (lane & 3);
        if (lane < 4) {
            sm->red_m[warp][h0] = m_run[nt][0];
            sm->red_m[warp][h0 + 1] = m_run[nt][1];
            sm->red_l[warp][h0] = l0;
            sm->red_l[warp][h0 + 1] = l1;
        }
#pragma unroll
        for (int mt = 0; mt < HD / 16; ++mt) {
            const int d0 = mt * 16 + (lane >> 2);
            float *base = red_o + (warp * HD) * 16;
            base[d0 * 16 + h0] = o[mt][nt][0];
            base[d0 * 16 + h0 + 1] = o[mt][nt][1];
            base[(d0 + 8) * 16 + h0] = o[mt][nt][2];
            base[(d0 + 8) * 16 + h0 + 1] = o[mt][nt][3];
        }
    }
    __syncthreads();
    const long long slot = ((static_cast<long long>(b) * p.Hkv + kvh) * p.n_parts + part) * g;
    for (int e = tid; e < g * HD; e += kDecThreads) {
        const int hh = e / HD, dd = e % HD;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sm->red_m[w][hh]);
        float acc = 0.f, sum = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) {
                const float mw = sm->red_m[w][hh];
                const float wt = (mw == -INFINITY) ? 0.f : ex2f(mw - M);
                acc += wt * red_o[(w * HD + dd) * 16 + hh];
                sum += wt * sm->red_l[w][hh];
            }
        }
        p.ws_o[(slot + hh) * HD + dd] = acc;
        if (dd == 0) {
            p.ws_ml[(slot + hh) * 2 + 0] = M;
            p.ws_ml[(slot + hh) * 2 + 1] = sum;
        }
    }
    __syncthreads();  // shared memory is reused by the next segment
    }  // kvh
    }  // b
}

template <int HD>
__global__ void __launch_bounds__(HD) decode_merge_kernel(const __grid_constant__ DecodeParams p) {
    const int hq = blockIdx.x, b = blockIdx.y, dd = threadIdx.x;
    const int L = p.cache_len[b];
    const long long oi = (static_cast<long long>(b) * p.Hq + hq);
    if (!dec_len_ok(p, L)) {
        p.o[oi * HD + dd] = __float2bfloat16(__int_as_float(0x7fc00000));
        if (p.lse != nullptr && dd == 0) p.lse[oi] = __int_as_float(0x7fc00000);
        return;
    }
    const int g = p.group, kvh = hq / g, hh = hq % g;
    // The split kernel's partition: this segment's units and the blocks that hold them.
    const long long total = dec_total_units(p);
    const long long U = dec_units_per_block(total, p.grid_blocks);
    long long seg0 = 0;
    for (int bb = 0; bb < b; ++bb) {
        const DecRanges r = dec_ranges(p, p.cache_len[bb]);
        seg0 += static_cast<long long>(p.Hkv) * (r.len1 + r.len2);
    }
    const DecRanges rg = dec_ranges(p, L);
    const long long V = rg.len1 + rg.len2;
    seg0 += kvh * V;
    const int n_parts = static_cast<int>((seg0 + V - 1) / U - seg0 / U) + 1;
    const long long base = (static_cast<long long>(b) * p.Hkv + kvh) * p.n_parts;
    float M = -INFINITY;
    for (int c = 0; c < n_parts; ++c) M = fmaxf(M, p.ws_ml[((base + c) * g + hh) * 2]);
    float acc = 0.f, sum = 0.f;
    for (int c = 0; c < n_parts; ++c) {
        const long long pi = (base + c) * g + hh;
        const float mc = p.ws_ml[pi * 2];
        const float w = (mc == -INFINITY) ? 0.f : ex2f(mc - M);
        sum += w * p.ws_ml[pi * 2 + 1];
        acc += w * p.ws_o[pi * HD + dd];
    }
    p.o[oi * HD + dd] = __float2bfloat16_rn(acc / sum);
    if (p.lse != nullptr && dd == 0) p.lse[oi] = (M + __log2f(sum)) * 0.69314718055994531f;
}

template <int HD>
constexpr size_t decode_smem_bytes() {
    return sizeof(DecodeSmem<HD>) + 128;
}

}  // namespace yr
