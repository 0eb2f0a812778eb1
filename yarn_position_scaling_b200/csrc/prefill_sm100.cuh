// prefill_sm100.cuh -- causal / windowed GQA attention prefill for sm_100a with
// rotary position embedding applied to Q inside the kernel.
//
// One CTA owns two 128-row query tiles (Q0, Q1) and walks the key/value tiles
// their rows can see.  Q0 and Q1 are rows [0, 128) and [128, 256) of a 256-row block
// of one (batch, head), or (head pairs, for windowed calls with an even number of
// query heads per KV head) the same 128 rows of two query heads of one KV group, which
// see exactly the same key tiles.  Roles:
//   warp 8      TMA producer: Q tiles once, then K~/V tiles through a 2-stage ring
//   warp 9      MMA issuer: S_t = Q_t K~^T and O_t += P_t V with tcgen05.mma,
//               accumulators in tensor memory (TMEM); the whole warp runs the
//               loop and one elected lane issues
//   warps 10-11 build the per-lane rotation table for the Q prologue
//   warps 0-3   softmax for Q0, warps 4-7 softmax for Q1: each thread owns one
//               query row (= one TMEM lane), so row max and row sum need no
//               shuffles; P is written back over S in TMEM as fp16
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+d), O1 [256+d,256+2d).
// The MMA issue order S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ... lets one
// softmax group work while the tensor cores serve the other ("ping-pong"); each
// S_t(j+1) follows its PV_t(j) directly, since it overwrites the P that PV reads.
//
// The keys may be one block of a longer sequence (ring attention): key n sits at
// position k_pos0 + n; masks work relative to key 0, only Q's rotation uses the
// absolute position, and a query tile that sees none of the keys writes o = 0 and
// lse = -inf.  The output is bf16, or fp32 for such block partials.
//
// Online softmax ("Long Context" concept page, key math: scores never reach
// HBM; "long-context-models", context parallelism: running row maxima,
// normalisation sums and output accumulators): a row's reference max only
// moves when its probabilities against the current reference would not fit
// fp16 (some p > 2^15), so O is rescaled rarely and most tiles need no row max.
//
// A row with no reference yet tries 0 and keeps it when its tile sum lies in
// [128, 2^15] (then its largest p is at least 1).  Masked tiles apply a per-row
// bit mask built from the causal, window and sink bounds.
//
// Rotation ("Arch_03_Long_Context", RoPE slide): pair (2i, 2i+1) of the query
// at position m turns by m * theta'_i (or pair (i, i + d/2) in the half-split
// layout, a separate instantiation of the kernel).  Each softmax warp reduces the angle of
// every pair at its first row in fp64 (turns minus the nearest integer) and takes its
// fp32 sin/cos; a row at lane l of the warp adds l * theta'_i by angle addition with
// (cos, sin)(l * theta'_i) from a table the two idle warps of the load/MMA warpgroup
// build once per CTA, so the prologue takes one sin/cos per pair and warp instead of
// one per element.  A rotated value that does not fit fp16 sets the range bit of the
// device status word.  Rarely run
// paths are kept small (rolled loops, compact masks): their instructions are
// fetched cold.
//
// Every wait is bounded (wall clock + a CTA abort flag + the device status
// word); a CTA that gives up drains its own copies and MMAs, frees TMEM and
// returns.
#pragma once
#include "sm100_ptx.cuh"

namespace yr {

constexpr int kBlockM = 128;
constexpr int kBlockN = 128;
constexpr int kQTiles = 2;
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kPrefillThreads = 384;  // 3 warpgroups: softmax Q0, softmax Q1, load/MMA
// Register split (setmaxnreg): the softmax warpgroups grow, the load/MMA one
// shrinks.  256 * 192 + 128 * 112 = 63488 <= 384 * 168 registers at launch; the
// host checks the launched count before the first launch.
constexpr int kRegsSoftmax = 192;
constexpr int kRegsOther = 112;
constexpr int kMinLaunchRegs = (256 * kRegsSoftmax + 128 * kRegsOther + 383) / 384;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxPairs = 64;
constexpr int kSubTileBytes = 128 * 128;  // 128 rows x 64 16-bit columns, 128-byte swizzle
// Upper bound on a row's probabilities within one tile before its reference max
// must move: P is stored as fp16 (max 65504), so 2^15 leaves a factor of two.
constexpr float kPBound = 32768.0f;

struct alignas(64) PrefillParams {
    CUtensorMap tm_q;  // bf16 [B][Hq][T][d] (4-D, caller strides)
    CUtensorMap tm_k;  // fp16 [B*Hkv][T][d] rotated keys (workspace)
    CUtensorMap tm_v;  // fp16 [B*Hkv][T][d] values (workspace)
    __nv_bfloat16 *o;
    long long osb, osh, ost;
    float *o32;  // if set: O as fp32 [B][Hq][T][d] (contiguous) instead of o
    float *lse;
    float *q_dbg;
    int B, Hq, Hkv, T, group;  // T: query rows
    // Masks work in key-index coordinates: key n of the workspace sits at position
    // k_pos0 + n, query row r at k_pos0 + q_off + r.  Only the rotation of Q needs the
    // absolute position, so it adds k_pos0 back (0 unless the keys are a block of a
    // longer sequence, as in ring attention).
    int Tk, q_off;             // keys, and the offset of query row 0 from key 0
    int k_pos0;
    int causal, window, n_sink;
    int n_qblocks;
    int kv_major;  // CTA order: 1 = by KV head first (grouped heads), 0 = by query block
    // 1: the CTA's two query tiles are heads h and h + 1 of one KV group at the same 128
    // rows (so both see exactly the same key tiles); 0: rows [0, 128) and [128, 256) of one
    // head.  n_qblocks counts 128-row blocks with head pairs, 256-row blocks without.
    int head_pair;
    int alibi;     // 1: add the ALiBi bias -m_h (i - j) to the logits
    // Split-KV: each (batch, head, query block) item is cut into n_split CTAs that take
    // equal shares of its key tiles; CTA s writes its normalised fp32 partial to
    // o32 + s * split_rows * d and its log-sum-exp to lse + s * split_rows, and a merge
    // kernel combines them.  n_split = 1: one CTA per item.
    int n_split;
    long long split_rows;
    float sl2;  // softmax_scale * log2(e)
    unsigned long long timeout_ns;
    // Failure-detection test hook, compiled only into the test build (YR_FAULT_HOOKS):
    // CTA 0's producer issues no copy for this key tile index (-1: off), so a wait that
    // nothing will complete runs out of time.
    int fault_drop_tile;
    double turns[64];
};

template <int HD>
struct PrefillSmem {
    static constexpr int kSub = HD / 64;
    uint8_t q[kQTiles][kSub][kSubTileBytes];
    uint8_t k[kKStages][kSub][kSubTileBytes];
    uint8_t v[kVStages][kSub][kSubTileBytes];
    uint64_t q_full[kQTiles], q_ready[kQTiles];
    uint64_t lanes_ready;
    uint64_t k_full[kKStages], k_empty[kKStages];
    uint64_t v_full[kVStages], v_empty[kVStages];
    uint64_t s_full[kQTiles], p_full[kQTiles], o_done[kQTiles];
    // Q rotation: per softmax warp, the angle (turns, reduced) of each pair at the
    // warp's first row, and the pair's rotations per position in fp32.
    float2 q_cs0[8][kMaxPairs];       // per softmax warp: (cos, sin) of pair i at its first row
    float2 lane_cs[kMaxPairs][32];    // (cos, sin) of lane * theta'_i, lane 0..31
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort;
};

// Key tiles one CTA visits, the n starting at position `first` (0, or the start of this
// CTA's share under split-KV) of the item's sequence.  Without a window the sequence is
// the tiles from lo on.  With a window it is the window's tiles after its first (fully
// visible to every row of a head-paired CTA), then the window's first tile, then the sink
// tiles [0, sink_end): a row's first tile is then a full one, on which reference 0 is
// normally kept, and the masked tiles (diagonal, window edge, sinks) come last and in a
// row (order-balanced A/B, 20 rounds: +1.7% / +2.7% on the windowed 64K YaRN / RoPE
// workloads; the online softmax takes its tiles in any order).
struct TilePlan {
    int sink_end, lo, n, first;
    int n_win;  // tiles of the window (lo .. lo + n_win - 1) when windowed, else 0
};

// q0 and last_row are query positions.
__device__ __forceinline__ TilePlan plan_tiles(const PrefillParams &p, int q0, int last_row) {
    TilePlan tp;
    // The last key any row may see: its own position (causal) or the last key, whichever
    // comes first (the keys can end before the rows when they are one block of a longer
    // sequence).
    const int hi = (p.causal ? min(last_row, p.Tk - 1) : p.Tk - 1) / kBlockN;
    if (p.window > 0) {
        const int first_key = max(0, q0 - p.window + 1);
        tp.lo = first_key / kBlockN;
        const int sink_tiles = (p.n_sink + kBlockN - 1) / kBlockN;
        tp.sink_end = min(min(sink_tiles, tp.lo), hi + 1);
    } else {
        tp.lo = 0;
        tp.sink_end = 0;
    }
    tp.n = tp.sink_end + max(0, hi - tp.lo + 1);
    tp.first = 0;
    tp.n_win = p.window > 0 ? tp.n - tp.sink_end : 0;
    return tp;
}
__device__ __forceinline__ int tile_at(const TilePlan &tp, int idx) {
    const int g = tp.first + idx;
    if (tp.n_win > 0) {
        if (g < tp.n_win - 1) return tp.lo + 1 + g;
        return g == tp.n_win - 1 ? tp.lo : g - tp.n_win;
    }
    return g < tp.sink_end ? g : tp.lo + (g - tp.sink_end);
}

// Does any (row, key) pair of rows [r_lo, r_hi] x tile j pass the visibility rule?
__device__ __forceinline__ bool tile_visible(const PrefillParams &p, int r_lo, int r_hi, int j) {
    if (r_lo > r_hi) return false;
    const int k_lo = j * kBlockN;
    const int k_hi = min(k_lo + kBlockN - 1, p.Tk - 1);
    if (k_lo > p.Tk - 1) return false;
    if (!p.causal) return true;
    if (k_lo > r_hi) return false;
    if (p.window > 0) {
        const int d_min = max(0, max(r_lo, k_lo) - k_hi);
        if (!(d_min < p.window || k_lo < p.n_sink)) return false;
    }
    return true;
}
// Is every pair visible (no masking needed)?
__device__ __forceinline__ bool tile_full(const PrefillParams &p, int r_lo, int r_hi, int j) {
    const int k_lo = j * kBlockN;
    const int k_hi = k_lo + kBlockN - 1;
    if (k_hi > p.Tk - 1) return false;
    if (p.causal && k_hi > r_lo) return false;
    if (p.window > 0 && !(r_hi - k_lo < p.window || k_hi < p.n_sink)) return false;
    return true;
}

// Query head of tile t of a CTA whose tile 0 has head h.  (Evaluated where it is used: a
// variable held across the softmax loop costs the d = 64 kernel a spill.)
__device__ __forceinline__ int tile_head(const PrefillParams &p, int h, int t) {
    return t == 0 ? h : h + p.head_pair;
}

// Bits 0..min(c, 31) set (0 for c < 0): columns at or below c of a 32-column word.
__device__ __forceinline__ uint32_t cols_upto(int c) {
    if (c < 0) return 0u;
    if (c >= 31) return 0xFFFFFFFFu;
    return (2u << c) - 1u;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// (a0, a1) += (b0, b1) as one packed f32x2 add: same per-lane rounding as two
// scalar adds, half the instructions in the row-sum chains.
__device__ __forceinline__ void add_f32x2(float &a0, float &a1, float b0, float b1) {
    uint64_t a = (static_cast<uint64_t>(__float_as_uint(a1)) << 32) | __float_as_uint(a0);
    const uint64_t b = (static_cast<uint64_t>(__float_as_uint(b1)) << 32) | __float_as_uint(b0);
    asm("add.rn.f32x2 %0, %0, %1;" : "+l"(a) : "l"(b));
    a0 = __uint_as_float(static_cast<uint32_t>(a));
    a1 = __uint_as_float(static_cast<uint32_t>(a >> 32));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

template <int HD, bool kHalfPairs>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    prefill_attn_kernel(const __grid_constant__ PrefillParams p) {
    using Smem = PrefillSmem<HD>;
    constexpr int kSub = Smem::kSub;
    extern __shared__ uint8_t smem_raw[];
    Smem *sm = reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Split-KV: the shares of one item are adjacent CTAs.
    const int split = p.n_split > 1 ? static_cast<int>(blockIdx.x) % p.n_split : 0;
    const int item = p.n_split > 1 ? static_cast<int>(blockIdx.x) / p.n_split
                                   : static_cast<int>(blockIdx.x);
    int qb, b, h;  // h: the head of query tile 0 (tile 1's is h + head_pair)
    if (p.kv_major) {
        // Grouped heads: one (batch, KV head) after another, its query blocks
        // heaviest first and the query heads (or head pairs) of its group adjacent, so
        // the CTAs resident at any time read the K/V of one or two KV heads, which stay
        // in L2.
        const int units = p.head_pair ? p.group / 2 : p.group;  // head units per KV head
        const int per_kv = p.n_qblocks * units;
        const int bk = item / per_kv;
        const int rem = item % per_kv;
        qb = p.n_qblocks - 1 - rem / units;
        b = bk / p.Hkv;
        h = (bk % p.Hkv) * p.group + (rem % units) * (p.head_pair ? 2 : 1);
    } else {
        // Heaviest causal blocks first, the heads of one query block adjacent.
        const int bh_count = p.B * p.Hq;
        qb = p.n_qblocks - 1 - item / bh_count;
        const int rem = item % bh_count;
        b = rem / p.Hq;
        h = rem % p.Hq;
    }
    const int kvh = h / p.group;
    // Query tiles by position: row r of the query tensor sits at position q_off + r.
    const int block_rows = p.head_pair ? kBlockM : kQTiles * kBlockM;
    const int q0 = p.q_off + qb * block_rows;
    const int last_pos = min(q0 + block_rows - 1, p.q_off + p.T - 1);
    TilePlan tp = plan_tiles(p, q0, last_pos);
    if (p.n_split > 1) {
        const int per = (tp.n + p.n_split - 1) / p.n_split;
        tp.first = min(split * per, tp.n);
        tp.n = min(per, tp.n - tp.first);
    }
    int r_lo[kQTiles], r_hi[kQTiles];
#pragma unroll
    for (int t = 0; t < kQTiles; ++t) {
        r_lo[t] = p.head_pair ? q0 : q0 + t * kBlockM;
        r_hi[t] = min(r_lo[t] + kBlockM - 1, last_pos);
    }

    if (threadIdx.x == 0) {
        for (int t = 0; t < kQTiles; ++t) {
            mbar_init(&sm->q_full[t], 1);
            mbar_init(&sm->q_ready[t], kBlockM / 32);  // one arrival per softmax warp
            mbar_init(&sm->s_full[t], 1);
            mbar_init(&sm->p_full[t], kBlockM / 32);
            mbar_init(&sm->o_done[t], 1);
        }
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&sm->k_full[s], 1);
            mbar_init(&sm->k_empty[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&sm->v_full[s], 1);
            mbar_init(&sm->v_empty[s], 1);
        }
        mbar_init(&sm->mma_done, 1);
        mbar_init(&sm->lanes_ready, 2);  // warps 10 and 11
        sm->abort = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tmem_alloc(&sm->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        prefetch_tensormap(&p.tm_q);
        prefetch_tensormap(&p.tm_k);
        prefetch_tensormap(&p.tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;
    volatile int *abort = &sm->abort;

    if (warp >= 8) {
      // load/MMA warpgroup (warps 8-11; 10 and 11 build the rotation table): shrink first
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
      if (warp >= 10) {
        // ------------------------------------------ per-lane rotation table
        // (cos, sin) of lane * theta'_i for lane 0..31: angle reduced in fp64 (turns
        // minus the nearest integer), one fp32 sin/cos per entry, for all CTAs' rows.
        for (int e = (warp - 10) * 32 + lane; e < (HD / 2) * 32; e += 64) {
            const int i = e >> 5, l = e & 31;
            const double tr = static_cast<double>(l) * p.turns[i];
            float sn, cs;
            __sincosf(static_cast<float>((tr - rint(tr)) * 6.283185307179586), &sn, &cs);
            sm->lane_cs[i][l] = make_float2(cs, sn);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->lanes_ready);
      } else if (warp == 8) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            bool ok = true;
            for (int t = 0; t < kQTiles; ++t) {
                if (r_lo[t] > r_hi[t]) continue;
                mbar_arrive_expect_tx(&sm->q_full[t], kSub * kSubTileBytes);
                for (int s = 0; s < kSub; ++s)
                    tma_load_4d(sm->q[t][s], &p.tm_q, &sm->q_full[t], s * 64, r_lo[t] - p.q_off,
                                tile_head(p, h, t), b, pol_q);
            }
            const int kv_plane = b * p.Hkv + kvh;
            int issued_k[kKStages] = {}, issued_v[kVStages] = {};
            for (int idx = 0; idx < tp.n && ok; ++idx) {
                const int j = tile_at(tp, idx);
                const int ks = idx % kKStages, vs = idx % kVStages;
#ifdef YR_FAULT_HOOKS
                if (idx == p.fault_drop_tile && blockIdx.x == 0) continue;
#endif
                ok = mbar_wait(&sm->k_empty[ks], ((idx / kKStages) & 1) ^ 1, abort, p.timeout_ns);
                if (!ok) break;
                mbar_arrive_expect_tx(&sm->k_full[ks], kSub * kSubTileBytes);
                for (int s = 0; s < kSub; ++s)
                    tma_load_3d(sm->k[ks][s], &p.tm_k, &sm->k_full[ks], s * 64, j * kBlockN,
                                kv_plane, pol_kv);
                ++issued_k[ks];
                ok = mbar_wait(&sm->v_empty[vs], ((idx / kVStages) & 1) ^ 1, abort, p.timeout_ns);
                if (!ok) break;
                mbar_arrive_expect_tx(&sm->v_full[vs], kSub * kSubTileBytes);
                for (int s = 0; s < kSub; ++s)
                    tma_load_3d(sm->v[vs][s], &p.tm_v, &sm->v_full[vs], s * 64, j * kBlockN,
                                kv_plane, pol_kv);
                ++issued_v[vs];
            }
            if (!ok) {
                raise_status(kStatusTimeoutLoad);
                sm->abort = 1;
            }
            // Drain: every copy this thread issued must land before the CTA exits.
            bool drained = true;
            for (int t = 0; t < kQTiles; ++t)
                if (r_lo[t] <= r_hi[t]) drained &= mbar_wait_drain(&sm->q_full[t], 0, p.timeout_ns);
            for (int s = 0; s < kKStages; ++s)
                if (issued_k[s])
                    drained &= mbar_wait_drain(&sm->k_full[s], (issued_k[s] - 1) & 1, p.timeout_ns);
            for (int s = 0; s < kVStages; ++s)
                if (issued_v[s])
                    drained &= mbar_wait_drain(&sm->v_full[s], (issued_v[s] - 1) & 1, p.timeout_ns);
            if (!drained) raise_status(kStatusTimeoutDrain);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ------------------------------------------------------- MMA issuer
        // The whole warp runs this loop, so its control flow and every operand
        // descriptor are warp-uniform; one elected lane issues the tcgen05.mma
        // and tcgen05.commit instructions.
        const bool leader = elect_one();
        constexpr uint32_t idesc_s = idesc_f16_f32(kBlockM, kBlockN, false, false);
        constexpr uint32_t idesc_o = idesc_f16_f32(kBlockM, HD, false, true);
        constexpr uint32_t kStageBytes = kSub * kSubTileBytes;
        const uint64_t desc_q0 = sw128_desc(smem_u32(sm->q[0][0]), 16, 1024);
        const uint64_t desc_q1 = sw128_desc(smem_u32(sm->q[1][0]), 16, 1024);
        const uint64_t desc_k = sw128_desc(smem_u32(sm->k[0][0]), 16, 1024);
        const uint64_t desc_v = sw128_desc(smem_u32(sm->v[0][0]), kSubTileBytes, 1024);
        bool ok = true;
        bool vis[kQTiles];
        int pv_count[kQTiles] = {0, 0};
        for (int t = 0; t < kQTiles; ++t)
            if (ok && r_lo[t] <= r_hi[t])
                ok = __all_sync(0xffffffffu, mbar_wait(&sm->q_ready[t], 0, abort, p.timeout_ns));
        tc_fence_after();

        // Descriptors advance by (byte offset >> 4) in their start-address field.
        auto issue_s = [&](int t, int ks) {
            const uint64_t da = t == 0 ? desc_q0 : desc_q1;
            const uint64_t db = desc_k + ((ks * kStageBytes) >> 4);
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * kSubTileBytes + (kk & 3) * 32) >> 4;
                    mma_ss(tmem + t * kBlockN, da + off, db + off, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm->s_full[t]);
            }
            __syncwarp();
        };
        auto issue_pv = [&](int t, int vs) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(&sm->p_full[t], pv_count[t] & 1, abort, p.timeout_ns)))
                return false;
            tc_fence_after();
            const uint64_t db = desc_v + ((vs * kStageBytes) >> 4);
            const uint32_t first = pv_count[t] > 0 ? 1u : 0u;
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < kBlockN / 16; ++kk)
                    mma_ts(tmem + 2 * kBlockN + t * HD, tmem + t * kBlockN + kk * 8,
                           db + ((kk * 2048) >> 4), idesc_o, kk > 0 ? 1u : first);
                mma_commit(&sm->o_done[t]);
            }
            __syncwarp();
            ++pv_count[t];
            return true;
        };

        // Tensor-pipe order: S0(0) S1(0) | PV0(0) S0(1) PV1(0) S1(1) | PV0(1) S0(2) ...
        // S_t(i+1) overwrites the P that PV_t(i) reads; tcgen05 MMAs from one thread
        // run in issue order, so it is issued right behind PV_t(i), with nothing in
        // between: the next tile's bookkeeping and its K and V waits are done while
        // this tile's softmax runs, before the wait for P.
        if (tp.n > 0) {
            const int j = tile_at(tp, 0);
            for (int t = 0; t < kQTiles; ++t) vis[t] = tile_visible(p, r_lo[t], r_hi[t], j);
            ok = __all_sync(0xffffffffu, mbar_wait(&sm->k_full[0], 0, abort, p.timeout_ns));
            if (ok) {
                tc_fence_after();
                if (vis[0]) issue_s(0, 0);
                if (vis[1]) issue_s(1, 0);
                if (leader) mma_commit(&sm->k_empty[0]);
                __syncwarp();
            }
        }
        for (int idx = 0; idx < tp.n && ok; ++idx) {
            const int vs = idx % kVStages;
            const int ks1 = (idx + 1) % kKStages;
            const bool has_next = idx + 1 < tp.n;
            bool vis1[kQTiles] = {false, false};
            if (has_next) {
                const int j1 = tile_at(tp, idx + 1);
                for (int t = 0; t < kQTiles; ++t) vis1[t] = tile_visible(p, r_lo[t], r_hi[t], j1);
            }
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&sm->v_full[vs], (idx / kVStages) & 1, abort, p.timeout_ns));
            if (ok && has_next)
                ok = __all_sync(0xffffffffu, mbar_wait(&sm->k_full[ks1], ((idx + 1) / kKStages) & 1,
                                                       abort, p.timeout_ns));
            if (!ok) break;
            tc_fence_after();
            if (vis[0] && !(ok = issue_pv(0, vs))) break;
            if (vis1[0]) issue_s(0, ks1);
            if (vis[1] && !(ok = issue_pv(1, vs))) break;
            if (leader) mma_commit(&sm->v_empty[vs]);
            if (vis1[1]) issue_s(1, ks1);
            if (leader && has_next) mma_commit(&sm->k_empty[ks1]);
            __syncwarp();
            vis[0] = vis1[0];
            vis[1] = vis1[1];
        }
        if (!ok) {
            if (leader) {
                raise_status(kStatusTimeoutMma);
                sm->abort = 1;
            }
        }
        // Drain: all MMAs issued above complete before TMEM/smem go away.
        if (leader) mma_commit(&sm->mma_done);
        __syncwarp();
        if (!__all_sync(0xffffffffu, mbar_wait_drain(&sm->mma_done, 0, p.timeout_ns)) && leader)
            raise_status(kStatusTimeoutDrain);
      }
    } else {
        // ------------------------------------------------- softmax warpgroups
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        const int t = warp >> 2;
        const int my_lo = t == 0 ? r_lo[0] : r_lo[1];
        const int my_hi = t == 0 ? r_hi[0] : r_hi[1];
        const int lane_base = (warp & 3) * 32;
        const int r = lane_base + lane;  // row within the tile = TMEM lane
        const int pos = my_lo + r;       // position of this thread's query row
        const int row = pos - p.q_off;   // its index in the query tensor
        const uint32_t tm_lane = static_cast<uint32_t>(lane_base) << 16;
        const uint32_t tm_s = tmem + tm_lane + t * kBlockN;
        const uint32_t tm_o = tmem + tm_lane + 2 * kBlockN + t * HD;
        const bool tile_live = my_lo <= my_hi;
        bool ok = true;

        if (tile_live) {
            // Rotate this row of Q in shared memory: bf16 in, fp16 out, in place.
            ok = mbar_wait(&sm->q_full[t], 0, abort, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                float *dbg = (p.q_dbg != nullptr && row < p.T)
                                 ? p.q_dbg + ((static_cast<long long>(b) * p.Hq + tile_head(p, h, t)) * p.T +
                                              row) * HD
                                 : nullptr;
                // Angle of pair i at this row = the warp's first row's angle plus
                // lane * theta'_i: (cos, sin) of the first (fp64-reduced, fp32 sin/cos, once
                // per warp and pair) times (cos, sin) of the lane's offset (a table built
                // once per CTA), by angle addition.
                float2 *cs0 = sm->q_cs0[warp];
                const int pos0 = pos - lane;
                for (int i = lane; i < HD / 2; i += 32) {
                    const double tr = static_cast<double>(pos0 + p.k_pos0) * p.turns[i];
                    float sn, cs;
                    __sincosf(static_cast<float>((tr - rint(tr)) * 6.283185307179586), &sn, &cs);
                    cs0[i] = make_float2(cs, sn);
                }
                __syncwarp();
                ok = __all_sync(0xffffffffu, mbar_wait(&sm->lanes_ready, 0, abort, p.timeout_ns));
                bool bad = false;  // a rotated value of this row does not fit fp16
                // sin/cos of pair i's angle at this row
                auto pair_sincos = [&](int i, float &sn, float &cs) {
                    const float2 a = cs0[i], l = sm->lane_cs[i][lane];
                    cs = fmaf(a.x, l.x, -a.y * l.y);
                    sn = fmaf(a.y, l.x, a.x * l.y);
                };
                // 16-byte chunk g (elements 8g .. 8g+7) of this row in the swizzled tile
                auto q_chunk = [&](int g) {
                    return reinterpret_cast<uint4 *>(sm->q[t][g >> 3] + r * 128 +
                                                     (((g & 7) ^ (r & 7)) << 4));
                };
                if constexpr (kHalfPairs) {
                    // Pairs (i, i + d/2): chunk c holds the first elements of pairs
                    // 8c .. 8c+7, chunk c + d/16 their second elements.
#pragma unroll 1
                    for (int c = 0; c < HD / 16; ++c) {
                        uint4 *plo = q_chunk(c), *phi = q_chunk(c + HD / 16);
                        const uint4 rlo = *plo, rhi = *phi;
                        const uint32_t wl[4] = {rlo.x, rlo.y, rlo.z, rlo.w};
                        const uint32_t wh[4] = {rhi.x, rhi.y, rhi.z, rhi.w};
                        float ylo[8], yhi[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const uint32_t bits_lo = (e & 1) ? (wl[e >> 1] & 0xFFFF0000u) : (wl[e >> 1] << 16);
                            const uint32_t bits_hi = (e & 1) ? (wh[e >> 1] & 0xFFFF0000u) : (wh[e >> 1] << 16);
                            const float a = __uint_as_float(bits_lo), bb = __uint_as_float(bits_hi);
                            float sn, cs;
                            pair_sincos(c * 8 + e, sn, cs);
                            ylo[e] = a * cs - bb * sn;
                            yhi[e] = a * sn + bb * cs;
                            bad |= f16_out_of_range(ylo[e]) | f16_out_of_range(yhi[e]);
                        }
                        *plo = make_uint4(pack_half2(ylo[0], ylo[1]), pack_half2(ylo[2], ylo[3]),
                                          pack_half2(ylo[4], ylo[5]), pack_half2(ylo[6], ylo[7]));
                        *phi = make_uint4(pack_half2(yhi[0], yhi[1]), pack_half2(yhi[2], yhi[3]),
                                          pack_half2(yhi[4], yhi[5]), pack_half2(yhi[6], yhi[7]));
                        if (dbg) {
                            float4 *dl = reinterpret_cast<float4 *>(dbg + c * 8);
                            float4 *dh = reinterpret_cast<float4 *>(dbg + HD / 2 + c * 8);
                            dl[0] = make_float4(ylo[0], ylo[1], ylo[2], ylo[3]);
                            dl[1] = make_float4(ylo[4], ylo[5], ylo[6], ylo[7]);
                            dh[0] = make_float4(yhi[0], yhi[1], yhi[2], yhi[3]);
                            dh[1] = make_float4(yhi[4], yhi[5], yhi[6], yhi[7]);
                        }
                    }
                } else {
                    // Pairs (2i, 2i+1): chunk c holds pairs 4c .. 4c+3.
#pragma unroll 1
                    for (int c = 0; c < HD / 8; ++c) {
                        uint4 *ptr = q_chunk(c);
                        const uint4 raw = *ptr;
                        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
                        uint32_t out[4];
                        float y[8];
#pragma unroll
                        for (int pp = 0; pp < 4; ++pp) {
                            const float a = __uint_as_float(w[pp] << 16);
                            const float bb = __uint_as_float(w[pp] & 0xFFFF0000u);
                            float sn, cs;
                            pair_sincos(c * 4 + pp, sn, cs);
                            y[2 * pp] = a * cs - bb * sn;
                            y[2 * pp + 1] = a * sn + bb * cs;
                            bad |= f16_out_of_range(y[2 * pp]) | f16_out_of_range(y[2 * pp + 1]);
                            out[pp] = pack_half2(y[2 * pp], y[2 * pp + 1]);
                        }
                        *ptr = make_uint4(out[0], out[1], out[2], out[3]);
                        if (dbg) {
                            float4 *d4 = reinterpret_cast<float4 *>(dbg + c * 8);
                            d4[0] = make_float4(y[0], y[1], y[2], y[3]);
                            d4[1] = make_float4(y[4], y[5], y[6], y[7]);
                        }
                    }
                }
                if (__any_sync(0xffffffffu, bad) && lane == 0) raise_status(kStatusRange);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->q_ready[t]);
            }
        }

        // ALiBi slope of this head, m_h = 2^(-8 (h+1) / Hq), over the softmax scale.
        const float alibi_coef =
            p.alibi ? exp2f(-8.0f * static_cast<float>(tile_head(p, h, t) + 1) /
                            static_cast<float>(p.Hq)) *
                          1.4426950408889634f / p.sl2
                    : 0.0f;
        float m_run = -INFINITY;  // reference max of this row, log2 units (score * sl2)
        float l_run = 0.0f;       // sum of exp2(score * sl2 - m_run) so far
        int it = 0;
        const float sl2 = p.sl2;
        for (int idx = 0; idx < tp.n && ok && tile_live; ++idx) {
            const int j = tile_at(tp, idx);
            if (!tile_visible(p, my_lo, my_hi, j)) continue;
            ok = mbar_wait(&sm->s_full[t], it & 1, abort, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            float s[kBlockN];
            {
                // The whole score row in one TMEM load (measured ~1% faster at 128K than
                // four 32-column loads).
                static_assert(kBlockN == 128, "one 128-column TMEM load per score row");
                uint32_t raw[kBlockN];
                tmem_ld128(tm_s, raw);
                tmem_ld_wait();
                reg_fence128(raw);
#pragma unroll
                for (int e = 0; e < kBlockN; ++e) s[e] = __uint_as_float(raw[e]);
            }
            if (p.alibi) {
                // ALiBi: logit - m_h (pos - n), folded into the raw score as
                // s + (m_h / softmax_scale) (n - pos).  Far keys get a large negative
                // score whose rounding does not matter: their weight is ~0.
                const float b0 = alibi_coef * static_cast<float>(j * kBlockN - pos);
#pragma unroll
                for (int c = 0; c < kBlockN; ++c) s[c] += fmaf(alibi_coef, static_cast<float>(c), b0);
            }
            if (!tile_full(p, my_lo, my_hi, j)) {
                // Visible columns of this row as a bit mask: c <= c_hi (causal, in range)
                // and (c >= c_lo or c < c_sink) (window, sinks); one select per score.
                const int k0 = j * kBlockN;
                int c_hi = p.Tk - 1 - k0;
                if (p.causal) c_hi = min(c_hi, pos - k0);
                const int c_lo = p.window > 0 ? pos - p.window + 1 - k0 : -(1 << 30);
                const int c_sink = p.window > 0 ? p.n_sink - k0 : -(1 << 30);
#pragma unroll
                for (int w32 = 0; w32 < kBlockN / 32; ++w32) {
                    const uint32_t vis = cols_upto(c_hi - 32 * w32) &
                                         (~cols_upto(c_lo - 1 - 32 * w32) | cols_upto(c_sink - 1 - 32 * w32));
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (!((vis >> e) & 1u)) s[w32 * 32 + e] = -INFINITY;
                }
            }
            auto exps_to_tmem = [&](float m_ref_in) -> float {
                // Scalar FMAs feed the scalar ex2 (measured on sm_100a, a packed f32x2
                // FMA there costs about twice as many cycles per element); the row
                // sums take packed adds.
                const float m_ref = (m_ref_in == -INFINITY) ? 0.0f : m_ref_in;
                const float neg_m = -m_ref;
                float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < kBlockN / 32; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float p0 = ex2(fmaf(s[c * 32 + 2 * e], sl2, neg_m));
                        const float p1 = ex2(fmaf(s[c * 32 + 2 * e + 1], sl2, neg_m));
                        add_f32x2(acc[(2 * e) & 7], acc[(2 * e + 1) & 7], p0, p1);
                        pk[e] = pack_half2(p0, p1);
                    }
                    tmem_st16(tm_s + c * 16, pk);
                }
                return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
            };
            // A row with a reference max takes its exponentials against it without
            // looking at this tile's max: P only has to fit fp16, and since every
            // p <= l_tile, l_tile <= kPBound proves it does.  A row with no reference
            // yet tries 0 (log2 units) and keeps it when kBlockN <= l_tile <= kPBound:
            // then its largest p is at least 1, as with the exact max, so the small p
            // keep the precision they would have had.
            // Rows that fail, in warps where any row fails, take the tile max, move
            // their reference to it and redo P (rare: a row's running max grows
            // slowly, and typical scores pass the first test).
            const bool fresh = m_run == -INFINITY;
            float l_tile = exps_to_tmem(m_run);  // reference 0 for a fresh row
            bool over = fresh ? !(l_tile >= static_cast<float>(kBlockN) && l_tile <= kPBound)
                              : !(l_tile <= kPBound);
            if (fresh && !over) m_run = 0.0f;
            if (__any_sync(0xffffffffu, over)) {
                // Tile max in four independent chains of three-input max: s[0..3] start
                // the chains, s[4..123] go eight per step, s[124..127] close them.
                static_assert(kBlockN % 8 == 0, "tile max covers the tile in steps of 8");
                float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
                for (int c = 4; c + 8 <= kBlockN - 4; c += 8) {
                    m4[0] = fmax3(m4[0], s[c], s[c + 1]);
                    m4[1] = fmax3(m4[1], s[c + 2], s[c + 3]);
                    m4[2] = fmax3(m4[2], s[c + 4], s[c + 5]);
                    m4[3] = fmax3(m4[3], s[c + 6], s[c + 7]);
                }
                m4[0] = fmax3(m4[0], s[kBlockN - 4], s[kBlockN - 3]);
                m4[1] = fmax3(m4[1], s[kBlockN - 2], s[kBlockN - 1]);
                const float m_tile = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * sl2;
                const bool first = m_run == -INFINITY;
                const bool move = first || (over && m_tile > m_run);
                const float m_new = move ? fmaxf(m_run, m_tile) : m_run;
                const bool rescale = !first && m_new > m_run;
                const float alpha = rescale ? ex2(m_run - m_new) : 1.0f;
                tmem_st_wait();
                l_tile = exps_to_tmem(m_new);
                if (it > 0 && __any_sync(0xffffffffu, rescale)) {
                    // O holds P V up to the previous tile: wait for it, then rescale.
                    ok = mbar_wait(&sm->o_done[t], (it - 1) & 1, abort, p.timeout_ns);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    tc_fence_after();
                    uint32_t raw[32];
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        tmem_ld32_sync(tm_o + c * 32, raw);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
                        tmem_st32(tm_o + c * 32, raw);
                    }
                }
                // Rows seen for the first time have O = 0 and l = 0: nothing to rescale.
                l_run *= alpha;
                m_run = m_new;
            }
            l_run += l_tile;
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->p_full[t]);
            ++it;
        }
        if (!ok) {
            raise_status(kStatusTimeoutSoftmax);
            sm->abort = 1;
        }
        // Epilogue: O / l -> bf16 (or fp32), and the log-sum-exp in natural-log units.
        const long long orow_idx =
            (static_cast<long long>(b) * p.Hq + tile_head(p, h, t)) * p.T + row + split * p.split_rows;
        if (ok && tile_live && it > 0) {
            ok = mbar_wait(&sm->o_done[t], (it - 1) & 1, abort, p.timeout_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc_fence_after();
                const float inv_l = (l_run > 0.0f) ? 1.0f / l_run : 0.0f;
                __nv_bfloat16 *orow = p.o + b * p.osb + tile_head(p, h, t) * p.osh +
                                      static_cast<long long>(row) * p.ost;
                uint32_t raw[32];
#pragma unroll
                for (int c = 0; c < HD / 32; ++c) {
                    tmem_ld32_sync(tm_o + c * 32, raw);
                    if (row < p.T && p.o32 != nullptr) {
                        float4 *dst = reinterpret_cast<float4 *>(p.o32 + orow_idx * HD + c * 32);
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4)
                            dst[q4] = make_float4(__uint_as_float(raw[4 * q4]) * inv_l,
                                                  __uint_as_float(raw[4 * q4 + 1]) * inv_l,
                                                  __uint_as_float(raw[4 * q4 + 2]) * inv_l,
                                                  __uint_as_float(raw[4 * q4 + 3]) * inv_l);
                    } else if (row < p.T) {
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                __nv_bfloat162 v2 = __floats2bfloat162_rn(
                                    __uint_as_float(raw[q4 * 8 + 2 * e]) * inv_l,
                                    __uint_as_float(raw[q4 * 8 + 2 * e + 1]) * inv_l);
                                pk[e] = *reinterpret_cast<uint32_t *>(&v2);
                            }
                            *reinterpret_cast<uint4 *>(orow + c * 32 + q4 * 8) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    }
                }
                if (p.lse != nullptr && row < p.T) {
                    const float m_ref = (m_run == -INFINITY) ? 0.0f : m_run;
                    p.lse[orow_idx] = (l_run > 0.0f) ? (m_ref + __log2f(l_run)) * 0.69314718055994531f
                                                     : -INFINITY;
                }
            } else {
                raise_status(kStatusTimeoutSoftmax);
                sm->abort = 1;
            }
        } else if (ok && tile_live && row < p.T) {
            // No key of this call is visible to the whole query tile (possible only when
            // the keys are one block of a longer sequence): o = 0, lse = -inf.
            if (p.o32 != nullptr) {
                float4 *dst = reinterpret_cast<float4 *>(p.o32 + orow_idx * HD);
#pragma unroll 1
                for (int c = 0; c < HD / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
            } else {
                __nv_bfloat16 *orow = p.o + b * p.osb + tile_head(p, h, t) * p.osh +
                                      static_cast<long long>(row) * p.ost;
#pragma unroll 1
                for (int c = 0; c < HD / 8; ++c)
                    *reinterpret_cast<uint4 *>(orow + c * 8) = make_uint4(0u, 0u, 0u, 0u);
            }
            if (p.lse != nullptr) p.lse[orow_idx] = -INFINITY;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

// Dynamic shared memory per CTA.  At least 116 KB, so that one CTA holds an SM
// (and all 512 TMEM columns) at a time for either head size.
template <int HD>
constexpr size_t prefill_smem_bytes() {
    return sizeof(PrefillSmem<HD>) + 1024 > 116 * 1024 ? sizeof(PrefillSmem<HD>) + 1024
                                                        : 116 * 1024;
}

}  // namespace yr
