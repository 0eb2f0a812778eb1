/*
 * yarnattn.h -- C ABI of libyarnattn.so: YaRN-RoPE causal grouped-query
 * attention on NVIDIA B200 (sm_100a).
 *
 * The library computes exact scaled-dot-product attention with rotary position
 * embedding applied to Q and K inside its kernels, in two forms: a prefill over
 * a whole sequence and a single-token decode over a KV cache.  It needs no
 * framework: arguments are plain pointers and sizes.  Device pointers must come
 * from the CUDA device that is current on the calling thread; `stream` is a
 * cudaStream_t (NULL = the legacy default stream).  Every compute call is
 * asynchronous on that stream and returns as soon as its kernels are queued.
 *
 * Ownership: the caller owns every buffer, including workspaces; the library
 * allocates no device memory and keeps no pointer after a call returns.
 *
 * Errors: every entry point returns YR_OK (0) or a negative YR_E* code, and
 * then yr_last_error() gives a message for the calling thread.  Arguments are
 * checked on the host before anything is launched.  Kernels never trap: a
 * kernel whose internal wait exceeds its time limit stops, records the fact in
 * a device status word and returns; yr_device_status() reads (and clears) it.
 *
 * Sources: the web pages on long-context position scaling --
 *   "LLM context window mechanics" (position wall; memory wall),
 *   "Long Context" concept page (key math),
 *   "Arch_03_Long_Context" slides (RoPE, PI, NTK-aware, YaRN, sliding window,
 *   attention sinks), "Long context (engineering 100k+ tokens)" (sec. 2 RoPE
 *   scaling, sec. 5 sinks), "long-context-models" (position enters attention).
 */
#ifndef YARNATTN_H
#define YARNATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define YR_OK 0
#define YR_EINVAL (-1)        /* an argument is out of range or inconsistent */
#define YR_EUNSUPPORTED (-2)  /* valid but not implemented (head_dim, device) */
#define YR_ECUDA (-3)         /* a CUDA runtime/driver call failed */
#define YR_ETIMEOUT (-4)      /* a kernel gave up on an internal wait */
#define YR_ERANGE (-5)        /* a prefill operand fell outside the fp16 range (see below) */

/* Position methods ("Arch_03_Long_Context": RoPE, PI, NTK-aware and YaRN slides). */
#define YR_ROPE 0  /* theta_i = base^(-2i/d) */
#define YR_PI 1    /* theta_i / s: positions compressed by the extension factor s */
#define YR_NTK 2   /* (base * s^(d/(d-2)))^(-2i/d) */
#define YR_YARN 3  /* per-band ramp between theta_i and theta_i / s, plus temperature */
/* Table variants ("Arch_03_Long_Context" NTK-aware slide, last sentence: dynamic NTK;
 * "Long context (engineering 100k+ tokens)" and "long-context-models": LongRoPE). */
#define YR_NTK_DYNAMIC 4  /* NTK-aware with s = max(1, L_cur / L_train) */
#define YR_YARN_DIMRAMP 5 /* YaRN with the ramp linear in the pair index (floor/ceil band edges) */
#define YR_FACTORS 6      /* theta_i / f_i with caller-supplied per-dimension factors */
/* ALiBi ("Arch_03_Long_Context", ALiBi slide; "long-context-models"): no rotation; the
 * kernels subtract m_h (i - j) from the scaled logit of query position i and key j,
 * with m_h = 2^(-8 (h+1) / Hq) for query head h. */
#define YR_ALIBI 7

#define YR_MAX_HEAD_DIM 128

/* Which elements of a head vector form the rotated pairs.  The pages print the
 * interleaved form ("Arch_03_Long_Context", RoPE slide: pair (2i, 2i+1)); the
 * half-split form (i, i + d/2), in which the first half of the vector holds the
 * first element of every pair, is the common alternative layout of the same
 * rotation.  Pair i turns by position * theta'_i in both. */
#define YR_PAIR_INTERLEAVED 0
#define YR_PAIR_HALF 1

/* Method parameters, named after the pages' rope_scaling config (type, factor,
 * original_max_position_embeddings) and the problem statement. */
typedef struct yr_rope_params {
    int head_dim;   /* d: even, 2 .. 128 for the table; the kernels take 64 or 128 */
    double base;    /* RoPE base, > 1 (10000 for Llama-2, 500000 for Llama-3) */
    int L_train;    /* original training context length (YaRN band split) */
    double scale;   /* s = L_target / L_train, >= 1 */
    int method;     /* YR_ROPE, YR_PI, YR_NTK or YR_YARN */
    double alpha;   /* YaRN ramp start, in rotations per L_train (pages: 1) */
    double beta;    /* YaRN ramp end (pages: 32); must exceed alpha */
    int L_cur;      /* YR_NTK_DYNAMIC: current sequence length (>= 1); else unused */
    const double *factors; /* YR_FACTORS: d/2 host doubles f_i > 0, read during the call */
    double attn_factor;    /* YR_FACTORS: mscale (attention temperature); <= 0 means 1 */
    int pairs;             /* YR_PAIR_INTERLEAVED (0, default) or YR_PAIR_HALF */
} yr_rope_params;

/* Frequency and temperature table, built on the host in double precision and
 * passed by value into the kernels. */
typedef struct yr_rope_table {
    int head_dim;
    int method;
    double inv_freq[YR_MAX_HEAD_DIM / 2]; /* theta'_i, radians per position */
    double turns[YR_MAX_HEAD_DIM / 2];    /* theta'_i / (2 pi): rotations per position */
    double mscale;                        /* 0.1 ln s + 1 for both YaRN forms, the caller's
                                             factor for YR_FACTORS, else 1 */
    double softmax_scale;                 /* mscale^2 / sqrt(d): the logit multiplier */
    uint64_t digest;                      /* FNV-1a of the parameters (position-config identity) */
    int pairs;                            /* YR_PAIR_INTERLEAVED or YR_PAIR_HALF: every kernel
                                             that rotates follows it */
} yr_rope_table;

/*
 * rope_freq_table -- fill `out` from `p` (host only; no CUDA).
 *   RoPE theta_i = base^(-2i/d) ("LLM context window mechanics", position wall;
 *   "Arch_03_Long_Context", RoPE slide).  PI theta_i / s (PI slide).  NTK
 *   (base s^(d/(d-2)))^(-2i/d) (NTK-aware slide).  YaRN: r_i = L_train theta_i /
 *   (2 pi), gamma_i = clamp((r_i - alpha)/(beta - alpha), 0, 1), theta'_i =
 *   gamma_i theta_i + (1 - gamma_i) theta_i / s, and mscale = 0.1 ln s + 1
 *   (YaRN slide and steps table).  softmax_scale = mscale^2 / sqrt(d).
 *   Dynamic NTK: NTK with s = max(1, L_cur / L_train) ("Arch_03_Long_Context",
 *   NTK-aware slide).  YaRN dimension ramp: i_edge(r) = d ln(L_train / (2 pi
 *   r)) / (2 ln base), low = floor(i_edge(beta)), high = ceil(i_edge(alpha)),
 *   gamma_i = 1 - clamp((i - low)/(high - low), 0, 1) ("LLM context window
 *   mechanics", the structure of its YaRN code).  Factors: theta'_i = theta_i /
 *   f_i and mscale = attn_factor (LongRoPE's per-dimension interpolation factors,
 *   "Long context (engineering 100k+ tokens)" and "long-context-models").
 *   ALiBi: every theta'_i = 0 (no rotation), mscale = 1; the attention entry
 *   points add the per-head linear bias when they see this method.
 *   pairs: copied into the table; the kernels rotate pairs (2i, 2i+1) or
 *   (i, i + d/2) accordingly (the q/k debug outputs and the rotated-key cache
 *   keep the caller's element order).
 *   The digest hashes the parameters, so a server can fold the position policy
 *   into its engine identity ("long-context-models", operational failure modes).
 * Errors: YR_EINVAL for NULL pointers, odd/out-of-range head_dim, base <= 1,
 *   scale < 1, unknown method, for either YaRN form L_train < 1 or beta <=
 *   alpha, for dynamic NTK L_train < 1 or L_cur < 1, for YR_FACTORS a NULL
 *   factors pointer or a factor that is not a positive finite number, and for a
 *   pairs value other than YR_PAIR_INTERLEAVED or YR_PAIR_HALF.
 */
int yr_rope_freq_table(const yr_rope_params *p, yr_rope_table *out);

/*
 * attn_prefill_workspace_bytes -- bytes of device workspace yr_attn_prefill
 * needs: the rotated keys and the values, each [B, Hkv, T, d] in fp16.
 * Returns 0 for invalid sizes.
 */
size_t yr_attn_prefill_workspace_bytes(int B, int Hkv, int T, int d);

/*
 * attn_prefill -- O = softmax(softmax_scale * (R_m q_m) . (R_n k_n)) V over the
 * visible keys n of every query m.
 *   Rotation R_p on each pair (2i, 2i+1) by p * theta'_i ("Arch_03_Long_Context",
 *   RoPE slide; "long-context-models", position enters attention).
 *   Visibility: n <= m when causal; with window W > 0 also (m - n < W or
 *   n < n_sink) ("Arch_03_Long_Context", sliding window and sink slides;
 *   "Long context (engineering 100k+ tokens)", sec. 5).  Query head h reads KV
 *   head h / (Hq / Hkv) (grouped-query attention).
 * Arguments (device pointers unless stated):
 *   q  bf16 [B, Hq, T, d]    strides q_strides[3] = {b, h, t} in elements
 *   k  bf16 [B, Hkv, T, d]   strides k_strides[3]
 *   v  bf16 [B, Hkv, T, d]   strides v_strides[3]
 *   o  bf16 [B, Hq, T, d]    strides o_strides[3]   (output)
 *   lse      fp32 [B, Hq, T] contiguous, natural-log sum of exp of the logits (nullable)
 *   k_cache  bf16 [B, Hkv, T, d] strides kc_strides[3]: receives the rotated keys,
 *            e.g. to seed a decode cache (nullable)
 *   q_rot_dbg fp32 [B, Hq, T, d] contiguous: the rotated queries as the kernel
 *            computed them, before rounding (nullable; for tests)
 *   k_rot_dbg fp32 [B, Hkv, T, d] contiguous: the same for the keys (nullable)
 *   A NULL strides pointer means contiguous.  d (the last dim) has unit stride;
 *   the other strides must be multiples of 8 elements and every base pointer
 *   16-byte aligned.
 *   tab: from yr_rope_freq_table with tab->head_dim == d.
 *   causal: 1 or 0; window (W) >= 0 with 0 = none; n_sink >= 0.  window > 0
 *   requires causal; n_sink > 0 requires window > 0.
 *   workspace: >= yr_attn_prefill_workspace_bytes(B, Hkv, T, d) bytes, 256-byte
 *   aligned.  It is overwritten; its contents after the call are unspecified.
 * Precision: inputs and outputs bf16; rotation angles reduced in fp64; rotated
 *   q/k, the probabilities and v enter the tensor cores as fp16; all sums fp32.
 *   |rotated q|, |rotated k| and |v| must stay below 65520, the fp16 range: a
 *   value outside it (or a NaN) sets the range bit of the device status word,
 *   which yr_device_status() then reports as YR_ERANGE; the output of such a
 *   call is unspecified.  The probabilities are kept within fp16 by the kernel.
 * Errors: YR_EINVAL (shapes, strides, alignment, flags, workspace too small),
 *   YR_EUNSUPPORTED (d not 64 or 128, device not sm_100), YR_ECUDA.
 */
int yr_attn_prefill(const void *q, const void *k, const void *v, void *o, float *lse,
                    void *k_cache, float *q_rot_dbg, float *k_rot_dbg,
                    int B, int Hq, int Hkv, int T, int d,
                    const int64_t *q_strides, const int64_t *k_strides,
                    const int64_t *v_strides, const int64_t *o_strides,
                    const int64_t *kc_strides,
                    const yr_rope_table *tab, int causal, int window, int n_sink,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * prefill_prepare_kv -- first half of yr_attn_prefill: rotate every key by its
 * position (k~_n = R_n k_n, "Arch_03_Long_Context", RoPE slide) and lay the
 * rotated keys and the values out in `workspace` as fp16 [B, Hkv, T, d].
 * Optionally also writes the rotated keys as bf16 to k_cache (caller strides)
 * and as fp32 to k_rot_dbg (contiguous).  Arguments, alignment and errors as in
 * yr_attn_prefill.  Useful on its own when several query blocks attend to the
 * same keys: prepare once, then call yr_prefill_attend per block.
 */
int yr_prefill_prepare_kv(const void *k, const void *v, void *k_cache, float *k_rot_dbg,
                          int B, int Hkv, int T, int d,
                          const int64_t *k_strides, const int64_t *v_strides,
                          const int64_t *kc_strides, const yr_rope_table *tab,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * prefill_attend -- second half of yr_attn_prefill: rotate the queries inside
 * the attention kernel and attend over the keys and values that
 * yr_prefill_prepare_kv left in `workspace` (which must have been prepared with
 * the same B, Hkv, T, d and table, on this stream or with the ordering made
 * explicit by the caller).  Arguments, alignment and errors as in
 * yr_attn_prefill; `workspace` is only read.
 */
int yr_prefill_attend(const void *q, void *o, float *lse, float *q_rot_dbg,
                      int B, int Hq, int Hkv, int T, int d,
                      const int64_t *q_strides, const int64_t *o_strides,
                      const yr_rope_table *tab, int causal, int window, int n_sink,
                      const void *workspace, size_t workspace_bytes, void *stream);

/*
 * attn_prefill_chunk -- prefill of a chunk of Tq new tokens per sequence after a
 * cached prefix ("LLM context window mechanics", deployment notes: cache prefix KV
 * pairs; "Long context (engineering 100k+ tokens)", sec. 6 prefix caching and its
 * exercise on chunked prefill).  The tokens sit at positions P0 .. P0+Tq-1: the
 * call rotates q and k_new at those positions, writes the rotated keys (bf16) and
 * v_new into cache slots P0 .. P0+Tq-1, and returns causal attention of each new
 * query over keys 0 .. its position, with the window/sink rule of yr_attn_prefill.
 * Slots 0 .. P0-1 are taken as already rotated.  With P0 = 0 it is a causal
 * yr_attn_prefill that also fills the cache; with Tq = 1 it is one decode step.
 * Arguments (device pointers, contiguous):
 *   q, o bf16 [B, Hq, Tq, d]; k_new, v_new bf16 [B, Hkv, Tq, d]
 *   k_cache, v_cache bf16 [B, Hkv, T_max, d], 0 <= P0 and P0 + Tq <= T_max
 *   lse fp32 [B, Hq, Tq] (nullable)
 *   workspace: >= yr_attn_prefill_workspace_bytes(B, Hkv, P0 + Tq, d) bytes,
 *     256-byte aligned; it receives fp16 copies of all P0 + Tq keys and values.
 * Errors: YR_EINVAL for NULL or misaligned pointers, sizes out of range, Hq not a
 *   multiple of Hkv, a window/sink combination yr_attn_prefill rejects, or a
 *   small workspace; YR_EUNSUPPORTED for d not 64/128 or a non-sm_100 device.
 */
int yr_attn_prefill_chunk(const void *q, const void *k_new, const void *v_new,
                          void *k_cache, void *v_cache, void *o, float *lse,
                          int B, int Hq, int Hkv, int Tq, int d, int P0, int T_max,
                          const yr_rope_table *tab, int window, int n_sink,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * attn_prefill_chunk_fp16cache -- yr_attn_prefill_chunk for a serving loop that
 * keeps, next to the bf16 cache, a second copy of it in the fp16 operand format
 * of the attention kernel, so that a call moves only its own Tq rows instead of
 * converting the whole cached prefix into a workspace ("Long context (engineering
 * 100k+ tokens)", sec. 6: prefix caching, chunked prefill).
 *   k_cache16, v_cache16: fp16 [B, Hkv, T_max, d], contiguous, 256-byte aligned,
 *     caller-owned.  Slots 0 .. cache16_len-1 must hold fp16 copies of the keys
 *     and values of those slots, as an earlier call of this function left them;
 *     the call converts slots cache16_len .. P0-1 from the bf16 caches, then
 *     writes the chunk's rotated keys and values into slots P0 .. P0+Tq-1 of both
 *     copies.  The keys it appends are their fp32 rotation rounded once to fp16
 *     in the copy and to bf16 in the cache (the precision yr_attn_prefill_chunk
 *     attends them with), so later chunks read them at fp16 precision.
 *     Afterwards slots 0 .. P0+Tq-1 of the fp16 copy are valid, so the next chunk
 *     passes cache16_len = P0 + Tq.  Slots a decode step appended to the bf16
 *     cache in between are picked up by passing the last valid length.
 *   0 <= cache16_len <= P0.
 *   workspace (nullable, 256-byte aligned): room for split-KV partials.  A short
 *     chunk after a long prefix has few (sequence, head, 256-row query block)
 *     items -- 32 for one 256-token chunk of a 32-head model -- too few for the
 *     GPU's SMs; with a workspace the call cuts each item's keys into up to 16
 *     shares run as separate CTAs, each leaving an fp32 partial output and its
 *     log-sum-exp, and merges them (the online-softmax combination of partial
 *     results, as in ring attention).  yr_attn_prefill_chunk_split_bytes() gives
 *     the bytes for the most shares; a smaller workspace limits the shares, NULL
 *     means none.  The result differs from the unsplit one only by fp32 rounding.
 *   Other arguments, results and errors as yr_attn_prefill_chunk.
 */
size_t yr_attn_prefill_chunk_split_bytes(int B, int Hq, int Tq, int d);
int yr_attn_prefill_chunk_fp16cache(const void *q, const void *k_new, const void *v_new,
                                    void *k_cache, void *v_cache, void *k_cache16,
                                    void *v_cache16, int cache16_len, void *o, float *lse,
                                    int B, int Hq, int Hkv, int Tq, int d, int P0, int T_max,
                                    const yr_rope_table *tab, int window, int n_sink,
                                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * prefill_prepare_kv_at -- yr_prefill_prepare_kv for a block of keys that starts at
 * absolute position k_pos0 (key t is rotated at k_pos0 + t): the step a worker of
 * ring attention / context parallelism ("long-context-models", section "Context
 * parallelism distributes exact attention"; "Long context (engineering 100k+
 * tokens)", sec. 3) runs once on its own slice of the sequence before the blocks
 * circulate.  With k_pos0 = 0 it is yr_prefill_prepare_kv.  Arguments, layout and
 * errors as there; YR_EINVAL also for k_pos0 < 0 or k_pos0 + T > 2^30.
 */
int yr_prefill_prepare_kv_at(const void *k, const void *v, void *k_cache, float *k_rot_dbg,
                             int B, int Hkv, int T, int d,
                             const int64_t *k_strides, const int64_t *v_strides,
                             const int64_t *kc_strides, const yr_rope_table *tab, int k_pos0,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * prefill_attend_block -- attention of T query rows at absolute positions
 * q_pos0 .. q_pos0+T-1 to the Tk keys and values of one block, at positions
 * k_pos0 .. k_pos0+Tk-1, that yr_prefill_prepare_kv_at(.., T = Tk, k_pos0, ..) left
 * in `workspace` (only read).  The queries are rotated at their absolute positions;
 * the causal, window and sink rules of yr_attn_prefill apply to absolute positions
 * (sinks are the first n_sink positions of the whole sequence).  o is the block's
 * own softmax-normalised output, kept in fp32 so that merging adds no rounding, and
 * lse (natural log, nullable) its log-sum-exp; a row with no visible key in the
 * block gets o = 0, lse = -inf.  yr_attn_merge folds such partials into the result.
 * Arguments: q bf16 [B, Hq, T, d] with optional strides as in yr_attn_prefill;
 *   o fp32 [B, Hq, T, d] contiguous; lse fp32 [B, Hq, T];
 *   workspace >= yr_attn_prefill_workspace_bytes(B, Hkv, Tk, d).
 * Errors: as yr_attn_prefill; YR_EINVAL also for Tk < 1, negative positions or
 *   positions past 2^30, and causal blocks with q_pos0 < k_pos0 (a block wholly
 *   in the future has no visible key: the caller skips it).
 */
int yr_prefill_attend_block(const void *q, float *o, float *lse,
                            int B, int Hq, int Hkv, int T, int Tk, int d,
                            const int64_t *q_strides,
                            const yr_rope_table *tab, int causal, int window, int n_sink,
                            int q_pos0, int k_pos0,
                            const void *workspace, size_t workspace_bytes, void *stream);

/*
 * attn_merge -- fold one block's partial attention (o_part, lse_part) into a
 * running result (o_acc, lse_acc) by their log-sum-exp weights, the online-softmax
 * combination of ring attention (sections above):
 *   L = log(e^lse_acc + e^lse_part),
 *   o_acc = e^(lse_acc - L) o_acc + e^(lse_part - L) o_part,  lse_acc = L,
 * row by row; rows where both lse are -inf are left alone, and a side whose lse is
 * -inf is not read.  init != 0 takes the
 * accumulator as empty without reading it (the first block: o_acc, lse_acc are
 * then just written); otherwise a row with lse_acc = -inf is empty and its o_acc
 * is not read.  If o_out is non-NULL it also receives the merged rows as bf16
 * (round to nearest even), e.g. on the last block.
 * Arguments (device pointers, contiguous, rows = B * Hq * T of the block call):
 *   o_part fp32 [rows, d]; lse_part fp32 [rows]; o_acc fp32 [rows, d];
 *   lse_acc fp32 [rows]; o_out bf16 [rows, d] (nullable).
 *   o pointers 16-byte aligned, lse pointers 4-byte aligned.
 * Errors: YR_EINVAL for NULL or misaligned pointers or rows < 1; YR_EUNSUPPORTED
 *   for d not 64/128 or a non-sm_100 device.
 */
int yr_attn_merge(const float *o_part, const float *lse_part, float *o_acc, float *lse_acc,
                  void *o_out, long long rows, int d, int init, void *stream);

/*
 * host_prefill -- prefill of prompts that live in host memory: q, k, v are read
 * from host buffers and o is written to a host buffer, with the copies inside the
 * call ("LLM context window mechanics", production lessons: a 128K prompt's first
 * request pays its whole prefill).  The work is cut into units of (sequence, group
 * of KV heads with their query heads); each unit's host-to-device copy, its
 * yr_attn_prefill (on `stream`) and its device-to-host copy run on three streams,
 * so the transfers of some units overlap the kernels of others, and a call's first
 * units overlap the previous call's last ones.
 *   A plan is made once per shape and reused:
 *   yr_host_prefill_workspace_bytes(B, Hq, Hkv, T, d, units_per_batch) -- device
 *     bytes the plan needs (q, k, v, o on the device plus a unit's prefill
 *     workspace); 0 for invalid sizes.  units_per_batch <= 0 means min(Hkv, 8).
 *   yr_host_prefill_create(&plan, B, Hq, Hkv, T, d, units_per_batch, workspace,
 *     workspace_bytes) -- workspace: caller-owned device memory of at least that
 *     many bytes, 256-byte aligned, kept for the plan's life.  The plan creates two
 *     streams and three events per unit on the current device (no device memory).
 *   yr_host_prefill_run(plan, q, k, v, o, tab, causal, window, n_sink, stream) --
 *     q, o: host [B, Hq, T, d] bf16; k, v: host [B, Hkv, T, d] bf16; contiguous.
 *     Page-locked (pinned) host memory lets the copies run asynchronously; with
 *     pageable memory they still work but do not overlap.  Asynchronous: work on
 *     `stream` after the call waits for the whole result; synchronise `stream`
 *     before reading o or changing q, k, v.  Other arguments and errors as
 *     yr_attn_prefill; YR_EINVAL also when called on another device than the
 *     plan's.  One host thread at a time per plan.
 *   yr_host_prefill_destroy(plan) -- waits for the plan's copies, frees its streams
 *     and events (NULL is accepted).
 */
typedef struct yr_host_prefill yr_host_prefill;
size_t yr_host_prefill_workspace_bytes(int B, int Hq, int Hkv, int T, int d,
                                       int units_per_batch);
int yr_host_prefill_create(yr_host_prefill **plan, int B, int Hq, int Hkv, int T, int d,
                           int units_per_batch, void *workspace, size_t workspace_bytes);
int yr_host_prefill_run(yr_host_prefill *plan, const void *q, const void *k, const void *v,
                        void *o, const yr_rope_table *tab, int causal, int window, int n_sink,
                        void *stream);
int yr_host_prefill_destroy(yr_host_prefill *plan);

/*
 * attn_decode_workspace_bytes -- bytes of device workspace yr_attn_decode needs
 * for its split-KV partial results with a cache of T_max slots.  0 if invalid.
 */
size_t yr_attn_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int T_max);

/*
 * attn_decode -- one new token per sequence, attending over its KV cache
 * ("Long Context" concept page: decode is memory-bound on the cache).
 *   The new token of sequence b sits at position L_b = cache_len[b]: the call
 *   rotates q_new and k_new by R_{L_b}, writes the rotated key and v_new into
 *   cache slot L_b, and returns attention of the rotated query over the keys
 *   0 .. L_b (slots 0 .. L_b-1 are taken as already rotated), with the
 *   window/sink rule of yr_attn_prefill taken at query position L_b.  It does
 *   not advance cache_len; the caller does.
 *   Split-KV: each (sequence, KV head, chunk of keys) yields a partial
 *   (max, sum, unnormalised output) for all Hq/Hkv query heads of the group;
 *   a second kernel merges them with log-sum-exp weights.
 * Arguments (device pointers, contiguous):
 *   q_new bf16 [B, Hq, d]; k_new, v_new bf16 [B, Hkv, d]
 *   k_cache, v_cache bf16 [B, Hkv, T_max, d] (slot L_b is written)
 *   cache_len int32 [B], each 0 <= L_b <= T_max - 1 (not checked on the host:
 *     the kernels skip a sequence whose length is out of range and record it
 *     in the device status word)
 *   o bf16 [B, Hq, d] (output); lse fp32 [B, Hq] (nullable)
 *   q_rot_dbg fp32 [B, Hq, d]: the rotated queries before rounding (nullable)
 *   tab: from yr_rope_freq_table with tab->head_dim == d.
 *   window >= 0 (0 = none), n_sink >= 0 (requires window > 0).
 *   workspace: >= yr_attn_decode_workspace_bytes(...) bytes, 256-byte aligned.
 * Errors: YR_EINVAL, YR_EUNSUPPORTED (d not 64 or 128, Hq/Hkv > 16, no sm_100),
 *   YR_ECUDA.
 */
int yr_attn_decode(const void *q_new, const void *k_new, const void *v_new,
                   void *k_cache, void *v_cache, const int32_t *cache_len,
                   void *o, float *lse, float *q_rot_dbg,
                   int B, int Hq, int Hkv, int d, int T_max,
                   const yr_rope_table *tab, int window, int n_sink,
                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * attn_decode_noalloc -- yr_attn_decode for callers that cannot allocate device
 * memory.  The pages have no counterpart: this is an interface for embedding.
 * Some callers cannot call cudaMalloc: a plugin inside a host application that
 * owns every byte of device memory and hands its plugins no scratch allocator,
 * or a latency-bound serving loop that may not allocate once it is running
 * (cudaMalloc can synchronise the device).  This entry point allocates nothing:
 * the caller still passes inputs, caches and outputs, and the split-KV partial
 * results go to a fixed scratch array inside the library instead of a workspace.
 *   Limit: the scratch is YR_DECODE_NOALLOC_SCRATCH_BYTES (16 MiB) per device,
 *   held by every GPU that loads the library until the process exits.  A call
 *   that needs more -- yr_attn_decode_workspace_bytes(B, Hq, Hkv, d, T_max)
 *   bytes -- returns YR_EINVAL without launching anything (e.g. 16 sequences of
 *   32768 slots with 128 query and 8 KV heads of d=128 need just over 16 MiB).
 *   The scratch is per CUDA context: each device's primary context, and any
 *   context the host application makes current, has its own copy.  The first
 *   call in each context looks up the scratch address in that context with the
 *   CUDA runtime; make that first call before any stream capture.
 *   Every call shares the one array, which keeps the last call's contents: calls
 *   that overlap on the GPU (other streams, other host threads) race on it, so
 *   order them.  Nothing in it needs to start at zero, because each call writes
 *   every partial result it reads back.
 * Other arguments, results and errors as yr_attn_decode.
 */
#define YR_DECODE_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
int yr_attn_decode_noalloc(const void *q_new, const void *k_new, const void *v_new,
                           void *k_cache, void *v_cache, const int32_t *cache_len,
                           void *o, float *lse, float *q_rot_dbg,
                           int B, int Hq, int Hkv, int d, int T_max,
                           const yr_rope_table *tab, int window, int n_sink, void *stream);

/*
 * device_status -- synchronise `stream`, then read and clear the device status
 * word of the current device.  Returns YR_OK, YR_ETIMEOUT (a kernel gave up on
 * a wait; yr_last_error names where), YR_ERANGE (a prefill, chunk or block call
 * met a rotated query or key, or a value, outside the fp16 range), YR_EINVAL (a
 * decode cache length was out of range), or YR_ECUDA.  When several bits are
 * set the first of those codes is returned and the message names them all.
 */
int yr_device_status(void *stream);

/* Message for the last error on the calling thread ("" if none). */
const char *yr_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int yr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* YARNATTN_H */
