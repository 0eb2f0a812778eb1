/*
 * yarn_oracle.c -- plain fp64 CPU oracle for YaRN-RoPE causal GQA attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline of the benchmark may load this library.  It shares no code with
 * the CUDA path and is deliberately slow: every quantity is computed straight
 * from its definition in double precision, with no tiling, no fusion and no
 * online softmax.
 *
 * Sources (the web pages on long-context position scaling):
 *   [P1] "LLM context window mechanics" -- sections "The memory wall,
 *        quantified" and "The position wall: RoPE and interpolation".
 *   [P2] "Long Context" concept page -- "Key math / How it works".
 *   [P3] "Arch_03_Long_Context" slide deck -- the RoPE, Position
 *        Interpolation, NTK-aware, YaRN, sliding-window and sink slides.
 *   [P4] "Long context (engineering 100k+ tokens)" -- section 2 (RoPE
 *        scaling tricks) and section 5 (attention sinks).
 *   [P5] "long-context-models" -- "Position enters attention" and
 *        "Memory grows even with efficient attention".
 *
 * Readings taken where the pages are silent, garbled or disagree (each is
 * also listed with its reason in the design notes of the repository):
 *   - YaRN band split follows [P3] YaRN slide + the steps table (alpha=1,
 *     beta=32), with the ramp linear in r = L_train / lambda_i; [P1]'s
 *     printed code is garbled and is not followed.
 *   - The temperature multiplies the logits by (0.1 ln s + 1)^2 / sqrt(d)
 *     (equivalently mscale on both rotated q and k).
 *   - Pairs are interleaved (2i, 2i+1) as on the [P3] RoPE slide; every
 *     rotating function also takes the half-split layout (i, i + d/2), the
 *     common alternative the pages do not print (a `pairs` argument, 1 = half).
 *   - Window: key n is visible to query m iff n <= m (causal) and
 *     (m - n < W or n < n_sink); positions are absolute.
 *   - GQA: query head h reads KV head floor(h / (Hq/Hkv)).
 *
 * Parity status per function:
 *   oracle_rope_theta   pinned (closed forms, s=1 reductions, NTK worked
 *                       number, band endpoints).  The YaRN ramp interior is
 *                       a reading of the pages (they print no value inside
 *                       it); the oracle's ramp is pinned to that reading's
 *                       closed form at constructed points (a base that puts a
 *                       pair at r = alpha + f (beta - alpha) must give
 *                       f theta + (1 - f) theta / s).
 *   oracle_rope_theta_ext  dynamic NTK pinned (RoPE at or below L_train, equal
 *                       to NTK at L_cur = s L_train, the page's ~82,000 base);
 *                       dimension-ramp YaRN pinned outside its ramp and at the
 *                       ramp's midpoint (a linear ramp's closed form), its
 *                       edges pinned against the r-space band edges; factors
 *                       pinned by f = 1 (RoPE), f = s (PI) and f = theta /
 *                       theta'(YaRN) (YaRN's frequencies).
 *   oracle_rotate_rows  pinned (page's rotation matrix, complex-number
 *                       form, orthogonality, relative-position invariance);
 *                       the half-split layout pinned by its own complex form
 *                       (z_i = x_i + i x_{i+d/2}), by equality with the
 *                       interleaved rotation of the permuted vector, and by
 *                       relative-position invariance.
 *   oracle_attn_rows    pinned (library SDPA special case, closed-form
 *                       means, page's "4 + last 4096" sink count, T=1).
 *   oracle_attn_rotated_f64 pinned (equals oracle_attn_rows on its own
 *                       rotation of bf16 inputs; library SDPA on operands that
 *                       are not bf16 values; closed-form means for q = 0).
 *   oracle_decode       pinned (equals the prefill row at the same position).
 *   oracle_prefill_chunk pinned (Tq = 1 is decode; P0 = 0 is the full
 *                       prefill; torch float64 SDPA on the assembled keys).
 *   ALiBi (slopes argument of the three attention functions, and
 *   oracle_alibi_slopes) pinned: the page's geometric series, torch float64
 *   SDPA with the additive bias, zero slopes give plain attention, and the
 *   output is invariant to a common shift of all positions.
 *   oracle_kv_cache_bytes pinned (the pages' ~69 GB / ~17 GB / 40 GiB).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_ROPE 0
#define OR_PI 1
#define OR_NTK 2
#define OR_YARN 3
#define OR_NTK_DYNAMIC 4
#define OR_YARN_DIMRAMP 5
#define OR_FACTORS 6

static double bf16_bits_to_double(uint16_t bits)
{
    /* bf16 is the upper half of an IEEE binary32: widening is exact. */
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Per-pair rotation frequencies theta'_i (i = 0 .. d/2-1), the attention
 * temperature mscale and the softmax logit scale.
 *   RoPE  theta_i = base^(-2i/d)                       [P1] position wall; [P3] RoPE slide
 *   PI    theta'_i = theta_i / s                        [P1]; [P3] PI slide (angles of m/s); [P4] sec. 2
 *   NTK   theta'_i = (base * s^(d/(d-2)))^(-2i/d)       [P3] NTK-aware slide
 *   YaRN  r_i = L_train * theta_i / (2 pi) = L_train / lambda_i   ([P3] YaRN slide: lambda_i = 2 pi / theta_i)
 *         gamma_i = clamp((r_i - alpha) / (beta - alpha), 0, 1)
 *         theta'_i = gamma_i * theta_i + (1 - gamma_i) * theta_i / s
 *         (short wavelengths unchanged, long wavelengths interpolated as PI,
 *          linear ramp between; alpha = 1, beta = 32 per the steps table)
 *   Dynamic NTK  NTK with s = max(1, L_cur / L_train), the current sequence
 *         length over the training length            [P3] NTK-aware slide, last sentence
 *   YaRN, dimension ramp  the same band split with the ramp linear in the pair
 *         index: i_edge(r) = d ln(L_train / (2 pi r)) / (2 ln base) is the
 *         (fractional) index where r_i = r; low = floor(i_edge(beta)),
 *         high = ceil(i_edge(alpha)); gamma_i = 1 - clamp((i - low) / (high - low), 0, 1)
 *         ([P1]'s code structure: band-edge indices from a log ratio, floor
 *          and ceil, a linear ramp over the index)
 *   Per-dimension factors  theta'_i = theta_i / f_i for caller-supplied f_i > 0
 *         ([P4] LongRoPE: searched non-uniform interpolation factors per
 *          dimension; [P5] LongRoPE); mscale = the caller's attention factor,
 *         1 when none is given
 *   mscale = 0.1 ln s + 1 for both YaRN forms, else 1  [P1] position wall; [P3] YaRN slide
 *   softmax_scale = mscale^2 / sqrt(d)
 * Returns 0, or -1 for an invalid argument (odd or non-positive d, s < 1,
 * base <= 1, beta <= alpha or L_train < 1 for the YaRN forms and dynamic NTK,
 * L_cur < 1 for dynamic NTK, missing or non-positive factors).
 */
int oracle_rope_theta_ext(int d, double base, int L_train, double s, int method,
                          double alpha, double beta, int L_cur, const double *factors,
                          double attn_factor, double *theta, double *mscale,
                          double *softmax_scale)
{
    if (d <= 0 || (d % 2) != 0) return -1;
    if (!(s >= 1.0) || !(base > 1.0)) return -1;
    if (method < OR_ROPE || method > OR_FACTORS) return -1;
    const int yarn = method == OR_YARN || method == OR_YARN_DIMRAMP;
    if (yarn && (!(beta > alpha) || L_train < 1)) return -1;
    if (method == OR_NTK_DYNAMIC && (L_train < 1 || L_cur < 1)) return -1;
    const int half = d / 2;
    if (method == OR_FACTORS) {
        if (factors == NULL) return -1;
        for (int i = 0; i < half; ++i)
            if (!(factors[i] > 0.0)) return -1;
    }
    /* Band-edge indices of the dimension ramp. */
    double low = 0.0, high = 1.0;
    if (method == OR_YARN_DIMRAMP) {
        const double i_beta = (double)d * log((double)L_train / (2.0 * M_PI * beta)) / (2.0 * log(base));
        const double i_alpha = (double)d * log((double)L_train / (2.0 * M_PI * alpha)) / (2.0 * log(base));
        low = floor(i_beta);
        high = ceil(i_alpha);
        if (low < 0.0) low = 0.0;
        if (high > (double)(half - 1)) high = (double)(half - 1);
        if (!(high > low)) high = low + 1.0;
    }
    const double s_dyn = (method == OR_NTK_DYNAMIC && (double)L_cur > (double)L_train)
                             ? (double)L_cur / (double)L_train
                             : 1.0;
    for (int i = 0; i < half; ++i) {
        const double expo = -2.0 * (double)i / (double)d;
        const double th = pow(base, expo);
        double out = th;
        if (method == OR_PI) {
            out = th / s;
        } else if (method == OR_NTK) {
            const double base_ntk = base * pow(s, (double)d / (double)(d - 2));
            out = pow(base_ntk, expo);
        } else if (method == OR_NTK_DYNAMIC) {
            const double base_ntk = base * pow(s_dyn, (double)d / (double)(d - 2));
            out = pow(base_ntk, expo);
        } else if (method == OR_YARN) {
            const double r = (double)L_train * th / (2.0 * M_PI);
            double g = (r - alpha) / (beta - alpha);
            if (g < 0.0) g = 0.0;
            if (g > 1.0) g = 1.0;
            out = g * th + (1.0 - g) * th / s;
        } else if (method == OR_YARN_DIMRAMP) {
            double ramp = ((double)i - low) / (high - low);
            if (ramp < 0.0) ramp = 0.0;
            if (ramp > 1.0) ramp = 1.0;
            const double g = 1.0 - ramp;
            out = g * th + (1.0 - g) * th / s;
        } else if (method == OR_FACTORS) {
            out = th / factors[i];
        }
        theta[i] = out;
    }
    double m = 1.0;
    if (yarn) m = 0.1 * log(s) + 1.0;
    if (method == OR_FACTORS && attn_factor > 0.0) m = attn_factor;
    if (mscale) *mscale = m;
    if (softmax_scale) *softmax_scale = m * m / sqrt((double)d);
    return 0;
}

/* The four fixed-table methods (RoPE, PI, NTK, YaRN). */
int oracle_rope_theta(int d, double base, int L_train, double s, int method,
                      double alpha, double beta, double *theta,
                      double *mscale, double *softmax_scale)
{
    if (method < OR_ROPE || method > OR_YARN) return -1;
    return oracle_rope_theta_ext(d, base, L_train, s, method, alpha, beta, 0, NULL, 0.0,
                                 theta, mscale, softmax_scale);
}

/*
 * Rotate one d-vector x at (possibly fractional) position p.  Pair i turns by
 * the angle p theta_i:
 *   [y_a]   [cos(p theta_i)  -sin(p theta_i)] [x_a]
 *   [y_b] = [sin(p theta_i)   cos(p theta_i)] [x_b]
 * with (a, b) = (2i, 2i+1) for interleaved pairs (pairs = 0, [P3] RoPE slide:
 * R_m,i on pair (2i, 2i+1); [P5] "Position enters attention"), or
 * (a, b) = (i, i + d/2) for the half-split layout (pairs = 1: the first half of
 * the vector holds the first element of every pair, the second half the second
 * element; the same rotation, another assignment of elements to pairs).
 */
static void rotate_vec(const double *x, double p, const double *theta, int d, int pairs,
                       double *y)
{
    for (int i = 0; i < d / 2; ++i) {
        const double phi = p * theta[i];
        const double c = cos(phi), sn = sin(phi);
        const int ia = pairs ? i : 2 * i;
        const int ib = pairs ? i + d / 2 : 2 * i + 1;
        const double a = x[ia], b = x[ib];
        y[ia] = a * c - b * sn;
        y[ib] = a * sn + b * c;
    }
}

/* Rotate n rows of bf16 bits (row stride d) at positions pos[r]. */
void oracle_rotate_rows(const uint16_t *x, long n, int d, const double *pos,
                        const double *theta, int pairs, double *out)
{
#pragma omp parallel
    {
        double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
        for (long r = 0; r < n; ++r) {
            for (int j = 0; j < d; ++j) tmp[j] = bf16_bits_to_double(x[r * d + j]);
            rotate_vec(tmp, pos[r], theta, d, pairs, out + r * d);
        }
        free(tmp);
    }
}

/* Same, for rows already in double precision. */
void oracle_rotate_rows_f64(const double *x, long n, int d, const double *pos,
                            const double *theta, int pairs, double *out)
{
    for (long r = 0; r < n; ++r) rotate_vec(x + r * d, pos[r], theta, d, pairs, out + r * d);
}

/*
 * Key n is visible to query m:
 *   causal: n <= m  ([P3] ALiBi slide "only attend to past")
 *   window W > 0: additionally m - n < W, or n < n_sink
 *   ([P3] sliding-window and StreamingLLM slides; [P4] sec. 5
 *    "always keep the first K tokens and the last W")
 */
/*
 * ALiBi slopes for H heads: one slope per head, falling geometrically from
 * 2^(-8/H) by a factor 2^(-8/H) per head ([P3] ALiBi slide), i.e.
 * m_h = 2^(-8 (h+1) / H).  ALiBi adds
 * -m_h * (i - j) to the scaled logit of query position i and key position j
 * and rotates nothing.
 */
void oracle_alibi_slopes(int H, double *m)
{
    for (int h = 0; h < H; ++h) m[h] = pow(2.0, -8.0 * (double)(h + 1) / (double)H);
}

static int visible(long m, long n, int causal, int window, int n_sink)
{
    if (causal && n > m) return 0;
    if (window > 0 && !((m - n) < (long)window || n < (long)n_sink)) return 0;
    return 1;
}

/*
 * Exact attention for a list of query rows.
 *   q [B,Hq,T,d], k and v [B,Hkv,T,d]: contiguous bf16 bit patterns.
 *   rows: n_rows flat indices (b*Hq + h)*T + m, or NULL for every row.
 *   For each row: q~ = R_m q, k~_n = R_n k_n, s_n = softmax_scale * q~.k~_n
 *   over visible n, P = exp(s - max) / sum, O = sum_n P_n v_n,
 *   LSE = max + ln(sum).   ([P3] "Q K^T / sqrt(d_k)" table slide; [P2]
 *   key math; [P5] memory section: exact self-attention.)
 *   o [n_rows, d], lse [n_rows] (nullable), q_rot [n_rows, d] (nullable).
 * Returns 0, -1 on bad arguments, -2 on allocation failure.
 */
int oracle_attn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     int B, int Hq, int Hkv, int T, int d,
                     const double *theta, double softmax_scale,
                     int causal, int window, int n_sink,
                     const int64_t *rows, long n_rows,
                     double *o, double *lse, double *q_rot, const double *slopes, int pairs)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || d < 2 || (d % 2) || (Hq % Hkv)) return -1;
    const int group = Hq / Hkv;
    const long total = (long)B * Hq * T;
    if (rows == NULL) n_rows = total;

    /* Which (b, kv head) pairs are needed and up to which key. */
    const long n_kv = (long)B * Hkv;
    long *need = (long *)calloc((size_t)n_kv, sizeof(long));
    if (!need) return -2;
    for (long r = 0; r < n_rows; ++r) {
        const long flat = rows ? (long)rows[r] : r;
        if (flat < 0 || flat >= total) { free(need); return -1; }
        const long m = flat % T, bh = flat / T;
        const long b = bh / Hq, h = bh % Hq;
        const long kv = b * Hkv + h / group;
        const long last = causal ? m + 1 : T;
        if (last > need[kv]) need[kv] = last;
    }
    /* Rotated keys k~_n = R_n k_n for the needed prefixes. */
    double **krot = (double **)calloc((size_t)n_kv, sizeof(double *));
    if (!krot) { free(need); return -2; }
    int fail = 0;
    for (long kv = 0; kv < n_kv; ++kv) {
        if (need[kv] == 0) continue;
        krot[kv] = (double *)malloc(sizeof(double) * (size_t)need[kv] * d);
        if (!krot[kv]) { fail = 1; break; }
    }
    if (fail) {
        for (long kv = 0; kv < n_kv; ++kv) free(krot[kv]);
        free(krot); free(need);
        return -2;
    }
    for (long kv = 0; kv < n_kv; ++kv) {
        const long cnt = need[kv];
        if (!cnt) continue;
        const uint16_t *kb = k + kv * (long)T * d;
        double *dst = krot[kv];
#pragma omp parallel
        {
            double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
            for (long n = 0; n < cnt; ++n) {
                for (int j = 0; j < d; ++j) tmp[j] = bf16_bits_to_double(kb[n * d + j]);
                rotate_vec(tmp, (double)n, theta, d, pairs, dst + n * d);
            }
            free(tmp);
        }
    }

#pragma omp parallel
    {
        double *qv = (double *)malloc(sizeof(double) * (size_t)d);
        double *qr = (double *)malloc(sizeof(double) * (size_t)d);
        double *sc = (double *)malloc(sizeof(double) * (size_t)T);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < n_rows; ++r) {
            const long flat = rows ? (long)rows[r] : r;
            const long m = flat % T, bh = flat / T;
            const long b = bh / Hq, h = bh % Hq;
            const long kv = b * Hkv + h / group;
            const uint16_t *qrow = q + flat * d;
            for (int j = 0; j < d; ++j) qv[j] = bf16_bits_to_double(qrow[j]);
            rotate_vec(qv, (double)m, theta, d, pairs, qr);
            if (q_rot) memcpy(q_rot + r * d, qr, sizeof(double) * (size_t)d);
            const long kmax = causal ? m + 1 : T;
            const double *kr = krot[kv];
            const uint16_t *vb = v + kv * (long)T * d;
            double mx = -INFINITY;
            for (long n = 0; n < kmax; ++n) {
                if (!visible(m, n, causal, window, n_sink)) { sc[n] = -INFINITY; continue; }
                double dot = 0.0;
                for (int j = 0; j < d; ++j) dot += qr[j] * kr[n * d + j];
                sc[n] = softmax_scale * dot;
                if (slopes) sc[n] -= slopes[h] * (double)(m - n);
                if (sc[n] > mx) mx = sc[n];
            }
            double z = 0.0;
            for (int j = 0; j < d; ++j) acc[j] = 0.0;
            for (long n = 0; n < kmax; ++n) {
                if (sc[n] == -INFINITY) continue;
                const double p = exp(sc[n] - mx);
                z += p;
                for (int j = 0; j < d; ++j) acc[j] += p * bf16_bits_to_double(vb[n * d + j]);
            }
            for (int j = 0; j < d; ++j) o[r * d + j] = acc[j] / z;
            if (lse) lse[r] = mx + log(z);
        }
        free(qv); free(qr); free(sc); free(acc);
    }
    for (long kv = 0; kv < n_kv; ++kv) free(krot[kv]);
    free(krot);
    free(need);
    return 0;
}

/*
 * Exact attention on operands given in double precision, the queries and keys
 * already rotated: the definition of oracle_attn_rows without its rotation step.
 *   q_rot [B,Hq,T,d], k_rot [B,Hkv,T,d], v [B,Hkv,T,d], contiguous doubles.
 *   For each row: s_n = softmax_scale * q_rot_m . k_rot_n (minus slopes[h] (m - n)
 *   when slopes is given) over visible n, P = exp(s - max) / sum, O = sum_n P_n v_n,
 *   LSE = max + ln(sum).  ([P3] "Q K^T / sqrt(d_k)" table slide; [P2] key math.)
 * With the oracle's own rotation of bf16 inputs it is oracle_attn_rows; with
 * operands rounded in a stated way first (a test's choice) it gives exact
 * attention of those rounded operands.
 *   rows: n_rows flat indices (b*Hq + h)*T + m, or NULL for every row.
 * Returns 0, -1 on bad arguments, -2 on allocation failure.
 */
int oracle_attn_rotated_f64(const double *q_rot, const double *k_rot, const double *v,
                            int B, int Hq, int Hkv, int T, int d, double softmax_scale,
                            int causal, int window, int n_sink,
                            const int64_t *rows, long n_rows,
                            double *o, double *lse, const double *slopes)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || d < 1 || (Hq % Hkv)) return -1;
    const int group = Hq / Hkv;
    const long total = (long)B * Hq * T;
    if (rows == NULL) n_rows = total;
    for (long r = 0; r < n_rows; ++r) {
        const long flat = rows ? (long)rows[r] : r;
        if (flat < 0 || flat >= total) return -1;
    }
    int fail = 0;
#pragma omp parallel
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)T);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        if (!sc || !acc) {
#pragma omp atomic write
            fail = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < n_rows; ++r) {
            if (!sc || !acc) continue;
            const long flat = rows ? (long)rows[r] : r;
            const long m = flat % T, bh = flat / T;
            const long b = bh / Hq, h = bh % Hq;
            const long kv = b * Hkv + h / group;
            const double *qr = q_rot + flat * d;
            const double *kr = k_rot + kv * (long)T * d;
            const double *vb = v + kv * (long)T * d;
            double mx = -INFINITY;
            for (long n = 0; n < T; ++n) {
                if (!visible(m, n, causal, window, n_sink)) { sc[n] = -INFINITY; continue; }
                double dot = 0.0;
                for (int j = 0; j < d; ++j) dot += qr[j] * kr[n * d + j];
                sc[n] = softmax_scale * dot;
                if (slopes) sc[n] -= slopes[h] * (double)(m - n);
                if (sc[n] > mx) mx = sc[n];
            }
            double z = 0.0;
            for (int j = 0; j < d; ++j) acc[j] = 0.0;
            for (long n = 0; n < T; ++n) {
                if (sc[n] == -INFINITY) continue;
                const double p = exp(sc[n] - mx);
                z += p;
                for (int j = 0; j < d; ++j) acc[j] += p * vb[n * d + j];
            }
            for (int j = 0; j < d; ++j) o[r * d + j] = acc[j] / z;
            if (lse) lse[r] = mx + log(z);
        }
        free(sc);
        free(acc);
    }
    return fail ? -2 : 0;
}

/*
 * Single-token decode over a KV cache.
 *   q_new [B,Hq,d]; k_new, v_new [B,Hkv,d]; caches [B,Hkv,T_max,d] whose
 *   slots 0 .. L_b-1 hold keys that are already rotated (and values).
 *   The new token sits at position L_b = cache_len[b]: q~ = R_L q_new,
 *   k~ = R_L k_new; it attends over the L_b cached keys plus the new one,
 *   with the visibility rule above taken at query position L_b.
 *   ([P2] "decode is memory-bound on the cache"; [P1] memory wall.)
 *   o [B,Hq,d]; lse [B,Hq]; k_rot_new [B,Hkv,d] and q_rot_new [B,Hq,d]
 *   are nullable.  Returns 0, -1 on bad arguments, -2 on allocation failure.
 */
int oracle_decode(const uint16_t *q_new, const uint16_t *k_new, const uint16_t *v_new,
                  const uint16_t *k_cache, const uint16_t *v_cache, int T_max,
                  const int32_t *cache_len, int B, int Hq, int Hkv, int d,
                  const double *theta, double softmax_scale, int window, int n_sink,
                  double *o, double *lse, double *k_rot_new, double *q_rot_new,
                  const double *slopes, int pairs)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || d < 2 || (d % 2) || (Hq % Hkv) || T_max < 1) return -1;
    for (int b = 0; b < B; ++b)
        if (cache_len[b] < 0 || cache_len[b] + 1 > T_max) return -1;
    const int group = Hq / Hkv;
    int bad = 0;
#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)d);
        double *qr = (double *)malloc(sizeof(double) * (size_t)d);
        double *kn = (double *)malloc(sizeof(double) * (size_t)d);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        double *sc = (double *)malloc(sizeof(double) * ((size_t)T_max + 1));
        if (!x || !qr || !kn || !acc || !sc) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for collapse(2) schedule(dynamic, 1)
        for (int b = 0; b < B; ++b) {
            for (int h = 0; h < Hq; ++h) {
                if (bad) continue;
                const long L = cache_len[b];
                const int kv = h / group;
                const long qi = (long)b * Hq + h, ki = (long)b * Hkv + kv;
                for (int j = 0; j < d; ++j) x[j] = bf16_bits_to_double(q_new[qi * d + j]);
                rotate_vec(x, (double)L, theta, d, pairs, qr);
                if (q_rot_new) memcpy(q_rot_new + qi * d, qr, sizeof(double) * (size_t)d);
                for (int j = 0; j < d; ++j) x[j] = bf16_bits_to_double(k_new[ki * d + j]);
                rotate_vec(x, (double)L, theta, d, pairs, kn);
                if (k_rot_new && (h % group) == 0) memcpy(k_rot_new + ki * d, kn, sizeof(double) * (size_t)d);
                const uint16_t *kc = k_cache + ki * (long)T_max * d;
                const uint16_t *vc = v_cache + ki * (long)T_max * d;
                double mx = -INFINITY;
                for (long n = 0; n <= L; ++n) {
                    if (!visible(L, n, 1, window, n_sink)) { sc[n] = -INFINITY; continue; }
                    double dot = 0.0;
                    if (n < L)
                        for (int j = 0; j < d; ++j) dot += qr[j] * bf16_bits_to_double(kc[n * d + j]);
                    else
                        for (int j = 0; j < d; ++j) dot += qr[j] * kn[j];
                    sc[n] = softmax_scale * dot;
                    if (slopes) sc[n] -= slopes[h] * (double)(L - n);
                    if (sc[n] > mx) mx = sc[n];
                }
                double z = 0.0;
                for (int j = 0; j < d; ++j) acc[j] = 0.0;
                for (long n = 0; n <= L; ++n) {
                    if (sc[n] == -INFINITY) continue;
                    const double p = exp(sc[n] - mx);
                    z += p;
                    if (n < L)
                        for (int j = 0; j < d; ++j) acc[j] += p * bf16_bits_to_double(vc[n * d + j]);
                    else
                        for (int j = 0; j < d; ++j) acc[j] += p * bf16_bits_to_double(v_new[ki * d + j]);
                }
                for (int j = 0; j < d; ++j) o[qi * d + j] = acc[j] / z;
                if (lse) lse[qi] = mx + log(z);
            }
        }
        free(x); free(qr); free(kn); free(acc); free(sc);
    }
    return bad ? -2 : 0;
}

/*
 * Prefill of a chunk against a rotated cache prefix: the Tq new tokens of each
 * sequence sit at positions P0 .. P0+Tq-1 ([P1] deployment notes: cache
 * prefix KV pairs; [P4] sec. 6 prefix caching and its exercise on chunked
 * prefill).  Cache slots 0 .. P0-1 hold keys that were rotated when they were
 * written, and their values (bf16, used as given, as decode reads them); the
 * chunk's keys are rotated at their positions.  Query i (position P0 + i) sees
 * key n iff n <= P0 + i and (window == 0 or P0 + i - n < window or n < n_sink).
 *   q      bf16 [B][Hq][Tq][d]        k_new, v_new  bf16 [B][Hkv][Tq][d]
 *   cache  bf16 [B][Hkv][T_max][d]    (P0 + Tq <= T_max)
 *   o      [B][Hq][Tq][d], lse [B][Hq][Tq] (natural log), k_rot_new [B][Hkv][Tq][d]
 * Returns 0, -1 for invalid arguments, -2 when out of memory.
 */
int oracle_prefill_chunk(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                         const uint16_t *k_cache, const uint16_t *v_cache, int T_max, int P0,
                         int B, int Hq, int Hkv, int Tq, int d,
                         const double *theta, double softmax_scale, int window, int n_sink,
                         double *o, double *lse, double *k_rot_new, const double *slopes,
                         int pairs)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Tq < 1 || d < 2 || (d % 2) || (Hq % Hkv)) return -1;
    if (P0 < 0 || (long)P0 + Tq > (long)T_max) return -1;
    const int group = Hq / Hkv;
    const long n_kv = (long)B * Hkv;
    /* The chunk's rotated keys, k~_{P0+i} = R_{P0+i} k_i. */
    double *krot = (double *)malloc(sizeof(double) * (size_t)n_kv * Tq * d);
    if (!krot) return -2;
#pragma omp parallel
    {
        double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for collapse(2) schedule(static)
        for (long kv = 0; kv < n_kv; ++kv) {
            for (long i = 0; i < Tq; ++i) {
                const uint16_t *src = k_new + (kv * Tq + i) * d;
                for (int j = 0; j < d; ++j) tmp[j] = bf16_bits_to_double(src[j]);
                rotate_vec(tmp, (double)(P0 + i), theta, d, pairs, krot + (kv * Tq + i) * d);
            }
        }
        free(tmp);
    }
    if (k_rot_new) memcpy(k_rot_new, krot, sizeof(double) * (size_t)n_kv * Tq * d);
    const long Tk = (long)P0 + Tq;
    int bad = 0;
#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)d);
        double *qr = (double *)malloc(sizeof(double) * (size_t)d);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        double *sc = (double *)malloc(sizeof(double) * (size_t)Tk);
        if (!x || !qr || !acc || !sc) {
#pragma omp atomic write
            bad = 1;
        }
#pragma omp for collapse(3) schedule(dynamic, 4)
        for (int b = 0; b < B; ++b) {
            for (int h = 0; h < Hq; ++h) {
                for (long i = 0; i < Tq; ++i) {
                    if (bad) continue;
                    const long m = (long)P0 + i;
                    const long kv = (long)b * Hkv + h / group;
                    const long qi = ((long)b * Hq + h) * Tq + i;
                    for (int j = 0; j < d; ++j) x[j] = bf16_bits_to_double(q[qi * d + j]);
                    rotate_vec(x, (double)m, theta, d, pairs, qr);
                    const uint16_t *kc = k_cache + kv * (long)T_max * d;
                    const uint16_t *vc = v_cache + kv * (long)T_max * d;
                    const double *kn = krot + kv * (long)Tq * d;
                    const uint16_t *vn = v_new + kv * (long)Tq * d;
                    double mx = -INFINITY;
                    for (long n = 0; n <= m; ++n) {
                        if (!visible(m, n, 1, window, n_sink)) { sc[n] = -INFINITY; continue; }
                        double dot = 0.0;
                        if (n < P0)
                            for (int j = 0; j < d; ++j) dot += qr[j] * bf16_bits_to_double(kc[n * d + j]);
                        else
                            for (int j = 0; j < d; ++j) dot += qr[j] * kn[(n - P0) * d + j];
                        sc[n] = softmax_scale * dot;
                        if (slopes) sc[n] -= slopes[h] * (double)(m - n);
                        if (sc[n] > mx) mx = sc[n];
                    }
                    double z = 0.0;
                    for (int j = 0; j < d; ++j) acc[j] = 0.0;
                    for (long n = 0; n <= m; ++n) {
                        if (sc[n] == -INFINITY) continue;
                        const double p = exp(sc[n] - mx);
                        z += p;
                        if (n < P0)
                            for (int j = 0; j < d; ++j) acc[j] += p * bf16_bits_to_double(vc[n * d + j]);
                        else
                            for (int j = 0; j < d; ++j) acc[j] += p * bf16_bits_to_double(vn[(n - P0) * d + j]);
                    }
                    for (int j = 0; j < d; ++j) o[qi * d + j] = acc[j] / z;
                    if (lse) lse[qi] = mx + log(z);
                }
            }
        }
        free(x); free(qr); free(acc); free(sc);
    }
    free(krot);
    return bad ? -2 : 0;
}

/*
 * KV-cache bytes = 2 * n_layers * n_kv_heads * head_dim * seq_len * batch *
 * dtype_bytes  ([P1] memory wall, kv_cache_gb; [P2] key math 2 L n_kv d_h s b p;
 * [P5] M_KV = 2 L S H_kv D B).
 */
double oracle_kv_cache_bytes(double n_layers, double n_kv_heads, double head_dim,
                             double seq_len, double batch, double dtype_bytes)
{
    return 2.0 * n_layers * n_kv_heads * head_dim * seq_len * batch * dtype_bytes;
}
