// rope_table.cpp -- host-side frequency and temperature table (no CUDA).
//
//   RoPE   theta_i = base^(-2i/d), i = 0 .. d/2-1
//          ("LLM context window mechanics", position wall; "Arch_03_Long_Context",
//           RoPE slide)
//   PI     theta_i / s  (PI slide: positions divided by s = L_target / L_train)
//   NTK    (base * s^(d/(d-2)))^(-2i/d)  (NTK-aware slide)
//   YaRN   r_i = L_train / lambda_i with lambda_i = 2 pi / theta_i; the share
//          gamma_i = clamp((r_i - alpha) / (beta - alpha), 0, 1) of each band
//          keeps its frequency, the rest is interpolated as in PI:
//          theta'_i = theta_i * (gamma_i + (1 - gamma_i) / s); the attention
//          temperature mscale = 0.1 ln s + 1 (YaRN slide, steps table)
//   Dynamic NTK  NTK with s = max(1, L_cur / L_train) (NTK-aware slide, last
//          sentence: s follows the current sequence length)
//   YaRN, dimension ramp  the YaRN band split with the ramp linear in the pair
//          index between floor(i_edge(beta)) and ceil(i_edge(alpha)), where
//          i_edge(r) = d ln(L_train / (2 pi r)) / (2 ln base) is the index at
//          which L_train / lambda_i = r ("LLM context window mechanics": its YaRN
//          code finds band-edge indices from a log ratio with floor and ceil)
//   Factors  theta_i / f_i with caller-supplied f_i, mscale = attn_factor
//          (LongRoPE: searched per-dimension interpolation factors)
//   ALiBi  no rotation (theta' = 0); the kernels add the per-head linear bias
//          (ALiBi slide)
//   softmax_scale = mscale^2 / sqrt(d): the temperature on both rotated q and k.
//   The pair layout (interleaved (2i, 2i+1) or half-split (i, i + d/2)) is
//   carried in the table for the kernels; it does not change any frequency.
// The table also carries theta'_i / (2 pi) (rotations per position), which the
// kernels multiply by the position in fp64 to reduce the angle exactly.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <string>

#include "../../include/yarnattn.h"

namespace yr_host {
void set_error(const std::string &msg);
}

namespace {

uint64_t fnv1a(uint64_t h, const void *data, size_t n) {
    const unsigned char *p = static_cast<const unsigned char *>(data);
    for (size_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= 0x100000001b3ull;
    }
    return h;
}

}  // namespace

extern "C" int yr_rope_freq_table(const yr_rope_params *p, yr_rope_table *out) {
    if (p == nullptr || out == nullptr) {
        yr_host::set_error("yr_rope_freq_table: NULL argument");
        return YR_EINVAL;
    }
    const int d = p->head_dim;
    if (d < 2 || d > YR_MAX_HEAD_DIM || (d % 2) != 0) {
        yr_host::set_error("yr_rope_freq_table: head_dim must be even and in [2, 128]");
        return YR_EINVAL;
    }
    if (!(p->base > 1.0) || !std::isfinite(p->base)) {
        yr_host::set_error("yr_rope_freq_table: base must be a finite number > 1");
        return YR_EINVAL;
    }
    if (!(p->scale >= 1.0) || !std::isfinite(p->scale)) {
        yr_host::set_error("yr_rope_freq_table: scale must be a finite number >= 1");
        return YR_EINVAL;
    }
    if (p->method < YR_ROPE || p->method > YR_ALIBI) {
        yr_host::set_error("yr_rope_freq_table: unknown method");
        return YR_EINVAL;
    }
    const bool yarn = p->method == YR_YARN || p->method == YR_YARN_DIMRAMP;
    if (yarn && (p->L_train < 1 || !(p->beta > p->alpha))) {
        yr_host::set_error("yr_rope_freq_table: YaRN needs L_train >= 1 and beta > alpha");
        return YR_EINVAL;
    }
    if (p->method == YR_NTK_DYNAMIC && (p->L_train < 1 || p->L_cur < 1)) {
        yr_host::set_error("yr_rope_freq_table: dynamic NTK needs L_train >= 1 and L_cur >= 1");
        return YR_EINVAL;
    }
    if (p->pairs != YR_PAIR_INTERLEAVED && p->pairs != YR_PAIR_HALF) {
        yr_host::set_error("yr_rope_freq_table: pairs must be YR_PAIR_INTERLEAVED or YR_PAIR_HALF");
        return YR_EINVAL;
    }
    if (p->method == YR_FACTORS) {
        if (p->factors == nullptr) {
            yr_host::set_error("yr_rope_freq_table: YR_FACTORS needs d/2 factors");
            return YR_EINVAL;
        }
        for (int i = 0; i < d / 2; ++i) {
            if (!(p->factors[i] > 0.0) || !std::isfinite(p->factors[i])) {
                yr_host::set_error("yr_rope_freq_table: every factor must be a positive finite number");
                return YR_EINVAL;
            }
        }
    }
    yr_rope_table t;
    std::memset(&t, 0, sizeof t);
    t.head_dim = d;
    t.method = p->method;
    t.pairs = p->pairs;
    const double two_pi = 2.0 * M_PI;
    const double ln_base = std::log(p->base);
    const double s = p->scale;
    // NTK-aware: the whole exponent scales the log of the base; the dynamic form
    // takes s from the current length.
    const double s_ntk =
        p->method == YR_NTK_DYNAMIC
            ? (p->L_cur > p->L_train ? static_cast<double>(p->L_cur) / p->L_train : 1.0)
            : s;
    const double ln_base_ntk = ln_base + (static_cast<double>(d) / (d - 2)) * std::log(s_ntk);
    // Dimension ramp: band-edge pair indices, clamped to the table.
    double ramp_lo = 0.0, ramp_hi = 1.0;
    if (p->method == YR_YARN_DIMRAMP) {
        auto i_edge = [&](double r) {
            return static_cast<double>(d) * std::log(p->L_train / (two_pi * r)) / (2.0 * ln_base);
        };
        ramp_lo = std::max(0.0, std::floor(i_edge(p->beta)));
        ramp_hi = std::min(static_cast<double>(d / 2 - 1), std::ceil(i_edge(p->alpha)));
        if (!(ramp_hi > ramp_lo)) ramp_hi = ramp_lo + 1.0;
    }
    for (int i = 0; i < d / 2; ++i) {
        const double e = -2.0 * i / d;
        const double theta = std::exp(e * ln_base);
        double th = theta;
        switch (p->method) {
            case YR_PI:
                th = theta / s;
                break;
            case YR_NTK:
            case YR_NTK_DYNAMIC:
                th = std::exp(e * ln_base_ntk);
                break;
            case YR_YARN: {
                const double r = p->L_train / (two_pi / theta);
                double gamma = (r - p->alpha) / (p->beta - p->alpha);
                gamma = gamma < 0.0 ? 0.0 : (gamma > 1.0 ? 1.0 : gamma);
                th = theta * (gamma + (1.0 - gamma) / s);
                break;
            }
            case YR_YARN_DIMRAMP: {
                double ramp = (i - ramp_lo) / (ramp_hi - ramp_lo);
                ramp = ramp < 0.0 ? 0.0 : (ramp > 1.0 ? 1.0 : ramp);
                const double gamma = 1.0 - ramp;
                th = theta * (gamma + (1.0 - gamma) / s);
                break;
            }
            case YR_FACTORS:
                th = theta / p->factors[i];
                break;
            case YR_ALIBI:
                th = 0.0;  // position enters as a bias on the logits, not a rotation
                break;
            default:
                break;
        }
        t.inv_freq[i] = th;
        t.turns[i] = th / two_pi;
    }
    t.mscale = yarn ? 0.1 * std::log(s) + 1.0 : 1.0;
    if (p->method == YR_FACTORS && p->attn_factor > 0.0) t.mscale = p->attn_factor;
    t.softmax_scale = t.mscale * t.mscale / std::sqrt(static_cast<double>(d));
    // Position-policy identity: a hash of the parameters that shape the table.
    uint64_t hsh = 0xcbf29ce484222325ull;
    // Fields a method does not use are hashed as constants, so equal tables
    // share a digest.
    const bool dyn = p->method == YR_NTK_DYNAMIC;
    const bool fac = p->method == YR_FACTORS;
    const bool uses_s = p->method == YR_PI || p->method == YR_NTK || yarn;
    const int32_t fields_i[4] = {p->head_dim, (yarn || dyn) ? p->L_train : 0, p->method,
                                 dyn ? p->L_cur : 0};
    const double fields_d[5] = {p->base, uses_s ? p->scale : 1.0, yarn ? p->alpha : 0.0,
                                yarn ? p->beta : 0.0, fac ? t.mscale : 0.0};
    hsh = fnv1a(hsh, fields_i, sizeof fields_i);
    hsh = fnv1a(hsh, fields_d, sizeof fields_d);
    if (fac) hsh = fnv1a(hsh, p->factors, sizeof(double) * (d / 2));
    if (p->pairs != YR_PAIR_INTERLEAVED) hsh = fnv1a(hsh, &p->pairs, sizeof p->pairs);
    t.digest = hsh;
    *out = t;
    return YR_OK;
}
