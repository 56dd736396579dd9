// tables.cu -- host-side position-encoding tables for lazy_attn_cfg:
// RoPE frequencies (the default base^(-2i/d) table and Llama-3.1 frequency
// scaling) and ALiBi head slopes.
//
// Source: gist.science, "LazyAttention: Efficient Retrieval-Augmented
// Generation with Deferred Positional Encoding", Technical Summary, Key
// Contributions -- the deferred encoding carries over to other relative
// positional encodings (RoPE variants, ALiBi).  The pages fix no table; the
// rules below are the published ones each function names.
#include <cmath>

#include "lazy_attn.h"

extern "C" {

int lazy_rope_theta(double base, int head_dim, double *theta) {
    if (!theta || head_dim <= 0 || (head_dim & 1) || !(base > 1.0) || !std::isfinite(base)) return LAZY_EINVAL;
    for (int i = 0; i < head_dim / 2; ++i) theta[i] = std::pow(base, -2.0 * i / head_dim);
    return LAZY_OK;
}

// Llama-3.1 frequency scaling ("llama3" rope type of the Llama 3.1 model
// configuration).  A default frequency f has wavelength 2 pi / f; wavelengths
// shorter than original_max / high_freq_factor keep f, those longer than
// original_max / low_freq_factor get f / factor, and in between the frequency
// moves linearly in original_max / wavelength from f / factor (at
// low_freq_factor) to f (at high_freq_factor).
int lazy_rope_theta_llama31(double base, int head_dim, double factor, double low_freq_factor,
                            double high_freq_factor, double original_max_position, double *theta) {
    if (!(factor > 0.0) || !(low_freq_factor > 0.0) || !(high_freq_factor > low_freq_factor) ||
        !(original_max_position > 0.0) || !std::isfinite(factor) || !std::isfinite(high_freq_factor) ||
        !std::isfinite(original_max_position))
        return LAZY_EINVAL;
    const int rc = lazy_rope_theta(base, head_dim, theta);
    if (rc != LAZY_OK) return rc;
    const double two_pi = 6.283185307179586476925286766559;
    const double short_wl = original_max_position / high_freq_factor;
    const double long_wl = original_max_position / low_freq_factor;
    for (int i = 0; i < head_dim / 2; ++i) {
        const double f = theta[i];
        const double wl = two_pi / f;
        if (wl < short_wl) continue;
        if (wl > long_wl) {
            theta[i] = f / factor;
        } else {
            const double t = (original_max_position / wl - low_freq_factor) / (high_freq_factor - low_freq_factor);
            theta[i] = t * f + (1.0 - t) * f / factor;
        }
    }
    return LAZY_OK;
}

// ALiBi head slopes (Press, Smith and Lewis, "Train Short, Test Long:
// Attention with Linear Biases", 2022): for n heads with n a power of two,
// slope k (k = 1..n) is 2^(-8k/n).  Otherwise the p slopes of the largest
// power of two p below n come first, then every second slope (the 1st, 3rd,
// 5th, ...) of the 2p-head rule, n - p of them.
int lazy_alibi_slopes(int num_heads, double *slopes) {
    if (!slopes || num_heads <= 0) return LAZY_EINVAL;
    int p = 1;
    while (2 * p <= num_heads) p *= 2;
    for (int k = 0; k < p; ++k) slopes[k] = std::exp2(-8.0 * (k + 1) / p);
    for (int k = p; k < num_heads; ++k) slopes[k] = std::exp2(-8.0 * (2 * (k - p) + 1) / (2 * p));
    return LAZY_OK;
}

}  // extern "C"
