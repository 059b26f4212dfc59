// RoPE device helpers.
//
// The rotation (page "Qwen2架构解析" on intelliparadigm.com, §2.3; page "Qwen2
// architecture introduction" on aicoding.csdn.net, §3.5.2 and §4.1.3 step 3):
// row x at position m is rotated pair by pair, dimension i with i + d/2, by the
// angle m * theta^(-2i/d):
//     x'_i       = x_i cos(phi) - x_{i+d/2} sin(phi)
//     x'_{i+d/2} = x_{i+d/2} cos(phi) + x_i sin(phi)
// One cos/sin value serves Q and K alike (page "Qwen2 / Qwen3 的实测配置差异与三个坑",
// docs.keinmal.top, closing note of pitfall 3).
//
// Accuracy: the angle m * f is formed in double precision and reduced into
// [-pi, pi] with 2*pi held as an unevaluated sum of two doubles (the
// Cody & Waite argument reduction), so the single-precision sincosf that
// follows sees a small argument; cos and sin then carry ~1e-7 absolute error
// at any position below 2^31.
#pragma once

#include <cstdint>

namespace gqa {

constexpr double kTwoPiHi = 6.283185307179586;        // the double nearest 2*pi
constexpr double kTwoPiLo = 2.4492935982947064e-16;   // 2*pi - kTwoPiHi
constexpr double kInvTwoPi = 0.15915494309189535;     // 1 / (2*pi), rounded

// YaRN scaling of the frequencies, for contexts beyond the trained window (page "Qwen-2 explained",
// yudonglee.me, §6.2: f'_i = f_i / s * alpha_i with a per-pair ramp alpha_i from 1 to s; page "Qwen2
// architecture introduction", aicoding.csdn.net, §5.3: the attention logits are rescaled with the
// length).  The pages give neither the ramp's bounds nor the rescaling: both follow the published YaRN
// method.  alpha_i = 1 + gamma_i (s - 1), gamma_i = clamp((r_i - 1) / (32 - 1), 0, 1), where r_i =
// orig * f_i / (2 pi) is the number of turns pair i makes over the original window: pairs turning 32
// times or more keep their frequency, pairs turning at most once are interpolated by s.  The logits are
// scaled by mscale^2, mscale = 0.1 ln(s) + 1 (applied by the callers).  factor <= 1: no scaling.
constexpr double kYarnTurnsSlow = 1.0;
constexpr double kYarnTurnsFast = 32.0;

struct RopeSpec {
    double log2_theta;   // log2 of the RoPE base
    double factor;       // YaRN factor s (1 = plain RoPE)
    double orig;         // original (trained) window, in positions
};

// The (possibly scaled) frequency of pair i: theta^(-2i/d), times alpha_i / s under YaRN.
__device__ __forceinline__ double rope_freq(int i, int d, const RopeSpec& r) {
    double f = exp2(-(2.0 * static_cast<double>(i) / static_cast<double>(d)) * r.log2_theta);
    if (r.factor > 1.0) {
        const double turns = r.orig * f * kInvTwoPi;
        double g = (turns - kYarnTurnsSlow) / (kYarnTurnsFast - kYarnTurnsSlow);
        g = g < 0.0 ? 0.0 : (g > 1.0 ? 1.0 : g);
        f = f / r.factor * (1.0 + g * (r.factor - 1.0));
    }
    return f;
}

// cos and sin of the angle pos * f.
__device__ __forceinline__ void rope_cossin(double pos, double f, float& c, float& s) {
    const double phi = pos * f;
    const double k = rint(phi * kInvTwoPi);
    double r = fma(-k, kTwoPiHi, phi);
    r = fma(-k, kTwoPiLo, r);
    sincosf(static_cast<float>(r), &s, &c);
}

// (x, y) rotated by the angle with cosine c and sine s.
__device__ __forceinline__ void rope_rotate(float x, float y, float c, float s, float& xr, float& yr) {
    xr = fmaf(x, c, -y * s);
    yr = fmaf(y, c, x * s);
}

}  // namespace gqa
