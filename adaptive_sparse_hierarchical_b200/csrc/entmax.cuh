// entmax.cuh -- alpha-entmax threshold helpers shared by the routing kernels and the backward
// pass (DashAttention, xllm-io paper review, section 3: the background alpha-entmax formula).
//
// Threshold tau: the mass f(t) = sum_c [x_c - t]_+^{1/(alpha-1)} is continuous and strictly
// decreasing where positive; f(max x - 1) >= 1 and f(max x - nvis^{-(alpha-1)}) <= 1.  Newton
// steps (below) from the left end of that bracket finish to float precision.
#pragma once

#include "dash_common.cuh"

namespace dash {
namespace {

constexpr int kMaxIter = 32;

__device__ __forceinline__ float ent_pow(float u, float p, int mode)
{
    // mode 1: alpha = 2 (power 1); mode 2: alpha = 1.5 (power 2); else general power
    return mode == 1 ? u : mode == 2 ? u * u : exp2f(p * __log2f(u));
}
__device__ __forceinline__ float ent_dpow(float u, float p, int mode)
{
    // u^(p-1)
    return mode == 1 ? 1.f : mode == 2 ? u : exp2f((p - 1.f) * __log2f(u));
}
__device__ __forceinline__ int ent_mode(float alpha) { return alpha == 2.f ? 1 : alpha == 1.5f ? 2 : 0; }

// Threshold tau of alpha-entmax for one row, cooperatively.  each(fn) applies fn(x) to this
// thread's entries; red(f, fd) sums both over the cooperating threads (uniform results).
// Newton steps on g(t) = f(t)^(alpha-1), f(t) = sum [x - t]_+^p, p = 1/(alpha-1): g is a p-norm
// of (x - t)_+, hence convex and decreasing, and exactly linear while the support is fixed, so
// from t = max x - 1 (where f >= 1) the iterates rise monotonically to the root in a few steps.
// The bracket [lo, hi] guards against rounding; a step leaving it falls back to bisection.
template <typename Each, typename Red>
__device__ float entmax_threshold(Each each, Red red, float mx, int nv, float alpha)
{
    const float p = 1.f / (alpha - 1.f);
    const int mode = ent_mode(alpha);
    float lo = mx - 1.f;
    float hi = mx - exp2f(-(alpha - 1.f) * __log2f((float)nv));
    float t = lo;
    for (int it = 0; it < kMaxIter; ++it) {
        float f = 0.f, fd = 0.f;
        each([&](float x) {
            const float u = x - t;
            if (u > 0.f) { f += ent_pow(u, p, mode); fd += ent_dpow(u, p, mode); }
        });
        red(f, fd);
        if (f >= 1.f) lo = t; else hi = t;
        float tn = 0.5f * (lo + hi);
        if (fd > 0.f && f > 0.f) {
            const float gg = mode == 2 ? sqrtf(f) : mode == 1 ? f : exp2f((alpha - 1.f) * __log2f(f));
            tn = t + (gg - 1.f) * f / (gg * fd);
        }
        if (fabsf(tn - t) <= 2e-7f * fmaxf(1.f, fabsf(t)) || fabsf(f - 1.f) <= 1e-6f) { t = tn; break; }
        if (!(tn > lo && tn < hi)) tn = 0.5f * (lo + hi);
        t = tn;
    }
    return t;
}

// Warp-cooperative threshold of one row held in shared memory, x[0..nv).
__device__ float warp_threshold(const float* x, int nv, float alpha)
{
    const int lane = threadIdx.x & 31;
    float mx = -INFINITY;
    for (int c = lane; c < nv; c += 32) mx = fmaxf(mx, x[c]);
    mx = warp_max(mx);
    return entmax_threshold(
        [&](auto fn) { for (int c = lane; c < nv; c += 32) fn(x[c]); },
        [](float& a, float& b) { a = warp_sum(a); b = warp_sum(b); }, mx, nv, alpha);
}

}  // namespace
}  // namespace dash
