// entmax.cuh -- alpha-entmax threshold helpers shared by the routing kernels and the backward
// pass (DashAttention, xllm-io paper review, section 3: the background alpha-entmax formula).
//
// Threshold tau: the mass f(t) = sum_c [x_c - t]_+^{1/(alpha-1)} is continuous and strictly
// decreasing where positive; f(max x - 1) >= 1 and f(max x - nvis^{-(alpha-1)}) <= 1.  Newton
// steps (below) from the left end of that bracket finish to float precision; for alpha = 2 and
// alpha = 1.5 a closed-form root on the current support ends the solve as soon as the support
// is found.
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

// Partial sums of the threshold solve over the entries x > t of a row (u = x - t > 0):
// f = sum u^p, fd = sum u^(p-1), n = their count, um = the smallest u.
struct EntSums {
    float f, fd, n, um;
};
__device__ __forceinline__ EntSums ent_zero() { return EntSums{0.f, 0.f, 0.f, INFINITY}; }
__device__ __forceinline__ void ent_add(EntSums& a, float u, float p, int mode)
{
    if (u > 0.f) {
        a.f += ent_pow(u, p, mode);
        a.fd += ent_dpow(u, p, mode);
        a.n += 1.f;
        a.um = fminf(a.um, u);
    }
}
__device__ __forceinline__ void ent_merge(EntSums& a, const EntSums& b)
{
    a.f += b.f;
    a.fd += b.fd;
    a.n += b.n;
    a.um = fminf(a.um, b.um);
}

// One step of the threshold solve from t, given the sums S over {x > t} of the whole row;
// returns true when t is final.  [lo, hi] brackets the root (f(lo) >= 1 >= f(hi)).
//  * Exact finish (alpha = 2 and alpha = 1.5, where f is a polynomial on a fixed support): the
//    root of sum_S (u - d)^p = 1 with S taken as the support, d = (f - 1)/n for p = 1 and the
//    smaller root of n d^2 - 2 fd d + (f - 1) = 0 for p = 2, written without cancellation as
//    (f - 1)/(fd + sqrt(fd^2 - n (f - 1))).  When f(t) >= 1 and d <= um, every entry of S stays
//    at or above t + d and every other entry is at or below t, so f(t + d) = 1 exactly: t + d is
//    the threshold and S the support.
//  * Otherwise a Newton step on g(t) = f(t)^(alpha-1): g is a p-norm of (x - t)_+, convex and
//    decreasing, and linear while the support is fixed, so from t = max x - 1 (where f >= 1) the
//    iterates rise monotonically to the root; g' = -f^(alpha-2) fd, so the step (g - 1)/(-g')
//    is (g - 1) f / (g fd).  A step that leaves the bracket falls back to bisection.
// Sums with n = 0 (a caller that leaves out the count and the minimum) take Newton steps only.
__device__ __forceinline__ bool ent_step(const EntSums& S, float& t, float& lo, float& hi, float alpha, int mode)
{
    if (S.f >= 1.f) lo = t; else hi = t;
    if (mode != 0 && S.f >= 1.f && S.n > 0.f) {
        float d = -1.f;
        if (mode == 1) d = (S.f - 1.f) / S.n;
        else {
            const float disc = S.fd * S.fd - S.n * (S.f - 1.f);
            if (disc >= 0.f) d = (S.f - 1.f) / (S.fd + sqrtf(disc));
        }
        if (d >= 0.f && d <= S.um) {
            t += d;
            return true;
        }
    }
    float tn = 0.5f * (lo + hi);
    if (S.fd > 0.f && S.f > 0.f) {
        const float gg = mode == 2 ? sqrtf(S.f) : mode == 1 ? S.f : exp2f((alpha - 1.f) * __log2f(S.f));
        tn = t + (gg - 1.f) * S.f / (gg * S.fd);
    }
    if (fabsf(tn - t) <= 2e-7f * fmaxf(1.f, fabsf(t)) || fabsf(S.f - 1.f) <= 1e-6f) {
        t = tn;
        return true;
    }
    if (!(tn > lo && tn < hi)) tn = 0.5f * (lo + hi);
    t = tn;
    return false;
}

// Threshold tau of alpha-entmax for one row, cooperatively.  each(fn) applies fn(x) to this
// thread's entries; red(S) combines the partial sums over the cooperating threads (uniform
// results).  Steps of ent_step from t = max x - 1.
template <typename Each, typename Red>
__device__ float entmax_threshold(Each each, Red red, float mx, int nv, float alpha)
{
    const float p = 1.f / (alpha - 1.f);
    const int mode = ent_mode(alpha);
    float lo = mx - 1.f;
    float hi = mx - exp2f(-(alpha - 1.f) * __log2f((float)nv));
    float t = lo;
    for (int it = 0; it < kMaxIter; ++it) {
        EntSums S = ent_zero();
        each([&](float x) { ent_add(S, x - t, p, mode); });
        red(S);
        if (ent_step(S, t, lo, hi, alpha, mode)) break;
    }
    return t;
}

// Sums of a warp's partial EntSums (uniform over the warp).
__device__ __forceinline__ void ent_warp_reduce(EntSums& S)
{
    S.f = warp_sum(S.f);
    S.fd = warp_sum(S.fd);
    S.n = warp_sum(S.n);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) S.um = fminf(S.um, __shfl_xor_sync(0xffffffffu, S.um, o));
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
        [](EntSums& S) { ent_warp_reduce(S); }, mx, nv, alpha);
}

}  // namespace
}  // namespace dash
