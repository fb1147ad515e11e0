// stage1.cu -- Stage 1 entmax chunk routing with the GQA average.
//
// DashAttention (xllm-io paper review, section 3, Eq. 6, the "Stage 1" kernel row and
// Proposition 4.1):
//   zbar_{i,c}^(h) = <q_i^(h), kbar_c^(r)>/sqrt(d)              for complete chunks c < floor(i/B)
//   what_i^(h)     = alpha-entmax(gamma zbar_i^(h)) = [(alpha-1) gamma zbar - tau]_+^{1/(alpha-1)}
//   w_i^(r)        = mean over the g_q heads of group r; routed set R = {c : w_c > 0}
//   bias_c         = (log w_c - mean_{c' in R} log w_c') / sigma
// The output is one ascending list of (chunk, bias) per (position, KV head): the heads of a
// group share one sparse support.
//
// Threshold tau: the mass f(t) = sum_c [x_c - t]_+^{1/(alpha-1)} is continuous and strictly
// decreasing where positive; f(max x - 1) >= 1 and f(max x - nvis^{-(alpha-1)}) <= 1.  A fixed
// number of bisection steps narrows that bracket to about 1e-6 of its width, then Newton steps
// from the left end (the tangent of a convex decreasing function stays below it, so the steps
// never pass the root) finish to float precision.
#include "dash_common.cuh"

namespace dash {
namespace {

constexpr int kBisect = 20;
constexpr int kNewton = 2;

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

// Warp-cooperative threshold of one row held in shared memory, x[0..nv).  Returns tau.
__device__ float warp_threshold(const float* x, int nv, float alpha)
{
    const int lane = threadIdx.x & 31;
    const float p = 1.f / (alpha - 1.f);
    const int mode = ent_mode(alpha);
    float mx = -INFINITY;
    for (int c = lane; c < nv; c += 32) mx = fmaxf(mx, x[c]);
    mx = warp_max(mx);
    float lo = mx - 1.f;
    float hi = mx - exp2f(-(alpha - 1.f) * __log2f((float)nv));
    for (int it = 0; it < kBisect; ++it) {
        const float t = 0.5f * (lo + hi);
        float f = 0.f;
        for (int c = lane; c < nv; c += 32) {
            float u = x[c] - t;
            if (u > 0.f) f += ent_pow(u, p, mode);
        }
        f = warp_sum(f);
        if (f >= 1.f) lo = t; else hi = t;
    }
    float t = lo;
    for (int it = 0; it < kNewton; ++it) {
        float f = 0.f, fd = 0.f;
        for (int c = lane; c < nv; c += 32) {
            float u = x[c] - t;
            if (u > 0.f) { f += ent_pow(u, p, mode); fd += ent_dpow(u, p, mode); }
        }
        f = warp_sum(f) - 1.f;
        fd = warp_sum(fd) * p;
        if (fd > 0.f) t = fminf(fmaxf(t + f / fd, lo), hi);
    }
    return t;
}

// Ordered compaction of one position's routed chunks by one warp; writes the list, the count
// and the optional bitmask row.  wsum(c) returns the sum over heads of the head weights.
template <typename WF>
__device__ void warp_emit(WF wsum, int nv, float inv_g, float inv_sigma, int* idx, float* bias,
                          int* count, uint32_t* mask_row, int words)
{
    const int lane = threadIdx.x & 31;
    float slog = 0.f;
    int cnt = 0;
    for (int c = lane; c < nv; c += 32) {
        float w = wsum(c) * inv_g;
        if (w > 0.f) { slog += __logf(w); ++cnt; }
    }
    slog = warp_sum(slog);
    cnt = warp_isum(cnt);
    const float mu = cnt > 0 ? slog / cnt : 0.f;
    int base = 0;
    for (int c0 = 0; c0 < nv; c0 += 32) {
        const int c = c0 + lane;
        float w = c < nv ? wsum(c) * inv_g : 0.f;
        const bool on = w > 0.f;
        const uint32_t m = __ballot_sync(0xffffffffu, on);
        if (on) {
            const int k = base + __popc(m & ((1u << lane) - 1u));
            idx[k] = c;
            bias[k] = (__logf(w) - mu) * inv_sigma;
        }
        if (mask_row && lane == 0) mask_row[c0 >> 5] = m;
        base += __popc(m);
    }
    if (mask_row)
        for (int wd = ((nv + 31) >> 5) + lane; wd < words; wd += 32) mask_row[wd] = 0u;
    if (lane == 0) *count = base;
}

// ------------------------------------------------------------------------------------------
// Prefill: one block per (sequence, KV head, block of P positions); rows = P * g query rows.
// Shared memory: scaled query rows [rows][D], one summary tile [32][D+4], logits [rows][Ts].
// ------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) route_prefill_kernel(Shape s, const T* __restrict__ Q,
                                                            const float* __restrict__ kbar,
                                                            Routes rt, int P, int Ts)
{
    extern __shared__ float4 smem4[];
    float* qsm = reinterpret_cast<float*>(smem4);
    float* ktile = qsm + P * s.g * D;
    float* S = ktile + 32 * (D + 4);
    const int rows = P * s.g;
    const int nblk = (s.n + P - 1) / P;
    const int br = blockIdx.x % (s.batch * s.hkv);
    const int pb = nblk - 1 - blockIdx.x / (s.batch * s.hkv);   // heaviest blocks first
    const int b = br / s.hkv, r = br % s.hkv;
    const int i0 = pb * P;
    const int ilast = min(i0 + P, s.n) - 1;
    const int nvmax = min(ilast / s.B, s.T);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int* counts = rt.counts + (long long)br * s.n;
    int* idx = rt.idx + (long long)br * rt.cap;
    float* bias = rt.bias + (long long)br * rt.cap;
    uint32_t* bm = rt.bitmask ? rt.bitmask + (long long)br * s.n * rt.words : nullptr;

    if (nvmax == 0) {
        for (int p = tid; p < P && i0 + p < s.n; p += blockDim.x) counts[i0 + p] = 0;
        if (bm)
            for (int k = tid; k < P * rt.words; k += blockDim.x)
                if (i0 + k / rt.words < s.n) bm[(long long)i0 * rt.words + k] = 0u;
        return;
    }
    // scaled query rows: x = (alpha-1) * gamma / sqrt(d) * <q, kbar>
    const float xs = (s.alpha - 1.f) * s.gamma * rsqrtf((float)D);
    constexpr int EPL = Vec<T>::N;
    for (int v = tid; v < rows * (D / EPL); v += blockDim.x) {
        const int row = v / (D / EPL), e0 = (v % (D / EPL)) * EPL;
        const int p = row / s.g, h = row % s.g, i = i0 + p;
        float q[EPL];
        if (i < s.n) {
            Vec<T>::load(Q + (long long)b * s.qs[0] + (long long)i * s.qs[1] +
                             (long long)(r * s.g + h) * s.qs[2] + e0, q);
        } else {
            for (int e = 0; e < EPL; ++e) q[e] = 0.f;
        }
        for (int e = 0; e < EPL; ++e) qsm[row * D + e0 + e] = q[e] * xs;
    }
    const float* kb = kbar + (long long)br * s.T * D;
    for (int c0 = 0; c0 < nvmax; c0 += 32) {
        __syncthreads();
        for (int v = tid; v < 32 * (D / 4); v += blockDim.x) {
            const int cc = v / (D / 4), e = (v % (D / 4)) * 4;
            float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
            if (c0 + cc < nvmax) val = *reinterpret_cast<const float4*>(kb + (long long)(c0 + cc) * D + e);
            *reinterpret_cast<float4*>(ktile + cc * (D + 4) + e) = val;
        }
        __syncthreads();
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.f;
        const float* kr = ktile + lane * (D + 4);
#pragma unroll 4
        for (int e = 0; e < D; e += 4) {
            const float4 kv = *reinterpret_cast<const float4*>(kr + e);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int row = warp + 8 * k;
                if (row < rows) {
                    const float4 qv = *reinterpret_cast<const float4*>(qsm + row * D + e);
                    acc[k] += qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
                }
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int row = warp + 8 * k;
            if (row < rows) S[row * Ts + c0 + lane] = acc[k];
        }
    }
    __syncthreads();
    // thresholds, one warp per row; head weights overwrite the logits in place
    for (int row = warp; row < rows; row += 8) {
        const int i = i0 + row / s.g;
        if (i >= s.n) continue;
        const int nv = min(i / s.B, s.T);
        if (nv == 0) continue;
        float* x = S + row * Ts;
        const float tau = warp_threshold(x, nv, s.alpha);
        const float p = 1.f / (s.alpha - 1.f);
        const int mode = ent_mode(s.alpha);
        for (int c = lane; c < nv; c += 32) {
            const float u = x[c] - tau;
            x[c] = u > 0.f ? ent_pow(u, p, mode) : 0.f;
        }
    }
    __syncthreads();
    // GQA average, bias and ordered compaction, one warp per position
    for (int p = warp; p < P; p += 8) {
        const int i = i0 + p;
        if (i >= s.n) continue;
        const int nv = min(i / s.B, s.T);
        const float* W = S + p * s.g * Ts;
        const int g = s.g;
        auto wsum = [&](int c) {
            float a = 0.f;
            for (int h = 0; h < g; ++h) a += W[h * Ts + c];
            return a;
        };
        const long long off = tri_offset(i, s.B);
        warp_emit(wsum, nv, 1.f / g, s.inv_sigma, idx + off, bias + off, counts + i,
                  bm ? bm + (long long)i * rt.words : nullptr, rt.words);
    }
}

// ------------------------------------------------------------------------------------------
// Decode: the single query of sequence b sits at position L_b - 1 (L_b = seqlens[b]) and sees
// the cached summaries of chunks c < floor((L_b - 1)/B).
// (a) logits: one block per (32-chunk tile, sequence, KV head), all g heads of the group.
// ------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) dec_logits_kernel(Shape s, const T* __restrict__ q,
                                                         const float* __restrict__ kbar, int kbar_T,
                                                         const int* __restrict__ seqlens, float* X)
{
    __shared__ float qsm[16 * D];
    __shared__ __align__(16) float ktile[32 * (D + 4)];
    const int br = blockIdx.y, b = br / s.hkv, r = br % s.hkv;
    const int nv = min((seqlens[b] - 1) / s.B, kbar_T);
    const int c0 = blockIdx.x * 32;
    if (c0 >= nv) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float xs = (s.alpha - 1.f) * s.gamma * rsqrtf((float)D);
    for (int v = tid; v < s.g * D; v += blockDim.x)
        qsm[v] = to_f(q[((long long)b * s.hq + r * s.g) * D + v]) * xs;
    const float* kb = kbar + (long long)br * kbar_T * D;
    for (int v = tid; v < 32 * (D / 4); v += blockDim.x) {
        const int cc = v / (D / 4), e = (v % (D / 4)) * 4;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c0 + cc < nv) val = *reinterpret_cast<const float4*>(kb + (long long)(c0 + cc) * D + e);
        *reinterpret_cast<float4*>(ktile + cc * (D + 4) + e) = val;
    }
    __syncthreads();
    const float* kr = ktile + lane * (D + 4);
    for (int h = warp; h < s.g; h += 8) {
        float acc = 0.f;
#pragma unroll 8
        for (int e = 0; e < D; e += 4) {
            const float4 kv = *reinterpret_cast<const float4*>(kr + e);
            const float4 qv = *reinterpret_cast<const float4*>(qsm + h * D + e);
            acc += qv.x * kv.x + qv.y * kv.y + qv.z * kv.z + qv.w * kv.w;
        }
        if (c0 + lane < nv) X[((long long)br * s.g + h) * kbar_T + c0 + lane] = acc;
    }
}

// (b) threshold: one block per (head, sequence, KV head); block-wide reductions.
__device__ float block_sum(float v, float* red)
{
    v = warp_sum(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = lane < nw ? red[lane] : 0.f;
    return warp_sum(t);
}
__device__ float block_max(float v, float* red)
{
    v = warp_max(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = lane < nw ? red[lane] : -INFINITY;
    return warp_max(t);
}

__global__ void __launch_bounds__(256) dec_tau_kernel(Shape s, int kbar_T, const int* __restrict__ seqlens,
                                                      float* X)
{
    __shared__ float red[32];
    const int h = blockIdx.x, br = blockIdx.y, b = br / s.hkv;
    const int nv = min((seqlens[b] - 1) / s.B, kbar_T);
    if (nv <= 0) return;
    float* x = X + ((long long)br * s.g + h) * kbar_T;
    const float p = 1.f / (s.alpha - 1.f);
    const int mode = ent_mode(s.alpha);
    float mx = -INFINITY;
    for (int c = threadIdx.x; c < nv; c += blockDim.x) mx = fmaxf(mx, x[c]);
    mx = block_max(mx, red);
    float lo = mx - 1.f, hi = mx - exp2f(-(s.alpha - 1.f) * __log2f((float)nv));
    for (int it = 0; it < kBisect; ++it) {
        const float t = 0.5f * (lo + hi);
        float f = 0.f;
        for (int c = threadIdx.x; c < nv; c += blockDim.x) {
            const float u = x[c] - t;
            if (u > 0.f) f += ent_pow(u, p, mode);
        }
        f = block_sum(f, red);
        if (f >= 1.f) lo = t; else hi = t;
    }
    float t = lo;
    for (int it = 0; it < kNewton; ++it) {
        float f = 0.f, fd = 0.f;
        for (int c = threadIdx.x; c < nv; c += blockDim.x) {
            const float u = x[c] - t;
            if (u > 0.f) { f += ent_pow(u, p, mode); fd += ent_dpow(u, p, mode); }
        }
        f = block_sum(f, red) - 1.f;
        fd = block_sum(fd, red) * p;
        if (fd > 0.f) t = fminf(fmaxf(t + f / fd, lo), hi);
    }
    __syncthreads();
    for (int c = threadIdx.x; c < nv; c += blockDim.x) {
        const float u = x[c] - t;
        x[c] = u > 0.f ? ent_pow(u, p, mode) : 0.f;
    }
}

// (c) GQA average, bias and compaction: one warp per (sequence, KV head).
__global__ void __launch_bounds__(32) dec_emit_kernel(Shape s, int kbar_T, const int* __restrict__ seqlens,
                                                      const float* __restrict__ X, Routes rt)
{
    const int br = blockIdx.x, b = br / s.hkv;
    const int nv = max(0, min((seqlens[b] - 1) / s.B, kbar_T));
    const float* W = X + (long long)br * s.g * kbar_T;
    const int g = s.g;
    auto wsum = [&](int c) {
        float a = 0.f;
        for (int h = 0; h < g; ++h) a += W[(long long)h * kbar_T + c];
        return a;
    };
    warp_emit(wsum, nv, 1.f / g, s.inv_sigma, rt.idx + (long long)br * rt.cap,
              rt.bias + (long long)br * rt.cap, rt.counts + br,
              rt.bitmask ? rt.bitmask + (long long)br * rt.words : nullptr, rt.words);
}

template <typename T, int D>
cudaError_t route_prefill_t(const Shape& s, const void* Q, const float* kbar, const Routes& rt,
                            cudaStream_t st)
{
    int P = 0;
    const size_t smem = route_prefill_smem(s, &P);
    if (P == 0) return cudaErrorInvalidValue;
    const int Ts = (s.T + 31) / 32 * 32;
    auto k = route_prefill_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long nblk = (s.n + P - 1) / P;
    const unsigned grid = (unsigned)(nblk * s.batch * s.hkv);
    if (grid == 0) return cudaSuccess;
    k<<<grid, 256, smem, st>>>(s, (const T*)Q, kbar, rt, P, Ts);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t dec_route_t(const Shape& s, const void* q, const float* kbar, int kbar_T,
                        const int* seqlens, const Routes& rt, float* X, cudaStream_t st)
{
    if (kbar_T > 0) {
        dim3 g1((kbar_T + 31) / 32, s.batch * s.hkv);
        dec_logits_kernel<T, D><<<g1, 256, 0, st>>>(s, (const T*)q, kbar, kbar_T, seqlens, X);
        dim3 g2(s.g, s.batch * s.hkv);
        dec_tau_kernel<<<g2, 256, 0, st>>>(s, kbar_T, seqlens, X);
    }
    dec_emit_kernel<<<s.batch * s.hkv, 32, 0, st>>>(s, kbar_T, seqlens, X, rt);
    return cudaGetLastError();
}

}  // namespace

size_t route_prefill_smem(const Shape& s, int* positions_per_block)
{
    const int Ts = (s.T + 31) / 32 * 32;
    const size_t limit = 200 * 1024;
    int best = 0;
    size_t bytes = 0;
    for (int P = 1; P * s.g <= 64; ++P) {
        size_t need = sizeof(float) * ((size_t)P * s.g * s.d + 32 * (size_t)(s.d + 4) + (size_t)P * s.g * Ts);
        if (need > limit) break;
        best = P;
        bytes = need;
    }
    *positions_per_block = best;
    return bytes;
}

cudaError_t launch_route_prefill(const Shape& s, int dtype, const void* Q, const float* kbar,
                                 const Routes& rt, cudaStream_t st)
{
    if (dtype == DASH_BF16)
        return s.d == 128 ? route_prefill_t<__nv_bfloat16, 128>(s, Q, kbar, rt, st)
                          : route_prefill_t<__nv_bfloat16, 64>(s, Q, kbar, rt, st);
    return s.d == 128 ? route_prefill_t<float, 128>(s, Q, kbar, rt, st)
                      : route_prefill_t<float, 64>(s, Q, kbar, rt, st);
}

cudaError_t launch_route_decode(const Shape& s, int dtype, const void* q, const float* kbar, int kbar_T,
                                const int* seqlens, const Routes& rt, float* X, cudaStream_t st)
{
    if (dtype == DASH_BF16)
        return s.d == 128 ? dec_route_t<__nv_bfloat16, 128>(s, q, kbar, kbar_T, seqlens, rt, X, st)
                          : dec_route_t<__nv_bfloat16, 64>(s, q, kbar, kbar_T, seqlens, rt, X, st);
    return s.d == 128 ? dec_route_t<float, 128>(s, q, kbar, kbar_T, seqlens, rt, X, st)
                      : dec_route_t<float, 64>(s, q, kbar, kbar_T, seqlens, rt, X, st);
}

}  // namespace dash
