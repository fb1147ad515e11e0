// stage0.cu -- Stage 0 chunk summaries and the incremental summary update.
//
// DashAttention (xllm-io paper review, section 3, Eq. 4 and the "Stage 0" kernel row):
//   kbar_c^(r) = sum_{t in chunk c} softmax_t(<qbar^(r), k_t>/sqrt(d)) k_t
// The keys double as values, so one pass over each key serves both the logit and the weighted
// sum (online softmax); a finished chunk's summary is written once and never recomputed.
//
// A key of d elements is read as 16-byte vectors by d*sizeof(T)/16 lanes, so a warp covers
// 32*16/(d*sizeof(T)) keys per load instruction; each lane group keeps its own online-softmax state
// and the groups merge at the end.
#include "dash_common.cuh"

namespace dash {
namespace {

template <typename T, int D>
struct KeyLanes {
    static constexpr int EPL = Vec<T>::N;   // elements per lane
    static constexpr int LPK = D / EPL;     // lanes per key
    static constexpr int KPI = 32 / LPK;    // keys per warp step
};

// Online-softmax state of one lane group: base-2 scaled logits, fp32.
template <int EPL>
struct Run {
    float m, l, acc[EPL];
    __device__ void init() { m = -INFINITY; l = 0.f; for (int e = 0; e < EPL; ++e) acc[e] = 0.f; }
    __device__ void push(float a2, const float* k)
    {
        float mn = fmaxf(m, a2);
        float sc = exp2f(m - mn), p = exp2f(a2 - mn);
        l = l * sc + p;
        for (int e = 0; e < EPL; ++e) acc[e] = acc[e] * sc + p * k[e];
        m = mn;
    }
    __device__ void merge(float m2, float l2, const float* acc2)
    {
        float mn = fmaxf(m, m2);
        if (mn == -INFINITY) return;
        float s1 = exp2f(m - mn), s2 = exp2f(m2 - mn);
        l = l * s1 + l2 * s2;
        for (int e = 0; e < EPL; ++e) acc[e] = acc[e] * s1 + acc2[e] * s2;
        m = mn;
    }
};

// One block (4 warps) per (sequence, KV head, chunk): warp w takes the w-th quarter of the chunk's
// keys with all of its loads in flight at once (8 per lane), keeps an online-softmax state per
// lane group, and the four warps' states merge through shared memory.
template <typename T, int D>
__global__ void __launch_bounds__(128) stage0_kernel(Shape s, const T* __restrict__ K,
                                                     const float* __restrict__ qbar,
                                                     const int* __restrict__ len, float* kbar,
                                                     int kbar_T, float* state, __nv_bfloat16* planes,
                                                     float* knorm)
{
    using L = KeyLanes<T, D>;
    __shared__ float wst[4][D + 2];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long item = blockIdx.x;
    const int per = kbar_T + 1;
    if (item >= (long long)s.batch * s.hkv * per) return;
    const int c = (int)(item % per);
    const int r = (int)((item / per) % s.hkv);
    const int b = (int)(item / ((long long)per * s.hkv));
    const int n = len ? len[b] : s.n;
    const int cfull = min(n / s.B, kbar_T);
    const bool complete = c < cfull;
    if (!complete && !(state && c == n / s.B)) return;   // block-uniform
    const int t0 = c * s.B, t1c = complete ? t0 + s.B : n;

    const int grp = lane / L::LPK, sub = lane % L::LPK;
    const float qscale = kLog2e * rsqrtf((float)D);
    float qv[L::EPL];
    for (int e = 0; e < L::EPL; ++e) qv[e] = qbar[r * D + sub * L::EPL + e] * qscale;

    Run<L::EPL> run;
    run.init();
    // the chunk's keys are consecutive rows (of a page, for paged caches: a chunk never
    // straddles two pages), so one base serves the whole chunk; no page lookup for an empty
    // chunk, and a chunk on an unmapped page reads nothing (its summary is left undefined)
    const long long koff = t1c > t0 ? kv_off(s, s.ks, s.kps, b, t0, r) : 0;
    const T* kb = K + (koff < 0 ? 0 : koff) + sub * L::EPL;
    const int t1 = koff < 0 ? t0 : t1c;
    // this warp's quarter of [t0, t1)
    const int len_all = t1 - t0, q = (len_all + 3) / 4;
    const int w0 = t0 + min(len_all, warp * q), w1 = t0 + min(len_all, (warp + 1) * q);
    constexpr int U = 8;
    // the loop bounds are warp-uniform so that every lane reaches the shuffles
    for (int base = w0; base < w1; base += U * L::KPI) {
        // all U loads first (rows past the quarter re-read its last row and are not pushed)
        uint4 raw[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int tt = min(base + u * L::KPI + grp, w1 - 1);
            raw[u] = Vec<T>::raw(kb + (long long)(tt - t0) * s.ks[1]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            int tt = base + u * L::KPI + grp;
            float kv[L::EPL];
            Vec<T>::cvt(raw[u], kv);
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < L::EPL; ++e) dot += qv[e] * kv[e];
#pragma unroll
            for (int o = L::LPK / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            if (tt < w1) run.push(dot, kv);
        }
    }
    // merge the lane groups (lanes sub, sub+LPK, sub+2LPK, ... hold the same elements)
#pragma unroll
    for (int o = L::LPK; o < 32; o <<= 1) {
        float m2 = __shfl_xor_sync(0xffffffffu, run.m, o);
        float l2 = __shfl_xor_sync(0xffffffffu, run.l, o);
        float a2[L::EPL];
        for (int e = 0; e < L::EPL; ++e) a2[e] = __shfl_xor_sync(0xffffffffu, run.acc[e], o);
        run.merge(m2, l2, a2);
    }
    // merge the four warps' states in warp order
    if (grp == 0) {
        for (int e = 0; e < L::EPL; ++e) wst[warp][sub * L::EPL + e] = run.acc[e];
        if (sub == 0) { wst[warp][D] = run.m; wst[warp][D + 1] = run.l; }
    }
    __syncthreads();
    if (warp != 0 || grp != 0) return;
    for (int w = 1; w < 4; ++w) {
        float a2[L::EPL];
        for (int e = 0; e < L::EPL; ++e) a2[e] = wst[w][sub * L::EPL + e];
        run.merge(wst[w][D], wst[w][D + 1], a2);
    }
    if (complete) {
        float* out = kbar + (((long long)b * s.hkv + r) * kbar_T + c) * D + sub * L::EPL;
        const float inv = 1.f / run.l;
        for (int e = 0; e < L::EPL; ++e) out[e] = run.acc[e] * inv;
        if (planes) {
            // the summary split exactly into three bf16 planes (hi + mid + lo), [b][r][3][T][D]
            __nv_bfloat16* pl = planes + ((long long)(b * s.hkv + r) * 3 * kbar_T + c) * D + sub * L::EPL;
            const long long ps = (long long)kbar_T * D;
            for (int e = 0; e < L::EPL; ++e) {
                const float v = run.acc[e] * inv;
                const __nv_bfloat16 hi = __float2bfloat16_rn(v);
                const float rem = v - __bfloat162float(hi);
                const __nv_bfloat16 mid = __float2bfloat16_rn(rem);
                pl[e] = hi;
                pl[ps + e] = mid;
                pl[2 * ps + e] = __float2bfloat16_rn(rem - __bfloat162float(mid));
            }
        }
        if (knorm) {
            // the largest Euclidean norm of a summary of this (sequence, KV head): non-negative
            // floats order as their bit patterns, so an unsigned maximum of the bits
            float ss = 0.f;
            for (int e = 0; e < L::EPL; ++e) {
                const float v = run.acc[e] * inv;
                ss = fmaf(v, v, ss);
            }
            constexpr unsigned kGrp = L::LPK >= 32 ? 0xffffffffu : ((1u << L::LPK) - 1u);
#pragma unroll
            for (int o = L::LPK / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(kGrp, ss, o);
            if (sub == 0)
                atomicMax(reinterpret_cast<unsigned*>(knorm) + (b * s.hkv + r), __float_as_uint(sqrtf(ss)));
        }
    } else {
        float* st = state + ((long long)b * s.hkv + r) * (D + 2);
        for (int e = 0; e < L::EPL; ++e) st[sub * L::EPL + e] = run.acc[e];
        if (sub == 0) { st[D] = run.m; st[D + 1] = run.l; }
    }
}

// One block per sequence, one warp per KV head.
template <typename T, int D>
__global__ void append_kernel(Shape s, const T* __restrict__ k_new, const T* __restrict__ v_new,
                              const float* __restrict__ qbar, T* Kc, T* Vc, float* kbar, int kbar_T,
                              float* state, int* seqlens)
{
    pdl_launch_dependents();   // the decode routing that follows waits for this grid itself
    const int b = blockIdx.x, r = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = seqlens[b];
    const bool ok = L < s.n;
    if (r < s.hkv && ok) {
        constexpr int EPL = Vec<T>::N, PIECES = D / EPL;
        const T* kn = k_new + ((long long)b * s.hkv + r) * D;
        const T* vn = v_new + ((long long)b * s.hkv + r) * D;
        const long long ko = kv_off(s, s.ks, s.kps, b, L, r), vo = kv_off(s, s.vs, s.vps, b, L, r);
        if (lane < PIECES && ko >= 0 && vo >= 0) {   // (an unmapped page is not written)
            reinterpret_cast<uint4*>(Kc + ko)[lane] = reinterpret_cast<const uint4*>(kn)[lane];
            reinterpret_cast<uint4*>(Vc + vo)[lane] = reinterpret_cast<const uint4*>(vn)[lane];
        }
        constexpr int E = D / 32;
        float kv[E], dot = 0.f;
        for (int e = 0; e < E; ++e) {
            kv[e] = to_f(kn[lane + 32 * e]);
            dot += qbar[r * D + lane + 32 * e] * kv[e];
        }
        const float a2 = warp_sum(dot) * kLog2e * rsqrtf((float)D);
        float* st = state + ((long long)b * s.hkv + r) * (D + 2);
        const float m = st[D], l = st[D + 1];
        const float mn = fmaxf(m, a2), sc = exp2f(m - mn), p = exp2f(a2 - mn);
        const float ln = l * sc + p;
        float acc[E];
        for (int e = 0; e < E; ++e) acc[e] = st[lane + 32 * e] * sc + p * kv[e];
        __syncwarp();
        if ((L + 1) % s.B == 0) {
            const int c = (L + 1) / s.B - 1;
            float* out = kbar + (((long long)b * s.hkv + r) * kbar_T + c) * D;
            const float inv = 1.f / ln;
            for (int e = 0; e < E; ++e) { out[lane + 32 * e] = acc[e] * inv; st[lane + 32 * e] = 0.f; }
            if (lane == 0) { st[D] = -INFINITY; st[D + 1] = 0.f; }
        } else {
            for (int e = 0; e < E; ++e) st[lane + 32 * e] = acc[e];
            if (lane == 0) { st[D] = mn; st[D + 1] = ln; }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && ok) seqlens[b] = L + 1;
}

template <typename T>
cudaError_t stage0_t(const Shape& s, const void* K, const float* qbar, const int* len, float* kbar,
                     int kbar_T, float* state, __nv_bfloat16* planes, float* knorm, cudaStream_t st)
{
    const long long items = (long long)s.batch * s.hkv * (kbar_T + 1);
    const unsigned grid = (unsigned)items;
    if (grid == 0) return cudaSuccess;
    if (s.d == 128)
        stage0_kernel<T, 128><<<grid, 128, 0, st>>>(s, (const T*)K, qbar, len, kbar, kbar_T, state, planes, knorm);
    else
        stage0_kernel<T, 64><<<grid, 128, 0, st>>>(s, (const T*)K, qbar, len, kbar, kbar_T, state, planes, knorm);
    return cudaGetLastError();
}

template <typename T>
cudaError_t append_t(const Shape& s, const void* kn, const void* vn, const float* qbar, void* Kc,
                     void* Vc, float* kbar, int kbar_T, float* state, int* seqlens, cudaStream_t st)
{
    const unsigned threads = 32u * (unsigned)s.hkv;
    if (s.d == 128)
        append_kernel<T, 128><<<s.batch, threads, 0, st>>>(s, (const T*)kn, (const T*)vn, qbar, (T*)Kc,
                                                           (T*)Vc, kbar, kbar_T, state, seqlens);
    else
        append_kernel<T, 64><<<s.batch, threads, 0, st>>>(s, (const T*)kn, (const T*)vn, qbar, (T*)Kc,
                                                          (T*)Vc, kbar, kbar_T, state, seqlens);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stage0(const Shape& s, int dtype, const void* K, const float* qbar,
                          const int* len, float* kbar, int kbar_T, float* state, cudaStream_t st,
                          __nv_bfloat16* planes, float* knorm)
{
    return dtype == DASH_BF16 ? stage0_t<__nv_bfloat16>(s, K, qbar, len, kbar, kbar_T, state, planes, knorm, st)
                              : stage0_t<float>(s, K, qbar, len, kbar, kbar_T, state, planes, knorm, st);
}

cudaError_t launch_append(const Shape& s, int dtype, const void* k_new, const void* v_new,
                          const float* qbar, void* Kc, void* Vc, float* kbar, int kbar_T,
                          float* state, int* seqlens, cudaStream_t st)
{
    return dtype == DASH_BF16
               ? append_t<__nv_bfloat16>(s, k_new, v_new, qbar, Kc, Vc, kbar, kbar_T, state, seqlens, st)
               : append_t<float>(s, k_new, v_new, qbar, Kc, Vc, kbar, kbar_T, state, seqlens, st);
}

}  // namespace dash
