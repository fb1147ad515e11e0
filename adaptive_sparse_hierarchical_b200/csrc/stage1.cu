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
// decreasing where positive; f(max x - 1) >= 1 and f(max x - nvis^{-(alpha-1)}) <= 1.  Newton
// steps on f^(alpha-1) from the left end (the tangent of a convex decreasing function stays
// below it, so the steps never pass the root) finish to float precision; for alpha = 2 and 1.5
// the closed-form root on the current support ends the solve once the support is found
// (entmax.cuh, ent_step).
#include <algorithm>
#include <cstdlib>

#include "dash_common.cuh"
#include "entmax.cuh"
#include "stage2_mma.cuh"

namespace dash {
namespace {

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

// A block of positions [i0, ilast] is recomputed only where the long-row kernel flagged one of
// the position blocks (redo_p positions each) that it overlaps; redo == null runs every block.
__device__ __forceinline__ bool redo_wanted(const unsigned char* redo, int redo_p, const Shape& s, int br, int i0,
                                            int ilast)
{
    if (!redo) return true;
    const unsigned char* rr = redo + (long long)br * ((s.n + redo_p - 1) / redo_p);
    for (int tb = i0 / redo_p; tb <= ilast / redo_p; ++tb)
        if (rr[tb]) return true;
    return false;
}

// ------------------------------------------------------------------------------------------
// Prefill: one block per (sequence, KV head, block of P positions); rows = P * g query rows.
// Shared memory: scaled query rows [rows][D], one summary tile [32][D+4], logits [rows][Ts].
// ------------------------------------------------------------------------------------------
template <typename T, int D>
__device__ void route_prefill_block(Shape s, const T* __restrict__ Q, const float* __restrict__ kbar, Routes rt,
                                    int P, int Ts, const unsigned char* redo, int redo_p, int blk)
{
    extern __shared__ float4 smem4[];
    float* qsm = reinterpret_cast<float*>(smem4);
    float* ktile = qsm + P * s.g * D;
    float* S = ktile + 32 * (D + 4);
    const int rows = P * s.g;
    const int nblk = (s.n + P - 1) / P;
    const int br = blk % (s.batch * s.hkv);
    const int pb = nblk - 1 - blk / (s.batch * s.hkv);   // heaviest blocks first
    const int b = br / s.hkv, r = br % s.hkv;
    const int i0 = pb * P;
    const int ilast = min(i0 + P, s.n) - 1;
    const int nvmax = min(ilast / s.B, s.T);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int* counts = rt.counts + (long long)br * s.n;
    int* idx = rt.idx + (long long)br * rt.cap;
    float* bias = rt.bias + (long long)br * rt.cap;
    uint32_t* bm = rt.bitmask ? rt.bitmask + (long long)br * s.n * rt.words : nullptr;
    if (!redo_wanted(redo, redo_p, s, br, i0, ilast)) return;

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

// Block number blk of the launch order above; with a list (list[0] entries from list[1] on), a
// fixed grid walks the listed block numbers instead of one block per position block.
template <typename T, int D>
__global__ void __launch_bounds__(256) route_prefill_kernel(Shape s, const T* __restrict__ Q,
                                                            const float* __restrict__ kbar,
                                                            Routes rt, int P, int Ts,
                                                            const unsigned char* redo, int redo_p, const int* list)
{
    if (!list) {
        route_prefill_block<T, D>(s, Q, kbar, rt, P, Ts, redo, redo_p, blockIdx.x);
        return;
    }
    const int nl = list[0];
    for (int w = blockIdx.x; w < nl; w += gridDim.x) {
        route_prefill_block<T, D>(s, Q, kbar, rt, P, Ts, nullptr, 1, list[1 + w]);
        __syncthreads();   // shared memory is reused by the next listed block
    }
}

// Threshold from a compacted candidate list: tau >= max x - 1, so entries at or below max - 1
// never enter the support and never contribute to the mass; the warp copies the others (about a
// sixth of a typical row) to its scratch list once and takes the Newton passes over that list.
template <int NPL>
__device__ float warp_threshold_compact(const float (&xr)[NPL], int nv, float alpha, float* scratch)
{
    const int lane = threadIdx.x & 31;
    float mx = xr[0];
#pragma unroll
    for (int k = 1; k < NPL; ++k) mx = fmaxf(mx, xr[k]);
    mx = warp_max(mx);
    const float lo = mx - 1.f;
    int m = 0;
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
        const bool keep = xr[k] > lo;
        const uint32_t bal = __ballot_sync(0xffffffffu, keep);
        if (keep) scratch[m + __popc(bal & ((1u << lane) - 1u))] = xr[k];
        m += __popc(bal);
    }
    __syncwarp();
    const float t = entmax_threshold(
        [&](auto fn) { for (int c = lane; c < m; c += 32) fn(scratch[c]); },
        [](EntSums& S) { ent_warp_reduce(S); }, mx, nv, alpha);
    __syncwarp();   // scratch is reused by the warp's next row
    return t;
}

// Register-resident threshold: row x[0..nv) with nv <= 32*NPL, NPL values per lane (-inf pads).
template <int NPL>
__device__ float warp_threshold_reg(const float (&xr)[NPL], int nv, float alpha)
{
    float mx = xr[0];
#pragma unroll
    for (int k = 1; k < NPL; ++k) mx = fmaxf(mx, xr[k]);
    mx = warp_max(mx);
    return entmax_threshold(
        [&](auto fn) {
#pragma unroll
            for (int k = 0; k < NPL; ++k) fn(xr[k]);
        },
        [](EntSums& S) { ent_warp_reduce(S); }, mx, nv, alpha);
}

// ------------------------------------------------------------------------------------------
// Prefill, bf16 queries: the chunk logits run on the tensor cores.  A query is exact in bf16;
// each fp32 summary is split exactly into three bf16 planes (hi + mid + lo = kbar, 8 mantissa
// bits each; written by Stage 0), so three bf16 MMAs with fp32 accumulation reproduce the fp32
// dot product.  Block = 8 warps, ROWS = 16*RG query rows = ROWS/g positions of one (sequence,
// KV head); 32-chunk plane tiles are staged with cp.async.  Shared memory: one tile (three
// swizzled bf16 planes) and the logits [ROWS][Ts].  Rows of up to 512 visible chunks solve the
// threshold from registers.
// ------------------------------------------------------------------------------------------
template <int D, int RG>
__device__ void route_prefill_tc_block(Shape s, const __nv_bfloat16* __restrict__ Q,
                                       const __nv_bfloat16* __restrict__ planes, Routes rt, int Ts,
                                       const unsigned char* redo, int redo_p, int blk)
{
    constexpr int ROWS = 16 * RG;
    constexpr int TCH = 32;                    // chunks per staged tile
    constexpr int PLANE = TCH * D * 2;
    extern __shared__ __align__(128) char smem[];
    char* kt = smem;
    float* S = reinterpret_cast<float*>(smem + 3 * PLANE);
    float* scratch = S + ROWS * Ts + (threadIdx.x >> 5) * 512;   // per-warp candidate list
    const int G = s.g, P = ROWS / G;
    const int nblk = (s.n + P - 1) / P;
    const int br = blk % (s.batch * s.hkv);
    const int pb = nblk - 1 - blk / (s.batch * s.hkv);   // heaviest blocks first
    const int b = br / s.hkv, r = br % s.hkv;
    const int i0 = pb * P;
    const int ilast = min(i0 + P, s.n) - 1;
    const int nvmax = min(ilast / s.B, s.T);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int* counts = rt.counts + (long long)br * s.n;
    int* idx = rt.idx + (long long)br * rt.cap;
    float* bias = rt.bias + (long long)br * rt.cap;
    uint32_t* bm = rt.bitmask ? rt.bitmask + (long long)br * s.n * rt.words : nullptr;
    if (!redo_wanted(redo, redo_p, s, br, i0, ilast)) return;
    if (nvmax == 0) {
        for (int p = tid; p < P && i0 + p < s.n; p += blockDim.x) counts[i0 + p] = 0;
        if (bm)
            for (int k = tid; k < P * rt.words; k += blockDim.x)
                if (i0 + k / rt.words < s.n) bm[(long long)i0 * rt.words + k] = 0u;
        return;
    }
    const int rg = warp % RG;
    uint32_t qf[D / 16][4];
    load_q_frags<D>(qf, [&](int rr) -> const __nv_bfloat16* {
        const int R = rg * 16 + rr, i = i0 + R / G;
        if (i >= s.n) return nullptr;
        return Q + (long long)b * s.qs[0] + (long long)i * s.qs[1] + (long long)(r * G + R % G) * s.qs[2];
    });
    const float xs = (s.alpha - 1.f) * s.gamma * rsqrtf((float)D);
    const __nv_bfloat16* pg = planes + (long long)br * 3 * s.T * D;
    const int mi = lane >> 3, rr8 = lane & 7, t4 = lane & 3;
    for (int c0 = 0; c0 < nvmax; c0 += TCH) {
        __syncthreads();
        for (int v = tid; v < 3 * TCH * (D / 8); v += 256) {
            const int pl = v / (TCH * (D / 8)), rem = v % (TCH * (D / 8));
            const int cc = rem / (D / 8), col = (rem % (D / 8)) * 8;
            const bool ok = c0 + cc < s.T;
            cp_async16_zfill(kt + pl * PLANE + swz<D>(cc, col),
                             ok ? pg + ((long long)pl * s.T + c0 + cc) * D + col : pg, ok);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        for (int u = warp; u < RG * (TCH / 16); u += 8) {
            const int slice = u / RG;
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = swz<D>(slice * 16 + rr8 + (mi >> 1) * 8, kk * 16 + (mi & 1) * 8);
#pragma unroll
                for (int pl = 0; pl < 3; ++pl) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(smem_u32(kt + pl * PLANE) + off, b0, b1, b2, b3);
                    mma_bf16(acc[0], qf[kk], b0, b1);
                    mma_bf16(acc[1], qf[kk], b2, b3);
                }
            }
            const int ra = rg * 16 + (lane >> 2), rb = ra + 8;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int col = c0 + slice * 16 + j * 8 + 2 * t4;
                *reinterpret_cast<float2*>(S + ra * Ts + col) = make_float2(acc[j][0] * xs, acc[j][1] * xs);
                *reinterpret_cast<float2*>(S + rb * Ts + col) = make_float2(acc[j][2] * xs, acc[j][3] * xs);
            }
        }
    }
    __syncthreads();
    const float p = 1.f / (s.alpha - 1.f);
    const int mode = ent_mode(s.alpha);
    for (int row = warp; row < ROWS; row += 8) {
        const int i = i0 + row / G;
        if (i >= s.n) continue;
        const int nv = min(i / s.B, s.T);
        if (nv == 0) continue;
        float* x = S + row * Ts;
        if (nv <= 512) {
            float xr[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) xr[k] = lane + 32 * k < nv ? x[lane + 32 * k] : -INFINITY;
            const float tau = warp_threshold_compact<16>(xr, nv, s.alpha, scratch);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const float u = xr[k] - tau;
                if (lane + 32 * k < nv) x[lane + 32 * k] = u > 0.f ? ent_pow(u, p, mode) : 0.f;
            }
        } else {
            const float tau = warp_threshold(x, nv, s.alpha);
            for (int c = lane; c < nv; c += 32) {
                const float u = x[c] - tau;
                x[c] = u > 0.f ? ent_pow(u, p, mode) : 0.f;
            }
        }
    }
    __syncthreads();
    for (int pp = warp; pp < P; pp += 8) {
        const int i = i0 + pp;
        if (i >= s.n) continue;
        const int nv = min(i / s.B, s.T);
        const float* W = S + pp * G * Ts;
        auto wsum = [&](int c) {
            float a = 0.f;
            for (int h = 0; h < G; ++h) a += W[h * Ts + c];
            return a;
        };
        const long long off = tri_offset(i, s.B);
        warp_emit(wsum, nv, 1.f / G, s.inv_sigma, idx + off, bias + off, counts + i,
                  bm ? bm + (long long)i * rt.words : nullptr, rt.words);
    }
}

// ------------------------------------------------------------------------------------------
// Decode: the single query of sequence b sits at position L_b - 1 (L_b = seqlens[b]) and sees
// the cached summaries of chunks c < floor((L_b - 1)/B).
// (a) logits: one block per (32-chunk tile, sequence, KV head), all g heads of the group.
// ------------------------------------------------------------------------------------------
template <int D, int RG>
__global__ void __launch_bounds__(256) route_prefill_tc_kernel(Shape s, const __nv_bfloat16* __restrict__ Q,
                                                               const __nv_bfloat16* __restrict__ planes,
                                                               Routes rt, int Ts,
                                                               const unsigned char* redo, int redo_p, const int* list)
{
    if (!list) {
        route_prefill_tc_block<D, RG>(s, Q, planes, rt, Ts, redo, redo_p, blockIdx.x);
        return;
    }
    const int nl = list[0];
    for (int w = blockIdx.x; w < nl; w += gridDim.x) {
        route_prefill_tc_block<D, RG>(s, Q, planes, rt, Ts, nullptr, 1, list[1 + w]);
        __syncthreads();   // shared memory is reused by the next listed block
    }
}

// The block numbers (launch order of the two kernels above, P positions per block) whose
// positions overlap a position block that the long-row kernel flagged: appended to list[1..],
// list[0] counting them (zero on entry).  The order of the list does not matter.
__global__ void __launch_bounds__(256) redo_compact_kernel(Shape s, int P, const unsigned char* __restrict__ redo,
                                                           int redo_p, int* list)
{
    const int nblk = (s.n + P - 1) / P;
    const long long total = (long long)nblk * s.batch * s.hkv;
    const long long f = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (f >= total) return;
    const int br = (int)(f % (s.batch * s.hkv));
    const int pb = nblk - 1 - (int)(f / (s.batch * s.hkv));
    const int i0 = pb * P, ilast = min(i0 + P, s.n) - 1;
    if (redo_wanted(redo, redo_p, s, br, i0, ilast)) list[1 + atomicAdd(list, 1)] = (int)f;
}

// Launch of a routing kernel over every position block (redo == null), or over the blocks that
// overlap a flagged one: compacted into redo_list first, then a fixed grid of a few blocks per SM.
template <typename Launch>
cudaError_t launch_redo(const Shape& s, int P, long long grid, const unsigned char* redo, int redo_p, int* redo_list,
                        cudaStream_t st, Launch launch)
{
    if (grid <= 0) return cudaSuccess;
    if (!redo || !redo_list) return launch((unsigned)grid, redo, (const int*)nullptr);
    if (cudaMemsetAsync(redo_list, 0, sizeof(int), st) != cudaSuccess) return cudaErrorUnknown;
    redo_compact_kernel<<<(unsigned)((grid + 255) / 256), 256, 0, st>>>(s, P, redo, redo_p, redo_list);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        nsm = 148;
    return launch((unsigned)std::min<long long>(grid, 2LL * nsm), (const unsigned char*)nullptr, (const int*)redo_list);
}

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

// (b) thresholds, GQA average, bias and ordered compaction for one (sequence, KV head): the
// logits of the g heads are copied to shared memory, one warp per head solves its threshold,
// then the whole block averages the heads and writes the ascending route list.
__global__ void __launch_bounds__(512) dec_route_kernel(Shape s, int kbar_T, const int* __restrict__ seqlens,
                                                        const float* __restrict__ X, Routes rt)
{
    extern __shared__ float xsm[];   // [g][kbar_T]
    __shared__ float red_f[16];
    __shared__ int red_i[16], wpos[17];
    const int br = blockIdx.x, b = br / s.hkv, G = s.g;
    const int nv = max(0, min((seqlens[b] - 1) / s.B, kbar_T));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
    const float* Xb = X + (long long)br * G * kbar_T;
    for (int v = tid; v < G * nv; v += blockDim.x) {
        const int h = v / nv, c = v % nv;
        xsm[h * kbar_T + c] = Xb[(long long)h * kbar_T + c];
    }
    __syncthreads();
    if (nv > 0 && warp < G) {
        float* x = xsm + warp * kbar_T;
        const float tau = warp_threshold(x, nv, s.alpha);
        const float p = 1.f / (s.alpha - 1.f);
        const int mode = ent_mode(s.alpha);
        for (int c = lane; c < nv; c += 32) {
            const float u = x[c] - tau;
            x[c] = u > 0.f ? ent_pow(u, p, mode) : 0.f;
        }
    }
    __syncthreads();
    const float inv_g = 1.f / G;
    auto wof = [&](int c) {
        float a = 0.f;
        for (int h = 0; h < G; ++h) a += xsm[h * kbar_T + c];
        return a * inv_g;
    };
    float sl = 0.f;
    int cnt = 0;
    for (int c = tid; c < nv; c += blockDim.x) {
        const float w = wof(c);
        if (w > 0.f) { sl += __logf(w); ++cnt; }
    }
    sl = warp_sum(sl);
    cnt = warp_isum(cnt);
    if (lane == 0) { red_f[warp] = sl; red_i[warp] = cnt; }
    __syncthreads();
    float tot = 0.f;
    int tcnt = 0;
    for (int k = 0; k < nw; ++k) { tot += red_f[k]; tcnt += red_i[k]; }
    const float mu = tcnt > 0 ? tot / tcnt : 0.f;
    int* idx = rt.idx + (long long)br * rt.cap;
    float* bias = rt.bias + (long long)br * rt.cap;
    uint32_t* mrow = rt.bitmask ? rt.bitmask + (long long)br * rt.words : nullptr;
    int base = 0;
    for (int c0 = 0; c0 < nv; c0 += blockDim.x) {
        const int c = c0 + tid;
        const float w = c < nv ? wof(c) : 0.f;
        const bool on = w > 0.f;
        const uint32_t m = __ballot_sync(0xffffffffu, on);
        if (lane == 0) red_i[warp] = __popc(m);
        __syncthreads();
        if (tid == 0) {
            wpos[0] = 0;
            for (int k = 0; k < nw; ++k) wpos[k + 1] = wpos[k] + red_i[k];
        }
        __syncthreads();
        if (on) {
            const int k = base + wpos[warp] + __popc(m & ((1u << lane) - 1u));
            idx[k] = c;
            bias[k] = (__logf(w) - mu) * s.inv_sigma;
        }
        if (mrow && lane == 0 && c0 + 32 * warp < nv) mrow[(c0 + 32 * warp) >> 5] = m;
        base += wpos[nw];
        __syncthreads();
    }
    if (mrow)
        for (int wd = ((nv + 31) >> 5) + tid; wd < rt.words; wd += blockDim.x) mrow[wd] = 0u;
    if (tid == 0) rt.counts[br] = base;
}

template <typename T, int D>
cudaError_t route_prefill_t(const Shape& s, const void* Q, const float* kbar, const Routes& rt,
                            cudaStream_t st, const unsigned char* redo = nullptr, int redo_p = 1, int* redo_list = nullptr)
{
    int P = 0;
    const size_t smem = route_prefill_smem(s, &P);
    if (P == 0) return cudaErrorInvalidValue;
    const int Ts = (s.T + 31) / 32 * 32;
    auto k = route_prefill_kernel<T, D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long nblk = (s.n + P - 1) / P;
    return launch_redo(s, P, nblk * s.batch * s.hkv, redo, redo_p, redo_list, st,
                       [&](unsigned grid, const unsigned char* rd, const int* list) {
                           k<<<grid, 256, smem, st>>>(s, (const T*)Q, kbar, rt, P, Ts, rd, redo_p, list);
                           return cudaGetLastError();
                       });
}

// Shared memory of the tensor-core routing kernel for RG row groups.
size_t route_tc_smem(const Shape& s, int RG)
{
    const int Ts = (s.T + 31) / 32 * 32 + 8;
    return 3 * (size_t)32 * s.d * 2 + (size_t)16 * RG * Ts * 4 + 8 * 512 * 4;
}

template <int D, int RG>
cudaError_t route_tc_t(const Shape& s, const void* Q, const __nv_bfloat16* planes, const Routes& rt, cudaStream_t st,
                       const unsigned char* redo, int redo_p, int* redo_list)
{
    const size_t smem = route_tc_smem(s, RG);
    const int Ts = (s.T + 31) / 32 * 32 + 8;
    auto k = route_prefill_tc_kernel<D, RG>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int P = 16 * RG / s.g;
    const long long nblk = (s.n + P - 1) / P;
    return launch_redo(s, P, nblk * s.batch * s.hkv, redo, redo_p, redo_list, st,
                       [&](unsigned grid, const unsigned char* rd, const int* list) {
                           k<<<grid, 256, smem, st>>>(s, (const __nv_bfloat16*)Q, planes, rt, Ts, rd, redo_p, list);
                           return cudaGetLastError();
                       });
}

template <int D>
cudaError_t route_tc_d(const Shape& s, const void* Q, const __nv_bfloat16* planes, const Routes& rt,
                       cudaStream_t st, bool* used, const unsigned char* redo = nullptr, int redo_p = 1,
                       int* redo_list = nullptr)
{
    constexpr size_t kLimit = 225 * 1024;
    *used = true;
    if (32 >= s.g && route_tc_smem(s, 2) <= kLimit) return route_tc_t<D, 2>(s, Q, planes, rt, st, redo, redo_p, redo_list);
    if (16 >= s.g && route_tc_smem(s, 1) <= kLimit) return route_tc_t<D, 1>(s, Q, planes, rt, st, redo, redo_p, redo_list);
    *used = false;
    return cudaSuccess;
}

// (b') threshold of one head's row, one block of 256 threads per (head, sequence, KV head); the
// row stays in registers (up to 16 values per thread) and each Newton step reduces over the block.
__global__ void __launch_bounds__(256) dec_tau_block_kernel(Shape s, int kbar_T, const int* __restrict__ seqlens,
                                                            float* X)
{
    __shared__ float4 red[2][8];
    const int h = blockIdx.x, br = blockIdx.y, b = br / s.hkv;
    const int nv = min((seqlens[b] - 1) / s.B, kbar_T);
    if (nv <= 0) return;
    float* x = X + ((long long)br * s.g + h) * kbar_T;
    constexpr int NPL = 16;
    float xr[NPL];
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
        const int c = threadIdx.x + 256 * k;
        xr[k] = c < nv ? x[c] : -INFINITY;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int phase = 0;
    auto bsum = [&](EntSums& S) {
        ent_warp_reduce(S);
        if (lane == 0) red[phase][warp] = make_float4(S.f, S.fd, S.n, S.um);
        __syncthreads();
        S = ent_zero();
        for (int w = 0; w < 8; ++w) {
            const float4 v = red[phase][w];
            ent_merge(S, EntSums{v.x, v.y, v.z, v.w});
        }
        phase ^= 1;   // alternate buffers: the next reduction cannot overwrite values still being read
    };
    float mx = xr[0];
#pragma unroll
    for (int k = 1; k < NPL; ++k) mx = fmaxf(mx, xr[k]);
    {
        const float m2 = warp_max(mx);
        if (lane == 0) red[phase][warp].x = m2;
        __syncthreads();
        mx = -INFINITY;
        for (int w = 0; w < 8; ++w) mx = fmaxf(mx, red[phase][w].x);
        phase ^= 1;
    }
    const float tau = entmax_threshold(
        [&](auto fn) {
#pragma unroll
            for (int k = 0; k < NPL; ++k) fn(xr[k]);
        },
        bsum, mx, nv, s.alpha);
    const float p = 1.f / (s.alpha - 1.f);
    const int mode = ent_mode(s.alpha);
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
        const int c = threadIdx.x + 256 * k;
        const float u = xr[k] - tau;
        if (c < nv) x[c] = u > 0.f ? ent_pow(u, p, mode) : 0.f;
    }
}

// (c') GQA average, bias and ordered compaction from the head weights in global memory: one
// block of 1024 threads per (sequence, KV head).
__global__ void __launch_bounds__(1024) dec_emit_block_kernel(Shape s, int kbar_T, const int* __restrict__ seqlens,
                                                              const float* __restrict__ X, Routes rt)
{
    __shared__ float red_f[32];
    __shared__ int red_i[32], wpos[33];
    const int br = blockIdx.x, b = br / s.hkv, G = s.g;
    const int nv = max(0, min((seqlens[b] - 1) / s.B, kbar_T));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
    const float* Xb = X + (long long)br * G * kbar_T;
    const float inv_g = 1.f / G;
    auto wof = [&](int c) {
        float a = 0.f;
        for (int h = 0; h < G; ++h) a += Xb[(long long)h * kbar_T + c];
        return a * inv_g;
    };
    float sl = 0.f;
    int cnt = 0;
    for (int c = tid; c < nv; c += blockDim.x) {
        const float w = wof(c);
        if (w > 0.f) { sl += __logf(w); ++cnt; }
    }
    sl = warp_sum(sl);
    cnt = warp_isum(cnt);
    if (lane == 0) { red_f[warp] = sl; red_i[warp] = cnt; }
    __syncthreads();
    float tot = 0.f;
    int tcnt = 0;
    for (int k = 0; k < nw; ++k) { tot += red_f[k]; tcnt += red_i[k]; }
    const float mu = tcnt > 0 ? tot / tcnt : 0.f;
    int* idx = rt.idx + (long long)br * rt.cap;
    float* bias = rt.bias + (long long)br * rt.cap;
    uint32_t* mrow = rt.bitmask ? rt.bitmask + (long long)br * rt.words : nullptr;
    int base = 0;
    for (int c0 = 0; c0 < nv; c0 += blockDim.x) {
        const int c = c0 + tid;
        const float w = c < nv ? wof(c) : 0.f;
        const bool on = w > 0.f;
        const uint32_t m = __ballot_sync(0xffffffffu, on);
        __syncthreads();
        if (lane == 0) red_i[warp] = __popc(m);
        __syncthreads();
        if (tid == 0) {
            wpos[0] = 0;
            for (int k = 0; k < nw; ++k) wpos[k + 1] = wpos[k] + red_i[k];
        }
        __syncthreads();
        if (on) {
            const int k = base + wpos[warp] + __popc(m & ((1u << lane) - 1u));
            idx[k] = c;
            bias[k] = (__logf(w) - mu) * s.inv_sigma;
        }
        if (mrow && lane == 0 && c0 + 32 * warp < nv) mrow[(c0 + 32 * warp) >> 5] = m;
        base += wpos[nw];
    }
    if (mrow)
        for (int wd = ((nv + 31) >> 5) + tid; wd < rt.words; wd += blockDim.x) mrow[wd] = 0u;
    if (tid == 0) rt.counts[br] = base;
}

template <typename T, int D>
cudaError_t dec_route_t(const Shape& s, const void* q, const float* kbar, int kbar_T,
                        const int* seqlens, const Routes& rt, float* X, cudaStream_t st)
{
    if (kbar_T > 0) {
        dim3 g1((kbar_T + 31) / 32, s.batch * s.hkv);
        dec_logits_kernel<T, D><<<g1, 256, 0, st>>>(s, (const T*)q, kbar, kbar_T, seqlens, X);
    }
    if (kbar_T <= 16 * 256) {
        if (kbar_T > 0) dec_tau_block_kernel<<<dim3(s.g, s.batch * s.hkv), 256, 0, st>>>(s, kbar_T, seqlens, X);
        dec_emit_block_kernel<<<s.batch * s.hkv, 1024, 0, st>>>(s, kbar_T, seqlens, X, rt);
        return cudaGetLastError();
    }
    const size_t smem = (size_t)s.g * (kbar_T > 0 ? kbar_T : 1) * 4;
    cudaError_t e = cudaFuncSetAttribute(dec_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dec_route_kernel<<<s.batch * s.hkv, 32 * s.g, smem, st>>>(s, kbar_T, seqlens, X, rt);
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

// DASH_LONG_ROUTE=off keeps rows of more than 512 chunks on the per-shape kernels (for comparison)
static bool long_route_off()
{
    static const bool off = [] {
        const char* v = getenv("DASH_LONG_ROUTE");
        return v && v[0] == 'o';
    }();
    return off;
}

cudaError_t launch_route_prefill(const Shape& s, int dtype, const void* Q, const float* kbar,
                                 const __nv_bfloat16* planes, const float* knorm, const Routes& rt,
                                 unsigned char* redo, int* redo_list, void* spill, int* err, cudaStream_t st)
{
    if (planes && route_tcgen05_supported(s, dtype) && !legacy_stage2())
        return launch_route_prefill_tcgen05(s, Q, planes, rt, err, st);
    // rows of more than 512 chunks: the long-row tcgen05 kernel, then the kernels below only for
    // the position blocks whose candidate lists overflowed
    const unsigned char* mask = nullptr;
    int mask_p = 1;
    if (planes && knorm && redo && route_long_supported(s, dtype) && !legacy_stage2() && !long_route_off()) {
        cudaError_t e = launch_route_prefill_long(s, Q, planes, knorm, rt, redo, err, spill, st);
        if (e != cudaSuccess) return e;
        mask = redo;
        mask_p = route_long_positions(s);
    }
    if (dtype == DASH_BF16 && planes) {
        bool used = false;
        int* list = mask ? redo_list : nullptr;
        cudaError_t e = s.d == 128 ? route_tc_d<128>(s, Q, planes, rt, st, &used, mask, mask_p, list)
                                   : route_tc_d<64>(s, Q, planes, rt, st, &used, mask, mask_p, list);
        if (used) return e;
        // very long rows (T * 16 rows of logits beyond shared memory): CUDA-core variant
        return s.d == 128 ? route_prefill_t<__nv_bfloat16, 128>(s, Q, kbar, rt, st, mask, mask_p, list)
                          : route_prefill_t<__nv_bfloat16, 64>(s, Q, kbar, rt, st, mask, mask_p, list);
    }
    return s.d == 128 ? route_prefill_t<float, 128>(s, Q, kbar, rt, st)
                      : route_prefill_t<float, 64>(s, Q, kbar, rt, st);
}

cudaError_t launch_route_decode(const Shape& s, int dtype, const void* q, const float* kbar, int kbar_T,
                                const int* seqlens, const Routes& rt, float* X, int* status, cudaStream_t st)
{
    // DASH_DEC_ROUTE=heads keeps the per-head kernels below (the long-context path) for comparison
    static const bool per_head = [] {
        const char* e = getenv("DASH_DEC_ROUTE");
        return e && e[0] == 'h';
    }();
    if (!per_head && dec_route_cluster_supported(s, kbar_T))
        return launch_route_decode_cluster(s, dtype, q, kbar, kbar_T, seqlens, rt, status, st);
    if (status && cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return cudaGetLastError();
    if (dtype == DASH_BF16)
        return s.d == 128 ? dec_route_t<__nv_bfloat16, 128>(s, q, kbar, kbar_T, seqlens, rt, X, st)
                          : dec_route_t<__nv_bfloat16, 64>(s, q, kbar, kbar_T, seqlens, rt, X, st);
    return s.d == 128 ? dec_route_t<float, 128>(s, q, kbar, kbar_T, seqlens, rt, X, st)
                      : dec_route_t<float, 64>(s, q, kbar, kbar_T, seqlens, rt, X, st);
}

}  // namespace dash
