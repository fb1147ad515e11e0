// stage1_decode.cu -- Stage 1 of incremental decoding in one launch: chunk logits, entmax
// thresholds, GQA average, bias and the ascending route list of every (sequence, KV head).
//
// DashAttention (xllm-io paper review, section 3, Eq. 6 and Proposition 4.1; decoding: the query
// at position L-1 routes over the cached summaries of the complete chunks c < floor((L-1)/B)):
//   x_c^(h) = (alpha-1) gamma <q^(h), kbar_c>/sqrt(d),  what^(h) = [x^(h) - tau^(h)]_+^{1/(alpha-1)}
//   w = mean over the g heads of the group,  R = {w > 0},  bias_c = (log w_c - mean_R log w)/sigma
//
// One thread-block cluster of 4 blocks per (sequence, KV head); block `rank` owns the chunk slice
// [rank * per, (rank + 1) * per) (per a multiple of 32) and keeps the g x per logits in shared
// memory.  The quantities that need the whole row are combined through distributed shared
// memory, always in rank order: each head's maximum; the entries above max - 1 (the only ones
// the support can reach), which every block pushes into the shared memory of block h % 4 so that
// it solves head h's threshold alone from local memory; the sum of log w and the routed count
// before each slice.  Five cluster barriers in all.
#include <cooperative_groups.h>
#include <type_traits>

#include "dash_common.cuh"
#include "entmax.cuh"
#include "stage2_mma.cuh"

namespace cg = cooperative_groups;

namespace dash {
namespace {

constexpr int kRanks = 4;        // blocks per cluster (small clusters: all of them fit on the GPU at once)
constexpr int kThr = 512;        // 16 warps: warp h owns head h in the per-head phases
constexpr int kMaxG = 16;
constexpr int kSlots = 16 / kRanks;   // heads each block solves (head h: block h % kRanks, slot h / kRanks)

struct Cross {                   // per block, read by the other blocks of the cluster
    float mx[kMaxG];             // slice maximum of each head's logits
    int cc[kSlots][kRanks];      // [head slot][source block]: entries pushed into gbuf
    float tau[kMaxG];            // thresholds of the heads this block solved (h % 8 == rank)
    float slog;                  // slice sum of log w over routed chunks
    int cnt;                     // routed chunks in the slice
};

// Shared-memory layout (floats): x [g][per] logits (row 0 later the group weights), gbuf
// [head slots][source blocks][per]: the entries above max - 1 of the heads this block solves,
// pushed there by every block of the cluster.
__host__ __device__ inline size_t route_cluster_smem(int g, int per)
{
    const int slots = (g + kRanks - 1) / kRanks;
    return ((size_t)g * per + (size_t)slots * kRanks * per) * 4;
}

// (hi, mid, lo) bf16 pairs with hi + mid + lo == (x0, x1) exactly, by truncation: hi keeps the
// top 8 significand bits of x, r = x - hi is exact and has at most 16, mid keeps r's top 8 and
// lo = r - mid the remaining 8 (all exactly representable in bf16).  Integer masks, subtractions
// and byte permutes only.
__device__ __forceinline__ void split3(float x0, float x1, uint32_t& hi, uint32_t& mid, uint32_t& lo)
{
    const float h0 = __uint_as_float(__float_as_uint(x0) & 0xffff0000u);
    const float h1 = __uint_as_float(__float_as_uint(x1) & 0xffff0000u);
    const float r0 = x0 - h0, r1 = x1 - h1;
    const float m0 = __uint_as_float(__float_as_uint(r0) & 0xffff0000u);
    const float m1 = __uint_as_float(__float_as_uint(r1) & 0xffff0000u);
    const float l0 = r0 - m0, l1 = r1 - m1;
    hi = __byte_perm(__float_as_uint(h0), __float_as_uint(h1), 0x7632);
    mid = __byte_perm(__float_as_uint(m0), __float_as_uint(m1), 0x7632);
    lo = __byte_perm(__float_as_uint(l0), __float_as_uint(l1), 0x7632);
}

template <typename T, int D>
__global__ void __cluster_dims__(kRanks, 1, 1) __launch_bounds__(kThr, 1)
    dec_route_cluster_kernel(Shape s, const T* __restrict__ q, const float* __restrict__ kbar, int kbar_T,
                             const int* __restrict__ seqlens, Routes rt, int per, int* status)
{
    // the append of this step (the previous kernel) may still run: seqlens and the caches are
    // read after its completion
    pdl_wait();
    pdl_launch_dependents();
    // the step's status word starts at 0 here (the later kernels of the step may set it)
    if (status && blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
    extern __shared__ __align__(16) float dyn[];
    __shared__ __align__(16) float qs[kMaxG * D];
    __shared__ Cross cx;
    __shared__ float tau[kMaxG], gmax[kMaxG];
    __shared__ int wsum[kThr / 32 + 1];
    __shared__ float fsum[kThr / 32];
    __shared__ float2 npart[2][kSlots * kRanks];      // Newton partial sums [step parity][slot, source]
    __shared__ int ndone[kSlots];
    cg::cluster_group cl = cg::this_cluster();
    const int rank = (int)cl.block_rank();
    const int br = blockIdx.x / kRanks, b = br / s.hkv, r = br % s.hkv, G = s.g;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nv = max(0, min((seqlens[b] - 1) / s.B, kbar_T));
    const int c_lo = rank * per, c_hi = min(nv, c_lo + per), nloc = max(0, c_hi - c_lo);
    const float xs = (s.alpha - 1.f) * s.gamma * rsqrtf((float)D);
    const float p = 1.f / (s.alpha - 1.f);
    const int mode = s.alpha == 2.f ? 1 : s.alpha == 1.5f ? 2 : 0;
    float* xsm = dyn;
    float* gbuf = dyn + (size_t)G * per;

    // ---- logits of this slice ---------------------------------------------------------------
    // bf16 queries are exact in bf16 and k̄ splits exactly into three bf16 planes, so the logits
    // come from m16n8k16 MMAs (16 head rows x 8 chunks, fp32 accumulation): warp w takes the
    // 8-chunk tiles w, w + 16, ...; each lane loads its B fragments straight from global memory
    // (per tile the warp reads the tile's 8 rows once, in whole 32-byte sectors, 16 loads in
    // flight per lane).  fp32 queries: CUDA cores, one thread per (chunk, 4 heads).
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    const float* kb = kbar + ((long long)br * kbar_T + c_lo) * D;
    if constexpr (kBf16) {
        uint32_t qf[D / 16][4];
        const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(q) + ((long long)b * s.hq + r * G) * D;
        load_q_frags<D>(qf, [&](int h) -> const __nv_bfloat16* { return h < G ? qb + (long long)h * D : nullptr; });
        const int g8 = lane >> 2, t4 = lane & 3;
        // the next tile's fragments are loaded while the current tile is computed
        float2 u[D / 16][2], un[D / 16][2];
        auto load_tile = [&](int nt, float2 (&dst)[D / 16][2]) {
            const int row = nt * 8 + g8;
            const bool ok = nt * 8 < nloc && row < nloc;
            const float* kr = kb + (long long)row * D + 2 * t4;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                dst[kk][0] = ok ? __ldg(reinterpret_cast<const float2*>(kr + kk * 16)) : make_float2(0.f, 0.f);
                dst[kk][1] = ok ? __ldg(reinterpret_cast<const float2*>(kr + kk * 16 + 8)) : make_float2(0.f, 0.f);
            }
        };
        load_tile(warp, u);
        for (int nt = warp; nt * 8 < nloc; nt += kThr / 32) {
            load_tile(nt + kThr / 32, un);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t h0, m0, l0, h1, m1, l1;
                split3(u[kk][0].x, u[kk][0].y, h0, m0, l0);
                split3(u[kk][1].x, u[kk][1].y, h1, m1, l1);
                mma_bf16(acc, qf[kk], l0, l1);
                mma_bf16(acc, qf[kk], m0, m1);
                mma_bf16(acc, qf[kk], h0, h1);
            }
            const int c = nt * 8 + 2 * t4;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int h = g8 + (e >> 1) * 8, cc = c + (e & 1);
                if (h < G && cc < nloc) xsm[h * per + cc] = acc[e] * xs;
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) { u[kk][0] = un[kk][0]; u[kk][1] = un[kk][1]; }
        }
    } else {
        for (int v = tid; v < G * D; v += kThr) qs[v] = to_f(q[((long long)b * s.hq + r * G) * D + v]) * xs;
        __syncthreads();
        const int hb = tid & 3;
        for (int c = tid >> 2; c < nloc && 4 * hb < G; c += kThr / 4) {
            const float4* kr = reinterpret_cast<const float4*>(kb + (long long)c * D);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int e4 = 0; e4 < D / 4; ++e4) {
                const float4 a = __ldg(kr + e4);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 qv = *reinterpret_cast<const float4*>(qs + min(4 * hb + j, G - 1) * D + 4 * e4);
                    acc[j] = fmaf(qv.x, a.x, fmaf(qv.y, a.y, fmaf(qv.z, a.z, fmaf(qv.w, a.w, acc[j]))));
                }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (4 * hb + j < G) xsm[(4 * hb + j) * per + c] = acc[j];
        }
    }
    __syncthreads();

    // ---- per-head maximum over the row (warp h: head h) ---------------------------------------
    if (warp < G) {
        float m = -INFINITY;
        for (int c = lane; c < nloc; c += 32) m = fmaxf(m, xsm[warp * per + c]);
        m = warp_max(m);
        if (lane == 0) cx.mx[warp] = m;
    }
    cl.sync();
    // ---- entries above max - 1 (the only ones that can enter the support: tau >= max - 1):
    // pushed, in index order, into region [rank] of head h's solver (block h % 8), with the count
    if (warp < G) {
        const float mr = lane < kRanks ? cl.map_shared_rank(&cx, lane)->mx[warp] : -INFINITY;
        const float m = warp_max(mr);
        if (lane == 0) gmax[warp] = m;
        const int slot = warp / kRanks;
        float* dst = cl.map_shared_rank(gbuf, warp % kRanks) + ((size_t)slot * kRanks + rank) * per;
        int n = 0;
        for (int c0 = 0; c0 < nloc; c0 += 32) {
            const int c = c0 + lane;
            const float v = c < nloc ? xsm[warp * per + c] : -INFINITY;
            const bool on = v > m - 1.f;
            const uint32_t bal = __ballot_sync(0xffffffffu, on);
            if (on) dst[n + __popc(bal & ((1u << lane) - 1u))] = v;
            n += __popc(bal);
        }
        if (lane == 0) cl.map_shared_rank(&cx, warp % kRanks)->cc[slot][rank] = n;
    }
    cl.sync();
    // ---- thresholds: block `rank` solves heads h = rank + kRanks slot on the pushed entries; warp
    // (slot, k) sums over source block k's entries, the partials are added in k order, and every
    // thread of the slot takes the same Newton step (entmax.cuh, ent_step; the closed-form finish
    // is left out here: its count and minimum reductions cost more on these ~700-entry lists than
    // the steps they save) from max - 1 -----------------------------------------------------------
    static_assert(kSlots * kRanks == kThr / 32, "one warp per (head slot, source block)");
    {
        const int slot = warp / kRanks, k = warp % kRanks, h = rank + kRanks * slot;
        const bool active = h < G && nv > 0;
        const float* gl = gbuf + ((size_t)slot * kRanks + k) * per;
        const int nk = active ? cx.cc[slot][k] : 0;
        const float mxh = active ? gmax[h] : 0.f;
        float lo = mxh - 1.f, t = lo;
        float hi = active ? mxh - exp2f(-(s.alpha - 1.f) * __log2f((float)nv)) : 0.f;
        bool dn = !active;
        if (tid < kSlots) ndone[tid] = !(rank + kRanks * tid < G && nv > 0);
        __syncthreads();
        for (int it = 0; it < 32; ++it) {
            bool all = true;
#pragma unroll
            for (int j = 0; j < kSlots; ++j) all = all && ndone[j];
            if (all) break;
            const int ph = it & 1;
            float f = 0.f, fd = 0.f;
            for (int j = lane; j < nk; j += 32) {
                const float u = gl[j] - t;
                if (u > 0.f) { f += ent_pow(u, p, mode); fd += ent_dpow(u, p, mode); }
            }
            f = warp_sum(f);
            fd = warp_sum(fd);
            if (lane == 0) npart[ph][slot * kRanks + k] = make_float2(f, fd);
            __syncthreads();   // a parity slot is rewritten two steps later, after the next barrier
            EntSums S = ent_zero();   // n = 0: Newton steps only
            for (int kk = 0; kk < kRanks; ++kk) { S.f += npart[ph][slot * kRanks + kk].x; S.fd += npart[ph][slot * kRanks + kk].y; }
            if (!dn) dn = ent_step(S, t, lo, hi, s.alpha, mode);
            // every thread of a slot holds the same state; the slot's first warp reports it
            if (k == 0 && lane == 0) ndone[slot] = dn;
            __syncthreads();
        }
        if (active && k == 0 && lane == 0) cx.tau[h] = t;
    }
    cl.sync();
    if (tid < G) tau[tid] = cl.map_shared_rank(&cx, tid % kRanks)->tau[tid];
    __syncthreads();

    // ---- group weights w_c, slice sums of log w and routed counts ----------------------------
    float sl = 0.f;
    int cn = 0;
    const float inv_g = 1.f / G;
    for (int c = tid; c < nloc; c += kThr) {
        float a = 0.f;
        for (int h = 0; h < G; ++h) {
            const float u = xsm[h * per + c] - tau[h];
            a += u > 0.f ? ent_pow(u, p, mode) : 0.f;
        }
        const float w = a * inv_g;
        xsm[c] = w;   // row 0 is only read by this thread from here on
        if (w > 0.f) { sl += __logf(w); ++cn; }
    }
    sl = warp_sum(sl);
    cn = warp_isum(cn);
    if (lane == 0) { wsum[warp] = cn; fsum[warp] = sl; }
    __syncthreads();
    if (tid == 0) {
        int tot = 0;
        float a = 0.f;
        for (int k = 0; k < kThr / 32; ++k) { tot += wsum[k]; a += fsum[k]; }
        cx.cnt = tot;
        cx.slog = a;
    }
    cl.sync();
    // the 8 blocks' sums, fetched in parallel (lane k reads block k) and added in rank order
    float tot_log = 0.f;
    int tot_cnt = 0, before = 0;
    {
        float ls = 0.f;
        int lc = 0;
        if (lane < kRanks) {
            const Cross* o = cl.map_shared_rank(&cx, lane);
            ls = o->slog;
            lc = o->cnt;
        }
        for (int k = 0; k < kRanks; ++k) {
            const float a = __shfl_sync(0xffffffffu, ls, k);
            const int c = __shfl_sync(0xffffffffu, lc, k);
            tot_log += a;
            tot_cnt += c;
            if (k < rank) before += c;
        }
    }
    const float mu = tot_cnt > 0 ? tot_log / tot_cnt : 0.f;

    // ---- ascending compaction of this slice at offset `before` --------------------------------
    int* idx = rt.idx + (long long)br * rt.cap;
    float* bias = rt.bias + (long long)br * rt.cap;
    uint32_t* mrow = rt.bitmask ? rt.bitmask + (long long)br * rt.words : nullptr;
    int base = before;
    for (int c0 = 0; c0 < nloc; c0 += kThr) {
        const int c = c0 + tid;
        const float w = c < nloc ? xsm[c] : 0.f;
        const bool on = w > 0.f;
        const uint32_t m = __ballot_sync(0xffffffffu, on);
        __syncthreads();
        if (lane == 0) wsum[warp] = __popc(m);
        __syncthreads();
        if (tid == 0) {
            int acc = 0;
            for (int k = 0; k < kThr / 32; ++k) { const int v = wsum[k]; wsum[k] = acc; acc += v; }
            wsum[kThr / 32] = acc;
        }
        __syncthreads();
        if (on) {
            const int k = base + wsum[warp] + __popc(m & ((1u << lane) - 1u));
            idx[k] = c_lo + c;
            bias[k] = (__logf(w) - mu) * s.inv_sigma;
        }
        if (mrow && lane == 0 && c0 + 32 * warp < nloc) mrow[(c_lo + c0 + 32 * warp) >> 5] = m;
        base += wsum[kThr / 32];
    }
    if (rank == 0) {
        if (tid == 0) rt.counts[br] = tot_cnt;
        if (mrow)
            for (int wd = ((nv + 31) >> 5) + tid; wd < rt.words; wd += kThr) mrow[wd] = 0u;
    }
    cl.sync();   // no block leaves while another may still read its shared memory
}

template <typename T, int D>
cudaError_t launch_t(const Shape& s, const void* q, const float* kbar, int kbar_T, const int* seqlens,
                     const Routes& rt, int* status, cudaStream_t st)
{
    const int per = dec_route_cluster_per(kbar_T);
    const size_t smem = route_cluster_smem(s.g, per);
    auto k = dec_route_cluster_kernel<T, D>;
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_after(k, dim3(kRanks * s.batch * s.hkv), dim3(kThr), smem, st, s, (const T*)q, kbar, kbar_T,
                        seqlens, rt, per, status);
}

}  // namespace

int dec_route_cluster_per(int kbar_T)
{
    const int per = (kbar_T + kRanks - 1) / kRanks;
    return per > 0 ? (per + 31) / 32 * 32 : 32;
}

bool dec_route_cluster_supported(const Shape& s, int kbar_T)
{
    if (s.g < 1 || s.g > kMaxG || (s.d != 64 && s.d != 128)) return false;
    const size_t smem = route_cluster_smem(s.g, dec_route_cluster_per(kbar_T));
    return smem + sizeof(float) * kMaxG * s.d + 1024 <= 227 * 1024;
}

cudaError_t launch_route_decode_cluster(const Shape& s, int dtype, const void* q, const float* kbar, int kbar_T,
                                        const int* seqlens, const Routes& rt, int* status, cudaStream_t st)
{
    if (dtype == DASH_BF16)
        return s.d == 128 ? launch_t<__nv_bfloat16, 128>(s, q, kbar, kbar_T, seqlens, rt, status, st)
                          : launch_t<__nv_bfloat16, 64>(s, q, kbar, kbar_T, seqlens, rt, status, st);
    return s.d == 128 ? launch_t<float, 128>(s, q, kbar, kbar_T, seqlens, rt, status, st)
                      : launch_t<float, 64>(s, q, kbar, kbar_T, seqlens, rt, status, st);
}

}  // namespace dash
