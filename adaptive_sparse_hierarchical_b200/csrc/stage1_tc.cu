// stage1_tc.cu -- Stage 1 routing for prefill on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// DashAttention (xllm-io paper review, section 3, Eq. 6 and the "Stage 1" kernel row: the row of
// chunk logits is kept on chip, the entmax threshold is solved in place, the GQA group is
// averaged, then the support is pruned):
//   x_c^(h) = (alpha-1) gamma <q_i^(h), kbar_c>/sqrt(d)  for c < floor(i/B)
//   what^(h) = [x^(h) - tau^(h)]_+^{1/(alpha-1)},  w = mean over the group,  R = {w > 0}
//   bias_c = (log w_c - mean_{c' in R} log w_c') / sigma                       (Prop. 4.1)
//
// One block = 128 query rows = (128/g positions) x (g heads) of one (sequence, KV head).
//   warp 0     TMA: the Q tile once, then 128-chunk tiles of the three exact bf16 planes of the
//              summaries (hi + mid + lo = kbar) into a 3-stage ring, one plane per stage
//   warp 1     allocates TMEM and issues, from one thread, X[:, tile] += Q . plane^T for the
//              three planes (M=128, N=128, K=16 steps), so X holds the fp32 logits of every
//              visible chunk, one row per TMEM lane
//   warps 2-17 four warps per TMEM lane quarter (32 rows), each reading every fourth 32-column
//              piece of its rows: max, Newton steps on f(t)^(alpha-1) and the head weights, the
//              partial sums of a row combined in shared memory in a fixed order (the passes are
//              warp-uniform because tcgen05.ld is a warp instruction); the g rows of a position
//              are g neighbouring lanes, summed by a shuffle reduce-scatter into shared memory;
//              then one warp per position writes the ascending route list (mean log weight,
//              bias, bitmask).
// Every mbarrier wait is bounded; on time-out the block records an error code and leaves.
#include <climits>
#include <cudaTypedefs.h>

#include "dash_common.cuh"
#include "entmax.cuh"
#include "tc_ptx.cuh"

namespace dash {

namespace {

constexpr int kR = 128, kCT = 128, kDd = 128;
constexpr int kQB = kR * kDd * 2;               // Q tile, two 16 KB d-halves
constexpr int kPlaneHalf = kCT * 64 * 2;        // [128 chunks][64 d] bf16 = 16 KB
constexpr int kStage = 2 * kPlaneHalf;          // one plane of a tile, two d-halves = 32 KB
constexpr int kNS = 3;                          // ring stages
constexpr int kOffQ1 = 0, kOffRing = kQB, kOffW = kOffRing + kNS * kStage;
constexpr int kCand = 48;   // candidate list length per row and warp: 16 x 32 x 48 floats fill the ring
static_assert(16 * 32 * kCand * 4 <= kNS * kStage && kCand % 4 == 0, "candidate lists must fit the ring");
static_assert(16 + 16 * kNS + 8 <= 96, "barriers below the TMEM slot");
constexpr int kMisc = 128 + 3 * 4 * kR * 16;    // barriers, TMEM slot, abort flag, reduction slots
// one M = 128, N = 128 MMA per (tile, plane, 16-wide k step): narrower MMAs accumulating into one
// tile form dependent chains that run well below the tensor rate
constexpr uint32_t kIdescX = tc::idesc_bf16(128, kCT, false, false);

// Sum over the g neighbouring lanes of a position of 32 values, reduce-scattered: afterwards
// lane (h = lane % g) holds the sums of the 32/g columns starting at *off.
template <int G>
__device__ __forceinline__ void group_reduce_scatter(float (&v)[32], int lane, int* off)
{
    int o = 0;
    int width = 32;
#pragma unroll
    for (int st = 1; st < G; st <<= 1) {
        const int half = width >> 1;
        const bool hi = (lane & st) != 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (j < half) {
                const float send = hi ? v[j] : v[half + j];
                const float keep = hi ? v[half + j] : v[j];
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, st);
            }
        }
        if (hi) o += half;
        width = half;
    }
    *off = o;
}

template <int G>
__global__ void __launch_bounds__(576, 1) route_prefill_tcgen05_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                       const __grid_constant__ CUtensorMap tmP,
                                                                       Shape s, Routes rt, int Tw, int* err)
{
    extern __shared__ char smem_raw[];
    char* sm = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = tc::smem_addr(sm);
    constexpr int P = kR / G;
    float* wbuf = reinterpret_cast<float*>(sm + kOffW);            // [P][Tw] group sums of the head weights
    char* misc = sm + kOffW + P * Tw * 4;
    float4* red = reinterpret_cast<float4*>(misc + 128);          // [3][4][kR] partial solve sums / max
    const uint32_t bar0 = tc::smem_addr(misc);
    const uint32_t q_full = bar0, x_ready = bar0 + 8;
    const uint32_t full0 = bar0 + 16, empty0 = bar0 + 16 + 8 * kNS;   // [kNS] each
    const uint32_t drain = bar0 + 16 + 16 * kNS;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + 96);
    volatile int* abort = reinterpret_cast<volatile int*>(misc + 100);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nblk = (s.n + P - 1) / P;
    const int br = blockIdx.x % (s.batch * s.hkv);
    const int pb = nblk - 1 - blockIdx.x / (s.batch * s.hkv);     // heaviest blocks first
    const int b = br / s.hkv, r = br % s.hkv;
    const int i0 = pb * P;
    const int ilast = min(i0 + P, s.n) - 1;
    const int nvmax = min(ilast / s.B, s.T);
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
    const int ntiles = (nvmax + kCT - 1) / kCT;
    uint32_t ncols = 32;
    while (ncols < (uint32_t)(ntiles * kCT)) ncols <<= 1;

    if (tid == 0) {
        tc::mbar_init(q_full, 1);
        tc::mbar_init(x_ready, 1);
        for (int k = 0; k < kNS; ++k) { tc::mbar_init(full0 + 8 * k, 1); tc::mbar_init(empty0 + 8 * k, 1); }
        tc::mbar_init(drain, 1);
        *abort = 0;
        tc::mbar_fence_init();
    }
    if (warp == 1) {
        __syncwarp();
        tc::tmem_alloc(tc::smem_addr(tmem_slot), ncols);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tc::prefetch_tmap(&tmQ);
            tc::prefetch_tmap(&tmP);
            tc::mbar_expect_tx(q_full, kQB);
            tc::tma_load_4d(base + kOffQ1, &tmQ, q_full, 0, r * G, i0, b);
            tc::tma_load_4d(base + kOffQ1 + kQB / 2, &tmQ, q_full, 64, r * G, i0, b);
            int last[kNS];
#pragma unroll
            for (int k = 0; k < kNS; ++k) last[k] = -1;
            bool pok = true;
            // one ring stage per (tile, plane); chunks past T read as zeros (never used)
            for (int gs = 0; pok && gs < 3 * ntiles; ++gs) {
                const int st = gs % kNS, t = gs / 3, pl = gs % 3;
                if (gs >= kNS && !tc::mbar_wait(empty0 + 8 * st, ((gs / kNS) - 1) & 1, abort, err, 21)) { pok = false; break; }
                last[st] = gs;
                const uint32_t dst = base + kOffRing + st * kStage, fb = full0 + 8 * st;
                tc::mbar_expect_tx(fb, kStage);
                tc::tma_load_4d(dst, &tmP, fb, 0, t * kCT, br * 3 + pl, 0);
                tc::tma_load_4d(dst + kPlaneHalf, &tmP, fb, 64, t * kCT, br * 3 + pl, 0);
            }
            if (*abort) {
                for (int k = 0; k < kNS; ++k)
                    if (last[k] >= 0)
                        for (long long it = 0; it < (1ll << 22); ++it)
                            if (tc::mbar_try(full0 + 8 * k, (last[k] / kNS) & 1)) break;
                for (long long it = 0; it < (1ll << 22); ++it)
                    if (tc::mbar_try(q_full, 0)) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // descriptors of the Q tile and ring stage 0; a stage / K-step moves only the start
            // address field (16-byte units, no carry), so each MMA is issued after one add
            const uint64_t dQ = tc::sw128_desc(base + kOffQ1, 16, 1024);
            const uint64_t dP0 = tc::sw128_desc(base + kOffRing, 16, 1024);
            bool ok = tc::mbar_wait(q_full, 0, abort, err, 22);
            for (int gs = 0; ok && gs < 3 * ntiles; ++gs) {
                const int st = gs % kNS, t = gs / 3, pl = gs % 3;
                if (!tc::mbar_wait(full0 + 8 * st, (gs / kNS) & 1, abort, err, 23)) { ok = false; break; }
                tc::fence_after_sync();
                const uint64_t dp = dP0 + (uint64_t)((st * kStage) >> 4);
                const uint32_t xd = tmem + t * kCT;
#pragma unroll
                for (int kk = 0; kk < kDd / 16; ++kk)
                    tc::mma_f16_ss(xd, dQ + (uint64_t)(((kk >> 2) * (kQB / 2) + (kk & 3) * 32) >> 4),
                                   dp + (uint64_t)(((kk >> 2) * kPlaneHalf + (kk & 3) * 32) >> 4), kIdescX,
                                   (pl > 0 || kk > 0) ? 1u : 0u);
                tc::mma_commit(empty0 + 8 * st);
            }
            if (ok) tc::mma_commit(x_ready);
            else {
                tc::mma_commit(drain);
                for (long long it = 0; it < (1ll << 22); ++it)
                    if (tc::mbar_try(drain, 0)) break;
            }
        }
    } else {
        // ---- four warps per 32 rows: warp (2 + 4 cq + q) reads TMEM lanes 32 (warp % 4) .. +31
        // and the column pieces pc with pc % 4 == cq; partial max / f / f' of a row are combined
        // through shared memory in a fixed order, so the four warps take identical Newton steps
        const int q4 = warp & 3, cq = (warp - 2) >> 2;
        const int row = q4 * 32 + lane;
        const int pl = row / G;
        const int i = i0 + pl;
        const int nv = i < s.n ? min(i / s.B, s.T) : 0;
        int nvw = nv;   // column bound, uniform over the warp and over the four warps of the rows
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) nvw = max(nvw, __shfl_xor_sync(0xffffffffu, nvw, o));
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        const float xs = (s.alpha - 1.f) * s.gamma * rsqrtf((float)kDd);
        const float p = 1.f / (s.alpha - 1.f);
        const int mode = s.alpha == 2.f ? 1 : s.alpha == 1.5f ? 2 : 0;
        tc::mbar_wait(x_ready, 0, abort, err, 24);
        asm volatile("bar.sync 1, 512;" ::: "memory");
        const bool ok = *abort == 0;   // same value in every worker: all waits ended before the barrier
        const uint32_t gbar = 2 + q4;
        auto group_sync = [&]() { asm volatile("bar.sync %0, 128;" ::"r"(gbar) : "memory"); };
        if (ok) {
            tc::fence_after_sync();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            const int npieces = (nvw + 31) / 32;
            auto load_piece = [&](int pc, float (&v)[32]) {
                tc::tmem_ld32(lane_base + pc * 32, v);
                tc::tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = pc * 32 + e < nv ? v[e] * xs : -INFINITY;
            };
            // row maximum
            float mx = -INFINITY;
            for (int pc = cq; pc < npieces; pc += 4) {
                float v[32];
                load_piece(pc, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) mx = fmaxf(mx, v[e]);
            }
            red[(2 * 4 + cq) * kR + row].x = mx;
            group_sync();
            mx = fmaxf(fmaxf(red[(2 * 4 + 0) * kR + row].x, red[(2 * 4 + 1) * kR + row].x),
                       fmaxf(red[(2 * 4 + 2) * kR + row].x, red[(2 * 4 + 3) * kR + row].x));
            // entries at or below max - 1 never enter the support (tau >= max - 1): each thread
            // copies the others of its pieces into a list in shared memory (over the Q / plane
            // ring, idle once X is complete; entry k of lane l at [k][l]), padded with -inf to a
            // multiple of four; a warp whose rows overflow kCand keeps reading TMEM instead
            float lo = mx - 1.f;
            float* cl = reinterpret_cast<float*>(sm + kOffRing) + (warp - 2) * kCand * 32 + lane;
            int m = 0;
            for (int pc = cq; pc < npieces; pc += 4) {
                float v[32];
                load_piece(pc, v);
                uint32_t mask = 0u;
#pragma unroll
                for (int e = 0; e < 32; ++e) mask |= (v[e] > lo ? 1u : 0u) << e;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int k = m + __popc(mask & ((1u << e) - 1u));
                    if (((mask >> e) & 1u) && k < kCand) cl[k * 32] = v[e];
                }
                m += __popc(mask);
            }
            const bool listed = __all_sync(0xffffffffu, m <= kCand);
            const int m4 = (m + 3) >> 2;
            for (int k = m; k < 4 * m4 && k < kCand; ++k) cl[k * 32] = -INFINITY;
            // the solve from t = max - 1 (entmax.cuh, ent_step: Newton on f^(alpha-1), closed-form
            // finish for alpha = 2 and 1.5); every lane keeps stepping until the whole warp is done
            float hi = nv > 0 ? mx - exp2f(-(s.alpha - 1.f) * __log2f((float)nv)) : 0.f;
            float t = lo;
            bool done = nv == 0;
            for (int it = 0; it < 32 && !__all_sync(0xffffffffu, done); ++it) {
                EntSums S = ent_zero();
                if (listed && mode == 2) {
#pragma unroll 2
                    for (int k = 0; k < m4; ++k) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float u = cl[(4 * k + j) * 32] - t;
                            const float up = fmaxf(u, 0.f);
                            S.f = fmaf(up, up, S.f);
                            S.fd += up;
                            S.n += u > 0.f ? 1.f : 0.f;
                            S.um = fminf(S.um, u > 0.f ? u : INFINITY);
                        }
                    }
                } else if (listed) {
                    for (int k = 0; k < 4 * m4; ++k) ent_add(S, cl[k * 32] - t, p, mode);
                } else {
                    for (int pc = cq; pc < npieces; pc += 4) {
                        float v[32];
                        load_piece(pc, v);
#pragma unroll
                        for (int e = 0; e < 32; ++e) ent_add(S, v[e] - t, p, mode);
                    }
                }
                float4* slot = red + (it & 1) * 4 * kR;
                slot[cq * kR + row] = make_float4(S.f, S.fd, S.n, S.um);
                group_sync();
                const float4 r0 = slot[row], r1 = slot[kR + row], r2 = slot[2 * kR + row], r3 = slot[3 * kR + row];
                S.f = (r0.x + r1.x) + (r2.x + r3.x);
                S.fd = (r0.y + r1.y) + (r2.y + r3.y);
                S.n = (r0.z + r1.z) + (r2.z + r3.z);
                S.um = fminf(fminf(r0.w, r1.w), fminf(r2.w, r3.w));
                if (!done) done = ent_step(S, t, lo, hi, s.alpha, mode);
            }
            // head weights of this warp's pieces, summed over the position's g lanes, into wbuf
            for (int pc = cq; pc < npieces; pc += 4) {
                float v[32];
                load_piece(pc, v);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float u = v[e] - t;
                    v[e] = u > 0.f ? ent_pow(u, p, mode) : 0.f;
                }
                int off;
                group_reduce_scatter<G>(v, lane, &off);
#pragma unroll
                for (int j = 0; j < 32 / G; ++j) wbuf[pl * Tw + pc * 32 + off + j] = v[j];
            }
        }
        asm volatile("bar.sync 1, 512;" ::: "memory");
        if (ok) {
            // one warp per position: GQA average, bias and the ordered route list
            for (int pp = warp - 2; pp < P; pp += 16) {
                const int ip = i0 + pp;
                if (ip >= s.n) continue;
                const int nvp = min(ip / s.B, s.T);
                const float* W = wbuf + pp * Tw;
                const float inv_g = 1.f / G;
                float slog = 0.f;
                int cnt = 0;
                for (int c = lane; c < nvp; c += 32) {
                    const float w = W[c] * inv_g;
                    if (w > 0.f) { slog += __logf(w); ++cnt; }
                }
                slog = warp_sum(slog);
                cnt = warp_isum(cnt);
                const float mu = cnt > 0 ? slog / cnt : 0.f;
                const long long toff = tri_offset(ip, s.B);
                uint32_t* mrow = bm ? bm + (long long)ip * rt.words : nullptr;
                int basec = 0;
                for (int c0 = 0; c0 < nvp; c0 += 32) {
                    const int c = c0 + lane;
                    const float w = c < nvp ? W[c] * inv_g : 0.f;
                    const bool on = w > 0.f;
                    const uint32_t m = __ballot_sync(0xffffffffu, on);
                    if (on) {
                        const int k = basec + __popc(m & ((1u << lane) - 1u));
                        idx[toff + k] = c;
                        bias[toff + k] = (__logf(w) - mu) * s.inv_sigma;
                    }
                    if (mrow && lane == 0) mrow[c0 >> 5] = m;
                    basec += __popc(m);
                }
                if (mrow)
                    for (int wd = ((nvp + 31) >> 5) + lane; wd < rt.words; wd += 32) mrow[wd] = 0u;
                if (lane == 0) counts[ip] = basec;
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, ncols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_r()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

template <int G>
cudaError_t launch_g(const Shape& s, const void* Q, const __nv_bfloat16* planes, const Routes& rt, int* err,
                     cudaStream_t st)
{
    auto fn = encode_fn_r();
    if (!fn) return cudaErrorInvalidValue;
    constexpr int P = kR / G;
    CUtensorMap mq, mp;
    {
        cuuint64_t dims[4] = {128, (cuuint64_t)s.hq, (cuuint64_t)s.n, (cuuint64_t)s.batch};
        cuuint64_t strides[3] = {(cuuint64_t)s.qs[2] * 2, (cuuint64_t)s.qs[1] * 2, (cuuint64_t)s.qs[0] * 2};
        if (s.batch == 1) strides[2] = strides[1] * (cuuint64_t)s.n;
        cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)P, 1};
        cuuint32_t es[4] = {1, 1, 1, 1};
        if (fn(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(Q), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        // planes [b*hkv*3][T][128] viewed as (d, chunk, plane-row, 1)
        cuuint64_t dims[4] = {128, (cuuint64_t)s.T, (cuuint64_t)s.batch * s.hkv * 3, 1};
        cuuint64_t strides[3] = {128 * 2, (cuuint64_t)s.T * 128 * 2, (cuuint64_t)s.T * 128 * 2 * s.batch * s.hkv * 3};
        cuuint32_t box[4] = {64, (cuuint32_t)kCT, 1, 1};   // 128 chunks x 64 d
        cuuint32_t es[4] = {1, 1, 1, 1};
        if (fn(&mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<__nv_bfloat16*>(planes), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const int Tw = (s.T + 31) / 32 * 32;
    const size_t smem = 1024 + kOffW + (size_t)P * Tw * 4 + kMisc;
    auto k = route_prefill_tcgen05_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long nblk = (s.n + P - 1) / P;
    const unsigned grid = (unsigned)(nblk * s.batch * s.hkv);
    if (grid == 0) return cudaSuccess;
    k<<<grid, 576, smem, st>>>(mq, mp, s, rt, Tw, err);
    return cudaGetLastError();
}

}  // namespace

bool route_tcgen05_supported(const Shape& s, int dtype)
{
    if (dtype != DASH_BF16 || s.d != 128 || s.T > 512 || s.T < 1) return false;
    if (!(s.g == 1 || s.g == 2 || s.g == 4 || s.g == 8 || s.g == 16)) return false;
    const int P = kR / s.g, Tw = (s.T + 31) / 32 * 32;
    return 1024 + kOffW + (size_t)P * Tw * 4 + kMisc <= 227 * 1024 && encode_fn_r() != nullptr;
}

cudaError_t launch_route_prefill_tcgen05(const Shape& s, const void* Q, const __nv_bfloat16* planes, const Routes& rt,
                                         int* err, cudaStream_t st)
{
    switch (s.g) {
    case 1: return launch_g<1>(s, Q, planes, rt, err, st);
    case 2: return launch_g<2>(s, Q, planes, rt, err, st);
    case 4: return launch_g<4>(s, Q, planes, rt, err, st);
    case 8: return launch_g<8>(s, Q, planes, rt, err, st);
    default: return launch_g<16>(s, Q, planes, rt, err, st);
    }
}

}  // namespace dash
