// stage1_tc_long.cu -- Stage 1 routing for prefill on tcgen05 when a row has more chunk logits
// than tensor memory holds (T > 512 chunks).
//
// DashAttention (xllm-io paper review, section 3, Eq. 6 and Prop. 4.1), as in stage1_tc.cu:
//   x_c^(h) = (alpha-1) gamma <q_i^(h), kbar_c>/sqrt(d) for c < floor(i/B),
//   what^(h) = [x^(h) - tau^(h)]_+^{1/(alpha-1)},  w = mean over the group,  R = {w > 0},
//   bias_c = (log w_c - mean_R log w)/sigma.
//
// One block = 128 query rows = (128/g positions) x (g heads) of one (sequence, KV head).  The
// logits X = Q k̄^T stream through two 256-column halves of TMEM in blocks of 256 chunks
// (three exact bf16 planes of k̄, TMA-staged), three times: pass 0 takes each row's maximum,
// pass 1 copies the entries above (max - 1) -- the only ones the support can reach -- into
// per-thread lists in shared memory, Newton on f^(alpha-1) then runs on the lists, and pass 2
// forms the head weights, sums them over the g heads of each position and writes the block's
// routed chunks (ascending) with log w; the bias is fixed up with the mean once all blocks are
// written.  The MMAs of one block overlap the processing of the previous one.  A block whose
// lists overflow flags its tile in `redo` and writes nothing; the per-shape routing kernels
// then recompute the flagged tiles.
// Roles (18 warps): warp 0 TMA producer, warp 1 TMEM allocation + MMA issue, warps 2-17 four
// warps per TMEM lane quarter (32 rows), each reading every fourth 32-column piece of a block.
// Every mbarrier wait is bounded; on time-out the block records an error code and leaves.
#include <climits>
#include <cudaTypedefs.h>

#include "dash_common.cuh"
#include "tc_ptx.cuh"

namespace dash {

namespace {

constexpr int kR = 128, kCT = 64, kDd = 128;
constexpr int kPlaneHalf = kCT * 64 * 2;        // [64 chunks][64 d] bf16 = 8 KB
constexpr int kStage = 2 * kPlaneHalf;          // one plane of a tile, two d-halves = 16 KB
constexpr int kNS = 4;                          // ring stages
constexpr int kBW = 192;                        // chunks per block = columns of a TMEM half
constexpr int kTPB = kBW / kCT;                 // 64-chunk tiles per block
constexpr int kPieces = kBW / 32;               // 32-column pieces per block
// TMEM: X halves at columns [0, 192) and [192, 384); the Q tile (the MMAs' A operand, 128 rows x
// 128 bf16, two per 32-bit column) at [384, 448)
constexpr int kColQ = 2 * kBW;
constexpr int kOffRing = 0, kOffLists = kOffRing + kNS * kStage;
constexpr uint32_t kIdescX = tc::idesc_bf16(128, 64, false, false);
// after every pass but the first the workers post whether another pass over the blocks follows
// (kPlanGo) or not (kPlanStop); at most kMaxExtract extraction passes per set of rows in play
constexpr int kPlanStop = 0, kPlanGo = 1;
constexpr int kMaxExtract = 2;

// candidate list entries per (worker warp, lane); the lists also hold the weights buffer
// [P][kBW] of the emission pass (the lists are dead by then)
constexpr int kCap = 72;
constexpr int kOffMisc = kOffLists + 16 * 32 * kCap * 4;
// misc: barriers (kBarBytes), tmem slot / abort / overflow / plan (16 B), red [3][4][kR] float2
// (12 KB), per position: running log-sum, count, list base (3 x 32 words)
constexpr int kBarBytes = 8 * (1 + 2 * kNS + 2 + 2 + 2);   // q_full, full/empty ring, x_ready/x_free, drain, dec
constexpr int kMiscBase = (kBarBytes + 15) / 16 * 16;
constexpr int kMiscBytes = kMiscBase + 16 + 3 * 4 * kR * 8 + 3 * 32 * 4;
constexpr size_t kLongSmem = 1024 + kOffMisc + kMiscBytes;
static_assert(kLongSmem <= 227 * 1024, "shared memory of the long-row routing kernel");
static_assert((kR / 4) * kBW * 4 <= 16 * 32 * kCap * 4, "weights buffer inside the lists");

__device__ __forceinline__ float pw(float u, float p, int mode)
{
    return mode == 1 ? u : mode == 2 ? u * u : exp2f(p * __log2f(u));
}
__device__ __forceinline__ float dpw(float u, float p, int mode)
{
    return mode == 1 ? 1.f : mode == 2 ? u : exp2f((p - 1.f) * __log2f(u));
}

// Lower bound on the root of f_S(t) = sum_{x in S} [x - t]_+^p = 1 over a subset S of a row's
// logits: this thread's list (entry k at cl[32 k], m entries) and three more values (the other
// column sets' maxima).  f_S <= f everywhere, so that root is itself a lower bound on the row's
// tau.  g = f_S^(alpha-1) is convex and decreasing (a p-norm of the [x - t]_+), so Newton steps
// on g taken from a point left of its root stay left of it: three steps from t0 (where f_S >= 1)
// give a bound good enough to cut a list; -inf when f_S(t0) < 1 (nothing to gain).
__device__ __noinline__ float subset_bound(const float* cl, int m, float om0, float om1, float om2, float t0,
                                           float p, int mode, float am1)
{
    float t = t0;
    for (int it = 0; it < 3; ++it) {
        float f = 0.f, fd = 0.f;
        for (int k = 0; k < m; ++k) {
            const float u = cl[32 * k] - t;
            if (u > 0.f) { f += pw(u, p, mode); fd += dpw(u, p, mode); }
        }
        const float om[3] = {om0, om1, om2};
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const float u = om[j] - t;
            if (u > 0.f) { f += pw(u, p, mode); fd += dpw(u, p, mode); }
        }
        if (f < 1.f) return it == 0 ? -INFINITY : t;
        if (!(fd > 0.f)) break;
        const float gg = mode == 2 ? sqrtf(f) : mode == 1 ? f : exp2f(am1 * __log2f(f));
        const float tn = t + (gg - 1.f) * f / (gg * fd);
        if (!(tn > t)) break;
        t = tn;
    }
    return t;
}

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
__global__ void __launch_bounds__(576, 1) route_prefill_long_kernel(const __grid_constant__ CUtensorMap tmP,
                                                                    const __nv_bfloat16* __restrict__ Q,
                                                                    Shape s, Routes rt, unsigned char* redo,
                                                                    int* err)
{
    extern __shared__ char smem_raw[];
    char* sm = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = tc::smem_addr(sm);
    constexpr int P = kR / G, CAP = kCap;
    float* lists = reinterpret_cast<float*>(sm + kOffLists);            // [16 warps][CAP][32 lanes]
    float* wbuf = lists;                                                // [P][kBW] group sums of one block
    char* misc = sm + kOffMisc;
    const uint32_t bar0 = tc::smem_addr(misc);
    const uint32_t q_full = bar0, full0 = bar0 + 8, empty0 = full0 + 8 * kNS;   // ring [kNS] each
    const uint32_t x_ready0 = empty0 + 8 * kNS, x_free0 = x_ready0 + 16;       // TMEM halves [2] each
    const uint32_t drain = x_free0 + 16;
    const uint32_t dec = drain + 8;                                             // pass decisions
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + kMiscBase);
    volatile int* abort = reinterpret_cast<volatile int*>(misc + kMiscBase + 4);
    int* overflow = reinterpret_cast<int*>(misc + kMiscBase + 8);
    volatile int* plan_word = reinterpret_cast<volatile int*>(misc + kMiscBase + 12);
    float2* red = reinterpret_cast<float2*>(misc + kMiscBase + 16);                  // [3][4][kR]
    float* pslog = reinterpret_cast<float*>(misc + kMiscBase + 16 + 3 * 4 * kR * 8);  // [P] log-sum so far
    int* pcnt = reinterpret_cast<int*>(pslog + 32);                        // [P] entries so far

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntile128 = (s.n + P - 1) / P;
    const int br = blockIdx.x % (s.batch * s.hkv);
    const int pb = ntile128 - 1 - blockIdx.x / (s.batch * s.hkv);     // heaviest blocks first
    const int b = br / s.hkv, r = br % s.hkv;
    const int i0 = pb * P;
    const int ilast = min(i0 + P, s.n) - 1;
    const int nvmax = min(ilast / s.B, s.T);
    int* counts = rt.counts + (long long)br * s.n;
    int* idx = rt.idx + (long long)br * rt.cap;
    float* bias = rt.bias + (long long)br * rt.cap;
    uint32_t* bm = rt.bitmask ? rt.bitmask + (long long)br * s.n * rt.words : nullptr;
    unsigned char* my_redo = redo + (long long)br * ntile128 + pb;
    if (nvmax == 0) {
        if (tid == 0) *my_redo = 0;
        for (int p = tid; p < P && i0 + p < s.n; p += blockDim.x) counts[i0 + p] = 0;
        if (bm)
            for (int k = tid; k < P * rt.words; k += blockDim.x)
                if (i0 + k / rt.words < s.n) bm[(long long)i0 * rt.words + k] = 0u;
        return;
    }
    const int ntiles = (nvmax + kCT - 1) / kCT;
    const int nbk = (ntiles + kTPB - 1) / kTPB;   // 256-chunk blocks

    if (tid == 0) {
        tc::mbar_init(q_full, 128);   // the four warps that write the Q rows into TMEM
        for (int k = 0; k < kNS; ++k) {
            tc::mbar_init(full0 + 8 * k, 1);
            tc::mbar_init(empty0 + 8 * k, 1);
        }
        for (int k = 0; k < 2; ++k) {
            tc::mbar_init(x_ready0 + 8 * k, 1);
            tc::mbar_init(x_free0 + 8 * k, 512);
        }
        tc::mbar_init(drain, 1);
        tc::mbar_init(dec, 1);
        *abort = 0;
        *overflow = 0;
        tc::mbar_fence_init();
    }
    if (tid < P) { pslog[tid] = 0.f; pcnt[tid] = 0; }
    if (warp == 1) {
        __syncwarp();
        tc::tmem_alloc(tc::smem_addr(tmem_slot), 512);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---- TMA producer: Q once, then the plane tiles of every block, once per pass ----------
        if (lane == 0) {
            tc::prefetch_tmap(&tmP);
            int last[kNS];
#pragma unroll
            for (int j = 0; j < kNS; ++j) last[j] = -1;
            int gs = 0;   // ring stage counter: one stage per (tile, plane)
            bool pok = true;
            for (int k = 0; pok; ++k) {
                for (int t = 0; pok && t < ntiles; ++t) {
                    for (int pl = 0; pl < 3; ++pl, ++gs) {
                        const int st = gs % kNS;
                        if (gs >= kNS && !tc::mbar_wait(empty0 + 8 * st, ((gs / kNS) - 1) & 1, abort, err, 31)) { pok = false; break; }
                        last[st] = gs;
                        const uint32_t dst = base + kOffRing + st * kStage, fb = full0 + 8 * st;
                        tc::mbar_expect_tx(fb, kStage);
                        tc::tma_load_4d(dst, &tmP, fb, 0, t * kCT, br * 3 + pl, 0);
                        tc::tma_load_4d(dst + kPlaneHalf, &tmP, fb, 64, t * kCT, br * 3 + pl, 0);
                    }
                }
                if (!pok || k == 0) continue;
                // the workers' decision after pass k
                if (!tc::mbar_wait(dec, (k - 1) & 1, abort, err, 36)) break;
                if (*plan_word == kPlanStop) break;
            }
            if (*abort) {
                for (int j = 0; j < kNS; ++j)
                    if (last[j] >= 0)
                        for (long long it = 0; it < (1ll << 22); ++it)
                            if (tc::mbar_try(full0 + 8 * j, (last[j] / kNS) & 1)) break;
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer: TMEM half u & 1 takes the u-th block of the pass sequence ------------
        if (lane == 0) {
            const uint64_t dP0 = tc::sw128_desc(base + kOffRing, 16, 1024);
            bool ok = tc::mbar_wait(q_full, 0, abort, err, 32);
            int gs = 0, u = 0;
            for (int k = 0; ok; ++k) {
                for (int kb = 0; ok && kb < nbk; ++kb, ++u) {
                    const int hlf = u & 1;
                    // the half's previous use (u - 2) has been read by every worker
                    if (u >= 2 && !tc::mbar_wait(x_free0 + 8 * hlf, ((u >> 1) - 1) & 1, abort, err, 33)) { ok = false; break; }
                    for (int t = kb * kTPB; ok && t < min(ntiles, (kb + 1) * kTPB); ++t) {
                        const uint32_t xd = tmem + hlf * kBW + (t - kb * kTPB) * kCT;
                        for (int pl = 0; pl < 3; ++pl, ++gs) {
                            const int st = gs % kNS;
                            if (!tc::mbar_wait(full0 + 8 * st, (gs / kNS) & 1, abort, err, 34)) { ok = false; break; }
                            tc::fence_after_sync();
                            const uint64_t dp = dP0 + (uint64_t)((st * kStage) >> 4);
#pragma unroll
                            for (int kk = 0; kk < kDd / 16; ++kk)
                                tc::mma_f16_ts(xd, tmem + kColQ + kk * 8,
                                               dp + (uint64_t)(((kk >> 2) * kPlaneHalf + (kk & 3) * 32) >> 4),
                                               kIdescX, (pl > 0 || kk > 0) ? 1u : 0u);
                            tc::mma_commit(empty0 + 8 * st);
                        }
                    }
                    if (ok) tc::mma_commit(x_ready0 + 8 * hlf);
                }
                if (!ok || k == 0) continue;
                if (!tc::mbar_wait(dec, (k - 1) & 1, abort, err, 37)) break;
                if (*plan_word == kPlanStop) break;
            }
            // every MMA this thread issued completes before TMEM is released
            tc::mma_commit(drain);
            for (long long it = 0; it < (1ll << 22); ++it)
                if (tc::mbar_try(drain, 0)) break;
        }
    } else {
        // ---- workers: four warps per TMEM lane quarter; warp (q4, cq) takes pieces lp % 4 == cq of
        // each 256-column block (two of its eight 32-column pieces) -----------------------------
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
        const uint32_t gbar = 2 + q4;
        auto group_sync = [&]() { asm volatile("bar.sync %0, 128;" ::"r"(gbar) : "memory"); };
        auto workers_sync = [&]() { asm volatile("bar.sync 1, 512;" ::: "memory"); };
        // true in every worker iff pred holds in every worker (named barrier 6 over the 512 workers)
        auto workers_all = [&](bool pred) {
            uint32_t rv;
            asm volatile("{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
                         "bar.red.and.pred po, 6, 512, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}\n"
                         : "=r"(rv)
                         : "r"((uint32_t)pred)
                         : "memory");
            return rv != 0;
        };
        // Lists: region (cq, q4) holds [CAP][32 lanes]; the regions of quarters q4 and q4 ^ 2 sit
        // side by side, so that with only half of the rows in play a thread's list runs on into
        // its idle partner's region (capacity 2 CAP).
        if (cq == 0) {
            // row (position i0 + row / g, head r g + row % g) of the Q tile into this lane of TMEM
            // columns [kColQ, kColQ + 64): the row's bf16 pairs are already the 32-bit columns
            uint4 qw[16];
            const __nv_bfloat16* qrow = Q + (long long)b * s.qs[0] + (long long)i * s.qs[1] + (long long)(r * G + row % G) * s.qs[2];
#pragma unroll
            for (int k = 0; k < 16; ++k)
                qw[k] = i < s.n ? __ldg(reinterpret_cast<const uint4*>(qrow) + k) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::tmem_st16(lane_base + kColQ + 16 * k, reinterpret_cast<const uint32_t*>(qw + 4 * k));
            tc::tmem_wait_st();
            tc::fence_before_sync();
            tc::mbar_arrive(q_full);
        }
        float* const own_list = lists + ((cq * 2 + (q4 & 1)) * 2 + (q4 >> 1)) * CAP * 32 + lane;
        float* const pair_list = lists + ((cq * 2 + (q4 & 1)) * 2) * CAP * 32 + lane;
        float* cl = own_list;   // this thread's list, entry k at cl[32 k]
        int cap = CAP;
        float mx = -INFINITY, lo = 0.f, t = 0.f;
        float hi = 0.f;
        float om[3] = {-INFINITY, -INFINITY, -INFINITY};   // the other three column sets' row maxima
        float lo_t = 0.f;   // this thread's list cut: lo, raised by its own subset bounds
        int m = 0;
        bool ok = true, emitted = false, redo_me = false;
        int kind = 0;   // pass kind: 0 row maximum, 1 candidate extraction, 2 weights and emission
        int half = -1;  // rows in play: all (-1), or the quarters q4 >> 1 == half
        int nextract = 0;
        for (int k = 0, u = 0;; ++k) {
            const bool active = half < 0 || (q4 >> 1) == half;
            for (int kb = 0; kb < nbk; ++kb, ++u) {
                const int hlf = u & 1;
                const bool got = ok && tc::mbar_wait(x_ready0 + 8 * hlf, (u >> 1) & 1, abort, err, 35);
                ok = workers_all(got);   // uniform: a time-out anywhere stops every worker together
                if (ok && active) {
                    tc::fence_after_sync();
                    // the pieces of this block whose global index (column / 32) is cq mod 4;
                    // column = kb * kBW + 32 lp + e
                    for (int lp = 0; lp < kPieces; ++lp) {
                        if ((kb * kPieces + lp) % 4 != cq) continue;
                        const int c0 = kb * kBW + lp * 32;
                        // columns past every row of the warp: never read (the g rows of a position
                        // sit in one warp, and the emission stops at the position's own bound)
                        if (c0 >= nvw) continue;
                        float v[32];
                        tc::tmem_ld32(lane_base + hlf * kBW + lp * 32, v);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = c0 + e < nv ? v[e] * xs : -INFINITY;
                        if (kind == 0) {
#pragma unroll
                            for (int e = 0; e < 32; ++e) mx = fmaxf(mx, v[e]);
                        } else if (kind == 1) {
                            // entries above the cut, compacted by prefix popcount (no serial chain)
                            uint32_t mask = 0u;
#pragma unroll
                            for (int e = 0; e < 32; ++e) mask |= (v[e] > lo_t ? 1u : 0u) << e;
                            if (m + __popc(mask) > cap && m <= cap) {
                                // list full: raise the cut to this thread's subset bound on tau
                                // (less the margin below) and drop the entries under it
                                const float tb = subset_bound(cl, m, om[0], om[1], om[2], lo_t, p, mode, s.alpha - 1.f);
                                const float cut = tb - 1e-3f * fmaxf(1.f, fabsf(tb));
                                if (cut > lo_t) {
                                    lo_t = cut;
                                    int j = 0;
                                    for (int kk = 0; kk < m; ++kk) {
                                        const float x = cl[32 * kk];
                                        if (x > cut) cl[32 * j++] = x;
                                    }
                                    m = j;
                                    mask = 0u;
#pragma unroll
                                    for (int e = 0; e < 32; ++e) mask |= (v[e] > lo_t ? 1u : 0u) << e;
                                }
                            }
                            if (mask) {
#pragma unroll
                                for (int e = 0; e < 32; ++e) {
                                    const int kk = m + __popc(mask & ((1u << e) - 1u));
                                    if (((mask >> e) & 1u) && kk < cap) cl[kk * 32] = v[e];
                                }
                                m += __popc(mask);
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                const float uu = v[e] - t;
                                v[e] = uu > 0.f ? pw(uu, p, mode) : 0.f;
                            }
                            int off;
                            group_reduce_scatter<G>(v, lane, &off);
#pragma unroll
                            for (int j = 0; j < 32 / G; ++j) wbuf[pl * kBW + lp * 32 + off + j] = v[j];
                        }
                    }
                }
                // TMEM half read: the MMAs of use u + 2 may overwrite it
                tc::fence_before_sync();
                tc::mbar_arrive(x_free0 + 8 * hlf);

                if (kind == 2 && ok) {
                    // ---- this block's routed chunks of each position in play: warp per position,
                    // ascending, log w for now (the bias needs the mean over all blocks) ---------
                    workers_sync();
                    for (int pp = warp - 2; pp < P; pp += 16) {
                        const int ip = i0 + pp;
                        if (ip >= s.n || (half >= 0 && ((pp * G) >> 6) != half)) continue;
                        const int nvp = min(ip / s.B, s.T);
                        const float* Wp = wbuf + pp * kBW;
                        const float inv_g = 1.f / G;
                        const long long toff = tri_offset(ip, s.B);
                        uint32_t* mrow = bm ? bm + (long long)ip * rt.words : nullptr;
                        int basec = pcnt[pp];
                        float slog = 0.f;
                        for (int j0 = 0; j0 < kBW; j0 += 32) {
                            const int c = kb * kBW + j0 + lane;
                            if (kb * kBW + j0 >= nvp) break;
                            const float w = c < nvp ? Wp[j0 + lane] * inv_g : 0.f;
                            const bool on = w > 0.f;
                            const uint32_t msk = __ballot_sync(0xffffffffu, on);
                            if (on) {
                                const int kk = basec + __popc(msk & ((1u << lane) - 1u));
                                const float lw = __logf(w);
                                idx[toff + kk] = c;
                                bias[toff + kk] = lw;
                                slog += lw;
                            }
                            if (mrow && lane == 0) mrow[c >> 5] = msk;
                            basec += __popc(msk);
                        }
                        slog = warp_sum(slog);
                        __syncwarp();
                        if (lane == 0) { pslog[pp] += slog; pcnt[pp] = basec; }
                        __syncwarp();
                    }
                    workers_sync();   // wbuf is rewritten by the next block
                }
            }
            if (kind == 0) {
                // row maximum over the four warps of the rows; the first lists start at max - 1
                // (tau >= max - 1: the largest entry alone already gives f(max - 1) >= 1)
                red[(2 * 4 + cq) * kR + row].x = mx;
                group_sync();
#pragma unroll
                for (int j = 0; j < 3; ++j) om[j] = red[(2 * 4 + ((cq + 1 + j) & 3)) * kR + row].x;
                mx = fmaxf(fmaxf(mx, om[0]), fmaxf(om[1], om[2]));
                lo = mx - 1.f;
                lo_t = lo;
                hi = nv > 0 ? mx - exp2f(-(s.alpha - 1.f) * __log2f((float)nv)) : 0.f;
                kind = 1;
                continue;   // an extraction pass always follows
            }
            bool stop = false;
            if (kind == 1) {
                // ---- after an extraction pass: threshold on the lists.  A list that overflowed
                // dropped entries, and the root on the entries kept is then a lower bound on tau
                // (a subset's f is smaller everywhere) from which the next extraction starts ------
                if (active && m > cap) atomicOr(overflow, 1);
                workers_sync();
                const bool over = *overflow != 0;
                ++nextract;
                if (ok && active) {
                    const int mm = min(m, cap);
                    const int m4 = (mm + 3) >> 2;
                    for (int kk = mm; kk < 4 * m4; ++kk) cl[kk * 32] = -INFINITY;
                    // every list holds all of its column set's entries above the largest of the
                    // four cuts (each cut is at most tau), so the solve starts there
                    red[(2 * 4 + cq) * kR + row].y = lo_t;
                    group_sync();
                    lo = fmaxf(fmaxf(red[(2 * 4 + 0) * kR + row].y, red[(2 * 4 + 1) * kR + row].y),
                               fmaxf(red[(2 * 4 + 2) * kR + row].y, red[(2 * 4 + 3) * kR + row].y));
                    // Newton on g(t) = f(t)^(alpha-1) from t = lo (see stage1.cu), the four warps'
                    // partial sums combined in a fixed order; every row of the quarter steps until
                    // all have converged (the group barriers stay matched)
                    float lo_n = lo, hi_n = hi;
                    t = lo;
                    bool done = nv == 0;
                    for (int it = 0; it < 32 && !__all_sync(0xffffffffu, done); ++it) {
                        float f = 0.f, fd = 0.f;
                        if (mode == 2) {
                            for (int kk = 0; kk < m4; ++kk) {
                                const float u0 = fmaxf(cl[(4 * kk) * 32] - t, 0.f), u1 = fmaxf(cl[(4 * kk + 1) * 32] - t, 0.f);
                                const float u2 = fmaxf(cl[(4 * kk + 2) * 32] - t, 0.f), u3 = fmaxf(cl[(4 * kk + 3) * 32] - t, 0.f);
                                f += u0 * u0 + u1 * u1 + u2 * u2 + u3 * u3;
                                fd += (u0 + u1) + (u2 + u3);
                            }
                        } else {
                            for (int kk = 0; kk < 4 * m4; ++kk) {
                                const float uu = cl[kk * 32] - t;
                                if (uu > 0.f) { f += pw(uu, p, mode); fd += dpw(uu, p, mode); }
                            }
                        }
                        float2* slot = red + (it & 1) * 4 * kR;
                        slot[cq * kR + row] = make_float2(f, fd);
                        group_sync();
                        const float2 r0 = slot[row], r1 = slot[kR + row], r2 = slot[2 * kR + row], r3 = slot[3 * kR + row];
                        f = (r0.x + r1.x) + (r2.x + r3.x);
                        fd = (r0.y + r1.y) + (r2.y + r3.y);
                        if (!done) {
                            if (f >= 1.f) lo_n = t; else hi_n = t;
                            float tn = 0.5f * (lo_n + hi_n);
                            if (fd > 0.f && f > 0.f) {
                                const float gg = mode == 2 ? sqrtf(f) : mode == 1 ? f : exp2f((s.alpha - 1.f) * __log2f(f));
                                tn = t + (gg - 1.f) * f / (gg * fd);
                            }
                            if (fabsf(tn - t) <= 2e-7f * fmaxf(1.f, fabsf(t)) || fabsf(f - 1.f) <= 1e-6f) { t = tn; done = true; }
                            else {
                                if (!(tn > lo_n && tn < hi_n)) tn = 0.5f * (lo_n + hi_n);
                                t = tn;
                            }
                        }
                    }
                    if (over) {
                        // the next lists keep the entries above the bound, less a margin far
                        // above the solve's rounding (f' at the root is at least 1/(alpha-1))
                        lo = fmaxf(lo, t - 1e-3f * fmaxf(1.f, fabsf(t)));
                    }
                }
                if (!ok) stop = true;
                else if (!over) kind = 2;
                else if (nextract < kMaxExtract) { lo_t = lo; m = 0; }
                else if (half < 0) {
                    // a column set holds more of the support than its list: redo the rows in two
                    // halves, each thread of the half in play taking its idle partner's list too
                    half = 0;
                    nextract = 0;
                    lo_t = lo;
                    m = 0;
                    cl = pair_list;
                    cap = 2 * CAP;
                } else { stop = true; redo_me = true; }
            } else {
                // ---- after a weights pass
                if (!ok) stop = true;
                else if (half == 0) { half = 1; kind = 1; nextract = 0; lo_t = lo; m = 0; }
                else { stop = true; emitted = true; }
            }
            workers_sync();   // every worker has read the overflow word
            if (tid == 64) {
                *overflow = 0;
                *plan_word = stop ? kPlanStop : kPlanGo;
                tc::mbar_arrive(dec);
            }
            if (stop) break;
        }
        // ---- bias = (log w - mean log w) / sigma over each position's list; counts; bitmask tail
        if (emitted) {
            for (int pp = warp - 2; pp < P; pp += 16) {
                const int ip = i0 + pp;
                if (ip >= s.n) continue;
                const int nvp = min(ip / s.B, s.T);
                const int cnt = pcnt[pp];
                const float mu = cnt > 0 ? pslog[pp] / cnt : 0.f;
                const long long toff = tri_offset(ip, s.B);
                for (int kk = lane; kk < cnt; kk += 32) bias[toff + kk] = (bias[toff + kk] - mu) * s.inv_sigma;
                uint32_t* mrow = bm ? bm + (long long)ip * rt.words : nullptr;
                if (mrow)
                    for (int wd = ((nvp + 31) >> 5) + lane; wd < rt.words; wd += 32) mrow[wd] = 0u;
                if (lane == 0) counts[ip] = cnt;
            }
        }
        if (tid == 64) *my_redo = (unsigned char)(redo_me ? 1 : 0);
    }
    // ---- teardown -----------------------------------------------------------------------------
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_l()
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
cudaError_t launch_long_g(const Shape& s, const void* Q, const __nv_bfloat16* planes, const Routes& rt,
                          unsigned char* redo, int* err, cudaStream_t st)
{
    auto fn = encode_fn_l();
    if (!fn) return cudaErrorInvalidValue;
    constexpr int P = kR / G;
    CUtensorMap mp;
    {
        // planes [b*hkv*3][T][128] viewed as (d, chunk, plane-row, 1)
        cuuint64_t dims[4] = {128, (cuuint64_t)s.T, (cuuint64_t)s.batch * s.hkv * 3, 1};
        cuuint64_t strides[3] = {128 * 2, (cuuint64_t)s.T * 128 * 2, (cuuint64_t)s.T * 128 * 2 * s.batch * s.hkv * 3};
        cuuint32_t box[4] = {64, (cuuint32_t)kCT, 1, 1};
        cuuint32_t es[4] = {1, 1, 1, 1};
        if (fn(&mp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<__nv_bfloat16*>(planes), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const size_t smem = kLongSmem;
    auto k = route_prefill_long_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long nblk = (s.n + P - 1) / P;
    const unsigned grid = (unsigned)(nblk * s.batch * s.hkv);
    if (grid == 0) return cudaSuccess;
    k<<<grid, 576, smem, st>>>(mp, static_cast<const __nv_bfloat16*>(Q), s, rt, redo, err);
    return cudaGetLastError();
}

}  // namespace

bool route_long_supported(const Shape& s, int dtype)
{
    if (dtype != DASH_BF16 || s.d != 128 || s.T <= 512) return false;
    if (!(s.g == 4 || s.g == 8 || s.g == 16)) return false;
    return encode_fn_l() != nullptr;
}

int route_long_positions(const Shape& s) { return kR / s.g; }

cudaError_t launch_route_prefill_long(const Shape& s, const void* Q, const __nv_bfloat16* planes, const Routes& rt,
                                      unsigned char* redo, int* err, cudaStream_t st)
{
    switch (s.g) {
    case 4: return launch_long_g<4>(s, Q, planes, rt, redo, err, st);
    case 8: return launch_long_g<8>(s, Q, planes, rt, redo, err, st);
    default: return launch_long_g<16>(s, Q, planes, rt, redo, err, st);
    }
}

}  // namespace dash
