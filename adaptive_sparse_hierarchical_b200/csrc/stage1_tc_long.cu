// stage1_tc_long.cu -- Stage 1 routing for prefill on tcgen05 when a row has more chunk logits
// than tensor memory holds (T > 512 chunks).
//
// DashAttention (xllm-io paper review, section 3, Eq. 6 and Prop. 4.1), as in stage1_tc.cu:
//   x_c^(h) = (alpha-1) gamma <q_i^(h), kbar_c>/sqrt(d) for c < floor(i/B),
//   what^(h) = [x^(h) - tau^(h)]_+^{1/(alpha-1)},  w = mean over the group,  R = {w > 0},
//   bias_c = (log w_c - mean_R log w)/sigma.
//
// One block = 128 query rows = (128/g positions) x (g heads) of one (sequence, KV head).  The
// logits X = Q k̄^T stream through two 192-column halves of TMEM in blocks of 192 chunks,
// TMA-staged bf16 planes of k̄ (hi + mid + lo = k̄ exactly).  Pass 0 takes each row's maximum
// from the hi plane alone: |x - x_hi| <= xs 2^-8 |q| |k̄_c| (bf16 rounding of k̄, plus a margin
// for the fp32 accumulation), so with the largest |k̄_c| of the (sequence, KV head) from Stage 0
// that maximum less the bound is a lower bound on the exact one.  Pass 1 (all three planes)
// copies the entries above (that bound - 1) -- a superset of the only ones the support can
// reach, tau >= max - 1 -- with their chunk indices into per-thread lists in shared memory; the
// threshold is solved on the lists, and the head weights, their sums over the g heads of each
// position and the routed chunks (ascending, with log w) all come from the lists: one warp per
// position merges the position's 4 g ascending lists; the bias is fixed up with the mean after.
// The MMAs of one block overlap the processing of the previous one.  A block whose lists
// overflow flags its tile in `redo` and writes nothing; the per-shape routing kernels then
// recompute the flagged tiles.
// Roles (18 warps): warp 0 TMA producer, warp 1 TMEM allocation + MMA issue, warps 2-17 four
// warps per TMEM lane quarter (32 rows), each reading every fourth 32-column piece of a block.
// Every mbarrier wait is bounded; on time-out the block records an error code and leaves.
#include <algorithm>
#include <climits>
#include <cudaTypedefs.h>

#include "dash_common.cuh"
#include "entmax.cuh"
#include "tc_ptx.cuh"

namespace dash {

namespace {

constexpr int kR = 128, kDd = 128;
constexpr int kBW = 192;                        // chunks per block = columns of a TMEM half = MMA N
constexpr int kStage = kBW * 64 * 2;            // ring stage: [192 chunks][64 d] bf16 of one plane = 24 KB
constexpr int kNS = 2;                          // ring stages
constexpr int kPieces = kBW / 32;               // 32-column pieces per block
// TMEM: X halves at columns [0, 192) and [256, 448); the Q tile (the MMAs' A operand, 128 rows x
// 128 bf16, two per 32-bit column) at [448, 512)
constexpr int kHalfCol = 256;
constexpr int kColQ = 448;
constexpr int kOffRing = 0, kOffLists = kOffRing + kNS * kStage;
// one MMA per (block, plane, 16-wide k step): M = 128 rows, N = 192 chunks.  Narrow N = 64 MMAs
// accumulating into one tile form a dependent chain that runs at a fraction of the tensor rate.
constexpr uint32_t kIdescX = tc::idesc_bf16(128, kBW, false, false);
// after every pass but the first the workers post whether another pass over the blocks follows
// (kPlanGo) or not (kPlanStop); at most kMaxExtract extraction passes per set of rows in play
constexpr int kPlanStop = 0, kPlanGo = 1;
constexpr int kMaxExtract = 2;

// candidate list entries per (worker warp, lane): a logit (fp32) and its chunk index (16 bits)
constexpr int kCap = 52;
constexpr int kOffIdx = kOffLists + 16 * 32 * kCap * 4;
constexpr int kOffMisc = kOffIdx + 16 * 32 * kCap * 2;
// misc: barriers (kBarBytes), tmem slot / abort / overflow / plan (16 B), red [2][4][kR] float4
// (16 KB), per position: log-sum and count (2 x 32 words, then 32 spare), per row |q| (kR)
constexpr int kBarBytes = 8 * (1 + 2 * kNS + 2 + 2 + 2);   // q_full, full/empty ring, x_ready/x_free, drain, dec
constexpr int kMiscBase = (kBarBytes + 15) / 16 * 16;
constexpr int kMiscBytes = kMiscBase + 16 + 2 * 4 * kR * 16 + 3 * 32 * 4 + kR * 4;
constexpr size_t kLongSmem = 1024 + kOffMisc + kMiscBytes;
static_assert(kLongSmem <= 227 * 1024, "shared memory of the long-row routing kernel");
static_assert(4 * 4 * kR * 4 <= kNS * kStage, "published list lengths, bases, capacities and spill columns inside the plane ring");
// spill areas in global memory: one per SM id below kSpillAreas (one block per SM)
constexpr int kSpillAreas = 160;
static_assert(kCap % 4 == 0, "lists are padded to a multiple of four entries");
// |x - x_hi| <= xs (2^-8 |q| |k̄_c|  +  fp32 accumulation error): coefficient of xs |q| max|k̄_c|
constexpr float kHiPlaneBound = 0.00390625f + 0.0009765625f;

// Lower bound on the root of f_S(t) = sum_{x in S} [x - t]_+^p = 1 over a subset S of a row's
// logits: this thread's list (entry k at cl[32 k], m entries) and three more values (the other
// column sets' maxima).  f_S <= f everywhere, so that root is itself a lower bound on the row's
// tau.  g = f_S^(alpha-1) is convex and decreasing (a p-norm of the [x - t]_+), so Newton steps
// on g taken from a point left of its root stay left of it: three steps from t0 (where f_S >= 1)
// give a bound good enough to cut a list; -inf when f_S(t0) < 1 (nothing to gain).
// Entries past the shared-memory capacity cap sit in the thread's spill slots gv[512 (k - cap)].
__device__ __noinline__ float subset_bound(const float* cl, int cap, const float* gv, int m, float om0, float om1,
                                           float om2, float t0, float p, int mode, float am1)
{
    float t = t0;
    for (int it = 0; it < 3; ++it) {
        float f = 0.f, fd = 0.f;
        for (int k = 0; k < m; ++k) {
            const float u = (k < cap ? cl[32 * k] : gv[(long long)(k - cap) * 512]) - t;
            if (u > 0.f) { f += ent_pow(u, p, mode); fd += ent_dpow(u, p, mode); }
        }
        const float om[3] = {om0, om1, om2};
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const float u = om[j] - t;
            if (u > 0.f) { f += ent_pow(u, p, mode); fd += ent_dpow(u, p, mode); }
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
                                                                    const float* __restrict__ knorm, Shape s,
                                                                    Routes rt, unsigned char* redo, int* err,
                                                                    float* spill_v, unsigned short* spill_i,
                                                                    int spill_cap)
{
    extern __shared__ char smem_raw[];
    char* sm = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = tc::smem_addr(sm);
    constexpr int P = kR / G, CAP = kCap;
    float* lists = reinterpret_cast<float*>(sm + kOffLists);            // [16 warps][CAP][32 lanes]
    unsigned short* lidx = reinterpret_cast<unsigned short*>(sm + kOffIdx);   // chunk index of each entry
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
    float4* red = reinterpret_cast<float4*>(misc + kMiscBase + 16);                  // [2][4][kR]
    float* pslog = reinterpret_cast<float*>(misc + kMiscBase + 16 + 2 * 4 * kR * 16);  // [P] log-sum so far
    int* pcnt = reinterpret_cast<int*>(pslog + 32);                        // [P] entries so far
    float* qnorm = pslog + 3 * 32;                                         // [kR] |q| of each row

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
    const int nbk = (nvmax + kBW - 1) / kBW;   // 192-chunk blocks

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
            int gs = 0;   // ring stage counter: one stage per (block, plane, d-half)
            bool pok = true;
            for (int k = 0; pok; ++k) {
                const int npl = k == 0 ? 1 : 3;   // the row-maximum pass reads the hi plane alone
                for (int kb = 0; pok && kb < nbk; ++kb) {
                    for (int j = 0; j < 2 * npl; ++j, ++gs) {
                        const int st = gs % kNS;
                        if (gs >= kNS && !tc::mbar_wait(empty0 + 8 * st, ((gs / kNS) - 1) & 1, abort, err, 31)) { pok = false; break; }
                        last[st] = gs;
                        const uint32_t dst = base + kOffRing + st * kStage, fb = full0 + 8 * st;
                        tc::mbar_expect_tx(fb, kStage);
                        // chunks past T read as zeros (their columns are never used)
                        tc::tma_load_4d(dst, &tmP, fb, 64 * (j & 1), kb * kBW, br * 3 + (j >> 1), 0);
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
                const int npl = k == 0 ? 1 : 3;
                for (int kb = 0; ok && kb < nbk; ++kb, ++u) {
                    const int hlf = u & 1;
                    // the half's previous use (u - 2) has been read by every worker
                    if (u >= 2 && !tc::mbar_wait(x_free0 + 8 * hlf, ((u >> 1) - 1) & 1, abort, err, 33)) { ok = false; break; }
                    const uint32_t xd = tmem + hlf * kHalfCol;
                    for (int j = 0; j < 2 * npl; ++j, ++gs) {
                        // stage j: plane j / 2, d-half j % 2 (k steps 4 (j % 2) .. + 3)
                        const int st = gs % kNS;
                        if (!tc::mbar_wait(full0 + 8 * st, (gs / kNS) & 1, abort, err, 34)) { ok = false; break; }
                        tc::fence_after_sync();
                        const uint64_t dp = dP0 + (uint64_t)((st * kStage) >> 4);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc::mma_f16_ts(xd, tmem + kColQ + (4 * (j & 1) + kk) * 8, dp + (uint64_t)((kk * 32) >> 4),
                                           kIdescX, (j > 0 || kk > 0) ? 1u : 0u);
                        tc::mma_commit(empty0 + 8 * st);
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
            // columns [kColQ, kColQ + 64): the row's bf16 pairs are already the 32-bit columns;
            // its Euclidean norm for the hi-plane bound
            uint4 qw[16];
            const __nv_bfloat16* qrow = Q + (long long)b * s.qs[0] + (long long)i * s.qs[1] + (long long)(r * G + row % G) * s.qs[2];
#pragma unroll
            for (int k = 0; k < 16; ++k)
                qw[k] = i < s.n ? __ldg(reinterpret_cast<const uint4*>(qrow) + k) : make_uint4(0u, 0u, 0u, 0u);
            float qq = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const uint32_t w4[4] = {qw[k].x, qw[k].y, qw[k].z, qw[k].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float lo16 = __uint_as_float(w4[j] << 16), hi16 = __uint_as_float(w4[j] & 0xffff0000u);
                    qq = fmaf(lo16, lo16, fmaf(hi16, hi16, qq));
                }
            }
            qnorm[row] = sqrtf(qq);
#pragma unroll
            for (int k = 0; k < 4; ++k) tc::tmem_st16(lane_base + kColQ + 16 * k, reinterpret_cast<const uint32_t*>(qw + 4 * k));
            tc::tmem_wait_st();
            tc::fence_before_sync();
            tc::mbar_arrive(q_full);
        }
        const int own_off = ((cq * 2 + (q4 & 1)) * 2 + (q4 >> 1)) * CAP * 32 + lane;
        const int pair_off = ((cq * 2 + (q4 & 1)) * 2) * CAP * 32 + lane;
        float* cl = lists + own_off;            // this thread's list, entry k at cl[32 k]
        unsigned short* ci = lidx + own_off;    // and its chunk index at ci[32 k]
        int cap = CAP;
        // entries past the shared-memory capacity spill to this thread's slots of its SM's area in
        // global memory (one block per SM, so the SM id names the area): entry k >= cap at
        // gv[512 (k - cap)], up to gcap of them (none when the SM id is past the areas).  This
        // relies on a block staying on its SM; a block resumed elsewhere after compute
        // preemption could share an area (claiming areas atomically per block would lift that).
        unsigned smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        const bool spills = spill_v && spill_i && spill_cap > 0 && smid < (unsigned)kSpillAreas;
        const int gcap = spills ? spill_cap : 0;
        const long long gbase = spills ? (long long)smid * spill_cap * 512 : 0;
        float* const gv = spills ? spill_v + gbase + (tid - 64) : nullptr;
        unsigned short* const gi = spills ? spill_i + gbase + (tid - 64) : nullptr;
        auto LV = [&](int k) -> float& { return k < cap ? cl[32 * k] : gv[(long long)(k - cap) * 512]; };
        auto LI = [&](int k) -> unsigned short& { return k < cap ? ci[32 * k] : gi[(long long)(k - cap) * 512]; };
        float mx = -INFINITY, lo = 0.f, t = 0.f;
        float hi = 0.f;
        float om[3] = {-INFINITY, -INFINITY, -INFINITY};   // lower bounds on the other column sets' maxima
        float lo_t = 0.f;   // this thread's list cut: lo, raised by its own subset bounds
        int m = 0;
        bool ok = true, emitted = false, redo_me = false;
        int kind = 0;   // pass kind: 0 row maximum (hi plane), 1 candidate extraction
        int half = -1;  // rows in play: all (-1), or the quarters q4 >> 1 == half
        int nextract = 0;
        const float kmax = __ldg(knorm + br);   // largest |k̄_c| of this (sequence, KV head)
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
                        // columns past every row of the warp: never read (the g rows of a position
                        // sit in one warp, and the emission stops at the position's own bound);
                        // 16 columns per TMEM load keep the register footprint low
#pragma unroll 1
                        for (int hh = 0; hh < 2; ++hh) {
                            const int c0 = kb * kBW + lp * 32 + 16 * hh;
                            if (c0 >= nvw) break;
                            float v[16];
                            tc::tmem_ld16(lane_base + hlf * kHalfCol + lp * 32 + 16 * hh, v);
                            tc::tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; ++e) v[e] = c0 + e < nv ? v[e] * xs : -INFINITY;
                            if (kind == 0) {
#pragma unroll
                                for (int e = 0; e < 16; ++e) mx = fmaxf(mx, v[e]);
                                continue;
                            }
                            // entries above the cut, compacted by prefix popcount (no serial chain)
                            uint32_t mask = 0u;
#pragma unroll
                            for (int e = 0; e < 16; ++e) mask |= (v[e] > lo_t ? 1u : 0u) << e;
                            if (m + __popc(mask) > cap + gcap && m <= cap + gcap) {
                                // list full: raise the cut to this thread's subset bound on tau
                                // (less the margin below) and drop the entries under it
                                const float tb = subset_bound(cl, cap, gv, m, om[0], om[1], om[2], lo_t, p, mode,
                                                              s.alpha - 1.f);
                                const float cut = tb - 1e-3f * fmaxf(1.f, fabsf(tb));
                                if (cut > lo_t) {
                                    lo_t = cut;
                                    int j = 0;
                                    for (int kk = 0; kk < m; ++kk) {
                                        const float x = LV(kk);
                                        if (x > cut) {
                                            LI(j) = LI(kk);
                                            LV(j++) = x;
                                        }
                                    }
                                    m = j;
                                    mask = 0u;
#pragma unroll
                                    for (int e = 0; e < 16; ++e) mask |= (v[e] > lo_t ? 1u : 0u) << e;
                                }
                            }
                            if (mask) {
                                if (m + __popc(mask) <= cap) {   // the common case: shared memory only
#pragma unroll
                                    for (int e = 0; e < 16; ++e) {
                                        const int kk = m + __popc(mask & ((1u << e) - 1u));
                                        if ((mask >> e) & 1u) {
                                            cl[kk * 32] = v[e];
                                            ci[kk * 32] = (unsigned short)(c0 + e);
                                        }
                                    }
                                } else {
#pragma unroll
                                    for (int e = 0; e < 16; ++e) {
                                        const int kk = m + __popc(mask & ((1u << e) - 1u));
                                        if (((mask >> e) & 1u) && kk < cap + gcap) {
                                            LV(kk) = v[e];
                                            LI(kk) = (unsigned short)(c0 + e);
                                        }
                                    }
                                }
                                m += __popc(mask);
                            }
                        }
                    }
                }
                // TMEM half read: the MMAs of use u + 2 may overwrite it
                tc::fence_before_sync();
                tc::mbar_arrive(x_free0 + 8 * hlf);
            }
            if (kind == 0) {
                // row maximum over the four warps of the rows, from the hi plane: less the bound on
                // |x - x_hi| it is a lower bound on the exact maximum, so the lists start at that
                // value - 1 (tau >= max - 1: the largest entry alone gives f(max - 1) >= 1)
                red[cq * kR + row].x = mx;
                group_sync();
#pragma unroll
                for (int j = 0; j < 3; ++j) om[j] = red[((cq + 1 + j) & 3) * kR + row].x;
                mx = fmaxf(fmaxf(mx, om[0]), fmaxf(om[1], om[2]));
                const float eb = xs * kHiPlaneBound * qnorm[row] * kmax + 1e-6f * fmaxf(1.f, fabsf(mx));
#pragma unroll
                for (int j = 0; j < 3; ++j) om[j] -= eb;
                lo = mx - eb - 1.f;
                lo_t = lo;
                hi = nv > 0 ? mx + eb - exp2f(-(s.alpha - 1.f) * __log2f((float)nv)) : 0.f;
                kind = 1;
                continue;   // an extraction pass always follows
            }
            // ---- after an extraction pass: threshold on the lists.  A list that overflowed
            // dropped entries, and the root on the entries kept is then a lower bound on tau
            // (a subset's f is smaller everywhere) from which the next extraction starts ----------
            if (active && m > cap + gcap) atomicOr(overflow, 1);
            workers_sync();   // also orders the reads of the maxima before the slots are reused
            const bool over = *overflow != 0;
            ++nextract;
            if (ok && active) {
                const int mm = min(m, cap + gcap);   // entries kept: shared memory, then spill slots
                const int ms = min(mm, cap);
                const int m4 = (ms + 3) >> 2;
                for (int kk = ms; kk < 4 * m4; ++kk) cl[kk * 32] = -INFINITY;
                // every list holds all of its column set's entries above the largest of the
                // four cuts (each cut is at most tau), so the solve starts there
                red[(4 + cq) * kR + row].y = lo_t;
                group_sync();
                lo = fmaxf(fmaxf(red[(4 + 0) * kR + row].y, red[(4 + 1) * kR + row].y),
                           fmaxf(red[(4 + 2) * kR + row].y, red[(4 + 3) * kR + row].y));
                // the solve from t = lo (entmax.cuh, ent_step), the four warps' partial sums
                // combined in a fixed order; every row of the quarter steps until all are done
                // (the group barriers stay matched).  Iteration 0 writes slot 0, read last before
                // the barrier above; slot 1 (the cuts) is rewritten only after iteration 0's barrier.
                float lo_n = lo, hi_n = hi;
                t = lo;
                bool done = nv == 0;
                for (int it = 0; it < 32 && !__all_sync(0xffffffffu, done); ++it) {
                    EntSums S = ent_zero();
                    if (mode == 2) {
                        for (int kk = 0; kk < m4; ++kk) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float uu = cl[(4 * kk + j) * 32] - t;
                                const float up = fmaxf(uu, 0.f);
                                S.f = fmaf(up, up, S.f);
                                S.fd += up;
                                S.n += uu > 0.f ? 1.f : 0.f;
                                S.um = fminf(S.um, uu > 0.f ? uu : INFINITY);
                            }
                        }
                    } else {
                        for (int kk = 0; kk < 4 * m4; ++kk) ent_add(S, cl[kk * 32] - t, p, mode);
                    }
                    for (int kk = cap; kk < mm; ++kk) ent_add(S, gv[(long long)(kk - cap) * 512] - t, p, mode);
                    float4* slot = red + (it & 1) * 4 * kR;
                    slot[cq * kR + row] = make_float4(S.f, S.fd, S.n, S.um);
                    group_sync();
                    const float4 r0 = slot[row], r1 = slot[kR + row], r2 = slot[2 * kR + row], r3 = slot[3 * kR + row];
                    S.f = (r0.x + r1.x) + (r2.x + r3.x);
                    S.fd = (r0.y + r1.y) + (r2.y + r3.y);
                    S.n = (r0.z + r1.z) + (r2.z + r3.z);
                    S.um = fminf(fminf(r0.w, r1.w), fminf(r2.w, r3.w));
                    if (!done) done = ent_step(S, t, lo_n, hi_n, s.alpha, mode);
                }
                if (over) {
                    // the next lists keep the entries above the bound, less a margin far
                    // above the solve's rounding (f' at the root is at least 1/(alpha-1))
                    lo = fmaxf(lo, t - 1e-3f * fmaxf(1.f, fabsf(t)));
                }
            }
            bool stop = false;
            if (!ok) stop = true;
            else if (!over) {
                // ---- every list holds its column set's whole support: the route lists come from
                // a merge of each position's 4 g lists (4 column sets x g heads, each ascending in
                // chunk index).  One warp per position: every step takes the smallest chunk any
                // list shows (a warp minimum), sums the head weights of the lists that show it in
                // a fixed butterfly order (deterministic), writes the entry and advances those
                // lists.  Entries at or below their row's threshold are skipped.  The lists' bases,
                // lengths and thresholds are published in the (idle) plane ring.
                int* pub_len = reinterpret_cast<int*>(sm + kOffRing);      // [4][kR]
                int* pub_off = pub_len + 4 * kR;                            // [4][kR] list base (entries)
                int* pub_cap = pub_off + 4 * kR;                            // [4][kR] shared-memory entries
                int* pub_sp = pub_cap + 4 * kR;                             // [4][kR] spill column (tid - 64)
                if (active) {
                    // the list in place becomes the support alone, each entry its head weight
                    const int mm = min(m, cap + gcap);
                    int j = 0;
                    if (mm <= cap) {   // the common case: shared memory only
                        for (int k = 0; k < mm; ++k) {
                            const float uu = cl[32 * k] - t;
                            if (uu > 0.f) {
                                ci[32 * j] = ci[32 * k];
                                cl[32 * j++] = ent_pow(uu, p, mode);
                            }
                        }
                    } else {
                        for (int k = 0; k < mm; ++k) {
                            const float uu = LV(k) - t;
                            if (uu > 0.f) {
                                LI(j) = LI(k);
                                LV(j++) = ent_pow(uu, p, mode);
                            }
                        }
                    }
                    pub_len[cq * kR + row] = j;
                    pub_off[cq * kR + row] = (int)(cl - lists);
                    pub_cap[cq * kR + row] = cap;
                    pub_sp[cq * kR + row] = tid - 64;
                }
                workers_sync();
                for (int pp = warp - 2; pp < P; pp += 16) {
                    const int ip = i0 + pp;
                    if (ip >= s.n || (half >= 0 && ((pp * G) >> 6) != half)) continue;
                    const int nvp = min(ip / s.B, s.T);
                    // lane l holds list l (and l + 32 when 4 g = 64): column set li / G, head li % G.
                    // A chunk lies in one column set, so the lists showing it are the G lanes
                    // (li / G) * G .. + G - 1 of one group, summed by a butterfly inside the group.
                    constexpr int NL = (4 * G + 31) / 32;   // lists per lane
                    constexpr int GW = G < 32 ? G : 32;     // lanes of a group
                    int lcur[NL] = {}, llen[NL] = {}, loff[NL] = {}, lcap[NL] = {}, lsp[NL] = {}, lc[NL] = {};
                    float lx[NL] = {};
                    auto advance = [&](int j) {
                        if (lcur[j] < llen[j]) {
                            const int k = lcur[j]++;
                            if (k < lcap[j]) {
                                const int e = loff[j] + 32 * k;
                                lc[j] = lidx[e];
                                lx[j] = lists[e];
                            } else {
                                const long long e = gbase + (long long)(k - lcap[j]) * 512 + lsp[j];
                                lc[j] = spill_i[e];
                                lx[j] = spill_v[e];
                            }
                        } else {
                            lc[j] = INT_MAX;
                        }
                    };
#pragma unroll
                    for (int j = 0; j < NL; ++j) {
                        const int li = lane + 32 * j;
                        const bool has = li < 4 * G;
                        const int rr = pp * G + (has ? li % G : 0), cs = has ? li / G : 0;
                        lcur[j] = 0;
                        llen[j] = has ? pub_len[cs * kR + rr] : 0;
                        loff[j] = has ? pub_off[cs * kR + rr] : 0;
                        lcap[j] = has ? pub_cap[cs * kR + rr] : 0;
                        lsp[j] = has ? pub_sp[cs * kR + rr] : 0;
                        advance(j);
                    }
                    const float inv_g = 1.f / G;
                    const long long toff = tri_offset(ip, s.B);
                    uint32_t* mrow = bm ? bm + (long long)ip * rt.words : nullptr;
                    if (mrow) {
                        for (int wd = lane; wd < rt.words; wd += 32) mrow[wd] = 0u;
                        __syncwarp();
                    }
                    int kk = 0, wcur = -1;
                    uint32_t wbits = 0u;
                    float slog = 0.f;
                    for (;;) {
                        int c = lc[0];
#pragma unroll
                        for (int j = 1; j < NL; ++j) c = min(c, lc[j]);
                        const int cmin = __reduce_min_sync(0xffffffffu, c);
                        if (cmin == INT_MAX || cmin >= nvp) break;
                        float w = 0.f;
#pragma unroll
                        for (int j = 0; j < NL; ++j)
                            if (lc[j] == cmin) {
                                w += lx[j];
                                advance(j);
                            }
                        const uint32_t on = __ballot_sync(0xffffffffu, w != 0.f);
#pragma unroll
                        for (int o = GW / 2; o > 0; o >>= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
                        const int src = on ? ((__ffs(on) - 1) / GW) * GW : 0;
                        w = __shfl_sync(0xffffffffu, w, src);
                        if (!(w > 0.f)) continue;   // weights that underflow route nothing
                        // the sum of log w for the mean: lane kk % 32 takes entry kk, and the 32
                        // partial sums are added in a tree at the end (few roundings per term)
                        const float lw = __logf(w * inv_g);
                        if (lane == (kk & 31)) slog += lw;
                        if (lane == 0) {
                            idx[toff + kk] = cmin;
                            bias[toff + kk] = lw;
                            if (mrow) {
                                if ((cmin >> 5) != wcur) {
                                    if (wcur >= 0) mrow[wcur] = wbits;
                                    wcur = cmin >> 5;
                                    wbits = 0u;
                                }
                                wbits |= 1u << (cmin & 31);
                            }
                        }
                        ++kk;
                    }
                    slog = warp_sum(slog);
                    if (lane == 0) {
                        if (mrow && wcur >= 0) mrow[wcur] = wbits;
                        pslog[pp] = slog;
                        pcnt[pp] = kk;
                    }
                    __syncwarp();
                }
                workers_sync();   // the published lists are read; the ring may be refilled
                // the ring is written by TMA again only after this pass's decision; order this
                // thread's generic accesses to it before those asynchronous-proxy writes
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                if (half == 0) {
                    // the second half of the rows: extraction passes of its own
                    half = 1;
                    nextract = 0;
                    lo_t = lo;
                    m = 0;
                } else {
                    stop = true;
                    emitted = true;
                }
            } else if (nextract < kMaxExtract) {
                lo_t = lo;
                m = 0;
            } else if (half < 0) {
                // a column set holds more of the support than its list: redo the rows in two
                // halves, each thread of the half in play taking its idle partner's list too
                half = 0;
                nextract = 0;
                lo_t = lo;
                m = 0;
                cl = lists + pair_off;
                ci = lidx + pair_off;
                cap = 2 * CAP;
            } else {
                stop = true;
                redo_me = true;
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
cudaError_t launch_long_g(const Shape& s, const void* Q, const __nv_bfloat16* planes, const float* knorm,
                          const Routes& rt, unsigned char* redo, int* err, void* spill, cudaStream_t st)
{
    auto fn = encode_fn_l();
    if (!fn) return cudaErrorInvalidValue;
    constexpr int P = kR / G;
    CUtensorMap mp;
    {
        // planes [b*hkv*3][T][128] viewed as (d, chunk, plane-row, 1)
        cuuint64_t dims[4] = {128, (cuuint64_t)s.T, (cuuint64_t)s.batch * s.hkv * 3, 1};
        cuuint64_t strides[3] = {128 * 2, (cuuint64_t)s.T * 128 * 2, (cuuint64_t)s.T * 128 * 2 * s.batch * s.hkv * 3};
        cuuint32_t box[4] = {64, (cuuint32_t)kBW, 1, 1};
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
    const int sc = spill ? route_long_spill_entries(s) : 0;
    float* sv = spill ? static_cast<float*>(spill) : nullptr;
    unsigned short* si = spill ? reinterpret_cast<unsigned short*>(sv + (size_t)kSpillAreas * sc * 512) : nullptr;
    k<<<grid, 576, smem, st>>>(mp, static_cast<const __nv_bfloat16*>(Q), knorm, s, rt, redo, err, sv, si, sc);
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

int route_long_spill_entries(const Shape& s)
{
    // a thread's column set holds at most ceil(T / 128) pieces of 32 chunks
    const long long most = (long long)(s.T + 127) / 128 * 32 - kCap;
    return (int)std::max(0LL, std::min<long long>(most, 460));
}

size_t route_long_spill_bytes(const Shape& s)
{
    return (size_t)kSpillAreas * route_long_spill_entries(s) * 512 * (4 + 2);
}

cudaError_t launch_route_prefill_long(const Shape& s, const void* Q, const __nv_bfloat16* planes, const float* knorm,
                                      const Routes& rt, unsigned char* redo, int* err, void* spill, cudaStream_t st)
{
    switch (s.g) {
    case 4: return launch_long_g<4>(s, Q, planes, knorm, rt, redo, err, spill, st);
    case 8: return launch_long_g<8>(s, Q, planes, knorm, rt, redo, err, spill, st);
    default: return launch_long_g<16>(s, Q, planes, knorm, rt, redo, err, spill, st);
    }
}

}  // namespace dash
