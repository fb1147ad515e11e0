// stage2_tc.cu -- Stage 2 prefill on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// DashAttention (xllm-io paper review, section 3, Proposition 4.1 and the "Stage 2" kernel row):
// per query row, o = softmax(<q,k_j>/sqrt(d) + d_j) V over the tokens of the routed chunks
// (d_j = the chunk's bias) and the diagonal tokens c(i)B..i (d_j = 0), in one online-softmax pass
// over the routed chunks.
//
// One block = 128 query rows = (128/g positions) x (g heads) of one (sequence, KV head); the
// heads of a position share one routing list, so the block walks the union of its positions'
// routed chunks plus their diagonal chunks, ascending, in tiles of 64 keys.  Rows that did not
// route a tile get -inf there.  Roles (6 warps):
//   warp 0      TMA producer: the Q tile once, then K and V tiles into a 4-slot ring
//   warp 1      allocates TMEM and issues the MMAs from one thread:
//               S = Q K^T  (M=128, N=64, K=128; two S buffers in TMEM)
//               O += P V   (M=128, N=128, K=64; O accumulates in TMEM)
//   warps 2-5   softmax, one thread per row (TMEM lane): S from TMEM, bias / causal mask,
//               running max and sum in base 2, P (bf16) to shared memory; O in TMEM is rescaled
//               only when a row's maximum grows by more than 2^8, otherwise the stale maximum
//               is kept (values stay <= 2^8, exact in the final normalisation).
// Every mbarrier wait is bounded; on time-out the block records an error code and leaves.
#include <climits>
#include <cstdlib>
#include <cudaTypedefs.h>

#include "dash_common.cuh"
#include "tc_ptx.cuh"

namespace dash {
namespace {

constexpr int kRows = 128, kKT = 64, kD = 128, kNS = 2;
constexpr int kQBytes = kRows * kD * 2;           // 32 KB, two 16 KB d-halves
constexpr int kKVHalf = kKT * 64 * 2;             // 8 KB: [64 keys][64 d]
constexpr int kSlot = 4 * kKVHalf;                // K (2 halves) + V (2 halves) = 32 KB
constexpr int kTmemCols = 256;                    // S0 [0,64), S1 [64,128), O [128,256); P_k over S_k
constexpr int kOffQ = 0, kOffSlots = kQBytes;
constexpr int kOffScratch = kOffSlots;            // set-up scratch (the union bitmask) in the ring
constexpr int kOffBar = kOffSlots + kNS * kSlot;  // 98304: two blocks fit on one SM
constexpr int kNumBars = 1 + 2 * kNS + 2 + 2 + 2 + 2 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;  // tmem base, abort, njobs
constexpr int kOffPos = kOffMisc + 32;             // the block's positions (128 / g of them)
constexpr int kOffJobs = kOffPos + 4 * kRows;

constexpr uint32_t kIdescS = tc::idesc_bf16(128, 64, false, false);
constexpr uint32_t kIdescPV = tc::idesc_bf16(128, 128, false, true);

// 2^x on the special-function unit (flush-to-zero; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed fp32 pairs (sm_100 f32x2 instructions: one issue slot for two lanes of arithmetic) and
// the three-input maximum: the softmax below is bound by instruction issue.
__device__ __forceinline__ unsigned long long f2(float a, float b)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void unf2(unsigned long long r, float& a, float& b)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b, unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ unsigned long long fadd2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// K and V of a slot have their own barriers.  With as many slots as S buffers (2), slot k % 2 holds
// job k's K until S_k is done and its V until P V_k is done, so the producer waits on s_full and
// pv_done themselves (two commits per job); neither can run a phase ahead of the producer's wait,
// since the next phase needs the load it has yet to issue.
static_assert(kNS == 2, "slot k % kNS must be S buffer k % 2");
struct Bars {
    uint32_t q_full, k_full[kNS], v_full[kNS], s_full[2], s_free[2], p_full[2], pv_done[2], drain;
};

__device__ __forceinline__ Bars make_bars(uint32_t base)
{
    Bars b;
    uint32_t a = base + kOffBar;
    b.q_full = a; a += 8;
    for (int k = 0; k < kNS; ++k) { b.k_full[k] = a; a += 8; }
    for (int k = 0; k < kNS; ++k) { b.v_full[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.s_full[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.s_free[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.p_full[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.pv_done[k] = a; a += 8; }
    b.drain = a;
    return b;
}

// Position order for the 128-row tiles (one block per window of kWinTiles tiles of P positions of
// one (sequence, KV head)).  Rows of a tile share the union of their positions' routed chunks, so
// positions with similar routes should share tiles.  A sparse window (under 1/8 of the visible
// chunks routed) is sorted by (first routed chunk, routed count, position): queries that route
// the same chunks -- the same keys region -- land in the same tiles, whatever their distance.
// Denser windows keep each run of 8 tiles and sort it by (routed count, position), so that
// positions with few routes (e.g. queries matching a few strong chunks) share tiles.  perm[br][k]
// = the position at slot k.
constexpr int kWinTiles = 64, kSubTiles = 8;
__global__ void __launch_bounds__(1024) group_positions_kernel(Shape s, Routes rt, int P, int* __restrict__ perm)
{
    __shared__ unsigned long long key[kWinTiles * 16];
    __shared__ int red[2][32];
    const int br = blockIdx.y, tid = threadIdx.x;
    const int Wn = kWinTiles * P, w0 = blockIdx.x * Wn, nw = min(Wn, s.n - w0);
    const int* counts = rt.counts + (long long)br * s.n;
    const int* ridx = rt.idx + (long long)br * rt.cap;
    int cs = 0, vs = 0;
    for (int j = tid; j < nw; j += blockDim.x) {
        const int i = w0 + j;
        cs += counts[i];
        vs += min(i / s.B, s.T);
    }
    for (int o = 16; o > 0; o >>= 1) {
        cs += __shfl_xor_sync(0xffffffffu, cs, o);
        vs += __shfl_xor_sync(0xffffffffu, vs, o);
    }
    if ((tid & 31) == 0) { red[0][tid >> 5] = cs; red[1][tid >> 5] = vs; }
    __syncthreads();
    long long csum = 0, vsum = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) { csum += red[0][w]; vsum += red[1][w]; }
    const bool sparse = 8 * csum < vsum;
    for (int j = tid; j < nw; j += blockDim.x) {
        const int i = w0 + j, c = counts[i];
        const unsigned long long first = c > 0 ? (unsigned long long)ridx[tri_offset(i, s.B)] : (unsigned long long)s.T;
        key[j] = sparse ? (first << 40) | ((unsigned long long)c << 20) | (unsigned long long)j
                        : ((unsigned long long)c << 20) | (unsigned long long)j;
    }
    __syncthreads();
    const int span = sparse ? Wn : kSubTiles * P;   // positions ranked together
    for (int j = tid; j < nw; j += blockDim.x) {
        const int g0 = j / span * span, g1 = min(nw, g0 + span);
        const unsigned long long kj = key[j];
        int rank = 0;
        for (int q = g0; q < g1; ++q) rank += key[q] < kj;
        perm[(long long)br * s.n + w0 + g0 + rank] = w0 + j;
    }
}

// A position's routed chunks in ascending order, from the ascending chunk list (MASK = false: the
// k-th entry) or from the bit-packed block mask M_i (MASK = true: the k-th set bit, taken in order
// by a scan over the position's mask words).  The bias of the k-th routed chunk is the k-th entry of
// the bias list either way, so both sources give identical results.
template <bool MASK>
struct ChunkSource {
    const int* li;
    const uint32_t* mw;
    uint32_t word;
    int wi, words;
    __device__ __forceinline__ void init(const int* li_, const uint32_t* mw_, int words_, bool any)
    {
        li = li_; mw = mw_; words = words_; wi = 0;
        word = MASK && any ? mw[0] : 0u;
    }
    // chunk id of entry k; entries are requested in increasing order, one after the other
    __device__ __forceinline__ int at(int k)
    {
        if constexpr (MASK) {
            (void)k;
            while (word == 0u) {
                if (++wi >= words) return INT_MAX;
                word = mw[wi];
            }
            const int b = __ffs(word) - 1;
            word &= word - 1u;
            return (wi << 5) + b;
        } else {
            return li[k];
        }
    }
};

// CPT = chunks per 64-key tile: 1 for chunks of 64 or 128 keys (a chunk is one or two jobs), 2 for
// 32-key chunks (a job covers two neighbouring chunks, each row with its own bias per half).
// MASK = true: the routed support comes from the bit-packed block mask instead of the chunk lists.
template <int CPT, bool MASK>
__global__ void __launch_bounds__(192, 2) attend_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                   const __grid_constant__ CUtensorMap tmQ1,
                                                                   const __grid_constant__ CUtensorMap tmK,
                                                                   const __grid_constant__ CUtensorMap tmV,
                                                                   Shape s, Routes rt,
                                                                   __nv_bfloat16* __restrict__ O, int* err,
                                                                   const int* __restrict__ perm)
{
    extern __shared__ char smem_raw[];
    char* sm = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = tc::smem_addr(sm);
    const Bars bar = make_bars(base);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + kOffMisc + 4);
    int* njobs_s = reinterpret_cast<int*>(sm + kOffMisc + 8);
    int* jobs = reinterpret_cast<int*>(sm + kOffJobs);
    int* spos = reinterpret_cast<int*>(sm + kOffPos);
    uint32_t* umask = reinterpret_cast<uint32_t*>(sm + kOffScratch);   // scratch until the first TMA

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = s.g, P = kRows / G;
    const int nblk = (s.n + P - 1) / P;
    const int br = blockIdx.x % (s.batch * s.hkv);
    const int pb = nblk - 1 - blockIdx.x / (s.batch * s.hkv);   // heaviest blocks first
    const int b = br / s.hkv, r = br % s.hkv;
    const int i0 = pb * P;
    const int* counts = rt.counts + (long long)br * s.n;
    const int* ridx = rt.idx + (long long)br * rt.cap;
    const float* rbias = rt.bias + (long long)br * rt.cap;
    const uint32_t* rmask = MASK ? rt.bitmask + (long long)br * s.n * rt.words : nullptr;
    const int W = (s.T + 32) >> 5;
    const int NH = CPT == 1 ? s.B / kKT : 1;   // jobs per union unit (chunk, or 64-key tile)
    const int UB = CPT == 1 ? s.B : kKT;       // keys per union unit

    // ---- set-up: barriers, TMEM, union of the block's routed + diagonal chunks --------------
    if (tid == 0) {
        tc::mbar_init(bar.q_full, 1);
        for (int k = 0; k < kNS; ++k) {
            tc::mbar_init(bar.k_full[k], 1);
            tc::mbar_init(bar.v_full[k], 1);
        }
        for (int k = 0; k < 2; ++k) {
            tc::mbar_init(bar.s_full[k], 1);
            tc::mbar_init(bar.s_free[k], 128);
            tc::mbar_init(bar.p_full[k], 128);
            tc::mbar_init(bar.pv_done[k], 1);
        }
        tc::mbar_init(bar.drain, 1);
        *abort = 0;
        tc::mbar_fence_init();
    }
    if (warp == 1) {
        __syncwarp();
        tc::tmem_alloc(tc::smem_addr(tmem_slot), kTmemCols);
    }
    for (int w = tid; w < W; w += blockDim.x) umask[w] = 0u;
    // the block's positions: slots pb*P .. pb*P+P-1 of the grouped order (positions past the end
    // of the sequence stay in place and are masked)
    for (int p = tid; p < P; p += blockDim.x) {
        const int k = i0 + p;
        spos[p] = perm && k < s.n ? perm[(long long)br * s.n + k] : k;
    }
    __syncthreads();
    if constexpr (MASK) {
        // union units from the positions' mask words (chunks; pairs of chunks when CPT = 2)
        for (int e = tid; e < P * rt.words; e += blockDim.x) {
            const int i = spos[e / rt.words];
            if (i >= s.n) continue;
            uint32_t w = rmask[(long long)i * rt.words + e % rt.words];
            while (w) {
                const int c = ((e % rt.words) << 5) + __ffs(w) - 1;
                w &= w - 1u;
                const int u = c / CPT;
                atomicOr(&umask[u >> 5], 1u << (u & 31));
            }
        }
        if (tid < P && spos[tid] < s.n) {
            const int u = (spos[tid] / s.B) / CPT;
            atomicOr(&umask[u >> 5], 1u << (u & 31));
        }
    } else {
        // union units from the positions' lists: blockDim / P threads per position, all positions
        // at once (one round trip for the counts, one for the entries)
        const int tpp = max(1, (int)blockDim.x / P);
        for (int p = tid / tpp; p < P; p += (int)blockDim.x / tpp) {
            const int sub = tid % tpp;
            const int i = spos[p];
            if (i >= s.n) continue;
            const int cnt = counts[i];
            const int* li = ridx + tri_offset(i, s.B);
            for (int k = sub; k < cnt; k += tpp) {
                const int u = li[k] / CPT;
                atomicOr(&umask[u >> 5], 1u << (u & 31));
            }
            if (sub == 0) {
                const int u = (i / s.B) / CPT;
                atomicOr(&umask[u >> 5], 1u << (u & 31));
            }
        }
    }
    __syncthreads();
    if (warp == 0) {   // ordered bitmask -> list of chunk ids
        int basec = 0;
        for (int w0 = 0; w0 < W; w0 += 32) {
            const uint32_t bits = w0 + lane < W ? umask[w0 + lane] : 0u;
            const int pc = __popc(bits);
            int incl = pc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            int at = basec + incl - pc;
            uint32_t bb = bits;
            while (bb) {
                const int bit = __ffs(bb) - 1;
                jobs[at++] = ((w0 + lane) << 5) + bit;
                bb &= bb - 1u;
            }
            basec += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) *njobs_s = basec * NH;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int njobs = *njobs_s;

    if (warp == 0) {
        // ---- TMA producer ------------------------------------------------------------------
        if (lane == 0 && njobs > 0) {
            tc::prefetch_tmap(&tmQ);
            tc::prefetch_tmap(&tmK);
            tc::prefetch_tmap(&tmV);
            tc::mbar_expect_tx(bar.q_full, kQBytes);
            if (perm) {
                // one box of g rows per position (g = 8 or 16 keeps every box 1024-byte aligned)
                tc::prefetch_tmap(&tmQ1);
                for (int p = 0; p < P; ++p) {
                    tc::tma_load_4d(base + kOffQ + p * G * 128, &tmQ1, bar.q_full, 0, r * G, spos[p], b);
                    tc::tma_load_4d(base + kOffQ + kQBytes / 2 + p * G * 128, &tmQ1, bar.q_full, 64, r * G, spos[p], b);
                }
            } else {
                tc::tma_load_4d(base + kOffQ, &tmQ, bar.q_full, 0, r * G, i0, b);
                tc::tma_load_4d(base + kOffQ + kQBytes / 2, &tmQ, bar.q_full, 64, r * G, i0, b);
            }
            // issue order K_0, K_1, V_0, K_2, V_1, ...: K runs one job ahead of V.  K_{k+1} needs
            // S_{k-1} done, V_k needs P V_{k-2} done, and P V_{k-2} is issued before S_k, so no
            // wait in this order blocks a load that could already go.
            int lastk[kNS], lastv[kNS];
            for (int k = 0; k < kNS; ++k) lastk[k] = lastv[k] = -1;
            auto load_k = [&](int k) -> bool {
                const int slot = k % kNS;
                if (k >= kNS && !tc::mbar_wait(bar.s_full[slot], ((k / kNS) - 1) & 1, abort, err, 1, s.polls)) return false;
                lastk[slot] = k;
                const int key0 = jobs[k / NH] * UB + (k % NH) * kKT;
                const uint32_t dst = base + kOffSlots + slot * kSlot;
                tc::mbar_expect_tx(bar.k_full[slot], 2 * kKVHalf);
                tc::tma_load_4d(dst, &tmK, bar.k_full[slot], 0, r, key0, b);
                tc::tma_load_4d(dst + kKVHalf, &tmK, bar.k_full[slot], 64, r, key0, b);
                return true;
            };
            auto load_v = [&](int k) -> bool {
                const int slot = k % kNS;
                if (k >= kNS && !tc::mbar_wait(bar.pv_done[slot], ((k / kNS) - 1) & 1, abort, err, 10, s.polls)) return false;
                lastv[slot] = k;
                const int key0 = jobs[k / NH] * UB + (k % NH) * kKT;
                const uint32_t dst = base + kOffSlots + slot * kSlot + 2 * kKVHalf;
                tc::mbar_expect_tx(bar.v_full[slot], 2 * kKVHalf);
                tc::tma_load_4d(dst, &tmV, bar.v_full[slot], 0, r, key0, b);
                tc::tma_load_4d(dst + kKVHalf, &tmV, bar.v_full[slot], 64, r, key0, b);
                return true;
            };
            bool pok = load_k(0);
            for (int k = 0; pok && k < njobs; ++k) {
                if (k + 1 < njobs && !load_k(k + 1)) break;
                pok = load_v(k);
            }
            if (*abort) {
                // let this block's TMA copies still in flight land before its shared memory goes away
                for (int k = 0; k < kNS; ++k) {
                    if (lastk[k] >= 0)
                        for (long long it = 0; it < (1ll << 22); ++it)
                            if (tc::mbar_try(bar.k_full[k], (lastk[k] / kNS) & 1)) break;
                    if (lastv[k] >= 0)
                        for (long long it = 0; it < (1ll << 22); ++it)
                            if (tc::mbar_try(bar.v_full[k], (lastv[k] / kNS) & 1)) break;
                }
                for (long long it = 0; it < (1ll << 22); ++it)
                    if (tc::mbar_try(bar.q_full, 0)) break;
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer --------------------------------------------------------------------
        if (lane == 0 && njobs > 0) {
            // descriptors of Q and slot 0; a slot / K-step moves only the start-address field
            // (16-byte units, no carry), so each MMA is issued after one add
            const uint64_t dQ = tc::sw128_desc(base + kOffQ, 16, 1024);
            const uint64_t dK0 = tc::sw128_desc(base + kOffSlots, 16, 1024);
            const uint64_t dV0 = tc::sw128_desc(base + kOffSlots + 2 * kKVHalf, kKVHalf, 1024);
            auto issue_pv = [&](int j) -> bool {
                const int pbuf = j & 1;
                if (!tc::mbar_wait(bar.p_full[pbuf], (j >> 1) & 1, abort, err, 2, s.polls)) return false;
                if (!tc::mbar_wait(bar.v_full[j % kNS], (j / kNS) & 1, abort, err, 13, s.polls)) return false;
                tc::fence_after_sync();
                const uint64_t dv = dV0 + (uint64_t)(((j % kNS) * kSlot) >> 4);
                // P_j (bf16, 2 per column) sits in the first 32 columns of S buffer pbuf
                tc::mma_f16_ts(tmem + 128, tmem + pbuf * 64, dv, kIdescPV, j > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 1; kk < kKT / 16; ++kk)
                    tc::mma_f16_ts(tmem + 128, tmem + pbuf * 64 + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), kIdescPV, 1u);
                tc::mma_commit(bar.pv_done[pbuf]);
                return true;
            };
            bool ok = tc::mbar_wait(bar.q_full, 0, abort, err, 3, s.polls);
            for (int k = 0; ok && k < njobs; ++k) {
                const int slot = k % kNS, sb = k & 1;
                if (!tc::mbar_wait(bar.k_full[slot], (k / kNS) & 1, abort, err, 4, s.polls)) { ok = false; break; }
                if (k >= 2 && !tc::mbar_wait(bar.s_free[sb], ((k - 2) >> 1) & 1, abort, err, 5, s.polls)) { ok = false; break; }
                tc::fence_after_sync();
                const uint64_t dk = dK0 + (uint64_t)((slot * kSlot) >> 4);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    tc::mma_f16_ss(tmem + sb * 64, dQ + (uint64_t)(((kk >> 2) * (kQBytes / 2) + (kk & 3) * 32) >> 4),
                                   dk + (uint64_t)(((kk >> 2) * kKVHalf + (kk & 3) * 32) >> 4), kIdescS, kk > 0 ? 1u : 0u);
                tc::mma_commit(bar.s_full[sb]);
                if (k >= 1 && !issue_pv(k - 1)) { ok = false; break; }
            }
            if (ok) ok = issue_pv(njobs - 1);
            if (!ok) {
                // drain the MMAs already issued before TMEM is released
                tc::mma_commit(bar.drain);
                for (long long it = 0; it < (1ll << 22); ++it)
                    if (tc::mbar_try(bar.drain, 0)) break;
            }
        }
    } else {
        // ---- softmax: one thread per row ---------------------------------------------------
        const int q4 = warp & 3;
        const int row = q4 * 32 + lane;
        const int pl = row / G, h = row % G;
        const int i = spos[pl];
        const bool valid = i < s.n;
        const int diag = i / s.B;
        const int* li = ridx + (valid ? tri_offset(i, s.B) : 0);
        const float* lb = rbias + (valid ? tri_offset(i, s.B) : 0);
        const int cnt = valid ? counts[i] : 0;
        ChunkSource<MASK> cs;
        cs.init(li, MASK ? rmask + (long long)(valid ? i : 0) * rt.words : nullptr, rt.words, cnt > 0);
        // the row's next two routed chunks stay in registers, so the global load of an entry is
        // issued at least one tile before the entry is compared
        int cur = 0;
        int nxt = cnt > 0 ? cs.at(0) : INT_MAX;
        float nbias = cnt > 0 ? lb[0] : 0.f;
        int nxt2 = cnt > 1 ? cs.at(1) : INT_MAX;
        float nbias2 = cnt > 1 ? lb[1] : 0.f;
        // two chunks per job: entries cur+2, cur+3 as well, and the queue only shifts at the end
        // of a job, so no compare waits on a load issued in the same job
        int nxt3 = CPT > 1 && cnt > 2 ? cs.at(2) : INT_MAX;
        float nbias3 = CPT > 1 && cnt > 2 ? lb[2] : 0.f;
        int nxt4 = CPT > 1 && cnt > 3 ? cs.at(3) : INT_MAX;
        float nbias4 = CPT > 1 && cnt > 3 ? lb[3] : 0.f;
        const float scale2 = kLog2e * rsqrtf((float)kD);
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int k = 0; k < njobs; ++k) {
            const int sb = k & 1;
            // waits are made warp-uniform: the tcgen05 loads and stores below are .sync.aligned
            if (!__all_sync(0xffffffffu, tc::mbar_wait(bar.s_full[sb], (k >> 1) & 1, abort, err, 6, s.polls))) { ok = false; break; }
            tc::fence_after_sync();
            float v[64];
            tc::tmem_ld32(lane_base + sb * 64, v);
            tc::tmem_ld32(lane_base + sb * 64 + 32, v + 32);
            tc::tmem_wait_ld();
            tc::fence_before_sync();
            tc::mbar_arrive(bar.s_free[sb]);
            const int c = jobs[k / NH];
            const int j0 = c * UB + (k % NH) * kKT;
            float bias2 = -INFINITY, bias2b = -INFINITY;   // per 32-key half (equal when CPT == 1)
            bool causal = false;
            int adv = 0;   // entries of the row's list consumed by this job (CPT > 1)
            if (CPT == 1) {
                if (valid) {
                    if (nxt == c) bias2 = nbias * kLog2e;
                    else if (c == diag) { bias2 = 0.f; causal = j0 + kKT - 1 > i; }
                }
                bias2b = bias2;
            } else if (valid) {
                const int c0 = c * 2, c1 = c0 + 1;
                const bool m0 = nxt == c0;
                const int nn = m0 ? nxt2 : nxt;
                const float nb = m0 ? nbias2 : nbias;
                const bool m1 = nn == c1;
                bias2 = m0 ? nbias * kLog2e : c0 == diag ? 0.f : -INFINITY;
                bias2b = m1 ? nb * kLog2e : c1 == diag ? 0.f : -INFINITY;
                causal = (c0 == diag || c1 == diag) && j0 + kKT - 1 > i;
                adv = (m0 ? 1 : 0) + (m1 ? 1 : 0);
            }
            if (causal) {
                // diagonal tile: keys past the query are masked
#pragma unroll
                for (int e = 0; e < 64; ++e)
                    if (j0 + e > i) v[e] = -INFINITY;
            }
            // tile maximum of the biased logits: max over raw scores (three-input tree), then scale
            // (scale2 > 0)
            float mx8[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const float t1 = fmax3(v[a], v[a + 8], v[a + 16]), t2 = fmax3(v[a + 24], v[a + 32], v[a + 40]);
                mx8[a] = fmax3(fmax3(v[a + 48], v[a + 56], t1), t2, t2);
            }
            float mt;
            if (CPT == 1) {
                const float smax = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
                mt = bias2 == -INFINITY ? -INFINITY : fmaf(smax, scale2, bias2);
            } else {
                // the two halves' maxima (columns 0-31 and 32-63), each with its own bias
                float ha = -INFINITY, hb = -INFINITY;
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    ha = fmax3(ha, v[e], v[e + 1]);
                    hb = fmax3(hb, v[32 + e], v[32 + e + 1]);
                }
                const float ma = bias2 == -INFINITY ? -INFINITY : fmaf(ha, scale2, bias2);
                const float mb = bias2b == -INFINITY ? -INFINITY : fmaf(hb, scale2, bias2b);
                mt = fmaxf(ma, mb);
            }
            const bool need = (m != -INFINITY) && (mt > m + 8.f);
            if (m == -INFINITY) m = mt;
            if (__any_sync(0xffffffffu, need)) {
                // rescale O: wait until the previous P V has landed
                if (!__all_sync(0xffffffffu, tc::mbar_wait(bar.pv_done[(k - 1) & 1], ((k - 1) >> 1) & 1, abort, err, 7, s.polls))) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const float f = need ? ex2_approx(m - mt) : 1.f;
                if (need) { l *= f; m = mt; }
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {
                    float o[32];
                    tc::tmem_ld32(lane_base + 128 + cb * 32, o);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= f;
                    tc::tmem_st32(lane_base + 128 + cb * 32, o);
                }
            }
            // p = 2^(s*scale2 + bias2 - m): one FMA and one ex2 per element; P (bf16 pairs) goes to
            // the first 32 columns of this job's S buffer.  A warp whose rows all skip the tile
            // writes zeros without computing.
            const uint32_t pdst = lane_base + sb * 64;
            if (__all_sync(0xffffffffu, bias2 == -INFINITY && bias2b == -INFINITY)) {
                uint32_t z[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) z[e] = 0u;
                tc::tmem_st16(pdst, z);
                tc::tmem_st16(pdst + 16, z);
            } else {
                const float mref = m == -INFINITY ? 0.f : m;
                // pairs of columns in f32x2: x = s * scale2 + off, then 2^x per lane, the running
                // sums in two packed accumulators
                const unsigned long long sc2 = f2(scale2, scale2);
                unsigned long long ls2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const float off = (half == 0 ? bias2 : bias2b) - mref;
                    const unsigned long long off2 = f2(off, off);
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float x0, x1;
                        unf2(ffma2(f2(v[32 * half + 2 * e], v[32 * half + 2 * e + 1]), sc2, off2), x0, x1);
                        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                        ls2[e & 1] = fadd2(ls2[e & 1], f2(p0, p1));
                        __nv_bfloat162 t2 = __floats2bfloat162_rn(p0, p1);
                        pk[e] = *reinterpret_cast<uint32_t*>(&t2);
                    }
                    tc::tmem_st16(pdst + 16 * half, pk);
                }
                float a0, a1, b0, b1;
                unf2(ls2[0], a0, a1);
                unf2(ls2[1], b0, b1);
                l += (a0 + a1) + (b0 + b1);
            }
            tc::tmem_wait_st();
            tc::fence_before_sync();
            tc::mbar_arrive(bar.p_full[sb]);
            if (CPT == 1) {
                if (k % NH == NH - 1 && nxt == c) {
                    ++cur;
                    nxt = nxt2;
                    nbias = nbias2;
                    nxt2 = cur + 1 < cnt ? cs.at(cur + 1) : INT_MAX;
                    nbias2 = cur + 1 < cnt ? lb[cur + 1] : 0.f;
                }
            } else if (adv == 1) {
                ++cur;
                nxt = nxt2; nbias = nbias2;
                nxt2 = nxt3; nbias2 = nbias3;
                nxt3 = nxt4; nbias3 = nbias4;
                nxt4 = cur + 3 < cnt ? cs.at(cur + 3) : INT_MAX;
                nbias4 = cur + 3 < cnt ? lb[cur + 3] : 0.f;
            } else if (adv == 2) {
                cur += 2;
                nxt = nxt3; nbias = nbias3;
                nxt2 = nxt4; nbias2 = nbias4;
                nxt3 = cur + 2 < cnt ? cs.at(cur + 2) : INT_MAX;
                nbias3 = cur + 2 < cnt ? lb[cur + 2] : 0.f;
                nxt4 = cur + 3 < cnt ? cs.at(cur + 3) : INT_MAX;
                nbias4 = cur + 3 < cnt ? lb[cur + 3] : 0.f;
            }
        }
        // ---- epilogue: O / l -> bf16 --------------------------------------------------------
        if (ok && njobs > 0 &&
            __all_sync(0xffffffffu, tc::mbar_wait(bar.pv_done[(njobs - 1) & 1], ((njobs - 1) >> 1) & 1, abort, err, 9, s.polls))) {
            tc::fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16* orow = valid ? O + (long long)b * s.os[0] + (long long)i * s.os[1] +
                                              (long long)(r * G + h) * s.os[2]
                                        : nullptr;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
                float o[32];
                tc::tmem_ld32(lane_base + 128 + cb * 32, o);
                tc::tmem_wait_ld();
                if (orow) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 w4;
                        __nv_bfloat162 a0 = __floats2bfloat162_rn(o[e] * inv, o[e + 1] * inv);
                        __nv_bfloat162 a1 = __floats2bfloat162_rn(o[e + 2] * inv, o[e + 3] * inv);
                        __nv_bfloat162 a2 = __floats2bfloat162_rn(o[e + 4] * inv, o[e + 5] * inv);
                        __nv_bfloat162 a3 = __floats2bfloat162_rn(o[e + 6] * inv, o[e + 7] * inv);
                        w4.x = *reinterpret_cast<uint32_t*>(&a0);
                        w4.y = *reinterpret_cast<uint32_t*>(&a1);
                        w4.z = *reinterpret_cast<uint32_t*>(&a2);
                        w4.w = *reinterpret_cast<uint32_t*>(&a3);
                        *reinterpret_cast<uint4*>(orow + cb * 32 + e) = w4;
                    }
                }
            }
        }
    }
    // ---- teardown -----------------------------------------------------------------------------
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

bool cluster_disabled()
{
    // DASH_CLUSTER=0 keeps positions in sequence order (no grouping; comparison runs and tests)
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("DASH_CLUSTER");
        v = (e && e[0] == '0') ? 1 : 0;
    }
    return v == 1;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 4-D map over a [batch, n, heads, 128] bf16 tensor (element strides st), box (64 d, bh heads,
// bp positions, 1), 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* map, const void* ptr, int batch, int n, int heads, const long long st[3], int bh,
              int bp)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {128, (cuuint64_t)heads, (cuuint64_t)n, (cuuint64_t)batch};
    cuuint64_t strides[3] = {(cuuint64_t)st[2] * 2, (cuuint64_t)st[1] * 2, (cuuint64_t)st[0] * 2};
    if (batch == 1) strides[2] = strides[1] * (cuuint64_t)n;   // unused dimension: any legal stride
    cuuint32_t box[4] = {64, (cuuint32_t)bh, (cuuint32_t)bp, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult rc = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return rc == CUDA_SUCCESS;
}

}  // namespace

bool s2_make_map(CUtensorMap* map, const void* ptr, int batch, int n, int heads, const long long st[3], int bh, int bp)
{
    return make_map(map, ptr, batch, n, heads, st, bh, bp);
}

bool s2_encode_available() { return encode_fn() != nullptr; }

bool s2_grouping_enabled(const Shape& s) { return (s.g == 8 || s.g == 16) && !cluster_disabled(); }

cudaError_t launch_group_positions(const Shape& s, const Routes& rt, int P, int* perm, cudaStream_t st)
{
    if (s.n <= 0) return cudaSuccess;
    const int Wn = kWinTiles * P;
    group_positions_kernel<<<dim3((s.n + Wn - 1) / Wn, s.batch * s.hkv), 1024, 0, st>>>(s, rt, P, perm);
    return cudaGetLastError();
}

// union units (chunks, or 64-key tiles of two 32-key chunks) a block's job list may hold
int attend_units(const Shape& s) { return (s.B >= kKT ? s.T : s.T / 2) + 2; }

bool attend_tc_supported(const Shape& s, int dtype)
{
    return dtype == DASH_BF16 && s.d == 128 && (s.B == 32 || s.B == 64 || s.B == 128) && s.g >= 1 && s.g <= 16 &&
           (kRows % s.g) == 0 && encode_fn() != nullptr && attend_units(s) * 4 <= 16 * 1024;
}

size_t attend_tc_smem(const Shape& s)
{
    return 1024 + kOffJobs + (size_t)attend_units(s) * 4;
}

cudaError_t launch_attend_prefill_tc(const Shape& s, const void* Q, const void* K, const void* V, void* O,
                                     const Routes& rt, int* perm, int* err, cudaStream_t st, bool mask)
{
    CUtensorMap mq, mq1, mk, mv;
    const int P = kRows / s.g;
    const bool group = perm && (s.g == 8 || s.g == 16) && !cluster_disabled();
    if (group && s.n > 0) {
        const int Wn = kWinTiles * P;
        group_positions_kernel<<<dim3((s.n + Wn - 1) / Wn, s.batch * s.hkv), 1024, 0, st>>>(s, rt, P, perm);
        const cudaError_t eg = cudaGetLastError();
        if (eg != cudaSuccess) return eg;
    }
    if (!make_map(&mq, Q, s.batch, s.n, s.hq, s.qs, s.g, P) || !make_map(&mq1, Q, s.batch, s.n, s.hq, s.qs, s.g, 1) ||
        !make_map(&mk, K, s.batch, s.n, s.hkv, s.ks, 1, kKT) || !make_map(&mv, V, s.batch, s.n, s.hkv, s.vs, 1, kKT))
        return cudaErrorInvalidValue;
    const size_t smem = attend_tc_smem(s);
    if (mask && !rt.bitmask) return cudaErrorInvalidValue;
    auto kern = s.B >= kKT ? (mask ? attend_prefill_tc_kernel<1, true> : attend_prefill_tc_kernel<1, false>)
                           : (mask ? attend_prefill_tc_kernel<2, true> : attend_prefill_tc_kernel<2, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long nblk = (s.n + P - 1) / P;
    const unsigned grid = (unsigned)(nblk * s.batch * s.hkv);
    if (grid == 0) return cudaSuccess;
    kern<<<grid, 192, smem, st>>>(mq, mq1, mk, mv, s, rt, (__nv_bfloat16*)O, err, group ? (const int*)perm : nullptr);
    return cudaGetLastError();
}

}  // namespace dash
