// stage2_pair.cu -- Stage 2 prefill on the sm_100a tensor cores (tcgen05 + TMEM + TMA): one block
// per PAIR of 128-row query tiles that walk one shared list of 128-key jobs.
//
// DashAttention (xllm-io paper review, section 3, Proposition 4.1 and the "Stage 2" kernel row):
// per query row, o = softmax(<q,k_j>/sqrt(d) + d_j) V over the tokens of the routed chunks
// (d_j = the chunk's bias) and the diagonal tokens c(i)B..i (d_j = 0), in one online-softmax pass
// over the routed chunks.
//
// A tile = 128 query rows = (128/g positions) x (g heads) of one (sequence, KV head).  The heads
// of a position share one routing list, so a tile's rows need the union of its positions' routed
// chunks plus their diagonal chunks.  The block's two tiles hold 2 * 128/g consecutive positions
// of the (route-grouped) position order and walk the union over both, ascending, in jobs of 128
// keys (128/B chunks per job).  Each K and V tile that is loaded serves both tiles (256 rows),
// which halves the L2-to-shared-memory traffic per FLOP of a one-tile walk; rows that did not
// route a job's chunk get -inf there.
//
// TMEM (512 columns): tile u keeps S_u in columns [256u, 256u+128) (P_u as bf16 pairs in columns
// [0, 32) and [64, 96) of it: each 64-key half over the start of its own S columns) and O_u in
// [256u+128, 256u+256).  Roles (20 warps):
//   warp 0      TMA producer: both Q tiles once, then per job K and V (two-slot rings)
//   warp 1      TMEM owner; one thread issues the MMAs (S = Q K^T: M=128, N=128, K=128;
//               O += P V: M=128, N=128, K=128 with P from TMEM) in the order
//                 S_0(0) S_1(0) | PV_0(j) S_0(j+1) PV_1(j) S_1(j+1) | ...
//               so that one tile's softmax runs while the tensor core works on the other tile
//   warp 2      routing: one lane per position walks the position's routed chunks and writes,
//               for every job, each position's bias per chunk of the job (log2 units; 0 on the
//               position's diagonal chunk; -inf where it did not route the chunk) into a ring of
//               kRD jobs in shared memory, ahead of the softmax
//   warp 3      idle after the set-up
//   warps 4-19  softmax, two threads per row: tile u = (warp-4)/8 takes the 64-key half
//               hf = ((warp-4)/4) % 2 of every job for the rows of TMEM lane quarter warp % 4.
//               Per job: the half's maximum of the biased logits, exchanged with the other half
//               through shared memory; the row's running maximum m moves only when the job
//               exceeds it by more than 2^8 (O and the sums are then rescaled), otherwise the
//               stale maximum is kept (values stay <= 2^8, exact in the final normalisation);
//               p = 2^(s - m) as bf16 pairs into the half's 32 P columns of TMEM.
// (The two halves' P columns lie inside each half's own S columns, so neither half writes where
// the other still reads S.)
// MASK = true reads the routed support from the bit-packed block mask (one bit per (position,
// chunk), 32 chunks per word) instead of the ascending chunk lists; the biases are read in the
// same ascending order, so both variants compute identical results.
// Every wait is bounded (mbarriers only, no named barriers between roles or halves); on time-out
// the block records an error code and leaves.
#include <climits>

#include "dash_common.cuh"
#include "tc_ptx.cuh"

namespace dash {
namespace {

constexpr int kRows = 128, kD = 128, kJK = 128;        // rows per tile, head dim, keys per job
constexpr int kQBytes = kRows * kD * 2;                 // 32 KB per tile: two d-halves of [128 rows][64 d]
constexpr int kKVHalf = kJK * 64 * 2;                   // 16 KB: [128 keys][64 d]
constexpr int kKVBytes = 2 * kKVHalf;                   // 32 KB: K (or V) of one job
constexpr int kOffQ = 0;
constexpr int kOffK = 2 * kQBytes;                      // 64 KB: K ring, 2 slots
constexpr int kOffV = kOffK + 2 * kKVBytes;             // 128 KB: V ring, 2 slots
constexpr int kRD = 8;                                  // jobs of routing data prepared ahead
constexpr int kNumBars = 1 + 2 * 4 + 2 * 5 + kRD + 1;
constexpr int kOffBar = kOffV + 2 * kKVBytes;           // 192 KB
constexpr int kOffMisc = kOffBar + kNumBars * 8;        // tmem base, abort, jobs, units
constexpr int kOffX = kOffMisc + 32;                    // [2 job parity][2 tiles][2 halves][128 rows] maxima
constexpr int kOffL = kOffX + 2 * 2 * 2 * kRows * 4;    // [2 tiles][2 halves][128 rows] row sums
constexpr int kOffRB = kOffL + 2 * 2 * kRows * 4;       // route ring [kRD][J][2P] floats, then positions, units
constexpr int kThreads = 640;
constexpr int kMaxP2 = 64;                              // positions per pair: 2 * 128 / g, g >= 4
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescS = tc::idesc_bf16(128, 128, false, false);
constexpr uint32_t kIdescPV = tc::idesc_bf16(128, 128, false, true);

__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
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

// K slot j % 2 holds K_j until S_0(j) and S_1(j) are done (k_free); V slot j % 2 holds V_j until
// PV_0(j) and PV_1(j) are done (v_free).  Per tile u: s_full (S_u of a job is in TMEM), xchg (the
// tile's 256 softmax threads posted their half maxima), p_full (they wrote P_u), pv_done (PV_u
// completed), lsum (the two halves' row sums are posted, at the end).  route[k]: the routing data
// of job j (k = j % kRD) is in shared memory.
struct Bars {
    uint32_t q_full, k_full[2], v_full[2], k_free[2], v_free[2];
    uint32_t s_full[2], xchg[2], p_full[2], pv_done[2], lsum[2];
    uint32_t route[kRD], drain;
};

__device__ __forceinline__ Bars make_bars(uint32_t base)
{
    Bars b;
    uint32_t a = base + kOffBar;
    b.q_full = a; a += 8;
    for (int k = 0; k < 2; ++k) { b.k_full[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.v_full[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.k_free[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.v_free[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.s_full[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.xchg[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.p_full[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.pv_done[k] = a; a += 8; }
    for (int k = 0; k < 2; ++k) { b.lsum[k] = a; a += 8; }
    for (int k = 0; k < kRD; ++k) { b.route[k] = a; a += 8; }
    b.drain = a;
    return b;
}

// A position's routed chunks in ascending order with their biases, from the chunk list (MASK =
// false) or from the bit-packed mask (MASK = true; the bias of the k-th routed chunk is the k-th
// entry of the position's bias list in both cases).  Two banks of four entries: the current bank
// is consumed while the next one's loads are in flight, and the banks swap only when the current
// one is used up, so no instruction reads a register whose load was issued shortly before.
template <bool MASK>
struct RouteQueue {
    int cc[4], nc[4];
    float cb[4], nb[4];
    int k, cnt, next;
    const int* li;
    const float* lb;
    const uint32_t* mw;
    uint32_t word, word2;
    int wi, words;

    __device__ __forceinline__ int fetch_chunk()
    {
        if constexpr (MASK) {
            while (word == 0u) {
                if (++wi >= words) return INT_MAX;
                word = word2;
                word2 = wi + 1 < words ? mw[wi + 1] : 0u;
            }
            const int b = __ffs(word) - 1;
            word &= word - 1u;
            return (wi << 5) + b;
        } else {
            return li[next];
        }
    }
    __device__ __forceinline__ void fill_next()
    {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (next < cnt) {
                nc[q] = fetch_chunk();
                nb[q] = lb[next];
                ++next;
            } else {
                nc[q] = INT_MAX;
                nb[q] = 0.f;
            }
        }
    }
    __device__ __forceinline__ void swap_banks()
    {
#pragma unroll
        for (int q = 0; q < 4; ++q) { cc[q] = nc[q]; cb[q] = nb[q]; }
        k = 0;
        fill_next();
    }
    __device__ __forceinline__ void init(const int* li_, const float* lb_, const uint32_t* mw_, int words_, int cnt_)
    {
        li = li_; lb = lb_; mw = mw_; words = words_; cnt = cnt_; next = 0; wi = 0;
        word = (MASK && cnt > 0) ? mw[0] : 0u;
        word2 = (MASK && cnt > 0 && words > 1) ? mw[1] : 0u;
        fill_next();
        swap_banks();
    }
    __device__ __forceinline__ int front() const { return k == 0 ? cc[0] : k == 1 ? cc[1] : k == 2 ? cc[2] : cc[3]; }
    __device__ __forceinline__ float front_bias() const { return k == 0 ? cb[0] : k == 1 ? cb[1] : k == 2 ? cb[2] : cb[3]; }
    __device__ __forceinline__ void pop() { if (++k == 4) swap_banks(); }
};

// J = chunks per 128-key job (128 / B).
template <int J, bool MASK>
__global__ void __launch_bounds__(kThreads, 1) attend_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                                  const __grid_constant__ CUtensorMap tmQ1,
                                                                  const __grid_constant__ CUtensorMap tmK,
                                                                  const __grid_constant__ CUtensorMap tmV,
                                                                  Shape s, Routes rt,
                                                                  __nv_bfloat16* __restrict__ O, int* err,
                                                                  const int* __restrict__ perm)
{
    constexpr int SEG = kJK / J;   // keys per chunk of a job (= B)
    extern __shared__ char smem_raw[];
    char* sm = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = tc::smem_addr(sm);
    const Bars bar = make_bars(base);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffMisc);
    volatile int* abort = reinterpret_cast<volatile int*>(sm + kOffMisc + 4);
    int* njobs_s = reinterpret_cast<int*>(sm + kOffMisc + 8);
    int* nunits_s = reinterpret_cast<int*>(sm + kOffMisc + 12);
    float* xsh = reinterpret_cast<float*>(sm + kOffX);
    float* lsh = reinterpret_cast<float*>(sm + kOffL);
    uint32_t* umask = reinterpret_cast<uint32_t*>(sm + kOffK);   // set-up scratch until the first TMA

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = s.g, P = kRows / G, P2 = 2 * P;
    float* rb = reinterpret_cast<float*>(sm + kOffRB);            // [kRD][J][P2]
    int* spos = reinterpret_cast<int*>(sm + kOffRB + kRD * J * P2 * 4);
    uint16_t* jobs = reinterpret_cast<uint16_t*>(sm + kOffRB + kRD * J * P2 * 4 + 4 * P2);
    const int nblk = (s.n + P - 1) / P;
    const int npairs = (nblk + 1) / 2;
    const int br = blockIdx.x % (s.batch * s.hkv);
    const int pp = npairs - 1 - blockIdx.x / (s.batch * s.hkv);   // heaviest pairs first
    const int b = br / s.hkv, r = br % s.hkv;
    const int i0 = pp * P2;
    const int* counts = rt.counts + (long long)br * s.n;
    const int* ridx = rt.idx + (long long)br * rt.cap;
    const float* rbias = rt.bias + (long long)br * rt.cap;
    const uint32_t* rmask = MASK ? rt.bitmask + (long long)br * s.n * rt.words : nullptr;
    const int W = (s.T + 32) >> 5;

    // ---- set-up: barriers, TMEM, union of the pair's routed + diagonal chunks ------------------
    if (tid == 0) {
        tc::mbar_init(bar.q_full, 1);
        for (int k = 0; k < 2; ++k) {
            tc::mbar_init(bar.k_full[k], 1);
            tc::mbar_init(bar.v_full[k], 1);
            tc::mbar_init(bar.k_free[k], 1);
            tc::mbar_init(bar.v_free[k], 1);
            tc::mbar_init(bar.s_full[k], 1);
            tc::mbar_init(bar.xchg[k], 256);
            tc::mbar_init(bar.p_full[k], 256);
            tc::mbar_init(bar.pv_done[k], 1);
            tc::mbar_init(bar.lsum[k], 256);
        }
        for (int k = 0; k < kRD; ++k) tc::mbar_init(bar.route[k], 1);
        tc::mbar_init(bar.drain, 1);
        *abort = 0;
        tc::mbar_fence_init();
    }
    if (warp == 1) {
        __syncwarp();
        tc::tmem_alloc(tc::smem_addr(tmem_slot), kTmemCols);
    }
    for (int w = tid; w < W; w += blockDim.x) umask[w] = 0u;
    // slots i0 .. i0 + 2P - 1 of the grouped order (positions past the end stay in place, masked)
    for (int p = tid; p < P2; p += blockDim.x) {
        const int k = i0 + p;
        spos[p] = perm && k < s.n ? perm[(long long)br * s.n + k] : k;
    }
    __syncthreads();
    if constexpr (MASK) {
        // union = OR of the positions' mask words
        for (int e = tid; e < P2 * rt.words; e += blockDim.x) {
            const int i = spos[e / rt.words];
            if (i >= s.n) continue;
            const uint32_t w = rmask[(long long)i * rt.words + e % rt.words];
            if (w) atomicOr(&umask[e % rt.words], w);
        }
        if (tid < P2 && spos[tid] < s.n) {
            const int c = spos[tid] / s.B;
            atomicOr(&umask[c >> 5], 1u << (c & 31));
        }
    } else {
        // the positions' list lengths and their prefix sums (scratch in the V ring), then every
        // list entry by a flat index, several independent loads per thread in flight
        int* pcnt = reinterpret_cast<int*>(sm + kOffV);
        int* poff = pcnt + kMaxP2;
        for (int p = tid; p < P2; p += blockDim.x) {
            const int i = spos[p];
            pcnt[p] = i < s.n ? counts[i] : 0;
            if (i < s.n) {
                const int c = i / s.B;
                atomicOr(&umask[c >> 5], 1u << (c & 31));
            }
        }
        __syncthreads();
        if (warp == 0) {
            int basec = 0;
            for (int p0 = 0; p0 < P2; p0 += 32) {
                const int v = p0 + lane < P2 ? pcnt[p0 + lane] : 0;
                int incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                if (p0 + lane < P2) poff[p0 + lane] = basec + incl - v;
                basec += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) poff[P2] = basec;
        }
        __syncthreads();
        const int total = poff[P2];
        auto entry = [&](int e) -> int {   // chunk id of flat entry e (binary search over poff)
            int lo = 0, hi = P2 - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (poff[mid] <= e) lo = mid; else hi = mid - 1;
            }
            return ridx[tri_offset(spos[lo], s.B) + (e - poff[lo])];
        };
        for (int e0 = tid; e0 < total; e0 += 4 * blockDim.x) {
            int c[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int e = e0 + q * blockDim.x;
                c[q] = e < total ? entry(e) : -1;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (c[q] >= 0) atomicOr(&umask[c[q] >> 5], 1u << (c[q] & 31));
        }
    }
    __syncthreads();
    if (warp == 0) {   // ordered bitmask -> list of chunk ids, padded to whole jobs
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
                jobs[at++] = (uint16_t)(((w0 + lane) << 5) + bit);
                bb &= bb - 1u;
            }
            basec += __shfl_sync(0xffffffffu, incl, 31);
        }
        __syncwarp();
        // padding entries repeat the last unit (real keys, finite values); every row masks them
        const int nj = (basec + J - 1) / J;
        if (lane < nj * J - basec) jobs[basec + lane] = basec > 0 ? jobs[basec - 1] : (uint16_t)0;
        if (lane == 0) {
            *njobs_s = nj;
            *nunits_s = basec;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int njobs = *njobs_s;
    const int nunits = *nunits_s;

    if (warp == 0) {
        // ---- TMA producer ----------------------------------------------------------------------
        if (lane == 0 && njobs > 0) {
            tc::prefetch_tmap(&tmQ);
            tc::prefetch_tmap(&tmK);
            tc::prefetch_tmap(&tmV);
            tc::mbar_expect_tx(bar.q_full, 2 * kQBytes);
            if (perm) {
                // one box of g rows per position (g = 8 or 16 keeps every box 1024-byte aligned)
                tc::prefetch_tmap(&tmQ1);
                for (int p = 0; p < P2; ++p) {
                    const uint32_t dst = base + kOffQ + (p / P) * kQBytes + (p % P) * G * 128;
                    tc::tma_load_4d(dst, &tmQ1, bar.q_full, 0, r * G, spos[p], b);
                    tc::tma_load_4d(dst + kQBytes / 2, &tmQ1, bar.q_full, 64, r * G, spos[p], b);
                }
            } else {
                for (int u = 0; u < 2; ++u) {
                    const uint32_t dst = base + kOffQ + u * kQBytes;
                    tc::tma_load_4d(dst, &tmQ, bar.q_full, 0, r * G, i0 + u * P, b);
                    tc::tma_load_4d(dst + kQBytes / 2, &tmQ, bar.q_full, 64, r * G, i0 + u * P, b);
                }
            }
            // loads in the order of first use: K_0, V_0, K_1, V_1, ...; slot j % 2 is refilled
            // once both tiles' MMAs of job j - 2 that read it have completed
            int lastk[2] = {-1, -1}, lastv[2] = {-1, -1};
            for (int j = 0; j < njobs; ++j) {
                const int slot = j & 1;
                if (j >= 2 && !tc::mbar_wait(bar.k_free[slot], ((j >> 1) - 1) & 1, abort, err, 21)) break;
                lastk[slot] = j;
                tc::mbar_expect_tx(bar.k_full[slot], kKVBytes);
#pragma unroll
                for (int sg = 0; sg < J; ++sg) {
                    const int key0 = jobs[j * J + sg] * SEG;
                    const uint32_t dst = base + kOffK + slot * kKVBytes + sg * SEG * 128;
                    tc::tma_load_4d(dst, &tmK, bar.k_full[slot], 0, r, key0, b);
                    tc::tma_load_4d(dst + kKVHalf, &tmK, bar.k_full[slot], 64, r, key0, b);
                }
                if (j >= 2 && !tc::mbar_wait(bar.v_free[slot], ((j >> 1) - 1) & 1, abort, err, 22)) break;
                lastv[slot] = j;
                tc::mbar_expect_tx(bar.v_full[slot], kKVBytes);
#pragma unroll
                for (int sg = 0; sg < J; ++sg) {
                    const int key0 = jobs[j * J + sg] * SEG;
                    const uint32_t dst = base + kOffV + slot * kKVBytes + sg * SEG * 128;
                    tc::tma_load_4d(dst, &tmV, bar.v_full[slot], 0, r, key0, b);
                    tc::tma_load_4d(dst + kKVHalf, &tmV, bar.v_full[slot], 64, r, key0, b);
                }
            }
            if (*abort) {
                // let this block's TMA copies still in flight land before its shared memory goes away
                for (int k = 0; k < 2; ++k) {
                    if (lastk[k] >= 0)
                        for (long long it = 0; it < (1ll << 22); ++it)
                            if (tc::mbar_try(bar.k_full[k], (lastk[k] >> 1) & 1)) break;
                    if (lastv[k] >= 0)
                        for (long long it = 0; it < (1ll << 22); ++it)
                            if (tc::mbar_try(bar.v_full[k], (lastv[k] >> 1) & 1)) break;
                }
                for (long long it = 0; it < (1ll << 22); ++it)
                    if (tc::mbar_try(bar.q_full, 0)) break;
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer --------------------------------------------------------------------------
        if (lane == 0 && njobs > 0) {
            // descriptors of Q_0 and of slot 0; a tile, slot or K-step moves only the start-address
            // field (16-byte units, no carry), so each MMA is issued after one add
            const uint64_t dQ0 = tc::sw128_desc(base + kOffQ, 16, 1024);
            const uint64_t dK0 = tc::sw128_desc(base + kOffK, 16, 1024);
            const uint64_t dV0 = tc::sw128_desc(base + kOffV, kKVHalf, 1024);
            auto issue_s = [&](int u, int j) {
                const uint64_t dq = dQ0 + (uint64_t)((u * kQBytes) >> 4);
                const uint64_t dk = dK0 + (uint64_t)(((j & 1) * kKVBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk)
                    tc::mma_f16_ss(tmem + 256u * u, dq + (uint64_t)(((kk >> 2) * (kQBytes / 2) + (kk & 3) * 32) >> 4),
                                   dk + (uint64_t)(((kk >> 2) * kKVHalf + (kk & 3) * 32) >> 4), kIdescS,
                                   kk > 0 ? 1u : 0u);
                tc::mma_commit(bar.s_full[u]);
            };
            auto issue_pv = [&](int u, int j) {
                const uint64_t dv = dV0 + (uint64_t)(((j & 1) * kKVBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < kJK / 16; ++kk)   // P of keys 16kk.. : columns 8kk (+32 for the upper half)
                    tc::mma_f16_ts(tmem + 256u * u + 128u, tmem + 256u * u + kk * 8 + (kk >= 4 ? 32u : 0u),
                                   dv + (uint64_t)((kk * 2048) >> 4), kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                tc::mma_commit(bar.pv_done[u]);
            };
            bool ok = tc::mbar_wait(bar.q_full, 0, abort, err, 23) && tc::mbar_wait(bar.k_full[0], 0, abort, err, 24);
            if (ok) {
                tc::fence_after_sync();
                issue_s(0, 0);
                issue_s(1, 0);
                tc::mma_commit(bar.k_free[0]);
            }
            for (int j = 0; ok && j < njobs; ++j) {
                const bool more = j + 1 < njobs;
                if (!tc::mbar_wait(bar.p_full[0], j & 1, abort, err, 25) ||
                    !tc::mbar_wait(bar.v_full[j & 1], (j >> 1) & 1, abort, err, 26)) { ok = false; break; }
                tc::fence_after_sync();
                issue_pv(0, j);
                if (more) {
                    if (!tc::mbar_wait(bar.k_full[(j + 1) & 1], ((j + 1) >> 1) & 1, abort, err, 27)) { ok = false; break; }
                    tc::fence_after_sync();
                    issue_s(0, j + 1);
                }
                if (!tc::mbar_wait(bar.p_full[1], j & 1, abort, err, 28)) { ok = false; break; }
                tc::fence_after_sync();
                issue_pv(1, j);
                tc::mma_commit(bar.v_free[j & 1]);
                if (more) {
                    issue_s(1, j + 1);
                    tc::mma_commit(bar.k_free[(j + 1) & 1]);
                }
            }
            if (!ok) {
                // drain the MMAs already issued before TMEM is released
                tc::mma_commit(bar.drain);
                for (long long it = 0; it < (1ll << 22); ++it)
                    if (tc::mbar_try(bar.drain, 0)) break;
            }
        }
    } else if (warp == 2) {
        // ---- routing: lane = position (and position + 32 when the pair has 64) ------------------
        constexpr int kPerLane = kMaxP2 / 32;
        RouteQueue<MASK> rq[kPerLane];
        int diag[kPerLane];
        bool vld[kPerLane];
#pragma unroll
        for (int q = 0; q < kPerLane; ++q) {
            const int p = lane + 32 * q;
            const int i = p < P2 ? spos[p] : INT_MAX;
            vld[q] = i < s.n;
            diag[q] = vld[q] ? i / s.B : -1;
            const long long toff = vld[q] ? tri_offset(i, s.B) : 0;
            rq[q].init(ridx + toff, rbias + toff, MASK ? rmask + (long long)(vld[q] ? i : 0) * rt.words : nullptr,
                       rt.words, vld[q] ? counts[i] : 0);
        }
        for (int j = 0; j < njobs; ++j) {
            const int slot = j % kRD;
            // slot reuse: both tiles' softmax of job j - kRD has finished reading it
            if (j >= kRD && !__all_sync(0xffffffffu, tc::mbar_wait(bar.p_full[0], (j - kRD) & 1, abort, err, 32) &&
                                                         tc::mbar_wait(bar.p_full[1], (j - kRD) & 1, abort, err, 33)))
                break;
            float* dst = rb + slot * J * P2;
#pragma unroll
            for (int sg = 0; sg < J; ++sg) {
                const int e = j * J + sg;
                const int unit = jobs[e];
#pragma unroll
                for (int q = 0; q < kPerLane; ++q) {
                    const int p = lane + 32 * q;
                    float b2 = -INFINITY;
                    if (vld[q] && e < nunits) {
                        if (rq[q].front() == unit) {
                            b2 = rq[q].front_bias() * kLog2e;
                            rq[q].pop();
                        } else if (unit == diag[q]) {
                            b2 = 0.f;
                        }
                    }
                    if (p < P2) dst[sg * P2 + p] = b2;
                }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar.route[slot]);
        }
    } else if (warp >= 4) {
        // ---- softmax: tile u, key half hf, two threads per row ------------------------------------
        const int w4 = warp - 4;
        const int u = w4 >> 3, hf = (w4 >> 2) & 1;
        const int q4 = warp & 3;                  // TMEM lane quarter this warp may access
        const int row = q4 * 32 + lane;
        const int pl = row / G, h = row % G;
        const int pidx = u * P + pl;
        const int i = spos[pidx];
        const bool valid = i < s.n;
        const int diag = valid ? i / s.B : -1;
        const float scale2 = kLog2e * rsqrtf((float)kD);
        const uint32_t tbase = tmem + ((uint32_t)(q4 * 32) << 16) + 256u * u;
        // S of this half: columns 64 hf + [0, 64); its P (bf16 pairs) over the first 32 of them,
        // which only this half reads; O of this half: 128 + 64 hf + [0, 64)
        const uint32_t scol = 64u * hf, pcol = 64u * hf, ocol = 128u + 64u * hf;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < njobs; ++j) {
            const int slot = j % kRD;
            // waits are made warp-uniform: the tcgen05 loads and stores below are .sync.aligned
            if (!__all_sync(0xffffffffu, tc::mbar_wait(bar.route[slot], (j / kRD) & 1, abort, err, 34) &&
                                             tc::mbar_wait(bar.s_full[u], j & 1, abort, err, 29))) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            // this half's two 32-key blocks: bias (log2 units; -inf: not routed or padding) and
            // the block's first key when it lies on the row's diagonal chunk (causal mask)
            float b2[2];
            int j0[2];
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                const int kin = 64 * hf + 32 * cb;           // first key of the block within the job
                const int sg = kin / SEG;
                b2[cb] = rb[(slot * J + sg) * P2 + pidx];
                const int unit = jobs[j * J + sg];
                j0[cb] = unit == diag ? unit * SEG + kin % SEG : -1;
            }
            // pass 1: the half's maximum of the biased logits
            float xm = -INFINITY;
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                if (__all_sync(0xffffffffu, b2[cb] == -INFINITY)) continue;
                float v[32];
                tc::tmem_ld32(tbase + scol + 32 * cb, v);
                tc::tmem_wait_ld();
                if (j0[cb] >= 0) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (j0[cb] + e > i) v[e] = -INFINITY;
                }
                float a = fmax3(v[0], v[1], v[2]);
#pragma unroll
                for (int e = 3; e < 31; e += 2) a = fmax3(a, v[e], v[e + 1]);
                a = fmaxf(a, v[31]);
                if (b2[cb] != -INFINITY) xm = fmaxf(xm, fmaf(a, scale2, b2[cb]));
            }
            // the row's maximum over both halves (shared memory, per job parity)
            float* xs = xsh + (((j & 1) * 2 + u) * 2) * kRows;
            xs[hf * kRows + row] = xm;
            tc::mbar_arrive(bar.xchg[u]);
            if (!__all_sync(0xffffffffu, tc::mbar_wait(bar.xchg[u], j & 1, abort, err, 35))) { ok = false; break; }
            const float xr = fmaxf(xs[row], xs[kRows + row]);
            // the running maximum moves when the job exceeds it by more than 2^8 (or holds the
            // row's first used key); O (this half's 64 columns) and l are rescaled
            const bool need = xr != -INFINITY && (m == -INFINITY || xr > m + 8.f);
            if (__any_sync(0xffffffffu, need)) {
                const float f = need && m != -INFINITY ? ex2_approx(m - xr) : 1.f;
                if (__any_sync(0xffffffffu, f != 1.f)) {
                    // PV_u(j-1) has completed: it precedes S_u(j) on the tensor pipe
                    if (!__all_sync(0xffffffffu, tc::mbar_wait(bar.pv_done[u], (j - 1) & 1, abort, err, 30))) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
#pragma unroll
                    for (int ob = 0; ob < 2; ++ob) {
                        float o[32];
                        tc::tmem_ld32(tbase + ocol + 32 * ob, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= f;
                        tc::tmem_st32(tbase + ocol + 32 * ob, o);
                    }
                }
                l *= f;
                if (need) m = xr;
            }
            // pass 2: p = 2^(s*scale2 + bias2 - m), bf16 pairs into this half's 32 P columns; a
            // block that no row of the warp uses is written as zeros without computing
            const float mref = m == -INFINITY ? 0.f : m;
            const unsigned long long sc2 = f2(scale2, scale2);
            unsigned long long ls2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                uint32_t pk[16];
                if (__all_sync(0xffffffffu, b2[cb] == -INFINITY)) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) pk[e] = 0u;
                } else {
                    float v[32];
                    tc::tmem_ld32(tbase + scol + 32 * cb, v);
                    tc::tmem_wait_ld();
                    if (j0[cb] >= 0) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (j0[cb] + e > i) v[e] = -INFINITY;
                    }
                    const float off = b2[cb] - mref;
                    const unsigned long long off2 = f2(off, off);
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float x0, x1;
                        unf2(ffma2(f2(v[2 * e], v[2 * e + 1]), sc2, off2), x0, x1);
                        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                        ls2[e & 1] = fadd2(ls2[e & 1], f2(p0, p1));
                        __nv_bfloat162 t2 = __floats2bfloat162_rn(p0, p1);
                        pk[e] = *reinterpret_cast<uint32_t*>(&t2);
                    }
                }
                tc::tmem_st16(tbase + pcol + 16 * cb, pk);
            }
            float a0, a1, c0, c1;
            unf2(ls2[0], a0, a1);
            unf2(ls2[1], c0, c1);
            l += (a0 + a1) + (c0 + c1);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            tc::mbar_arrive(bar.p_full[u]);
        }
        // ---- epilogue: the two halves' sums, O / l -> bf16 (each half writes its 64 columns) -----
        if (ok && njobs > 0) {
            lsh[(u * 2 + hf) * kRows + row] = l;
            tc::mbar_arrive(bar.lsum[u]);
            if (__all_sync(0xffffffffu, tc::mbar_wait(bar.lsum[u], 0, abort, err, 36) &&
                                            tc::mbar_wait(bar.pv_done[u], (njobs - 1) & 1, abort, err, 31))) {
                tc::fence_after_sync();
                const float lt = lsh[(u * 2) * kRows + row] + lsh[(u * 2 + 1) * kRows + row];
                const float inv = lt > 0.f ? 1.f / lt : 0.f;
                __nv_bfloat16* orow = valid ? O + (long long)b * s.os[0] + (long long)i * s.os[1] +
                                                  (long long)(r * G + h) * s.os[2] + 64 * hf
                                            : nullptr;
#pragma unroll
                for (int ob = 0; ob < 2; ++ob) {
                    float o[32];
                    tc::tmem_ld32(tbase + ocol + 32 * ob, o);
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
                            *reinterpret_cast<uint4*>(orow + 32 * ob + e) = w4;
                        }
                    }
                }
            }
        }
    }
    // ---- teardown ---------------------------------------------------------------------------------
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

size_t pair_smem(const Shape& s)
{
    const int P2 = 2 * (kRows / s.g), J = s.B >= kJK ? 1 : kJK / s.B;
    return 1024 + (size_t)kOffRB + (size_t)kRD * J * P2 * 4 + 4 * (size_t)P2 + 2 * (size_t)(s.T + 2 + 4);
}

template <int J, bool MASK>
cudaError_t launch_j(const Shape& s, const CUtensorMap& mq, const CUtensorMap& mq1, const CUtensorMap& mk,
                     const CUtensorMap& mv, const Routes& rt, void* O, int* err, const int* perm, cudaStream_t st)
{
    auto kern = attend_pair_kernel<J, MASK>;
    const size_t smem = pair_smem(s);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int P = kRows / s.g;
    const long long nblk = (s.n + P - 1) / P;
    const unsigned grid = (unsigned)((nblk + 1) / 2 * s.batch * s.hkv);
    if (grid == 0) return cudaSuccess;
    kern<<<grid, kThreads, smem, st>>>(mq, mq1, mk, mv, s, rt, (__nv_bfloat16*)O, err, perm);
    return cudaGetLastError();
}

cudaError_t launch_attend_prefill_pair_impl(const Shape& s, const void* Q, const void* K, const void* V, void* O,
                                            const Routes& rt, int* perm, int* err, bool mask, cudaStream_t st)
{
    const int P = kRows / s.g;
    const bool group = perm && s2_grouping_enabled(s);
    if (group) {
        const cudaError_t eg = launch_group_positions(s, rt, P, perm, st);
        if (eg != cudaSuccess) return eg;
    }
    CUtensorMap mq, mq1, mk, mv;
    if (!s2_make_map(&mq, Q, s.batch, s.n, s.hq, s.qs, s.g, P) || !s2_make_map(&mq1, Q, s.batch, s.n, s.hq, s.qs, s.g, 1) ||
        !s2_make_map(&mk, K, s.batch, s.n, s.hkv, s.ks, 1, s.B) || !s2_make_map(&mv, V, s.batch, s.n, s.hkv, s.vs, 1, s.B))
        return cudaErrorInvalidValue;
    const int* pm = group ? perm : nullptr;
    if (mask) {
        switch (s.B) {
        case 32: return launch_j<4, true>(s, mq, mq1, mk, mv, rt, O, err, pm, st);
        case 64: return launch_j<2, true>(s, mq, mq1, mk, mv, rt, O, err, pm, st);
        default: return launch_j<1, true>(s, mq, mq1, mk, mv, rt, O, err, pm, st);
        }
    }
    switch (s.B) {
    case 32: return launch_j<4, false>(s, mq, mq1, mk, mv, rt, O, err, pm, st);
    case 64: return launch_j<2, false>(s, mq, mq1, mk, mv, rt, O, err, pm, st);
    default: return launch_j<1, false>(s, mq, mq1, mk, mv, rt, O, err, pm, st);
    }
}

}  // namespace

bool attend_pair_supported(const Shape& s, int dtype)
{
    return dtype == DASH_BF16 && s.d == kD && (s.B == 32 || s.B == 64 || s.B == 128) &&
           (s.g == 4 || s.g == 8 || s.g == 16) && s.T + 8 < 65536 && s2_encode_available() &&
           pair_smem(s) <= 227 * 1024;
}

cudaError_t launch_attend_prefill_pair(const Shape& s, const void* Q, const void* K, const void* V, void* O,
                                       const Routes& rt, int* perm, int* err, cudaStream_t st)
{
    return launch_attend_prefill_pair_impl(s, Q, K, V, O, rt, perm, err, false, st);
}

cudaError_t launch_attend_prefill_mask(const Shape& s, const void* Q, const void* K, const void* V, void* O,
                                       const Routes& rt, int* perm, int* err, cudaStream_t st)
{
    if (!rt.bitmask) return cudaErrorInvalidValue;
    return launch_attend_prefill_pair_impl(s, Q, K, V, O, rt, perm, err, true, st);
}

}  // namespace dash
