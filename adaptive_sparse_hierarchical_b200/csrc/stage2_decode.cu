// stage2_decode.cu -- Stage 2 of incremental decoding, bf16, d = 128, HBM-bound.
//
// DashAttention (xllm-io paper review, section 3, Prop. 4.1 and the "Stage 2" kernel row:
// decoding splits the routed chunks along KV to expose parallelism).  The single query of
// sequence b (g heads of KV head r) attends over its routed chunks (bias d_c) and the diagonal
// tokens of its own chunk.  One block per (split, sequence, KV head): a TMA producer warp keeps a
// 6-slot ring of 64-key K/V tiles (192 KB) in flight; three consumer warps take the split's tiles
// round-robin, each with its own online softmax over 16 rows (the g heads, padded), using
// m16n8k16 bf16 MMAs; the three states are merged in shared memory into the split's partial
// (o, m, l), which the merge kernel combines across splits.
#include <climits>
#include <cudaTypedefs.h>

#include "dash_common.cuh"
#include "stage2_mma.cuh"
#include "tc_ptx.cuh"

namespace dash {
namespace {

constexpr int kNSd = 6;           // ring slots
constexpr int kHalf = 64 * 64 * 2;
constexpr int kSlotB = 4 * kHalf; // K halves + V halves = 32 KB
constexpr int kCons = 3;          // consumer warps; job k goes to warp k % kCons and slot k % kNSd
// Every slot must have a single consumer that takes its jobs in order, so that a wait on the
// slot's "full" barrier is never more than one phase ahead (phase parity would alias otherwise).
static_assert(kNSd % kCons == 0, "each ring slot needs exactly one consumer warp");

// Byte offset of element (row, col) of a [64 rows][128 cols] bf16 tile stored by TMA as two
// 128-byte-swizzled halves of 64 columns.
__device__ __forceinline__ uint32_t sw_off(int row, int col)
{
    const int half = col >> 6, c = col & 63;
    return (uint32_t)(half * kHalf + row * 128 + ((((c >> 3) ^ (row & 7))) << 4) + (c & 7) * 2);
}

// Persistent: gridDim.x blocks (one per SM) split the concatenated tile list of all (sequence,
// KV head) pairs evenly.  Pair br owns tiles [P[br], P[br+1]) with P the prefix sum of
// (count + 1) * B/64 (the +1 is the diagonal chunk).  A block walks its range segment by segment;
// for each pair it touches it writes one partial (o, m, l) per head at part[br][block].
constexpr int kMaxBR = 64;
constexpr int kMaxJobs = 2048;   // per-block tile table in shared memory

__global__ void __launch_bounds__(32 * (1 + kCons), 1)
dec_attend_tma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, Shape s,
                      const __nv_bfloat16* __restrict__ q, const int* __restrict__ seqlens, Routes rt,
                      float* __restrict__ part, int* err)
{
    extern __shared__ char smem_raw[];
    char* sm = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = tc::smem_addr(sm);
    const uint32_t bar_full = base + kNSd * kSlotB, bar_empty = bar_full + 8 * kNSd;
    volatile int* abort = reinterpret_cast<volatile int*>(sm + kNSd * kSlotB + 16 * kNSd);
    float* mrg = reinterpret_cast<float*>(sm + kNSd * kSlotB + 16 * kNSd + 16);   // [kCons][16][2]
    int* pre = reinterpret_cast<int*>(mrg + kCons * 16 * 2);                         // [kMaxBR + 1]
    float* osm = reinterpret_cast<float*>(pre + kMaxBR + 1);                         // [16][128]
    int* jkey = reinterpret_cast<int*>(osm + 16 * 128);                              // [kMaxJobs] first key
    float* jbias = reinterpret_cast<float*>(jkey + kMaxJobs);                        // [kMaxJobs] bias, NaN = diagonal

    const int BR = s.batch * s.hkv, G = s.g, NH = s.B / 64;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();   // the routes of this step
    pdl_launch_dependents();
    // tile counts of the (sequence, KV head) pairs: one load per thread, all in flight at once
    // (blockDim >= kMaxBR >= BR), then their prefix in shared memory
    static_assert(32 * (1 + kCons) >= kMaxBR, "one thread per pair");
    if (threadIdx.x < BR) pre[threadIdx.x + 1] = (rt.counts[threadIdx.x] + 1) * NH;
    __syncthreads();
    if (threadIdx.x == 0) {
        pre[0] = 0;
        for (int x = 1; x <= BR; ++x) pre[x] += pre[x - 1];
        for (int k = 0; k < kNSd; ++k) { tc::mbar_init(bar_full + 8 * k, 1); tc::mbar_init(bar_empty + 8 * k, 1); }
        *abort = 0;
        tc::mbar_fence_init();
    }
    __syncthreads();
    const long long total = pre[BR];
    const int j_lo = (int)(total * blockIdx.x / gridDim.x), j_hi = (int)(total * (blockIdx.x + 1) / gridDim.x);
    if (j_lo >= j_hi) return;
    auto seg_of = [&](int j) {
        int x = 0;
        while (pre[x + 1] <= j) ++x;
        return x;
    };
    // first key and bias of every tile of this block's range, looked up once (NaN bias marks the
    // pair's diagonal chunk); ranges beyond the table fall back to looking tiles up on the fly
    const int njobs = j_hi - j_lo;
    const bool table = njobs <= kMaxJobs;
    auto lookup = [&](int j, int x, int* key0, float* bias) {
        const int t = j - pre[x], e = t / NH;
        const int cnt = rt.counts[x];
        if (e < cnt) {
            *key0 = rt.idx[(long long)x * rt.cap + e] * s.B + (t % NH) * 64;
            *bias = rt.bias[(long long)x * rt.cap + e];
        } else {
            *key0 = ((seqlens[x / s.hkv] - 1) / s.B) * s.B + (t % NH) * 64;
            *bias = __int_as_float(0x7fc00000);
        }
    };
    if (table) {
        for (int k = threadIdx.x; k < njobs; k += blockDim.x) {
            const int j = j_lo + k;
            lookup(j, seg_of(j), &jkey[k], &jbias[k]);
        }
        __syncthreads();
    }
    auto job = [&](int k, int x, int* key0, float* bias) {
        if (table) { *key0 = jkey[k]; *bias = jbias[k]; }
        else lookup(j_lo + k, x, key0, bias);
    };

    if (warp == 0) {
        if (lane == 0) {
            tc::prefetch_tmap(&tmK);
            tc::prefetch_tmap(&tmV);
            const uint64_t pol = tc::l2_evict_first_policy();
            int last[kNSd];
            for (int k = 0; k < kNSd; ++k) last[k] = -1;
            int x = seg_of(j_lo);
            for (int k = 0; k < j_hi - j_lo; ++k) {
                const int j = j_lo + k;
                while (pre[x + 1] <= j) ++x;
                const int slot = k % kNSd;
                if (k >= kNSd && !tc::mbar_wait(bar_empty + 8 * slot, ((k / kNSd) - 1) & 1, abort, err, 11)) break;
                last[slot] = k;
                int key0;
                float bdummy;
                job(k, x, &key0, &bdummy);
                const int bb = x / s.hkv, r = x % s.hkv;
                // coordinates (row, sequence), or (row in page, page) for paged caches: a 64-key
                // tile never straddles two pages (the page size is a multiple of 64 and of B)
                int c2 = key0, c3 = bb;
                if (s.pt) {
                    c2 = key0 % s.psz;
                    c3 = s.pt[(long long)bb * s.pmax + key0 / s.psz];
                }
                const uint32_t dst = base + slot * kSlotB, fb = bar_full + 8 * slot;
                tc::mbar_expect_tx(fb, kSlotB);
                // the routed K/V tiles are a stream of several times L2 read once per step: evict
                // them first, so the chunk summaries that the next step's routing reads stay in L2
                tc::tma_load_4d_hint(dst, &tmK, fb, 0, r, c2, c3, pol);
                tc::tma_load_4d_hint(dst + kHalf, &tmK, fb, 64, r, c2, c3, pol);
                tc::tma_load_4d_hint(dst + 2 * kHalf, &tmV, fb, 0, r, c2, c3, pol);
                tc::tma_load_4d_hint(dst + 3 * kHalf, &tmV, fb, 64, r, c2, c3, pol);
            }
            if (*abort)   // let copies still in flight land before the block's shared memory goes away
                for (int k = 0; k < kNSd; ++k)
                    if (last[k] >= 0)
                        for (long long it = 0; it < (1ll << 22); ++it)
                            if (tc::mbar_try(bar_full + 8 * k, (last[k] / kNSd) & 1)) break;
        }
        return;
    }
    // ---- consumers ------------------------------------------------------------------------------
    const int cw = warp - 1;
    const int ra = lane >> 2, rb = ra + 8, t4 = lane & 3;
    const float scale2 = kLog2e * rsqrtf(128.f);
    const int mi = lane >> 3, rr8 = lane & 7;
    // a segment is the part of one pair's tiles inside this block's range
    for (int x = seg_of(j_lo); x < BR && pre[x] < j_hi; ++x) {
        const int s_lo = max(j_lo, pre[x]), s_hi = min(j_hi, pre[x + 1]);
        const int bb = x / s.hkv, r = x % s.hkv;
        const int L = seqlens[bb], i = L - 1;
        uint32_t qf[8][4];
        load_q_frags<128>(qf, [&](int rr) -> const __nv_bfloat16* {
            return rr < G ? q + ((long long)bb * s.hq + r * G + rr) * 128 : nullptr;
        });
        WarpAcc<128> acc;
        acc.init();
        // job index k counts tiles from j_lo: warp k % kCons, slot k % kNSd
        int k0 = s_lo - j_lo;
        k0 += ((cw - k0) % kCons + kCons) % kCons;
        for (int k = k0; k < s_hi - j_lo; k += kCons) {
            const int slot = k % kNSd;
            if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_full + 8 * slot, (k / kNSd) & 1, abort, err, 12))) break;
            char* tile = sm + slot * kSlotB;
            int j0;
            float jb;
            job(k, x, &j0, &jb);
            RowMode md;
            if (jb == jb) { md.bias2 = jb * kLog2e; md.jmax = INT_MAX; }
            else {
                md.bias2 = 0.f;
                md.jmax = i;
                // keys past the query may be unwritten cache slots: zero their V rows
                for (int row = max(0, i + 1 - j0); row < 64; ++row)
                    for (int cc = lane; cc < 16; cc += 32)
                        *reinterpret_cast<uint4*>(tile + 2 * kHalf + (cc >> 3) * kHalf + row * 128 + ((cc & 7) << 4)) =
                            make_uint4(0u, 0u, 0u, 0u);
                __syncwarp();
            }
            RowMode off;
            off.bias2 = -INFINITY;
            off.jmax = INT_MAX;
            const RowMode mA = ra < G ? md : off, mB = rb < G ? md : off;
            float sv[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) sv[j][0] = sv[j][1] = sv[j][2] = sv[j][3] = 0.f;
            const uint32_t kb = tc::smem_addr(tile), vb = kb + 2 * kHalf;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
                for (int nn = 0; nn < 8; nn += 2) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kb + sw_off(nn * 8 + rr8 + (mi >> 1) * 8, kk * 16 + (mi & 1) * 8), b0, b1, b2, b3);
                    mma_bf16(sv[nn], qf[kk], b0, b1);
                    mma_bf16(sv[nn + 1], qf[kk], b2, b3);
                }
            }
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const RowMode& m = q2 < 2 ? mA : mB;
                    float xv = sv[j][q2] * scale2 + m.bias2;
                    if (j0 + j * 8 + 2 * t4 + (q2 & 1) > m.jmax) xv = -INFINITY;
                    sv[j][q2] = xv;
                    mx[q2 >> 1] = fmaxf(mx[q2 >> 1], xv);
                }
            float corr[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
                const float mn = fmaxf(acc.m[h], mx[h]);
                const float bse = mn == -INFINITY ? 0.f : mn;
                corr[h] = exp2f(acc.m[h] - bse);
                acc.m[h] = mn;
                mx[h] = bse;
                acc.l[h] *= corr[h];
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                acc.o[j][0] *= corr[0]; acc.o[j][1] *= corr[0];
                acc.o[j][2] *= corr[1]; acc.o[j][3] *= corr[1];
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    const float pv = exp2f(sv[j][q2] - mx[q2 >> 1]);
                    sv[j][q2] = pv;
                    acc.l[q2 >> 1] += pv;
                }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t a[4];
                a[0] = pack_bf16(sv[2 * kk][0], sv[2 * kk][1]);
                a[1] = pack_bf16(sv[2 * kk][2], sv[2 * kk][3]);
                a[2] = pack_bf16(sv[2 * kk + 1][0], sv[2 * kk + 1][1]);
                a[3] = pack_bf16(sv[2 * kk + 1][2], sv[2 * kk + 1][3]);
#pragma unroll
                for (int nn = 0; nn < 16; nn += 2) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vb + sw_off(kk * 16 + rr8 + (mi & 1) * 8, nn * 8 + (mi >> 1) * 8), b0, b1, b2, b3);
                    mma_bf16(acc.o[nn], a, b0, b1);
                    mma_bf16(acc.o[nn + 1], a, b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar_empty + 8 * slot);
        }
        // ---- merge the consumer warps' states of this segment (fixed order: deterministic) ----
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            acc.l[h] += __shfl_xor_sync(0xffffffffu, acc.l[h], 1);
            acc.l[h] += __shfl_xor_sync(0xffffffffu, acc.l[h], 2);
        }
        if (t4 == 0) {
            mrg[(cw * 16 + ra) * 2] = acc.m[0];
            mrg[(cw * 16 + rb) * 2] = acc.m[1];
            mrg[(cw * 16 + ra) * 2 + 1] = acc.l[0];
            mrg[(cw * 16 + rb) * 2 + 1] = acc.l[1];
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kCons));
        // common maximum per row, then the warps add their rescaled sums one after another
        float sc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = h ? rb : ra;
            float M = -INFINITY;
            for (int w = 0; w < kCons; ++w) M = fmaxf(M, mrg[(w * 16 + row) * 2]);
            sc[h] = acc.m[h] == -INFINITY ? 0.f : exp2f(acc.m[h] - M);
        }
        for (int w = 0; w < kCons; ++w) {
            if (cw == w) {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int col = j * 8 + 2 * t4;
                    float* oa = osm + ra * 128 + col;
                    float* ob = osm + rb * 128 + col;
                    if (w == 0) {
                        oa[0] = acc.o[j][0] * sc[0]; oa[1] = acc.o[j][1] * sc[0];
                        ob[0] = acc.o[j][2] * sc[1]; ob[1] = acc.o[j][3] * sc[1];
                    } else {
                        oa[0] += acc.o[j][0] * sc[0]; oa[1] += acc.o[j][1] * sc[0];
                        ob[0] += acc.o[j][2] * sc[1]; ob[1] += acc.o[j][3] * sc[1];
                    }
                }
            }
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kCons));
        }
        float* pb = part + ((long long)x * gridDim.x + blockIdx.x) * G * 130;
        for (int v = threadIdx.x - 32; v < G * 128; v += 32 * kCons) {
            const int row = v >> 7, col = v & 127;
            pb[row * 130 + col] = osm[row * 128 + col];
        }
        if (threadIdx.x - 32 < G) {
            const int row = threadIdx.x - 32;
            float M = -INFINITY, Lr = 0.f;
            for (int w = 0; w < kCons; ++w) M = fmaxf(M, mrg[(w * 16 + row) * 2]);
            for (int w = 0; w < kCons; ++w) {
                const float mw = mrg[(w * 16 + row) * 2];
                if (mw != -INFINITY) Lr += mrg[(w * 16 + row) * 2 + 1] * exp2f(mw - M);
            }
            pb[row * 130 + 128] = M;
            pb[row * 130 + 129] = Lr;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kCons));   // osm / mrg are reused by the next segment
    }
}

// Merge of the per-block partials of each pair: one block per (pair, head), one thread per
// column.  Every thread finds the pair's blocks and the common maximum / sum itself (the few
// partial (m, l) values are broadcast loads), so the merge is one chain of loads, no barrier.
template <int D>
__global__ void __launch_bounds__(D) dec_merge_kernel(Shape s, const float* __restrict__ part, int nblocks,
                                                      Routes rt, __nv_bfloat16* __restrict__ O)
{
    pdl_wait();   // the partials of this step
    const int x = blockIdx.x / s.g, row = blockIdx.x % s.g, G = s.g, NH = s.B / 64;
    const int b = x / s.hkv, r = x % s.hkv, col = threadIdx.x;
    // tiles before this pair and in all: the pairs' counts loaded by the block's threads at once,
    // summed by warp shuffles, then over the warps in order
    __shared__ long long wsum_lo[D / 32], wsum_tot[D / 32];
    long long lo_p = 0, tot_p = 0;
    for (int y = threadIdx.x; y < s.batch * s.hkv; y += D) {
        const long long c = (long long)(rt.counts[y] + 1) * NH;
        if (y < x) lo_p += c;
        tot_p += c;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo_p += __shfl_xor_sync(0xffffffffu, lo_p, o);
        tot_p += __shfl_xor_sync(0xffffffffu, tot_p, o);
    }
    if ((threadIdx.x & 31) == 0) { wsum_lo[threadIdx.x >> 5] = lo_p; wsum_tot[threadIdx.x >> 5] = tot_p; }
    __syncthreads();
    long long lo = 0, total = 0;
#pragma unroll
    for (int w = 0; w < D / 32; ++w) { lo += wsum_lo[w]; total += wsum_tot[w]; }
    const long long hi = lo + (long long)(rt.counts[x] + 1) * NH;
    // block c covers tiles [total c / n, total (c+1) / n); it wrote a partial for this pair iff
    // that range is nonempty and meets [lo, hi)
    auto jlo = [&](int c) { return total * c / nblocks; };
    int c0 = (int)(lo * nblocks / total), c1 = (int)((hi - 1) * nblocks / total);
    while (c0 > 0 && jlo(c0) > lo) --c0;
    while (c0 + 1 < nblocks && jlo(c0 + 1) <= lo) ++c0;
    while (c1 + 1 < nblocks && jlo(c1 + 1) <= hi - 1) ++c1;
    while (c1 > 0 && jlo(c1) > hi - 1) --c1;
    const bool all_nonempty = total >= nblocks;
    const float* basep = part + (long long)x * nblocks * G * 130 + (long long)row * 130;
    const long long sstride = (long long)G * 130;
    // one pass with a running maximum; four partials' loads in flight at a time
    float M = -INFINITY, Lsum = 0.f, o = 0.f;
    for (int c = c0; c <= c1; c += 4) {
        float mk[4], lk[4], ok[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int cc = c + q;
            const bool use = cc <= c1 && (all_nonempty || jlo(cc) < jlo(cc + 1));
            mk[q] = use ? basep[cc * sstride + 128] : -INFINITY;
            lk[q] = use ? basep[cc * sstride + 129] : 0.f;
            ok[q] = use ? basep[cc * sstride + col] : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (mk[q] == -INFINITY) continue;
            if (mk[q] > M) {
                const float sc = exp2f(M - mk[q]);
                Lsum *= sc;
                o *= sc;
                M = mk[q];
            }
            const float w = exp2f(mk[q] - M);
            Lsum += lk[q] * w;
            o += ok[q] * w;
        }
    }
    O[((long long)b * s.hq + r * G + row) * D + col] = __float2bfloat16_rn(Lsum > 0.f ? o / Lsum : 0.f);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_d()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 4-D map (d, head, row, sequence) over a contiguous cache, or (d, head, row in page, page) over
// a paged pool (ps = elements between pages)
bool map_kv(CUtensorMap* map, const void* ptr, const Shape& s, const long long st[3], long long ps)
{
    auto fn = encode_fn_d();
    if (!fn) return false;
    cuuint64_t dims[4] = {128, (cuuint64_t)s.hkv, (cuuint64_t)s.n, (cuuint64_t)s.batch};
    cuuint64_t strides[3] = {(cuuint64_t)st[2] * 2, (cuuint64_t)st[1] * 2, (cuuint64_t)st[0] * 2};
    if (s.batch == 1) strides[2] = strides[1] * (cuuint64_t)s.n;
    if (s.pt) {
        dims[2] = (cuuint64_t)s.psz;
        dims[3] = (cuuint64_t)s.npages;
        strides[2] = (cuuint64_t)ps * 2;
    }
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool dec_tma_supported(const Shape& s, int dtype)
{
    return dtype == DASH_BF16 && s.d == 128 && (s.B == 64 || s.B == 128) && s.g <= 16 &&
           s.batch * s.hkv <= kMaxBR && encode_fn_d() != nullptr;
}

int dec_tma_blocks()
{
    static int n = 0;
    if (!n) {
        int dev = 0, sms = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        n = sms > 0 ? (sms > 1024 ? 1024 : sms) : 148;
    }
    return n;
}

cudaError_t launch_dec_attend_tma(const Shape& s, const void* q, const void* Kc, const void* Vc, const int* seqlens,
                                  const Routes& rt, float* part, void* O, int* err, cudaStream_t st)
{
    CUtensorMap mk, mv;
    if (!map_kv(&mk, Kc, s, s.ks, s.kps) || !map_kv(&mv, Vc, s, s.vs, s.vps)) return cudaErrorInvalidValue;
    const size_t smem = 1024 + kNSd * kSlotB + 16 * kNSd + 16 + kCons * 16 * 2 * 4 + (kMaxBR + 1) * 4 +
                        16 * 128 * 4 + 2 * kMaxJobs * 4;
    cudaError_t e = cudaFuncSetAttribute(dec_attend_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int nb = dec_tma_blocks();
    e = launch_after(dec_attend_tma_kernel, dim3(nb), dim3(32 * (1 + kCons)), smem, st, mk, mv, s,
                     (const __nv_bfloat16*)q, seqlens, rt, part, err);
    if (e != cudaSuccess) return e;
    return launch_after(dec_merge_kernel<128>, dim3(s.batch * s.hkv * s.g), dim3(128), 0, st, s, (const float*)part,
                        nb, rt, (__nv_bfloat16*)O);
}

}  // namespace dash
