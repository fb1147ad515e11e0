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

constexpr int kCPS = 16;          // route entries (chunks) per split
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

__global__ void __launch_bounds__(32 * (1 + kCons), 1)
dec_attend_tma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, Shape s,
                      const __nv_bfloat16* __restrict__ q, const int* __restrict__ seqlens, Routes rt,
                      float* __restrict__ part, int splits, int* err)
{
    extern __shared__ char smem_raw[];
    char* sm = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t base = tc::smem_addr(sm);
    const uint32_t bar_full = base + kNSd * kSlotB, bar_empty = bar_full + 8 * kNSd;
    volatile int* abort = reinterpret_cast<volatile int*>(sm + kNSd * kSlotB + 16 * kNSd);
    float* mrg = reinterpret_cast<float*>(sm + kNSd * kSlotB + 16 * kNSd + 16);   // [kCons][16][2]

    const int br = blockIdx.y, sp = blockIdx.x, b = br / s.hkv, r = br % s.hkv;
    const int L = seqlens[b], i = L - 1, G = s.g;
    const int cnt = rt.counts[br];
    const int e0 = sp * kCPS, e1 = min(e0 + kCPS, cnt + 1);
    if (e0 >= e1 || L <= 0) return;
    const int NH = s.B / 64;
    const int njobs = (e1 - e0) * NH;
    const int* li = rt.idx + (long long)br * rt.cap;
    const float* lb = rt.bias + (long long)br * rt.cap;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int k = 0; k < kNSd; ++k) { tc::mbar_init(bar_full + 8 * k, 1); tc::mbar_init(bar_empty + 8 * k, 1); }
        *abort = 0;
        tc::mbar_fence_init();
    }
    __syncthreads();
    auto chunk_of = [&](int e) { return e < cnt ? li[e] : i / s.B; };

    if (warp == 0) {
        if (lane == 0) {
            tc::prefetch_tmap(&tmK);
            tc::prefetch_tmap(&tmV);
            int last[kNSd];
            for (int k = 0; k < kNSd; ++k) last[k] = -1;
            for (int k = 0; k < njobs; ++k) {
                const int slot = k % kNSd;
                if (k >= kNSd && !tc::mbar_wait(bar_empty + 8 * slot, ((k / kNSd) - 1) & 1, abort, err, 11)) break;
                last[slot] = k;
                const int key0 = chunk_of(e0 + k / NH) * s.B + (k % NH) * 64;
                const uint32_t dst = base + slot * kSlotB, fb = bar_full + 8 * slot;
                tc::mbar_expect_tx(fb, kSlotB);
                tc::tma_load_4d(dst, &tmK, fb, 0, r, key0, b);
                tc::tma_load_4d(dst + kHalf, &tmK, fb, 64, r, key0, b);
                tc::tma_load_4d(dst + 2 * kHalf, &tmV, fb, 0, r, key0, b);
                tc::tma_load_4d(dst + 3 * kHalf, &tmV, fb, 64, r, key0, b);
            }
            if (*abort)   // let copies still in flight land before the block's shared memory goes away
                for (int k = 0; k < kNSd; ++k)
                    if (last[k] >= 0)
                        for (long long it = 0; it < (1ll << 22); ++it)
                            if (tc::mbar_try(bar_full + 8 * k, (last[k] / kNSd) & 1)) break;
        }
    } else {
        const int cw = warp - 1;
        const int ra = lane >> 2, rb = ra + 8, t4 = lane & 3;
        uint32_t qf[8][4];
        load_q_frags<128>(qf, [&](int rr) -> const __nv_bfloat16* {
            return rr < G ? q + ((long long)b * s.hq + r * G + rr) * 128 : nullptr;
        });
        WarpAcc<128> acc;
        acc.init();
        const float scale2 = kLog2e * rsqrtf(128.f);
        const int mi = lane >> 3, rr8 = lane & 7;
        for (int k = cw; k < njobs; k += kCons) {
            const int slot = k % kNSd;
            if (!__all_sync(0xffffffffu, tc::mbar_wait(bar_full + 8 * slot, (k / kNSd) & 1, abort, err, 12))) break;
            char* tile = sm + slot * kSlotB;
            const int e = e0 + k / NH, c = chunk_of(e);
            const int j0 = c * s.B + (k % NH) * 64;
            RowMode md;
            if (e < cnt) { md.bias2 = lb[e] * kLog2e; md.jmax = INT_MAX; }
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
            // S = Q K^T over 64 keys
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
                    float x = sv[j][q2] * scale2 + m.bias2;
                    if (j0 + j * 8 + 2 * t4 + (q2 & 1) > m.jmax) x = -INFINITY;
                    sv[j][q2] = x;
                    mx[q2 >> 1] = fmaxf(mx[q2 >> 1], x);
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
                    const float p = exp2f(sv[j][q2] - mx[q2 >> 1]);
                    sv[j][q2] = p;
                    acc.l[q2 >> 1] += p;
                }
            // O += P V
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
        // merge the consumer warps: max and sum per row, then the rescaled outputs
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            acc.l[h] += __shfl_xor_sync(0xffffffffu, acc.l[h], 1);
            acc.l[h] += __shfl_xor_sync(0xffffffffu, acc.l[h], 2);
        }
        if (t4 == 0) {
            mrg[(cw * 16 + ra) * 2] = acc.m[0];
            mrg[(cw * 16 + rb) * 2] = acc.m[1];
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kCons));
        float M[2], sc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = h ? rb : ra;
            M[h] = -INFINITY;
            for (int w = 0; w < kCons; ++w) M[h] = fmaxf(M[h], mrg[(w * 16 + row) * 2]);
            sc[h] = M[h] == -INFINITY ? 0.f : exp2f(acc.m[h] - M[h]);
        }
        float* osm = reinterpret_cast<float*>(sm);   // ring is idle now: [16][128] output sums
        // one snapshot of the abort flag for all consumer threads: the branch below holds barriers
        volatile int* snap = reinterpret_cast<volatile int*>(sm + kNSd * kSlotB + 16 * kNSd + 8);
        if (threadIdx.x == 32) *snap = *abort;
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kCons));
        if (!*snap) {
            for (int v = threadIdx.x - 32; v < 16 * 128; v += 32 * kCons) osm[v] = 0.f;
            if (t4 == 0) {
                mrg[(cw * 16 + ra) * 2 + 1] = acc.l[0] * sc[0];
                mrg[(cw * 16 + rb) * 2 + 1] = acc.l[1] * sc[1];
            }
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kCons));
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int col = j * 8 + 2 * t4;
                atomicAdd(&osm[ra * 128 + col], acc.o[j][0] * sc[0]);
                atomicAdd(&osm[ra * 128 + col + 1], acc.o[j][1] * sc[0]);
                atomicAdd(&osm[rb * 128 + col], acc.o[j][2] * sc[1]);
                atomicAdd(&osm[rb * 128 + col + 1], acc.o[j][3] * sc[1]);
            }
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kCons));
            float* pb = part + ((long long)br * splits + sp) * G * 130;
            for (int v = threadIdx.x - 32; v < G * 128; v += 32 * kCons) {
                const int row = v >> 7, col = v & 127;
                pb[row * 130 + col] = osm[row * 128 + col];
            }
            if (threadIdx.x - 32 < G) {
                const int row = threadIdx.x - 32;
                float Mr = -INFINITY, Lr = 0.f;
                for (int w = 0; w < kCons; ++w) Mr = fmaxf(Mr, mrg[(w * 16 + row) * 2]);
                for (int w = 0; w < kCons; ++w) Lr += mrg[(w * 16 + row) * 2 + 1];
                pb[row * 130 + 128] = Mr;
                pb[row * 130 + 129] = Lr;
            }
        }
    }
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

bool map_kv(CUtensorMap* map, const void* ptr, const Shape& s, const long long st[3])
{
    auto fn = encode_fn_d();
    if (!fn) return false;
    cuuint64_t dims[4] = {128, (cuuint64_t)s.hkv, (cuuint64_t)s.n, (cuuint64_t)s.batch};
    cuuint64_t strides[3] = {(cuuint64_t)st[2] * 2, (cuuint64_t)st[1] * 2, (cuuint64_t)st[0] * 2};
    if (s.batch == 1) strides[2] = strides[1] * (cuuint64_t)s.n;
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool dec_tma_supported(const Shape& s, int dtype)
{
    return dtype == DASH_BF16 && s.d == 128 && (s.B == 64 || s.B == 128) && s.g <= 16 && encode_fn_d() != nullptr;
}

int dec_tma_splits(const Shape& s, int kbar_T)
{
    (void)s;
    return (kbar_T + 1 + kCPS - 1) / kCPS;
}

int dec_tma_cps() { return kCPS; }

cudaError_t launch_dec_attend_tma(const Shape& s, const void* q, const void* Kc, const void* Vc, const int* seqlens,
                                  const Routes& rt, float* part, int splits, int* err, cudaStream_t st)
{
    CUtensorMap mk, mv;
    if (!map_kv(&mk, Kc, s, s.ks) || !map_kv(&mv, Vc, s, s.vs)) return cudaErrorInvalidValue;
    const size_t smem = 1024 + kNSd * kSlotB + 16 * kNSd + 16 + kCons * 16 * 2 * 4;
    cudaError_t e = cudaFuncSetAttribute(dec_attend_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(splits, s.batch * s.hkv);
    dec_attend_tma_kernel<<<grid, 32 * (1 + kCons), smem, st>>>(mk, mv, s, (const __nv_bfloat16*)q, seqlens, rt, part,
                                                              splits, err);
    return cudaGetLastError();
}

}  // namespace dash
