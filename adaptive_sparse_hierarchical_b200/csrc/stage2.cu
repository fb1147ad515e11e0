// stage2.cu -- Stage 2 prior-induced sparse softmax (Proposition 4.1 bias form) for prefill
// and decode, plus the fp32 CUDA-core variant.
//
// DashAttention (xllm-io paper review, section 3, Eq. 9 / Prop. 4.1 and the "Stage 2" kernel
// row: a masked FlashAttention pass over the routed chunks with a per-chunk bias; decoding uses
// a split-KV variant).  For query row (i, h) of KV group r:
//   o = sum_{j in R u D} exp(z_j + d_j) v_j / sum exp(z_j + d_j),  z_j = <q,k_j>/sqrt(d),
//   d_j = bias of chunk c(j) for routed tokens, 0 for the diagonal tokens c(i)B..i.
#include <climits>
#include <cstdlib>

#include "stage2_mma.cuh"

namespace dash {
namespace {

// First set bit >= c in a shared bitmask of `words` words, or -1.
__device__ __forceinline__ int next_set(const uint32_t* mask, int words, int c)
{
    int w = c >> 5;
    if (w >= words) return -1;
    uint32_t bits = mask[w] & (0xffffffffu << (c & 31));
    while (bits == 0u) {
        if (++w >= words) return -1;
        bits = mask[w];
    }
    return (w << 5) + __ffs(bits) - 1;
}

// Routing cursor of one query row: walks the row's ascending chunk list.
struct Cursor {
    const int* idx;
    const float* bias;
    int cnt, cur, next;
    float nbias;
    __device__ void init(const int* i_, const float* b_, int n_)
    {
        idx = i_; bias = b_; cnt = n_; cur = 0;
        next = cnt > 0 ? idx[0] : INT_MAX;
        nbias = cnt > 0 ? bias[0] : 0.f;
    }
    __device__ void advance_past(int c)
    {
        if (next == c) {
            ++cur;
            next = cur < cnt ? idx[cur] : INT_MAX;
            nbias = cur < cnt ? bias[cur] : 0.f;
        }
    }
};

__device__ __forceinline__ RowMode row_mode(bool valid, const Cursor& cu, int c, int diag, int i)
{
    RowMode m;
    m.jmax = INT_MAX;
    if (!valid) m.bias2 = -INFINITY;
    else if (cu.next == c) m.bias2 = cu.nbias * kLog2e;
    else if (c == diag) { m.bias2 = 0.f; m.jmax = i; }
    else m.bias2 = -INFINITY;
    return m;
}

// ------------------------------------------------------------------------------------------
// Prefill, bf16 tensor cores.  Block = 4 warps = 64 rows = (64/g positions) x (g heads) of one
// (sequence, KV head).  The block visits the union of its positions' routed chunks and their
// diagonal chunks in ascending order, double-buffering K/V tiles of KT keys in shared memory;
// a warp skips a tile when none of its rows uses it.
// ------------------------------------------------------------------------------------------
template <int KT, int D>
__global__ void __launch_bounds__(128) attend_prefill_mma_kernel(Shape s, const __nv_bfloat16* __restrict__ Q,
                                                                 const __nv_bfloat16* __restrict__ K,
                                                                 const __nv_bfloat16* __restrict__ V,
                                                                 __nv_bfloat16* __restrict__ O, Routes rt)
{
    constexpr int TILE = KT * D * 2;
    extern __shared__ __align__(128) char smem[];
    char* sK0 = smem;
    uint32_t* umask = reinterpret_cast<uint32_t*>(smem + 4 * TILE);
    const int W = (s.T + 32) >> 5;   // chunk ids 0..T (T is a partial last chunk)
    const int G = s.g, P = 64 / G;
    const int nblk = (s.n + P - 1) / P;
    const int br = blockIdx.x % (s.batch * s.hkv);
    const int pb = nblk - 1 - blockIdx.x / (s.batch * s.hkv);
    const int b = br / s.hkv, r = br % s.hkv;
    const int i0 = pb * P;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int* counts = rt.counts + (long long)br * s.n;
    const int* ridx = rt.idx + (long long)br * rt.cap;
    const float* rbias = rt.bias + (long long)br * rt.cap;

    for (int w = tid; w < W; w += 128) umask[w] = 0u;
    __syncthreads();
    for (int p = 0; p < P; ++p) {
        const int i = i0 + p;
        if (i >= s.n) break;
        const int cnt = counts[i];
        const int* li = ridx + tri_offset(i, s.B);
        for (int k = tid; k < cnt; k += 128) atomicOr(&umask[li[k] >> 5], 1u << (li[k] & 31));
        if (tid == 0) atomicOr(&umask[(i / s.B) >> 5], 1u << ((i / s.B) & 31));
    }
    __syncthreads();

    // the lane's two rows
    const int RA = warp * 16 + (lane >> 2), RB = RA + 8;
    const int iA = i0 + RA / G, iB = i0 + RB / G;
    const bool vA = iA < s.n, vB = iB < s.n;
    Cursor cA, cB;
    cA.init(ridx + (vA ? tri_offset(iA, s.B) : 0), rbias + (vA ? tri_offset(iA, s.B) : 0), vA ? counts[iA] : 0);
    cB.init(ridx + (vB ? tri_offset(iB, s.B) : 0), rbias + (vB ? tri_offset(iB, s.B) : 0), vB ? counts[iB] : 0);
    const int dA = iA / s.B, dB = iB / s.B;

    uint32_t qf[D / 16][4];
    load_q_frags<D>(qf, [&](int rr) -> const __nv_bfloat16* {
        const int R = warp * 16 + rr, i = i0 + R / G;
        if (i >= s.n) return nullptr;
        return Q + (long long)b * s.qs[0] + (long long)i * s.qs[1] + (long long)(r * G + R % G) * s.qs[2];
    });
    WarpAcc<D> acc;
    acc.init();
    const float scale2 = kLog2e * rsqrtf((float)D);
    const int NH = s.B / KT;
    const __nv_bfloat16* Kb = K + (long long)b * s.ks[0] + (long long)r * s.ks[2];
    const __nv_bfloat16* Vb = V + (long long)b * s.vs[0] + (long long)r * s.vs[2];

    int c = next_set(umask, W, 0), hh = 0, buf = 0;
    if (c >= 0) {
        const long long j0 = (long long)c * s.B;
        const int nv = (int)min((long long)KT, s.n - j0);
        load_tile<KT, D, 128>(sK0, Kb + j0 * s.ks[1], s.ks[1], nv, Kb, tid);
        load_tile<KT, D, 128>(sK0 + 2 * TILE, Vb + j0 * s.vs[1], s.vs[1], nv, Vb, tid);
    }
    cp_async_commit();
    while (c >= 0) {
        // next job
        int nc = c, nh = hh + 1;
        if (nh == NH) { nh = 0; nc = next_set(umask, W, c + 1); }
        if (nc >= 0) {
            const long long j0 = (long long)nc * s.B + nh * KT;
            const int nv = (int)min((long long)KT, s.n - j0);
            load_tile<KT, D, 128>(sK0 + (buf ^ 1) * TILE, Kb + j0 * s.ks[1], s.ks[1], nv, Kb, tid);
            load_tile<KT, D, 128>(sK0 + (2 + (buf ^ 1)) * TILE, Vb + j0 * s.vs[1], s.vs[1], nv, Vb, tid);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const RowMode ma = row_mode(vA, cA, c, dA, iA), mb = row_mode(vB, cB, c, dB, iB);
        const bool use = (ma.bias2 != -INFINITY) || (mb.bias2 != -INFINITY);
        if (__any_sync(0xffffffffu, use))
            tile_step<KT, D>(acc, qf, sK0 + buf * TILE, sK0 + (2 + buf) * TILE, c * s.B + hh * KT, ma, mb, scale2);
        if (hh == NH - 1) { cA.advance_past(c); cB.advance_past(c); }
        __syncthreads();
        c = nc; hh = nh; buf ^= 1;
    }
    cp_async_wait<0>();

    // normalise and store
    const int t = lane & 3;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        acc.l[h] += __shfl_xor_sync(0xffffffffu, acc.l[h], 1);
        acc.l[h] += __shfl_xor_sync(0xffffffffu, acc.l[h], 2);
    }
    const float invA = acc.l[0] > 0.f ? 1.f / acc.l[0] : 0.f;
    const float invB = acc.l[1] > 0.f ? 1.f / acc.l[1] : 0.f;
    __nv_bfloat16* oA = vA ? O + (long long)b * s.os[0] + (long long)iA * s.os[1] + (long long)(r * G + RA % G) * s.os[2] : nullptr;
    __nv_bfloat16* oB = vB ? O + (long long)b * s.os[0] + (long long)iB * s.os[1] + (long long)(r * G + RB % G) * s.os[2] : nullptr;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const int col = j * 8 + 2 * t;
        if (oA) *reinterpret_cast<uint32_t*>(oA + col) = pack_bf16(acc.o[j][0] * invA, acc.o[j][1] * invA);
        if (oB) *reinterpret_cast<uint32_t*>(oB + col) = pack_bf16(acc.o[j][2] * invB, acc.o[j][3] * invB);
    }
}

// ------------------------------------------------------------------------------------------
// Decode, bf16 tensor cores, split along the route list (the pages' split-KV decoding
// variant).  Block = one warp = the g (<= 16) heads of one (sequence, KV head); split sp takes
// route entries [sp*CPS, sp*CPS + CPS) where entry `count` stands for the diagonal chunk.
// Each split writes an unnormalised partial (o, running max m, running sum l) per head.
// ------------------------------------------------------------------------------------------
constexpr int kDecCPS = 8;

template <int KT, int D>
__global__ void __launch_bounds__(32) dec_attend_mma_kernel(Shape s, const __nv_bfloat16* __restrict__ q,
                                                            const __nv_bfloat16* __restrict__ Kc,
                                                            const __nv_bfloat16* __restrict__ Vc,
                                                            const int* __restrict__ seqlens, Routes rt,
                                                            float* __restrict__ part, int splits)
{
    constexpr int TILE = KT * D * 2;
    extern __shared__ __align__(128) char smem[];
    const int br = blockIdx.y, sp = blockIdx.x, b = br / s.hkv, r = br % s.hkv;
    const int L = seqlens[b], i = L - 1, G = s.g;
    const int cnt = rt.counts[br];
    const int e0 = sp * kDecCPS, e1 = min(e0 + kDecCPS, cnt + 1);
    if (e0 >= e1) return;
    const int lane = threadIdx.x;
    const int* li = rt.idx + (long long)br * rt.cap;
    const float* lb = rt.bias + (long long)br * rt.cap;
    const int ra = lane >> 2, rb = ra + 8;
    uint32_t qf[D / 16][4];
    load_q_frags<D>(qf, [&](int rr) -> const __nv_bfloat16* {
        return rr < G ? q + ((long long)b * s.hq + r * G + rr) * D : nullptr;
    });
    WarpAcc<D> acc;
    acc.init();
    const float scale2 = kLog2e * rsqrtf((float)D);
    const int NH = s.B / KT;
    const __nv_bfloat16* Kb = Kc + (long long)b * s.ks[0] + (long long)r * s.ks[2];
    const __nv_bfloat16* Vb = Vc + (long long)b * s.vs[0] + (long long)r * s.vs[2];
    auto chunk_of = [&](int e) { return e < cnt ? li[e] : i / s.B; };
    const int jobs = (e1 - e0) * NH;
    {
        const long long j0 = (long long)chunk_of(e0) * s.B;
        const int nv = (int)min((long long)KT, (long long)L - j0);
        load_tile<KT, D, 32>(smem, Kb + j0 * s.ks[1], s.ks[1], nv, Kb, lane);
        load_tile<KT, D, 32>(smem + 2 * TILE, Vb + j0 * s.vs[1], s.vs[1], nv, Vb, lane);
    }
    cp_async_commit();
    for (int jb = 0; jb < jobs; ++jb) {
        const int buf = jb & 1;
        if (jb + 1 < jobs) {
            const int e = e0 + (jb + 1) / NH, h = (jb + 1) % NH;
            const long long j0 = (long long)chunk_of(e) * s.B + h * KT;
            const int nv = (int)min((long long)KT, (long long)L - j0);
            load_tile<KT, D, 32>(smem + (buf ^ 1) * TILE, Kb + j0 * s.ks[1], s.ks[1], nv, Kb, lane);
            load_tile<KT, D, 32>(smem + (2 + (buf ^ 1)) * TILE, Vb + j0 * s.vs[1], s.vs[1], nv, Vb, lane);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncwarp();
        const int e = e0 + jb / NH, h = jb % NH;
        RowMode md;
        if (e < cnt) { md.bias2 = lb[e] * kLog2e; md.jmax = INT_MAX; }
        else { md.bias2 = 0.f; md.jmax = i; }
        RowMode off;
        off.bias2 = -INFINITY;
        off.jmax = INT_MAX;
        tile_step<KT, D>(acc, qf, smem + buf * TILE, smem + (2 + buf) * TILE, chunk_of(e) * s.B + h * KT,
                         ra < G ? md : off, rb < G ? md : off, scale2);
        __syncwarp();
    }
    cp_async_wait<0>();
    const int t = lane & 3;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        acc.l[h] += __shfl_xor_sync(0xffffffffu, acc.l[h], 1);
        acc.l[h] += __shfl_xor_sync(0xffffffffu, acc.l[h], 2);
    }
    float* pa = part + (((long long)br * splits + sp) * G + ra) * (D + 2);
    float* pb = part + (((long long)br * splits + sp) * G + rb) * (D + 2);
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const int col = j * 8 + 2 * t;
        if (ra < G) { pa[col] = acc.o[j][0]; pa[col + 1] = acc.o[j][1]; }
        if (rb < G) { pb[col] = acc.o[j][2]; pb[col + 1] = acc.o[j][3]; }
    }
    if (t == 0) {
        if (ra < G) { pa[D] = acc.m[0]; pa[D + 1] = acc.l[0]; }
        if (rb < G) { pb[D] = acc.m[1]; pb[D + 1] = acc.l[1]; }
    }
}

// Log-sum-exp merge of the split partials; one block per (sequence, query head): the split
// weights 2^(m_k - M) / L are computed once into shared memory, then each thread merges one
// output column.
template <typename T, int D>
__global__ void __launch_bounds__(128) dec_combine_kernel(Shape s, const float* __restrict__ part, int splits,
                                                          int cps, Routes rt, T* __restrict__ O)
{
    __shared__ float wk[1024];
    __shared__ float red[4];
    const int br = blockIdx.x / s.g, row = blockIdx.x % s.g, G = s.g;
    const int b = br / s.hkv, r = br % s.hkv;
    const int nsp = min((rt.counts[br] + 1 + cps - 1) / cps, 1024);
    const float* base = part + (long long)br * splits * G * (D + 2) + (long long)row * (D + 2);
    const long long sstride = (long long)G * (D + 2);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float M = -INFINITY;
    for (int k = tid; k < nsp; k += blockDim.x) M = fmaxf(M, base[k * sstride + D]);
    M = warp_max(M);
    if (lane == 0) red[warp] = M;
    __syncthreads();
    M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    __syncthreads();
    float Lsum = 0.f;
    for (int k = tid; k < nsp; k += blockDim.x) {
        const float w = exp2f(base[k * sstride + D] - M);
        wk[k] = w;
        Lsum += base[k * sstride + D + 1] * w;
    }
    Lsum = warp_sum(Lsum);
    if (lane == 0) red[warp] = Lsum;
    __syncthreads();
    Lsum = red[0] + red[1] + red[2] + red[3];
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    for (int col = tid; col < D; col += blockDim.x) {
        float o = 0.f;
        for (int k = 0; k < nsp; ++k) o += base[k * sstride + col] * wk[k];
        O[((long long)b * s.hq + r * G + row) * D + col] = from_f<T>(o * inv);
    }
}

// ------------------------------------------------------------------------------------------
// fp32 inputs: CUDA-core kernel, one warp per query row (prefill rows, or decode rows when
// seqlens != null).  32 keys per step, one key per lane for the logits, one output column
// slice per lane for P V.
// ------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(128) attend_rows_kernel(Shape s, const T* __restrict__ Q,
                                                          const T* __restrict__ K, const T* __restrict__ V,
                                                          T* __restrict__ O, Routes rt,
                                                          const int* __restrict__ seqlens)
{
    __shared__ float qsh[4][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 4 + warp;
    int b, i, h;
    const T* qp;
    T* op;
    const int* li;
    const float* lb;
    int cnt;
    if (seqlens) {
        if (row >= (long long)s.batch * s.hq) return;
        b = (int)(row / s.hq); h = (int)(row % s.hq); i = seqlens[b] - 1;
        qp = Q + row * D;
        op = O + row * D;
        const int br = b * s.hkv + h / s.g;
        li = rt.idx + (long long)br * rt.cap; lb = rt.bias + (long long)br * rt.cap; cnt = rt.counts[br];
    } else {
        if (row >= (long long)s.batch * s.n * s.hq) return;
        b = (int)(row / ((long long)s.n * s.hq)); i = (int)((row / s.hq) % s.n); h = (int)(row % s.hq);
        qp = Q + (long long)b * s.qs[0] + (long long)i * s.qs[1] + (long long)h * s.qs[2];
        op = O + (long long)b * s.os[0] + (long long)i * s.os[1] + (long long)h * s.os[2];
        const int br = b * s.hkv + h / s.g;
        const long long off = (long long)br * rt.cap + tri_offset(i, s.B);
        li = rt.idx + off; lb = rt.bias + off; cnt = rt.counts[(long long)br * s.n + i];
    }
    const int r = h / s.g;
    const float sc = kLog2e * rsqrtf((float)D);
    for (int e = lane; e < D; e += 32) qsh[warp][e] = to_f(qp[e]) * sc;
    __syncwarp();
    const T* Kb = K + (long long)b * s.ks[0] + (long long)r * s.ks[2];
    const T* Vb = V + (long long)b * s.vs[0] + (long long)r * s.vs[2];
    float m = -INFINITY, l = 0.f, acc[D / 32];
#pragma unroll
    for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
    auto range = [&](int j0, int j1, float bias2) {
        for (int jb = j0; jb < j1; jb += 32) {
            const int j = jb + lane;
            float sv = -INFINITY;
            if (j < j1) {
                const T* kr = Kb + (long long)j * s.ks[1];
                float dot = 0.f;
                for (int e = 0; e < D; e += Vec<T>::N) {
                    float kv[Vec<T>::N];
                    Vec<T>::load(kr + e, kv);
                    for (int u = 0; u < Vec<T>::N; ++u) dot += qsh[warp][e + u] * kv[u];
                }
                sv = dot + bias2;
            }
            const float mn = fmaxf(m, warp_max(sv));
            const float corr = exp2f(m - mn);
            const float p = exp2f(sv - mn);
            l = l * corr + warp_sum(p);
#pragma unroll
            for (int e = 0; e < D / 32; ++e) acc[e] *= corr;
            const int jn = min(32, j1 - jb);
            for (int jj = 0; jj < jn; ++jj) {
                const float pj = __shfl_sync(0xffffffffu, p, jj);
                const T* vr = Vb + (long long)(jb + jj) * s.vs[1];
#pragma unroll
                for (int e = 0; e < D / 32; ++e) acc[e] += pj * to_f(vr[lane + 32 * e]);
            }
            m = mn;
        }
    };
    // chunks shorter than a warp (B = 1: each chunk is one token, B = 16): 32 / B listed chunks
    // per step, lane -> (entry k0 + lane / B, key lane % B), each lane with its chunk's bias
    auto gather = [&](int k0) {
        const int e = k0 + lane / s.B;
        const bool ok = e < cnt;
        const int j = ok ? li[e] * s.B + lane % s.B : 0;
        float sv = -INFINITY;
        if (ok) {
            const T* kr = Kb + (long long)j * s.ks[1];
            float dot = 0.f;
            for (int x = 0; x < D; x += Vec<T>::N) {
                float kv[Vec<T>::N];
                Vec<T>::load(kr + x, kv);
                for (int u = 0; u < Vec<T>::N; ++u) dot += qsh[warp][x + u] * kv[u];
            }
            sv = dot + lb[e] * kLog2e;
        }
        const float mn = fmaxf(m, warp_max(sv));   // lane 0 always holds a listed key
        const float corr = exp2f(m - mn);
        const float p = ok ? exp2f(sv - mn) : 0.f;
        l = l * corr + warp_sum(p);
#pragma unroll
        for (int x = 0; x < D / 32; ++x) acc[x] *= corr;
        const int nl = min(32, (cnt - k0) * s.B);
        for (int jj = 0; jj < nl; ++jj) {
            const float pj = __shfl_sync(0xffffffffu, p, jj);
            const int tj = __shfl_sync(0xffffffffu, j, jj);
            const T* vr = Vb + (long long)tj * s.vs[1];
#pragma unroll
            for (int x = 0; x < D / 32; ++x) acc[x] += pj * to_f(vr[lane + 32 * x]);
        }
        m = mn;
    };
    if (s.B < 32)
        for (int k = 0; k < cnt; k += 32 / s.B) gather(k);
    else
        for (int k = 0; k < cnt; ++k) range(li[k] * s.B, li[k] * s.B + s.B, lb[k] * kLog2e);
    range((i / s.B) * s.B, i + 1, 0.f);
    const float inv = 1.f / l;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) op[lane + 32 * e] = from_f<T>(acc[e] * inv);
}

template <int KT, int D>
cudaError_t prefill_mma_t(const Shape& s, const void* Q, const void* K, const void* V, void* O,
                          const Routes& rt, cudaStream_t st)
{
    const int W = (s.T + 32) >> 5;
    const size_t smem = 4 * (size_t)KT * D * 2 + (size_t)W * 4;
    auto k = attend_prefill_mma_kernel<KT, D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int P = 64 / s.g;
    const long long nblk = (s.n + P - 1) / P;
    const unsigned grid = (unsigned)(nblk * s.batch * s.hkv);
    if (grid == 0) return cudaSuccess;
    k<<<grid, 128, smem, st>>>(s, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
                               (__nv_bfloat16*)O, rt);
    return cudaGetLastError();
}

template <int D>
cudaError_t prefill_bf16_d(const Shape& s, const void* Q, const void* K, const void* V, void* O,
                           const Routes& rt, cudaStream_t st)
{
    switch (s.B) {
    case 16: return prefill_mma_t<16, D>(s, Q, K, V, O, rt, st);
    case 32: return prefill_mma_t<32, D>(s, Q, K, V, O, rt, st);
    default: return prefill_mma_t<64, D>(s, Q, K, V, O, rt, st);
    }
}

template <int KT, int D>
cudaError_t dec_mma_t(const Shape& s, const void* q, const void* Kc, const void* Vc, const int* seqlens,
                      const Routes& rt, const DecodeWs& ws, void* O, cudaStream_t st)
{
    const size_t smem = 4 * (size_t)KT * D * 2;
    auto k = dec_attend_mma_kernel<KT, D>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(ws.splits, s.batch * s.hkv);
    k<<<grid, 32, smem, st>>>(s, (const __nv_bfloat16*)q, (const __nv_bfloat16*)Kc, (const __nv_bfloat16*)Vc,
                              seqlens, rt, ws.part, ws.splits);
    dec_combine_kernel<__nv_bfloat16, D><<<s.batch * s.hkv * s.g, 128, 0, st>>>(s, ws.part, ws.splits, kDecCPS,
                                                                                 rt, (__nv_bfloat16*)O);
    return cudaGetLastError();
}

template <int D>
cudaError_t dec_bf16_d(const Shape& s, const void* q, const void* Kc, const void* Vc, const int* seqlens,
                       const Routes& rt, const DecodeWs& ws, void* O, cudaStream_t st)
{
    switch (s.B) {
    case 16: return dec_mma_t<16, D>(s, q, Kc, Vc, seqlens, rt, ws, O, st);
    case 32: return dec_mma_t<32, D>(s, q, Kc, Vc, seqlens, rt, ws, O, st);
    default: return dec_mma_t<64, D>(s, q, Kc, Vc, seqlens, rt, ws, O, st);
    }
}

template <typename T, int D>
cudaError_t rows_t(const Shape& s, const void* Q, const void* K, const void* V, void* O, const Routes& rt,
                   const int* seqlens, cudaStream_t st)
{
    const long long rows = seqlens ? (long long)s.batch * s.hq : (long long)s.batch * s.n * s.hq;
    const unsigned grid = (unsigned)((rows + 3) / 4);
    if (grid == 0) return cudaSuccess;
    attend_rows_kernel<T, D><<<grid, 128, 0, st>>>(s, (const T*)Q, (const T*)K, (const T*)V, (T*)O, rt, seqlens);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_prefill(const Shape& s, int dtype, const void* Q, const void* K, const void* V,
                                  void* O, const Routes& rt, int* perm, int* err, cudaStream_t st)
{
    if (pair_stage2() && attend_pair_supported(s, dtype))
        return launch_attend_prefill_pair(s, Q, K, V, O, rt, perm, err, st);
    if (attend_tc_supported(s, dtype) && !legacy_stage2())
        return launch_attend_prefill_tc(s, Q, K, V, O, rt, perm, err, st);
    if (s.B == 1)   // one token per chunk (Stage 1 is entmax over tokens): the row kernel
        return dtype == DASH_BF16
                   ? (s.d == 128 ? rows_t<__nv_bfloat16, 128>(s, Q, K, V, O, rt, nullptr, st)
                                 : rows_t<__nv_bfloat16, 64>(s, Q, K, V, O, rt, nullptr, st))
                   : (s.d == 128 ? rows_t<float, 128>(s, Q, K, V, O, rt, nullptr, st)
                                 : rows_t<float, 64>(s, Q, K, V, O, rt, nullptr, st));
    if (dtype == DASH_BF16)
        return s.d == 128 ? prefill_bf16_d<128>(s, Q, K, V, O, rt, st) : prefill_bf16_d<64>(s, Q, K, V, O, rt, st);
    return s.d == 128 ? rows_t<float, 128>(s, Q, K, V, O, rt, nullptr, st)
                      : rows_t<float, 64>(s, Q, K, V, O, rt, nullptr, st);
}

bool pair_stage2()
{
    // DASH_STAGE2=pair selects the paired-tile tcgen05 kernel (two tiles per block, 128-key jobs)
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("DASH_STAGE2");
        v = (e && e[0] == 'p') ? 1 : 0;
    }
    return v == 1;
}

bool attend_mask_supported(const Shape& s, int dtype)
{
    if (pair_stage2() && attend_pair_supported(s, dtype)) return true;
    return attend_tc_supported(s, dtype) && !legacy_stage2();
}

cudaError_t launch_attend_prefill_bitmask(const Shape& s, int dtype, const void* Q, const void* K, const void* V,
                                          void* O, const Routes& rt, int* perm, int* err, cudaStream_t st)
{
    if (pair_stage2() && attend_pair_supported(s, dtype))
        return launch_attend_prefill_mask(s, Q, K, V, O, rt, perm, err, st);
    if (attend_tc_supported(s, dtype) && !legacy_stage2())
        return launch_attend_prefill_tc(s, Q, K, V, O, rt, perm, err, st, true);
    return cudaErrorNotSupported;
}

bool legacy_stage2()
{
    // DASH_STAGE2=mma selects the warp-level mma.sync kernel for comparison runs.
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("DASH_STAGE2");
        v = (e && e[0] == 'm') ? 1 : 0;
    }
    return v == 1;
}

int decode_splits(const Shape& s, int kbar_T)
{
    (void)s;
    return (kbar_T + 1 + kDecCPS - 1) / kDecCPS;
}

cudaError_t launch_decode(const Shape& s, int dtype, const void* q, const void* Kc, const void* Vc,
                          const float* kbar, int kbar_T, const int* seqlens, void* O, const Routes& rt,
                          const DecodeWs& ws, cudaStream_t st)
{
    cudaError_t e = launch_route_decode(s, dtype, q, kbar, kbar_T, seqlens, rt, ws.x, ws.err, st);
    if (e != cudaSuccess) return e;
    if (dec_tma_supported(s, dtype) && (!legacy_stage2() || s.pt)) {   // paged caches: the TMA path only
        e = launch_dec_attend_tma(s, q, Kc, Vc, seqlens, rt, ws.part, O, ws.err, st);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    if (s.pt) return cudaErrorInvalidValue;
    if (s.B == 1)
        return dtype == DASH_BF16
                   ? (s.d == 128 ? rows_t<__nv_bfloat16, 128>(s, q, Kc, Vc, O, rt, seqlens, st)
                                 : rows_t<__nv_bfloat16, 64>(s, q, Kc, Vc, O, rt, seqlens, st))
                   : (s.d == 128 ? rows_t<float, 128>(s, q, Kc, Vc, O, rt, seqlens, st)
                                 : rows_t<float, 64>(s, q, Kc, Vc, O, rt, seqlens, st));
    if (dtype == DASH_BF16)
        return s.d == 128 ? dec_bf16_d<128>(s, q, Kc, Vc, seqlens, rt, ws, O, st)
                          : dec_bf16_d<64>(s, q, Kc, Vc, seqlens, rt, ws, O, st);
    return s.d == 128 ? rows_t<float, 128>(s, q, Kc, Vc, O, rt, seqlens, st)
                      : rows_t<float, 64>(s, q, Kc, Vc, O, rt, seqlens, st);
}

}  // namespace dash
