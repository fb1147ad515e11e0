// backward.cu -- gradients of the DashAttention prefill forward with respect to Q, K, V and the
// Stage 0 query qbar.
//
// DashAttention (xllm-io paper review, section 3): the output of Eq. 9 / Proposition 4.1 is
// differentiable in q, k, v and in the prior, so the gradient reaches the Stage 1 entmax scores
// and through them the Stage 0 summaries; the Stage 2 kernel row says that the training
// backward reuses the routed support (the entmax Jacobian is sparse).  The routed set R is
// piecewise constant in the inputs and is taken from the forward call's route lists.
//
// Chain for L = sum dO . O, per pair (b, KV head r), position i, head h of the group:
//   Stage 2:  p = softmax(z + d) over R u D, z = <q, k_j>/sqrt(d);  dv_j += p_j dO;
//             ds_j = p_j (dO . v_j - Delta), Delta = sum_t p_t dO . v_t;  dq += ds_j k_j/sqrt(d);
//             dk_j += ds_j q/sqrt(d);  dbias_c = sum over the group's heads and chunk c's tokens.
//   bias:     dlog w_c = (dbias_c - mean_R dbias)/sigma, dw_c = dlog w_c / w_c, dwhat^(h) = dw/g.
//   entmax:   dtheta = s*dwhat - s (s . dwhat)/sum s, s_c = what_c^(2 - alpha) on the support,
//             theta = gamma zbar:  dzbar = gamma dtheta;  dq += dzbar_c kbar_c/sqrt(d);
//             dkbar_c += dzbar_c q/sqrt(d).
//   Stage 0:  dk_t += pi_t dkbar_c + pi_t (k_t . dkbar_c - kbar_c . dkbar_c) qbar/sqrt(d);
//             dqbar += pi_t (k_t . dkbar_c - kbar_c . dkbar_c) k_t/sqrt(d).
//
// Kernels (fp32 arithmetic on the CUDA cores):
//   bwd_rows_kernel    one block per (position, pair): log-sum-exp and Delta per head, dQ of
//                      Stage 2, dbias per routed chunk, the recomputed per-head entmax weights
//                      (threshold solved again from the forward's summaries), dzbar, and the
//                      Stage 1 part of dQ.  dQ is written once, complete.
//   bwd_tcount / bwd_tscan / bwd_tfill   the routed lists transposed per chunk (positions in
//                      ascending order, deterministic) so that keys gather their queries.
//   bwd_keys_kernel    one block per (32-key tile, pair): dK, dV of Stage 2 from the routed and
//                      diagonal queries of the tile's chunk; the chunk's first tile also sums
//                      dkbar.  No atomics: each tile owns its keys.
//   bwd_stage0_kernel  one block per (chunk, pair): the Stage 0 terms added into dK, and a dqbar
//                      partial per chunk; bwd_qbar_reduce sums the partials in a fixed order.
#include "dash_common.cuh"
#include "entmax.cuh"

namespace dash {
namespace {

constexpr int kBW = 4;        // warps per block
constexpr int kMaxE = 4;      // d / 32 elements per lane in the Stage 0 kernel (d <= 128)

template <typename T>
__device__ __forceinline__ void load_lane(const T* row, int nE, float* out)
{
    const int lane = threadIdx.x & 31;
    for (int k = 0; k < nE; ++k) out[k] = to_f(row[lane + 32 * k]);
}

// ------------------------------------------------------------------------------------------
// Query-major pass.  Dynamic shared memory (floats):
//   qs[g*d], gs[g*d]            the position's query and output-gradient rows
//   red[kBW*g*3]                per-warp (max, sum, sum p*dp) of pass 1
//   lse[g], del[g]              log-sum-exp and Delta per head
//   dbias[T], wsum[T]           per routed entry: bias gradient, GQA-averaged weight
//   xl[g*T]                     (alpha-1) gamma zbar per head and visible chunk
//   dz[g*T]                     dzbar per head and routed entry
//   tau[g], s12[kBW*g*2], misc[kBW]
//   dqp[kBW*g*d]                per-warp dQ partials
// ------------------------------------------------------------------------------------------
template <typename T, int G, int D>
__global__ void __launch_bounds__(32 * kBW) bwd_rows_kernel(Shape s, const T* __restrict__ Q, const T* __restrict__ K,
                                                           const T* __restrict__ V, const T* __restrict__ dO,
                                                           const float* __restrict__ kbar, Routes rt,
                                                           float* __restrict__ dQ, float* __restrict__ lse_out,
                                                           float* __restrict__ del_out, float* __restrict__ dzbar)
{
    extern __shared__ float smf[];
    constexpr int nE = D / 32;
    const int B = s.B, Tn = s.T > 0 ? s.T : 1;
    float* qs = smf;
    float* gs = qs + G * D;
    float* red = gs + G * D;
    float* lse = red + kBW * G * 3;
    float* del = lse + G;
    float* dbias = del + G;
    float* wsum = dbias + Tn;
    float* xl = wsum + Tn;
    float* dz = xl + G * Tn;
    float* tau = dz + G * Tn;
    float* s12 = tau + G;
    float* misc = s12 + kBW * G * 2;
    float* dqp = misc + kBW;

    const int i = blockIdx.x, x = blockIdx.y;
    const int b = x / s.hkv, r = x % s.hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float scale = rsqrtf((float)D);
    const int ci = i / B, nvis = min(ci, s.T);
    // (the lists come from the forward call; a count beyond the visible chunks is clamped so that
    // a bad list cannot index past the shared-memory rows)
    const int cnt = nvis > 0 ? min(max(rt.counts[(long long)x * s.n + i], 0), nvis) : 0;
    const long long lbase = (long long)x * rt.cap + tri_offset(i, B);

    for (int t = threadIdx.x; t < G * D; t += blockDim.x) {
        const int h = t / D, e = t % D;
        const int hq = r * G + h;
        qs[t] = to_f(Q[(long long)b * s.qs[0] + (long long)i * s.qs[1] + (long long)hq * s.qs[2] + e]);
        gs[t] = to_f(dO[(long long)b * s.os[0] + (long long)i * s.os[1] + (long long)hq * s.os[2] + e]);
    }
    __syncthreads();

    // units: routed entries 0..cnt-1 (B tokens each), then the diagonal (tokens ci*B .. i)
    auto unit = [&](int u, int* j0, int* j1, float* bias) {
        if (u < cnt) {
            const int c = min(max(rt.idx[lbase + u], 0), nvis - 1);
            *j0 = c * B; *j1 = c * B + B; *bias = rt.bias[lbase + u];
        } else {
            *j0 = ci * B; *j1 = i + 1; *bias = 0.f;
        }
    };
    auto kv_row = [&](const T* base, const long long st[3], int j) {
        return base + (long long)b * st[0] + (long long)j * st[1] + (long long)r * st[2];
    };

    // pass 1: per head, the running max / sum and sum of p * dp (Delta = dO . o)
    float m[G], l[G], a[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { m[h] = -INFINITY; l[h] = 0.f; a[h] = 0.f; }
    for (int u = warp; u <= cnt; u += kBW) {
        int j0, j1;
        float bias;
        unit(u, &j0, &j1, &bias);
        for (int j = j0; j < j1; ++j) {
            float kv[nE], vv[nE];
            load_lane(kv_row(K, s.ks, j), nE, kv);
            load_lane(kv_row(V, s.vs, j), nE, vv);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float sd = 0.f, pd = 0.f;
#pragma unroll
                for (int k = 0; k < nE; ++k) {
                    sd += qs[h * D + lane + 32 * k] * kv[k];
                    pd += gs[h * D + lane + 32 * k] * vv[k];
                }
                const float z = warp_sum(sd) * scale + bias, dp = warp_sum(pd);
                const float mn = fmaxf(m[h], z), sc = __expf(m[h] - mn), pe = __expf(z - mn);
                l[h] = l[h] * sc + pe;
                a[h] = a[h] * sc + pe * dp;
                m[h] = mn;
            }
        }
    }
    if (lane == 0)
        for (int h = 0; h < G; ++h) {
            red[(warp * G + h) * 3 + 0] = m[h];
            red[(warp * G + h) * 3 + 1] = l[h];
            red[(warp * G + h) * 3 + 2] = a[h];
        }
    __syncthreads();
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int w = 0; w < kBW; ++w) M = fmaxf(M, red[(w * G + h) * 3]);
        float L = 0.f, A = 0.f;
        for (int w = 0; w < kBW; ++w) {
            const float f = __expf(red[(w * G + h) * 3] - M);
            L += red[(w * G + h) * 3 + 1] * f;
            A += red[(w * G + h) * 3 + 2] * f;
        }
        lse[h] = M + __logf(L);
        del[h] = A / L;
        const long long o = ((long long)b * s.hq + r * G + h) * s.n + i;
        lse_out[o] = lse[h];
        del_out[o] = del[h];
    }
    __syncthreads();

    // pass 2: ds, the Stage 2 part of dQ, and dbias per routed entry
    float dq[G][nE];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int k = 0; k < nE; ++k) dq[h][k] = 0.f;
    for (int u = warp; u <= cnt; u += kBW) {
        int j0, j1;
        float bias;
        unit(u, &j0, &j1, &bias);
        float db = 0.f;
        for (int j = j0; j < j1; ++j) {
            float kv[nE], vv[nE];
            load_lane(kv_row(K, s.ks, j), nE, kv);
            load_lane(kv_row(V, s.vs, j), nE, vv);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float sd = 0.f, pd = 0.f;
#pragma unroll
                for (int k = 0; k < nE; ++k) {
                    sd += qs[h * D + lane + 32 * k] * kv[k];
                    pd += gs[h * D + lane + 32 * k] * vv[k];
                }
                const float z = warp_sum(sd) * scale + bias, dp = warp_sum(pd);
                const float p = __expf(z - lse[h]);
                const float ds = p * (dp - del[h]);
                db += ds;
#pragma unroll
                for (int k = 0; k < nE; ++k) dq[h][k] += ds * kv[k] * scale;
            }
        }
        if (u < cnt && lane == 0) dbias[u] = db;
    }
    __syncthreads();

    // Stage 1: logits of every visible chunk, the thresholds, the weights of the routed entries
    if (cnt > 0) {
        const float am1 = s.alpha - 1.f, pw = 1.f / am1;
        const int mode = ent_mode(s.alpha);
        const float* kb0 = kbar + (long long)x * s.T * D;
        for (int c = warp; c < nvis; c += kBW) {
            float kv[nE];
            for (int k = 0; k < nE; ++k) kv[k] = kb0[(long long)c * D + lane + 32 * k];
            for (int h = 0; h < G; ++h) {
                float sd = 0.f;
                for (int k = 0; k < nE; ++k) sd += qs[h * D + lane + 32 * k] * kv[k];
                sd = warp_sum(sd);
                if (lane == 0) xl[h * Tn + c] = am1 * (s.gamma * sd * scale);
            }
        }
        __syncthreads();
        for (int h = warp; h < G; h += kBW) {
            const float t = warp_threshold(xl + h * Tn, nvis, s.alpha);
            if (lane == 0) tau[h] = t;
        }
        __syncthreads();
        // GQA-averaged weight of each routed entry and the mean of dbias over the entries
        float dsum = 0.f;
        for (int e = threadIdx.x; e < cnt; e += blockDim.x) {
            const int c = min(max(rt.idx[lbase + e], 0), nvis - 1);
            float w = 0.f;
            for (int h = 0; h < G; ++h) {
                const float u = xl[h * Tn + c] - tau[h];
                if (u > 0.f) w += ent_pow(u, pw, mode);
            }
            wsum[e] = w / G;
            dsum += dbias[e];
        }
        dsum = warp_sum(dsum);
        if (lane == 0) misc[warp] = dsum;
        __syncthreads();
        float mdb = 0.f;
        for (int w = 0; w < kBW; ++w) mdb += misc[w];
        mdb /= cnt;
        // per head: sum s and sum s * dwhat over the support
        float S1[G], S2[G];
#pragma unroll
        for (int h = 0; h < G; ++h) { S1[h] = 0.f; S2[h] = 0.f; }
        for (int e = threadIdx.x; e < cnt; e += blockDim.x) {
            const int c = min(max(rt.idx[lbase + e], 0), nvis - 1);
            const float dw = wsum[e] > 0.f ? s.inv_sigma * (dbias[e] - mdb) / wsum[e] / G : 0.f;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float u = xl[h * Tn + c] - tau[h];
                if (u > 0.f) {
                    const float sv = ent_dpow(u, pw, mode);   // what^(2 - alpha) = u^((2 - alpha)/(alpha - 1))
                    S1[h] += sv;
                    S2[h] += sv * dw;
                }
            }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float a1 = warp_sum(S1[h]), a2 = warp_sum(S2[h]);
            if (lane == 0) { s12[(warp * G + h) * 2] = a1; s12[(warp * G + h) * 2 + 1] = a2; }
        }
        __syncthreads();
        for (int e = threadIdx.x; e < cnt; e += blockDim.x) {
            const int c = min(max(rt.idx[lbase + e], 0), nvis - 1);
            const float dw = wsum[e] > 0.f ? s.inv_sigma * (dbias[e] - mdb) / wsum[e] / G : 0.f;
            for (int h = 0; h < G; ++h) {
                float t1 = 0.f, t2 = 0.f;
                for (int w = 0; w < kBW; ++w) { t1 += s12[(w * G + h) * 2]; t2 += s12[(w * G + h) * 2 + 1]; }
                const float u = xl[h * Tn + c] - tau[h];
                float v = 0.f;
                if (u > 0.f && t1 > 0.f) {
                    const float sv = ent_dpow(u, pw, mode);
                    v = s.gamma * (sv * dw - sv * t2 / t1);
                }
                dz[e * G + h] = v;
                dzbar[(lbase + e) * G + h] = v;
            }
        }
        __syncthreads();
        // the Stage 1 part of dQ
        for (int e = warp; e < cnt; e += kBW) {
            const int c = min(max(rt.idx[lbase + e], 0), nvis - 1);
            float kv[nE];
#pragma unroll
            for (int k = 0; k < nE; ++k) kv[k] = kb0[(long long)c * D + lane + 32 * k];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float v = dz[e * G + h] * scale;
#pragma unroll
                for (int k = 0; k < nE; ++k) dq[h][k] += v * kv[k];
            }
        }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int k = 0; k < nE; ++k) dqp[(warp * G + h) * D + lane + 32 * k] = dq[h][k];
    __syncthreads();
    for (int t = threadIdx.x; t < G * D; t += blockDim.x) {
        const int h = t / D, e = t % D;
        float v = 0.f;
        for (int w = 0; w < kBW; ++w) v += dqp[(w * G + h) * D + e];
        dQ[(((long long)b * s.n + i) * s.hq + r * G + h) * D + e] = v;
    }
}

// ------------------------------------------------------------------------------------------
// Transposed route lists: for each (pair, complete chunk c), the positions that route c in
// ascending order and the entry index of c in each position's list.
// ------------------------------------------------------------------------------------------
__global__ void bwd_tcount_kernel(Shape s, Routes rt, int* __restrict__ tcnt)
{
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)s.batch * s.hkv * s.n) return;
    const int x = (int)(t / s.n), i = (int)(t % s.n);
    if (i / s.B == 0) return;
    const int cnt = min(rt.counts[t], min(i / s.B, s.T));
    const long long base = (long long)x * rt.cap + tri_offset(i, s.B);
    for (int e = 0; e < cnt; ++e) {
        const int c = rt.idx[base + e];
        if (c >= 0 && c < s.T) atomicAdd(&tcnt[(long long)x * s.T + c], 1);
    }
}

// one block per pair: exclusive prefix sum of the chunk counts (toff has T + 1 entries)
__global__ void __launch_bounds__(1024) bwd_tscan_kernel(Shape s, const int* __restrict__ tcnt, int* __restrict__ toff)
{
    __shared__ int part[1024];
    const int x = blockIdx.x, T = s.T;
    const int per = (T + blockDim.x - 1) / blockDim.x;
    const int c0 = threadIdx.x * per, c1 = min(T, c0 + per);
    int sum = 0;
    for (int c = c0; c < c1; ++c) sum += tcnt[(long long)x * T + c];
    part[threadIdx.x] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int k = 0; k < (int)blockDim.x; ++k) { const int v = part[k]; part[k] = acc; acc += v; }
        toff[(long long)x * (T + 1) + T] = acc;
    }
    __syncthreads();
    int acc = part[threadIdx.x];
    for (int c = c0; c < c1; ++c) {
        toff[(long long)x * (T + 1) + c] = acc;
        acc += tcnt[(long long)x * T + c];
    }
}

// one warp per (chunk, pair): scan positions (c+1)B .. n-1 in order, binary-search c in each
// position's ascending list, append the hits
__global__ void bwd_tfill_kernel(Shape s, Routes rt, const int* __restrict__ toff, int* __restrict__ tpos,
                                 int* __restrict__ tent)
{
    const int c = blockIdx.x, x = blockIdx.y, lane = threadIdx.x;
    int out = toff[(long long)x * (s.T + 1) + c];
    const long long obase = (long long)x * rt.cap;
    for (int i0 = (c + 1) * s.B; i0 < s.n; i0 += 32) {
        const int i = i0 + lane;
        int e = -1;
        if (i < s.n) {
            const int cnt = min(rt.counts[(long long)x * s.n + i], min(i / s.B, s.T));
            const int* lst = rt.idx + (long long)x * rt.cap + tri_offset(i, s.B);
            int lo = 0, hi = cnt;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (lst[mid] < c) lo = mid + 1; else hi = mid;
            }
            if (lo < cnt && lst[lo] == c) e = lo;
        }
        const uint32_t hit = __ballot_sync(0xffffffffu, e >= 0);
        if (e >= 0) {
            const int k = out + __popc(hit & ((1u << lane) - 1u));
            tpos[obase + k] = i;
            tent[obase + k] = e;
        }
        out += __popc(hit);
    }
}

// ------------------------------------------------------------------------------------------
// Key-major pass: dK, dV (Stage 2) and dkbar.  One block per (KT-key tile, pair).  Lane jj owns
// key j0 + jj; each warp walks its share of the queries and keeps private accumulators.
// Dynamic shared memory (floats): Ks[KT][D+1], Vs[KT][D+1], dKa[kBW][KT][D+1], dVa[kBW][KT][D+1],
// qv[kBW][D], gv[kBW][D], dkb[kBW][D].
// ------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(32 * kBW) bwd_keys_kernel(Shape s, const T* __restrict__ Q, const T* __restrict__ K,
                                                           const T* __restrict__ V, const T* __restrict__ dO, Routes rt,
                                                           const float* __restrict__ lse_in, const float* __restrict__ del_in,
                                                           const float* __restrict__ dzbar, const int* __restrict__ toff,
                                                           const int* __restrict__ tpos, const int* __restrict__ tent,
                                                           float* __restrict__ dK, float* __restrict__ dV,
                                                           float* __restrict__ dkbar, int KT)
{
    extern __shared__ float smf[];
    constexpr int P = D + 1;
    const int G = s.g, B = s.B;
    float* Ks = smf;
    float* Vs = Ks + KT * P;
    float* dKa = Vs + KT * P;
    float* dVa = dKa + kBW * KT * P;
    float* qv = dVa + kBW * KT * P;
    float* gv = qv + kBW * D;
    float* dkb = gv + kBW * D;

    const int j0 = blockIdx.x * KT, x = blockIdx.y;
    const int b = x / s.hkv, r = x % s.hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float scale = rsqrtf((float)D);
    const int jn = min(KT, s.n - j0);
    const int c = j0 / B;
    const bool first = (j0 % B) == 0 && c < s.T;   // this tile sums the chunk's dkbar

    for (int t = threadIdx.x; t < KT * D; t += blockDim.x) {
        const int jj = t / D, e = t % D;
        float kvv = 0.f, vvv = 0.f;
        if (jj < jn) {
            const long long j = j0 + jj;
            kvv = to_f(K[(long long)b * s.ks[0] + j * s.ks[1] + (long long)r * s.ks[2] + e]);
            vvv = to_f(V[(long long)b * s.vs[0] + j * s.vs[1] + (long long)r * s.vs[2] + e]);
        }
        Ks[jj * P + e] = kvv;
        Vs[jj * P + e] = vvv;
    }
    for (int t = threadIdx.x; t < kBW * KT * P; t += blockDim.x) { dKa[t] = 0.f; dVa[t] = 0.f; }
    for (int t = threadIdx.x; t < kBW * D; t += blockDim.x) dkb[t] = 0.f;
    __syncthreads();

    // queries: the routed ones of chunk c (transposed list), then the diagonal ones
    int r0 = 0, r1 = 0;
    if (c < s.T) {
        r0 = toff[(long long)x * (s.T + 1) + c];
        r1 = toff[(long long)x * (s.T + 1) + c + 1];
    }
    const int nr = r1 - r0;
    const int d0 = j0, d1 = min(s.n, (c + 1) * B);   // diagonal queries with i >= j0
    const int nq = nr + max(0, d1 - d0);
    float* q_w = qv + warp * D;
    float* g_w = gv + warp * D;
    float* dka = dKa + warp * KT * P;
    float* dva = dVa + warp * KT * P;
    for (int u = warp; u < nq; u += kBW) {
        int i;
        float bias = 0.f;
        long long ent = -1;
        if (u < nr) {
            i = tpos[(long long)x * rt.cap + r0 + u];
            const int e = tent[(long long)x * rt.cap + r0 + u];
            ent = (long long)x * rt.cap + tri_offset(i, B) + e;
            bias = rt.bias[ent];
        } else {
            i = d0 + (u - nr);
        }
        for (int h = 0; h < G; ++h) {
            const int hq = r * G + h;
            __syncwarp();
            for (int e = lane; e < D; e += 32) {
                q_w[e] = to_f(Q[(long long)b * s.qs[0] + (long long)i * s.qs[1] + (long long)hq * s.qs[2] + e]);
                g_w[e] = to_f(dO[(long long)b * s.os[0] + (long long)i * s.os[1] + (long long)hq * s.os[2] + e]);
            }
            __syncwarp();
            const long long o = ((long long)b * s.hq + hq) * s.n + i;
            const float lse = lse_in[o], dl = del_in[o];
            if (first && ent >= 0) {
                const float v = dzbar[ent * G + h] * scale;
                for (int e = lane; e < D; e += 32) dkb[warp * D + e] += v * q_w[e];
            }
            const int jj = lane;
            const bool valid = jj < jn && (ent >= 0 || j0 + jj <= i);
            if (valid) {
                float sd = 0.f, pd = 0.f;
#pragma unroll 16
                for (int e = 0; e < D; ++e) {
                    sd += q_w[e] * Ks[jj * P + e];
                    pd += g_w[e] * Vs[jj * P + e];
                }
                const float p = __expf(sd * scale + bias - lse);
                const float ds = p * (pd - dl) * scale;
#pragma unroll 16
                for (int e = 0; e < D; ++e) {
                    dva[jj * P + e] += p * g_w[e];
                    dka[jj * P + e] += ds * q_w[e];
                }
            }
        }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < jn * D; t += blockDim.x) {
        const int jj = t / D, e = t % D;
        float a = 0.f, v = 0.f;
        for (int w = 0; w < kBW; ++w) { a += dKa[(w * KT + jj) * P + e]; v += dVa[(w * KT + jj) * P + e]; }
        const long long o = (((long long)b * s.n + j0 + jj) * s.hkv + r) * D + e;
        dK[o] = a;
        dV[o] = v;
    }
    if (first)
        for (int e = threadIdx.x; e < D; e += blockDim.x) {
            float a = 0.f;
            for (int w = 0; w < kBW; ++w) a += dkb[w * D + e];
            dkbar[((long long)x * s.T + c) * D + e] = a;
        }
}

// ------------------------------------------------------------------------------------------
// Stage 0 backward: one block per (complete chunk, pair).  Shared memory (floats):
// gk[D] (dkbar_c), kb[D] (kbar_c), qb[D], at[B], part[kBW][D].
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(32 * kBW) bwd_stage0_kernel(Shape s, const T* __restrict__ K,
                                                             const float* __restrict__ qbar,
                                                             const float* __restrict__ kbar,
                                                             const float* __restrict__ dkbar, float* __restrict__ dK,
                                                             float* __restrict__ qpart)
{
    __shared__ float gk[128], kb[128], qb[128], at[128], part[kBW][128], misc[2];
    const int c = blockIdx.x, x = blockIdx.y;
    const int b = x / s.hkv, r = x % s.hkv;
    const int D = s.d, B = s.B, nE = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float scale = rsqrtf((float)D);
    for (int e = threadIdx.x; e < D; e += blockDim.x) {
        gk[e] = dkbar[((long long)x * s.T + c) * D + e];
        kb[e] = kbar[((long long)x * s.T + c) * D + e];
        qb[e] = qbar[r * D + e];
        for (int w = 0; w < kBW; ++w) part[w][e] = 0.f;
    }
    __syncthreads();
    auto krow = [&](int t) { return K + (long long)b * s.ks[0] + (long long)(c * B + t) * s.ks[1] + (long long)r * s.ks[2]; };
    for (int t = warp; t < B; t += kBW) {
        float kv[kMaxE];
        load_lane(krow(t), nE, kv);
        float a = 0.f;
        for (int k = 0; k < nE; ++k) a += qb[lane + 32 * k] * kv[k];
        a = warp_sum(a);
        if (lane == 0) at[t] = a * scale;
    }
    if (warp == 0) {
        float kg = 0.f;
        for (int e = lane; e < D; e += 32) kg += kb[e] * gk[e];
        kg = warp_sum(kg);
        if (lane == 0) misc[0] = kg;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float mx = -INFINITY, den = 0.f;
        for (int t = 0; t < B; ++t) mx = fmaxf(mx, at[t]);
        for (int t = 0; t < B; ++t) { at[t] = __expf(at[t] - mx); den += at[t]; }
        misc[1] = 1.f / den;
    }
    __syncthreads();
    const float kbg = misc[0], inv = misc[1];
    for (int t = warp; t < B; t += kBW) {
        float kv[kMaxE];
        load_lane(krow(t), nE, kv);
        float kg = 0.f;
        for (int k = 0; k < nE; ++k) kg += kv[k] * gk[lane + 32 * k];
        kg = warp_sum(kg);
        const float pi = at[t] * inv, da = pi * (kg - kbg);
        float* out = dK + (((long long)b * s.n + c * B + t) * s.hkv + r) * D;
        for (int k = 0; k < nE; ++k) {
            const int e = lane + 32 * k;
            out[e] += pi * gk[e] + da * qb[e] * scale;
            part[warp][e] += da * kv[k] * scale;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < D; e += blockDim.x) {
        float a = 0.f;
        for (int w = 0; w < kBW; ++w) a += part[w][e];
        qpart[((long long)x * s.T + c) * D + e] = a;
    }
}

// dqbar[r] = sum over sequences and chunks of the partials, in a fixed order
__global__ void bwd_qbar_reduce_kernel(Shape s, const float* __restrict__ qpart, float* __restrict__ dqbar)
{
    const int r = blockIdx.x, e = threadIdx.x;
    if (e >= s.d) return;
    float a = 0.f;
    for (int b = 0; b < s.batch; ++b)
        for (int c = 0; c < s.T; ++c) a += qpart[(((long long)b * s.hkv + r) * s.T + c) * s.d + e];
    dqbar[r * s.d + e] = a;
}

template <typename T, int G, int D>
cudaError_t rows_g(const Shape& s, const T* Q, const T* K, const T* V, const T* dO, const float* kbar, const Routes& rt,
                   float* dQ, const BackwardWs& ws, cudaStream_t st)
{
    const size_t smem = backward_rows_smem(s);
    cudaError_t e = cudaFuncSetAttribute(bwd_rows_kernel<T, G, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_rows_kernel<T, G, D><<<dim3(s.n, s.batch * s.hkv), 32 * kBW, smem, st>>>(s, Q, K, V, dO, kbar, rt, dQ, ws.lse,
                                                                                ws.del, ws.dzbar);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t rows_d(const Shape& s, const T* Q, const T* K, const T* V, const T* dO, const float* kbar, const Routes& rt,
                   float* dQ, const BackwardWs& ws, cudaStream_t st)
{
    switch (s.g) {
    case 1: return rows_g<T, 1, D>(s, Q, K, V, dO, kbar, rt, dQ, ws, st);
    case 2: return rows_g<T, 2, D>(s, Q, K, V, dO, kbar, rt, dQ, ws, st);
    case 4: return rows_g<T, 4, D>(s, Q, K, V, dO, kbar, rt, dQ, ws, st);
    case 8: return rows_g<T, 8, D>(s, Q, K, V, dO, kbar, rt, dQ, ws, st);
    case 16: return rows_g<T, 16, D>(s, Q, K, V, dO, kbar, rt, dQ, ws, st);
    default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t backward_t(const Shape& s, const T* Q, const T* K, const T* V, const T* dO, const float* qbar,
                       const float* kbar, const Routes& rt, float* dQ, float* dK, float* dV, float* dqbar,
                       const BackwardWs& ws, cudaStream_t st)
{
    const int pairs = s.batch * s.hkv;
    cudaError_t e;
    if (s.T > 0) {
        e = cudaMemsetAsync(ws.tcnt, 0, sizeof(int) * (size_t)pairs * s.T, st);
        if (e != cudaSuccess) return e;
        const long long tot = (long long)pairs * s.n;
        bwd_tcount_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(s, rt, ws.tcnt);
        bwd_tscan_kernel<<<pairs, 1024, 0, st>>>(s, ws.tcnt, ws.toff);
        bwd_tfill_kernel<<<dim3(s.T, pairs), 32, 0, st>>>(s, rt, ws.toff, ws.tpos, ws.tent);
    }
    e = s.d == 128 ? rows_d<T, 128>(s, Q, K, V, dO, kbar, rt, dQ, ws, st)
                   : rows_d<T, 64>(s, Q, K, V, dO, kbar, rt, dQ, ws, st);
    if (e != cudaSuccess) return e;
    const int KT = s.B >= 32 ? 32 : s.B;
    const size_t keys_smem = backward_keys_smem(s);
    auto keys = s.d == 128 ? bwd_keys_kernel<T, 128> : bwd_keys_kernel<T, 64>;
    e = cudaFuncSetAttribute(keys, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)keys_smem);
    if (e != cudaSuccess) return e;
    keys<<<dim3((s.n + KT - 1) / KT, pairs), 32 * kBW, keys_smem, st>>>(
        s, Q, K, V, dO, rt, ws.lse, ws.del, ws.dzbar, ws.toff, ws.tpos, ws.tent, dK, dV, ws.dkbar, KT);
    if (s.T > 0)
        bwd_stage0_kernel<T><<<dim3(s.T, pairs), 32 * kBW, 0, st>>>(s, K, qbar, kbar, ws.dkbar, dK, ws.qpart);
    bwd_qbar_reduce_kernel<<<s.hkv, 128, 0, st>>>(s, ws.qpart, dqbar);
    return cudaGetLastError();
}

}  // namespace

size_t backward_rows_smem(const Shape& s)
{
    const size_t G = s.g, D = s.d, Tn = s.T > 0 ? s.T : 1;
    return sizeof(float) * (2 * G * D + kBW * G * 3 + 2 * G + 2 * Tn + 2 * G * Tn + G + kBW * G * 2 + kBW + kBW * G * D);
}

size_t backward_keys_smem(const Shape& s)
{
    const size_t KT = s.B >= 32 ? 32 : s.B, P = s.d + 1;
    return sizeof(float) * (2 * KT * P + 2 * kBW * KT * P + 3 * kBW * (size_t)s.d);
}

cudaError_t launch_backward(const Shape& s, int dtype, const void* Q, const void* K, const void* V, const void* dO,
                            const float* qbar, const float* kbar, const Routes& rt, float* dQ, float* dK, float* dV,
                            float* dqbar, const BackwardWs& ws, cudaStream_t st)
{
    if (dtype == DASH_BF16)
        return backward_t(s, static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
                          static_cast<const __nv_bfloat16*>(V), static_cast<const __nv_bfloat16*>(dO), qbar, kbar, rt,
                          dQ, dK, dV, dqbar, ws, st);
    return backward_t(s, static_cast<const float*>(Q), static_cast<const float*>(K), static_cast<const float*>(V),
                      static_cast<const float*>(dO), qbar, kbar, rt, dQ, dK, dV, dqbar, ws, st);
}

}  // namespace dash
