// dash_common.cuh -- shared device helpers and internal launcher declarations of the
// B200 DashAttention library.  Internal only: the public interface is include/dash.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/dash.h"

namespace dash {

constexpr float kLog2e = 1.4426950408889634f;

// Shape and hyper-parameters as the kernels see them.
struct Shape {
    int batch, n, hq, hkv, g, d, B, T;   // T = floor(n / B) complete chunks
    float alpha, gamma, inv_sigma;
    long long qs[3], ks[3], vs[3], os[3];
    // paged decode caches (pt == null: contiguous [b][t][head][d] by ks / vs)
    const int* pt;                       // page table [batch][pmax]
    int psz, pmax, npages;               // page size (tokens), pages per sequence, pool pages
    long long kps, vps;                  // elements between pages of the K / V pools
    long long polls;                     // poll limit of the bounded waits of the Stage 2 tcgen05 kernels
};

// Poll limit the next launches' Shapes carry (dash_set_wait_limit; the default is kWaitPolls).
long long wait_limit();

// Element offset of token t of sequence b, KV head r in a K (st = ks, ps = kps) or V cache; -1
// when the token's page is unmapped (a page id outside [0, npages), or t beyond the table), so
// that callers skip the access instead of leaving the pool.
__device__ __forceinline__ long long kv_off(const Shape& s, const long long st[3], long long ps, int b, long long t,
                                            int r)
{
    if (!s.pt) return (long long)b * st[0] + t * st[1] + (long long)r * st[2];
    const long long slot = t / s.psz;
    if (slot >= s.pmax) return -1;
    const int pg = s.pt[(long long)b * s.pmax + slot];
    if (pg < 0 || pg >= s.npages) return -1;
    return (long long)pg * ps + (t % s.psz) * st[1] + (long long)r * st[2];
}

// Route storage: where Stage 1 writes and Stage 2 reads.
struct Routes {
    int* counts;        // [b, hkv, rows]
    int* idx;           // [b, hkv, cap]
    float* bias;        // [b, hkv, cap]
    uint32_t* bitmask;  // [b, hkv, rows, words] or null
    long long cap;      // entries per (b, r)
    int words;          // ceil(T / 32)
};

// Start of position i's list inside one (b, r) route arena: positions with c = floor(i/B)
// hold c entries each, so the lists before i take B * c*(c-1)/2 + (i - c*B) * c entries.
__host__ __device__ inline long long tri_offset(int i, int B)
{
    long long c = i / B;
    return (long long)B * (c * (c - 1) / 2) + (long long)(i - c * B) * c;
}

// Programmatic dependent launch: a kernel launched with launch_after() may start while the
// previous kernel of the stream still runs; it calls pdl_wait() (every thread, before any early
// exit) ahead of its first access to that kernel's results, so completion stays transitive along
// the stream.  pdl_launch_dependents() lets the next such kernel start early.  Both are no-ops
// for kernels launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... P, typename... A>
inline cudaError_t launch_after(void (*k)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, A... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, args...);
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ int warp_isum(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// 16-byte vector of elements of type T converted to fp32.
template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void load(const float* p, float* out)
    {
        float4 v = *reinterpret_cast<const float4*>(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
    // the raw 16 bytes, and their conversion (split so that several loads can be in flight)
    __device__ __forceinline__ static uint4 raw(const float* p) { return *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ static void cvt(uint4 v, float* out)
    {
        out[0] = __uint_as_float(v.x); out[1] = __uint_as_float(v.y);
        out[2] = __uint_as_float(v.z); out[3] = __uint_as_float(v.w);
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void cvt(uint4 v, float* out)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            out[2 * k] = __uint_as_float(w[k] << 16);
            out[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 raw(const __nv_bfloat16* p) { return *reinterpret_cast<const uint4*>(p); }
    __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* out)
    {
        cvt(*reinterpret_cast<const uint4*>(p), out);
    }
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Shape and hyper-parameter checks shared by every entry point (DASH_OK or a DASH_E* status).
int check_params(const dash_params* p);

// ---- launchers (each returns cudaGetLastError() of its launches) -------------------------
// Stage 0: summaries of complete chunks of positions [0, len_b) and, if state != null, the
// running state of the incomplete chunk.  len == null means every sequence has length s.n.
// planes (optional, bf16 [b][hkv][3][T][d]): each summary split exactly into hi + mid + lo.
cudaError_t launch_stage0(const Shape& s, int dtype, const void* K, const float* qbar,
                          const int* len, float* kbar, int kbar_T, float* state, cudaStream_t st,
                          __nv_bfloat16* planes = nullptr, float* knorm = nullptr);
cudaError_t launch_append(const Shape& s, int dtype, const void* k_new, const void* v_new,
                          const float* qbar, void* Kc, void* Vc, float* kbar, int kbar_T,
                          float* state, int* seqlens, cudaStream_t st);
// Stage 1 for prefill: routes of every position.
// redo: one byte per (sequence, KV head, position block) for the long-row kernel's overflow flags
// knorm: per (sequence, KV head) the largest Euclidean norm of a summary (written by Stage 0
// with the planes; the long-row kernel's hi-plane bound)
// redo_list: scratch of 1 + batch * h_kv * n ints for the list of position blocks to recompute
// spill: route_long_spill_bytes(s) of scratch for the long-row kernel's candidate lists (or null)
cudaError_t launch_route_prefill(const Shape& s, int dtype, const void* Q, const float* kbar,
                                 const __nv_bfloat16* planes, const float* knorm, const Routes& rt,
                                 unsigned char* redo, int* redo_list, void* spill, int* err, cudaStream_t st);
// tcgen05 / TMEM variant of Stage 1 (bf16, d = 128, at most 512 complete chunks)
bool route_tcgen05_supported(const Shape& s, int dtype);
cudaError_t launch_route_prefill_tcgen05(const Shape& s, const void* Q, const __nv_bfloat16* planes, const Routes& rt,
                                         int* err, cudaStream_t st);
size_t route_prefill_smem(const Shape& s, int* positions_per_block);
// tcgen05 variant for rows of more than 512 chunks (bf16, d = 128, g in {4, 8, 16}): blocks of
// route_long_positions(s) positions; a block whose candidate lists overflow sets its redo byte
// and writes nothing, and launch_route_prefill recomputes those blocks with the kernels above.
bool route_long_supported(const Shape& s, int dtype);
int route_long_positions(const Shape& s);
cudaError_t launch_route_prefill_long(const Shape& s, const void* Q, const __nv_bfloat16* planes, const float* knorm,
                                      const Routes& rt, unsigned char* redo, int* err, void* spill, cudaStream_t st);
// per-thread spill entries of the long-row kernel's candidate lists and the bytes of their areas
int route_long_spill_entries(const Shape& s);
size_t route_long_spill_bytes(const Shape& s);
// Stage 2 for prefill.
// perm: workspace of batch * h_kv * n ints (the tensor-core path's grouped position order)
cudaError_t launch_attend_prefill(const Shape& s, int dtype, const void* Q, const void* K,
                                  const void* V, void* O, const Routes& rt, int* perm, int* err, cudaStream_t st);
// tcgen05 / TMEM / TMA variant (bf16, d = 128, chunk 64 or 128); err receives a non-zero code
// when one of its bounded waits times out.
bool attend_tc_supported(const Shape& s, int dtype);
// perm: workspace of batch * h_kv * n ints for the grouped position order (null: sequence order)
// mask = true: the routed support is read from rt.bitmask (the bit-packed block mask) instead of
// the chunk lists, with identical results.
cudaError_t launch_attend_prefill_tc(const Shape& s, const void* Q, const void* K, const void* V, void* O,
                                     const Routes& rt, int* perm, int* err, cudaStream_t st, bool mask = false);
bool legacy_stage2();
bool pair_stage2();
// Stage 2 driven by the bit-packed block mask on the tensor-core kernel the list-driven Stage 2 uses
// for these shapes; cudaErrorNotSupported where neither tensor-core kernel applies.
bool attend_mask_supported(const Shape& s, int dtype);
cudaError_t launch_attend_prefill_bitmask(const Shape& s, int dtype, const void* Q, const void* K, const void* V,
                                          void* O, const Routes& rt, int* perm, int* err, cudaStream_t st);
// Helpers of the tensor-core Stage 2 kernels (stage2_tc.cu): a 4-D TMA map over a
// [batch, n, heads, 128] bf16 tensor with box (64 d, bh heads, bp positions, 1) and 128-byte
// swizzle; whether positions are grouped by route similarity before tiling; the grouping launch.
bool s2_make_map(CUtensorMap* map, const void* ptr, int batch, int n, int heads, const long long st[3], int bh, int bp);
bool s2_encode_available();
bool s2_grouping_enabled(const Shape& s);
cudaError_t launch_group_positions(const Shape& s, const Routes& rt, int P, int* perm, cudaStream_t st);
// Paired-tile Stage 2 (stage2_pair.cu): one block per two 128-row tiles sharing one key walk of
// 128-key jobs (bf16, d = 128, chunk 32 / 64 / 128, g in {4, 8, 16}); selected by DASH_STAGE2=pair.
bool attend_pair_supported(const Shape& s, int dtype);
cudaError_t launch_attend_prefill_pair(const Shape& s, const void* Q, const void* K, const void* V, void* O,
                                       const Routes& rt, int* perm, int* err, cudaStream_t st);
// The same kernel driven by the bit-packed block mask rt.bitmask (plus the bias lists) instead of
// the chunk lists.
cudaError_t launch_attend_prefill_mask(const Shape& s, const void* Q, const void* K, const void* V, void* O,
                                       const Routes& rt, int* perm, int* err, cudaStream_t st);
// Decode: Stage 1 (logits, thresholds, GQA aggregation) and Stage 2 (split + merge).
struct DecodeWs {
    float* x;        // [b, hkv, g, T]  scaled logits, then head weights
    float* part;     // [b, hkv, splits, g, d + 2]
    int splits;      // partial slots per (b, r)
    int* err;        // status word of bounded waits
};
// Decode Stage 2 with TMA-fed K/V rings (bf16, d = 128, chunk 64 or 128).
bool dec_tma_supported(const Shape& s, int dtype);
int dec_tma_blocks();   // persistent blocks (the SM count); partial slots per pair
cudaError_t launch_dec_attend_tma(const Shape& s, const void* q, const void* Kc, const void* Vc, const int* seqlens,
                                  const Routes& rt, float* part, void* O, int* err, cudaStream_t st);
// status: the decode call's status word, set to 0 by the routing launch before later kernels run
cudaError_t launch_route_decode(const Shape& s, int dtype, const void* q, const float* kbar, int kbar_T,
                                const int* seqlens, const Routes& rt, float* X, int* status, cudaStream_t st);
// Decode Stage 1 in one launch (8-block clusters per (sequence, KV head); g <= 16, d = 64 / 128).
int dec_route_cluster_per(int kbar_T);
bool dec_route_cluster_supported(const Shape& s, int kbar_T);
cudaError_t launch_route_decode_cluster(const Shape& s, int dtype, const void* q, const float* kbar, int kbar_T,
                                        const int* seqlens, const Routes& rt, int* status, cudaStream_t st);
cudaError_t launch_decode(const Shape& s, int dtype, const void* q, const void* Kc, const void* Vc,
                          const float* kbar, int kbar_T, const int* seqlens, void* O,
                          const Routes& rt, const DecodeWs& ws, cudaStream_t st);
int decode_splits(const Shape& s, int kbar_T);

// Backward pass (backward.cu): scratch of one call, all in the caller's workspace.
struct BackwardWs {
    float* lse;    // [b, h_q, n] log-sum-exp of each row's biased logits
    float* del;    // [b, h_q, n] Delta = dO . O
    float* dzbar;  // [b, h_kv, route capacity, g] gradient of the chunk logits, per routed entry
    int* tcnt;     // [b, h_kv, T] routing positions per chunk
    int* toff;     // [b, h_kv, T + 1] their offsets
    int* tpos;     // [b, h_kv, route capacity] positions routing each chunk, ascending
    int* tent;     // [b, h_kv, route capacity] the chunk's entry index in each position's list
    float* dkbar;  // [b, h_kv, T, d]
    float* qpart;  // [b, h_kv, T, d] dqbar partial per chunk
};
size_t backward_rows_smem(const Shape& s);
size_t backward_keys_smem(const Shape& s);
cudaError_t launch_backward(const Shape& s, int dtype, const void* Q, const void* K, const void* V, const void* dO,
                            const float* qbar, const float* kbar, const Routes& rt, float* dQ, float* dK, float* dV,
                            float* dqbar, const BackwardWs& ws, cudaStream_t st);

}  // namespace dash
