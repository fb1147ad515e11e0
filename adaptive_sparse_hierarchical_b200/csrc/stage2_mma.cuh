// stage2_mma.cuh -- warp-level bf16 tensor-core tile step of Stage 2 (biased online softmax).
//
// DashAttention (xllm-io paper review, section 3, Proposition 4.1 and the "Stage 2" kernel row):
// o_i = sum_j softmax_j(<q_i,k_j>/sqrt(d) + d_ij) v_j over the routed chunks' tokens (d_ij =
// the chunk's bias) and the diagonal tokens c(i)B..i (d_ij = 0), one online softmax pass.
//
// A warp owns 16 query rows; rows of one position share the routing (the GQA group's union
// support).  For each K/V tile of KT keys staged in shared memory the warp computes
// S = Q K^T (m16n8k16 bf16 MMAs, fp32 accumulate), applies per-row bias / causal mask, updates
// the running max and sum in base 2 and accumulates O += P V.
#pragma once
#include "dash_common.cuh"

namespace dash {

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(sdst)), "l"(gsrc));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of element (row, col) of a [rows][D] bf16 tile whose 16-byte column groups are
// XOR-swizzled by (row & 7), so that ldmatrix rows at one column hit distinct banks.
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int col)
{
    const int grp = (col >> 3) ^ (row & 7);
    return (uint32_t)(row * D * 2 + grp * 16 + (col & 7) * 2);
}

// 16-byte async copy that writes zeros instead of reading when `valid` is false.
__device__ __forceinline__ void cp_async16_zfill(void* sdst, const void* gsrc, bool valid)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(sdst)), "l"(gsrc),
                 "r"(valid ? 16 : 0));
}

// Copy a [KT][D] bf16 tile (rows = keys j0.., row stride `ld` elements) into swizzled smem.
// Rows >= nvalid are not read (they lie past the sequence) and are zero-filled, so masked keys
// can never inject non-finite values into P V.
// `safe` is any readable address (the sequence's first row); a zero-filled copy points there.
template <int KT, int D, int NT>
__device__ __forceinline__ void load_tile(char* sdst, const __nv_bfloat16* src, long long ld, int nvalid,
                                          const __nv_bfloat16* safe, int tid)
{
    constexpr int PIECES = KT * D / 8;
#pragma unroll
    for (int v = tid; v < PIECES; v += NT) {
        const int row = v / (D / 8), col = (v % (D / 8)) * 8;
        const bool ok = row < nvalid;
        cp_async16_zfill(sdst + swz<D>(row, col), ok ? src + (long long)row * ld + col : safe, ok);
    }
}

// Per-row routing decision for one tile: additive base-2 bias, or masked, plus a causal limit.
struct RowMode {
    float bias2;   // bias * log2(e); -inf masks the whole tile for this row
    int jmax;      // keys with index > jmax are masked (causal diagonal); INT_MAX otherwise
};

// Warp state for 16 rows: running max/sum (base 2) for the lane's two rows, O accumulators.
template <int D>
struct WarpAcc {
    float m[2], l[2];
    float o[D / 8][4];
    __device__ void init()
    {
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    }
};

// One tile step.  qf: Q fragments [D/16][4]; sK, sV: swizzled tiles; j0: first key index;
// modes for the lane's rows (lane>>2) and (lane>>2)+8; scale2 = log2(e)/sqrt(d).
template <int KT, int D>
__device__ __forceinline__ void tile_step(WarpAcc<D>& acc, const uint32_t (*qf)[4], const char* sK,
                                          const char* sV, int j0, RowMode ma, RowMode mb, float scale2)
{
    const int lane = threadIdx.x & 31;
    float s[KT / 8][4];
#pragma unroll
    for (int j = 0; j < KT / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
    const uint32_t kbase = smem_u32(sK), vbase = smem_u32(sV);
    const int mi = lane >> 3, rr = lane & 7;
    // S = Q K^T
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
        for (int nn = 0; nn < KT / 8; nn += 2) {
            uint32_t b0, b1, b2, b3;
            const int key = nn * 8 + rr + (mi >> 1) * 8;
            const int col = kk * 16 + (mi & 1) * 8;
            ldsm_x4(kbase + swz<D>(key, col), b0, b1, b2, b3);
            mma_bf16(s[nn], qf[kk], b0, b1);
            mma_bf16(s[nn + 1], qf[kk], b2, b3);
        }
    }
    // bias, causal mask, online softmax (rows ra = lane>>2 and rb = ra + 8)
    const int t = lane & 3;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < KT / 8; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int key = j0 + j * 8 + 2 * t + (e & 1);
            const RowMode& md = (e < 2) ? ma : mb;
            float v = s[j][e] * scale2 + md.bias2;
            if (key > md.jmax) v = -INFINITY;
            s[j][e] = v;
            mx[e >> 1] = fmaxf(mx[e >> 1], v);
        }
    }
    float corr[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
        const float mn = fmaxf(acc.m[h], mx[h]);
        const float base = mn == -INFINITY ? 0.f : mn;
        corr[h] = exp2f(acc.m[h] - base);
        acc.m[h] = mn;
        mx[h] = base;
        acc.l[h] *= corr[h];
    }
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        acc.o[j][0] *= corr[0]; acc.o[j][1] *= corr[0];
        acc.o[j][2] *= corr[1]; acc.o[j][3] *= corr[1];
    }
#pragma unroll
    for (int j = 0; j < KT / 8; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float p = exp2f(s[j][e] - mx[e >> 1]);
            s[j][e] = p;
            acc.l[e >> 1] += p;
        }
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < KT / 16; ++kk) {
        uint32_t a[4];
        a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int nn = 0; nn < D / 8; nn += 2) {
            uint32_t b0, b1, b2, b3;
            const int key = kk * 16 + rr + (mi & 1) * 8;
            const int col = nn * 8 + (mi >> 1) * 8;
            ldsm_x4_t(vbase + swz<D>(key, col), b0, b1, b2, b3);
            mma_bf16(acc.o[nn], a, b0, b1);
            mma_bf16(acc.o[nn + 1], a, b2, b3);
        }
    }
}

// Q fragments of the warp's 16 rows straight from global memory; rowptr(r) gives row r's
// d-vector or null for an absent row.
template <int D, typename RP>
__device__ __forceinline__ void load_q_frags(uint32_t (*qf)[4], RP rowptr)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const __nv_bfloat16* ra = rowptr(g);
    const __nv_bfloat16* rb = rowptr(g + 8);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int c0 = kk * 16 + 2 * t;
        qf[kk][0] = ra ? *reinterpret_cast<const uint32_t*>(ra + c0) : 0u;
        qf[kk][1] = rb ? *reinterpret_cast<const uint32_t*>(rb + c0) : 0u;
        qf[kk][2] = ra ? *reinterpret_cast<const uint32_t*>(ra + c0 + 8) : 0u;
        qf[kk][3] = rb ? *reinterpret_cast<const uint32_t*>(rb + c0 + 8) : 0u;
    }
}

}  // namespace dash
