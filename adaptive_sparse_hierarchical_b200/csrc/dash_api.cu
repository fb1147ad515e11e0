// dash_api.cu -- the C ABI declared in include/dash.h: argument checks, workspace layout and
// the launch sequence of each entry point.  No allocation, no synchronisation.
#include <cmath>
#include <cstdint>

#include "dash_common.cuh"

using namespace dash;

namespace {

bool pow2_group(int g) { return g == 1 || g == 2 || g == 4 || g == 8 || g == 16; }

}  // namespace

#include <atomic>

namespace dash {

namespace {
std::atomic<long long> g_wait_limit{1ll << 23};
}

long long wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }

// Shape checks shared by every entry point.
int check_params(const dash_params* p)
{
    if (!p) return DASH_EINVAL;
    if (p->batch < 1 || p->seqlen < 1 || p->h_q < 1 || p->h_kv < 1 || p->h_q % p->h_kv) return DASH_EINVAL;
    if (!(p->alpha > 1.f && p->alpha <= 2.f)) return DASH_EINVAL;
    if (!(p->gamma >= 0.f) || !std::isfinite(p->gamma)) return DASH_EINVAL;
    if (!(p->inv_sigma >= 0.f) || !std::isfinite(p->inv_sigma)) return DASH_EINVAL;
    if (p->dtype != DASH_F32 && p->dtype != DASH_BF16) return DASH_EINVAL;
    if (p->chunk < 1 || p->d_h < 1) return DASH_EINVAL;
    if (p->d_h != 64 && p->d_h != 128) return DASH_EUNSUPPORTED;
    if (p->chunk != 1 && p->chunk != 16 && p->chunk != 32 && p->chunk != 64 && p->chunk != 128)
        return DASH_EUNSUPPORTED;
    if (!pow2_group(p->h_q / p->h_kv)) return DASH_EUNSUPPORTED;
    return DASH_OK;
}

}  // namespace dash

namespace {

constexpr size_t kAlign = 256;
inline size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int esize(int dtype) { return dtype == DASH_BF16 ? 2 : 4; }

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }
bool aligned4(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; }

bool strides_ok(const long long st[3], int dtype)
{
    for (int k = 0; k < 3; ++k)
        if (st[k] < 0 || (st[k] * esize(dtype)) % 16) return false;
    return true;
}

Shape make_shape(const dash_params* p)
{
    Shape s;
    s.batch = p->batch; s.n = p->seqlen; s.hq = p->h_q; s.hkv = p->h_kv; s.g = p->h_q / p->h_kv;
    s.d = p->d_h; s.B = p->chunk; s.T = p->seqlen / p->chunk;
    s.alpha = p->alpha; s.gamma = p->gamma; s.inv_sigma = p->inv_sigma;
    for (int k = 0; k < 3; ++k) {
        s.qs[k] = p->q_strides[k]; s.ks[k] = p->k_strides[k];
        s.vs[k] = p->v_strides[k]; s.os[k] = p->o_strides[k];
    }
    s.pt = nullptr;
    s.psz = s.pmax = s.npages = 0;
    s.kps = s.vps = 0;
    s.polls = wait_limit();
    return s;
}

// Paged caches: checks of the page description (null: contiguous caches, nothing to check) and
// the Shape fields the kernels address the pools with.
int check_paged(const dash_params* p, const dash_paged_kv* pk)
{
    if (!pk) return DASH_OK;
    if (!pk->page_table || pk->page_size <= 0 || pk->max_pages <= 0 || pk->num_pages <= 0) return DASH_EINVAL;
    if (pk->page_size % 64 || pk->page_size % p->chunk) return DASH_EUNSUPPORTED;
    if ((long long)pk->max_pages * pk->page_size < p->seqlen) return DASH_EINVAL;
    if (p->dtype != DASH_BF16 || p->d_h != 128) return DASH_EUNSUPPORTED;
    if (pk->k_page_stride <= 0 || pk->v_page_stride <= 0 || (pk->k_page_stride * 2) % 16 || (pk->v_page_stride * 2) % 16)
        return DASH_EALIGN;
    if (reinterpret_cast<uintptr_t>(pk->page_table) & 3u) return DASH_EALIGN;
    return DASH_OK;
}

void apply_paged(Shape& s, const dash_paged_kv* pk)
{
    if (!pk) return;
    s.pt = pk->page_table;
    s.psz = pk->page_size;
    s.pmax = pk->max_pages;
    s.npages = pk->num_pages;
    s.kps = pk->k_page_stride;
    s.vps = pk->v_page_stride;
}

long long route_cap(const dash_params* p)
{
    // sum_{i < n} floor(i / B) = tri_offset(n, B)
    return tri_offset(p->seqlen, p->chunk);
}

struct PrefillLayout { size_t kbar, counts, idx, bias, err, knorm, planes, redo, perm, spill, total; };
PrefillLayout prefill_layout(const dash_params* p)
{
    PrefillLayout L;
    const size_t bh = (size_t)p->batch * p->h_kv;
    const size_t T = (size_t)(p->seqlen / p->chunk);
    const size_t cap = (size_t)route_cap(p);
    L.kbar = 0;
    L.counts = L.kbar + up(bh * T * p->d_h * 4);
    L.idx = L.counts + up(bh * (size_t)p->seqlen * 4);
    L.bias = L.idx + up(bh * cap * 4);
    L.err = L.bias + up(bh * cap * 4);
    L.knorm = L.err + 16;   // the status word, then one float per (sequence, KV head)
    L.planes = L.err + up(16 + bh * 4);
    L.redo = L.planes + up(bh * 3 * T * p->d_h * 2);
    L.perm = L.redo + up(bh * (size_t)p->seqlen);   // one flag per position block at most
    // Stage 2's position order; before Stage 2 rewrites it, Stage 1's list of position blocks to
    // recompute (one count + one int per block at most)
    L.spill = L.perm + up(bh * (size_t)p->seqlen * 4 + 16);
    // the long-row Stage 1 kernel's candidate-list spill areas (shapes it can serve)
    const int g = p->h_kv > 0 ? p->h_q / p->h_kv : 0;
    const bool long_rows = p->dtype == DASH_BF16 && p->d_h == 128 && T > 512 && (g == 4 || g == 8 || g == 16);
    L.total = L.spill + (long_rows ? up(route_long_spill_bytes(make_shape(p))) : 0);
    return L;
}

struct DecodeLayout { size_t x, part, counts, idx, bias, err, total; int splits; };
DecodeLayout decode_layout(const dash_params* p)
{
    DecodeLayout L;
    const Shape s = make_shape(p);
    const size_t bh = (size_t)p->batch * p->h_kv;
    const size_t T = (size_t)s.T;
    // partial slots per (sequence, KV head): the split kernel's splits, or one per persistent block
    L.splits = decode_splits(s, s.T);
    if (dec_tma_blocks() > L.splits) L.splits = dec_tma_blocks();
    L.x = 0;
    L.part = L.x + up(bh * s.g * (T > 0 ? T : 1) * 4);
    L.counts = L.part + up(bh * (size_t)L.splits * s.g * (p->d_h + 2) * 4);
    L.idx = L.counts + up(bh * 4);
    L.bias = L.idx + up(bh * (T > 0 ? T : 1) * 4);
    L.err = L.bias + up(bh * (T > 0 ? T : 1) * 4);
    L.total = L.err + kAlign;
    return L;
}

struct BackwardLayout { size_t lse, del, dzbar, tcnt, toff, tpos, tent, dkbar, qpart, total; };
BackwardLayout backward_layout(const dash_params* p)
{
    BackwardLayout L;
    const size_t bh = (size_t)p->batch * p->h_kv, rows = (size_t)p->batch * p->h_q * p->seqlen;
    const size_t T = (size_t)(p->seqlen / p->chunk), Tn = T > 0 ? T : 1;
    const size_t cap = (size_t)route_cap(p) > 0 ? (size_t)route_cap(p) : 1;
    const size_t g = (size_t)(p->h_q / p->h_kv);
    L.lse = 0;
    L.del = L.lse + up(rows * 4);
    L.dzbar = L.del + up(rows * 4);
    L.tcnt = L.dzbar + up(bh * cap * g * 4);
    L.toff = L.tcnt + up(bh * Tn * 4);
    L.tpos = L.toff + up(bh * (Tn + 1) * 4);
    L.tent = L.tpos + up(bh * cap * 4);
    L.dkbar = L.tent + up(bh * cap * 4);
    L.qpart = L.dkbar + up(bh * Tn * p->d_h * 4);
    L.total = L.qpart + up(bh * Tn * p->d_h * 4);
    return L;
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? DASH_OK : DASH_ELAUNCH; }

}  // namespace

extern "C" {

size_t dash_workspace_size(const dash_params* p, int op)
{
    if (check_params(p) != DASH_OK) return 0;
    if (op == DASH_OP_PREFILL) return prefill_layout(p).total;
    if (op == DASH_OP_DECODE) return decode_layout(p).total;
    if (op == DASH_OP_BACKWARD) return backward_layout(p).total;
    return 0;
}

long long dash_error_word_offset(const dash_params* p, int op)
{
    if (check_params(p) != DASH_OK) return -1;
    if (op == DASH_OP_PREFILL) return (long long)prefill_layout(p).err;
    if (op == DASH_OP_DECODE) return (long long)decode_layout(p).err;
    return -1;
}

long long dash_prefill_order_offset(const dash_params* p)
{
    if (check_params(p) != DASH_OK) return -1;
    const Shape s = make_shape(p);
    if (!attend_tc_supported(s, p->dtype) || legacy_stage2() || pair_stage2() || !s2_grouping_enabled(s)) return -1;
    return (long long)prefill_layout(p).perm;
}

long long dash_route_capacity(const dash_params* p)
{
    if (check_params(p) != DASH_OK) return 0;
    return route_cap(p);
}

int dash_prefill_stage(const dash_params* p, int stage, const void* Q, const void* K, const void* V,
                       const float* qbar, void* O, float* kbar_out, const dash_route_out* route, void* workspace,
                       size_t ws_bytes, void* stream);

int dash_prefill(const dash_params* p, const void* Q, const void* K, const void* V, const float* qbar,
                 void* O, float* kbar_out, const dash_route_out* route, void* workspace, size_t ws_bytes,
                 void* stream)
{
    return dash_prefill_stage(p, -1, Q, K, V, qbar, O, kbar_out, route, workspace, ws_bytes, stream);
}

int dash_prefill_stage(const dash_params* p, int stage, const void* Q, const void* K, const void* V,
                       const float* qbar, void* O, float* kbar_out, const dash_route_out* route, void* workspace,
                       size_t ws_bytes, void* stream)
{
    if (stage < -1 || stage > DASH_STAGE2_BITMASK) return DASH_EINVAL;
    int rc = check_params(p);
    if (rc != DASH_OK) return rc;
    if (!Q || !K || !V || !qbar || !O) return DASH_EINVAL;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(qbar)) return DASH_EALIGN;
    if (!strides_ok(p->q_strides, p->dtype) || !strides_ok(p->k_strides, p->dtype) ||
        !strides_ok(p->v_strides, p->dtype) || !strides_ok(p->o_strides, p->dtype))
        return DASH_EALIGN;
    const Shape s = make_shape(p);
    int P = 0;
    route_prefill_smem(s, &P);
    if (P == 0) return DASH_EUNSUPPORTED;
    const PrefillLayout L = prefill_layout(p);
    if (!workspace || ws_bytes < L.total) return DASH_EWORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return DASH_EALIGN;
    if (kbar_out && !aligned16(kbar_out)) return DASH_EALIGN;
    char* ws = static_cast<char*>(workspace);
    float* kbar = kbar_out ? kbar_out : reinterpret_cast<float*>(ws + L.kbar);
    Routes rt;
    rt.counts = route && route->counts ? route->counts : reinterpret_cast<int*>(ws + L.counts);
    rt.idx = route && route->chunk_idx ? route->chunk_idx : reinterpret_cast<int*>(ws + L.idx);
    rt.bias = route && route->bias ? route->bias : reinterpret_cast<float*>(ws + L.bias);
    rt.bitmask = route ? route->bitmask : nullptr;
    rt.cap = route_cap(p);
    rt.words = (s.T + 31) / 32;
    if (!aligned4(rt.counts) || !aligned4(rt.idx) || !aligned4(rt.bias) || (rt.bitmask && !aligned4(rt.bitmask)))
        return DASH_EALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // bf16: Stage 0 also writes the summaries as three exact bf16 planes for Stage 1's MMAs
    __nv_bfloat16* planes = p->dtype == DASH_BF16 ? reinterpret_cast<__nv_bfloat16*>(ws + L.planes) : nullptr;
    int* err = reinterpret_cast<int*>(ws + L.err);
    float* knorm = reinterpret_cast<float*>(ws + L.knorm);
    if (stage == -1 || stage == DASH_STAGE0) {
        // a prefill starts here: clear the status word of the bounded waits and the per-(sequence,
        // KV head) summary norms that Stage 0 raises
        if (cudaMemsetAsync(err, 0, L.planes - L.err, st) != cudaSuccess) return DASH_ELAUNCH;
        rc = launch_status(launch_stage0(s, p->dtype, K, qbar, nullptr, kbar, s.T, nullptr, st, planes,
                                         planes ? knorm : nullptr));
        if (rc != DASH_OK) return rc;
    }
    if (stage == -1 || stage == DASH_STAGE1) {
        unsigned char* redo = reinterpret_cast<unsigned char*>(ws + L.redo);
        void* spill = L.total > L.spill ? ws + L.spill : nullptr;
        rc = launch_status(launch_route_prefill(s, p->dtype, Q, kbar, planes, planes ? knorm : nullptr, rt, redo,
                                                reinterpret_cast<int*>(ws + L.perm), spill, err, st));
        if (rc != DASH_OK) return rc;
    }
    if (stage == -1 || stage == DASH_STAGE2)
        rc = launch_status(launch_attend_prefill(s, p->dtype, Q, K, V, O, rt,
                                                 reinterpret_cast<int*>(ws + L.perm), err, st));
    if (stage == DASH_STAGE2_BITMASK) {
        if (!rt.bitmask) return DASH_EINVAL;
        if (!attend_mask_supported(s, p->dtype)) return DASH_EUNSUPPORTED;
        rc = launch_status(launch_attend_prefill_bitmask(s, p->dtype, Q, K, V, O, rt,
                                                         reinterpret_cast<int*>(ws + L.perm), err, st));
    }
    return rc;
}

static int summary_build(const dash_params* p, const dash_paged_kv* pk, const void* K_cache, const float* qbar,
                         const int* seqlens, float* kbar_cache, float* partial_state, void* stream)
{
    int rc = check_params(p);
    if (rc != DASH_OK) return rc;
    if ((rc = check_paged(p, pk)) != DASH_OK) return rc;
    if (!K_cache || !qbar || !seqlens || !kbar_cache || !partial_state) return DASH_EINVAL;
    if (!aligned16(K_cache) || !strides_ok(p->k_strides, p->dtype) || !aligned16(qbar)) return DASH_EALIGN;
    if (!aligned4(seqlens) || !aligned4(kbar_cache) || !aligned4(partial_state)) return DASH_EALIGN;
    Shape s = make_shape(p);
    apply_paged(s, pk);
    return launch_status(launch_stage0(s, p->dtype, K_cache, qbar, seqlens, kbar_cache, s.T, partial_state,
                                       static_cast<cudaStream_t>(stream)));
}

int dash_summary_build(const dash_params* p, const void* K_cache, const float* qbar, const int* seqlens,
                       float* kbar_cache, float* partial_state, void* stream)
{
    return summary_build(p, nullptr, K_cache, qbar, seqlens, kbar_cache, partial_state, stream);
}

int dash_summary_build_paged(const dash_params* p, const dash_paged_kv* pk, const void* K_pool, const float* qbar,
                             const int* seqlens, float* kbar_cache, float* partial_state, void* stream)
{
    if (!pk) return DASH_EINVAL;
    return summary_build(p, pk, K_pool, qbar, seqlens, kbar_cache, partial_state, stream);
}

static int summary_append(const dash_params* p, const dash_paged_kv* pk, const void* k_new, const void* v_new,
                          const float* qbar, void* K_cache, void* V_cache, float* kbar_cache, float* partial_state,
                          int* seqlens, void* stream)
{
    int rc = check_params(p);
    if (rc != DASH_OK) return rc;
    if ((rc = check_paged(p, pk)) != DASH_OK) return rc;
    if (!k_new || !v_new || !qbar || !K_cache || !V_cache || !kbar_cache || !partial_state || !seqlens)
        return DASH_EINVAL;
    if (p->h_kv > 32) return DASH_EUNSUPPORTED;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(K_cache) || !aligned16(V_cache) || !aligned16(qbar))
        return DASH_EALIGN;
    if (!strides_ok(p->k_strides, p->dtype) || !strides_ok(p->v_strides, p->dtype)) return DASH_EALIGN;
    if (!aligned4(seqlens) || !aligned4(kbar_cache) || !aligned4(partial_state)) return DASH_EALIGN;
    Shape s = make_shape(p);
    apply_paged(s, pk);
    return launch_status(launch_append(s, p->dtype, k_new, v_new, qbar, K_cache, V_cache, kbar_cache, s.T,
                                       partial_state, seqlens, static_cast<cudaStream_t>(stream)));
}

int dash_summary_append(const dash_params* p, const void* k_new, const void* v_new, const float* qbar,
                        void* K_cache, void* V_cache, float* kbar_cache, float* partial_state, int* seqlens,
                        void* stream)
{
    return summary_append(p, nullptr, k_new, v_new, qbar, K_cache, V_cache, kbar_cache, partial_state, seqlens,
                          stream);
}

int dash_summary_append_paged(const dash_params* p, const dash_paged_kv* pk, const void* k_new, const void* v_new,
                              const float* qbar, void* K_pool, void* V_pool, float* kbar_cache, float* partial_state,
                              int* seqlens, void* stream)
{
    if (!pk) return DASH_EINVAL;
    return summary_append(p, pk, k_new, v_new, qbar, K_pool, V_pool, kbar_cache, partial_state, seqlens, stream);
}

static int decode(const dash_params* p, const dash_paged_kv* pk, const void* q, const void* K_cache,
                  const void* V_cache, const float* kbar_cache, const int* seqlens, void* O,
                  const dash_route_out* route, void* workspace, size_t ws_bytes, void* stream)
{
    int rc = check_params(p);
    if (rc != DASH_OK) return rc;
    if ((rc = check_paged(p, pk)) != DASH_OK) return rc;
    if (!q || !K_cache || !V_cache || !kbar_cache || !seqlens || !O) return DASH_EINVAL;
    if (!aligned16(q) || !aligned16(K_cache) || !aligned16(V_cache) || !aligned16(O) || !aligned16(kbar_cache))
        return DASH_EALIGN;
    if (!strides_ok(p->k_strides, p->dtype) || !strides_ok(p->v_strides, p->dtype)) return DASH_EALIGN;
    if (!aligned4(seqlens)) return DASH_EALIGN;
    // the routing step keeps every head's logits of one (sequence, KV head) in shared memory
    if ((size_t)(p->h_q / p->h_kv) * (size_t)(p->seqlen / p->chunk) * 4 > 225 * 1024) return DASH_EUNSUPPORTED;
    const DecodeLayout L = decode_layout(p);
    if (L.splits > 1024) return DASH_EUNSUPPORTED;   // the merge step holds at most 1024 split weights
    if (!workspace || ws_bytes < L.total) return DASH_EWORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return DASH_EALIGN;
    Shape s = make_shape(p);
    apply_paged(s, pk);
    if (pk && !dec_tma_supported(s, p->dtype)) return DASH_EUNSUPPORTED;   // paged: the TMA attend only
    char* ws = static_cast<char*>(workspace);
    Routes rt;
    rt.counts = route && route->counts ? route->counts : reinterpret_cast<int*>(ws + L.counts);
    rt.idx = route && route->chunk_idx ? route->chunk_idx : reinterpret_cast<int*>(ws + L.idx);
    rt.bias = route && route->bias ? route->bias : reinterpret_cast<float*>(ws + L.bias);
    rt.bitmask = route ? route->bitmask : nullptr;
    rt.cap = s.T;
    rt.words = (s.T + 31) / 32;
    DecodeWs dw;
    dw.x = reinterpret_cast<float*>(ws + L.x);
    dw.part = reinterpret_cast<float*>(ws + L.part);
    dw.splits = L.splits;
    dw.err = reinterpret_cast<int*>(ws + L.err);   // cleared by the routing launch
    return launch_status(launch_decode(s, p->dtype, q, K_cache, V_cache, kbar_cache, s.T, seqlens, O, rt, dw,
                                       static_cast<cudaStream_t>(stream)));
}

int dash_decode(const dash_params* p, const void* q, const void* K_cache, const void* V_cache,
                const float* kbar_cache, const int* seqlens, void* O, const dash_route_out* route,
                void* workspace, size_t ws_bytes, void* stream)
{
    return decode(p, nullptr, q, K_cache, V_cache, kbar_cache, seqlens, O, route, workspace, ws_bytes, stream);
}

int dash_decode_paged(const dash_params* p, const dash_paged_kv* pk, const void* q, const void* K_pool,
                      const void* V_pool, const float* kbar_cache, const int* seqlens, void* O,
                      const dash_route_out* route, void* workspace, size_t ws_bytes, void* stream)
{
    if (!pk) return DASH_EINVAL;
    return decode(p, pk, q, K_pool, V_pool, kbar_cache, seqlens, O, route, workspace, ws_bytes, stream);
}

long long dash_set_wait_limit(long long polls)
{
    if (polls < 0) return -1;
    return g_wait_limit.exchange(polls);
}

const char* dash_status_string(int status)
{
    switch (status) {
    case DASH_OK: return "ok";
    case DASH_EINVAL: return "invalid argument";
    case DASH_EUNSUPPORTED: return "unsupported configuration (d_h, chunk, group size or sequence too long)";
    case DASH_EWORKSPACE: return "workspace missing or too small";
    case DASH_EALIGN: return "pointer or stride misaligned";
    case DASH_ELAUNCH: return "kernel launch failed";
    default: return "unknown status";
    }
}

}  // extern "C"

extern "C" int dash_backward(const dash_params* p, const void* Q, const void* K, const void* V, const float* qbar,
                             const void* dO, const float* kbar, const dash_route_out* route, float* dQ, float* dK,
                             float* dV, float* dqbar, void* workspace, size_t ws_bytes, void* stream)
{
    int rc = check_params(p);
    if (rc != DASH_OK) return rc;
    if (!Q || !K || !V || !qbar || !dO || !kbar || !route || !route->counts || !route->chunk_idx || !route->bias ||
        !dQ || !dK || !dV || !dqbar)
        return DASH_EINVAL;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dO) || !aligned16(qbar)) return DASH_EALIGN;
    if (!strides_ok(p->q_strides, p->dtype) || !strides_ok(p->k_strides, p->dtype) ||
        !strides_ok(p->v_strides, p->dtype) || !strides_ok(p->o_strides, p->dtype))
        return DASH_EALIGN;
    if (!aligned4(kbar) || !aligned4(route->counts) || !aligned4(route->chunk_idx) || !aligned4(route->bias) ||
        !aligned4(dQ) || !aligned4(dK) || !aligned4(dV) || !aligned4(dqbar))
        return DASH_EALIGN;
    const Shape s = make_shape(p);
    // shared memory of the query-major kernel grows with the group's chunk logits (g * T floats)
    if (backward_rows_smem(s) > 220 * 1024 || backward_keys_smem(s) > 220 * 1024) return DASH_EUNSUPPORTED;
    const BackwardLayout L = backward_layout(p);
    if (!workspace || ws_bytes < L.total) return DASH_EWORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return DASH_EALIGN;
    char* ws = static_cast<char*>(workspace);
    BackwardWs bw;
    bw.lse = reinterpret_cast<float*>(ws + L.lse);
    bw.del = reinterpret_cast<float*>(ws + L.del);
    bw.dzbar = reinterpret_cast<float*>(ws + L.dzbar);
    bw.tcnt = reinterpret_cast<int*>(ws + L.tcnt);
    bw.toff = reinterpret_cast<int*>(ws + L.toff);
    bw.tpos = reinterpret_cast<int*>(ws + L.tpos);
    bw.tent = reinterpret_cast<int*>(ws + L.tent);
    bw.dkbar = reinterpret_cast<float*>(ws + L.dkbar);
    bw.qpart = reinterpret_cast<float*>(ws + L.qpart);
    Routes rt;
    rt.counts = route->counts;
    rt.idx = route->chunk_idx;
    rt.bias = route->bias;
    rt.bitmask = nullptr;
    rt.cap = route_cap(p);
    rt.words = (s.T + 31) / 32;
    return launch_status(launch_backward(s, p->dtype, Q, K, V, dO, qbar, kbar, rt, dQ, dK, dV, dqbar, bw,
                                         static_cast<cudaStream_t>(stream)));
}
