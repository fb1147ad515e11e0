// dash_noalloc.cu -- dash_decode_noalloc: the decode step of dash_decode without a caller
// workspace.  Its scratch (per-head logits and weights, routing lists, split partials) lives in
// one file-scope device array of fixed size, so the call needs no device allocation at all.
//
// Who needs this: a host program that has no way to obtain device memory for a workspace --
// for example a plugin loaded into a runtime that owns every device allocation and offers the
// plugin no allocator, or a service that must not grow its device footprint after start-up.
// Such a caller still owns the inputs and outputs (caches, query, output); only the scratch is
// provided by the library.
//
// Limits and rules:
//   * scratch capacity kNoAllocScratchBytes (16 MiB) per GPU, held by every GPU that loads the
//     library until the process exits; larger requests are rejected with DASH_EWORKSPACE;
//   * all calls on one GPU share the array: two calls whose kernels overlap on the GPU (other
//     streams, other host threads) race on it and must be serialised by the caller;
//   * the array keeps the previous call's contents; every scratch value a call reads is written
//     earlier in the same call, so nothing has to start at zero;
//   * the first call on each device looks up the array's device address (cudaGetSymbolAddress,
//     with that device current) and caches it; make that first call before any stream capture.
#include <mutex>

#include "dash_common.cuh"

using namespace dash;

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;
constexpr size_t kAlignNA = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

inline size_t upna(size_t x) { return (x + kAlignNA - 1) / kAlignNA * kAlignNA; }

// Device address of this GPU's scratch array (looked up once per device).
void* scratch_for_current_device()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int dash_decode_noalloc(const dash_params* p, const void* q, const void* K_cache, const void* V_cache,
                                   const float* kbar_cache, const int* seqlens, void* O, void* stream)
{
    if (!p) return DASH_EINVAL;
    if (p->batch < 1 || p->seqlen < 1 || p->h_q < 1 || p->h_kv < 1 || p->h_q % p->h_kv) return DASH_EINVAL;
    if (!(p->alpha > 1.f && p->alpha <= 2.f) || !(p->gamma >= 0.f) || !(p->inv_sigma >= 0.f)) return DASH_EINVAL;
    if (p->dtype != DASH_F32 && p->dtype != DASH_BF16) return DASH_EINVAL;
    // the remaining shape checks, and the launches, are those of dash_decode
    const int g = p->h_q / p->h_kv;
    const size_t T = (size_t)(p->seqlen / (p->chunk > 0 ? p->chunk : 1));
    const size_t Tn = T > 0 ? T : 1;
    const size_t bh = (size_t)p->batch * p->h_kv;
    size_t splits = (T + 1 + 7) / 8;
    if ((size_t)dec_tma_blocks() > splits) splits = (size_t)dec_tma_blocks();
    const size_t off_part = upna(bh * g * Tn * 4);
    const size_t off_counts = off_part + upna(bh * splits * g * ((size_t)p->d_h + 2) * 4);
    const size_t off_idx = off_counts + upna(bh * 4);
    const size_t off_bias = off_idx + upna(bh * Tn * 4);
    const size_t total = off_bias + upna(bh * Tn * 4) + kAlignNA;   // + status word
    if (total > kNoAllocScratchBytes) return DASH_EWORKSPACE;
    void* scratch = scratch_for_current_device();
    if (!scratch) return DASH_ELAUNCH;
    return dash_decode(p, q, K_cache, V_cache, kbar_cache, seqlens, O, nullptr, scratch, kNoAllocScratchBytes, stream);
}
