// dash_noalloc.cu -- dash_decode_noalloc: the decode step of dash_decode without a caller
// workspace.  Its scratch (per-head logits and weights, routing lists, split partials, the status
// word of the bounded waits) lives in one file-scope device array of fixed size, so the call
// needs no device allocation at all.
//
// Who needs this: a host program that has no way to obtain device memory for a workspace --
// for example a plugin loaded into a runtime that owns every device allocation and offers the
// plugin no allocator, or a service that must not grow its device footprint after start-up.
// Such a caller still owns the inputs and outputs (caches, query, output, status word); only the
// scratch is provided by the library.
//
// Limits and rules:
//   * scratch capacity kNoAllocScratchBytes (16 MiB) per GPU, held by every GPU that loads the
//     library until the process exits; a request whose decode workspace
//     (dash_workspace_size(p, DASH_OP_DECODE)) is larger is rejected with DASH_EWORKSPACE;
//   * all calls on one GPU share the array: two calls whose kernels overlap on the GPU (other
//     streams, other host threads) race on it and must be serialised by the caller;
//   * the array keeps the previous call's contents; every scratch value a call reads is written
//     earlier in the same call (the routing kernel clears the status word first), so nothing
//     has to start at zero;
//   * the array's device address is looked up with cudaGetSymbolAddress the first time a call
//     runs under a given (device, CUDA context) pair, with that device current, and cached for
//     that pair; make that first call before any stream capture.
#include <cuda.h>

#include <mutex>

#include "dash_common.cuh"

using namespace dash;

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;
constexpr int kCacheSlots = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

struct ScratchAddr {
    int dev;
    CUcontext ctx;
    void* ptr;
};

std::mutex g_mu;
ScratchAddr g_cache[kCacheSlots] = {};
int g_used = 0;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry point (no link dependency on libcuda).
CtxGetCurrentFn ctx_get_current()
{
    static CtxGetCurrentFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    }
    return fn;
}

// Device address of the scratch array in the current device's current context.  The host-side
// name g_decode_scratch is only a stand-in for the symbol; kernels get this address instead.
void* scratch_for_current_context()
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
    CtxGetCurrentFn get = ctx_get_current();
    if (!get) return nullptr;
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (ctx)
        for (int k = 0; k < g_used; ++k)
            if (g_cache[k].dev == dev && g_cache[k].ctx == ctx) return g_cache[k].ptr;
    // first call under this (device, context): the lookup also binds the runtime's primary context
    // to this thread when no context was current yet, so the context is read again afterwards
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return nullptr;
    if (!ctx && (get(&ctx) != CUDA_SUCCESS || !ctx)) return nullptr;
    if (g_used < kCacheSlots) g_cache[g_used++] = ScratchAddr{dev, ctx, p};
    return p;
}

}  // namespace

extern "C" int dash_decode_noalloc(const dash_params* p, const void* q, const void* K_cache, const void* V_cache,
                                   const float* kbar_cache, const int* seqlens, void* O, int* status, void* stream)
{
    const int prc = check_params(p);
    if (prc != DASH_OK) return prc;
    // the size of dash_decode's workspace for these parameters (one layout for both entry points)
    const size_t need = dash_workspace_size(p, DASH_OP_DECODE);
    if (need == 0) return DASH_EINVAL;
    if (need > kNoAllocScratchBytes) return DASH_EWORKSPACE;
    const long long err_off = dash_error_word_offset(p, DASH_OP_DECODE);
    if (err_off < 0 || (size_t)err_off + sizeof(int) > need) return DASH_EINVAL;
    if (status && (reinterpret_cast<uintptr_t>(status) & 3u)) return DASH_EALIGN;
    void* scratch = scratch_for_current_context();
    if (!scratch) return DASH_ELAUNCH;
    const int rc = dash_decode(p, q, K_cache, V_cache, kbar_cache, seqlens, O, nullptr, scratch, kNoAllocScratchBytes,
                               stream);
    if (rc != DASH_OK || !status) return rc;
    // the call's status word, copied into the caller's int on the same stream (device to device)
    if (cudaMemcpyAsync(status, static_cast<char*>(scratch) + err_off, sizeof(int), cudaMemcpyDeviceToDevice,
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return DASH_ELAUNCH;
    return DASH_OK;
}
