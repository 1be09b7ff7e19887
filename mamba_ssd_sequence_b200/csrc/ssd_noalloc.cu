// ssd_fwd_noalloc: the general SIMT forward path run on a fixed scratch
// buffer that lives in the library itself, for callers that cannot allocate
// device memory (see include/ssd.h).
//
// The scratch is a file-scope __device__ array.  In host code its name is
// only a host-side stand-in, never a device address, so the address handed
// to the kernels comes from cudaGetSymbolAddress, looked up with the context
// current.  A __device__ symbol's address belongs to the context the module
// was loaded into, so the address is remembered per context -- keyed by the
// context's ID, which the driver never reuses within a process -- and looked
// up again for a context not seen before: a plugin whose host application
// creates its own contexts, or any context made after cudaDeviceReset.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "ssd_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB per GPU
constexpr int kCacheSlots = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct CacheSlot {
    unsigned long long ctx_id;
    void *ptr;
};
CacheSlot g_cache[kCacheSlots] = {};
int g_cache_next = 0;
std::mutex g_scratch_mutex;

// Device address of g_noalloc_scratch in the calling thread's current context
// (nullptr on error).  The first call in a context loads the library's module
// there if it is not loaded yet.
void *scratch_for_current_context() {
    unsigned long long id = 0;
    if (!ssd::current_context_id(&id)) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    for (const CacheSlot &s : g_cache)
        if (s.ptr != nullptr && s.ctx_id == id) return s.ptr;
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_cache[g_cache_next] = CacheSlot{id, p};
    g_cache_next = (g_cache_next + 1) % kCacheSlots;
    return p;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int ssd_fwd_noalloc(const void *q, const void *k, const void *v, const float *dt_p,
                               const float *A_log, const float *dt_bias, const float *D, int B,
                               int H, int N, int d_h, int dtype, int order, int normalize,
                               int chunk, void *out, void *stream) {
    using namespace ssd;
    if (!q || !k || !v || !dt_p || !A_log || !dt_bias || !out) return SSD_ERR_NULL;
    // make_plan validates shape, dtype, order and chunk
    Plan chosen{};
    const int rc = make_plan(B, H, N, d_h, dtype, order, normalize, chunk, 0, 0, &chosen);
    if (rc != SSD_OK) return rc;
    if ((size_t)N / chunk > (size_t)kMaxSimtChunks) return SSD_ERR_SHAPE;
    const void *ptrs[] = {q, k, v, dt_p, A_log, dt_bias, out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return SSD_ERR_ALIGN;
    if (D && !aligned16(D)) return SSD_ERR_ALIGN;

    // this entry point always runs the SIMT path, with the same scratch layout
    // as ssd_fwd's SIMT path
    Plan p{};
    simt_layout(B, H, N, d_h, order, chunk, &p);
    if (p.total > kNoAllocScratchBytes) return SSD_ERR_WORKSPACE;

    void *scratch = scratch_for_current_context();
    if (!scratch) return SSD_ERR_CUDA;
    FwdArgs a{q, k, v, dt_p, A_log, dt_bias, D, nullptr, 0, nullptr, nullptr, nullptr, nullptr,
              B, H, N, d_h, dtype, order, normalize ? 1 : 0,
              chunk, out, scratch, kNoAllocScratchBytes, static_cast<cudaStream_t>(stream)};
    return launch_simt(a, p);
}
