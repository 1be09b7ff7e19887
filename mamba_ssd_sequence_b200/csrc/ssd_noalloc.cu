// ssd_fwd_noalloc: the general SIMT forward path run on a fixed scratch
// buffer that lives in the library itself, for callers that cannot allocate
// device memory (see include/ssd.h).
//
// The scratch is a file-scope __device__ array.  In host code its name is
// only a host-side stand-in, never a device address, so the address handed
// to the kernels comes from cudaGetSymbolAddress, looked up once per device
// (with that device current) on the first call made on it.
#include <cuda_runtime.h>

#include <mutex>

#include "ssd_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB per GPU
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void *g_scratch_dev_ptr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of g_noalloc_scratch on the current device (nullptr on error).
void *scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_dev_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return nullptr;
        g_scratch_dev_ptr[dev] = p;
    }
    return g_scratch_dev_ptr[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int ssd_fwd_noalloc(const void *q, const void *k, const void *v, const float *dt_p,
                               const float *A_log, const float *dt_bias, const float *D, int B,
                               int H, int N, int d_h, int dtype, int order, int normalize,
                               int chunk, void *out, void *stream) {
    using namespace ssd;
    if (!q || !k || !v || !dt_p || !A_log || !dt_bias || !out) return SSD_ERR_NULL;
    // ssd_workspace_bytes validates shape, dtype, order and chunk (0 = invalid)
    if (ssd_workspace_bytes(B, H, N, d_h, dtype, order, chunk) == 0) {
        if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_DTYPE;
        if (order != 1 && order != 2) return SSD_ERR_ORDER;
        if (chunk != 64 && chunk != 128 && chunk != 256) return SSD_ERR_CHUNK;
        return SSD_ERR_SHAPE;
    }
    const void *ptrs[] = {q, k, v, dt_p, A_log, dt_bias, out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return SSD_ERR_ALIGN;
    if (D && !aligned16(D)) return SSD_ERR_ALIGN;

    // Layout of the SIMT path's scratch: status block, chunk-local decay,
    // chunk totals, per-chunk carried states (with the normaliser column).
    const size_t BH = (size_t)B * H, nc = (size_t)N / chunk;
    const size_t Dphi = order == 1 ? (size_t)d_h : (size_t)d_h * d_h;
    Plan p{};
    p.path = PATH_SIMT;
    p.n_launches = 4;
    p.acs_off = kStatusBytes;
    p.lam_off = align_up(p.acs_off + BH * N * sizeof(float), 256);
    p.state_off = align_up(p.lam_off + BH * nc * sizeof(float), 256);
    p.total = align_up(p.state_off + BH * nc * Dphi * (d_h + 1) * sizeof(float), 256);
    if (p.total > kNoAllocScratchBytes) return SSD_ERR_WORKSPACE;

    void *scratch = scratch_for_current_device();
    if (!scratch) return SSD_ERR_CUDA;
    FwdArgs a{q, k, v, dt_p, A_log, dt_bias, D, nullptr, 0, nullptr, nullptr, nullptr, nullptr,
              B, H, N, d_h, dtype, order, normalize ? 1 : 0,
              chunk, out, scratch, kNoAllocScratchBytes, static_cast<cudaStream_t>(stream)};
    return launch_simt(a, p);
}
