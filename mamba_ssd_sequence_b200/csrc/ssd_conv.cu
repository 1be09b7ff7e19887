// Causal depthwise 1-D convolution over tokens with optional SiLU: the
// prologue Q, K, V = SiLU(conv_1d(h W_QKV)) of 2Mamba2Furious Algorithm 3 and
// the window-2 convolution q^c_t = conv_1d(q_t, q_{t-1}) of the Algorithm 6
// page, applied to one [B, H, N, d_h] tensor:
//     u = bias[c] + sum_{j < width} w[c][j] x[t - j, c]   (x before token 0 is 0)
//     out = SiLU(u) or u
// One CTA per tile of kTile consecutive tokens of one (b, h): the tile and the
// width - 1 rows before it are contiguous in memory, so one bulk copy brings
// them into shared memory (every input row is read from HBM once); the
// threads then take (token, 8-channel group) items with 16-byte shared loads
// and global stores.  All CTAs of a call are resident at once, each with its
// copy in flight, which keeps HBM busy.  HBM-bound.
#include <cuda_bf16.h>
#include <math.h>

#include "ptx.cuh"
#include "ssd_internal.h"
#include "ssd_math.cuh"

namespace ssd {
namespace {

constexpr int kConvThreads = 256;

__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ void store8(float *p, const float (&y)[8]) {
    *reinterpret_cast<float4 *>(p) = make_float4(y[0], y[1], y[2], y[3]);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(y[4], y[5], y[6], y[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&y)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 b = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&b);
    }
    *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

constexpr int kTile = 128;   // tokens per CTA
constexpr int kMaxWidth = 4;

template <typename T>
__global__ void __launch_bounds__(kConvThreads)
conv1d_kernel(const T *__restrict__ x, const float *__restrict__ w, const float *__restrict__ bias, int H,
              int N, int d, int width, int silu, T *__restrict__ out) {
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm);
    T *xs = reinterpret_cast<T *>(sm + 128);  // row r: token t0 - (kMaxWidth - 1) + r
    const int tiles = (N + kTile - 1) / kTile;
    const int tile = (int)(blockIdx.x % tiles);
    const long long bhrow = blockIdx.x / tiles;  // b H + h
    const int h = (int)(bhrow % H);
    const int t0 = tile * kTile, tn = min(kTile, N - t0);
    const int halo = min(kMaxWidth - 1, t0);  // rows before the tile that exist
    const int tid = threadIdx.x;
    const uint32_t bytes = (uint32_t)((halo + tn) * d * sizeof(T));
    if (tid == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        ptx::mbar_arrive_expect_tx(bar, bytes);
        ptx::bulk_load(xs + (kMaxWidth - 1 - halo) * d, x + ((size_t)bhrow * N + t0 - halo) * d, bytes, bar);
    }
    // rows before token 0 are zero
    for (int e = tid; e < (kMaxWidth - 1 - halo) * d; e += kConvThreads) xs[e] = T(0.0f);
    // the head's weights, tap-major, and bias through shared memory (coalesced
    // loads while the tile is in flight); a thread then keeps one channel
    // group (kConvThreads is a multiple of d / 8) in registers
    float *sw = reinterpret_cast<float *>(sm + 128 + (size_t)(kTile + kMaxWidth - 1) * d * sizeof(T));
    for (int i = tid; i < d * width; i += kConvThreads) sw[(i % width) * d + i / width] = __ldg(w + (size_t)h * d * width + i);
    for (int i = tid; i < d; i += kConvThreads) sw[kMaxWidth * d + i] = bias ? __ldg(bias + h * d + i) : 0.0f;
    const bool ok = ptx::mbar_wait_bounded(bar, 0);
    __syncthreads();  // the zero rows and the weights too
    if (!ok) return;  // never expected: the copy lands unless the device faults
    const int g8 = d / 8;
    const int c0 = (tid % g8) * 8, k0 = tid / g8, kstep = kConvThreads / g8;
    float wr[kMaxWidth][8], bs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        bs[e] = sw[kMaxWidth * d + c0 + e];
#pragma unroll
        for (int j = 0; j < kMaxWidth; ++j) wr[j][e] = j < width ? sw[j * d + c0 + e] : 0.0f;
    }
    for (int k = k0; k < tn; k += kstep) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = bs[e];
#pragma unroll
        for (int j = 0; j < kMaxWidth; ++j) {
            if (j < width) {
                float xv[8];
                load8(xs + (k + kMaxWidth - 1 - j) * d + c0, xv);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(wr[j][e], xv[e], acc[e]);
            }
        }
        if (silu) {
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = silu_fast(acc[e]);
        }
        store8(out + ((size_t)bhrow * N + t0 + k) * d + c0, acc);
    }
}

}  // namespace
}  // namespace ssd

using namespace ssd;

extern "C" int ssd_conv1d(const void *x, const float *w, const float *bias, int B, int H, int N, int d_h,
                          int width, int silu, int dtype, void *out, void *stream) {
    if (!x || !w || !out) return SSD_ERR_NULL;
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_DTYPE;
    if (B < 1 || H < 1 || N < 1 || (d_h != 16 && d_h != 32 && d_h != 64) || width < 1 || width > 4)
        return SSD_ERR_SHAPE;
    if ((long long)B * H * N * d_h >= (1ll << 40)) return SSD_ERR_SHAPE;
    const uintptr_t ax = reinterpret_cast<uintptr_t>(x), ao = reinterpret_cast<uintptr_t>(out);
    if ((ax & 15u) || (ao & 15u) || (reinterpret_cast<uintptr_t>(w) & 3u) ||
        (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
        return SSD_ERR_ALIGN;
    const size_t bytes = (size_t)B * H * N * d_h * (dtype == SSD_F32 ? 4 : 2);
    if (ax < ao + bytes && ao < ax + bytes) return SSD_ERR_SHAPE;  // out must not overlap x
    const long long grid = (long long)B * H * ((N + kTile - 1) / kTile);
    if (grid >= (1ll << 31)) return SSD_ERR_SHAPE;
    const size_t esize = dtype == SSD_F32 ? 4 : 2;
    const size_t smem = 128 + (size_t)(kTile + kMaxWidth - 1) * d_h * esize + (size_t)(kMaxWidth + 1) * d_h * 4;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == SSD_F32) {
        if (cudaFuncSetAttribute(conv1d_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return SSD_ERR_CUDA;
        conv1d_kernel<float><<<(unsigned)grid, kConvThreads, smem, s>>>(static_cast<const float *>(x), w, bias, H, N,
                                                                        d_h, width, silu, static_cast<float *>(out));
    } else {
        if (cudaFuncSetAttribute(conv1d_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return SSD_ERR_CUDA;
        conv1d_kernel<__nv_bfloat16><<<(unsigned)grid, kConvThreads, smem, s>>>(
            static_cast<const __nv_bfloat16 *>(x), w, bias, H, N, d_h, width, silu,
            static_cast<__nv_bfloat16 *>(out));
    }
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
