// Causal depthwise 1-D convolution over tokens with optional SiLU: the
// prologue Q, K, V = SiLU(conv_1d(h W_QKV)) of 2Mamba2Furious Algorithm 3 and
// the window-2 convolution q^c_t = conv_1d(q_t, q_{t-1}) of the Algorithm 6
// page, applied to one [B, H, N, d_h] tensor:
//     u = bias[c] + sum_{j < width} w[c][j] x[t - j, c]   (x before token 0 is 0)
//     out = SiLU(u) or u
// One thread per (b, h, t) and 8 consecutive channels, 16-byte loads for
// bf16.  HBM-bound: it reads x once (the width-1 earlier rows hit L1/L2) and
// writes out once.
#include <cuda_bf16.h>
#include <math.h>

#include "ssd_internal.h"

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

template <typename T>
__global__ void __launch_bounds__(kConvThreads)
conv1d_kernel(const T *__restrict__ x, const float *__restrict__ w, const float *__restrict__ bias, int H,
              int N, int d, int width, int silu, long long n_items, T *__restrict__ out) {
    const long long item = (long long)blockIdx.x * kConvThreads + threadIdx.x;
    if (item >= n_items) return;
    const int g8 = d / 8;
    const int cg = (int)(item % g8);
    const long long row = item / g8;       // (b, h, t) flattened
    const int t = (int)(row % N);
    const int h = (int)((row / N) % H);
    const int c0 = cg * 8;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = bias ? bias[h * d + c0 + e] : 0.0f;
    for (int j = 0; j < width && j <= t; ++j) {
        float xv[8];
        load8(x + (size_t)(row - j) * d + c0, xv);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(w[(size_t)(h * d + c0 + e) * width + j], xv[e], acc[e]);
    }
    if (silu) {
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = acc[e] / (1.0f + expf(-acc[e]));
    }
    store8(out + (size_t)row * d + c0, acc);
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
    const long long n_items = (long long)B * H * N * (d_h / 8);
    const unsigned grid = (unsigned)((n_items + kConvThreads - 1) / kConvThreads);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == SSD_F32)
        conv1d_kernel<float><<<grid, kConvThreads, 0, s>>>(static_cast<const float *>(x), w, bias, H, N, d_h,
                                                            width, silu, n_items, static_cast<float *>(out));
    else
        conv1d_kernel<__nv_bfloat16><<<grid, kConvThreads, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(x), w, bias, H, N, d_h, width, silu, n_items,
            static_cast<__nv_bfloat16 *>(out));
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
