// One recurrent step per (b, h) of the SSD operator: the token-by-token form
// of 2Mamba2Furious Algorithm 6, used for generation after a prefill:
//     h <- a h + phi(k) (f v)^T,   z <- a z + phi(k),
//     y  = phi(q)^T h  [/ phi(q) . z]  [+ D (.) v]
// with a = exp(log-decay) (A dt of Algorithm 3, or a given value, Algorithm 4)
// and f = dt under value discretisation (Algorithm 4), else 1.
//
// The step reads and writes the whole state once, so it is bound by HBM:
// order 2 at d_h = 64 keeps 4096 x 64 fp32 per head.  Two launches:
//   decode_state_kernel   grid (B*H, S): CTA s updates state rows
//                         [s R, s R + R) with 16-byte accesses and writes its
//                         partial readout phi(q)^T h (and phi(q) . z) to the
//                         workspace;
//   decode_output_kernel  grid (B*H): sums the S partials, normalises, adds
//                         the residual and stores y.
#include <cuda_bf16.h>
#include <math.h>

#include "ptx.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kDecThreads = 256;
// float4s of state a thread updates: a CTA holds at most 64 rows of d_h <= 64
// columns, 1024 float4s
constexpr int kPerThread = 4;

__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}
__device__ __forceinline__ float load_elem(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_elem(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16 *p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// State rows per CTA: the whole state for order 1, 64 feature rows for order 2.
__host__ __device__ inline int rows_per_cta(int d, int order) { return order == 1 ? d : 64; }
__host__ __device__ inline int slices(int d, int order) {
    return order == 1 ? 1 : (d * d) / 64;
}

template <typename T>
__global__ void __launch_bounds__(kDecThreads)
decode_state_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                    const float *__restrict__ dt_p, const float *__restrict__ A_log,
                    const float *__restrict__ dt_bias, const float *__restrict__ log_decay,
                    int value_dt, int H, int d, int order, float *__restrict__ h,
                    float *__restrict__ z, float *__restrict__ part) {
    __shared__ float qs[64], ks[64], vs[64];
    __shared__ float red[kDecThreads / 32][65];
    const int bh = blockIdx.x, s = blockIdx.y, hd = bh % H;
    const int S = gridDim.y;
    const int R = rows_per_cta(d, order);
    const int Dphi = order == 1 ? d : d * d;
    const int m0 = s * R;
    const int tid = threadIdx.x;
    const int d4 = d / 4;
    const int n4 = R * d4;  // float4s of this CTA's state rows
    float4 *hb = reinterpret_cast<float4 *>(h + ((size_t)bh * Dphi + m0) * d);
    // this thread's state loads go out first (n4 <= kPerThread kDecThreads):
    // they depend on nothing else, so their latency overlaps the token's
    float4 xv[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int e = tid + u * kDecThreads;
        if (e < n4) xv[u] = __ldcs(hb + e);
    }
    const float zv = (z && tid < R) ? z[(size_t)bh * Dphi + m0 + tid] : 0.0f;
    if (tid < d) {
        qs[tid] = load_elem(q, (size_t)bh * d + tid);
        ks[tid] = load_elem(k, (size_t)bh * d + tid);
        vs[tid] = load_elem(v, (size_t)bh * d + tid);
    }
    // decay and value factor of this token
    float dt = 0.0f;
    if (value_dt || !log_decay) dt = softplus_f(dt_p[bh] + dt_bias[hd]);
    const float a = expf(log_decay ? log_decay[bh] : -expf(A_log[hd]) * dt);
    const float f = value_dt ? dt : 1.0f;
    __syncthreads();

    // each thread keeps the partial readout of one column group
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int c4 = tid % d4;  // column group of this thread: the same for all its elements
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int e = tid + u * kDecThreads;
        if (e >= n4) break;
        const int r = e / d4;
        const int m = m0 + r;
        const float fk = order == 1 ? ks[m] : ks[m / d] * ks[m % d];
        const float fq = order == 1 ? qs[m] : qs[m / d] * qs[m % d];
        const float w = fk * f;
        float4 x = xv[u];
        x.x = fmaf(a, x.x, w * vs[4 * c4 + 0]);
        x.y = fmaf(a, x.y, w * vs[4 * c4 + 1]);
        x.z = fmaf(a, x.z, w * vs[4 * c4 + 2]);
        x.w = fmaf(a, x.w, w * vs[4 * c4 + 3]);
        __stcs(hb + e, x);
        acc.x = fmaf(fq, x.x, acc.x);
        acc.y = fmaf(fq, x.y, acc.y);
        acc.z = fmaf(fq, x.z, acc.z);
        acc.w = fmaf(fq, x.w, acc.w);
    }
    float nacc = 0.0f;
    if (z && tid < R) {  // R <= 64 < kDecThreads: one normaliser entry per thread, loaded at the start
        const int m = m0 + tid;
        const float fk = order == 1 ? ks[m] : ks[m / d] * ks[m % d];
        const float fq = order == 1 ? qs[m] : qs[m / d] * qs[m % d];
        const float zn = fmaf(a, zv, fk);
        z[(size_t)bh * Dphi + m] = zn;
        nacc = fq * zn;
    }
    // reduce the column groups: lanes tid, tid ^ d4, ... hold the same group
    // (d4 divides 32), then the warps through shared memory
    const int lane = tid & 31, wid = tid >> 5;
    for (int o = d4; o < 32; o <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) nacc += __shfl_xor_sync(0xffffffffu, nacc, o);
    if (lane < d4) {  // rows of 65 floats: scalar stores (a row is not 16-byte aligned)
        red[wid][4 * lane + 0] = acc.x;
        red[wid][4 * lane + 1] = acc.y;
        red[wid][4 * lane + 2] = acc.z;
        red[wid][4 * lane + 3] = acc.w;
    }
    if (lane == 0) red[wid][d] = nacc;
    __syncthreads();
    if (tid <= d) {
        float y = 0.0f;
#pragma unroll
        for (int w = 0; w < kDecThreads / 32; ++w) y += red[w][tid];
        part[((size_t)bh * S + s) * (d + 1) + tid] = y;
    }
    ptx::pdl_launch_dependents();  // the output kernel waits for this grid before it reads part
}

// Block (65, 4): thread (c, g) sums column c (c = d: the normaliser) over the
// slices s = g, g + 4, ..., so that four independent chains of loads are in
// flight per column rather than one chain over all S slices.
template <typename T>
__global__ void __launch_bounds__(65 * 4)
decode_output_kernel(const T *__restrict__ v, const float *__restrict__ D,
                     const float *__restrict__ part, int H, int d, int S,
                     int normalize, T *__restrict__ out) {
    __shared__ float red[4][65];
    const int bh = blockIdx.x, c = threadIdx.x, g = threadIdx.y;
    ptx::pdl_wait();  // every partial of the state kernel is visible
    const float *p = part + (size_t)bh * S * (d + 1);
    float acc = 0.0f;
    if (c <= d) {
#pragma unroll 4
        for (int s = g; s < S; s += 4) acc += p[(size_t)s * (d + 1) + c];
    }
    red[g][c] = acc;
    __syncthreads();
    if (g == 0 && c <= d) red[0][c] = (red[0][c] + red[1][c]) + (red[2][c] + red[3][c]);
    __syncthreads();
    if (g == 0 && c < d) {
        float y = red[0][c];
        if (normalize) y /= red[0][d];
        if (D) y = fmaf(D[(bh % H) * d + c], load_elem(v, (size_t)bh * d + c), y);
        store_elem(out, (size_t)bh * d + c, y);
    }
}

template <typename T>
int run_decode(const FwdArgs &a, float *h, float *z) {
    const int BH = a.B * a.H;
    const int S = slices(a.d, a.order);
    float *part = reinterpret_cast<float *>(static_cast<char *>(a.workspace) + kStatusBytes);
    decode_state_kernel<T><<<dim3(BH, S), kDecThreads, 0, a.stream>>>(
        static_cast<const T *>(a.q), static_cast<const T *>(a.k), static_cast<const T *>(a.v), a.dt_p,
        a.A_log, a.dt_bias, a.log_decay, a.value_dt, a.H, a.d, a.order, h, z, part);
    // launched as a programmatic dependent: its CTAs may start while the state
    // kernel drains, and each waits (griddepcontrol.wait) before reading part
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t c2 = {};
    c2.gridDim = dim3(BH);
    c2.blockDim = dim3(65, 4);
    c2.stream = a.stream;
    c2.attrs = pdl;
    c2.numAttrs = 1;
    if (cudaLaunchKernelEx(&c2, decode_output_kernel<T>, static_cast<const T *>(a.v), a.D, (const float *)part, a.H,
                           a.d, S, a.normalize, static_cast<T *>(a.out)) != cudaSuccess)
        return SSD_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace

size_t decode_workspace(int B, int H, int d, int order) {
    return align_up((size_t)B * H * slices(d, order) * (d + 1) * sizeof(float), 256);
}

int launch_decode(const FwdArgs &a, float *h, float *z) {
    if (a.dtype == SSD_F32) return run_decode<float>(a, h, z);
    return run_decode<__nv_bfloat16>(a, h, z);
}

}  // namespace ssd
