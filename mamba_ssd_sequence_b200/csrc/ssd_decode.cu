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

#include "ssd_internal.h"

namespace ssd {
namespace {

constexpr int kDecThreads = 256;

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
    __shared__ float ys[65];
    const int bh = blockIdx.x, s = blockIdx.y, hd = bh % H;
    const int S = gridDim.y;
    const int R = rows_per_cta(d, order);
    const int Dphi = order == 1 ? d : d * d;
    const int m0 = s * R;
    const int tid = threadIdx.x;
    if (tid < d) {
        qs[tid] = load_elem(q, (size_t)bh * d + tid);
        ks[tid] = load_elem(k, (size_t)bh * d + tid);
        vs[tid] = load_elem(v, (size_t)bh * d + tid);
    }
    if (tid <= d) ys[tid] = 0.0f;
    // decay and value factor of this token
    float dt = 0.0f;
    if (value_dt || !log_decay) dt = softplus_f(dt_p[bh] + dt_bias[hd]);
    const float a = expf(log_decay ? log_decay[bh] : -expf(A_log[hd]) * dt);
    const float f = value_dt ? dt : 1.0f;
    __syncthreads();

    const int d4 = d / 4;
    const int n4 = R * d4;  // float4s of this CTA's state rows
    float4 *hb = reinterpret_cast<float4 *>(h + ((size_t)bh * Dphi + m0) * d);
    // each thread keeps the partial readout of one column group
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int c4 = tid % d4;  // column group of this thread: the same for all its elements
    for (int e = tid; e < n4; e += kDecThreads) {
        const int r = e / d4;
        const int m = m0 + r;
        const float fk = order == 1 ? ks[m] : ks[m / d] * ks[m % d];
        const float fq = order == 1 ? qs[m] : qs[m / d] * qs[m % d];
        const float w = fk * f;
        float4 x = hb[e];
        x.x = fmaf(a, x.x, w * vs[4 * c4 + 0]);
        x.y = fmaf(a, x.y, w * vs[4 * c4 + 1]);
        x.z = fmaf(a, x.z, w * vs[4 * c4 + 2]);
        x.w = fmaf(a, x.w, w * vs[4 * c4 + 3]);
        hb[e] = x;
        acc.x = fmaf(fq, x.x, acc.x);
        acc.y = fmaf(fq, x.y, acc.y);
        acc.z = fmaf(fq, x.z, acc.z);
        acc.w = fmaf(fq, x.w, acc.w);
    }
    float nacc = 0.0f;
    if (z) {
        for (int r = tid; r < R; r += kDecThreads) {
            const int m = m0 + r;
            const float fk = order == 1 ? ks[m] : ks[m / d] * ks[m % d];
            const float fq = order == 1 ? qs[m] : qs[m / d] * qs[m % d];
            float *zp = z + (size_t)bh * Dphi + m;
            const float zn = fmaf(a, *zp, fk);
            *zp = zn;
            nacc = fmaf(fq, zn, nacc);
        }
    }
    // reduce the column groups (kDecThreads is a multiple of d4, so each
    // thread's group is fixed) and the normaliser through shared memory
    atomicAdd(&ys[4 * c4 + 0], acc.x);
    atomicAdd(&ys[4 * c4 + 1], acc.y);
    atomicAdd(&ys[4 * c4 + 2], acc.z);
    atomicAdd(&ys[4 * c4 + 3], acc.w);
    if (z) atomicAdd(&ys[d], nacc);
    __syncthreads();
    if (tid <= d) part[((size_t)bh * S + s) * (d + 1) + tid] = ys[tid];
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
    decode_output_kernel<T><<<BH, dim3(65, 4), 0, a.stream>>>(static_cast<const T *>(a.v), a.D, part, a.H,
                                                              a.d, S, a.normalize, static_cast<T *>(a.out));
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
