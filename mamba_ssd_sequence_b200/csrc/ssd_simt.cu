// General SIMT (CUDA-core, fp32 arithmetic) path of the SSD forward operator,
// and kernel (a), the chunked decay.
//
// The path runs for every supported shape and is the one used for fp32
// inputs, where the tolerance (1e-4 of max|y|) rules out bf16/tf32 tensor
// cores.  It evaluates the chunked ("state passing") decomposition of
// 2Mamba2Furious Algorithms 1/5 with the decay of Algorithm 3 in four
// launches:
//   (a) chunk_cumsum  : acs_t = chunk-local inclusive cumsum of A*dt,
//                       lam_c = the chunk's total;
//   (b) chunk_state   : U_c = sum_{j in c} exp(lam_c - acs_j) phi(k_j) [v_j, 1]^T,
//                       the chunk's own contribution to the carried state
//                       (the column of ones carries the normaliser state);
//   (c) state_scan    : S_c = state entering chunk c,
//                       S_0 = 0, S_{c+1} = exp(lam_c) S_c + U_c  (Algorithm 6
//                       applied chunk by chunk);
//   (d) chunk_output  : y_i = sum_{j in c, j<=i} (q_i.k_j)^p exp(acs_i-acs_j) v_j
//                             + exp(acs_i) phi(q_i)^T S_c,
//                       the same for the row sum, then /row sum, + D*v.
// phi is the identity (order 1) or the tensor square (order 2), whose inner
// product with phi(k) is (q.k)^2.
// Mamba-2S options (Algorithm 4): a given per-token log-decay replaces A*dt
// in (a); with value discretisation, v_j is multiplied by dt_j in (b) and
// (d) (not in the normaliser column, not in the D residual).
#include <cuda_bf16.h>
#include <math.h>

#include "ssd_internal.h"
#include "ssd_math.cuh"

namespace ssd {
namespace {

__device__ __forceinline__ float load_elem(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_elem(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16 *p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
}

// softplus(x) = log(1 + e^x) in the overflow-free form.
__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

// ---------------------------------------------------------------- kernel (a)
// Chunk-local inclusive cumsum of the per-token log-decay, and chunk totals.
// 256 threads per CTA, kCumU blocks of 1024 tokens per CTA: in block u,
// thread t takes the four consecutive tokens 4t..4t+3 (16-byte loads and
// stores); every block's loads are issued before any is used.  One block per
// CTA measured fastest: more keep more loads in flight per thread but leave
// small problems with too few CTAs.  A chunk of C
// tokens is C/4 threads: a
// segment of 16 or 32 lanes for C = 64 or 128, two warps for C = 256.
// Chunks are contiguous in the flattened [B H N] order and never straddle a
// head, since N % C == 0.  Index arithmetic is in I: 32-bit when B H N <
// 2^31 (integer division by N being the costly step), else 64-bit.
constexpr int kCumU = 1;

template <typename I>
__global__ void __launch_bounds__(256)
chunk_cumsum_kernel(const float *__restrict__ dt_p, const float *__restrict__ A_log,
                    const float *__restrict__ dt_bias, const float *__restrict__ log_decay, int H,
                    int N, int chunk_shift, I total, float *__restrict__ acs,
                    float *__restrict__ chunk_sum, DeviceStatus *status) {
    __shared__ float warp_tot[kCumU][8];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    if (status && blockIdx.x == 0 && t == 0) {
        status->code = 0;
        status->detail = 0;
    }
    const int chunk = 1 << chunk_shift;
    I tok0[kCumU];
    float4 x[kCumU];
    int h[kCumU];
#pragma unroll
    for (int u = 0; u < kCumU; ++u) {
        tok0[u] = (((I)blockIdx.x * kCumU + (I)u) * 256 + (I)t) * 4;
        h[u] = 0;
        x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (tok0[u] < total) {  // total is a multiple of 64: whole chunks only
            x[u] = __ldg(reinterpret_cast<const float4 *>((log_decay ? log_decay : dt_p) + tok0[u]));
            h[u] = (int)((tok0[u] / (I)N) % (I)H);
        }
    }
    const int seg = chunk / 4;  // threads per chunk
    const int width = seg < 32 ? seg : 32;
    float a[kCumU][4], before[kCumU];
#pragma unroll
    for (int u = 0; u < kCumU; ++u) {
        if (log_decay) {
            a[u][0] = x[u].x, a[u][1] = x[u].y, a[u][2] = x[u].z, a[u][3] = x[u].w;
        } else {
            const bool live = tok0[u] < total;
            const float A = live ? -expf(__ldg(A_log + h[u])) : 0.0f;
            const float bias = live ? __ldg(dt_bias + h[u]) : 0.0f;
            a[u][0] = A * softplus_fast(x[u].x + bias);
            a[u][1] = A * softplus_fast(x[u].y + bias);
            a[u][2] = A * softplus_fast(x[u].z + bias);
            a[u][3] = A * softplus_fast(x[u].w + bias);
        }
        a[u][1] += a[u][0];
        a[u][2] += a[u][1];
        a[u][3] += a[u][2];
        // inclusive scan of the thread totals within each chunk's lanes
        float run = a[u][3];
        for (int o = 1; o < width; o <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, run, o, width);
            if ((lane & (width - 1)) >= o) run += y;
        }
        before[u] = run - a[u][3];
        if (lane == 31) warp_tot[u][warp] = run;
    }
    if (seg > 32) {  // C = 256: the second warp of a chunk adds the first's total
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kCumU; ++u)
            if (warp & 1) before[u] += warp_tot[u][warp - 1];
    }
#pragma unroll
    for (int u = 0; u < kCumU; ++u) {
        if (tok0[u] < total) {
            const float bf = before[u];
            *reinterpret_cast<float4 *>(acs + tok0[u]) =
                make_float4(a[u][0] + bf, a[u][1] + bf, a[u][2] + bf, a[u][3] + bf);
            if ((((int)tok0[u] + 4) & (chunk - 1)) == 0) chunk_sum[tok0[u] >> chunk_shift] = a[u][3] + bf;
        }
    }
}

// ---------------------------------------------------------------- kernel (b)
constexpr int kThreads = 256;
constexpr int kJT = 32;      // tokens per shared-memory tile
constexpr int kStateTM = 16; // state rows per block in chunk_state
constexpr int kMaxOut = 5;   // ceil(16 * 65 / 256)

template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_state_kernel(const T *__restrict__ k, const T *__restrict__ v,
                   const float *__restrict__ acs, const float *__restrict__ lam,
                   const float *__restrict__ dt_p, const float *__restrict__ dt_bias,
                   int value_dt, int H, int N, int d, int order, int chunk,
                   float *__restrict__ states) {
    __shared__ float ks[kJT * 64];
    __shared__ float vs[kJT * 64];
    __shared__ float ws[kJT];
    __shared__ float fs[kJT];  // value factor dt_j (1 without value discretisation)
    const int mt = blockIdx.x, c = blockIdx.y, bh = blockIdx.z;
    const int nc = N / chunk;
    const int Dphi = order == 1 ? d : d * d;
    const int ld = d + 1;
    const int m0 = mt * kStateTM;
    const int n_out = kStateTM * ld;
    const float lam_c = lam[(size_t)bh * nc + c];
    const size_t tok0 = (size_t)bh * N + (size_t)c * chunk;

    int om[kMaxOut], oc[kMaxOut];
    float acc[kMaxOut];
#pragma unroll
    for (int r = 0; r < kMaxOut; ++r) {
        int o = threadIdx.x + r * kThreads;
        om[r] = m0 + o / ld;
        oc[r] = o % ld;
        acc[r] = 0.0f;
        if (o >= n_out || om[r] >= Dphi) om[r] = -1;
    }
    for (int j0 = 0; j0 < chunk; j0 += kJT) {
        __syncthreads();
        for (int e = threadIdx.x; e < kJT * d; e += kThreads) {
            int jj = e / d, cc = e % d;
            ks[jj * d + cc] = load_elem(k, (tok0 + j0 + jj) * d + cc);
            vs[jj * d + cc] = load_elem(v, (tok0 + j0 + jj) * d + cc);
        }
        if (threadIdx.x < kJT) {
            const size_t tj = tok0 + j0 + threadIdx.x;
            ws[threadIdx.x] = expf(lam_c - acs[tj]);
            fs[threadIdx.x] = value_dt ? softplus_f(dt_p[tj] + dt_bias[(bh % H)]) : 1.0f;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kMaxOut; ++r) {
            if (om[r] < 0) continue;
            const int m = om[r], cc = oc[r];
            const int ma = order == 1 ? m : m / d, mb = order == 1 ? -1 : m % d;
            float s = acc[r];
            for (int jj = 0; jj < kJT; ++jj) {
                float f = ks[jj * d + ma];
                if (mb >= 0) f *= ks[jj * d + mb];
                float vv = cc < d ? vs[jj * d + cc] * fs[jj] : 1.0f;
                s = fmaf(ws[jj] * f, vv, s);
            }
            acc[r] = s;
        }
    }
    float *dst = states + ((size_t)bh * nc + c) * (size_t)Dphi * ld;
#pragma unroll
    for (int r = 0; r < kMaxOut; ++r)
        if (om[r] >= 0) dst[(size_t)om[r] * ld + oc[r]] = acc[r];
}

// ---------------------------------------------------------------- kernel (c)
// One thread per state element; walks the chunks in order, replacing each
// chunk's own contribution U_c by the state entering the chunk.  Element e
// of a state is row m = e / (d+1), column e % (d+1) (column d is the
// normaliser state).  The scan starts from the carried state h0 / z0 (zero
// when NULL) and leaves the state after the last chunk in h_out / z_out.
__global__ void state_scan_kernel(float *__restrict__ states, const float *__restrict__ lam,
                                  int nc, size_t elems_per_state, int BH, int d,
                                  const float *__restrict__ h0, const float *__restrict__ z0,
                                  float *__restrict__ h_out, float *__restrict__ z_out) {
    const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int bh = blockIdx.y;
    if (e >= elems_per_state || bh >= BH) return;
    const size_t m = e / (d + 1), col = e % (d + 1);
    const size_t Dphi = elems_per_state / (d + 1);
    float *base = states + (size_t)bh * nc * elems_per_state + e;
    const float *lb = lam + (size_t)bh * nc;
    float h = 0.0f;
    if (col < (size_t)d && h0) h = h0[((size_t)bh * Dphi + m) * d + col];
    if (col == (size_t)d && z0) h = z0[(size_t)bh * Dphi + m];
    for (int c = 0; c < nc; ++c) {
        float u = base[(size_t)c * elems_per_state];
        base[(size_t)c * elems_per_state] = h;
        h = fmaf(expf(lb[c]), h, u);
    }
    if (col < (size_t)d && h_out) h_out[((size_t)bh * Dphi + m) * d + col] = h;
    if (col == (size_t)d && z_out) z_out[(size_t)bh * Dphi + m] = h;
}

// ---------------------------------------------------------------- kernel (d)
constexpr int kTI = 16;  // output rows per block
constexpr int kTM2 = 32; // state rows per shared-memory tile

template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_output_kernel(const T *__restrict__ q, const T *__restrict__ k,
                    const T *__restrict__ v, const float *__restrict__ acs,
                    const float *__restrict__ states, const float *__restrict__ D,
                    const float *__restrict__ dt_p, const float *__restrict__ dt_bias,
                    int value_dt, int carried, int H, int N, int d, int order, int normalize,
                    int chunk, T *__restrict__ out) {
    __shared__ float qs[kTI * 64];
    __shared__ float ks[kJT * 64];
    __shared__ float vs[kJT * 64];
    __shared__ float fs[kJT];  // value factor dt_j (1 without value discretisation)
    __shared__ float ps[kTI * kJT];
    __shared__ float ss[kTM2 * 65];
    __shared__ float ys[kTI * 65];
    __shared__ float acs_i[kTI];

    const int it = blockIdx.x, c = blockIdx.y, bh = blockIdx.z, h = bh % H;
    const int nc = N / chunk;
    const int Dphi = order == 1 ? d : d * d;
    const int ld = d + 1;
    const int i0 = it * kTI;  // first row of this block inside the chunk
    const size_t tok0 = (size_t)bh * N + (size_t)c * chunk;
    const int n_out = kTI * ld;

    for (int e = threadIdx.x; e < kTI * d; e += kThreads)
        qs[e] = load_elem(q, (tok0 + i0) * d + e);
    if (threadIdx.x < kTI) acs_i[threadIdx.x] = acs[tok0 + i0 + threadIdx.x];

    int oi[kMaxOut], oc[kMaxOut];
    float acc[kMaxOut], off[kMaxOut];
#pragma unroll
    for (int r = 0; r < kMaxOut; ++r) {
        int o = threadIdx.x + r * kThreads;
        oi[r] = o < n_out ? o / ld : -1;
        oc[r] = o % ld;
        acc[r] = 0.0f;
        off[r] = 0.0f;
    }

    // intra-chunk part: tokens j of this chunk with j <= last row of the block
    const int j_end = i0 + kTI;
    for (int j0 = 0; j0 < j_end; j0 += kJT) {
        __syncthreads();
        for (int e = threadIdx.x; e < kJT * d; e += kThreads) {
            int jj = e / d, cc = e % d;
            ks[jj * d + cc] = load_elem(k, (tok0 + j0 + jj) * d + cc);
            vs[jj * d + cc] = load_elem(v, (tok0 + j0 + jj) * d + cc);
        }
        if (threadIdx.x < kJT)
            fs[threadIdx.x] = value_dt ? softplus_f(dt_p[tok0 + j0 + threadIdx.x] + dt_bias[h]) : 1.0f;
        __syncthreads();
        for (int e = threadIdx.x; e < kTI * kJT; e += kThreads) {
            int ii = e / kJT, jj = e % kJT;
            int i = i0 + ii, j = j0 + jj;
            float w = 0.0f;
            if (j <= i) {
                float s = 0.0f;
                for (int cc = 0; cc < d; ++cc) s = fmaf(qs[ii * d + cc], ks[jj * d + cc], s);
                float sc = order == 1 ? s : s * s;
                w = sc * expf(acs_i[ii] - acs[tok0 + j]);
            }
            ps[e] = w;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kMaxOut; ++r) {
            if (oi[r] < 0) continue;
            float s = acc[r];
            const int ii = oi[r], cc = oc[r];
            for (int jj = 0; jj < kJT; ++jj) {
                float vv = cc < d ? vs[jj * d + cc] * fs[jj] : 1.0f;
                s = fmaf(ps[ii * kJT + jj], vv, s);
            }
            acc[r] = s;
        }
    }

    // carried-state part: phi(q_i)^T S_c, scaled by exp(acs_i) (chunk 0 only
    // has one when a state was carried into the sequence)
    if (c > 0 || carried) {
        const float *S = states + ((size_t)bh * nc + c) * (size_t)Dphi * ld;
        for (int m0 = 0; m0 < Dphi; m0 += kTM2) {
            __syncthreads();
            for (int e = threadIdx.x; e < kTM2 * ld; e += kThreads) {
                int mm = e / ld;
                ss[e] = (m0 + mm < Dphi) ? S[(size_t)m0 * ld + e] : 0.0f;
            }
            __syncthreads();
#pragma unroll
            for (int r = 0; r < kMaxOut; ++r) {
                if (oi[r] < 0) continue;
                const int ii = oi[r], cc = oc[r];
                float s = off[r];
                const int mlim = min(kTM2, Dphi - m0);
                for (int mm = 0; mm < mlim; ++mm) {
                    int m = m0 + mm;
                    float f;
                    if (order == 1) f = qs[ii * d + m];
                    else f = qs[ii * d + m / d] * qs[ii * d + m % d];
                    s = fmaf(f, ss[mm * ld + cc], s);
                }
                off[r] = s;
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kMaxOut; ++r)
        if (oi[r] >= 0) ys[oi[r] * ld + oc[r]] = fmaf(expf(acs_i[oi[r]]), off[r], acc[r]);
    __syncthreads();
    for (int e = threadIdx.x; e < kTI * d; e += kThreads) {
        int ii = e / d, cc = e % d;
        float y = ys[ii * ld + cc];
        if (normalize) y = y / ys[ii * ld + d];
        size_t gi = (tok0 + i0 + ii) * d + cc;
        if (D) y = fmaf(D[h * d + cc], load_elem(v, gi), y);
        store_elem(out, gi, y);
    }
}

template <typename T>
int run_simt(const FwdArgs &a, const Plan &p) {
    char *ws = static_cast<char *>(a.workspace);
    float *acs = reinterpret_cast<float *>(ws + p.acs_off);
    float *lam = reinterpret_cast<float *>(ws + p.lam_off);
    float *states = reinterpret_cast<float *>(ws + p.state_off);
    DeviceStatus *status = reinterpret_cast<DeviceStatus *>(ws);
    const int BH = a.B * a.H, nc = a.N / a.chunk;
    const int Dphi = a.order == 1 ? a.d : a.d * a.d;
    int rc = launch_chunk_cumsum(a.dt_p, a.A_log, a.dt_bias, a.log_decay, a.B, a.H, a.N, a.chunk,
                                 acs, lam, status, a.stream);
    if (rc != SSD_OK) return rc;
    const T *q = static_cast<const T *>(a.q);
    const T *k = static_cast<const T *>(a.k);
    const T *v = static_cast<const T *>(a.v);
    dim3 g1((Dphi + kStateTM - 1) / kStateTM, nc, BH);
    chunk_state_kernel<T><<<g1, kThreads, 0, a.stream>>>(k, v, acs, lam, a.dt_p, a.dt_bias,
                                                         a.value_dt, a.H, a.N, a.d, a.order,
                                                         a.chunk, states);
    const size_t elems = (size_t)Dphi * (a.d + 1);
    dim3 g2((unsigned)((elems + 255) / 256), BH);
    state_scan_kernel<<<g2, 256, 0, a.stream>>>(states, lam, nc, elems, BH, a.d, a.h0, a.z0, a.h_out,
                                                a.z_out);
    dim3 g3(a.chunk / kTI, nc, BH);
    chunk_output_kernel<T><<<g3, kThreads, 0, a.stream>>>(
        q, k, v, acs, states, a.D, a.dt_p, a.dt_bias, a.value_dt, (a.h0 || a.z0) ? 1 : 0, a.H, a.N, a.d,
        a.order, a.normalize, a.chunk, static_cast<T *>(a.out));
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace

int launch_chunk_cumsum(const float *dt_p, const float *A_log, const float *dt_bias,
                        const float *log_decay, int B, int H, int N, int chunk, float *acs,
                        float *chunk_sum, DeviceStatus *status, cudaStream_t stream) {
    const size_t total = (size_t)B * H * N;
    const int shift = chunk == 64 ? 6 : chunk == 128 ? 7 : 8;
    const unsigned grid = (unsigned)((total + 1024 * kCumU - 1) / (1024 * kCumU));
    if (total < (1ull << 31))
        chunk_cumsum_kernel<uint32_t><<<grid, 256, 0, stream>>>(dt_p, A_log, dt_bias, log_decay, H, N, shift,
                                                                (uint32_t)total, acs, chunk_sum, status);
    else
        chunk_cumsum_kernel<size_t><<<grid, 256, 0, stream>>>(dt_p, A_log, dt_bias, log_decay, H, N, shift,
                                                              total, acs, chunk_sum, status);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

int launch_simt(const FwdArgs &a, const Plan &p) {
    if (a.dtype == SSD_F32) return run_simt<float>(a, p);
    return run_simt<__nv_bfloat16>(a, p);
}

}  // namespace ssd
