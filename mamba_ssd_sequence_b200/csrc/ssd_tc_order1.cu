// Order-1 tensor-core path (tcgen05 + TMEM, TMA) of the SSD forward operator
// for bf16 inputs, d_h = 64, chunk = 128.
//
// One CTA per (batch, head) walks that head's chunks in order, keeping the
// carried state h (d_h x d_h, fp32) in tensor memory, so every q/k/v tile is
// read from HBM exactly once and the state never leaves the SM.  Per chunk
// (2Mamba2Furious, Algorithms 1, 3, 4 and 6; the chunked split is the
// standard state-passing form of the semiseparable mask):
//   acs_t   = chunk-local inclusive cumsum of A*dt          (kernel (a), fused)
//   S       = Q K^T                                        (tcgen05, TMEM)
//   P_ij    = S_ij exp(acs_i - acs_j) [i >= j]              (CUDA cores -> smem bf16)
//   Y       = P V                                          (tcgen05, TMEM)
//   Y_off   = Q h_{c-1}                                    (tcgen05, TMEM)
//   h_c     = exp(lam_c) h_{c-1} + K'^T V,  K'_j = exp(lam_c - acs_j) k_j
//                                                          (tcgen05, accumulating in TMEM)
//   y_i     = Y_i + exp(acs_i) Y_off_i  [/ row sum] [+ D v_i]  (epilogue, TMA store)
// All exponentials are of non-positive arguments (chunk-local differences),
// so nothing overflows.  The normaliser state z (d_h floats) is kept in
// shared memory in fp32.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

using namespace ptx;

constexpr int kC = 128;         // chunk length (rows of every tile)
constexpr int kD = 64;          // head dim
constexpr int kThreads = 128;   // one thread per chunk row / TMEM lane
constexpr uint32_t kTileBytes = kC * kD * 2;  // 16 KiB bf16 tile
constexpr uint32_t kStageBytes = 3 * kTileBytes;

// shared-memory map (offsets from a 1024-aligned base)
constexpr uint32_t kOffStage = 0;                               // 2 x {Q, K, V}
constexpr uint32_t kOffP = kOffStage + 2 * kStageBytes;         // P: 2 column blocks
constexpr uint32_t kOffKp = kOffP + 2 * kTileBytes;             // K' (MN-major operand)
constexpr uint32_t kOffHs = kOffKp + kTileBytes;                // h_{c-1} bf16, 64 x 64
constexpr uint32_t kOffMisc = kOffHs + kD * kD * 2;
constexpr uint32_t kSmemBytes = kOffMisc + 1024 + 1024;         // misc + alignment slack

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S: 128 x 128 fp32
constexpr uint32_t kColY = 128;    // Y: 128 x 64
constexpr uint32_t kColYoff = 192; // Y_off: 128 x 64
constexpr uint32_t kColH = 256;    // h: 64 x 64 (M=64 layout: rows at lanes 32w + 0..15)

constexpr float kLog2e = 1.4426950408889634f;

struct Misc {
    float acs2[kC];      // chunk-local cumsum, log2 units
    float z[kD];         // normaliser state
    float wtot[4];
    uint64_t bar_tma[2];
    uint64_t bar_s;
    uint64_t bar_mma;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) {  // K-major, 128B swizzle
    return make_sdesc(saddr, 16, 1024);
}
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr) {  // MN-major, 128B swizzle
    return make_sdesc(saddr, kTileBytes, 1024);
}

__device__ __forceinline__ void unpack8(uint4 u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ uint4 pack8(const float *f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                      pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
}

__device__ __forceinline__ void record_timeout(DeviceStatus *status, int where, Misc *misc) {
    if (status) {
        atomicCAS(&status->code, 0, (int)SSD_ERR_TIMEOUT);
        atomicExch(&status->detail, where);
    }
    misc->abort_flag = 1;
}

__global__ void __launch_bounds__(kThreads, 1)
tc_order1_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                 const float *__restrict__ dt_p, const float *__restrict__ A_log,
                 const float *__restrict__ dt_bias, const float *__restrict__ Dres, int H, int N,
                 int normalize, DeviceStatus *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Misc *misc = reinterpret_cast<Misc *>(smem + kOffMisc);
    const uint32_t sbase = smem_u32(smem);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, h = bh % H;
    const int nc = N / kC;
    const int row0 = bh * N;

    if (tid == 0) {
        if (bh == 0 && status) {
            status->code = 0;
            status->detail = 0;
        }
        mbar_init(&misc->bar_tma[0], 1);
        mbar_init(&misc->bar_tma[1], 1);
        mbar_init(&misc->bar_s, 1);
        mbar_init(&misc->bar_mma, 1);
        misc->abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_o);
    }
    if (warp == 0) {
        tmem_alloc(&misc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (tid < kD) misc->z[tid] = 0.0f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;
    const uint32_t t_lane = (uint32_t)(warp * 32) << 16;

    const float A2 = -expf(A_log[h]) * kLog2e;  // decay rate in log2 units
    const float bias = dt_bias[h];
    float dt_next = dt_p[(size_t)row0 + tid];

    constexpr uint32_t idesc_S = make_idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t idesc_Y = make_idesc_bf16(128, 64, 0, 1);
    constexpr uint32_t idesc_U = make_idesc_bf16(64, 64, 1, 1);

    if (tid == 0) {
        mbar_arrive_expect_tx(&misc->bar_tma[0], kStageBytes);
        tma_load_2d(smem + kOffStage, &tm_q, 0, row0, &misc->bar_tma[0]);
        tma_load_2d(smem + kOffStage + kTileBytes, &tm_k, 0, row0, &misc->bar_tma[0]);
        tma_load_2d(smem + kOffStage + 2 * kTileBytes, &tm_v, 0, row0, &misc->bar_tma[0]);
    }

    for (int c = 0; c < nc; ++c) {
        const int st = c & 1;
        uint8_t *sQ = smem + kOffStage + st * kStageBytes;
        uint8_t *sK = sQ + kTileBytes;
        uint8_t *sV = sK + kTileBytes;
        const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);

        // ---- decay: chunk-local inclusive cumsum (log2 units), one token per thread
        const float dtv = dt_next;
        if (c + 1 < nc) dt_next = dt_p[(size_t)row0 + (size_t)(c + 1) * kC + tid];
        float acs2 = A2 * softplus_f(dtv + bias);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            float y = __shfl_up_sync(0xffffffffu, acs2, o);
            if (lane >= o) acs2 += y;
        }
        if (lane == 31) misc->wtot[warp] = acs2;
        __syncthreads();
        for (int w = 0; w < warp; ++w) acs2 += misc->wtot[w];
        misc->acs2[tid] = acs2;

        // ---- q/k/v of this chunk
        if (!mbar_wait_bounded(&misc->bar_tma[st], (c >> 1) & 1)) record_timeout(status, 1, misc);
        __syncthreads();  // acs2[] complete; abort flag visible
        if (misc->abort_flag) break;
        const float lam2 = misc->acs2[kC - 1];

        if (tid == 0) {
            if (c + 1 < nc) {  // prefetch the next chunk into the other stage
                bulk_wait_group_read0();  // staging of chunk c-1's output has been read
                uint8_t *nQ = smem + kOffStage + (st ^ 1) * kStageBytes;
                const int nrow = row0 + (c + 1) * kC;
                mbar_arrive_expect_tx(&misc->bar_tma[st ^ 1], kStageBytes);
                tma_load_2d(nQ, &tm_q, 0, nrow, &misc->bar_tma[st ^ 1]);
                tma_load_2d(nQ + kTileBytes, &tm_k, 0, nrow, &misc->bar_tma[st ^ 1]);
                tma_load_2d(nQ + 2 * kTileBytes, &tm_v, 0, nrow, &misc->bar_tma[st ^ 1]);
            }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks)
                mma_bf16(tmem + kColS, desc_k(aQ + ks * 32), desc_k(aK + ks * 32), idesc_S, ks > 0);
            mma_commit(&misc->bar_s);
        }

        // ---- K'_j = exp(lam - acs_j) k_j (row tid), same layout as K
        {
            const float wj = exp2f(lam2 - acs2);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 u = *reinterpret_cast<const uint4 *>(sK + sw128_chunk(tid, ch));
                float f[8];
                unpack8(u, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] *= wj;
                *reinterpret_cast<uint4 *>(smem + kOffKp + sw128_chunk(tid, ch)) = pack8(f);
            }
        }
        // ---- h_{c-1}: bf16 copy for Y_off, then scale by exp(lam) in place
        if (c > 0) {
            const float decay = exp2f(lam2);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float hv[32];
                tmem_ld32(tmem + t_lane + kColH + half * 32, hv);
                tmem_wait_ld();
                if (lane < 16) {
                    const int m = warp * 16 + lane;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4 *>(smem + kOffHs + sw128_chunk(m, half * 4 + q4)) =
                            pack8(hv + q4 * 8);
                }
#pragma unroll
                for (int e = 0; e < 32; ++e) hv[e] *= decay;
                tmem_st32(tmem + t_lane + kColH + half * 32, hv);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // h (+)= K'^T V      (M = 64, N = 64, K = 128 tokens; both MN-major)
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks)
                mma_bf16(tmem + kColH, desc_mn(sbase + kOffKp + ks * 2048), desc_mn(aV + ks * 2048),
                         idesc_U, (c > 0 || ks > 0) ? 1u : 0u);
            // Y_off = Q h_{c-1}  (M = 128, N = 64, K = 64)
            if (c > 0) {
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks)
                    mma_bf16(tmem + kColYoff, desc_k(aQ + ks * 32),
                             desc_mn(sbase + kOffHs + ks * 2048), idesc_Y, ks > 0);
            }
        }

        // ---- P = S (.) exp(acs_i - acs_j) [i >= j], row tid, bf16 into smem
        if (!mbar_wait_bounded(&misc->bar_s, c & 1)) record_timeout(status, 2, misc);
        tc_fence_after();
        float rowsum = 0.0f;
#pragma unroll
        for (int jb = 0; jb < kC / 32; ++jb) {
            uint8_t *pblk = smem + kOffP + (jb >> 1) * kTileBytes;
            if (jb > warp) {  // every column of this block is above the diagonal
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    *reinterpret_cast<uint4 *>(pblk + sw128_chunk(tid, (jb & 1) * 4 + q4)) =
                        make_uint4(0, 0, 0, 0);
                continue;
            }
            float sv[32];
            tmem_ld32(tmem + t_lane + kColS + jb * 32, sv);
            tmem_wait_ld();
#pragma unroll
            for (int u = 0; u < 32; ++u) {
                const int j = jb * 32 + u;
                const float p = (j <= tid) ? sv[u] * exp2f(acs2 - misc->acs2[j]) : 0.0f;
                sv[u] = p;
                rowsum += p;
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
                *reinterpret_cast<uint4 *>(pblk + sw128_chunk(tid, (jb & 1) * 4 + q4)) =
                    pack8(sv + q4 * 8);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // Y = P V  (M = 128, N = 64, K = 128 tokens)
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks)
                mma_bf16(tmem + kColY, desc_k(sbase + kOffP + (ks >> 2) * kTileBytes + (ks & 3) * 32),
                         desc_mn(aV + ks * 2048), idesc_Y, ks > 0);
            mma_commit(&misc->bar_mma);
        }

        // ---- normaliser: q_i . z_{c-1}, then z_c = exp(lam) z_{c-1} + sum_j w_j k_j (fp32)
        float qz = 0.0f;
        if (normalize) {
            if (c > 0) {
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float f[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sQ + sw128_chunk(tid, ch)), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) qz = fmaf(f[e], misc->z[ch * 8 + e], qz);
                }
            }
            __syncthreads();
            if (tid < kD) {
                float s = 0.0f;
                for (int j = 0; j < kC; ++j) {
                    const uint16_t kb =
                        *reinterpret_cast<const uint16_t *>(sK + sw128_offset(j, tid));
                    s = fmaf(exp2f(lam2 - misc->acs2[j]), __uint_as_float((uint32_t)kb << 16), s);
                }
                misc->z[tid] = fmaf(exp2f(lam2), misc->z[tid], s);
            }
        }

        // ---- epilogue
        if (!mbar_wait_bounded(&misc->bar_mma, c & 1)) record_timeout(status, 3, misc);
        tc_fence_after();
        {
            const float eoff = exp2f(acs2);
            float y[64];
            tmem_ld32(tmem + t_lane + kColY, *reinterpret_cast<float(*)[32]>(y));
            tmem_ld32(tmem + t_lane + kColY + 32, *reinterpret_cast<float(*)[32]>(y + 32));
            tmem_wait_ld();
            if (c > 0) {
                float yo[32];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tmem_ld32(tmem + t_lane + kColYoff + half * 32, yo);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) y[half * 32 + e] = fmaf(eoff, yo[e], y[half * 32 + e]);
                }
            }
            if (normalize) {
                const float inv = 1.0f / fmaf(eoff, qz, rowsum);
#pragma unroll
                for (int e = 0; e < 64; ++e) y[e] *= inv;
            }
            if (Dres) {
                const float *Dh = Dres + h * kD;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    float f[8];
                    unpack8(*reinterpret_cast<const uint4 *>(sV + sw128_chunk(tid, ch)), f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[ch * 8 + e] = fmaf(__ldg(Dh + ch * 8 + e), f[e], y[ch * 8 + e]);
                }
            }
            // stage the bf16 row in the (now free) Q buffer and store the tile with TMA
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
                *reinterpret_cast<uint4 *>(sQ + sw128_chunk(tid, ch)) = pack8(y + ch * 8);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tma_store_2d(&tm_o, sQ, 0, row0 + c * kC);
            bulk_commit_group();
        }
    }

    if (tid == 0) bulk_wait_group0();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// [rows, 64] bf16 row-major tensor, boxes of box_rows x 64, 128-byte swizzle.
bool make_tmap_rows64(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {64, rows};
    cuuint64_t strides[1] = {64 * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool tc_order1_supports(int B, int H, int N, int d, int dtype, int chunk) {
    return dtype == SSD_BF16 && d == kD && chunk == kC && (long long)B * H * N < (1ll << 31);
}

size_t tc_order1_workspace(int, int, int, int, int) { return 0; }

int launch_tc_order1(const FwdArgs &a, const Plan &) {
    const uint64_t rows = (uint64_t)a.B * a.H * a.N;
    CUtensorMap tq, tk, tv, to;
    if (!make_tmap_rows64(&tq, a.q, rows, kC) || !make_tmap_rows64(&tk, a.k, rows, kC) ||
        !make_tmap_rows64(&tv, a.v, rows, kC) || !make_tmap_rows64(&to, a.out, rows, kC))
        return SSD_ERR_CUDA;
    static bool attr_set = false;
    if (!attr_set) {
        if (cudaFuncSetAttribute(tc_order1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes) != cudaSuccess)
            return SSD_ERR_CUDA;
        attr_set = true;
    }
    DeviceStatus *status = reinterpret_cast<DeviceStatus *>(a.workspace);
    tc_order1_kernel<<<a.B * a.H, kThreads, kSmemBytes, a.stream>>>(
        tq, tk, tv, to, a.dt_p, a.A_log, a.dt_bias, a.D, a.H, a.N, a.normalize, status);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace ssd
