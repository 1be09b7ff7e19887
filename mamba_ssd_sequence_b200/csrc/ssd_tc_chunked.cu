// Chunk-parallel order-1 tensor-core path of the SSD forward operator for
// bf16 inputs, d_h = 64, chunk C in {128, 256}, no normaliser.
//
// The chunked form of 2Mamba2Furious (thelatestinai.com summary page,
// Algorithms 3-5) splits the masked product into work that is independent per
// chunk and one short recurrence over chunk states.  Three launches:
//   (1) chunk_state_kernel, one CTA per chunk c of a head:
//         acs_t = chunk-local inclusive cumsum of A dt (log2 units), lam = acs_{C-1}
//         U_c   = sum_j 2^(lam - acs_j) k_j v_j^T          (tcgen05, M = N = 64, K = C)
//   (2) state_pass_kernel: h_{-1} = 0, hin_c = bf16(h_{c-1}),
//         h_c = 2^lam_c h_{c-1} + U_c                      (fp32, elementwise over the 64 x 64 state)
//   (3) chunk_scan_kernel, persistent, one 128-row output tile per step:
//         S = Q K^T over the keys of the chunk up to the tile's last row   (tcgen05)
//         P_ij = S_ij 2^(acs_i - acs_j) [j <= i]           (CUDA cores)
//         Y = P V,  Z = Q hin                               (tcgen05)
//         y_i = Y_i + 2^acs_i Z_i [+ D v_i]
// The decay of an off-diagonal 32 x 32 block of P is factorised through the
// block's last key r: 2^(acs_i - acs_j) = 2^(acs_i - acs_r) 2^(acs_r - acs_j),
// both factors <= 1 because acs falls along the chunk, so one exp2 per row and
// per column replaces one per element; diagonal blocks take the exact
// per-element exp2.  Every wait is bounded; a timeout sets the status word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "ptx.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

using namespace ptx;

constexpr int kD = 64;
constexpr uint32_t kRowB = 128;         // bytes per bf16 row of 64
constexpr uint32_t kBox = 128 * kRowB;  // one TMA box: 128 rows, 16 KiB
constexpr uint32_t kHinBytes = 64 * kRowB;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) { return make_sdesc(saddr, 16, 1024); }
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr) { return make_sdesc(saddr, 8192, 1024); }

__device__ void set_timeout(DeviceStatus *status, int where, int *abort_flag) {
    if (status) {
        atomicCAS(&status->code, 0, (int)SSD_ERR_TIMEOUT);
        atomicCAS(&status->detail, 0, where);
    }
    if (abort_flag) *reinterpret_cast<volatile int *>(abort_flag) = 1;
}

// =====================================================================
// (1) chunk states
// =====================================================================
template <int C>
struct StateMisc {
    float wtot[4];
    uint64_t full, mma;
    uint32_t tmem;
};

template <int C>
__global__ void __launch_bounds__(128)
chunk_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const float *__restrict__ dt_p, const float *__restrict__ A_log,
                   const float *__restrict__ dt_bias, int H, int N, float *__restrict__ U,
                   float *__restrict__ lam_out, DeviceStatus *status) {
    constexpr int KP = C / 128;  // keys per thread
    constexpr uint32_t K_OFF = 0, V_OFF = C * kRowB, MISC_OFF = 2 * C * kRowB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    StateMisc<C> *misc = reinterpret_cast<StateMisc<C> *>(smem + MISC_OFF);
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nc = N / C;
    const int tile = blockIdx.x, bh = tile / nc, c = tile % nc, h = bh % H;
    const int row = bh * N + c * C;

    if (tid == 0) {
        if (tile == 0 && status) {
            status->code = 0;
            status->detail = 0;
        }
        mbar_init(&misc->full, 1);
        mbar_init(&misc->mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&misc->tmem, 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem;

    if (tid == 0) {
        mbar_arrive_expect_tx(&misc->full, 2 * C * kRowB);
#pragma unroll
        for (int b = 0; b < KP; ++b) {
            tma_load_2d(smem + K_OFF + b * kBox, &tm_k, 0, row + 128 * b, &misc->full);
            tma_load_2d(smem + V_OFF + b * kBox, &tm_v, 0, row + 128 * b, &misc->full);
        }
    }
    // decay of keys [KP tid, KP tid + KP): inclusive scan over the chunk
    const float A2 = -expf(A_log[h]) * kLog2e;
    const float bias = dt_bias[h];
    float a[KP];
    float run = 0.0f;
#pragma unroll
    for (int e = 0; e < KP; ++e) {
        run += A2 * softplus_f(dt_p[(size_t)row + KP * tid + e] + bias);
        a[e] = run;
    }
    float incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) misc->wtot[warp] = incl;
    __syncthreads();
    float pre = incl - run;
    for (int w = 0; w < warp; ++w) pre += misc->wtot[w];
    const float lam = misc->wtot[0] + misc->wtot[1] + misc->wtot[2] + misc->wtot[3];

    const bool ok = mbar_wait_bounded(&misc->full, 0);
    if (__syncthreads_or(!ok)) {
        if (tid == 0) set_timeout(status, 100, nullptr);
    } else {
        // K'_j = 2^(lam - acs_j) k_j in place (a whole 128-byte row shares one factor)
#pragma unroll
        for (int e = 0; e < KP; ++e) {
            const float w = ex2_approx(lam - (pre + a[e]));
            const float2 w2 = make_float2(w, w);
            uint4 *rowp = reinterpret_cast<uint4 *>(smem + K_OFF + (KP * tid + e) * kRowB);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                uint4 x = rowp[ch];
                uint32_t wv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = __fmul2_rn(bf2_to_f2(wv[q]), w2);
                    wv[q] = pack_bf16x2(f.x, f.y);
                }
                rowp[ch] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            constexpr uint32_t idU = make_idesc_bf16(64, 64, 1, 1);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tmem, desc_mn(sbase + K_OFF + ks * 2048), desc_mn(sbase + V_OFF + ks * 2048), idU,
                         ks > 0);
            mma_commit(&misc->mma);
        }
        const bool ok2 = mbar_wait_bounded(&misc->mma, 0);
        if (__syncthreads_or(!ok2)) {
            if (tid == 0) set_timeout(status, 101, nullptr);
            // the product may still be running: wait for it once more before TMEM goes
            mbar_wait_bounded(&misc->mma, 0);
        } else {
            tc_fence_after();
            // M = 64 accumulator: row m sits in lane 32 (m / 16) + m % 16
            float v0[32], v1[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16), v0);
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32, v1);
            tmem_wait_ld();
            if (lane < 16) {
                float4 *dst = reinterpret_cast<float4 *>(U + ((size_t)tile * 64 + warp * 16 + lane) * 64);
#pragma unroll
                for (int q = 0; q < 8; ++q) dst[q] = make_float4(v0[4 * q], v0[4 * q + 1], v0[4 * q + 2], v0[4 * q + 3]);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    dst[8 + q] = make_float4(v1[4 * q], v1[4 * q + 1], v1[4 * q + 2], v1[4 * q + 3]);
            }
            if (tid == 0) lam_out[tile] = lam;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 64);
}

// =====================================================================
// (2) state passing: one thread per 4 state entries of a head
// =====================================================================
__global__ void __launch_bounds__(256)
state_pass_kernel(const float *__restrict__ U, const float *__restrict__ lam, __nv_bfloat16 *__restrict__ hin,
                  int nc) {
    const int bh = blockIdx.x;
    const int e = (blockIdx.y * 256 + threadIdx.x) * 4;  // 4 consecutive entries of the 64 x 64 state
    const float4 *u = reinterpret_cast<const float4 *>(U + (size_t)bh * nc * 4096 + e);
    uint2 *out = reinterpret_cast<uint2 *>(hin + (size_t)bh * nc * 4096 + e);
    const float *lm = lam + (size_t)bh * nc;
    float4 hs = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int c = 0; c < nc; ++c) {
        const float4 uc = __ldg(u + (size_t)c * 1024);
        const float f = ex2_approx(__ldg(lm + c));
        out[(size_t)c * 1024] = make_uint2(pack_bf16x2(hs.x, hs.y), pack_bf16x2(hs.z, hs.w));
        hs.x = fmaf(f, hs.x, uc.x);
        hs.y = fmaf(f, hs.y, uc.y);
        hs.z = fmaf(f, hs.z, uc.z);
        hs.w = fmaf(f, hs.w, uc.w);
    }
}

// =====================================================================
// (3) chunk scan: persistent, warp-specialised
// =====================================================================
constexpr int kScanThreads = 64 + 256;  // TMA warp, MMA warp, 8 compute warps

template <int C>
struct ScanCfg {
    static constexpr int NKB = C / 128;             // 128-key blocks per chunk
    static constexpr int NRB = C / 128;             // 128-row tiles per chunk
    static constexpr int NSB = C == 128 ? 2 : 1;    // S buffers in TMEM
    static constexpr int STAGES = C == 128 ? 3 : 2;
    static constexpr uint32_t Q_OFF = 0;                          // Q tile; P of keys [0,128) later
    static constexpr uint32_t K_OFF = kBox;                       // NKB boxes
    static constexpr uint32_t H_OFF = K_OFF + NKB * kBox;         // hin, 64 rows
    static constexpr uint32_t V_OFF = H_OFF + kHinBytes;          // NKB boxes
    static constexpr uint32_t STAGE = V_OFF + NKB * kBox;
    static constexpr uint32_t P1_OFF = STAGES * STAGE;            // P of keys [128,256) (C = 256)
    static constexpr uint32_t MISC_OFF = P1_OFF + (NKB - 1) * 2 * kBox;
    static constexpr uint32_t MISC_BYTES = 16 * C + 1024;
    static constexpr uint32_t SMEM = MISC_OFF + MISC_BYTES + 1024;
    static constexpr uint32_t COL_S = 0;    // NSB x 128 (C = 128) or 256 (C = 256)
    static constexpr uint32_t COL_Z = 256;  // 2 x 64
    static constexpr uint32_t COL_Y = 384;  // 2 x 64
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(STAGE % 1024 == 0, "stage alignment");
};

template <int C>
struct ScanMisc {
    float acs[2][C];
    float colf[2][C];
    float wtot[2][8];
    uint64_t stage_full[ScanCfg<C>::STAGES], stage_empty[ScanCfg<C>::STAGES];
    uint64_t s_full[ScanCfg<C>::NSB], p_full[ScanCfg<C>::NKB], y_full[2], ep_done[2];
    uint64_t drain;
    uint32_t tmem;
    int abort_flag;
};

struct TileIdx {
    int bh, c, rb;
};
template <int C>
__device__ __forceinline__ TileIdx tile_idx(int t, int nc) {
    constexpr int NRB = ScanCfg<C>::NRB;
    TileIdx x;
    x.rb = t % NRB;
    x.c = (t / NRB) % nc;
    x.bh = t / (NRB * nc);
    return x;
}

template <int C>
__global__ void __launch_bounds__(kScanThreads, 1)
chunk_scan_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_h,
                  const __nv_bfloat16 *__restrict__ vglob, __nv_bfloat16 *__restrict__ out,
                  const float *__restrict__ dt_p, const float *__restrict__ A_log,
                  const float *__restrict__ dt_bias, const float *__restrict__ Dres, int H, int N,
                  int n_tiles, DeviceStatus *status) {
    using K = ScanCfg<C>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    ScanMisc<C> *misc = reinterpret_cast<ScanMisc<C> *>(smem + K::MISC_OFF);
    const volatile int *abort_flag = &misc->abort_flag;
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nc = N / C;

    if (tid == 0) {
        for (int i = 0; i < K::STAGES; ++i) {
            mbar_init(&misc->stage_full[i], 1);
            mbar_init(&misc->stage_empty[i], 1);
        }
        for (int i = 0; i < K::NSB; ++i) mbar_init(&misc->s_full[i], 1);
        for (int i = 0; i < K::NKB; ++i) mbar_init(&misc->p_full[i], 256);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&misc->y_full[i], 1);
            mbar_init(&misc->ep_done[i], 256);
        }
        mbar_init(&misc->drain, 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc->tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            prefetch_tmap(&tm_h);
            int i = 0;
            for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
                const int st = i % K::STAGES;
                if (i >= K::STAGES &&
                    !mbar_wait_abortable(&misc->stage_empty[st], ((i / K::STAGES) - 1) & 1, abort_flag)) {
                    set_timeout(status, 110, &misc->abort_flag);
                    break;
                }
                const TileIdx x = tile_idx<C>(t, nc);
                const int nkb = x.rb + 1;
                const int crow = x.bh * N + x.c * C;
                uint8_t *sp = smem + st * K::STAGE;
                mbar_arrive_expect_tx(&misc->stage_full[st], kBox + kHinBytes + 2 * nkb * kBox);
                tma_load_2d(sp + K::Q_OFF, &tm_q, 0, crow + 128 * x.rb, &misc->stage_full[st]);
                for (int kb = 0; kb < nkb; ++kb) {
                    tma_load_2d(sp + K::K_OFF + kb * kBox, &tm_k, 0, crow + 128 * kb, &misc->stage_full[st]);
                    tma_load_2d(sp + K::V_OFF + kb * kBox, &tm_v, 0, crow + 128 * kb, &misc->stage_full[st]);
                }
                tma_load_2d(sp + K::H_OFF, &tm_h, 0, (x.bh * nc + x.c) * 64, &misc->stage_full[st]);
            }
            // copies still in flight after an abort land before the CTA exits (bounded)
            for (int j = i > K::STAGES ? i - K::STAGES : 0; j < i; ++j)
                mbar_wait_bounded(&misc->stage_full[j % K::STAGES], (j / K::STAGES) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS128 = make_idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idS256 = make_idesc_bf16(128, 256, 0, 0);
            constexpr uint32_t idO = make_idesc_bf16(128, 64, 0, 1);
            uint32_t np[K::NKB];
            for (int kb = 0; kb < K::NKB; ++kb) np[kb] = 0;
            bool ok = true;
            int i = 0;
            for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++i) {
                const int st = i % K::STAGES, sb = i % K::NSB, tb = i & 1;
                const TileIdx x = tile_idx<C>(t, nc);
                const int nkb = x.rb + 1;
                const uint32_t sp = sbase + st * K::STAGE;
                if (!(ok = mbar_wait_abortable(&misc->stage_full[st], (i / K::STAGES) & 1, abort_flag))) break;
                if (i >= 2 && !(ok = mbar_wait_abortable(&misc->ep_done[tb], ((i >> 1) - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
                const uint32_t colS = K::COL_S + (C == 128 ? sb * 128 : 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + colS, desc_k(sp + K::Q_OFF + ks * 32), desc_k(sp + K::K_OFF + ks * 32),
                             nkb == 2 ? idS256 : idS128, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma_bf16(tmem + K::COL_Z + tb * 64, desc_k(sp + K::Q_OFF + ks * 32),
                             desc_mn(sp + K::H_OFF + ks * 2048), idO, ks > 0);
                mma_commit(&misc->s_full[sb]);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!(ok = mbar_wait_abortable(&misc->p_full[kb], np[kb] & 1, abort_flag))) break;
                    ++np[kb];
                    tc_fence_after();
                    const uint32_t pb = kb == 0 ? sp + K::Q_OFF : sbase + K::P1_OFF;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16(tmem + K::COL_Y + tb * 64, desc_k(pb + (ks >> 2) * kBox + (ks & 3) * 32),
                                 desc_mn(sp + K::V_OFF + kb * kBox + ks * 2048), idO, (kb > 0 || ks > 0));
                }
                if (!ok) break;
                mma_commit(&misc->y_full[tb]);
                mma_commit(&misc->stage_empty[st]);
            }
            if (!ok) {
                set_timeout(status, 120, &misc->abort_flag);
                // products still in flight finish before TMEM is released (bounded)
                mma_commit(&misc->drain);
                mbar_wait_bounded(&misc->drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------ compute warps
        const int ct = tid - 64;           // 0..255
        const int w = ct >> 5;             // 0..7
        const int g = warp & 3;            // TMEM lane quarter
        const int hf = (warp - 2) >> 2;    // half of the columns
        const uint32_t lane_off = (uint32_t)(g * 32) << 16;
        const int r = g * 32 + lane;       // row of the 128-row tile
        const bool elected = ct == 0;

        int i = 0;
        int pt = -1, pi = 0;  // tile whose epilogue is pending, and its local index
        auto epilogue = [&](int t, int li) -> bool {
            const TileIdx x = tile_idx<C>(t, nc);
            const int tb = li & 1;
            const bool bad = !mbar_wait_abortable(&misc->y_full[tb], (li >> 1) & 1, abort_flag);
            if (named_bar_any(1, 256, bad)) return false;
            tc_fence_after();
            const int h = x.bh % H;
            const int ir = 128 * x.rb + r;
            const size_t grow = (size_t)x.bh * N + (size_t)x.c * C + ir;
            const float e = ex2_approx(misc->acs[li & 1][ir]);
            float yv[32], zv[32];
            tmem_ld32(tmem + lane_off + K::COL_Y + tb * 64 + hf * 32, yv);
            tmem_ld32(tmem + lane_off + K::COL_Z + tb * 64 + hf * 32, zv);
            uint4 vr[4];
            float dh[32];
            if (Dres) {
                const uint4 *vp = reinterpret_cast<const uint4 *>(vglob + grow * kD + hf * 32);
                const float4 *dp = reinterpret_cast<const float4 *>(Dres + h * kD + hf * 32);
#pragma unroll
                for (int q = 0; q < 4; ++q) vr[q] = __ldg(vp + q);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 d4 = __ldg(dp + q);
                    dh[4 * q] = d4.x;
                    dh[4 * q + 1] = d4.y;
                    dh[4 * q + 2] = d4.z;
                    dh[4 * q + 3] = d4.w;
                }
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&misc->ep_done[tb]);
            uint4 *op = reinterpret_cast<uint4 *>(out + grow * kD + hf * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t wv[4];
                const uint32_t vw[4] = {vr[q].x, vr[q].y, vr[q].z, vr[q].w};
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int cc = q * 8 + 2 * p;
                    float y0 = fmaf(e, zv[cc], yv[cc]);
                    float y1 = fmaf(e, zv[cc + 1], yv[cc + 1]);
                    if (Dres) {
                        const float2 vf = bf2_to_f2(vw[p]);
                        y0 = fmaf(dh[cc], vf.x, y0);
                        y1 = fmaf(dh[cc + 1], vf.y, y1);
                    }
                    wv[p] = pack_bf16x2(y0, y1);
                }
                op[q] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
            return true;
        };

        // raw decay input of thread ct's key for tile t (0 past the tile's keys)
        auto load_decay = [&](int t) -> float {
            if (t >= n_tiles) return 0.0f;
            const TileIdx x = tile_idx<C>(t, nc);
            if (ct >= 128 * (x.rb + 1)) return 0.0f;
            const int h = x.bh % H;
            return -expf(A_log[h]) * kLog2e * softplus_f(dt_p[(size_t)x.bh * N + (size_t)x.c * C + ct] + dt_bias[h]);
        };
        bool failed = false;
        float a_next = load_decay(blockIdx.x);
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
            const TileIdx x = tile_idx<C>(t, nc);
            const int nkb = x.rb + 1;
            const int sb = i % K::NSB, ab = i & 1;
            // ---- decay of keys [0, 128 nkb): thread ct owns key ct
            float a = a_next;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, a, o);
                if (lane >= o) a += y;
            }
            if (lane == 31) misc->wtot[ab][w] = a;
            named_bar_sync(1, 256);
            for (int ww = 0; ww < w; ++ww) a += misc->wtot[ab][ww];
            const float aref = __shfl_sync(0xffffffffu, a, 31);  // acs of this 32-key block's last key
            if (ct < C) {
                misc->acs[ab][ct] = a;
                misc->colf[ab][ct] = ex2_approx(aref - a);
            }
            a_next = load_decay(t + gridDim.x);  // consumed at the next tile
            // ---- S of this tile
            const bool bad = !mbar_wait_abortable(&misc->s_full[sb], (i / K::NSB) & 1, abort_flag);
            if (named_bar_any(1, 256, bad)) {  // also publishes acs[] and colf[]
                failed = true;
                break;
            }
            tc_fence_after();
            const int ir = 128 * x.rb + r;  // chunk-local row
            const float ai = misc->acs[ab][ir];
            const int W32 = 4 * x.rb + g;  // 32-row block of this warp, chunk-local
            for (int kb = 0; kb < nkb; ++kb) {
                uint8_t *pb = kb == 0 ? smem + (i % K::STAGES) * K::STAGE + K::Q_OFF : smem + K::P1_OFF;
                const uint32_t colS = K::COL_S + (C == 128 ? sb * 128 : kb * 128);
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    const int q = 2 * hf + pc;        // 32-key piece of the 128-key block
                    const int P32 = 4 * kb + q;       // chunk-local 32-key block
                    const int k0 = 32 * P32;
                    uint32_t pk[16];
                    if (P32 > W32) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    } else {
                        float sv[32];
                        tmem_ld32(tmem + lane_off + colS + 32 * q, sv);
                        tmem_wait_ld();
                        if (P32 < W32) {
                            const float rowf = ex2_approx(ai - misc->acs[ab][k0 + 31]);
                            const float2 rf2 = make_float2(rowf, rowf);
                            const float4 *cf = reinterpret_cast<const float4 *>(&misc->colf[ab][k0]);
#pragma unroll
                            for (int e4 = 0; e4 < 8; ++e4) {
                                const float4 c4 = cf[e4];
                                const float2 p0 = __fmul2_rn(__fmul2_rn(make_float2(sv[4 * e4], sv[4 * e4 + 1]),
                                                                        make_float2(c4.x, c4.y)), rf2);
                                const float2 p1 = __fmul2_rn(__fmul2_rn(make_float2(sv[4 * e4 + 2], sv[4 * e4 + 3]),
                                                                        make_float2(c4.z, c4.w)), rf2);
                                pk[2 * e4] = pack_bf16x2(p0.x, p0.y);
                                pk[2 * e4 + 1] = pack_bf16x2(p1.x, p1.y);
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 32; e += 2) {
                                const int j = k0 + e;
                                float p0 = sv[e] * ex2_approx(ai - misc->acs[ab][j]);
                                float p1 = sv[e + 1] * ex2_approx(ai - misc->acs[ab][j + 1]);
                                if (j > ir) p0 = 0.0f;
                                if (j + 1 > ir) p1 = 0.0f;
                                pk[e >> 1] = pack_bf16x2(p0, p1);
                            }
                        }
                    }
                    uint8_t *atom = pb + (q >> 1) * kBox;
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc)
                        *reinterpret_cast<uint4 *>(atom + sw128_chunk(r, (q & 1) * 4 + cc)) =
                            make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
                }
                tc_fence_before();
                fence_proxy_async_smem();
                mbar_arrive(&misc->p_full[kb]);
            }
            // ---- the previous tile's epilogue overlaps this tile's P V
            if (pt >= 0 && !epilogue(pt, pi)) {
                failed = true;
                break;
            }
            pt = t;
            pi = i;
        }
        if (!failed && pt >= 0 && !epilogue(pt, pi)) failed = true;
        if (failed && elected) set_timeout(status, 130, &misc->abort_flag);
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
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

// [rows, 64] bf16 row-major tensor read in boxes of `box_rows` rows, 128-byte swizzle.
bool make_tmap64(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {64, rows};
    cuuint64_t strides[1] = {64 * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                     estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Sets the dynamic shared-memory limit of `fn` once per device.
template <typename F>
bool smem_attr_once(F fn, int bytes, std::atomic<uint64_t> &done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load() & bit) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return false;
    done.fetch_or(bit);
    return true;
}

int num_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

template <int C>
int launch_c(const FwdArgs &a, const Plan &p) {
    using K = ScanCfg<C>;
    const int BH = a.B * a.H, nc = a.N / C;
    const uint64_t rows = (uint64_t)BH * a.N;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    DeviceStatus *status = reinterpret_cast<DeviceStatus *>(ws);
    float *lam = reinterpret_cast<float *>(ws + p.lam_off);
    float *U = reinterpret_cast<float *>(ws + p.state_off);
    __nv_bfloat16 *hin = reinterpret_cast<__nv_bfloat16 *>(ws + p.aux_off);
    CUtensorMap tq, tk, tv, th;
    if (!make_tmap64(&tq, a.q, rows, 128) || !make_tmap64(&tk, a.k, rows, 128) ||
        !make_tmap64(&tv, a.v, rows, 128) || !make_tmap64(&th, hin, (uint64_t)BH * nc * 64, 64))
        return SSD_ERR_CUDA;
    static std::atomic<uint64_t> attr1{0}, attr3{0};
    constexpr int smem1 = 2 * C * kRowB + 1024 + 1024;
    if (!smem_attr_once(chunk_state_kernel<C>, smem1, attr1) ||
        !smem_attr_once(chunk_scan_kernel<C>, (int)K::SMEM, attr3))
        return SSD_ERR_CUDA;
    const int sms = num_sms();
    if (sms <= 0) return SSD_ERR_CUDA;

    chunk_state_kernel<C><<<BH * nc, 128, smem1, a.stream>>>(tk, tv, a.dt_p, a.A_log, a.dt_bias, a.H, a.N, U,
                                                             lam, status);
    state_pass_kernel<<<dim3(BH, 4), 256, 0, a.stream>>>(U, lam, hin, nc);
    const int n_tiles = BH * nc * K::NRB;
    const int grid = n_tiles < sms ? n_tiles : sms;
    chunk_scan_kernel<C><<<grid, kScanThreads, K::SMEM, a.stream>>>(
        tq, tk, tv, th, static_cast<const __nv_bfloat16 *>(a.v), static_cast<__nv_bfloat16 *>(a.out), a.dt_p,
        a.A_log, a.dt_bias, a.D, a.H, a.N, n_tiles, status);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace

bool tc_chunked_supports(int B, int H, int N, int d, int dtype, int chunk) {
    return dtype == SSD_BF16 && d == kD && (chunk == 128 || chunk == 256) && (long long)B * H * N < (1ll << 31);
}

// lam (n_chunks floats), U (n_chunks x 64 x 64 fp32), hin (n_chunks x 64 x 64 bf16)
void tc_chunked_layout(int B, int H, int N, int chunk, Plan *p) {
    const size_t n = (size_t)B * H * (N / chunk);
    p->acs_off = kStatusBytes;
    p->lam_off = kStatusBytes;
    p->state_off = align_up(p->lam_off + n * sizeof(float), 256);
    p->aux_off = align_up(p->state_off + n * 4096 * sizeof(float), 256);
    p->total = align_up(p->aux_off + n * 4096 * 2, 256);
}

int launch_tc_chunked(const FwdArgs &a, const Plan &p) {
    if (a.normalize || a.order != 1) return SSD_ERR_UNSUPPORTED;
    return a.chunk == 256 ? launch_c<256>(a, p) : launch_c<128>(a, p);
}

}  // namespace ssd
