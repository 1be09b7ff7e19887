// Chunk-parallel order-1 tensor-core path of the SSD forward operator for
// bf16 inputs, d_h = 64, chunk C in {128, 256}, no normaliser.
//
// The chunked form of 2Mamba2Furious (thelatestinai.com summary page,
// Algorithms 3-5) splits the masked product into work that is independent per
// chunk and one short recurrence over chunk states.  Three launches:
//   (1) chunk_state_kernel, persistent, one compute group per chunk c of a head:
//         acs_t = chunk-local inclusive cumsum of A dt (log2 units), lam = acs_{C-1}
//         U_c   = sum_j 2^(lam - acs_j) k_j v_j^T          (tcgen05, M = N = 64, K = C;
//                                                          accumulated in fp32, stored as bf16)
//   (2) state_pass_kernel: h_{-1} = h0 (or 0), hin_c = bf16(h_{c-1}),
//         h_c = 2^lam_c h_{c-1} + U_c                      (fp32, elementwise over the 64 x 64 state)
//         and h_out = h of the last chunk when asked for
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
// Mamba-2S options (Algorithm 4): a given per-token log-decay replaces A dt
// in (1); with value discretisation the factor dt_j multiplies key j's
// weight in U (through K') and in P (through the per-key factors).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "ptx.cuh"
#include "ssd_internal.h"
#include "ssd_math.cuh"

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
// (1) chunk states: persistent, warp-specialised
//   warp 0: TMA producer (ring of K, V chunk tiles)
//   warp 1: MMA issuer (U_c^T = V^T K' into the owning group's TMEM accumulator)
//   NG compute groups of 4 warps taking chunks round-robin: decay scan, K'
//   scaling in place, U epilogue.  While one group waits for its product the
//   others work, which hides most of each chunk's latency chain.
// U is stored transposed, U^T[n][k] (value index n, feature index k), which
// is the K-major layout the output kernel's MMA takes for the state.
// With the convolution prologue fused (CV), the stages hold the raw q, k, v
// tiles; the group convolves them in place (conv_tile), stores the results
// for the scan, and writes K' into the Q slot once Q's store has read it.
// =====================================================================
constexpr int kStateGroup = 128;

template <int C, bool CV>
struct StateCfg {
    static constexpr int NG = C == 128 ? 4 : 2;
    static constexpr int THREADS = 64 + NG * kStateGroup;
    static constexpr int STAGES = CV ? (C == 128 ? 4 : 2) : (C == 128 ? 6 : 3);
    static constexpr uint32_t TILE = C * kRowB;
    static constexpr uint32_t STAGE = (CV ? 3 : 2) * TILE;  // K, V [, Q]
    static constexpr uint32_t MISC_OFF = STAGES * STAGE;
    static constexpr uint32_t MISC_BYTES = 4 * NG * C + 1024;
    static constexpr uint32_t SMEM = MISC_OFF + MISC_BYTES + 1024;
    static_assert(SMEM <= 232448, "shared memory budget");
};

template <int C, bool CV>
struct StateMisc {
    static constexpr int NG = StateCfg<C, CV>::NG;
    float wk[NG][C];  // per group: 2^(lam - acs_j) per key
    float wtot[NG][4];
    uint64_t stage_full[StateCfg<C, CV>::STAGES], stage_empty[StateCfg<C, CV>::STAGES];
    uint64_t kp_full[NG], u_full[NG], u_free[NG];
    uint64_t drain;
    uint32_t tmem;
    int abort_flag;
};
static_assert(sizeof(StateMisc<128, false>) <= StateCfg<128, false>::MISC_BYTES, "misc block");
static_assert(sizeof(StateMisc<256, false>) <= StateCfg<256, false>::MISC_BYTES, "misc block");
static_assert(sizeof(StateMisc<128, true>) <= StateCfg<128, true>::MISC_BYTES, "misc block");

// Raw inputs and taps of the fused convolution (see ConvParams).
struct ConvTaps {
    const __nv_bfloat16 *x[3];
    const float *w[3], *bias[3];
    int width, silu;
};

// The causal depthwise convolution (+ SiLU) of one C-row bf16 tile, in place
// in the 128-byte swizzle of its TMA box.  Lane l of warp gw of the 128-thread
// group owns the 4-byte word l of each row (channels 2 l, 2 l + 1) in rows
// [gw C/4, (gw + 1) C/4), so a warp reads and writes whole rows.  Every thread
// first reads its taps and the three rows before its range (another warp's
// rows, or, for the first warp, the three tokens before the chunk from global
// memory: zero at the start of a head); after the group's barrier it walks its
// own rows in order, eight loads ahead, so every tap sees unconvolved values.
// The arithmetic is the standalone convolution's (bias, then one fused
// multiply-add per tap from j = 0, then silu_fast), so the two agree bit for
// bit.
template <int C>
__device__ __forceinline__ void conv_tile(uint8_t *tile, const __nv_bfloat16 *xraw, const float *w,
                                          const float *bias, int width, int silu, int h, bool head_start,
                                          size_t row0, int gt, int bar) {
    constexpr int R = C / 4;  // rows per warp
    const int wd = gt & 31, r0 = (gt >> 5) * R;
    auto word = [&](int r) {
        return reinterpret_cast<uint32_t *>(tile + r * kRowB + ((((wd >> 2) ^ (r & 7)) & 7) << 4) + (wd & 3) * 4);
    };
    uint32_t hb[3];  // rows r0 - 3, r0 - 2, r0 - 1
#pragma unroll
    for (int i = 0; i < 3; ++i) {
        const int r = r0 - 3 + i;
        if (r >= 0) {
            hb[i] = *word(r);
        } else if (!head_start) {
            hb[i] = __ldg(reinterpret_cast<const uint32_t *>(xraw + (row0 + r) * kD) + wd);
        } else {
            hb[i] = 0u;
        }
    }
    const int c = h * kD + 2 * wd;
    const float2 bs = bias ? make_float2(__ldg(bias + c), __ldg(bias + c + 1)) : make_float2(0.0f, 0.0f);
    float2 wr[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        wr[j] = j < width ? make_float2(__ldg(w + (size_t)c * width + j), __ldg(w + (size_t)(c + 1) * width + j))
                          : make_float2(0.0f, 0.0f);
    named_bar_sync(bar, kStateGroup);
    float2 x1 = bf2_to_f2(hb[2]), x2 = bf2_to_f2(hb[1]), x3 = bf2_to_f2(hb[0]);  // x[r-1], x[r-2], x[r-3]
#pragma unroll 1
    for (int i0 = 0; i0 < R; i0 += 8) {
        uint32_t xs[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) xs[k] = *word(r0 + i0 + k);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float2 xc = bf2_to_f2(xs[k]);
            float2 acc = __ffma2_rn(wr[0], xc, bs);
            if (width > 1) acc = __ffma2_rn(wr[1], x1, acc);
            if (width > 2) acc = __ffma2_rn(wr[2], x2, acc);
            if (width > 3) acc = __ffma2_rn(wr[3], x3, acc);
            if (silu) acc = make_float2(silu_fast(acc.x), silu_fast(acc.y));
            *word(r0 + i0 + k) = pack_bf16x2(acc.x, acc.y);
            x3 = x2;
            x2 = x1;
            x1 = xc;
        }
    }
    fence_proxy_async_smem();  // the TMA store of the tile and the MMA read it
}

template <int C, bool CV>
__global__ void __launch_bounds__(StateCfg<C, CV>::THREADS, 1)
chunk_state_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_xq,
                   const __grid_constant__ CUtensorMap tm_sq, const __grid_constant__ CUtensorMap tm_sk,
                   const __grid_constant__ CUtensorMap tm_sv, const ConvTaps cv,
                   const float *__restrict__ dt_p, const float *__restrict__ A_log,
                   const float *__restrict__ dt_bias, const float *__restrict__ log_decay, int value_dt,
                   int H, int N, int n_chunks, float *__restrict__ acs_out, float *__restrict__ vfac_out,
                   __nv_bfloat16 *__restrict__ Ut, float *__restrict__ lam_out, DeviceStatus *status, int dbg_skip,
                   unsigned long long wait_ns) {
    using K = StateCfg<C, CV>;
    constexpr int NG = K::NG;
    constexpr int KP = C / 128;  // keys per thread in the decay scan
    pdl_launch_dependents();  // the state pass waits for this grid before it reads anything
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    StateMisc<C, CV> *misc = reinterpret_cast<StateMisc<C, CV> *>(smem + K::MISC_OFF);
    const volatile int *abort_flag = &misc->abort_flag;
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nc = N / C;

    if (tid == 0) {
        if (blockIdx.x == 0 && status) {
            status->code = 0;
            status->detail = 0;
        }
        for (int i = 0; i < K::STAGES; ++i) {
            mbar_init(&misc->stage_full[i], 1);
            // released by the U product (tcgen05.commit) and by the compute group
            // once U^T, staged over K', has been stored
            mbar_init(&misc->stage_empty[i], 2);
        }
        for (int b = 0; b < NG; ++b) {
            mbar_init(&misc->kp_full[b], kStateGroup);
            mbar_init(&misc->u_full[b], 1);
            mbar_init(&misc->u_free[b], kStateGroup);
        }
        mbar_init(&misc->drain, 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc->tmem, 64 * NG);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            prefetch_tmap(&tm_u);
            if (CV) {
                prefetch_tmap(&tm_xq);
                prefetch_tmap(&tm_sq);
                prefetch_tmap(&tm_sk);
                prefetch_tmap(&tm_sv);
            }
            int i = 0;
            for (int t = blockIdx.x; t < n_chunks; t += gridDim.x, ++i) {
                const int st = i % K::STAGES;
                if (i >= K::STAGES &&
                    !mbar_wait_abortable(&misc->stage_empty[st], ((i / K::STAGES) - 1) & 1, abort_flag, wait_ns)) {
                    set_timeout(status, 100, &misc->abort_flag);
                    break;
                }
                if (i == dbg_skip) continue;  // failure test: this step is never published
                const int row = t * C;  // chunks are contiguous row blocks of [B H N, d]
                uint8_t *sp = smem + st * K::STAGE;
                mbar_arrive_expect_tx(&misc->stage_full[st], K::STAGE);
#pragma unroll
                for (int b = 0; b < C / 128; ++b) {
                    tma_load_2d(sp + b * kBox, &tm_k, 0, row + 128 * b, &misc->stage_full[st]);
                    tma_load_2d(sp + K::TILE + b * kBox, &tm_v, 0, row + 128 * b, &misc->stage_full[st]);
                    if (CV) tma_load_2d(sp + 2 * K::TILE + b * kBox, &tm_xq, 0, row + 128 * b, &misc->stage_full[st]);
                }
            }
            for (int j = i > K::STAGES ? i - K::STAGES : 0; j < i; ++j)
                if (j != dbg_skip) mbar_wait_bounded(&misc->stage_full[j % K::STAGES], (j / K::STAGES) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idU = make_idesc_bf16(64, 64, 1, 1);
            bool ok = true;
            int i = 0;
            for (int t = blockIdx.x; t < n_chunks; t += gridDim.x, ++i) {
                const int st = i % K::STAGES, ub = i % NG, use = i / NG;
                if (!(ok = mbar_wait_abortable(&misc->kp_full[ub], use & 1, abort_flag, wait_ns))) break;
                if (use >= 1 && !(ok = mbar_wait_abortable(&misc->u_free[ub], (use - 1) & 1, abort_flag, wait_ns))) break;
                tc_fence_after();
                const uint32_t sp = sbase + st * K::STAGE;
                const uint32_t kp = sp + (CV ? 2 * K::TILE : 0u);  // K' (in the Q slot with the convolution)
                // D[n][k] = sum_j v_jn k'_jk: A = V (MN-major), B = K' (MN-major)
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tmem + 64 * ub, desc_mn(sp + K::TILE + ks * 2048), desc_mn(kp + ks * 2048), idU,
                             ks > 0);
                mma_commit(&misc->u_full[ub]);
                mma_commit(&misc->stage_empty[st]);
            }
            if (!ok) {
                set_timeout(status, 101, &misc->abort_flag);
                mma_commit(&misc->drain);
                mbar_wait_bounded(&misc->drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------ compute groups
        const int gi = (warp - 2) >> 2;      // group: chunks i with i % NG == gi
        const int gt = (tid - 64) & 127;     // thread in the group
        const int gw = gt >> 5;              // warp in the group
        const int g = warp & 3;              // TMEM lane quarter
        const uint32_t lane_off = (uint32_t)(g * 32) << 16;
        const int bar = 1 + gi;
        bool failed = false;

        // raw inputs of a chunk, fetched one chunk ahead: dt projections (when
        // dt is used), given log-decays (when given), A_log and dt_bias
        struct Raw {
            float dt[KP], ld[KP], alog, bias;
        };
        auto fetch = [&](int t) -> Raw {
            Raw x;
#pragma unroll
            for (int e = 0; e < KP; ++e) x.dt[e] = x.ld[e] = 0.0f;
            x.alog = x.bias = 0.0f;
            if (t >= n_chunks) return x;
            const int h = (t / nc) % H;
            if (A_log) x.alog = __ldg(A_log + h);
            if (dt_bias) x.bias = __ldg(dt_bias + h);
#pragma unroll
            for (int e = 0; e < KP; ++e) {
                if (dt_p) x.dt[e] = __ldg(dt_p + (size_t)t * C + KP * gt + e);
                if (log_decay) x.ld[e] = __ldg(log_decay + (size_t)t * C + KP * gt + e);
            }
            return x;
        };

        int i = gi;
        Raw raw_next = fetch(blockIdx.x + gi * gridDim.x);
        for (int t = blockIdx.x + gi * gridDim.x; t < n_chunks; t += NG * gridDim.x, i += NG) {
            const int st = i % K::STAGES, use = i / NG;
            const Raw raw = raw_next;
            raw_next = fetch(t + NG * gridDim.x);
            // ---- decay: inclusive scan of A dt over the chunk (log2 units)
            const float A2 = -expf(raw.alog) * kLog2e;
            float a[KP], vf[KP];
            float run = 0.0f;
#pragma unroll
            for (int e = 0; e < KP; ++e) {
                const float dt = (value_dt || !log_decay) ? softplus_f(raw.dt[e] + raw.bias) : 0.0f;
                // one explicit fused multiply-add, so every instantiation of
                // this kernel rounds the decay the same way
                run = log_decay ? fmaf(raw.ld[e], kLog2e, run) : fmaf(A2, dt, run);
                a[e] = run;
                vf[e] = value_dt ? dt : 1.0f;
            }
            float incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            if (lane == 31) misc->wtot[gi][gw] = incl;
            named_bar_sync(bar, kStateGroup);
            float pre = incl - run, lam = 0.0f;
#pragma unroll
            for (int ww = 0; ww < 4; ++ww) {
                const float x = misc->wtot[gi][ww];
                if (ww < gw) pre += x;
                lam += x;
            }
#pragma unroll
            for (int e = 0; e < KP; ++e) {
                const float acs = pre + a[e];
                acs_out[(size_t)t * C + KP * gt + e] = acs;
                if (value_dt) vfac_out[(size_t)t * C + KP * gt + e] = vf[e];
                misc->wk[gi][KP * gt + e] = ex2_approx(lam - acs) * vf[e];
            }
            if (gt == 0) lam_out[t] = lam;
            // ---- K'_j = 2^(lam - acs_j) k_j in place: eight lanes per 128-byte row
            bool bad = !mbar_wait_abortable(&misc->stage_full[st], (i / K::STAGES) & 1, abort_flag, wait_ns);
            if (named_bar_any(bar, kStateGroup, bad)) {  // also publishes wk[]
                failed = true;
                break;
            }
            uint8_t *sk = smem + st * K::STAGE;
            uint8_t *skp = sk;  // K'
            if constexpr (CV) {
                // q, k, v = SiLU(conv(x)) in place; each tile goes to the
                // workspace as soon as it is complete (one bulk group per tile)
                uint8_t *sv = sk + K::TILE, *sq = sk + 2 * K::TILE;
                const int h = (t / nc) % H;
                const bool head_start = (t % nc) == 0;
                const size_t row0 = (size_t)t * C;
                conv_tile<C>(sq, cv.x[0], cv.w[0], cv.bias[0], cv.width, cv.silu, h, head_start, row0, gt, bar);
                conv_tile<C>(sk, cv.x[1], cv.w[1], cv.bias[1], cv.width, cv.silu, h, head_start, row0, gt, bar);
                if (gt == 0) {  // every thread's q rows are final (the barrier inside the k tile's pass)
#pragma unroll
                    for (int b = 0; b < C / 128; ++b) tma_store_2d(&tm_sq, sq + b * kBox, 0, t * C + 128 * b);
                    bulk_commit_group();
                }
                conv_tile<C>(sv, cv.x[2], cv.w[2], cv.bias[2], cv.width, cv.silu, h, head_start, row0, gt, bar);
                named_bar_sync(bar, kStateGroup);
                if (gt == 0) {
#pragma unroll
                    for (int b = 0; b < C / 128; ++b) {
                        tma_store_2d(&tm_sk, sk + b * kBox, 0, t * C + 128 * b);
                        tma_store_2d(&tm_sv, sv + b * kBox, 0, t * C + 128 * b);
                    }
                    bulk_commit_group();
                    bulk_wait_group_read<1>();  // the q tile has been read: K' may overwrite it
                }
                named_bar_sync(bar, kStateGroup);
                skp = sq;
            }
#pragma unroll 4
            for (int it = 0; it < C / 16; ++it) {
                const int j = it * 16 + (gt >> 3);
                const float wj = misc->wk[gi][j];
                const float2 w2 = make_float2(wj, wj);
                const uint4 x = *(reinterpret_cast<const uint4 *>(sk + j * kRowB) + (gt & 7));
                uint32_t wv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f = __fmul2_rn(bf2_to_f2(wv[q]), w2);
                    wv[q] = pack_bf16x2(f.x, f.y);
                }
                *(reinterpret_cast<uint4 *>(skp + j * kRowB) + (gt & 7)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&misc->kp_full[gi]);
            // ---- U^T epilogue: rows 16 g + lane (lanes 0-15) of the M = 64 accumulator
            bad = !mbar_wait_abortable(&misc->u_full[gi], use & 1, abort_flag, wait_ns);
            if (named_bar_any(bar, kStateGroup, bad)) {
                failed = true;
                break;
            }
            tc_fence_after();
            float v0[32], v1[32];
            tmem_ld32(tmem + lane_off + 64 * gi, v0);
            tmem_ld32(tmem + lane_off + 64 * gi + 32, v1);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&misc->u_free[gi]);
            // U^T rows n = 16 g + lane, rounded to bf16 and staged over K' (read
            // by the finished product) as one 64 x 64 box in the 128-byte swizzle
            if (lane < 16) {
                const int n = g * 16 + lane;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float *v = q < 4 ? v0 + 8 * q : v1 + 8 * (q - 4);
                    *reinterpret_cast<uint4 *>(skp + sw128_chunk(n, q)) =
                        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                   pack_bf16x2(v[6], v[7]));
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(bar, kStateGroup);
            if (gt == 0) {
                tma_store_2d(&tm_u, skp, 0, t * 64);
                bulk_commit_group();
                bulk_wait_group_read0();
                mbar_arrive(&misc->stage_empty[st]);
            }
        }
        if (gt == 0) bulk_wait_group0();  // every U^T tile has reached global memory
        if (failed && gt == 0) set_timeout(status, 102, &misc->abort_flag);
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 64 * NG);
}

// =====================================================================
// (2) state passing: one thread per 4 state entries of a head
// =====================================================================
constexpr int kPassBatch = 16;  // chunks whose inputs are in flight at once
__global__ void __launch_bounds__(256)
state_pass_kernel(const __nv_bfloat16 *__restrict__ U, const float *__restrict__ lam, __nv_bfloat16 *__restrict__ hin,
                  int nc, const float *__restrict__ h0, float *__restrict__ h_out) {
    pdl_launch_dependents();  // the chunk scan waits for this grid before it reads hin
    pdl_wait();               // U and lam of the chunk-state kernel
    const int bh = blockIdx.x;
    const int e = (blockIdx.y * 256 + threadIdx.x) * 4;  // 4 consecutive entries of the 64 x 64 state
    const uint2 *u = reinterpret_cast<const uint2 *>(U + (size_t)bh * nc * 4096 + e);
    uint2 *out = reinterpret_cast<uint2 *>(hin + (size_t)bh * nc * 4096 + e);
    const float *lm = lam + (size_t)bh * nc;
    // the state carried into the sequence (h0 is [k][n]; this thread holds
    // entries (n, k..k+3) of the transposed state)
    const int n_ = e / 64, k_ = e % 64;
    float4 hs = make_float4(0.f, 0.f, 0.f, 0.f);
    if (h0) {
        const float *hp = h0 + (size_t)bh * 4096 + (size_t)k_ * 64 + n_;
        hs = make_float4(hp[0], hp[64], hp[128], hp[192]);
    }
    // 16 chunks' inputs (bf16 U, 8 bytes a thread) are in flight before the
    // dependent updates run: a head of up to 16 chunks costs one L2 round trip
    for (int c0 = 0; c0 < nc; c0 += kPassBatch) {
        uint2 ub[kPassBatch];
        float fb[kPassBatch];
#pragma unroll
        for (int j = 0; j < kPassBatch; ++j) {
            if (c0 + j < nc) {
                ub[j] = __ldg(u + (size_t)(c0 + j) * 1024);
                fb[j] = __ldg(lm + c0 + j);
            }
        }
#pragma unroll
        for (int j = 0; j < kPassBatch; ++j) {
            if (c0 + j < nc) {
                const float f = ex2_approx(fb[j]);
                out[(size_t)(c0 + j) * 1024] = make_uint2(pack_bf16x2(hs.x, hs.y), pack_bf16x2(hs.z, hs.w));
                const float2 u01 = bf2_to_f2(ub[j].x), u23 = bf2_to_f2(ub[j].y);
                hs.x = fmaf(f, hs.x, u01.x);
                hs.y = fmaf(f, hs.y, u01.y);
                hs.z = fmaf(f, hs.z, u23.x);
                hs.w = fmaf(f, hs.w, u23.y);
            }
        }
    }
    if (h_out) {
        float *hp = h_out + (size_t)bh * 4096 + (size_t)k_ * 64 + n_;
        hp[0] = hs.x;
        hp[64] = hs.y;
        hp[128] = hs.z;
        hp[192] = hs.w;
    }
}

// =====================================================================
// (3) chunk scan: persistent, warp-specialised
//   warp 0: TMA producer.
//   warp 1: MMA issuer.  It polls its barriers and issues whichever product
//     is ready: S' = Q [K ; hin^T]^T (scores and the state readout Z = Q hin
//     in one N = 192 product), or Y = P V with P read from TMEM.
//   NG compute groups of 8 warps (two for C = 128, one for C = 256) taking
//     tiles round-robin: P from S (written back to TMEM as bf16), then the
//     epilogue of the same tile.
// Keeping P in TMEM and reading Q once for both S and Z roughly halves the
// shared-memory operand traffic of the tensor core, which bounds this kernel.
// =====================================================================
template <int C>
struct ScanCfg {
    static constexpr int NG = C == 128 ? 2 : 1;      // compute groups
    static constexpr int THREADS = 64 + 256 * NG;
    static constexpr int NKB = C / 128;              // 128-key blocks per chunk
    static constexpr int NRB = C / 128;              // 128-row tiles per chunk
    static constexpr int NSB = C == 128 ? 2 : 1;     // S' buffers in TMEM
    static constexpr int STAGES = C == 128 ? 3 : 2;
    // Per stage: Q | K slots (NKB boxes) | hin^T (64 rows) | V slots (NKB boxes).
    // The last K slot is followed directly by hin^T, so [K ; hin^T] is one
    // B operand of 192 rows.  A tile with nkb key blocks puts key block kb in
    // K slot NKB - nkb + kb.
    static constexpr uint32_t Q_OFF = 0;
    static constexpr uint32_t K_OFF = kBox;
    static constexpr uint32_t H_OFF = K_OFF + NKB * kBox;
    static constexpr uint32_t V_OFF = H_OFF + kHinBytes;
    static constexpr uint32_t STAGE = V_OFF + NKB * kBox;
    // C = 256 (two stages) stages each group's output tile in a slot of its
    // own, so that a stage is free as soon as its P V product completes;
    // C = 128 (three stages) stages it over the stage's Q box, which keeps
    // the residual rows at hand in the stage's V box.
    static constexpr bool OUT_SLOT = C == 256;
    // C = 256 (one compute group): the group runs tile i's P and then tile
    // i - 1's epilogue, so each tile's P V completes behind the next tile's
    // P; Z then lives in a TMEM slot per tile parity (see below)
    static constexpr bool PIPE = C == 256;
    static constexpr uint32_t Y_OFF = STAGES * STAGE;
    static constexpr uint32_t MISC_OFF = Y_OFF + (OUT_SLOT ? NG * kBox : 0);
    static constexpr uint32_t MISC_BYTES = 28 * NG * C + 1024;
    static constexpr uint32_t SMEM = MISC_OFF + MISC_BYTES + 1024;
    // TMEM: C = 128: S' buffers at 0 and 192 (keys at +0, Z at +128);
    //       C = 256: keys k at 128 (2 - nkb) + k, Z of tile j at 256 + 64 (j % 2)
    //       (a product of its own: the next tile's scores need only this
    //       tile's P V done, not its epilogue).  Y buffers at 384, 448.
    static constexpr uint32_t COL_Y = 384;
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(STAGE % 1024 == 0, "stage alignment");
};

// Per group, two alternating tile slots: a thread may write its group's next
// tile's entries while a slower one still reads the current tile's.
template <int C>
struct ScanMisc {
    static constexpr int NG = ScanCfg<C>::NG;
    float acs[NG][2][C];
    float colf[NG][2][C];   // 2^(acs_r - acs_j) f_j, r the last key of j's 32-key block
    float vf[NG][2][C];     // value factor f_j of key j (dt_j, or 1)
    float dres[NG][2][64];  // D of the tile's head
    uint64_t stage_full[ScanCfg<C>::STAGES], stage_empty[ScanCfg<C>::STAGES];
    uint64_t s_full[ScanCfg<C>::NSB], p_full[NG][ScanCfg<C>::NKB], y_full[2], ep_done[2];
    uint64_t drain;
    uint32_t tmem;
    int abort_flag;
};
static_assert(sizeof(ScanMisc<128>) <= ScanCfg<128>::MISC_BYTES, "misc block");
static_assert(sizeof(ScanMisc<256>) <= ScanCfg<256>::MISC_BYTES, "misc block");

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
// TMEM column of key 0 of a tile's scores, and of its state readout Z
template <int C>
__device__ __forceinline__ uint32_t key_col(int sb, int nkb) {
    return C == 128 ? (uint32_t)sb * 192u : 128u * (uint32_t)(2 - nkb);
}
template <int C>
__device__ __forceinline__ uint32_t z_col(int sb, int j) {
    return C == 128 ? (uint32_t)sb * 192u + 128u : 256u + 64u * (uint32_t)(j & 1);
}

template <int C>
__global__ void __launch_bounds__(ScanCfg<C>::THREADS, 1)
chunk_scan_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_h,
                  const __grid_constant__ CUtensorMap tm_out, const __nv_bfloat16 *__restrict__ vglob,
                  const float *__restrict__ acs_in, const float *__restrict__ vfac_in,
                  const float *__restrict__ Dres, int H, int N, int n_tiles, DeviceStatus *status, int dbg_skip,
                  unsigned long long wait_ns) {
    using K = ScanCfg<C>;
    constexpr int NG = K::NG;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    ScanMisc<C> *misc = reinterpret_cast<ScanMisc<C> *>(smem + K::MISC_OFF);
    const volatile int *abort_flag = &misc->abort_flag;
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nc = N / C;
    // number of tiles this CTA processes
    // a contiguous range of tiles per CTA: the row blocks of a chunk (and the
    // chunks of a head) follow one another on one SM, so key blocks a later
    // tile shares with an earlier one are still in L2
    const int tile0 = (int)((long long)blockIdx.x * n_tiles / gridDim.x);
    const int my_tiles = (int)((long long)(blockIdx.x + 1) * n_tiles / gridDim.x) - tile0;

    if (tid == 0) {
        for (int i = 0; i < K::STAGES; ++i) {
            mbar_init(&misc->stage_full[i], 1);
            // released by the P V product (tcgen05.commit) and, with the output
            // staged over Q, by the compute group once that tile has been stored
            mbar_init(&misc->stage_empty[i], K::OUT_SLOT ? 1 : 2);
        }
        for (int i = 0; i < K::NSB; ++i) mbar_init(&misc->s_full[i], 1);
        for (int gi = 0; gi < NG; ++gi)
            for (int kb = 0; kb < K::NKB; ++kb) mbar_init(&misc->p_full[gi][kb], 256);
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
            prefetch_tmap(&tm_out);
            pdl_wait();  // hin (state pass) and everything before it are visible
            int i = 0;
            for (; i < my_tiles; ++i) {
                const int t = tile0 + i;
                const int st = i % K::STAGES;
                if (i >= K::STAGES &&
                    !mbar_wait_abortable(&misc->stage_empty[st], ((i / K::STAGES) - 1) & 1, abort_flag, wait_ns)) {
                    set_timeout(status, 110, &misc->abort_flag);
                    break;
                }
                if (i == dbg_skip) continue;  // failure test: this step is never published
                const TileIdx x = tile_idx<C>(t, nc);
                const int nkb = x.rb + 1;
                const int crow = x.bh * N + x.c * C;
                uint8_t *sp = smem + st * K::STAGE;
                mbar_arrive_expect_tx(&misc->stage_full[st], kBox + kHinBytes + 2 * nkb * kBox);
                tma_load_2d(sp + K::Q_OFF, &tm_q, 0, crow + 128 * x.rb, &misc->stage_full[st]);
                for (int kb = 0; kb < nkb; ++kb) {
                    tma_load_2d(sp + K::K_OFF + (K::NKB - nkb + kb) * kBox, &tm_k, 0, crow + 128 * kb,
                                &misc->stage_full[st]);
                    tma_load_2d(sp + K::V_OFF + kb * kBox, &tm_v, 0, crow + 128 * kb, &misc->stage_full[st]);
                }
                tma_load_2d(sp + K::H_OFF, &tm_h, 0, (x.bh * nc + x.c) * 64, &misc->stage_full[st]);
            }
            // copies still in flight after an abort land before the CTA exits (bounded)
            for (int j = i > K::STAGES ? i - K::STAGES : 0; j < i; ++j)
                if (j != dbg_skip) mbar_wait_bounded(&misc->stage_full[j % K::STAGES], (j / K::STAGES) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS128 = make_idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idS192 = make_idesc_bf16(128, 192, 0, 0);
            constexpr uint32_t idZ = make_idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t idO = make_idesc_bf16(128, 64, 0, 1);
            uint32_t np[NG][K::NKB];
            for (int gi = 0; gi < NG; ++gi)
                for (int kb = 0; kb < K::NKB; ++kb) np[gi][kb] = 0;
            int next_s = 0, next_pv = 0, pv_kb = 0;
            bool ok = true;
            uint64_t idle_since = globaltimer_ns();
            uint32_t spins = 0;
            while (next_pv < my_tiles) {
                bool progress = false;
                // ---- Y = P V for tile next_pv, one 128-key block at a time
                if (next_pv < next_s) {
                    const int i = next_pv, gi = i % NG, tb = i & 1, st = i % K::STAGES;
                    const TileIdx x = tile_idx<C>(tile0 + i, nc);
                    const int nkb = x.rb + 1;
                    if (mbar_test(&misc->p_full[gi][pv_kb], np[gi][pv_kb] & 1)) {
                        ++np[gi][pv_kb];
                        tc_fence_after();
                        const uint32_t sp = sbase + st * K::STAGE;
                        const uint32_t pcol = key_col<C>(i % K::NSB, nkb) + 128 * pv_kb;
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks)
                            mma_bf16_ts(tmem + K::COL_Y + tb * 64, tmem + pcol + 64 * (ks >> 2) + 8 * (ks & 3),
                                        desc_mn(sp + K::V_OFF + pv_kb * kBox + ks * 2048), idO,
                                        (pv_kb > 0 || ks > 0));
                        if (++pv_kb == nkb) {
                            mma_commit(&misc->y_full[tb]);
                            mma_commit(&misc->stage_empty[st]);
                            ++next_pv;
                            pv_kb = 0;
                        }
                        progress = true;
                    }
                }
                // ---- S' for tile next_s.  C = 128: its TMEM buffer is free once
                // tile next_s - NSB is done.  C = 256: the key columns once the
                // previous tile's P V is done, its Z slot once tile next_s - 2 is.
                if (next_s < my_tiles) {
                    const int j = next_s, st = j % K::STAGES;
                    const int jp = j - K::NSB;  // previous user of the S' buffer
                    const bool buf_free =
                        !K::PIPE ? (jp < 0 || mbar_test(&misc->ep_done[jp & 1], (jp >> 1) & 1))
                                 : ((j < 1 || mbar_test(&misc->y_full[(j - 1) & 1], ((j - 1) >> 1) & 1)) &&
                                    (j < 2 || mbar_test(&misc->ep_done[j & 1], ((j - 2) >> 1) & 1)));
                    if (buf_free && mbar_test(&misc->stage_full[st], (j / K::STAGES) & 1)) {
                        tc_fence_after();
                        const TileIdx x = tile_idx<C>(tile0 + j, nc);
                        const int nkb = x.rb + 1;
                        const int sb = j % K::NSB;
                        const uint32_t sp = sbase + st * K::STAGE;
                        const uint32_t kc = key_col<C>(sb, nkb);
                        if (nkb == 2) {
                            // keys [0, 128) of a 256-key row block: plain scores from K slot 0
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_bf16(tmem + kc, desc_k(sp + K::Q_OFF + ks * 32), desc_k(sp + K::K_OFF + ks * 32),
                                         idS128, ks > 0);
                        }
                        const uint32_t kl = sp + K::K_OFF + (K::NKB - 1) * kBox;
                        if (!K::PIPE) {
                            // last key block and the state readout: B = [K slot NKB - 1 ; hin^T]
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_bf16(tmem + kc + 128 * (nkb - 1), desc_k(sp + K::Q_OFF + ks * 32),
                                         desc_k(kl + ks * 32), idS192, ks > 0);
                        } else {
                            // last key block, then the state readout into the tile's Z slot
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_bf16(tmem + kc + 128 * (nkb - 1), desc_k(sp + K::Q_OFF + ks * 32),
                                         desc_k(kl + ks * 32), idS128, ks > 0);
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                mma_bf16(tmem + z_col<C>(sb, j), desc_k(sp + K::Q_OFF + ks * 32),
                                         desc_k(sp + K::H_OFF + ks * 32), idZ, ks > 0);
                        }
                        mma_commit(&misc->s_full[sb]);
                        ++next_s;
                        progress = true;
                    }
                }
                if (progress) {
                    idle_since = 0;
                    spins = 0;
                } else {
                    __nanosleep(32);  // nothing ready: leave the issue slots to the compute groups
                }
                if (!progress && (++spins & 63u) == 0) {
                    const uint64_t now = globaltimer_ns();
                    if (idle_since == 0) idle_since = now;
                    if (*abort_flag || now - idle_since > wait_ns) {
                        ok = false;
                        break;
                    }
                }
            }
            if (!ok) {
                set_timeout(status, 120, &misc->abort_flag);
                // products still in flight finish before TMEM is released (bounded)
                mma_commit(&misc->drain);
                mbar_wait_bounded(&misc->drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------ compute groups
        const int gi = (warp - 2) >> 3;    // group: tiles i with i % NG == gi
        const int ct = (tid - 64) & 255;   // thread in the group; key ct of the tile
        const int gw = ct >> 5;            // warp in the group
        const int g = warp & 3;            // TMEM lane quarter
        const int hf = gw >> 2;            // half of the columns
        const uint32_t lane_off = (uint32_t)(g * 32) << 16;
        const int r = g * 32 + lane;       // row of the 128-row tile
        const int bar = 1 + gi;

        // Raw inputs of a tile, fetched one tile ahead: acs of key ct and four entries of D.
        struct Raw {
            float acs, vf;
            float4 d;
        };
        auto fetch = [&](int i) -> Raw {
            Raw x{0.0f, 1.0f, make_float4(0.f, 0.f, 0.f, 0.f)};
            if (i >= my_tiles) return x;
            const TileIdx ti = tile_idx<C>(tile0 + i, nc);
            if (ct < 128 * (ti.rb + 1)) {
                const size_t key = (size_t)ti.bh * N + (size_t)ti.c * C + ct;
                x.acs = __ldg(acs_in + key);
                if (vfac_in) x.vf = __ldg(vfac_in + key);
            }
            if (Dres && ct < 16) x.d = __ldg(reinterpret_cast<const float4 *>(Dres + (ti.bh % H) * kD) + ct);
            return x;
        };

        bool failed = false;
        int pend_st = -1;  // thread ct = 0: stage of an output store not yet waited for
        auto epilogue = [&](int j) -> bool {
            const TileIdx x = tile_idx<C>(tile0 + j, nc);
            const int sb = j % K::NSB, tb = j & 1, slot = (j / NG) & 1;
            const int ir = 128 * x.rb + r;
            uint8_t *sp = smem + (j % K::STAGES) * K::STAGE;
            const float ai = misc->acs[gi][slot][ir];
        // ---- epilogue of tile j: y = Y + 2^acs_i Z [+ D v], columns [32 hf, 32 hf + 32)
            // With an output slot the stage may be refilled once P V completes,
            // so the residual rows v_i (still in L2) are fetched from global
            // memory while P V runs; otherwise they are read from the V box.
            uint4 vres[4] = {};
            if (K::OUT_SLOT && Dres) {
                const uint4 *vp = reinterpret_cast<const uint4 *>(
                                      vglob + ((size_t)x.bh * N + (size_t)x.c * C + 128 * x.rb + r) * kD) +
                                  4 * hf;
#pragma unroll
                for (int q = 0; q < 4; ++q) vres[q] = __ldg(vp + q);
            }
            bool bad = !mbar_wait_abortable(&misc->y_full[tb], (j >> 1) & 1, abort_flag, wait_ns);
            // the V box is read below: observe the stage's TMA completion here too
            // (long complete; the stage cannot be refilled before this group releases it)
            if (!K::OUT_SLOT)
                bad = bad || !mbar_wait_abortable(&misc->stage_full[j % K::STAGES], (j / K::STAGES) & 1, abort_flag, wait_ns);
            if (named_bar_any(bar, 256, bad)) return false;
            tc_fence_after();
            const float e = ex2_approx(ai);
            const float *dh = &misc->dres[gi][slot][hf * 32];
            // residual v_i: row r of V box rb (this tile's own tokens).  y is
            // staged in the swizzled layout of the TMA store, over Q (dead since
            // S' completed) or in the group's slot, whose previous store was
            // read before this group signalled P of this tile complete.
            const uint8_t *vrow = sp + K::V_OFF + x.rb * kBox;
            uint8_t *ytile = K::OUT_SLOT ? smem + K::Y_OFF + gi * kBox : sp + K::Q_OFF;
            const uint32_t zc = tmem + lane_off + z_col<C>(sb, j) + 32 * hf;
            const uint32_t yc = tmem + lane_off + K::COL_Y + 64 * tb + 32 * hf;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float yv[16], zv[16];
                tmem_ld16(yc + 16 * half, yv);
                tmem_ld16(zc + 16 * half, zv);
                tmem_wait_ld();
                if (half == 1) {
                    tc_fence_before();
                    mbar_arrive(&misc->ep_done[tb]);
                }
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    const int q = 2 * half + q2;
                    uint32_t wv[4];
                    uint4 vq = vres[q];
                    if (!K::OUT_SLOT && Dres) vq = *reinterpret_cast<const uint4 *>(vrow + sw128_chunk(r, 4 * hf + q));
                    const uint32_t vw[4] = {vq.x, vq.y, vq.z, vq.w};
#pragma unroll
                    for (int pp = 0; pp < 4; ++pp) {
                        const int cl = q2 * 8 + 2 * pp;  // column within the half
                        float y0 = fmaf(e, zv[cl], yv[cl]);
                        float y1 = fmaf(e, zv[cl + 1], yv[cl + 1]);
                        if (Dres) {
                            const float2 vf = bf2_to_f2(vw[pp]);
                            y0 = fmaf(dh[16 * half + cl], vf.x, y0);
                            y1 = fmaf(dh[16 * half + cl + 1], vf.y, y1);
                        }
                        wv[pp] = pack_bf16x2(y0, y1);
                    }
                    *reinterpret_cast<uint4 *>(ytile + sw128_chunk(r, 4 * hf + q)) =
                        make_uint4(wv[0], wv[1], wv[2], wv[3]);
                }
            }
            // one TMA store per tile; its read of the tile (and, staged over Q,
            // the stage's release) is settled before the group's next S
            fence_proxy_async_smem();
            named_bar_sync(bar, 256);
            if (ct == 0) {
                tma_store_2d(&tm_out, ytile, 0, x.bh * N + x.c * C + 128 * x.rb);
                bulk_commit_group();
                pend_st = j % K::STAGES;
            }
            return true;
        };

        pdl_wait();  // acs (chunk-state kernel) is visible
        Raw raw_next = fetch(gi);
        for (int i = gi; i < my_tiles; i += NG) {
            const TileIdx x = tile_idx<C>(tile0 + i, nc);
            const int nkb = x.rb + 1;
            const int sb = i % K::NSB, slot = (i / NG) & 1;
            const Raw raw = raw_next;
            raw_next = fetch(i + NG);
            const int ir = 128 * x.rb + r;  // chunk-local row
            uint8_t *sp = smem + (i % K::STAGES) * K::STAGE;
            if (Dres && ct < 16) *reinterpret_cast<float4 *>(&misc->dres[gi][slot][4 * ct]) = raw.d;
            // chunk-local cumulative decay of key ct, and its factor to the end of its 32-key block
            const float aref = __shfl_sync(0xffffffffu, raw.acs, 31);
            if (ct < C) {
                misc->acs[gi][slot][ct] = raw.acs;
                misc->colf[gi][slot][ct] = ex2_approx(aref - raw.acs) * raw.vf;
                misc->vf[gi][slot][ct] = raw.vf;
            }
            // ---- the group's previous output store: its read of shared memory is
            // waited for here, where the group waits for S anyway, rather than
            // right after the store, which held the whole group at its next barrier
            if (ct == 0 && pend_st >= 0) {
                bulk_wait_group_read0();
                if (!K::OUT_SLOT) mbar_arrive(&misc->stage_empty[pend_st]);
                pend_st = -1;
            }
            // ---- S of this tile
            bool bad = !mbar_wait_abortable(&misc->s_full[sb], (i / K::NSB) & 1, abort_flag, wait_ns);
            if (named_bar_any(bar, 256, bad)) {  // also publishes acs[], colf[], dres[]
                failed = true;
                break;
            }
            tc_fence_after();
            const float *acs = misc->acs[gi][slot];
            const float ai = acs[ir];
            const int W32 = 4 * x.rb + g;  // 32-row block of this warp, chunk-local
            const uint32_t kc = key_col<C>(sb, nkb);
            for (int kb = 0; kb < nkb; ++kb) {
                // this warp reads S columns [64 hf, 64 hf + 64) of the key block and
                // writes their bf16 P over the first 32 of them (in order, so
                // nothing is overwritten before this warp has read it)
                const uint32_t cb = tmem + lane_off + kc + 128 * kb + 64 * hf;
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    const int q = 2 * hf + pc;   // 32-key piece of the 128-key block
                    const int P32 = 4 * kb + q;  // chunk-local 32-key block
                    const int k0 = 32 * P32;
                    uint32_t pk[16];
                    if (P32 > W32) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                    } else {
                        float sv[32];
                        tmem_ld32(cb + 32 * pc, sv);
                        tmem_wait_ld();
                        if (P32 < W32) {
                            const float rowf = ex2_approx(ai - acs[k0 + 31]);
                            const float2 rf2 = make_float2(rowf, rowf);
                            const float4 *cf = reinterpret_cast<const float4 *>(&misc->colf[gi][slot][k0]);
#pragma unroll
                            for (int e4 = 0; e4 < 8; ++e4) {
                                const float4 c4 = cf[e4];
                                const float2 p0 = __fmul2_rn(
                                    __fmul2_rn(make_float2(sv[4 * e4], sv[4 * e4 + 1]), make_float2(c4.x, c4.y)), rf2);
                                const float2 p1 = __fmul2_rn(
                                    __fmul2_rn(make_float2(sv[4 * e4 + 2], sv[4 * e4 + 3]), make_float2(c4.z, c4.w)),
                                    rf2);
                                pk[2 * e4] = pack_bf16x2(p0.x, p0.y);
                                pk[2 * e4 + 1] = pack_bf16x2(p1.x, p1.y);
                            }
                        } else {
                            const float4 *a4p = reinterpret_cast<const float4 *>(&acs[k0]);
                            const float4 *v4p = reinterpret_cast<const float4 *>(&misc->vf[gi][slot][k0]);
#pragma unroll
                            for (int e4 = 0; e4 < 8; ++e4) {
                                const float4 a4 = a4p[e4], v4 = v4p[e4];
                                const int j = k0 + 4 * e4;
                                const float2 f0 = __fmul2_rn(make_float2(ex2_approx(ai - a4.x), ex2_approx(ai - a4.y)),
                                                             make_float2(v4.x, v4.y));
                                const float2 f1 = __fmul2_rn(make_float2(ex2_approx(ai - a4.z), ex2_approx(ai - a4.w)),
                                                             make_float2(v4.z, v4.w));
                                float2 p0 = __fmul2_rn(make_float2(sv[4 * e4], sv[4 * e4 + 1]), f0);
                                float2 p1 = __fmul2_rn(make_float2(sv[4 * e4 + 2], sv[4 * e4 + 3]), f1);
                                if (j > ir) p0.x = 0.0f;
                                if (j + 1 > ir) p0.y = 0.0f;
                                if (j + 2 > ir) p1.x = 0.0f;
                                if (j + 3 > ir) p1.y = 0.0f;
                                pk[2 * e4] = pack_bf16x2(p0.x, p0.y);
                                pk[2 * e4 + 1] = pack_bf16x2(p1.x, p1.y);
                            }
                        }
                    }
                    tmem_st16(cb + 16 * pc, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&misc->p_full[gi][kb]);
            }
            if (!K::PIPE) {
                if (!epilogue(i)) {
                    failed = true;
                    break;
                }
            } else if (i - NG >= gi && !epilogue(i - NG)) {
                failed = true;
                break;
            }
        }
        // the last tile's epilogue (one tile behind)
        if (K::PIPE && !failed && my_tiles > gi && !epilogue(gi + (my_tiles - 1 - gi) / NG * NG)) failed = true;
        if (ct == 0) bulk_wait_group0();  // every output tile has reached global memory
        if (failed && ct == 0) set_timeout(status, 130, &misc->abort_flag);
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------- host side
// [rows, 64] bf16 row-major tensor read in boxes of `box_rows` rows, 128-byte swizzle.
bool make_tmap64(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
    return encode_tmap_2d(m, base, true, 64, rows, 64, box_rows, 128);
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

template <int C, bool CV>
int launch_c(const FwdArgs &a, const Plan &p) {
    using K = ScanCfg<C>;
    using SK = StateCfg<C, CV>;
    const int BH = a.B * a.H, nc = a.N / C;
    const uint64_t rows = (uint64_t)BH * a.N;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    DeviceStatus *status = reinterpret_cast<DeviceStatus *>(ws);
    float *lam = reinterpret_cast<float *>(ws + p.lam_off);
    float *acs = reinterpret_cast<float *>(ws + p.acs_off);
    float *vfac = a.value_dt ? reinterpret_cast<float *>(ws + p.vfac_off) : nullptr;
    __nv_bfloat16 *U = reinterpret_cast<__nv_bfloat16 *>(ws + p.state_off);
    __nv_bfloat16 *hin = reinterpret_cast<__nv_bfloat16 *>(ws + p.aux_off);
    CUtensorMap tq, tk, tv, th, to;
    if (!make_tmap64(&tq, a.q, rows, 128) || !make_tmap64(&tk, a.k, rows, 128) ||
        !make_tmap64(&tv, a.v, rows, 128) || !make_tmap64(&th, hin, (uint64_t)BH * nc * 64, 64) ||
        !make_tmap64(&to, a.out, rows, 128))
        return SSD_ERR_CUDA;
    CUtensorMap tu;
    if (!make_tmap64(&tu, U, (uint64_t)BH * nc * 64, 64)) return SSD_ERR_CUDA;
    // With the convolution fused, the chunk-state kernel reads the raw
    // activations and stores the convolved q, k, v (a.q, a.k, a.v, in the
    // workspace) through the scan's maps, which the scan then reads.
    CUtensorMap txq = tk, txk = tk, txv = tv;
    ConvTaps taps{};
    if (CV) {
        if (!make_tmap64(&txq, a.conv->x[0], rows, 128) || !make_tmap64(&txk, a.conv->x[1], rows, 128) ||
            !make_tmap64(&txv, a.conv->x[2], rows, 128))
            return SSD_ERR_CUDA;
        for (int i = 0; i < 3; ++i) {
            taps.x[i] = static_cast<const __nv_bfloat16 *>(a.conv->x[i]);
            taps.w[i] = a.conv->w[i];
            taps.bias[i] = a.conv->bias[i];
        }
        taps.width = a.conv->width;
        taps.silu = a.conv->silu;
    }
    static std::atomic<uint64_t> attr1{0}, attr3{0};
    if (!smem_attr_once(chunk_state_kernel<C, CV>, (int)SK::SMEM, attr1) ||
        !smem_attr_once(chunk_scan_kernel<C>, (int)K::SMEM, attr3))
        return SSD_ERR_CUDA;
    const int sms = num_sms();
    if (sms <= 0) return SSD_ERR_CUDA;

    const int n_chunks = BH * nc;
    const unsigned long long wait_ns = a.wait_ns ? a.wait_ns : 1000000000ull;
    chunk_state_kernel<C, CV><<<n_chunks < sms ? n_chunks : sms, SK::THREADS, SK::SMEM, a.stream>>>(
        txk, txv, tu, txq, tq, tk, tv, taps, a.dt_p, a.A_log, a.dt_bias, a.log_decay, a.value_dt, a.H, a.N,
        n_chunks, acs, vfac, U, lam, status, a.dbg_skip, wait_ns);
    // The state pass and the chunk scan are launched as programmatic dependents:
    // their CTAs may start while the previous kernel drains, and each waits
    // (griddepcontrol.wait) before it reads that kernel's results.
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t c2 = {};
    c2.gridDim = dim3(BH, 4);
    c2.blockDim = dim3(256);
    c2.stream = a.stream;
    c2.attrs = pdl;
    c2.numAttrs = 1;
    const cudaError_t e2 = cudaLaunchKernelEx(&c2, state_pass_kernel, (const __nv_bfloat16 *)U, (const float *)lam,
                                              hin, nc, a.h0, a.h_out);
    if (e2 != cudaSuccess)
        return SSD_ERR_CUDA;
    const int n_tiles = BH * nc * K::NRB;
    const int grid = n_tiles < sms ? n_tiles : sms;
    cudaLaunchConfig_t c3 = {};
    c3.gridDim = dim3(grid);
    c3.blockDim = dim3(K::THREADS);
    c3.dynamicSmemBytes = K::SMEM;
    c3.stream = a.stream;
    c3.attrs = pdl;
    c3.numAttrs = 1;
    if (cudaLaunchKernelEx(&c3, chunk_scan_kernel<C>, tq, tk, tv, th, to, (const __nv_bfloat16 *)a.v,
                           (const float *)acs, (const float *)vfac, a.D, a.H, a.N, n_tiles, status, a.dbg_skip,
                           wait_ns) != cudaSuccess)
        return SSD_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace

// The convolution prologue is fused at chunk 128.  At chunk 256 only two
// stages of raw q, k, v tiles fit in shared memory, and the convolution,
// which then runs on two groups per SM, outlasts the loads: there the
// standalone convolution followed by the operator is faster.
bool tc_order1_fuses_conv(int chunk) { return chunk == 128; }

bool tc_order1_supports(int B, int H, int N, int d, int dtype, int chunk) {
    return dtype == SSD_BF16 && d == kD && (chunk == 128 || chunk == 256) && (long long)B * H * N < (1ll << 31);
}

// lam (n_chunks floats), acs and vfac (B H N floats each), U (n_chunks x 64
// x 64 bf16), hin (n_chunks x 64 x 64 bf16)
void tc_order1_layout(int B, int H, int N, int chunk, Plan *p) {
    const size_t n = (size_t)B * H * (N / chunk);
    p->lam_off = kStatusBytes;
    p->acs_off = align_up(p->lam_off + n * sizeof(float), 256);
    p->vfac_off = align_up(p->acs_off + (size_t)B * H * N * sizeof(float), 256);
    p->state_off = align_up(p->vfac_off + (size_t)B * H * N * sizeof(float), 256);
    p->aux_off = align_up(p->state_off + n * 4096 * 2, 256);
    p->total = align_up(p->aux_off + n * 4096 * 2, 256);
}

int launch_tc_order1(const FwdArgs &a, const Plan &p) {
    if (a.normalize || a.order != 1) return SSD_ERR_UNSUPPORTED;
    if (a.conv) return a.chunk == 128 ? launch_c<128, true>(a, p) : SSD_ERR_UNSUPPORTED;
    return a.chunk == 256 ? launch_c<256, false>(a, p) : launch_c<128, false>(a, p);
}

}  // namespace ssd
