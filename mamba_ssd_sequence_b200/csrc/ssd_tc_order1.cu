// Order-1 tensor-core path (tcgen05 + TMEM, TMA) of the SSD forward operator
// for bf16 inputs, d_h = 64, chunk = 128, no normaliser.
//
// Each (batch, head) is split into R segments of whole chunks; one CTA per
// segment.  A CTA first folds the chunks before its segment into the carried
// state (K and V only, no output), then produces its own chunks; so it never
// waits for another CTA, and the state it carries never leaves the SM.  Per
// chunk c (2Mamba2Furious, Algorithms 1, 3, 4 and 6, evaluated in the
// chunked state-passing form of the semiseparable mask):
//   acs_t = chunk-local inclusive cumsum of A*dt (log2 units)  (kernel (a), fused)
//   S     = Q K^T                                  tcgen05, fp32 in TMEM
//   P_ij  = S_ij 2^(acs_i - acs_j) [i >= j]        CUDA cores, bf16 back into TMEM
//   U_c   = K'^T V,   K'_j = 2^(lam_c - acs_j) k_j  tcgen05 (the chunk's own state term)
//   h_c   = 2^(lam_c) h_{c-1} + U_c                 CUDA cores, fp32
//   Y     = P V + Q' h_{c-1},  Q'_i = 2^(acs_i) q_i  tcgen05 (P from TMEM)
//   y_i   = Y_i [+ D v_i]                           epilogue, 16-byte stores
//
// Warp roles (608 threads): warp 0 issues TMA loads into a 3-stage ring;
// warps 1 and 2 each issue the MMAs of one compute group in a fixed order
// (blocking, bounded waits: no polling); warps 3-10 and 11-18 are two compute
// groups that take even and odd chunks (ping-pong), so one group's
// exponentials overlap the other's MMAs and epilogue.  In a group the two
// warps that share a TMEM lane quarter split each row's columns.  Each group
// keeps its own copy of the carried state and advances it two chunks at a
// time, h_{c-1} = 2^(lam_{c-1}) h_{c-2} + U_{c-1}, where U_{c-1} is the other
// group's chunk term read from TMEM: the only cross-group dependency is an
// MMA result, never a chain of group-to-group hand-offs.  All exponentials
// are of non-positive arguments (chunk-local differences).  Every wait is
// bounded; a timeout sets SSD_ERR_TIMEOUT in the workspace status and all
// roles leave their loops.
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

constexpr int kC = 128;             // chunk length = rows of every tile
constexpr int kD = 64;              // head dim
constexpr int kStages = 3;          // TMA ring depth
constexpr int kGroupThreads = 256;  // one compute group: 8 warps, 2 per TMEM lane quarter
constexpr int kFirstGroupWarp = 3;
constexpr int kThreads = 32 * kFirstGroupWarp + 2 * kGroupThreads;
constexpr uint32_t kTileBytes = kC * kD * 2;  // 16 KiB bf16 tile
constexpr uint32_t kStageBytes = 3 * kTileBytes;

constexpr uint32_t kHRow = kD + 4;                               // padded fp32 row of h
constexpr uint32_t kOffStage = 0;                                // kStages x {Q, K, V}
constexpr uint32_t kOffHs = kOffStage + kStages * kStageBytes;   // 2 x h_{c-1} bf16 (64 x 64)
constexpr uint32_t kOffH32 = kOffHs + 2 * kD * kD * 2;           // 2 x own state h (fp32)
constexpr uint32_t kOffDres = kOffH32 + 2 * kD * kHRow * 4;      // D of this head (fp32)
constexpr uint32_t kOffMisc = kOffDres + kD * 4;
constexpr uint32_t kSmemBytes = kOffMisc + 2048 + 1024;          // misc + alignment slack

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // 2 x 128: S (fp32), then P (bf16 pairs) at [32, 96)
constexpr uint32_t kColP = 32;    // offset of P inside an S slot
constexpr uint32_t kColY = 256;   // 2 x 64: Y
constexpr uint32_t kColU = 384;   // 2 x 64: U (M = 64 layout, rows at lanes 32g + 0..15)

constexpr float kLog2e = 1.4426950408889634f;

struct Misc {
    float acs2[2][kC];
    float wtot[2][4];
    float lam_red[2][4];
    uint64_t stage_full[kStages];
    uint64_t stage_empty[kStages];
    uint64_t s_full[2], kp_full[2], p_full[2], u_full[2], u_free[2], hs_full[2], y_full[2],
        y_free[2];
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Misc) <= 2048, "misc block");

__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}
__device__ __forceinline__ uint64_t desc_k(uint32_t saddr) { return make_sdesc(saddr, 16, 1024); }
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr) {
    return make_sdesc(saddr, kTileBytes, 1024);
}
// bf16 pair (low, high) -> float2
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t f2_to_bf2(float2 v) { return pack_bf16x2(v.x, v.y); }

// Scales columns [32 hf, 32 hf + 32) of row `row` of a 128B-swizzled bf16 tile.
__device__ __forceinline__ void scale_half_row_inplace(uint8_t *tile, int row, int hf, float s) {
    const float2 s2 = make_float2(s, s);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 *p = reinterpret_cast<uint4 *>(tile + sw128_chunk(row, hf * 4 + q));
        uint4 u = *p;
        u.x = f2_to_bf2(__fmul2_rn(bf2_to_f2(u.x), s2));
        u.y = f2_to_bf2(__fmul2_rn(bf2_to_f2(u.y), s2));
        u.z = f2_to_bf2(__fmul2_rn(bf2_to_f2(u.z), s2));
        u.w = f2_to_bf2(__fmul2_rn(bf2_to_f2(u.w), s2));
        *p = u;
    }
}

// P for 16 columns (tokens j0 .. j0+15, all inside column block jb) of this
// thread's row, from the S values `sv` already loaded; writes 8 packed bf16
// columns of TMEM at column j0 / 2.  Blocks entirely above the diagonal
// (jb > g) are written as zeros.
__device__ __forceinline__ void build_p16(uint32_t tP, int j0, int jb, int g, int row, float acs2,
                                          const float *acs_row, const float (&sv)[16]) {
    uint32_t pk[8];
    if (jb > g) {
#pragma unroll
        for (int e = 0; e < 8; ++e) pk[e] = 0u;
    } else {
        const float2 ai = make_float2(acs2, acs2);
        const float4 *ac = reinterpret_cast<const float4 *>(acs_row + j0);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const float4 aj = ac[q4];
            const float2 d0 = __fadd2_rn(ai, make_float2(-aj.x, -aj.y));
            const float2 d1 = __fadd2_rn(ai, make_float2(-aj.z, -aj.w));
            float2 p0 = __fmul2_rn(make_float2(sv[q4 * 4], sv[q4 * 4 + 1]),
                                   make_float2(ex2_approx(d0.x), ex2_approx(d0.y)));
            float2 p1 = __fmul2_rn(make_float2(sv[q4 * 4 + 2], sv[q4 * 4 + 3]),
                                   make_float2(ex2_approx(d1.x), ex2_approx(d1.y)));
            if (jb == g) {  // the diagonal block: keep j <= i
                const int j = j0 + q4 * 4;
                if (j > row) p0.x = 0.0f;
                if (j + 1 > row) p0.y = 0.0f;
                if (j + 2 > row) p1.x = 0.0f;
                if (j + 3 > row) p1.y = 0.0f;
            }
            pk[q4 * 2] = f2_to_bf2(p0);
            pk[q4 * 2 + 1] = f2_to_bf2(p1);
        }
    }
    tmem_st8(tP + j0 / 2, pk);
}

__device__ void raise_timeout(Misc *misc, DeviceStatus *status, int where) {
    if (status) {
        atomicCAS(&status->code, 0, (int)SSD_ERR_TIMEOUT);
        atomicCAS(&status->detail, 0, where);
    }
    *reinterpret_cast<volatile int *>(&misc->abort_flag) = 1;
}

__global__ void __launch_bounds__(kThreads, 1)
tc_order1_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16 *__restrict__ out,
                 const float *__restrict__ dt_p, const float *__restrict__ A_log,
                 const float *__restrict__ dt_bias, const float *__restrict__ Dres, int H, int N,
                 int BH, int R, DeviceStatus *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Misc *misc = reinterpret_cast<Misc *>(smem + kOffMisc);
    const volatile int *abort_flag = &misc->abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x % BH, seg = blockIdx.x / BH, h = bh % H;
    const int nc = N / kC;
    const int row0 = bh * N;
    // This CTA produces the outputs of chunks [c_begin, c_end) of its head.
    // Chunks [0, c_begin) are only folded into the carried state (K and V
    // are read, no output), so the CTA starts its own segment from the exact
    // state without waiting for another CTA.
    const int c_begin = (seg * nc) / R, c_end = ((seg + 1) * nc) / R;
    // index of own chunk c among the own chunks of its parity (phases of the
    // barriers that only own chunks use)
    auto own_idx = [&](int c) { return (c - (c_begin + ((c ^ c_begin) & 1))) >> 1; };

    if (tid == 0) {
        if (blockIdx.x == 0 && status) {
            status->code = 0;
            status->detail = 0;
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&misc->stage_full[i], 1);
            mbar_init(&misc->stage_empty[i], kGroupThreads);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&misc->s_full[s], 1);
            mbar_init(&misc->kp_full[s], kGroupThreads);
            mbar_init(&misc->p_full[s], kGroupThreads);
            mbar_init(&misc->u_full[s], 1);
            mbar_init(&misc->u_free[s], 2 * kGroupThreads);
            mbar_init(&misc->hs_full[s], kGroupThreads);
            mbar_init(&misc->y_full[s], 1);
            mbar_init(&misc->y_free[s], kGroupThreads);
        }
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    {
        float *sD = reinterpret_cast<float *>(smem + kOffDres);
        float *sH32 = reinterpret_cast<float *>(smem + kOffH32);
        for (int i = tid; i < kD; i += kThreads) sD[i] = Dres ? Dres[h * kD + i] : 0.0f;
        for (int i = tid; i < 2 * kD * (int)kHRow; i += kThreads) sH32[i] = 0.0f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            for (int c = 0; c < c_end; ++c) {
                const int st = c % kStages;
                if (c >= kStages &&
                    !mbar_wait_abortable(&misc->stage_empty[st], ((c / kStages) - 1) & 1, abort_flag)) {
                    raise_timeout(misc, status, 10);
                    break;
                }
                uint8_t *dst = smem + kOffStage + st * kStageBytes;
                const int r = row0 + c * kC;
                const bool own = c >= c_begin;
                mbar_arrive_expect_tx(&misc->stage_full[st], own ? kStageBytes : 2 * kTileBytes);
                if (own) tma_load_2d(dst, &tm_q, 0, r, &misc->stage_full[st]);
                tma_load_2d(dst + kTileBytes, &tm_k, 0, r, &misc->stage_full[st]);
                tma_load_2d(dst + 2 * kTileBytes, &tm_v, 0, r, &misc->stage_full[st]);
            }
        }
    } else if (warp < 3) {
        // ------------------------------------------------------ MMA issuers
        // Warp 1 issues every MMA of group 0's chunks, warp 2 of group 1's, in
        // chunk order: S, U, P V, Q' h.  Same-thread issue order keeps the
        // slot reuse of S / P, Y and h_{c-1} in order; U slots are shared with
        // the other group and are guarded by u_free.
        const int s = warp - 1;
        if (lane == 0) {
            constexpr uint32_t idesc_S = make_idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idesc_Y = make_idesc_bf16(128, 64, 0, 1);
            constexpr uint32_t idesc_U = make_idesc_bf16(64, 64, 1, 1);
            const uint32_t sbase = smem_u32(smem);
            bool ok = true;
            for (int c = s; ok && c < c_end; c += 2) {
                const int k = c >> 1, st = c % kStages;
                const bool own = c >= c_begin;
                const int ko = own ? own_idx(c) : 0;
                const uint32_t aQ = sbase + kOffStage + st * kStageBytes;
                const uint32_t aK = aQ + kTileBytes, aV = aK + kTileBytes;
                if (own) {  // S = Q K^T
                    if (!(ok = mbar_wait_abortable(&misc->stage_full[st], (c / kStages) & 1, abort_flag)))
                        break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks)
                        mma_bf16(tmem + kColS + s * 128, desc_k(aQ + ks * 32), desc_k(aK + ks * 32),
                                 idesc_S, ks > 0);
                    mma_commit(&misc->s_full[s]);
                }
                // U_c = K'^T V   (M = 64, N = 64, K = 128 tokens; K' and V MN-major)
                if (!(ok = mbar_wait_abortable(&misc->kp_full[s], k & 1, abort_flag))) break;
                if (c >= 2 && !(ok = mbar_wait_abortable(&misc->u_free[s], (k - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_bf16(tmem + kColU + s * 64, desc_mn(aK + ks * 2048), desc_mn(aV + ks * 2048),
                             idesc_U, ks > 0);
                mma_commit(&misc->u_full[s]);
                if (!own) continue;
                // Y = P V   (A = P from TMEM, 8 packed columns per 16 tokens)
                if (!(ok = mbar_wait_abortable(&misc->p_full[s], ko & 1, abort_flag))) break;
                if (ko >= 1 && !(ok = mbar_wait_abortable(&misc->y_free[s], (ko - 1) & 1, abort_flag)))
                    break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_bf16_ts(tmem + kColY + s * 64, tmem + kColS + s * 128 + kColP + ks * 8,
                                desc_mn(aV + ks * 2048), idesc_Y, ks > 0);
                // Y += Q' h_{c-1}
                if (!(ok = mbar_wait_abortable(&misc->hs_full[s], ko & 1, abort_flag))) break;
                tc_fence_after();
                if (c >= 1) {
                    const uint32_t aH = sbase + kOffHs + s * (kD * kD * 2);
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks)
                        mma_bf16(tmem + kColY + s * 64, desc_k(aQ + ks * 32), desc_mn(aH + ks * 2048),
                                 idesc_Y, 1);
                }
                mma_commit(&misc->y_full[s]);
            }
            if (!ok) raise_timeout(misc, status, 20 + s);
        }
    } else if (warp >= kFirstGroupWarp) {
        // ------------------------------------------------------ compute groups
        const int s = (warp - kFirstGroupWarp) >> 3;  // 0: even chunks, 1: odd chunks
        const int wi = (warp - kFirstGroupWarp) & 7;  // warp inside the group
        const int g = warp & 3;                       // TMEM lane quarter = row block
        const int hf = wi >> 2;                       // which half of each row's columns
        const int row = g * 32 + lane;                // chunk row owned (shared by the halves)
        const int wt = wi * 32 + lane;                // 0..255 inside the group
        const int bar_id = 1 + s;                     // group barrier
        const uint32_t lane_off = (uint32_t)(g * 32) << 16;
        const float A2 = -expf(A_log[h]) * kLog2e;
        const float bias = dt_bias[h];
        // own carried state h_{c-2}, fp32 in shared memory (row m = 16g + lane)
        float *hown = reinterpret_cast<float *>(smem + kOffH32) + s * kD * kHRow;
        const float *sD = reinterpret_cast<const float *>(smem + kOffDres);
        // half 0 scans this chunk's decay; half 1 sums the previous chunk's
        // (the other group's), so each loads one dt per chunk, one ahead
        const int dt_off = hf == 0 ? 0 : -1;
        float dt_next = (s + dt_off >= 0 && s + dt_off < c_end)
                            ? dt_p[(size_t)row0 + (s + dt_off) * kC + row] : 0.0f;

        for (int c = s; c < c_end; c += 2) {
            const int k = c >> 1, st = c % kStages;
            const bool own = c >= c_begin;  // produce outputs (else: state only)
            const int ko = own ? own_idx(c) : 0;
            uint8_t *sQ = smem + kOffStage + st * kStageBytes;
            uint8_t *sK = sQ + kTileBytes;
            uint8_t *sV = sK + kTileBytes;
            const float dtv = dt_next;
            const int cn = c + 2 + dt_off;
            if (cn < c_end) dt_next = dt_p[(size_t)row0 + (size_t)cn * kC + row];

            // ---- decay: scan of this chunk (half 0), total of chunk c-1 (half 1)
            float a = (hf == 0 || c >= 1) ? A2 * softplus_f(dtv + bias) : 0.0f;
            if (hf == 0) {
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, a, o);
                    if (lane >= o) a += y;
                }
                if (lane == 31) misc->wtot[s][g] = a;
            } else {
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                if (lane == 0) misc->lam_red[s][g] = a;
            }
            named_bar_sync(bar_id, kGroupThreads);
            const float lam2 = misc->wtot[s][0] + misc->wtot[s][1] + misc->wtot[s][2] + misc->wtot[s][3];
            const float lam2_prev = misc->lam_red[s][0] + misc->lam_red[s][1] + misc->lam_red[s][2] +
                                    misc->lam_red[s][3];
            if (hf == 0) {
                for (int w = 0; w < g; ++w) a += misc->wtot[s][w];
                misc->acs2[s][row] = a;
            }

            // ---- wait for this chunk's tiles and for S = Q K^T (after which Q and K
            //      may be rewritten in place)
            bool bad = !mbar_wait_abortable(&misc->stage_full[st], (c / kStages) & 1, abort_flag);
            bad = bad || (own && !mbar_wait_abortable(&misc->s_full[s], ko & 1, abort_flag));
            if (named_bar_any(bar_id, kGroupThreads, bad)) {
                if (wt == 0) raise_timeout(misc, status, 32 + s);
                break;
            }
            tc_fence_after();
            const float acs2 = misc->acs2[s][row];

            // ---- K'_j = 2^(lam - acs_j) k_j, in place in the stage's K tile (half row)
            scale_half_row_inplace(sK, row, hf, ex2_approx(lam2 - acs2));
            fence_proxy_async_smem();
            mbar_arrive(&misc->kp_full[s]);

            if (own) {
                // ---- P = S (.) 2^(acs_i - acs_j) [i >= j] -> bf16 pairs back into TMEM,
                // at columns [32, 96) of the S slot (token j at 32 + j / 2).  Half 0
                // covers tokens 0-63 and writes columns 32-63, which only it reads
                // (S columns 0-63); half 1 covers tokens 64-127 and writes 64-95
                // (inside its S columns 64-127).  The 16-token pieces go in an
                // order in which every write lands on S values already consumed.
                const uint32_t tS = tmem + lane_off + kColS + s * 128;
#pragma unroll 1
                for (int t = 0; t < 4; ++t) {
                    // half 0: tokens 48, 32, 16, 0; half 1: 64, 80, 96, 112
                    const int j0 = hf == 0 ? 48 - 16 * t : 64 + 16 * t;
                    const int jb = j0 >> 5;
                    float sv[16];
                    if (jb <= g) {
                        tmem_ld16(tS + j0, sv);
                        tmem_wait_ld();
                    }
                    build_p16(tS + kColP, j0, jb, g, row, acs2, misc->acs2[s], sv);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&misc->p_full[s]);

                // ---- Q'_i = 2^(acs_i) q_i, in place (the S MMA of this chunk is done)
                scale_half_row_inplace(sQ, row, hf, ex2_approx(acs2));
            }

            // ---- carried state: h_{c-1} (bf16, for Y) and own h_c; this warp does
            //      columns [32 hf, 32 hf + 32) of rows m = 16g + lane (lane < 16)
            bad = (c >= 1) && !mbar_wait_abortable(&misc->u_full[s ^ 1], ((c - 1) >> 1) & 1, abort_flag);
            bad = bad || !mbar_wait_abortable(&misc->u_full[s], k & 1, abort_flag);
            if (named_bar_any(bar_id, kGroupThreads, bad)) {
                if (wt == 0) raise_timeout(misc, status, 34 + s);
                break;
            }
            tc_fence_after();
            {
                const float dp = ex2_approx(lam2_prev), dc = ex2_approx(lam2);
                const float2 dprev = make_float2(dp, dp), dcur = make_float2(dc, dc);
                const uint32_t tUo = tmem + lane_off + kColU + (s ^ 1) * 64 + hf * 32;
                const uint32_t tUs = tmem + lane_off + kColU + s * 64 + hf * 32;
                uint8_t *sH = smem + kOffHs + s * (kD * kD * 2);
                const int m = g * 16 + lane;  // state row (valid for lane < 16)
#pragma unroll
                for (int qt = 0; qt < 2; ++qt) {
                    float uo[16], us[16];
                    if (c >= 1) tmem_ld16(tUo + qt * 16, uo);
                    tmem_ld16(tUs + qt * 16, us);
                    tmem_wait_ld();
                    if (lane < 16) {
                        const int col0 = hf * 32 + qt * 16;
                        uint32_t hb[8];
#pragma unroll
                        for (int e4 = 0; e4 < 4; ++e4) {
                            float4 *hp4 = reinterpret_cast<float4 *>(hown + m * kHRow + col0 + e4 * 4);
                            const float4 hv = *hp4;
                            float2 h0 = make_float2(0.0f, 0.0f), h1 = h0;
                            if (c >= 1) {
                                h0 = __ffma2_rn(dprev, make_float2(hv.x, hv.y),
                                                make_float2(uo[e4 * 4], uo[e4 * 4 + 1]));
                                h1 = __ffma2_rn(dprev, make_float2(hv.z, hv.w),
                                                make_float2(uo[e4 * 4 + 2], uo[e4 * 4 + 3]));
                            }
                            hb[e4 * 2] = f2_to_bf2(h0);
                            hb[e4 * 2 + 1] = f2_to_bf2(h1);
                            const float2 n0 = __ffma2_rn(dcur, h0, make_float2(us[e4 * 4], us[e4 * 4 + 1]));
                            const float2 n1 = __ffma2_rn(dcur, h1, make_float2(us[e4 * 4 + 2], us[e4 * 4 + 3]));
                            *hp4 = make_float4(n0.x, n0.y, n1.x, n1.y);
                        }
                        if (own && c >= 1) {
                            *reinterpret_cast<uint4 *>(sH + sw128_chunk(m, col0 / 8)) =
                                make_uint4(hb[0], hb[1], hb[2], hb[3]);
                            *reinterpret_cast<uint4 *>(sH + sw128_chunk(m, col0 / 8 + 1)) =
                                make_uint4(hb[4], hb[5], hb[6], hb[7]);
                        }
                    }
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            mbar_arrive(&misc->u_free[s]);
            if (c >= 1) mbar_arrive(&misc->u_free[s ^ 1]);
            if (!own) {
                // state-only chunk: U_c has been read (u_full), so the stage is free
                mbar_arrive(&misc->stage_empty[st]);
                continue;
            }
            mbar_arrive(&misc->hs_full[s]);

            // ---- epilogue: y = Y [+ D v], bf16, 16-byte stores straight to HBM
            bad = !mbar_wait_abortable(&misc->y_full[s], ko & 1, abort_flag);
            if (named_bar_any(bar_id, kGroupThreads, bad)) {
                if (wt == 0) raise_timeout(misc, status, 36 + s);
                break;
            }
            tc_fence_after();
            {
                float y0[16], y1[16];
                tmem_ld16(tmem + lane_off + kColY + s * 64 + hf * 32, y0);
                tmem_ld16(tmem + lane_off + kColY + s * 64 + hf * 32 + 16, y1);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&misc->y_free[s]);
                const float4 *Dh = reinterpret_cast<const float4 *>(sD);
                uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)(row0 + c * kC + row) * kD + hf * 32);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int ch = hf * 4 + q4;
                    const float *yy = q4 < 2 ? (y0 + q4 * 8) : (y1 + (q4 - 2) * 8);
                    uint32_t w[4];
                    if (Dres) {
                        const uint4 vv = *reinterpret_cast<const uint4 *>(sV + sw128_chunk(row, ch));
                        const float4 d0 = Dh[2 * ch], d1 = Dh[2 * ch + 1];
                        const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
                        const float2 dd[4] = {make_float2(d0.x, d0.y), make_float2(d0.z, d0.w),
                                              make_float2(d1.x, d1.y), make_float2(d1.z, d1.w)};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w[e] = f2_to_bf2(__ffma2_rn(dd[e], bf2_to_f2(vw[e]),
                                                        make_float2(yy[2 * e], yy[2 * e + 1])));
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) w[e] = pack_bf16x2(yy[2 * e], yy[2 * e + 1]);
                    }
                    dst[q4] = make_uint4(w[0], w[1], w[2], w[3]);
                }
                mbar_arrive(&misc->stage_empty[st]);  // this thread is done with the stage
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
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

// Segments per head: enough CTAs to cover the SMs, as long as the extra
// state-only work (segment r re-folds r earlier segments) stays small.
int segments_per_head(int BH, int nc) {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            sms = 148;
    }
    int R = 1;
    while (R < 2 && BH * (R * 2) <= sms && nc >= R * 2 * 2) R *= 2;
    return R;
}

int launch_tc_order1(const FwdArgs &a, const Plan &) {
    if (a.normalize) return SSD_ERR_UNSUPPORTED;
    const uint64_t rows = (uint64_t)a.B * a.H * a.N;
    CUtensorMap tq, tk, tv;
    if (!make_tmap_rows64(&tq, a.q, rows, kC) || !make_tmap_rows64(&tk, a.k, rows, kC) ||
        !make_tmap_rows64(&tv, a.v, rows, kC))
        return SSD_ERR_CUDA;
    static std::atomic<uint64_t> attr_set{0};  // one bit per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSD_ERR_CUDA;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_set.load() & bit)) {
        if (cudaFuncSetAttribute(tc_order1_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes) != cudaSuccess)
            return SSD_ERR_CUDA;
        attr_set.fetch_or(bit);
    }
    DeviceStatus *status = reinterpret_cast<DeviceStatus *>(a.workspace);
    const int BH = a.B * a.H;
    const int R = segments_per_head(BH, a.N / kC);
    tc_order1_kernel<<<BH * R, kThreads, kSmemBytes, a.stream>>>(
        tq, tk, tv, static_cast<__nv_bfloat16 *>(a.out), a.dt_p, a.A_log, a.dt_bias, a.D, a.H, a.N, BH, R, status);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace ssd
