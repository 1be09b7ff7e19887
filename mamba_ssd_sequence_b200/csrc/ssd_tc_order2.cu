// Order-2 (2Mamba, squared scores) tensor-core path (tcgen05 + TMEM, TMA) of
// the SSD forward operator for bf16 inputs, d_h = 32, chunk = 64.
//
// Order 2 squares the score: w_ij = (q_i . k_j)^2 2^(acs_i - acs_j), whose
// recurrent form (2Mamba2Furious, Algorithm 6) carries the state
// h = sum_j 2^(A_t - A_j) (k_j (x) k_j) v_j^T of d_h^2 x d_h values, plus the
// normaliser state z = sum_j 2^(A_t - A_j) (k_j (x) k_j).  One CTA per
// (batch, head) keeps h and z in tensor memory (fp32) and walks the chunks
// in order.  Per chunk of C = 64 tokens:
//   acs_t = chunk-local inclusive cumsum of A dt (log2 units)   (kernel (a), fused)
//   S     = Q K^T                                      tcgen05 (M = 64)
//   P_ij  = S_ij^2 2^(acs_i - acs_j) [i >= j],  r_i = sum_j P_ij   CUDA cores
//   Y     = P V                                        tcgen05
//   then, over the state's feature rows in slabs of 128 (feature (a, b) = a d + b):
//     hb    = bf16(h_slab)  (the state entering the chunk); h_slab *= 2^lam
//     Fk    = [w_j k_ja k_jb]_{j, (a,b)},  w_j = 2^(lam - acs_j)
//     Fq    = [2^acs_i q_ia q_ib]_{i, (a,b)}
//     h_slab += Fk^T V,   z_slab += Fk^T 1             tcgen05 (M = 128)
//     Y     += Fq hb,     n_off += Fq zb               tcgen05 (M = 64)
//   y_i = Y_i / (r_i + n_off_i) [+ D v_i]             epilogue
// The (q . k)^2 of the intra-chunk part is the same inner product as
// (q (x) q) . (k (x) k) of the feature form (Algorithm 5 vs Algorithm 6).
// All exponentials are of non-positive arguments.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "ptx.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

using namespace ptx;

constexpr int kC = 64;                  // chunk length
constexpr int kD = 32;                  // head dim
constexpr int kF = kD * kD;             // feature rows of the state (1024)
constexpr int kSlab = 128;              // feature rows per slab (one M = 128 tile)
constexpr int kSlabs = kF / kSlab;      // 8
constexpr int kStages = 4;
constexpr int kThreads = 192;           // warp 0: TMA, warp 1: TMEM owner, warps 2-5: compute
constexpr uint32_t kTile = kC * kD * 2;          // 4 KiB: 64 rows x 64 B (64-byte swizzle)
constexpr uint32_t kStageBytes = 3 * kTile;

// shared memory map (1024-aligned pieces)
constexpr uint32_t kOffStage = 0;
constexpr uint32_t kOffP = kOffStage + kStages * kStageBytes;     // 64 x 64 bf16, 128B swizzle
constexpr uint32_t kOffFk = kOffP + 8192;                          // 2 x 16 KiB
constexpr uint32_t kOffFq = kOffFk + 2 * 16384;                    // 2 x 16 KiB
constexpr uint32_t kOffHb = kOffFq + 2 * 16384;                    // 2 x 128 x 64 B (64B swizzle)
constexpr uint32_t kOffZb = kOffHb + 2 * 8192;                     // 2 x 128 x 32 B (32B swizzle)
constexpr uint32_t kOffOnes = kOffZb + 2 * 4096;                   // 64 x 32 B (32B swizzle)
constexpr uint32_t kOffMisc = kOffOnes + 2048;
constexpr uint32_t kSmemBytes = kOffMisc + 2048 + 1024;

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColH = 0;                     // 8 slabs x 32: h (M = 128)
constexpr uint32_t kColZ = kColH + kSlabs * kD;   // 8 slabs x 16: z (column 0 used)
constexpr uint32_t kColS = kColZ + kSlabs * 16;   // 64: S (M = 64)
constexpr uint32_t kColY = kColS + 64;            // 32: Y (M = 64)
constexpr uint32_t kColN = kColY + kD;            // 16: normaliser off-chunk term (M = 64)
static_assert(kColN + 16 <= kTmemCols, "TMEM budget");

constexpr float kLog2e = 1.4426950408889634f;

struct Misc {
    float acs2[kC];
    float rsum[kC];
    float Dh[kD];
    float wtot[2];
    uint64_t stage_full[kStages];
    uint64_t stage_empty[kStages];
    uint64_t mma_bar;
    uint64_t slab_bar[2];
    uint32_t tmem_base;
    int abort_flag;
};
static_assert(sizeof(Misc) <= 2048, "misc block");

__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// swizzle modes of the tcgen05 shared-memory descriptor
constexpr uint32_t kSw128 = 2, kSw64 = 4, kSw32 = 6;

__device__ void raise_timeout(Misc *misc, DeviceStatus *status, int where) {
    if (status) {
        atomicCAS(&status->code, 0, (int)SSD_ERR_TIMEOUT);
        atomicCAS(&status->detail, 0, where);
    }
    *reinterpret_cast<volatile int *>(&misc->abort_flag) = 1;
}

__global__ void __launch_bounds__(kThreads, 1)
tc_order2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16 *__restrict__ out,
                 const float *__restrict__ dt_p, const float *__restrict__ A_log,
                 const float *__restrict__ dt_bias, const float *__restrict__ Dres, int H, int N,
                 int normalize, DeviceStatus *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Misc *misc = reinterpret_cast<Misc *>(smem + kOffMisc);
    const volatile int *abort_flag = &misc->abort_flag;
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
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&misc->stage_full[i], 1);
            mbar_init(&misc->stage_empty[i], 1);
        }
        mbar_init(&misc->mma_bar, 1);
        mbar_init(&misc->slab_bar[0], 1);
        mbar_init(&misc->slab_bar[1], 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    // constant B operand [1, 0, ..., 0] per token (64 rows x 16 bf16, 32B swizzle)
    for (int i = tid; i < kC * 2; i += kThreads) {
        const int r = i >> 1, ch = i & 1;
        const uint32_t one = ch == 0 ? 0x3F80u : 0u;  // bf16 1.0 in the first element
        *reinterpret_cast<uint4 *>(smem + kOffOnes + sw32_chunk(r, ch)) = make_uint4(one, 0, 0, 0);
    }
    if (tid < kD) misc->Dh[tid] = Dres ? Dres[h * kD + tid] : 0.0f;
    fence_proxy_async_smem();
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
            for (int c = 0; c < nc; ++c) {
                const int st = c % kStages;
                if (c >= kStages &&
                    !mbar_wait_abortable(&misc->stage_empty[st], ((c / kStages) - 1) & 1, abort_flag)) {
                    raise_timeout(misc, status, 10);
                    break;
                }
                uint8_t *dst = smem + kOffStage + st * kStageBytes;
                const int r = row0 + c * kC;
                mbar_arrive_expect_tx(&misc->stage_full[st], kStageBytes);
                tma_load_2d(dst, &tm_q, 0, r, &misc->stage_full[st]);
                tma_load_2d(dst + kTile, &tm_k, 0, r, &misc->stage_full[st]);
                tma_load_2d(dst + 2 * kTile, &tm_v, 0, r, &misc->stage_full[st]);
            }
        }
    } else if (warp >= 2) {
        // ------------------------------------------------------ compute group
        const int ct = tid - 64;                  // 0..127
        const int g = warp & 3;                   // TMEM lane quarter
        const uint32_t lane_off = (uint32_t)(g * 32) << 16;
        const int frow = g * 32 + lane;           // feature row of a slab (M = 128 layout)
        const int mrow = g * 16 + lane;           // chunk row in the M = 64 layout (lane < 16)
        const bool mrow_ok = lane < 16;
        const float A2 = -expf(A_log[h]) * kLog2e;
        const float bias = dt_bias[h];
        const bool elected = ct == 0;

        constexpr uint32_t idS = make_idesc_bf16(64, 64, 0, 0);
        constexpr uint32_t idPV = make_idesc_bf16(64, kD, 0, 1);
        constexpr uint32_t idU = make_idesc_bf16(128, kD, 1, 1);
        constexpr uint32_t idZ = make_idesc_bf16(128, 16, 1, 1);
        constexpr uint32_t idT = make_idesc_bf16(64, kD, 0, 1);
        constexpr uint32_t idTz = make_idesc_bf16(64, 16, 0, 1);

        uint32_t mma_uses = 0, slab_uses[2] = {0, 0};
        auto wait_mma = [&](uint64_t *bar, uint32_t uses) -> bool {
            return mbar_wait_abortable(bar, (uses - 1) & 1, abort_flag);
        };

        float dt_next = (ct < kC && nc > 0) ? dt_p[(size_t)row0 + ct] : 0.0f;
        for (int c = 0; c < nc; ++c) {
            const int st = c % kStages;
            uint8_t *sQ = smem + kOffStage + st * kStageBytes;
            uint8_t *sK = sQ + kTile;
            uint8_t *sV = sK + kTile;
            const uint32_t aQ = smem_u32(sQ), aK = aQ + kTile, aV = aK + kTile;
            const float dtv = dt_next;
            if (ct < kC && c + 1 < nc) dt_next = dt_p[(size_t)row0 + (size_t)(c + 1) * kC + ct];

            // ---- decay (tokens 0..63 on threads 0..63: warps 2 and 3)
            float a = 0.0f;
            if (ct < kC) {
                a = A2 * softplus_f(dtv + bias);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, a, o);
                    if (lane >= o) a += y;
                }
                if (lane == 31) misc->wtot[ct >> 5] = a;
            }
            named_bar_sync(1, 128);
            if (ct >= 32 && ct < kC) a += misc->wtot[0];
            if (ct < kC) misc->acs2[ct] = a;
            const float lam2 = misc->wtot[0] + misc->wtot[1];

            bool bad = !mbar_wait_abortable(&misc->stage_full[st], (c / kStages) & 1, abort_flag);
            if (named_bar_any(1, 128, bad)) {
                if (elected) raise_timeout(misc, status, 30);
                break;
            }
            // ---- S = Q K^T
            if (elected) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kD / 16; ++ks)
                    mma_bf16(tmem + kColS, make_sdesc(aQ + ks * 32, 16, 512, kSw64),
                             make_sdesc(aK + ks * 32, 16, 512, kSw64), idS, ks > 0);
                mma_commit(&misc->mma_bar);
            }
            ++mma_uses;
            bad = !wait_mma(&misc->mma_bar, mma_uses);
            if (named_bar_any(1, 128, bad)) {
                if (elected) raise_timeout(misc, status, 31);
                break;
            }
            tc_fence_after();

            // ---- P = S^2 2^(acs_i - acs_j) [i >= j] (rows of the M = 64 layout), row sums
            {
                float sv[32];
                float rs = 0.0f;
                const float ai = misc->acs2[mrow & 63];
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    tmem_ld32(tmem + lane_off + kColS + half * 32, sv);
                    tmem_wait_ld();
                    if (mrow_ok) {
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const int j = half * 32 + e;
                            float p0 = sv[e] * sv[e] * ex2_approx(ai - misc->acs2[j]);
                            float p1 = sv[e + 1] * sv[e + 1] * ex2_approx(ai - misc->acs2[j + 1]);
                            if (j > mrow) p0 = 0.0f;
                            if (j + 1 > mrow) p1 = 0.0f;
                            rs += p0 + p1;
                            pk[e >> 1] = pack_bf16x2(p0, p1);
                        }
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            *reinterpret_cast<uint4 *>(smem + kOffP + sw128_chunk(mrow, half * 4 + q4)) =
                                make_uint4(pk[q4 * 4], pk[q4 * 4 + 1], pk[q4 * 4 + 2], pk[q4 * 4 + 3]);
                    }
                }
                if (mrow_ok) misc->rsum[mrow] = rs;
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, 128);
            // ---- Y = P V
            if (elected) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_bf16(tmem + kColY, make_sdesc(sbase + kOffP + ks * 32, 16, 1024, kSw128),
                             make_sdesc(aV + ks * 1024, 16, 512, kSw64), idPV, ks > 0);
            }

            // ---- state slabs
            const float acs_tok = misc->acs2[ct & 63];        // token of this thread in F*
            const float wk = ex2_approx(lam2 - acs_tok);       // w_j for F_k
            const float sq = ex2_approx(acs_tok);              // 2^acs_i for F_q
            const float dec = ex2_approx(lam2);                // decay of the whole chunk
            const int tok = ct & 63, blk = ct >> 6;
            float kr[kD], qr[kD];                              // this token's k and q rows
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                const uint4 ku = *reinterpret_cast<const uint4 *>(sK + sw64_chunk(tok, ch));
                const uint4 qu = *reinterpret_cast<const uint4 *>(sQ + sw64_chunk(tok, ch));
                const uint32_t kw[4] = {ku.x, ku.y, ku.z, ku.w}, qw[4] = {qu.x, qu.y, qu.z, qu.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kf = bf2_to_f2(kw[e]), qf = bf2_to_f2(qw[e]);
                    kr[ch * 8 + 2 * e] = kf.x;
                    kr[ch * 8 + 2 * e + 1] = kf.y;
                    qr[ch * 8 + 2 * e] = qf.x;
                    qr[ch * 8 + 2 * e + 1] = qf.y;
                }
            }
            for (int sl = 0; sl < kSlabs; ++sl) {
                const int b = sl & 1;
                if (slab_uses[b] > 0) {
                    bad = !wait_mma(&misc->slab_bar[b], slab_uses[b]);
                    if (named_bar_any(1, 128, bad)) {
                        if (elected) raise_timeout(misc, status, 32);
                        goto done;
                    }
                    tc_fence_after();
                }
                // h_{c-1} of this slab to bf16 (64B-swizzled rows), then h *= 2^lam; same for z
                {
                    float hv[32];
                    tmem_ld32(tmem + lane_off + kColH + sl * kD, hv);
                    float zv = normalize ? tmem_ld1(tmem + lane_off + kColZ + sl * 16) : 0.0f;
                    tmem_wait_ld();
                    if (c >= 1) {
                        uint8_t *hb = smem + kOffHb + b * 8192;
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch)
                            *reinterpret_cast<uint4 *>(hb + sw64_chunk(frow, ch)) =
                                make_uint4(pack_bf16x2(hv[ch * 8], hv[ch * 8 + 1]),
                                           pack_bf16x2(hv[ch * 8 + 2], hv[ch * 8 + 3]),
                                           pack_bf16x2(hv[ch * 8 + 4], hv[ch * 8 + 5]),
                                           pack_bf16x2(hv[ch * 8 + 6], hv[ch * 8 + 7]));
                        if (normalize) {
                            uint8_t *zb = smem + kOffZb + b * 4096;
                            *reinterpret_cast<uint4 *>(zb + sw32_chunk(frow, 0)) =
                                make_uint4(pack_bf16x2(zv, 0.0f), 0u, 0u, 0u);
                            *reinterpret_cast<uint4 *>(zb + sw32_chunk(frow, 1)) = make_uint4(0u, 0u, 0u, 0u);
                        }
                        const float2 d2 = make_float2(dec, dec);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 r2 = __fmul2_rn(make_float2(hv[e], hv[e + 1]), d2);
                            hv[e] = r2.x;
                            hv[e + 1] = r2.y;
                        }
                        tmem_st32(tmem + lane_off + kColH + sl * kD, hv);
                        if (normalize) tmem_st1(tmem + lane_off + kColZ + sl * 16, zv * dec);
                    }
                }
                // F_k and F_q: this thread writes token `tok`, 64-feature block `blk`
                // (features (a, b) with a = 4 sl + 2 blk + {0, 1}, b = 0..31)
                {
                    const int a0 = sl * 4 + blk * 2;
                    uint8_t *fk = smem + kOffFk + b * 16384 + blk * 8192;
                    uint8_t *fq = smem + kOffFq + b * 16384 + blk * 8192;
#pragma unroll
                    for (int aa = 0; aa < 2; ++aa) {
                        const int ai = a0 + aa;  // k_{j,a} and q_{i,a} read back from the tiles
                        const uint32_t eo = sw64_chunk(tok, ai >> 3) + (ai & 7) * 2;
                        const float ka = __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t *>(sK + eo) << 16);
                        const float qa = __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t *>(sQ + eo) << 16);
                        const float sk = wk * ka, sqq = sq * qa;
                        const float2 sk2 = make_float2(sk, sk), sq2 = make_float2(sqq, sqq);
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch) {
                            uint32_t wk4[4], wq4[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int bb = ch * 8 + 2 * e;
                                const float2 kv = __fmul2_rn(make_float2(kr[bb], kr[bb + 1]), sk2);
                                const float2 qv = __fmul2_rn(make_float2(qr[bb], qr[bb + 1]), sq2);
                                wk4[e] = pack_bf16x2(kv.x, kv.y);
                                wq4[e] = pack_bf16x2(qv.x, qv.y);
                            }
                            const int cidx = aa * 4 + ch;  // 16B chunk in the 128B row
                            *reinterpret_cast<uint4 *>(fk + sw128_chunk(tok, cidx)) =
                                make_uint4(wk4[0], wk4[1], wk4[2], wk4[3]);
                            *reinterpret_cast<uint4 *>(fq + sw128_chunk(tok, cidx)) =
                                make_uint4(wq4[0], wq4[1], wq4[2], wq4[3]);
                        }
                    }
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar_sync(1, 128);
                if (elected) {
                    tc_fence_after();
                    const uint32_t fkA = sbase + kOffFk + b * 16384;
                    const uint32_t fqA = sbase + kOffFq + b * 16384;
                    // h_slab += Fk^T V  (A: features x tokens, MN-major, two 64-feature groups)
#pragma unroll
                    for (int ks = 0; ks < kC / 16; ++ks)
                        mma_bf16(tmem + kColH + sl * kD, make_sdesc(fkA + ks * 2048, 8192, 1024, kSw128),
                                 make_sdesc(aV + ks * 1024, 16, 512, kSw64), idU, (c > 0 || ks > 0));
                    if (normalize) {
#pragma unroll
                        for (int ks = 0; ks < kC / 16; ++ks)
                            mma_bf16(tmem + kColZ + sl * 16, make_sdesc(fkA + ks * 2048, 8192, 1024, kSw128),
                                     make_sdesc(sbase + kOffOnes + ks * 512, 16, 256, kSw32), idZ,
                                     (c > 0 || ks > 0));
                    }
                    if (c >= 1) {
                        // Y += Fq hb ;  n_off += Fq zb   (A: tokens x features, K-major)
                        const uint32_t hbB = sbase + kOffHb + b * 8192;
                        const uint32_t zbB = sbase + kOffZb + b * 4096;
#pragma unroll
                        for (int ks = 0; ks < kSlab / 16; ++ks) {
                            const uint64_t adesc =
                                make_sdesc(fqA + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kSw128);
                            mma_bf16(tmem + kColY, adesc, make_sdesc(hbB + ks * 1024, 16, 512, kSw64), idT, 1);
                            if (normalize)
                                mma_bf16(tmem + kColN, adesc, make_sdesc(zbB + ks * 512, 16, 256, kSw32), idTz,
                                         (sl > 0 || ks > 0));
                        }
                    }
                    mma_commit(&misc->slab_bar[b]);
                }
                ++slab_uses[b];
            }
            // ---- all MMAs of the chunk done
            if (elected) mma_commit(&misc->mma_bar);
            ++mma_uses;
            bad = !wait_mma(&misc->mma_bar, mma_uses);
            if (named_bar_any(1, 128, bad)) {
                if (elected) raise_timeout(misc, status, 33);
                break;
            }
            tc_fence_after();

            // ---- epilogue: y = Y / (r + n_off) [+ D v], bf16 stores (rows of the M = 64 layout)
            {
                float yv[32];
                tmem_ld32(tmem + lane_off + kColY, yv);
                const float noff = (normalize && c >= 1) ? tmem_ld1(tmem + lane_off + kColN) : 0.0f;
                tmem_wait_ld();
                if (mrow_ok) {
                    const float inv = normalize ? 1.0f / (misc->rsum[mrow] + noff) : 1.0f;
                    uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)(row0 + c * kC + mrow) * kD);
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        const uint4 vu = *reinterpret_cast<const uint4 *>(sV + sw64_chunk(mrow, ch));
                        const uint32_t vw[4] = {vu.x, vu.y, vu.z, vu.w};
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int cc = ch * 8 + 2 * e;
                            float y0 = yv[cc] * inv, y1 = yv[cc + 1] * inv;
                            if (Dres) {
                                const float2 vf = bf2_to_f2(vw[e]);
                                y0 = fmaf(misc->Dh[cc], vf.x, y0);
                                y1 = fmaf(misc->Dh[cc + 1], vf.y, y1);
                            }
                            w[e] = pack_bf16x2(y0, y1);
                        }
                        dst[ch] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(1, 128);
            if (elected) mbar_arrive(&misc->stage_empty[st]);
        }
    done:;
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

// [rows, 32] bf16 row-major tensor, boxes of 64 rows, 64-byte swizzle.
bool make_tmap_rows32(CUtensorMap *m, const void *base, uint64_t rows) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {kD, rows};
    cuuint64_t strides[1] = {kD * 2};
    cuuint32_t box[2] = {kD, kC};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool tc_order2_supports(int B, int H, int N, int d, int dtype, int chunk) {
    return dtype == SSD_BF16 && d == kD && chunk == kC && (long long)B * H * N < (1ll << 31);
}

size_t tc_order2_workspace(int, int, int, int, int) { return 0; }

int launch_tc_order2(const FwdArgs &a, const Plan &) {
    const uint64_t rows = (uint64_t)a.B * a.H * a.N;
    CUtensorMap tq, tk, tv;
    if (!make_tmap_rows32(&tq, a.q, rows) || !make_tmap_rows32(&tk, a.k, rows) ||
        !make_tmap_rows32(&tv, a.v, rows))
        return SSD_ERR_CUDA;
    static bool attr_set = false;
    if (!attr_set) {
        if (cudaFuncSetAttribute(tc_order2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes) != cudaSuccess)
            return SSD_ERR_CUDA;
        attr_set = true;
    }
    DeviceStatus *status = reinterpret_cast<DeviceStatus *>(a.workspace);
    tc_order2_kernel<<<a.B * a.H, kThreads, kSmemBytes, a.stream>>>(
        tq, tk, tv, static_cast<__nv_bfloat16 *>(a.out), a.dt_p, a.A_log, a.dt_bias, a.D, a.H,
        a.N, a.normalize, status);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace ssd
