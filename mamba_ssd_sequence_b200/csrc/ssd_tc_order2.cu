// Order-2 (2Mamba, squared scores) tensor-core path (tcgen05 + TMEM, TMA) of
// the SSD forward operator for bf16 inputs, d_h in {32, 64}, chunk = 64.
//
// Order 2 squares the score: w_ij = (q_i . k_j)^2 2^(acs_i - acs_j), whose
// recurrent form (2Mamba2Furious, Algorithm 6) carries the state
// h = sum_j 2^(A_t - A_j) (k_j (x) k_j) v_j^T of d_h^2 x d_h values, plus the
// normaliser state z = sum_j 2^(A_t - A_j) (k_j (x) k_j).  The state of one
// head does not fit one SM at d_h = 64 (1 MiB), so a thread-block cluster of
// R = d_h^2 / 512 CTAs shares a head: CTA r keeps feature rows
// [512 r, 512 r + 512) of h and z in tensor memory (fp32) -- feature (a, b)
// is row a d_h + b -- and the cluster walks the chunks together.  Per chunk
// of C = 64 tokens, every CTA:
//   acs_t = chunk-local inclusive cumsum of A dt (log2 units)   (kernel (a), fused)
//   S     = Q K^T                                      tcgen05 (M = 64)
//   P_ij  = S_ij^2 2^(acs_i - acs_j) [i >= j],  r_i = sum_j P_ij   CUDA cores
//   Y     = P V                                        tcgen05
//   over its 4 slabs of 128 feature rows:
//     hb    = bf16(h_slab)  (the state entering the chunk); h_slab *= 2^lam
//     Fk    = [w_j k_ja k_jb]_{j, (a,b)},  w_j = 2^(lam - acs_j)
//     Fq    = [2^acs_i q_ia q_ib]_{i, (a,b)}
//     h_slab += Fk^T V,   z_slab += Fk^T 1             tcgen05 (M = 128)
//     T     += Fq hb,     Tn += Fq zb                  tcgen05 (M = 64)
// The cluster then sums the partial T, Tn of its CTAs through distributed
// shared memory: CTA r owns rows [64 r / R, 64 (r + 1) / R) of the chunk and
// writes y_i = (Y_i + sum T_i) / (r_i + sum Tn_i) [+ D v_i].  The
// (q . k)^2 of the intra-chunk part is the same inner product as
// (q (x) q) . (k (x) k) of the feature form (Algorithm 5 vs Algorithm 6).
// Options: a per-token log-decay and value discretisation (Algorithm 4; V is
// scaled by dt in shared memory); a carried state h0, z0 enters as the state
// before chunk 0, and h_out, z_out receive the state after the last chunk.
// All exponentials are of non-positive arguments.  Every wait is bounded.
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

constexpr int kC = 64;          // chunk length
constexpr int kFs = 512;        // feature rows per CTA
constexpr int kSlab = 128;      // feature rows per slab (one M = 128 tile)
constexpr int kNs = kFs / kSlab;
constexpr int kStages = 2;
constexpr int kTeam = 256;      // compute threads: warps 2-9
constexpr int kThreads = 64 + kTeam;
constexpr uint32_t kSw128 = 2, kSw64 = 4, kSw32 = 6;  // descriptor swizzle modes
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct Cfg {
    static constexpr int R = D * D / kFs;              // CTAs per head
    static constexpr int ROWS = kC / R;                // output rows owned per CTA
    static constexpr uint32_t RB = D * 2;              // bytes per bf16 row of q/k/v/hb
    static constexpr uint32_t SW = RB == 128 ? kSw128 : kSw64;
    static constexpr uint32_t SBO = 8 * RB;            // 8-row swizzle atom
    static constexpr uint32_t TILE = kC * RB;          // q/k/v tile
    static constexpr uint32_t STAGE = 3 * TILE;
    static constexpr int PR = D + 4;                   // padded row (floats) of a partial
    // shared memory map
    static constexpr uint32_t OFF_STAGE = 0;
    static constexpr uint32_t OFF_P = OFF_STAGE + kStages * STAGE;       // 64 x 64 bf16
    static constexpr uint32_t OFF_FK = OFF_P + 8192;                      // 2 x 16 KiB
    static constexpr uint32_t OFF_FQ = OFF_FK + 2 * 16384;                // 2 x 16 KiB
    static constexpr uint32_t OFF_HB = OFF_FQ + 2 * 16384;                // 2 x 128 rows
    // z entering the chunk, one 128-row tile per buffer in hb's layout with z in
    // column 0 and zeros elsewhere: hb and zb form one B operand of 2 D columns
    // (two MN atoms LBO_HZ bytes apart), so T and Tn come from one product
    static constexpr uint32_t OFF_ZB = OFF_HB + 2 * kSlab * RB;           // 2 x 128 rows
    static constexpr uint32_t LBO_HZ = OFF_ZB - OFF_HB;
    static constexpr uint32_t OFF_ONES = OFF_ZB + 2 * kSlab * RB;         // 64 x 32 B
    static constexpr uint32_t OFF_PART = OFF_ONES + 2048;                 // 2 x 64 x PR fp32
    static constexpr uint32_t OFF_RES = OFF_PART + 2 * kC * PR * 4;       // ROWS x PR fp32
    static constexpr uint32_t OFF_MISC = (OFF_RES + ROWS * PR * 4 + 1023) / 1024 * 1024;
    static constexpr uint32_t SMEM = OFF_MISC + 2048 + 1024;
    // tensor memory columns
    static constexpr uint32_t COL_H = 0;                   // kNs x D   h    (M = 128)
    static constexpr uint32_t COL_Z = COL_H + kNs * D;     // kNs x 16  z    (M = 128)
    static constexpr uint32_t COL_S = COL_Z + kNs * 16;    // 64: S, then Y = P V (M = 64)
    static constexpr uint32_t COL_T = COL_S + 64;          // 2 D: partial readout [T | Tn 0...] (M = 64)
    static constexpr uint32_t COL_TN = COL_T + D;          // Tn: first column of the second half
    static_assert(COL_T + 2 * D <= 512, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct Misc {
    float acs2[kC];
    float vfac[kC];  // value factor dt_j of the chunk's tokens (value discretisation)
    float rsum[2][kC];
    float Dh[64];
    float wtot[2];
    uint64_t stage_full[kStages], stage_empty[kStages];
    uint64_t s_full, p_full, y_free, chunk_done;
    uint64_t slab_full[2], slab_done[2];
    uint64_t ready[2], consumed[2];
    uint64_t drain;
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
__device__ __forceinline__ float bf16_at(const uint8_t *p) {
    return __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t *>(p) << 16);
}
template <uint32_t RB>
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t ch) {
    if constexpr (RB == 128) return sw128_chunk(row, ch);
    else return sw64_chunk(row, ch);
}

__device__ void raise_timeout(Misc *misc, DeviceStatus *status, int where) {
    if (status) {
        atomicCAS(&status->code, 0, (int)SSD_ERR_TIMEOUT);
        atomicCAS(&status->detail, 0, where);
    }
    *reinterpret_cast<volatile int *>(&misc->abort_flag) = 1;
}

// kState: the call carries a state in or out (a separate instantiation, so
// that calls without one run none of its code).
template <int D, bool kState>
__global__ void __launch_bounds__(kThreads, 1)
tc_order2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16 *__restrict__ vglob,
                 __nv_bfloat16 *__restrict__ out,
                 const float *__restrict__ dt_p, const float *__restrict__ A_log,
                 const float *__restrict__ dt_bias, const float *__restrict__ Dres,
                 const float *__restrict__ log_decay, int value_dt, int H, int N,
                 int normalize, const float *__restrict__ h0, const float *__restrict__ z0,
                 float *__restrict__ h_out, float *__restrict__ z_out, DeviceStatus *status) {
    using K = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Misc *misc = reinterpret_cast<Misc *>(smem + K::OFF_MISC);
    const volatile int *abort_flag = &misc->abort_flag;
    const uint32_t sbase = smem_u32(smem);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int bh = blockIdx.x / K::R, h = bh % H;
    const int nc = N / kC;
    const int row0 = bh * N;
    // a carried state enters before chunk 0 exactly as the state of a previous
    // chunk does; the normaliser state is tracked when it is used or asked for
    const bool carry = kState && (h0 != nullptr || z0 != nullptr);
    const bool track_z = normalize || (kState && (z0 != nullptr || z_out != nullptr));

    if (tid == 0) {
        if (blockIdx.x == 0 && status) {
            status->code = 0;
            status->detail = 0;
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&misc->stage_full[i], 1);
            mbar_init(&misc->stage_empty[i], 1);
        }
        mbar_init(&misc->s_full, 1);
        mbar_init(&misc->p_full, kTeam);
        mbar_init(&misc->y_free, kTeam);
        mbar_init(&misc->chunk_done, 1);
        mbar_init(&misc->drain, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&misc->slab_full[b], kTeam);
            mbar_init(&misc->slab_done[b], 1);
            mbar_init(&misc->ready[b], K::R);
            mbar_init(&misc->consumed[b], K::R);
        }
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc->tmem_base, 512);
        tmem_relinquish();
    }
    // zb tiles: zero once; only column 0 of each row is written later
    for (int i = tid; i < (int)(2 * kSlab * K::RB / 16); i += kThreads)
        reinterpret_cast<uint4 *>(smem + K::OFF_ZB)[i] = make_uint4(0u, 0u, 0u, 0u);
    // constant B operand: [1, 0, ..., 0] per token (64 rows x 16 bf16, 32B swizzle)
    for (int i = tid; i < kC * 2; i += kThreads) {
        const int r = i >> 1, ch = i & 1;
        *reinterpret_cast<uint4 *>(smem + K::OFF_ONES + sw32_chunk(r, ch)) =
            make_uint4(ch == 0 ? 0x3F80u : 0u, 0u, 0u, 0u);
    }
    if (tid < D) misc->Dh[tid] = Dres ? Dres[h * D + tid] : 0.0f;
    fence_proxy_async_smem();
    tc_fence_before();
    cluster_sync_all();  // every CTA's barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            int issued = 0;
            for (int c = 0; c < nc; ++c) {
                const int st = c % kStages;
                if (c >= kStages &&
                    !mbar_wait_abortable(&misc->stage_empty[st], ((c / kStages) - 1) & 1, abort_flag)) {
                    raise_timeout(misc, status, 10);
                    break;
                }
                uint8_t *dst = smem + K::OFF_STAGE + st * K::STAGE;
                const int r = row0 + c * kC;
                mbar_arrive_expect_tx(&misc->stage_full[st], K::STAGE);
                tma_load_2d(dst, &tm_q, 0, r, &misc->stage_full[st]);
                tma_load_2d(dst + K::TILE, &tm_k, 0, r, &misc->stage_full[st]);
                tma_load_2d(dst + 2 * K::TILE, &tm_v, 0, r, &misc->stage_full[st]);
                ++issued;
            }
            // copies still in flight after an abort land before the CTA exits (bounded)
            for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
                mbar_wait_bounded(&misc->stage_full[c % kStages], (c / kStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = make_idesc_bf16(64, 64, 0, 0);
            constexpr uint32_t idPV = make_idesc_bf16(64, D, 0, 1);
            constexpr uint32_t idU = make_idesc_bf16(128, D, 1, 1);
            constexpr uint32_t idZ = make_idesc_bf16(128, 16, 1, 1);
            constexpr uint32_t idT = make_idesc_bf16(64, D, 0, 1);
            constexpr uint32_t idT2 = make_idesc_bf16(64, 2 * D, 0, 1);  // [T | Tn] in one product
            uint32_t slab_uses[2] = {0, 0};
            bool ok = true;
            for (int c = 0; ok && c < nc; ++c) {
                const int st = c % kStages;
                const uint32_t aQ = sbase + K::OFF_STAGE + st * K::STAGE;
                const uint32_t aK = aQ + K::TILE, aV = aK + K::TILE;
                if (!(ok = mbar_wait_abortable(&misc->stage_full[st], (c / kStages) & 1, abort_flag))) break;
                if (c >= 1 && !(ok = mbar_wait_abortable(&misc->y_free, (c - 1) & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)
                    mma_bf16(tmem + K::COL_S, make_sdesc(aQ + ks * 32, 16, K::SBO, K::SW),
                             make_sdesc(aK + ks * 32, 16, K::SBO, K::SW), idS, ks > 0);
                mma_commit(&misc->s_full);
                if (!(ok = mbar_wait_abortable(&misc->p_full, c & 1, abort_flag))) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_bf16(tmem + K::COL_S, make_sdesc(sbase + K::OFF_P + ks * 32, 16, 1024, kSw128),
                             make_sdesc(aV + ks * 16 * K::RB, 16, K::SBO, K::SW), idPV, ks > 0);
                for (int sl = 0; sl < kNs; ++sl) {
                    const int b = sl & 1;
                    if (!(ok = mbar_wait_abortable(&misc->slab_full[b], slab_uses[b] & 1, abort_flag))) break;
                    ++slab_uses[b];
                    tc_fence_after();
                    const uint32_t fkA = sbase + K::OFF_FK + b * 16384;
                    const uint32_t fqA = sbase + K::OFF_FQ + b * 16384;
                    // h_slab += Fk^T V  (A: features x tokens, MN-major, two 64-feature groups)
#pragma unroll
                    for (int ks = 0; ks < kC / 16; ++ks)
                        mma_bf16(tmem + K::COL_H + sl * D, make_sdesc(fkA + ks * 2048, 8192, 1024, kSw128),
                                 make_sdesc(aV + ks * 16 * K::RB, 16, K::SBO, K::SW), idU,
                                 (c > 0 || carry || ks > 0));
                    if (track_z) {
#pragma unroll
                        for (int ks = 0; ks < kC / 16; ++ks)
                            mma_bf16(tmem + K::COL_Z + sl * 16, make_sdesc(fkA + ks * 2048, 8192, 1024, kSw128),
                                     make_sdesc(sbase + K::OFF_ONES + ks * 512, 16, 256, kSw32), idZ,
                                     (c > 0 || carry || ks > 0));
                    }
                    if (c >= 1 || carry) {
                        // [T | Tn] += Fq [hb | zb]   (A: tokens x features, K-major;
                        // B: the hb and zb tiles as two MN atoms)
                        const uint32_t hbB = sbase + K::OFF_HB + b * kSlab * K::RB;
#pragma unroll
                        for (int ks = 0; ks < kSlab / 16; ++ks) {
                            const uint64_t adesc =
                                make_sdesc(fqA + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024, kSw128);
                            mma_bf16(tmem + K::COL_T, adesc,
                                     make_sdesc(hbB + ks * 16 * K::RB, K::LBO_HZ, K::SBO, K::SW),
                                     normalize ? idT2 : idT, (sl > 0 || ks > 0));
                        }
                    }
                    mma_commit(&misc->slab_done[b]);
                }
                if (!ok) break;
                mma_commit(&misc->chunk_done);
            }
            if (!ok) {
                raise_timeout(misc, status, 20);
                // matrix products still in flight finish before TMEM is released (bounded)
                mma_commit(&misc->drain);
                mbar_wait_bounded(&misc->drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------ compute team
        const int ct = tid - 64;                    // 0..255
        const int g = warp & 3;                     // TMEM lane quarter
        const int hf = (warp - 2) >> 2;             // which half of the columns
        const uint32_t lane_off = (uint32_t)(g * 32) << 16;
        const int frow = g * 32 + lane;             // feature row of a slab (M = 128 layout)
        const int mrow = g * 16 + lane;             // chunk row (M = 64 layout, lane < 16)
        const bool mrow_ok = lane < 16;
        const bool own_row = mrow_ok && mrow / K::ROWS == (int)rank;
        const float A2 = log_decay ? 0.0f : -expf(A_log[h]) * kLog2e;
        const float bias = dt_bias ? dt_bias[h] : 0.0f;  // given whenever dt is used
        const bool elected = ct == 0;
        const int tok = ct & 63, q4 = ct >> 6;      // feature generation: token, 32-feature part
        uint32_t slab_uses[2] = {0, 0};
        float *part0 = reinterpret_cast<float *>(smem + K::OFF_PART);
        float *res = reinterpret_cast<float *>(smem + K::OFF_RES);

        // per-token decay input: the dt projection, or the given log-decay (Algorithm 4)
        const float *dsrc = log_decay ? log_decay : dt_p;
        float dt_next = (ct < kC && nc > 0) ? dsrc[(size_t)row0 + ct] : 0.0f;
        // the dt projection for the value factor, when it is not already dsrc
        const bool vdt_own = value_dt && log_decay;
        float vdt_next = (vdt_own && ct < kC && nc > 0) ? dt_p[(size_t)row0 + ct] : 0.0f;
        bool failed = false;
        // Own rows of chunk cc: sum the R partials (distributed shared memory),
        // release them, then y = (Y + T) / (r + Tn) [+ D v].
        static_assert(K::ROWS * (D / 8) <= kTeam, "one output item per thread");
        auto reduce_output = [&](int cc) -> bool {
            // this thread's output item and its residual input, fetched before the waits
            const int o_rr = ct / (D / 8), o_ch = ct % (D / 8);
            const bool o_live = ct < K::ROWS * (D / 8);
            const size_t o_grow = (size_t)row0 + (size_t)cc * kC + rank * K::ROWS + o_rr;
            uint4 vu = make_uint4(0u, 0u, 0u, 0u);
            if (Dres && o_live) vu = __ldg(reinterpret_cast<const uint4 *>(vglob + o_grow * D + o_ch * 8));
            const bool bad = !mbar_wait_cluster(&misc->ready[cc & 1], (cc >> 1) & 1, abort_flag);
            if (named_bar_any(1, kTeam, bad)) {
                if (elected) raise_timeout(misc, status, 34);
                return false;
            }
            {
                constexpr int NV = D / 4 + 1;  // float4 groups of a row, plus the normaliser
                const uint32_t pb = smem_u32(part0 + (cc & 1) * kC * K::PR);
                for (int it = ct; it < K::ROWS * NV; it += kTeam) {
                    const int rr = it / NV, v = it % NV;
                    const int row = rank * K::ROWS + rr;
                    const uint32_t off = (uint32_t)(row * K::PR + (v < D / 4 ? v * 4 : D)) * 4u;
                    // all R remote loads are issued before any is used, so their
                    // latencies overlap
                    if (v < D / 4) {
                        float4 x[K::R];
#pragma unroll
                        for (int r2 = 0; r2 < K::R; ++r2) x[r2] = ld_dsmem_f4(mapa_shared(pb + off, r2));
                        float4 acc = x[0];
#pragma unroll
                        for (int r2 = 1; r2 < K::R; ++r2) {
                            acc.x += x[r2].x;
                            acc.y += x[r2].y;
                            acc.z += x[r2].z;
                            acc.w += x[r2].w;
                        }
                        *reinterpret_cast<float4 *>(res + rr * K::PR + v * 4) = acc;
                    } else {
                        float x[K::R];
#pragma unroll
                        for (int r2 = 0; r2 < K::R; ++r2) x[r2] = ld_dsmem_f1(mapa_shared(pb + off, r2));
                        float acc = x[0];
#pragma unroll
                        for (int r2 = 1; r2 < K::R; ++r2) acc += x[r2];
                        res[rr * K::PR + D] = acc;
                    }
                }
            }
            named_bar_sync(1, kTeam);
            if (ct < K::R) {
                fence_acq_rel_cluster();
                mbar_arrive_cluster(mapa_shared(smem_u32(&misc->consumed[cc & 1]), ct));
            }
            if (o_live) {
                const int rr = o_rr, ch = o_ch;
                const size_t grow = o_grow;
                const float *rrow = res + rr * K::PR;
                const float inv = normalize ? 1.0f / rrow[D] : 1.0f;
                const uint32_t vw[4] = {vu.x, vu.y, vu.z, vu.w};
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c2 = ch * 8 + 2 * e;
                    float y0 = rrow[c2] * inv, y1 = rrow[c2 + 1] * inv;
                    if (Dres) {
                        const float2 vf = bf2_to_f2(vw[e]);
                        y0 = fmaf(misc->Dh[c2], vf.x, y0);
                        y1 = fmaf(misc->Dh[c2 + 1], vf.y, y1);
                    }
                    w[e] = pack_bf16x2(y0, y1);
                }
                *reinterpret_cast<uint4 *>(out + grow * D + ch * 8) = make_uint4(w[0], w[1], w[2], w[3]);
            }
            named_bar_sync(1, kTeam);  // res is reused by the next reduction
            return true;
        };
        for (int c = 0; c < nc; ++c) {
            const int st = c % kStages;
            uint8_t *sQ = smem + K::OFF_STAGE + st * K::STAGE;
            uint8_t *sK = sQ + K::TILE;
            uint8_t *sV = sK + K::TILE;
            const float dtv = dt_next;
            if (ct < kC && c + 1 < nc) dt_next = dsrc[(size_t)row0 + (size_t)(c + 1) * kC + ct];
            const float vdt = vdt_own ? vdt_next : dtv;
            if (vdt_own && ct < kC && c + 1 < nc) vdt_next = dt_p[(size_t)row0 + (size_t)(c + 1) * kC + ct];

            bool bad = !mbar_wait_abortable(&misc->stage_full[st], (c / kStages) & 1, abort_flag);
            // ---- decay (tokens 0..63 on threads 0..63)
            float a = 0.0f;
            if (ct < kC) {
                a = log_decay ? dtv * kLog2e : A2 * softplus_f(dtv + bias);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, a, o);
                    if (lane >= o) a += y;
                }
                if (lane == 31) misc->wtot[ct >> 5] = a;
                if (value_dt) misc->vfac[ct] = softplus_f(vdt + bias);
            }
            if (named_bar_any(1, kTeam, bad)) {  // also publishes wtot[] and vfac[]
                if (elected) raise_timeout(misc, status, 30);
                break;
            }
            if (value_dt) {
                // value discretisation: V <- diag(dt) V in place, before P V and the
                // state products read it (both wait for p_full below); the
                // normaliser and the D residual use the raw scores and v
                constexpr int CPR = D / 8;  // 16-byte chunks per row
                for (int t = ct; t < kC * CPR; t += kTeam) {
                    const int r = t / CPR, ch = t % CPR;
                    uint4 *pv = reinterpret_cast<uint4 *>(sV + swz<K::RB>(r, ch));
                    const float f = misc->vfac[r];
                    const float2 f2 = make_float2(f, f);
                    const uint4 x = *pv;
                    uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 y = __fmul2_rn(bf2_to_f2(w[e]), f2);
                        w[e] = pack_bf16x2(y.x, y.y);
                    }
                    *pv = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            if (ct >= 32 && ct < kC) a += misc->wtot[0];
            if (ct < kC) misc->acs2[ct] = a;
            const float lam2 = misc->wtot[0] + misc->wtot[1];

            // ---- P = S^2 2^(acs_i - acs_j) [i >= j]: row mrow, columns [32 hf, 32 hf + 32)
            bad = !mbar_wait_abortable(&misc->s_full, c & 1, abort_flag);
            if (named_bar_any(1, kTeam, bad)) {  // also publishes acs2[]
                if (elected) raise_timeout(misc, status, 31);
                break;
            }
            tc_fence_after();
            {
                float sv[32];
                tmem_ld32(tmem + lane_off + K::COL_S + hf * 32, sv);
                tmem_wait_ld();
                if (own_row) {  // rows of other CTAs are never read back from Y
                    const float ai = misc->acs2[mrow];
                    float rs = 0.0f;
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        const int j = hf * 32 + e;
                        float p0 = sv[e] * sv[e] * ex2_approx(ai - misc->acs2[j]);
                        float p1 = sv[e + 1] * sv[e + 1] * ex2_approx(ai - misc->acs2[j + 1]);
                        if (j > mrow) p0 = 0.0f;
                        if (j + 1 > mrow) p1 = 0.0f;
                        rs += p0 + p1;
                        pk[e >> 1] = pack_bf16x2(p0, p1);
                    }
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        *reinterpret_cast<uint4 *>(smem + K::OFF_P + sw128_chunk(mrow, hf * 4 + k4)) =
                            make_uint4(pk[k4 * 4], pk[k4 * 4 + 1], pk[k4 * 4 + 2], pk[k4 * 4 + 3]);
                    misc->rsum[hf][mrow] = rs;
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            mbar_arrive(&misc->p_full);

            // ---- state slabs
            const float acs_tok = misc->acs2[tok];
            const float wk = ex2_approx(lam2 - acs_tok);   // w_j for F_k
            const float sqs = ex2_approx(acs_tok);         // 2^acs_i for F_q
            const float dec = ex2_approx(lam2);            // decay over the whole chunk
            for (int sl = 0; sl < kNs; ++sl) {
                const int b = sl & 1;
                if (slab_uses[b] > 0) {
                    bad = !mbar_wait_abortable(&misc->slab_done[b], (slab_uses[b] - 1) & 1, abort_flag);
                    if (named_bar_any(1, kTeam, bad)) {
                        if (elected) raise_timeout(misc, status, 32);
                        goto done;
                    }
                    tc_fence_after();
                }
                // h_{c-1} of this slab -> bf16, then h *= 2^lam (columns [hf D/2, hf D/2 + D/2));
                // z likewise (column 0, half 0 only).  Before chunk 0 the state
                // is the carried one, read from global memory (zero if absent).
                if (c >= 1 || carry) {
                    constexpr int HC = D / 2;
                    float hv[HC];
                    float zv = 0.0f;
                    const uint32_t ta = tmem + lane_off + K::COL_H + sl * D + hf * HC;
                    const size_t m = (size_t)bh * D * D + rank * kFs + sl * kSlab + frow;  // feature row
                    if (c >= 1) {
                        if constexpr (HC == 32) tmem_ld32(ta, hv);
                        else tmem_ld16(ta, hv);
                        if (track_z && hf == 0) zv = tmem_ld1(tmem + lane_off + K::COL_Z + sl * 16);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int j = 0; j < HC; j += 4) {
                            const float4 x = h0 ? *reinterpret_cast<const float4 *>(h0 + m * D + hf * HC + j)
                                                : make_float4(0.f, 0.f, 0.f, 0.f);
                            hv[j] = x.x;
                            hv[j + 1] = x.y;
                            hv[j + 2] = x.z;
                            hv[j + 3] = x.w;
                        }
                        if (track_z && hf == 0 && z0) zv = z0[m];
                    }
                    uint8_t *hb = smem + K::OFF_HB + b * kSlab * K::RB;
#pragma unroll
                    for (int ch = 0; ch < HC / 8; ++ch)
                        *reinterpret_cast<uint4 *>(hb + swz<K::RB>(frow, hf * (HC / 8) + ch)) =
                            make_uint4(pack_bf16x2(hv[ch * 8], hv[ch * 8 + 1]),
                                       pack_bf16x2(hv[ch * 8 + 2], hv[ch * 8 + 3]),
                                       pack_bf16x2(hv[ch * 8 + 4], hv[ch * 8 + 5]),
                                       pack_bf16x2(hv[ch * 8 + 6], hv[ch * 8 + 7]));
                    const float2 d2 = make_float2(dec, dec);
#pragma unroll
                    for (int e = 0; e < HC; e += 2) {
                        const float2 r2 = __fmul2_rn(make_float2(hv[e], hv[e + 1]), d2);
                        hv[e] = r2.x;
                        hv[e + 1] = r2.y;
                    }
                    if constexpr (HC == 32) tmem_st32(ta, hv);
                    else tmem_st16(ta, hv);
                    if (track_z && hf == 0) {
                        // column 0 of the zb row; the rest of the tile stays zero
                        uint8_t *zb = smem + K::OFF_ZB + b * kSlab * K::RB;
                        *reinterpret_cast<uint4 *>(zb + swz<K::RB>(frow, 0)) =
                            make_uint4(pack_bf16x2(zv, 0.0f), 0u, 0u, 0u);
                        tmem_st1(tmem + lane_off + K::COL_Z + sl * 16, zv * dec);
                    }
                }
                // features: token `tok`, slab-local features [32 q4, 32 q4 + 32)
                {
                    const int fl0 = q4 * 32;
                    const int a = (int)(rank * kFs + sl * kSlab + fl0) / D;  // first index of the pair
                    const int b0 = (rank * kFs + sl * kSlab + fl0) % D;
                    const float ka = bf16_at(sK + swz<K::RB>(tok, a >> 3) + (a & 7) * 2);
                    const float qa = bf16_at(sQ + swz<K::RB>(tok, a >> 3) + (a & 7) * 2);
                    const float2 sk2 = make_float2(wk * ka, wk * ka), sq2 = make_float2(sqs * qa, sqs * qa);
                    uint8_t *fk = smem + K::OFF_FK + b * 16384 + (fl0 >> 6) * 8192;
                    uint8_t *fq = smem + K::OFF_FQ + b * 16384 + (fl0 >> 6) * 8192;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        const int bb = b0 + ch * 8;
                        const uint4 ku = *reinterpret_cast<const uint4 *>(sK + swz<K::RB>(tok, bb >> 3));
                        const uint4 qu = *reinterpret_cast<const uint4 *>(sQ + swz<K::RB>(tok, bb >> 3));
                        const uint32_t kw[4] = {ku.x, ku.y, ku.z, ku.w}, qw[4] = {qu.x, qu.y, qu.z, qu.w};
                        uint32_t ok4[4], oq4[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 kv = __fmul2_rn(bf2_to_f2(kw[e]), sk2);
                            const float2 qv = __fmul2_rn(bf2_to_f2(qw[e]), sq2);
                            ok4[e] = pack_bf16x2(kv.x, kv.y);
                            oq4[e] = pack_bf16x2(qv.x, qv.y);
                        }
                        const int cidx = ((fl0 & 63) >> 3) + ch;  // 16B chunk in the 128B feature row
                        *reinterpret_cast<uint4 *>(fk + sw128_chunk(tok, cidx)) =
                            make_uint4(ok4[0], ok4[1], ok4[2], ok4[3]);
                        *reinterpret_cast<uint4 *>(fq + sw128_chunk(tok, cidx)) =
                            make_uint4(oq4[0], oq4[1], oq4[2], oq4[3]);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                fence_proxy_async_smem();
                mbar_arrive(&misc->slab_full[b]);
                ++slab_uses[b];
            }

            // ---- the previous chunk's cluster reduction and output run here,
            // while this chunk's last slab products are still on the tensor core
            if (c >= 1 && !reduce_output(c - 1)) {
                failed = true;
                break;
            }

            // ---- this CTA's partial (plus Y and r on its own rows) into part[c & 1]
            bad = !mbar_wait_abortable(&misc->chunk_done, c & 1, abort_flag);
            bad = bad || (c >= 2 && !mbar_wait_cluster(&misc->consumed[c & 1], ((c >> 1) - 1) & 1, abort_flag));
            if (named_bar_any(1, kTeam, bad)) {
                if (elected) raise_timeout(misc, status, 33);
                failed = true;
                break;
            }
            tc_fence_after();
            {
                constexpr int HC = D / 2;
                float tv[HC], yv[HC];
                const uint32_t tt = tmem + lane_off + K::COL_T + hf * HC;
                const uint32_t ty = tmem + lane_off + K::COL_S + hf * HC;
                if constexpr (HC == 32) {
                    tmem_ld32(tt, tv);
                    tmem_ld32(ty, yv);
                } else {
                    tmem_ld16(tt, tv);
                    tmem_ld16(ty, yv);
                }
                const float tn = (normalize && hf == 0) ? tmem_ld1(tmem + lane_off + K::COL_TN) : 0.0f;
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&misc->y_free);
                if (mrow_ok) {
                    float *prow = part0 + (c & 1) * kC * K::PR + mrow * K::PR;
#pragma unroll
                    for (int e = 0; e < HC; e += 4) {
                        float4 v = (c >= 1 || carry) ? make_float4(tv[e], tv[e + 1], tv[e + 2], tv[e + 3])
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                        if (own_row) {
                            v.x += yv[e];
                            v.y += yv[e + 1];
                            v.z += yv[e + 2];
                            v.w += yv[e + 3];
                        }
                        *reinterpret_cast<float4 *>(prow + hf * HC + e) = v;
                    }
                    if (hf == 0)
                        prow[D] = ((c >= 1 || carry) ? tn : 0.0f) +
                                  (own_row ? misc->rsum[0][mrow] + misc->rsum[1][mrow] : 0.0f);
                }
            }
            named_bar_sync(1, kTeam);
            // thread r announces this CTA's partial to cluster CTA r; the R remote
            // arrivals (each a cluster-scope release) run in parallel
            if (ct < K::R) {
                fence_acq_rel_cluster();
                mbar_arrive_cluster(mapa_shared(smem_u32(&misc->ready[c & 1]), ct));
            }
            // the stage is no longer read: features are built, the products are
            // done and the output reads v from global memory
            if (elected) mbar_arrive(&misc->stage_empty[st]);
        }
        if (!failed && nc >= 1) reduce_output(nc - 1);
        // the state after the last token: TMEM holds it once the last chunk's
        // products are done (waited for above)
        if (kState && !failed && (h_out || z_out)) {
            tc_fence_after();
            constexpr int HC = D / 2;
            for (int sl = 0; sl < kNs; ++sl) {
                const size_t m = (size_t)bh * D * D + rank * kFs + sl * kSlab + frow;
                if (h_out) {
                    float hv[HC];
                    const uint32_t ta = tmem + lane_off + K::COL_H + sl * D + hf * HC;
                    if constexpr (HC == 32) tmem_ld32(ta, hv);
                    else tmem_ld16(ta, hv);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < HC; j += 4)
                        *reinterpret_cast<float4 *>(h_out + m * D + hf * HC + j) =
                            make_float4(hv[j], hv[j + 1], hv[j + 2], hv[j + 3]);
                }
                if (z_out) {
                    const float zv = tmem_ld1(tmem + lane_off + K::COL_Z + sl * 16);
                    tmem_wait_ld();
                    if (hf == 0) z_out[m] = zv;
                }
            }
        }
    done:;
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync_all();  // no CTA leaves while another may still read its shared memory
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

// [rows, d] bf16 row-major tensor, boxes of 64 rows, swizzle = row bytes.
bool make_tmap(CUtensorMap *m, const void *base, uint64_t rows, int d) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {(cuuint32_t)d, kC};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     d == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D>
int launch_d(const FwdArgs &a) {
    using K = Cfg<D>;
    const uint64_t rows = (uint64_t)a.B * a.H * a.N;
    CUtensorMap tq, tk, tv;
    if (!make_tmap(&tq, a.q, rows, D) || !make_tmap(&tk, a.k, rows, D) || !make_tmap(&tv, a.v, rows, D))
        return SSD_ERR_CUDA;
    const bool state = a.h0 || a.z0 || a.h_out || a.z_out;
    auto kern = state ? tc_order2_kernel<D, true> : tc_order2_kernel<D, false>;
    static std::atomic<uint64_t> attr_set{0};  // one bit per device and instantiation
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SSD_ERR_CUDA;
    const uint64_t bit = 1ull << (2 * (dev & 31) + (state ? 1 : 0));
    if (!(attr_set.load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::SMEM) != cudaSuccess)
            return SSD_ERR_CUDA;
        attr_set.fetch_or(bit);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B * a.H * K::R);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = K::SMEM;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = K::R;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    DeviceStatus *status = reinterpret_cast<DeviceStatus *>(a.workspace);
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv,
                                       static_cast<const __nv_bfloat16 *>(a.v),
                                       static_cast<__nv_bfloat16 *>(a.out), a.dt_p, a.A_log,
                                       a.dt_bias, a.D, a.log_decay, a.value_dt, a.H, a.N, a.normalize,
                                       a.h0, a.z0, a.h_out, a.z_out, status);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace

bool tc_order2_supports(int B, int H, int N, int d, int dtype, int chunk) {
    return dtype == SSD_BF16 && (d == 32 || d == 64) && chunk == kC &&
           (long long)B * H * N < (1ll << 31);
}

size_t tc_order2_workspace(int, int, int, int, int) { return 0; }

int launch_tc_order2(const FwdArgs &a, const Plan &) {
    return a.d == 64 ? launch_d<64>(a) : launch_d<32>(a);
}

}  // namespace ssd
