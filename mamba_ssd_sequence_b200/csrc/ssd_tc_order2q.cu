// Order-2 (2Mamba, squared scores) operator in its masked quadratic form
// (2Mamba2Furious, Algorithm 5: the causal, decay-masked score matrix with
// the scores squared) as tcgen05/TMEM tensor-core tiles, for calls that carry
// no state in or out: bf16, d_h = D in {32, 64}, N a multiple of 128.
//
//   w_ij = (q_i . k_j)^2 2^(A_i - A_j)  for j <= i        (A: cumulative log2-decay)
//   y_i  = sum_j w_ij f_j v_j  [/ sum_j w_ij]  [+ D (.) v_i]   (f_j = dt_j under value
//                                                          discretisation, else 1)
// The chunked state form (ssd_tc_order2.cu) carries a D^2 x D state per head;
// this form never builds it.  Per 128-row query tile I of a head it walks the
// key tiles J = I, I - 1, ... as a flash-style loop, the tensor core doing
//   S = Q_I K_J^T      (M = 128, N = 128, K = D; into one of two TMEM buffers)
//   Y += P V_J         (M = 128, N = D, K = 128; P read from TMEM)
// while eight compute warps form P = S^2 (.) decay from the other buffer and
// write it back over S as bf16.  The decay of a key tile factors through its
// last key: for J < I,
//   2^(A_i - A_j) = 2^(a_i + G_J) 2^(lam_J - a_j),
// with a the tile-local inclusive cumulative decay, lam_J the decay over
// tile J and G_J the decay over the tiles strictly between J and I; both
// factors are <= 1.  The diagonal tile takes the exact per-element factor
// and the causal mask.  Once G_J < -200 every weight of tile J and of all
// earlier tiles is below 2^-200 times a squared score, which rounds to a zero
// bf16 P: those tiles are skipped (the row sum changes below fp32
// resolution).  The row sums of w (the normaliser, without f) accumulate in
// registers.  Kernel (a) runs first (quad_decay_kernel): the tile-local
// cumulative decay, lam per tile, the factor 2^(lam - a) and f per token.
//
// Roles (320 threads): warp 0 TMA (Q tiles, double-buffered; K, V tiles
// through a ring of four stages); warp 1 MMA issue (S of step s + 1 goes
// out before P V of step s); warps 2-9 the compute team (P, then each
// query tile's epilogue: y = Y / n [+ D v], staged in shared memory and
// written by one TMA store).  CTAs take the query tiles one at a time from a
// counter in the workspace (which kernel (a) zeroes), the latest tiles, whose
// key ranges are the longest, first: where a head's decay skips its early
// tiles, work per query tile differs from head to head.  Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "ptx.cuh"
#include "ssd_internal.h"

namespace ssd {
namespace {

using namespace ptx;

constexpr int kT = 128;              // tokens per tile
constexpr int kNS = 4;               // K, V stages
constexpr int kSB = 2;               // S buffers in TMEM
constexpr int kCT = 256;             // compute threads
constexpr int kQThreads = 64 + kCT;
constexpr uint32_t kQBar = 1;        // named barrier of the compute team
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSkipLog2 = -200.0f;  // key tiles whose decay to the query tile is below 2^this are skipped

template <int D>
struct QCfg {
    static constexpr uint32_t RB = D * 2;                  // bytes per bf16 row
    static constexpr uint32_t SW = RB == 128 ? 2u : 4u;    // descriptor swizzle: 128 or 64 bytes
    static constexpr uint32_t SBO = 8 * RB;                // 8-row swizzle atom
    static constexpr uint32_t TILE = kT * RB;              // one 128-row tile
    static constexpr uint32_t OFF_Q = 0;                   // 2 x TILE
    static constexpr uint32_t OFF_KV = 2 * TILE;           // kNS x (K | V | key factors)
    // per stage: the key tile, the value tile, then the key tile's 2^(lam - a_j),
    // a_j and f_j (128 floats each), brought by the same TMA transaction
    static constexpr uint32_t FAC = 3 * kT * 4;
    static constexpr uint32_t STAGE = (2 * TILE + FAC + 1023) / 1024 * 1024;
    static constexpr uint32_t OFF_OUT = OFF_KV + kNS * STAGE;  // 2 x TILE: output staging per Y buffer
    static constexpr uint32_t OFF_MISC = OFF_OUT + 2 * TILE;
    static constexpr uint32_t SMEM = OFF_MISC + 2048 + 1024;
    // TMEM: S buffers at 128 b (P packed over columns [64 h, 64 h + 32) of
    // each half h), then the two Y buffers
    static constexpr uint32_t COL_Y = 128 * kSB;
    static_assert(COL_Y + 2 * D <= 512, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(STAGE % 1024 == 0 && TILE % 1024 == 0, "swizzle atoms");
};

struct QMisc {
    uint64_t item_full[2], item_empty[2];  // the work item the TMA warp took, to the other roles
    long long item[2];
    uint64_t q_full[2], q_empty[2];
    uint64_t st_full[kNS], st_empty[kNS];
    uint64_t s_full[kSB], p_full[kSB], pv_done[kSB];
    uint64_t y_full[2], ep_done[2];
    uint64_t drain;
    float rs[2][kT];  // the two column halves' row sums of w
    uint32_t tmem;
    int abort_flag;
};
static_assert(sizeof(QMisc) <= 2048, "misc block");

__device__ __forceinline__ float softplus_f(float x) {
    return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
template <uint32_t RB>
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t ch) {
    if constexpr (RB == 128) return sw128_chunk(row, ch);
    else return sw64_chunk(row, ch);
}

__device__ void q_timeout(DeviceStatus *status, int where, int *abort_flag) {
    if (status) {
        atomicCAS(&status->code, 0, (int)SSD_ERR_TIMEOUT);
        atomicCAS(&status->detail, 0, where);
    }
    *reinterpret_cast<volatile int *>(abort_flag) = 1;
}

// The key tiles of query tile I of a head: J = I, I - 1, ..., while the decay
// over the tiles strictly between J and I stays >= 2^kSkipLog2.  Every role
// walks them with the same arithmetic, so all agree on the steps.
struct Walk {
    const float *lam_h;  // the head's tile totals
    int I, J;
    float G;  // log2-decay over tiles J + 1 .. I - 1
    __device__ __forceinline__ bool next() {  // advance to the next key tile; false when done
        if (J == 0) return false;
        --J;
        if (J <= I - 2) {
            G += lam_h[J + 1];
            if (G < kSkipLog2) return false;
        }
        return true;
    }
};


// Kernel (a) of this path: per 128-token tile of a head, the tile-local
// inclusive cumulative log2-decay a_t, the tile total lam, the key factor
// 2^(lam - a_t) and the value factor f_t = dt_t (value discretisation).
__global__ void __launch_bounds__(kT)
quad_decay_kernel(const float *__restrict__ dt_p, const float *__restrict__ A_log,
                  const float *__restrict__ dt_bias, const float *__restrict__ log_decay, int value_dt, int H,
                  int N, float *__restrict__ acs, float *__restrict__ colf, float *__restrict__ fval,
                  float *__restrict__ lam, int *__restrict__ next_item) {
    __shared__ float wsum[kT / 32];
    __shared__ float total_s;
    const int NT = N / kT;
    const int tile = blockIdx.x, bh = tile / NT, h = bh % H;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const size_t tok = (size_t)tile * kT + t;
    if (tile == 0 && t == 0) *next_item = 0;  // the work counter of the kernel that follows
    float dt = 0.0f;
    if (!log_decay || value_dt) dt = softplus_f(dt_p[tok] + dt_bias[h]);
    const float a = log_decay ? log_decay[tok] * kLog2e : (-expf(A_log[h]) * kLog2e) * dt;
    float incl = a;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    float off = 0.0f;
    for (int i = 0; i < w; ++i) off += wsum[i];
    incl += off;
    if (t == kT - 1) total_s = incl;  // lam: the last token's inclusive sum, so 2^(lam - a) = 1 there
    __syncthreads();
    const float total = total_s;
    acs[tok] = incl;
    colf[tok] = ex2_approx(total - incl);
    if (value_dt) fval[tok] = dt;
    if (t == kT - 1) lam[tile] = total;
}

template <int D>
__global__ void __launch_bounds__(kQThreads, 1)
tc_order2q_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                  const __nv_bfloat16 *__restrict__ vglob, const float *__restrict__ acs,
                  const float *__restrict__ colf, const float *__restrict__ fval, const float *__restrict__ lam,
                  const float *__restrict__ Dres, int BH, int H, int N, int normalize, int *__restrict__ next_item,
                  DeviceStatus *status, int dbg_skip, unsigned long long wait_ns) {
    using K = QCfg<D>;
    constexpr uint32_t RB = K::RB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    QMisc *misc = reinterpret_cast<QMisc *>(smem + K::OFF_MISC);
    const volatile int *abort_flag = &misc->abort_flag;
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int NT = N / kT;
    // work items t = 0, 1, ...: query tile I = NT - 1 - t / BH of head bh = t %
    // BH, longest key ranges first; CTAs take them one at a time from a
    // counter (the key ranges of different heads end at different tiles)
    const long long n_items = (long long)BH * NT;
    const int cta = (int)blockIdx.x;

    if (tid == 0) {
        if (cta == 0 && status) {
            status->code = 0;
            status->detail = 0;
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&misc->item_full[i], 1);
            mbar_init(&misc->item_empty[i], 1 + kCT);
            mbar_init(&misc->q_full[i], 1);
            mbar_init(&misc->q_empty[i], 1);
            mbar_init(&misc->y_full[i], 1);
            mbar_init(&misc->ep_done[i], kCT);
        }
        for (int i = 0; i < kSB; ++i) {
            mbar_init(&misc->s_full[i], 1);
            mbar_init(&misc->p_full[i], kCT);
            mbar_init(&misc->pv_done[i], 1);
        }
        for (int i = 0; i < kNS; ++i) {
            mbar_init(&misc->st_full[i], 1);
            mbar_init(&misc->st_empty[i], 1);
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

    auto item_of = [&](long long t, int &I, int &bh) {
        I = NT - 1 - (int)(t / BH);
        bh = (int)(t % BH);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
            prefetch_tmap(&tm_out);
            long long kv = 0, ti = 0;
            bool ok = true;
            for (;; ++ti) {
                const int slot = (int)(ti & 1);
                if (ti >= 2 && !mbar_wait_abortable(&misc->item_empty[slot], (uint32_t)(((ti >> 1) - 1) & 1),
                                                    abort_flag, wait_ns)) {
                    ok = false;
                    break;
                }
                const long long t = atomicAdd(next_item, 1);
                misc->item[slot] = t;
                mbar_arrive(&misc->item_full[slot]);
                if (t >= n_items) break;
                int I, bh;
                item_of(t, I, bh);
                const int qb = (int)(ti & 1);
                if (ti >= 2 && !mbar_wait_abortable(&misc->q_empty[qb], (uint32_t)(((ti >> 1) - 1) & 1), abort_flag,
                                                    wait_ns)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&misc->q_full[qb], K::TILE);
                tma_load_2d(smem + K::OFF_Q + qb * K::TILE, &tm_q, 0, bh * N + I * kT, &misc->q_full[qb]);
                Walk wk{lam + (size_t)bh * NT, I, I, 0.0f};
                do {
                    const int st = (int)(kv % kNS);
                    if (kv >= kNS && !mbar_wait_abortable(&misc->st_empty[st], (uint32_t)(((kv / kNS) - 1) & 1),
                                                          abort_flag, wait_ns)) {
                        ok = false;
                        break;
                    }
                    if (kv != dbg_skip) {  // failure test: this stage is never published
                        uint8_t *sp = smem + K::OFF_KV + st * K::STAGE;
                        const size_t key0 = (size_t)bh * N + (size_t)wk.J * kT;
                        mbar_arrive_expect_tx(&misc->st_full[st], 2 * K::TILE + (fval ? 3 : 2) * kT * 4);
                        tma_load_2d(sp, &tm_k, 0, (int)key0, &misc->st_full[st]);
                        tma_load_2d(sp + K::TILE, &tm_v, 0, (int)key0, &misc->st_full[st]);
                        bulk_load(sp + 2 * K::TILE, colf + key0, kT * 4, &misc->st_full[st]);
                        bulk_load(sp + 2 * K::TILE + kT * 4, acs + key0, kT * 4, &misc->st_full[st]);
                        if (fval) bulk_load(sp + 2 * K::TILE + 2 * kT * 4, fval + key0, kT * 4, &misc->st_full[st]);
                    }
                    ++kv;
                } while (wk.next());
            }
            if (!ok) q_timeout(status, 201, &misc->abort_flag);
            // copies still in flight after an abort land before the CTA exits (bounded)
            for (long long j = kv > kNS ? kv - kNS : 0; j < kv; ++j)
                if (j != dbg_skip) mbar_wait_bounded(&misc->st_full[j % kNS], (uint32_t)((j / kNS) & 1));
            if (ok && ti >= 1) mbar_wait_bounded(&misc->q_full[(ti - 1) & 1], (uint32_t)(((ti - 1) >> 1) & 1));
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = make_idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idPV = make_idesc_bf16(128, D, 0, 1);
            constexpr uint64_t kStepRows = (16 * RB) >> 4;  // descriptor units per 16 rows
            bool ok = true;
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                ok = ok && mbar_wait_abortable(bar, parity, abort_flag, wait_ns);
                return ok;
            };
            struct Pend {
                long long s, ti;
                int st, first, last;
            };
            Pend pv{-1, 0, 0, 0, 0};
            // Y += P V of step p.s (its P in S buffer s % kSB, its V in stage st)
            auto issue_pv = [&](const Pend &p) {
                const int sb = (int)(p.s % kSB), yb = (int)(p.ti & 1);
                if (!wait(&misc->p_full[sb], (uint32_t)((p.s / kSB) & 1))) return;
                if (p.first && p.ti >= 2 && !wait(&misc->ep_done[yb], (uint32_t)(((p.ti >> 1) - 1) & 1))) return;
                tc_fence_after();
                const uint64_t dV = make_sdesc(sbase + K::OFF_KV + p.st * K::STAGE + K::TILE, 16, K::SBO, K::SW);
#pragma unroll
                for (int ks = 0; ks < kT / 16; ++ks)
                    mma_bf16_ts(tmem + K::COL_Y + D * yb, tmem + 128 * sb + 64 * (ks >> 2) + 8 * (ks & 3),
                                dV + ks * kStepRows, idPV, (!p.first || ks > 0) ? 1u : 0u);
                mma_commit(&misc->pv_done[sb]);
                mma_commit(&misc->st_empty[p.st]);
                if (p.last) {
                    mma_commit(&misc->y_full[yb]);
                    mma_commit(&misc->q_empty[p.ti & 1]);
                }
            };
            long long kv = 0, s = 0, ti = 0;
            for (; ok; ++ti) {
                const int slot = (int)(ti & 1);
                if (!wait(&misc->item_full[slot], (uint32_t)((ti >> 1) & 1))) break;
                const long long t = misc->item[slot];
                mbar_arrive(&misc->item_empty[slot]);
                if (t >= n_items) break;
                int I, bh;
                item_of(t, I, bh);
                const int qb = (int)(ti & 1);
                if (!wait(&misc->q_full[qb], (uint32_t)((ti >> 1) & 1))) break;
                const uint64_t dQ = make_sdesc(sbase + K::OFF_Q + qb * K::TILE, 16, K::SBO, K::SW);
                Walk wk{lam + (size_t)bh * NT, I, I, 0.0f};
                bool more = true;
                while (more && ok) {
                    const int sb = (int)(s % kSB), st = (int)(kv % kNS);
                    const bool first = wk.J == I;
                    more = wk.next();
                    // the S buffer: the P V of step s - kSB has read its P
                    if (s >= kSB && !wait(&misc->pv_done[sb], (uint32_t)(((s / kSB) - 1) & 1))) break;
                    if (!wait(&misc->st_full[st], (uint32_t)((kv / kNS) & 1))) break;
                    tc_fence_after();
                    const uint64_t dK = make_sdesc(sbase + K::OFF_KV + st * K::STAGE, 16, K::SBO, K::SW);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks)
                        mma_bf16(tmem + 128 * sb, dQ + ks * 2, dK + ks * 2, idS, ks > 0 ? 1u : 0u);
                    mma_commit(&misc->s_full[sb]);
                    if (pv.s >= 0) issue_pv(pv);
                    pv = Pend{s, ti, st, first ? 1 : 0, more ? 0 : 1};
                    ++s;
                    ++kv;
                }
            }
            if (ok && pv.s >= 0) issue_pv(pv);
            if (!ok) {
                q_timeout(status, 202, &misc->abort_flag);
                // products still in flight finish before TMEM is released (bounded)
                mma_commit(&misc->drain);
                mbar_wait_bounded(&misc->drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------ compute team
        const int g = warp & 3;              // TMEM lane quarter
        const int hf = (warp - 2) >> 2;      // half of the key (and output) columns
        const uint32_t lane_off = (uint32_t)(g * 32) << 16;
        const int r = g * 32 + lane;         // row of the query tile
        const int ct = tid - 64;
        bool failed = false;
        long long s = 0, ti = 0;
        for (;; ++ti) {
            const int slot = (int)(ti & 1);
            const bool badi = !mbar_wait_abortable(&misc->item_full[slot], (uint32_t)((ti >> 1) & 1), abort_flag,
                                                   wait_ns);
            if (named_bar_any(kQBar, kCT, badi)) {
                failed = true;
                break;
            }
            const long long t = misc->item[slot];
            mbar_arrive(&misc->item_empty[slot]);
            if (t >= n_items) break;
            int I, bh;
            item_of(t, I, bh);
            const size_t qtok = (size_t)bh * N + (size_t)I * kT;  // first token of the query tile
            const float ai = acs[qtok + r];
            float rsum = 0.0f;
            Walk wk{lam + (size_t)bh * NT, I, I, 0.0f};
            bool more = true;
            while (more) {
                const int sb = (int)(s % kSB), st = (int)(s % kNS);
                const int J = wk.J;
                const float Gd = wk.G;
                more = wk.next();
                bool bad = !mbar_wait_abortable(&misc->s_full[sb], (uint32_t)((s / kSB) & 1), abort_flag, wait_ns);
                // the stage's key factors are read below: observe its TMA completion
                // too (long complete; the stage is refilled only after this P)
                bad = bad || !mbar_wait_abortable(&misc->st_full[st], (uint32_t)((s / kNS) & 1), abort_flag, wait_ns);
                if (named_bar_any(kQBar, kCT, bad)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                // the key tile's factors: [0, 128) 2^(lam - a_j), [128, 256) a_j, [256, 384) f_j
                const float *fac = reinterpret_cast<const float *>(smem + K::OFF_KV + st * K::STAGE + 2 * K::TILE);
                const float rowf = ex2_approx(ai + Gd);
                const float2 rf2 = make_float2(rowf, rowf);
                float2 rs2 = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    float sv[32];
                    tmem_ld32(tmem + lane_off + 128 * sb + 64 * hf + 32 * pc, sv);
                    tmem_wait_ld();
                    const int kb = 64 * hf + 32 * pc;  // key of sv[0] in the tile
                    const float4 *cf = reinterpret_cast<const float4 *>(fac + (J == I ? kT : 0) + kb);
                    const float4 *fv = reinterpret_cast<const float4 *>(fac + 2 * kT + kb);
                    uint32_t pk[16];
#pragma unroll
                    for (int e4 = 0; e4 < 8; ++e4) {
                        const float4 c4 = cf[e4];
                        float2 w01, w23;
                        if (J == I) {  // exact decay and the causal mask
                            const int jj = kb + 4 * e4;
                            w01 = make_float2(jj <= r ? ex2_approx(ai - c4.x) : 0.0f,
                                              jj + 1 <= r ? ex2_approx(ai - c4.y) : 0.0f);
                            w23 = make_float2(jj + 2 <= r ? ex2_approx(ai - c4.z) : 0.0f,
                                              jj + 3 <= r ? ex2_approx(ai - c4.w) : 0.0f);
                        } else {
                            w01 = __fmul2_rn(make_float2(c4.x, c4.y), rf2);
                            w23 = __fmul2_rn(make_float2(c4.z, c4.w), rf2);
                        }
                        const float2 x01 = make_float2(sv[4 * e4], sv[4 * e4 + 1]);
                        const float2 x23 = make_float2(sv[4 * e4 + 2], sv[4 * e4 + 3]);
                        float2 q01 = __fmul2_rn(__fmul2_rn(x01, x01), w01);
                        float2 q23 = __fmul2_rn(__fmul2_rn(x23, x23), w23);
                        rs2 = __fadd2_rn(rs2, __fadd2_rn(q01, q23));
                        if (fval) {
                            const float4 f4 = fv[e4];
                            q01 = __fmul2_rn(q01, make_float2(f4.x, f4.y));
                            q23 = __fmul2_rn(q23, make_float2(f4.z, f4.w));
                        }
                        pk[2 * e4] = pack_bf16x2(q01.x, q01.y);
                        pk[2 * e4 + 1] = pack_bf16x2(q23.x, q23.y);
                    }
                    // P of keys [kb, kb + 32) as bf16 pairs over columns
                    // [64 hf + 16 pc, +16), which this warp has already read
                    tmem_st16(tmem + lane_off + 128 * sb + 64 * hf + 16 * pc, pk);
                }
                rsum += rs2.x + rs2.y;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&misc->p_full[sb]);
                ++s;
            }
            if (failed) break;
            // ---- epilogue of query tile I: y = Y / n [+ D v]
            const int yb = (int)(ti & 1);
            misc->rs[hf][r] = rsum;
            // the residual row (still in L2) while the last P V runs
            constexpr int NQ = D / 16;  // 16-byte chunks of this thread's half row
            uint4 vres[NQ];
            if (Dres) {
                const uint4 *vp = reinterpret_cast<const uint4 *>(vglob + (qtok + r) * D + hf * (D / 2));
#pragma unroll
                for (int q = 0; q < NQ; ++q) vres[q] = __ldg(vp + q);
            }
            if (ct == 0) bulk_wait_group_read0();  // the staging buffer's previous store has read it
            const bool bad = !mbar_wait_abortable(&misc->y_full[yb], (uint32_t)((ti >> 1) & 1), abort_flag, wait_ns);
            if (named_bar_any(kQBar, kCT, bad)) {  // also publishes rs[][]
                failed = true;
                break;
            }
            tc_fence_after();
            const float n = misc->rs[0][r] + misc->rs[1][r];
            const float inv = normalize ? 1.0f / n : 1.0f;
            float yv[D / 2];
            if constexpr (D == 64) {
                tmem_ld32(tmem + lane_off + K::COL_Y + D * yb + 32 * hf, yv);
            } else {
                tmem_ld16(tmem + lane_off + K::COL_Y + D * yb + 16 * hf, yv);
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&misc->ep_done[yb]);
            const int hh = bh % H;
            uint8_t *ytile = smem + K::OFF_OUT + yb * K::TILE;
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
                const uint32_t vw[4] = {vres[q].x, vres[q].y, vres[q].z, vres[q].w};
                uint32_t wv[4];
#pragma unroll
                for (int pp = 0; pp < 4; ++pp) {
                    const int cl = 8 * q + 2 * pp;  // column within the half
                    float y0 = yv[cl] * inv, y1 = yv[cl + 1] * inv;
                    if (Dres) {
                        const float2 vf = bf2_to_f2(vw[pp]);
                        y0 = fmaf(Dres[hh * D + hf * (D / 2) + cl], vf.x, y0);
                        y1 = fmaf(Dres[hh * D + hf * (D / 2) + cl + 1], vf.y, y1);
                    }
                    wv[pp] = pack_bf16x2(y0, y1);
                }
                *reinterpret_cast<uint4 *>(ytile + swz<RB>(r, NQ * hf + q)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
            fence_proxy_async_smem();
            named_bar_sync(kQBar, kCT);  // the tile is staged; rs[][] may be rewritten
            if (ct == 0) {
                tma_store_2d(&tm_out, ytile, 0, (int)qtok);
                bulk_commit_group();
            }
        }
        if (ct == 0) bulk_wait_group0();  // every output tile has reached global memory
        if (failed && ct == 0) q_timeout(status, 203, &misc->abort_flag);
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------- host side
// [rows, D] bf16, 128-row boxes, swizzled to match the descriptors
bool make_tmap_q(CUtensorMap *m, const void *base, uint64_t rows, int d) {
    return encode_tmap_2d(m, base, true, (uint64_t)d, rows, (uint32_t)d, kT, d == 64 ? 128 : 64);
}

template <int D>
int launch_q(const FwdArgs &a, const Plan &p) {
    using K = QCfg<D>;
    const int BH = a.B * a.H, NT = a.N / kT;
    const uint64_t rows = (uint64_t)BH * a.N;
    CUtensorMap tq, tk, tv, to;
    if (!make_tmap_q(&tq, a.q, rows, D) || !make_tmap_q(&tk, a.k, rows, D) || !make_tmap_q(&tv, a.v, rows, D) ||
        !make_tmap_q(&to, a.out, rows, D))
        return SSD_ERR_CUDA;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    float *acs = reinterpret_cast<float *>(ws + p.acs_off);
    float *colf = reinterpret_cast<float *>(ws + p.state_off);
    float *fval = a.value_dt ? reinterpret_cast<float *>(ws + p.vfac_off) : nullptr;
    float *lam = reinterpret_cast<float *>(ws + p.lam_off);
    int *next_item = reinterpret_cast<int *>(ws + p.aux_off);
    static std::atomic<uint64_t> attr_set{0};  // one bit per device
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return SSD_ERR_CUDA;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(attr_set.load() & bit)) {
        if (cudaFuncSetAttribute(tc_order2q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)K::SMEM) !=
            cudaSuccess)
            return SSD_ERR_CUDA;
        attr_set.fetch_or(bit);
    }
    quad_decay_kernel<<<BH * NT, kT, 0, a.stream>>>(a.dt_p, a.A_log, a.dt_bias, a.log_decay, a.value_dt, a.H, a.N,
                                                   acs, colf, fval, lam, next_item);
    // the CTAs split the query tiles of all heads among themselves
    const long long items = (long long)BH * NT;
    const int grid = items < sms ? (int)items : sms;
    DeviceStatus *status = reinterpret_cast<DeviceStatus *>(a.workspace);
    const unsigned long long wait_ns = a.wait_ns ? a.wait_ns : 1000000000ull;
    tc_order2q_kernel<D><<<grid, kQThreads, K::SMEM, a.stream>>>(
        tq, tk, tv, to, static_cast<const __nv_bfloat16 *>(a.v), acs, colf, fval, lam, a.D, BH, a.H, a.N,
        a.normalize, next_item, status, a.dbg_skip, wait_ns);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace

bool tc_order2q_supports(int B, int H, int N, int d, int dtype) {
    return dtype == SSD_BF16 && (d == 32 || d == 64) && N % kT == 0 && (long long)B * H * N < (1ll << 31) &&
           (long long)B * H <= 65535;
}

// status block | acs (B H N) | key factors (B H N) | value factors (B H N) |
// lam (B H N / 128) | the work counter
void tc_order2q_layout(int B, int H, int N, Plan *p) {
    const size_t tok = (size_t)B * H * N;
    p->acs_off = kStatusBytes;
    p->state_off = align_up(p->acs_off + tok * sizeof(float), 256);
    p->vfac_off = align_up(p->state_off + tok * sizeof(float), 256);
    p->lam_off = align_up(p->vfac_off + tok * sizeof(float), 256);
    p->aux_off = align_up(p->lam_off + tok / kT * sizeof(float), 256);
    p->total = p->aux_off + 256;
}

int launch_tc_order2q(const FwdArgs &a, const Plan &p) {
    if (a.order != 2 || a.h0 || a.z0 || a.h_out || a.z_out) return SSD_ERR_UNSUPPORTED;
    return a.d == 64 ? launch_q<64>(a, p) : launch_q<32>(a, p);
}

}  // namespace ssd
