// Order-2 (2Mamba, squared scores) tensor-core path (tcgen05 + TMEM, TMA) of
// the SSD forward operator for bf16 inputs, d_h = D in {32, 64}, chunk = 64.
//
// Order 2 squares the score: w_ij = (q_i . k_j)^2 2^(acs_i - acs_j), whose
// recurrent form (2Mamba2Furious, Algorithm 6) carries the state
// h = sum_j 2^(A_t - A_j) (k_j (x) k_j) v_j^T of D^2 x D values and the
// normaliser state z = sum_j 2^(A_t - A_j) (k_j (x) k_j).  One head's state
// does not fit one SM at D = 64 (1 MiB), so R = D^2 / 512 CTAs share a head:
// each keeps 512 of the D^2 feature rows of h in tensor memory (fp32), as
// four slabs of 128 rows, and z of those features in registers.  The feature
// of TMEM lane L of slab s of CTA r is (a, b) with
//     a = r (512 / D) + 4 (L / D) + s,   b = L % D,
// so the four slabs of a lane share b, and a warp shares a.
//
// Per chunk c of 64 tokens (acs_t = chunk-local inclusive cumsum of A dt in
// log2 units, lam = acs_63; kernel (a), fused), every CTA, slab by slab:
//   state build   h <- 2^lam h + Fk^T V                    tcgen05, M = 128
//                 Fk[j][(a,b)] = 2^(lam - acs_j) k_ja k_jb (A operand in TMEM)
//                 z <- 2^lam z + sum_j Fk[j]               CUDA cores (fp32)
//   readout       [T | Tn] += Fq [hb | zb]                 tcgen05, M = 64
//                 Fq[i][(a,b)] = 2^acs_i q_ia q_ib         (A operand in smem)
//                 hb, zb = bf16 of the state entering the chunk (B in smem)
// and one CTA of the head (c mod R) adds the chunk's own quadratic part:
//   S = Q K^T,  P_ij = S_ij^2 2^(acs_i - acs_j) [i >= j],  T += P V,
// with the row sums of P added to Tn.  The R partial [T | Tn] of a chunk are
// summed across the head's CTAs -- through distributed shared memory within
// a thread-block cluster at D = 32, through L2 with counters at D = 64 (where
// a cluster of 8 per head would not fit all heads at once) -- and CTA r
// writes rows [64r/R, 64(r+1)/R):   y_i = T_i / Tn_i (normaliser on) [+ D v_i].
// The (q . k)^2 of the quadratic part and (q (x) q) . (k (x) k) of the state
// part are the same inner product (Algorithm 5 against Algorithm 6).
//
// Roles (576 threads): warp 0 the decay warp (kernel (a): the chunk's decay,
// key weights and value discretisation, one chunk ahead; it also requests the
// Q, K, V tiles); warp 1 MMA issue; warps 2-9 the state team (slabs 0, 2 and
// slabs 1, 3: state conversion and scaling, Fk, z); warps 10-13 the query team
// (Fq, P); warps 14-17 the output team (partials, reduction across the head's
// CTAs, output).  Every slab has a buffer of its own in each ring, so a slab's
// preparation for chunk c waits only for that slab's products of chunk c - 1.
// Options: a per-token log-decay and value discretisation (Algorithm 4; V is
// scaled by dt in shared memory, the normaliser and the residual use the raw
// scores and v); a carried state h0, z0 enters as the state before chunk 0,
// and h_out, z_out receive the state after the last chunk.  All exponentials
// are of non-positive arguments.  Every wait is bounded.
#include <cuda.h>
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
constexpr int kMaxStages = 3;   // Q, K, V tile ring (3 at d_h 32, 2 at d_h 64)
constexpr int kNQ = 3;          // Fq ring
constexpr int kNP = 4;          // partial ring of the reduction through L2
constexpr int kSTT = 256;       // state team: warps 2-9
constexpr int kQ1T = 128;       // query team: warps 10-13
constexpr int kQ2T = 128;       // output team: warps 14-17
constexpr int kQ1W0 = (64 + kSTT) / 32;
constexpr int kQ2W0 = kQ1W0 + kQ1T / 32;
constexpr int kThreads = kQ2W0 * 32 + kQ2T;      // warp 0 decay and TMA, warp 1 MMA, the teams
constexpr uint32_t kSw128 = 2, kSw64 = 4;        // descriptor swizzle modes
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kHalf1 = 16u << 16;           // lane offset of the second M = 64 tile
constexpr uint32_t kBarQ2 = 1;                   // named barrier of the output team
constexpr size_t kCounterStride = 64;            // bytes of reduction counters per head
static_assert((2 * kNP + 1) * 4 <= kCounterStride, "counters of a head");

template <int D>
struct Cfg {
    static constexpr int R = D * D / kFs;          // CTAs per head
    static constexpr int ROWS = kC / R;            // output rows owned per CTA
    static constexpr int NA = kFs / D;             // values of a per CTA
    static constexpr uint32_t RB = D * 2;          // bytes per bf16 row of q/k/v/hb
    static constexpr uint32_t SW = RB == 128 ? kSw128 : kSw64;
    static constexpr uint32_t SBO = 8 * RB;        // 8-row swizzle atom
    static constexpr uint32_t TILE = kC * RB;      // q/k/v tile
    static constexpr uint32_t STAGE = 3 * TILE;    // Q | K | V
    static constexpr uint32_t HBT = kSlab * RB;    // hb tile of one slab
    static constexpr int NT = D + 8;               // readout columns: T, Tn, zeros
    static constexpr int PR = D + 4;               // padded partial row (floats)
    static constexpr bool GLOBAL = D == 64;        // reduction through L2 (no cluster)
    static constexpr int STAGES = D == 64 ? 2 : 3;  // Q, K, V tile ring
    // shared memory map (bytes from a 1024-aligned base)
    static constexpr uint32_t OFF_STAGE = 0;
    static constexpr uint32_t OFF_HB = STAGES * STAGE;                  // kNs x 128 rows
    // z of slab s in logical 16-byte chunk s of each row: the readout's
    // descriptor for slab s starts its second N atom 16 s bytes in
    static constexpr uint32_t OFF_ZB = OFF_HB + kNs * HBT;              // 128 rows
    static constexpr uint32_t OFF_FQ = OFF_ZB + HBT;                    // kNQ x 16 KiB
    static constexpr uint32_t OFF_P = OFF_FQ + kNQ * 16384;             // 64 x 64 bf16
    static constexpr uint32_t OFF_PART = OFF_P + 8192;                  // 2 x 64 x PR (cluster only)
    static constexpr uint32_t OFF_RES = OFF_PART + (GLOBAL ? 0 : 2 * kC * PR * 4);  // ROWS x PR
    static constexpr uint32_t OFF_WK = (OFF_RES + ROWS * PR * 4 + 15) / 16 * 16;      // 2 x NA x 32
    // K^T as bf16 pairs of consecutive tokens, per chunk parity: row b holds the
    // 32 pairs of column b, 16-byte chunk j of row b at position j ^ (b % 8)
    static constexpr uint32_t OFF_KT = OFF_WK + 2 * NA * 32 * 4;                      // 2 x D x 128 B
    static constexpr uint32_t OFF_MISC = (OFF_KT + 2 * D * 128 + 1023) / 1024 * 1024;
    static constexpr uint32_t SMEM = OFF_MISC + 2048 + 1024;
    // tensor memory columns.  The readout and S are M = 64 accumulators
    // sharing columns: the readout in lanes 0-15 of each quarter, S in lanes
    // 16-31 (the second M = 64 tile).
    static constexpr uint32_t COL_H = 0;                  // kNs x D    h            (M = 128)
    static constexpr uint32_t COL_FK = kNs * D;           // kNs x 32   Fk^T ring    (M = 128)
    static constexpr uint32_t COL_T = COL_FK + kNs * 32;  // NT         [T | Tn]     (M = 64, lanes 0-15)
    static constexpr uint32_t COL_S = COL_T;              // 64         S            (M = 64, lanes 16-31)
    static_assert(COL_T + NT <= 512 && COL_S + 64 <= 512, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(OFF_HB % 1024 == 0 && OFF_ZB % 1024 == 0 && OFF_FQ % 1024 == 0 && OFF_P % 1024 == 0,
                  "swizzle atoms");
};

struct Misc {
    float acs2[2][kC];   // chunk-local cumsum per chunk parity (decay warp -> query team)
    float vfac[kC];      // value factors dt_j of the decay warp's current chunk
    float rsum[kC];      // row sums of P (chunks whose quadratic part this CTA adds)
    float Dh[64];        // D of the head
    float lam2[2];       // chunk total per chunk parity (state team reads it)
    uint64_t stage_full[kMaxStages], stage_empty[kMaxStages];
    uint64_t decay_ready[2], decay_free[2];
    uint64_t st_ready[kNs], slab_done[kNs], q_ready[kNQ];
    uint64_t t_full, t_free, s_full, p_full;
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
__device__ __forceinline__ uint32_t bf16_bits_at(const uint8_t *p) {
    return (uint32_t)*reinterpret_cast<const uint16_t *>(p);
}
__device__ __forceinline__ float bf16_at(const uint8_t *p) { return __uint_as_float(bf16_bits_at(p) << 16); }
template <uint32_t RB>
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t ch) {
    if constexpr (RB == 128) return sw128_chunk(row, ch);
    else return sw64_chunk(row, ch);
}
// byte offset of element `col` of `row` in a swizzled bf16 tile
template <uint32_t RB>
__device__ __forceinline__ uint32_t swz_elem(uint32_t row, uint32_t col) {
    return swz<RB>(row, col >> 3) + (col & 7u) * 2u;
}

// Waits until the counter reaches `target`; gives up (false) on a raised
// abort flag (this CTA's or the head's) or after limit_ns of wall time.
__device__ bool counter_wait(const uint32_t *cnt, uint32_t target, const volatile int *abort,
                             const uint32_t *head_abort, unsigned long long limit_ns) {
    if (ld_acquire_gpu(cnt) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (ld_acquire_gpu(cnt) >= target) return true;
        if ((it & 63u) == 63u) {
            if (*abort || ld_acquire_gpu(head_abort)) return false;
            if (globaltimer_ns() - t0 > limit_ns) return false;
        }
        __nanosleep(32);
    }
}

// Records a timeout (the first one wins) and raises the abort flags: this
// CTA's, and every other CTA's of the head (the cluster's through
// distributed shared memory, or the head's flag in global memory).
template <bool kGlobal, int R>
__device__ void raise_timeout(Misc *misc, DeviceStatus *status, int where, uint32_t *head_abort) {
    if (status) {
        atomicCAS(&status->code, 0, (int)SSD_ERR_TIMEOUT);
        atomicCAS(&status->detail, 0, where);
    }
    if constexpr (kGlobal) {
        *reinterpret_cast<volatile int *>(&misc->abort_flag) = 1;
        atomicExch(head_abort, 1u);
    } else {
        const uint32_t a = smem_u32(&misc->abort_flag);
        for (int r = 0; r < R; ++r) st_dsmem_u32(mapa_shared(a, (uint32_t)r), 1u);
        fence_acq_rel_cluster();
    }
}

// kState: the call carries a state in or out (a separate instantiation, so
// that calls without one run none of its code).
template <int D, bool kState>
__global__ void __launch_bounds__(kThreads, 1)
tc_order2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16 *__restrict__ vglob,
                 __nv_bfloat16 *__restrict__ out, const float *__restrict__ dt_p,
                 const float *__restrict__ A_log, const float *__restrict__ dt_bias,
                 const float *__restrict__ Dres, const float *__restrict__ log_decay, int value_dt,
                 int H, int N, int normalize, const float *__restrict__ h0, const float *__restrict__ z0,
                 float *__restrict__ h_out, float *__restrict__ z_out, DeviceStatus *status,
                 uint32_t *__restrict__ counters, float *__restrict__ gpart, int dbg_skip,
                 unsigned long long wait_ns) {
    using K = Cfg<D>;
    constexpr int R = K::R;
    constexpr uint32_t RB = K::RB;
    constexpr bool GL = K::GLOBAL;
    constexpr int kStages = K::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Misc *misc = reinterpret_cast<Misc *>(smem + K::OFF_MISC);
    const volatile int *abort_flag = &misc->abort_flag;
    const uint32_t sbase = smem_u32(smem);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = GL ? (uint32_t)(blockIdx.x % R) : cluster_ctarank();
    const int bh = blockIdx.x / R, h = bh % H;
    const int nc = N / kC;
    const int row0 = bh * N;
    // a carried state enters before chunk 0 exactly as the state of a previous chunk does
    const bool carry = kState && (h0 != nullptr || z0 != nullptr);
    // per head: ready[kNP], consumed[kNP] (per slot of the partial ring), abort
    uint32_t *hcnt = GL ? counters + bh * (kCounterStride / 4) : nullptr;
    uint32_t *head_abort = GL ? hcnt + 2 * kNP : nullptr;
    auto timeout = [&](int where) { raise_timeout<GL, R>(misc, status, where, head_abort); };

    if (tid == 0) {
        if (blockIdx.x == 0 && status) {
            status->code = 0;
            status->detail = 0;
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&misc->stage_full[i], 1);
            mbar_init(&misc->stage_empty[i], 1 + kSTT + kQ1T + 32);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&misc->decay_ready[b], 32);
            mbar_init(&misc->decay_free[b], kSTT + kQ1T);
            mbar_init(&misc->ready[b], R);
            mbar_init(&misc->consumed[b], R);
        }
        for (int s = 0; s < kNs; ++s) {
            mbar_init(&misc->st_ready[s], kSTT / 2);
            mbar_init(&misc->slab_done[s], 1);
        }
        for (int e = 0; e < kNQ; ++e) mbar_init(&misc->q_ready[e], kQ1T);
        mbar_init(&misc->t_full, 1);
        mbar_init(&misc->t_free, kQ2T);
        mbar_init(&misc->s_full, 1);
        mbar_init(&misc->p_full, kQ1T);
        mbar_init(&misc->drain, 1);
        misc->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc->tmem_base, 512);
        tmem_relinquish();
    }
    if (tid < D) misc->Dh[tid] = Dres ? Dres[h * D + tid] : 0.0f;
    tc_fence_before();
    if constexpr (GL) __syncthreads();
    else cluster_sync_all();  // every CTA's barriers exist before any remote access
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ decay warp and TMA
        // kernel (a): chunk-local inclusive cumsum of the log-decay (log2 units),
        // the chunk total, the key weights wk[a][j / 2] = bf16 pair of
        // 2^(lam - acs_j) k_ja, and V <- diag(dt) V under value discretisation.
        // The same warp requests the chunks' Q, K, V tiles: a chunk's tiles
        // before its decay step needs them (waiting for their stage if it must),
        // and the next chunks' whenever their stage is already free.
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
        }
        int issued = 0;  // chunks whose tiles have been requested
        // requests tiles for chunks issued .. upto; waits for a busy stage only
        // when `block` (false: stops at the first busy one)
        auto request = [&](int upto, bool block) -> bool {
            while (issued <= upto && issued < nc) {
                const int st = issued % kStages;
                if (issued >= kStages) {
                    const uint32_t par = ((issued / kStages) - 1) & 1;
                    if (block) {
                        const bool good = mbar_wait_abortable(&misc->stage_empty[st], par, abort_flag, wait_ns);
                        if (!__all_sync(0xffffffffu, good)) return false;
                    } else if (!__shfl_sync(0xffffffffu, (int)mbar_test(&misc->stage_empty[st], par), 0)) {
                        return true;
                    }
                }
                if (lane == 0) {
                    uint8_t *dst = smem + K::OFF_STAGE + st * K::STAGE;
                    const int r = row0 + issued * kC;
                    mbar_arrive_expect_tx(&misc->stage_full[st], K::STAGE);
                    tma_load_2d(dst, &tm_q, 0, r, &misc->stage_full[st]);
                    tma_load_2d(dst + K::TILE, &tm_k, 0, r, &misc->stage_full[st]);
                    tma_load_2d(dst + 2 * K::TILE, &tm_v, 0, r, &misc->stage_full[st]);
                }
                __syncwarp();
                ++issued;
            }
            return true;
        };
        const float A2 = log_decay ? 0.0f : -expf(A_log[h]) * kLog2e;
        const float bias = dt_bias ? dt_bias[h] : 0.0f;  // given whenever dt is used
        const float *dsrc = log_decay ? log_decay : dt_p;
        const bool vdt_own = value_dt && log_decay;  // the dt projection, when it is not dsrc
        float2 dnext = make_float2(0.f, 0.f), vnext = make_float2(0.f, 0.f);
        if (nc > 0) {
            dnext = *reinterpret_cast<const float2 *>(dsrc + (size_t)row0 + 2 * lane);
            if (vdt_own) vnext = *reinterpret_cast<const float2 *>(dt_p + (size_t)row0 + 2 * lane);
        }
        bool ok = request(kStages - 1, true);
        for (int c = 0; ok && c < nc; ++c) {
            const int st = c % kStages;
            if (!(ok = request(c, true))) break;
            const float2 dv = dnext, vv = vdt_own ? vnext : dnext;
            if (c + 1 < nc) {
                dnext = *reinterpret_cast<const float2 *>(dsrc + (size_t)row0 + (size_t)(c + 1) * kC + 2 * lane);
                if (vdt_own) vnext = *reinterpret_cast<const float2 *>(dt_p + (size_t)row0 + (size_t)(c + 1) * kC + 2 * lane);
            }
            // tokens 2 lane and 2 lane + 1
            const float a0 = log_decay ? dv.x * kLog2e : A2 * softplus_f(dv.x + bias);
            const float a1 = log_decay ? dv.y * kLog2e : A2 * softplus_f(dv.y + bias);
            float incl = a0 + a1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const float lam = __shfl_sync(0xffffffffu, incl, 31);
            if (c >= 2) {
                ok = mbar_wait_abortable(&misc->decay_free[c & 1], ((c >> 1) - 1) & 1, abort_flag, wait_ns);
                if (!__all_sync(0xffffffffu, ok)) break;
            }
            misc->acs2[c & 1][2 * lane] = incl - a1;
            misc->acs2[c & 1][2 * lane + 1] = incl;
            if (value_dt) {
                misc->vfac[2 * lane] = softplus_f(vv.x + bias);
                misc->vfac[2 * lane + 1] = softplus_f(vv.y + bias);
            }
            if (lane == 0) misc->lam2[c & 1] = lam;
            ok = mbar_wait_abortable(&misc->stage_full[st], (c / kStages) & 1, abort_flag, wait_ns);
            if (!__all_sync(0xffffffffu, ok)) break;
            __syncwarp();
            uint8_t *sK = smem + K::OFF_STAGE + st * K::STAGE + K::TILE;
            uint8_t *sV = sK + K::TILE;
            const float *acs = misc->acs2[c & 1];
            uint32_t *wk = reinterpret_cast<uint32_t *>(smem + K::OFF_WK) + (c & 1) * K::NA * 32;
            // K^T pairs and key weights: lane l holds token pair (2l, 2l + 1); for
            // every column b, kT[b][l] = bf16 pair (k_2l,b, k_2l+1,b), and for the
            // CTA's a, wk[a][l] = bf16 pair (2^(lam - acs_2l) k_2l,a, same for 2l + 1)
            {
                const int j = 2 * lane;
                const float w0 = ex2_approx(lam - acs[j]), w1 = ex2_approx(lam - acs[j + 1]);
                uint32_t *kT = reinterpret_cast<uint32_t *>(smem + K::OFF_KT) + (c & 1) * D * 32;
#pragma unroll 2
                for (int ch = 0; ch < D / 8; ++ch) {
                    const uint4 r0 = *reinterpret_cast<const uint4 *>(sK + swz<RB>(j, ch));
                    const uint4 r1 = *reinterpret_cast<const uint4 *>(sK + swz<RB>(j + 1, ch));
                    const uint32_t a0[4] = {r0.x, r0.y, r0.z, r0.w}, a1[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int b = 8 * ch + e;
                        const uint32_t lo = (e & 1) ? (a0[e >> 1] >> 16) : (a0[e >> 1] & 0xFFFFu);
                        const uint32_t hi = (e & 1) ? (a1[e >> 1] & 0xFFFF0000u) : (a1[e >> 1] << 16);
                        kT[b * 32 + ((((lane >> 2) ^ b) & 7) << 2) + (lane & 3)] = lo | hi;
                        const int al = b - (int)rank * K::NA;
                        if (al >= 0 && al < K::NA)
                            wk[al * 32 + lane] = pack_bf16x2(w0 * __uint_as_float(lo << 16), w1 * __uint_as_float(hi));
                    }
                }
            }
            if (value_dt) {
                // value discretisation: V <- diag(dt) V in place, before any product reads it
                constexpr int CPR = D / 8;  // 16-byte chunks per row
                for (int t = lane; t < kC * CPR; t += 32) {
                    const int r = t / CPR, ch = t % CPR;
                    uint4 *pv = reinterpret_cast<uint4 *>(sV + swz<RB>(r, ch));
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
                fence_proxy_async_smem();
            }
            mbar_arrive(&misc->decay_ready[c & 1]);
            mbar_arrive(&misc->stage_empty[st]);
            request(c + kStages, false);
        }
        if (!ok) timeout(50);
        // copies still in flight after an abort land before the CTA exits (bounded)
        for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
            mbar_wait_bounded(&misc->stage_full[c % kStages], (c / kStages) & 1);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idBuild = make_idesc_bf16(128, D, 0, 1);
            constexpr uint32_t idRead = make_idesc_bf16(64, K::NT, 0, 1);
            constexpr uint32_t idS = make_idesc_bf16(64, 64, 0, 0);
            constexpr uint32_t idPV = make_idesc_bf16(64, D, 0, 1);
            constexpr uint64_t kStepRows = (16 * RB) >> 4;  // descriptor units per 16 rows
            const uint64_t dP = make_sdesc(sbase + K::OFF_P, 16, 1024, kSw128);
            const uint64_t dFq = make_sdesc(sbase + K::OFF_FQ, 16, 1024, kSw128);
            const uint32_t tT = tmem + K::COL_T, tS = tmem + kHalf1 + K::COL_S;
            bool ok = true;
            int kown = 0;
            auto wait = [&](uint64_t *bar, uint32_t parity) {
                ok = ok && mbar_wait_abortable(bar, parity, abort_flag, wait_ns);
                return ok;
            };
            for (int c = 0; ok && c < nc; ++c) {
                const int st = c % kStages, c3 = c % kNQ;
                const bool has_read = c >= 1 || carry;
                const bool owner = (c % R) == (int)rank;
                const uint32_t acc = (c >= 1 || carry) ? 1u : 0u;
                if (!wait(&misc->stage_full[st], (c / kStages) & 1)) break;
                const uint32_t soff = K::OFF_STAGE + st * K::STAGE;
                const uint64_t dQ = make_sdesc(sbase + soff, 16, K::SBO, K::SW);
                const uint64_t dK = make_sdesc(sbase + soff + K::TILE, 16, K::SBO, K::SW);
                const uint64_t dV = make_sdesc(sbase + soff + 2 * K::TILE, 16, K::SBO, K::SW);
                if (owner) {  // S = Q K^T into the second M = 64 tile of the readout's columns
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks)
                        mma_bf16(tS, dQ + ks * 2, dK + ks * 2, idS, ks > 0 ? 1u : 0u);
                    mma_commit(&misc->s_full);
                }
                // state builds of the four slabs (they do not touch the readout's columns)
#pragma unroll
                for (int s = 0; s < kNs; ++s) {
                    if (!wait(&misc->st_ready[s], c & 1)) break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < kC / 16; ++ks)
                        mma_bf16_ts(tmem + K::COL_H + s * D, tmem + K::COL_FK + s * 32 + ks * 8, dV + ks * kStepRows,
                                    idBuild, (acc | (ks > 0 ? 1u : 0u)));
                }
                if (!ok) break;
                if (c >= 1 && !wait(&misc->t_free, (c - 1) & 1)) break;  // previous partial read
                // readouts, slab by slab; each slab's buffers are released by slab_done
#pragma unroll
                for (int s = 0; s < kNs; ++s) {
                    const int it = 4 * c + s, e = (c3 + s) % kNQ;
                    if (!wait(&misc->q_ready[e], (it / kNQ) & 1)) break;
                    tc_fence_after();
                    if (has_read) {
                        const uint64_t dA = dFq + (((uint32_t)e * 16384u) >> 4);
                        const uint64_t dB = make_sdesc(sbase + K::OFF_HB + s * K::HBT,
                                                       (K::OFF_ZB + 16u * s) - (K::OFF_HB + s * K::HBT), K::SBO, K::SW);
#pragma unroll
                        for (int ks = 0; ks < kSlab / 16; ++ks)
                            mma_bf16(tT, dA + (((ks >> 2) * 8192u + (ks & 3) * 32u) >> 4), dB + ks * kStepRows, idRead,
                                     (s > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(&misc->slab_done[s]);
                    if (s == 1 && owner) {
                        if (!wait(&misc->p_full, kown & 1)) break;
                        tc_fence_after();
#pragma unroll
                        for (int ks = 0; ks < kC / 16; ++ks)
                            mma_bf16(tT, dP + ks * 2, dV + ks * kStepRows, idPV, (has_read || ks > 0) ? 1u : 0u);
                        ++kown;
                    }
                }
                if (!ok) break;
                mma_commit(&misc->t_full);
                mma_commit(&misc->stage_empty[st]);
            }
            if (!ok) {
                timeout(20);
                // products still in flight finish before TMEM is released (bounded)
                mma_commit(&misc->drain);
                mbar_wait_bounded(&misc->drain, 0);
            }
        }
    } else if (warp < kQ1W0) {
        // ------------------------------------------------------------ state team
        const int q = warp & 3;                      // TMEM lane quarter
        const int hh = (warp - 2) >> 2;              // slabs hh and hh + 2
        const int L = q * 32 + lane;                 // lane of every slab
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const int bcol = L % D;                      // b of this lane's features
        const int lg = L / D;                        // a = rank NA + 4 lg + s
        bool ok = true;
        auto wait = [&](uint64_t *bar, uint32_t parity) {
            ok = ok && mbar_wait_abortable(bar, parity, abort_flag, wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            return ok;
        };
        auto feature = [&](int s) -> size_t {  // global feature row of slab s
            return (size_t)bh * D * D + (size_t)(rank * K::NA + 4 * lg + s) * D + bcol;
        };
        // z of this lane's features (slabs hh, hh + 2): the state entering the next chunk
        float zr[2];
#pragma unroll
        for (int si = 0; si < 2; ++si) zr[si] = (kState && z0) ? z0[feature(hh + 2 * si)] : 0.0f;
        for (int c = 0; c < nc; ++c) {
            const int st = c % kStages;
            if (!wait(&misc->stage_full[st], (c / kStages) & 1)) break;
            mbar_arrive(&misc->stage_empty[st]);
            if (!wait(&misc->decay_ready[c & 1], (c >> 1) & 1)) break;
            const float dec = ex2_approx(misc->lam2[c & 1]);
            const uint32_t *wk = reinterpret_cast<const uint32_t *>(smem + K::OFF_WK) + (c & 1) * K::NA * 32;
            const uint8_t *kTrow = smem + K::OFF_KT + (c & 1) * D * 128 + bcol * 128;  // k_jb pairs of column b
#pragma unroll
            for (int si = 0; si < 2; ++si) {
                const int s = hh + 2 * si;
                if (c >= 1 && !wait(&misc->slab_done[s], (c - 1) & 1)) break;
                tc_fence_after();
                // ---- the state entering the chunk -> hb, zb (bf16); the state *= 2^lam
                if (c >= 1 || carry) {
                    uint8_t *hb = smem + K::OFF_HB + s * K::HBT;
#pragma unroll
                    for (int half = 0; half < D / 32; ++half) {
                        float hv[32];
                        const uint32_t ta = tmem + lane_off + K::COL_H + s * D + 32 * half;
                        if (c >= 1) {
                            tmem_ld32(ta, hv);
                            tmem_wait_ld();
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; j += 4) {
                                const float4 x = h0 ? *reinterpret_cast<const float4 *>(h0 + feature(s) * D + 32 * half + j)
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                                hv[j] = x.x;
                                hv[j + 1] = x.y;
                                hv[j + 2] = x.z;
                                hv[j + 3] = x.w;
                            }
                        }
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch)
                            *reinterpret_cast<uint4 *>(hb + swz<RB>(L, 4 * half + ch)) =
                                make_uint4(pack_bf16x2(hv[ch * 8], hv[ch * 8 + 1]), pack_bf16x2(hv[ch * 8 + 2], hv[ch * 8 + 3]),
                                           pack_bf16x2(hv[ch * 8 + 4], hv[ch * 8 + 5]),
                                           pack_bf16x2(hv[ch * 8 + 6], hv[ch * 8 + 7]));
                        const float2 d2 = make_float2(dec, dec);
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 r2 = __fmul2_rn(make_float2(hv[e], hv[e + 1]), d2);
                            hv[e] = r2.x;
                            hv[e + 1] = r2.y;
                        }
                        tmem_st32(ta, hv);
                    }
                    *reinterpret_cast<uint4 *>(smem + K::OFF_ZB + swz<RB>(L, s)) =
                        make_uint4(pack_bf16x2(zr[si], 0.0f), 0u, 0u, 0u);
                }
                // ---- Fk^T row of feature (a, b) over the 64 tokens, and z
                {
                    const uint4 *wr = reinterpret_cast<const uint4 *>(wk + (4 * lg + s) * 32);
                    float2 zs = make_float2(0.f, 0.f);
                    // eight steps of four token pairs: two 16-byte loads, four
                    // products, one 4-column store (few registers live at a time)
#pragma unroll 2
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const uint4 w = wr[q4];
                        const uint4 kq = *reinterpret_cast<const uint4 *>(kTrow + (((q4 ^ bcol) & 7) << 4));
                        const uint32_t f0 = mul_bf16x2(w.x, kq.x), f1 = mul_bf16x2(w.y, kq.y);
                        const uint32_t f2 = mul_bf16x2(w.z, kq.z), f3 = mul_bf16x2(w.w, kq.w);
                        zs = __fadd2_rn(zs, __fadd2_rn(__fadd2_rn(bf2_to_f2(f0), bf2_to_f2(f1)),
                                                       __fadd2_rn(bf2_to_f2(f2), bf2_to_f2(f3))));
                        tmem_st4(tmem + lane_off + K::COL_FK + s * 32 + 4 * q4, f0, f1, f2, f3);
                    }
                    zr[si] = fmaf(zr[si], dec, zs.x + zs.y);
                }
                tmem_wait_st();
                tc_fence_before();
                fence_proxy_async_smem();
                if (4 * c + s != dbg_skip) mbar_arrive(&misc->st_ready[s]);
            }
            if (!ok) break;
            mbar_arrive(&misc->decay_free[c & 1]);
        }
        // the state after the last token: TMEM holds h once the last products are done
        if (kState && ok && (h_out || z_out)) {
#pragma unroll
            for (int si = 0; si < 2; ++si) {
                const int s = hh + 2 * si;
                if (!wait(&misc->slab_done[s], (nc - 1) & 1)) break;
                tc_fence_after();
                if (h_out) {
#pragma unroll
                    for (int half = 0; half < D / 32; ++half) {
                        float hv[32];
                        tmem_ld32(tmem + lane_off + K::COL_H + s * D + 32 * half, hv);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4 *>(h_out + feature(s) * D + 32 * half + j) =
                                make_float4(hv[j], hv[j + 1], hv[j + 2], hv[j + 3]);
                    }
                }
                if (z_out) z_out[feature(s)] = zr[si];
            }
        }
    } else if (warp < kQ2W0) {
        // ------------------------------------------------------------ query team
        const int q1 = tid - kQ1W0 * 32;             // 0..127
        const int qq = warp & 3;                     // TMEM lane quarter
        const uint32_t lane_off = (uint32_t)(qq * 32) << 16;
        // Fq: thread q1 writes row tk of the 64-feature atom `at` of every slab
        const int tk = q1 & 63, at = q1 >> 6;
        bool ok = true;
        int kown = 0;
        auto wait = [&](uint64_t *bar, uint32_t parity) {
            ok = ok && mbar_wait_abortable(bar, parity, abort_flag, wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            return ok;
        };
        for (int c = 0; c < nc; ++c) {
            const int st = c % kStages, c3 = c % kNQ;
            const bool owner = (c % R) == (int)rank;
            if (!wait(&misc->stage_full[st], (c / kStages) & 1)) break;
            if (!wait(&misc->decay_ready[c & 1], (c >> 1) & 1)) break;
            const uint8_t *sQ = smem + K::OFF_STAGE + st * K::STAGE;
            const float *acs = misc->acs2[c & 1];
            // this thread's query row (bf16 pairs) and 2^acs of its token
            uint32_t qr[D / 2];
#pragma unroll
            for (int ch = 0; ch < D / 8; ++ch) {
                const uint4 x = *reinterpret_cast<const uint4 *>(sQ + swz<RB>(tk, ch));
                qr[4 * ch] = x.x;
                qr[4 * ch + 1] = x.y;
                qr[4 * ch + 2] = x.z;
                qr[4 * ch + 3] = x.w;
            }
            const float ut = ex2_approx(acs[tk]);
            for (int s = 0; s < kNs; ++s) {
                if (s == 2 && owner) {
                    // ---- quadratic part of the chunk: P = S^2 2^(acs_i - acs_j) [i >= j]
                    if (!wait(&misc->s_full, kown & 1)) break;
                    tc_fence_after();
                    float sv0[32], sv1[32];
                    tmem_ld32(tmem + lane_off + K::COL_S, sv0);
                    tmem_ld32(tmem + lane_off + K::COL_S + 32, sv1);
                    tmem_wait_ld();
                    tc_fence_before();
                    if (lane >= 16) {  // rows of the second M = 64 tile
                        const int i = 16 * qq + lane - 16;
                        const float ai = acs[i];
                        float rs = 0.0f;
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 8; e += 2) {
                                const int j = ch * 8 + e;
                                const float x0 = j < 32 ? sv0[j & 31] : sv1[j & 31];
                                const float x1 = j + 1 < 32 ? sv0[(j + 1) & 31] : sv1[(j + 1) & 31];
                                float p0 = x0 * x0 * ex2_approx(ai - acs[j]);
                                float p1 = x1 * x1 * ex2_approx(ai - acs[j + 1]);
                                if (j > i) p0 = 0.0f;
                                if (j + 1 > i) p1 = 0.0f;
                                rs += p0 + p1;
                                pk[e >> 1] = pack_bf16x2(p0, p1);
                            }
                            *reinterpret_cast<uint4 *>(smem + K::OFF_P + sw128_chunk(i, ch)) =
                                make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                        misc->rsum[i] = rs;
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(&misc->p_full);
                    ++kown;
                }
                const int it = 4 * c + s, e = (c3 + s) % kNQ;
                // the Fq buffer's previous user (iteration it - kNQ) has been read
                if (it >= kNQ && !wait(&misc->slab_done[(it - kNQ) & 3], ((it - kNQ) >> 2) & 1)) break;
                // ---- Fq slab s (K-major, 64 x 128): feature k of the slab is
                // (a = rank NA + 4 (k / D) + s, b = k % D); this thread writes row tk
                // of atom at, i.e. k = 64 at + kk for kk in [0, 64)
                constexpr int NAA = 64 / D;  // values of a in one 64-feature atom
                uint32_t ca[NAA];
#pragma unroll
                for (int ag = 0; ag < NAA; ++ag) {
                    const int av = rank * K::NA + 4 * (NAA * at + ag) + s;
                    const float cv = ut * bf16_at(sQ + swz_elem<RB>(tk, av));
                    ca[ag] = pack_bf16x2(cv, cv);
                }
                uint8_t *fq = smem + K::OFF_FQ + e * 16384 + at * 8192;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const int kk = 8 * ch;
                    const uint32_t cp = ca[kk / D];
                    const int qp = (kk % D) / 2;  // first bf16 pair of q_ib
                    *reinterpret_cast<uint4 *>(fq + sw128_chunk(tk, ch)) =
                        make_uint4(mul_bf16x2(cp, qr[qp]), mul_bf16x2(cp, qr[qp + 1]), mul_bf16x2(cp, qr[qp + 2]),
                                   mul_bf16x2(cp, qr[qp + 3]));
                }
                fence_proxy_async_smem();
                mbar_arrive(&misc->q_ready[e]);
            }
            if (!ok) break;
            mbar_arrive(&misc->decay_free[c & 1]);
            mbar_arrive(&misc->stage_empty[st]);
        }
        if (!ok) timeout(30);
    } else {
        // ------------------------------------------------------------ output team
        const int q2 = tid - kQ2W0 * 32;             // 0..127
        const int qq = warp & 3;
        const uint32_t lane_off = (uint32_t)(qq * 32) << 16;
        const bool row_t = lane < 16;                // holds a row of the M = 64 readout
        const int row = 16 * qq + lane;
        float *res = reinterpret_cast<float *>(smem + K::OFF_RES);
        bool failed = false;
        int kown = 0;
        auto team_ok = [&](bool good) { return !named_bar_any(kBarQ2, kQ2T, !good); };
        static_assert(K::ROWS * (D / 8) <= kQ2T, "one output item per thread");
        constexpr int NV = D / 4 + 1;  // float4 groups of a row, plus the normaliser
        // residual input of this thread's output item of chunk cc (fetched
        // ahead of the waits that precede its use)
        auto load_residual = [&](int cc) -> uint4 {
            uint4 vu = make_uint4(0u, 0u, 0u, 0u);
            if (Dres && cc >= 0 && cc < nc && q2 < K::ROWS * (D / 8)) {
                const size_t o_grow = (size_t)row0 + (size_t)cc * kC + rank * K::ROWS + q2 / (D / 8);
                vu = __ldg(reinterpret_cast<const uint4 *>(vglob + o_grow * D + (q2 % (D / 8)) * 8));
            }
            return vu;
        };
        // y of chunk cc from the summed rows in res: y = T / Tn [+ D v]
        auto write_output = [&](int cc, uint4 vu) {
            const int o_rr = q2 / (D / 8), o_ch = q2 % (D / 8);
            if (q2 < K::ROWS * (D / 8)) {
                const size_t o_grow = (size_t)row0 + (size_t)cc * kC + rank * K::ROWS + o_rr;
                const float *rrow = res + o_rr * K::PR;
                const float inv = normalize ? 1.0f / rrow[D] : 1.0f;
                const uint32_t vw[4] = {vu.x, vu.y, vu.z, vu.w};
                uint32_t w[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c2 = o_ch * 8 + 2 * e;
                    float y0 = rrow[c2] * inv, y1 = rrow[c2 + 1] * inv;
                    if (Dres) {
                        const float2 vf = bf2_to_f2(vw[e]);
                        y0 = fmaf(misc->Dh[c2], vf.x, y0);
                        y1 = fmaf(misc->Dh[c2 + 1], vf.y, y1);
                    }
                    w[e] = pack_bf16x2(y0, y1);
                }
                *reinterpret_cast<uint4 *>(out + o_grow * D + o_ch * 8) = make_uint4(w[0], w[1], w[2], w[3]);
            }
        };
        // ---- this CTA's partial [T | Tn] of chunk c, read from TMEM into
        // `dst_row` (this thread's row); releases the readout's columns
        auto drain = [&](int c, float *dst_row, bool owner) {
            const bool has_read = c >= 1 || carry;
            const float rs = (owner && row_t) ? misc->rsum[row] : 0.0f;
#pragma unroll
            for (int part = 0; part < D / 16; ++part) {
                float tv[16];
                tmem_ld16(tmem + lane_off + K::COL_T + 16 * part, tv);
                tmem_wait_ld();
                if (row_t)
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4 *>(dst_row + 16 * part + e) =
                            (has_read || owner) ? make_float4(tv[e], tv[e + 1], tv[e + 2], tv[e + 3])
                                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            const float tn = tmem_ld1(tmem + lane_off + K::COL_T + D);
            tmem_wait_ld();
            if (row_t) dst_row[D] = (has_read ? tn : 0.0f) + rs;
            tc_fence_before();
            mbar_arrive(&misc->t_free);
        };
        if constexpr (GL) {
            // reduction through L2: partials[bh][c % kNP][rank][row][PR].  Per
            // slot of the ring, ready counts the CTAs' published partials and
            // consumed their finished reductions; each use of a slot adds
            // exactly R to both, because a slot is rewritten only after all R
            // CTAs have reduced its previous chunk (CTAs may run ahead of one
            // another by up to kNP chunks).  Software pipeline: iteration c
            // drains chunk c, publishes chunk c - 1 (its stores were issued an
            // iteration earlier) and reduces chunk c - 2 (its loads are issued
            // before the drain, so their latency overlaps it).
            static_assert(K::ROWS * (D / 4) == kQ2T && K::ROWS * R <= kQ2T, "one float4 group per thread");
            uint32_t *ready_cnt = hcnt, *consumed_cnt = hcnt + kNP;
            float *hpart = gpart + (size_t)bh * kNP * R * kC * K::PR;
            const int g_rr = q2 / (D / 4), g_v = q2 % (D / 4);   // this thread's float4 group of T
            const int n_rr = q2 / R, n_r2 = q2 % R;               // this thread's Tn term (q2 < ROWS R)
            for (int c = 0; c <= nc + 1; ++c) {
                const int cr = c - 2;
                float4 x[R];
                float xn = 0.0f;
                uint4 vu = make_uint4(0u, 0u, 0u, 0u);
                if (cr >= 0) {
                    bool good = true;
                    if (q2 == 0)
                        good = counter_wait(ready_cnt + cr % kNP, (uint32_t)(R * (cr / kNP + 1)), abort_flag, head_abort,
                                            wait_ns);
                    if (!team_ok(good)) {
                        failed = true;
                        break;
                    }
                    const float *cpart = hpart + (size_t)(cr % kNP) * R * kC * K::PR;
                    const size_t goff = (size_t)(rank * K::ROWS + g_rr) * K::PR + 4 * g_v;
#pragma unroll
                    for (int r2 = 0; r2 < R; ++r2)
                        x[r2] = __ldcg(reinterpret_cast<const float4 *>(cpart + (size_t)r2 * kC * K::PR + goff));
                    if (q2 < K::ROWS * R)
                        xn = __ldcg(cpart + ((size_t)n_r2 * kC + rank * K::ROWS + n_rr) * K::PR + D);
                    vu = load_residual(cr);
                }
                if (c < nc) {
                    const bool owner = (c % R) == (int)rank;
                    bool good = mbar_wait_abortable(&misc->t_full, c & 1, abort_flag, wait_ns);
                    if (owner) good = good && mbar_wait_abortable(&misc->p_full, kown & 1, abort_flag, wait_ns);
                    // every CTA has reduced the slot's previous chunk, c - kNP
                    if (c >= kNP && q2 == 0)
                        good = good && counter_wait(consumed_cnt + c % kNP, (uint32_t)(R * (c / kNP)), abort_flag,
                                                    head_abort, wait_ns);
                    if (!team_ok(good)) {
                        failed = true;
                        break;
                    }
                    tc_fence_after();
                    drain(c, hpart + (((size_t)(c % kNP) * R + rank) * kC + row) * K::PR, owner);
                    if (owner) ++kown;
                }
                // every thread's stores of chunk c - 1 precede this barrier (they
                // preceded the previous one); one release publishes them
                named_bar_sync(kBarQ2, kQ2T);
                if (q2 == 0 && c >= 1 && c <= nc) red_release_gpu_add(ready_cnt + (c - 1) % kNP, 1u);
                if (cr >= 0) {
                    float4 acc4 = x[0];
#pragma unroll
                    for (int r2 = 1; r2 < R; ++r2) {
                        acc4.x += x[r2].x;
                        acc4.y += x[r2].y;
                        acc4.z += x[r2].z;
                        acc4.w += x[r2].w;
                    }
                    *reinterpret_cast<float4 *>(res + g_rr * K::PR + 4 * g_v) = acc4;
                    // Tn of row n_rr: the R terms sit on R consecutive lanes
#pragma unroll
                    for (int o = 1; o < R; o <<= 1) xn += __shfl_xor_sync(0xffffffffu, xn, o);
                    if (q2 < K::ROWS * R && n_r2 == 0) res[n_rr * K::PR + D] = xn;
                    named_bar_sync(kBarQ2, kQ2T);
                    if (q2 == 0) red_release_gpu_add(consumed_cnt + cr % kNP, 1u);
                    write_output(cr, vu);
                    named_bar_sync(kBarQ2, kQ2T);  // res is reused by the next chunk
                }
            }
        } else {
            // reduction through distributed shared memory within the cluster
            float *part0 = reinterpret_cast<float *>(smem + K::OFF_PART);
            for (int c = 0; c < nc; ++c) {
                const bool owner = (c % R) == (int)rank;
                const uint4 vu = load_residual(c);
                bool good = mbar_wait_abortable(&misc->t_full, c & 1, abort_flag, wait_ns);
                if (owner) good = good && mbar_wait_abortable(&misc->p_full, kown & 1, abort_flag, wait_ns);
                if (c >= 2)
                    good = good && mbar_wait_cluster(&misc->consumed[c & 1], ((c >> 1) - 1) & 1, abort_flag, wait_ns);
                if (!team_ok(good)) {
                    failed = true;
                    break;
                }
                tc_fence_after();
                drain(c, part0 + (c & 1) * kC * K::PR + row * K::PR, owner);
                if (owner) ++kown;
                named_bar_sync(kBarQ2, kQ2T);
                // thread r announces this CTA's partial to cluster CTA r
                if (q2 < R) {
                    fence_acq_rel_cluster();
                    mbar_arrive_cluster(mapa_shared(smem_u32(&misc->ready[c & 1]), (uint32_t)q2));
                }
                good = mbar_wait_cluster(&misc->ready[c & 1], (c >> 1) & 1, abort_flag, wait_ns);
                if (!team_ok(good)) {
                    failed = true;
                    break;
                }
                const uint32_t pb = smem_u32(part0 + (c & 1) * kC * K::PR);
                for (int itm = q2; itm < K::ROWS * NV; itm += kQ2T) {
                    const int rr = itm / NV, v = itm % NV;
                    const uint32_t off = (uint32_t)((rank * K::ROWS + rr) * K::PR + (v < D / 4 ? v * 4 : D)) * 4u;
                    if (v < D / 4) {
                        float4 x[R];
#pragma unroll
                        for (int r2 = 0; r2 < R; ++r2) x[r2] = ld_dsmem_f4(mapa_shared(pb + off, (uint32_t)r2));
                        float4 acc4 = x[0];
#pragma unroll
                        for (int r2 = 1; r2 < R; ++r2) {
                            acc4.x += x[r2].x;
                            acc4.y += x[r2].y;
                            acc4.z += x[r2].z;
                            acc4.w += x[r2].w;
                        }
                        *reinterpret_cast<float4 *>(res + rr * K::PR + v * 4) = acc4;
                    } else {
                        float x[R];
#pragma unroll
                        for (int r2 = 0; r2 < R; ++r2) x[r2] = ld_dsmem_f1(mapa_shared(pb + off, (uint32_t)r2));
                        float accs = x[0];
#pragma unroll
                        for (int r2 = 1; r2 < R; ++r2) accs += x[r2];
                        res[rr * K::PR + D] = accs;
                    }
                }
                named_bar_sync(kBarQ2, kQ2T);
                if (q2 < R) {
                    fence_acq_rel_cluster();
                    mbar_arrive_cluster(mapa_shared(smem_u32(&misc->consumed[c & 1]), (uint32_t)q2));
                }
                write_output(c, vu);
                named_bar_sync(kBarQ2, kQ2T);  // res is reused by the next chunk
            }
        }
        if (failed && q2 == 0) timeout(40);
    }

    __syncwarp();
    tc_fence_before();
    if constexpr (GL) __syncthreads();
    else cluster_sync_all();  // no CTA leaves while another may still read its shared memory
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------- host side
// [rows, d] bf16 tiles of kC rows, swizzled to match the descriptors
bool make_tmap(CUtensorMap *m, const void *base, uint64_t rows, int d) {
    return encode_tmap_2d(m, base, true, (uint64_t)d, rows, (uint32_t)d, kC, d == 64 ? 128 : 64);
}

// Workspace of the reduction through L2 (D = 64): per head, 64 bytes of
// counters [ready[kNP], consumed[kNP], abort], then the partial ring
// [B H][kNP][R][64][PR] fp32.
size_t counters_bytes(int BH) { return align_up((size_t)BH * kCounterStride, 256); }
size_t partials_bytes(int BH) { return (size_t)BH * kNP * Cfg<64>::R * kC * Cfg<64>::PR * sizeof(float); }

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
    const int BH = a.B * a.H;
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    uint32_t *counters = nullptr;
    float *gpart = nullptr;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(BH * K::R);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = K::SMEM;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    if constexpr (K::GLOBAL) {
        // the head's CTAs wait on one another through L2: a cooperative launch
        // guarantees that all of them are resident (or the launch fails)
        counters = reinterpret_cast<uint32_t *>(ws + kStatusBytes);
        gpart = reinterpret_cast<float *>(ws + kStatusBytes + counters_bytes(BH));
        if (cudaMemsetAsync(counters, 0, counters_bytes(BH), a.stream) != cudaSuccess) return SSD_ERR_CUDA;
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    } else {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = K::R;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    DeviceStatus *status = reinterpret_cast<DeviceStatus *>(a.workspace);
    const unsigned long long wait_ns = a.wait_ns ? a.wait_ns : 1000000000ull;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, static_cast<const __nv_bfloat16 *>(a.v),
                                       static_cast<__nv_bfloat16 *>(a.out), a.dt_p, a.A_log, a.dt_bias, a.D,
                                       a.log_decay, a.value_dt, a.H, a.N, a.normalize, a.h0, a.z0, a.h_out,
                                       a.z_out, status, counters, gpart, a.dbg_skip, wait_ns);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace

bool tc_order2_supports(int B, int H, int N, int d, int dtype, int chunk) {
    return dtype == SSD_BF16 && (d == 32 || d == 64) && chunk == kC &&
           (long long)B * H * N < (1ll << 31);
}

size_t tc_order2_workspace(int B, int H, int, int d, int) {
    if (d != 64) return 0;
    const int BH = B * H;
    return counters_bytes(BH) + partials_bytes(BH);
}

int launch_tc_order2(const FwdArgs &a, const Plan &) {
    return a.d == 64 ? launch_d<64>(a) : launch_d<32>(a);
}

}  // namespace ssd
