// Internal declarations shared by the entry points and the kernel files of
// libssd.so.  Nothing here is part of the public ABI (see include/ssd.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ssd.h"

namespace ssd {

// Arguments of one forward call after validation.
// The causal depthwise convolution (+ SiLU) that produces q, k, v from the
// raw activations x (the prologue Q, K, V = SiLU(conv_1d(h W_QKV))): w and
// bias per input as for ssd_conv1d().
struct ConvParams {
    const void *x[3];     // raw q, k, v: [B, H, N, d_h]
    const float *w[3];    // [H*d_h, width]
    const float *bias[3]; // [H*d_h] or NULL
    int width, silu;
};

struct FwdArgs {
    const void *q, *k, *v;
    const float *dt_p, *A_log, *dt_bias, *D;
    const float *log_decay;  // per-token log-decay, or NULL (A * dt)
    int value_dt;            // contract with v * dt
    const float *h0, *z0;    // carried state in, or NULL (zero)
    float *h_out, *z_out;    // carried state out, or NULL
    int B, H, N, d, dtype, order, normalize, chunk;
    void *out;
    void *workspace;
    size_t workspace_bytes;
    cudaStream_t stream;
    // failure-detection test hook (ssd_debug_fwd): the iteration whose
    // publication a producer skips (-1: none), and the bounded waits' limit in
    // nanoseconds (0: the default of one second)
    int dbg_skip = -1;
    unsigned long long wait_ns = 0;
    // with the convolution fused (order-1 tensor-core path): q, k, v above
    // are the workspace buffers that receive the convolved activations, which
    // the chunk-state kernel computes from conv->x and stores for the scan
    const ConvParams *conv = nullptr;
};

// Device status block at the start of every workspace: status code (an
// ssd_status value, 0 = fine) and a detail word (where a wait gave up).
struct DeviceStatus {
    int code;
    int detail;
    int pad[2];
};

constexpr size_t kStatusBytes = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

enum Path { PATH_SIMT = 0, PATH_TC_ORDER1 = 1, PATH_TC_ORDER2 = 2, PATH_TC_ORDER2Q = 3 };

// Workspace plan for one call: which path runs and where its buffers sit.
struct Plan {
    int path;
    int n_launches;
    size_t acs_off, lam_off, state_off, aux_off, vfac_off, total;
};

// Fills `plan` for the arguments and returns SSD_OK, or the status that
// rejects them (SSD_ERR_SHAPE etc. for invalid shapes, SSD_ERR_UNSUPPORTED
// when no kernel exists).  state: SSD_STATE_H / SSD_STATE_Z bits of the
// state arguments in use.
int make_plan(int B, int H, int N, int d, int dtype, int order, int normalize, int chunk,
              int value_dt, int state, Plan *plan);

// Scratch layout of the SIMT path: status block, chunk-local decay, chunk
// totals, per-chunk carried states with the normaliser column.  Fills the
// offsets and the total of `p` (path and launch count included).
void simt_layout(int B, int H, int N, int d, int order, int chunk, Plan *p);

// The SIMT path puts the chunk index in gridDim.y.
constexpr int kMaxSimtChunks = 65535;

// Path launchers (each returns an ssd_status).
int launch_simt(const FwdArgs &a, const Plan &p);
int launch_tc_order2(const FwdArgs &a, const Plan &p);
bool tc_order2_supports(int B, int H, int N, int d, int dtype, int chunk);
size_t tc_order2_workspace(int B, int H, int N, int d, int chunk);
int launch_tc_order2q(const FwdArgs &a, const Plan &p);
bool tc_order2q_supports(int B, int H, int N, int d, int dtype);
void tc_order2q_layout(int B, int H, int N, Plan *p);
int launch_tc_order1(const FwdArgs &a, const Plan &p);
bool tc_order1_fuses_conv(int chunk);
bool tc_order1_supports(int B, int H, int N, int d, int dtype, int chunk);
void tc_order1_layout(int B, int H, int N, int chunk, Plan *p);

// 2-D TMA tensor map of a row-major [rows, cols] bf16 (or fp32) tensor read or
// written in boxes of box_rows x box_cols, with the 0, 32, 64 or 128-byte
// swizzle (ssd_tmap.cu).  False when the driver rejects it.
bool encode_tmap_2d(CUtensorMap *m, const void *base, bool bf16, uint64_t cols, uint64_t rows,
                    uint32_t box_cols, uint32_t box_rows, int swizzle_bytes);

// The ID of the calling thread's current CUDA context (the driver never
// reuses one within a process); when no context is current, the current
// device's primary context is made current first.  False on a driver error.
bool current_context_id(unsigned long long *id);

// Decode step (ssd_decode.cu).
size_t decode_workspace(int B, int H, int d, int order);
int launch_decode(const FwdArgs &a, float *h, float *z);

// Kernel (a): chunk-local inclusive cumsum of A*dt and the chunk totals.
// When `status` is non-NULL, block (0,0) thread 0 clears it.
// log_decay (may be NULL) replaces A*dt by a given per-token log-decay.
int launch_chunk_cumsum(const float *dt_p, const float *A_log, const float *dt_bias,
                        const float *log_decay, int B, int H, int N, int chunk, float *acs,
                        float *chunk_sum, DeviceStatus *status, cudaStream_t stream);

}  // namespace ssd
