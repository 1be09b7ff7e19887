// C entry points of libssd.so: argument validation, workspace planning and
// dispatch to the kernel paths.  The operator and the conventions are
// documented in include/ssd.h.
#include <cuda_runtime.h>

#include "ssd_internal.h"

namespace ssd {

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int check_shape(int B, int H, int N, int d, int dtype, int order, int chunk) {
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_DTYPE;
    if (order != 1 && order != 2) return SSD_ERR_ORDER;
    if (chunk != 64 && chunk != 128 && chunk != 256) return SSD_ERR_CHUNK;
    if (B < 1 || H < 1 || N < 1) return SSD_ERR_SHAPE;
    if (d != 16 && d != 32 && d != 64) return SSD_ERR_SHAPE;
    if (N % chunk != 0) return SSD_ERR_SHAPE;
    if ((long long)B * H > 65535) return SSD_ERR_SHAPE;
    if ((long long)B * H * N * d >= (1ll << 40)) return SSD_ERR_SHAPE;
    return SSD_OK;
}

void simt_layout(int B, int H, int N, int d, int order, int chunk, Plan *p) {
    const size_t BH = (size_t)B * H, nc = (size_t)N / chunk;
    const size_t Dphi = order == 1 ? (size_t)d : (size_t)d * d;
    p->path = PATH_SIMT;
    p->n_launches = 4;
    p->acs_off = kStatusBytes;
    p->lam_off = align_up(p->acs_off + BH * N * sizeof(float), 256);
    p->state_off = align_up(p->lam_off + BH * nc * sizeof(float), 256);
    p->total = align_up(p->state_off + BH * nc * Dphi * (d + 1) * sizeof(float), 256);
}

int make_plan(int B, int H, int N, int d, int dtype, int order, int normalize, int chunk,
              int value_dt, int state, Plan *plan) {
    const int rc = check_shape(B, H, N, d, dtype, order, chunk);
    if (rc != SSD_OK) return rc;
    Plan p{};
    if (order == 1 && !normalize && !(state & SSD_STATE_Z) &&
        tc_order1_supports(B, H, N, d, dtype, chunk)) {
        p.path = PATH_TC_ORDER1;
        p.n_launches = 3;
        tc_order1_layout(B, H, N, chunk, &p);
    } else if (order == 2 && tc_order2_supports(B, H, N, d, dtype, chunk)) {
        p.path = PATH_TC_ORDER2;
        p.n_launches = 1;
        p.acs_off = p.lam_off = p.state_off = kStatusBytes;
        p.total = kStatusBytes + tc_order2_workspace(B, H, N, d, chunk);
    } else {
        if (N / chunk > kMaxSimtChunks) return SSD_ERR_SHAPE;
        simt_layout(B, H, N, d, order, chunk, &p);
    }
    *plan = p;
    return SSD_OK;
}

}  // namespace ssd

using namespace ssd;

extern "C" {

size_t ssd_workspace_bytes_ex(int B, int H, int N, int d_h, int dtype, int order, int chunk,
                              int flags, int state) {
    if ((flags & ~SSD_VALUE_DT) != 0 || (state & ~(SSD_STATE_H | SSD_STATE_Z)) != 0) return 0;
    // the size covers both settings of `normalize`, which can select different paths
    size_t need = 0;
    for (int norm = 0; norm < 2; ++norm) {
        Plan p;
        if (make_plan(B, H, N, d_h, dtype, order, norm, chunk, flags & SSD_VALUE_DT, state, &p) != SSD_OK)
            return 0;
        if (p.total > need) need = p.total;
    }
    return need;
}

size_t ssd_workspace_bytes(int B, int H, int N, int d_h, int dtype, int order, int chunk) {
    return ssd_workspace_bytes_ex(B, H, N, d_h, dtype, order, chunk, 0, 0);
}

int ssd_fwd_path(int B, int H, int N, int d_h, int dtype, int order, int chunk,
                 int *n_launches) {
    Plan p;
    if (make_plan(B, H, N, d_h, dtype, order, 0, chunk, 0, 0, &p) != SSD_OK) return -1;
    if (n_launches) *n_launches = p.n_launches;
    return p.path;
}

}  // extern "C"

namespace {

int fwd_common(const void *q, const void *k, const void *v, const float *dt_p, const float *A_log,
               const float *dt_bias, const float *D, const float *log_decay, int B, int H, int N,
               int d_h, int dtype, int order, int normalize, int chunk, int flags, const float *h0,
               const float *z0, float *h_out, float *z_out, void *out, void *workspace,
               size_t workspace_bytes, void *stream, int dbg_skip, unsigned long long wait_ns,
               const ConvParams *conv = nullptr) {
    if ((flags & ~SSD_VALUE_DT) != 0) return SSD_ERR_FLAGS;
    const int value_dt = (flags & SSD_VALUE_DT) ? 1 : 0;
    if (!q || !k || !v || !out) return SSD_ERR_NULL;
    const bool need_dt = !log_decay || value_dt;  // dt feeds the decay and/or the values
    if (need_dt && (!dt_p || !dt_bias)) return SSD_ERR_NULL;
    if (!log_decay && !A_log) return SSD_ERR_NULL;
    int rc = check_shape(B, H, N, d_h, dtype, order, chunk);
    if (rc != SSD_OK) return rc;
    if (!workspace) return SSD_ERR_WORKSPACE;
    const void *ptrs[] = {q, k, v, out, dt_p, A_log, dt_bias, D, log_decay, h0, z0, h_out, z_out};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSD_ERR_ALIGN;
    const int state = ((h0 || h_out) ? SSD_STATE_H : 0) | ((z0 || z_out) ? SSD_STATE_Z : 0);
    Plan p;
    rc = make_plan(B, H, N, d_h, dtype, order, normalize, chunk, value_dt, state, &p);
    if (rc != SSD_OK) return rc;
    if (workspace_bytes < p.total) return SSD_ERR_WORKSPACE;
    FwdArgs a{q, k, v, need_dt ? dt_p : nullptr, log_decay ? nullptr : A_log,
              need_dt ? dt_bias : nullptr, D, log_decay, value_dt, h0, z0, h_out, z_out,
              B, H, N, d_h, dtype, order, normalize ? 1 : 0, chunk, out, workspace,
              workspace_bytes, static_cast<cudaStream_t>(stream)};
    a.dbg_skip = dbg_skip;
    a.wait_ns = wait_ns;
    if (conv) {
        // q, k, v are the workspace buffers for the convolved activations:
        // the order-1 tensor-core path at chunk 128 computes them inside its
        // chunk-state kernel; the other paths run the standalone convolution
        // first
        if (p.path == PATH_TC_ORDER1 && tc_order1_fuses_conv(chunk)) {
            a.conv = conv;
        } else {
            const void *dst[3] = {q, k, v};
            for (int i = 0; i < 3; ++i) {
                rc = ssd_conv1d(conv->x[i], conv->w[i], conv->bias[i], B, H, N, d_h, conv->width, conv->silu,
                                dtype, const_cast<void *>(dst[i]), stream);
                if (rc != SSD_OK) return rc;
            }
        }
    }
    switch (p.path) {
    case PATH_TC_ORDER1: return launch_tc_order1(a, p);
    case PATH_TC_ORDER2: return launch_tc_order2(a, p);
    default: return launch_simt(a, p);
    }
}

}  // namespace

extern "C" {

int ssd_fwd_state(const void *q, const void *k, const void *v, const float *dt_p,
                  const float *A_log, const float *dt_bias, const float *D, const float *log_decay,
                  int B, int H, int N, int d_h, int dtype, int order, int normalize, int chunk,
                  int flags, const float *h0, const float *z0, float *h_out, float *z_out,
                  void *out, void *workspace, size_t workspace_bytes, void *stream) {
    return fwd_common(q, k, v, dt_p, A_log, dt_bias, D, log_decay, B, H, N, d_h, dtype, order, normalize,
                      chunk, flags, h0, z0, h_out, z_out, out, workspace, workspace_bytes, stream, -1, 0);
}

int ssd_debug_fwd(const void *q, const void *k, const void *v, const float *dt_p,
                  const float *A_log, const float *dt_bias, const float *D, int B, int H, int N,
                  int d_h, int dtype, int order, int normalize, int chunk, void *out,
                  void *workspace, size_t workspace_bytes, void *stream, int skip_publish,
                  long long wait_ns) {
    if (wait_ns < 0) return SSD_ERR_SHAPE;
    if (!dt_p || !A_log || !dt_bias) return SSD_ERR_NULL;
    return fwd_common(q, k, v, dt_p, A_log, dt_bias, D, nullptr, B, H, N, d_h, dtype, order, normalize,
                      chunk, 0, nullptr, nullptr, nullptr, nullptr, out, workspace, workspace_bytes, stream,
                      skip_publish, (unsigned long long)wait_ns);
}

int ssd_fwd_ex(const void *q, const void *k, const void *v, const float *dt_p,
               const float *A_log, const float *dt_bias, const float *D, const float *log_decay,
               int B, int H, int N, int d_h, int dtype, int order, int normalize, int chunk,
               int flags, void *out, void *workspace, size_t workspace_bytes, void *stream) {
    return ssd_fwd_state(q, k, v, dt_p, A_log, dt_bias, D, log_decay, B, H, N, d_h, dtype, order,
                         normalize, chunk, flags, nullptr, nullptr, nullptr, nullptr, out, workspace,
                         workspace_bytes, stream);
}

static size_t act_bytes(int B, int H, int N, int d_h, int dtype) {
    return align_up((size_t)B * H * N * d_h * (dtype == SSD_F32 ? 4 : 2), 256);
}

size_t ssd_fwd_conv_workspace_bytes(int B, int H, int N, int d_h, int dtype, int order, int chunk,
                                    int flags) {
    const size_t base = ssd_workspace_bytes_ex(B, H, N, d_h, dtype, order, chunk, flags, 0);
    return base ? base + 3 * act_bytes(B, H, N, d_h, dtype) : 0;
}

int ssd_fwd_conv(const void *xq, const void *xk, const void *xv, const ssd_conv_params *conv,
                 const float *dt_p, const float *A_log, const float *dt_bias, const float *D,
                 const float *log_decay, int B, int H, int N, int d_h, int dtype, int order,
                 int normalize, int chunk, int flags, void *out, void *workspace,
                 size_t workspace_bytes, void *stream) {
    if (!xq || !xk || !xv || !conv || !out) return SSD_ERR_NULL;
    if (!conv->w[0] || !conv->w[1] || !conv->w[2]) return SSD_ERR_NULL;
    if (conv->width < 1 || conv->width > 4) return SSD_ERR_SHAPE;
    if ((flags & ~SSD_VALUE_DT) != 0) return SSD_ERR_FLAGS;
    int rc = check_shape(B, H, N, d_h, dtype, order, chunk);
    if (rc != SSD_OK) return rc;
    const void *x16[] = {xq, xk, xv};
    for (const void *p : x16)
        if (!aligned16(p)) return SSD_ERR_ALIGN;
    for (int i = 0; i < 3; ++i)
        if ((reinterpret_cast<uintptr_t>(conv->w[i]) & 3u) || (reinterpret_cast<uintptr_t>(conv->bias[i]) & 3u))
            return SSD_ERR_ALIGN;
    if (!workspace) return SSD_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSD_ERR_ALIGN;
    const size_t need = ssd_fwd_conv_workspace_bytes(B, H, N, d_h, dtype, order, chunk, flags);
    if (need == 0) return SSD_ERR_SHAPE;
    if (workspace_bytes < need) return SSD_ERR_WORKSPACE;
    // the convolved q, k, v sit after the operator's own workspace
    const size_t act = act_bytes(B, H, N, d_h, dtype);
    uint8_t *qc = static_cast<uint8_t *>(workspace) + (need - 3 * act);
    const ConvParams cp{{xq, xk, xv}, {conv->w[0], conv->w[1], conv->w[2]},
                        {conv->bias[0], conv->bias[1], conv->bias[2]}, conv->width, conv->silu ? 1 : 0};
    return fwd_common(qc, qc + act, qc + 2 * act, dt_p, A_log, dt_bias, D, log_decay, B, H, N, d_h, dtype,
                      order, normalize, chunk, flags, nullptr, nullptr, nullptr, nullptr, out, workspace,
                      need - 3 * act, stream, -1, 0, &cp);
}

size_t ssd_decode_workspace_bytes(int B, int H, int d_h, int order) {
    if (B < 1 || H < 1 || (long long)B * H > 65535) return 0;
    if ((d_h != 16 && d_h != 32 && d_h != 64) || (order != 1 && order != 2)) return 0;
    return kStatusBytes + decode_workspace(B, H, d_h, order);
}

int ssd_decode_step(const void *q, const void *k, const void *v, const float *dt_p,
                    const float *A_log, const float *dt_bias, const float *D,
                    const float *log_decay, int B, int H, int d_h, int dtype, int order,
                    int normalize, int flags, float *h, float *z, void *out, void *workspace,
                    size_t workspace_bytes, void *stream) {
    if ((flags & ~SSD_VALUE_DT) != 0) return SSD_ERR_FLAGS;
    const int value_dt = (flags & SSD_VALUE_DT) ? 1 : 0;
    if (!q || !k || !v || !out || !h) return SSD_ERR_NULL;
    if (normalize && !z) return SSD_ERR_NULL;
    const bool need_dt = !log_decay || value_dt;
    if (need_dt && (!dt_p || !dt_bias)) return SSD_ERR_NULL;
    if (!log_decay && !A_log) return SSD_ERR_NULL;
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_DTYPE;
    if (order != 1 && order != 2) return SSD_ERR_ORDER;
    const size_t need = ssd_decode_workspace_bytes(B, H, d_h, order);
    if (need == 0) return SSD_ERR_SHAPE;
    if (!workspace) return SSD_ERR_WORKSPACE;
    const void *ptrs[] = {q, k, v, out, h, z, D};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_ALIGN;
    const void *ptrs4[] = {dt_p, A_log, dt_bias, log_decay};  // per-token / per-head scalars
    for (const void *p : ptrs4)
        if (p && (reinterpret_cast<uintptr_t>(p) & 3u) != 0) return SSD_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SSD_ERR_ALIGN;
    if (workspace_bytes < need) return SSD_ERR_WORKSPACE;
    FwdArgs a{q, k, v, need_dt ? dt_p : nullptr, log_decay ? nullptr : A_log,
              need_dt ? dt_bias : nullptr, D, log_decay, value_dt, nullptr, nullptr, nullptr,
              nullptr, B, H, 1, d_h, dtype, order, normalize ? 1 : 0, 64, out, workspace,
              workspace_bytes, static_cast<cudaStream_t>(stream)};
    return launch_decode(a, h, z);
}

int ssd_fwd(const void *q, const void *k, const void *v, const float *dt_p,
            const float *A_log, const float *dt_bias, const float *D, int B, int H, int N,
            int d_h, int dtype, int order, int normalize, int chunk, void *out,
            void *workspace, size_t workspace_bytes, void *stream) {
    if (!dt_p || !A_log || !dt_bias) return SSD_ERR_NULL;
    return ssd_fwd_ex(q, k, v, dt_p, A_log, dt_bias, D, nullptr, B, H, N, d_h, dtype, order,
                      normalize, chunk, 0, out, workspace, workspace_bytes, stream);
}

int ssd_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                 const float *dt_p_host, const float *A_log_host, const float *dt_bias_host,
                 const float *D_host, int B, int H, int N, int d_h, int dtype, int order,
                 int normalize, int chunk, void *out_host, void *d_q, void *d_k, void *d_v,
                 float *d_dt_p, float *d_A_log, float *d_dt_bias, float *d_D, void *d_out,
                 void *workspace, size_t workspace_bytes, void *stream) {
    if (!q_host || !k_host || !v_host || !dt_p_host || !A_log_host || !dt_bias_host ||
        !out_host)
        return SSD_ERR_NULL;
    if (D_host && !d_D) return SSD_ERR_NULL;
    int rc = check_shape(B, H, N, d_h, dtype, order, chunk);
    if (rc != SSD_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t elem = dtype == SSD_F32 ? 4 : 2;
    const size_t act = (size_t)B * H * N * d_h * elem;
    const size_t tok = (size_t)B * H * N * sizeof(float);
    const size_t hp = (size_t)H * sizeof(float);
    struct Copy { void *dst; const void *src; size_t n; } h2d[] = {
        {d_q, q_host, act}, {d_k, k_host, act}, {d_v, v_host, act}, {d_dt_p, dt_p_host, tok},
        {d_A_log, A_log_host, hp}, {d_dt_bias, dt_bias_host, hp},
        {d_D, D_host, (size_t)H * d_h * sizeof(float)}};
    for (const Copy &c : h2d) {
        if (!c.src) continue;
        if (!c.dst) return SSD_ERR_NULL;
        if (cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return SSD_ERR_CUDA;
    }
    rc = ssd_fwd(d_q, d_k, d_v, d_dt_p, d_A_log, d_dt_bias, D_host ? d_D : nullptr, B, H, N,
                 d_h, dtype, order, normalize, chunk, d_out, workspace, workspace_bytes, stream);
    if (rc != SSD_OK) return rc;
    if (cudaMemcpyAsync(out_host, d_out, act, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return SSD_ERR_CUDA;
    return SSD_OK;
}

int ssd_chunk_cumsum(const float *dt_p, const float *A_log, const float *dt_bias, int B, int H,
                     int N, int chunk, float *acs, float *chunk_sum, void *stream) {
    if (!dt_p || !A_log || !dt_bias || !acs || !chunk_sum) return SSD_ERR_NULL;
    if (chunk != 64 && chunk != 128 && chunk != 256) return SSD_ERR_CHUNK;
    if (B < 1 || H < 1 || N < 1 || N % chunk != 0 || (long long)B * H > 65535)
        return SSD_ERR_SHAPE;
    if (!aligned16(dt_p) || !aligned16(acs)) return SSD_ERR_ALIGN;  // 16-byte vector accesses
    return launch_chunk_cumsum(dt_p, A_log, dt_bias, nullptr, B, H, N, chunk, acs, chunk_sum, nullptr,
                               static_cast<cudaStream_t>(stream));
}

int ssd_status_from_workspace(const void *workspace, void *stream) {
    if (!workspace) return SSD_ERR_NULL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return SSD_ERR_CUDA;
    DeviceStatus st;
    if (cudaMemcpy(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SSD_ERR_CUDA;
    return st.code;
}

const char *ssd_status_str(int status) {
    switch (status) {
    case SSD_OK: return "SSD_OK";
    case SSD_ERR_NULL: return "SSD_ERR_NULL: a required pointer is NULL";
    case SSD_ERR_SHAPE: return "SSD_ERR_SHAPE: B, H, N or d_h out of range, or N % chunk != 0";
    case SSD_ERR_DTYPE: return "SSD_ERR_DTYPE: dtype must be SSD_F32 or SSD_BF16";
    case SSD_ERR_ORDER: return "SSD_ERR_ORDER: order must be 1 or 2";
    case SSD_ERR_CHUNK: return "SSD_ERR_CHUNK: chunk must be 64, 128 or 256";
    case SSD_ERR_ALIGN: return "SSD_ERR_ALIGN: device pointer not 16-byte aligned (workspace: 256)";
    case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing or too small";
    case SSD_ERR_CUDA: return "SSD_ERR_CUDA: CUDA runtime or launch error";
    case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: a bounded device-side wait gave up";
    case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: no kernel for this combination";
    case SSD_ERR_FLAGS: return "SSD_ERR_FLAGS: unknown bits in the flags of ssd_fwd_ex";
    default: return "unknown ssd status";
    }
}

}  // extern "C"
