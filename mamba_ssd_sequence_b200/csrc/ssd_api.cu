// C entry points of libssd.so: argument validation, workspace planning and
// dispatch to the kernel paths.  The operator and the conventions are
// documented in include/ssd.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "ssd_internal.h"

namespace ssd {

namespace drv {
typedef CUresult (*PfnCtxGetCurrent)(CUcontext *);
typedef CUresult (*PfnCtxGetId)(CUcontext, unsigned long long *);

template <typename F>
F driver_fn(const char *name) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<F>(p);
}
}  // namespace drv

bool current_context_id(unsigned long long *id) {
    static drv::PfnCtxGetCurrent get_ctx = drv::driver_fn<drv::PfnCtxGetCurrent>("cuCtxGetCurrent");
    static drv::PfnCtxGetId get_id = drv::driver_fn<drv::PfnCtxGetId>("cuCtxGetId");
    if (!get_ctx || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return false;
    if (ctx == nullptr) {
        // no context current on this thread yet: make the runtime's primary
        // context of the current device current (this allocates nothing)
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return false;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    }
    return get_id(ctx, id) == CUDA_SUCCESS;
}

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
    } else if (order == 2 && state == 0 && tc_order2q_supports(B, H, N, d, dtype)) {
        // without a carried state the masked quadratic form needs no D^2 x D state
        p.path = PATH_TC_ORDER2Q;
        p.n_launches = 2;
        tc_order2q_layout(B, H, N, &p);
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
               const ConvParams *conv = nullptr, int state_hint = 0) {
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
    const int state = ((h0 || h_out) ? SSD_STATE_H : 0) | ((z0 || z_out) ? SSD_STATE_Z : 0) | state_hint;
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
    case PATH_TC_ORDER2Q: return launch_tc_order2q(a, p);
    default: return launch_simt(a, p);
    }
}

// ---- ssd_fwd_host: slices of heads whose copies overlap the previous
// slice's forward pass and output copy (PCIe carries both directions at once)

constexpr int kMaxHostSlices = 4;
constexpr size_t kMinPipelinedBytes = 4u << 20;  // below this one slice is as fast

struct HostSlice {
    int b0, nb, h0, nh;
};
struct HostSlices {
    int n;
    HostSlice s[kMaxHostSlices];
};

// Whole batches when B >= 2; for B = 1, ranges of heads that start at a
// multiple of 4 (A_log, dt_bias and D stay 16-byte aligned).
HostSlices host_slices(int B, int H, size_t act_bytes) {
    HostSlices r{};
    r.n = 1;
    r.s[0] = HostSlice{0, B, 0, H};
    if (act_bytes < kMinPipelinedBytes) return r;
    if (B >= 2) {
        r.n = B < kMaxHostSlices ? B : kMaxHostSlices;
        for (int g = 0; g < r.n; ++g) {
            const int b0 = (int)((long long)B * g / r.n), b1 = (int)((long long)B * (g + 1) / r.n);
            r.s[g] = HostSlice{b0, b1 - b0, 0, H};
        }
    } else if (H >= 8) {
        const int quads = H / 4;  // whole groups of four heads; the last slice takes the rest
        r.n = quads < kMaxHostSlices ? quads : kMaxHostSlices;
        for (int g = 0; g < r.n; ++g) {
            const int h0 = 4 * (int)((long long)quads * g / r.n);
            const int h1 = g + 1 == r.n ? H : 4 * (int)((long long)quads * (g + 1) / r.n);
            r.s[g] = HostSlice{0, 1, h0, h1 - h0};
        }
    }
    return r;
}

// The copy stream and events of ssd_fwd_host, one set per CUDA context (keyed
// by the context's ID, which the driver never reuses), created on first use
// and kept until exit; nullptr when they cannot be made (or after 16
// contexts), and the call then runs as one slice.  The mutex serialises the enqueueing of one call, so
// that two host threads never interleave their event records.
struct HostPipe {
    unsigned long long ctx_id;
    cudaStream_t copy;
    cudaEvent_t entry, ready[kMaxHostSlices];
    std::mutex *mutex;
};
constexpr int kPipeSlots = 16;
HostPipe g_pipes[kPipeSlots] = {};
int g_pipe_count = 0;
std::mutex g_pipe_mutex;

const HostPipe *host_pipe() {
    unsigned long long id = 0;
    if (!current_context_id(&id)) return nullptr;
    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    for (int i = 0; i < g_pipe_count; ++i)
        if (g_pipes[i].ctx_id == id) return &g_pipes[i];
    if (g_pipe_count == kPipeSlots) return nullptr;
    HostPipe p{};
    p.ctx_id = id;
    if (cudaStreamCreateWithFlags(&p.copy, cudaStreamNonBlocking) != cudaSuccess) {
        cudaGetLastError();  // not sticky: the caller goes on with one slice
        return nullptr;
    }
    cudaEvent_t *ev[1 + kMaxHostSlices];
    ev[0] = &p.entry;
    for (int i = 0; i < kMaxHostSlices; ++i) ev[1 + i] = &p.ready[i];
    for (int i = 0; i < 1 + kMaxHostSlices; ++i) {
        if (cudaEventCreateWithFlags(ev[i], cudaEventDisableTiming) != cudaSuccess) {
            for (int j = 0; j < i; ++j) cudaEventDestroy(*ev[j]);
            cudaStreamDestroy(p.copy);
            cudaGetLastError();
            return nullptr;
        }
    }
    p.mutex = new std::mutex;
    g_pipes[g_pipe_count] = p;
    return &g_pipes[g_pipe_count++];
}

// Each slice's forward pass rewrites the status word; the slot after it in
// the status block keeps the first failure (first: the first slice; last:
// copy the kept status back into the word ssd_status_from_workspace reads).
__global__ void keep_status_kernel(DeviceStatus *st, int first, int last) {
    if (threadIdx.x != 0) return;
    DeviceStatus *kept = st + 4;  // bytes 64-79 of the 256-byte status block
    if (first || kept->code == 0) *kept = *st;
    if (last) *st = *kept;
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
                  long long wait_ns, int path) {
    if (wait_ns < 0) return SSD_ERR_SHAPE;
    if (path != -1 && path != PATH_TC_ORDER2) return SSD_ERR_UNSUPPORTED;
    if (!dt_p || !A_log || !dt_bias) return SSD_ERR_NULL;
    // path 2: the path a call with a carried state takes (the chunked order-2
    // kernel), selected as if a state were carried, though none is
    return fwd_common(q, k, v, dt_p, A_log, dt_bias, D, nullptr, B, H, N, d_h, dtype, order, normalize,
                      chunk, 0, nullptr, nullptr, nullptr, nullptr, out, workspace, workspace_bytes, stream,
                      skip_publish, (unsigned long long)wait_ns, nullptr, path == PATH_TC_ORDER2 ? SSD_STATE_H : 0);
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
    if (!d_q || !d_k || !d_v || !d_dt_p || !d_A_log || !d_dt_bias || !d_out) return SSD_ERR_NULL;
    if (D_host && !d_D) return SSD_ERR_NULL;
    int rc = check_shape(B, H, N, d_h, dtype, order, chunk);
    if (rc != SSD_OK) return rc;
    {
        // the whole problem is validated before anything is enqueued
        Plan p;
        rc = make_plan(B, H, N, d_h, dtype, order, normalize, chunk, 0, 0, &p);
        if (rc != SSD_OK) return rc;
        if (!workspace) return SSD_ERR_WORKSPACE;
        if (workspace_bytes < p.total) return SSD_ERR_WORKSPACE;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t elem = dtype == SSD_F32 ? 4 : 2;
    const size_t row_act = (size_t)N * d_h * elem;  // one (b, h) row of q, k, v or out
    const size_t row_tok = (size_t)N * sizeof(float);
    HostSlices sl = host_slices(B, H, (size_t)B * H * row_act);
    const HostPipe *pipe = sl.n > 1 ? host_pipe() : nullptr;
    if (!pipe) sl = host_slices(B, H, 0);  // no copy stream (or none needed): one slice
    // one stream (the caller's) when there is a single slice; otherwise the
    // inputs go in on the library's copy stream, after the caller's earlier work
    cudaStream_t cs = pipe ? pipe->copy : s;
    std::unique_lock<std::mutex> lock;
    if (pipe) {
        lock = std::unique_lock<std::mutex>(*pipe->mutex);
        if (cudaEventRecord(pipe->entry, s) != cudaSuccess || cudaStreamWaitEvent(cs, pipe->entry, 0) != cudaSuccess)
            return SSD_ERR_CUDA;
    }
    auto h2d = [&](void *dst, const void *src, size_t n) {
        return cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, cs) == cudaSuccess;
    };
    const size_t hp = (size_t)H * sizeof(float);
    if (!h2d(d_A_log, A_log_host, hp) || !h2d(d_dt_bias, dt_bias_host, hp) ||
        (D_host && !h2d(d_D, D_host, (size_t)H * d_h * sizeof(float))))
        return SSD_ERR_CUDA;
    for (int g = 0; g < sl.n; ++g) {
        const HostSlice &c = sl.s[g];
        // slice rows (b, h) for b in [b0, b0 + nb), h in [h0, h0 + nh): contiguous
        // when the slice is whole batches (nh = H) or one batch (nb = 1)
        const size_t r0 = (size_t)c.b0 * H + c.h0, nr = (size_t)c.nb * c.nh;
        auto act = [&](const void *base) { return static_cast<const char *>(base) + r0 * row_act; };
        auto dact = [&](void *base) { return static_cast<char *>(base) + r0 * row_act; };
        if (!h2d(dact(d_q), act(q_host), nr * row_act) || !h2d(dact(d_k), act(k_host), nr * row_act) ||
            !h2d(dact(d_v), act(v_host), nr * row_act) ||
            !h2d(reinterpret_cast<char *>(d_dt_p) + r0 * row_tok,
                 reinterpret_cast<const char *>(dt_p_host) + r0 * row_tok, nr * row_tok))
            return SSD_ERR_CUDA;
        if (pipe && (cudaEventRecord(pipe->ready[g], cs) != cudaSuccess ||
                     cudaStreamWaitEvent(s, pipe->ready[g], 0) != cudaSuccess))
            return SSD_ERR_CUDA;
        rc = ssd_fwd(dact(d_q), dact(d_k), dact(d_v), reinterpret_cast<float *>(reinterpret_cast<char *>(d_dt_p) +
                                                                                  r0 * row_tok),
                     d_A_log + c.h0, d_dt_bias + c.h0, D_host ? d_D + (size_t)c.h0 * d_h : nullptr, c.nb, c.nh, N,
                     d_h, dtype, order, normalize, chunk, dact(d_out), workspace, workspace_bytes, stream);
        if (rc != SSD_OK) return rc;
        if (sl.n > 1)  // the first failure among the slices is the one the status word keeps
            keep_status_kernel<<<1, 32, 0, s>>>(static_cast<DeviceStatus *>(workspace), g == 0, g == sl.n - 1);
        if (cudaMemcpyAsync(static_cast<char *>(out_host) + r0 * row_act, dact(d_out), nr * row_act,
                            cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return SSD_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
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
