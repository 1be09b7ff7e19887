/*
 * ssd.h -- C ABI of libssd.so, the B200 (sm_100a) implementation of the
 * forward pass of the causal, decay-masked linear-attention ("SSD") operator
 * of Mamba-2 / Mamba-2S / 2Mamba.
 *
 * The operator (2Mamba2Furious, Mongaras & Larson 2026; Algorithm 1 "Linear
 * attention", Algorithm 3 "Mamba-2 Forward Pass", Algorithm 4 "Mamba-2S",
 * Algorithm 5 "2Mamba"), per batch b and head h, for rows i and columns j of
 * one sequence of N tokens:
 *
 *     A_h    = -exp(A_log[h])                              (Algorithm 3)
 *     dt_t   = softplus(dt_p[b,h,t] + dt_bias[h])          (Algorithm 3)
 *     A^CS_t = sum_{tau <= t} A_h dt_tau   (inclusive)     (Algorithm 3)
 *     w_ij   = (q_i . k_j)^order * exp(A^CS_i - A^CS_j) * [i >= j]
 *                                                   (Algorithms 1, 4 and 5)
 *     y_i    = sum_j w_ij v_j                              (Algorithm 1 / 5)
 *     y_i   /= sum_j w_ij            when normalize != 0   (Algorithm 1 / 5)
 *     y_ic  += D[h*d_h + c] v_ic     when D != NULL        (Algorithm 3, D_res)
 *
 * order 1 is plain linear attention with the Mamba-2 decay mask; order 2 is
 * 2Mamba's squared score, whose recurrent form (Algorithm 6 "2Mamba
 * Inference") carries a d_h^2 x d_h state.  The library evaluates it in
 * chunks of `chunk` tokens: a quadratic form inside each chunk plus a state
 * carried across chunks.  The result does not depend on `chunk` except
 * through rounding.
 *
 * Conventions for every entry point:
 *  - Layouts are row-major and contiguous: q, k, v, out are [B, H, N, d_h];
 *    dt_p is [B, H, N]; A_log and dt_bias are [H]; D is [H*d_h].
 *  - Pointers marked "device" must point to device memory of the current
 *    CUDA device, 16-byte aligned.  The caller owns every buffer; the library
 *    allocates no memory and keeps no state between calls, so calls on
 *    different streams with different buffers are independent.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as
 *    void*, NULL = the legacy default stream).  The return value reports
 *    argument validation and launch errors only; errors detected on the
 *    device are read back with ssd_status_from_workspace().
 *  - Arithmetic is fp32 for the decay, the scores' products and all
 *    accumulation; bf16 inputs feed the tensor cores as bf16 (the score
 *    matrix P and the carried state are rounded to bf16 as MMA operands) and
 *    the output is rounded to the input dtype with round-to-nearest-even.
 */
#ifndef SSD_B200_H
#define SSD_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum {
    SSD_OK = 0,
    SSD_ERR_NULL = 1,        /* a required pointer is NULL */
    SSD_ERR_SHAPE = 2,       /* B, H, N or d_h out of range, or N % chunk != 0 */
    SSD_ERR_DTYPE = 3,       /* dtype is not SSD_F32 or SSD_BF16 */
    SSD_ERR_ORDER = 4,       /* order is not 1 or 2 */
    SSD_ERR_CHUNK = 5,       /* chunk is not 64, 128 or 256 */
    SSD_ERR_ALIGN = 6,       /* a device pointer is not 16-byte aligned */
    SSD_ERR_WORKSPACE = 7,   /* workspace NULL or smaller than ssd_workspace_bytes() */
    SSD_ERR_CUDA = 8,        /* a CUDA runtime call or kernel launch failed */
    SSD_ERR_TIMEOUT = 9,     /* a device-side wait ran out (read back from the workspace) */
    SSD_ERR_UNSUPPORTED = 10, /* a valid combination the library has no kernel for */
    SSD_ERR_FLAGS = 11       /* unknown bits in the flags of ssd_fwd_ex() */
} ssd_status;

/* Option bits of ssd_fwd_ex(). */
typedef enum {
    /* Value discretisation (2Mamba2Furious, Algorithm 4: V_dt = V (.) dt):
     * the contraction uses v_t * dt_t, dt_t = softplus(dt_p[t] + dt_bias[h]).
     * The row normaliser and the D residual still use the raw scores and the
     * raw v. */
    SSD_VALUE_DT = 1
} ssd_flags;

/* Element type of q, k, v and out. */
typedef enum { SSD_F32 = 0, SSD_BF16 = 1 } ssd_dtype;

/*
 * Bytes of device workspace ssd_fwd() needs for this problem (either
 * normalize setting).  Depends only on the arguments.  Returns 0 when the arguments are invalid (ssd_fwd
 * would reject them).  Supported: B, H >= 1; N >= 1 with N % chunk == 0;
 * d_h in {16, 32, 64}; order in {1, 2}; chunk in {64, 128, 256}.
 */
size_t ssd_workspace_bytes(int B, int H, int N, int d_h, int dtype, int order, int chunk);

/* State arguments of ssd_fwd_state() that are in use (bit mask). */
typedef enum { SSD_STATE_H = 1, SSD_STATE_Z = 2 } ssd_state_mask;

/*
 * Bytes of device workspace ssd_fwd_ex() / ssd_fwd_state() need: `flags` as
 * passed to them, `state` = SSD_STATE_H if h0 or h_out is given, | SSD_STATE_Z
 * if z0 or z_out is given (0 for ssd_fwd_ex).  Either normalize setting.
 * 0 for invalid arguments.
 */
size_t ssd_workspace_bytes_ex(int B, int H, int N, int d_h, int dtype, int order, int chunk,
                              int flags, int state);

/*
 * Forward pass of the operator above.
 *   q, k, v    device, [B, H, N, d_h], element type `dtype`
 *   dt_p       device, [B, H, N] fp32 (the per-token dt projection, Algorithm 3)
 *   A_log      device, [H] fp32
 *   dt_bias    device, [H] fp32
 *   D          device, [H*d_h] fp32, or NULL for no residual
 *   normalize  nonzero: divide each row by its row sum (Algorithm 1, y / N)
 *   chunk      chunk length in tokens (64, 128 or 256), N % chunk == 0; the
 *              order-2 path in the masked quadratic form (ssd_fwd_path() = 3)
 *              does not chunk the sequence, and its result does not depend
 *              on it
 *   out        device, [B, H, N, d_h], element type `dtype`; must not alias
 *              an input
 *   workspace  device, at least ssd_workspace_bytes(...) bytes, 256-byte
 *              aligned; its contents on entry do not matter.  The first 16
 *              bytes receive the device status read by
 *              ssd_status_from_workspace().
 * Returns SSD_OK or an error code; on error nothing is enqueued.
 */
int ssd_fwd(const void *q, const void *k, const void *v,
            const float *dt_p, const float *A_log, const float *dt_bias,
            const float *D,
            int B, int H, int N, int d_h, int dtype,
            int order, int normalize, int chunk,
            void *out, void *workspace, size_t workspace_bytes,
            void *stream);

/*
 * The operator with the Mamba-2S options of 2Mamba2Furious Algorithm 4.
 * Same arguments and conventions as ssd_fwd(), plus:
 *   log_decay  device, [B, H, N] fp32, or NULL.  When given, the per-token
 *              log-decay a_t = log_decay[t] (natural log, normally <= 0, e.g.
 *              -softplus(h W_A)) replaces A_h * dt_t, so the mask is
 *              exp(cumsum(a)_i - cumsum(a)_j); A_log is then not read and may
 *              be NULL.
 *   flags      0 or SSD_VALUE_DT.  dt_p and dt_bias must be given when
 *              log_decay is NULL or SSD_VALUE_DT is set; otherwise they may
 *              be NULL.
 * ssd_fwd(...) is ssd_fwd_ex(..., log_decay = NULL, flags = 0).
 * workspace_bytes must be at least ssd_workspace_bytes_ex(..., flags, 0).
 * Paths: both options run on the tensor-core paths where the shape allows
 * (value discretisation scales V by dt on chip); otherwise on the SIMT path.
 * Errors as ssd_fwd(), plus SSD_ERR_FLAGS for unknown flag bits.
 */
int ssd_fwd_ex(const void *q, const void *k, const void *v,
               const float *dt_p, const float *A_log, const float *dt_bias,
               const float *D, const float *log_decay,
               int B, int H, int N, int d_h, int dtype,
               int order, int normalize, int chunk, int flags,
               void *out, void *workspace, size_t workspace_bytes,
               void *stream);

/*
 * ssd_fwd() with the activations in HOST memory: enqueues the host-to-device
 * copies of q, k, v, dt_p, A_log, dt_bias and D (when non-NULL) into the
 * caller's device buffers, the forward pass, and the device-to-host copy of
 * the result into out_host.  Host buffers should be pinned (cudaHostAlloc /
 * torch pin_memory) for the copies to be asynchronous.  The d_* buffers are
 * device buffers of the shapes listed for ssd_fwd(); every d_* but d_D must
 * be non-NULL, and d_D may be NULL only when D_host is NULL.
 *
 * When q, k and v hold 4 MiB or more, the heads go through in up to four
 * slices (whole batches when B >= 2; ranges of heads starting at multiples of
 * 4 when B = 1 and H >= 8): a slice's input copies run on a copy stream of
 * the library while the previous slice's forward pass and output copy run on
 * `stream`, so the two directions of the host link overlap.  The copy
 * stream and its events are created on the first such call in a CUDA context
 * (per context, kept until exit; where they cannot be created the call runs
 * as one slice on `stream`) and wait for the work enqueued on `stream`
 * before the call; every later step of the call is enqueued on `stream`, so
 * synchronising `stream` before reading out_host suffices, as for one slice.
 * Concurrent calls from several host threads in one context are serialised
 * while they enqueue.  The status word of the workspace
 * (ssd_status_from_workspace) reports the first slice that failed.
 * Errors: as ssd_fwd(), checked on the whole problem before anything is
 * enqueued; SSD_ERR_CUDA when a copy or an event record or wait fails.
 */
int ssd_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                 const float *dt_p_host, const float *A_log_host,
                 const float *dt_bias_host, const float *D_host,
                 int B, int H, int N, int d_h, int dtype,
                 int order, int normalize, int chunk,
                 void *out_host,
                 void *d_q, void *d_k, void *d_v, float *d_dt_p,
                 float *d_A_log, float *d_dt_bias, float *d_D, void *d_out,
                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * Chunked decay (Algorithm 3, last line, evaluated per chunk):
 *   acs[b,h,t]       = sum over tau in t's chunk, tau <= t, of A_h dt_tau
 *                      (the chunk-local inclusive cumulative sum, fp32)
 *   chunk_sum[b,h,c] = the same sum over the whole chunk c (= acs at the
 *                      chunk's last token)
 * A^CS_i - A^CS_j for i, j in one chunk equals acs[i] - acs[j]; across chunks
 * the global value is recovered by adding the chunk_sum of the chunks in
 * between.  dt_p, A_log, dt_bias, acs ([B,H,N]) and chunk_sum ([B,H,N/chunk])
 * are device pointers; dt_p and acs 16-byte aligned (SSD_ERR_ALIGN
 * otherwise).  chunk in {64, 128, 256}; N % chunk == 0.
 */
int ssd_chunk_cumsum(const float *dt_p, const float *A_log, const float *dt_bias,
                     int B, int H, int N, int chunk,
                     float *acs, float *chunk_sum, void *stream);

/*
 * Synchronises `stream`, then reads the device status that the kernels of
 * the last ssd_fwd() on this workspace wrote (SSD_OK or SSD_ERR_TIMEOUT when
 * a bounded inter-block wait gave up; the output is then incomplete).
 * Returns SSD_ERR_CUDA if the synchronisation itself fails.
 */
int ssd_status_from_workspace(const void *workspace, void *stream);

/*
 * ssd_fwd() for callers that cannot allocate device memory: a library or
 * plugin whose host application owns the device memory pool and forbids
 * cudaMalloc, or code that must not risk the device-wide synchronisation
 * that cudaMalloc / cudaFree can cause.  The operator has no counterpart of
 * this call on the pages; it only changes where the scratch lives.
 *
 * It runs the general SIMT path (four kernels) on a scratch buffer built
 * into the library: a fixed 16 MiB array in device memory, which every GPU
 * that loads the library holds until the process exits.  Nothing is
 * allocated and no workspace is passed; inputs and output are the caller's
 * device buffers, with the shapes and rules of ssd_fwd().
 *  - Problems whose scratch (the same as ssd_fwd's SIMT path: about
 *    4*B*H*N + 4*B*H*(N/chunk)*d_h^order*(d_h+1) bytes) exceeds 16 MiB are
 *    rejected with SSD_ERR_WORKSPACE before anything is enqueued.
 *  - It runs in the CUDA context current on the calling thread (the
 *    runtime's primary context, or a context the host application made
 *    itself with the driver API).  The first call in each context looks up
 *    the buffer's device address there (cudaGetSymbolAddress, which also
 *    loads the library's module into that context if needed); make that
 *    first call before any stream capture.  Later calls in the same context
 *    reuse the address; a new context -- one created later, or the primary
 *    context re-created after cudaDeviceReset -- gets its own lookup.
 *  - All calls on one device share the one buffer and it keeps the last
 *    call's contents (the kernels write everything they later read).  Calls
 *    that can overlap on the GPU -- on different streams without ordering
 *    between them -- race on it and give wrong results; serialise them.
 *  - The path has no device-side waits, so there is no device status to
 *    read back.
 */
int ssd_fwd_noalloc(const void *q, const void *k, const void *v,
                    const float *dt_p, const float *A_log, const float *dt_bias,
                    const float *D,
                    int B, int H, int N, int d_h, int dtype,
                    int order, int normalize, int chunk,
                    void *out, void *stream);

/*
 * ssd_fwd_ex() with the carried state in and out (prefill before decode;
 * 2Mamba2Furious Algorithm 6, whose state update H_t = a_t H_{t-1} +
 * phi(k_t) v_t^T this continues).  Extra arguments, each may be NULL:
 *   h0     device, [B, H, D_phi, d_h] fp32, the state carried into token 0
 *          (D_phi = d_h for order 1, d_h^2 for order 2; feature (a, b) of
 *          order 2 is row a*d_h + b).  NULL = zero.
 *   z0     device, [B, H, D_phi] fp32, the normaliser state carried in.
 *          NULL = zero.
 *   h_out  device, [B, H, D_phi, d_h] fp32, receives the state after token
 *          N-1.  May equal h0 (updated in place).
 *   z_out  device, [B, H, D_phi] fp32, the normaliser state after token N-1.
 *          May equal z0.
 * With value discretisation the state accumulates phi(k) (dt v)^T; the
 * normaliser state never sees dt.  Paths: order 1 with h0/h_out only, and
 * order 2 with any state, run on the tensor-core paths where the shape
 * allows; z0/z_out for order 1 run on the SIMT path.  Errors as
 * ssd_fwd_ex().
 */
int ssd_fwd_state(const void *q, const void *k, const void *v,
                  const float *dt_p, const float *A_log, const float *dt_bias,
                  const float *D, const float *log_decay,
                  int B, int H, int N, int d_h, int dtype,
                  int order, int normalize, int chunk, int flags,
                  const float *h0, const float *z0, float *h_out, float *z_out,
                  void *out, void *workspace, size_t workspace_bytes,
                  void *stream);

/*
 * Bytes of device workspace ssd_decode_step() needs (0 for invalid
 * arguments: d_h in {16, 32, 64}, order in {1, 2}, B, H >= 1).
 */
size_t ssd_decode_workspace_bytes(int B, int H, int d_h, int order);

/*
 * One recurrent step per (b, h): the token-by-token form of 2Mamba2Furious
 * Algorithm 6 used for generation after a prefill.
 *   q, k, v    device, [B, H, d_h], element type `dtype`
 *   dt_p       device, [B, H] fp32 (may be NULL when log_decay is given and
 *              SSD_VALUE_DT is not set); A_log, dt_bias [H] fp32 as in
 *              ssd_fwd_ex(); log_decay device [B, H] fp32 or NULL
 *   D          device, [H*d_h] fp32, or NULL
 *   h          device, [B, H, D_phi, d_h] fp32, updated in place:
 *              h <- a h + phi(k) (f v)^T, a = exp(log-decay), f = dt or 1
 *   z          device, [B, H, D_phi] fp32, updated in place when given:
 *              z <- a z + phi(k); required when normalize != 0, may be NULL
 *              otherwise
 *   out        device, [B, H, d_h], element type `dtype`:
 *              y = phi(q)^T h [/ phi(q) . z] [+ D (.) v]
 *   workspace  device, >= ssd_decode_workspace_bytes(), 256-byte aligned
 * The step reads and writes the whole state once (memory-bound: order 2 at
 * d_h = 64 moves 2 MiB per head).  Two launches.  Errors as ssd_fwd_ex().
 */
int ssd_decode_step(const void *q, const void *k, const void *v,
                    const float *dt_p, const float *A_log, const float *dt_bias,
                    const float *D, const float *log_decay,
                    int B, int H, int d_h, int dtype, int order, int normalize, int flags,
                    float *h, float *z, void *out,
                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * Causal depthwise convolution over tokens with optional SiLU, the prologue
 * Q, K, V = SiLU(conv_1d(h W_QKV)) of 2Mamba2Furious Algorithm 3 and the
 * window-2 convolution conv_1d(q_t, q_{t-1}) of its Algorithm 6 page.  Apply
 * it to each of q, k, v before ssd_fwd, or call ssd_fwd_conv(), which fuses
 * it into the order-1 tensor-core path.
 *   x      device, [B, H, N, d_h], element type `dtype` (pre-convolution)
 *   w      device, [H*d_h, width] fp32; w[c][j] multiplies token t - j of
 *          channel c = h*d_h + channel (j = 0 is the current token)
 *   bias   device, [H*d_h] fp32, or NULL
 *   width  1..4 (the pages use 2)
 *   silu   nonzero: out = SiLU(u) = u / (1 + e^-u), else out = u
 *   out    device, [B, H, N, d_h], `dtype`; must not overlap x
 * Tokens before the first of each (b, h) count as zero.  Asynchronous on
 * `stream`.  Returns SSD_OK, SSD_ERR_NULL, SSD_ERR_DTYPE, SSD_ERR_SHAPE
 * (sizes, width, or out overlapping x), SSD_ERR_ALIGN (x, out 16 bytes;
 * w, bias 4 bytes) or SSD_ERR_CUDA.
 */
int ssd_conv1d(const void *x, const float *w, const float *bias, int B, int H, int N, int d_h,
               int width, int silu, int dtype, void *out, void *stream);

/* Taps of the convolution prologue of ssd_fwd_conv(), one set per input. */
typedef struct {
    const float *w[3];    /* for q, k, v: device, [H*d_h, width] fp32, as w of ssd_conv1d() */
    const float *bias[3]; /* device, [H*d_h] fp32, or NULL */
    int width;            /* 1..4 (the pages use 2) */
    int silu;             /* nonzero: SiLU after each convolution */
} ssd_conv_params;

/*
 * Bytes of device workspace ssd_fwd_conv() needs: the operator's
 * (ssd_workspace_bytes_ex(..., flags, 0)) plus room for the convolved q, k,
 * v.  0 for invalid arguments.
 */
size_t ssd_fwd_conv_workspace_bytes(int B, int H, int N, int d_h, int dtype, int order, int chunk,
                                    int flags);

/*
 * The operator with its convolution prologue, 2Mamba2Furious Algorithm 3
 * (Q, K, V = SiLU(conv_1d(h W_QKV))) and the window-2 conv_1d(q_t, q_{t-1})
 * of its Algorithm 6 page:
 *   q = act(conv(xq)), k = act(conv(xk)), v = act(conv(xv)),
 * each exactly as ssd_conv1d() computes it (rounded to `dtype`), then
 * ssd_fwd_ex(q, k, v, ...) with the remaining arguments.
 *   xq, xk, xv  device, [B, H, N, d_h], `dtype`, the activations before the
 *               convolution, 16-byte aligned
 *   conv        host pointer to the taps (w, bias: 4-byte aligned)
 *   workspace   at least ssd_fwd_conv_workspace_bytes(...) bytes; the
 *               convolved q, k, v are left in its last three
 *               B*H*N*d_h-element blocks (each rounded up to 256 bytes)
 * On the order-1 tensor-core path at chunk 128 (bf16, d_h = 64) the
 * convolution is fused: the chunk-state kernel reads the raw tiles, convolves
 * them in shared memory with a three-token halo and stores the results, which
 * the chunk scan reads; the separate convolution passes disappear.  Other
 * shapes, chunk 256 included, run ssd_conv1d() three times, then the
 * operator.  The result equals
 * ssd_conv1d() on each input followed by ssd_fwd_ex(), bit for bit.  Errors
 * as ssd_fwd_ex(), plus SSD_ERR_NULL for missing taps and SSD_ERR_SHAPE for
 * a width outside 1..4.
 */
int ssd_fwd_conv(const void *xq, const void *xk, const void *xv, const ssd_conv_params *conv,
                 const float *dt_p, const float *A_log, const float *dt_bias, const float *D,
                 const float *log_decay, int B, int H, int N, int d_h, int dtype, int order,
                 int normalize, int chunk, int flags, void *out, void *workspace,
                 size_t workspace_bytes, void *stream);

/*
 * Test hook for the device-side failure detection; the pages have no
 * counterpart.  ssd_fwd() with three arguments that only failure tests use:
 *   skip_publish  >= 0: on the tensor-core paths, one producer inside the
 *                 kernels skips its publication at that pipeline step, so
 *                 the consumer's bounded wait runs out; -1: none (the call
 *                 is then ssd_fwd())
 *   wait_ns       limit of every bounded device-side wait in nanoseconds
 *                 (0: the default of one second)
 *   path          -1: the path ssd_fwd() takes; 2: the path of a call that
 *                 carries a state (the chunked order-2 kernel), although
 *                 none is carried (the workspace must then be sized with
 *                 ssd_workspace_bytes_ex(..., state = SSD_STATE_H));
 *                 other values return SSD_ERR_UNSUPPORTED
 * A wait that runs out never traps: it records SSD_ERR_TIMEOUT in the
 * workspace status, every role of the kernel stops, the copies and matrix
 * products already in flight complete, the tensor memory is freed and the
 * kernel returns.  ssd_status_from_workspace() then reports
 * SSD_ERR_TIMEOUT; the output is incomplete.  The same workspace can be
 * used by the next call (every call resets the status).  Other errors as
 * ssd_fwd(), plus SSD_ERR_SHAPE for a negative wait_ns.
 */
int ssd_debug_fwd(const void *q, const void *k, const void *v,
                  const float *dt_p, const float *A_log, const float *dt_bias,
                  const float *D,
                  int B, int H, int N, int d_h, int dtype,
                  int order, int normalize, int chunk,
                  void *out, void *workspace, size_t workspace_bytes,
                  void *stream, int skip_publish, long long wait_ns, int path);

/* Human-readable name of a status code (static string, never NULL). */
const char *ssd_status_str(int status);

/*
 * Which kernel sequence ssd_fwd() runs for these arguments: 0 = the general
 * SIMT path (any supported shape, fp32 or bf16), 1 = the order-1 tcgen05
 * path (chunk states, state passing, chunk outputs: three launches),
 * 2 = the chunked order-2 tcgen05 path (one launch: the D^2 x D state of a
 * head spread over a cluster of CTAs; calls that carry a state in or out
 * take it), 3 = the order-2 tcgen05 path in the masked quadratic form
 * (Algorithm 5; two launches: the decay factors, then a flash-style loop
 * over key tiles; bf16, d_h in {32, 64}, N a multiple of 128, no carried
 * state); -1 when the arguments are invalid.
 * *n_launches (may be NULL) receives the number of kernels one call launches.
 */
int ssd_fwd_path(int B, int H, int N, int d_h, int dtype, int order, int chunk,
                 int *n_launches);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_H */
