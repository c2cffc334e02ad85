/*
 * libtitansmem: chunked write-and-read of the Titans neural long-term memory
 * on NVIDIA B200 (sm_100a).
 *
 * The memory M is a bias-free MLP of depth L (1..4) per stream, where a stream
 * is one (batch entry, head) pair. Depth 1 is the linear map W. Between layers
 * the activation is SiLU; after the last layer there is none. Widths are
 * n_0 = d_h, n_1..n_{L-1} = expansion * d_h, n_L = d_h.
 *   ("Titans, explained", glossary entry "M — the memory"; "titans-pytorch"
 *    review: the "simple 1-4 layer MLP" neural memory)
 *
 * One call processes T tokens per stream in chunks of C tokens. For every
 * token t of a chunk:
 *   u_t = grad_W || M(k_t) - v_t ||^2, taken at the chunk-start weights
 *         ("Titans, explained", step 2 "Measure surprise" and step 6 "Make it
 *          trainable in parallel")
 *   S_t = eta_t S_{t-1} - theta_t u_t        (step 3, momentum)
 *   W_t = (1 - alpha_t) W_{t-1} + S_t        (step 4, forget then write)
 *   y_t = M(q_t) through the chunk-start weights, no write   (step 5)
 * The chunk of token t starts at t - (t mod C), tokens counted from 0
 *   ("Attack of the Titans", section "Parallel training").
 * The chunk-start weights are those at the end of the previous chunk (W0 for
 * the first chunk of a call). Momentum S carries across chunks and calls.
 *
 * State layout ("parameter vector", P floats per stream): layer l = 1..L is a
 * row-major [n_l x n_{l-1}] block, blocks end to end in layer order, so layer l
 * starts at offset sum_{m<l} n_m n_{m-1}. tm_param_count() returns P.
 *
 * Carrying (W_end, S_end) of one call into (W0, S0) of the next, with the split
 * on a chunk boundary, equals one longer call ("titans-pytorch" review, section
 * "NeuralMemory as a standalone module": mem_state is state you carry forward).
 *
 * Threading: a tm_ctx may be used from one host thread at a time. Calls are
 * asynchronous on the given stream; calls that overlap on the GPU must not
 * share a workspace.
 */
#ifndef TITANSMEM_H
#define TITANSMEM_H

#include <stddef.h>

#if defined(__GNUC__)
#define TM_API __attribute__((visibility("default")))
#else
#define TM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tm_ctx tm_ctx; /* opaque; owned by the library */

typedef enum {
  TM_OK = 0,
  TM_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size ...                 */
  TM_ERR_UNSUPPORTED = 2,  /* valid but not implemented (shape, dtype, path)   */
  TM_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch, sync ...)    */
  TM_ERR_OOM = 4,          /* host allocation failed, or workspace too small   */
  TM_ERR_TIMEOUT = 5,      /* a bounded device-side wait expired               */
  TM_ERR_DEVICE = 6        /* the device reported an internal consistency error */
} tm_status;

typedef enum { TM_ACT_SILU = 0 } tm_act;

typedef enum {
  TM_F32 = 0,  /* k, v, q are float32; fp32 arithmetic throughout            */
  TM_BF16 = 1  /* k, v, q are bfloat16; tensor-core path, fp32 state        */
} tm_dtype;

typedef enum {
  TM_PATH_AUTO = 0,        /* TM_BF16: cluster kernel, else layered kernels, else SIMT     */
  TM_PATH_SIMT = 1,        /* fp32 CUDA-core kernel for any supported shape and dtype      */
  TM_PATH_TC = 2,          /* tcgen05 cluster kernel, state resident on chip (L = 2,
                              d in {64, 128}, hidden = 64 G, C = 64); else unsupported     */
  TM_PATH_TC_LAYERED = 3,  /* tcgen05 batched GEMMs per chunk; state in W_end / S_end
                              (widths multiples of 64, C a multiple of 64 up to 256); when
                              every width is at most 256 the forward and backward of a
                              chunk run as one fused launch, then one update launch per
                              layer; else unsupported                                      */
  TM_PATH_TC_PHASED = 4,   /* as TM_PATH_TC_LAYERED, but every forward, backward and
                              update phase its own launch (same results; for comparison)   */
  TM_PATH_TC_GLOBAL = 5    /* as TM_PATH_TC, but the CTAs of a stream exchange through
                              global memory instead of a cluster's shared memory (all
                              B*H*hidden/64 CTAs must fit on the SMs at once, else
                              unsupported). TM_PATH_TC itself uses this form, beside the
                              clusters, for the streams whose clusters do not fit at once */
} tm_path;

/*
 * Create a context for a memory of depth L (1..4), head dimension d_h and
 * hidden expansion (ignored for L == 1). Host-only: allocates the small host
 * object *out and nothing on the device.
 * Supported: d_h in [1, 1024] and a multiple of 4; expansion * d_h <= 4096.
 * Returns TM_ERR_INVALID_ARG for out == NULL or out-of-range values.
 */
TM_API tm_status tm_create(int L, int d_h, int expansion, tm_act act, tm_ctx **out);

/* Destroy a context (NULL is accepted). Host-only. */
TM_API tm_status tm_destroy(tm_ctx *ctx);

/* P, the number of floats in one stream's parameter vector; 0 for NULL. */
TM_API size_t tm_param_count(const tm_ctx *ctx);

/* Select the kernel family used by tm_run (default TM_PATH_AUTO). Host-only. */
TM_API tm_status tm_set_path(tm_ctx *ctx, tm_path path);

/* The kernel family tm_run would use for these arguments. Host-only. */
TM_API tm_status tm_query_path(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                        tm_path *out);

/*
 * Number of kernel launches one tm_run of this problem makes (no counterpart
 * in the method's description; for profiling and accounting). Host-only;
 * same errors as tm_query_path. The layered paths split the B*H streams into
 * up to 8 groups run on concurrent CUDA streams (one group's forward and
 * backward beside another group's update); the environment variable
 * TM_TCL_GROUPS (1..8), read once per process, overrides the split.
 */
TM_API tm_status tm_launch_count(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                                 long long *out);

/*
 * Bytes of device workspace tm_run needs for this problem. Host-only. The
 * workspace holds the device status word (first 256 bytes) plus per-stream
 * activations of the CUDA-core path.
 */
TM_API tm_status tm_workspace_size(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                            size_t *bytes);

/*
 * Run the chunked write-and-read for B*H independent streams on `stream`
 * (a cudaStream_t, NULL = legacy default stream). Asynchronous; allocates no
 * device buffers. On the layered paths (TM_PATH_TC_LAYERED, TM_PATH_TC_PHASED)
 * a call that repeats this context's previous call exactly (shapes, every
 * pointer, path, wait limit) captures its launch sequence into a CUDA graph
 * kept by the context (its resources are the CUDA runtime's), and identical
 * calls after it replay that graph on `stream`; any other call, and any call
 * made while `stream` is being captured by the caller, launches directly. The
 * graph reads whatever the pointers hold when it runs. Calls on one context
 * must not run concurrently.
 *
 *   k, q   [B, H, T, d_h]  in_dtype, device     keys and queries
 *   v      [B, H, T, d_h]  in_dtype, device     values
 *   theta, eta, alpha [B, H, T] float32, device  per-token gates
 *   W0, S0 [B, H, P] float32, device             state at the start of the call
 *   y      [B, H, T, d_h] float32, device        reads M(q_t), output
 *   W_end, S_end [B, H, P] float32, device       state after the last token
 *   workspace: device buffer of at least tm_workspace_size() bytes, 256-byte
 *              aligned; contents on entry are ignored.
 *
 * All pointers must be 16-byte aligned. W_end may equal W0 and S_end may equal
 * S0 (in-place update); no other aliasing is allowed, and y must not overlap
 * any input. Requires 1 <= C <= 256 and T >= 1. Chunks start at multiples
 * of C; when C does not divide T the last chunk is shorter (T % C tokens). On
 * the tensor-core paths the whole chunks run first and that last chunk runs
 * after them on the CUDA-core kernel, from the state they left.
 *
 * Errors: argument problems return at once with no launch (TM_ERR_OOM when
 * workspace_bytes is too small). A device-side error (an expired bounded wait,
 * an internal check) is recorded in the workspace's status word, which every
 * tm_run clears on `stream` before its kernels start; call tm_sync() after a
 * tm_run to learn that call's device-side status.
 */
TM_API tm_status tm_run(tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                 const void *k, const void *v, const void *q,
                 const float *theta, const float *eta, const float *alpha,
                 const float *W0, const float *S0,
                 float *y, float *W_end, float *S_end,
                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * tm_run without a workspace, for callers that must not allocate device
 * memory where they run the memory (a latency-bound serving loop, where
 * cudaMalloc/cudaFree may synchronize the device; a framework whose memory
 * manager owns all device memory). This entry point has no counterpart in the
 * method's description: it only changes where the scratch lives.
 *
 * Same arguments and semantics as tm_run, minus the workspace. It always runs
 * the CUDA-core (fp32) kernel, whose per-stream activations go to a fixed
 * 16 MiB array inside the library's device memory (held by every GPU that
 * loads the library until the process exits). Problems that need more than
 * 16 MiB of activations are refused with TM_ERR_OOM before any CUDA call.
 * Allocates nothing and calls no allocating routine.
 *
 * The first call on each device looks up the array's device address (again
 * after the device's context has been reset, e.g. by cudaDeviceReset, which
 * may move the array); make that first call before any stream capture. All
 * calls on a device share the
 * array (it keeps the last call's contents; every call clears its status
 * word): calls whose kernels overlap on the GPU race and must be serialised
 * by the caller. Device-side errors are not reported through tm_sync (there
 * is no caller workspace); argument errors are returned as by tm_run.
 */
TM_API tm_status tm_run_noalloc(tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                                const void *k, const void *v, const void *q,
                                const float *theta, const float *eta, const float *alpha,
                                const float *W0, const float *S0,
                                float *y, float *W_end, float *S_end, void *stream);

/*
 * The write-and-read with every input and output in HOST memory: the same
 * operation and results as tm_run (bit for bit: the state is carried on the
 * device between segments, and carrying the state equals one longer call,
 * "titans-pytorch" review, "NeuralMemory as a standalone module"), with the
 * host <-> device copies inside the call and overlapped with the kernels.
 *
 * T is walked in segments of `segment_tokens` tokens per stream (a multiple
 * of C, or >= T; the last segment takes the rest). With segment_tokens = 0
 * the library chooses: middle segments of about T / 16 whole chunks, and the
 * first and last three ramping up from and down to an eighth of that, so that
 * the copies no kernel runs beside (the first segment's inputs, the last
 * one's reads) are short. While the kernels run segment i, the
 * inputs of segment i + 1 are copied in on one side stream and the reads y
 * of segment i - 1 copied out on another (one cudaMemcpy2DAsync per tensor
 * and segment). W0/S0 go in before the first segment, W_end/S_end come out
 * after the last.
 *
 *   k, v, q, theta, eta, alpha, W0, S0   host memory, layouts as for tm_run
 *   y, W_end, S_end                       host memory, outputs
 *   workspace: device buffer of at least tm_host_workspace_size() bytes,
 *              256-byte aligned (tm_run's workspace for one segment, the
 *              carried state and two sets of segment buffers).
 *
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister) for
 * the copies to overlap the kernels; pageable memory gives the same results
 * without the overlap. Aliasing rules as for tm_run (W_end may equal W0, S_end
 * S0). Asynchronous: the outputs are complete once `stream` has reached the
 * point of the call (cudaStreamSynchronize or an event); the inputs must stay
 * unchanged until then. Errors as for tm_run; tm_sync(ctx, workspace, stream)
 * reports device-side errors of all segments. The context's calls must not run
 * concurrently.
 */
TM_API tm_status tm_host_workspace_size(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                                        int segment_tokens, size_t *bytes);
TM_API tm_status tm_run_host(tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                             const void *k, const void *v, const void *q,
                             const float *theta, const float *eta, const float *alpha,
                             const float *W0, const float *S0,
                             float *y, float *W_end, float *S_end,
                             int segment_tokens, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Wait for `stream`, then read and clear the device status word in
 * `workspace`. Returns TM_OK, TM_ERR_TIMEOUT or TM_ERR_DEVICE from the
 * kernels, or TM_ERR_CUDA if the stream itself reports an error.
 */
TM_API tm_status tm_sync(tm_ctx *ctx, void *workspace, void *stream);

/*
 * Gradients of the memory layer for an outer model that trains through it
 * ("Titans, explained" and "Attack of the Titans" train the memory's inputs,
 * k, v, q and the data-dependent gates, through the write-and-read; no
 * kernel form is given). For the run tm_run(k, v, q, gates, W0, S0) -> (y,
 * W_end, S_end) and upstream gradients dy, dW_end, dS_end, returns the
 * gradients of J = sum_t <dy_t, y_t> + <dW_end, W_end> + <dS_end, S_end>:
 *
 *   dy                [B, H, T, d_h] float32     gradient of the reads y
 *   dW_end, dS_end    [B, H, P] float32          gradient of the final state
 *   dk, dv, dq        [B, H, T, d_h] float32     outputs
 *   dtheta, deta, dalpha [B, H, T] float32       outputs
 *   dW0, dS0          [B, H, P] float32          outputs
 *   other arguments as for tm_run (chunk size C, a shorter last chunk allowed)
 *
 * Supported: every depth 1 to 4 (the surprise is itself a gradient, so the
 * backward takes second derivatives through the MLP), any C the forward
 * accepts; TM_ERR_UNSUPPORTED otherwise. Arithmetic: fp32 throughout for fp32
 * inputs or TM_PATH_SIMT; for bf16 inputs on the other paths the chunk's
 * matrix products run on the tensor cores with TF32 operands (rounded to
 * nearest, fp32's exponent range) and fp32 accumulation, the rest in fp32.
 * The forward is recomputed inside (chunk-start states kept in the workspace:
 * tm_backward_workspace_size()); tm_sync(ctx, workspace, stream) reports a
 * device-side error of the call (its waits are bounded).
 * Pointers 16-byte aligned; outputs must not overlap inputs or each other.
 * Errors as for tm_run. Asynchronous on `stream`; allocates nothing.
 */
TM_API tm_status tm_backward_workspace_size(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                                            size_t *bytes);
TM_API tm_status tm_backward(tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype, const void *k,
                             const void *v, const void *q, const float *theta, const float *eta,
                             const float *alpha, const float *W0, const float *S0, const float *dy,
                             const float *dW_end, const float *dS_end, float *dk, float *dv, float *dq,
                             float *dtheta, float *deta, float *dalpha, float *dW0, float *dS0, void *workspace,
                             size_t workspace_bytes, void *stream);

/*
 * One decode step: a single token per stream, the chunk size C = 1 form of
 * the write-and-read ("Titans, explained" steps 2-6: surprise of the token at
 * the current weights, momentum and forgetting, then the update). With the
 * state (W, S) before the token: y = M_W(q) (the read sees none of this
 * token's write), then S <- eta S - theta u and W <- (1 - alpha) W + S with
 * u = grad_W ||M_W(k) - v||^2, in place. Same results as tm_run with T = C = 1
 * and W_end = W0, S_end = S0 (fp32 arithmetic throughout), as one launch that
 * reads and writes every parameter of W and S once.
 *
 *   k, v, q   [B, H, d_h] in_dtype, device      the token of each stream
 *   theta, eta, alpha [B, H] float32, device
 *   W, S      [B, H, P] float32, device         state, updated in place
 *   y         [B, H, d_h] float32, device       output
 *
 * Supported: depth 1 (any d_h multiple of 4 up to 4096), or depth 2 with
 * d_h in {64, 128} and hidden = 64 G, G in {1, 2, 4, 8} (one thread-block
 * cluster of G CTAs per stream); TM_ERR_UNSUPPORTED otherwise (use tm_run
 * with T = C = 1). Pointers 16-byte aligned; y must not overlap any input or
 * the state, W not S. Errors: TM_ERR_INVALID_ARG (no launch), TM_ERR_CUDA.
 * Asynchronous on `stream`; allocates nothing.
 */
TM_API tm_status tm_decode_step(tm_ctx *ctx, int B, int H, tm_dtype in_dtype, const void *k, const void *v,
                                const void *q, const float *theta, const float *eta, const float *alpha,
                                float *W, float *S, float *y, void *stream);

/*
 * The step before the memory: a short depthwise causal convolution of the
 * projected keys, values and queries, followed by L2 normalisation of every
 * key and query row ("Titans, explained", step 1: "the projections are
 * followed by a short depthwise convolution, and keys and queries are
 * l2-normalized"). One fused launch for the three tensors; allocates nothing.
 *
 *   x_in  (k_in, v_in, q_in)  [B, H, T, d] in_dtype, device
 *   filt  (filt_k, ...)       [H, d, width] float32, device: out[t, c] =
 *                             sum_{j=0}^{width-1} filt[h, c, j] x[t - j, c]
 *   hist  (hist_k, ...)       [B, H, width-1, d] in_dtype, device, or NULL:
 *                             the last width-1 tokens before this call
 *                             (NULL = zeros); row width-1+t holds token t < 0
 *   x_out (k_out, ...)        [B, H, T, d] in_dtype, device; must not overlap
 *                             any input. A zero key/query row stays zero.
 * Requires 1 <= width <= 8, T >= 1, 16-byte aligned pointers, and d in
 * {32, 64} or a multiple of 128 up to 768 (TM_ERR_UNSUPPORTED otherwise). Returns TM_ERR_INVALID_ARG for bad arguments (no launch),
 * TM_ERR_CUDA if the launch fails.
 */
TM_API tm_status tm_prologue(int B, int H, int T, int d, int width, tm_dtype in_dtype,
                             const void *k_in, const void *v_in, const void *q_in,
                             const float *filt_k, const float *filt_v, const float *filt_q,
                             const void *hist_k, const void *hist_v, const void *hist_q,
                             void *k_out, void *v_out, void *q_out, void *stream);

/*
 * Test hook for failure handling (process-wide, host-only). inject_timeout != 0
 * makes every CTA of the tensor-core kernels (the cluster walker and the
 * layered forward/backward, per-phase and update kernels) first wait on a
 * barrier that nothing completes, so the bounded wait expires, the kernel
 * records TM_ERR_TIMEOUT, issues nothing further, cleans up and returns;
 * tm_sync() then reports it. wait_limit_ns sets the time limit of each
 * device-side wait (0 = default 2 s). Affects launches issued after the call.
 */
TM_API tm_status tm_set_debug(int inject_timeout, unsigned long long wait_limit_ns);

/* Static, NUL-terminated description of a status code. */
TM_API const char *tm_status_string(tm_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
TM_API int tm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TITANSMEM_H */
