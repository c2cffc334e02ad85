// Internal declarations shared by the library's translation units (host side).
#pragma once
#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/titansmem.h"

namespace tmem {

constexpr int kMaxL = 4;
constexpr int kMaxC = 256;
constexpr int kMaxGroups = 8;         // layered path: concurrent groups of streams
constexpr size_t kStatusBytes = 256;  // device status word lives here

// Device status codes written by kernels (first error wins).
enum DevStatus : int {
  kDevOk = 0,
  kDevTimeout = 1,     // a bounded wait ran out
  kDevBadConfig = 2,   // kernel received a shape it was not built for
};

struct Problem {
  int L;
  int dims[kMaxL + 1];
  size_t layer_off[kMaxL + 1];
  size_t P;
  int B, H, T, C;
  int T_run;              // tokens per stream the launch processes (from t_begin); T is the stride
  int t_begin;            // CUDA-core path: first token of each stream
  int streams;
  tm_dtype in_dtype;
  const void *k, *v, *q;
  const void *k16, *q16;  // tensor-core paths: fp16 copies of k and q (workspace)
  const float *theta, *eta, *alpha;
  const float *W0, *S0;
  float *y, *W_end, *S_end;
  int *status;            // device status word
  void *scratch;          // per-stream activations (SIMT path)
  int fuse_fb;            // layered path: fused forward + backward launch where supported
  int tc_global;          // cluster-kernel path: every stream exchanges through global memory
  int bw_tc;              // backward: the chunk's products on tcgen05 (TF32) rather than fp32 FFMA
  // layered path: CUDA streams and events (owned by the context) for groups
  // 1.. of the streams; group 0 runs on the caller's stream
  void *side_streams[kMaxGroups - 1];
  void *ev_fork;
  void *ev_join[kMaxGroups - 1];
  size_t scratch_bytes;
};

// Shape checks of tm_run, shared with the other C entry points.
bool problem_from_ctx(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype dt, Problem *out);
// Aliasing rules of tm_run's buffers for problem p (shapes filled in): y
// overlaps no input or other output; W_end / S_end equal W0 / S0 exactly or
// overlap nothing else. False if a rule is broken.
bool run_aliasing_ok(const Problem &p, const void *k, const void *v, const void *q, const float *theta,
                     const float *eta, const float *alpha, const float *W0, const float *S0, const float *y,
                     const float *W_end, const float *S_end);

// fp16 copies of the keys and queries for the tensor-core paths: workspace
// bytes (both copies, 256-byte aligned) and the conversion launch (p.k, p.q
// bf16 -> p.k16, p.q16).
size_t tokens_f16_bytes(const Problem &p);
cudaError_t tokens_f16_launch(const Problem &p, cudaStream_t stream);

// SIMT (CUDA-core, fp32) path.
size_t simt_scratch_bytes(const Problem &p);
cudaError_t simt_launch(const Problem &p, cudaStream_t stream);

// Tensor-core (tcgen05) path.
bool tc_supported(const Problem &p);
size_t tc_scratch_bytes(const Problem &p);
int tc_launch_count(const Problem &p);
cudaError_t tc_launch(const Problem &p, cudaStream_t stream);
// Layer-by-layer tensor-core path 
bool tcl_supported(const Problem &p);
size_t tcl_scratch_bytes(const Problem &p);
cudaError_t tcl_launch(const Problem &p, cudaStream_t stream);
int tcl_group_count(const Problem &p);   // CUDA streams tcl_launch uses
long long tcl_launch_count(const Problem &p);
// Test hooks of the layered kernels, as tc_set_debug below.
void tcl_set_debug(int inject_timeout, unsigned long long wait_ns);
unsigned long long tcl_wait_ns();
int tcl_inject();

// Gradients of the memory layer (depths 1 to 4) with respect to its inputs.
bool backward_supported(const Problem &p);
size_t backward_scratch_bytes(const Problem &p);
cudaError_t backward_launch(const Problem &p, const float *dy, const float *dW_end, const float *dS_end,
                            float *dk, float *dv, float *dq, float *dtheta, float *deta, float *dalpha,
                            float *dW0, float *dS0, cudaStream_t stream);

// One-token decode step (C = 1), state updated in place.
bool decode_supported(const Problem &p);
cudaError_t decode_launch(const Problem &p, const void *k, const void *v, const void *q, const float *theta,
                          const float *eta, const float *alpha, float *W, float *S, float *y, cudaStream_t st);

// Depthwise causal convolution + L2 normalisation before the memory.
bool prologue_supported_d(int d);
cudaError_t prologue_launch(int streams, int H, int T, int d, int w, bool bf16, const void *const in[3],
                            const float *const filt[3], const void *const hist[3], void *const out[3],
                            cudaStream_t stream);

// Test hooks of the tensor-core path: make the first wait of every CTA one
// that nothing completes, and/or shorten the per-wait time limit (0 = 2 s).
void tc_set_debug(int inject_timeout, unsigned long long wait_ns);

}  // namespace tmem
