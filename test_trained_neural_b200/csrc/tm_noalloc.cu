// tm_run_noalloc: the write-and-read for callers that must not allocate
// device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the memory:
// a serving loop with a latency budget (cudaMalloc and cudaFree may
// synchronize the device and stall every stream), or code embedded in a
// framework whose memory manager owns all device memory and forbids outside
// allocations. tm_run needs a caller-provided workspace for the CUDA-core
// kernel's per-stream activations; this entry point instead uses a fixed
// array that lives in the library's own device memory, so the caller only
// passes inputs and outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it until the process exits. All calls on a device share it
// and it keeps the contents of the last call; the status word at its start is
// cleared by every call, the activation area is fully written before it is
// read. Calls whose kernels overlap on the GPU (different streams, or
// different host threads) race on the array and must be serialised by the
// caller.
#include <mutex>

#include <cuda.h>

#include "tm_internal.h"

namespace {

constexpr size_t kScratchMax = 16u << 20;  // activation bytes the array holds
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[tmem::kStatusBytes + kScratchMax];

// Device address of g_noalloc_scratch per device, and the id of the CUDA
// context it was looked up in. In host code the symbol itself is only a
// host-side stand-in; the address comes from cudaGetSymbolAddress with that
// device current. A context created after a reset of the device (for
// example cudaDeviceReset) loads the module afresh and the array may move,
// so the address is looked up again whenever the current context's id
// differs from the one recorded.
struct ScratchAddr {
  void *ptr = nullptr;
  unsigned long long ctx_id = 0;
};
ScratchAddr g_scratch_dev[kMaxDevices];
std::mutex g_scratch_mu;

// Id of the CUDA context current on this thread; 0 if none is current yet.
// The two driver functions are resolved through the runtime, so that the
// library loads on machines without the driver library.
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_current || !get_id) {
    void *a = nullptr, *b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qb != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return 0;
    }
    get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    get_id = reinterpret_cast<CtxGetIdFn>(b);
  }
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

tm_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr &e = g_scratch_dev[dev];
  const unsigned long long id = current_ctx_id();
  if (!e.ptr || id == 0 || id != e.ctx_id) {
    // set-up for this device (and context): cudaGetSymbolAddress also makes
    // the device's primary context current when no context is yet
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return TM_ERR_CUDA;
    e.ptr = ptr;
    e.ctx_id = current_ctx_id();
  }
  *out = e.ptr;
  return TM_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

tm_status tm_run_noalloc(tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                         const void *k, const void *v, const void *q, const float *theta,
                         const float *eta, const float *alpha, const float *W0, const float *S0,
                         float *y, float *W_end, float *S_end, void *stream) {
  tmem::Problem p;
  if (!tmem::problem_from_ctx(ctx, B, H, T, C, in_dtype, &p)) return TM_ERR_INVALID_ARG;
  const void *ptrs[] = {k, v, q, theta, eta, alpha, W0, S0, y, W_end, S_end};
  for (const void *x : ptrs)
    if (!x || !aligned16(x)) return TM_ERR_INVALID_ARG;
  // Problems whose activations do not fit the fixed array are refused before
  // any CUDA call.
  const size_t need = tmem::simt_scratch_bytes(p);
  if (need > kScratchMax) return TM_ERR_OOM;
  // the same aliasing rules as tm_run
  if (!tmem::run_aliasing_ok(p, k, v, q, theta, eta, alpha, W0, S0, y, W_end, S_end)) return TM_ERR_INVALID_ARG;
  void *base = nullptr;
  tm_status st = scratch_address(&base);
  if (st != TM_OK) return st;
  p.k = k;
  p.v = v;
  p.q = q;
  p.theta = theta;
  p.eta = eta;
  p.alpha = alpha;
  p.W0 = W0;
  p.S0 = S0;
  p.y = y;
  p.W_end = W_end;
  p.S_end = S_end;
  p.status = static_cast<int *>(base);
  p.scratch = static_cast<unsigned char *>(base) + tmem::kStatusBytes;
  p.scratch_bytes = kScratchMax;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(p.status, 0, sizeof(int), s) != cudaSuccess) return TM_ERR_CUDA;
  return tmem::simt_launch(p, s) == cudaSuccess ? TM_OK : TM_ERR_CUDA;
}

}  // extern "C"
