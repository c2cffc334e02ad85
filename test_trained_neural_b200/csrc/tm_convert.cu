// Keys and queries as fp16 for the tensor-core paths.
//
// The tensor-core kernels take fp16 operands (10 mantissa bits) with fp32
// accumulation; keys and queries arrive as bf16. This pass writes fp16
// copies of both into the workspace once per call, so that the chunk kernels
// can feed them to the tensor cores by TMA as they are. bf16 -> fp16 is exact
// for the values here (unit-norm rows: every component lies well inside
// fp16's normal range, up to rare components below 6.1e-5 that become fp16
// subnormals with an absolute error under 3e-8).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "tm_internal.h"

namespace tmem {
namespace {

__device__ __forceinline__ uint4 to_f16x8(uint4 u) {
  const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&u);
  uint4 o;
  __half2 *h = reinterpret_cast<__half2 *>(&o);
#pragma unroll
  for (int e = 0; e < 4; ++e) h[e] = __float22half2_rn(__bfloat1622float2(b[e]));
  return o;
}

// Grid-stride over 16-byte pieces (8 elements) of k then q; each thread keeps
// four independent loads in flight before it converts and stores them.
constexpr int CV_UNROLL = 4;
__global__ void __launch_bounds__(256) tokens_f16_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ q,
                                                         uint4 *__restrict__ k16, uint4 *__restrict__ q16, long long n8) {
  const long long total = 2 * n8, stride = (long long)gridDim.x * blockDim.x;
  for (long long base = (long long)blockIdx.x * blockDim.x + threadIdx.x; base < total; base += stride * CV_UNROLL) {
    uint4 u[CV_UNROLL];
#pragma unroll
    for (int r = 0; r < CV_UNROLL; ++r) {
      const long long i = base + r * stride;
      if (i < total) u[r] = i < n8 ? __ldcs(k + i) : __ldcs(q + (i - n8));
    }
#pragma unroll
    for (int r = 0; r < CV_UNROLL; ++r) {
      const long long i = base + r * stride;
      if (i < total) (i < n8 ? k16[i] : q16[i - n8]) = to_f16x8(u[r]);
    }
  }
}

}  // namespace

size_t tokens_f16_bytes(const Problem &p) {
  const size_t one = (size_t)p.streams * (size_t)p.T * (size_t)p.dims[0] * 2;
  return 2 * ((one + 255) / 256 * 256);
}

cudaError_t tokens_f16_launch(const Problem &p, cudaStream_t stream) {
  const size_t n = (size_t)p.streams * (size_t)p.T * (size_t)p.dims[0];   // a multiple of 4 (d % 4 == 0)
  if (n % 8 != 0 || !p.k16 || !p.q16) return cudaErrorInvalidValue;
  const long long n8 = (long long)(n / 8);
  long long blocks = (2 * n8 + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;     // 8 CTAs of 256 threads per SM
  tokens_f16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
      static_cast<const uint4 *>(p.k), static_cast<const uint4 *>(p.q), static_cast<uint4 *>(const_cast<void *>(p.k16)),
      static_cast<uint4 *>(const_cast<void *>(p.q16)), n8);
  return cudaGetLastError();
}

}  // namespace tmem
