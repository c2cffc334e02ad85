// The step before the memory: short depthwise causal convolution of the
// projected keys, values and queries, then L2 normalisation of keys and
// queries ("Titans, explained", step 1). One kernel for the three tensors.
//
// Layout of the work: a thread owns 4 consecutive channels, so a row of d
// channels is handled by d/4 threads (a "row group"); a CTA holds RL row groups
// side by side and each row group computes RB = 8 consecutive output rows.
// A thread loads its 4 channels of the RB + 7 input rows it needs straight
// from global memory (8- or 16-byte loads; rows before the tile come from the
// neighbouring thread's rows through L1/L2, rows before the sequence from the
// caller's history or zeros), keeps them and its 4 x w filter taps in
// registers, forms every output row once and stores it with one vector store.
// The L2 norm of a key or query row is reduced with shuffles inside the row
// group when d <= 128, otherwise per warp and then across the group's warps
// through shared memory. HBM traffic is one read of the inputs and one write
// of the outputs: the kernel is bound by HBM bandwidth.
#include <cuda_bf16.h>

#include <type_traits>

#include "tm_internal.h"

namespace tmem {
namespace {

constexpr int RB = 8;        // output rows per row group
constexpr int MAXW_ALL = 8;  // largest filter width
constexpr int NT = 256;      // target threads per CTA

struct ProArgs {
  int T, d, w, H, bf16;
  const void *in[3];
  const float *filt[3];      // [H, d, w]
  const void *hist[3];       // [streams, w-1, d] or null
  void *out[3];
};

// Predicated loads into registers that already hold zero: every load of a
// thread issues back to back, and a row outside the sequence (or a tap beyond
// the filter) simply stays zero, with no branch whose join would wait on it.
__device__ __forceinline__ void ld_pred(float &x, const float *p, bool pred) {
  asm("{\n .reg .pred q;\n setp.ne.b32 q, %1, 0;\n @q ld.global.nc.f32 %0, [%2];\n}"
      : "+f"(x) : "r"((int)pred), "l"(p));
}
__device__ __forceinline__ void ld_pred(uint2 &x, const void *p, bool pred) {
  asm("{\n .reg .pred q;\n setp.ne.b32 q, %2, 0;\n @q ld.global.nc.v2.u32 {%0, %1}, [%3];\n}"
      : "+r"(x.x), "+r"(x.y) : "r"((int)pred), "l"(p));
}
__device__ __forceinline__ void ld_pred(uint4 &x, const void *p, bool pred) {
  asm("{\n .reg .pred q;\n setp.ne.b32 q, %4, 0;\n @q ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%5];\n}"
      : "+r"(x.x), "+r"(x.y), "+r"(x.z), "+r"(x.w) : "r"((int)pred), "l"(p));
}

// 4 channels of one row as raw bits: two words of bf16 pairs or four fp32 words
template <bool BF16> struct Raw;
template <> struct Raw<true> {
  uint2 u = make_uint2(0u, 0u);
  __device__ __forceinline__ void to_f32(float x[4]) const {
    x[0] = __uint_as_float(u.x << 16);
    x[1] = __uint_as_float(u.x & 0xffff0000u);
    x[2] = __uint_as_float(u.y << 16);
    x[3] = __uint_as_float(u.y & 0xffff0000u);
  }
};
template <> struct Raw<false> {
  uint4 u = make_uint4(0u, 0u, 0u, 0u);
  __device__ __forceinline__ void to_f32(float x[4]) const {
    x[0] = __uint_as_float(u.x);
    x[1] = __uint_as_float(u.y);
    x[2] = __uint_as_float(u.z);
    x[3] = __uint_as_float(u.w);
  }
};

template <bool BF16>
__device__ __forceinline__ void store4(void *p, long long i, const float o[4]) {
  if constexpr (BF16) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(o[0], o[1]);
    const __nv_bfloat162 b = __floats2bfloat162_rn(o[2], o[3]);
    uint2 u;
    u.x = *reinterpret_cast<const unsigned *>(&a);
    u.y = *reinterpret_cast<const unsigned *>(&b);
    *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p) + i) = u;
  } else {
    *reinterpret_cast<float4 *>(static_cast<float *>(p) + i) = make_float4(o[0], o[1], o[2], o[3]);
  }
}

template <typename T>
__device__ __forceinline__ T pick(int z, T a, T b, T c) { return z == 0 ? a : (z == 1 ? b : c); }

// MAXW: taps held in registers (4 or 8; taps beyond the filter width are zero);
// RBT: output rows per row group (more rows amortise the w - 1 halo rows and
// the CTA's start over more work, fewer rows give small problems more CTAs)
template <bool BF16, bool WIDE, int MAXW, int RBT = RB>
__global__ void __launch_bounds__(NT, (!WIDE && MAXW == 4) ? 3 : 2) prologue_kernel(const ProArgs a) {
  using El = typename std::conditional<BF16, __nv_bfloat16, float>::type;
  __shared__ float part[NT / 32][RBT];        // per-warp partial sums of squares (d > 128)
  const int s = blockIdx.y, z = blockIdx.z;
  const int d = a.d, w = a.w, T = a.T;
  const int d4 = d / 4;
  const int g = threadIdx.x % d4, rl = threadIdx.x / d4;
  const int RL = blockDim.x / d4;
  const int c = 4 * g;
  const long long tb = (long long)(blockIdx.x * RL + rl) * RBT;   // first output row
  const El *in = static_cast<const El *>(pick(z, a.in[0], a.in[1], a.in[2]));
  const El *hist = static_cast<const El *>(pick(z, a.hist[0], a.hist[1], a.hist[2]));
  const float *fp = pick(z, a.filt[0], a.filt[1], a.filt[2]) + ((long long)(s % a.H) * d + c) * w;
  void *out = pick(z, a.out[0], a.out[1], a.out[2]);
  const long long base = (long long)s * T * d;

  // raw[i] holds input row tb - (MAXW - 1) + i; only rows i >= MAXW - w feed a tap
  Raw<BF16> raw[RBT + MAXW - 1];
#pragma unroll
  for (int i = 0; i < RBT + MAXW - 1; ++i) {
    const long long t = tb - (MAXW - 1) + i;
    const bool live = i + w >= MAXW && t < T && (t >= 0 || hist != nullptr);
    const El *p = t >= 0 ? in + base + t * d + c : hist + ((long long)s * (w - 1) + (w - 1 + t)) * d + c;
    ld_pred(raw[i].u, p, live);
  }
  float f[MAXW][4];
#pragma unroll
  for (int j = 0; j < MAXW; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      f[j][e] = 0.f;
      ld_pred(f[j][e], fp + e * w + (j < w ? j : 0), j < w);
    }

  const bool norm = z != 1;                  // keys and queries: unit L2 norm per row
  if constexpr (!WIDE && MAXW == 4) {
    // a row group lies inside one warp: each output row is formed, reduced
    // with shuffles, scaled and stored on its own (few live registers, so
    // more CTAs and more loads in flight per SM)
    const int width = d4;
#pragma unroll
    for (int r = 0; r < RBT; ++r) {
      float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < MAXW; ++j) {
        float x[4];
        raw[r + MAXW - 1 - j].to_f32(x);
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = fmaf(f[j][e], x[e], o[e]);
      }
      if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) ss = fmaf(o[e], o[e], ss);
        for (int off = width / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        const float scale = ss > 0.f ? 1.f / sqrtf(ss) : 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] *= scale;
      }
      const long long t = tb + r;
      if (t < T) store4<BF16>(out, base + t * d + c, o);
    }
    return;
  } else {
  float o[RBT][4];
#pragma unroll
  for (int r = 0; r < RBT; ++r)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[r][e] = 0.f;
#pragma unroll
  for (int i = 0; i < RBT + MAXW - 1; ++i) {
    float x[4];
    raw[i].to_f32(x);
#pragma unroll
    for (int j = 0; j < MAXW; ++j) {
      const int r = i + j - (MAXW - 1);      // output row that input row i feeds through tap j
      if (r < 0 || r >= RBT) continue;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[r][e] = fmaf(f[j][e], x[e], o[r][e]);
    }
  }

  if (norm) {
    float ss[RBT];
#pragma unroll
    for (int r = 0; r < RBT; ++r) {
      ss[r] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) ss[r] = fmaf(o[r][e], o[r][e], ss[r]);
    }
    const int width = d4 < 32 ? d4 : 32;
#pragma unroll
    for (int r = 0; r < RBT; ++r)
      for (int off = width / 2; off > 0; off >>= 1) ss[r] += __shfl_xor_sync(0xffffffffu, ss[r], off);
    if (d4 > 32) {                           // row group spans d4/32 whole warps
      const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
      if (lane == 0)
#pragma unroll
        for (int r = 0; r < RBT; ++r) part[warp][r] = ss[r];
      __syncthreads();
      const int w0 = rl * (d4 / 32);
#pragma unroll
      for (int r = 0; r < RBT; ++r) {
        float t = 0.f;
        for (int k = 0; k < d4 / 32; ++k) t += part[w0 + k][r];
        ss[r] = t;
      }
    }
#pragma unroll
    for (int r = 0; r < RBT; ++r) {
      const float scale = ss[r] > 0.f ? 1.f / sqrtf(ss[r]) : 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[r][e] *= scale;
    }
  }
#pragma unroll
  for (int r = 0; r < RBT; ++r) {
    const long long t = tb + r;
    if (t < T) store4<BF16>(out, base + t * d + c, o[r]);
  }
  }
}

int rows_groups_per_cta(int d) {
  const int d4 = d / 4;
  return d4 >= NT ? 1 : NT / d4;
}

}  // namespace

bool prologue_supported_d(int d) {
  return d == 32 || d == 64 || (d % 128 == 0 && d >= 128 && d <= 768);
}

cudaError_t prologue_launch(int streams, int H, int T, int d, int w, bool bf16, const void *const in[3],
                            const float *const filt[3], const void *const hist[3], void *const out[3],
                            cudaStream_t stream) {
  if (!prologue_supported_d(d) || w < 1 || w > MAXW_ALL) return cudaErrorNotSupported;
  ProArgs a;
  a.T = T;
  a.d = d;
  a.w = w;
  a.H = H;
  a.bf16 = bf16 ? 1 : 0;
  for (int i = 0; i < 3; ++i) {
    a.in[i] = in[i];
    a.filt[i] = filt[i];
    a.hist[i] = hist[i];
    a.out[i] = out[i];
  }
  const int RL = rows_groups_per_cta(d);
  const bool wide = d / 4 > 32, short_filter = w <= 4;
  // bf16, d <= 128, short filter, at least 2^20 rows per tensor: 16 rows per
  // row group (measured on 16 streams x 262144 tokens of d = 128: 3.06 ->
  // 2.79 ms; on 32 x 8192 tokens of d = 64 the 8-row form stays faster)
  const bool long_rows = bf16 && !wide && short_filter && (long long)streams * T >= (1LL << 20);
  const int rows = RL * (long_rows ? 2 * RB : RB);
  dim3 grid((unsigned)((T + rows - 1) / rows), (unsigned)streams, 3);
  const dim3 block((unsigned)(RL * (d / 4)));
  auto go = [&](auto kern) { kern<<<grid, block, 0, stream>>>(a); };
  if (long_rows) {
    go(prologue_kernel<true, false, 4, 2 * RB>);
  } else if (bf16) {
    if (wide) short_filter ? go(prologue_kernel<true, true, 4>) : go(prologue_kernel<true, true, 8>);
    else short_filter ? go(prologue_kernel<true, false, 4>) : go(prologue_kernel<true, false, 8>);
  } else {
    if (wide) short_filter ? go(prologue_kernel<false, true, 4>) : go(prologue_kernel<false, true, 8>);
    else short_filter ? go(prologue_kernel<false, false, 4>) : go(prologue_kernel<false, false, 8>);
  }
  return cudaGetLastError();
}

}  // namespace tmem
