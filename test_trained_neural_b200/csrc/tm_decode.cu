// One decode step: a single token per stream (the chunk size C = 1 form of
// the memory's write-and-read, "Titans, explained" steps 2-6; "Attack of the
// Titans", the per-token surprise update). Per stream, with the state (W, S)
// before the token:
//   y = M_W(q)                                   read through the old weights
//   u = grad_W ||M_W(k) - v||^2                  the token's surprise
//   S <- eta S - theta u,  W <- (1 - alpha) W + S   (in place)
// which is tm_run with T = C = 1, as one launch and with the ideal traffic:
// every parameter of W and S read once and written once.
//
// Depth 2, M(x) = W2 silu(W1 x), hidden = 64 G: one thread-block cluster of G
// CTAs per stream, CTA j staging its slice of the state in shared memory
// (rows 64j.. of W1 and S1, columns 64j.. of W2 and S2). It forms its 64
// hidden units for the key and the query, its partial sums of layer 2 for
// both, and writes them into every CTA of the cluster (remote shared-memory
// stores, then one cluster barrier); every CTA sums the G partials in the
// same order, so all hold the same Z2 and G2 = 2 (Z2 - v); CTA 0 writes y.
// The backward to its hidden units and the updates of its slices run in
// shared memory; the slices are written back once.
// Depth 1 (linear memory): rows of W are independent; a warp owns a row.
#include <cuda_bf16.h>

#include "tm_internal.h"
#include "tm_sm100.cuh"

namespace tmem {
namespace {

using namespace sm100;

constexpr int DT = 256;      // threads per CTA
constexpr int DHS = 64;      // hidden units per CTA (depth 2)

struct DecArgs {
  int d, hid, G, bf16;
  long long P;
  const void *k, *v, *q;
  const float *theta, *eta, *alpha;
  float *W, *S, *y;
};

__device__ __forceinline__ float ld_tok(const void *p, int bf16, long long i) {
  return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]) : static_cast<const float *>(p)[i];
}
__device__ __forceinline__ float sigm_f(float z) { return 1.f / (1.f + expf(-z)); }
// 16-byte asynchronous copy global -> shared (all of a thread's copies in
// flight at once), and the wait for every copy issued so far.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <int D>
struct DecLayout {
  static constexpr int W1 = 0;                  // [64][D]
  static constexpr int S1 = W1 + DHS * D;
  static constexpr int W2 = S1 + DHS * D;       // [D][64]
  static constexpr int S2 = W2 + D * DHS;
  static constexpr int K = S2 + D * DHS;        // k, q, v [D]
  static constexpr int Q = K + D;
  static constexpr int V = Q + D;
  static constexpr int X1 = V + D;              // [64] silu(z1) of the key
  static constexpr int XQ = X1 + DHS;           // [64] of the query
  static constexpr int SP = XQ + DHS;           // [64] silu'(z1)
  static constexpr int G1 = SP + DHS;           // [64] layer-1 gradient
  static constexpr int PZ = G1 + DHS;           // [D] this CTA's partial Z2, then [D] partial y
  static constexpr int G2 = PZ + 2 * D;         // [D]
  static constexpr int RECV = G2 + D;           // [8][2][D] partials of every CTA
  static constexpr int RED = RECV + 8 * 2 * D;  // [4][64] partial sums of the backward
  static constexpr int TOTAL = RED + 4 * DHS;   // floats
};

template <int D>
__global__ void __launch_bounds__(DT, 1) decode2_kernel(const DecArgs a) {
  using Lay = DecLayout<D>;
  extern __shared__ __align__(16) float sm[];
  const int G = a.G;
  const int j = (int)cluster_rank();
  const int s = blockIdx.x / G;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int hid = a.hid;
  float *W1s = sm + Lay::W1, *S1s = sm + Lay::S1, *W2s = sm + Lay::W2, *S2s = sm + Lay::S2;
  float *kk = sm + Lay::K, *qq = sm + Lay::Q, *vv = sm + Lay::V;
  float *x1 = sm + Lay::X1, *xq = sm + Lay::XQ, *sp1 = sm + Lay::SP, *g1 = sm + Lay::G1;
  float *pz = sm + Lay::PZ, *g2 = sm + Lay::G2, *recv = sm + Lay::RECV, *red = sm + Lay::RED;

  float *W = a.W + (long long)s * a.P, *S = a.S + (long long)s * a.P;
  float *W1g = W + (long long)DHS * j * D, *S1g = S + (long long)DHS * j * D;   // rows of W1 [hid x D]
  float *W2g = W + (long long)hid * D, *S2g = S + (long long)hid * D;           // W2 [D x hid]

  // Consecutive steps are launched with programmatic serialization: the next
  // step may be launched now, and this one reads nothing (state or token)
  // before the previous kernel of the stream has completed.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // stage the slices (asynchronous 16-byte copies, all in flight) and the token
  for (int i = tid; i < DHS * D / 4; i += DT) {
    cp_async16(W1s + 4 * i, W1g + 4 * i);
    cp_async16(S1s + 4 * i, S1g + 4 * i);
  }
  for (int i = tid; i < D * (DHS / 4); i += DT) {
    const int r = i / (DHS / 4), c4 = i % (DHS / 4);
    const long long g = (long long)r * hid + DHS * j + 4 * c4;
    cp_async16(W2s + 4 * i, W2g + g);
    cp_async16(S2s + 4 * i, S2g + g);
  }
  for (int i = tid; i < D; i += DT) {
    kk[i] = ld_tok(a.k, a.bf16, (long long)s * D + i);
    qq[i] = ld_tok(a.q, a.bf16, (long long)s * D + i);
    vv[i] = ld_tok(a.v, a.bf16, (long long)s * D + i);
  }
  const float th = a.theta[s], et = a.eta[s], al = a.alpha[s];
  cp_async_wait_all();
  __syncthreads();

  // layer 1: this CTA's 64 hidden units for the key and the query
  for (int r = warp; r < DHS; r += DT / 32) {
    float zk = 0.f, zq = 0.f;
    for (int c = lane; c < D; c += 32) {
      const float w = W1s[r * D + c];
      zk = fmaf(w, kk[c], zk);
      zq = fmaf(w, qq[c], zq);
    }
    zk = warp_sum(zk);
    zq = warp_sum(zq);
    if (lane == 0) {
      const float sg = sigm_f(zk);
      x1[r] = zk * sg;
      sp1[r] = sg * (1.f + zk * (1.f - sg));
      xq[r] = zq * sigm_f(zq);
    }
  }
  __syncthreads();
  // layer 2: partial sums over this CTA's 64 hidden units
  for (int r = warp; r < D; r += DT / 32) {
    const float w0 = W2s[r * DHS + lane], w1 = W2s[r * DHS + lane + 32];
    float z = fmaf(w0, x1[lane], w1 * x1[lane + 32]);
    float yq = fmaf(w0, xq[lane], w1 * xq[lane + 32]);
    z = warp_sum(z);
    yq = warp_sum(yq);
    if (lane == 0) {
      pz[r] = z;
      pz[D + r] = yq;
    }
  }
  __syncthreads();
  // every CTA of the cluster receives this CTA's partials in slot j
  {
    const uint32_t dst = smem_u32(recv + j * 2 * D);
    for (int i = tid; i < G * (2 * D / 4); i += DT) {
      const int p = i / (2 * D / 4), e4 = i % (2 * D / 4);
      const float4 v4 = reinterpret_cast<const float4 *>(pz)[e4];
      st_cluster_v4(mapa(dst + 16u * e4, (uint32_t)p),
                    make_uint4(__float_as_uint(v4.x), __float_as_uint(v4.y), __float_as_uint(v4.z),
                               __float_as_uint(v4.w)));
    }
  }
  cluster_arrive_release();
  cluster_wait_acquire();
  // Z2 and y: the G partials summed in slot order (identical in every CTA)
  for (int r = tid; r < D; r += DT) {
    float z = 0.f, yq = 0.f;
    for (int p = 0; p < G; ++p) {
      z += recv[p * 2 * D + r];
      yq += recv[p * 2 * D + D + r];
    }
    g2[r] = 2.f * (z - vv[r]);
    if (j == 0) a.y[(long long)s * D + r] = yq;
  }
  __syncthreads();
  // backward to this CTA's hidden units: g1 = (W2^T G2) . silu'(z1); thread
  // (part, c) sums rows part, part + 4, ... (consecutive c: no bank conflicts)
  {
    const int c = tid % DHS, part = tid / DHS;
    float acc = 0.f;
    for (int r = part; r < D; r += DT / DHS) acc = fmaf(W2s[r * DHS + c], g2[r], acc);
    red[part * DHS + c] = acc;
  }
  __syncthreads();
  if (tid < DHS) g1[tid] = (red[tid] + red[DHS + tid] + red[2 * DHS + tid] + red[3 * DHS + tid]) * sp1[tid];
  __syncthreads();
  // updates of the slices, written back once
  const float keep = 1.f - al;
  for (int i = tid; i < DHS * D / 4; i += DT) {
    const int r = (4 * i) / D, c = (4 * i) % D;
    const float4 w4 = reinterpret_cast<const float4 *>(W1s)[i], s4 = reinterpret_cast<const float4 *>(S1s)[i];
    const float gr = th * g1[r];
    float4 sn, wn;
    sn.x = fmaf(et, s4.x, -gr * kk[c]);
    sn.y = fmaf(et, s4.y, -gr * kk[c + 1]);
    sn.z = fmaf(et, s4.z, -gr * kk[c + 2]);
    sn.w = fmaf(et, s4.w, -gr * kk[c + 3]);
    wn.x = fmaf(keep, w4.x, sn.x);
    wn.y = fmaf(keep, w4.y, sn.y);
    wn.z = fmaf(keep, w4.z, sn.z);
    wn.w = fmaf(keep, w4.w, sn.w);
    reinterpret_cast<float4 *>(S1g)[i] = sn;
    reinterpret_cast<float4 *>(W1g)[i] = wn;
  }
  for (int i = tid; i < D * (DHS / 4); i += DT) {
    const int r = i / (DHS / 4), c = 4 * (i % (DHS / 4));
    const float4 w4 = reinterpret_cast<const float4 *>(W2s)[i], s4 = reinterpret_cast<const float4 *>(S2s)[i];
    const float gr = th * g2[r];
    float4 sn, wn;
    sn.x = fmaf(et, s4.x, -gr * x1[c]);
    sn.y = fmaf(et, s4.y, -gr * x1[c + 1]);
    sn.z = fmaf(et, s4.z, -gr * x1[c + 2]);
    sn.w = fmaf(et, s4.w, -gr * x1[c + 3]);
    wn.x = fmaf(keep, w4.x, sn.x);
    wn.y = fmaf(keep, w4.y, sn.y);
    wn.z = fmaf(keep, w4.z, sn.z);
    wn.w = fmaf(keep, w4.w, sn.w);
    const long long g = (long long)r * hid + DHS * j + c;
    *reinterpret_cast<float4 *>(S2g + g) = sn;
    *reinterpret_cast<float4 *>(W2g + g) = wn;
  }
}

// Depth 1: a warp per row of W [d x d]; CTA = 8 rows of one stream.
__global__ void __launch_bounds__(DT) decode1_kernel(const DecArgs a, int rows_per_cta) {
  const int d = a.d;
  const int ctas = (d + rows_per_cta - 1) / rows_per_cta;
  const int s = blockIdx.x / ctas;
  const int r = (blockIdx.x % ctas) * rows_per_cta + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  // launched with programmatic serialization, as the depth-2 step
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (r >= d) return;
  float *Wr = a.W + (long long)s * a.P + (long long)r * d;
  float *Sr = a.S + (long long)s * a.P + (long long)r * d;
  const long long t = (long long)s * d;
  float zk = 0.f, zq = 0.f;
  for (int c = lane; c < d; c += 32) {
    const float w = Wr[c];
    zk = fmaf(w, ld_tok(a.k, a.bf16, t + c), zk);
    zq = fmaf(w, ld_tok(a.q, a.bf16, t + c), zq);
  }
  zk = warp_sum(zk);
  zq = warp_sum(zq);
  if (lane == 0) a.y[t + r] = zq;
  const float gr = a.theta[s] * 2.f * (zk - ld_tok(a.v, a.bf16, t + r));
  const float et = a.eta[s], keep = 1.f - a.alpha[s];
  for (int c = lane; c < d; c += 32) {
    const float sn = fmaf(et, Sr[c], -gr * ld_tok(a.k, a.bf16, t + c));
    Sr[c] = sn;
    Wr[c] = fmaf(keep, Wr[c], sn);
  }
}

template <int D>
cudaError_t launch2(const DecArgs &a, int streams, cudaStream_t st) {
  const size_t smem = (size_t)DecLayout<D>::TOTAL * sizeof(float);
  static bool attr_done = false;   // per process (one device)
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(decode2_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(streams * a.G));
  cfg.blockDim = dim3(DT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)a.G;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode2_kernel<D>, a);
}

}  // namespace

bool decode_supported(const Problem &p) {
  if (p.L == 1) return p.dims[0] % 4 == 0 && p.dims[0] <= 4096;
  if (p.L != 2) return false;
  const int d = p.dims[0], h = p.dims[1];
  if (d != 64 && d != 128) return false;
  if (h % DHS) return false;
  const int G = h / DHS;
  return G == 1 || G == 2 || G == 4 || G == 8;
}

cudaError_t decode_launch(const Problem &p, const void *k, const void *v, const void *q, const float *theta,
                          const float *eta, const float *alpha, float *W, float *S, float *y, cudaStream_t st) {
  if (!decode_supported(p)) return cudaErrorNotSupported;
  DecArgs a;
  a.d = p.dims[0];
  a.hid = p.L == 2 ? p.dims[1] : 0;
  a.G = p.L == 2 ? p.dims[1] / DHS : 1;
  a.bf16 = p.in_dtype == TM_BF16 ? 1 : 0;
  a.P = (long long)p.P;
  a.k = k;
  a.v = v;
  a.q = q;
  a.theta = theta;
  a.eta = eta;
  a.alpha = alpha;
  a.W = W;
  a.S = S;
  a.y = y;
  if (p.L == 1) {
    const int rows = DT / 32;
    const int ctas = (a.d + rows - 1) / rows;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.streams * ctas));
    cfg.blockDim = dim3(DT);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode1_kernel, a, rows);
  }
  return a.d == 64 ? launch2<64>(a, p.streams, st) : launch2<128>(a, p.streams, st);
}

}  // namespace tmem
