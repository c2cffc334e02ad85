// tcgen05 tensor-core chunk walker for depth-2 memories, M(x) = W2 silu(W1 x).
//
// One thread-block cluster of G CTAs walks one stream (batch entry, head).
// CTA j of the cluster owns hidden units [64 j, 64 j + 64): rows of W1 and
// columns of W2, so hidden = 64 G. Per chunk of C = 64 tokens:
//
//   A1  TMA loads keys and queries of the chunk as one 128-row fp16 tile
//       (keys rows 0-63, queries rows 64-127), 128-byte swizzle.
//   A5  the control warp turns the chunk's gates into per-token coefficients
//       with warp shuffles (division-free reverse scan).
//   A2  Z1 = [K;Q] W1_j^T        M=128 N=64  K=d   (keys and queries share W)
//       X1 = silu(Z1)            epilogue, fp16 to shared memory
//       Z2_j = X1 W2_j^T         M=128 N=d   K=64  (this CTA's partial sum)
//       all-reduce of Z2 over the cluster with bulk copies between the CTAs'
//       shared memories (the copy engine, mbarrier transaction counts, no
//       thread-level cluster fences): each CTA stages its partial as fp16 rows
//       and pushes rows [128/G p, 128/G (p+1)) to CTA p (reduce-scatter); CTA p
//       sums them in fp32, writes y for query rows and G2 = 2 (Z2 - V) for key
//       rows, and pushes its G2 rows to every CTA (all-gather) (A3). (Per-thread
//       asynchronous remote stores, st.async, measured slower here: 8.3 against
//       7.3 us per chunk.)
//   A4  G1 = (G2 W2_j) . silu'(Z1_K)        M=128(64 used) N=64 K=d
//   A6+A7 the fp32 state of this CTA's slice, [W | S], lives in TMEM for the
//       whole stream. Before the weight-update contractions of a chunk the
//       epilogue pre-scales it in place, W <- B W + c_S S, S <- A S (off the
//       critical path), and the contractions accumulate onto it:
//       [W2' | S2']   = [W2 | S2]   + G2^T [-c X1_K | -e X1_K]   M=d N=128 K=64
//       [W1' | S1']^T = [W1 | S1]^T + K^T  [-c G1   | -e G1]     M=d N=128 K=64
//       (c_i, e_i fold the momentum and forget gates of the chunk into the
//        operands), so the tensor core itself emits the updated state; the
//       epilogue only writes the fp16 copy of W' the next chunk multiplies with.
//   A8  the loop over chunks; TMA for chunk c+1 overlaps the write-back.
//       W_end / S_end are written once, after the last chunk.
//
// ("Titans, explained" steps 2-6; "Attack of the Titans", "Parallel training":
//  gradients at the chunk-start weights written as matrix products, decay
//  products folded per token.)
//
// Operand format: every contraction takes fp16 operands (10 mantissa bits)
// with fp32 accumulation. Keys and queries arrive as bf16 and are converted to
// fp16 once per call before this kernel; weights, activations, gradients and
// the exchanged partial sums are rounded to fp16. (With bf16's 7 mantissa bits
// the rounding of these operands, although unbiased, drifts the state along a
// near-symmetry of the depth-2 memory - W1 -> A W1, W2 -> W2 A^-1 for the
// nearly linear SiLU at small pre-activations - by several percent over
// thousands of chunks; fp16 cuts that drift eightfold at the same cost.)
//
// Warp roles: warps 0-15 epilogue (warp w reads TMEM lanes 32 (w % 4) .. +31
// and a quarter w / 4 of the slice's 64 hidden columns; warps 0-7 also stage
// and reduce the layer-2 exchange by column halves), warp 16 control (TMA,
// MMA issue by lane 0, scan).
// Every wait is bounded; on expiry the kernel records TM_ERR_TIMEOUT in the
// status word, drains its copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstring>

#include "tm_internal.h"
#include "tm_sm100.cuh"

namespace tmem {
namespace {

using namespace sm100;

constexpr int C = 64;           // chunk size of this kernel
constexpr int HS = 64;          // hidden units per CTA
constexpr int EPI_WARPS = 16;   // warp w: TMEM lanes 32 (w % 4) .., hidden columns quarter w / 4
constexpr int XCH_WARPS = 8;    // the first 8 stage and reduce the layer-2 exchange (column halves)
constexpr int NTHREADS = (EPI_WARPS + 1) * 32;
constexpr int XCH_THREADS = XCH_WARPS * 32;
constexpr int CPT = HS / (EPI_WARPS / 4);   // hidden columns of a slice per epilogue thread (16)
constexpr uint32_t TMEM_COLS = 512;

struct TcArgs {
  int T, P, G;
  int nchunks;                   // chunks per stream to process (T is the token stride)
  const __nv_bfloat16 *v;
  const float *theta, *eta, *alpha;
  const float *W0, *S0;
  float *y, *W, *S;
  int *status;
  unsigned long long wait_ns;
  int inject_timeout;
  // Exchange through global memory (streams whose cluster does not fit
  // beside the others): per stream, receive buffers and G2 rows, double
  // buffered by chunk parity, and monotonic arrival counters.
  unsigned char *xrecv;          // [stream][dest][parity][G x 2 x RP x d] fp16
  unsigned char *xg2;            // [stream][parity][64 x d] fp16, row-block layout
  unsigned *xflag;               // [stream][G + 1] counters, 128 bytes apart
};

// Exchange buffer sizes per stream (bytes) and counter stride (in unsigned).
constexpr int XFLAG_STRIDE = 32;
__host__ __device__ constexpr size_t xrecv_bytes(int D, int G) { return (size_t)G * 2 * (2 * 128 * D); }
__host__ __device__ constexpr size_t xg2_bytes(int D) { return (size_t)2 * 64 * D * 2; }
__host__ __device__ constexpr size_t xflag_bytes(int G) { return (size_t)(G + 1) * XFLAG_STRIDE * 4; }

// Per-chunk coefficients. sig is a power of two that the S part of the
// TMEM state carries for this chunk (S_tmem = sig S) and that the -e X1 and
// -e G1 operands are multiplied by: e_i = theta_i prod_{j>i} eta_j reaches
// 1e-6 for the first tokens of a chunk, and e_i x_i would otherwise fall among
// fp16's subnormals, whose coarse spacing biases the momentum update; sig puts
// theta_max sig in [8, 16).
struct Coefs {
  float c[C];
  float e[C];
  float Bw, As, cS, sig;
};

// The power of two 2^k with tmax 2^k in [8, 16), k clamped to [0, 40]; 1 when
// tmax is not positive.
__device__ __forceinline__ float chunk_scale(float tmax) {
  if (!(tmax > 0.f)) return 1.f;
  int ex;
  frexpf(tmax, &ex);                 // tmax = m 2^ex, m in [0.5, 1)
  int k = 4 - ex;
  k = k < 0 ? 0 : (k > 40 ? 40 : k);
  return ldexpf(1.f, k);
}

// Shared-memory map (bytes from a 1024-aligned base). Feature dims of the
// d-wide buffers are allocated as 128 even for d = 64 so that the padded
// M = 128 operands stay inside their own buffer.
template <int D>
struct Layout {
  static constexpr int FD = 128;
  static constexpr uint32_t W1 = 0;                          // W1_j^T [D x 64 hid] R=D
  static constexpr uint32_t W2 = W1 + D * 64 * 2;            // W2_j   [D x 64 hid] R=D
  static constexpr uint32_t XKQ = W2 + D * 64 * 2;           // [128 tok x FD]  R=128
  static constexpr uint32_t X1 = XKQ + 128 * FD * 2;         // [128 tok x 64]  R=128
  static constexpr uint32_t X1S = X1 + 128 * 64 * 2;         // [64 tok x 128]  R=64
  static constexpr uint32_t G2 = X1S + 64 * 128 * 2;         // [64 tok x FD]   R=64
  static constexpr uint32_t G1S = G2 + 64 * FD * 2;          // [64 tok x 128]  R=64
  static constexpr uint32_t SEND = G1S + 64 * 128 * 2;       // [128 x D] fp16 partial Z2
  static constexpr uint32_t RECV = SEND + 128 * D * 2;       // G x [128/G x D] fp16
  static constexpr uint32_t G2OWN = RECV + 128 * D * 2;      // owned rows of G2, RB atoms
  static constexpr uint32_t COEF = G2OWN + 64 * D * 2;       // 2 x Coefs
  static constexpr uint32_t BARS = COEF + 2 * sizeof(Coefs);
  static constexpr uint32_t NBARS = 16;
  static constexpr uint32_t MISC = BARS + NBARS * 8;         // tmem slot, abort flag
  static constexpr uint32_t TOTAL = MISC + 64;
};

enum Bar {
  B_TMA = 0, B_COEF, B_F1, B_X1, B_F2, B_QFREE, B_RECV, B_G2OWN, B_G2, B_B1, B_G1, B_U2, B_U1,
  B_UPD, B_FIN, B_NEVER, B_COUNT
};

// sigmoid(z) = 1/2 + tanh(z/2)/2, with the hardware tanh approximation (one
// MUFU operation; its error is far below the fp16 rounding of the results).
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigm(float z) { return fmaf(0.5f, tanh_approx(0.5f * z), 0.5f); }

// Two fp32 values as one fp16 pair (round to nearest even): the operand
// format of every tensor-core contraction here.
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint4 pack8(const float *v) {
  return make_uint4(pack_h2(v[0], v[1]), pack_h2(v[2], v[3]), pack_h2(v[4], v[5]),
                    pack_h2(v[6], v[7]));
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
// N (a multiple of 16) consecutive TMEM columns of this thread's lane.
template <int N>
__device__ __forceinline__ void tmem_ldn(uint32_t taddr, float (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N / 16; ++i) tmem_ld16(taddr + 16 * i, *reinterpret_cast<float(*)[16]>(&v[16 * i]));
}
template <int N>
__device__ __forceinline__ void tmem_stn(uint32_t taddr, const float (&v)[N]) {
#pragma unroll
  for (int i = 0; i < N / 16; ++i) tmem_st16(taddr + 16 * i, *reinterpret_cast<const float(*)[16]>(&v[16 * i]));
}
__device__ __forceinline__ void arrive_remote_release(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                   bar_cluster_addr)
               : "memory");
}
__device__ __forceinline__ bool try_wait_acquire_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Copy `bytes` from this CTA's shared memory into CTA-of-cluster shared memory
// (dst, bar are shared::cluster addresses); completion counts on the remote bar.
__device__ __forceinline__ void bulk_push(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "r"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// Global-memory exchange: bulk copy shared -> global, completion, proxy fence,
// release counter, acquire poll, bulk copy global -> shared.
__device__ __forceinline__ void bulk_store_global(void *gdst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_and_wait() {
  asm volatile("cp.async.bulk.commit_group;\n\tcp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void bulk_load_global(uint32_t dst, const void *gsrc, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(gsrc), "r"(bytes), "r"(bar)
      : "memory");
}
// One arrival per warp on a local barrier, after every lane's shared-memory
// writes have been made visible to the tensor cores (async proxy).
__device__ __forceinline__ void warp_arrive_local(uint64_t *bar, int lane) {
  fence_proxy_async_smem();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}
// Bounded wait that also gives up as soon as another thread of the CTA has
// flagged an abort. cluster_scope selects acquire.cluster semantics.
__device__ bool wait_bar(uint64_t *bar, uint32_t parity, const TcArgs &a, volatile int *abort_flag,
                         bool cluster_scope = false) {
  const uint32_t addr = smem_u32(bar);
  auto probe = [&]() {
    return cluster_scope ? try_wait_acquire_cluster(addr, parity) : mbar_try_wait(bar, parity);
  };
  if (probe()) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (probe()) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > a.wait_ns) {
      atomicCAS(a.status, 0, kDevTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}

// Bounded wait until a global arrival counter reaches target (acquire).
__device__ bool wait_flag(const unsigned *flag, unsigned target, const TcArgs &a, volatile int *abort_flag) {
  if ((int)(ld_acquire(flag) - target) >= 0) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if ((int)(ld_acquire(flag) - target) >= 0) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > a.wait_ns) {
      atomicCAS(a.status, 0, kDevTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}

// A5 with warp shuffles. Lane l holds tokens 2l and 2l+1 of the chunk.
//   pa_i = prod_{j>i} (1 - alpha_j), pe_i = prod_{j>i} eta_j,
//   r_i  = pa_i + eta_{i+1} r_{i+1}, r_{C-1} = 1   (an affine map per token,
//          composed from the right with an inclusive suffix scan),
//   c_i = theta_i r_i, e_i = theta_i pe_i,
//   Bw = prod (1 - alpha), As = prod eta, cS = eta_0 r_0.
__device__ void coef_scan_warp(Coefs &cf, const float *th, const float *et, const float *al,
                               int lane) {
  const int i0 = 2 * lane, i1 = 2 * lane + 1;
  const float t0 = th[i0], t1 = th[i1], e0 = et[i0], e1 = et[i1];
  const float f0 = 1.f - al[i0], f1 = 1.f - al[i1];
  // inclusive suffix products over lanes of the pair products
  float pf = f0 * f1, pe = e0 * e1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    float xf = __shfl_down_sync(0xffffffffu, pf, o);
    float xe = __shfl_down_sync(0xffffffffu, pe, o);
    if (lane + o < 32) { pf *= xf; pe *= xe; }
  }
  // exclusive suffix (products strictly after this lane's pair)
  float nf = __shfl_down_sync(0xffffffffu, pf, 1);
  float ne = __shfl_down_sync(0xffffffffu, pe, 1);
  if (lane == 31) { nf = 1.f; ne = 1.f; }
  const float pa1 = nf, pa0 = f1 * nf;   // pa for tokens i1 and i0
  const float pe1 = ne, pe0 = e1 * ne;
  // affine maps g_i(x) = pa_i + b_i x with b_i = eta_{i+1}; the last token's
  // map is the constant 1. Compose the pair (g_i0 o g_i1), then suffix-scan.
  const float eta_next = __shfl_down_sync(0xffffffffu, e0, 1);  // eta of token i1 + 1
  const float b1 = (lane == 31) ? 0.f : eta_next;
  const float a1 = (lane == 31) ? 1.f : pa1;
  const float a0 = pa0, b0 = e1;                // b_{i0} = eta_{i0 + 1} = eta_{i1}
  // pair = g_i0 o g_i1: (a0 + b0 a1, b0 b1)
  float A = a0 + b0 * a1, Bm = b0 * b1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    float xa = __shfl_down_sync(0xffffffffu, A, o);
    float xb = __shfl_down_sync(0xffffffffu, Bm, o);
    if (lane + o < 32) { A = A + Bm * xa; Bm = Bm * xb; }
  }
  // A now equals r_{i0} (the composition ends in a constant map)
  float An = __shfl_down_sync(0xffffffffu, A, 1);
  const float r0 = A;
  const float r1 = (lane == 31) ? 1.f : (a1 + b1 * An);
  cf.c[i0] = t0 * r0;
  cf.c[i1] = t1 * r1;
  cf.e[i0] = t0 * pe0;
  cf.e[i1] = t1 * pe1;
  float tmax = fmaxf(t0, t1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
  if (lane == 0) {
    cf.Bw = pa0 * f0;
    cf.As = pe0 * e0;
    cf.cS = e0 * r0;
    cf.sig = chunk_scale(tmax);
  }
}

// XG = false: the G CTAs of a stream form a cluster and exchange through
// each other's shared memory. XG = true: the same walker without a cluster,
// the exchange going through global memory (used for streams whose cluster
// does not fit beside the others; all G CTAs of a stream must be resident).
template <int D, int G, bool XG>
// 17 warps: registers are allocated for whole groups of four warps (20
// warps), so 96 registers a thread fill the SM's 64 K (one CTA per SM)
__global__ void __launch_bounds__(NTHREADS, 1)
    tc_chunk_kernel(const TcArgs a, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_q) {
  using Lay = Layout<D>;
  // Reduce-scatter of Z2 by rows: CTA p owns rows [RP p, RP (p + 1)) of the
  // 128 (keys 0-63, queries 64-127); owners of key rows produce G2 rows.
  constexpr int RP = 128 / G;                      // rows owned per CTA
  constexpr int RPK = RP < 64 ? RP : 64;           // key rows owned by a key owner
  constexpr int NQO = G >= 2 ? G / 2 : 0;          // owners of query rows only
  constexpr int NPT = RP * D / 8 / XCH_THREADS;    // 16-byte chunks reduced per exchange thread
  constexpr int SWZ = (D / 16 < 8 ? D / 16 : 8) - 1; // chunk swizzle mask of a half row
  static_assert(NPT >= 1 && RP * D / 8 % XCH_THREADS == 0, "reduce split");
  static_assert(CPT % 16 == 0, "epilogue column split");
  constexpr int NSIG = 2 * G * (RP >= 32 ? RP / 32 : 1);   // row pushes a CTA receives per chunk
  constexpr int NKO = RP >= C ? 1 : C / RP;                 // CTAs owning key rows
  constexpr uint32_t XDEST = 2 * 128 * D;                   // bytes of one receive buffer
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *sm =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(sm);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Lay::BARS);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + Lay::MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + Lay::MISC + 4);
  Coefs *coefs = reinterpret_cast<Coefs *>(sm + Lay::COEF);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const uint32_t j = XG ? (uint32_t)(blockIdx.x % G) : cluster_rank();
  const int stream = blockIdx.x / G;
  unsigned *const xfl = XG ? a.xflag + (size_t)stream * (G + 1) * XFLAG_STRIDE : nullptr;
  unsigned char *const xrv = XG ? a.xrecv + (size_t)stream * xrecv_bytes(D, G) : nullptr;
  unsigned char *const xg2 = XG ? a.xg2 + (size_t)stream * xg2_bytes(D) : nullptr;
  const int T = a.T, nchunks = a.nchunks, P = a.P;
  const int Hd = HS * G;             // hidden width
  float *Wg = a.W + (long long)stream * P;
  float *Sg = a.S + (long long)stream * P;
  const float *W0g = a.W0 + (long long)stream * P;
  const float *S0g = a.S0 + (long long)stream * P;
  const long long tok0 = (long long)stream * T;

  if (tid == 0) {
    mbar_init(&bars[B_TMA], 1);
    mbar_init(&bars[B_COEF], 32);
    mbar_init(&bars[B_F1], 1);
    mbar_init(&bars[B_X1], EPI_WARPS);
    mbar_init(&bars[B_F2], 1);
    mbar_init(&bars[B_RECV], 1);
    mbar_init(&bars[B_G2OWN], EPI_WARPS);
    mbar_init(&bars[B_G2], 1);
    mbar_init(&bars[B_QFREE], NQO > 0 ? NQO : 1);
    mbar_init(&bars[B_B1], 1);
    mbar_init(&bars[B_G1], EPI_WARPS);
    mbar_init(&bars[B_U2], 1);
    mbar_init(&bars[B_U1], 1);
    mbar_init(&bars[B_UPD], EPI_WARPS);
    mbar_init(&bars[B_FIN], 1);
    mbar_init(&bars[B_NEVER], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  // Zero the operand rows that padded M = 128 contractions read but never use,
  // so that they hold finite values: the second feature block of XKQ and G2
  // for d = 64.
  if (D < 128) {
    for (uint32_t off = tid * 16; off < 128 * 128 * 2; off += NTHREADS * 16)
      st_shared_v4(sbase + Lay::XKQ + off, make_uint4(0, 0, 0, 0));
    for (uint32_t off = tid * 16; off < 64 * 128 * 2; off += NTHREADS * 16)
      st_shared_v4(sbase + Lay::G2 + off, make_uint4(0, 0, 0, 0));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (!XG) {
    cluster_arrive_release();   // every CTA's barriers are initialised
    cluster_wait_acquire();
    // every CTA of this grid is resident: a kernel launched after this one
    // with programmatic serialization (the global-exchange walker for the
    // streams that did not fit) may take the SMs left free
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  const uint32_t tm = *tmem_slot;
  const uint32_t t_z1 = tm + 0, t_z2 = tm + 64, t_g1 = tm + 192, t_s2 = tm + 256, t_s1 = tm + 384;

  if (warp < EPI_WARPS) {
    // ---------------------------------------------------------------- epilogue warps
    const int q = warp & 3, h = warp >> 2;
    const int row = 32 * q + lane;                     // TMEM lane of this thread
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    // TMEM-resident state: lane d, columns [W | S] of the slice; this thread
    // holds hidden units CPT h .. CPT h + CPT - 1 of row d.
    //   t_s2: W2[d][64 j + n] (n < 64), S2 at n + 64
    //   t_s1: W1[64 j + n][d] (n < 64), S1 at n + 64
    if (row < D) {
      float w[CPT], sv[CPT];
      const long long g2 = (long long)Hd * D + (long long)row * Hd + HS * j + CPT * h;
#pragma unroll
      for (int i4 = 0; i4 < CPT / 4; ++i4) {
        const float4 a4 = *reinterpret_cast<const float4 *>(W0g + g2 + 4 * i4);
        const float4 b4 = *reinterpret_cast<const float4 *>(S0g + g2 + 4 * i4);
        w[4 * i4] = a4.x; w[4 * i4 + 1] = a4.y; w[4 * i4 + 2] = a4.z; w[4 * i4 + 3] = a4.w;
        sv[4 * i4] = b4.x; sv[4 * i4 + 1] = b4.y; sv[4 * i4 + 2] = b4.z; sv[4 * i4 + 3] = b4.w;
      }
      tmem_stn(t_s2 + lane_base + CPT * h, w);
      tmem_stn(t_s2 + lane_base + 64 + CPT * h, sv);
#pragma unroll
      for (int k8 = 0; k8 < CPT / 8; ++k8)
        st_shared_v4(sbase + Lay::W2 + rb_chunk(D, row, (CPT / 8) * h + k8), pack8(&w[8 * k8]));
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const long long g1 = (long long)(HS * j + CPT * h + i) * D + row;
        w[i] = W0g[g1];
        sv[i] = S0g[g1];
      }
      tmem_stn(t_s1 + lane_base + CPT * h, w);
      tmem_stn(t_s1 + lane_base + 64 + CPT * h, sv);
#pragma unroll
      for (int k8 = 0; k8 < CPT / 8; ++k8)
        st_shared_v4(sbase + Lay::W1 + rb_chunk(D, row, (CPT / 8) * h + k8), pack8(&w[8 * k8]));
      tmem_wait_st();
    }
    warp_arrive_local(&bars[B_UPD], lane);
    float sig_prev = 1.f;                              // S_tmem = sig_prev S (S0 loaded as is)

    for (int cch = 0; cch < nchunks; ++cch) {
      const uint32_t par = cch & 1;
      const long long tb = tok0 + (long long)cch * C;
      // Load the values V this thread needs in the reduce step now, so the
      // loads have the whole forward pass to land.
      uint4 vv[NPT];
#pragma unroll
      for (int i = 0; i < NPT; ++i) {
        const int k = tid + i * XCH_THREADS, gr = (int)j * RP + k / (D / 8), c = k % (D / 8);
        if (tid < XCH_THREADS && gr < C) vv[i] = *reinterpret_cast<const uint4 *>(a.v + (tb + gr) * D + 8 * c);
      }
      if (!wait_bar(&bars[B_COEF], par, a, abort_flag)) break;
      const Coefs &cf = coefs[par];
      // -------- A7, first half: W <- B W + c_S S, S <- A S in TMEM. Runs while
      // F1 executes; the accumulating contractions later add the writes. S
      // moves from the previous chunk's scale to this chunk's (exact: powers of
      // two).
      const float sig = cf.sig, inv_prev = 1.f / sig_prev;
      const float cS_t = cf.cS * inv_prev, As_t = cf.As * (sig * inv_prev);
      sig_prev = sig;
      if (row < D) {
#pragma unroll
        for (int layer = 0; layer < 2; ++layer) {
          const uint32_t ts = (layer ? t_s1 : t_s2) + lane_base + CPT * h;
          float w[CPT], sv[CPT];
          tmem_ldn(ts, w);
          tmem_ldn(ts + 64, sv);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < CPT; ++i) {
            w[i] = cf.Bw * w[i] + cS_t * sv[i];
            sv[i] = As_t * sv[i];
          }
          tmem_stn(ts, w);
          tmem_stn(ts + 64, sv);
        }
        tmem_wait_st();
      }
      // -------- E1: X1 = silu(Z1); key rows also give -c X1 and -e X1
      if (!wait_bar(&bars[B_F1], par, a, abort_flag)) break;
      tc_fence_after();
      {
        float z[CPT];
        tmem_ldn(t_z1 + lane_base + CPT * h, z);
        tmem_wait_ld();
        float x[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) x[i] = z[i] * sigm(z[i]);
#pragma unroll
        for (int k8 = 0; k8 < CPT / 8; ++k8)
          st_shared_v4(sbase + Lay::X1 + rb_chunk(128, row, (CPT / 8) * h + k8), pack8(&x[8 * k8]));
        // X1 feeds the next MMA: publish it first
        warp_arrive_local(&bars[B_X1], lane);
        // the scaled copies are only needed by the W2 update, much later (they
        // reach the tensor cores through the fence of the B_G2OWN arrival)
        if (row < C) {
          const float ci = -cf.c[row], ei = -cf.e[row] * sig;
          float s8[8];
#pragma unroll
          for (int k8 = 0; k8 < CPT / 8; ++k8) {
#pragma unroll
            for (int i = 0; i < 8; ++i) s8[i] = ci * x[8 * k8 + i];
            st_shared_v4(sbase + Lay::X1S + rb_chunk(64, row, (CPT / 8) * h + k8), pack8(s8));
#pragma unroll
            for (int i = 0; i < 8; ++i) s8[i] = ei * x[8 * k8 + i];
            st_shared_v4(sbase + Lay::X1S + rb_chunk(64, row, 8 + (CPT / 8) * h + k8), pack8(s8));
          }
        }
      }
      // -------- E2: stage this CTA's partial Z2 as fp16, [half][row][d/2]
      // (16-byte chunk index XOR row), and let each warp bulk-copy the rows it
      // staged into their owners' receive buffers (reduce-scatter by rows:
      // CTA p owns rows [RP p, RP p + RP)).
      if (!wait_bar(&bars[B_F2], par, a, abort_flag)) break;
      tc_fence_after();
      // Query rows (warps of lane quarters 2, 3) reuse send and receive space
      // that the query owners read in the previous chunk: wait for their
      // release (normally long given). Key rows need no such wait: the key
      // owners' G2 of the previous chunk already proved it.
      // (The global exchange double-buffers by chunk parity instead: a peer
      // writes chunk c+2 only after this CTA's push of chunk c+1, which
      // follows its reads of chunk c.)
      // Only the first XCH_WARPS warps (column halves h = 0, 1) stage and push.
      if (!XG && NQO > 0 && warp < XCH_WARPS && q >= 2 && cch > 0 &&
          !wait_bar(&bars[B_QFREE], (uint32_t)((cch - 1) & 1), a, abort_flag, true))
        break;
      if (warp < XCH_WARPS) {
        constexpr int HALF = D / 2;                    // columns of Z2 per thread
        const uint32_t srow = sbase + Lay::SEND + (uint32_t)(h * 128 * D + row * D);
#pragma unroll
        for (int c16 = 0; c16 < HALF / 16; ++c16) {
          float z[16];
          tmem_ld16(t_z2 + lane_base + HALF * h + 16 * c16, z);
          tmem_wait_ld();
#pragma unroll
          for (int k8 = 0; k8 < 2; ++k8)
            st_shared_v4(srow + (uint32_t)(((2 * c16 + k8) ^ (row & SWZ)) << 4), pack8(&z[8 * k8]));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          constexpr int RPP = RP < 32 ? RP : 32;       // rows per push
#pragma unroll
          for (int i = 0; i < 32 / RPP; ++i) {
            const int r0 = 32 * q + i * RPP, p = r0 / RP, rin = r0 - p * RP;
            const uint32_t off = (uint32_t)(j * 2 * RP * D + h * RP * D + rin * D);
            const uint32_t src = sbase + Lay::SEND + (uint32_t)(h * 128 * D + r0 * D);
            if constexpr (XG)
              bulk_store_global(xrv + (size_t)(p * 2 + (int)par) * XDEST + off, src, (uint32_t)(RPP * D));
            else
              bulk_push(mapa(sbase + Lay::RECV + off, (uint32_t)p), src, (uint32_t)(RPP * D),
                        mapa(smem_u32(&bars[B_RECV]), (uint32_t)p));
          }
          if constexpr (XG) {
            // the rows are in global memory before the owners are told
            bulk_commit_and_wait();
            fence_proxy_async_global();
#pragma unroll
            for (int i = 0; i < 32 / RPP; ++i) red_release_add(xfl + ((32 * q + i * RPP) / RP) * XFLAG_STRIDE, 1u);
          }
        }
        __syncwarp();
      }
      // -------- reduce my rows over the G partials (fp32 sums, fixed order):
      // y for query rows, G2 = 2 (Z2 - V) for key rows (A3)
      if (XG ? !wait_flag(xfl + j * XFLAG_STRIDE, (unsigned)(NSIG * (cch + 1)), a, abort_flag)
             : !wait_bar(&bars[B_RECV], par, a, abort_flag))
        break;
      {
        float acc[NPT][8];
#pragma unroll
        for (int i = 0; i < NPT; ++i) {
          if (tid >= XCH_THREADS) break;
          const int k = tid + i * XCH_THREADS, r = k / (D / 8), c = k % (D / 8);
          uint4 pv[G];
#pragma unroll
          for (int s2 = 0; s2 < G; ++s2) {
            const uint32_t off = (uint32_t)(s2 * 2 * RP * D + (c / (D / 16)) * RP * D + r * D +
                                            (((c % (D / 16)) ^ (r & SWZ)) << 4));
            if constexpr (XG)
              pv[s2] = __ldcg(reinterpret_cast<const uint4 *>(xrv + (size_t)(j * 2 + par) * XDEST + off));
            else
              pv[s2] = *reinterpret_cast<const uint4 *>(sm + Lay::RECV + off);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
#pragma unroll
          for (int s2 = 0; s2 < G; ++s2) {
            const __half *pb = reinterpret_cast<const __half *>(&pv[s2]);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[i][e] += __half2float(pb[e]);
          }
          const int gr = (int)j * RP + r;
          if (gr < C) {
            const __nv_bfloat16 *vb = reinterpret_cast<const __nv_bfloat16 *>(&vv[i]);
            float g[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) g[e] = 2.f * (acc[i][e] - __bfloat162float(vb[e]));
            st_shared_v4(sbase + Lay::G2OWN + rb_chunk(RPK, r, c), pack8(g));
          }
        }
        warp_arrive_local(&bars[B_G2OWN], lane);
        // reads y of my query rows
#pragma unroll
        for (int i = 0; i < NPT; ++i) {
          if (tid >= XCH_THREADS) break;
          const int k = tid + i * XCH_THREADS, r = k / (D / 8), c = k % (D / 8);
          const int gr = (int)j * RP + r;
          if (gr >= C) {
            float *yp = a.y + (tb + (gr - C)) * D + 8 * c;
            *reinterpret_cast<float4 *>(yp) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
            *reinterpret_cast<float4 *>(yp + 4) = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
          }
        }
      }
      // -------- E3: G1 = (G2 W2_j) . silu'(Z1) on key rows -> [-c G1 | -e G1]
      if (!wait_bar(&bars[B_B1], par, a, abort_flag)) break;
      tc_fence_after();
      if (row < C) {
        float gp[CPT], z[CPT];
        tmem_ldn(t_g1 + lane_base + CPT * h, gp);
        tmem_ldn(t_z1 + lane_base + CPT * h, z);
        tmem_wait_ld();
        const float ci = -cf.c[row], ei = -cf.e[row] * sig;
        float g1[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
          const float s = sigm(z[i]);
          g1[i] = gp[i] * (s * (1.f + z[i] * (1.f - s)));
        }
        float s8[8];
#pragma unroll
        for (int k8 = 0; k8 < CPT / 8; ++k8) {
#pragma unroll
          for (int i = 0; i < 8; ++i) s8[i] = ci * g1[8 * k8 + i];
          st_shared_v4(sbase + Lay::G1S + rb_chunk(64, row, (CPT / 8) * h + k8), pack8(s8));
#pragma unroll
          for (int i = 0; i < 8; ++i) s8[i] = ei * g1[8 * k8 + i];
          st_shared_v4(sbase + Lay::G1S + rb_chunk(64, row, 8 + (CPT / 8) * h + k8), pack8(s8));
        }
      }
      warp_arrive_local(&bars[B_G1], lane);
      // -------- A7, second half: the fp16 copies of W2' and W1' for the next chunk
      if (!wait_bar(&bars[B_U2], par, a, abort_flag)) break;
      tc_fence_after();
      if (row < D) {
        float w[CPT];
        tmem_ldn(t_s2 + lane_base + CPT * h, w);
        tmem_wait_ld();
#pragma unroll
        for (int k8 = 0; k8 < CPT / 8; ++k8)
          st_shared_v4(sbase + Lay::W2 + rb_chunk(D, row, (CPT / 8) * h + k8), pack8(&w[8 * k8]));
      }
      if (!wait_bar(&bars[B_U1], par, a, abort_flag)) break;
      tc_fence_after();
      if (row < D) {
        float w[CPT];
        tmem_ldn(t_s1 + lane_base + CPT * h, w);
        tmem_wait_ld();
#pragma unroll
        for (int k8 = 0; k8 < CPT / 8; ++k8)
          st_shared_v4(sbase + Lay::W1 + rb_chunk(D, row, (CPT / 8) * h + k8), pack8(&w[8 * k8]));
      }
      warp_arrive_local(&bars[B_UPD], lane);
    }
    // -------- W_end, S_end: write the TMEM-resident state back once
    if (!*abort_flag && row < D) {
      tc_fence_after();
      float w[CPT], sv[CPT];
      const float inv_sig = 1.f / sig_prev;            // S_tmem = sig S of the last chunk
      {
        const uint32_t ts = t_s2 + lane_base + CPT * h;
        tmem_ldn(ts, w);
        tmem_ldn(ts + 64, sv);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < CPT; ++i) sv[i] *= inv_sig;
        const long long g2 = (long long)Hd * D + (long long)row * Hd + HS * j + CPT * h;
#pragma unroll
        for (int i4 = 0; i4 < CPT / 4; ++i4) {
          *reinterpret_cast<float4 *>(Wg + g2 + 4 * i4) = make_float4(w[4 * i4], w[4 * i4 + 1], w[4 * i4 + 2], w[4 * i4 + 3]);
          *reinterpret_cast<float4 *>(Sg + g2 + 4 * i4) = make_float4(sv[4 * i4], sv[4 * i4 + 1], sv[4 * i4 + 2], sv[4 * i4 + 3]);
        }
      }
      {
        const uint32_t ts = t_s1 + lane_base + CPT * h;
        tmem_ldn(ts, w);
        tmem_ldn(ts + 64, sv);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
          sv[i] *= inv_sig;
          const long long g1 = (long long)(HS * j + CPT * h + i) * D + row;
          Wg[g1] = w[i];
          Sg[g1] = sv[i];
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- control warp
    const uint32_t i_f1 = idesc_f16(128, 64, false, true);
    const uint32_t i_f2 = idesc_f16(128, D, false, false);
    const uint32_t i_b1 = idesc_f16(128, 64, false, true);
    const uint32_t i_dw = idesc_f16(128, 128, true, true);
    const uint32_t xkq = sbase + Lay::XKQ, x1 = sbase + Lay::X1, x1s = sbase + Lay::X1S;
    const uint32_t g2 = sbase + Lay::G2, g1s = sbase + Lay::G1S;
    const uint32_t w1 = sbase + Lay::W1, w2 = sbase + Lay::W2;
    constexpr uint32_t TILE_BYTES = 2u * C * D * 2u;
    auto issue_tma = [&](int cch) {
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars[B_TMA], TILE_BYTES);
        const int y0 = (int)(tok0 + (long long)cch * C);
#pragma unroll
        for (int fb = 0; fb < D / 64; ++fb) {
          tma_load_2d(sm + Lay::XKQ + fb * 128 * 128, &map_k, &bars[B_TMA], 64 * fb, y0);
          tma_load_2d(sm + Lay::XKQ + fb * 128 * 128 + 64 * 128, &map_q, &bars[B_TMA], 64 * fb, y0);
        }
      }
      __syncwarp();
    };
    auto scan = [&](int cch) {
      const long long tb = tok0 + (long long)cch * C;
      coef_scan_warp(coefs[cch & 1], a.theta + tb, a.eta + tb, a.alpha + tb, lane);
      __syncwarp();
      mbar_arrive(&bars[B_COEF]);
    };
    if (lane == 0) { prefetch_tmap(&map_k); prefetch_tmap(&map_q); }
    int tma_inflight = 0;
    issue_tma(0);
    tma_inflight = 1;
    scan(0);
    int cch = 0;
    for (; cch < nchunks; ++cch) {
      const uint32_t par = cch & 1;
      if (a.inject_timeout) {
        // Test hook: wait on a barrier nothing ever completes.
        if (!wait_bar(&bars[B_NEVER], 0, a, abort_flag)) break;
      }
      if (!wait_bar(&bars[B_TMA], par, a, abort_flag)) break;
      tma_inflight = 0;
      if (!wait_bar(&bars[B_UPD], par, a, abort_flag)) break;
      tc_fence_after();
      // this chunk's incoming bytes: G partial blocks, and all 64 rows of G2
      if (lane == 0) {
        if (!XG) mbar_arrive_expect_tx(&bars[B_RECV], (uint32_t)(G * RP * D * 2));
        mbar_arrive_expect_tx(&bars[B_G2], (uint32_t)(C * D * 2));
      }
      __syncwarp();
      // A2 first half: Z1 = [K;Q] W1_j^T
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          umma_f16(t_z1, desc_kmajor(xkq, 128, ks), desc_mnmajor(w1, D, ks), i_f1, ks > 0);
        umma_commit(&bars[B_F1]);
      }
      __syncwarp();
      if (!wait_bar(&bars[B_X1], par, a, abort_flag)) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < HS / 16; ++ks)
          umma_f16(t_z2, desc_kmajor(x1, 128, ks), desc_kmajor(w2, D, ks), i_f2, ks > 0);
        umma_commit(&bars[B_F2]);
      }
      __syncwarp();
      // Coefficients of the next chunk while F2 and the all-reduce run. Only
      // after B_X1: the epilogue has then consumed this chunk's B_COEF phase,
      // so B_COEF can never run two phases ahead of its waiters.
      if (cch + 1 < nchunks) scan(cch + 1);
      // all-gather of G2: key owners push their rows (whole 1 KB swizzle
      // atoms) to every CTA; query owners report that they are done reading
      // their receive buffer (B_QFREE, off the critical path).
      if (!wait_bar(&bars[B_G2OWN], par, a, abort_flag)) break;
      if (lane == 0) {
        if ((int)j * RP < C && XG) {
          // G2 rows to global memory, then one arrival for every reader
#pragma unroll
          for (int fb = 0; fb < D / 64; ++fb)
            bulk_store_global(xg2 + (size_t)par * (64 * D * 2) + fb * 64 * 128 + j * (uint32_t)(RP * 128),
                              sbase + Lay::G2OWN + (uint32_t)(fb * RPK * 128), (uint32_t)(RPK * 128));
          bulk_commit_and_wait();
          fence_proxy_async_global();
          red_release_add(xfl + G * XFLAG_STRIDE, 1u);
        } else if ((int)j * RP < C) {
#pragma unroll
          for (int i = 0; i < G; ++i) {
            const uint32_t p = (j + (uint32_t)i) % G;
#pragma unroll
            for (int fb = 0; fb < D / 64; ++fb)
              bulk_push(mapa(sbase + Lay::G2 + (uint32_t)(fb * 64 * 128) + j * (uint32_t)(RP * 128), p),
                        sbase + Lay::G2OWN + (uint32_t)(fb * RPK * 128), (uint32_t)(RPK * 128),
                        mapa(smem_u32(&bars[B_G2]), p));
          }
        } else if (!XG) {
          // done reading this chunk's receive buffer: query rows of the next
          // chunk may be pushed here
#pragma unroll
          for (int i = 0; i < G; ++i)
            arrive_remote_release(mapa(smem_u32(&bars[B_QFREE]), (j + (uint32_t)i) % G));
        }
      }
      __syncwarp();
      if constexpr (XG) {
        // every key owner's rows of this chunk are out: copy G2 in
        int ok = 1;
        if (lane == 0) {
          ok = wait_flag(xfl + G * XFLAG_STRIDE, (unsigned)(NKO * (cch + 1)), a, abort_flag) ? 1 : 0;
          if (ok) {
            fence_proxy_async_global();
            bulk_load_global(g2, xg2 + (size_t)par * (64 * D * 2), (uint32_t)(C * D * 2), smem_u32(&bars[B_G2]));
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      }
      // G2 complete in this CTA's shared memory
      if (!wait_bar(&bars[B_G2], par, a, abort_flag, !XG)) break;
      tc_fence_after();
      if (lane == 0) {
        // A4: G1 pre-activation gradient = G2 W2_j
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          umma_f16(t_g1, desc_kmajor(g2, 64, ks), desc_mnmajor(w2, D, ks), i_b1, ks > 0);
        umma_commit(&bars[B_B1]);
        // A6+A7 for W2: [W2 | S2] += G2^T [-c X1_K | -e X1_K] onto the pre-scaled state
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          umma_f16(t_s2, desc_mnmajor(g2, 64, ks), desc_mnmajor(x1s, 64, ks), i_dw, 1);
        umma_commit(&bars[B_U2]);
      }
      __syncwarp();
      if (!wait_bar(&bars[B_G1], par, a, abort_flag)) break;
      tc_fence_after();
      if (lane == 0) {
        // A6+A7 for W1: [W1 | S1]^T += K^T [-c G1 | -e G1] onto the pre-scaled state
#pragma unroll
        for (int ks = 0; ks < C / 16; ++ks)
          umma_f16(t_s1, desc_mnmajor(xkq, 128, ks), desc_mnmajor(g1s, 64, ks), i_dw, 1);
        umma_commit(&bars[B_U1]);
      }
      __syncwarp();
      // the key/query tile is free once U1 is done: prefetch the next chunk
      if (!wait_bar(&bars[B_U1], par, a, abort_flag)) break;
      if (cch + 1 < nchunks) {
        issue_tma(cch + 1);
        tma_inflight = 1;
      }
    }
    // Drain: no copy or MMA may be in flight when the CTA leaves. These waits
    // ignore the abort flag but stay bounded in time.
    if (tma_inflight && !mbar_wait(&bars[B_TMA], (uint32_t)(cch & 1), a.wait_ns))
      atomicCAS(a.status, 0, kDevTimeout);
    if (lane == 0) umma_commit(&bars[B_FIN]);
    __syncwarp();
    if (!mbar_wait(&bars[B_FIN], 0, a.wait_ns)) atomicCAS(a.status, 0, kDevTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (!XG) {
    // no CTA leaves while a peer may still write into its shared memory
    cluster_arrive_release();
    cluster_wait_acquire();
  }
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, TMEM_COLS);
  // launched behind the cluster walker: do not complete before it, so that
  // later work in the stream sees both done
  if constexpr (XG) asm volatile("griddepcontrol.wait;" ::: "memory");
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D map over [rows x d] fp16 tokens (the converted keys or queries), box =
// 64 features x 64 tokens, 128B swizzle.
bool make_token_map(CUtensorMap *map, const void *base, long long rows, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  std::memset(map, 0, sizeof *map);
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)C};
  cuuint32_t es[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int cluster_size(const Problem &p) { return p.dims[1] / HS; }

template <int D, int G, bool XG>
cudaError_t launch_dg(int streams, cudaStream_t stream, const TcArgs &a, const CUtensorMap &mk,
                      const CUtensorMap &mq, bool after_primary) {
  using Lay = Layout<D>;
  const size_t smem = Lay::TOTAL + 1024;
  auto kern = tc_chunk_kernel<D, G, XG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(streams * G));
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  if (!XG) {
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = G;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
  } else if (after_primary) {
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, a, mk, mq);
}

template <int D, int G>
int max_clusters_dg() {
  using Lay = Layout<D>;
  const size_t smem = Lay::TOTAL + 1024;
  auto kern = tc_chunk_kernel<D, G, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(G * 64));
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = G;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// Clusters of this shape that can be resident at once (0 if unknown), and
// the SM count; both cached per process.
int max_clusters(int d, int G) {
  static int cache[2][9] = {};
  static bool done[2][9] = {};
  const int di = d == 64 ? 0 : 1;
  if (!done[di][G]) {
    int n = 0;
    switch (G) {
      case 1: n = d == 64 ? max_clusters_dg<64, 1>() : max_clusters_dg<128, 1>(); break;
      case 2: n = d == 64 ? max_clusters_dg<64, 2>() : max_clusters_dg<128, 2>(); break;
      case 4: n = d == 64 ? max_clusters_dg<64, 4>() : max_clusters_dg<128, 4>(); break;
      case 8: n = max_clusters_dg<128, 8>(); break;
    }
    cache[di][G] = n;
    done[di][G] = true;
  }
  return cache[di][G];
}

int sm_count() {
  static int n = -1;
  if (n < 0) {
    int dev = 0;
    n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
  }
  return n;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// Streams run by the global-exchange walker: with `all`, every stream (when
// all CTAs fit on the SMs at once); otherwise the streams beyond the
// clusters that fit, when their CTAs fit on the SMs those clusters leave.
int global_streams(const Problem &p, bool all) {
  const int G = cluster_size(p), sms = sm_count();
  if (all) return (sms > 0 && p.streams * G <= sms) ? p.streams : -1;
  const int mx = max_clusters(p.dims[0], G);
  if (mx <= 0 || p.streams <= mx) return 0;
  const int rest = p.streams - mx;
  return rest * G <= sms - mx * G ? rest : 0;
}

size_t exchange_bytes(int d, int G, int nx) {
  if (nx <= 0) return 0;
  return up256((size_t)nx * xflag_bytes(G)) + up256((size_t)nx * xg2_bytes(d)) +
         up256((size_t)nx * xrecv_bytes(d, G));
}

}  // namespace

bool tc_supported(const Problem &p) {
  if (p.in_dtype != TM_BF16 || p.L != 2 || p.C != C) return false;
  const int d = p.dims[0], h = p.dims[1];
  if (d != 64 && d != 128) return false;
  if (h % HS != 0) return false;
  const int G = h / HS;
  const bool shape = d == 64 ? (G == 1 || G == 2 || G == 4) : (G == 1 || G == 2 || G == 4 || G == 8);
  if (!shape) return false;
  return !p.tc_global || global_streams(p, true) >= 0;
}

int tc_launch_count(const Problem &p) {
  const int nx = global_streams(p, p.tc_global != 0);
  if (nx < 0) return 0;
  return (p.streams - nx > 0 ? 1 : 0) + (nx > 0 ? 1 : 0);
}

size_t tc_scratch_bytes(const Problem &p) {
  const int nx = global_streams(p, p.tc_global != 0);
  return exchange_bytes(p.dims[0], cluster_size(p), nx);
}

static unsigned long long g_wait_ns = 2000000000ull;  // 2 s per wait
static int g_inject_timeout = 0;

void tc_set_debug(int inject_timeout, unsigned long long wait_ns) {
  g_inject_timeout = inject_timeout;
  g_wait_ns = wait_ns ? wait_ns : 2000000000ull;
}

namespace {

template <int D, int G>
cudaError_t launch_both(const Problem &p, cudaStream_t stream, int nc, int nx, unsigned char *xbuf) {
  const size_t td = (size_t)p.T * D;
  TcArgs base;
  std::memset(&base, 0, sizeof base);
  base.T = p.T;
  base.nchunks = p.T_run / C;
  base.P = (int)p.P;
  base.G = G;
  base.status = p.status;
  base.wait_ns = g_wait_ns;
  base.inject_timeout = g_inject_timeout;
  // streams [s0, s0 + n) of the problem
  auto run = [&](int s0, int n, bool xg, bool after) -> cudaError_t {
    CUtensorMap mk, mq;
    const __half *k = static_cast<const __half *>(p.k16) + (size_t)s0 * td;
    const __half *q = static_cast<const __half *>(p.q16) + (size_t)s0 * td;
    if (!make_token_map(&mk, k, (long long)n * p.T, D) || !make_token_map(&mq, q, (long long)n * p.T, D))
      return cudaErrorInvalidValue;
    TcArgs a = base;
    a.v = static_cast<const __nv_bfloat16 *>(p.v) + (size_t)s0 * td;
    a.theta = p.theta + (size_t)s0 * p.T;
    a.eta = p.eta + (size_t)s0 * p.T;
    a.alpha = p.alpha + (size_t)s0 * p.T;
    a.W0 = p.W0 + (size_t)s0 * p.P;
    a.S0 = p.S0 + (size_t)s0 * p.P;
    a.y = p.y + (size_t)s0 * td;
    a.W = p.W_end + (size_t)s0 * p.P;
    a.S = p.S_end + (size_t)s0 * p.P;
    if (!xg) return launch_dg<D, G, false>(n, stream, a, mk, mq, false);
    a.xflag = reinterpret_cast<unsigned *>(xbuf);
    a.xg2 = xbuf + up256((size_t)n * xflag_bytes(G));
    a.xrecv = a.xg2 + up256((size_t)n * xg2_bytes(D));
    return launch_dg<D, G, true>(n, stream, a, mk, mq, after);
  };
  cudaError_t e = cudaSuccess;
  if (nx > 0) {
    e = cudaMemsetAsync(xbuf, 0, (size_t)nx * xflag_bytes(G), stream);
    if (e != cudaSuccess) return e;
  }
  if (nc > 0) e = run(0, nc, false, false);
  if (e == cudaSuccess && nx > 0) e = run(nc, nx, true, nc > 0);
  return e;
}

}  // namespace

cudaError_t tc_launch(const Problem &p, cudaStream_t stream) {
  if (!tc_supported(p)) return cudaErrorNotSupported;
  const int G = cluster_size(p), d = p.dims[0];
  const int nx = global_streams(p, p.tc_global != 0);
  if (nx < 0) return cudaErrorNotSupported;
  const int nc = p.streams - nx;
  unsigned char *xbuf = static_cast<unsigned char *>(p.scratch);
  if (nx > 0 && (!xbuf || p.scratch_bytes < exchange_bytes(d, G, nx))) return cudaErrorInvalidValue;
  switch (G) {
    case 1: return d == 64 ? launch_both<64, 1>(p, stream, nc, nx, xbuf) : launch_both<128, 1>(p, stream, nc, nx, xbuf);
    case 2: return d == 64 ? launch_both<64, 2>(p, stream, nc, nx, xbuf) : launch_both<128, 2>(p, stream, nc, nx, xbuf);
    case 4: return d == 64 ? launch_both<64, 4>(p, stream, nc, nx, xbuf) : launch_both<128, 4>(p, stream, nc, nx, xbuf);
    case 8: return launch_both<128, 8>(p, stream, nc, nx, xbuf);
  }
  return cudaErrorNotSupported;
}

}  // namespace tmem
