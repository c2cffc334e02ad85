// Layer-by-layer tensor-core path: the chunk recurrence as a sequence of
// batched tcgen05 GEMMs with fused epilogues, one launch per phase.
//
// For memories whose per-stream state cannot stay on chip (wide heads, deep
// memories with many streams), every chunk of every stream runs as:
//   forward    l = 1..L  Z_l = X_{l-1} W_l^T over the chunk's [keys; queries]
//              (epilogue: X_l = silu(Z_l) and silu'(Z_l) for key rows; for the
//               last layer y for query rows and G_L = 2 (Z_L - V) for key rows)
//   backward   l = L..2  G_{l-1} = (G_l W_l) . silu'(Z_{l-1})
//   update     l = 1..L  [U_W | U_S] = [-c G_l | -e G_l]^T X_{l-1}, epilogue
//              W' = B W + c_S S + U_W, S' = A S + U_S (fp32 state in the
//              caller's W_end / S_end) and the fp16 copy of W' for the next chunk
// ("Titans, explained" steps 2-6; "Attack of the Titans", "Parallel
//  training"). Launch order on one stream orders the phases. For widths up to
// 256 one fused kernel runs a tile's whole forward and backward; wider layers
// run one launch per phase (one output tile per CTA: TMA loads with the
// 128-byte swizzle into a ring of shared-memory stages, tcgen05 MMAs into
// TMEM, an epilogue from TMEM); one launch updates every layer. Each stream's
// tiles are independent (batched over streams).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdlib>
#include <cstring>
#include <vector>

#include "tm_internal.h"
#include "tm_sm100.cuh"

namespace tmem {
namespace {

using namespace sm100;

// Operand format of every contraction: fp16 (10 mantissa bits), fp32
// accumulation. The keys and queries arrive as bf16 and are converted to fp16
// once per call; the weight copies, activations, silu' and gradients the
// kernels exchange are fp16. Values stay bf16 (read by the epilogues only).
using op_t = __half;

constexpr int NT = 256;          // 8 warps: warp w reads TMEM lanes 32 (w % 4) .. +31,
                                 // columns half w / 4 of the tile
constexpr int KB = 64;           // K block (one 128-byte swizzle atom of 2-byte elements)
constexpr int kMaxSplit = 4;     // CTAs per output tile sharing a per-phase GEMM's reduction

enum Kind { K_FWD = 0, K_FWD_LAST = 1, K_BWD = 2 };

struct GemmArgs {
  int kind;
  int C, T, chunk;               // chunk size, tokens per stream, chunk index
  int M, N, K;                   // per-stream GEMM: rows, cols, reduction
  int streams, ksplit;           // grid z = streams x ksplit: K is split over ksplit CTAs per tile
  float *part;                   // [tiles, ksplit, 128, N] fp32 partial tiles (ksplit > 1)
  unsigned *cnt;                 // [tiles] arrivals per tile; the last CTA resets it to 0
  int n_out;                     // row length of the epilogue's outputs
  int a_rows_per_stream;         // rows of the A source per stream
  int b_rows_per_stream;
  int a_split_kq;                // layer-1 forward: rows < C from k, else from q
  // epilogue operands
  op_t *x_out;                   // [streams, 2C, n] activations (forward)
  op_t *sp_out;                  // [streams, C, n] silu'(Z) of key rows (forward)
  const op_t *sp_in;             // [streams, C, n] silu' of the layer below (backward)
  op_t *g_out, *gc_out, *ge_out; // [streams, C, n] G, -c G, -e G
  float *y;                      // [streams, T, d] reads (last forward)
  const __nv_bfloat16 *v;        // [streams, T, d] values (last forward)
  const float *coef;             // [streams, T, 2] (c, e) per token
  int *status;
  unsigned long long wait_ns;
  int inject;                    // test hook: every CTA's first wait is one that nothing completes
};

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigm(float z) { return fmaf(0.5f, tanh_approx(0.5f * z), 0.5f); }

// SiLU and its derivative of a pair of pre-activations in half precision,
// for outputs that are fp16 operands anyway: with s = sigmoid(z) =
// 1/2 + tanh(z/2)/2, x = z s and s' = s (1 + z (1 - s)). Returns the pairs
// of x and s' as fp16 bits.
__device__ __forceinline__ void silu_pair_h2(float z0, float z1, uint32_t &x, uint32_t &sp) {
  const __half2 z = __floats2half2_rn(z0, z1);
  const __half2 half = __float2half2_rn(0.5f), one = __float2half2_rn(1.0f);
  __half2 h = __hmul2(z, half), t;
  const uint32_t hb = *reinterpret_cast<const uint32_t *>(&h);
  uint32_t tb;
  asm("tanh.approx.f16x2 %0, %1;" : "=r"(tb) : "r"(hb));
  t = *reinterpret_cast<const __half2 *>(&tb);
  const __half2 sg = __hfma2(t, half, half);
  const __half2 xx = __hmul2(z, sg);
  const __half2 dd = __hmul2(sg, __hfma2(z, __hsub2(one, sg), one));
  x = *reinterpret_cast<const uint32_t *>(&xx);
  sp = *reinterpret_cast<const uint32_t *>(&dd);
}

// Two fp32 values as one fp16 pair (round to nearest even).
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint4 pack8(const float *v) {
  return make_uint4(pack_h2(v[0], v[1]), pack_h2(v[2], v[3]), pack_h2(v[4], v[5]),
                    pack_h2(v[6], v[7]));
}

__device__ bool wait_b(uint64_t *bar, uint32_t par, const GemmArgs &a) {
  if (mbar_wait(bar, par, a.wait_ns)) return true;
  atomicCAS(a.status, 0, kDevTimeout);
  return false;
}

// Test hook of failure handling: a wait on a barrier that nothing ever
// completes. It runs out after the wait limit and is recorded like any other
// expired wait; the caller then issues nothing and leaves through its abort
// path. Returns false (the wait did not succeed).
__device__ bool injected_wait(uint64_t *never, int *status, unsigned long long wait_ns) {
  if (mbar_wait(never, 0, wait_ns)) return true;
  atomicCAS(status, 0, kDevTimeout);
  return false;
}

// Shared-memory stage: A tile [128 rows x 64 k] (K-major); B tile up to
// [256 x 64] (K-major) or [64 x 256] (MN-major). All in the row-block layout.
constexpr uint32_t A_BYTES = 128 * KB * 2;       // 16 KB
constexpr uint32_t B_BYTES = 256 * KB * 2;       // 32 KB
constexpr uint32_t STAGE_BYTES_MM = A_BYTES + B_BYTES;       // 48 KB, 4 stages
constexpr int STAGES_MAX = 4;

// A tile loads. mt: 128-row tile index.
__device__ __forceinline__ void load_stage(const GemmArgs &a, const CUtensorMap *mA,
                                           const CUtensorMap *mA2, const CUtensorMap *mB,
                                           unsigned char *st, uint64_t *bar, int s, int mt,
                                           int nt, int kb) {
  const int kind = a.kind;
  // A: K-major [128 rows x 64] (rows = tokens); two 64-row pieces.
  for (int piece = 0; piece < 2; ++piece) {
    const int r = 128 * mt + 64 * piece;         // row of the per-stream matrix
    if (a.a_split_kq) {
      const CUtensorMap *src = r < a.C ? mA : mA2;
      const int rr = (r < a.C ? r : r - a.C) + s * a.T + a.chunk * a.C;
      tma_load_2d(st + piece * 64 * 128, src, bar, kb * KB, rr);
    } else {
      tma_load_2d(st + piece * 64 * 128, mA, bar, kb * KB, s * a.a_rows_per_stream + r);
    }
  }
  if (kind == K_BWD) {
    // B: W_l as [K = n_l rows, N = n_{l-1} features], MN-major; 64 K rows per stage
    const int brow0 = s * a.b_rows_per_stream + kb * KB;
    for (int f = 0; f < a.N / 64; ++f)
      tma_load_2d(st + A_BYTES + f * 64 * 128, mB, bar, a.N * nt + 64 * f, brow0);
  } else {
    // B: W_l rows = N (K-major), up to 256 rows in 64-row pieces
    for (int piece = 0; piece < a.N / 64; ++piece)
      tma_load_2d(st + A_BYTES + piece * 64 * 128, mB, bar, kb * KB,
                  s * a.b_rows_per_stream + a.N * nt + 64 * piece);
  }
}

// One output tile (stream s, row tile mt, column tile nt) of a phase GEMM.
// KIND is one of the phases.
template <int KIND>
__device__ __forceinline__ void gemm_tile(const GemmArgs &a, const CUtensorMap &mA, const CUtensorMap &mA2,
                                          const CUtensorMap &mB, const int s, const int mt, const int nt) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *sm =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[STAGES_MAX], empty[STAGES_MAX], done, never;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  constexpr int kind = KIND;
  // this CTA's share of the reduction: K blocks [kb0, kb0 + nk)
  const int nkt = a.K / KB;
  const int kz = blockIdx.z / a.streams;
  const int kb0 = nkt * kz / a.ksplit, nk = nkt * (kz + 1) / a.ksplit - kb0;
  const uint32_t ncols = 256u;
  constexpr int STAGES = 4;
  constexpr uint32_t STAGE_BYTES = STAGE_BYTES_MM;

  if (tid == 0) {
    for (int i = 0; i < STAGES_MAX; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(&done, 1);
    mbar_init(&never, 1);
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&tslot, ncols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tslot;
  bool ok = true;
  // Programmatic dependent launch: everything above overlapped the previous
  // kernel's tail; its outputs are read only after this wait.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (tid == 0) {
    if (a.inject) ok = injected_wait(&never, a.status, a.wait_ns);
    const uint32_t tx = (uint32_t)(A_BYTES + (uint32_t)a.N * KB * 2);
    uint32_t idesc;
    if (kind == K_BWD) idesc = idesc_f16(128, a.N, false, true);
    else idesc = idesc_f16(128, a.N, false, false);
    for (int kb = 0; kb < nk && kb < STAGES && ok; ++kb) {
      mbar_arrive_expect_tx(&full[kb], tx);
      load_stage(a, &mA, &mA2, &mB, sm + kb * STAGE_BYTES, &full[kb], s, mt, nt, kb0 + kb);
    }
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int st = kb % STAGES;
      const uint32_t ph = (uint32_t)((kb / STAGES) & 1);
      if (!wait_b(&full[st], ph, a)) { ok = false; break; }
      tc_fence_after();
      const uint32_t base = smem_u32(sm + st * STAGE_BYTES);
      for (int ks = 0; ks < KB / 16; ++ks) {
        if (kind == K_BWD) {
          umma_f16(tm, desc_kmajor(base, 128, ks), desc_mnmajor(base + A_BYTES, 64, ks), idesc,
                    (kb | ks) != 0);
        } else {
          umma_f16(tm, desc_kmajor(base, 128, ks), desc_kmajor(base + A_BYTES, a.N, ks), idesc,
                    (kb | ks) != 0);
        }
      }
      umma_commit(&empty[st]);
      if (kb + STAGES < nk) {
        if (!wait_b(&empty[st], ph, a)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[st], tx);
        load_stage(a, &mA, &mA2, &mB, sm + st * STAGE_BYTES, &full[st], s, mt, nt, kb0 + kb + STAGES);
      }
    }
    umma_commit(&done);
  }
  __syncwarp();
  // the next kernel may start its prologue now (it waits for our completion
  // before reading anything we write)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // ------------------------------------------------------------ epilogue
  if (!mbar_wait(&done, 0, a.wait_ns)) { atomicCAS(a.status, 0, kDevTimeout); ok = false; }
  tc_fence_after();
  ok = __syncthreads_and(ok) != 0;               // an expired wait anywhere skips the epilogue
  const int row = 32 * (warp & 3) + lane;        // TMEM lane = output row of the tile
  const uint32_t lb = (uint32_t)(32 * (warp & 3)) << 16;
  const int half = warp >> 2;                    // this warp's half of the tile's columns
  const int cbeg = half * (a.N / 2), cend = cbeg + a.N / 2;
  // Split K: every CTA of the tile stores its partial sums; the last to
  // arrive adds them up (in split order, so the result does not depend on
  // the arrival order) and runs the epilogue.
  const int tile = (s * gridDim.y + mt) * gridDim.x + nt;
  const float *parts = nullptr;
  if (ok && a.ksplit > 1) {
    __shared__ int last;
    float *mine = a.part + ((long long)tile * a.ksplit + kz) * 128 * a.N + (long long)row * a.N;
    for (int c0 = cbeg; c0 < cend; c0 += 16) {
      float z[16];
      tmem_ld16(tm + lb + c0, z);
      tmem_wait_ld();
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4)
        __stcg(reinterpret_cast<float4 *>(mine + c0 + 4 * i4), make_float4(z[4 * i4], z[4 * i4 + 1], z[4 * i4 + 2], z[4 * i4 + 3]));
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const unsigned prev = atomicAdd(a.cnt + tile, 1u);
      last = prev == (unsigned)a.ksplit - 1;
      if (last) a.cnt[tile] = 0;                 // every CTA of the tile has arrived: ready for the next launch
    }
    __syncthreads();
    if (!last) ok = false;                       // not an error: another CTA finishes the tile
    __threadfence();
    parts = a.part + (long long)tile * a.ksplit * 128 * a.N + (long long)row * a.N;
  }
  // the tile's 16 sums from column c0 on, for this thread's row
  auto sums = [&](int c0, float (&z)[16]) {
    if (parts == nullptr) {
      tmem_ld16(tm + lb + c0, z);
      tmem_wait_ld();
      return;
    }
    // every partial of the 16 columns requested at once (at most 4 splits),
    // then added in split order
    float4 v[kMaxSplit][4];
#pragma unroll
    for (int k = 0; k < kMaxSplit; ++k)
      if (k < a.ksplit) {
        const float4 *src = reinterpret_cast<const float4 *>(parts + (long long)k * 128 * a.N + c0);
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) v[k][i4] = __ldcg(src + i4);
      }
#pragma unroll
    for (int i4 = 0; i4 < 4; ++i4) {
      z[4 * i4] = v[0][i4].x; z[4 * i4 + 1] = v[0][i4].y; z[4 * i4 + 2] = v[0][i4].z; z[4 * i4 + 3] = v[0][i4].w;
    }
#pragma unroll
    for (int k = 1; k < kMaxSplit; ++k)
      if (k < a.ksplit) {
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          z[4 * i4] += v[k][i4].x; z[4 * i4 + 1] += v[k][i4].y; z[4 * i4 + 2] += v[k][i4].z; z[4 * i4 + 3] += v[k][i4].w;
        }
      }
  };
  if (ok) {
    if constexpr (kind == K_FWD || kind == K_FWD_LAST || kind == K_BWD) {
      const int r = 128 * mt + row;              // row of the per-stream matrix
      const bool key = r < a.C;
      const bool valid = (kind == K_BWD) ? key : (r < 2 * a.C);
      for (int c0 = cbeg; c0 < cend; c0 += 16) {
        float z[16];
        sums(c0, z);
        if (!valid) continue;
        const int col = a.N * nt + c0;           // column in the per-stream output
        if (kind == K_FWD) {
          float x[16], sp[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float sg = sigm(z[i]);
            x[i] = z[i] * sg;
            sp[i] = sg * (1.f + z[i] * (1.f - sg));
          }
          op_t *xo = a.x_out + ((long long)s * 2 * a.C + r) * a.n_out + col;
          *reinterpret_cast<uint4 *>(xo) = pack8(x);
          *reinterpret_cast<uint4 *>(xo + 8) = pack8(x + 8);
          if (key) {
            op_t *so = a.sp_out + ((long long)s * a.C + r) * a.n_out + col;
            *reinterpret_cast<uint4 *>(so) = pack8(sp);
            *reinterpret_cast<uint4 *>(so + 8) = pack8(sp + 8);
          }
        } else {
          float g[16];
          long long tok = (long long)s * a.T + (long long)a.chunk * a.C + (key ? r : r - a.C);
          if (kind == K_FWD_LAST) {
            if (!key) {
              float *yo = a.y + tok * a.n_out + col;
#pragma unroll
              for (int i4 = 0; i4 < 4; ++i4)
                *reinterpret_cast<float4 *>(yo + 4 * i4) = make_float4(z[4 * i4], z[4 * i4 + 1], z[4 * i4 + 2], z[4 * i4 + 3]);
              continue;
            }
            const uint4 v0 = *reinterpret_cast<const uint4 *>(a.v + tok * a.n_out + col);
            const uint4 v1 = *reinterpret_cast<const uint4 *>(a.v + tok * a.n_out + col + 8);
            const __nv_bfloat16 *vb0 = reinterpret_cast<const __nv_bfloat16 *>(&v0);
            const __nv_bfloat16 *vb1 = reinterpret_cast<const __nv_bfloat16 *>(&v1);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              g[i] = 2.f * (z[i] - __bfloat162float(vb0[i]));
              g[8 + i] = 2.f * (z[8 + i] - __bfloat162float(vb1[i]));
            }
          } else {
            const op_t *spi = a.sp_in + ((long long)s * a.C + r) * a.n_out + col;
            const uint4 s0 = *reinterpret_cast<const uint4 *>(spi);
            const uint4 s1 = *reinterpret_cast<const uint4 *>(spi + 8);
            const op_t *sb0 = reinterpret_cast<const op_t *>(&s0);
            const op_t *sb1 = reinterpret_cast<const op_t *>(&s1);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              g[i] = z[i] * __half2float(sb0[i]);
              g[8 + i] = z[8 + i] * __half2float(sb1[i]);
            }
          }
          const float2 ce = *reinterpret_cast<const float2 *>(a.coef + 2 * tok);
          float gc[16], ge[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) { gc[i] = -ce.x * g[i]; ge[i] = -ce.y * g[i]; }
          const long long o = ((long long)s * a.C + r) * a.n_out + col;
          *reinterpret_cast<uint4 *>(a.g_out + o) = pack8(g);
          *reinterpret_cast<uint4 *>(a.g_out + o + 8) = pack8(g + 8);
          *reinterpret_cast<uint4 *>(a.gc_out + o) = pack8(gc);
          *reinterpret_cast<uint4 *>(a.gc_out + o + 8) = pack8(gc + 8);
          *reinterpret_cast<uint4 *>(a.ge_out + o) = pack8(ge);
          *reinterpret_cast<uint4 *>(a.ge_out + o + 8) = pack8(ge + 8);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, ncols);
}

// Forward and backward phases: one launch per layer, grid = (column tiles,
// row tiles, streams).
template <int KIND>
__global__ void __launch_bounds__(NT, 1)
    tcl_gemm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap mA,
                    const __grid_constant__ CUtensorMap mA2, const __grid_constant__ CUtensorMap mB) {
  gemm_tile<KIND>(a, mA, mA2, mB, blockIdx.z % a.streams, blockIdx.y, blockIdx.x);
}

// ------------------------------------------------------------------------
// The state update of every layer of a chunk, in one launch. One CTA per
// tile of 128 rows x N columns of one layer's W_l (tiles numbered layer, then
// stream, row tile, column tile) forms the weight-update contractions
//   U_W = sum_i (-c_i g_i) x_i^T,  U_S = sum_i (-e_i g_i) x_i^T
// on tcgen05 (A = the MN-major -c G and -e G of the tile's rows, B = the
// layer's inputs X; accumulators in TMEM columns 0.. and 128..), then
//   W' = B W + c_S S + U_W,  S' = A S + U_S
// and the fp16 copy of W' that the next chunk's forward reads.
// The fp32 state tile travels by TMA both ways. Its loads (32-column boxes,
// 128-byte swizzle) are issued when the CTA starts, beside the contraction's
// operands: the previous chunk's update of these rows completed before the
// kernels between it and this launch could start, so they need not wait for
// the preceding kernel. After the MMAs, the thread that owns a row's TMEM
// lane updates that row in shared memory (16-byte chunk j of row r sits at
// j ^ (r % 8): conflict-free across the 8 rows a quarter-warp touches), and
// the tile goes back to global memory by TMA stores. Every state byte is read
// once and written once and a tile's loads are all in flight together.
constexpr int UP_NT = 256;
constexpr uint32_t UP_BOX = 128 * 128;         // one box slot: 128 rows x 128 bytes
struct UpLayer {
  int M, N, mtiles, ntiles, first;             // rows of W_l, tile width, tiles per stream, first tile
  int b_rows_per_stream;                       // rows of the X source per stream
  long long b_row_off;                         // first X row of the chunk (layer 1 reads the keys)
};
struct UpArgs {
  UpLayer l[kMaxL];
  int L, C, chunk, nchunks;
  const float *scal;                           // [streams, nchunks, 4] (B, A, c_S, -)
  int *status;
  unsigned long long wait_ns;
  int inject;                                  // test hook, as in GemmArgs
};
struct UpMaps {
  CUtensorMap a[kMaxL], a2[kMaxL], b[kMaxL];   // -c G_l, -e G_l [S*C, d_l]; X_{l-1} (fp16, 64 x 64 boxes)
  CUtensorMap w[kMaxL], s[kMaxL];              // fp32 W_l, S_l as {cols, rows, stream}, 32-column boxes
  CUtensorMap wb[kMaxL];                       // fp16 W_l as {cols, rows, stream}, 64-column boxes
};
__host__ __device__ constexpr uint32_t up_stage_bytes(int N) { return 2 * A_BYTES + (uint32_t)N * KB * 2; }
__host__ __device__ constexpr int up_stages(int nk) { return nk <= 2 ? 2 : 3; }
// dynamic shared memory: the operand ring, then the W and S tiles
__host__ __device__ constexpr size_t up_smem(int N, int nk) {
  return (size_t)up_stages(nk) * up_stage_bytes(N) + 2 * (size_t)(N / 32) * UP_BOX + 1024;
}
// tile width: 128 columns when the ring and both state tiles fit (C <= 128)
__host__ __device__ constexpr int up_width(int cols, int C) { return cols % 128 == 0 && C <= 128 ? 128 : 64; }

__device__ __forceinline__ bool up_wait(uint64_t *bar, uint32_t par, const UpArgs &a) {
  if (mbar_wait(bar, par, a.wait_ns)) return true;
  atomicCAS(a.status, 0, kDevTimeout);
  return false;
}

__global__ void __launch_bounds__(UP_NT, 1)
    tcl_update_kernel(const __grid_constant__ UpArgs a, const __grid_constant__ UpMaps m) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *sm =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[3], empty[3], done, stb, never;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int t = blockIdx.x;
  int l = 0;
  while (l + 1 < a.L && t >= a.l[l + 1].first) ++l;
  const UpLayer &ly = a.l[l];
  const int per = ly.mtiles * ly.ntiles, i = t - ly.first;
  const int s = i / per, mt = (i % per) / ly.ntiles, nt = i % ly.ntiles;
  const int N = ly.N, nk = a.C / KB, STAGES = up_stages(nk);
  const uint32_t SB = up_stage_bytes(N);
  unsigned char *wt = sm + STAGES * SB;        // W tile: N / 32 boxes
  unsigned char *st = wt + (N / 32) * UP_BOX;  // S tile
  unsigned char *wbt = sm;                     // fp16 W' tile (N / 64 boxes), in the ring once the MMAs are done
  const int R = ly.M < 128 ? ly.M : 128;       // rows of a box
  const int rows = ly.M - 128 * mt < 128 ? ly.M - 128 * mt : 128;   // rows of this tile

  if (tid == 0) {
    for (int k = 0; k < 3; ++k) { mbar_init(&full[k], 1); mbar_init(&empty[k], 1); }
    mbar_init(&done, 1);
    mbar_init(&stb, 1);
    mbar_init(&never, 1);
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&tslot, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tslot;
  bool ok = true;
  if (tid == 0) {
    if (a.inject) ok = injected_wait(&never, a.status, a.wait_ns);
    if (ok) {
      mbar_arrive_expect_tx(&stb, 2u * (uint32_t)(N / 32) * (uint32_t)R * 128u);
      for (int b = 0; b < N / 32; ++b) {
        tma_load_3d(wt + b * UP_BOX, &m.w[l], &stb, N * nt + 32 * b, 128 * mt, s);
        tma_load_3d(st + b * UP_BOX, &m.s[l], &stb, N * nt + 32 * b, 128 * mt, s);
      }
    } else {
      mbar_arrive(&stb);                       // nothing issued: release the state-tile waiters
    }
  }
  // the operands are the preceding kernel's outputs
  asm volatile("griddepcontrol.wait;" ::: "memory");
  int issued = 0, consumed = 0;                // operand stages requested / seen complete (thread 0)
  if (tid == 0) {
    const uint32_t idesc = idesc_f16(128, N, true, true);
    auto load = [&](int stg, int kb) {
      unsigned char *d = sm + stg * SB;
      const int row0 = s * a.C + kb * KB;
      for (int f = 0; f < 2; ++f) {
        tma_load_2d(d + f * 64 * 128, &m.a[l], &full[stg], 128 * mt + 64 * f, row0);
        tma_load_2d(d + A_BYTES + f * 64 * 128, &m.a2[l], &full[stg], 128 * mt + 64 * f, row0);
      }
      const int brow0 = (int)(s * ly.b_rows_per_stream + ly.b_row_off) + kb * KB;
      for (int f = 0; f < N / 64; ++f)
        tma_load_2d(d + 2 * A_BYTES + f * 64 * 128, &m.b[l], &full[stg], N * nt + 64 * f, brow0);
    };
    for (int kb = 0; kb < nk && kb < STAGES && ok; ++kb) {
      mbar_arrive_expect_tx(&full[kb], SB);
      load(kb, kb);
      ++issued;
    }
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int stg = kb % STAGES;
      const uint32_t ph = (uint32_t)((kb / STAGES) & 1);
      if (!up_wait(&full[stg], ph, a)) { ok = false; break; }
      ++consumed;
      tc_fence_after();
      const uint32_t base = smem_u32(sm + stg * SB);
      for (int ks = 0; ks < KB / 16; ++ks) {
        const uint64_t bd = desc_mnmajor(base + 2 * A_BYTES, 64, ks);
        umma_f16(tm, desc_mnmajor(base, 64, ks), bd, idesc, (kb | ks) != 0);
        umma_f16(tm + 128, desc_mnmajor(base + A_BYTES, 64, ks), bd, idesc, (kb | ks) != 0);
      }
      umma_commit(&empty[stg]);
      if (kb + STAGES < nk) {
        if (!up_wait(&empty[stg], ph, a)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[stg], SB);
        load(stg, kb + STAGES);
        ++issued;
      }
    }
    umma_commit(&done);
  }
  __syncwarp();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (!up_wait(&done, 0, a)) ok = false;
  if (!up_wait(&stb, 0, a)) ok = false;
  tc_fence_after();
  ok = __syncthreads_and(ok) != 0;
  if (ok) {
    const float4 sc = *reinterpret_cast<const float4 *>(a.scal + 4 * ((long long)s * a.nchunks + a.chunk));
    const int q = warp & 3, h = warp >> 2;     // TMEM lanes 32q.. (rows); column half h
    const int r = 32 * q + lane;
    const uint32_t lb = (uint32_t)(32 * q) << 16;
    for (int gi = 0; gi < N / 64; ++gi) {
      const int cg = (N / 2) * h + 32 * gi;    // first of this thread's 32 columns
      float u0[16], u1[16], v0[16], v1[16];
      tmem_ld16(tm + lb + (uint32_t)cg, u0);
      tmem_ld16(tm + lb + (uint32_t)cg + 16, u1);
      tmem_ld16(tm + lb + 128 + (uint32_t)cg, v0);
      tmem_ld16(tm + lb + 128 + (uint32_t)cg + 16, v1);
      tmem_wait_ld();
      if (r >= rows) continue;
      unsigned char *wr = wt + (cg / 32) * UP_BOX + r * 128;
      unsigned char *sr = st + (cg / 32) * UP_BOX + r * 128;
      unsigned char *br = wbt + (cg / 64) * UP_BOX + r * 128;
      const int c16 = (cg % 64) / 8;           // 16-byte chunk of the fp16 row that column cg starts
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t o = (uint32_t)((j ^ (r & 7)) << 4);
        const float *uw = j < 4 ? u0 + 4 * j : u1 + 4 * (j - 4);
        const float *us = j < 4 ? v0 + 4 * j : v1 + 4 * (j - 4);
        const float4 w = *reinterpret_cast<const float4 *>(wr + o);
        const float4 x = *reinterpret_cast<const float4 *>(sr + o);
        const float4 wn = make_float4(sc.x * w.x + sc.z * x.x + uw[0], sc.x * w.y + sc.z * x.y + uw[1],
                                      sc.x * w.z + sc.z * x.z + uw[2], sc.x * w.w + sc.z * x.w + uw[3]);
        const float4 sn = make_float4(sc.y * x.x + us[0], sc.y * x.y + us[1], sc.y * x.z + us[2],
                                      sc.y * x.w + us[3]);
        *reinterpret_cast<float4 *>(wr + o) = wn;
        *reinterpret_cast<float4 *>(sr + o) = sn;
        const uint32_t ob = (uint32_t)((((c16 + (j >> 1)) ^ (r & 7)) << 4) + (j & 1) * 8);
        *reinterpret_cast<uint2 *>(br + ob) = make_uint2(pack_h2(wn.x, wn.y), pack_h2(wn.z, wn.w));
      }
    }
  }
  fence_proxy_async_smem();                    // the updated tiles are read by the TMA stores
  __syncthreads();
  if (tid == 0 && ok) {
    for (int b = 0; b < N / 32; ++b) {
      tma_store_3d(&m.w[l], wt + b * UP_BOX, N * nt + 32 * b, 128 * mt, s);
      tma_store_3d(&m.s[l], st + b * UP_BOX, N * nt + 32 * b, 128 * mt, s);
    }
    for (int b = 0; b < N / 64; ++b) tma_store_3d(&m.wb[l], wbt + b * UP_BOX, N * nt + 64 * b, 128 * mt, s);
    tma_store_commit_wait_read();
  }
  if (!ok && tid == 0) {
    // after an expired wait: copies and MMAs this CTA started may still be
    // using its shared memory; give them (again bounded) time to finish
    for (int k = consumed; k < issued; ++k) mbar_wait(&full[k % STAGES], (uint32_t)((k / STAGES) & 1), a.wait_ns);
    mbar_wait(&stb, 0, a.wait_ns);
    mbar_wait(&done, 0, a.wait_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 256);
}

// ------------------------------------------------------------------------
// The state update of every layer of a chunk, pipelined (chunks of at most 128
// tokens). One CTA per unit = (layer l, stream, block of 128 rows of W_l, a
// range of up to `tpu` 64-column tiles). The contraction's A operands, -c G
// and -e G of the block's rows over the whole chunk (K = C), are loaded once.
// The MMAs run per 64-column tile (X columns in one of two slots, reused as
// soon as the tile's MMAs are done; the U_W | U_S accumulators in one of two
// TMEM pairs); the fp32 W and S stream through four slots of 32-column half
// tiles, so that up to four half tiles of state are in flight while one is
// updated and stored:
//   warp 0      TMA loads (state half tiles first: they do not depend on the
//               previous kernel; the operands after griddepcontrol.wait)
//   warp 1      TMEM allocation; MMA issue (M = 128 rows, N = 64, K = C)
//   warp 2      TMA stores of W' and S' per half tile, each slot freed once
//               its stores have read it
//   warps 4-11  epilogue: the thread owning TMEM lane r (row r) and 16 of a
//               half tile's 32 columns computes W' = B W + c_S S + U_W,
//               S' = A S + U_S in place, and writes the fp16 W' of its 16
//               columns (32 contiguous bytes) straight to global memory
// Every wait is bounded and also gives up once another role has flagged an
// abort; after an abort the producer waits (bounded) for its copies in
// flight and the MMA warp for its MMAs before TMEM is freed.
constexpr int UP2_NT = 384;
constexpr int UP2_EPI0 = 4;                    // first epilogue warp
constexpr int UP2_WS = 4;                      // state half-tile slots
struct Up2Layer {
  int M, mtiles, ntiles, nranges, first;       // rows of W_l, 128-row blocks, 64-column tiles, ranges, first unit
  int b_rows_per_stream;                       // rows of the X source per stream
  long long b_row_off;                         // first X row of the chunk (layer 1 reads the keys)
  op_t *wb;                                    // fp16 copy of W_l, [streams, M, 64 ntiles] row-major
};
struct Up2Args {
  Up2Layer l[kMaxL];
  int L, C, chunk, nchunks, tpu;
  const float *scal;                           // [streams, nchunks, 4] (B, A, c_S, -)
  int *status;
  unsigned long long wait_ns;
  int inject;                                  // test hook, as in GemmArgs
};
// shared memory: A operands, two X slots, four state slots
__host__ __device__ constexpr uint32_t up2_a_bytes(int C) { return 2u * (uint32_t)C * 128u; }
__host__ __device__ constexpr uint32_t up2_x_bytes(int C) { return (uint32_t)(C > 128 ? C : 128) * 128u; }
__host__ __device__ constexpr uint32_t up2_ws_bytes() { return 2u * UP_BOX; }   // W and S, 32 columns each
__host__ __device__ constexpr size_t up2_smem(int C) {
  return 2 * (size_t)up2_a_bytes(C) + 2 * (size_t)up2_x_bytes(C) + UP2_WS * (size_t)up2_ws_bytes() + 1024;
}

// Bounded wait that also returns (false) once *abort is set; on expiry it
// records TM_ERR_TIMEOUT and sets *abort.
__device__ bool up2_wait(uint64_t *bar, uint32_t par, const Up2Args &a, volatile int *abort) {
  if (mbar_try_wait(bar, par)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (mbar_try_wait(bar, par)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > a.wait_ns) {
      atomicCAS(a.status, 0, kDevTimeout);
      *abort = 1;
      return false;
    }
  }
}

__global__ void __launch_bounds__(UP2_NT, 1)
    tcl_update2_kernel(const __grid_constant__ Up2Args a, const __grid_constant__ UpMaps m) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *sm =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t a_full, x_full[2], mma_done[2], acc_free[2];
  __shared__ uint64_t ws_full[UP2_WS], epi_done[UP2_WS], ws_free[UP2_WS], fin, never;
  __shared__ uint32_t tslot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  // this CTA's unit
  const int u = blockIdx.x;
  int l = 0;
  while (l + 1 < a.L && u >= a.l[l + 1].first) ++l;
  const Up2Layer &ly = a.l[l];
  const int per = ly.mtiles * ly.nranges, i = u - ly.first;
  const int s = i / per, mt = (i % per) / ly.nranges, rg = i % ly.nranges;
  const int j0 = rg * a.tpu, j1 = (j0 + a.tpu < ly.ntiles) ? j0 + a.tpu : ly.ntiles;
  const int nt = j1 - j0;                      // 64-column tiles of this unit
  const int nh = 2 * nt;                       // 32-column half tiles
  const int C = a.C;
  const int R = ly.M < 128 ? ly.M : 128;       // rows of a state box
  const int rows = ly.M - 128 * mt < 128 ? ly.M - 128 * mt : 128;
  const uint32_t AB = up2_a_bytes(C), XB = up2_x_bytes(C);
  unsigned char *a_cg = sm, *a_eg = sm + AB;
  auto x_slot = [&](int b) { return sm + 2 * AB + b * XB; };
  auto w_slot = [&](int b) { return sm + 2 * AB + 2 * XB + b * up2_ws_bytes(); };
  auto s_slot = [&](int b) { return w_slot(b) + UP_BOX; };
  const uint32_t ws_bytes = 2u * (uint32_t)R * 128u;
  const uint32_t x_bytes = (uint32_t)C * 128u;

  if (tid == 0) {
    mbar_init(&a_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&x_full[b], 1);
      mbar_init(&mma_done[b], 1);
      mbar_init(&acc_free[b], 8);
    }
    for (int b = 0; b < UP2_WS; ++b) {
      mbar_init(&ws_full[b], 1);
      mbar_init(&epi_done[b], 8);
      mbar_init(&ws_free[b], 1);
    }
    mbar_init(&fin, 1);
    mbar_init(&never, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&tslot, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tslot;
  volatile int *abort = &abort_flag;

  // state half tiles of the first UP2_WS half tiles: issued before the wait
  // for the preceding kernel (this chunk's forward/backward), which does not
  // write them
  int ws_armed[UP2_WS] = {0, 0, 0, 0}, x_armed[2] = {0, 0}, a_armed = 0;
  auto load_ws = [&](int h2) {                 // half tile h2 into slot h2 % UP2_WS
    const int b = h2 % UP2_WS, col = 64 * j0 + 32 * h2;
    mbar_arrive_expect_tx(&ws_full[b], ws_bytes);
    tma_load_3d(w_slot(b), &m.w[l], &ws_full[b], col, 128 * mt, s);
    tma_load_3d(s_slot(b), &m.s[l], &ws_full[b], col, 128 * mt, s);
    ++ws_armed[b];
  };
  if (warp == 0 && lane == 0) {
    if (a.inject && !injected_wait(&never, a.status, a.wait_ns)) *abort = 1;
    for (int h2 = 0; h2 < nh && h2 < UP2_WS && !*abort; ++h2) load_ws(h2);
    // the unit's later half tiles wait for a free slot; bring them into L2 now
    // so that their loads, when the slots free up, do not wait on DRAM
    for (int h2 = UP2_WS; h2 < nh && !*abort; ++h2) {
      tma_prefetch_l2_3d(&m.w[l], 64 * j0 + 32 * h2, 128 * mt, s);
      tma_prefetch_l2_3d(&m.s[l], 64 * j0 + 32 * h2, 128 * mt, s);
    }
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !*abort) {
      const long long brow = (long long)s * ly.b_rows_per_stream + ly.b_row_off;
      mbar_arrive_expect_tx(&a_full, 2u * AB);
      for (int f = 0; f < 2; ++f)
        for (int kp = 0; kp < C / 64; ++kp) {
          tma_load_2d(a_cg + f * C * 128 + kp * 64 * 128, &m.a[l], &a_full, 128 * mt + 64 * f, s * C + 64 * kp);
          tma_load_2d(a_eg + f * C * 128 + kp * 64 * 128, &m.a2[l], &a_full, 128 * mt + 64 * f, s * C + 64 * kp);
        }
      a_armed = 1;
      for (int jj = 0; jj < nt; ++jj) {
        const int b = jj & 1;
        // the slot's previous X (tile jj - 2) has been read by its MMAs
        if (jj >= 2 && !up2_wait(&mma_done[b], (uint32_t)(((jj - 2) >> 1) & 1), a, abort)) break;
        mbar_arrive_expect_tx(&x_full[b], x_bytes);
        for (int kp = 0; kp < C / 64; ++kp)
          tma_load_2d(x_slot(b) + kp * 64 * 128, &m.b[l], &x_full[b], 64 * (j0 + jj), (int)(brow + 64 * kp));
        ++x_armed[b];
        bool ok = true;
        for (int h2 = 2 * jj; h2 < 2 * jj + 2; ++h2) {
          if (h2 < UP2_WS) continue;           // issued before the wait
          if (!up2_wait(&ws_free[h2 % UP2_WS], (uint32_t)(((h2 - UP2_WS) / UP2_WS) & 1), a, abort)) { ok = false; break; }
          load_ws(h2);
        }
        if (!ok) break;
      }
    }
    if (lane == 0 && *abort) {
      // copies still in flight into this CTA's shared memory finish first
      if (a_armed) mbar_wait(&a_full, 0, a.wait_ns);
      for (int b = 0; b < 2; ++b)
        if (x_armed[b]) mbar_wait(&x_full[b], (uint32_t)((x_armed[b] - 1) & 1), a.wait_ns);
      for (int b = 0; b < UP2_WS; ++b)
        if (ws_armed[b]) mbar_wait(&ws_full[b], (uint32_t)((ws_armed[b] - 1) & 1), a.wait_ns);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(128, 64, true, true);
      const uint32_t acg = smem_u32(a_cg), aeg = smem_u32(a_eg);
      bool ok = up2_wait(&a_full, 0, a, abort);
      for (int jj = 0; jj < nt && ok; ++jj) {
        const int b = jj & 1;
        if (!up2_wait(&x_full[b], (uint32_t)((jj >> 1) & 1), a, abort)) break;
        if (jj >= 2 && !up2_wait(&acc_free[b], (uint32_t)(((jj - 2) >> 1) & 1), a, abort)) break;
        tc_fence_after();
        const uint32_t xb = smem_u32(x_slot(b));
        const uint32_t acc = tm + 128u * (uint32_t)b;
        for (int ks = 0; ks < C / 16; ++ks) {
          const uint64_t bd = desc_mnmajor(xb, C, ks);
          umma_f16(acc, desc_mnmajor(acg, C, ks), bd, idesc, ks != 0);
          umma_f16(acc + 64, desc_mnmajor(aeg, C, ks), bd, idesc, ks != 0);
        }
        umma_commit(&mma_done[b]);
      }
      // every MMA this CTA issued has completed before TMEM is freed
      umma_commit(&fin);
      mbar_wait(&fin, 0, a.wait_ns);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ stores
    // One bulk group per half tile (its W' and S'); a group's slot is released
    // once the next group has been issued and the earlier ones have read
    // their sources, so one group stays in flight while the next is stored.
    if (lane == 0) {
      int pend = -1;                           // slot of the newest group, released one group later
      for (int h2 = 0; h2 < nh; ++h2) {
        const int b = h2 % UP2_WS, col = 64 * j0 + 32 * h2;
        if (!up2_wait(&epi_done[b], (uint32_t)((h2 / UP2_WS) & 1), a, abort)) break;
        tma_store_3d(&m.w[l], w_slot(b), col, 128 * mt, s);
        tma_store_3d(&m.s[l], s_slot(b), col, 128 * mt, s);
        bulk_commit_group();
        bulk_wait_group_read<1>();             // every group but this one has read its slot
        if (pend >= 0) mbar_arrive(&ws_free[pend]);
        pend = b;
      }
      bulk_wait_group_read<0>();
      if (pend >= 0) mbar_arrive(&ws_free[pend]);
    }
    __syncwarp();
  } else if (warp >= UP2_EPI0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3, h = (warp - UP2_EPI0) >> 2;
    const int r = 32 * q + lane;               // TMEM lane = row of the block
    const uint32_t lb = (uint32_t)(32 * q) << 16;
    const float4 sc = *reinterpret_cast<const float4 *>(a.scal + 4 * ((long long)s * a.nchunks + a.chunk));
    bool ok = true;
    for (int jj = 0; jj < nt && ok; ++jj) {
      const int xb = jj & 1;
      if (!up2_wait(&mma_done[xb], (uint32_t)((jj >> 1) & 1), a, abort)) break;
      for (int hs = 0; hs < 2; ++hs) {
        const int h2 = 2 * jj + hs, b = h2 % UP2_WS;
        if (!up2_wait(&ws_full[b], (uint32_t)((h2 / UP2_WS) & 1), a, abort)) { ok = false; break; }
        tc_fence_after();
        // this thread's 16 columns of the half tile: U_W and U_S
        float uw[16], us[16];
        const uint32_t acc = tm + lb + 128u * (uint32_t)xb + 32u * (uint32_t)hs + 16u * (uint32_t)h;
        tmem_ld16(acc, uw);
        tmem_ld16(acc + 64, us);
        tmem_wait_ld();
        if (hs == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_free[xb]);   // the MMAs of tile jj + 2 may overwrite the pair
        }
        if (r < rows) {
          unsigned char *wr = w_slot(b) + r * 128;
          unsigned char *sr = s_slot(b) + r * 128;
          uint32_t hw[8];                      // fp16 W' of this thread's 16 columns
#pragma unroll
          for (int jc = 0; jc < 4; ++jc) {
            const uint32_t o = (uint32_t)(((4 * h + jc) ^ (r & 7)) << 4);
            const float4 w = *reinterpret_cast<const float4 *>(wr + o);
            const float4 x = *reinterpret_cast<const float4 *>(sr + o);
            const float4 wn = make_float4(sc.x * w.x + sc.z * x.x + uw[4 * jc], sc.x * w.y + sc.z * x.y + uw[4 * jc + 1],
                                          sc.x * w.z + sc.z * x.z + uw[4 * jc + 2], sc.x * w.w + sc.z * x.w + uw[4 * jc + 3]);
            const float4 sn = make_float4(sc.y * x.x + us[4 * jc], sc.y * x.y + us[4 * jc + 1],
                                          sc.y * x.z + us[4 * jc + 2], sc.y * x.w + us[4 * jc + 3]);
            *reinterpret_cast<float4 *>(wr + o) = wn;
            *reinterpret_cast<float4 *>(sr + o) = sn;
            hw[2 * jc] = pack_h2(wn.x, wn.y);
            hw[2 * jc + 1] = pack_h2(wn.z, wn.w);
          }
          op_t *dst = ly.wb + (long long)s * ly.M * (64 * ly.ntiles) + (long long)(128 * mt + r) * (64 * ly.ntiles) +
                      64 * (j0 + jj) + 32 * hs + 16 * h;
          *reinterpret_cast<uint4 *>(dst) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4 *>(dst + 8) = make_uint4(hw[4], hw[5], hw[6], hw[7]);
        }
        fence_proxy_async_smem();              // the TMA stores read these rows
        __syncwarp();
        if (lane == 0) mbar_arrive(&epi_done[b]);
      }
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tm, 256);
}

// ------------------------------------------------------------------------
// The state update with the contraction transposed (chunks of at most 128
// tokens, every layer input width a multiple of 128). One CTA per unit =
// (layer l, stream, block of 128 columns of W_l, block of up to 256 rows):
//   U_W^T = X^T (-c G),  U_S^T = X^T (-e G)   (M = 128 columns, N = rows, K = C)
// so that TMEM lane i holds column i of the block and TMEM column j row j.
// A warp then owns 32 consecutive columns: it reads a row's W and S from a
// staged slot as one 128-byte piece and writes W', S' (fp32) and the fp16 copy
// of W' straight to global memory, each a whole row piece per instruction.
// The state streams through 16-row slots (16 KB: W and S of 16 rows x 128
// columns); once the MMAs have read the operands, their shared memory becomes
// more slots, so most of a unit's state is in flight at once, and a slot is
// refilled as soon as its four readers are done with it.
//   warps 0-15  epilogue: warp w owns TMEM lanes (columns) 32 (w % 4) .. +31
//               and the 16-row chunks i = w / 4, w / 4 + 4, ... (UP3_RQ = 4 row groups)
//   warp 16     TMA loads (the first slots' state before waiting for the
//               preceding kernel, which does not write it; the operands after)
//   warp 17     TMEM allocation; MMA issue, rows 0-127 and 128-255 committed
//               separately so that the epilogue starts on the first half
// Every wait is bounded and gives up once another role has flagged an abort.
constexpr int UP3_EPI = 16;                    // epilogue warps
constexpr int UP3_RQ = UP3_EPI / 4;            // row groups (each reads every column of its chunks)
constexpr int UP3_NT = (UP3_EPI + 2) * 32;
constexpr int UP3_SLOT = 16384;                // W and S of 16 rows x 128 fp32 columns
constexpr int UP3_NSLOT_MEM = 14;              // slots' worth of dynamic shared memory
constexpr int UP3_NS = 12;                     // slots in the ring (a multiple of the row groups)
static_assert(UP3_NS % UP3_RQ == 0, "a slot is always read by the same row group");
constexpr size_t UP3_SMEM = (size_t)UP3_NSLOT_MEM * UP3_SLOT + 1024;
struct Up3Layer {
  int M, cols, rblocks, cblocks, first;        // rows and columns of W_l, 256-row and 128-column blocks, first unit
  int b_rows_per_stream;                       // rows of the X source per stream
  long long b_row_off;                         // first X row of the chunk (layer 1 reads the keys)
  float *w, *s;                                // fp32 W_l, S_l of stream 0 (stream stride P)
  op_t *wb;                                    // fp16 copy of W_l, [streams, M, cols]
};
struct Up3Args {
  Up3Layer l[kMaxL];
  int L, C, chunk, nchunks;
  long long P;
  const float *scal;                           // [streams, nchunks, 4] (B, A, c_S, -)
  int *status;
  unsigned long long wait_ns;
  int inject;                                  // test hook, as in GemmArgs
};
struct Up3Maps {
  CUtensorMap a[kMaxL], a2[kMaxL], b[kMaxL];   // -c G_l, -e G_l [S*C, d_l]; X_{l-1} (fp16, 64 x 64 boxes)
  CUtensorMap w[kMaxL], s[kMaxL];              // fp32 W_l, S_l as {cols, rows, stream}, 128 x 16 boxes
};
// operand bytes: X^T (128 columns x C) and -c G, -e G (256 rows x C each), fp16
__host__ __device__ constexpr uint32_t up3_op_bytes(int C) { return 1280u * (uint32_t)C; }
// slots before the operand region (the rest of the ring overlays the operands)
__host__ __device__ constexpr int up3_dedicated(int C) {
  return UP3_NSLOT_MEM - (int)((up3_op_bytes(C) + UP3_SLOT - 1) / UP3_SLOT);
}

__device__ bool up3_wait(uint64_t *bar, uint32_t par, const Up3Args &a, volatile int *abort) {
  if (mbar_try_wait(bar, par)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (mbar_try_wait(bar, par)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > a.wait_ns) {
      atomicCAS(a.status, 0, kDevTimeout);
      *abort = 1;
      return false;
    }
  }
}

__global__ void __launch_bounds__(UP3_NT, 1)
    tcl_update3_kernel(const __grid_constant__ Up3Args a, const __grid_constant__ Up3Maps m) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *sm =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[UP3_NS], freed[UP3_NS], op_full[2], mma_done[2], fin, never;
  __shared__ uint32_t tslot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  // this CTA's unit
  const int u = blockIdx.x;
  int l = 0;
  while (l + 1 < a.L && u >= a.l[l + 1].first) ++l;
  const Up3Layer &ly = a.l[l];
  const int per = ly.rblocks * ly.cblocks, i0 = u - ly.first;
  const int s = i0 / per, rb = (i0 % per) / ly.cblocks, cb = i0 % ly.cblocks;
  const int N = ly.M - 256 * rb < 256 ? ly.M - 256 * rb : 256;   // rows of this unit (a multiple of 64)
  const int nch = N / 16;                      // 16-row chunks
  const int nhalf = N > 128 ? 2 : 1;
  const int C = a.C;
  const int NSD = up3_dedicated(C);
  unsigned char *opa = sm + NSD * UP3_SLOT;    // X^T: 2 feature blocks of 64 columns x C
  unsigned char *opc = opa + 256 * C;          // -c G: up to 4 feature blocks of 64 rows x C
  unsigned char *ope = opc + 512 * C;          // -e G
  auto slot_w = [&](int b) { return sm + b * UP3_SLOT; };

  if (tid == 0) {
    for (int b = 0; b < UP3_NS; ++b) {
      mbar_init(&full[b], 1);
      mbar_init(&freed[b], 4);                 // the four warps reading the slot's columns
    }
    mbar_init(&op_full[0], 1);
    mbar_init(&op_full[1], 1);
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
    mbar_init(&fin, 1);
    mbar_init(&never, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == UP3_EPI + 1) { tmem_alloc(&tslot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tslot;
  volatile int *abort = &abort_flag;

  int armed = 0, op_armed = 0;                 // chunks whose loads were issued; operand halves issued
  auto load_chunk = [&](int i) {               // rows 16 i .. 16 i + 15 of the unit into slot i % NS
    const int b = i % UP3_NS;
    unsigned char *dst = slot_w(b);
    mbar_arrive_expect_tx(&full[b], (uint32_t)UP3_SLOT);
    tma_load_3d(dst, &m.w[l], &full[b], 128 * cb, 256 * rb + 16 * i, s);
    tma_load_3d(dst + UP3_SLOT / 2, &m.s[l], &full[b], 128 * cb, 256 * rb + 16 * i, s);
    armed = i + 1;
  };
  if (warp == UP3_EPI && lane == 0) {
    if (a.inject && !injected_wait(&never, a.status, a.wait_ns)) *abort = 1;
    for (int i = 0; i < nch && i < NSD && !*abort; ++i) load_chunk(i);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == UP3_EPI) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !*abort) {
      const long long brow = (long long)s * ly.b_rows_per_stream + ly.b_row_off;
      // operands in two halves, so that the MMAs of rows 0-127 start while
      // those of rows 128-255 are still arriving: X^T and the first rows of
      // -c G, -e G, then the remaining rows
      for (int h = 0; h < nhalf; ++h) {
        const int f0 = 2 * h, f1 = (N / 64 < f0 + 2) ? N / 64 : f0 + 2;
        mbar_arrive_expect_tx(&op_full[h], (uint32_t)((h == 0 ? 256 * C : 0) + 2 * (f1 - f0) * 128 * C));
        for (int kp = 0; kp < C / 64; ++kp) {
          if (h == 0)
            for (int f = 0; f < 2; ++f)
              tma_load_2d(opa + f * C * 128 + kp * 64 * 128, &m.b[l], &op_full[0], 128 * cb + 64 * f, (int)(brow + 64 * kp));
          for (int f = f0; f < f1; ++f) {
            tma_load_2d(opc + f * C * 128 + kp * 64 * 128, &m.a[l], &op_full[h], 256 * rb + 64 * f, s * C + 64 * kp);
            tma_load_2d(ope + f * C * 128 + kp * 64 * 128, &m.a2[l], &op_full[h], 256 * rb + 64 * f, s * C + 64 * kp);
          }
        }
        op_armed = h + 1;
      }
      // the later chunks wait for slots (over the operands, or refills); bring
      // them into L2 behind the operands so that those loads do not wait on DRAM
      for (int i = armed; i < nch; ++i) {
        tma_prefetch_l2_3d(&m.w[l], 128 * cb, 256 * rb + 16 * i, s);
        tma_prefetch_l2_3d(&m.s[l], 128 * cb, 256 * rb + 16 * i, s);
      }
      bool ops_free = false;                   // the MMAs have read the operand region
      for (int i = armed; i < nch; ++i) {
        const int b = i % UP3_NS, use = i / UP3_NS;
        bool ok;
        if (use == 0) {                        // first use of a slot over the operands
          ok = ops_free || up3_wait(&mma_done[nhalf - 1], 0, a, abort);
          ops_free = ok;
        } else {
          ok = up3_wait(&freed[b], (uint32_t)((use - 1) & 1), a, abort);
        }
        if (!ok) break;
        load_chunk(i);
      }
    }
    if (lane == 0 && *abort) {
      // copies still in flight into this CTA's shared memory finish first
      for (int h = 0; h < op_armed; ++h) mbar_wait(&op_full[h], 0, a.wait_ns);
      for (int i = 0; i < armed; ++i)
        if (i + UP3_NS >= armed) mbar_wait(&full[i % UP3_NS], (uint32_t)((i / UP3_NS) & 1), a.wait_ns);
    }
    __syncwarp();
  } else if (warp == UP3_EPI + 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t xa = smem_u32(opa), gc = smem_u32(opc), ge = smem_u32(ope);
      for (int h = 0; h < nhalf; ++h) {
        if (!up3_wait(&op_full[h], 0, a, abort)) break;
        tc_fence_after();
        const int nh = N - 128 * h < 128 ? N - 128 * h : 128;
        const uint32_t idesc = idesc_f16(128, nh, true, true);
        const uint32_t boff = (uint32_t)(2 * h) * (uint32_t)C * 128u;   // feature blocks 2h, 2h + 1
        for (int ks = 0; ks < C / 16; ++ks) {
          const uint64_t ad = desc_mnmajor(xa, C, ks);
          umma_f16(tm + 128u * (uint32_t)h, ad, desc_mnmajor(gc + boff, C, ks), idesc, ks != 0);
          umma_f16(tm + 256u + 128u * (uint32_t)h, ad, desc_mnmajor(ge + boff, C, ks), idesc, ks != 0);
        }
        umma_commit(&mma_done[h]);
      }
      // every MMA this CTA issued has completed before TMEM is freed
      umma_commit(&fin);
      mbar_wait(&fin, 0, a.wait_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int lq = warp & 3, rq = warp >> 2;
    const int col = 32 * lq + lane;            // column of the block = TMEM lane
    const uint32_t lb = (uint32_t)(32 * lq) << 16;
    const float4 sc = *reinterpret_cast<const float4 *>(a.scal + 4 * ((long long)s * a.nchunks + a.chunk));
    const long long gcol = 128LL * cb + col;
    float *wout = ly.w + (long long)s * a.P + gcol;
    float *sout = ly.s + (long long)s * a.P + gcol;
    op_t *bout = ly.wb + (long long)s * ly.M * ly.cols + gcol;
    const int cols = ly.cols;
    int seen = 0;                              // halves of the accumulator known complete
    for (int i = rq; i < nch; i += UP3_RQ) {
      const int h = 16 * i >= 128 ? 1 : 0;
      if (seen <= h) {
        if (!up3_wait(&mma_done[h], 0, a, abort)) break;
        seen = h + 1;
      }
      const int b = i % UP3_NS;
      if (!up3_wait(&full[b], (uint32_t)((i / UP3_NS) & 1), a, abort)) break;
      tc_fence_after();
      float uw[16], us[16];
      tmem_ld16(tm + lb + 16u * (uint32_t)i, uw);
      tmem_ld16(tm + lb + 256u + 16u * (uint32_t)i, us);
      tmem_wait_ld();
      const float *ws_ = reinterpret_cast<const float *>(slot_w(b)) + col;
      const float *ss_ = ws_ + UP3_SLOT / 8;   // S follows W in the slot (8 KB = 2048 floats)
      const int o0 = (256 * rb + 16 * i) * cols;   // element offset of the chunk's first row
      float *wo = wout + o0, *so = sout + o0;
      op_t *bo = bout + o0;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float w = ws_[128 * r], x = ss_[128 * r];
        const float wn = sc.x * w + sc.z * x + uw[r];
        const float sn = sc.y * x + us[r];
        *wo = wn;
        *so = sn;
        *bo = __float2half_rn(wn);
        wo += cols;
        so += cols;
        bo += cols;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&freed[b]);   // the slot may be refilled
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  if (warp == UP3_EPI + 1) tmem_dealloc(tm, 512);
}

// ------------------------------------------------------------------------
// Fused forward + backward of one chunk, for memories whose every layer is at
// most 256 wide. One CTA per (128-row tile of the chunk's [keys; queries],
// stream) runs the whole chain that the per-phase kernels run as 2L - 1
// launches: the tile's rows stay in shared memory (fp16, row-block layout,
// overwritten in place by each epilogue) and the accumulator in TMEM, while
// the fp16 weights stream through a ring of TMA stages whose prefetch runs
// ahead across layer boundaries (the next layer's slices land during the
// current epilogue). Rows of a tile are independent through every layer, so
// no other CTA is involved.
//   forward  l = 1..L: Z_l = X_{l-1} W_l^T (K-major W slices of 64 columns)
//   backward l = L..2: G_{l-1} = (G_l W_l) . silu'(Z_{l-1}) (MN-major W slices
//            of 64 rows); tiles without key rows stop after the forward.
// Outputs are those the update GEMMs read: X_l and silu'(Z_l) of key rows,
// -c G_l and -e G_l; and y for query rows.
constexpr int FB_STAGES = 5;    // 64 KB tile + 5 x 32 KB ring: one slice of the next phase lands early
constexpr uint32_t FB_STAGE = 256 * KB * 2;          // 32 KB: one 64-wide slice of W_l
constexpr uint32_t FB_ABUF = 128 * 256 * 2;          // 64 KB: the tile's rows
constexpr size_t FB_SMEM = FB_ABUF + FB_STAGES * FB_STAGE + 1024;
constexpr int FB_MAXD = 256;
constexpr int FB_EPI = 512;          // 16 epilogue warps: warp w reads TMEM lanes 32 (w % 4) ..
                                     // +31, columns quarter w / 4 of the phase's output
constexpr int FB_NT = FB_EPI + 32;   // and one producer warp (TMA loads, MMA issue)

struct FbArgs {
  int L, C, T, chunk;
  int dims[kMaxL + 1];
  op_t *x_out[kMaxL + 1];            // [streams, 2C, d_l], key rows written (l = 1..L-1)
  op_t *sp_out[kMaxL + 1];           // silu'(Z_l) of key rows, [streams, d_l / 8, C, 8]: 16-byte
                                     // pieces of a row, consecutive rows adjacent (written and read
                                     // back by the same thread; a warp's 32 rows are 512 contiguous bytes)
  op_t *gc_out[kMaxL + 1];           // [streams, C, d_l] -c G_l
  op_t *ge_out[kMaxL + 1];           // [streams, C, d_l] -e G_l
  float *y;                          // [streams, T, d]
  const __nv_bfloat16 *v;            // [streams, T, d]
  const float *coef;                 // [streams, T, 2]
  int *status;
  unsigned long long wait_ns;
  int inject;                        // test hook, as in GemmArgs
};

struct FbMaps {
  CUtensorMap k, q;
  CUtensorMap w[kMaxL + 1];          // w[l]: fp16 W_l of every stream, [streams * d_l, d_{l-1}]
};

struct FbPhase {
  int bwd, l, ns, N;                 // backward?, layer, 64-wide K slices, output width
};

__device__ __forceinline__ FbPhase fb_phase(const FbArgs &a, int p) {
  FbPhase f;
  if (p < a.L) {
    f.bwd = 0; f.l = p + 1; f.ns = a.dims[p] / KB; f.N = a.dims[p + 1];
  } else {
    f.bwd = 1; f.l = a.L - (p - a.L); f.ns = a.dims[f.l] / KB; f.N = a.dims[f.l - 1];
  }
  return f;
}

// Issue the TMA loads of global weight slice g (counting slices over all
// phases of this tile) into stage g % FB_STAGES.
__device__ __forceinline__ void fb_load_slice(const FbArgs &a, const FbMaps &m, unsigned char *ring,
                                              uint64_t *full, int s, int g) {
  int p = 0, kb = g;
  FbPhase f = fb_phase(a, 0);
  while (kb >= f.ns) { kb -= f.ns; f = fb_phase(a, ++p); }
  const int st = g % FB_STAGES;
  unsigned char *dst = ring + st * FB_STAGE;
  const CUtensorMap *mw = &m.w[f.l];
  const int dl = a.dims[f.l];
  mbar_arrive_expect_tx(&full[st], (uint32_t)f.N * KB * 2);
  if (!f.bwd) {
    for (int piece = 0; piece < f.N / 64; ++piece)   // rows of W_l, K-major slice kb
      tma_load_2d(dst + piece * 64 * 128, mw, &full[st], kb * KB, s * dl + 64 * piece);
  } else {
    for (int blk = 0; blk < f.N / 64; ++blk)         // 64 rows (K) of W_l, MN-major
      tma_load_2d(dst + blk * 64 * 128, mw, &full[st], 64 * blk, s * dl + kb * KB);
  }
}

__device__ __forceinline__ void st_shared_v4(unsigned char *p, uint4 v) {
  *reinterpret_cast<uint4 *>(p) = v;
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(FB_EPI) : "memory"); }

__global__ void __launch_bounds__(FB_NT, 1)
    tcl_fb_kernel(const __grid_constant__ FbArgs a, const __grid_constant__ FbMaps m) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *abuf =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char *ring = abuf + FB_ABUF;
  __shared__ uint64_t full[FB_STAGES], empty[FB_STAGES], xbar, done, ready, flushed, never;
  __shared__ uint32_t tslot;
  __shared__ int abort_flag;
  __shared__ float2 cef[128];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int mt = blockIdx.x, s = blockIdx.y;
  const int C = a.C, L = a.L;
  const bool has_keys = 128 * mt < C;
  const int nphase = has_keys ? 2 * L - 1 : L;
  // key rows of this tile (keys precede queries)
  const int nkey = C - 128 * mt >= 128 ? 128 : (C - 128 * mt > 0 ? C - 128 * mt : 0);
  // silu'(Z_l) of key rows for the backward: the last two hidden layers keep
  // it in TMEM (fp16 pairs in columns 256-383 and 384-511, beside the
  // accumulator in 0-255); earlier layers go through global memory
  auto sp_slot = [&](int l) -> int { return L - 1 - l < 2 ? 256 + 128 * ((L - 1 - l) & 1) : -1; };

  if (tid == 0) {
    for (int i = 0; i < FB_STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(&xbar, 1);
    mbar_init(&done, 1);
    mbar_init(&ready, FB_EPI / 32);
    mbar_init(&flushed, FB_EPI / 32);
    mbar_init(&never, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&tslot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tslot;
  // The tile's input rows (fp16 keys or queries) were converted before the
  // chunk walk began, and every kernel of the walk waits for its predecessor
  // before it signals its dependents, so they can be requested before waiting
  // for the preceding kernel (the weights cannot).
  auto load_x = [&]() {
    const int d0 = a.dims[0];
    mbar_arrive_expect_tx(&xbar, (uint32_t)(128 * d0 * 2));
    for (int piece = 0; piece < 2; ++piece) {
      const int r = 128 * mt + 64 * piece;
      const CUtensorMap *src = r < C ? &m.k : &m.q;
      const int row = s * a.T + a.chunk * C + (r < C ? r : r - C);
      for (int f = 0; f < d0 / 64; ++f)
        tma_load_2d(abuf + f * 128 * 128 + piece * 64 * 128, src, &xbar, 64 * f, row);
    }
  };
  if (warp == FB_EPI / 32 && lane == 0 && !a.inject) load_x();
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == FB_EPI / 32) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && a.inject && !injected_wait(&never, a.status, a.wait_ns)) {
      abort_flag = 1;                            // nothing issued yet; release the epilogue
      mbar_arrive(&done);
    } else if (lane == 0) {
      int total = 0;
      for (int p = 0; p < nphase; ++p) total += fb_phase(a, p).ns;
      int issued = 0, consumed = 0;
      if (a.inject) load_x();
      for (; issued < total && issued < FB_STAGES; ++issued) fb_load_slice(a, m, ring, full, s, issued);
      bool ok = true;
      for (int p = 0; p < nphase && ok; ++p) {
        const FbPhase f = fb_phase(a, p);
        // the tile holds this phase's A operand: the input rows, or the
        // previous epilogue's output
        ok = p == 0 ? mbar_wait(&xbar, 0, a.wait_ns) : mbar_wait(&ready, (uint32_t)((p - 1) & 1), a.wait_ns);
        tc_fence_after();
        const uint32_t idesc = idesc_f16(128, f.N, false, f.bwd != 0);
        const uint32_t abase = smem_u32(abuf);
        // A phase has at most FB_STAGES slices and all of them were requested
        // before it began (the refills below run a phase ahead), so the MMAs
        // of a phase issue back to back.
        for (int kb = 0; kb < f.ns && ok; ++kb) {
          const int g = consumed;
          const int st = g % FB_STAGES;
          if (!mbar_wait(&full[st], (uint32_t)((g / FB_STAGES) & 1), a.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t bb = smem_u32(ring + st * FB_STAGE);
          for (int ks = 0; ks < KB / 16; ++ks) {
            const uint64_t ad = desc_kmajor(abase + kb * 128 * 128, 128, ks);
            const uint64_t bd = f.bwd ? desc_mnmajor(bb, 64, ks) : desc_kmajor(bb, f.N, ks);
            umma_f16(tm, ad, bd, idesc, (kb | ks) != 0);
          }
          umma_commit(&empty[st]);
          ++consumed;
        }
        if (!ok) { atomicCAS(a.status, 0, kDevTimeout); abort_flag = 1; }
        umma_commit(&done);
        // the last phase is under way: let the update launch behind this
        // kernel start (its state loads do not depend on this kernel; it waits
        // for this grid's completion before it reads the outputs)
        if (p == nphase - 1) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        // refill the consumed stages with the next phase's slices as the MMAs
        // finish; they land while the epilogue runs
        while (ok && issued < total && issued - FB_STAGES <= consumed - 1) {
          const int j = issued - FB_STAGES;
          if (!mbar_wait(&empty[j % FB_STAGES], (uint32_t)((j / FB_STAGES) & 1), a.wait_ns)) {
            ok = false;
            atomicCAS(a.status, 0, kDevTimeout);
            abort_flag = 1;
          } else {
            fb_load_slice(a, m, ring, full, s, issued++);
          }
        }
      }
      // after an abort: wait (bounded) for the copies still in flight into this CTA
      for (int g = consumed; g < issued; ++g)
        mbar_wait(&full[g % FB_STAGES], (uint32_t)((g / FB_STAGES) & 1), a.wait_ns);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int row = 32 * (warp & 3) + lane;      // TMEM lane = row of the tile
    const uint32_t lb = (uint32_t)(32 * (warp & 3)) << 16;
    const int quarter = warp >> 2;
    const int r = 128 * mt + row;                // row of the stream's [keys; queries]
    const bool key = r < C;
    const long long tok = (long long)s * a.T + (long long)a.chunk * C + (key ? r : r - C);
    if (tid < nkey)
      cef[tid] = *reinterpret_cast<const float2 *>(a.coef + 2 * ((long long)s * a.T + (long long)a.chunk * C + 128 * mt + tid));
    epi_sync();
    // Global traffic of the tile's outputs that the update reads (X, -c G,
    // -e G) leaves from the tile in shared memory after the next phase's MMAs
    // have been released (they only read the tile too). Each warp stores the
    // part of the tile it wrote itself (its 32 rows, its quarter of the
    // columns), whole row pieces per instruction, so that no warp waits for
    // another before it overwrites the tile in the next epilogue, unless the
    // next phase's width differs: then its column quarters overlap other
    // warps' old ones, and every warp waits (bounded) until all have flushed
    // (mbarrier `flushed`, one arrival per warp and phase).
    int pend_kind = 0, pend_l = 0, pend_N = 0;   // 1: X_l, 2: -c G_l and -e G_l
    auto flush = [&]() {
      if (!pend_kind || nkey == 0) return;
      const int N = pend_N, nchw = N / 4 / 8;    // 16-byte chunks of this warp's quarter of a row
      const int ch0 = quarter * nchw;
      for (int i = lane; i < 32 * nchw; i += 32) {
        const int rr = 32 * (warp & 3) + i / nchw;   // tile row
        const int ch = ch0 + i % nchw;
        if (rr >= nkey) continue;
        const uint4 u = *reinterpret_cast<const uint4 *>(abuf + rb_chunk(128, rr, ch));
        if (pend_kind == 1) {
          *reinterpret_cast<uint4 *>(a.x_out[pend_l] + ((long long)s * 2 * C + 128 * mt + rr) * N + 8 * ch) = u;
        } else {
          const op_t *hb = reinterpret_cast<const op_t *>(&u);
          const float2 k2 = cef[rr];
          float vc[8], ve[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float g = __half2float(hb[j]);
            vc[j] = -k2.x * g;
            ve[j] = -k2.y * g;
          }
          const long long o = ((long long)s * C + 128 * mt + rr) * N + 8 * ch;
          *reinterpret_cast<uint4 *>(a.gc_out[pend_l] + o) = pack8(vc);
          *reinterpret_cast<uint4 *>(a.ge_out[pend_l] + o) = pack8(ve);
        }
      }
      pend_kind = 0;
    };
    for (int p = 0; p < nphase; ++p) {
      const FbPhase f = fb_phase(a, p);
      const int N = f.N, cbeg = quarter * (N / 4), cend = cbeg + N / 4;
      // (every warp handles TMEM lanes 32 (warp % 4).. and columns [cbeg, cend))
      const bool last_fwd = !f.bwd && f.l == L;
      const bool grad = f.bwd || last_fwd;
      // this thread's other operand of a gradient phase (V, or silu' of the
      // layer below, which this same thread stored going forward), requested
      // before the MMAs finish
      uint4 aux[8];
      const int spt = f.bwd ? sp_slot(f.l - 1) : -1;      // silu' of the layer below in TMEM?
      if (grad && key && spt < 0) {
        // fp16 silu' (backward) or bf16 values (last forward), 8 per 16 bytes
        if (f.bwd) {
          const uint4 *src = reinterpret_cast<const uint4 *>(a.sp_out[f.l - 1] + (long long)s * C * N) + (cbeg / 8) * C + r;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (8 * i < N / 4) aux[i] = src[(long long)i * C];
        } else {
          const uint4 *src = reinterpret_cast<const uint4 *>(a.v + tok * N + cbeg);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (8 * i < N / 4) aux[i] = src[i];
        }
      }
      const bool width_change = pend_kind != 0 && nkey > 0 && pend_N != N;
      flush();                                   // the previous phase's outputs
      __syncwarp();
      if (lane == 0) mbar_arrive(&flushed);
      // one lane per warp waits for this phase's MMAs and, when the width
      // changes, for every warp's flush of the old outputs
      if (lane == 0 && (!mbar_wait(&done, (uint32_t)(p & 1), a.wait_ns) ||
                        (width_change && !mbar_wait(&flushed, (uint32_t)(p & 1), a.wait_ns)))) {
        atomicCAS(a.status, 0, kDevTimeout);
        abort_flag = 1;
      }
      __syncwarp();
      if (*(volatile int *)&abort_flag) break;
      tc_fence_after();
#pragma unroll
      for (int step = 0; step < FB_MAXD / 4 / 16; ++step) {
        const int c0 = cbeg + 16 * step;
        if (c0 >= cend) break;
        float z[16];
        tmem_ld16(tm + lb + c0, z);
        tmem_wait_ld();
        if (!grad) {
          // hidden layer: X = silu(Z) for every row (the next operand), and
          // silu'(Z) of key rows straight out; both are fp16 operands, so they
          // are computed in half precision, two at a time
          uint32_t xh[8], sh[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) silu_pair_h2(z[2 * i], z[2 * i + 1], xh[i], sh[i]);
#pragma unroll
          for (int i = 0; i < 2; ++i)
            st_shared_v4(abuf + rb_chunk(128, row, c0 / 8 + i), make_uint4(xh[4 * i], xh[4 * i + 1], xh[4 * i + 2], xh[4 * i + 3]));
          if (key) {
            const int slot = sp_slot(f.l);
            if (slot >= 0) {
              tmem_st8(tm + lb + (uint32_t)(slot + c0 / 2), sh);
            } else {
              uint4 *so = reinterpret_cast<uint4 *>(a.sp_out[f.l] + (long long)s * C * N) + (c0 / 8) * C + r;
              so[0] = make_uint4(sh[0], sh[1], sh[2], sh[3]);
              so[C] = make_uint4(sh[4], sh[5], sh[6], sh[7]);
            }
          }
        } else if (!key) {
          if (last_fwd) {                        // query row of the last layer: the read y
            float *yo = a.y + tok * N + c0;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              *reinterpret_cast<float4 *>(yo + 4 * i) = make_float4(z[4 * i], z[4 * i + 1], z[4 * i + 2], z[4 * i + 3]);
          }
        } else {
          // G_L = 2 (Z_L - V) or G_{l-1} = (G_l W_l) . silu'(Z_{l-1})
          if (spt >= 0) {
            uint32_t pk[8];
            tmem_ld8(tm + lb + (uint32_t)(spt + c0 / 2), pk);
            tmem_wait_ld();
            aux[2 * step] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            aux[2 * step + 1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const uint4 u = aux[2 * step + i];
            const op_t *hh = reinterpret_cast<const op_t *>(&u);
            const __nv_bfloat16 *hb = reinterpret_cast<const __nv_bfloat16 *>(&u);
            float g[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float h = f.bwd ? __half2float(hh[j]) : __bfloat162float(hb[j]);
              g[j] = f.bwd ? z[8 * i + j] * h : 2.f * (z[8 * i + j] - h);
            }
            st_shared_v4(abuf + rb_chunk(128, row, c0 / 8 + i), pack8(g));
          }
        }
      }
      if (!grad) tmem_wait_st();                 // silu' stored into TMEM above
      // the tile (generic-proxy writes) is read by the next phase's MMAs:
      // every warp reports its part
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ready);
      pend_kind = grad ? 2 : (nkey > 0 ? 1 : 0);
      pend_l = f.bwd ? f.l - 1 : f.l;
      pend_N = N;
      if (grad && !has_keys) pend_kind = 0;
    }
    if (!*(volatile int *)&abort_flag) flush();
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 512);
}

// A5 for every chunk of every stream at once: one warp per (stream, chunk),
// lane l holding tokens m l .. m l + m - 1 of the chunk (m = C / 32, 0-based i
// within the chunk):
//   pa_i = prod_{j>i}(1 - alpha_j), pe_i = prod_{j>i} eta_j,
//   r_{C-1} = 1, r_i = pa_i + eta_{i+1} r_{i+1};  c_i = theta_i r_i, e_i = theta_i pe_i;
//   B = prod(1 - alpha), A = prod eta, c_S = eta_0 r_0.
// The suffix products are a suffix scan over lanes of each lane's products;
// r is a chain of affine maps x -> pa_i + eta_{i+1} x, composed within each
// lane, suffix-scanned over lanes, then unrolled within the lane. No division.
constexpr int COEF_MAXM = kMaxC / 32;
__global__ void tcl_coef_kernel(const float *theta, const float *eta, const float *alpha, int streams,
                                int T, int C, int nchunks, float *coef, float *scal) {
  const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (long long)streams * nchunks) return;   // the whole warp leaves together
  const long long s = wid / nchunks, ch = wid % nchunks;
  const long long t0 = s * T + ch * C;
  const int m = C / 32;
  float th[COEF_MAXM], et[COEF_MAXM], om[COEF_MAXM];
  float Pa = 1.f, Pe = 1.f;
#pragma unroll
  for (int k = 0; k < COEF_MAXM; ++k)
    if (k < m) {
      const long long t = t0 + (long long)lane * m + k;
      th[k] = theta[t];
      et[k] = eta[t];
      om[k] = 1.f - alpha[t];
      Pa *= om[k];
      Pe *= et[k];
    }
  // products over the lanes after this one
  float xa = Pa, xe = Pe;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float ya = __shfl_down_sync(0xffffffffu, xa, o), ye = __shfl_down_sync(0xffffffffu, xe, o);
    if (lane + o < 32) { xa *= ya; xe *= ye; }
  }
  float na = __shfl_down_sync(0xffffffffu, xa, 1), ne = __shfl_down_sync(0xffffffffu, xe, 1);
  if (lane == 31) { na = 1.f; ne = 1.f; }
  float pa[COEF_MAXM], pe[COEF_MAXM], bn[COEF_MAXM];
  const float eta_after = __shfl_down_sync(0xffffffffu, et[0], 1);   // eta of the next lane's first token
  float A = 0.f, Bm = 1.f;                       // this lane's maps composed: x -> A + Bm x
#pragma unroll
  for (int k = COEF_MAXM - 1; k >= 0; --k)
    if (k < m) {
      pa[k] = na;
      pe[k] = ne;
      na *= om[k];
      ne *= et[k];
      bn[k] = k + 1 < m ? et[k + 1] : (lane == 31 ? 0.f : eta_after);   // eta_{i+1}; 0 past the chunk
      A = pa[k] + bn[k] * A;
      Bm = bn[k] * Bm;
    }
  // suffix scan of the lanes' maps: FA = r at this lane's first token
  float FA = A, FB = Bm;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float ya = __shfl_down_sync(0xffffffffu, FA, o), yb = __shfl_down_sync(0xffffffffu, FB, o);
    if (lane + o < 32) { FA = FA + FB * ya; FB = FB * yb; }
  }
  float r = __shfl_down_sync(0xffffffffu, FA, 1);   // r just after this lane's tokens (unused by lane 31)
#pragma unroll
  for (int k = COEF_MAXM - 1; k >= 0; --k)
    if (k < m) {
      r = pa[k] + bn[k] * r;
      const long long t = t0 + (long long)lane * m + k;
      *reinterpret_cast<float2 *>(coef + 2 * t) = make_float2(th[k] * r, th[k] * pe[k]);
      if (lane == 0 && k == 0)
        *reinterpret_cast<float4 *>(scal + 4 * wid) = make_float4(pa[0] * om[0], pe[0] * et[0], et[0] * r, 0.f);
    }
}

// Copy W0/S0 into W_end/S_end (unless in place) and build the fp16 operand
// copies, stored layer-major ([streams, n_l, n_{l-1}] per layer) so that one
// 2-D tensor map covers a layer of every stream.
struct InitArgs {
  const float *W0, *S0;
  float *W, *S;
  op_t *Wbf;
  long long P;
  long long streams;
  int L;
  long long off[kMaxL + 1];      // layer offsets inside a parameter vector
  long long boff[kMaxL + 1];     // layer offsets inside the fp16 copy
};

__global__ void tcl_init_kernel(const InitArgs a) {
  const long long total = a.streams * a.P;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const float w = a.W0[i];
    if (a.W != a.W0) a.W[i] = w;
    if (a.S != a.S0) a.S[i] = a.S0[i];
    const long long s = i / a.P, j = i % a.P;
    int l = 0;
    while (l + 1 < a.L && j >= a.off[l + 1]) ++l;
    const long long within = j - a.off[l];
    const long long per = a.off[l + 1] - a.off[l];
    a.Wbf[a.boff[l] + s * per + within] = __float2half_rn(w);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_l() {
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

// 2-D fp16 map over [rows x cols], box = 64 columns x box_rows rows, 128B swizzle.
bool map2d(CUtensorMap *m, const void *base, long long rows, int cols, int box_rows) {
  EncodeTiledFn fn = encode_fn_l();
  if (!fn) return false;
  std::memset(m, 0, sizeof *m);
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over `streams` matrices [rows x cols] of el-byte elements, matrix
// s at base + s * stream_stride elements; box = box_cols x box_rows x 1 with
// the 128-byte swizzle (box_cols * el = 128).
bool map3d(CUtensorMap *m, CUtensorMapDataType dt, int el, const void *base, int cols, int rows, int streams,
           long long stream_stride, int box_cols, int box_rows) {
  EncodeTiledFn fn = encode_fn_l();
  if (!fn || box_cols * el != 128) return false;
  std::memset(m, 0, sizeof *m);
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)streams};
  cuuint64_t strides[2] = {(cuuint64_t)cols * el, (cuuint64_t)stream_stride * el};
  cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over `streams` fp32 matrices [rows x cols] (matrix s at base + s *
// stream_stride elements), box = box_cols x box_rows x 1, no swizzle: rows of
// the box land in shared memory one after another (box_cols * 4 bytes each).
bool map3d_f32_plain(CUtensorMap *m, const float *base, int cols, int rows, int streams, long long stream_stride,
                     int box_cols, int box_rows) {
  EncodeTiledFn fn = encode_fn_l();
  if (!fn || (box_cols * 4) % 16 != 0 || box_cols > 256 || box_rows > 256) return false;
  std::memset(m, 0, sizeof *m);
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)streams};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 4, (cuuint64_t)stream_stride * 4};
  cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Workspace carve-up (bytes, 256-aligned pieces), per problem.
struct Carve {
  size_t coef, scal, wbf, x[kMaxL + 1], sp[kMaxL + 1], g[kMaxL + 1], gc[kMaxL + 1], ge[kMaxL + 1];
  size_t part, cnt, cnt_bytes;       // split-K partial sums and per-tile arrival counters
  size_t total;
};

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

bool fb_ok(const Problem &p);

// Widest output tile of a per-phase GEMM that divides n and still gives about
// one CTA per SM (S streams, mtiles row tiles).
int phase_tile(int n, int mtiles, int S) {
  for (int t = 256; t >= 64; t /= 2) {
    if (n % t) continue;
    if ((long long)S * mtiles * (n / t) >= 128 || t == 64) return t;
  }
  return 64;
}
// Split of a per-phase GEMM's reduction over several CTAs per output tile,
// for grids that leave most SMs idle and long reductions (K >= 1024): the
// partial tiles cost a store, a fence and a re-read, which shorter
// reductions do not earn back.
int phase_ksplit(long long ctas, int nk) {
  if (ctas >= 64 || nk < 16) return 1;
  for (int ks = kMaxSplit; ks >= 2; --ks)
    if (ctas * ks <= 148) return ks;
  return 1;
}
// Largest partial-sum buffer (bytes) and tile count of the split phases.
void phase_split_sizes(const Problem &p, size_t *part_bytes, size_t *tiles) {
  *part_bytes = 0;
  *tiles = 0;
  if (p.fuse_fb && fb_ok(p)) return;           // the fused kernel runs instead
  const int C = p.C, S = p.streams;
  auto one = [&](int n_out, int M, int K) {
    const int mtiles = (M + 127) / 128, N = phase_tile(n_out, mtiles, S);
    const long long ctas = (long long)S * mtiles * (n_out / N);
    const int ks = phase_ksplit(ctas, K / KB);
    if (ks > 1) {
      const size_t b = (size_t)ctas * ks * 128 * N * sizeof(float);
      if (b > *part_bytes) *part_bytes = b;
      if ((size_t)ctas > *tiles) *tiles = (size_t)ctas;
    }
  };
  for (int l = 1; l <= p.L; ++l) one(p.dims[l], 2 * C, p.dims[l - 1]);
  for (int l = p.L; l >= 2; --l) one(p.dims[l - 1], C, p.dims[l]);
}

Carve carve(const Problem &p) {
  Carve c{};
  size_t off = 0;
  const size_t S = (size_t)p.streams;
  auto take = [&](size_t bytes) { size_t o = off; off += up256(bytes); return o; };
  c.coef = take(S * p.T * 2 * sizeof(float));
  c.scal = take(S * (p.T / p.C) * 4 * sizeof(float));
  c.wbf = take(S * p.P * 2);
  for (int l = 1; l < p.L; ++l) {
    c.x[l] = take(S * 2 * p.C * p.dims[l] * 2);
    c.sp[l] = take(S * p.C * p.dims[l] * 2);
  }
  for (int l = 1; l <= p.L; ++l) {
    c.g[l] = take(S * p.C * p.dims[l] * 2);
    c.gc[l] = take(S * p.C * p.dims[l] * 2);
    c.ge[l] = take(S * p.C * p.dims[l] * 2);
  }
  size_t pb, nt;
  phase_split_sizes(p, &pb, &nt);
  c.part = pb ? take(pb) : 0;
  c.cnt = nt ? take(nt * sizeof(unsigned)) : 0;
  c.cnt_bytes = nt * sizeof(unsigned);
  c.total = off;
  return c;
}

bool dims_ok(const Problem &p) {
  for (int l = 0; l <= p.L; ++l)
    if (p.dims[l] % 64 != 0) return false;
  return true;
}

constexpr size_t SMEM_BYTES = 4 * STAGE_BYTES_MM + 1024;

bool fb_ok(const Problem &p) {
  for (int l = 0; l <= p.L; ++l)
    if (p.dims[l] > FB_MAXD) return false;
  return true;
}

cudaError_t launch_fb(const FbArgs &a, const FbMaps &m, int streams, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * a.C / 128), (unsigned)streams);
  cfg.blockDim = dim3(FB_NT);
  cfg.dynamicSmemBytes = FB_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tcl_fb_kernel, a, m);
}

cudaError_t launch_gemm(const GemmArgs &a, const CUtensorMap &mA, const CUtensorMap &mA2,
                        const CUtensorMap &mB, int streams, int mtiles, int ntiles, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ntiles, (unsigned)mtiles, (unsigned)(streams * a.ksplit));
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  switch (a.kind) {
    case K_FWD: return cudaLaunchKernelEx(&cfg, tcl_gemm_kernel<K_FWD>, a, mA, mA2, mB);
    case K_FWD_LAST: return cudaLaunchKernelEx(&cfg, tcl_gemm_kernel<K_FWD_LAST>, a, mA, mA2, mB);
    case K_BWD: return cudaLaunchKernelEx(&cfg, tcl_gemm_kernel<K_BWD>, a, mA, mA2, mB);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_up2(const Up2Args &a, const UpMaps &m, int units, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)units);
  cfg.blockDim = dim3(UP2_NT);
  cfg.dynamicSmemBytes = up2_smem(a.C);
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tcl_update2_kernel, a, m);
}

cudaError_t launch_up3(const Up3Args &a, const Up3Maps &m, int units, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)units);
  cfg.blockDim = dim3(UP3_NT);
  cfg.dynamicSmemBytes = UP3_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tcl_update3_kernel, a, m);
}

cudaError_t launch_up(const UpArgs &a, const UpMaps &m, int tiles, size_t smem, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)tiles);
  cfg.blockDim = dim3(UP_NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tcl_update_kernel, a, m);
}

}  // namespace

bool tcl_supported(const Problem &p) {
  if (p.in_dtype != TM_BF16) return false;
  if (p.C % 64 != 0 || p.C > 256) return false;
  if (!dims_ok(p)) return false;
  for (int l = 0; l <= p.L; ++l)
    if (p.dims[l] > 4096) return false;
  return true;
}


static unsigned long long g_tcl_wait_ns = 2000000000ull;
static int g_tcl_inject = 0;

namespace {

// Column tiles per unit of the pipelined update: 4 (longer pipelines) unless
// that leaves fewer than 32 CTAs per launch; TM_TCL_TPU (1..16), read once
// per process, overrides.
int up2_tiles_per_unit(const Problem &p) {
  static int forced = -1;
  if (forced < 0) {
    const char *e = std::getenv("TM_TCL_TPU");
    forced = e ? std::atoi(e) : 0;
    if (forced < 0 || forced > 16) forced = 0;
  }
  if (forced) return forced;
  for (int tpu = 4; tpu > 1; tpu /= 2) {
    long long units = 0;
    for (int l = 1; l <= p.L; ++l)
      units += (long long)p.streams * ((p.dims[l] + 127) / 128) * ((p.dims[l - 1] / 64 + tpu - 1) / tpu);
    if (units >= 32) return tpu;
  }
  return 1;
}

// One group of streams: its slice of every tensor, its own workspace carve
// and CUDA stream, and everything its launches need.
struct TclGroup {
  Problem p;
  cudaStream_t st;
  Carve cv;
  unsigned char *ws;
  float *coef, *scal;
  op_t *wbf;
  int L, C, T, S, nchunks;
  InitArgs ia;
  CUtensorMap mk, mq, mwb[kMaxL + 1], mx[kMaxL + 1], mg[kMaxL + 1], mgc[kMaxL + 1], mge[kMaxL + 1];
  GemmArgs base;
  UpArgs ua;
  UpMaps um;
  int up_tiles;
  size_t up_smem_bytes;
  bool up2;                      // pipelined update kernel (C <= 128)
  bool up3;                      // transposed update kernel (C <= 128, input widths multiples of 128)
  Up3Args ua3;
  Up3Maps um3;
  int up3_units;
  Up2Args ua2;
  int up2_units;
  bool fused;
  FbArgs fa;
  FbMaps fm;

  op_t *bf(size_t off) const { return reinterpret_cast<op_t *>(ws + off); }
  // Widest tile that divides n and still gives about one CTA per SM.
  int tile_for(int n, int mtiles) const { return phase_tile(n, mtiles, S); }
  cudaError_t setup();
  cudaError_t chunk(int ch);
};

cudaError_t TclGroup::setup() {
  cv = carve(p);
  ws = static_cast<unsigned char *>(p.scratch);
  coef = reinterpret_cast<float *>(ws + cv.coef);
  scal = reinterpret_cast<float *>(ws + cv.scal);
  wbf = reinterpret_cast<op_t *>(ws + cv.wbf);
  L = p.L; C = p.C; T = p.T; S = p.streams; nchunks = p.T_run / C;
  const int d = p.dims[0];
  cudaStream_t stream = st;

  ia.W0 = p.W0; ia.S0 = p.S0; ia.W = p.W_end; ia.S = p.S_end; ia.Wbf = wbf;
  ia.P = (long long)p.P; ia.streams = S; ia.L = L;
  long long bo = 0;
  for (int l = 0; l <= L; ++l) ia.off[l] = (long long)p.layer_off[l];
  for (int l = 0; l < L; ++l) {
    ia.boff[l] = bo;
    bo += (long long)S * p.dims[l + 1] * p.dims[l];
  }
  ia.boff[L] = bo;
  tcl_init_kernel<<<592, 256, 0, stream>>>(ia);
  const long long nct = (long long)S * nchunks;
  tcl_coef_kernel<<<(unsigned)((nct * 32 + 127) / 128), 128, 0, stream>>>(p.theta, p.eta, p.alpha, S, T, C,
                                                                          nchunks, coef, scal);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  // tensor maps, built once per call
  if (!map2d(&mk, p.k16, (long long)S * T, d, 64) || !map2d(&mq, p.q16, (long long)S * T, d, 64))
    return cudaErrorInvalidValue;
  for (int l = 1; l <= L; ++l) {
    const int nl = p.dims[l], np = p.dims[l - 1];
    if (!map2d(&mwb[l], wbf + ia.boff[l - 1], (long long)S * nl, np, 64)) return cudaErrorInvalidValue;
    if (!map2d(&mg[l], bf(cv.g[l]), (long long)S * C, nl, 64) ||
        !map2d(&mgc[l], bf(cv.gc[l]), (long long)S * C, nl, 64) ||
        !map2d(&mge[l], bf(cv.ge[l]), (long long)S * C, nl, 64))
      return cudaErrorInvalidValue;
    if (l < L && !map2d(&mx[l], bf(cv.x[l]), (long long)S * 2 * C, nl, 64)) return cudaErrorInvalidValue;
  }

  std::memset(&base, 0, sizeof base);
  base.C = C;
  base.T = T;
  base.streams = S;
  base.ksplit = 1;
  if (cv.part) base.part = reinterpret_cast<float *>(ws + cv.part);
  if (cv.cnt) {
    base.cnt = reinterpret_cast<unsigned *>(ws + cv.cnt);
    err = cudaMemsetAsync(base.cnt, 0, cv.cnt_bytes, stream);   // each split tile's last CTA resets its counter
    if (err != cudaSuccess) return err;
  }
  base.coef = coef;
  base.status = p.status;
  base.wait_ns = g_tcl_wait_ns;
  base.inject = g_tcl_inject;
  base.y = p.y;
  base.v = reinterpret_cast<const __nv_bfloat16 *>(p.v);

  // the update launch: per layer, tiles of 128 rows of W_l x (128 or 64) columns
  std::memset(&ua, 0, sizeof ua);
  std::memset(&um, 0, sizeof um);
  ua.L = L;
  ua.C = C;
  ua.nchunks = nchunks;
  ua.scal = scal;
  ua.status = p.status;
  ua.wait_ns = g_tcl_wait_ns;
  ua.inject = g_tcl_inject;
  up_tiles = 0;
  up_smem_bytes = 0;
  for (int l = 1; l <= L; ++l) {
    UpLayer &u = ua.l[l - 1];
    const int nl = p.dims[l], np = p.dims[l - 1];
    u.M = nl;
    u.N = up_width(np, C);
    u.mtiles = (nl + 127) / 128;
    u.ntiles = np / u.N;
    u.first = up_tiles;
    u.b_rows_per_stream = l == 1 ? T : 2 * C;
    up_tiles += S * u.mtiles * u.ntiles;
    um.a[l - 1] = mgc[l];
    um.a2[l - 1] = mge[l];
    um.b[l - 1] = l == 1 ? mk : mx[l - 1];
    const int br = nl < 128 ? nl : 128;
    if (!map3d(&um.w[l - 1], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.W_end + p.layer_off[l - 1], np, nl, S,
               (long long)p.P, 32, br) ||
        !map3d(&um.s[l - 1], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.S_end + p.layer_off[l - 1], np, nl, S,
               (long long)p.P, 32, br) ||
        !map3d(&um.wb[l - 1], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, wbf + ia.boff[l - 1], np, nl, S,
               (long long)nl * np, 64, br))
      return cudaErrorInvalidValue;
    const size_t sm = up_smem(u.N, C / KB);
    if (sm > up_smem_bytes) up_smem_bytes = sm;
  }

  // the pipelined update: units of (layer, stream, 128-row block, range of
  // up to tpu 64-column tiles)
  up2 = C <= 128;
  if (up2) {
    std::memset(&ua2, 0, sizeof ua2);
    ua2.L = L;
    ua2.C = C;
    ua2.nchunks = nchunks;
    ua2.scal = scal;
    ua2.status = p.status;
    ua2.wait_ns = g_tcl_wait_ns;
    ua2.inject = g_tcl_inject;
    ua2.tpu = up2_tiles_per_unit(p);
    up2_units = 0;
    for (int l = 1; l <= L; ++l) {
      Up2Layer &u = ua2.l[l - 1];
      u.M = p.dims[l];
      u.mtiles = (p.dims[l] + 127) / 128;
      u.ntiles = p.dims[l - 1] / 64;
      u.nranges = (u.ntiles + ua2.tpu - 1) / ua2.tpu;
      u.first = up2_units;
      u.b_rows_per_stream = l == 1 ? T : 2 * C;
      u.wb = wbf + ia.boff[l - 1];
      up2_units += S * u.mtiles * u.nranges;
    }
  }

  // the transposed update: units of (layer, stream, 256-row block, 128-column block)
  up3 = up2;
  for (int l = 1; l <= L; ++l)
    if (p.dims[l - 1] % 128 != 0 || p.dims[l] % 64 != 0) up3 = false;
  if (up3) {
    std::memset(&ua3, 0, sizeof ua3);
    std::memset(&um3, 0, sizeof um3);
    ua3.L = L;
    ua3.C = C;
    ua3.nchunks = nchunks;
    ua3.P = (long long)p.P;
    ua3.scal = scal;
    ua3.status = p.status;
    ua3.wait_ns = g_tcl_wait_ns;
    ua3.inject = g_tcl_inject;
    up3_units = 0;
    for (int l = 1; l <= L; ++l) {
      Up3Layer &u = ua3.l[l - 1];
      u.M = p.dims[l];
      u.cols = p.dims[l - 1];
      u.rblocks = (u.M + 255) / 256;
      u.cblocks = u.cols / 128;
      u.first = up3_units;
      u.b_rows_per_stream = l == 1 ? T : 2 * C;
      u.w = p.W_end + p.layer_off[l - 1];
      u.s = p.S_end + p.layer_off[l - 1];
      u.wb = wbf + ia.boff[l - 1];
      up3_units += S * u.rblocks * u.cblocks;
      um3.a[l - 1] = mgc[l];
      um3.a2[l - 1] = mge[l];
      um3.b[l - 1] = l == 1 ? mk : mx[l - 1];
      if (!map3d_f32_plain(&um3.w[l - 1], u.w, u.cols, u.M, S, (long long)p.P, 128, 16) ||
          !map3d_f32_plain(&um3.s[l - 1], u.s, u.cols, u.M, S, (long long)p.P, 128, 16))
        return cudaErrorInvalidValue;
    }
  }

  fused = p.fuse_fb && fb_ok(p);
  if (fused) {
    std::memset(&fa, 0, sizeof fa);
    std::memset(&fm, 0, sizeof fm);
    fa.L = L;
    fa.C = C;
    fa.T = T;
    for (int l = 0; l <= L; ++l) fa.dims[l] = p.dims[l];
    for (int l = 1; l <= L; ++l) {
      if (l < L) { fa.x_out[l] = bf(cv.x[l]); fa.sp_out[l] = bf(cv.sp[l]); }
      fa.gc_out[l] = bf(cv.gc[l]);
      fa.ge_out[l] = bf(cv.ge[l]);
      fm.w[l] = mwb[l];
    }
    fm.k = mk;
    fm.q = mq;
    fa.y = p.y;
    fa.v = reinterpret_cast<const __nv_bfloat16 *>(p.v);
    fa.coef = coef;
    fa.status = p.status;
    fa.wait_ns = g_tcl_wait_ns;
    fa.inject = g_tcl_inject;
  }
  return cudaSuccess;
}

cudaError_t TclGroup::chunk(int ch) {
  cudaStream_t stream = st;
  cudaError_t err = cudaSuccess;
  if (fused) {
    fa.chunk = ch;
    err = launch_fb(fa, fm, S, stream);
    if (err != cudaSuccess) return err;
  }
  // forward of keys and queries, layer by layer
  for (int l = 1; l <= L && !fused; ++l) {
    GemmArgs a = base;
    const int nl = p.dims[l], np = p.dims[l - 1];
    a.kind = l < L ? K_FWD : K_FWD_LAST;
    a.chunk = ch;
    a.N = tile_for(nl, 2 * C / 128);
    a.K = np;
    a.M = 2 * C;
    a.n_out = nl;
    a.a_split_kq = l == 1;
    a.a_rows_per_stream = 2 * C;
    a.b_rows_per_stream = nl;
    a.ksplit = base.cnt ? phase_ksplit((long long)S * (2 * C / 128) * (nl / a.N), np / KB) : 1;
    if (l < L) { a.x_out = bf(cv.x[l]); a.sp_out = bf(cv.sp[l]); }
    a.g_out = bf(cv.g[L]); a.gc_out = bf(cv.gc[L]); a.ge_out = bf(cv.ge[L]);
    err = launch_gemm(a, l == 1 ? mk : mx[l - 1], mq, mwb[l], S, 2 * C / 128, nl / a.N, stream);
    if (err != cudaSuccess) return err;
  }
  // backward to every hidden layer
  for (int l = L; l >= 2 && !fused; --l) {
    GemmArgs a = base;
    const int nl = p.dims[l], np = p.dims[l - 1];
    a.kind = K_BWD;
    a.chunk = ch;
    a.N = tile_for(np, (C + 127) / 128);
    a.K = nl;
    a.M = C;
    a.n_out = np;
    a.a_rows_per_stream = C;
    a.b_rows_per_stream = nl;
    a.ksplit = base.cnt ? phase_ksplit((long long)S * ((C + 127) / 128) * (np / a.N), nl / KB) : 1;
    a.sp_in = bf(cv.sp[l - 1]);
    a.g_out = bf(cv.g[l - 1]); a.gc_out = bf(cv.gc[l - 1]); a.ge_out = bf(cv.ge[l - 1]);
    err = launch_gemm(a, mg[l], mg[l], mwb[l], S, (C + 127) / 128, np / a.N, stream);
    if (err != cudaSuccess) return err;
  }
  // weight-update contractions of every layer, with the fused state update
  if (up3) {
    ua3.chunk = ch;
    ua3.l[0].b_row_off = (long long)ch * C;
    return launch_up3(ua3, um3, up3_units, stream);
  }
  if (up2) {
    ua2.chunk = ch;
    ua2.l[0].b_row_off = (long long)ch * C;
    return launch_up2(ua2, um, up2_units, stream);
  }
  ua.chunk = ch;
  ua.l[0].b_row_off = (long long)ch * C;
  return launch_up(ua, um, up_tiles, up_smem_bytes, stream);
}

// Streams split into groups issued on separate CUDA streams: one group's
// (latency-bound) forward/backward kernel runs beside another group's
// (bandwidth-bound) update. TM_TCL_GROUPS (1..8) overrides the choice.
int tcl_groups(const Problem &p) {
  static int forced = -1;
  if (forced < 0) {
    const char *e = std::getenv("TM_TCL_GROUPS");
    forced = e ? std::atoi(e) : 0;
    if (forced < 0 || forced > kMaxGroups) forced = 0;
  }
  // about eight streams per group (measured on the depth-4 workload, 64
  // streams: 1 group 32.5 ms, 2: 30.8, 4: 26.4, 8: 25.4)
  int g = forced ? forced : p.streams / 8;
  if (g > kMaxGroups) g = kMaxGroups;
  if (g > p.streams) g = p.streams;
  return g < 1 ? 1 : g;
}

Problem group_slice(const Problem &p, int g, int groups) {
  const int s0 = (int)((long long)p.streams * g / groups), s1 = (int)((long long)p.streams * (g + 1) / groups);
  Problem q = p;
  const size_t el = p.in_dtype == TM_BF16 ? 2 : 4;
  const size_t td = (size_t)p.T * p.dims[0];
  q.streams = s1 - s0;
  q.B = 1;
  q.H = q.streams;
  q.k = static_cast<const char *>(p.k) + s0 * td * el;
  q.v = static_cast<const char *>(p.v) + s0 * td * el;
  q.q = static_cast<const char *>(p.q) + s0 * td * el;
  q.k16 = static_cast<const char *>(p.k16) + s0 * td * 2;   // fp16 copies
  q.q16 = static_cast<const char *>(p.q16) + s0 * td * 2;
  q.theta = p.theta + (size_t)s0 * p.T;
  q.eta = p.eta + (size_t)s0 * p.T;
  q.alpha = p.alpha + (size_t)s0 * p.T;
  q.W0 = p.W0 + (size_t)s0 * p.P;
  q.S0 = p.S0 + (size_t)s0 * p.P;
  q.W_end = p.W_end + (size_t)s0 * p.P;
  q.S_end = p.S_end + (size_t)s0 * p.P;
  q.y = p.y + (size_t)s0 * td;
  return q;
}

size_t group_bytes(const Problem &p, int groups) {
  size_t m = 0;
  for (int g = 0; g < groups; ++g) {
    const size_t b = carve(group_slice(p, g, groups)).total;
    if (b > m) m = b;
  }
  return m;
}

}  // namespace

size_t tcl_scratch_bytes(const Problem &p) {
  const int G = tcl_groups(p);
  return (size_t)G * group_bytes(p, G);
}

int tcl_group_count(const Problem &p) { return tcl_supported(p) ? tcl_groups(p) : 1; }

long long tcl_launch_count(const Problem &p) {
  // per group: init and coefficient kernels, then per chunk the fused
  // forward + backward (or 2L - 1 phase launches) and one update launch
  const long long per_chunk = (p.fuse_fb && fb_ok(p)) ? 2 : 2LL * p.L;
  return (long long)tcl_group_count(p) * (2 + per_chunk * (p.T_run / p.C));
}

cudaError_t tcl_launch(const Problem &p, cudaStream_t stream) {
  if (!tcl_supported(p)) return cudaErrorNotSupported;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaSuccess;
    const void *kerns[3] = {(const void *)tcl_gemm_kernel<K_FWD>, (const void *)tcl_gemm_kernel<K_FWD_LAST>,
                            (const void *)tcl_gemm_kernel<K_BWD>};
    for (const void *k : kerns) {
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
      if (e != cudaSuccess) return e;
    }
    e = cudaFuncSetAttribute(tcl_fb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FB_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tcl_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)up_smem(128, 2));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tcl_update2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)up2_smem(128));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tcl_update3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)UP3_SMEM);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const int G = tcl_groups(p);
  if (G > 1 && (!p.side_streams[G - 2] || !p.ev_fork || !p.ev_join[G - 2])) return cudaErrorInvalidValue;
  const size_t gb = group_bytes(p, G);
  std::vector<TclGroup> groups((size_t)G);
  cudaError_t err = cudaSuccess;
  if (G > 1) {
    err = cudaEventRecord(static_cast<cudaEvent_t>(p.ev_fork), stream);
    for (int g = 1; g < G && err == cudaSuccess; ++g)
      err = cudaStreamWaitEvent(static_cast<cudaStream_t>(p.side_streams[g - 1]),
                                static_cast<cudaEvent_t>(p.ev_fork), 0);
    if (err != cudaSuccess) return err;
  }
  for (int g = 0; g < G && err == cudaSuccess; ++g) {
    TclGroup &t = groups[(size_t)g];
    t.p = group_slice(p, g, G);
    t.p.scratch = static_cast<unsigned char *>(p.scratch) + (size_t)g * gb;
    t.p.scratch_bytes = gb;
    t.st = g == 0 ? stream : static_cast<cudaStream_t>(p.side_streams[g - 1]);
    err = t.setup();
  }
  // launches of the groups interleaved chunk by chunk
  const int nchunks = p.T_run / p.C;
  for (int ch = 0; ch < nchunks && err == cudaSuccess; ++ch)
    for (int g = 0; g < G && err == cudaSuccess; ++g) err = groups[(size_t)g].chunk(ch);
  if (G > 1) {
    // join (also after an error, so that the caller's stream never runs ahead
    // of work already queued on the side streams)
    for (int g = 1; g < G; ++g) {
      cudaEvent_t ev = static_cast<cudaEvent_t>(p.ev_join[g - 1]);
      if (cudaEventRecord(ev, static_cast<cudaStream_t>(p.side_streams[g - 1])) == cudaSuccess)
        cudaStreamWaitEvent(stream, ev, 0);
    }
  }
  return err;
}

void tcl_set_debug(int inject_timeout, unsigned long long wait_ns) {
  g_tcl_inject = inject_timeout ? 1 : 0;
  g_tcl_wait_ns = wait_ns ? wait_ns : 2000000000ull;
}
unsigned long long tcl_wait_ns() { return g_tcl_wait_ns; }
int tcl_inject() { return g_tcl_inject; }

}  // namespace tmem
