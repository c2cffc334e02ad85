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
//              caller's W_end / S_end) and the bf16 copy of W' for the next chunk
// ("Titans, explained" steps 2-6; "Attack of the Titans", "Parallel
//  training"). Launch order on one stream orders the phases; every kernel is
// one output tile per CTA: TMA loads (128-byte swizzle) into a ring of
// shared-memory stages, tcgen05 MMAs into TMEM, a 4-warp epilogue. Each
// stream's tiles are independent (batched over streams).
#include <cuda.h>
#include <cuda_bf16.h>

#include <cstring>

#include "tm_internal.h"
#include "tm_sm100.cuh"

namespace tmem {
namespace {

using namespace sm100;

constexpr int NT = 256;          // 8 warps: warp w reads TMEM lanes 32 (w % 4) .. +31,
                                 // columns half w / 4 of the tile
constexpr int KB = 64;           // K block (one 128-byte swizzle atom of bf16)

enum Kind { K_FWD = 0, K_FWD_LAST = 1, K_BWD = 2, K_DW = 3 };

struct GemmArgs {
  int kind;
  int C, T, chunk;               // chunk size, tokens per stream, chunk index
  int M, N, K;                   // per-stream GEMM: rows, cols, reduction
  int n_out;                     // row length of the epilogue's outputs
  int a_rows_per_stream;         // rows of the A source per stream
  int b_rows_per_stream;
  int a_split_kq;                // layer-1 forward: rows < C from k, else from q
  long long b_row_off;           // added to B's row coordinate (update of layer 1: keys)
  // epilogue operands
  __nv_bfloat16 *x_out;          // [streams, 2C, n] activations (forward)
  __nv_bfloat16 *sp_out;         // [streams, C, n] silu'(Z) of key rows (forward)
  const __nv_bfloat16 *sp_in;    // [streams, C, n] silu' of the layer below (backward)
  __nv_bfloat16 *g_out, *gc_out, *ge_out;  // [streams, C, n] G, -c G, -e G
  float *y;                      // [streams, T, d] reads (last forward)
  const __nv_bfloat16 *v;        // [streams, T, d] values (last forward)
  const float *coef;             // [streams, T, 2] (c, e) per token
  const float *scal;             // [streams, nchunks, 4] (B, A, cS, -)
  float *W, *S;                  // fp32 state of this layer: [streams] x P stride
  __nv_bfloat16 *Wbf;            // bf16 copy of this layer: [streams, M, N]
  long long P, layer_off;
  int nchunks;
  int *status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigm(float z) { return fmaf(0.5f, tanh_approx(0.5f * z), 0.5f); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint4 pack8(const float *v) {
  return make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                    pack_bf16(v[6], v[7]));
}

__device__ bool wait_b(uint64_t *bar, uint32_t par, const GemmArgs &a) {
  if (mbar_wait(bar, par, a.wait_ns)) return true;
  atomicCAS(a.status, 0, kDevTimeout);
  return false;
}

// Shared-memory stage: A tile [128 rows x 64 k] (K-major) or, for the update
// GEMM, two MN-major A tiles [64 tokens x 128] (c and e); B tile up to
// [256 x 64] (K-major) or [64 x 256] (MN-major). All in the row-block layout.
constexpr uint32_t A_BYTES = 128 * KB * 2;       // 16 KB
constexpr uint32_t B_BYTES = 256 * KB * 2;       // 32 KB
constexpr uint32_t STAGE_BYTES_DW = 2 * A_BYTES + B_BYTES;   // 64 KB, 3 stages
constexpr uint32_t STAGE_BYTES_MM = A_BYTES + B_BYTES;       // 48 KB, 4 stages
constexpr int STAGES_MAX = 4;

// A tile loads. mt: 128-row tile index (forward/backward) or 128-column tile
// of the transposed operand (update).
__device__ __forceinline__ void load_stage(const GemmArgs &a, const CUtensorMap *mA,
                                           const CUtensorMap *mA2, const CUtensorMap *mB,
                                           unsigned char *st, uint64_t *bar, int s, int mt,
                                           int nt, int kb) {
  const int kind = a.kind;
  if (kind == K_DW) {
    // A^T operands: -c G and -e G, rows = tokens (K), features = rows of W (M)
    // B: X_{l-1}, rows = tokens (K), features = N. All MN-major.
    const int row0 = s * a.a_rows_per_stream + kb * KB;
    for (int f = 0; f < 2; ++f) {
      tma_load_2d(st + f * 64 * 128, mA, bar, 128 * mt + 64 * f, row0);
      tma_load_2d(st + A_BYTES + f * 64 * 128, mA2, bar, 128 * mt + 64 * f, row0);
    }
    const int brow0 = (int)(s * a.b_rows_per_stream + a.b_row_off) + kb * KB;
    for (int f = 0; f < a.N / 64; ++f)
      tma_load_2d(st + 2 * A_BYTES + f * 64 * 128, mB, bar, a.N * nt + 64 * f, brow0);
    return;  // DW stage: [A_c | A_e | B]
  }
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

__global__ void __launch_bounds__(NT, 1)
    tcl_gemm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap mA,
                    const __grid_constant__ CUtensorMap mA2, const __grid_constant__ CUtensorMap mB) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *sm =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[STAGES_MAX], empty[STAGES_MAX], done;
  __shared__ uint32_t tslot;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int s = blockIdx.z, mt = blockIdx.y, nt = blockIdx.x;
  const int kind = a.kind;
  const int nk = a.K / KB;
  const uint32_t ncols = kind == K_DW ? 512u : 256u;
  const int STAGES = kind == K_DW ? 3 : 4;
  const uint32_t STAGE_BYTES = kind == K_DW ? STAGE_BYTES_DW : STAGE_BYTES_MM;

  if (tid == 0) {
    for (int i = 0; i < STAGES_MAX; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(&done, 1);
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
    const uint32_t tx = kind == K_DW ? (uint32_t)(2 * A_BYTES + (uint32_t)a.N * KB * 2)
                                     : (uint32_t)(A_BYTES + (uint32_t)a.N * KB * 2);
    uint32_t idesc;
    if (kind == K_DW) idesc = idesc_bf16(128, a.N, true, true);
    else if (kind == K_BWD) idesc = idesc_bf16(128, a.N, false, true);
    else idesc = idesc_bf16(128, a.N, false, false);
    for (int kb = 0; kb < nk && kb < STAGES; ++kb) {
      mbar_arrive_expect_tx(&full[kb], tx);
      load_stage(a, &mA, &mA2, &mB, sm + kb * STAGE_BYTES, &full[kb], s, mt, nt, kb);
    }
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int st = kb % STAGES;
      const uint32_t ph = (uint32_t)((kb / STAGES) & 1);
      if (!wait_b(&full[st], ph, a)) { ok = false; break; }
      tc_fence_after();
      const uint32_t base = smem_u32(sm + st * STAGE_BYTES);
      for (int ks = 0; ks < KB / 16; ++ks) {
        if (kind == K_DW) {
          const uint64_t bd = desc_mnmajor(base + 2 * A_BYTES, 64, ks);
          umma_bf16(tm, desc_mnmajor(base, 64, ks), bd, idesc, (kb | ks) != 0);
          umma_bf16(tm + 256, desc_mnmajor(base + A_BYTES, 64, ks), bd, idesc, (kb | ks) != 0);
        } else if (kind == K_BWD) {
          umma_bf16(tm, desc_kmajor(base, 128, ks), desc_mnmajor(base + A_BYTES, 64, ks), idesc,
                    (kb | ks) != 0);
        } else {
          umma_bf16(tm, desc_kmajor(base, 128, ks), desc_kmajor(base + A_BYTES, a.N, ks), idesc,
                    (kb | ks) != 0);
        }
      }
      umma_commit(&empty[st]);
      if (kb + STAGES < nk) {
        if (!wait_b(&empty[st], ph, a)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[st], tx);
        load_stage(a, &mA, &mA2, &mB, sm + st * STAGE_BYTES, &full[st], s, mt, nt, kb + STAGES);
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
  const int row = 32 * (warp & 3) + lane;        // TMEM lane = output row of the tile
  const uint32_t lb = (uint32_t)(32 * (warp & 3)) << 16;
  const int half = warp >> 2;                    // this warp's half of the tile's columns
  const int cbeg = half * (a.N / 2), cend = cbeg + a.N / 2;
  if (ok) {
    if (kind == K_FWD || kind == K_FWD_LAST || kind == K_BWD) {
      const int r = 128 * mt + row;              // row of the per-stream matrix
      const bool key = r < a.C;
      const bool valid = (kind == K_BWD) ? key : (r < 2 * a.C);
      for (int c0 = cbeg; c0 < cend; c0 += 16) {
        float z[16];
        tmem_ld16(tm + lb + c0, z);
        tmem_wait_ld();
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
          __nv_bfloat16 *xo = a.x_out + ((long long)s * 2 * a.C + r) * a.n_out + col;
          *reinterpret_cast<uint4 *>(xo) = pack8(x);
          *reinterpret_cast<uint4 *>(xo + 8) = pack8(x + 8);
          if (key) {
            __nv_bfloat16 *so = a.sp_out + ((long long)s * a.C + r) * a.n_out + col;
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
            const __nv_bfloat16 *spi = a.sp_in + ((long long)s * a.C + r) * a.n_out + col;
            const uint4 s0 = *reinterpret_cast<const uint4 *>(spi);
            const uint4 s1 = *reinterpret_cast<const uint4 *>(spi + 8);
            const __nv_bfloat16 *sb0 = reinterpret_cast<const __nv_bfloat16 *>(&s0);
            const __nv_bfloat16 *sb1 = reinterpret_cast<const __nv_bfloat16 *>(&s1);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              g[i] = z[i] * __bfloat162float(sb0[i]);
              g[8 + i] = z[8 + i] * __bfloat162float(sb1[i]);
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
    } else {
      // update: row of W_l = 128 mt + row, columns N nt + [0, N)
      const int wr = 128 * mt + row;
      const bool valid = wr < a.M;
      const float4 sc = *reinterpret_cast<const float4 *>(a.scal + 4 * ((long long)s * a.nchunks + a.chunk));
      float *Wl = a.W + (long long)s * a.P + a.layer_off;
      float *Sl = a.S + (long long)s * a.P + a.layer_off;
      for (int c0 = cbeg; c0 < cend; c0 += 64) {
        const int col = a.N * nt + c0;
        const long long g = (long long)wr * a.n_out + col;
        const int ncol = cend - c0 < 64 ? cend - c0 : 64;  // 64, or 32 for a 64-wide tile
        // all of this thread's W and S loads of the piece in flight at once
        float4 w4[16], s4[16];
        if (valid) {
#pragma unroll
          for (int i4 = 0; i4 < 16; ++i4) {
            if (4 * i4 < ncol) {
              w4[i4] = *reinterpret_cast<const float4 *>(Wl + g + 4 * i4);
              s4[i4] = *reinterpret_cast<const float4 *>(Sl + g + 4 * i4);
            }
          }
        }
#pragma unroll
        for (int q16 = 0; q16 < 4; ++q16) {
          if (16 * q16 >= ncol) break;
          float uw[16], us[16];
          tmem_ld16(tm + lb + c0 + 16 * q16, uw);
          tmem_ld16(tm + lb + 256 + c0 + 16 * q16, us);
          tmem_wait_ld();
          if (!valid) continue;
          float w[16], sv[16];
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) {
            const float4 a4 = w4[4 * q16 + i4], b4 = s4[4 * q16 + i4];
            w[4 * i4] = a4.x; w[4 * i4 + 1] = a4.y; w[4 * i4 + 2] = a4.z; w[4 * i4 + 3] = a4.w;
            sv[4 * i4] = b4.x; sv[4 * i4 + 1] = b4.y; sv[4 * i4 + 2] = b4.z; sv[4 * i4 + 3] = b4.w;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            w[i] = sc.x * w[i] + sc.z * sv[i] + uw[i];
            sv[i] = sc.y * sv[i] + us[i];
          }
          const long long gq = g + 16 * q16;
#pragma unroll
          for (int i4 = 0; i4 < 4; ++i4) {
            *reinterpret_cast<float4 *>(Wl + gq + 4 * i4) = make_float4(w[4 * i4], w[4 * i4 + 1], w[4 * i4 + 2], w[4 * i4 + 3]);
            *reinterpret_cast<float4 *>(Sl + gq + 4 * i4) = make_float4(sv[4 * i4], sv[4 * i4 + 1], sv[4 * i4 + 2], sv[4 * i4 + 3]);
          }
          __nv_bfloat16 *wb = a.Wbf + (long long)s * a.M * a.n_out + gq;
          *reinterpret_cast<uint4 *>(wb) = pack8(w);
          *reinterpret_cast<uint4 *>(wb + 8) = pack8(w + 8);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, ncols);
}

// A5 for every chunk of every stream at once: one thread per (stream, chunk)
// runs the reverse recurrence over its C tokens (0-based i within the chunk):
//   pa_i = prod_{j>i}(1 - alpha_j), pe_i = prod_{j>i} eta_j,
//   r_{C-1} = 1, r_i = pa_i + eta_{i+1} r_{i+1};  c_i = theta_i r_i, e_i = theta_i pe_i;
//   B = prod(1 - alpha), A = prod eta, c_S = eta_0 r_0.
__global__ void tcl_coef_kernel(const float *theta, const float *eta, const float *alpha, int streams,
                                int T, int C, float *coef, float *scal) {
  const int nchunks = T / C;
  const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= (long long)streams * nchunks) return;
  const long long s = id / nchunks, ch = id % nchunks;
  const long long t0 = s * T + ch * C;
  float pa = 1.f, pe = 1.f, r = 1.f;
  for (int i = C - 1; i >= 0; --i) {
    if (i < C - 1) {
      pa *= 1.f - alpha[t0 + i + 1];
      pe *= eta[t0 + i + 1];
      r = pa + eta[t0 + i + 1] * r;
    }
    coef[2 * (t0 + i)] = theta[t0 + i] * r;
    coef[2 * (t0 + i) + 1] = theta[t0 + i] * pe;
  }
  float *o = scal + 4 * id;
  o[0] = pa * (1.f - alpha[t0]);
  o[1] = pe * eta[t0];
  o[2] = eta[t0] * r;
  o[3] = 0.f;
}

// Copy W0/S0 into W_end/S_end (unless in place) and build the bf16 operand
// copies, stored layer-major ([streams, n_l, n_{l-1}] per layer) so that one
// 2-D tensor map covers a layer of every stream.
struct InitArgs {
  const float *W0, *S0;
  float *W, *S;
  __nv_bfloat16 *Wbf;
  long long P;
  long long streams;
  int L;
  long long off[kMaxL + 1];      // layer offsets inside a parameter vector
  long long boff[kMaxL + 1];     // layer offsets inside the bf16 copy
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
    a.Wbf[a.boff[l] + s * per + within] = __float2bfloat16_rn(w);
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

// 2-D bf16 map over [rows x cols], box = 64 columns x box_rows rows, 128B swizzle.
bool map2d(CUtensorMap *m, const void *base, long long rows, int cols, int box_rows) {
  EncodeTiledFn fn = encode_fn_l();
  if (!fn) return false;
  std::memset(m, 0, sizeof *m);
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Workspace carve-up (bytes, 256-aligned pieces), per problem.
struct Carve {
  size_t coef, scal, wbf, x[kMaxL + 1], sp[kMaxL + 1], g[kMaxL + 1], gc[kMaxL + 1], ge[kMaxL + 1];
  size_t total;
};

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

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
  c.total = off;
  return c;
}

bool dims_ok(const Problem &p) {
  for (int l = 0; l <= p.L; ++l)
    if (p.dims[l] % 64 != 0) return false;
  return true;
}

constexpr size_t SMEM_BYTES = 3 * STAGE_BYTES_DW + 1024;   // = 4 * STAGE_BYTES_MM + 1024

cudaError_t launch_gemm(const GemmArgs &a, const CUtensorMap &mA, const CUtensorMap &mA2,
                        const CUtensorMap &mB, int streams, int mtiles, int ntiles, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ntiles, (unsigned)mtiles, (unsigned)streams);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tcl_gemm_kernel, a, mA, mA2, mB);
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

size_t tcl_scratch_bytes(const Problem &p) { return carve(p).total; }

static unsigned long long g_tcl_wait_ns = 2000000000ull;

cudaError_t tcl_launch(const Problem &p, cudaStream_t stream) {
  if (!tcl_supported(p)) return cudaErrorNotSupported;
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(tcl_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const Carve cv = carve(p);
  unsigned char *ws = static_cast<unsigned char *>(p.scratch);
  float *coef = reinterpret_cast<float *>(ws + cv.coef);
  float *scal = reinterpret_cast<float *>(ws + cv.scal);
  __nv_bfloat16 *wbf = reinterpret_cast<__nv_bfloat16 *>(ws + cv.wbf);
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16 *>(ws + off); };
  const int L = p.L, C = p.C, T = p.T, S = p.streams, nchunks = T / C;
  const int d = p.dims[0];

  InitArgs ia;
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
  tcl_coef_kernel<<<(unsigned)((nct + 127) / 128), 128, 0, stream>>>(p.theta, p.eta, p.alpha, S, T, C,
                                                                     coef, scal);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;

  // tensor maps, built once per call
  CUtensorMap mk, mq, mwb[kMaxL + 1], mx[kMaxL + 1], mg[kMaxL + 1], mgc[kMaxL + 1], mge[kMaxL + 1];
  if (!map2d(&mk, p.k, (long long)S * T, d, 64) || !map2d(&mq, p.q, (long long)S * T, d, 64))
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
  // Widest tile that divides n and still gives about one CTA per SM.
  auto tile_for = [&](int n, int mtiles) {
    for (int t = 256; t >= 64; t /= 2) {
      if (n % t) continue;
      if ((long long)S * mtiles * (n / t) >= 128 || t == 64) return t;
    }
    return 64;
  };

  GemmArgs base;
  std::memset(&base, 0, sizeof base);
  base.C = C;
  base.T = T;
  base.coef = coef;
  base.scal = scal;
  base.W = p.W_end;
  base.S = p.S_end;
  base.P = (long long)p.P;
  base.nchunks = nchunks;
  base.status = p.status;
  base.wait_ns = g_tcl_wait_ns;
  base.y = p.y;
  base.v = reinterpret_cast<const __nv_bfloat16 *>(p.v);

  for (int ch = 0; ch < nchunks; ++ch) {
    // forward of keys and queries, layer by layer
    for (int l = 1; l <= L; ++l) {
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
      if (l < L) { a.x_out = bf(cv.x[l]); a.sp_out = bf(cv.sp[l]); }
      a.g_out = bf(cv.g[L]); a.gc_out = bf(cv.gc[L]); a.ge_out = bf(cv.ge[L]);
      err = launch_gemm(a, l == 1 ? mk : mx[l - 1], mq, mwb[l], S, 2 * C / 128, nl / a.N, stream);
      if (err != cudaSuccess) return err;
    }
    // backward to every hidden layer
    for (int l = L; l >= 2; --l) {
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
      a.sp_in = bf(cv.sp[l - 1]);
      a.g_out = bf(cv.g[l - 1]); a.gc_out = bf(cv.gc[l - 1]); a.ge_out = bf(cv.ge[l - 1]);
      err = launch_gemm(a, mg[l], mg[l], mwb[l], S, (C + 127) / 128, np / a.N, stream);
      if (err != cudaSuccess) return err;
    }
    // weight-update contractions with the fused state update
    for (int l = 1; l <= L; ++l) {
      GemmArgs a = base;
      const int nl = p.dims[l], np = p.dims[l - 1];
      a.kind = K_DW;
      a.chunk = ch;
      a.N = tile_for(np, (nl + 127) / 128);
      a.K = C;
      a.M = nl;
      a.n_out = np;
      a.a_rows_per_stream = C;
      a.b_rows_per_stream = l == 1 ? T : 2 * C;
      a.b_row_off = l == 1 ? (long long)ch * C : 0;
      a.layer_off = (long long)p.layer_off[l - 1];
      a.Wbf = wbf + ia.boff[l - 1];
      err = launch_gemm(a, mgc[l], mge[l], l == 1 ? mk : mx[l - 1], S, (nl + 127) / 128, np / a.N, stream);
      if (err != cudaSuccess) return err;
    }
  }
  return cudaSuccess;
}

void tcl_set_wait(unsigned long long wait_ns) { g_tcl_wait_ns = wait_ns ? wait_ns : 2000000000ull; }

}  // namespace tmem
