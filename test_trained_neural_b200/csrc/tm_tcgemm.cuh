// Tensor-core GEMM inside one CTA of 256 threads, for the reverse pass's
// chains of small products (the gradient of the chunked write-and-read):
//
//   out(m, n) = sum_k A(m, k) B(n, k),   A(m, k) = A[m sam + k sak],
//                                        B(n, k) = B[n sbn + k sbk],
//
// A and B fp32 in global memory (any strides), each output element handed to
// epi(m, n, value) exactly once: the contract of the CUDA-core tile loop it
// replaces. Output blocks of 128 rows x up to 256 columns; per block the
// reduction runs in rounds of 64: every thread loads its share of the round's
// A and B elements, rounds them to TF32 (cvt.rna: to nearest, 10 explicit
// mantissa bits, fp32's exponent range, so gradients of any magnitude keep
// their relative precision) and stores them K-major in the 128-byte-swizzled
// layout (16-byte chunk c of row r at c ^ (r % 8)); one thread issues the
// round's tcgen05.mma.kind::tf32 instructions (M = 128, N = the block's
// columns rounded up to 16, K = 8 each) accumulating in TMEM, and the CTA
// waits for them before the next round overwrites the operands. Then warp w
// reads TMEM lanes 32 (w % 4) .. (rows) of 32 columns at a time into shared
// memory, from where the CTA calls epi row by row, consecutive threads on
// consecutive columns (the epilogues' global stores coalesce). The k order of
// the sums is fixed, so results do not depend on timing. Rows and columns
// beyond M, N and reductions beyond K are zero.
//
// Shared state (TcGemm, in shared memory) is set up once per kernel by
// tcg_init and released by tcg_release: the TMEM columns (256) and the MMA
// barrier. Every wait is bounded: on expiry the CTA records kDevTimeout in
// the status word and the results are not valid (the kernel does not hang).
#pragma once
#include <cstdint>

#include "tm_internal.h"
#include "tm_sm100.cuh"

namespace tmem {

constexpr int TCG_NT = 256;                      // threads of the CTA
constexpr int TCG_KR = 64;                       // reduction per round (two 32-wide swizzle atoms)
constexpr uint32_t TCG_A_BYTES = 2u * 128u * 128u;   // 128 rows x 64 fp32
constexpr uint32_t TCG_B_BYTES = 2u * 256u * 128u;   // 256 rows x 64 fp32
constexpr size_t TCG_SMEM = TCG_A_BYTES + TCG_B_BYTES + 1024;   // dynamic shared memory

struct TcGemm {
  uint64_t bar;          // MMA completion
  uint64_t never;        // test hook: a barrier nothing completes
  int inject;            // test hook on: the CTA's first product first waits on `never`
  uint32_t uses;         // completed phases of bar
  uint32_t tmem;         // TMEM base (256 columns)
  int *status;
  unsigned long long wait_ns;
  unsigned char *a, *b;  // operand buffers (1024-byte aligned)
};

// Instruction descriptor, kind::tf32: TF32 A and B (format code 2), K-major,
// fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// Byte offset of element (r, k) (k < 64) in a K-major buffer of `rows` rows.
__device__ __forceinline__ uint32_t tcg_off(int rows, int r, int k) {
  return (uint32_t)(k >> 5) * (uint32_t)rows * 128u + (uint32_t)r * 128u +
         ((uint32_t)(((k & 31) >> 2) ^ (r & 7)) << 4) + (uint32_t)(k & 3) * 4u;
}

// Set up by the whole CTA at kernel start (dyn: the kernel's dynamic shared
// memory, TCG_SMEM bytes).
__device__ __forceinline__ void tcg_init(TcGemm &g, unsigned char *dyn, int *status, unsigned long long wait_ns,
                                         int inject) {
  using namespace sm100;
  unsigned char *al = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(dyn) + 1023) & ~uintptr_t(1023));
  if (threadIdx.x == 0) {
    mbar_init(&g.bar, 1);
    mbar_init(&g.never, 1);
    g.inject = inject;
    g.uses = 0;
    g.status = status;
    g.wait_ns = wait_ns;
    g.a = al;
    g.b = al + TCG_A_BYTES;
    fence_barrier_init();
  }
  if (threadIdx.x < 32) { tmem_alloc(&g.tmem, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

__device__ __forceinline__ void tcg_release(TcGemm &g) {
  using namespace sm100;
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) tmem_dealloc(g.tmem, 256);
}

// Rows of B's staging layout for an output block of np columns: np rounded
// up to a power of two (the MMA reads the first np), so that element indices
// split into row and k with shifts.
__device__ __forceinline__ int tcg_rows_b(int np) {
  int r = 16;
  while (r < np) r <<= 1;
  return r;
}

// Stage `total` elements (rows x 64 of the round) of one operand: batches of
// 16 loads per thread in flight before their stores. X(row, k) =
// src[(row0 + row) * s_row + (k0 + k) * s_k], times kscale[k0 + k] if given;
// zero outside rows_valid x K. kfast: consecutive threads take consecutive k
// (s_k == 1), else consecutive rows.
__device__ __forceinline__ void tcg_stage(unsigned char *dst, int rows_lay, int lg_rows, int total, bool kfast,
                                          const float *src, long long s_row, long long s_k, int row0,
                                          int rows_valid, int k0, int K, const float *kscale) {
  const int tid = threadIdx.x;
  for (int base = 0; base < total; base += TCG_NT * 16) {
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int e = base + j * TCG_NT + tid;
      const int r = kfast ? (e >> 6) : (e & (rows_lay - 1)), k = kfast ? (e & 63) : (e >> lg_rows);
      const int gk = k0 + k;
      v[j] = 0.f;
      if (e < total && r < rows_valid && gk < K) {
        v[j] = src[(long long)(row0 + r) * s_row + (long long)gk * s_k];
        if (kscale) v[j] *= kscale[gk];
      }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int e = base + j * TCG_NT + tid;
      const int r = kfast ? (e >> 6) : (e & (rows_lay - 1)), k = kfast ? (e & 63) : (e >> lg_rows);
      if (e < total) *reinterpret_cast<uint32_t *>(dst + tcg_off(rows_lay, r, k)) = to_tf32(v[j]);
    }
  }
}

// The reduction of output block (m0, n0) into TMEM columns 0.. (all rounds):
// staging, MMA issue and the wait. One copy for every call site (not inlined).
// Returns false if a wait ran out (status recorded).
__device__ __noinline__ bool tcg_block(TcGemm &g, int M, int N, int K, int m0, int n0, const float *A,
                                       long long sam, long long sak, const float *B, long long sbn,
                                       long long sbk, const float *kscale) {
  using namespace sm100;
  const int tid = threadIdx.x;
  const uint32_t abase = smem_u32(g.a), bbase = smem_u32(g.b);
  const int nb = N - n0 < 256 ? N - n0 : 256;
  const int np = (nb + 15) / 16 * 16;           // MMA N: a multiple of 16
  const int rb = tcg_rows_b(np);
  int lg_rb = 4;
  while ((1 << lg_rb) < rb) ++lg_rb;
  const uint32_t idesc = idesc_tf32(128, np);
  uint32_t uses = g.uses;                       // read by every thread; updated identically
  bool ok = true;
  if (g.inject && uses == 0 && !mbar_wait(&g.never, 0, g.wait_ns)) {
    // test hook: the wait ran out as a lost MMA completion would; recorded,
    // and the call goes on (its products are still issued and awaited)
    if (tid == 0) atomicCAS(g.status, 0, kDevTimeout);
    ok = false;
  }
  for (int k0 = 0; k0 < K; k0 += TCG_KR) {
    // ---- stage the round's operands (zeros outside M, N, K)
    tcg_stage(g.a, 128, 7, 128 * TCG_KR, sak == 1, A, sam, sak, m0, M - m0, k0, K, kscale);
    tcg_stage(g.b, rb, lg_rb, rb * TCG_KR, sbk == 1, B, sbn, sbk, n0, nb, k0, K, nullptr);
    fence_proxy_async_smem();                  // generic-proxy writes, read by the MMAs
    tc_fence_before();
    __syncthreads();
    // ---- one thread issues the round: 8 MMAs of K = 8 (32 bytes each)
    if (tid == 0) {
      tc_fence_after();
      for (int ks = 0; ks < TCG_KR / 8; ++ks)
        umma_tf32(g.tmem, desc_kmajor(abase, 128, ks), desc_kmajor(bbase, rb, ks), idesc,
                  (k0 > 0 || ks > 0) ? 1u : 0u);
      umma_commit(&g.bar);
    }
    // every thread waits: the operands are overwritten next round and TMEM
    // is read after the last one
    if (!mbar_wait(&g.bar, uses & 1u, g.wait_ns)) {
      if (ok && tid == 0) atomicCAS(g.status, 0, kDevTimeout);
      ok = false;
    }
    ++uses;
    tc_fence_after();
  }
  __syncthreads();                              // every thread has read g.uses
  if (tid == 0) g.uses = uses;
  __syncthreads();
  return ok;
}

// kscale (optional): A(m, k) is multiplied by kscale[k] before rounding.
template <class Epi>
__device__ void tc_gemm(TcGemm &g, int M, int N, int K, const float *A, long long sam, long long sak,
                        const float *B, long long sbn, long long sbk, Epi epi, const float *kscale = nullptr) {
  using namespace sm100;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  float *tile = reinterpret_cast<float *>(g.b);  // 128 x 65 fp32 once the MMAs are done
  for (int m0 = 0; m0 < M; m0 += 128) {
    for (int n0 = 0; n0 < N; n0 += 256) {
      tcg_block(g, M, N, K, m0, n0, A, sam, sak, B, sbn, sbk, kscale);
      const int nb = N - n0 < 256 ? N - n0 : 256;
      const int np = (nb + 15) / 16 * 16;
      const int row = 32 * (warp & 3) + lane;   // TMEM lane of this thread
      const uint32_t lb = (uint32_t)(32 * (warp & 3)) << 16;
      // 64 columns at a time through shared memory, so that the epilogue
      // visits consecutive columns with consecutive threads
      for (int c0 = 0; c0 < np; c0 += 64) {
        const int cw = np - c0 < 64 ? np - c0 : 64;   // a multiple of 16
        const int cs = 32 * (warp >> 2);              // this warp's 32 columns of the slab
        for (int q = 0; q < 32; q += 16) {
          if (cs + q >= cw) break;                    // warp-uniform
          float z[16];
          tmem_ld16(g.tmem + lb + (uint32_t)(c0 + cs + q), z);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) tile[row * 65 + cs + q + i] = z[i];
        }
        __syncthreads();
        // the block's valid rows only (often 64 of 128)
        const int rv = M - m0 < 128 ? M - m0 : 128;
#pragma unroll 4
        for (int e = tid; e < rv * 64; e += TCG_NT) {
          const int r = e >> 6, c = e & 63;
          if (c < cw && c0 + c < nb) epi(m0 + r, n0 + c0 + c, tile[r * 65 + c]);
        }
        __syncthreads();
      }
      // TMEM and the operand buffers are reused by the next block
      tc_fence_before();
      __syncthreads();
    }
  }
}

}  // namespace tmem
