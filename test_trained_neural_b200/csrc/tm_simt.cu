// CUDA-core (fp32 FFMA) persistent chunk walker for the Titans memory.
//
// One CTA per stream (batch entry, head). The CTA walks the chunks of its
// stream in order; inside a chunk it runs, with block-wide barriers between
// the steps:
//   A5  the gate-coefficient scan (division-free reverse recurrence),
//   A2  forward of the chunk's keys and queries through the chunk-start weights
//       (queries give the reads y, "Titans, explained" step 5),
//   A3  residual G_L = 2 (M(k) - v)   (step 2: loss ||M(k) - v||^2),
//   A4  backward G_{l-1} = (W_l^T G_l) . silu'(Z_{l-1}),
//   A6+A7 per layer one dual-accumulator contraction over the chunk's tokens,
//       U_W = sum_i c_i g_i x_i^T and U_S = sum_i e_i g_i x_i^T, whose epilogue
//       applies W' = B W + c_S S - U_W and S' = A S - U_S in place
//       (steps 3 and 4, unrolled over the chunk; "Attack of the Titans",
//        "Parallel training": gradients at the chunk start, decay products
//        collected per token).
// W and S live in the caller's W_end / S_end buffers (copied from W0 / S0 at
// the start unless they alias them). Activations of the chunk live in the
// per-stream scratch. Everything is fp32; bf16 inputs are widened on load.
//
// This kernel runs every supported shape and both input dtypes. It is the
// fp32 product path and the reference the tensor-core path is checked against
// on small shapes.
#include <cuda_bf16.h>

#include "tm_internal.h"
#include "tm_tcgemm.cuh"

namespace tmem {
namespace {

constexpr int NT = 256;        // threads per CTA
constexpr int TMt = 64;        // output tile rows
constexpr int TNt = 64;        // output tile cols
constexpr int TKt = 16;        // reduction tile
constexpr int PAD = 4;

struct Coef {
  float c[kMaxC];   // weight of token i's surprise in the W update
  float e[kMaxC];   // weight of token i's surprise in the S update
  float Bw;         // prod (1 - alpha)     : factor on W
  float As;         // prod eta             : factor on S in the S update
  float cS;         // eta_1 r_1            : factor on S in the W update
};

struct SmemT {
  float As[TKt][TMt + PAD];
  float Bs[TKt][TNt + PAD];
  Coef coef;
};

struct Net {
  int L;
  int dims[kMaxL + 1];
  long long off[kMaxL + 1];
  long long P;
  int maxw;
};

__device__ __forceinline__ float load_tok(const void *p, int bf16, long long i) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(p)[i]);
  return reinterpret_cast<const float *>(p)[i];
}

__device__ __forceinline__ float sigm(float z) { return 1.0f / (1.0f + expf(-z)); }
__device__ __forceinline__ float silu(float z) { return z * sigm(z); }
__device__ __forceinline__ float warp_sum_simt(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float silu_prime(float z) {
  float s = sigm(z);
  return s * (1.0f + z * (1.0f - s));
}

// out(m, n) = sum_k A(m, k) B(n, k); A(m,k) = A[m*sam + k*sak], B(n,k) = B[n*sbn + k*sbk].
// Every output element is handed to epi(m, n, value) exactly once.
template <class Epi>
__device__ void gemm(SmemT &sm, int M, int N, int K, const float *A, long long sam, long long sak,
                     const float *B, long long sbn, long long sbk, Epi epi) {
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  for (int m0 = 0; m0 < M; m0 += TMt) {
    for (int n0 = 0; n0 < N; n0 += TNt) {
      float acc[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
      for (int k0 = 0; k0 < K; k0 += TKt) {
        for (int e = tid; e < TMt * TKt; e += NT) {
          int mm, kk;
          if (sak == 1) { kk = e % TKt; mm = e / TKt; } else { mm = e % TMt; kk = e / TMt; }
          int gm = m0 + mm, gk = k0 + kk;
          sm.As[kk][mm] = (gm < M && gk < K) ? A[gm * sam + gk * sak] : 0.f;
        }
        for (int e = tid; e < TNt * TKt; e += NT) {
          int nn, kk;
          if (sbk == 1) { kk = e % TKt; nn = e / TKt; } else { nn = e % TNt; kk = e / TNt; }
          int gn = n0 + nn, gk = k0 + kk;
          sm.Bs[kk][nn] = (gn < N && gk < K) ? B[gn * sbn + gk * sbk] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TKt; ++kk) {
          float a[4], b[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) a[i] = sm.As[kk][ty + 16 * i];
#pragma unroll
          for (int j = 0; j < 4; ++j) b[j] = sm.Bs[kk][tx + 16 * j];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
          if (m < M && n < N) epi(m, n, acc[i][j]);
        }
    }
  }
}

// The weight update of one layer: U_W(r, c) = sum_i c_i G[i][r] X[i][c],
// U_S(r, c) = sum_i e_i G[i][r] X[i][c], then W' = Bw W + cS S - U_W and
// S' = As S - U_S for the [rows x cols] block at Wl / Sl.
__device__ void update_layer(SmemT &sm, int rows, int cols, int C, const float *G, const float *X,
                             float *Wl, float *Sl) {
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const Coef &cf = sm.coef;
  for (int m0 = 0; m0 < rows; m0 += TMt) {
    for (int n0 = 0; n0 < cols; n0 += TNt) {
      float aw[4][4], as[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) aw[i][j] = as[i][j] = 0.f;
      for (int k0 = 0; k0 < C; k0 += TKt) {
        for (int e = tid; e < TMt * TKt; e += NT) {
          int mm = e % TMt, kk = e / TMt;  // G[i][r]: r contiguous
          int gm = m0 + mm, gk = k0 + kk;
          sm.As[kk][mm] = (gm < rows && gk < C) ? G[(long long)gk * rows + gm] : 0.f;
        }
        for (int e = tid; e < TNt * TKt; e += NT) {
          int nn = e % TNt, kk = e / TNt;  // X[i][c]: c contiguous
          int gn = n0 + nn, gk = k0 + kk;
          sm.Bs[kk][nn] = (gn < cols && gk < C) ? X[(long long)gk * cols + gn] : 0.f;
        }
        __syncthreads();
        for (int kk = 0; kk < TKt && k0 + kk < C; ++kk) {
          float ci = cf.c[k0 + kk], ei = cf.e[k0 + kk];
          float a[4], b[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) a[i] = sm.As[kk][ty + 16 * i];
#pragma unroll
          for (int j = 0; j < 4; ++j) b[j] = sm.Bs[kk][tx + 16 * j];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float ab = a[i] * b[j];
              aw[i][j] = fmaf(ci, ab, aw[i][j]);
              as[i][j] = fmaf(ei, ab, as[i][j]);
            }
        }
        __syncthreads();
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          int r = m0 + ty + 16 * i, c = n0 + tx + 16 * j;
          if (r < rows && c < cols) {
            long long idx = (long long)r * cols + c;
            float w = Wl[idx], s = Sl[idx];
            Wl[idx] = cf.Bw * w + cf.cS * s - aw[i][j];
            Sl[idx] = cf.As * s - as[i][j];
          }
        }
    }
  }
}

// A5: per-token coefficients of one chunk from its gates (0-based i = 0..n-1):
//   pa_i = prod_{j>i} (1 - alpha_j),  pe_i = prod_{j>i} eta_j,
//   r_{n-1} = 1,  r_i = pa_i + eta_{i+1} r_{i+1},
//   c_i = theta_i r_i,  e_i = theta_i pe_i,
//   Bw = pa_0 (1 - alpha_0),  As = pe_0 eta_0,  cS = eta_0 r_0.
// Unrolling S_t = eta_t S_{t-1} - theta_t u_t and W_t = (1-alpha_t) W_{t-1} + S_t
// over the chunk gives W_end = Bw W + cS S - sum c_i u_i, S_end = As S - sum e_i u_i.
// No division, so alpha = 1 and eta = 0 are exact.
__device__ void chunk_coefficients(Coef &cf, const float *theta, const float *eta,
                                   const float *alpha, int n) {
  if (threadIdx.x != 0) return;
  float pa = 1.f, pe = 1.f, r = 1.f;
  for (int i = n - 1; i >= 0; --i) {
    if (i < n - 1) {
      pa *= 1.f - alpha[i + 1];
      pe *= eta[i + 1];
      r = pa + eta[i + 1] * r;
    }
    cf.c[i] = theta[i] * r;
    cf.e[i] = theta[i] * pe;
  }
  cf.Bw = pa * (1.f - alpha[0]);
  cf.As = pe * eta[0];
  cf.cS = eta[0] * r;
}

struct KArgs {
  Net net;
  int T, C, bf16;
  int t_begin;                   // first token of each stream to process
  const void *k, *v, *q;
  const float *theta, *eta, *alpha, *W0, *S0;
  float *y, *W, *S;
  float *scratch;
  long long scratch_per_stream;  // floats
  int *status;
};

__global__ void __launch_bounds__(NT) simt_chunk_kernel(KArgs a) {
  __shared__ SmemT sm;
  const Net &n = a.net;
  const int s = blockIdx.x;
  const int L = n.L, C = a.C, T = a.T;
  const int d_in = n.dims[0], d_out = n.dims[L];
  if (C > kMaxC || C < 1) {
    if (threadIdx.x == 0) atomicCAS(a.status, 0, kDevBadConfig);
    return;
  }
  float *W = a.W + (long long)s * n.P;
  float *S = a.S + (long long)s * n.P;
  if (a.W0 + (long long)s * n.P != W)
    for (long long i = threadIdx.x; i < n.P; i += NT) W[i] = a.W0[(long long)s * n.P + i];
  if (a.S0 + (long long)s * n.P != S)
    for (long long i = threadIdx.x; i < n.P; i += NT) S[i] = a.S0[(long long)s * n.P + i];

  // scratch layout (floats): X[0..L-1] (C x n_l), Z[1..L-1] (C x n_l),
  // Qa, Qb (C x maxw), Ga, Gb (C x maxw)
  float *base = a.scratch + (long long)s * a.scratch_per_stream;
  float *X[kMaxL], *Z[kMaxL];
  float *p = base;
  for (int l = 0; l < L; ++l) { X[l] = p; p += (long long)C * n.dims[l]; }
  for (int l = 1; l < L; ++l) { Z[l] = p; p += (long long)C * n.dims[l]; }
  float *Qa = p; p += (long long)C * n.maxw;
  float *Qb = p; p += (long long)C * n.maxw;
  float *Ga = p; p += (long long)C * n.maxw;
  float *Gb = p;
  __syncthreads();

  const long long tok_base = (long long)s * T;
  // chunks start at t_begin + multiples of C; the last one may be shorter
  for (int t0 = a.t_begin; t0 < T; t0 += C) {
    const long long tb = tok_base + t0;
    const int Cc = T - t0 < C ? T - t0 : C;       // tokens in this chunk
    chunk_coefficients(sm.coef, a.theta + tb, a.eta + tb, a.alpha + tb, Cc);
    for (int i = threadIdx.x; i < Cc * d_in; i += NT) {
      X[0][i] = load_tok(a.k, a.bf16, tb * d_in + i);
      Qa[i] = load_tok(a.q, a.bf16, tb * d_in + i);
    }
    __syncthreads();

    // A2 + A3: forward of the keys; keep pre-activations for the backward.
    float *Gcur = Ga;
    for (int l = 1; l <= L; ++l) {
      const float *Wl = W + n.off[l - 1];
      const int rows = n.dims[l], cols = n.dims[l - 1];
      if (l < L) {
        float *Zl = Z[l], *Xl = X[l];
        gemm(sm, Cc, rows, cols, X[l - 1], cols, 1, Wl, cols, 1,
             [&](int i, int r, float z) {
               Zl[(long long)i * rows + r] = z;
               Xl[(long long)i * rows + r] = silu(z);
             });
      } else {
        gemm(sm, Cc, rows, cols, X[l - 1], cols, 1, Wl, cols, 1,
             [&](int i, int r, float z) {
               float vv = load_tok(a.v, a.bf16, (tb + i) * d_out + r);
               Gcur[(long long)i * rows + r] = 2.f * (z - vv);
             });
      }
      __syncthreads();
    }
    // A2 (read half): forward of the queries through the same weights -> y.
    float *qin = Qa, *qout = Qb;
    for (int l = 1; l <= L; ++l) {
      const float *Wl = W + n.off[l - 1];
      const int rows = n.dims[l], cols = n.dims[l - 1];
      if (l < L) {
        gemm(sm, Cc, rows, cols, qin, cols, 1, Wl, cols, 1,
             [&](int i, int r, float z) { qout[(long long)i * rows + r] = silu(z); });
        float *tmp = qin; qin = qout; qout = tmp;
      } else {
        float *y = a.y + tb * d_out;
        gemm(sm, Cc, rows, cols, qin, cols, 1, Wl, cols, 1,
             [&](int i, int r, float z) { y[(long long)i * rows + r] = z; });
      }
      __syncthreads();
    }
    // A4: backward to every layer's pre-activation gradient.
    // G[l] for layer l is kept: the update of layer l needs it.
    float *Gl[kMaxL + 1];
    Gl[L] = Gcur;
    // Keep distinct buffers: layer L in Ga, then alternate through Gb and the
    // (no longer needed) query buffers.
    float *pool[3] = {Gb, Qa, Qb};
    for (int l = L; l >= 2; --l) {
      const float *Wl = W + n.off[l - 1];
      const int rows = n.dims[l], cols = n.dims[l - 1];
      float *Gout = pool[(L - l) % 3];
      const float *Zp = Z[l - 1];
      gemm(sm, Cc, cols, rows, Gl[l], rows, 1, Wl, 1, cols,
           [&](int i, int c, float g) {
             long long idx = (long long)i * cols + c;
             Gout[idx] = g * silu_prime(Zp[idx]);
           });
      Gl[l - 1] = Gout;
      __syncthreads();
    }
    // A6 + A7: per-layer dual contraction and fused state update.
    for (int l = 1; l <= L; ++l) {
      update_layer(sm, n.dims[l], n.dims[l - 1], Cc, Gl[l], X[l - 1], W + n.off[l - 1],
                   S + n.off[l - 1]);
    }
    __syncthreads();
  }
}


// ---------------------------------------------------------------------------
// Gradients of the linear memory (depth 1, W and S [d x d]) for an outer
// model training through it: given dy (of the reads), dW_end and dS_end, the
// gradients of J = sum <dy_t, y_t> + <dW_end, W_end> + <dS_end, S_end> with
// respect to k, v, q, the gates, W0 and S0. A forward pass stores the
// chunk-start state; the reverse pass carries (gW, gS) back through the
// chunks. Per chunk, with r_i = W k_i - v_i, u_i = 2 r_i k_i^T and
// m_i = -(c_i gW + e_i gS) k_i:
//   dq_i = W^T dy_i,  dv_i = -2 m_i,  dk_i = 2 W^T m_i - 2 c_i gW^T r_i - 2 e_i gS^T r_i
//   dc_i = -2 r_i^T gW k_i,  de_i = -2 r_i^T gS k_i
//   dB = <gW, W>, dcS = <gW, S>, dA = <gS, S>
//   gW <- B gW + 2 sum m_i k_i^T + sum dy_i q_i^T,   gS <- cS gW + A gS
// and (dc, de, dB, dA, dcS) go back through the coefficient scan to the gates.
struct BArgs {
  int d, T, C, bf16;
  int *status;                   // device status word (bounded waits of the tensor-core products)
  unsigned long long wait_ns;
  int inject;                    // test hook (tm_set_debug), tensor-core products only
  const void *k, *v, *q;
  const float *theta, *eta, *alpha, *W0, *S0, *dy, *dW_end, *dS_end;
  float *dk, *dv, *dq, *dtheta, *deta, *dalpha, *dW0, *dS0;
  float *scratch;
  long long scratch_per_stream;
};

__device__ float block_sum(float x, float *red) {
  x = warp_sum_simt(x);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();
  if (lane == 0) red[warp] = x;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < NT / 32) t = red[threadIdx.x];
  if (warp == 0) t = warp_sum_simt(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  const float r = red[0];
  __syncthreads();
  return r;
}

// Reverse-mode through the coefficient scan of one chunk (Cc tokens), one
// thread: from the gradients of c_i, e_i, B, A, c_S to theta, eta, alpha.
//   pa_i = prod_{j>i}(1 - alpha_j), pe_i = prod_{j>i} eta_j,
//   rho_{C-1} = 1, rho_i = pa_i + eta_{i+1} rho_{i+1};
//   c_i = theta_i rho_i, e_i = theta_i pe_i, B = pa_0 (1 - alpha_0),
//   A = pe_0 eta_0, c_S = eta_0 rho_0.
// pa .. drho: scratch of Cc floats each.
__device__ void gate_reverse(int Cc, const float *th, const float *et, const float *al, const float *dc,
                             const float *de, float dB, float dA, float dcS, float *dth, float *det, float *dal,
                             float *pa, float *pe, float *rho, float *dpa, float *dpe, float *drho) {
  pa[Cc - 1] = 1.f; pe[Cc - 1] = 1.f; rho[Cc - 1] = 1.f;
  for (int i = Cc - 2; i >= 0; --i) {
    pa[i] = pa[i + 1] * (1.f - al[i + 1]);
    pe[i] = pe[i + 1] * et[i + 1];
    rho[i] = pa[i] + et[i + 1] * rho[i + 1];
  }
  for (int i = 0; i < Cc; ++i) {
    dth[i] = dc[i] * rho[i] + de[i] * pe[i];
    drho[i] = dc[i] * th[i];
    dpe[i] = de[i] * th[i];
    dpa[i] = 0.f;
    det[i] = 0.f;
    dal[i] = 0.f;
  }
  dpa[0] += dB * (1.f - al[0]);
  dal[0] += -dB * pa[0];
  dpe[0] += dA * et[0];
  det[0] += dA * pe[0];
  det[0] += dcS * rho[0];
  drho[0] += dcS * et[0];
  for (int i = 0; i + 1 < Cc; ++i) {
    dpa[i] += drho[i];
    det[i + 1] += drho[i] * rho[i + 1];
    drho[i + 1] += drho[i] * et[i + 1];
    dpe[i + 1] += dpe[i] * et[i + 1];
    det[i + 1] += dpe[i] * pe[i + 1];
    dpa[i + 1] += dpa[i] * (1.f - al[i + 1]);
    dal[i + 1] += -dpa[i] * pa[i + 1];
  }
}

template <bool TC>
__global__ void __launch_bounds__(NT) backward1_kernel(BArgs a) {
  __shared__ SmemT sm;
  __shared__ float red[NT / 32];
  extern __shared__ __align__(1024) unsigned char tcg_dyn[];
  __shared__ TcGemm tg;
  if constexpr (TC) tcg_init(tg, tcg_dyn, a.status, a.wait_ns, a.inject);
  // the chunk's products: tcgen05 (TF32 operands, fp32 accumulation) or fp32 FFMA tiles
  auto mm = [&](int M_, int N_, int K_, const float *A_, long long sam, long long sak, const float *B_,
                long long sbn, long long sbk, auto epi) {
    if constexpr (TC) tc_gemm(tg, M_, N_, K_, A_, sam, sak, B_, sbn, sbk, epi);
    else gemm(sm, M_, N_, K_, A_, sam, sak, B_, sbn, sbk, epi);
  };
  // the forward pass's state update of one layer (A6 + A7): on the tensor
  // cores as two products, U_W with the tokens' c and U_S with their e
  auto upd = [&](int rows, int cols, int Cn, const float *G, const float *X, float *Wl, float *Sl) {
    if constexpr (TC) {
      const Coef &cf = sm.coef;
      tc_gemm(tg, rows, cols, Cn, G, 1, rows, X, 1, cols, [&](int r, int c, float u) {
        const long long idx = (long long)r * cols + c;
        Wl[idx] = cf.Bw * Wl[idx] + cf.cS * Sl[idx] - u;
      }, cf.c);
      tc_gemm(tg, rows, cols, Cn, G, 1, rows, X, 1, cols, [&](int r, int c, float u) {
        const long long idx = (long long)r * cols + c;
        Sl[idx] = cf.As * Sl[idx] - u;
      }, cf.e);
    } else {
      update_layer(sm, rows, cols, Cn, G, X, Wl, Sl);
    }
  };
  const int s = blockIdx.x, d = a.d, T = a.T, C = a.C, dd = d * d;
  const int nch = (T + C - 1) / C;
  float *p = a.scratch + (long long)s * a.scratch_per_stream;
  float *ckW = p; p += (long long)nch * dd;
  float *ckS = p; p += (long long)nch * dd;
  float *Wc = p; p += dd;
  float *Sc = p; p += dd;
  float *gW = p; p += dd;
  float *gS = p; p += dd;
  float *gWn = p; p += dd;
  float *K = p; p += (long long)C * d;
  float *V = p; p += (long long)C * d;
  float *Q = p; p += (long long)C * d;
  float *DY = p; p += (long long)C * d;
  float *R = p; p += (long long)C * d;
  float *Am = p; p += (long long)C * d;
  float *Bm = p; p += (long long)C * d;
  float *Mm = p; p += (long long)C * d;
  float *Pm = p; p += (long long)C * d;
  float *Qm = p; p += (long long)C * d;
  float *dc = p; p += C;
  float *de = p; p += C;
  float *pa = p; p += C;
  float *pe = p; p += C;
  float *rho = p; p += C;
  float *dpa = p; p += C;
  float *dpe = p; p += C;
  float *drho = p; p += C;
  const long long sw = (long long)s * dd, tok0 = (long long)s * T;

  auto load_chunk = [&](int t0, int Cc, bool grads) {
    for (int i = threadIdx.x; i < Cc * d; i += NT) {
      const long long g = (tok0 + t0) * d + i;
      K[i] = load_tok(a.k, a.bf16, g);
      V[i] = load_tok(a.v, a.bf16, g);
      if (grads) {
        Q[i] = load_tok(a.q, a.bf16, g);
        DY[i] = a.dy[g];
      }
    }
    __syncthreads();
  };
  // ---- forward: chunk-start states
  for (int i = threadIdx.x; i < dd; i += NT) {
    Wc[i] = a.W0[sw + i];
    Sc[i] = a.S0[sw + i];
  }
  __syncthreads();
  for (int c = 0; c < nch; ++c) {
    const int t0 = c * C, Cc = T - t0 < C ? T - t0 : C;
    for (int i = threadIdx.x; i < dd; i += NT) {
      ckW[(long long)c * dd + i] = Wc[i];
      ckS[(long long)c * dd + i] = Sc[i];
    }
    chunk_coefficients(sm.coef, a.theta + tok0 + t0, a.eta + tok0 + t0, a.alpha + tok0 + t0, Cc);
    load_chunk(t0, Cc, false);
    // G = 2 (K W^T - V): the surprise factor of every token
    mm(Cc, d, d, K, d, 1, Wc, d, 1, [&](int i, int r, float z) { R[i * d + r] = 2.f * (z - V[i * d + r]); });
    __syncthreads();
    upd(d, d, Cc, R, K, Wc, Sc);
    __syncthreads();
  }
  // ---- reverse
  for (int i = threadIdx.x; i < dd; i += NT) {
    gW[i] = a.dW_end[sw + i];
    gS[i] = a.dS_end[sw + i];
  }
  __syncthreads();
  for (int c = nch - 1; c >= 0; --c) {
    const int t0 = c * C, Cc = T - t0 < C ? T - t0 : C;
    const float *th = a.theta + tok0 + t0, *et = a.eta + tok0 + t0, *al = a.alpha + tok0 + t0;
    const float *W = ckW + (long long)c * dd, *S = ckS + (long long)c * dd;
    chunk_coefficients(sm.coef, th, et, al, Cc);
    load_chunk(t0, Cc, true);
    // residuals r_i and the products with gW, gS
    mm(Cc, d, d, K, d, 1, W, d, 1, [&](int i, int r, float z) { R[i * d + r] = z - V[i * d + r]; });
    mm(Cc, d, d, K, d, 1, gW, d, 1, [&](int i, int r, float z) { Am[i * d + r] = z; });
    mm(Cc, d, d, K, d, 1, gS, d, 1, [&](int i, int r, float z) { Bm[i * d + r] = z; });
    __syncthreads();
    mm(Cc, d, d, R, d, 1, gW, 1, d, [&](int i, int j, float z) { Pm[i * d + j] = z; });
    mm(Cc, d, d, R, d, 1, gS, 1, d, [&](int i, int j, float z) { Qm[i * d + j] = z; });
    for (int e = threadIdx.x; e < Cc * d; e += NT) {
      const int i = e / d;
      Mm[e] = -(sm.coef.c[i] * Am[e] + sm.coef.e[i] * Bm[e]);
    }
    __syncthreads();
    // coefficient gradients (warp per token) and the chunk scalars
    for (int i = threadIdx.x / 32; i < Cc; i += NT / 32) {
      float x = 0.f, y = 0.f;
      for (int r = threadIdx.x % 32; r < d; r += 32) {
        x = fmaf(R[i * d + r], Am[i * d + r], x);
        y = fmaf(R[i * d + r], Bm[i * d + r], y);
      }
      x = warp_sum_simt(x);
      y = warp_sum_simt(y);
      if (threadIdx.x % 32 == 0) {
        dc[i] = -2.f * x;
        de[i] = -2.f * y;
      }
    }
    float pw = 0.f, pws = 0.f, pss = 0.f;
    for (int e = threadIdx.x; e < dd; e += NT) {
      pw = fmaf(gW[e], W[e], pw);
      pws = fmaf(gW[e], S[e], pws);
      pss = fmaf(gS[e], S[e], pss);
    }
    const float dB = block_sum(pw, red), dcS = block_sum(pws, red), dA = block_sum(pss, red);
    // token gradients
    const long long gt = (tok0 + t0) * d;
    mm(Cc, d, d, Mm, d, 1, W, 1, d, [&](int i, int j, float z) {
      const int e = i * d + j;
      a.dk[gt + e] = 2.f * z - 2.f * sm.coef.c[i] * Pm[e] - 2.f * sm.coef.e[i] * Qm[e];
    });
    mm(Cc, d, d, DY, d, 1, W, 1, d, [&](int i, int j, float z) { a.dq[gt + i * d + j] = z; });
    for (int e = threadIdx.x; e < Cc * d; e += NT) a.dv[gt + e] = -2.f * Mm[e];
    // gates: back through the coefficient scan (one thread, in order)
    if (threadIdx.x == 0)
      gate_reverse(Cc, th, et, al, dc, de, dB, dA, dcS, a.dtheta + tok0 + t0, a.deta + tok0 + t0,
                   a.dalpha + tok0 + t0, pa, pe, rho, dpa, dpe, drho);
    // the state gradients at the chunk start
    const float Bw = sm.coef.Bw, As = sm.coef.As, cS = sm.coef.cS;
    mm(d, d, Cc, Mm, 1, d, K, 1, d, [&](int r, int j, float z) { gWn[r * d + j] = Bw * gW[r * d + j] + 2.f * z; });
    __syncthreads();
    mm(d, d, Cc, DY, 1, d, Q, 1, d, [&](int r, int j, float z) { gWn[r * d + j] += z; });
    __syncthreads();
    for (int e = threadIdx.x; e < dd; e += NT) {
      gS[e] = cS * gW[e] + As * gS[e];
      gW[e] = gWn[e];
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < dd; e += NT) {
    a.dW0[sw + e] = gW[e];
    a.dS0[sw + e] = gS[e];
  }
  if constexpr (TC) tcg_release(tg);
}


// ---------------------------------------------------------------------------
// The same gradients for the depth-2 memory M(x) = W2 silu(W1 x) (W1 [n x d],
// W2 [o x n]). Per token the surprise enters J through
//   J_i = g1^T a + g2^T b,  a = M1 k, b = M2 x1,  M_l = -(c_i gW_l + e_i gS_l),
// with z1 = W1 k, x1 = silu(z1), g2 = 2 (W2 x1 - v), h = W2^T g2,
// g1 = h . silu'(z1); reverse mode through these vector steps gives, for the
// chunk's tokens as matrices (rows = tokens):
//   dG1 = a;  dH = a . silu'(z1);  dSP = a . h;  dG2 = b + dH W2^T
//   dW2 += G2^T dH + 2 dG2^T X1;  dv = -2 dG2
//   dX1 = 2 dG2 W2 - c (G2 gW2) - e (G2 gS2)
//   dZ1 = dX1 . silu'(z1) + dSP . silu''(z1)
//   dW1 += dZ1^T K;  dk = dZ1 W1 - c (G1 gW1) - e (G1 gS1)
// and the reads y = W2 silu(W1 q) add their ordinary backward (dq, dW1, dW2).
// The coefficient, scalar, state and gate steps are those of depth 1.
__device__ __forceinline__ float silu_second(float z) {
  const float s = sigm(z);
  return s * (1.f - s) * (2.f + z * (1.f - 2.f * s));
}

struct BArgs2 {
  int d, n, o, T, C, bf16;
  int *status;                   // device status word (bounded waits of the tensor-core products)
  unsigned long long wait_ns;
  int inject;                    // test hook (tm_set_debug), tensor-core products only
  long long P;
  const void *k, *v, *q;
  const float *theta, *eta, *alpha, *W0, *S0, *dy, *dW_end, *dS_end;
  float *dk, *dv, *dq, *dtheta, *deta, *dalpha, *dW0, *dS0;
  float *scratch;
  long long scratch_per_stream;
};

__host__ __device__ inline long long backward2_floats(int d, int n, int o, int T, int C) {
  const long long P = (long long)n * d + (long long)o * n, nch = (T + C - 1) / C;
  const long long m = n > d ? (n > o ? n : o) : (d > o ? d : o);
  return 2 * nch * P + 5 * P + 20LL * C * m + 8LL * C;
}

template <bool TC>
__global__ void __launch_bounds__(NT) backward2_kernel(BArgs2 a) {
  __shared__ SmemT sm;
  __shared__ float red[NT / 32];
  extern __shared__ __align__(1024) unsigned char tcg_dyn[];
  __shared__ TcGemm tg;
  if constexpr (TC) tcg_init(tg, tcg_dyn, a.status, a.wait_ns, a.inject);
  // the chunk's products: tcgen05 (TF32 operands, fp32 accumulation) or fp32 FFMA tiles
  auto mm = [&](int M_, int N_, int K_, const float *A_, long long sam, long long sak, const float *B_,
                long long sbn, long long sbk, auto epi) {
    if constexpr (TC) tc_gemm(tg, M_, N_, K_, A_, sam, sak, B_, sbn, sbk, epi);
    else gemm(sm, M_, N_, K_, A_, sam, sak, B_, sbn, sbk, epi);
  };
  // the forward pass's state update of one layer (A6 + A7): on the tensor
  // cores as two products, U_W with the tokens' c and U_S with their e
  auto upd = [&](int rows, int cols, int Cn, const float *G, const float *X, float *Wl, float *Sl) {
    if constexpr (TC) {
      const Coef &cf = sm.coef;
      tc_gemm(tg, rows, cols, Cn, G, 1, rows, X, 1, cols, [&](int r, int c, float u) {
        const long long idx = (long long)r * cols + c;
        Wl[idx] = cf.Bw * Wl[idx] + cf.cS * Sl[idx] - u;
      }, cf.c);
      tc_gemm(tg, rows, cols, Cn, G, 1, rows, X, 1, cols, [&](int r, int c, float u) {
        const long long idx = (long long)r * cols + c;
        Sl[idx] = cf.As * Sl[idx] - u;
      }, cf.e);
    } else {
      update_layer(sm, rows, cols, Cn, G, X, Wl, Sl);
    }
  };
  const int s = blockIdx.x, d = a.d, n = a.n, o = a.o, T = a.T, C = a.C;
  const long long P = a.P, nd = (long long)n * d;
  const int nch = (T + C - 1) / C;
  const int m = n > d ? (n > o ? n : o) : (d > o ? d : o);
  float *p = a.scratch + (long long)s * a.scratch_per_stream;
  float *ckW = p; p += (long long)nch * P;
  float *ckS = p; p += (long long)nch * P;
  float *Wc = p; p += P;
  float *Sc = p; p += P;
  float *gW = p; p += P;
  float *gS = p; p += P;
  float *gWn = p; p += P;
  auto take = [&]() { float *r = p; p += (long long)C * m; return r; };
  float *K = take(), *V = take(), *Q = take(), *DY = take();
  float *Z1 = take(), *X1 = take(), *G2 = take(), *H = take(), *G1 = take();
  float *ZQ = take(), *XQ = take(), *KW1 = take(), *KS1 = take(), *XW2 = take(), *XS2 = take();
  float *T1 = take(), *T2 = take(), *TO = take();
  take(); take();
  float *dc = p; p += C;
  float *de = p; p += C;
  float *pa = p; p += C;
  float *pe = p; p += C;
  float *rho = p; p += C;
  float *dpa = p; p += C;
  float *dpe = p; p += C;
  float *drho = p; p += C;
  const long long sw = (long long)s * P, tok0 = (long long)s * T;

  auto load_chunk = [&](int t0, int Cc, bool grads) {
    for (int i = threadIdx.x; i < Cc * d; i += NT) {
      const long long g = (tok0 + t0) * d + i;
      K[i] = load_tok(a.k, a.bf16, g);
      if (grads) Q[i] = load_tok(a.q, a.bf16, g);
    }
    for (int i = threadIdx.x; i < Cc * o; i += NT) {
      const long long g = (tok0 + t0) * o + i;
      V[i] = load_tok(a.v, a.bf16, g);
      if (grads) DY[i] = a.dy[g];
    }
    __syncthreads();
  };
  // forward of the keys at (W1, W2): Z1, X1, G2, H = G2 W2, G1
  auto keys_forward = [&](int Cc, const float *W1, const float *W2) {
    mm(Cc, n, d, K, d, 1, W1, d, 1, [&](int i, int j, float z) {
      Z1[i * n + j] = z;
      X1[i * n + j] = silu(z);
    });
    __syncthreads();
    mm(Cc, o, n, X1, n, 1, W2, n, 1, [&](int i, int r, float z) { G2[i * o + r] = 2.f * (z - V[i * o + r]); });
    __syncthreads();
    mm(Cc, n, o, G2, o, 1, W2, 1, n, [&](int i, int j, float z) {
      H[i * n + j] = z;
      G1[i * n + j] = z * silu_prime(Z1[i * n + j]);
    });
    __syncthreads();
  };
  // ---- forward: chunk-start states
  for (long long i = threadIdx.x; i < P; i += NT) {
    Wc[i] = a.W0[sw + i];
    Sc[i] = a.S0[sw + i];
  }
  __syncthreads();
  for (int c = 0; c < nch; ++c) {
    const int t0 = c * C, Cc = T - t0 < C ? T - t0 : C;
    for (long long i = threadIdx.x; i < P; i += NT) {
      ckW[(long long)c * P + i] = Wc[i];
      ckS[(long long)c * P + i] = Sc[i];
    }
    chunk_coefficients(sm.coef, a.theta + tok0 + t0, a.eta + tok0 + t0, a.alpha + tok0 + t0, Cc);
    load_chunk(t0, Cc, false);
    keys_forward(Cc, Wc, Wc + nd);
    upd(o, n, Cc, G2, X1, Wc + nd, Sc + nd);
    upd(n, d, Cc, G1, K, Wc, Sc);
    __syncthreads();
  }
  // ---- reverse
  for (long long i = threadIdx.x; i < P; i += NT) {
    gW[i] = a.dW_end[sw + i];
    gS[i] = a.dS_end[sw + i];
  }
  __syncthreads();
  for (int c = nch - 1; c >= 0; --c) {
    const int t0 = c * C, Cc = T - t0 < C ? T - t0 : C;
    const float *th = a.theta + tok0 + t0, *et = a.eta + tok0 + t0, *al = a.alpha + tok0 + t0;
    const float *W1 = ckW + (long long)c * P, *W2 = W1 + nd;
    const float *S = ckS + (long long)c * P;
    const float *gW1 = gW, *gW2 = gW + nd, *gS1 = gS, *gS2 = gS + nd;
    chunk_coefficients(sm.coef, th, et, al, Cc);
    load_chunk(t0, Cc, true);
    keys_forward(Cc, W1, W2);
    mm(Cc, n, d, Q, d, 1, W1, d, 1, [&](int i, int j, float z) {
      ZQ[i * n + j] = z;
      XQ[i * n + j] = silu(z);
    });
    mm(Cc, n, d, K, d, 1, gW1, d, 1, [&](int i, int j, float z) { KW1[i * n + j] = z; });
    mm(Cc, n, d, K, d, 1, gS1, d, 1, [&](int i, int j, float z) { KS1[i * n + j] = z; });
    mm(Cc, o, n, X1, n, 1, gW2, n, 1, [&](int i, int r, float z) { XW2[i * o + r] = z; });
    mm(Cc, o, n, X1, n, 1, gS2, n, 1, [&](int i, int r, float z) { XS2[i * o + r] = z; });
    __syncthreads();
    // coefficient gradients: dc_i = -<gW, u_i>, de_i = -<gS, u_i>
    for (int i = threadIdx.x / 32; i < Cc; i += NT / 32) {
      float x = 0.f, y = 0.f;
      for (int j = threadIdx.x % 32; j < n; j += 32) {
        x = fmaf(G1[i * n + j], KW1[i * n + j], x);
        y = fmaf(G1[i * n + j], KS1[i * n + j], y);
      }
      for (int r = threadIdx.x % 32; r < o; r += 32) {
        x = fmaf(G2[i * o + r], XW2[i * o + r], x);
        y = fmaf(G2[i * o + r], XS2[i * o + r], y);
      }
      x = warp_sum_simt(x);
      y = warp_sum_simt(y);
      if (threadIdx.x % 32 == 0) {
        dc[i] = -x;
        de[i] = -y;
      }
    }
    __syncthreads();
    // a = M1 k (into KW1), b = M2 x1 (into XW2); dH (T1), dSP (T2)
    for (int e = threadIdx.x; e < Cc * n; e += NT) {
      const int i = e / n;
      const float av = -(sm.coef.c[i] * KW1[e] + sm.coef.e[i] * KS1[e]);
      KW1[e] = av;
      T1[e] = av * silu_prime(Z1[e]);
      T2[e] = av * H[e];
    }
    for (int e = threadIdx.x; e < Cc * o; e += NT) {
      const int i = e / o;
      XW2[e] = -(sm.coef.c[i] * XW2[e] + sm.coef.e[i] * XS2[e]);
    }
    __syncthreads();
    // dG2 = b + dH W2^T (TO)
    mm(Cc, o, n, T1, n, 1, W2, n, 1, [&](int i, int r, float z) { TO[i * o + r] = z + XW2[i * o + r]; });
    __syncthreads();
    // state gradient of W2: B gW2 + G2^T dH + 2 dG2^T X1 + DY^T XQ
    const float Bw = sm.coef.Bw, As = sm.coef.As, cS = sm.coef.cS;
    float *gWn1 = gWn, *gWn2 = gWn + nd;
    mm(o, n, Cc, G2, 1, o, T1, 1, n, [&](int r, int j, float z) { gWn2[r * n + j] = Bw * gW2[r * n + j] + z; });
    __syncthreads();
    mm(o, n, Cc, TO, 1, o, X1, 1, n, [&](int r, int j, float z) { gWn2[r * n + j] += 2.f * z; });
    __syncthreads();
    mm(o, n, Cc, DY, 1, o, XQ, 1, n, [&](int r, int j, float z) { gWn2[r * n + j] += z; });
    __syncthreads();
    const long long gt_in = (tok0 + t0) * d, gt_out = (tok0 + t0) * o;
    for (int e = threadIdx.x; e < Cc * o; e += NT) a.dv[gt_out + e] = -2.f * TO[e];
    // dX1 = 2 dG2 W2 - c (G2 gW2) - e (G2 gS2)  (into T1, dH no longer needed)
    mm(Cc, n, o, TO, o, 1, W2, 1, n, [&](int i, int j, float z) { T1[i * n + j] = 2.f * z; });
    __syncthreads();
    mm(Cc, n, o, G2, o, 1, gW2, 1, n, [&](int i, int j, float z) { T1[i * n + j] -= sm.coef.c[i] * z; });
    __syncthreads();
    mm(Cc, n, o, G2, o, 1, gS2, 1, n, [&](int i, int j, float z) { T1[i * n + j] -= sm.coef.e[i] * z; });
    __syncthreads();
    // dZ1 = dX1 . silu'(z1) + dSP . silu''(z1)  (T1)
    for (int e = threadIdx.x; e < Cc * n; e += NT) T1[e] = T1[e] * silu_prime(Z1[e]) + T2[e] * silu_second(Z1[e]);
    __syncthreads();
    // reads: dZQ = (DY W2) . silu'(zq)  (T2)
    mm(Cc, n, o, DY, o, 1, W2, 1, n, [&](int i, int j, float z) { T2[i * n + j] = z * silu_prime(ZQ[i * n + j]); });
    __syncthreads();
    // state gradient of W1: B gW1 + dZ1^T K + dZQ^T Q
    mm(n, d, Cc, T1, 1, n, K, 1, d, [&](int j, int mm, float z) { gWn1[j * d + mm] = Bw * gW1[j * d + mm] + z; });
    __syncthreads();
    mm(n, d, Cc, T2, 1, n, Q, 1, d, [&](int j, int mm, float z) { gWn1[j * d + mm] += z; });
    __syncthreads();
    // dk = dZ1 W1 - c (G1 gW1) - e (G1 gS1);  dq = dZQ W1
    mm(Cc, d, n, T1, n, 1, W1, 1, d, [&](int i, int mm, float z) { a.dk[gt_in + i * d + mm] = z; });
    __syncthreads();
    mm(Cc, d, n, G1, n, 1, gW1, 1, d, [&](int i, int mm, float z) { a.dk[gt_in + i * d + mm] -= sm.coef.c[i] * z; });
    __syncthreads();
    mm(Cc, d, n, G1, n, 1, gS1, 1, d, [&](int i, int mm, float z) { a.dk[gt_in + i * d + mm] -= sm.coef.e[i] * z; });
    __syncthreads();
    mm(Cc, d, n, T2, n, 1, W1, 1, d, [&](int i, int mm, float z) { a.dq[gt_in + i * d + mm] = z; });
    // chunk scalars
    float pw = 0.f, pws = 0.f, pss = 0.f;
    for (long long e = threadIdx.x; e < P; e += NT) {
      pw = fmaf(gW[e], W1[e], pw);
      pws = fmaf(gW[e], S[e], pws);
      pss = fmaf(gS[e], S[e], pss);
    }
    const float dB = block_sum(pw, red), dcS = block_sum(pws, red), dA = block_sum(pss, red);
    if (threadIdx.x == 0)
      gate_reverse(Cc, th, et, al, dc, de, dB, dA, dcS, a.dtheta + tok0 + t0, a.deta + tok0 + t0,
                   a.dalpha + tok0 + t0, pa, pe, rho, dpa, dpe, drho);
    for (long long e = threadIdx.x; e < P; e += NT) {
      gS[e] = cS * gW[e] + As * gS[e];
      gW[e] = gWn[e];
    }
    __syncthreads();
  }
  for (long long e = threadIdx.x; e < P; e += NT) {
    a.dW0[sw + e] = gW[e];
    a.dS0[sw + e] = gS[e];
  }
  if constexpr (TC) tcg_release(tg);
}


// ---------------------------------------------------------------------------
// The same gradients for any depth L (used for depths 3 and 4). With
// x_0 = k, z_l = W_l x_{l-1}, x_l = silu(z_l) (x_L = z_L), g_L = 2 (x_L - v),
// h_{l-1} = W_l^T g_l, g_{l-1} = h_{l-1} . silu'(z_{l-1}), the surprise enters
// J through sum_l g_l^T a_l with a_l = M_l x_{l-1}. Reverse mode:
//   dg_l = a_l, dx_{l-1} = M_l^T g_l                      (for every l)
//   l = 2..L:  dh = dg_{l-1} . silu'(z_{l-1});  dsp_{l-1} = dg_{l-1} . h_{l-1}
//              dW_l += g_l dh^T;  dg_l += dh W_l^T
//   dx_L += 2 dg_L;  dv = -2 dg_L
//   l = L..1:  dz = dx_l . silu'(z_l) + dsp_l . silu''(z_l)   (dz = dx_L at L)
//              dW_l += dz x_{l-1}^T;  dx_{l-1} += dz W_l;      dk = dx_0
// and the reads add their ordinary backward.
constexpr int BWL_ARRAYS = 2 + 9 * (kMaxL + 1) + 3;   // V, DY; 9 per level; P1, P2, dH

struct BArgsL {
  int L, T, C, bf16, maxw;
  int *status;                   // device status word (bounded waits of the tensor-core products)
  unsigned long long wait_ns;
  int inject;                    // test hook (tm_set_debug), tensor-core products only
  int dims[kMaxL + 1];
  long long off[kMaxL + 1];
  long long P;
  const void *k, *v, *q;
  const float *theta, *eta, *alpha, *W0, *S0, *dy, *dW_end, *dS_end;
  float *dk, *dv, *dq, *dtheta, *deta, *dalpha, *dW0, *dS0;
  float *scratch;
  long long scratch_per_stream;
};

__host__ __device__ inline long long backwardL_floats(long long P, int maxw, int T, int C) {
  const long long nch = (T + C - 1) / C;
  return 2 * nch * P + 5 * P + (long long)BWL_ARRAYS * C * maxw + 8LL * C;
}

template <bool TC>
__global__ void __launch_bounds__(NT) backwardL_kernel(BArgsL a) {
  __shared__ SmemT sm;
  __shared__ float red[NT / 32];
  extern __shared__ __align__(1024) unsigned char tcg_dyn[];
  __shared__ TcGemm tg;
  if constexpr (TC) tcg_init(tg, tcg_dyn, a.status, a.wait_ns, a.inject);
  // the chunk's products: tcgen05 (TF32 operands, fp32 accumulation) or fp32 FFMA tiles
  auto mm = [&](int M_, int N_, int K_, const float *A_, long long sam, long long sak, const float *B_,
                long long sbn, long long sbk, auto epi) {
    if constexpr (TC) tc_gemm(tg, M_, N_, K_, A_, sam, sak, B_, sbn, sbk, epi);
    else gemm(sm, M_, N_, K_, A_, sam, sak, B_, sbn, sbk, epi);
  };
  // the forward pass's state update of one layer (A6 + A7): on the tensor
  // cores as two products, U_W with the tokens' c and U_S with their e
  auto upd = [&](int rows, int cols, int Cn, const float *G, const float *X, float *Wl, float *Sl) {
    if constexpr (TC) {
      const Coef &cf = sm.coef;
      tc_gemm(tg, rows, cols, Cn, G, 1, rows, X, 1, cols, [&](int r, int c, float u) {
        const long long idx = (long long)r * cols + c;
        Wl[idx] = cf.Bw * Wl[idx] + cf.cS * Sl[idx] - u;
      }, cf.c);
      tc_gemm(tg, rows, cols, Cn, G, 1, rows, X, 1, cols, [&](int r, int c, float u) {
        const long long idx = (long long)r * cols + c;
        Sl[idx] = cf.As * Sl[idx] - u;
      }, cf.e);
    } else {
      update_layer(sm, rows, cols, Cn, G, X, Wl, Sl);
    }
  };
  const int s = blockIdx.x, L = a.L, T = a.T, C = a.C, mw = a.maxw;
  const int *nn = a.dims;
  const long long P = a.P;
  const int nch = (T + C - 1) / C;
  float *p = a.scratch + (long long)s * a.scratch_per_stream;
  float *ckW = p; p += (long long)nch * P;
  float *ckS = p; p += (long long)nch * P;
  float *Wc = p; p += P;
  float *Sc = p; p += P;
  float *gW = p; p += P;
  float *gS = p; p += P;
  float *gWn = p; p += P;
  auto take = [&]() { float *r = p; p += (long long)C * mw; return r; };
  float *V = take(), *DY = take();
  float *Xk[kMaxL + 1], *Zk[kMaxL + 1], *Gk[kMaxL + 1], *Hk[kMaxL + 1];
  float *Xq[kMaxL + 1], *Zq[kMaxL + 1], *dG[kMaxL + 1], *dSP[kMaxL + 1], *dX[kMaxL + 1], *dXq[kMaxL + 1];
  for (int l = 0; l <= kMaxL; ++l) {
    Xk[l] = take(); Zk[l] = take(); Gk[l] = take(); Hk[l] = take();
    Xq[l] = take(); Zq[l] = take(); dG[l] = take(); dSP[l] = take(); dX[l] = take();
  }
  for (int l = 0; l <= kMaxL; ++l) dXq[l] = dX[l];   // the reads reuse dX after the keys are done
  float *P1 = take(), *P2 = take(), *dH = take();
  float *dc = p; p += C;
  float *de = p; p += C;
  float *pa = p; p += C;
  float *pe = p; p += C;
  float *rho = p; p += C;
  float *dpa = p; p += C;
  float *dpe = p; p += C;
  float *drho = p; p += C;
  const long long sw = (long long)s * P, tok0 = (long long)s * T;
  const int d0 = nn[0], dL = nn[L];

  auto load_chunk = [&](int t0, int Cc, bool grads) {
    for (int i = threadIdx.x; i < Cc * d0; i += NT) {
      const long long g = (tok0 + t0) * d0 + i;
      Xk[0][i] = load_tok(a.k, a.bf16, g);
      if (grads) Xq[0][i] = load_tok(a.q, a.bf16, g);
    }
    for (int i = threadIdx.x; i < Cc * dL; i += NT) {
      const long long g = (tok0 + t0) * dL + i;
      V[i] = load_tok(a.v, a.bf16, g);
      if (grads) DY[i] = a.dy[g];
    }
    __syncthreads();
  };
  // forward of rows X[0] through W: Z[l], X[l] (X[L] = Z[L])
  auto forward = [&](int Cc, const float *W, float **X, float **Z) {
    for (int l = 1; l <= L; ++l) {
      const int r = nn[l], cl = nn[l - 1];
      float *Zl = Z[l], *Xl = X[l];
      const bool last = l == L;
      mm(Cc, r, cl, X[l - 1], cl, 1, W + a.off[l - 1], cl, 1, [&](int i, int j, float z) {
        Zl[i * r + j] = z;
        Xl[i * r + j] = last ? z : silu(z);
      });
      __syncthreads();
    }
  };
  // the keys' backward: G[L] = 2 (X[L] - V), H[l-1] = G[l] W_l, G[l-1] = H[l-1] . silu'(Z[l-1])
  auto keys_backward = [&](int Cc, const float *W) {
    for (int e = threadIdx.x; e < Cc * dL; e += NT) Gk[L][e] = 2.f * (Xk[L][e] - V[e]);
    __syncthreads();
    for (int l = L; l >= 2; --l) {
      const int r = nn[l], cl = nn[l - 1];
      float *Hl = Hk[l - 1], *Gl = Gk[l - 1], *Zl = Zk[l - 1];
      mm(Cc, cl, r, Gk[l], r, 1, W + a.off[l - 1], 1, cl, [&](int i, int j, float z) {
        Hl[i * cl + j] = z;
        Gl[i * cl + j] = z * silu_prime(Zl[i * cl + j]);
      });
      __syncthreads();
    }
  };
  // ---- forward: chunk-start states
  for (long long i = threadIdx.x; i < P; i += NT) {
    Wc[i] = a.W0[sw + i];
    Sc[i] = a.S0[sw + i];
  }
  __syncthreads();
  for (int c = 0; c < nch; ++c) {
    const int t0 = c * C, Cc = T - t0 < C ? T - t0 : C;
    for (long long i = threadIdx.x; i < P; i += NT) {
      ckW[(long long)c * P + i] = Wc[i];
      ckS[(long long)c * P + i] = Sc[i];
    }
    chunk_coefficients(sm.coef, a.theta + tok0 + t0, a.eta + tok0 + t0, a.alpha + tok0 + t0, Cc);
    load_chunk(t0, Cc, false);
    forward(Cc, Wc, Xk, Zk);
    keys_backward(Cc, Wc);
    for (int l = 1; l <= L; ++l) upd(nn[l], nn[l - 1], Cc, Gk[l], Xk[l - 1], Wc + a.off[l - 1], Sc + a.off[l - 1]);
    __syncthreads();
  }
  // ---- reverse
  for (long long i = threadIdx.x; i < P; i += NT) {
    gW[i] = a.dW_end[sw + i];
    gS[i] = a.dS_end[sw + i];
  }
  __syncthreads();
  for (int c = nch - 1; c >= 0; --c) {
    const int t0 = c * C, Cc = T - t0 < C ? T - t0 : C;
    const float *th = a.theta + tok0 + t0, *et = a.eta + tok0 + t0, *al = a.alpha + tok0 + t0;
    const float *W = ckW + (long long)c * P, *S = ckS + (long long)c * P;
    chunk_coefficients(sm.coef, th, et, al, Cc);
    load_chunk(t0, Cc, true);
    forward(Cc, W, Xk, Zk);
    keys_backward(Cc, W);
    forward(Cc, W, Xq, Zq);
    const float Bw = sm.coef.Bw, As = sm.coef.As, cS = sm.coef.cS;
    for (long long e = threadIdx.x; e < P; e += NT) gWn[e] = Bw * gW[e];
    for (int i = threadIdx.x; i < Cc; i += NT) { dc[i] = 0.f; de[i] = 0.f; }
    __syncthreads();
    // per layer: a_l = M_l x_{l-1} (dG[l]), dc, de, and dx_{l-1} = M_l^T g_l (dX[l-1])
    for (int l = 1; l <= L; ++l) {
      const int r = nn[l], cl = nn[l - 1];
      const float *gWl = gW + a.off[l - 1], *gSl = gS + a.off[l - 1];
      mm(Cc, r, cl, Xk[l - 1], cl, 1, gWl, cl, 1, [&](int i, int j, float z) { P1[i * r + j] = z; });
      mm(Cc, r, cl, Xk[l - 1], cl, 1, gSl, cl, 1, [&](int i, int j, float z) { P2[i * r + j] = z; });
      __syncthreads();
      for (int i = threadIdx.x / 32; i < Cc; i += NT / 32) {
        float x = 0.f, y = 0.f;
        for (int j = threadIdx.x % 32; j < r; j += 32) {
          x = fmaf(Gk[l][i * r + j], P1[i * r + j], x);
          y = fmaf(Gk[l][i * r + j], P2[i * r + j], y);
        }
        x = warp_sum_simt(x);
        y = warp_sum_simt(y);
        if (threadIdx.x % 32 == 0) { dc[i] -= x; de[i] -= y; }
      }
      for (int e = threadIdx.x; e < Cc * r; e += NT) {
        const int i = e / r;
        dG[l][e] = -(sm.coef.c[i] * P1[e] + sm.coef.e[i] * P2[e]);
      }
      __syncthreads();
      float *dXl = dX[l - 1];
      mm(Cc, cl, r, Gk[l], r, 1, gWl, 1, cl, [&](int i, int j, float z) { dXl[i * cl + j] = -sm.coef.c[i] * z; });
      __syncthreads();
      mm(Cc, cl, r, Gk[l], r, 1, gSl, 1, cl, [&](int i, int j, float z) { dXl[i * cl + j] -= sm.coef.e[i] * z; });
      __syncthreads();
    }
    // back through the keys' backward recursion
    for (int l = 2; l <= L; ++l) {
      const int r = nn[l], cl = nn[l - 1];
      for (int e = threadIdx.x; e < Cc * cl; e += NT) {
        dH[e] = dG[l - 1][e] * silu_prime(Zk[l - 1][e]);
        dSP[l - 1][e] = dG[l - 1][e] * Hk[l - 1][e];
      }
      __syncthreads();
      float *gWnl = gWn + a.off[l - 1], *dGl = dG[l];
      mm(r, cl, Cc, Gk[l], 1, r, dH, 1, cl, [&](int rr, int j, float z) { gWnl[rr * cl + j] += z; });
      __syncthreads();
      mm(Cc, r, cl, dH, cl, 1, W + a.off[l - 1], cl, 1, [&](int i, int rr, float z) { dGl[i * r + rr] += z; });
      __syncthreads();
    }
    const long long gout = (tok0 + t0) * dL, gin = (tok0 + t0) * d0;
    for (int e = threadIdx.x; e < Cc * dL; e += NT) {
      dX[L][e] = 2.f * dG[L][e];
      a.dv[gout + e] = -2.f * dG[L][e];
    }
    __syncthreads();
    // back through the keys' forward
    for (int l = L; l >= 1; --l) {
      const int r = nn[l], cl = nn[l - 1];
      float *dZ = dH;
      if (l == L) {
        for (int e = threadIdx.x; e < Cc * r; e += NT) dZ[e] = dX[L][e];
      } else {
        for (int e = threadIdx.x; e < Cc * r; e += NT)
          dZ[e] = dX[l][e] * silu_prime(Zk[l][e]) + dSP[l][e] * silu_second(Zk[l][e]);
      }
      __syncthreads();
      float *gWnl = gWn + a.off[l - 1], *dXl = dX[l - 1];
      mm(r, cl, Cc, dZ, 1, r, Xk[l - 1], 1, cl, [&](int rr, int j, float z) { gWnl[rr * cl + j] += z; });
      __syncthreads();
      mm(Cc, cl, r, dZ, r, 1, W + a.off[l - 1], 1, cl, [&](int i, int j, float z) { dXl[i * cl + j] += z; });
      __syncthreads();
    }
    for (int e = threadIdx.x; e < Cc * d0; e += NT) a.dk[gin + e] = dX[0][e];
    __syncthreads();
    // the reads: ordinary backward of y = M(q)
    for (int e = threadIdx.x; e < Cc * dL; e += NT) dXq[L][e] = DY[e];
    __syncthreads();
    for (int l = L; l >= 1; --l) {
      const int r = nn[l], cl = nn[l - 1];
      float *dZ = dH;
      for (int e = threadIdx.x; e < Cc * r; e += NT) dZ[e] = l == L ? dXq[L][e] : dXq[l][e] * silu_prime(Zq[l][e]);
      __syncthreads();
      float *gWnl = gWn + a.off[l - 1], *dXl = dXq[l - 1];
      mm(r, cl, Cc, dZ, 1, r, Xq[l - 1], 1, cl, [&](int rr, int j, float z) { gWnl[rr * cl + j] += z; });
      __syncthreads();
      mm(Cc, cl, r, dZ, r, 1, W + a.off[l - 1], 1, cl, [&](int i, int j, float z) { dXl[i * cl + j] = z; });
      __syncthreads();
    }
    for (int e = threadIdx.x; e < Cc * d0; e += NT) a.dq[gin + e] = dXq[0][e];
    // chunk scalars, gates, state gradients
    float pw = 0.f, pws = 0.f, pss = 0.f;
    for (long long e = threadIdx.x; e < P; e += NT) {
      pw = fmaf(gW[e], W[e], pw);
      pws = fmaf(gW[e], S[e], pws);
      pss = fmaf(gS[e], S[e], pss);
    }
    const float dB = block_sum(pw, red), dcS = block_sum(pws, red), dA = block_sum(pss, red);
    if (threadIdx.x == 0)
      gate_reverse(Cc, th, et, al, dc, de, dB, dA, dcS, a.dtheta + tok0 + t0, a.deta + tok0 + t0,
                   a.dalpha + tok0 + t0, pa, pe, rho, dpa, dpe, drho);
    for (long long e = threadIdx.x; e < P; e += NT) {
      gS[e] = cS * gW[e] + As * gS[e];
      gW[e] = gWn[e];
    }
    __syncthreads();
  }
  for (long long e = threadIdx.x; e < P; e += NT) {
    a.dW0[sw + e] = gW[e];
    a.dS0[sw + e] = gS[e];
  }
  if constexpr (TC) tcg_release(tg);
}

}  // namespace

size_t simt_scratch_bytes(const Problem &p) {
  long long per = 0;
  int maxw = 0;
  for (int l = 0; l <= p.L; ++l) maxw = p.dims[l] > maxw ? p.dims[l] : maxw;
  for (int l = 0; l < p.L; ++l) per += (long long)p.C * p.dims[l];
  for (int l = 1; l < p.L; ++l) per += (long long)p.C * p.dims[l];
  per += 4LL * p.C * maxw;
  per = (per + 63) / 64 * 64;
  return (size_t)per * sizeof(float) * (size_t)p.streams;
}

cudaError_t simt_launch(const Problem &p, cudaStream_t stream) {
  KArgs a;
  a.net.L = p.L;
  a.net.maxw = 0;
  for (int l = 0; l <= p.L; ++l) {
    a.net.dims[l] = p.dims[l];
    a.net.off[l] = (long long)p.layer_off[l];
    a.net.maxw = p.dims[l] > a.net.maxw ? p.dims[l] : a.net.maxw;
  }
  a.net.P = (long long)p.P;
  a.T = p.T;
  a.C = p.C;
  a.t_begin = p.t_begin;
  a.bf16 = p.in_dtype == TM_BF16;
  a.k = p.k; a.v = p.v; a.q = p.q;
  a.theta = p.theta; a.eta = p.eta; a.alpha = p.alpha;
  a.W0 = p.W0; a.S0 = p.S0;
  a.y = p.y; a.W = p.W_end; a.S = p.S_end;
  a.scratch = reinterpret_cast<float *>(p.scratch);
  a.scratch_per_stream = (long long)(simt_scratch_bytes(p) / sizeof(float) / (size_t)p.streams);
  a.status = p.status;
  simt_chunk_kernel<<<p.streams, NT, 0, stream>>>(a);
  return cudaGetLastError();
}

bool backward_supported(const Problem &p) { return p.L >= 1 && p.L <= kMaxL && p.C <= kMaxC; }

size_t backward_scratch_bytes(const Problem &p) {
  const long long d = p.dims[0], C = p.C, nch = (p.T + p.C - 1) / p.C;
  int maxw = 0;
  for (int l = 0; l <= p.L; ++l) maxw = p.dims[l] > maxw ? p.dims[l] : maxw;
  const long long per = p.L == 1   ? 2 * nch * d * d + 5 * d * d + 10 * C * d + 8 * C
                        : p.L == 2 ? backward2_floats(p.dims[0], p.dims[1], p.dims[2], p.T, p.C)
                                   : backwardL_floats((long long)p.P, maxw, p.T, p.C);
  return (size_t)(per * p.streams) * sizeof(float);
}

cudaError_t backward_launch(const Problem &p, const float *dy, const float *dW_end, const float *dS_end,
                            float *dk, float *dv, float *dq, float *dtheta, float *deta, float *dalpha,
                            float *dW0, float *dS0, cudaStream_t stream) {
  if (!backward_supported(p)) return cudaErrorNotSupported;
  if (p.bw_tc) {
    static bool attr_done = false;
    if (!attr_done) {
      const void *kerns[3] = {(const void *)backward1_kernel<true>, (const void *)backward2_kernel<true>,
                              (const void *)backwardL_kernel<true>};
      for (const void *k : kerns) {
        const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TCG_SMEM);
        if (e != cudaSuccess) return e;
      }
      attr_done = true;
    }
  }
  if (p.L >= 3) {
    BArgsL b;
    b.L = p.L;
    b.T = p.T;
    b.C = p.C;
    b.bf16 = p.in_dtype == TM_BF16 ? 1 : 0;
    b.maxw = 0;
    for (int l = 0; l <= kMaxL; ++l) {
      b.dims[l] = l <= p.L ? p.dims[l] : 0;
      b.off[l] = l <= p.L ? (long long)p.layer_off[l] : 0;
      if (l <= p.L && p.dims[l] > b.maxw) b.maxw = p.dims[l];
    }
    b.P = (long long)p.P;
    b.k = p.k; b.v = p.v; b.q = p.q;
    b.theta = p.theta; b.eta = p.eta; b.alpha = p.alpha;
    b.W0 = p.W0; b.S0 = p.S0;
    b.dy = dy; b.dW_end = dW_end; b.dS_end = dS_end;
    b.dk = dk; b.dv = dv; b.dq = dq; b.dtheta = dtheta; b.deta = deta; b.dalpha = dalpha;
    b.dW0 = dW0; b.dS0 = dS0;
    b.scratch = static_cast<float *>(p.scratch);
    b.scratch_per_stream = backwardL_floats(b.P, b.maxw, p.T, p.C);
    b.status = p.status;
    b.wait_ns = tcl_wait_ns();
    b.inject = tcl_inject();
    if (p.bw_tc) backwardL_kernel<true><<<p.streams, NT, TCG_SMEM, stream>>>(b);
    else backwardL_kernel<false><<<p.streams, NT, 0, stream>>>(b);
    return cudaGetLastError();
  }
  if (p.L == 2) {
    BArgs2 b;
    b.d = p.dims[0];
    b.n = p.dims[1];
    b.o = p.dims[2];
    b.T = p.T;
    b.C = p.C;
    b.bf16 = p.in_dtype == TM_BF16 ? 1 : 0;
    b.P = (long long)p.P;
    b.k = p.k; b.v = p.v; b.q = p.q;
    b.theta = p.theta; b.eta = p.eta; b.alpha = p.alpha;
    b.W0 = p.W0; b.S0 = p.S0;
    b.dy = dy; b.dW_end = dW_end; b.dS_end = dS_end;
    b.dk = dk; b.dv = dv; b.dq = dq; b.dtheta = dtheta; b.deta = deta; b.dalpha = dalpha;
    b.dW0 = dW0; b.dS0 = dS0;
    b.scratch = static_cast<float *>(p.scratch);
    b.scratch_per_stream = backward2_floats(b.d, b.n, b.o, p.T, p.C);
    b.status = p.status;
    b.wait_ns = tcl_wait_ns();
    b.inject = tcl_inject();
    if (p.bw_tc) backward2_kernel<true><<<p.streams, NT, TCG_SMEM, stream>>>(b);
    else backward2_kernel<false><<<p.streams, NT, 0, stream>>>(b);
    return cudaGetLastError();
  }
  BArgs a;
  const long long d = p.dims[0], C = p.C, nch = (p.T + p.C - 1) / p.C;
  a.d = (int)d;
  a.T = p.T;
  a.C = p.C;
  a.bf16 = p.in_dtype == TM_BF16 ? 1 : 0;
  a.k = p.k; a.v = p.v; a.q = p.q;
  a.theta = p.theta; a.eta = p.eta; a.alpha = p.alpha;
  a.W0 = p.W0; a.S0 = p.S0;
  a.dy = dy; a.dW_end = dW_end; a.dS_end = dS_end;
  a.dk = dk; a.dv = dv; a.dq = dq; a.dtheta = dtheta; a.deta = deta; a.dalpha = dalpha;
  a.dW0 = dW0; a.dS0 = dS0;
  a.scratch = static_cast<float *>(p.scratch);
  a.scratch_per_stream = 2 * nch * d * d + 5 * d * d + 10 * C * d + 8 * C;
  a.status = p.status;
  a.wait_ns = tcl_wait_ns();
  a.inject = tcl_inject();
  if (p.bw_tc) backward1_kernel<true><<<p.streams, NT, TCG_SMEM, stream>>>(a);
  else backward1_kernel<false><<<p.streams, NT, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace tmem
