// C-ABI of libtitansmem: argument checks, workspace accounting, kernel choice.
// The operation each entry point performs is documented in include/titansmem.h.
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "tm_internal.h"

struct tm_ctx {
  int L;
  int d;
  int expansion;
  int dims[tmem::kMaxL + 1];
  size_t layer_off[tmem::kMaxL + 1];
  size_t P;
  tm_path path;
  // layered path: side CUDA streams and events, created on first use on
  // device `dev`; one context's calls must not run concurrently
  int dev = -1;
  cudaStream_t side[tmem::kMaxGroups - 1] = {};
  cudaEvent_t ev_fork = nullptr;
  cudaEvent_t ev_join[tmem::kMaxGroups - 1] = {};
  // layered path: its per-chunk launches as one CUDA graph, captured when a
  // call repeats the previous call exactly (shapes, pointers, settings) and
  // replayed while calls keep repeating it; the launch sequence is long
  // (two launches per chunk and group) and the host's enqueue rate would
  // otherwise pace the GPU
  struct Key {
    int v[12];
    const void *ptr[12];
  };
  Key seen{}, graph_key{};
  bool has_seen = false;
  cudaStream_t cap = nullptr;
  cudaGraphExec_t exec = nullptr;
  // tm_run_host: copy streams (host -> device, device -> host) and the
  // events that order them against the kernels, created on first use on
  // device `hdev`
  int hdev = -1;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t h_start = nullptr, h_done = nullptr, h_state = nullptr;
  cudaEvent_t in_ready[2] = {}, in_free[2] = {}, y_ready[2] = {}, y_free[2] = {};
};

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb) {
  auto x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

tm_status check_shape(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype dt) {
  if (!ctx) return TM_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || T < 1 || C < 1) return TM_ERR_INVALID_ARG;
  if (C > tmem::kMaxC) return TM_ERR_INVALID_ARG;
  if (dt != TM_F32 && dt != TM_BF16) return TM_ERR_INVALID_ARG;
  if ((long long)B * H > (1LL << 31) - 1) return TM_ERR_INVALID_ARG;
  return TM_OK;
}

tmem::Problem make_problem(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype dt) {
  tmem::Problem p{};
  p.L = ctx->L;
  for (int l = 0; l <= ctx->L; ++l) {
    p.dims[l] = ctx->dims[l];
    p.layer_off[l] = ctx->layer_off[l];
  }
  p.P = ctx->P;
  p.B = B;
  p.H = H;
  p.T = T;
  p.C = C;
  p.streams = B * H;
  p.in_dtype = dt;
  p.fuse_fb = 1;
  p.tc_global = ctx->path == TM_PATH_TC_GLOBAL;
  // the tensor-core paths run the whole chunks; a shorter last chunk
  // (T % C tokens) runs after them on the CUDA-core kernel
  p.T_run = T - T % C;
  p.t_begin = 0;
  return p;
}

tm_path choose_path(const tm_ctx *ctx, const tmem::Problem &p) {
  if (ctx->path != TM_PATH_AUTO) return ctx->path;
  if (p.in_dtype == TM_BF16 && tmem::tc_supported(p)) return TM_PATH_TC;
  if (p.in_dtype == TM_BF16 && tmem::tcl_supported(p)) return TM_PATH_TC_LAYERED;
  return TM_PATH_SIMT;
}

bool path_supported(tm_path path, const tmem::Problem &p) {
  if (path == TM_PATH_TC || path == TM_PATH_TC_GLOBAL) return tmem::tc_supported(p);
  if (path == TM_PATH_TC_LAYERED || path == TM_PATH_TC_PHASED) return tmem::tcl_supported(p);
  return true;
}

bool tensor_path(tm_path path) {
  return path == TM_PATH_TC || path == TM_PATH_TC_GLOBAL || path == TM_PATH_TC_LAYERED ||
         path == TM_PATH_TC_PHASED;
}

// Bytes at the start of the workspace (after the status word) that hold the
// fp16 copies of keys and queries on the tensor-core paths.
size_t f16_bytes(tm_path path, const tmem::Problem &p) { return tensor_path(path) ? tmem::tokens_f16_bytes(p) : 0; }

// Workspace after the status word: the fp16 token copies (tensor-core paths),
// then the kernels' scratch. A tensor-core path with a shorter last chunk runs
// it afterwards on the CUDA-core kernel, in the same scratch space.
size_t scratch_bytes(tm_path path, const tmem::Problem &p) {
  size_t b = tmem::simt_scratch_bytes(p);
  if (!tensor_path(path)) return b;
  size_t m = (path == TM_PATH_TC || path == TM_PATH_TC_GLOBAL) ? tmem::tc_scratch_bytes(p)
                                                              : tmem::tcl_scratch_bytes(p);
  if (p.T_run < p.T && b > m) m = b;
  return f16_bytes(path, p) + m;
}

}  // namespace

namespace tmem {
// Validated problem description of a context, for entry points that live in
// other translation units.
bool problem_from_ctx(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype dt, Problem *out) {
  if (!out || check_shape(ctx, B, H, T, C, dt) != TM_OK) return false;
  *out = make_problem(ctx, B, H, T, C, dt);
  return true;
}

bool run_aliasing_ok(const Problem &p, const void *k, const void *v, const void *q, const float *theta,
                     const float *eta, const float *alpha, const float *W0, const float *S0, const float *y,
                     const float *W_end, const float *S_end) {
  const size_t tok_el = p.in_dtype == TM_BF16 ? 2 : 4;
  const size_t ntok = (size_t)p.streams * (size_t)p.T;
  const size_t d = (size_t)p.dims[0];
  const size_t tok_bytes = ntok * d * tok_el;
  const size_t y_bytes = ntok * d * 4;
  const size_t gate_bytes = ntok * 4;
  const size_t st_bytes = (size_t)p.streams * p.P * 4;
  // y must not overlap any input or other output.
  const void *ins[] = {k, v, q, theta, eta, alpha, W0, S0, W_end, S_end};
  const size_t insz[] = {tok_bytes, tok_bytes, tok_bytes, gate_bytes, gate_bytes, gate_bytes,
                         st_bytes, st_bytes, st_bytes, st_bytes};
  for (int i = 0; i < 10; ++i)
    if (ranges_overlap(y, y_bytes, ins[i], insz[i])) return false;
  // W_end may equal W0 exactly (in place) but not partially overlap anything else.
  if (W_end != W0 && ranges_overlap(W_end, st_bytes, W0, st_bytes)) return false;
  if (S_end != S0 && ranges_overlap(S_end, st_bytes, S0, st_bytes)) return false;
  if (ranges_overlap(W_end, st_bytes, S_end, st_bytes)) return false;
  if (ranges_overlap(W_end, st_bytes, S0, st_bytes)) return false;
  if (ranges_overlap(S_end, st_bytes, W0, st_bytes)) return false;
  // the state outputs must not overlap the token inputs or the gates
  const void *tin[] = {k, v, q, theta, eta, alpha};
  for (int i = 0; i < 6; ++i)
    if (ranges_overlap(W_end, st_bytes, tin[i], insz[i]) || ranges_overlap(S_end, st_bytes, tin[i], insz[i]))
      return false;
  return true;
}
}  // namespace tmem

extern "C" {

tm_status tm_create(int L, int d_h, int expansion, tm_act act, tm_ctx **out) {
  if (!out) return TM_ERR_INVALID_ARG;
  *out = nullptr;
  if (L < 1 || L > tmem::kMaxL || d_h < 1 || d_h > 1024 || d_h % 4 != 0) return TM_ERR_INVALID_ARG;
  if (act != TM_ACT_SILU) return TM_ERR_INVALID_ARG;
  if (L > 1 && (expansion < 1 || (long long)expansion * d_h > 4096)) return TM_ERR_INVALID_ARG;
  tm_ctx *c = new (std::nothrow) tm_ctx();
  if (!c) return TM_ERR_OOM;
  c->L = L;
  c->d = d_h;
  c->expansion = L > 1 ? expansion : 1;
  c->dims[0] = d_h;
  for (int l = 1; l < L; ++l) c->dims[l] = expansion * d_h;
  c->dims[L] = d_h;
  size_t off = 0;
  for (int l = 1; l <= L; ++l) {
    c->layer_off[l - 1] = off;
    off += (size_t)c->dims[l] * c->dims[l - 1];
  }
  c->layer_off[L] = off;
  c->P = off;
  c->path = TM_PATH_AUTO;
  *out = c;
  return TM_OK;
}

namespace {

void drop_graph(tm_ctx *ctx) {
  if (ctx->exec) cudaGraphExecDestroy(ctx->exec);
  ctx->exec = nullptr;
}

void release_host(tm_ctx *ctx) {
  cudaStream_t st[] = {ctx->h2d, ctx->d2h};
  for (cudaStream_t x : st)
    if (x) cudaStreamDestroy(x);
  ctx->h2d = ctx->d2h = nullptr;
  cudaEvent_t *evs[] = {&ctx->h_start, &ctx->h_done, &ctx->h_state, &ctx->in_ready[0], &ctx->in_ready[1],
                        &ctx->in_free[0], &ctx->in_free[1], &ctx->y_ready[0], &ctx->y_ready[1],
                        &ctx->y_free[0], &ctx->y_free[1]};
  for (cudaEvent_t *e : evs) {
    if (*e) cudaEventDestroy(*e);
    *e = nullptr;
  }
  ctx->hdev = -1;
}

// Copy streams and events of tm_run_host on the current device.
bool ensure_host(tm_ctx *ctx) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (ctx->hdev != dev) release_host(ctx);
  ctx->hdev = dev;
  cudaStream_t *st[] = {&ctx->h2d, &ctx->d2h};
  for (cudaStream_t *x : st)
    if (!*x && cudaStreamCreateWithFlags(x, cudaStreamNonBlocking) != cudaSuccess) return false;
  cudaEvent_t *evs[] = {&ctx->h_start, &ctx->h_done, &ctx->h_state, &ctx->in_ready[0], &ctx->in_ready[1],
                        &ctx->in_free[0], &ctx->in_free[1], &ctx->y_ready[0], &ctx->y_ready[1],
                        &ctx->y_free[0], &ctx->y_free[1]};
  for (cudaEvent_t *e : evs)
    if (!*e && cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
  return true;
}

void release_side(tm_ctx *ctx) {
  drop_graph(ctx);
  ctx->has_seen = false;
  if (ctx->cap) cudaStreamDestroy(ctx->cap);
  ctx->cap = nullptr;
  for (int i = 0; i < tmem::kMaxGroups - 1; ++i) {
    if (ctx->side[i]) cudaStreamDestroy(ctx->side[i]);
    if (ctx->ev_join[i]) cudaEventDestroy(ctx->ev_join[i]);
    ctx->side[i] = nullptr;
    ctx->ev_join[i] = nullptr;
  }
  if (ctx->ev_fork) cudaEventDestroy(ctx->ev_fork);
  ctx->ev_fork = nullptr;
  ctx->dev = -1;
}

// Side streams and events for `groups` concurrent groups, on the current device.
bool ensure_side(tm_ctx *ctx, int groups) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (ctx->dev != dev) release_side(ctx);
  ctx->dev = dev;
  if (groups > 1 && !ctx->ev_fork &&
      cudaEventCreateWithFlags(&ctx->ev_fork, cudaEventDisableTiming) != cudaSuccess)
    return false;
  for (int i = 0; i < groups - 1; ++i) {
    if (!ctx->side[i] && cudaStreamCreateWithFlags(&ctx->side[i], cudaStreamNonBlocking) != cudaSuccess)
      return false;
    if (!ctx->ev_join[i] && cudaEventCreateWithFlags(&ctx->ev_join[i], cudaEventDisableTiming) != cudaSuccess)
      return false;
  }
  return true;
}

tm_ctx::Key run_key(const tm_ctx *ctx, tm_path path, const tmem::Problem &p) {
  tm_ctx::Key k;
  std::memset(&k, 0, sizeof k);
  const unsigned long long w = tmem::tcl_wait_ns();
  const int v[] = {(int)path, p.B, p.H, p.T, p.C, (int)p.in_dtype, tmem::tcl_group_count(p), ctx->dev,
                   (int)(w & 0x7fffffff), (int)(w >> 31), p.T_run, tmem::tcl_inject()};
  std::memcpy(k.v, v, sizeof v);
  const void *ptr[] = {p.k, p.v, p.q, p.theta, p.eta, p.alpha, p.W0, p.S0, p.y, p.W_end, p.S_end, p.scratch};
  std::memcpy(k.ptr, ptr, sizeof ptr);
  return k;
}

bool same_key(const tm_ctx::Key &a, const tm_ctx::Key &b) { return std::memcmp(&a, &b, sizeof a) == 0; }

// Captures the layered launch sequence of `p` into ctx->exec. On any failure
// the capture is discarded and the caller launches directly.
bool capture_layered(tm_ctx *ctx, const tmem::Problem &p, const tm_ctx::Key &key) {
  drop_graph(ctx);
  if (!ctx->cap && cudaStreamCreateWithFlags(&ctx->cap, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (cudaStreamBeginCapture(ctx->cap, cudaStreamCaptureModeRelaxed) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const cudaError_t e = tmem::tcl_launch(p, ctx->cap);
  cudaGraph_t g = nullptr;
  const cudaError_t e2 = cudaStreamEndCapture(ctx->cap, &g);
  bool ok = e == cudaSuccess && e2 == cudaSuccess && g != nullptr;
  if (ok) ok = cudaGraphInstantiate(&ctx->exec, g, 0) == cudaSuccess;
  if (g) cudaGraphDestroy(g);
  if (!ok) {
    ctx->exec = nullptr;
    cudaGetLastError();
    return false;
  }
  ctx->graph_key = key;
  return true;
}

// The layered path: graph replay when the call repeats, else direct launches.
// While the caller captures `s` into a graph of its own, the launches go
// straight into that capture.
cudaError_t run_layered(tm_ctx *ctx, tm_path path, const tmem::Problem &p, cudaStream_t s) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return tmem::tcl_launch(p, s);
  }
  const tm_ctx::Key key = run_key(ctx, path, p);
  if (ctx->exec && same_key(key, ctx->graph_key)) return cudaGraphLaunch(ctx->exec, s);
  if (ctx->has_seen && same_key(key, ctx->seen) && capture_layered(ctx, p, key))
    return cudaGraphLaunch(ctx->exec, s);
  ctx->seen = key;
  ctx->has_seen = true;
  return tmem::tcl_launch(p, s);
}

}  // namespace

tm_status tm_destroy(tm_ctx *ctx) {
  if (ctx) {
    release_side(ctx);
    release_host(ctx);
  }
  delete ctx;
  return TM_OK;
}

size_t tm_param_count(const tm_ctx *ctx) { return ctx ? ctx->P : 0; }

tm_status tm_set_path(tm_ctx *ctx, tm_path path) {
  if (!ctx) return TM_ERR_INVALID_ARG;
  if (path != TM_PATH_AUTO && path != TM_PATH_SIMT && path != TM_PATH_TC && path != TM_PATH_TC_LAYERED &&
      path != TM_PATH_TC_PHASED && path != TM_PATH_TC_GLOBAL)
    return TM_ERR_INVALID_ARG;
  ctx->path = path;
  return TM_OK;
}

tm_status tm_query_path(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                        tm_path *out) {
  if (!out) return TM_ERR_INVALID_ARG;
  tm_status st = check_shape(ctx, B, H, T, C, in_dtype);
  if (st != TM_OK) return st;
  tmem::Problem p = make_problem(ctx, B, H, T, C, in_dtype);
  tm_path path = choose_path(ctx, p);
  if (!path_supported(path, p)) return TM_ERR_UNSUPPORTED;
  *out = path;
  return TM_OK;
}

tm_status tm_launch_count(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                          long long *out) {
  if (!out) return TM_ERR_INVALID_ARG;
  tm_status st = check_shape(ctx, B, H, T, C, in_dtype);
  if (st != TM_OK) return st;
  tmem::Problem p = make_problem(ctx, B, H, T, C, in_dtype);
  tm_path path = choose_path(ctx, p);
  if (!path_supported(path, p)) return TM_ERR_UNSUPPORTED;
  p.fuse_fb = path == TM_PATH_TC_LAYERED;
  long long n = 1;
  if (tensor_path(path)) {
    n = p.T_run == 0 ? 0
        : 1 + ((path == TM_PATH_TC_LAYERED || path == TM_PATH_TC_PHASED) ? tmem::tcl_launch_count(p)
                                                                         : tmem::tc_launch_count(p));
    if (p.T_run < p.T) n += 1;                 // the shorter last chunk
  }
  *out = n;
  return TM_OK;
}

tm_status tm_workspace_size(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                            size_t *bytes) {
  if (!bytes) return TM_ERR_INVALID_ARG;
  tm_status st = check_shape(ctx, B, H, T, C, in_dtype);
  if (st != TM_OK) return st;
  tmem::Problem p = make_problem(ctx, B, H, T, C, in_dtype);
  tm_path path = choose_path(ctx, p);
  if (!path_supported(path, p)) return TM_ERR_UNSUPPORTED;
  *bytes = tmem::kStatusBytes + scratch_bytes(path, p);
  return TM_OK;
}

}  // extern "C"

namespace {

// tm_run's work; clear_status = false keeps the device status word as it is
// (tm_run_host clears it once for all of its segments).
tm_status run_device(tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype, const void *k,
                     const void *v, const void *q, const float *theta, const float *eta,
                     const float *alpha, const float *W0, const float *S0, float *y, float *W_end,
                     float *S_end, void *workspace, size_t workspace_bytes, void *stream, bool clear_status) {
  tm_status st = check_shape(ctx, B, H, T, C, in_dtype);
  if (st != TM_OK) return st;
  const void *ptrs[] = {k, v, q, theta, eta, alpha, W0, S0, y, W_end, S_end, workspace};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return TM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TM_ERR_INVALID_ARG;

  tmem::Problem p = make_problem(ctx, B, H, T, C, in_dtype);
  const size_t y_bytes = (size_t)p.streams * (size_t)T * (size_t)ctx->d * 4;
  if (!tmem::run_aliasing_ok(p, k, v, q, theta, eta, alpha, W0, S0, y, W_end, S_end))
    return TM_ERR_INVALID_ARG;

  tm_path path = choose_path(ctx, p);
  if (!path_supported(path, p)) return TM_ERR_UNSUPPORTED;
  const size_t need = tmem::kStatusBytes + scratch_bytes(path, p);
  if (workspace_bytes < need) return TM_ERR_OOM;
  if (ranges_overlap(workspace, need, y, y_bytes)) return TM_ERR_INVALID_ARG;

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
  p.status = reinterpret_cast<int *>(workspace);
  const size_t f16b = f16_bytes(path, p);
  char *after_status = static_cast<char *>(workspace) + tmem::kStatusBytes;
  if (f16b) {
    p.k16 = after_status;
    p.q16 = after_status + f16b / 2;
  }
  p.scratch = after_status + f16b;
  p.scratch_bytes = workspace_bytes - tmem::kStatusBytes - f16b;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (clear_status && cudaMemsetAsync(p.status, 0, sizeof(int), s) != cudaSuccess) return TM_ERR_CUDA;
  // the tensor-core kernels read fp16 copies of the keys and queries
  if (f16b && p.T_run > 0 && tmem::tokens_f16_launch(p, s) != cudaSuccess) return TM_ERR_CUDA;
  p.fuse_fb = path == TM_PATH_TC_LAYERED;
  if (path == TM_PATH_TC_LAYERED || path == TM_PATH_TC_PHASED) {
    const int groups = tmem::tcl_group_count(p);
    if (!ensure_side(ctx, groups)) return TM_ERR_CUDA;
    if (groups > 1) {
      for (int i = 0; i < groups - 1; ++i) {
        p.side_streams[i] = ctx->side[i];
        p.ev_join[i] = ctx->ev_join[i];
      }
      p.ev_fork = ctx->ev_fork;
    }
  }
  cudaError_t err = cudaSuccess;
  if (!tensor_path(path)) {
    p.T_run = p.T;                             // the CUDA-core kernel runs the short chunk itself
    err = tmem::simt_launch(p, s);
  } else {
    if (p.T_run > 0)
      err = (path == TM_PATH_TC || path == TM_PATH_TC_GLOBAL) ? tmem::tc_launch(p, s) : run_layered(ctx, path, p, s);
    if (err == cudaSuccess && p.T_run < p.T) {
      // the shorter last chunk, from the state the whole chunks left
      tmem::Problem q = p;
      q.t_begin = p.T_run;
      if (p.T_run > 0) {
        q.W0 = p.W_end;
        q.S0 = p.S_end;
      }
      err = tmem::simt_launch(q, s);
    }
  }
  if (err != cudaSuccess) {
    // a failed launch leaves its error pending in the runtime: consume it
    // here (it is reported as TM_ERR_CUDA) so that later calls do not see it
    cudaGetLastError();
    return TM_ERR_CUDA;
  }
  return TM_OK;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// Segments of tm_run_host, as token counts in order. A caller's
// segment_tokens > 0 gives equal segments (the last one shorter). Otherwise
// the middle segments are about T / 16 (whole chunks) and the first and last
// three ramp up from and down to an eighth of that: the copies of the first
// segment's inputs and of the last one's reads are the only ones no kernel
// runs beside, so keeping those segments short leaves the host link busy for
// almost the whole call, while the middle ones stay long enough that each
// tm_run's fixed cost is small. Every segment but the last is a multiple of C.
std::vector<int> host_segments(int T, int C, int segment_tokens) {
  std::vector<int> lens;
  if (segment_tokens > 0) {
    const int seg = segment_tokens < T ? segment_tokens : T;
    for (int t = 0; t < T; t += seg) lens.push_back(T - t < seg ? T - t : seg);
    return lens;
  }
  const int Tc = T - T % C;                    // tokens in whole chunks
  const int base = ((T + 15) / 16 + C - 1) / C * C;
  auto down = [&](int x) { x = x / C * C; return x < C ? C : x; };
  const int ramp[3] = {down(base / 8), down(base / 4), down(base / 2)};
  const int ends = 2 * (ramp[0] + ramp[1] + ramp[2]);
  if (base >= Tc || Tc - ends < base) {
    // too short for a ramp: equal segments of about T / 16
    for (int t = 0; t < T; t += base) lens.push_back(T - t < base ? T - t : base);
    return lens;
  }
  for (int r : ramp) lens.push_back(r);
  int mid = Tc - ends;
  while (mid > 0) {
    const int n = mid < base ? mid : base;
    lens.push_back(n);
    mid -= n;
  }
  for (int i = 2; i >= 0; --i) lens.push_back(ramp[i]);
  lens.back() += T - Tc;                       // a shorter final chunk goes with the last segment
  return lens;
}

// Longest segment and whether every segment but the last is whole chunks.
int host_segment_max(const std::vector<int> &lens) {
  int m = 0;
  for (int n : lens) m = n > m ? n : m;
  return m;
}
bool host_segments_ok(const std::vector<int> &lens, int C) {
  for (size_t i = 0; i + 1 < lens.size(); ++i)
    if (lens[i] % C != 0) return false;
  return true;
}

// Device workspace of tm_run_host: tm_run's workspace for one segment first
// (so that its status word sits at the start), then the carried state and
// two sets of segment buffers.
struct HostCarve {
  size_t run, run_bytes, W, S, buf[2], k, v, q, th, et, al, y, total;
};

tm_status host_carve(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype dt, const std::vector<int> &lens,
                     HostCarve *c) {
  const int seg = host_segment_max(lens);
  size_t ws = 0;
  for (int t : lens) {
    size_t b = 0;
    const tm_status st = tm_workspace_size(ctx, B, H, t, C, dt, &b);
    if (st != TM_OK) return st;
    if (b > ws) ws = b;
  }
  const size_t S = (size_t)B * H, d = (size_t)ctx->d, el = dt == TM_BF16 ? 2 : 4, ts = (size_t)seg;
  std::memset(c, 0, sizeof *c);
  size_t off = 0;
  c->run = off;
  c->run_bytes = up256(ws);
  off += c->run_bytes;
  c->W = off;
  off += up256(S * ctx->P * 4);
  c->S = off;
  off += up256(S * ctx->P * 4);
  // offsets inside one set of segment buffers
  size_t o = 0;
  c->k = o; o += up256(S * ts * d * el);
  c->v = o; o += up256(S * ts * d * el);
  c->q = o; o += up256(S * ts * d * el);
  c->th = o; o += up256(S * ts * 4);
  c->et = o; o += up256(S * ts * 4);
  c->al = o; o += up256(S * ts * 4);
  c->y = o; o += up256(S * ts * d * 4);
  c->buf[0] = off;
  c->buf[1] = off + o;
  c->total = off + 2 * o;
  return TM_OK;
}

}  // namespace

extern "C" {

tm_status tm_run(tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype, const void *k,
                 const void *v, const void *q, const float *theta, const float *eta,
                 const float *alpha, const float *W0, const float *S0, float *y, float *W_end,
                 float *S_end, void *workspace, size_t workspace_bytes, void *stream) {
  return run_device(ctx, B, H, T, C, in_dtype, k, v, q, theta, eta, alpha, W0, S0, y, W_end, S_end, workspace,
                    workspace_bytes, stream, true);
}

tm_status tm_host_workspace_size(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                                 int segment_tokens, size_t *bytes) {
  if (!bytes || segment_tokens < 0) return TM_ERR_INVALID_ARG;
  tm_status st = check_shape(ctx, B, H, T, C, in_dtype);
  if (st != TM_OK) return st;
  const std::vector<int> lens = host_segments(T, C, segment_tokens);
  if (!host_segments_ok(lens, C)) return TM_ERR_INVALID_ARG;
  HostCarve c;
  st = host_carve(ctx, B, H, T, C, in_dtype, lens, &c);
  if (st != TM_OK) return st;
  *bytes = c.total;
  return TM_OK;
}

tm_status tm_run_host(tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype, const void *k,
                      const void *v, const void *q, const float *theta, const float *eta,
                      const float *alpha, const float *W0, const float *S0, float *y, float *W_end,
                      float *S_end, int segment_tokens, void *workspace, size_t workspace_bytes,
                      void *stream) {
  tm_status st = check_shape(ctx, B, H, T, C, in_dtype);
  if (st != TM_OK) return st;
  if (segment_tokens < 0) return TM_ERR_INVALID_ARG;
  const void *ptrs[] = {k, v, q, theta, eta, alpha, W0, S0, y, W_end, S_end, workspace};
  for (const void *x : ptrs)
    if (!x) return TM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TM_ERR_INVALID_ARG;
  const tmem::Problem p = make_problem(ctx, B, H, T, C, in_dtype);
  if (!tmem::run_aliasing_ok(p, k, v, q, theta, eta, alpha, W0, S0, y, W_end, S_end)) return TM_ERR_INVALID_ARG;
  const std::vector<int> lens = host_segments(T, C, segment_tokens);
  if (!host_segments_ok(lens, C)) return TM_ERR_INVALID_ARG;
  HostCarve c;
  st = host_carve(ctx, B, H, T, C, in_dtype, lens, &c);
  if (st != TM_OK) return st;
  if (workspace_bytes < c.total) return TM_ERR_OOM;
  {
    // every segment's path must be one tm_run supports
    tm_path path;
    for (size_t i = 0; i < lens.size(); ++i)
      if ((i == 0 || lens[i] != lens[i - 1]) && tm_query_path(ctx, B, H, lens[i], C, in_dtype, &path) != TM_OK)
        return TM_ERR_UNSUPPORTED;
  }
  if (!ensure_host(ctx)) return TM_ERR_CUDA;

  unsigned char *ws = static_cast<unsigned char *>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t S = (size_t)p.streams, d = (size_t)ctx->d, el = in_dtype == TM_BF16 ? 2 : 4;
  const size_t st_bytes = S * ctx->P * 4;
  float *dW = reinterpret_cast<float *>(ws + c.W), *dS = reinterpret_cast<float *>(ws + c.S);
  const int nseg = (int)lens.size();
  std::vector<size_t> start((size_t)nseg);
  for (int i = 0, t = 0; i < nseg; t += lens[(size_t)i], ++i) start[(size_t)i] = (size_t)t;
  auto seg_len = [&](int i) { return lens[(size_t)i]; };
  // One strided copy per tensor and segment: the segment's rows of every
  // stream, [S rows] x [n tokens x width] bytes.
  auto copy_in = [&](int i) -> cudaError_t {
    unsigned char *b = ws + c.buf[i & 1];
    const size_t t0 = start[(size_t)i], n = (size_t)seg_len(i);
    const void *src[6] = {k, v, q, theta, eta, alpha};
    const size_t off[6] = {c.k, c.v, c.q, c.th, c.et, c.al};
    const size_t w[6] = {d * el, d * el, d * el, 4, 4, 4};
    for (int j = 0; j < 6; ++j) {
      const cudaError_t e = cudaMemcpy2DAsync(b + off[j], n * w[j], static_cast<const unsigned char *>(src[j]) + t0 * w[j],
                                              (size_t)T * w[j], n * w[j], S, cudaMemcpyHostToDevice, ctx->h2d);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  };
  cudaError_t e = cudaEventRecord(ctx->h_start, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ctx->h2d, ctx->h_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ctx->d2h, ctx->h_start, 0);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dW, W0, st_bytes, cudaMemcpyHostToDevice, ctx->h2d);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dS, S0, st_bytes, cudaMemcpyHostToDevice, ctx->h2d);
  if (e == cudaSuccess) e = copy_in(0);
  if (e == cudaSuccess) e = cudaEventRecord(ctx->in_ready[0], ctx->h2d);
  st = e == cudaSuccess ? TM_OK : TM_ERR_CUDA;
  for (int i = 0; i < nseg && st == TM_OK; ++i) {
    const int b = i & 1, n = seg_len(i);
    unsigned char *bb = ws + c.buf[b];
    if (i + 1 < nseg) {
      // the next segment's inputs land while this one runs (its buffer was
      // last read by segment i - 1)
      e = cudaStreamWaitEvent(ctx->h2d, ctx->in_free[(i + 1) & 1], 0);
      if (e == cudaSuccess) e = copy_in(i + 1);
      if (e == cudaSuccess) e = cudaEventRecord(ctx->in_ready[(i + 1) & 1], ctx->h2d);
    }
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ctx->in_ready[b], 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ctx->y_free[b], 0);   // y buffer read out (segment i - 2)
    if (e != cudaSuccess) { st = TM_ERR_CUDA; break; }
    float *yb = reinterpret_cast<float *>(bb + c.y);
    st = run_device(ctx, B, H, n, C, in_dtype, bb + c.k, bb + c.v, bb + c.q, reinterpret_cast<float *>(bb + c.th),
                    reinterpret_cast<float *>(bb + c.et), reinterpret_cast<float *>(bb + c.al), dW, dS, yb, dW, dS,
                    ws + c.run, c.run_bytes, s, i == 0);
    if (st != TM_OK) break;
    e = cudaEventRecord(ctx->in_free[b], s);
    if (e == cudaSuccess) e = cudaEventRecord(ctx->y_ready[b], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ctx->d2h, ctx->y_ready[b], 0);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(y + start[(size_t)i] * d, (size_t)T * d * 4, yb, (size_t)n * d * 4, (size_t)n * d * 4, S,
                            cudaMemcpyDeviceToHost, ctx->d2h);
    if (e == cudaSuccess) e = cudaEventRecord(ctx->y_free[b], ctx->d2h);
    if (e != cudaSuccess) st = TM_ERR_CUDA;
  }
  if (st == TM_OK) {
    e = cudaEventRecord(ctx->h_state, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ctx->d2h, ctx->h_state, 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(W_end, dW, st_bytes, cudaMemcpyDeviceToHost, ctx->d2h);
    if (e == cudaSuccess) e = cudaMemcpyAsync(S_end, dS, st_bytes, cudaMemcpyDeviceToHost, ctx->d2h);
    if (e != cudaSuccess) st = TM_ERR_CUDA;
  }
  // join both copy streams into the caller's stream, also after an error
  if (cudaEventRecord(ctx->h_done, ctx->d2h) == cudaSuccess) cudaStreamWaitEvent(s, ctx->h_done, 0);
  if (cudaEventRecord(ctx->h_state, ctx->h2d) == cudaSuccess) cudaStreamWaitEvent(s, ctx->h_state, 0);
  return st;
}

tm_status tm_sync(tm_ctx *ctx, void *workspace, void *stream) {
  if (!ctx || !workspace) return TM_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int code = 0;
  if (cudaMemcpyAsync(&code, workspace, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return TM_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return TM_ERR_CUDA;
  if (code == tmem::kDevOk) return TM_OK;
  const int zero = 0;
  if (cudaMemcpyAsync(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return TM_ERR_CUDA;
  return code == tmem::kDevTimeout ? TM_ERR_TIMEOUT : TM_ERR_DEVICE;
}

tm_status tm_backward_workspace_size(const tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype,
                                     size_t *bytes) {
  if (!bytes) return TM_ERR_INVALID_ARG;
  tm_status st = check_shape(ctx, B, H, T, C, in_dtype);
  if (st != TM_OK) return st;
  const tmem::Problem p = make_problem(ctx, B, H, T, C, in_dtype);
  if (!tmem::backward_supported(p)) return TM_ERR_UNSUPPORTED;
  *bytes = tmem::kStatusBytes + tmem::backward_scratch_bytes(p);
  return TM_OK;
}

tm_status tm_backward(tm_ctx *ctx, int B, int H, int T, int C, tm_dtype in_dtype, const void *k, const void *v,
                      const void *q, const float *theta, const float *eta, const float *alpha, const float *W0,
                      const float *S0, const float *dy, const float *dW_end, const float *dS_end, float *dk,
                      float *dv, float *dq, float *dtheta, float *deta, float *dalpha, float *dW0, float *dS0,
                      void *workspace, size_t workspace_bytes, void *stream) {
  tm_status st = check_shape(ctx, B, H, T, C, in_dtype);
  if (st != TM_OK) return st;
  const void *ptrs[] = {k, v, q, theta, eta, alpha, W0, S0, dy, dW_end, dS_end, dk, dv, dq, dtheta, deta,
                        dalpha, dW0, dS0, workspace};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return TM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return TM_ERR_INVALID_ARG;
  tmem::Problem p = make_problem(ctx, B, H, T, C, in_dtype);
  if (!tmem::backward_supported(p)) return TM_ERR_UNSUPPORTED;
  const size_t need = tmem::kStatusBytes + tmem::backward_scratch_bytes(p);
  if (workspace_bytes < need) return TM_ERR_OOM;
  const size_t S = (size_t)p.streams, el = in_dtype == TM_BF16 ? 2 : 4, d = (size_t)p.dims[0];
  const size_t tokb = S * p.T * d * el, tokf = S * p.T * d * 4, gate = S * p.T * 4, state = S * p.P * 4;
  const void *ins[] = {k, v, q, theta, eta, alpha, W0, S0, dy, dW_end, dS_end, workspace};
  const size_t insz[] = {tokb, tokb, tokb, gate, gate, gate, state, state, tokf, state, state, need};
  const void *outs[] = {dk, dv, dq, dtheta, deta, dalpha, dW0, dS0};
  const size_t outsz[] = {tokf, tokf, tokf, gate, gate, gate, state, state};
  for (int i = 0; i < 8; ++i) {
    for (int j = 0; j < 12; ++j)
      if (ranges_overlap(outs[i], outsz[i], ins[j], insz[j])) return TM_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j)
      if (ranges_overlap(outs[i], outsz[i], outs[j], outsz[j])) return TM_ERR_INVALID_ARG;
  }
  p.k = k;
  p.v = v;
  p.q = q;
  p.theta = theta;
  p.eta = eta;
  p.alpha = alpha;
  p.W0 = W0;
  p.S0 = S0;
  p.scratch = static_cast<char *>(workspace) + tmem::kStatusBytes;
  p.scratch_bytes = workspace_bytes - tmem::kStatusBytes;
  // bf16 inputs on a tensor-core path: the reverse pass's products on tcgen05
  // (TF32 operands); fp32 inputs or TM_PATH_SIMT: fp32 FFMA throughout
  p.bw_tc = in_dtype == TM_BF16 && ctx->path != TM_PATH_SIMT;
  p.status = static_cast<int *>(workspace);
  if (cudaMemsetAsync(workspace, 0, sizeof(int), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return TM_ERR_CUDA;
  const cudaError_t e = tmem::backward_launch(p, dy, dW_end, dS_end, dk, dv, dq, dtheta, deta, dalpha, dW0, dS0,
                                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TM_OK : TM_ERR_CUDA;
}

tm_status tm_decode_step(tm_ctx *ctx, int B, int H, tm_dtype in_dtype, const void *k, const void *v,
                         const void *q, const float *theta, const float *eta, const float *alpha, float *W,
                         float *S, float *y, void *stream) {
  tm_status st = check_shape(ctx, B, H, 1, 1, in_dtype);
  if (st != TM_OK) return st;
  const void *ptrs[] = {k, v, q, theta, eta, alpha, W, S, y};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return TM_ERR_INVALID_ARG;
  const tmem::Problem p = make_problem(ctx, B, H, 1, 1, in_dtype);
  const size_t el = in_dtype == TM_BF16 ? 2 : 4;
  const size_t tok = (size_t)p.streams * p.dims[0] * el, gate = (size_t)p.streams * 4;
  const size_t state = (size_t)p.streams * p.P * 4, yb = (size_t)p.streams * p.dims[0] * 4;
  const void *ins[] = {k, v, q, theta, eta, alpha, W, S};
  const size_t insz[] = {tok, tok, tok, gate, gate, gate, state, state};
  for (int i = 0; i < 8; ++i)
    if (ranges_overlap(y, yb, ins[i], insz[i])) return TM_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (ranges_overlap(W, state, ins[i], insz[i]) || ranges_overlap(S, state, ins[i], insz[i]))
      return TM_ERR_INVALID_ARG;
  if (ranges_overlap(W, state, S, state)) return TM_ERR_INVALID_ARG;
  if (!tmem::decode_supported(p)) return TM_ERR_UNSUPPORTED;
  const cudaError_t e = tmem::decode_launch(p, k, v, q, theta, eta, alpha, W, S, y,
                                            reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TM_OK : TM_ERR_CUDA;
}

tm_status tm_prologue(int B, int H, int T, int d, int width, tm_dtype in_dtype, const void *k_in,
                      const void *v_in, const void *q_in, const float *filt_k, const float *filt_v,
                      const float *filt_q, const void *hist_k, const void *hist_v, const void *hist_q,
                      void *k_out, void *v_out, void *q_out, void *stream) {
  if (B < 1 || H < 1 || T < 1 || d < 1 || d > 768 || width < 1 || width > 8) return TM_ERR_INVALID_ARG;
  if (!tmem::prologue_supported_d(d)) return TM_ERR_UNSUPPORTED;
  if (in_dtype != TM_F32 && in_dtype != TM_BF16) return TM_ERR_INVALID_ARG;
  if ((long long)B * H > (1LL << 16) - 1 || T > (1 << 30)) return TM_ERR_INVALID_ARG;
  const void *in[3] = {k_in, v_in, q_in};
  const float *filt[3] = {filt_k, filt_v, filt_q};
  const void *hist[3] = {hist_k, hist_v, hist_q};
  void *out[3] = {k_out, v_out, q_out};
  const size_t el = in_dtype == TM_BF16 ? 2 : 4;
  const size_t tens = (size_t)B * H * T * d * el;
  for (int i = 0; i < 3; ++i) {
    if (!in[i] || !filt[i] || !out[i]) return TM_ERR_INVALID_ARG;
    const void *ps[] = {in[i], filt[i], out[i], hist[i]};
    for (const void *p : ps)
      if (p && (reinterpret_cast<uintptr_t>(p) & 15u)) return TM_ERR_INVALID_ARG;
    for (int j = 0; j < 3; ++j)
      if (ranges_overlap(out[i], tens, in[j], tens)) return TM_ERR_INVALID_ARG;
    for (int j = 0; j < i; ++j)
      if (ranges_overlap(out[i], tens, out[j], tens)) return TM_ERR_INVALID_ARG;
  }
  cudaError_t e = tmem::prologue_launch(B * H, H, T, d, width, in_dtype == TM_BF16, in, filt, hist, out,
                                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TM_OK : TM_ERR_CUDA;
}

tm_status tm_set_debug(int inject_timeout, unsigned long long wait_limit_ns) {
  tmem::tc_set_debug(inject_timeout, wait_limit_ns);
  tmem::tcl_set_debug(inject_timeout, wait_limit_ns);
  return TM_OK;
}

const char *tm_status_string(tm_status status) {
  switch (status) {
    case TM_OK: return "ok";
    case TM_ERR_INVALID_ARG: return "invalid argument";
    case TM_ERR_UNSUPPORTED: return "unsupported shape, dtype or path";
    case TM_ERR_CUDA: return "CUDA runtime error";
    case TM_ERR_OOM: return "out of memory or workspace too small";
    case TM_ERR_TIMEOUT: return "a bounded device-side wait expired";
    case TM_ERR_DEVICE: return "device-side consistency check failed";
  }
  return "unknown status";
}

int tm_version(void) { return 100; }

}  // extern "C"
