/*
 * Titans neural long-term memory: float64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY. This is the checker for the CUDA library, not part
 * of it. Only the tests, the smoke check and the benchmark's CPU-baseline leg
 * may load it. It shares no code, header or constant with the CUDA path.
 *
 * What it computes: the literal per-token recurrence of the memory, in float64,
 * one stream (batch entry, head) at a time.
 *
 *   memory M: an MLP of depth L without biases. z_l = W_l x_{l-1} and
 *   x_l = silu(z_l) between layers; the last layer has no activation.
 *   A depth-1 memory is the linear map W.
 *       ("Titans, explained", glossary entry "M — the memory"; "titans-pytorch"
 *        review: the "simple 1-4 layer MLP" memory)
 *   surprise:   u_t = grad_W || M(k_t) - v_t ||^2, a plain sum of squares with
 *               no 1/2 and no mean, taken at the chunk-start weights.
 *       ("Titans, explained", step 2 "Measure surprise"; step 6 "Make it
 *        trainable in parallel"; the "At the extremes" paragraph gives the
 *        linear case 2 (M k - v) k^T)
 *   momentum:   S_t = eta_t S_{t-1} - theta_t u_t
 *       ("Titans, explained", step 3 "Accumulate surprise with momentum")
 *   forget+write: W_t = (1 - alpha_t) W_{t-1} + S_t, using the new S_t
 *       ("Titans, explained", step 4 "Forget, then write")
 *   read:       y_t = M(q_t) through the weights at the start of the chunk,
 *               with no write ("Titans, explained", step 5 "Read without
 *               writing")
 *   chunking:   the chunk of token t starts at t - (t mod C) with 0-based t;
 *               every gradient inside the chunk is taken at the weights as they
 *               stood after the last token of the previous chunk ("Attack of
 *               the Titans", section "Parallel training": t' = t - (t mod b)).
 *
 * A partial last chunk (T not a multiple of C) is handled as a shorter chunk.
 * Every u_t, S_t and W_t is materialised as a full [P] vector, as written.
 *
 * Parameter layout: layer l (1-based) is a row-major [n_l x n_{l-1}] block, the
 * blocks laid end to end in layer order, P = sum_l n_l n_{l-1}.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F64 = 0, OR_F32 = 1, OR_BF16 = 2 };

#define OR_MAX_L 8

static double load_elem(const void *p, int dtype, size_t i) {
  if (dtype == OR_F64) return ((const double *)p)[i];
  if (dtype == OR_F32) return (double)((const float *)p)[i];
  uint32_t bits = ((uint32_t)((const uint16_t *)p)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }
static double silu(double z) { return z * sigmoid(z); }
/* d/dz [z s(z)] = s(z) + z s(z) (1 - s(z)) */
static double silu_prime(double z) {
  double s = sigmoid(z);
  return s * (1.0 + z * (1.0 - s));
}

typedef struct {
  int L;
  int dims[OR_MAX_L + 1];
  size_t off[OR_MAX_L + 1]; /* off[l-1] = start of layer l; off[L] = P */
  size_t P;
  int maxw;
} net_t;

/* Forward one vector through the weights Wf. xs[l] receives x_l (x_0 = input),
 * zs[l] receives z_l for l = 1..L. Returns nothing; x_L is the output. */
static void forward(const net_t *n, const double *Wf, double **xs, double **zs) {
  for (int l = 1; l <= n->L; ++l) {
    const double *Wl = Wf + n->off[l - 1];
    int rows = n->dims[l], cols = n->dims[l - 1];
    for (int r = 0; r < rows; ++r) {
      double acc = 0.0;
      const double *wr = Wl + (size_t)r * cols;
      for (int c = 0; c < cols; ++c) acc += wr[c] * xs[l - 1][c];
      zs[l][r] = acc;
      xs[l][r] = (l < n->L) ? silu(acc) : acc;
    }
  }
}

/* u = grad over all layers of || M(k) - v ||^2 at Wf, written into u[P].
 * xs/zs must hold the forward pass of k. g and gn are scratch of maxw. */
static void surprise(const net_t *n, const double *Wf, double **xs, double **zs,
                     const double *v, double *u, double *g, double *gn) {
  int L = n->L;
  int dL = n->dims[L];
  for (int i = 0; i < dL; ++i) g[i] = 2.0 * (xs[L][i] - v[i]);
  for (int l = L; l >= 1; --l) {
    int rows = n->dims[l], cols = n->dims[l - 1];
    double *ul = u + n->off[l - 1];
    for (int r = 0; r < rows; ++r)
      for (int c = 0; c < cols; ++c) ul[(size_t)r * cols + c] = g[r] * xs[l - 1][c];
    if (l > 1) {
      const double *Wl = Wf + n->off[l - 1];
      for (int c = 0; c < cols; ++c) {
        double acc = 0.0;
        for (int r = 0; r < rows; ++r) acc += Wl[(size_t)r * cols + c] * g[r];
        gn[c] = acc * silu_prime(zs[l - 1][c]);
      }
      memcpy(g, gn, sizeof(double) * cols);
    }
  }
}

typedef struct {
  const net_t *net;
  int n_streams, T, C, d_in, d_out;
  int tok_dtype, gate_dtype, state_dtype;
  const void *k, *v, *q, *theta, *eta, *alpha, *W0, *S0;
  double *y, *W_end, *S_end;
  double *u_trace, *S_trace, *W_trace; /* optional [n, T, P] */
  int next;
  pthread_mutex_t lock;
  int status;
} job_t;

static int run_stream(job_t *jb, int s) {
  const net_t *n = jb->net;
  size_t P = n->P;
  int T = jb->T, C = jb->C, d = jb->d_in, dout = jb->d_out, L = n->L;
  double *W = malloc(sizeof(double) * P), *S = malloc(sizeof(double) * P);
  double *Wf = malloc(sizeof(double) * P), *u = malloc(sizeof(double) * P);
  double *bufx = malloc(sizeof(double) * (size_t)(L + 1) * n->maxw);
  double *bufz = malloc(sizeof(double) * (size_t)(L + 1) * n->maxw);
  double *g = malloc(sizeof(double) * n->maxw), *gn = malloc(sizeof(double) * n->maxw);
  double *vt = malloc(sizeof(double) * dout);
  if (!W || !S || !Wf || !u || !bufx || !bufz || !g || !gn || !vt) {
    free(W); free(S); free(Wf); free(u); free(bufx); free(bufz); free(g); free(gn); free(vt);
    return 1;
  }
  double *xs[OR_MAX_L + 1], *zs[OR_MAX_L + 1];
  for (int l = 0; l <= L; ++l) {
    xs[l] = bufx + (size_t)l * n->maxw;
    zs[l] = bufz + (size_t)l * n->maxw;
  }
  for (size_t i = 0; i < P; ++i) {
    W[i] = load_elem(jb->W0, jb->state_dtype, (size_t)s * P + i);
    S[i] = load_elem(jb->S0, jb->state_dtype, (size_t)s * P + i);
  }
  for (int t = 0; t < T; ++t) {
    if (t % C == 0) memcpy(Wf, W, sizeof(double) * P); /* chunk-start weights */
    size_t tok = ((size_t)s * T + t);
    /* surprise of token t at the chunk-start weights */
    for (int i = 0; i < d; ++i) xs[0][i] = load_elem(jb->k, jb->tok_dtype, tok * d + i);
    for (int i = 0; i < dout; ++i) vt[i] = load_elem(jb->v, jb->tok_dtype, tok * dout + i);
    forward(n, Wf, xs, zs);
    surprise(n, Wf, xs, zs, vt, u, g, gn);
    double th = load_elem(jb->theta, jb->gate_dtype, tok);
    double et = load_elem(jb->eta, jb->gate_dtype, tok);
    double al = load_elem(jb->alpha, jb->gate_dtype, tok);
    /* momentum, then forget-and-write with the new momentum */
    for (size_t i = 0; i < P; ++i) S[i] = et * S[i] - th * u[i];
    for (size_t i = 0; i < P; ++i) W[i] = (1.0 - al) * W[i] + S[i];
    if (jb->u_trace) memcpy(jb->u_trace + tok * P, u, sizeof(double) * P);
    if (jb->S_trace) memcpy(jb->S_trace + tok * P, S, sizeof(double) * P);
    if (jb->W_trace) memcpy(jb->W_trace + tok * P, W, sizeof(double) * P);
    /* read through the chunk-start weights */
    for (int i = 0; i < d; ++i) xs[0][i] = load_elem(jb->q, jb->tok_dtype, tok * d + i);
    forward(n, Wf, xs, zs);
    memcpy(jb->y + tok * dout, xs[L], sizeof(double) * dout);
  }
  memcpy(jb->W_end + (size_t)s * P, W, sizeof(double) * P);
  memcpy(jb->S_end + (size_t)s * P, S, sizeof(double) * P);
  free(W); free(S); free(Wf); free(u); free(bufx); free(bufz); free(g); free(gn); free(vt);
  return 0;
}

static void *worker(void *arg) {
  job_t *jb = (job_t *)arg;
  for (;;) {
    pthread_mutex_lock(&jb->lock);
    int s = jb->next++;
    pthread_mutex_unlock(&jb->lock);
    if (s >= jb->n_streams) break;
    if (run_stream(jb, s)) {
      pthread_mutex_lock(&jb->lock);
      jb->status = 3;
      pthread_mutex_unlock(&jb->lock);
    }
  }
  return NULL;
}

/*
 * Run the recurrence for n_streams independent streams.
 *   dims[0..L]:  n_0 = input width (d of k and q), n_L = output width (d of v, y)
 *   k, q:        [n_streams, T, n_0] in tok_dtype;  v: [n_streams, T, n_L]
 *   theta, eta, alpha: [n_streams, T] in gate_dtype
 *   W0, S0:      [n_streams, P] in state_dtype
 *   y:           [n_streams, T, n_L] float64 out
 *   W_end, S_end:[n_streams, P] float64 out
 *   u_trace, S_trace, W_trace: optional [n_streams, T, P] float64 (NULL = off):
 *                u_t, S_t and W_t after token t.
 * dtype codes: 0 float64, 1 float32, 2 bfloat16 bits (uint16).
 * Returns 0 on success, 1 bad arguments, 3 out of host memory.
 */
int titans_oracle_run(int L, const int *dims, int n_streams, int T, int C,
                      int tok_dtype, const void *k, const void *v, const void *q,
                      int gate_dtype, const void *theta, const void *eta, const void *alpha,
                      int state_dtype, const void *W0, const void *S0,
                      double *y, double *W_end, double *S_end,
                      double *u_trace, double *S_trace, double *W_trace, int n_threads) {
  if (L < 1 || L > OR_MAX_L || !dims || n_streams < 0 || T < 0 || C < 1) return 1;
  net_t net;
  net.L = L;
  net.P = 0;
  net.maxw = 0;
  for (int l = 0; l <= L; ++l) {
    if (dims[l] < 1) return 1;
    net.dims[l] = dims[l];
    if (dims[l] > net.maxw) net.maxw = dims[l];
  }
  for (int l = 1; l <= L; ++l) {
    net.off[l - 1] = net.P;
    net.P += (size_t)dims[l] * dims[l - 1];
  }
  net.off[L] = net.P;
  if (n_streams == 0) return 0;
  job_t jb;
  memset(&jb, 0, sizeof jb);
  jb.net = &net;
  jb.n_streams = n_streams;
  jb.T = T;
  jb.C = C;
  jb.d_in = dims[0];
  jb.d_out = dims[L];
  jb.tok_dtype = tok_dtype;
  jb.gate_dtype = gate_dtype;
  jb.state_dtype = state_dtype;
  jb.k = k; jb.v = v; jb.q = q;
  jb.theta = theta; jb.eta = eta; jb.alpha = alpha;
  jb.W0 = W0; jb.S0 = S0;
  jb.y = y; jb.W_end = W_end; jb.S_end = S_end;
  jb.u_trace = u_trace; jb.S_trace = S_trace; jb.W_trace = W_trace;
  pthread_mutex_init(&jb.lock, NULL);
  if (n_threads < 1) n_threads = 1;
  if (n_threads > n_streams) n_threads = n_streams;
  pthread_t *th = malloc(sizeof(pthread_t) * n_threads);
  if (!th) return 3;
  int started = 0;
  for (int i = 0; i < n_threads - 1; ++i)
    if (pthread_create(&th[started], NULL, worker, &jb) == 0) ++started;
  /* the calling thread works too */
  worker(&jb);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
  pthread_mutex_destroy(&jb.lock);
  return jb.status;
}

/* Surprise of a single token at given weights: u = grad_W ||M(k) - v||^2,
 * float64 everywhere. Used by the tests to check the chunk closed form.
 * Returns 0, or 1 for bad arguments, 3 out of memory. */
int titans_oracle_surprise(int L, const int *dims, const double *W, const double *k,
                           const double *v, double *u) {
  if (L < 1 || L > OR_MAX_L || !dims) return 1;
  net_t net;
  net.L = L;
  net.P = 0;
  net.maxw = 0;
  for (int l = 0; l <= L; ++l) {
    net.dims[l] = dims[l];
    if (dims[l] > net.maxw) net.maxw = dims[l];
  }
  for (int l = 1; l <= L; ++l) {
    net.off[l - 1] = net.P;
    net.P += (size_t)dims[l] * dims[l - 1];
  }
  double *bufx = malloc(sizeof(double) * (size_t)(L + 1) * net.maxw);
  double *bufz = malloc(sizeof(double) * (size_t)(L + 1) * net.maxw);
  double *g = malloc(sizeof(double) * net.maxw), *gn = malloc(sizeof(double) * net.maxw);
  if (!bufx || !bufz || !g || !gn) {
    free(bufx); free(bufz); free(g); free(gn);
    return 3;
  }
  double *xs[OR_MAX_L + 1], *zs[OR_MAX_L + 1];
  for (int l = 0; l <= L; ++l) {
    xs[l] = bufx + (size_t)l * net.maxw;
    zs[l] = bufz + (size_t)l * net.maxw;
  }
  memcpy(xs[0], k, sizeof(double) * dims[0]);
  forward(&net, W, xs, zs);
  surprise(&net, W, xs, zs, v, u, g, gn);
  free(bufx); free(bufz); free(g); free(gn);
  return 0;
}
