/*
 * ss_oracle.c -- fp64 CPU oracle for the S6 selective-scan forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library; the two meet only through the seeded inputs handed to both.
 *
 * What it computes is the plain serial recurrence of the selective SSM,
 * widened exactly from the stored input dtype to double:
 *
 *   for every (b, d):  h[n] = h0[b,d,n]  (0 when no initial state is given)
 *     for t = 0 .. L-1:
 *       Delta  = softplus(delta[b,d,t] + delta_bias[d])   (or without softplus)
 *       h[n]   = exp(Delta * A[d,n]) * h[n] + Delta * B[b,n,t] * u[b,d,t]
 *       y      = sum_n C[b,n,t] * h[n] + D[d] * u[b,d,t]
 *       y      = y * z * sigmoid(z)                       (when z is given)
 *     last_state[b,d,n] = h[n]
 *
 * Passages followed (page title, section):
 *  - "从Transformer的痛点说起 ... Mamba" (pwwt.cn), sec. 2.2: ZOH gives
 *    A_bar = exp(Delta A); implementations simplify B_bar to Delta * B;
 *    recurrence h_t = A_bar h_{t-1} + B_bar x_t, y_t = C h_t.
 *  - same page, sec. 3.1: B_t, C_t, Delta_t are functions of x_t, with
 *    Delta_t = softplus(Linear(x_t)); A stays input independent.
 *  - same page, sec. 4.2 (pure-PyTorch SelectiveSSM): the bias of the Delta
 *    projection sits inside the softplus; A = -exp(A_log) is diagonal [D,N];
 *    the state starts at zero; the readout uses the state after the update
 *    that includes token t; the skip term x*D is added before the gate
 *    y * SiLU(z).
 *  - "Mamba 选择性机制" (discosf.com), sec. 1.1 and 3.1: the discrete
 *    recurrence and the associative operator it folds with.
 *  - "Mamba 深度解读报告" (zako-mio.github.io), sec. 2.4: the state is never
 *    materialised over (B,L,D,N); only y (B,L,D) is the output.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - softplus(x) = log(1 + e^x), evaluated as log1p(exp(x)) for x <= 30 and
 *    x + log1p(exp(-x)) above, both exact to double rounding.
 *  - softplus_flag == 0 means Delta = delta + delta_bias.
 *  - SiLU(z) = z / (1 + exp(-z)).
 *  - a null D, delta_bias or z means zero skip, zero bias and no gate.
 *  - with a short convolution (same page, sec. 3.3 block diagram and the
 *    sec. 4.2 code: a depthwise Conv1d of width W, padding W-1, cut to the
 *    first L outputs, then SiLU), the scan's input is
 *      u[b,d,t] = SiLU(conv_bias[d] + sum_{k<W} conv_w[d,k] x[b,d,t-(W-1)+k]),
 *    with x = 0 before t = 0 (Conv1d is a cross-correlation, so tap W-1
 *    meets the current token).
 *  - exact zero-order hold (zoh != 0; same page, sec. 2.2, the form before its
 *    simplification): B_bar = (Delta A)^-1 (exp(Delta A) - 1) Delta B, which
 *    for diagonal A is expm1(Delta A[d,n]) / A[d,n] * B[b,n,t], and Delta B
 *    where A[d,n] = 0 (its limit).  expm1 keeps it exact for small Delta A.
 *  - an initial state h0 replaces the zero state of the pure-PyTorch module;
 *    the pages keep h between calls for recurrent (one token at a time)
 *    inference ("从Transformer的痛点说起 ... Mamba", sec. 5.1 table and
 *    sec. 6.3, fourth note), and one such step is this recurrence with L = 1
 *    started from the carried state.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Stored input dtypes: 0 = IEEE binary32, 1 = bfloat16 (upper half of a
 * binary32).  Both widen to double without rounding. */
static double widen(const void* p, int dtype, int64_t i) {
  if (dtype == 1) {
    uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float*)p)[i];
}

static double softplus64(double x) {
  if (x <= 30.0) return log1p(exp(x));
  return x + log1p(exp(-x));
}

static double silu64(double z) { return z / (1.0 + exp(-z)); }

typedef struct {
  const void *u, *delta, *B, *C, *z;
  const float *A, *D, *delta_bias;
  int softplus_flag, dtype;
  int64_t batch, dim, seqlen;
  int dstate;
  const int64_t* channels; /* optional list of flat channel ids b*dim+d */
  int64_t n_channels;
  double* y;          /* [n_channels, seqlen] */
  double* last_state; /* [n_channels, dstate] or NULL */
  const double* h0;   /* [batch, dim, dstate] initial state or NULL (zero) */
  const float* conv_w; /* [dim, conv_width] or NULL: u is the scan input itself */
  const float* conv_b; /* [dim] or NULL */
  int conv_width;
  int zoh;            /* 1: exact zero-order hold for B_bar */
  int64_t next;       /* work counter (guarded by mu) */
  pthread_mutex_t mu;
} job_t;

/* One (b, d) channel: the serial recurrence, nothing reordered. */
/* The scan's input at step t of one channel: u itself, or the SiLU of the
 * causal depthwise convolution of x (stored in J->u) at t. */
static double scan_input(const job_t* J, int64_t row, int64_t d, int64_t t) {
  if (!J->conv_w) return widen(J->u, J->dtype, row + t);
  const int W = J->conv_width;
  double acc = J->conv_b ? (double)J->conv_b[d] : 0.0;
  for (int k = 0; k < W; ++k) {
    const int64_t s = t - (W - 1) + k;
    if (s >= 0) acc += (double)J->conv_w[d * W + k] * widen(J->u, J->dtype, row + s);
  }
  return silu64(acc);
}

static void run_channel(const job_t* J, int64_t slot, double* h) {
  const int64_t flat = J->channels ? J->channels[slot] : slot;
  const int64_t b = flat / J->dim, d = flat % J->dim;
  const int64_t L = J->seqlen;
  const int N = J->dstate;
  const int64_t row = (b * J->dim + d) * L;    /* u, delta, z: [B,D,L] */
  const int64_t bc_base = b * (int64_t)N * L;  /* B, C: [B,N,L] */
  const double bias = J->delta_bias ? (double)J->delta_bias[d] : 0.0;
  const double Dd = J->D ? (double)J->D[d] : 0.0;
  double* yrow = J->y + slot * L;

  for (int n = 0; n < N; ++n) h[n] = J->h0 ? J->h0[flat * N + n] : 0.0;
  for (int64_t t = 0; t < L; ++t) {
    const double x = widen(J->delta, J->dtype, row + t) + bias;
    const double dt = J->softplus_flag ? softplus64(x) : x;
    const double ut = scan_input(J, row, d, t);
    double s = 0.0;
    for (int n = 0; n < N; ++n) {
      const double a_bar = exp(dt * (double)J->A[d * N + n]);
      const double b_t = widen(J->B, J->dtype, bc_base + (int64_t)n * L + t);
      const double c_t = widen(J->C, J->dtype, bc_base + (int64_t)n * L + t);
      const double an = (double)J->A[d * N + n];
      const double b_bar = (J->zoh && an != 0.0) ? expm1(dt * an) / an * b_t : dt * b_t;
      h[n] = a_bar * h[n] + b_bar * ut;
      s += c_t * h[n];
    }
    s += Dd * ut;
    if (J->z) s *= silu64(widen(J->z, J->dtype, row + t));
    yrow[t] = s;
  }
  if (J->last_state)
    for (int n = 0; n < N; ++n) J->last_state[slot * N + n] = h[n];
}

static void* worker(void* arg) {
  job_t* J = (job_t*)arg;
  double* h = (double*)malloc(sizeof(double) * (size_t)J->dstate);
  if (!h) return NULL;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    const int64_t slot = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (slot >= J->n_channels) break;
    run_channel(J, slot, h);
  }
  free(h);
  return NULL;
}

/*
 * oracle_scan_fwd: returns 0 on success, -1 on a bad argument.
 *
 * u, delta, z : [batch, dim, seqlen] in `dtype` (0 f32, 1 bf16), L fastest;
 *               with conv_w, u holds the convolution's input x
 * B, C        : [batch, dstate, seqlen] in `dtype`
 * A           : [dim, dstate] f32;  D, delta_bias: [dim] f32 (nullable)
 * channels    : NULL for every channel (b*dim+d order), else n_channels flat
 *               channel ids; y and last_state then hold only those rows.
 * y           : [n_channels, seqlen] double
 * last_state  : [n_channels, dstate] double (nullable)
 * h0          : [batch, dim, dstate] double initial state, indexed by the
 *               full flat channel id even when `channels` is given (nullable:
 *               the state starts at zero)
 * conv_w      : [dim, conv_width] f32 taps of the short convolution, or NULL
 * conv_b      : [dim] f32 convolution bias (nullable)
 * conv_width  : 1..64 when conv_w is given
 * zoh         : nonzero for the exact zero-order-hold B_bar
 * nthreads    : worker threads (>= 1)
 */
int oracle_scan_fwd(const void* u, const void* delta, const float* A,
                    const void* B, const void* C, const float* D,
                    const void* z, const float* delta_bias, int softplus_flag,
                    int dtype, int64_t batch, int64_t dim, int64_t seqlen,
                    int dstate, const int64_t* channels, int64_t n_channels,
                    double* y, double* last_state, const double* h0,
                    const float* conv_w, const float* conv_b, int conv_width,
                    int zoh, int nthreads) {
  if (!u || !delta || !A || !B || !C || !y) return -1;
  if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0) return -1;
  if (dtype != 0 && dtype != 1) return -1;
  if (conv_w && (conv_width < 1 || conv_width > 64)) return -1;
  if (!channels) n_channels = batch * dim;
  if (n_channels <= 0) return -1;
  if (channels)
    for (int64_t i = 0; i < n_channels; ++i)
      if (channels[i] < 0 || channels[i] >= batch * dim) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;

  job_t J;
  memset(&J, 0, sizeof J);
  J.u = u; J.delta = delta; J.B = B; J.C = C; J.z = z;
  J.A = A; J.D = D; J.delta_bias = delta_bias;
  J.softplus_flag = softplus_flag; J.dtype = dtype;
  J.batch = batch; J.dim = dim; J.seqlen = seqlen; J.dstate = dstate;
  J.channels = channels; J.n_channels = n_channels;
  J.y = y; J.last_state = last_state; J.h0 = h0; J.next = 0;
  J.conv_w = conv_w; J.conv_b = conv_b; J.conv_width = conv_w ? conv_width : 0;
  J.zoh = zoh != 0;
  pthread_mutex_init(&J.mu, NULL);

  pthread_t tids[512];
  int started = 0;
  for (int i = 1; i < nthreads; ++i)
    if (pthread_create(&tids[started], NULL, worker, &J) == 0) ++started;
  worker(&J);
  for (int i = 0; i < started; ++i) pthread_join(tids[i], NULL);
  pthread_mutex_destroy(&J.mu);
  return 0;
}

/* The scalar pieces, exported so that tests can pin them one by one. */
double oracle_softplus(double x) { return softplus64(x); }
double oracle_silu(double z) { return silu64(z); }


/* ------------------------------------------------------------- backward --
 *
 * Reverse-mode derivative of the simplified-B_bar scan (h0 = 0, no
 * convolution) for a loss whose gradient with respect to y is dy (and, if
 * given, dlast with respect to the final state).  Per channel the forward
 * states h_t are recomputed and kept, then the adjoint g_t = dL/dh_t runs
 * backwards in time:
 *
 *   q_t  = C_t . h_t + D u_t,   y_t = q_t SiLU(z_t)
 *   dq_t = dy_t SiLU(z_t),      dz_t = dy_t q_t SiLU'(z_t)
 *   g_t[n] = dq_t C_t[n] + a_{t+1}[n] g_{t+1}[n]   (+ dlast[n] at t = L-1)
 *   with a_t[n] = exp(Delta_t A[n]):
 *     dDelta_t = sum_n g_t[n] (B_t[n] u_t + A[n] a_t[n] h_{t-1}[n])
 *     du_t     = dq_t D + sum_n g_t[n] Delta_t B_t[n]
 *     dA[n]   += g_t[n] Delta_t a_t[n] h_{t-1}[n]
 *     dB_t[n] += g_t[n] Delta_t u_t          (summed over channels d)
 *     dC_t[n] += dq_t h_t[n]                 (summed over channels d)
 *     dD      += dq_t u_t
 *     ddelta_t = dDelta_t softplus'(x_t) = dDelta_t sigmoid(x_t)  (flag on)
 *     dbias   += ddelta_t
 * SiLU'(z) = s (1 + z (1 - s)), s = sigmoid(z).  The pages describe this
 * backward only as recomputation instead of stored states ("Mamba 深度解读报告",
 * sec. 3.3; "Mamba 选择性机制", sec. 3.4); the derivative itself is the chain
 * rule applied to the forward above.
 */
typedef struct {
  const void *u, *delta, *B, *C, *z;
  const float *A, *D, *delta_bias;
  const double *dy, *dlast;
  int softplus_flag, dtype;
  int64_t batch, dim, seqlen;
  int dstate;
  double *du, *ddelta, *dz;         /* [batch, dim, L] */
  double *dA, *dB, *dC, *dD, *dbias; /* shared sums, merged under mu */
  int64_t next;
  pthread_mutex_t mu;
} bjob_t;

static double sigmoid64(double x) { return 1.0 / (1.0 + exp(-x)); }

static void bwd_channel(bjob_t* J, int64_t flat, double* hs, double* g, double* dA,
                        double* dB, double* dC, double* dD, double* dbias) {
  const int64_t b = flat / J->dim, d = flat % J->dim, L = J->seqlen;
  const int N = J->dstate;
  const int64_t row = (b * J->dim + d) * L, bc = b * (int64_t)N * L;
  const double bias = J->delta_bias ? (double)J->delta_bias[d] : 0.0;
  const double Dd = J->D ? (double)J->D[d] : 0.0;
  /* forward, keeping h_t for every t */
  for (int64_t t = 0; t < L; ++t) {
    const double x = widen(J->delta, J->dtype, row + t) + bias;
    const double dt = J->softplus_flag ? softplus64(x) : x;
    const double ut = widen(J->u, J->dtype, row + t);
    for (int n = 0; n < N; ++n) {
      const double prev = t ? hs[(t - 1) * N + n] : 0.0;
      hs[t * N + n] = exp(dt * (double)J->A[d * N + n]) * prev +
                      dt * widen(J->B, J->dtype, bc + (int64_t)n * L + t) * ut;
    }
  }
  /* adjoint, backwards */
  for (int n = 0; n < N; ++n) g[n] = J->dlast ? J->dlast[flat * N + n] : 0.0;
  for (int64_t t = L - 1; t >= 0; --t) {
    const double x = widen(J->delta, J->dtype, row + t) + bias;
    const double dt = J->softplus_flag ? softplus64(x) : x;
    const double ut = widen(J->u, J->dtype, row + t);
    double q = Dd * ut;
    for (int n = 0; n < N; ++n) q += widen(J->C, J->dtype, bc + (int64_t)n * L + t) * hs[t * N + n];
    double dq = J->dy[row + t];
    if (J->z) {
      const double zt = widen(J->z, J->dtype, row + t), sg = sigmoid64(zt);
      J->dz[row + t] = J->dy[row + t] * q * sg * (1.0 + zt * (1.0 - sg));
      dq = J->dy[row + t] * zt * sg;
    }
    double ddt = 0.0, du = dq * Dd;
    *dD += dq * ut;
    for (int n = 0; n < N; ++n) {
      const double an = (double)J->A[d * N + n];
      const double a = exp(dt * an);
      const double bt = widen(J->B, J->dtype, bc + (int64_t)n * L + t);
      const double ct = widen(J->C, J->dtype, bc + (int64_t)n * L + t);
      const double prev = t ? hs[(t - 1) * N + n] : 0.0;
      const double gt = g[n] + dq * ct; /* g[n] holds a_{t+1} g_{t+1} (+ dlast) */
      ddt += gt * (bt * ut + an * a * prev);
      du += gt * dt * bt;
      dA[d * N + n] += gt * dt * a * prev;
      dB[bc + (int64_t)n * L + t] += gt * dt * ut;
      dC[bc + (int64_t)n * L + t] += dq * hs[t * N + n];
      g[n] = a * gt;
    }
    const double dx = J->softplus_flag ? ddt * sigmoid64(x) : ddt;
    J->ddelta[row + t] = dx;
    J->du[row + t] = du;
    dbias[d] += dx;
  }
}

static void* bwd_worker(void* arg) {
  bjob_t* J = (bjob_t*)arg;
  const int N = J->dstate;
  const int64_t L = J->seqlen, D = J->dim;
  const size_t nbc = (size_t)J->batch * N * L;
  double* hs = (double*)malloc(sizeof(double) * (size_t)L * N);
  double* g = (double*)malloc(sizeof(double) * N);
  double* dA = (double*)calloc((size_t)D * N, sizeof(double));
  double* dB = (double*)calloc(nbc, sizeof(double));
  double* dC = (double*)calloc(nbc, sizeof(double));
  double* dD = (double*)calloc((size_t)D, sizeof(double));
  double* dbias = (double*)calloc((size_t)D, sizeof(double));
  if (hs && g && dA && dB && dC && dD && dbias) {
    for (;;) {
      pthread_mutex_lock(&J->mu);
      const int64_t flat = J->next++;
      pthread_mutex_unlock(&J->mu);
      if (flat >= J->batch * D) break;
      double dDd = 0.0;
      bwd_channel(J, flat, hs, g, dA, dB, dC, &dDd, dbias);
      dD[flat % D] += dDd;
    }
    pthread_mutex_lock(&J->mu);
    for (int64_t i = 0; i < D * N; ++i) J->dA[i] += dA[i];
    for (size_t i = 0; i < nbc; ++i) {
      J->dB[i] += dB[i];
      J->dC[i] += dC[i];
    }
    for (int64_t i = 0; i < D; ++i) {
      J->dD[i] += dD[i];
      J->dbias[i] += dbias[i];
    }
    pthread_mutex_unlock(&J->mu);
  }
  free(hs); free(g); free(dA); free(dB); free(dC); free(dD); free(dbias);
  return NULL;
}

/*
 * oracle_scan_bwd: returns 0, or -1 on a bad argument or memory shortage.
 * Inputs as oracle_scan_fwd (every channel); dy [batch, dim, L] and dlast
 * [batch, dim, N] (nullable) in double.  Outputs (double, overwritten):
 * du, ddelta, dz [batch, dim, L] (dz ignored without z); dA [dim, N];
 * dB, dC [batch, N, L]; dD, dbias [dim].
 */
int oracle_scan_bwd(const void* u, const void* delta, const float* A, const void* B,
                    const void* C, const float* D, const void* z, const float* delta_bias,
                    int softplus_flag, int dtype, int64_t batch, int64_t dim, int64_t seqlen,
                    int dstate, const double* dy, const double* dlast, double* du,
                    double* ddelta, double* dz, double* dA, double* dB, double* dC,
                    double* dD, double* dbias, int nthreads) {
  if (!u || !delta || !A || !B || !C || !dy || !du || !ddelta || !dA || !dB || !dC || !dD ||
      !dbias || (z && !dz))
    return -1;
  if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0) return -1;
  if (dtype != 0 && dtype != 1) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;
  memset(dA, 0, sizeof(double) * (size_t)(dim * dstate));
  memset(dB, 0, sizeof(double) * (size_t)(batch * dstate * seqlen));
  memset(dC, 0, sizeof(double) * (size_t)(batch * dstate * seqlen));
  memset(dD, 0, sizeof(double) * (size_t)dim);
  memset(dbias, 0, sizeof(double) * (size_t)dim);
  bjob_t J;
  memset(&J, 0, sizeof J);
  J.u = u; J.delta = delta; J.B = B; J.C = C; J.z = z;
  J.A = A; J.D = D; J.delta_bias = delta_bias; J.dy = dy; J.dlast = dlast;
  J.softplus_flag = softplus_flag; J.dtype = dtype;
  J.batch = batch; J.dim = dim; J.seqlen = seqlen; J.dstate = dstate;
  J.du = du; J.ddelta = ddelta; J.dz = dz;
  J.dA = dA; J.dB = dB; J.dC = dC; J.dD = dD; J.dbias = dbias;
  pthread_mutex_init(&J.mu, NULL);
  pthread_t tids[512];
  int started = 0;
  for (int i = 1; i < nthreads; ++i)
    if (pthread_create(&tids[started], NULL, bwd_worker, &J) == 0) ++started;
  bwd_worker(&J);
  for (int i = 0; i < started; ++i) pthread_join(tids[i], NULL);
  pthread_mutex_destroy(&J.mu);
  return 0;
}
