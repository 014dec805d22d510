/*
 * gdn_oracle.c -- CPU oracle for the chunked Gated DeltaNet (GDN) scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library; the two meet only through seeded inputs.
 *
 * What it computes (plain definition, token by token, in `real` = double or
 * long double, no blocking, no chunking, no reordering):
 *
 *   per (b, h):   S = state_in  (or 0)
 *     for t = 0 .. T-1:
 *       q^ = q_t / sqrt(max(|q_t|^2, 1e-12)),  k^ likewise
 *       a  = exp(g_t),  b = beta_t
 *       S  = a (I - b k^ k^T) S + b k^ v_t^T          (S is Dk x Dv)
 *       o_t = S^T q^
 *   state_out = S
 *
 * This is the Gated DeltaNet state update.  The pages describe GDN only in
 * words: a fixed-size memory that is updated recursively from the previous
 * state ("[논문리뷰] SANA-Streaming: Real-time Streaming Video Editing with
 * Hybrid Diffusion Transformer", 1. Key Terms & Definitions, "GDN"), used in
 * streaming as a forward scan that starts from the previous chunk's cache
 * ("SANA-Streaming：基于混合扩散Transformer的实时流式视频编辑系统",
 * 方法步骤详情, second step).  The decay a multiplies the old state before the
 * delta correction, and (I - b k k^T) acts on the left of S, the reading
 * under which S^T k = v holds after a unit-gate update.
 *
 * Bidirectional mode (same page, same step: "前向扫描（带上一chunk缓存）+
 * chunk内后向扫描"): out = forward scan from state_in + the same recurrence
 * run over the time-reversed chunk from a zero state (token t keeps its own
 * g_t and beta_t, its own term counted in both directions, plain sum);
 * state_out comes from the forward scan only.
 *
 * Gate-logit mode (the *_logits entry points): the g and beta arrays hold
 * the gate layer's two logits x_t, y_t instead, and the gates are
 *   g_t = -softplus(x_t) = -log(1 + e^{x_t}),   beta_t = sigmoid(y_t),
 * evaluated here in `real`.  The pages name the gate layer (it stays in BF16
 * under mixed-precision quantisation: same page, 实验结果) but do not write its
 * activations; these are the plainest maps onto g <= 0 and beta in (0, 1).
 *
 * Layouts: q, k [B,T,H,Dk]; v, out [B,T,H,Dv]; g, beta [B,T,H];
 * state [B,H,Dk,Dv]; all row-major, contiguous.  Inputs are float (the exact
 * values the device sees, bf16 values are exact in float); outputs are real.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#ifndef ORACLE_REAL
#define ORACLE_REAL double
#define ORACLE_SUFFIX(name) name
#endif
typedef ORACLE_REAL real;

#define ORACLE_EXP(x) ((real)expl((long double)(x)))
#define ORACLE_SQRT(x) ((real)sqrtl((long double)(x)))

typedef struct {
  const float *q, *k, *v, *g, *beta;
  const real *state_in;
  real *state_out, *out;
  int B, T, H, Dk, Dv;
  int bidir;
  int logits;               /* g, beta hold gate logits */
  int next;                 /* next (b,h) pair to take, guarded by lock */
  pthread_mutex_t lock;
} job_t;

/* x^ = x / sqrt(max(sum x^2, 1e-12)) */
static void l2_normalise(const float *x, int n, real *xhat) {
  real ss = 0;
  for (int i = 0; i < n; ++i) ss += (real)x[i] * (real)x[i];
  if (ss < (real)1e-12) ss = (real)1e-12;
  real inv = (real)1 / ORACLE_SQRT(ss);
  for (int i = 0; i < n; ++i) xhat[i] = (real)x[i] * inv;
}

/* The decay a = e^g and the write strength beta of one token: given
 * directly, or from the gate logits x, y as a = e^{-softplus(x)}, beta =
 * sigmoid(y) (each side of the softplus and sigmoid formed without
 * overflow). */
static real gate_decay(const job_t *J, size_t row) {
  const long double x = J->g[row];
  if (!J->logits) return ORACLE_EXP(x);
  const long double sp = x > 0 ? x + log1pl(expl(-x)) : log1pl(expl(x));
  return ORACLE_EXP(-sp);
}
static real gate_beta(const job_t *J, size_t row) {
  const long double y = J->beta[row];
  if (!J->logits) return (real)y;
  if (y >= 0) return (real)(1.0L / (1.0L + expl(-y)));
  const long double e = expl(y);
  return (real)(e / (1.0L + e));
}

/* One token of the recurrence: S = a (I - b k k^T) S + b k v^T, then
 * out[j] (+)= sum_i S[i][j] q[i].  x is scratch of length Dv. */
static void token_step(real *S, const real *khat, const real *qhat,
                       const float *v, real a, real b, int Dk, int Dv,
                       real *x, real *out, int accumulate) {
  /* x = k^T S  (row vector over the Dv columns) */
  for (int j = 0; j < Dv; ++j) x[j] = 0;
  for (int i = 0; i < Dk; ++i) {
    const real ki = khat[i];
    const real *Si = S + (size_t)i * Dv;
    for (int j = 0; j < Dv; ++j) x[j] += ki * Si[j];
  }
  /* S = a (S - b k x) + b k v^T */
  for (int i = 0; i < Dk; ++i) {
    const real ki = khat[i];
    real *Si = S + (size_t)i * Dv;
    for (int j = 0; j < Dv; ++j)
      Si[j] = a * (Si[j] - b * ki * x[j]) + b * ki * (real)v[j];
  }
  /* o = S^T q */
  for (int j = 0; j < Dv; ++j) x[j] = 0;
  for (int i = 0; i < Dk; ++i) {
    const real qi = qhat[i];
    const real *Si = S + (size_t)i * Dv;
    for (int j = 0; j < Dv; ++j) x[j] += qi * Si[j];
  }
  if (accumulate)
    for (int j = 0; j < Dv; ++j) out[j] += x[j];
  else
    for (int j = 0; j < Dv; ++j) out[j] = x[j];
}

static void scan_head(const job_t *J, int b, int h, real *S, real *khat,
                      real *qhat, real *x) {
  const int T = J->T, H = J->H, Dk = J->Dk, Dv = J->Dv;
  const size_t sbase = ((size_t)b * H + h) * (size_t)Dk * Dv;
  if (J->state_in)
    memcpy(S, J->state_in + sbase, sizeof(real) * (size_t)Dk * Dv);
  else
    memset(S, 0, sizeof(real) * (size_t)Dk * Dv);

  /* forward scan, carried state */
  for (int t = 0; t < T; ++t) {
    const size_t row = ((size_t)b * T + t) * H + h;
    l2_normalise(J->k + row * Dk, Dk, khat);
    l2_normalise(J->q + row * Dk, Dk, qhat);
    const real a = gate_decay(J, row);
    const real bt = gate_beta(J, row);
    token_step(S, khat, qhat, J->v + row * Dv, a, bt, Dk, Dv, x,
               J->out + row * Dv, 0);
  }
  if (J->state_out)
    memcpy(J->state_out + sbase, S, sizeof(real) * (size_t)Dk * Dv);

  if (!J->bidir) return;
  /* reverse scan over the same chunk, zero state, added into out */
  memset(S, 0, sizeof(real) * (size_t)Dk * Dv);
  for (int t = T - 1; t >= 0; --t) {
    const size_t row = ((size_t)b * T + t) * H + h;
    l2_normalise(J->k + row * Dk, Dk, khat);
    l2_normalise(J->q + row * Dk, Dk, qhat);
    const real a = gate_decay(J, row);
    const real bt = gate_beta(J, row);
    token_step(S, khat, qhat, J->v + row * Dv, a, bt, Dk, Dv, x,
               J->out + row * Dv, 1);
  }
}

static void *worker(void *arg) {
  job_t *J = (job_t *)arg;
  const int Dk = J->Dk, Dv = J->Dv;
  real *S = (real *)malloc(sizeof(real) * (size_t)Dk * Dv);
  real *khat = (real *)malloc(sizeof(real) * (size_t)Dk);
  real *qhat = (real *)malloc(sizeof(real) * (size_t)Dk);
  real *x = (real *)malloc(sizeof(real) * (size_t)Dv);
  if (S && khat && qhat && x) {
    for (;;) {
      pthread_mutex_lock(&J->lock);
      const int p = J->next++;
      pthread_mutex_unlock(&J->lock);
      if (p >= J->B * J->H) break;
      scan_head(J, p / J->H, p % J->H, S, khat, qhat, x);
    }
  }
  free(S); free(khat); free(qhat); free(x);
  return NULL;
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation failure.
 * nthreads <= 0 uses every online core.  state_in may be NULL (zero state);
 * state_out may be NULL. */
static int run(const float *q, const float *k, const float *v, const float *g,
               const float *beta, const real *state_in, real *state_out,
               real *out, int B, int T, int H, int Dk, int Dv, int bidir,
               int logits, int nthreads) {
  if (!q || !k || !v || !g || !beta || !out) return -1;
  if (B < 1 || T < 0 || H < 1 || Dk < 1 || Dv < 1) return -1;
  job_t J = {q, k, v, g, beta, state_in, state_out, out, B, T, H, Dk, Dv,
             bidir, logits, 0, PTHREAD_MUTEX_INITIALIZER};
  if (T == 0) {
    if (state_out) {
      const size_t n = (size_t)B * H * Dk * Dv;
      if (state_in) memcpy(state_out, state_in, sizeof(real) * n);
      else memset(state_out, 0, sizeof(real) * n);
    }
    return 0;
  }
  if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nthreads > B * H) nthreads = B * H;
  if (nthreads < 1) nthreads = 1;
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  if (!th) return -2;
  int started = 0;
  for (int i = 0; i < nthreads; ++i)
    if (pthread_create(&th[i], NULL, worker, &J) == 0) ++started;
  if (started == 0) worker(&J);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  free(th);
  return 0;
}

#define ORACLE_ENTRY(name, bidir, logits)                                      \
  int ORACLE_SUFFIX(name)(const float *q, const float *k, const float *v,      \
                          const float *g, const float *beta,                   \
                          const real *state_in, real *state_out, real *out,    \
                          int B, int T, int H, int Dk, int Dv, int nthreads) { \
    return run(q, k, v, g, beta, state_in, state_out, out, B, T, H, Dk, Dv,   \
               bidir, logits, nthreads);                                       \
  }
ORACLE_ENTRY(gdn_oracle_fwd, 0, 0)
ORACLE_ENTRY(gdn_oracle_bidir, 1, 0)
ORACLE_ENTRY(gdn_oracle_fwd_logits, 0, 1)
ORACLE_ENTRY(gdn_oracle_bidir_logits, 1, 1)

int ORACLE_SUFFIX(gdn_oracle_online_cores)(void) {
  return (int)sysconf(_SC_NPROCESSORS_ONLN);
}
