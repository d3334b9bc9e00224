/*
 * oracle.c -- plain, slow, fp64 CPU oracle of the Liger Attention forward pass
 * (prefill and decode) and of the prefill's gradient.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The product
 * (the CUDA library and its Python binding) never calls it, and the two share
 * no code, header, table or helper.
 *
 * Sources (web pages on Liger, by title and section):
 *   [N-gate]  "Liger: Linearizing Large Language Models to Gated Recurrent
 *             Structures" (Paper-Notes), section "核心思想：Key 投影复用构建门控",
 *             gate equation G_t = f(k_t) = f(x_t W_K), f = a parameter-free
 *             pooling such as the mean.
 *   [N-rec]   same page, section "统一的门控线性循环框架", recurrence
 *             S_t = G_t (.) S_{t-1} + phi(k_t)^T v_t,  o_t = phi(q_t) S_t,
 *             with phi = Softmax (no learned feature map).
 *   [N-vgate] same page, same section: Liger adapts to other gated recurrent
 *             structures (GLA, Mamba2, mLSTM, HGRN2, RWKV6) by the form of G_t;
 *             read here as GLA's per-dimension gate with the parameter-free
 *             pooling of the key taken per element: G_t[r] = sigmoid(k_t[r])
 *             acting on row r (key dimension) of S, so G_t (.) S_{t-1} is
 *             diag(G_t) S_{t-1}.
 *   [N-mix]   same page, section "Liger Attention：层内混合注意力",
 *             o_t = alpha*GRM + beta*SWA, alpha + beta = 1 (0.5 each), w = 64.
 *   [J-method] news article on Liger (Japanese), section "手法の説明":
 *             gate obtained by pooling the key projection; feature map
 *             simplified to a Softmax applied to Q and to K separately.
 *
 * Readings where the pages leave a step open (all listed in the design notes):
 *   - phi is a softmax over the head dimension, per token and head, no scale.
 *   - the pooled gate is sigmoid(mean_d k_t), a scalar per (token, kv head),
 *     formed in log space: log g = -softplus(-m).
 *   - "phi(k_t^T) v_t" is the outer product phi(k_t)^T v_t (d_k x d_v).
 *   - the state is updated before it is read (o_t uses S_t).
 *   - SWA: keys t-w+1 .. t (self included), scores q.k / sqrt(d), raw q, k.
 *   - beta = 1 - alpha; GQA: q head h reads kv head h / (Hq/Hkv).
 *   - varlen: state and window restart at each sequence start.
 *   - initial_state seeds the recurrence only; the window starts at the first
 *     token of the call.
 *
 * The gradient has no formula on the pages (the linearisation fine-tune they
 * describe trains through this layer): it is the reverse-mode derivative of the
 * same token-by-token evaluation, written out step by step.
 *
 * Everything is evaluated token by token, exactly in the order of the
 * recurrence, in double precision.  Work is split over POSIX threads by
 * (sequence, q head) for prefill and by batch row for decode.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ---- elementary pieces -------------------------------------------------- */

/* Softmax of x[0..d) into y, max-subtracted.  [N-rec] phi = Softmax. */
void oracle_feature_map(const double* x, int d, double* y) {
  double m = x[0];
  for (int i = 1; i < d; ++i) m = x[i] > m ? x[i] : m;
  double s = 0.0;
  for (int i = 0; i < d; ++i) { y[i] = exp(x[i] - m); s += y[i]; }
  for (int i = 0; i < d; ++i) y[i] /= s;
}

/* log of the pooled gate: log sigmoid(mean_d k).  [N-gate]
 * log sigmoid(m) = -log(1 + exp(-m)), written so that neither branch
 * overflows: for m >= 0 use -log1p(exp(-m)); for m < 0 use m - log1p(exp(m)). */
double oracle_log_gate(const double* k, int d) {
  double m = 0.0;
  for (int i = 0; i < d; ++i) m += k[i];
  m /= (double)d;
  if (m >= 0.0) return -log1p(exp(-m));
  return m - log1p(exp(m));
}

/* ---- prefill ------------------------------------------------------------ */

typedef struct {
  const double *q, *k, *v, *s0;
  const int* cu;
  int B, Hq, Hkv, T, d, w, n_seqs, gate_off;
  double alpha;
  double *out, *fs, *ring;
  int* pos;
  int unit_begin, unit_end;  /* units are (seq, q head) pairs */
} prefill_job;

static void prefill_unit(const prefill_job* J, int seq, int h) {
  const int d = J->d, Hq = J->Hq, Hkv = J->Hkv, w = J->w;
  const int G = Hq / Hkv, kv = h / G;
  /* token range [t0, t1) inside the [B, T] grid flattened over (b, t) */
  long t0, t1;
  if (J->cu) { t0 = J->cu[seq]; t1 = J->cu[seq + 1]; }
  else { t0 = (long)seq * J->T; t1 = t0 + J->T; }
  const long len = t1 - t0;

  double* S = (double*)malloc(sizeof(double) * d * d);
  double* pk = (double*)malloc(sizeof(double) * d);
  double* pq = (double*)malloc(sizeof(double) * d);
  double* sc = (double*)malloc(sizeof(double) * w);
  if (J->s0) memcpy(S, J->s0 + ((long)seq * Hq + h) * d * d, sizeof(double) * d * d);
  else memset(S, 0, sizeof(double) * d * d);
  const double inv_sqrt_d = 1.0 / sqrt((double)d);

  for (long t = t0; t < t1; ++t) {
    const double* qt = J->q + (t * Hq + h) * d;
    const double* kt = J->k + (t * Hkv + kv) * d;
    const double* vt = J->v + (t * Hkv + kv) * d;
    /* gated recurrent branch [N-gate], [N-rec] */
    const double g = J->gate_off == 1 ? 1.0 : exp(oracle_log_gate(kt, d));
    oracle_feature_map(kt, d, pk);
    oracle_feature_map(qt, d, pq);
    for (int r = 0; r < d; ++r) {
      /* gate_off == 2: one gate per key dimension, sigmoid(k[r]) on row r [N-vgate] */
      const double gr = J->gate_off == 2 ? exp(oracle_log_gate(kt + r, 1)) : g;
      for (int c = 0; c < d; ++c) S[r * d + c] = gr * S[r * d + c] + pk[r] * vt[c];
    }
    double* o = J->out + (t * Hq + h) * d;
    for (int c = 0; c < d; ++c) {
      double a = 0.0;
      for (int r = 0; r < d; ++r) a += pq[r] * S[r * d + c];
      o[c] = J->alpha * a;
    }
    /* sliding-window branch [N-mix] */
    long j0 = t - w + 1;
    if (j0 < t0) j0 = t0;
    double mx = -INFINITY;
    for (long j = j0; j <= t; ++j) {
      const double* kj = J->k + (j * Hkv + kv) * d;
      double s = 0.0;
      for (int i = 0; i < d; ++i) s += qt[i] * kj[i];
      s *= inv_sqrt_d;
      sc[j - j0] = s;
      if (s > mx) mx = s;
    }
    double l = 0.0;
    for (long j = j0; j <= t; ++j) { sc[j - j0] = exp(sc[j - j0] - mx); l += sc[j - j0]; }
    const double beta = 1.0 - J->alpha;
    for (int c = 0; c < d; ++c) {
      double a = 0.0;
      for (long j = j0; j <= t; ++j) a += sc[j - j0] * J->v[(j * Hkv + kv) * d + c];
      o[c] += beta * a / l;
    }
  }
  if (J->fs) memcpy(J->fs + ((long)seq * Hq + h) * d * d, S, sizeof(double) * d * d);
  /* ring and position: written once per (seq, kv head) by the group's first q head */
  if (h % G == 0 && J->ring) {
    double* rk = J->ring + (((long)seq * Hkv + kv) * 2 + 0) * w * d;
    double* rv = J->ring + (((long)seq * Hkv + kv) * 2 + 1) * w * d;
    memset(rk, 0, sizeof(double) * w * d);
    memset(rv, 0, sizeof(double) * w * d);
    long first = len > w ? len - w : 0;
    for (long p = first; p < len; ++p) {
      long t = t0 + p;
      memcpy(rk + (p % w) * d, J->k + (t * Hkv + kv) * d, sizeof(double) * d);
      memcpy(rv + (p % w) * d, J->v + (t * Hkv + kv) * d, sizeof(double) * d);
    }
  }
  if (h == 0 && J->pos) J->pos[seq] = (int)len;
  free(S); free(pk); free(pq); free(sc);
}

static void* prefill_worker(void* arg) {
  const prefill_job* J = (const prefill_job*)arg;
  for (int u = J->unit_begin; u < J->unit_end; ++u) prefill_unit(J, u / J->Hq, u % J->Hq);
  return NULL;
}

/*
 * Prefill over one batch.
 *   q [B, T, Hq, d], k and v [B, T, Hkv, d], out [B, T, Hq, d]   (row-major)
 *   With cu_seqlens (n_seqs + 1 offsets into the T axis), B must be 1 and the
 *   T axis holds n_seqs packed sequences; otherwise n_seqs = B.
 *   initial_state [n_seqs, Hq, d, d] or NULL (zero state).
 *   final_state   [n_seqs, Hq, d, d] or NULL; row = key dim, column = value dim.
 *   ring_out      [n_seqs, Hkv, 2, w, d] or NULL: the last min(len, w) keys and
 *                 values, position p at slot p mod w, other slots zero.
 *   pos_out       [n_seqs] or NULL: the sequence lengths.
 *   gate_off      gate form: 0 the pooled scalar gate sigmoid(mean_d k_t) [N-gate];
 *                 1 forces g = 1 (ungated linear attention, a test switch);
 *                 2 one gate per key dimension, sigmoid(k_t[r]) scaling row r of
 *                 the state [N-vgate].
 * Returns 0, or -1 on a bad argument.
 */
int oracle_prefill(const double* q, const double* k, const double* v, int B, int Hq, int Hkv,
                   int T, int d, int w, double alpha, const double* initial_state,
                   const int* cu_seqlens, int n_seqs, double* out, double* final_state,
                   double* ring_out, int* pos_out, int gate_off, int nthreads) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || T < 0 || d < 1 || w < 1) return -1;
  if (cu_seqlens) {
    if (B != 1 || n_seqs < 1 || cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != T) return -1;
    for (int i = 0; i < n_seqs; ++i)
      if (cu_seqlens[i + 1] < cu_seqlens[i]) return -1;
  } else {
    n_seqs = B;
  }
  const int units = n_seqs * Hq;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > units) nthreads = units;
  prefill_job base = {q, k, v, initial_state, cu_seqlens, B, Hq, Hkv, T, d, w, n_seqs,
                      gate_off, alpha, out, final_state, ring_out, pos_out, 0, 0};
  prefill_job* jobs = (prefill_job*)malloc(sizeof(prefill_job) * nthreads);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
  for (int i = 0; i < nthreads; ++i) {
    jobs[i] = base;
    jobs[i].unit_begin = (int)((long)units * i / nthreads);
    jobs[i].unit_end = (int)((long)units * (i + 1) / nthreads);
    pthread_create(&th[i], NULL, prefill_worker, &jobs[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  free(jobs); free(th);
  return 0;
}

/* ---- prefill backward ---------------------------------------------------- */

/* log sigmoid(m), overflow-free on both sides (the same form as the gate). */
static double log_sigmoid(double m) {
  if (m >= 0.0) return -log1p(exp(-m));
  return m - log1p(exp(m));
}

typedef struct {
  const double *q, *k, *v, *s0, *dout, *dfs;
  const int* cu;
  int Hq, Hkv, T, d, w, gate_off;
  double alpha;
  double *dq, *dk, *dv, *ds0;
  int unit_begin, unit_end;  /* units are (seq, kv head) pairs */
} backward_job;

/* One q head of one sequence: a forward sweep that keeps every state, then the
 * reverse sweep.  dq of the head is written; dk and dv of its kv head are
 * accumulated (the caller runs the heads of one kv head one after another). */
static void backward_head(const backward_job* J, long t0, long t1, int seq, int h) {
  const int d = J->d, Hq = J->Hq, Hkv = J->Hkv, w = J->w;
  const int G = Hq / Hkv, kv = h / G;
  const long len = t1 - t0;
  const long dd = (long)d * d;
  const double alpha = J->alpha, beta = 1.0 - J->alpha;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);

  /* Ss[i] = state after i tokens of the sequence (Ss[0] = initial state) */
  double* Ss = (double*)malloc(sizeof(double) * dd * (len + 1));
  double* dS = (double*)malloc(sizeof(double) * dd);
  double* pk = (double*)malloc(sizeof(double) * d);
  double* pq = (double*)malloc(sizeof(double) * d);
  double* dpk = (double*)malloc(sizeof(double) * d);
  double* dpq = (double*)malloc(sizeof(double) * d);
  double* p = (double*)malloc(sizeof(double) * w);
  double* dp = (double*)malloc(sizeof(double) * w);
  if (J->s0) memcpy(Ss, J->s0 + ((long)seq * Hq + h) * dd, sizeof(double) * dd);
  else memset(Ss, 0, sizeof(double) * dd);
  for (long t = t0; t < t1; ++t) {
    const double* kt = J->k + (t * Hkv + kv) * d;
    const double* vt = J->v + (t * Hkv + kv) * d;
    const double g = J->gate_off ? 1.0 : exp(oracle_log_gate(kt, d));
    oracle_feature_map(kt, d, pk);
    const double* prev = Ss + (t - t0) * dd;
    double* cur = Ss + (t - t0 + 1) * dd;
    for (int r = 0; r < d; ++r)
      for (int c = 0; c < d; ++c) cur[r * d + c] = g * prev[r * d + c] + pk[r] * vt[c];
  }

  /* gradient of the final state comes from the loss's second term */
  if (J->dfs) memcpy(dS, J->dfs + ((long)seq * Hq + h) * dd, sizeof(double) * dd);
  else memset(dS, 0, sizeof(double) * dd);
  for (long t = t1 - 1; t >= t0; --t) {
    const double* qt = J->q + (t * Hq + h) * d;
    const double* kt = J->k + (t * Hkv + kv) * d;
    const double* vt = J->v + (t * Hkv + kv) * d;
    const double* dot = J->dout + (t * Hq + h) * d;
    double* dqt = J->dq + (t * Hq + h) * d;
    double* dkt = J->dk + (t * Hkv + kv) * d;
    double* dvt = J->dv + (t * Hkv + kv) * d;
    const double* cur = Ss + (t - t0 + 1) * dd;
    const double* prev = Ss + (t - t0) * dd;
    oracle_feature_map(kt, d, pk);
    oracle_feature_map(qt, d, pq);

    /* read-out: out_t += alpha * phi(q_t) S_t */
    for (int r = 0; r < d; ++r) {
      double a = 0.0;
      for (int c = 0; c < d; ++c) a += cur[r * d + c] * dot[c];
      dpq[r] = alpha * a;
    }
    for (int r = 0; r < d; ++r)
      for (int c = 0; c < d; ++c) dS[r * d + c] += alpha * pq[r] * dot[c];

    /* update: S_t = g_t S_{t-1} + phi(k_t)^T v_t */
    for (int r = 0; r < d; ++r) {
      double a = 0.0;
      for (int c = 0; c < d; ++c) a += dS[r * d + c] * vt[c];
      dpk[r] = a;
    }
    for (int c = 0; c < d; ++c) {
      double a = 0.0;
      for (int r = 0; r < d; ++r) a += pk[r] * dS[r * d + c];
      dvt[c] += a;
    }
    double dg = 0.0;
    for (long e = 0; e < dd; ++e) dg += dS[e] * prev[e];
    double m = 0.0;
    for (int i = 0; i < d; ++i) m += kt[i];
    m /= (double)d;
    const double g = J->gate_off ? 1.0 : exp(log_sigmoid(m));
    for (long e = 0; e < dd; ++e) dS[e] *= g;   /* now the gradient of S_{t-1} */

    /* softmax feature maps: dx = phi (dphi - <dphi, phi>) */
    double a = 0.0, b = 0.0;
    for (int r = 0; r < d; ++r) { a += dpq[r] * pq[r]; b += dpk[r] * pk[r]; }
    for (int r = 0; r < d; ++r) {
      dqt[r] += pq[r] * (dpq[r] - a);
      dkt[r] += pk[r] * (dpk[r] - b);
    }
    /* gate: g = sigmoid(mean k), dg/dm = sigmoid(m) sigmoid(-m) */
    if (!J->gate_off) {
      const double gm = dg * exp(log_sigmoid(m) + log_sigmoid(-m)) / (double)d;
      for (int i = 0; i < d; ++i) dkt[i] += gm;
    }

    /* window branch: out_t += beta * sum_j p_j v_j, p = softmax_j(q_t.k_j / sqrt d) */
    long j0 = t - w + 1;
    if (j0 < t0) j0 = t0;
    double mx = -INFINITY;
    for (long j = j0; j <= t; ++j) {
      const double* kj = J->k + (j * Hkv + kv) * d;
      double s = 0.0;
      for (int i = 0; i < d; ++i) s += qt[i] * kj[i];
      s *= inv_sqrt_d;
      p[j - j0] = s;
      if (s > mx) mx = s;
    }
    double l = 0.0;
    for (long j = j0; j <= t; ++j) { p[j - j0] = exp(p[j - j0] - mx); l += p[j - j0]; }
    for (long j = j0; j <= t; ++j) p[j - j0] /= l;
    double pdp = 0.0;
    for (long j = j0; j <= t; ++j) {
      const double* vj = J->v + (j * Hkv + kv) * d;
      double s = 0.0;
      for (int c = 0; c < d; ++c) s += dot[c] * vj[c];
      dp[j - j0] = beta * s;
      pdp += p[j - j0] * dp[j - j0];
    }
    for (long j = j0; j <= t; ++j) {
      const double* kj = J->k + (j * Hkv + kv) * d;
      double* dkj = J->dk + (j * Hkv + kv) * d;
      double* dvj = J->dv + (j * Hkv + kv) * d;
      const double pj = p[j - j0];
      const double dsj = pj * (dp[j - j0] - pdp) * inv_sqrt_d;
      for (int i = 0; i < d; ++i) {
        dqt[i] += dsj * kj[i];
        dkj[i] += dsj * qt[i];
        dvj[i] += beta * pj * dot[i];
      }
    }
  }
  if (J->ds0) memcpy(J->ds0 + ((long)seq * Hq + h) * dd, dS, sizeof(double) * dd);
  free(Ss); free(dS); free(pk); free(pq); free(dpk); free(dpq); free(p); free(dp);
}

static void* backward_worker(void* arg) {
  const backward_job* J = (const backward_job*)arg;
  const int G = J->Hq / J->Hkv;
  for (int u = J->unit_begin; u < J->unit_end; ++u) {
    const int seq = u / J->Hkv, kv = u % J->Hkv;
    long t0, t1;
    if (J->cu) { t0 = J->cu[seq]; t1 = J->cu[seq + 1]; }
    else { t0 = (long)seq * J->T; t1 = t0 + J->T; }
    for (int h = kv * G; h < (kv + 1) * G; ++h) backward_head(J, t0, t1, seq, h);
  }
  return NULL;
}

/*
 * Gradients of the prefill with respect to q, k, v and the initial state, for
 * the loss  L = sum(d_out * out) + sum(d_final_state * final_state).
 * The pages give no backward pass (their linearisation fine-tune needs one);
 * this is reverse-mode differentiation of the token-by-token evaluation above.
 *   d_out [B, T, Hq, d]; d_final_state [n_seqs, Hq, d, d] or NULL (zero).
 *   dq [B, T, Hq, d], dk and dv [B, T, Hkv, d]: written (zeroed first).
 *   d_initial_state [n_seqs, Hq, d, d] or NULL.
 * Layouts, cu_seqlens, w, alpha and gate_off as in oracle_prefill.  Memory:
 * every state of a sequence is kept, len * d * d doubles per (sequence, head)
 * in flight.  Returns 0, or -1 on a bad argument.
 */
int oracle_prefill_backward(const double* q, const double* k, const double* v, int B, int Hq,
                            int Hkv, int T, int d, int w, double alpha,
                            const double* initial_state, const int* cu_seqlens, int n_seqs,
                            const double* d_out, const double* d_final_state, double* dq,
                            double* dk, double* dv, double* d_initial_state, int gate_off,
                            int nthreads) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || T < 0 || d < 1 || w < 1 || !d_out || gate_off == 2) return -1;
  if (cu_seqlens) {
    if (B != 1 || n_seqs < 1 || cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != T) return -1;
    for (int i = 0; i < n_seqs; ++i)
      if (cu_seqlens[i + 1] < cu_seqlens[i]) return -1;
  } else {
    n_seqs = B;
  }
  memset(dq, 0, sizeof(double) * (size_t)B * T * Hq * d);
  memset(dk, 0, sizeof(double) * (size_t)B * T * Hkv * d);
  memset(dv, 0, sizeof(double) * (size_t)B * T * Hkv * d);
  const int units = n_seqs * Hkv;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > units) nthreads = units;
  backward_job base = {q, k, v, initial_state, d_out, d_final_state, cu_seqlens, Hq, Hkv, T, d,
                       w, gate_off, alpha, dq, dk, dv, d_initial_state, 0, 0};
  backward_job* jobs = (backward_job*)malloc(sizeof(backward_job) * nthreads);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
  for (int i = 0; i < nthreads; ++i) {
    jobs[i] = base;
    jobs[i].unit_begin = (int)((long)units * i / nthreads);
    jobs[i].unit_end = (int)((long)units * (i + 1) / nthreads);
    pthread_create(&th[i], NULL, backward_worker, &jobs[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  free(jobs); free(th);
  return 0;
}

/* ---- decode ------------------------------------------------------------- */

typedef struct {
  const double *q, *k, *v;
  double *state, *ring, *out;
  int* pos;
  int Hq, Hkv, d, w, gate_off;
  double alpha;
  int b_begin, b_end;
} decode_job;

static void decode_row(const decode_job* J, int b) {
  const int d = J->d, Hq = J->Hq, Hkv = J->Hkv, w = J->w, G = Hq / Hkv;
  const long p = J->pos[b];
  double* pk = (double*)malloc(sizeof(double) * d);
  double* pq = (double*)malloc(sizeof(double) * d);
  double* sc = (double*)malloc(sizeof(double) * w);
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  /* append the new key/value to each kv head's ring first; the window of
   * token p is then positions max(0, p-w+1) .. p, all held by the ring */
  for (int kv = 0; kv < Hkv; ++kv) {
    double* rk = J->ring + (((long)b * Hkv + kv) * 2 + 0) * w * d;
    double* rv = J->ring + (((long)b * Hkv + kv) * 2 + 1) * w * d;
    memcpy(rk + (p % w) * d, J->k + ((long)b * Hkv + kv) * d, sizeof(double) * d);
    memcpy(rv + (p % w) * d, J->v + ((long)b * Hkv + kv) * d, sizeof(double) * d);
  }
  for (int h = 0; h < Hq; ++h) {
    const int kv = h / G;
    const double* qt = J->q + ((long)b * Hq + h) * d;
    const double* kt = J->k + ((long)b * Hkv + kv) * d;
    const double* vt = J->v + ((long)b * Hkv + kv) * d;
    double* S = J->state + ((long)b * Hq + h) * d * d;
    const double g = J->gate_off == 1 ? 1.0 : exp(oracle_log_gate(kt, d));
    oracle_feature_map(kt, d, pk);
    oracle_feature_map(qt, d, pq);
    for (int r = 0; r < d; ++r) {
      const double gr = J->gate_off == 2 ? exp(oracle_log_gate(kt + r, 1)) : g;   /* [N-vgate] */
      for (int c = 0; c < d; ++c) S[r * d + c] = gr * S[r * d + c] + pk[r] * vt[c];
    }
    double* o = J->out + ((long)b * Hq + h) * d;
    for (int c = 0; c < d; ++c) {
      double a = 0.0;
      for (int r = 0; r < d; ++r) a += pq[r] * S[r * d + c];
      o[c] = J->alpha * a;
    }
    const double* rk = J->ring + (((long)b * Hkv + kv) * 2 + 0) * w * d;
    const double* rv = J->ring + (((long)b * Hkv + kv) * 2 + 1) * w * d;
    long j0 = p - w + 1;
    if (j0 < 0) j0 = 0;
    double mx = -INFINITY;
    for (long j = j0; j <= p; ++j) {
      const double* kj = rk + (j % w) * d;
      double s = 0.0;
      for (int i = 0; i < d; ++i) s += qt[i] * kj[i];
      s *= inv_sqrt_d;
      sc[j - j0] = s;
      if (s > mx) mx = s;
    }
    double l = 0.0;
    for (long j = j0; j <= p; ++j) { sc[j - j0] = exp(sc[j - j0] - mx); l += sc[j - j0]; }
    const double beta = 1.0 - J->alpha;
    for (int c = 0; c < d; ++c) {
      double a = 0.0;
      for (long j = j0; j <= p; ++j) a += sc[j - j0] * rv[(j % w) * d + c];
      o[c] += beta * a / l;
    }
  }
  J->pos[b] = (int)(p + 1);
  free(pk); free(pq); free(sc);
}

static void* decode_worker(void* arg) {
  const decode_job* J = (const decode_job*)arg;
  for (int b = J->b_begin; b < J->b_end; ++b) decode_row(J, b);
  return NULL;
}

/*
 * One decode step for B independent sequences (one new token each).
 *   q [B, Hq, d], k and v [B, Hkv, d], out [B, Hq, d]
 *   state [B, Hq, d, d] in/out, ring [B, Hkv, 2, w, d] in/out, pos [B] in/out.
 * Returns 0, or -1 on a bad argument.
 */
int oracle_decode(const double* q, const double* k, const double* v, double* state, double* ring,
                  double* out, int* pos, int B, int Hq, int Hkv, int d, int w, double alpha,
                  int gate_off, int nthreads) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || d < 1 || w < 1) return -1;
  for (int b = 0; b < B; ++b)
    if (pos[b] < 0) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > B) nthreads = B;
  decode_job base = {q, k, v, state, ring, out, pos, Hq, Hkv, d, w, gate_off, alpha, 0, 0};
  decode_job* jobs = (decode_job*)malloc(sizeof(decode_job) * nthreads);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
  for (int i = 0; i < nthreads; ++i) {
    jobs[i] = base;
    jobs[i].b_begin = (int)((long)B * i / nthreads);
    jobs[i].b_end = (int)((long)B * (i + 1) / nthreads);
    pthread_create(&th[i], NULL, decode_worker, &jobs[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  free(jobs); free(th);
  return 0;
}
