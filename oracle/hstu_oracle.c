/*
 * HSTU layer forward -- CPU oracle in plain C, fp64 throughout.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct definition that the CUDA path
 * is checked against.  It is used by the tests, by `__graft_entry__.smoke()` and by the CPU-baseline
 * and reference legs of `bench.py`, and by nothing else.  It shares no code, header, table or helper with the CUDA
 * path and includes nothing from it.
 *
 * What it computes (per layer, for every sequence s of a jagged batch and local token indices
 * i, j in [0, n_s)), following "Actions Speak Louder than Words" (paper notes), section 3.1,
 * Eqs. 1-3, and the HSTU-layer section of "4.4 推荐模型的 Scaling" (equations and the HSTULayer
 * sketch):
 *
 *   Eq. 1   Z = X W1 + b1;  U | V | Q | K = SiLU(Z)         (column blocks, in that order)
 *   Eq. 2   AV_i = sum_{j<=i} scale * SiLU(q_i . k_j + bias(i, j)) * v_j     (per head, no softmax)
 *   Eq. 3   G_i = LayerNorm(AV_i) * U_i;   Y_i = G_i W2 + b2 + X_i           (residual between layers)
 *
 * bias(i, j) is either the relative attention bias rab^{p,t}
 *   pos[h][min(i-j, P-1)] + time[h][min(Tb-1, floor(log2(1 + max(t_i - t_j, 0))))]
 * or the GenRank ALiBi bias  -m_h * (i - j).
 *
 * Readings of the pages that this file fixes (the pages leave them open):
 *   - `scale` multiplies SiLU's output (the sketch divides by a constant after SiLU);
 *   - the causal mask is the summation range j <= i (the sketch zeroes masked weights after SiLU);
 *   - LayerNorm spans all H*dv columns with biased variance and epsilon `ln_eps`;
 *   - the time bucket is computed exactly on integer seconds (highest set bit of 1 + delta);
 *   - the rab tables are per head; the position index is i - j clamped to P-1.
 *
 * Layouts: every matrix is row-major.  X [T, d], W1 [d, n1] (d_in x d_out) with
 * n1 = 2*H*dv + 2*H*dqk, UVQK [T, n1] with columns [U: H*dv | V: H*dv | Q: H*dqk | K: H*dqk], each
 * block head-major (head h owns columns h*hd .. h*hd+hd-1), AV and G [T, H*dv], W2 [H*dv, d],
 * Y [T, d].  Tables: pos [H, P], time [H, Tb], alibi slopes [H].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* SiLU(x) = x * sigmoid(x) = x / (1 + e^{-x}).  phi_1 and phi_2 of Eqs. 1-2. */
static double silu(double x) { return x / (1.0 + exp(-x)); }

/* floor(log2(v)) for v >= 1: the index of the highest set bit. */
static int32_t floor_log2_u64(uint64_t v) {
  int32_t b = 0;
  while (v > 1) {
    v >>= 1;
    b++;
  }
  return b;
}

int32_t oracle_time_bucket(int64_t ti, int64_t tj, int32_t n_time_buckets) {
  int64_t delta = ti - tj;
  if (delta < 0) delta = 0;
  int32_t b = floor_log2_u64((uint64_t)delta + 1u);
  return b < n_time_buckets - 1 ? b : n_time_buckets - 1;
}

int32_t oracle_pos_bucket(int64_t i, int64_t j, int32_t n_pos_buckets) {
  int64_t p = i - j;
  if (p < 0) p = 0;
  return p < n_pos_buckets - 1 ? (int32_t)p : n_pos_buckets - 1;
}

/* bias(i, j) for head h; i, j are local indices, ts points at the sequence's first timestamp. */
static double bias_at(int32_t h, int64_t i, int64_t j, const int64_t* ts,
                      const double* pos_table, int32_t P, const double* time_table, int32_t Tb,
                      const double* alibi_slopes) {
  if (alibi_slopes) return -alibi_slopes[h] * (double)(i - j);
  double b = 0.0;
  if (pos_table) b += pos_table[(int64_t)h * P + oracle_pos_bucket(i, j, P)];
  if (time_table) b += time_table[(int64_t)h * Tb + oracle_time_bucket(ts[i], ts[j], Tb)];
  return b;
}

/* ---------------------------------------------------------------------------------------------
 * Eq. 1: one row of the pointwise projection, columns [c0, c1):  out[c] = SiLU(b1[c] + sum_k x[k] W1[k][c]).
 * f1 is one affine map (weight W1, bias b1); phi_1 is SiLU; the result splits into U, V, Q, K.
 * --------------------------------------------------------------------------------------------- */
static void f1_row_cols(int32_t d, int32_t n1, const double* x, const double* W1, const double* b1,
                        int32_t c0, int32_t c1, double* out /* indexed by c */) {
  for (int32_t c = c0; c < c1; c++) out[c] = b1 ? b1[c] : 0.0;
  for (int32_t k = 0; k < d; k++) {
    const double xk = x[k];
    const double* w = W1 + (int64_t)k * n1;
    for (int32_t c = c0; c < c1; c++) out[c] += xk * w[c];
  }
  for (int32_t c = c0; c < c1; c++) out[c] = silu(out[c]);
}

void oracle_f1(int64_t T, int32_t d, int32_t n1, const double* X, const double* W1,
               const double* b1, double* uvqk) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; t++) f1_row_cols(d, n1, X + t * d, W1, b1, 0, n1, uvqk + t * n1);
}

/* ---------------------------------------------------------------------------------------------
 * Eq. 2: pointwise aggregated attention for one output row.
 * AV_i[h] = sum_{j=0}^{i} scale * SiLU(q_i[h] . k_j[h] + bias_h(i, j)) * v_j[h].
 * `uvqk_seq` points at the sequence's first row (row stride n1).
 * --------------------------------------------------------------------------------------------- */
static void attention_row(int64_t i, int32_t H, int32_t dqk, int32_t dv, int32_t n1,
                          const double* uvqk_seq, const int64_t* ts, const double* pos_table,
                          int32_t P, const double* time_table, int32_t Tb,
                          const double* alibi_slopes, double scale, double* av_row) {
  const int32_t offV = H * dv, offQ = 2 * H * dv, offK = 2 * H * dv + H * dqk;
  for (int32_t h = 0; h < H; h++) {
    double* acc = av_row + (int64_t)h * dv;
    for (int32_t c = 0; c < dv; c++) acc[c] = 0.0;
    const double* q = uvqk_seq + i * n1 + offQ + (int64_t)h * dqk;
    for (int64_t j = 0; j <= i; j++) {
      const double* k = uvqk_seq + j * n1 + offK + (int64_t)h * dqk;
      const double* v = uvqk_seq + j * n1 + offV + (int64_t)h * dv;
      double s = 0.0;
      for (int32_t c = 0; c < dqk; c++) s += q[c] * k[c];
      s += bias_at(h, i, j, ts, pos_table, P, time_table, Tb, alibi_slopes);
      const double a = scale * silu(s);
      for (int32_t c = 0; c < dv; c++) acc[c] += a * v[c];
    }
  }
}

void oracle_attention(int64_t B, const int64_t* seq_offsets, int32_t H, int32_t dqk, int32_t dv,
                      const double* uvqk, const int64_t* timestamps, const double* pos_table,
                      int32_t P, const double* time_table, int32_t Tb, const double* alibi_slopes,
                      double scale, double* av) {
  const int32_t n1 = 2 * H * dv + 2 * H * dqk;
  const int64_t T = seq_offsets[B];
  /* rows are independent; the row -> sequence map is a search over the offsets */
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t r = 0; r < T; r++) {
    int64_t s = 0;
    while (seq_offsets[s + 1] <= r) s++;
    const int64_t start = seq_offsets[s];
    attention_row(r - start, H, dqk, dv, n1, uvqk + start * n1,
                  timestamps ? timestamps + start : NULL, pos_table, P, time_table, Tb,
                  alibi_slopes, scale, av + r * (int64_t)H * dv);
  }
}

/* ---------------------------------------------------------------------------------------------
 * Backward of Eq. 2 (training; "Actions Speak Louder than Words" paper notes, sections 3.4-3.5 and
 * the training-speed figures of section 4): given dAV = dL/dAV, with x_ij = q_i . k_j + bias(i, j)
 * and a_ij = scale * SiLU(x_ij) for j <= i (per head),
 *   dv_j   = sum_{i >= j} a_ij dAV_i
 *   dx_ij  = scale * SiLU'(x_ij) * (dAV_i . v_j),  SiLU'(x) = s(x) (1 + x (1 - s(x))), s = sigmoid
 *   dq_i   = sum_{j <= i} dx_ij k_j,   dk_j = sum_{i >= j} dx_ij q_i
 *   dpos[h][p] = sum of dx_ij over the pairs whose position bucket is p; dtime likewise.
 * ALiBi slopes are fixed hyperparameters: no gradient.  Outputs are [T, H*hd] (dq, dk, dv) and the
 * table shapes, fully overwritten.
 * --------------------------------------------------------------------------------------------- */
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

void oracle_attention_bwd(int64_t B, const int64_t* seq_offsets, int32_t H, int32_t dqk, int32_t dv,
                          const double* uvqk, const int64_t* timestamps, const double* pos_table,
                          int32_t P, const double* time_table, int32_t Tb,
                          const double* alibi_slopes, double scale, const double* dav, double* dq,
                          double* dk, double* dvv, double* dpos, double* dtime) {
  const int32_t n1 = 2 * H * dv + 2 * H * dqk;
  const int32_t offV = H * dv, offQ = 2 * H * dv, offK = 2 * H * dv + H * dqk;
  const int64_t T = seq_offsets[B];
  memset(dq, 0, sizeof(double) * (size_t)T * H * dqk);
  memset(dk, 0, sizeof(double) * (size_t)T * H * dqk);
  memset(dvv, 0, sizeof(double) * (size_t)T * H * dv);
  if (dpos) memset(dpos, 0, sizeof(double) * (size_t)H * P);
  if (dtime) memset(dtime, 0, sizeof(double) * (size_t)H * Tb);
  /* one (sequence, head) at a time; its pairs touch only its rows and head columns */
  for (int64_t s = 0; s < B; s++) {
    const int64_t a0 = seq_offsets[s], n = seq_offsets[s + 1] - seq_offsets[s];
    const double* u = uvqk + a0 * n1;
    const int64_t* ts = timestamps ? timestamps + a0 : NULL;
    for (int32_t h = 0; h < H; h++) {
      for (int64_t i = 0; i < n; i++) {
        const double* q = u + i * n1 + offQ + (int64_t)h * dqk;
        const double* g = dav + (a0 + i) * (int64_t)H * dv + (int64_t)h * dv;
        for (int64_t j = 0; j <= i; j++) {
          const double* k = u + j * n1 + offK + (int64_t)h * dqk;
          const double* v = u + j * n1 + offV + (int64_t)h * dv;
          double x = 0.0, gv = 0.0;
          for (int32_t c = 0; c < dqk; c++) x += q[c] * k[c];
          x += bias_at(h, i, j, ts, pos_table, P, time_table, Tb, alibi_slopes);
          for (int32_t c = 0; c < dv; c++) gv += g[c] * v[c];
          const double sg = sigmoid(x);
          const double a = scale * x * sg;
          const double dx = scale * sg * (1.0 + x * (1.0 - sg)) * gv;
          double* dvj = dvv + (a0 + j) * (int64_t)H * dv + (int64_t)h * dv;
          for (int32_t c = 0; c < dv; c++) dvj[c] += a * g[c];
          double* dqi = dq + (a0 + i) * (int64_t)H * dqk + (int64_t)h * dqk;
          double* dkj = dk + (a0 + j) * (int64_t)H * dqk + (int64_t)h * dqk;
          for (int32_t c = 0; c < dqk; c++) {
            dqi[c] += dx * k[c];
            dkj[c] += dx * q[c];
          }
          if (!alibi_slopes) {
            if (pos_table && dpos) dpos[(int64_t)h * P + oracle_pos_bucket(i, j, P)] += dx;
            if (time_table && dtime)
              dtime[(int64_t)h * Tb + oracle_time_bucket(ts[i], ts[j], Tb)] += dx;
          }
        }
      }
    }
  }
}

/* ---------------------------------------------------------------------------------------------
 * M-FALCON candidate scoring ("Actions Speak Louder than Words" paper notes, section 3.6; the
 * efficiency paragraph of "4.4 推荐模型的 Scaling"): m candidates are appended after a user's n
 * history tokens and scored in one pass; the attention mask lets each candidate see the history
 * but no other candidate, and the relative bias is modified for candidates.  Readings fixed here:
 *   - a candidate also sees itself (the causal mask keeps its diagonal; only the other
 *     candidates are removed);
 *   - every candidate takes the position n it would have as the single item appended after the
 *     history, so its position bias towards history token j uses n - j and towards itself 0, and
 *     its time bias uses its own timestamp t_c: bucket of t_c - t_j, and of 0 for itself;
 *   - with ALiBi the bias is -m_h (n - j), and 0 for itself.
 * Hence, per head,
 *   AV_c = sum_{j<n} scale * SiLU(q_c . k_j + bias(n, j)) v_j + scale * SiLU(q_c . k_c + bias(n, n)) v_c
 * which, for a single candidate, is the causal attention row of the sequence [history, candidate]
 * at index n.  Micro-batching the candidates and caching the history's K and V change neither.
 * --------------------------------------------------------------------------------------------- */

/* Bias between a query at position pi with timestamp ti and a key at position pj, timestamp tj. */
static double bias_pt(int32_t h, int64_t pi, int64_t pj, int64_t ti, int64_t tj,
                      const double* pos_table, int32_t P, const double* time_table, int32_t Tb,
                      const double* alibi_slopes) {
  if (alibi_slopes) return -alibi_slopes[h] * (double)(pi - pj);
  double b = 0.0;
  if (pos_table) b += pos_table[(int64_t)h * P + oracle_pos_bucket(pi, pj, P)];
  if (time_table) b += time_table[(int64_t)h * Tb + oracle_time_bucket(ti, tj, Tb)];
  return b;
}

void oracle_candidate_attention(int64_t B, const int64_t* hist_offsets,
                                const int64_t* cand_offsets, int32_t H, int32_t dqk, int32_t dv,
                                const double* uvqk_hist, const int64_t* hist_ts,
                                const double* uvqk_cand, const int64_t* cand_ts,
                                const double* pos_table, int32_t P, const double* time_table,
                                int32_t Tb, const double* alibi_slopes, double scale,
                                double* av_cand) {
  const int32_t n1 = 2 * H * dv + 2 * H * dqk;
  const int32_t offV = H * dv, offQ = 2 * H * dv, offK = 2 * H * dv + H * dqk;
  const int64_t Tc = cand_offsets[B];
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t c = 0; c < Tc; c++) {
    int64_t b = 0;
    while (cand_offsets[b + 1] <= c) b++;
    const int64_t h0 = hist_offsets[b], n = hist_offsets[b + 1] - hist_offsets[b];
    const int64_t tc = cand_ts ? cand_ts[c] : 0;
    const double* crow = uvqk_cand + c * n1;
    for (int32_t h = 0; h < H; h++) {
      double* acc = av_cand + c * (int64_t)H * dv + (int64_t)h * dv;
      for (int32_t e = 0; e < dv; e++) acc[e] = 0.0;
      const double* q = crow + offQ + (int64_t)h * dqk;
      /* keys 0 .. n-1: the history; key n: the candidate itself */
      for (int64_t j = 0; j <= n; j++) {
        const double* krow = j < n ? uvqk_hist + (h0 + j) * n1 : crow;
        const double* k = krow + offK + (int64_t)h * dqk;
        const double* v = krow + offV + (int64_t)h * dv;
        const int64_t tj = j < n ? (hist_ts ? hist_ts[h0 + j] : 0) : tc;
        double sc = 0.0;
        for (int32_t e = 0; e < dqk; e++) sc += q[e] * k[e];
        sc += bias_pt(h, n, j, tc, tj, pos_table, P, time_table, Tb, alibi_slopes);
        const double a = scale * silu(sc);
        for (int32_t e = 0; e < dv; e++) acc[e] += a * v[e];
      }
    }
  }
}

/* ---------------------------------------------------------------------------------------------
 * Stochastic Length ("Actions Speak Louder than Words" paper notes, section 3.3).  With
 * N_c = the longest sequence (passed in) and alpha in (1, 2], a sequence of n tokens is kept whole
 * when n <= N_c^(alpha/2); otherwise, with probability 1 - N_c^alpha / n^2, it is replaced by a
 * subsequence of floor(N_c^(alpha/2)) of its tokens (and kept whole with probability
 * N_c^alpha / n^2).  Readings fixed here (the pages leave them open):
 *   - the subsequence is a uniformly random subset of that size, kept in the original order;
 *   - the method's random draws are inputs: u[s] uniform in [0, 1) per sequence (subsample when
 *     u[s] >= N_c^alpha / n^2) and keys[t] uniform 32-bit words per token (the subset is the
 *     floor(N_c^(alpha/2)) tokens with the smallest (key, position) pairs, which is a uniform
 *     random subset when the keys are i.i.d.).
 * Output: the new offsets [B+1] and, for the new batch's row r, the source row index[r]; returns
 * the new token count.
 * --------------------------------------------------------------------------------------------- */
typedef struct {
  uint32_t key;
  int64_t pos;
} sl_entry;

static int sl_by_key(const void* a, const void* b) {
  const sl_entry* x = (const sl_entry*)a;
  const sl_entry* y = (const sl_entry*)b;
  if (x->key != y->key) return x->key < y->key ? -1 : 1;
  return x->pos < y->pos ? -1 : (x->pos > y->pos ? 1 : 0);
}

static int sl_by_pos(const void* a, const void* b) {
  const sl_entry* x = (const sl_entry*)a;
  const sl_entry* y = (const sl_entry*)b;
  return x->pos < y->pos ? -1 : (x->pos > y->pos ? 1 : 0);
}

int64_t oracle_stochastic_length(int64_t B, const int64_t* seq_offsets, int64_t max_len,
                                 double alpha, const double* u, const uint32_t* keys,
                                 int64_t* new_offsets, int64_t* index) {
  const double lf = pow((double)max_len, alpha / 2.0);   /* N_c^(alpha/2) */
  const int64_t L = (int64_t)floor(lf);
  int64_t r = 0;
  new_offsets[0] = 0;
  for (int64_t s = 0; s < B; s++) {
    const int64_t a = seq_offsets[s], n = seq_offsets[s + 1] - seq_offsets[s];
    const int sub = (double)n > lf && u[s] >= (lf * lf) / ((double)n * (double)n);
    if (!sub) {
      for (int64_t i = 0; i < n; i++) index[r++] = a + i;
    } else {
      sl_entry* e = (sl_entry*)malloc((size_t)n * sizeof(sl_entry));
      for (int64_t i = 0; i < n; i++) {
        e[i].key = keys[a + i];
        e[i].pos = i;
      }
      qsort(e, (size_t)n, sizeof(sl_entry), sl_by_key);   /* the L smallest come first */
      qsort(e, (size_t)L, sizeof(sl_entry), sl_by_pos);   /* back to sequence order */
      for (int64_t k = 0; k < L; k++) index[r++] = a + e[k].pos;
      free(e);
    }
    new_offsets[s + 1] = r;
  }
  return r;
}

/* ---------------------------------------------------------------------------------------------
 * Eq. 3, first half: G = LayerNorm(AV) * U.  Norm is a layer normalisation; the sketch normalises
 * the full d-wide row.  Mean and biased variance over the H*dv columns.
 * --------------------------------------------------------------------------------------------- */
static void ln_gate_row(int32_t w, const double* av, const double* u, const double* ln_w,
                        const double* ln_b, double eps, double* g) {
  double mean = 0.0;
  for (int32_t c = 0; c < w; c++) mean += av[c];
  mean /= (double)w;
  double var = 0.0;
  for (int32_t c = 0; c < w; c++) var += (av[c] - mean) * (av[c] - mean);
  var /= (double)w;
  const double rstd = 1.0 / sqrt(var + eps);
  for (int32_t c = 0; c < w; c++) g[c] = ((av[c] - mean) * rstd * ln_w[c] + ln_b[c]) * u[c];
}

void oracle_ln_gate(int64_t T, int32_t H, int32_t dqk, int32_t dv, const double* av,
                    const double* uvqk, const double* ln_w, const double* ln_b, double eps,
                    double* g) {
  const int32_t n1 = 2 * H * dv + 2 * H * dqk, w = H * dv;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; t++)
    ln_gate_row(w, av + t * w, uvqk + t * n1 /* U is block 0 */, ln_w, ln_b, eps, g + t * w);
}

/* ---------------------------------------------------------------------------------------------
 * Eq. 3, second half, plus the residual connection between layers: Y = G W2 + b2 + X.
 * --------------------------------------------------------------------------------------------- */
static void f2_row(int32_t w, int32_t d, const double* g, const double* W2, const double* b2,
                   const double* x, double* y) {
  for (int32_t c = 0; c < d; c++) y[c] = b2 ? b2[c] : 0.0;
  for (int32_t k = 0; k < w; k++) {
    const double gk = g[k];
    const double* wr = W2 + (int64_t)k * d;
    for (int32_t c = 0; c < d; c++) y[c] += gk * wr[c];
  }
  for (int32_t c = 0; c < d; c++) y[c] += x[c];
}

void oracle_f2(int64_t T, int32_t w, int32_t d, const double* g, const double* W2,
               const double* b2, const double* X, double* Y) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; t++) f2_row(w, d, g + t * w, W2, b2, X + t * d, Y + t * d);
}

/* ---------------------------------------------------------------------------------------------
 * The whole layer.  Intermediates are returned when the caller passes buffers for them.
 * Returns 0, or -1 on an allocation failure.
 * --------------------------------------------------------------------------------------------- */
int oracle_layer_fwd(int64_t B, const int64_t* seq_offsets, int32_t d, int32_t H, int32_t dqk,
                     int32_t dv, const double* X, const int64_t* timestamps, const double* W1,
                     const double* b1, const double* W2, const double* b2, const double* ln_w,
                     const double* ln_b, const double* pos_table, int32_t P,
                     const double* time_table, int32_t Tb, const double* alibi_slopes,
                     double scale, double ln_eps, double* Y, double* uvqk_out, double* av_out,
                     double* g_out) {
  const int64_t T = seq_offsets[B];
  const int32_t n1 = 2 * H * dv + 2 * H * dqk, w = H * dv;
  double* uvqk = uvqk_out ? uvqk_out : (double*)malloc(sizeof(double) * (size_t)(T * n1 + 1));
  double* av = av_out ? av_out : (double*)malloc(sizeof(double) * (size_t)(T * w + 1));
  double* g = g_out ? g_out : (double*)malloc(sizeof(double) * (size_t)(T * w + 1));
  if (!uvqk || !av || !g) return -1;
  oracle_f1(T, d, n1, X, W1, b1, uvqk);
  oracle_attention(B, seq_offsets, H, dqk, dv, uvqk, timestamps, pos_table, P, time_table, Tb,
                   alibi_slopes, scale, av);
  oracle_ln_gate(T, H, dqk, dv, av, uvqk, ln_w, ln_b, ln_eps, g);
  oracle_f2(T, w, d, g, W2, b2, X, Y);
  if (!uvqk_out) free(uvqk);
  if (!av_out) free(av);
  if (!g_out) free(g);
  return 0;
}

/* ---------------------------------------------------------------------------------------------
 * The layer on a sample of output rows (global token indices `rows[0..n_rows)`).  By causality,
 * output row i of sequence s needs U and Q of row i and V and K of rows 0..i of s only, so each
 * sampled row is evaluated exactly as oracle_layer_fwd would, computing just what it reads.
 * Y_rows is [n_rows, d]; av_rows (nullable) is [n_rows, H*dv].
 * --------------------------------------------------------------------------------------------- */
int oracle_layer_rows(int64_t B, const int64_t* seq_offsets, int32_t d, int32_t H, int32_t dqk,
                      int32_t dv, const double* X, const int64_t* timestamps, const double* W1,
                      const double* b1, const double* W2, const double* b2, const double* ln_w,
                      const double* ln_b, const double* pos_table, int32_t P,
                      const double* time_table, int32_t Tb, const double* alibi_slopes,
                      double scale, double ln_eps, const int64_t* rows, int64_t n_rows,
                      double* Y_rows, double* av_rows) {
  const int32_t n1 = 2 * H * dv + 2 * H * dqk, w = H * dv;
  const int32_t offV = H * dv, offQ = 2 * H * dv, offK = 2 * H * dv + H * dqk;
  for (int64_t s = 0; s < B; s++) {
    const int64_t start = seq_offsets[s], n = seq_offsets[s + 1] - start;
    int64_t last = -1; /* the largest sampled local index in this sequence */
    for (int64_t r = 0; r < n_rows; r++)
      if (rows[r] >= start && rows[r] < start + n && rows[r] - start > last) last = rows[r] - start;
    if (last < 0) continue;
    /* the sequence's rows 0..last: V and K for all of them, U and Q only where sampled */
    double* uvqk = (double*)calloc((size_t)((last + 1) * n1), sizeof(double));
    if (!uvqk) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j <= last; j++) {
      f1_row_cols(d, n1, X + (start + j) * d, W1, b1, offV, offQ, uvqk + j * n1); /* V */
      f1_row_cols(d, n1, X + (start + j) * d, W1, b1, offK, n1, uvqk + j * n1);   /* K */
    }
    for (int64_t r = 0; r < n_rows; r++) {
      if (rows[r] < start || rows[r] >= start + n) continue;
      const int64_t i = rows[r] - start;
      double* ui = (double*)malloc(sizeof(double) * (size_t)n1);
      double* avr = (double*)malloc(sizeof(double) * (size_t)w);
      double* g = (double*)malloc(sizeof(double) * (size_t)w);
      if (!ui || !avr || !g) return -1;
      f1_row_cols(d, n1, X + (start + i) * d, W1, b1, 0, offV, ui);                 /* U */
      f1_row_cols(d, n1, X + (start + i) * d, W1, b1, offQ, offK, uvqk + i * n1);   /* Q */
      attention_row(i, H, dqk, dv, n1, uvqk, timestamps ? timestamps + start : NULL, pos_table,
                    P, time_table, Tb, alibi_slopes, scale, avr);
      ln_gate_row(w, avr, ui, ln_w, ln_b, ln_eps, g);
      f2_row(w, d, g, W2, b2, X + (start + i) * d, Y_rows + r * d);
      if (av_rows) memcpy(av_rows + r * w, avr, sizeof(double) * (size_t)w);
      free(ui);
      free(avr);
      free(g);
    }
    free(uvqk);
  }
  return 0;
}

/* ---------------------------------------------------------------------------------------------
 * Action-oriented token assembly (GenRank, "item-action organisation"): the token at each
 * position is the sum of its item embedding and its action embedding, stored as bf16.
 * --------------------------------------------------------------------------------------------- */

/* Round to the nearest bf16 value (8 significant bits, ties to even), by definition: scale to an
 * integer number of bf16 quanta and round half to even with rint() (default rounding mode). */
double oracle_round_bf16(double x) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  frexp(x, &e);               /* x = m * 2^e, 0.5 <= |m| < 1 */
  int q = e - 8;              /* quantum 2^(e-8) keeps 8 significant bits */
  if (q < -133) q = -133;     /* subnormal range: fixed quantum 2^-133 */
  return ldexp(rint(ldexp(x, -q)), q);
}

void oracle_token_embed(int64_t T, int32_t d, const int64_t* item_ids, const int64_t* action_ids,
                        const double* item_table, const double* action_table, double* X) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; t++)
    for (int32_t c = 0; c < d; c++)
      X[t * d + c] = oracle_round_bf16(item_table[item_ids[t] * d + c] +
                                       action_table[action_ids[t] * d + c]);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
