/*
 * kvc_oracle.c -- plain, slow, float64 CPU oracle for observation-window
 * token scoring, selection and KV / hidden-state compaction.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What it follows (citations are to the pages the method is described on):
 *  - FastKV (gist.science 2502.01068), section 2.A "Token-Selective
 *    Propagation": at the TSP layer the importance of each context token is
 *    judged from the attention that a window of recent tokens pays to it, and
 *    the window tokens themselves always go forward with the selected ones.
 *  - FastKV, section 2.B "KV retention decoupled": two independent budgets
 *    (TSP rate, KV retention rate) rank the same scores.
 *  - FastKV abstract (chatpaper.ai / arXiv 2502.01068): the KV compression is
 *    GQA-aware, i.e. one retained set per KV head, shared by its query group.
 *  - StructKV (gist.science 2604.06746), section 2.A: the global in-degree
 *    centrality C_global is the sum of the per-layer attention contributions;
 *    section 2.B: per-layer attention entropy, sparsity and variance.
 * Numeric details the pages leave open are fixed as follows (plainest
 * reading): contributions are SUMMED over window rows and group heads; the
 * query head h belongs to KV head floor(h / G); the softmax of window row i
 * runs over every key at or before its own position (causal inside the
 * window); pooling is a zero-padded centred moving average over the prefix
 * (window keys excluded) divided by the kernel size; ties in the ranking go
 * to the lower position.
 *
 * Every floating-point step is float64.  bf16 inputs arrive as raw uint16
 * bit patterns and are widened exactly.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC.  Defining
 * ORACLE_MUTANT=n compiles a deliberately wrong variant; the pin tests use
 * those to show that each plausible mistake is caught.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

int oracle_mutant(void) { return ORACLE_MUTANT; }

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

static double bf16_to_f64(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* KV head that query head h reads (contiguous grouping). */
static int kv_head_of(int h, int H, int Hkv) {
#if ORACLE_MUTANT == 3
  (void)H;
  return h % Hkv; /* mutant: interleaved grouping */
#else
  return h / (H / Hkv);
#endif
}

/* s = scale * <q, k> */
static double logit(const double* q, const double* k, int d, double scale) {
  double acc = 0.0;
  for (int c = 0; c < d; ++c) acc += q[c] * k[c];
#if ORACLE_MUTANT == 2
  (void)scale;
  return acc; /* mutant: scale dropped */
#else
  return scale * acc;
#endif
}

/* Last key that window row i may see: its own position N - w + i. */
static int64_t last_visible(int64_t N, int w, int i) {
#if ORACLE_MUTANT == 1
  (void)w; (void)i;
  return N - 1; /* mutant: no causal mask inside the window */
#else
  return N - w + i;
#endif
}

/*
 * Window attention aggregate of one sequence.
 *   q : [w][H][d] bf16 bits, element (i, h, c) at q[i*q_si + h*q_sh + c]
 *   k : [N][Hkv][d] bf16 bits, element (j, g, c) at k[j*k_sn + g*k_sh + c]
 *   A : [Hkv][N] float64 out, A[g*N + j] =
 *         sum over query heads h of group g, window rows i with j <= N-w+i,
 *         of softmax_j( scale * q[i,h] . k[j,g] )
 * Returns 0 on success, -1 on bad arguments.
 */
int oracle_window_scores(const uint16_t* q, int64_t q_si, int64_t q_sh,
                         const uint16_t* k, int64_t k_sn, int64_t k_sh,
                         int64_t N, int H, int Hkv, int d, int w, double scale,
                         double* A) {
  if (!q || !k || !A || H <= 0 || Hkv <= 0 || H % Hkv || d <= 0 || w < 1 || w > N)
    return -1;
  const int G = H / Hkv;
  const int R = G * w; /* rows per KV head */
  double* kd = (double*)malloc(sizeof(double) * (size_t)N * d);
  double* qd = (double*)malloc(sizeof(double) * (size_t)R * d);
  double* m = (double*)malloc(sizeof(double) * R);
  double* l = (double*)malloc(sizeof(double) * R);
  int64_t* last = (int64_t*)malloc(sizeof(int64_t) * R);
  if (!kd || !qd || !m || !l || !last) {
    free(kd); free(qd); free(m); free(l); free(last);
    return -1;
  }
  for (int g = 0; g < Hkv; ++g) {
    /* widen this KV head's keys and its group's window queries */
    for (int64_t j = 0; j < N; ++j)
      for (int c = 0; c < d; ++c) kd[j * d + c] = bf16_to_f64(k[j * k_sn + (int64_t)g * k_sh + c]);
    int r = 0;
    for (int h = 0; h < H; ++h) {
      if (kv_head_of(h, H, Hkv) != g) continue;
      for (int i = 0; i < w; ++i, ++r) {
        for (int c = 0; c < d; ++c) qd[r * d + c] = bf16_to_f64(q[i * q_si + (int64_t)h * q_sh + c]);
        last[r] = last_visible(N, w, i);
      }
    }
    /* softmax normaliser of every row: max and sum of exp over visible keys */
#pragma omp parallel
    {
      double* s = (double*)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
      for (int rr = 0; rr < R; ++rr) {
        double mx = -INFINITY;
        for (int64_t j = 0; j <= last[rr]; ++j) {
          s[j] = logit(qd + rr * d, kd + j * d, d, scale);
          if (s[j] > mx) mx = s[j];
        }
        double sum = 0.0;
        for (int64_t j = 0; j <= last[rr]; ++j) sum += exp(s[j] - mx);
        m[rr] = mx;
        l[rr] = sum;
      }
      free(s);
    }
    /* A[g, j] = sum over rows of the normalised probability of key j */
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < N; ++j) {
      double a = 0.0;
      for (int rr = 0; rr < R; ++rr) {
        if (j > last[rr]) continue;
        a += exp(logit(qd + rr * d, kd + j * d, d, scale) - m[rr]) / l[rr];
      }
      A[(int64_t)g * N + j] = a;
    }
  }
  free(kd); free(qd); free(m); free(l); free(last);
  return 0;
}

/*
 * The same aggregate with each window row's softmax normaliser given instead
 * of computed: lse[i*ls_i + h*ls_h] = ln sum_{j <= N-w+i} exp(scale * q[i,h] . k[j,g])
 * for window row i of query head h (the log-sum-exp a causal prefill
 * attention produces for that query).  By the definition of the softmax,
 *   A[g*N + j] = sum over h of group g, i with j <= N-w+i, of
 *                exp(scale * q[i,h] . k[j,g] - lse[i,h]),
 * which equals oracle_window_scores when lse is the true log-sum-exp.  FastKV
 * section 2.A: the TSP layer runs full attention over the prompt, so these
 * normalisers exist before the token scores are formed.
 */
int oracle_window_scores_lse(const uint16_t* q, int64_t q_si, int64_t q_sh,
                             const uint16_t* k, int64_t k_sn, int64_t k_sh,
                             int64_t N, int H, int Hkv, int d, int w, double scale,
                             const double* lse, int64_t ls_i, int64_t ls_h, double* A) {
  if (!q || !k || !lse || !A || H <= 0 || Hkv <= 0 || H % Hkv || d <= 0 || w < 1 || w > N)
    return -1;
  const int G = H / Hkv;
  const int R = G * w;
  double* kd = (double*)malloc(sizeof(double) * (size_t)N * d);
  double* qd = (double*)malloc(sizeof(double) * (size_t)R * d);
  double* z = (double*)malloc(sizeof(double) * R);
  int64_t* last = (int64_t*)malloc(sizeof(int64_t) * R);
  if (!kd || !qd || !z || !last) {
    free(kd); free(qd); free(z); free(last);
    return -1;
  }
  for (int g = 0; g < Hkv; ++g) {
    for (int64_t j = 0; j < N; ++j)
      for (int c = 0; c < d; ++c) kd[j * d + c] = bf16_to_f64(k[j * k_sn + (int64_t)g * k_sh + c]);
    int r = 0;
    for (int h = 0; h < H; ++h) {
      if (kv_head_of(h, H, Hkv) != g) continue;
      for (int i = 0; i < w; ++i, ++r) {
        for (int c = 0; c < d; ++c) qd[r * d + c] = bf16_to_f64(q[i * q_si + (int64_t)h * q_sh + c]);
        last[r] = last_visible(N, w, i);
        z[r] = lse[(int64_t)i * ls_i + (int64_t)h * ls_h];
      }
    }
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < N; ++j) {
      double a = 0.0;
      for (int rr = 0; rr < R; ++rr) {
        if (j > last[rr]) continue;
        a += exp(logit(qd + rr * d, kd + j * d, d, scale) - z[rr]);
      }
      A[(int64_t)g * N + j] = a;
    }
  }
  free(kd); free(qd); free(z); free(last);
  return 0;
}

/* out[j] = sum_r rows[r*stride + j], r = 0..nrows-1 (TSP aggregate, C_global). */
void oracle_sum_rows(const double* rows, int nrows, int64_t stride, int64_t n, double* out) {
  for (int64_t j = 0; j < n; ++j) {
    double s = 0.0;
    for (int r = 0; r < nrows; ++r) s += rows[(int64_t)r * stride + j];
    out[j] = s;
  }
}

/*
 * Zero-padded centred moving average with odd kernel p:
 *   y[j] = (1/p) * sum_{t=-(p/2)}^{p/2} x[j+t],  x[.] = 0 outside [0, L).
 */
int oracle_avg_pool(const double* x, int64_t L, int p, double* y) {
  if (p < 1 || (p & 1) == 0) return -1;
  const int half = p / 2;
  for (int64_t j = 0; j < L; ++j) {
    double s = 0.0;
    int cnt = 0;
    for (int t = -half; t <= half; ++t) {
      int64_t u = j + t;
      if (u < 0 || u >= L) continue;
      s += x[u];
      ++cnt;
    }
#if ORACLE_MUTANT == 4
    y[j] = s / cnt; /* mutant: divide by the in-range count */
#else
    (void)cnt;
    y[j] = s / p;
#endif
  }
  return 0;
}

typedef struct {
  double s;
  int64_t j;
} keyed_t;

/* higher score first; equal scores: lower position first */
static int by_score_then_pos(const void* a, const void* b) {
  const keyed_t* x = (const keyed_t*)a;
  const keyed_t* y = (const keyed_t*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
#if ORACLE_MUTANT == 5
  return (x->j < y->j) ? 1 : (x->j > y->j) ? -1 : 0; /* mutant: higher position wins ties */
#else
  return (x->j < y->j) ? -1 : (x->j > y->j) ? 1 : 0;
#endif
}

static int cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/*
 * Top-k that always keeps the window.
 *   S   : ranking scores of the prefix positions 0..N-w-1 (already pooled)
 *   k   : budget INCLUDING the w window positions, k >= w
 *   idx : out, min(k, N) positions in ascending order: the k-w best prefix
 *         positions (score descending, ties to the lower position) together
 *         with the window N-w..N-1; if k >= N every position is kept.
 * Returns the number of indices written, or -1 on bad arguments.
 */
int64_t oracle_select_topk(const double* S, int64_t N, int w, int64_t k, int32_t* idx) {
  if (w < 1 || w > N || k < w) return -1;
  if (k >= N) {
    for (int64_t j = 0; j < N; ++j) idx[j] = (int32_t)j;
    return N;
  }
  const int64_t L = N - w;
  const int64_t kk = k - w;
  keyed_t* v = (keyed_t*)malloc(sizeof(keyed_t) * (size_t)(L > 0 ? L : 1));
  if (!v) return -1;
  for (int64_t j = 0; j < L; ++j) {
    v[j].s = S[j];
    v[j].j = j;
  }
  qsort(v, (size_t)L, sizeof(keyed_t), by_score_then_pos);
  int64_t n = 0;
  for (int64_t t = 0; t < kk; ++t) idx[n++] = (int32_t)v[t].j;
#if ORACLE_MUTANT == 6
  for (int t = 0; t < w - 1; ++t) idx[n++] = (int32_t)(L + t); /* mutant: last window token dropped */
  idx[n++] = (int32_t)v[kk].j;
#else
  for (int t = 0; t < w; ++t) idx[n++] = (int32_t)(L + t);
#endif
  qsort(idx, (size_t)n, sizeof(int32_t), cmp_i32);
  free(v);
  return n;
}

/*
 * Row gather (bit copy): out[r*row_elems + c] = src[idx[r]*src_stride + c];
 * idx[r] == -1 marks a padding row and writes zeros.  Returns the number of
 * indices outside [-1, nsrc) (those rows are written as zeros too).
 */
int64_t oracle_gather_rows(const uint16_t* src, int64_t src_stride, int64_t nsrc, int64_t row_elems,
                           const int32_t* idx, int64_t n, uint16_t* out) {
  int64_t bad = 0;
  for (int64_t r = 0; r < n; ++r) {
    int64_t j = idx[r];
    uint16_t* o = out + r * row_elems;
    if (j < 0 || j >= nsrc) {
      if (j != -1) ++bad;
      memset(o, 0, sizeof(uint16_t) * (size_t)row_elems);
      continue;
    }
    memcpy(o, src + j * src_stride, sizeof(uint16_t) * (size_t)row_elems);
  }
  return bad;
}

static int cmp_desc_f64(const void* a, const void* b) {
  double x = *(const double*)a, y = *(const double*)b;
  return (x < y) - (x > y);
}

/*
 * Per-row attention statistics on a_hat = A / mass_norm (mass_norm = w*G, the
 * exact total mass of one KV head's aggregate):
 *   out[0] entropy        -sum a ln a   (0 ln 0 = 0), nats
 *   out[1] top-1% mass     sum of the ceil(N/100) largest a
 *   out[2] variance        (1/N) sum (a - mean)^2
 */
int oracle_layer_stats(const double* A, int64_t N, double mass_norm, double* out) {
  if (N < 1 || !(mass_norm > 0)) return -1;
  double* a = (double*)malloc(sizeof(double) * (size_t)N);
  if (!a) return -1;
  double ent = 0.0, sum = 0.0;
  for (int64_t j = 0; j < N; ++j) {
    a[j] = A[j] / mass_norm;
    if (a[j] > 0) ent -= a[j] * log(a[j]);
    sum += a[j];
  }
  const double mean = sum / (double)N;
  double var = 0.0;
  for (int64_t j = 0; j < N; ++j) var += (a[j] - mean) * (a[j] - mean);
  var /= (double)N;
  qsort(a, (size_t)N, sizeof(double), cmp_desc_f64);
  const int64_t m = (N + 99) / 100;
  double top = 0.0;
  for (int64_t t = 0; t < m; ++t) top += a[t];
  out[0] = ent;
  out[1] = top;
  out[2] = var;
  free(a);
  return 0;
}

/*
 * Dynamic pivot detection, online  [StructKV section 2.B: the per-layer
 * attention entropy, sparsity and variance are watched, and the pivot layer
 * is where the entropy falls sharply while the sparsity rises].  The page
 * fixes neither the statistic per layer nor the threshold; reading taken:
 *   E_l, S_l = mean over the layer's KV-head rows of the entropy and of the
 *              top-1% mass (the sparsity measure), from the float outputs of
 *              the layer statistics, summed in float64 in head order;
 *   the pivot is the first layer l (1-based) with l_min <= l <= l_max and
 *   l >= 2 such that (E_{l-1} - E_l) >= tau * E_{l-1} and S_l > S_{l-1};
 *   if none qualifies, l_max.  Variance is monitored but not part of the rule
 *   (the page's detection sentence names only entropy and sparsity).
 * stats: [L][Hkv][3] float, per layer and KV head (entropy, top-1% mass,
 * variance).  Returns the pivot layer, or -1 on bad arguments.
 */
int oracle_pivot_layer(const float* stats, int L, int Hkv, double tau, int l_min, int l_max) {
  if (!stats || L < 1 || Hkv < 1 || !(tau >= 0) || l_min < 1 || l_max < l_min || l_max > L) return -1;
  double E_prev = 0.0, S_prev = 0.0;
  for (int l = 1; l <= l_max; ++l) {
    double E = 0.0, S = 0.0;
    for (int g = 0; g < Hkv; ++g) {
      E += (double)stats[((size_t)(l - 1) * Hkv + g) * 3 + 0];
      S += (double)stats[((size_t)(l - 1) * Hkv + g) * 3 + 1];
    }
    E /= (double)Hkv;
    S /= (double)Hkv;
    if (l >= 2 && l >= l_min && (E_prev - E) >= tau * E_prev && S > S_prev) return l;
    E_prev = E;
    S_prev = S;
  }
  return l_max;
}

/*
 * Decode attention over the compacted cache  [FastKV 2.B: the retained
 * entries form the KV cache the decoding steps read; FastKV abstract: one
 * retained set per KV head, shared by its query group].  One new query per
 * query head, every retained entry visible (positions are already applied to
 * K before compaction):
 *   out[h][c] = sum_r softmax_r( scale * q[h] . kc[g][r] ) vc[g][r][c],  g = h / G
 * q [H][d], kc and vc [Hkv][kk][d], contiguous bf16 bits; out [H][d] float64.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_decode_attention(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, int H, int Hkv,
                            int64_t kk, int d, double scale, double* out) {
  if (!q || !kc || !vc || !out || H <= 0 || Hkv <= 0 || H % Hkv || kk < 1 || d <= 0) return -1;
  double* qd = (double*)malloc(sizeof(double) * (size_t)d);
  double* kd = (double*)malloc(sizeof(double) * (size_t)d);
  double* s = (double*)malloc(sizeof(double) * (size_t)kk);
  if (!qd || !kd || !s) {
    free(qd); free(kd); free(s);
    return -1;
  }
  for (int h = 0; h < H; ++h) {
    const int g = kv_head_of(h, H, Hkv);
    for (int c = 0; c < d; ++c) qd[c] = bf16_to_f64(q[(int64_t)h * d + c]);
    double mx = -INFINITY;
    for (int64_t r = 0; r < kk; ++r) {
      for (int c = 0; c < d; ++c) kd[c] = bf16_to_f64(kc[((int64_t)g * kk + r) * d + c]);
      s[r] = logit(qd, kd, d, scale);
      if (s[r] > mx) mx = s[r];
    }
    double z = 0.0;
    for (int64_t r = 0; r < kk; ++r) z += exp(s[r] - mx);
    for (int c = 0; c < d; ++c) out[(int64_t)h * d + c] = 0.0;
    for (int64_t r = 0; r < kk; ++r) {
      const double p = exp(s[r] - mx) / z;
      for (int c = 0; c < d; ++c) out[(int64_t)h * d + c] += p * bf16_to_f64(vc[((int64_t)g * kk + r) * d + c]);
    }
  }
  free(qd); free(kd); free(s);
  return 0;
}

/*
 * Causal prefill attention of one sequence, with each query row's
 * log-sum-exp  [FastKV (gist.science 2502.01068) section 1: every layer runs
 * full (quadratic) attention over the prompt during prefill; section 2.A: the
 * TSP layer does so over the whole prompt, which is where the window rows'
 * normalisers come from; FastKV abstract: grouped-query heads].  Query i sees
 * keys j <= i:
 *   s_ij       = scale * q[i,h] . k[j,g],   g = h / G
 *   lse[i,h]   = ln sum_{j<=i} exp(s_ij)
 *   out[i,h,:] = sum_{j<=i} exp(s_ij - lse[i,h]) v[j,g,:]
 * q [N][H][d], k and v [N][Hkv][d], contiguous bf16 bits; out [N][H][d] and
 * lse [N][H] float64.  Returns 0, or -1 on bad arguments.
 */
int oracle_prefill_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t N, int H,
                             int Hkv, int d, double scale, double* out, double* lse) {
  if (!q || !k || !v || !out || !lse || N < 1 || H <= 0 || Hkv <= 0 || H % Hkv || d <= 0) return -1;
  double* kd = (double*)malloc(sizeof(double) * (size_t)N * Hkv * d);
  double* vd = (double*)malloc(sizeof(double) * (size_t)N * Hkv * d);
  if (!kd || !vd) {
    free(kd); free(vd);
    return -1;
  }
  for (int64_t e = 0; e < N * Hkv * d; ++e) {
    kd[e] = bf16_to_f64(k[e]);
    vd[e] = bf16_to_f64(v[e]);
  }
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 4) reduction(| : bad)
  for (int64_t ih = 0; ih < N * H; ++ih) {
    const int64_t i = ih / H;
    const int h = (int)(ih % H);
    const int g = kv_head_of(h, H, Hkv);
#if ORACLE_MUTANT == 9
    const int64_t last = i - 1 < 0 ? 0 : i - 1; /* mutant: the query's own key dropped */
#else
    const int64_t last = i;
#endif
    double* qd = (double*)malloc(sizeof(double) * (size_t)d);
    double* sv = (double*)malloc(sizeof(double) * (size_t)(last + 1));
    if (!qd || !sv) {
      free(qd); free(sv);
      bad = 1;
      continue;
    }
    for (int c = 0; c < d; ++c) qd[c] = bf16_to_f64(q[ih * d + c]);
    double mx = -INFINITY;
    for (int64_t j = 0; j <= last; ++j) {
      sv[j] = logit(qd, kd + (j * Hkv + g) * d, d, scale);
      if (sv[j] > mx) mx = sv[j];
    }
    double z = 0.0;
    for (int64_t j = 0; j <= last; ++j) z += exp(sv[j] - mx);
    lse[ih] = mx + log(z);
    double* o = out + ih * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int64_t j = 0; j <= last; ++j) {
      const double pj = exp(sv[j] - mx) / z;
      const double* vr = vd + (j * Hkv + g) * d;
      for (int c = 0; c < d; ++c) o[c] += pj * vr[c];
    }
    free(qd); free(sv);
  }
  free(kd); free(vd);
  return bad ? -1 : 0;
}

/*
 * Residual vector quantisation of retained K or V rows  [VQKV (gist.science
 * 2603.16435) section 2: each cached vector is mapped to nearest codewords
 * stage by stage, the first codebook taking the main approximation and every
 * later one the residual the earlier stages left].  The codebooks are inputs
 * (random ones in the tests: trained ones need data).  Reading taken: whole
 * head rows (d values), squared Euclidean distance, ties to the lowest index:
 *   r_1 = x,  c_s = argmin_m ||r_s - C_s[m]||^2,  r_{s+1} = r_s - C_s[c_s].
 * x [n][d] bf16 bits, row stride x_stride elements; C [S][M][d] float32;
 * codes [n][S] int32 out; gap [n][S] float64 out or NULL: the second-best
 * minus the best squared distance at each stage (+inf when M == 1).
 * Returns 0, or -1 on bad arguments.
 */
int oracle_rvq_encode(const uint16_t* x, int64_t x_stride, int64_t n, int d, const float* C, int S, int M,
                      int32_t* codes, double* gap) {
  if (!x || !C || !codes || n < 0 || d <= 0 || S < 1 || M < 1 || x_stride < d) return -1;
#pragma omp parallel
  {
    double* r = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < n; ++t) {
      for (int c = 0; c < d; ++c) r[c] = bf16_to_f64(x[t * x_stride + c]);
      for (int st = 0; st < S; ++st) {
        const float* Cs = C + (size_t)st * M * d;
        double best = INFINITY, second = INFINITY;
        int arg = 0;
        for (int m = 0; m < M; ++m) {
          double dist = 0.0;
          for (int c = 0; c < d; ++c) {
            const double e = r[c] - (double)Cs[(size_t)m * d + c];
            dist += e * e;
          }
#if ORACLE_MUTANT == 8
          if (dist <= best) { /* mutant: ties to the highest index */
#else
          if (dist < best) {
#endif
            second = best;
            best = dist;
            arg = m;
          } else if (dist < second) {
            second = dist;
          }
        }
        codes[t * S + st] = arg;
        if (gap) gap[t * S + st] = second - best;
#if ORACLE_MUTANT != 7
        for (int c = 0; c < d; ++c) r[c] -= (double)Cs[(size_t)arg * d + c];
#endif /* mutant 7: every stage encodes the row itself, not the residual */
      }
    }
    free(r);
  }
  return 0;
}

