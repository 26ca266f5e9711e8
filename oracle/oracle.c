/*
 * oracle/oracle.c -- plain, slow, fp64 CPU oracle for streaming sparse decode
 * attention.  TEST INFRASTRUCTURE ONLY: it may be used by tests/, the smoke
 * check and the CPU-baseline leg of the benchmark, never by the library.  It
 * shares no code with the CUDA path (its only input is bf16 data in logical,
 * token-major layout, made by the seeded generator).
 *
 * Every function states the passage it follows:
 *   [ART]      "ART (Attention Run-time Termination)", sections 2.1-2.4
 *   [SQZ]      "Squeezed Attention" blog Q&A, Q1/Q2 (offline clusters,
 *              online query-centroid comparison, attention over the chosen
 *              clusters' keys only)
 *   [FLUX]     "Flux Attention", section 2 (hard per-layer routing; sparse
 *              layers keep only a minimal KV set)
 *   [PULSAR]   "Pulsar Attention", Phase 1 (64-token sink) and Phase 2
 *              (exact online-softmax merge of per-shard partials)
 *   [SPARDA]   "SparDA", technical summary section 2 (a per-layer Forecast
 *              projection, one head per GQA group, picks the next layer's
 *              KV blocks ahead of time)
 *
 * Precision: fp64 throughout; inputs are bf16 (exact in fp64).  One
 * exception, orc_forecast: its output is a bf16 query that then decides
 * integer block ids, so it is computed in the precision the method's kernel
 * fixes (fp32 fused multiply-adds in input order, one rounding to bf16), and
 * both sides take the decision from the same bits.
 * Build: gcc -O2 -fPIC -shared -fopenmp -ffp-contract=off oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the OpenMP loops below use (1 without OpenMP), and a way to change
 * them for timing the oracle on one core.  Not part of any definition. */
int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

static double bf(uint16_t h) {
  union { float f; uint32_t u; } c;
  c.u = (uint32_t)h << 16;
  return (double)c.f;
}

/* ------------------------------------------------------------------------ */
/* Plain softmax attention over an explicit key set.                        */
/*   z_i = scale * q . k_i,  lse = log sum_i exp(z_i),                      */
/*   O = sum_i exp(z_i - lse) v_i.                                          */
/* Two passes (max, then sums) exactly as the definition reads.  An empty   */
/* key set gives O = 0, lse = -inf.                                         */
/* [ART] 2.1 (the quantity a tile-streaming kernel accumulates),            */
/* [SQZ] Q2 step 3 (exact attention over the selected keys).               */
/* ------------------------------------------------------------------------ */
static void attend_one(const uint16_t* q, int d, const uint16_t* K, const uint16_t* V,
                       const int64_t* idx, int64_t m, double scale, double* O, double* lse,
                       double* z /* scratch [m] */) {
  double M = -INFINITY;
  for (int64_t i = 0; i < m; ++i) {
    const uint16_t* k = K + idx[i] * (int64_t)d;
    double s = 0.0;
    for (int j = 0; j < d; ++j) s += bf(q[j]) * bf(k[j]);
    z[i] = scale * s;
    if (z[i] > M) M = z[i];
  }
  for (int j = 0; j < d; ++j) O[j] = 0.0;
  if (m == 0) {
    *lse = -INFINITY;
    return;
  }
  double sum = 0.0;
  for (int64_t i = 0; i < m; ++i) sum += exp(z[i] - M);
  double L = M + log(sum);
  for (int64_t i = 0; i < m; ++i) {
    double w = exp(z[i] - L);
    const uint16_t* v = V + idx[i] * (int64_t)d;
    for (int j = 0; j < d; ++j) O[j] += w * bf(v[j]);
  }
  *lse = L;
}

/*
 * Attention for a batch of independent units (OpenMP over units).
 * Unit u has nq query rows q[u][r][d]; its keys/values are K[u][Lk][d],
 * V[u][Lk][d]; row r of unit u attends the key indices
 * idx[(u*nq + r)*idx_stride + 0 .. m[u*nq + r]).
 * Outputs O[u][r][d], lse[u][r].
 */
void orc_attend(int64_t n_units, int nq, int d, const uint16_t* q, const uint16_t* K,
                const uint16_t* V, int64_t Lk, const int64_t* idx, const int64_t* m,
                int64_t idx_stride, double scale, double* O, double* lse) {
#pragma omp parallel
  {
    double* z = (double*)malloc(sizeof(double) * (size_t)(idx_stride > 0 ? idx_stride : 1));
#pragma omp for schedule(dynamic, 1) collapse(2)
    for (int64_t u = 0; u < n_units; ++u) {
      for (int r = 0; r < nq; ++r) {
        int64_t row = u * nq + r;
        attend_one(q + row * d, d, K + u * Lk * d, V + u * Lk * d, idx + row * idx_stride,
                   m[row], scale, O + row * d, lse + row, z);
      }
    }
    free(z);
  }
}

/* ------------------------------------------------------------------------ */
/* ART stability test on a probe trajectory.  [ART] 2.2 and 2.3.            */
/*   d_scale(t)     = | ||x_t|| - ||x_{t-1}|| | / ||x_{t-1}||               */
/*   d_direction(t) = 1 - cos(x_t, x_{t-1})                                  */
/*   pass(t) = d_scale < tau AND d_direction < phi   (both at once, strict)  */
/*   counter = pass ? counter + 1 : 0   (p CONSECUTIVE blocks)               */
/*   stop after block t when counter >= p.                                   */
/* Zero vectors: ||x_{t-1}|| = 0 gives d_scale = 0 if ||x_t|| = 0, else inf; */
/* a zero vector in the cosine gives 0 if both are zero, else 1.             */
/* ------------------------------------------------------------------------ */
static double norm8(const double* x, int n) {
  double s = 0.0;
  for (int i = 0; i < n; ++i) s += x[i] * x[i];
  return sqrt(s);
}

void orc_art_metrics(const double* xp, const double* x, int n, double* d_scale,
                     double* d_dir) {
  double a = norm8(x, n), b = norm8(xp, n);
  if (b == 0.0) *d_scale = (a == 0.0) ? 0.0 : INFINITY;
  else *d_scale = fabs(a - b) / b;
  if (a == 0.0 || b == 0.0) *d_dir = (a == 0.0 && b == 0.0) ? 0.0 : 1.0;
  else {
    double dot = 0.0;
    for (int i = 0; i < n; ++i) dot += x[i] * xp[i];
    *d_dir = 1.0 - dot / (a * b);
  }
}

/* How far one test is from flipping, relative to its thresholds: for a pass,
 * the smaller relative distance below tau / phi; for a fail, the larger
 * relative distance above (the metric that makes it fail). */
static double test_margin(double ds, double dc, double tau, double phi) {
  double rs = (tau > 0.0) ? (ds - tau) / tau : INFINITY;
  double rc = (phi > 0.0) ? (dc - phi) / phi : INFINITY;
  int pass = (ds < tau) && (dc < phi);
  if (pass) return fmin(-rs, -rc);
  return fmax(rs, rc);
}

/* Runs the stopping rule over a given trajectory x[T][n].  Returns the number
 * of blocks consumed (stop after block t -> t + 1; never -> T).  margin gets
 * the minimum test margin over the tests performed (INFINITY if none). */
int orc_art_stop(const double* x, int T, int n, double tau, double phi, int patience,
                 double* margin) {
  int counter = 0;
  double mg = INFINITY;
  for (int t = 1; t < T; ++t) {
    double ds, dc;
    orc_art_metrics(x + (int64_t)(t - 1) * n, x + (int64_t)t * n, n, &ds, &dc);
    double r = test_margin(ds, dc, tau, phi);
    if (r < mg) mg = r;
    int pass = (ds < tau) && (dc < phi);
    counter = pass ? counter + 1 : 0;
    if (counter >= patience) {
      if (margin) *margin = mg;
      return t + 1;
    }
  }
  if (margin) *margin = mg;
  return T;
}

/* ------------------------------------------------------------------------ */
/* Sequential ART decode for one query head.  [ART] 2.1-2.4.                */
/* blocks[0..nblk) is the effective traversal (the caller puts block 0      */
/* first, [ART] 2.4 "attention sinks").  Block j covers tokens              */
/* [j*bs, min(j*bs + bs, L)).  After folding each block into the running    */
/* online-softmax state (m, l, O), the probe is x_t = (O / l)[0:n_probe].   */
/* forced > 0: consume exactly `forced` blocks, ignoring the rule.          */
/* ------------------------------------------------------------------------ */
static void art_head(const uint16_t* q, int d, const uint16_t* K, const uint16_t* V, int64_t L,
                     int bs, const int32_t* blocks, int nblk, double scale, double tau,
                     double phi, int patience, int n_probe, int forced, double* O, double* lse,
                     int32_t* consumed, double* margin, double* xs /* scratch [nblk][n_probe] */) {
  double m = -INFINITY, l = 0.0;
  for (int j = 0; j < d; ++j) O[j] = 0.0;
  int counter = 0, used = nblk;
  double mg = INFINITY;
  for (int t = 0; t < nblk; ++t) {
    int64_t j0 = (int64_t)blocks[t] * bs, j1 = j0 + bs;
    if (j1 > L) j1 = L;
    for (int64_t i = j0; i < j1; ++i) { /* online softmax, one key at a time */
      const uint16_t* k = K + i * d;
      const uint16_t* v = V + i * d;
      double s = 0.0;
      for (int j = 0; j < d; ++j) s += bf(q[j]) * bf(k[j]);
      double z = scale * s;
      double mn = z > m ? z : m;
      double a = exp(m - mn), w = exp(z - mn);
      l = a * l + w;
      for (int j = 0; j < d; ++j) O[j] = a * O[j] + w * bf(v[j]);
      m = mn;
    }
    double* x = xs + (int64_t)t * n_probe;
    for (int j = 0; j < n_probe; ++j) x[j] = (l > 0.0) ? O[j] / l : 0.0;
    if (forced > 0) {
      if (t + 1 == forced) { used = forced; break; }
      continue;
    }
    if (t >= 1) {
      double ds, dc;
      orc_art_metrics(xs + (int64_t)(t - 1) * n_probe, x, n_probe, &ds, &dc);
      double r = test_margin(ds, dc, tau, phi);
      if (r < mg) mg = r;
      counter = (ds < tau && dc < phi) ? counter + 1 : 0;
      if (counter >= patience) { used = t + 1; break; }
    }
  }
  for (int j = 0; j < d; ++j) O[j] = (l > 0.0) ? O[j] / l : 0.0;
  *lse = (l > 0.0) ? m + log(l) : -INFINITY;
  *consumed = used;
  *margin = mg;
}

/*
 * ART for a batch of KV groups (OpenMP over groups x heads).  Group u has G
 * query heads q[u][G][d], keys/values K[u][L][d], V[u][L][d] with L = Ls[u],
 * traversal blocks[u][0 .. nblk[u]) (row stride blk_stride).
 * forced: NULL, or int [n_units][G] (>0 forces that many consumed blocks).
 * Outputs O[u][G][d], lse[u][G], consumed[u][G], margin[u][G].
 */
void orc_art(int64_t n_units, int G, int d, const uint16_t* q, const uint16_t* K,
             const uint16_t* V, int64_t Lk, const int64_t* Ls, int bs, const int32_t* blocks,
             const int32_t* nblk, int64_t blk_stride, double scale, double tau, double phi,
             int patience, int n_probe, const int32_t* forced, double* O, double* lse,
             int32_t* consumed, double* margin) {
#pragma omp parallel
  {
    double* xs = (double*)malloc(sizeof(double) * (size_t)(blk_stride + 1) * (size_t)n_probe);
#pragma omp for schedule(dynamic, 1) collapse(2)
    for (int64_t u = 0; u < n_units; ++u) {
      for (int g = 0; g < G; ++g) {
        int64_t row = u * G + g;
        art_head(q + row * d, d, K + u * Lk * d, V + u * Lk * d, Ls[u], bs,
                 blocks + u * blk_stride, nblk[u], scale, tau, phi, patience, n_probe,
                 forced ? forced[row] : 0, O + row * d, lse + row, consumed + row,
                 margin + row, xs);
      }
    }
    free(xs);
  }
}

/* ------------------------------------------------------------------------ */
/* Centroid selection for one KV group.  [SQZ] Q2 step 2: compare the query */
/* with every cluster centroid and keep the best clusters.  Reading used:   */
/* score_c = (sum over the group's query heads of q_g) . c_c, keep the k    */
/* largest, ties to the lower index, ids reported in ascending order.       */
/* scores[C] receives every score (fp64).                                   */
/* ------------------------------------------------------------------------ */
typedef struct { double s; int32_t i; } scored;

static int by_score_desc(const void* a, const void* b) {
  const scored* x = (const scored*)a;
  const scored* y = (const scored*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return (x->i > y->i) - (x->i < y->i);
}
static int by_int_asc(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

void orc_select(int64_t n_units, int G, int d, const uint16_t* q /*[u][G][d]*/,
                const uint16_t* cent /*[u][C][d]*/, int C, int k, int32_t* ids /*[u][k]*/,
                double* scores /*[u][C]*/) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t u = 0; u < n_units; ++u) {
    scored* s = (scored*)malloc(sizeof(scored) * (size_t)C);
    const uint16_t* qu = q + u * G * d;
    for (int c = 0; c < C; ++c) {
      const uint16_t* cc = cent + (u * C + c) * d;
      double acc = 0.0;
      for (int j = 0; j < d; ++j) {
        double qs = 0.0;
        for (int g = 0; g < G; ++g) qs += bf(qu[g * d + j]);
        acc += qs * bf(cc[j]);
      }
      s[c].s = acc;
      s[c].i = c;
      scores[u * C + c] = acc;
    }
    qsort(s, (size_t)C, sizeof(scored), by_score_desc);
    int kk = k < C ? k : C;
    for (int i = 0; i < kk; ++i) ids[u * k + i] = s[i].i;
    qsort(ids + u * k, (size_t)kk, sizeof(int32_t), by_int_asc);
    free(s);
  }
}

/* ------------------------------------------------------------------------ */
/* Exact merge of per-shard partials.  [PULSAR] Phase 2: each shard's local */
/* attention (O_i normalised, lse_i) is combined by the online-softmax      */
/* merge into the exact global attention:                                   */
/*   M = max_i lse_i,  w_i = exp(lse_i - M),                                 */
/*   O = sum_i w_i O_i / sum_i w_i,  lse = M + log sum_i w_i.                */
/* Empty shards (lse = -inf) have weight 0; all empty -> O = 0, lse = -inf.  */
/* ------------------------------------------------------------------------ */
void orc_merge(int S, int64_t N, int d, const double* o_parts /*[S][N][d]*/,
               const double* lse_parts /*[S][N]*/, double* out /*[N][d]*/, double* lse /*[N]*/) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    double M = -INFINITY;
    for (int s = 0; s < S; ++s)
      if (lse_parts[s * N + n] > M) M = lse_parts[s * N + n];
    for (int j = 0; j < d; ++j) out[n * d + j] = 0.0;
    if (M == -INFINITY) {
      lse[n] = -INFINITY;
      continue;
    }
    double W = 0.0;
    for (int s = 0; s < S; ++s) {
      double w = exp(lse_parts[s * N + n] - M);
      W += w;
      for (int j = 0; j < d; ++j) out[n * d + j] += w * o_parts[(s * N + n) * d + j];
    }
    for (int j = 0; j < d; ++j) out[n * d + j] /= W;
    lse[n] = M + log(W);
  }
}

/* ------------------------------------------------------------------------ */
/* Forecast projection.  [SPARDA] 2: layer l's Forecast head (one per GQA   */
/* group) maps the layer's activation x to a vector whose dot products with */
/* the next layer's block summaries rank the blocks to fetch:               */
/*   f[j] = bf16( sum_i w[i][j] x[i] ),                                     */
/* the sum taken in fp32 with one fused multiply-add per term, i ascending, */
/* and rounded to bf16 to nearest, ties to even.                            */
/* ------------------------------------------------------------------------ */
static uint16_t f32_to_bf16_rne(float f) {
  union { float f; uint32_t u; } c;
  c.f = f;
  if ((c.u & 0x7F800000u) == 0x7F800000u && (c.u & 0x007FFFFFu)) return (uint16_t)((c.u >> 16) | 0x40u);
  uint32_t lsb = (c.u >> 16) & 1u;
  return (uint16_t)((c.u + 0x7FFFu + lsb) >> 16);
}

void orc_forecast(int64_t n_units, int d, const uint16_t* x /*[u][d]*/, const uint16_t* w /*[u][d][d]*/,
                  uint16_t* f /*[u][d]*/) {
#pragma omp parallel for schedule(static)
  for (int64_t u = 0; u < n_units; ++u) {
    const uint16_t* wu = w + u * d * d;
    for (int j = 0; j < d; ++j) {
      float acc = 0.0f;
      for (int i = 0; i < d; ++i) {
        union { float f; uint32_t u; } a, b;
        a.u = (uint32_t)wu[(int64_t)i * d + j] << 16;
        b.u = (uint32_t)x[u * d + i] << 16;
        acc = fmaf(a.f, b.f, acc);
      }
      f[u * d + j] = f32_to_bf16_rne(acc);
    }
  }
}
