/*
 * fmms_oracle.c -- CPU oracle for the fused matmul-sample (FMMS) step of
 * "FlashSampling: Fast and Memory-Efficient Exact Sampling" (Ruiz et al.,
 * arXiv:2603.15854).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant generator with the CUDA path; the two meet only in
 * the seeded synthetic inputs.
 *
 * What it computes is the plain definition of the method, with the noise held
 * fixed (abstract: logits, plus Gumbel noise, then an argmax; "exact because
 * argmax decomposes over a partition"):
 *
 *   l[b,v] = sum_k h[b,k] * W[v,k]            fp64 from bf16 inputs (the bf16
 *                                             products are exact in fp64)
 *   x[b,v] = l[b,v] / T                        temperature (readus.org page,
 *                                             "API" section: temperature is an
 *                                             argument of the sampling call)
 *   s[b,v] = x[b,v] + g(r[b,v])  if v allowed, else -inf
 *                                             (readus.org page, "Top-K and
 *                                             masking": forbidden tokens are
 *                                             set to -inf before the noise)
 *   out[b] = smallest v with s[b,v] = max_v s[b,v], or -1 if none is allowed
 *
 * g(r) is the Gumbel transform of a 32-bit Philox word r:
 *   u = (r + 1) / (2^32 + 1)                   (readus.org page, "floating
 *   g = -log(-log(u))                           point precision" section)
 * evaluated in fp64 so that u never rounds to 0 or 1.
 *
 * The noise word r for (seed, step, row b, vocab index v) is word (v & 3) of
 * Philox4x32-10 with key = (seed lo32, seed hi32) and counter
 * (v >> 2, b, step, tag), tag 0 for token noise and 1 for group noise.  The
 * pages only say "Triton's Philox, keyed on a master seed and the thread's
 * grid coordinates" (readus.org page, "seed management"); keying on the
 * vocab index instead of a grid coordinate makes the noise a pure function
 * of (seed, step, row, token), so any tiling of the vocabulary sees the same
 * noise.  Philox4x32-10 itself follows Salmon, Moraes, Dror and Shaw,
 * "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11).
 *
 * Grouped sampling (Group-Gumbel-Max; readus.org page, "Group Gumbel Max"
 * section; abstract: "grouped variants ... are exact by hierarchical
 * factorization of the categorical distribution"):
 *   group g covers v in [floor(g V / G), floor((g+1) V / G))
 *   lse_g = log sum_{v in g, allowed} exp(x[b,v])        (the group "captain")
 *   i_g   = argmax_{v in g} s[b,v]
 *   g*    = argmax_g (lse_g + gumbel(word (g & 3) of Philox(key, (g>>2, b, step, 1))))
 *   out   = i_{g*}
 *
 * Parallelism: OpenMP over independent vocab entries or steps only; every
 * argmax scan runs sequentially in index order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon et al., SC'11).                                     */
/* ------------------------------------------------------------------------ */

/* Round multipliers and Weyl key increments of Philox4x32 as published. */
#define ORACLE_PHILOX_MUL_A 0xD2511F53u
#define ORACLE_PHILOX_MUL_B 0xCD9E8D57u
#define ORACLE_PHILOX_WEYL_A 0x9E3779B9u
#define ORACLE_PHILOX_WEYL_B 0xBB67AE85u

void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2],
                          uint32_t out[4]) {
  uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) { /* key schedule: bump between rounds */
      k0 += ORACLE_PHILOX_WEYL_A;
      k1 += ORACLE_PHILOX_WEYL_B;
    }
    /* S-box: two 32x32->64 multiplies, high halves mixed with the other
       counter words and the round key, low halves passed through. */
    uint64_t pa = (uint64_t)ORACLE_PHILOX_MUL_A * (uint64_t)x0;
    uint64_t pb = (uint64_t)ORACLE_PHILOX_MUL_B * (uint64_t)x2;
    uint32_t y0 = (uint32_t)(pb >> 32) ^ x1 ^ k0;
    uint32_t y1 = (uint32_t)pb;
    uint32_t y2 = (uint32_t)(pa >> 32) ^ x3 ^ k1;
    uint32_t y3 = (uint32_t)pa;
    x0 = y0; x1 = y1; x2 = y2; x3 = y3;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

void oracle_philox_batch(const uint32_t *ctrs, const uint32_t *keys,
                         uint32_t *outs, int64_t n) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    oracle_philox4x32_10(ctrs + 4 * i, keys + 2 * i, outs + 4 * i);
}

/* A 64-bit digest of the Philox words of the n consecutive counters
 * (c0 + i mod 2^32, c1, c2, c3), i = 0..n-1, under the key of `seed`:
 * the sum over i and j of word j of counter i times (4 i + j + 1), mod 2^64.
 * It lets a test compare two Philox implementations on billions of counters
 * without storing their words: for n <= 2^28 every weight is below 2^30, so
 * any single differing word changes the digest. */
uint64_t oracle_philox_digest(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                              uint64_t seed, int64_t n) {
  const uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};
  uint64_t total = 0;
#pragma omp parallel for schedule(static) reduction(+ : total)
  for (int64_t i = 0; i < n; ++i) {
    const uint32_t ctr[4] = {c0 + (uint32_t)i, c1, c2, c3};
    uint32_t out[4];
    oracle_philox4x32_10(ctr, key, out);
    for (int j = 0; j < 4; ++j) total += (uint64_t)out[j] * (uint64_t)(4 * i + j + 1);
  }
  return total;
}

/* The 32-bit noise word for (seed, step, row, index, tag). */
uint32_t oracle_noise_word(uint64_t seed, uint32_t step, uint32_t row,
                           uint32_t index, uint32_t tag) {
  uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};
  uint32_t ctr[4] = {index >> 2, row, step, tag};
  uint32_t out[4];
  oracle_philox4x32_10(ctr, key, out);
  return out[index & 3u];
}

/* ------------------------------------------------------------------------ */
/* Gumbel transform.                                                         */
/* ------------------------------------------------------------------------ */

/* g(r) = -log(-log u), u = (r + 1) / (2^32 + 1), in fp64.
 * For r >= 2^31 (u >= 1/2) the inner log is taken as log1p(-(1 - u)) with
 * 1 - u = (2^32 - r) / (2^32 + 1), so that the upper tail, where the argmax
 * lives, keeps full relative precision. */
double oracle_gumbel_from_u32(uint32_t r) {
  const double two32 = 4294967296.0;
  const double denom = 4294967297.0; /* 2^32 + 1 */
  double t; /* t = -log(u) > 0 */
  if (r >= 0x80000000u) {
    double one_minus_u = (two32 - (double)r) / denom;
    t = -log1p(-one_minus_u);
  } else {
    double u = ((double)r + 1.0) / denom;
    t = -log(u);
  }
  return -log(t);
}

void oracle_gumbel_batch(const uint32_t *r, double *g, int64_t n) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) g[i] = oracle_gumbel_from_u32(r[i]);
}

/* ------------------------------------------------------------------------ */
/* Logits.                                                                   */
/* ------------------------------------------------------------------------ */

static double bf16_to_double(uint16_t bits) {
  uint32_t w = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

/* l[v] = sum_k h[k] W[v,k] for one hidden row h, in fp64. */
static void logits_row(const uint16_t *h, const uint16_t *W, int d, int V,
                       double *l) {
#pragma omp parallel for schedule(static)
  for (int v = 0; v < V; ++v) {
    const uint16_t *w = W + (int64_t)v * d;
    double acc = 0.0;
    for (int k = 0; k < d; ++k) acc += bf16_to_double(h[k]) * bf16_to_double(w[k]);
    l[v] = acc;
  }
}

/* Logits of the listed rows: out[i*V + v] = l[rows[i], v]. */
void oracle_logits(const uint16_t *H, const uint16_t *W, int B, int d, int V,
                   const int32_t *rows, int nrows, double *out) {
  (void)B;
  for (int i = 0; i < nrows; ++i)
    logits_row(H + (int64_t)rows[i] * d, W, d, V, out + (int64_t)i * V);
}

/* ------------------------------------------------------------------------ */
/* Perturbed scores and flat sampling.                                       */
/* ------------------------------------------------------------------------ */

static int token_allowed(const uint32_t *mask, int V, int b, int v) {
  if (!mask) return 1;
  int words = (V + 31) / 32;
  return (int)((mask[(int64_t)b * words + (v >> 5)] >> (v & 31)) & 1u);
}

static uint64_t row_key(uint64_t seed, const uint64_t *row_seeds, int b) {
  return row_seeds ? row_seeds[b] : seed;
}

/* s[v] for row b given its logits l[v], with token noise of counter tag
 * `tag` (0 for the first sample of a row; sample k of a multi-sample call
 * uses 2k, keeping odd tags for group noise). */
static void scores_from_logits_tag(const double *l, int V, double T,
                                   uint64_t key, uint32_t step, int b,
                                   uint32_t tag, const uint32_t *mask,
                                   double *s) {
#pragma omp parallel for schedule(static)
  for (int v = 0; v < V; ++v) {
    if (!token_allowed(mask, V, b, v)) {
      s[v] = -INFINITY;
    } else {
      uint32_t r = oracle_noise_word(key, step, (uint32_t)b, (uint32_t)v, tag);
      s[v] = l[v] / T + oracle_gumbel_from_u32(r);
    }
  }
}

static void scores_from_logits(const double *l, int V, double T, uint64_t key,
                               uint32_t step, int b, const uint32_t *mask,
                               double *s) {
  scores_from_logits_tag(l, V, T, key, step, b, 0u, mask, s);
}

/* Perturbed scores of the listed rows: out[i*V + v] = s[rows[i], v]. */
void oracle_scores(const uint16_t *H, const uint16_t *W, int B, int d, int V,
                   double T, uint64_t seed, const uint64_t *row_seeds,
                   uint32_t step, const uint32_t *mask, const int32_t *rows,
                   int nrows, double *out) {
  (void)B;
  double *l = (double *)malloc(sizeof(double) * (size_t)V);
  for (int i = 0; i < nrows; ++i) {
    int b = rows[i];
    logits_row(H + (int64_t)b * d, W, d, V, l);
    scores_from_logits(l, V, T, row_key(seed, row_seeds, b), step, b, mask,
                       out + (int64_t)i * V);
  }
  free(l);
}

/* Sequential argmax in index order; ties go to the smallest index.  Also
 * reports the best and second-best score (the parity tolerance is stated on
 * their gap).  Returns -1 when every score is -inf. */
static int argmax_scan(const double *s, int lo, int hi, double *best,
                       double *second) {
  int arg = -1;
  double b1 = -INFINITY, b2 = -INFINITY;
  for (int v = lo; v < hi; ++v) {
    if (s[v] == -INFINITY) continue;
    if (arg < 0 || s[v] > b1) {
      b2 = b1;
      b1 = s[v];
      arg = v;
    } else if (s[v] > b2) {
      b2 = s[v];
    }
  }
  if (best) *best = b1;
  if (second) *second = b2;
  return arg;
}

/* Test entry point: the samplers' argmax scan over s[0, n), with its
 * best and second-best score (NULL pointers allowed). */
int oracle_argmax(const double *s, int n, double *best, double *second) {
  return argmax_scan(s, 0, n, best, second);
}

/* Flat FMMS sampling of the listed rows.
 * out_idx[i]   = sampled token of row rows[i] (or -1)
 * out_best[i]  = its perturbed score, out_second[i] = runner-up score. */
void oracle_sample(const uint16_t *H, const uint16_t *W, int B, int d, int V,
                   double T, uint64_t seed, const uint64_t *row_seeds,
                   uint32_t step, const uint32_t *mask, const int32_t *rows,
                   int nrows, int32_t *out_idx, double *out_best,
                   double *out_second) {
  (void)B;
  double *l = (double *)malloc(sizeof(double) * (size_t)V);
  double *s = (double *)malloc(sizeof(double) * (size_t)V);
  for (int i = 0; i < nrows; ++i) {
    int b = rows[i];
    logits_row(H + (int64_t)b * d, W, d, V, l);
    scores_from_logits(l, V, T, row_key(seed, row_seeds, b), step, b, mask, s);
    double b1, b2;
    out_idx[i] = argmax_scan(s, 0, V, &b1, &b2);
    if (out_best) out_best[i] = b1;
    if (out_second) out_second[i] = b2;
  }
  free(s);
  free(l);
}

/* Flat sampling of every row at each of the steps step0 .. step0+nsteps-1:
 * the same result as oracle_sample called once per step, with the logits
 * (which do not depend on the step) computed once.  out_idx[n*B + b],
 * out_best / out_second likewise.  Parallel over (step, row) pairs; each
 * pair's scores and argmax run on one thread. */
void oracle_sample_steps(const uint16_t *H, const uint16_t *W, int B, int d,
                         int V, double T, uint64_t seed,
                         const uint64_t *row_seeds, uint32_t step0,
                         int nsteps, const uint32_t *mask, int32_t *out_idx,
                         double *out_best, double *out_second) {
  double *l = (double *)malloc(sizeof(double) * (size_t)B * (size_t)V);
  for (int b = 0; b < B; ++b)
    logits_row(H + (int64_t)b * d, W, d, V, l + (int64_t)b * V);
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)V);
#pragma omp for schedule(static)
    for (int64_t i = 0; i < (int64_t)nsteps * B; ++i) {
      const int n = (int)(i / B), b = (int)(i % B);
      /* the nested parallel loop of the scores runs on this thread */
      scores_from_logits(l + (int64_t)b * V, V, T, row_key(seed, row_seeds, b),
                         step0 + (uint32_t)n, b, mask, s);
      double b1, b2;
      out_idx[i] = argmax_scan(s, 0, V, &b1, &b2);
      if (out_best) out_best[i] = b1;
      if (out_second) out_second[i] = b2;
    }
    free(s);
  }
  free(l);
}

/* Several samples per row: sample k draws with token-noise tag 2k, so the
 * samples are independent draws from the same softmax and sample 0 is the
 * single-sample result.  out_idx[i*S + k], out_best / out_second likewise
 * (readus.org page, API: the number of samples is an argument of the call). */
void oracle_sample_multi(const uint16_t *H, const uint16_t *W, int B, int d,
                         int V, int S, double T, uint64_t seed,
                         const uint64_t *row_seeds, uint32_t step,
                         const uint32_t *mask, const int32_t *rows, int nrows,
                         int32_t *out_idx, double *out_best,
                         double *out_second) {
  (void)B;
  double *l = (double *)malloc(sizeof(double) * (size_t)V);
  double *s = (double *)malloc(sizeof(double) * (size_t)V);
  for (int i = 0; i < nrows; ++i) {
    int b = rows[i];
    logits_row(H + (int64_t)b * d, W, d, V, l);
    for (int k = 0; k < S; ++k) {
      scores_from_logits_tag(l, V, T, row_key(seed, row_seeds, b), step, b,
                             2u * (uint32_t)k, mask, s);
      double b1, b2;
      out_idx[(int64_t)i * S + k] = argmax_scan(s, 0, V, &b1, &b2);
      if (out_best) out_best[(int64_t)i * S + k] = b1;
      if (out_second) out_second[(int64_t)i * S + k] = b2;
    }
  }
  free(s);
  free(l);
}

/* ------------------------------------------------------------------------ */
/* Top-k sampling.                                                           */
/* ------------------------------------------------------------------------ */

/* Order of the candidate selection: larger logit first, then smaller index. */
typedef struct {
  double l;
  int v;
} oracle_lv;

static int cmp_lv_desc(const void *a, const void *b) {
  const oracle_lv *x = (const oracle_lv *)a, *y = (const oracle_lv *)b;
  if (x->l > y->l) return -1;
  if (x->l < y->l) return 1;
  return (x->v < y->v) ? -1 : (x->v > y->v);
}

/* Top-k sampling (readus.org page, "Top-K and masking": a prefilter isolates
 * the candidates, then exact Gumbel-max runs on that subset): the candidates
 * of row b are its k allowed tokens with the largest logits (ties broken
 * toward the smaller index; all allowed tokens if fewer than k), and the
 * sample is the smallest-index argmax of x + g over them, with the same noise
 * as flat sampling.  The logit l orders the candidates (T > 0 keeps the order
 * of x = l / T). */
void oracle_sample_topk(const uint16_t *H, const uint16_t *W, int B, int d,
                        int V, int K, double T, uint64_t seed,
                        const uint64_t *row_seeds, uint32_t step,
                        const uint32_t *mask, const int32_t *rows, int nrows,
                        int32_t *out_idx, double *out_best, double *out_second) {
  (void)B;
  double *l = (double *)malloc(sizeof(double) * (size_t)V);
  double *s = (double *)malloc(sizeof(double) * (size_t)V);
  oracle_lv *cand = (oracle_lv *)malloc(sizeof(oracle_lv) * (size_t)V);
  for (int i = 0; i < nrows; ++i) {
    int b = rows[i];
    logits_row(H + (int64_t)b * d, W, d, V, l);
    scores_from_logits(l, V, T, row_key(seed, row_seeds, b), step, b, mask, s);
    int n = 0;
    for (int v = 0; v < V; ++v)
      if (token_allowed(mask, V, b, v)) {
        cand[n].l = l[v];
        cand[n].v = v;
        ++n;
      }
    qsort(cand, (size_t)n, sizeof(oracle_lv), cmp_lv_desc);
    int keep = n < K ? n : K;
    int arg = -1;
    double b1 = -INFINITY, b2 = -INFINITY;
    for (int j = 0; j < keep; ++j) {
      int v = cand[j].v;
      if (arg < 0 || s[v] > b1 || (s[v] == b1 && v < arg)) {
        if (arg >= 0) b2 = b1 > b2 ? b1 : b2;
        b1 = s[v];
        arg = v;
      } else if (s[v] > b2) {
        b2 = s[v];
      }
    }
    out_idx[i] = arg;
    if (out_best) out_best[i] = b1;
    if (out_second) out_second[i] = b2;
  }
  free(cand);
  free(s);
  free(l);
}

/* ------------------------------------------------------------------------ */
/* Grouped (Group-Gumbel-Max) sampling.                                      */
/* ------------------------------------------------------------------------ */

static int group_begin(int g, int V, int G) {
  return (int)(((int64_t)g * V) / G);
}

/* lse over allowed entries of x = l / T in [lo, hi), max-shifted, fp64. */
static double group_lse(const double *l, const double *s, int lo, int hi,
                        double T) {
  double m = -INFINITY;
  for (int v = lo; v < hi; ++v)
    if (s[v] != -INFINITY && l[v] / T > m) m = l[v] / T;
  if (m == -INFINITY) return -INFINITY;
  double acc = 0.0;
  for (int v = lo; v < hi; ++v)
    if (s[v] != -INFINITY) acc += exp(l[v] / T - m);
  return m + log(acc);
}

/* Grouped sampling of the listed rows.
 * summary[(i*G + g)*3 + {0,1,2}] = (max s in g, argmax in g, lse_g)
 * out_margin[i*2 + 0] = gap between the best and second-best group key
 *                       lse_g + group noise
 * out_margin[i*2 + 1] = gap between the best and second-best s inside the
 *                       chosen group
 * (either array may be NULL). */
void oracle_sample_grouped(const uint16_t *H, const uint16_t *W, int B, int d,
                           int V, int G, double T, uint64_t seed,
                           const uint64_t *row_seeds, uint32_t step,
                           const uint32_t *mask, const int32_t *rows,
                           int nrows, int32_t *out_idx, double *summary,
                           double *out_margin) {
  (void)B;
  double *l = (double *)malloc(sizeof(double) * (size_t)V);
  double *s = (double *)malloc(sizeof(double) * (size_t)V);
  for (int i = 0; i < nrows; ++i) {
    int b = rows[i];
    uint64_t key = row_key(seed, row_seeds, b);
    logits_row(H + (int64_t)b * d, W, d, V, l);
    scores_from_logits(l, V, T, key, step, b, mask, s);
    int gstar = -1, istar = -1;
    double k1 = -INFINITY, k2 = -INFINITY, in1 = 0.0, in2 = 0.0;
    for (int g = 0; g < G; ++g) {
      int lo = group_begin(g, V, G), hi = group_begin(g + 1, V, G);
      double gb1, gb2;
      int ig = argmax_scan(s, lo, hi, &gb1, &gb2);
      double lse = group_lse(l, s, lo, hi, T);
      if (summary) {
        summary[((int64_t)i * G + g) * 3 + 0] = gb1;
        summary[((int64_t)i * G + g) * 3 + 1] = (double)ig;
        summary[((int64_t)i * G + g) * 3 + 2] = lse;
      }
      if (lse == -INFINITY) continue; /* a fully masked group is never picked */
      uint32_t r = oracle_noise_word(key, step, (uint32_t)b, (uint32_t)g, 1u);
      double kg = lse + oracle_gumbel_from_u32(r);
      if (gstar < 0 || kg > k1) {
        k2 = k1;
        k1 = kg;
        gstar = g;
        istar = ig;
        in1 = gb1;
        in2 = gb2;
      } else if (kg > k2) {
        k2 = kg;
      }
    }
    out_idx[i] = istar;
    if (out_margin) {
      out_margin[2 * i + 0] = (gstar < 0) ? INFINITY : k1 - k2;
      out_margin[2 * i + 1] = (gstar < 0) ? INFINITY : in1 - in2;
    }
  }
  free(s);
  free(l);
}

/* ------------------------------------------------------------------------ */
/* Many draws of one row (for distribution tests).                           */
/* ------------------------------------------------------------------------ */

/* Draws row b once per step in [step0, step0 + nsteps) and counts outcomes:
 * counts[v] for v in [0, V), counts[V] for "no token" (-1).  G == 0 selects
 * flat sampling, G >= 1 grouped sampling.  The logits do not depend on the
 * step, so they are computed once. */
void oracle_histogram(const uint16_t *H, const uint16_t *W, int B, int d,
                      int V, int G, double T, uint64_t seed,
                      const uint64_t *row_seeds, int b, const uint32_t *mask,
                      uint32_t step0, int64_t nsteps, int64_t *counts) {
  (void)B;
  double *l = (double *)malloc(sizeof(double) * (size_t)V);
  logits_row(H + (int64_t)b * d, W, d, V, l);
  uint64_t key = row_key(seed, row_seeds, b);
  memset(counts, 0, sizeof(int64_t) * (size_t)(V + 1));
#pragma omp parallel
  {
    int64_t *local = (int64_t *)calloc((size_t)(V + 1), sizeof(int64_t));
    double *s = (double *)malloc(sizeof(double) * (size_t)V);
#pragma omp for schedule(static)
    for (int64_t n = 0; n < nsteps; ++n) {
      uint32_t step = step0 + (uint32_t)n;
      /* the samplers' own scores (the nested parallel loop runs on this thread) */
      scores_from_logits(l, V, T, key, step, b, mask, s);
      int pick;
      if (G <= 0) {
        pick = argmax_scan(s, 0, V, NULL, NULL);
      } else {
        int gstar = -1;
        double k1 = -INFINITY;
        pick = -1;
        for (int g = 0; g < G; ++g) {
          int lo = group_begin(g, V, G), hi = group_begin(g + 1, V, G);
          double lse = group_lse(l, s, lo, hi, T);
          if (lse == -INFINITY) continue;
          uint32_t r = oracle_noise_word(key, step, (uint32_t)b, (uint32_t)g, 1u);
          double kg = lse + oracle_gumbel_from_u32(r);
          if (gstar < 0 || kg > k1) {
            k1 = kg;
            gstar = g;
            pick = argmax_scan(s, lo, hi, NULL, NULL);
          }
        }
      }
      local[pick < 0 ? V : pick] += 1;
    }
#pragma omp critical
    for (int v = 0; v <= V; ++v) counts[v] += local[v];
    free(s);
    free(local);
  }
  free(l);
}

/* Number of OpenMP threads the oracle runs with. */
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
