/*
 * ksa_oracle.c -- plain fp64 CPU oracle for block top-k sparse decode
 * attention and LessIsMore unified selection.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke entry and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.  Every routine follows the plain definition of its step, with no
 * blocking, fusion or reordering beyond it, so that a reader can check it
 * against the sources by eye:
 *
 *  - Kinetics: Rethinking Test-Time Scaling Laws (press summary,
 *    news.43u.com.cn), section 5 "from theory to practice: block top-k":
 *    split the history into blocks, represent each block by its mean, keep the
 *    K' most relevant blocks, attend over those blocks only.
 *  - LessIsMore (press summary, techwalker.com), section 2 "unified head
 *    selection" and "stable recency window" and section 5 "selection layer":
 *    every head picks its top tokens, the picks are pooled by vote count, and
 *    the shared set is 75% voted tokens plus 25% most recent tokens.
 *
 * Readings taken where the sources are silent (each also listed in the design
 * notes):
 *  (R1) block relevance = dot product of the query with the block mean key;
 *  (R2) one selection per kv-head, scored with the sum of its G query heads;
 *  (R3) a partial tail block is averaged over its valid tokens only;
 *  (R4) seq_lens counts every cached token, the current one included;
 *  (R5) ties go to the lower index; selections are returned ascending;
 *  (R6) if k covers every block (or the budget covers every token) all are
 *       selected;
 *  (R7) softmax scale defaults to 1/sqrt(D);
 *  (R8) LessIsMore voted tokens are drawn from outside the recency window, so
 *       voted + window is exactly the budget;
 *  (R9) per-head selection ranks raw q.k (softmax is monotone per head);
 *  (R10) bf16 block summaries are a storage format of the block mean: each
 *        mean is replaced by the nearest bf16 value (ties to even) and the
 *        scores read the stored values;
 *  (R11) random-head aggregation: the random head of each row is an input
 *        drawn by the caller, and that head's own top-k set serves every head;
 *  (R12) attention recall of a selection is the share of the dense softmax
 *        weight (over every cached token) that falls on the selected tokens;
 *  (R13) fp8 block summaries are a storage format of the block mean: each
 *        block's D means are scaled by 2^-e, e the smallest exponent with
 *        max |mean| <= 448 2^e, rounded to the nearest e4m3 value (ties to
 *        even) and scaled back; the scores read the stored values.
 *
 * Inputs: bf16 values arrive as their 16-bit patterns and are widened to fp64
 * exactly.  All arrays are dense row-major.  Threads: OpenMP over independent
 * (batch, head) rows only; the arithmetic of a row is sequential.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- helpers ------------------------------------------------------------ */

/* A bf16 value is the top half of an IEEE binary32; widening is exact. */
static double bf16_to_f64(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static int num_blocks(int len, int bs) { return (len + bs - 1) / bs; }

void ksa_oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int ksa_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---- (A1) block summaries ----------------------------------------------- */
/*
 * Kinetics section 5: each block of bs cached keys is represented by its mean.
 * S[b,g,j,:] = (1/n_j) * sum_{t = j*bs}^{j*bs + n_j - 1} K[b,g,t,:],
 * n_j = min(bs, L_b - j*bs), for j < ceil(L_b/bs)  (reading R3).
 * Entries with j >= ceil(L_b/bs) are written as 0 and are not part of the
 * result.
 *   K: [B, Hkv, T, D] bf16 bits;  S: [B, Hkv, ceil(T/bs), D] fp64.
 */
void ksa_oracle_block_summaries(int B, int Hkv, int T, int D, int bs,
                                const uint16_t *K, const int32_t *seq_lens,
                                double *S) {
  const int nb_max = num_blocks(T, bs);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b) {
    for (int g = 0; g < Hkv; ++g) {
      const int L = seq_lens[b];
      const int nb = num_blocks(L, bs);
      for (int j = 0; j < nb_max; ++j) {
        double *out = S + (((size_t)b * Hkv + g) * nb_max + j) * D;
        for (int d = 0; d < D; ++d) out[d] = 0.0;
        if (j >= nb) continue;
        int n = L - j * bs;
        if (n > bs) n = bs;
        for (int t = j * bs; t < j * bs + n; ++t) {
          const uint16_t *krow = K + (((size_t)b * Hkv + g) * T + t) * D;
          for (int d = 0; d < D; ++d) out[d] += bf16_to_f64(krow[d]);
        }
        for (int d = 0; d < D; ++d) out[d] /= (double)n;
      }
    }
  }
}

/*
 * Optional bf16 storage of the summaries (R10).  A bf16 number is a binary32
 * whose low 16 bits are zero: sign, 8 exponent bits, 7 stored mantissa bits.
 * In the binade [2^(e-1), 2^e) the bf16 numbers are the multiples of
 * 2^(e-8); below 2^-126 the spacing stays 2^-133 (subnormals).  The value is
 * scaled onto that grid (exact), rounded to the nearest integer with ties to
 * the even one, and scaled back; results above the largest bf16 become
 * infinity.  Returns the 16-bit pattern.
 */
uint16_t ksa_oracle_round_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  const uint16_t sign = signbit(x) ? 0x8000 : 0;
  const double a = fabs(x);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7F80);
  int e;
  frexp(a, &e); /* a = f * 2^e with 0.5 <= f < 1 */
  int q = e - 8;
  if (q < -133) q = -133;
  const double m = ldexp(a, -q); /* a in units of the grid spacing, exact */
  double r = floor(m);
  const double frac = m - r;
  if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
  const double v = ldexp(r, q);
  if (v > 3.3895313892515355e38) return (uint16_t)(sign | 0x7F80); /* above the largest bf16 */
  const float f = (float)v; /* exact: v has at most 9 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(sign | (uint16_t)(u >> 16));
}

/* ---- (R13) fp8 e4m3 block summaries ----------------------------------------
 * e4m3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  Normal values
 * (1 + m/8) 2^(E-7) for E = 1..15 except E = 15, m = 7 (not a number), so the
 * largest is 1.75 * 2^8 = 448; subnormal values (m/8) 2^-6.  Every finite
 * value is therefore a multiple of its binade's spacing 2^(E-10) (2^-9 below
 * 2^-6).  Rounding: to the nearest value, ties to the even mantissa; a
 * magnitude above 448 is held at 448.  Returns the rounded value. */
double ksa_oracle_round_e4m3(double x) {
  if (isnan(x)) return x;
  const double a = fabs(x);
  if (a == 0.0) return x;
  int e;
  frexp(a, &e); /* a = f 2^e, 0.5 <= f < 1: binade [2^(e-1), 2^e) */
  int q = e - 4; /* spacing 2^(e-1-3) */
  if (q < -9) q = -9; /* subnormals share the spacing of the lowest binade */
  const double m = ldexp(a, -q); /* a in units of the spacing, exact */
  double r = floor(m);
  const double frac = m - r;
  if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
  double v = ldexp(r, q);
  if (v > 448.0) v = 448.0;
  return signbit(x) ? -v : v;
}

/* The block's scale exponent: the smallest e with max_d |mean_d| <= 448 2^e
 * (0 when the block mean is all zeros).  The stored block is the values
 * round_e4m3(mean_d 2^-e) with the scale 2^e. */
int ksa_oracle_e4m3_scale_exp(double amax) {
  if (!(amax > 0.0)) return 0;
  int e = (int)ceil(log2(amax / 448.0)) - 1;
  while (amax > ldexp(448.0, e)) ++e; /* settle e exactly against 448 2^e */
  while (e > -200 && amax <= ldexp(448.0, e - 1)) --e;
  return e;
}

/* Stored form of D-dim block means, in place: each block of D values becomes
 * round_e4m3(v 2^-e) 2^e with its own e. */
void ksa_oracle_store_fp8_blocks(size_t n_blocks, int D, double *S) {
  for (size_t j = 0; j < n_blocks; ++j) {
    double *m = S + j * (size_t)D;
    double amax = 0.0;
    for (int d = 0; d < D; ++d)
      if (fabs(m[d]) > amax) amax = fabs(m[d]);
    const int e = ksa_oracle_e4m3_scale_exp(amax);
    for (int d = 0; d < D; ++d) m[d] = ldexp(ksa_oracle_round_e4m3(ldexp(m[d], -e)), e);
  }
}

void ksa_oracle_round_bf16_array(size_t n, const double *in, uint16_t *out) {
  for (size_t i = 0; i < n; ++i) out[i] = ksa_oracle_round_bf16(in[i]);
}

/*
 * Paged KV cache (Kinetics section 5 integrates block top-k with paging: a
 * page holds one block).  Pages are [num_pages, Hkv, bs, D]; block_table
 * [B, max_blocks] names the page of logical block j of row b.  The logical
 * cache [B, Hkv, T = max_blocks*bs, D] is, for every t < L_b,
 *   K[b, g, t, :] = pages[block_table[b, t/bs], g, t % bs, :];
 * slots t >= L_b, and blocks whose page id is outside [0, num_pages), are
 * written as zero bits.  Every computation on a paged cache is the same
 * computation on this gathered cache.
 */
void ksa_oracle_gather_pages(int B, int Hkv, int D, int bs, int max_blocks, int num_pages,
                             const uint16_t *pages, const int32_t *block_table,
                             const int32_t *seq_lens, uint16_t *K) {
  const int T = max_blocks * bs;
  memset(K, 0, sizeof(uint16_t) * (size_t)B * Hkv * T * D);
  for (int b = 0; b < B; ++b) {
    int L = seq_lens[b];
    if (L > T) L = T;
    for (int t = 0; t < L; ++t) {
      const int page = block_table[(size_t)b * max_blocks + t / bs];
      if (page < 0 || page >= num_pages) continue;
      for (int g = 0; g < Hkv; ++g) {
        const uint16_t *src = pages + (((size_t)page * Hkv + g) * bs + t % bs) * D;
        memcpy(K + (((size_t)b * Hkv + g) * T + t) * D, src, sizeof(uint16_t) * (size_t)D);
      }
    }
  }
}

/* ---- (A2) block scores -------------------------------------------------- */
/*
 * Kinetics section 5: score every block against the query (R1, R2):
 * s[b,g,j] = sum_{h in group g} sum_d q[b,h,d] * S[b,g,j,d]  for j < NB_b,
 * group g = query heads [g*G, (g+1)*G), G = Hq/Hkv.  The softmax scale is a
 * positive constant and does not change the ranking, so it is left out.
 * Entries with j >= NB_b are written as -INFINITY.
 *   q: [B, Hq, D] bf16 bits;  S: [B, Hkv, nb_max, D];  s: [B, Hkv, nb_max].
 */
void ksa_oracle_block_scores(int B, int Hq, int Hkv, int D, int nb_max, int bs,
                             const uint16_t *q, const double *S,
                             const int32_t *seq_lens, double *scores) {
  const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b) {
    for (int g = 0; g < Hkv; ++g) {
      const int nb = num_blocks(seq_lens[b], bs);
      for (int j = 0; j < nb_max; ++j) {
        double s = -INFINITY;
        if (j < nb) {
          const double *srow = S + (((size_t)b * Hkv + g) * nb_max + j) * D;
          s = 0.0;
          for (int h = g * G; h < (g + 1) * G; ++h) {
            const uint16_t *qrow = q + ((size_t)b * Hq + h) * D;
            for (int d = 0; d < D; ++d) s += bf16_to_f64(qrow[d]) * srow[d];
          }
        }
        scores[((size_t)b * Hkv + g) * nb_max + j] = s;
      }
    }
  }
}

/* ---- (A3) top-k --------------------------------------------------------- */
/*
 * Kinetics section 5: keep the K' highest-scoring candidates.  Plain
 * definition: take the arg-max k times, each time among the candidates not
 * yet taken; among equal scores the lower index wins (R5).  The winners are
 * then listed in ascending index order.  If k >= n every candidate is taken
 * (R6).  Returns the number taken, min(k, n).
 */
static int cmp_int32(const void *a, const void *b) {
  int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
  return (x > y) - (x < y);
}

int ksa_oracle_topk(int n, const double *s, int k, int32_t *out) {
  int m = k < n ? k : n;
  if (m <= 0) return 0;
  char *taken = (char *)calloc((size_t)n, 1);
  for (int r = 0; r < m; ++r) {
    int best = -1;
    for (int j = 0; j < n; ++j) {
      if (taken[j]) continue;
      if (best < 0 || s[j] > s[best]) best = j; /* strict '>' keeps lower j */
    }
    taken[best] = 1;
    out[r] = best;
  }
  free(taken);
  qsort(out, (size_t)m, sizeof(int32_t), cmp_int32);
  return m;
}

/*
 * (A1 -> A2 -> A3) composed: block ids per (b, g), ascending, -1 padded.
 * summary_fmt: 0 exact means; 1 stored as bf16 (R10); 2 stored as fp8 e4m3
 * with a power-of-two scale per block (R13), before scoring.
 *   block_idx: [B, Hkv, k];  num_sel: [B, Hkv];
 *   scores_out (nullable): [B, Hkv, ceil(T/bs)].
 */
void ksa_oracle_select_blocks_ex(int B, int Hq, int Hkv, int D, int T, int bs,
                                 const uint16_t *q, const uint16_t *K,
                                 const int32_t *seq_lens, int k, int summary_fmt,
                                 int32_t *block_idx, int32_t *num_sel,
                                 double *scores_out) {
  const int nb_max = num_blocks(T, bs);
  const size_t n_sum = (size_t)B * Hkv * nb_max * D;
  double *S = (double *)malloc(sizeof(double) * n_sum);
  double *s = scores_out ? scores_out
                         : (double *)malloc(sizeof(double) * (size_t)B * Hkv * nb_max);
  ksa_oracle_block_summaries(B, Hkv, T, D, bs, K, seq_lens, S);
  if (summary_fmt == 1) {
    for (size_t i = 0; i < n_sum; ++i) S[i] = bf16_to_f64(ksa_oracle_round_bf16(S[i]));
  } else if (summary_fmt == 2) {
    ksa_oracle_store_fp8_blocks(n_sum / (size_t)D, D, S);
  }
  ksa_oracle_block_scores(B, Hq, Hkv, D, nb_max, bs, q, S, seq_lens, s);
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b) {
    for (int g = 0; g < Hkv; ++g) {
      int32_t *row = block_idx + ((size_t)b * Hkv + g) * k;
      for (int i = 0; i < k; ++i) row[i] = -1;
      const int nb = num_blocks(seq_lens[b], bs);
      num_sel[b * Hkv + g] =
          ksa_oracle_topk(nb, s + ((size_t)b * Hkv + g) * nb_max, k, row);
    }
  }
  free(S);
  if (!scores_out) free(s);
}

void ksa_oracle_select_blocks(int B, int Hq, int Hkv, int D, int T, int bs,
                              const uint16_t *q, const uint16_t *K,
                              const int32_t *seq_lens, int k,
                              int32_t *block_idx, int32_t *num_sel,
                              double *scores_out) {
  ksa_oracle_select_blocks_ex(B, Hq, Hkv, D, T, bs, q, K, seq_lens, k, 0, block_idx,
                              num_sel, scores_out);
}

/*
 * Kinetics section 5 compares block top-k with local attention, a fixed
 * pattern that attends only to the nearest tokens.  As a block selection:
 * every (b, g) keeps its last min(k, NB_b) blocks, NB_b - min(k, NB_b) ..
 * NB_b - 1, ascending and -1 padded.
 */
void ksa_oracle_select_window(int B, int Hkv, int bs, const int32_t *seq_lens, int k,
                              int32_t *block_idx, int32_t *num_sel) {
  for (int b = 0; b < B; ++b) {
    const int nb = num_blocks(seq_lens[b], bs);
    const int n = k < nb ? k : nb;
    for (int g = 0; g < Hkv; ++g) {
      int32_t *row = block_idx + ((size_t)b * Hkv + g) * k;
      for (int i = 0; i < k; ++i) row[i] = i < n ? nb - n + i : -1;
      num_sel[b * Hkv + g] = n;
    }
  }
}

/* ---- (A4/A5/A7/A8) attention over a selected token set ------------------ */
/*
 * Kinetics section 5 and LessIsMore section 5 "sparse attention layer":
 * ordinary softmax attention restricted to the selected tokens.
 * For query head h of row b (kv-head g = h / G) and token set T_sel:
 *   z_t = scale * sum_d q[b,h,d] * K[b,g,t,d]
 *   w_t = exp(z_t - max z) / sum_u exp(z_u - max z)
 *   out[b,h,:] = sum_t w_t * V[b,g,t,:],   lse[b,h] = max z + log sum exp(z - max z)
 * T_sel: idx == NULL means every t < L_b (dense).  Otherwise entry e of the
 * list (e < num_idx) names tokens [idx*tpi, idx*tpi + tpi), of which only
 * 0 <= t < L_b are kept (R4); negative entries are skipped.  The list is
 * [B, Hkv, cap] (shared == 0) or [B, cap] shared by all kv-heads (shared == 1).
 * An empty token set gives out = 0 and lse = -INFINITY.
 * wsum (nullable) receives sum_t w_t, which must be 1.
 */
void ksa_oracle_attention(int B, int Hq, int Hkv, int D, int T,
                          const uint16_t *q, const uint16_t *K,
                          const uint16_t *V, const int32_t *seq_lens,
                          const int32_t *idx, const int32_t *num_idx, int cap,
                          int tpi, int shared, double scale, double *out,
                          double *lse, double *wsum) {
  const int G = Hq / Hkv;
  if (scale == 0.0) scale = 1.0 / sqrt((double)D); /* R7 */
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < Hq; ++h) {
      const int g = h / G;
      const int L = seq_lens[b];
      /* collect the token set */
      int n_tok = 0;
      int32_t *tok;
      if (!idx) {
        tok = (int32_t *)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
        for (int t = 0; t < L; ++t) tok[n_tok++] = t;
      } else {
        const int32_t *list = shared ? idx + (size_t)b * cap
                                     : idx + ((size_t)b * Hkv + g) * cap;
        const int cnt = shared ? num_idx[b] : num_idx[b * Hkv + g];
        tok = (int32_t *)malloc(sizeof(int32_t) * (size_t)(cnt * tpi + 1));
        for (int e = 0; e < cnt; ++e) {
          if (list[e] < 0) continue;
          for (int u = 0; u < tpi; ++u) {
            long t = (long)list[e] * tpi + u;
            if (t < L) tok[n_tok++] = (int32_t)t;
          }
        }
      }
      const uint16_t *qrow = q + ((size_t)b * Hq + h) * D;
      double *o = out + ((size_t)b * Hq + h) * D;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      if (n_tok == 0) {
        if (lse) lse[b * Hq + h] = -INFINITY;
        if (wsum) wsum[b * Hq + h] = 0.0;
        free(tok);
        continue;
      }
      double *z = (double *)malloc(sizeof(double) * (size_t)n_tok);
      double zmax = -INFINITY;
      for (int i = 0; i < n_tok; ++i) {
        const uint16_t *krow = K + (((size_t)b * Hkv + g) * T + tok[i]) * D;
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += bf16_to_f64(qrow[d]) * bf16_to_f64(krow[d]);
        z[i] = scale * acc;
        if (z[i] > zmax) zmax = z[i];
      }
      double denom = 0.0;
      for (int i = 0; i < n_tok; ++i) denom += exp(z[i] - zmax);
      double ws = 0.0;
      for (int i = 0; i < n_tok; ++i) {
        const double w = exp(z[i] - zmax) / denom;
        ws += w;
        const uint16_t *vrow = V + (((size_t)b * Hkv + g) * T + tok[i]) * D;
        for (int d = 0; d < D; ++d) o[d] += w * bf16_to_f64(vrow[d]);
      }
      if (lse) lse[b * Hq + h] = zmax + log(denom);
      if (wsum) wsum[b * Hq + h] = ws;
      free(z);
      free(tok);
    }
  }
}

/* ---- (A6) LessIsMore unified selection ---------------------------------- */
/*
 * LessIsMore section 2 (unified head selection, stable recency window) and
 * section 5 (token selection layer), for one row b with L = seq_lens[b]:
 *  1. every query head h scores every token t < L with s_h[t] = q_h . K[g(h),t]
 *     (R9) and picks its top P tokens, ties to the lower t (R5);
 *  2. votes[t] = number of heads whose pick contains t;
 *  3. the recency window is W = [L - R, L);
 *  4. the voted part is the top (budget - R) tokens of [0, L - R) by votes,
 *     ties to the lower t (R8);
 *  5. the result is voted part + W, ascending; count = budget.
 * If L <= budget every token [0, L) is selected (R6).
 *   token_idx: [B, budget] ascending, -1 padded;  num_sel: [B];
 *   votes_out (nullable): [B, T], tokens t >= L get 0.
 */
typedef struct {
  double key; /* sort descending on key */
  int32_t t;  /* then ascending on t */
} ranked_t;

/* ---- (f4) attention recall ----------------------------------------------
 * LessIsMore, section 3 (accuracy and efficiency) and section 4 (mechanism
 * analysis) rate a token selection by attention recall: how much of a query
 * head's full softmax attention falls on the selected tokens.  Written as the
 * definition: the dense weights w_t = exp(z_t - max z) / sum_u exp(z_u - max z)
 * over every t < L_b, z_t = scale * <q_h, K_t>, then the sum of w_t over the
 * distinct selected tokens t < L_b.  Layouts of the selection as for
 * attention; shared = 2 means one list per query head [B, Hq, cap].
 * recall: [B, Hq]. */
void ksa_oracle_attention_recall(int B, int Hq, int Hkv, int D, int T,
                                 const uint16_t *q, const uint16_t *K,
                                 const int32_t *seq_lens, const int32_t *idx,
                                 const int32_t *num_idx, int cap, int tpi,
                                 int shared, double scale, double *recall) {
  const int G = Hq / Hkv;
  if (scale == 0.0) scale = 1.0 / sqrt((double)D); /* R7 */
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < Hq; ++h) {
      const int g = h / G;
      const int L = seq_lens[b];
      double *r = recall + (size_t)b * Hq + h;
      if (L <= 0) {
        *r = 0.0;
        continue;
      }
      /* the dense softmax over every cached token */
      double *w = (double *)malloc(sizeof(double) * (size_t)L);
      const uint16_t *qrow = q + ((size_t)b * Hq + h) * D;
      double zmax = -INFINITY;
      for (int t = 0; t < L; ++t) {
        const uint16_t *krow = K + (((size_t)b * Hkv + g) * T + t) * D;
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += bf16_to_f64(qrow[d]) * bf16_to_f64(krow[d]);
        w[t] = scale * acc;
        if (w[t] > zmax) zmax = w[t];
      }
      double denom = 0.0;
      for (int t = 0; t < L; ++t) {
        w[t] = exp(w[t] - zmax);
        denom += w[t];
      }
      /* the selected tokens, each counted once */
      char *sel = (char *)calloc((size_t)L, 1);
      const int32_t *list;
      int cnt;
      if (shared == 1) {
        list = idx + (size_t)b * cap;
        cnt = num_idx[b];
      } else if (shared == 2) {
        list = idx + ((size_t)b * Hq + h) * cap;
        cnt = num_idx[b * Hq + h];
      } else {
        list = idx + ((size_t)b * Hkv + g) * cap;
        cnt = num_idx[b * Hkv + g];
      }
      for (int e = 0; e < cnt; ++e) {
        if (list[e] < 0) continue;
        for (int u = 0; u < tpi; ++u) {
          const long t = (long)list[e] * tpi + u;
          if (t < L) sel[t] = 1;
        }
      }
      double mass = 0.0;
      for (int t = 0; t < L; ++t)
        if (sel[t]) mass += w[t] / denom;
      *r = mass;
      free(sel);
      free(w);
    }
  }
}

static int cmp_ranked(const void *a, const void *b) {
  const ranked_t *x = (const ranked_t *)a, *y = (const ranked_t *)b;
  if (x->key > y->key) return -1;
  if (x->key < y->key) return 1;
  return (x->t > y->t) - (x->t < y->t);
}

/*
 * Kinetics section 5's ideal token-level sparse attention: every query head h
 * keeps its own k highest-scoring tokens, s_t = sum_d q[b,h,d] * K[b,g,t,d]
 * over t < L_b (g = h / G), ties to the lower t (the same full stable ranking
 * as the LessIsMore per-head picks), listed ascending and -1 padded.  If
 * k >= L_b every token is kept.
 *   token_idx: [B, Hq, k];  num_sel: [B, Hq].
 */
void ksa_oracle_select_tokens_per_head(int B, int Hq, int Hkv, int D, int T,
                                       const uint16_t *q, const uint16_t *K,
                                       const int32_t *seq_lens, int k, int32_t *token_idx,
                                       int32_t *num_sel) {
  const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < Hq; ++h) {
      const int L = seq_lens[b];
      const int g = h / G;
      int32_t *row = token_idx + ((size_t)b * Hq + h) * k;
      for (int i = 0; i < k; ++i) row[i] = -1;
      ranked_t *r = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)(L > 0 ? L : 1));
      const uint16_t *qrow = q + ((size_t)b * Hq + h) * D;
      for (int t = 0; t < L; ++t) {
        const uint16_t *krow = K + (((size_t)b * Hkv + g) * T + t) * D;
        double sc = 0.0;
        for (int d = 0; d < D; ++d) sc += bf16_to_f64(qrow[d]) * bf16_to_f64(krow[d]);
        r[t].key = sc;
        r[t].t = t;
      }
      qsort(r, (size_t)L, sizeof(ranked_t), cmp_ranked);
      const int n = k < L ? k : L;
      for (int i = 0; i < n; ++i) row[i] = r[i].t;
      qsort(row, (size_t)n, sizeof(int32_t), cmp_int32);
      num_sel[(size_t)b * Hq + h] = n;
      free(r);
    }
  }
}

/*
 * LessIsMore section 4 (mechanism analysis) compares three ways of turning
 * the heads' choices into the set the sparse layers read: one randomly chosen
 * head's selection used for every head, a set kept per head (above), and the
 * unified vote (below).  Random-head aggregation (R11): row b takes query head
 * head_of_row[b]'s own top-k tokens, ranked as above, as the set shared by all
 * heads.
 *   head_of_row: [B], each in [0, Hq);  token_idx: [B, k];  num_sel: [B].
 */
void ksa_oracle_select_tokens_one_head(int B, int Hq, int Hkv, int D, int T,
                                       const uint16_t *q, const uint16_t *K,
                                       const int32_t *seq_lens, const int32_t *head_of_row,
                                       int k, int32_t *token_idx, int32_t *num_sel) {
  int32_t *all = (int32_t *)malloc(sizeof(int32_t) * (size_t)B * Hq * k);
  int32_t *cnt = (int32_t *)malloc(sizeof(int32_t) * (size_t)B * Hq);
  ksa_oracle_select_tokens_per_head(B, Hq, Hkv, D, T, q, K, seq_lens, k, all, cnt);
  for (int b = 0; b < B; ++b) {
    const int h = head_of_row[b];
    memcpy(token_idx + (size_t)b * k, all + ((size_t)b * Hq + h) * k, sizeof(int32_t) * (size_t)k);
    num_sel[b] = cnt[(size_t)b * Hq + h];
  }
  free(all);
  free(cnt);
}

void ksa_oracle_unified_select(int B, int Hq, int Hkv, int D, int T,
                               const uint16_t *q, const uint16_t *K,
                               const int32_t *seq_lens, int P, int budget,
                               int R, int32_t *token_idx, int32_t *num_sel,
                               int32_t *votes_out) {
  const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic)
  for (int b = 0; b < B; ++b) {
    const int L = seq_lens[b];
    int32_t *row = token_idx + (size_t)b * budget;
    for (int i = 0; i < budget; ++i) row[i] = -1;
    int32_t *votes = (int32_t *)calloc((size_t)(T > 0 ? T : 1), sizeof(int32_t));
    ranked_t *r = (ranked_t *)malloc(sizeof(ranked_t) * (size_t)(L > 0 ? L : 1));
    /* steps 1-2: per-head picks and votes (computed for every L so that the
       vote table can be inspected even when everything is selected) */
    const int p = P < L ? P : L;
    for (int h = 0; h < Hq; ++h) {
      const int g = h / G;
      const uint16_t *qrow = q + ((size_t)b * Hq + h) * D;
      for (int t = 0; t < L; ++t) {
        const uint16_t *krow = K + (((size_t)b * Hkv + g) * T + t) * D;
        double s = 0.0;
        for (int d = 0; d < D; ++d) s += bf16_to_f64(qrow[d]) * bf16_to_f64(krow[d]);
        r[t].key = s;
        r[t].t = t;
      }
      qsort(r, (size_t)L, sizeof(ranked_t), cmp_ranked);
      for (int i = 0; i < p; ++i) votes[r[i].t] += 1;
    }
    if (L <= budget) {
      for (int t = 0; t < L; ++t) row[t] = t;
      num_sel[b] = L;
    } else {
      /* steps 3-5 */
      const int n_cand = L - R;
      const int n_vote = budget - R;
      for (int t = 0; t < n_cand; ++t) {
        r[t].key = (double)votes[t];
        r[t].t = t;
      }
      qsort(r, (size_t)n_cand, sizeof(ranked_t), cmp_ranked);
      int32_t *pick = (int32_t *)malloc(sizeof(int32_t) * (size_t)(budget > 0 ? budget : 1));
      int n = 0;
      for (int i = 0; i < n_vote; ++i) pick[n++] = r[i].t;
      for (int t = L - R; t < L; ++t) pick[n++] = t;
      qsort(pick, (size_t)n, sizeof(int32_t), cmp_int32);
      memcpy(row, pick, sizeof(int32_t) * (size_t)n);
      num_sel[b] = n;
      free(pick);
    }
    if (votes_out) memcpy(votes_out + (size_t)b * T, votes, sizeof(int32_t) * (size_t)T);
    free(r);
    free(votes);
  }
}
