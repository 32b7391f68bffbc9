/*
 * L³ oracle: a plain, slow, fp64 CPU restatement of the Large Lookup Layer
 * forward pass and of the batch sort that groups tokens by ID.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's
 * CPU-baseline / reference leg load this file's library. The CUDA library
 * shares no code with it and never calls it.
 *
 * Sources ("L³: Large Lookup Layers", Tseng & De Sa, as summarised on the
 * kimjy99.github.io review and the papernotes.org note):
 *   - Method, eq. L³:  L3(x, t) = W_mix [ LayerNorm(W_up (V_t^T Softmax(K_t x))) ; x ]
 *     (kimjy99 review, Method; papernotes 整体框架).
 *   - K_t / V_t are d_t-row slices of the concatenated tables W_K [v x d_in] and
 *     W_V [v x d_emb] (kimjy99 review, §2 Efficient Training and Inference).
 *   - The batch is sorted by token ID so that the attention mask becomes
 *     block-diagonal, and the sort is undone at the end (sciencestack page,
 *     Fig. 3 caption; kimjy99 review §2).
 *
 * Readings where the pages are silent or garbled (all stated once more in the
 * repository's design notes):
 *   - W_up is d_up x d_emb (the review prints a shape that cannot multiply
 *     V_t^T p); W_mix columns 0..d_up-1 act on the LayerNorm output and
 *     columns d_up..d_up+d_in-1 on x, following the stacking order [LN ; x].
 *   - No 1/sqrt(d) scale in the softmax (none appears in any statement of
 *     the equation); no biases.
 *   - LayerNorm over d_up with biased variance, learned gamma/beta and an
 *     explicit eps.
 *   - Token IDs are 0-based; K_t = W_K[offsets[t] .. offsets[t+1]-1].
 *   - The sort is stable (equal IDs keep their original order) and groups
 *     come in ascending ID order.
 *
 * Every value is widened exactly to double before use (bf16 and fp32 both
 * embed exactly in fp64) and all arithmetic is fp64, in the order the
 * equation states it. Nothing is blocked, fused or reordered.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_F64 = 2 };
enum { ORACLE_OK = 0, ORACLE_BAD_ARG = 1, ORACLE_TOKEN_RANGE = 2, ORACLE_BAD_OFFSETS = 3,
       ORACLE_OOM = 4 };

/* element i of a tensor stored as fp32, bf16 (raw uint16 bits) or fp64 */
static double elem(const void *p, int dtype, int64_t i) {
  if (dtype == ORACLE_F32) return (double)((const float *)p)[i];
  if (dtype == ORACLE_F64) return ((const double *)p)[i];
  uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

int l3_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Forward pass for the tokens listed in sel[0..n_sel-1] (indices into the
 * batch); y_out is [n_sel x d_out] fp64. Each token is computed on its own:
 * the layer mixes channels only and never mixes tokens (papernotes, 整体框架).
 */
int l3_oracle_forward(int64_t n_sel, const int64_t *sel, int64_t n_tokens,
                      const int32_t *ids, const int32_t *offsets, int64_t vocab,
                      int64_t d_in, int64_t d_emb, int64_t d_up, int64_t d_out, int dtype,
                      const void *x, const void *W_K, const void *W_V, const void *W_up,
                      const void *ln_gamma, const void *ln_beta, const void *W_mix,
                      double eps, double *y_out, int n_threads) {
  if (n_sel < 0 || d_in <= 0 || d_emb <= 0 || d_up <= 0 || d_out <= 0) return ORACLE_BAD_ARG;
  int status = ORACLE_OK;
#ifdef _OPENMP
  if (n_threads <= 0) n_threads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
#endif
  for (int64_t q = 0; q < n_sel; ++q) {
    int64_t n = sel[q];
    double *y = y_out + q * d_out;
    if (n < 0 || n >= n_tokens || ids[n] < 0 || ids[n] >= vocab) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      status = ORACLE_TOKEN_RANGE;
      continue;
    }
    int32_t t = ids[n];
    int64_t off = offsets[t];
    int64_t d = (int64_t)offsets[t + 1] - off;
    if (d < 1) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      status = ORACLE_BAD_OFFSETS;
      continue;
    }
    double *s = malloc(sizeof(double) * d);
    double *a = malloc(sizeof(double) * d_emb);
    double *z = malloc(sizeof(double) * d_up);
    double *h = malloc(sizeof(double) * d_up);
    if (!s || !a || !z || !h) {
      free(s); free(a); free(z); free(h);
#ifdef _OPENMP
#pragma omp atomic write
#endif
      status = ORACLE_OOM;
      continue;
    }

    /* logits s = K_t x */
    for (int64_t j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int64_t i = 0; i < d_in; ++i)
        acc += elem(W_K, dtype, (off + j) * d_in + i) * elem(x, dtype, n * d_in + i);
      s[j] = acc;
    }
    /* p = softmax(s); subtracting the max is exact algebra */
    double mx = s[0];
    for (int64_t j = 1; j < d; ++j) mx = s[j] > mx ? s[j] : mx;
    double sum = 0.0;
    for (int64_t j = 0; j < d; ++j) {
      s[j] = exp(s[j] - mx);
      sum += s[j];
    }
    for (int64_t j = 0; j < d; ++j) s[j] /= sum;
    /* a = V_t^T p */
    for (int64_t e = 0; e < d_emb; ++e) {
      double acc = 0.0;
      for (int64_t j = 0; j < d; ++j) acc += s[j] * elem(W_V, dtype, (off + j) * d_emb + e);
      a[e] = acc;
    }
    /* z = W_up a */
    for (int64_t u = 0; u < d_up; ++u) {
      double acc = 0.0;
      for (int64_t e = 0; e < d_emb; ++e) acc += elem(W_up, dtype, u * d_emb + e) * a[e];
      z[u] = acc;
    }
    /* h = LayerNorm(z): mean, biased variance, gamma, beta */
    double mu = 0.0;
    for (int64_t u = 0; u < d_up; ++u) mu += z[u];
    mu /= (double)d_up;
    double var = 0.0;
    for (int64_t u = 0; u < d_up; ++u) var += (z[u] - mu) * (z[u] - mu);
    var /= (double)d_up;
    double rstd = 1.0 / sqrt(var + eps);
    for (int64_t u = 0; u < d_up; ++u)
      h[u] = elem(ln_gamma, dtype, u) * ((z[u] - mu) * rstd) + elem(ln_beta, dtype, u);
    /* y = W_mix [h ; x] */
    int64_t ld = d_up + d_in;
    for (int64_t o = 0; o < d_out; ++o) {
      double acc = 0.0;
      for (int64_t u = 0; u < d_up; ++u) acc += elem(W_mix, dtype, o * ld + u) * h[u];
      for (int64_t i = 0; i < d_in; ++i)
        acc += elem(W_mix, dtype, o * ld + d_up + i) * elem(x, dtype, n * d_in + i);
      y[o] = acc;
    }
    free(s); free(a); free(z); free(h);
  }
  return status;
}

/*
 * Stable counting sort of the batch by token ID, and the groups it forms
 * (sciencestack page, Fig. 3: sorting makes the mask block-diagonal).
 *   perm[i]            original index of the token at sorted position i
 *   inv_perm[n]        sorted position of original token n
 *   sorted_ids[i]      ids[perm[i]]
 *   group_ids[g]       g-th distinct ID present, ascending
 *   group_tok_start[g] first sorted position of group g; [G] = N
 *   seg_rows[g]        sum of d_t over groups before g; [G] = total rows
 * Array capacities: N for the per-token arrays, N + 1 for the group arrays.
 */
int l3_oracle_plan(const int32_t *ids, int64_t n_tokens, const int32_t *offsets, int64_t vocab,
                   int32_t *perm, int32_t *inv_perm, int32_t *sorted_ids, int32_t *group_ids,
                   int32_t *group_tok_start, int32_t *seg_rows, int64_t *G_out) {
  if (n_tokens < 0 || vocab <= 0) return ORACLE_BAD_ARG;
  for (int64_t n = 0; n < n_tokens; ++n)
    if (ids[n] < 0 || ids[n] >= vocab) return ORACLE_TOKEN_RANGE;
  int64_t *count = calloc((size_t)vocab, sizeof(int64_t));
  int64_t *next = malloc(sizeof(int64_t) * (size_t)vocab);
  if (!count || !next) {
    free(count); free(next);
    return ORACLE_OOM;
  }
  for (int64_t n = 0; n < n_tokens; ++n) count[ids[n]] += 1;
  int64_t run = 0;
  for (int64_t t = 0; t < vocab; ++t) {
    next[t] = run;
    run += count[t];
  }
  /* visiting tokens in original order keeps equal IDs in original order */
  for (int64_t n = 0; n < n_tokens; ++n) {
    int64_t pos = next[ids[n]]++;
    perm[pos] = (int32_t)n;
    sorted_ids[pos] = ids[n];
    inv_perm[n] = (int32_t)pos;
  }
  int64_t g = 0, start = 0, rows = 0;
  seg_rows[0] = 0;
  for (int64_t t = 0; t < vocab; ++t) {
    if (count[t] == 0) continue;
    group_ids[g] = (int32_t)t;
    group_tok_start[g] = (int32_t)start;
    start += count[t];
    rows += (int64_t)offsets[t + 1] - offsets[t];
    seg_rows[g + 1] = (int32_t)rows;
    ++g;
  }
  group_tok_start[g] = (int32_t)n_tokens;
  *G_out = g;
  free(count);
  free(next);
  return ORACLE_OK;
}
