/*
 * oracle.c -- plain float64 CPU definition of grouped-query causal attention
 * with rotary position embeddings and the cross-document mask.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's
 * CPU-baseline / reference legs may load this library. It shares no code,
 * header, table or constant with the CUDA library: nothing here is used to
 * compute a product result.
 *
 * What it computes, and where the pages state it:
 *
 *  - RoPE frequencies theta_k = base^(-2k/d) for k in [0, d/2 - 1]
 *    ("Llama 3.1 Architecture: Dense Scaling to 405B and 128K Context",
 *    section "Context Expansion", subsection "High Base Frequency"), with the
 *    base 500,000 of the 8K pre-training (same subsection; "The Llama 3 Herd of
 *    Models" overview, architecture chapter). d is read as the head dimension.
 *  - The rotation itself is the RoFormer one that page cites in its
 *    references: adjacent pairs (x_2k, x_2k+1) are turned by the angle
 *    p * theta_k, where p is the token's position.
 *  - Grouped-query attention: each KV head serves a consecutive block of
 *    Hq/Hkv query heads ("How Meta's Llama 3.1 405B Architecture Actually
 *    Works", GQA paragraph; 128 query heads over 8 KV heads on the
 *    architecture page's hyper-parameter chart).
 *  - Causal decoder attention with the cross-document mask ("The Llama 3 Herd
 *    of Models", architecture chapter summary): key j is visible to query i iff
 *    both sit in the same batch row and the same document and j <= i.
 *    Positions restart at 0 at each document start.
 *  - Scores are scaled by 1/sqrt(D) and normalised with a softmax over the
 *    visible keys.
 *  - Decode: one new query per sequence, rotated at position len, attends to
 *    the len cached keys (already rotated at positions 0..len-1) and values.
 *    With len = 0 the output is defined as 0.
 *
 * Everything is float64. The softmax is taken over the full masked row:
 * every key of the batch row is visited, masked keys get -inf.
 *
 * Parity status: every exported function is pinned by the CPU tests
 * (brute force against an independent torch formulation, invariants and
 * closed forms).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* theta_k = base^(-2k/D), k = 0 .. D/2 - 1 */
void oracle_rope_freqs(int D, double base, double *freqs) {
  for (int k = 0; k < D / 2; ++k) freqs[k] = pow(base, -2.0 * (double)k / (double)D);
}

/* Rotate one D-vector x at position p into y. */
static void rope_rotate_one(const double *x, double *y, int D, double p, const double *freqs) {
  for (int k = 0; k < D / 2; ++k) {
    double angle = p * freqs[k];
    double c = cos(angle), s = sin(angle);
    double x0 = x[2 * k], x1 = x[2 * k + 1];
    y[2 * k] = x0 * c - x1 * s;
    y[2 * k + 1] = x0 * s + x1 * c;
  }
}

/* Rotate n vectors of H heads each: x is [n, H, D]; vector i is at position pos[i]. */
void oracle_rope_rotate(const double *x, int64_t n, int H, int D, const double *pos, double base,
                        double *y) {
  double *freqs = (double *)malloc(sizeof(double) * (size_t)(D / 2));
  oracle_rope_freqs(D, base, freqs);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    for (int h = 0; h < H; ++h)
      rope_rotate_one(x + (i * H + h) * D, y + (i * H + h) * D, D, pos[i], freqs);
  free(freqs);
}

/*
 * Document layout from doc_offsets (cumulative document starts in flattened
 * B*S token coordinates, ending with the sentinel B*S; NULL = one document per
 * batch row). Writes, per token t, the row-local index of its document's first
 * token and its position t - start. Returns 0, or -1 when the offsets are
 * malformed (not starting at 0, not strictly increasing, not ending at B*S, or
 * a document that crosses a batch-row boundary).
 */
int oracle_doc_layout(const int32_t *offs, int B, int S, int32_t *doc_start, int32_t *pos) {
  const int64_t total = (int64_t)B * S;
  if (offs == NULL) {
    for (int64_t t = 0; t < total; ++t) {
      doc_start[t] = 0;
      pos[t] = (int32_t)(t % S);
    }
    return 0;
  }
  if (offs[0] != 0) return -1;
  int64_t d = 0;
  while ((int64_t)offs[d] < total) {
    int64_t start = offs[d], end = offs[d + 1];
    if (end <= start || end > total) return -1;
    if (start / S != (end - 1) / S) return -1; /* straddles two batch rows */
    for (int64_t t = start; t < end; ++t) {
      doc_start[t] = (int32_t)(start % S);
      pos[t] = (int32_t)(t - start);
    }
    ++d;
  }
  return 0;
}

/* Query head h reads KV head h / (Hq / Hkv): the replicated copy of that KV head. */
static int kv_head_of(int h, int Hq, int Hkv) { return h / (Hq / Hkv); }

/*
 * Attention weights of one query row over the S keys of its batch row.
 * qrot: rotated query [D]; krot: rotated keys of the batch row [S, Hkv, D];
 * doc_start: row-local doc starts of the batch row [S]; i: the query's row index.
 * w receives S weights (masked keys get exactly 0). If lse is not NULL it
 * receives log(sum over visible j of exp(s_ij)), the log of the softmax
 * denominator of the scaled scores.
 */
static void masked_softmax_row(const double *qrot, const double *krot, const int32_t *doc_start,
                               int S, int Hkv, int g, int D, int i, double *w, double *lse) {
  const double scale = 1.0 / sqrt((double)D);
  double m = -INFINITY;
  for (int j = 0; j < S; ++j) {
    int visible = (j <= i) && (doc_start[j] == doc_start[i]);
    if (!visible) {
      w[j] = -INFINITY;
      continue;
    }
    const double *kj = krot + ((int64_t)j * Hkv + g) * D;
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += qrot[d] * kj[d];
    w[j] = dot * scale;
    if (w[j] > m) m = w[j];
  }
  double sum = 0.0;
  for (int j = 0; j < S; ++j) {
    w[j] = (w[j] == -INFINITY) ? 0.0 : exp(w[j] - m);
    sum += w[j];
  }
  for (int j = 0; j < S; ++j) w[j] /= sum;
  if (lse) *lse = m + log(sum);
}

/* Rotate every key of the batch at its token position: k [B*S, Hkv, D]. */
static double *rotate_keys(const double *k, const int32_t *pos_i, int64_t n_tok, int Hkv, int D,
                           double base) {
  double *pos = (double *)malloc(sizeof(double) * (size_t)n_tok);
  for (int64_t t = 0; t < n_tok; ++t) pos[t] = (double)pos_i[t];
  double *krot = (double *)malloc(sizeof(double) * (size_t)n_tok * Hkv * D);
  oracle_rope_rotate(k, n_tok, Hkv, D, pos, base, krot);
  free(pos);
  return krot;
}

/*
 * Prefill. k, v: [B, S, Hkv, D]. doc_start, pos: per token [B*S] (from
 * oracle_doc_layout). Query rows: rows[r] is a flattened token index b*S+i and
 * q_rows holds that token's query [n_rows, Hq, D]; rows == NULL means all B*S
 * tokens in order. out: [n_rows, Hq, D].
 */
static void prefill_impl(const double *q_rows, const double *k, const double *v,
                         const int32_t *doc_start, const int32_t *pos, int B, int S, int Hq, int Hkv,
                         int D, double base, const int64_t *rows, int64_t n_rows, double *out,
                         double *lse_out) {
  const int64_t n_tok = (int64_t)B * S;
  double *krot = rotate_keys(k, pos, n_tok, Hkv, D, base);
  double *freqs = (double *)malloc(sizeof(double) * (size_t)(D / 2));
  oracle_rope_freqs(D, base, freqs);

#pragma omp parallel
  {
    double *w = (double *)malloc(sizeof(double) * (size_t)S);
    double *qrot = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
    for (int64_t rh = 0; rh < n_rows * Hq; ++rh) {
      const int64_t r = rh / Hq;
      const int h = (int)(rh % Hq);
      const int64_t t = rows ? rows[r] : r;
      const int b = (int)(t / S), i = (int)(t % S);
      const int g = kv_head_of(h, Hq, Hkv);
      rope_rotate_one(q_rows + (r * Hq + h) * D, qrot, D, (double)pos[t], freqs);
      const double *krow = krot + (int64_t)b * S * Hkv * D;
      masked_softmax_row(qrot, krow, doc_start + (int64_t)b * S, S, Hkv, g, D, i, w,
                         lse_out ? lse_out + r * Hq + h : NULL);
      double *o = out + (r * Hq + h) * D;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      const double *vrow = v + (int64_t)b * S * Hkv * D;
      for (int j = 0; j < S; ++j) {
        if (w[j] == 0.0) continue;
        const double *vj = vrow + ((int64_t)j * Hkv + g) * D;
        for (int d = 0; d < D; ++d) o[d] += w[j] * vj[d];
      }
    }
    free(w);
    free(qrot);
  }
  free(freqs);
  free(krot);
}

void oracle_prefill(const double *q_rows, const double *k, const double *v,
                    const int32_t *doc_start, const int32_t *pos, int B, int S, int Hq, int Hkv,
                    int D, double base, const int64_t *rows, int64_t n_rows, double *out) {
  prefill_impl(q_rows, k, v, doc_start, pos, B, S, Hq, Hkv, D, base, rows, n_rows, out, NULL);
}

/*
 * Prefill that also returns, per query row and head, the log-sum-exp of its
 * visible scaled scores: lse [n_rows, Hq] (natural logarithm). This is the
 * quantity that lets partial attentions over disjoint key sets be merged.
 */
void oracle_prefill_lse(const double *q_rows, const double *k, const double *v,
                        const int32_t *doc_start, const int32_t *pos, int B, int S, int Hq, int Hkv,
                        int D, double base, const int64_t *rows, int64_t n_rows, double *out,
                        double *lse) {
  prefill_impl(q_rows, k, v, doc_start, pos, B, S, Hq, Hkv, D, base, rows, n_rows, out, lse);
}

/*
 * The attention weights of one (b, h, i) row over its S keys (for the
 * invariant tests: they must sum to 1 and vanish outside the mask).
 * q: [B, S, Hq, D]; k: [B, S, Hkv, D].
 */
void oracle_prefill_weights(const double *q, const double *k, const int32_t *doc_start,
                            const int32_t *pos, int B, int S, int Hq, int Hkv, int D, double base,
                            int b, int h, int i, double *w) {
  const int64_t n_tok = (int64_t)B * S;
  double *krot = rotate_keys(k, pos, n_tok, Hkv, D, base);
  double *freqs = (double *)malloc(sizeof(double) * (size_t)(D / 2));
  double *qrot = (double *)malloc(sizeof(double) * (size_t)D);
  oracle_rope_freqs(D, base, freqs);
  const int64_t t = (int64_t)b * S + i;
  rope_rotate_one(q + (t * Hq + h) * D, qrot, D, (double)pos[t], freqs);
  masked_softmax_row(qrot, krot + (int64_t)b * S * Hkv * D, doc_start + (int64_t)b * S, S, Hkv,
                     kv_head_of(h, Hq, Hkv), D, i, w, NULL);
  free(qrot);
  free(freqs);
  free(krot);
}

/*
 * Decode. q: [B, Hq, D] (not rotated); kc, vc: [B, Hkv, Lmax, D], the keys
 * already rotated at their cache positions; lens: [B]. The query of sequence b
 * is rotated at position lens[b] and attends to cache rows 0 .. lens[b]-1.
 * out: [B, Hq, D].
 */
void oracle_decode(const double *q, const double *kc, const double *vc, const int32_t *lens, int B,
                   int Hq, int Hkv, int D, int Lmax, double base, double *out) {
  double *freqs = (double *)malloc(sizeof(double) * (size_t)(D / 2));
  oracle_rope_freqs(D, base, freqs);
  const double scale = 1.0 / sqrt((double)D);
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
    double *qrot = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < (int64_t)B * Hq; ++bh) {
      const int b = (int)(bh / Hq), h = (int)(bh % Hq);
      const int g = kv_head_of(h, Hq, Hkv);
      const int L = lens[b];
      double *o = out + bh * D;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      if (L <= 0) continue;
      rope_rotate_one(q + bh * D, qrot, D, (double)L, freqs);
      const double *kbase = kc + ((int64_t)b * Hkv + g) * Lmax * D;
      const double *vbase = vc + ((int64_t)b * Hkv + g) * Lmax * D;
      double m = -INFINITY;
      for (int n = 0; n < L; ++n) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qrot[d] * kbase[(int64_t)n * D + d];
        s[n] = dot * scale;
        if (s[n] > m) m = s[n];
      }
      double sum = 0.0;
      for (int n = 0; n < L; ++n) {
        s[n] = exp(s[n] - m);
        sum += s[n];
      }
      for (int n = 0; n < L; ++n) {
        const double wn = s[n] / sum;
        for (int d = 0; d < D; ++d) o[d] += wn * vbase[(int64_t)n * D + d];
      }
    }
    free(s);
    free(qrot);
  }
  free(freqs);
}
