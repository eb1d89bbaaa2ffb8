/*
 * mala_oracle.c -- plain, slow CPU oracle for MALA (MassAlloc Attention).
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the package smoke check and
 * the CPU-baseline leg of the benchmark may load this library. The product
 * path never calls it, and it shares no code with the CUDA sources.
 *
 * Everything is float64 with scalar loops: one query row, one key, one
 * accumulator at a time, in the order the method states. Tiles appear only
 * because the method's decisions are made per tile (T query rows x T keys);
 * there is no blocking beyond that.
 *
 * Sources (web pages on arXiv 2609.32712, "MassAlloc Attention: Let Attention
 * Allocate Its Own Compute"):
 *  [R1] agihunt.info summary, paragraph defining MALA: a tile is skipped when
 *       its largest per-key contribution ratio is below tau/Lq, Lq = number of
 *       keys the query can see; tau dimensionless, default 1.
 *  [R2] agihunt.info summary, forward paragraph; jaehun.me review, section
 *       "Forward: online sparse softmax": ratio = exp(tile row max - running
 *       max) / retained mass; skip only if all valid rows are below; skipped
 *       tiles leave m, l, O untouched; traversal from the diagonal toward
 *       earlier keys; the first legal tile is always kept; the final
 *       log-normalizer is written for backward.
 *  [R3] agihunt.info summary, backward paragraph; jaehun.me review, section
 *       "Backward: offline sparse probabilities": the same test with the
 *       final normalizer; no stored mask; kept tiles do the standard
 *       P / dP / dS / dQ / dK / dV work.
 *  [R4] jaehun.me review, section "Theoretical upper bound on forward omitted
 *       mass" (Proposition 1, appendix A.2).
 *  [R5] agihunt.info summary, limits paragraph; gpt-diffusion blog, "Contexto":
 *       tau -> 0 recovers FullAttn in both passes; decode uses the same rule.
 *
 * Readings where the pages are silent (each is listed with the design notes):
 *  - skip iff ratio < tau/Lq for every valid row (equality keeps);
 *  - the log form: (mt - m - ln l) < ln tau - ln Lq;
 *  - Lq = r + 1 for query position r (self-attention), Lq = Lc in decode;
 *  - backward has no forced keep of the diagonal tile (flag selects it);
 *  - D_r = <dO_r, O_r> with the forward output O;
 *  - decode tiles are 128 keys aligned from position 0, visited newest first;
 *    the rows of a decode tile are the query heads sharing one KV head.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define NEG_INF (-INFINITY)

static double dot(const double *a, const double *b, int d) {
  double s = 0.0;
  for (int k = 0; k < d; ++k) s += a[k] * b[k];
  return s;
}

static int imin(int a, int b) { return a < b ? a : b; }

int mala_oracle_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

/* log of the length-normalised threshold tau / Lq ([R1]); -inf at tau = 0. */
static double log_threshold(double tau, double Lq) {
  if (tau <= 0.0) return NEG_INF;
  return log(tau) - log(Lq);
}

/*
 * Forward over query blocks [qb0, qb1) of one (batch, head) slice.
 * Q, K, V: [L][d]. O: [L][d], LSE: [L] (rows of the given blocks written).
 * keep (may be NULL): [nb][nb] bytes, entry (i, j) = 1 if tile kept, written
 *   for i in the range and j <= i.
 * margin (may be NULL): [nb][nb], max over valid rows of
 *   (mt - m - ln l) - (ln tau - ln Lq), +inf for a forced keep.
 * force_first: keep the diagonal tile unconditionally ([R2]).
 */
int mala_oracle_fwd(const double *Q, const double *K, const double *V, int L,
                    int d, int T, double scale, double tau, int force_first,
                    double *O, double *LSE, uint8_t *keep, double *margin,
                    int qb0, int qb1) {
  if (L <= 0) return 0;
  const int nb = (L + T - 1) / T;
  if (qb1 > nb) qb1 = nb;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = qb1 - 1; i >= qb0; --i) {
    const int r0 = i * T, r1 = imin(L, (i + 1) * T), R = r1 - r0;
    double *m = malloc(sizeof(double) * R);
    double *l = malloc(sizeof(double) * R);
    double *mt = malloc(sizeof(double) * R);
    double *acc = calloc((size_t)R * d, sizeof(double));
    double *s = malloc(sizeof(double) * (size_t)R * T);
    for (int r = 0; r < R; ++r) { m[r] = NEG_INF; l[r] = 0.0; }

    /* key tiles from the diagonal toward earlier keys ([R2]) */
    for (int j = i; j >= 0; --j) {
      const int c0 = j * T;
      /* scores of every legal key of the tile ([R1]: QK is never skipped) */
      for (int r = 0; r < R; ++r) {
        const int row = r0 + r;
        const int c1 = imin((j + 1) * T, row + 1);
        double mx = NEG_INF;
        for (int c = c0; c < c1; ++c) {
          double v = scale * dot(Q + (size_t)row * d, K + (size_t)c * d, d);
          s[(size_t)r * T + (c - c0)] = v;
          if (v > mx) mx = v;
        }
        mt[r] = mx;
      }
      /* online skip test ([R2], log form) */
      int kept;
      double mu = NEG_INF;
      if (j == i && force_first) {
        kept = 1;
        mu = INFINITY;
      } else if (tau <= 0.0) {
        kept = 1; /* ln tau = -inf: nothing is ever below the threshold */
        mu = INFINITY;
      } else {
        kept = 0;
        for (int r = 0; r < R; ++r) {
          const double lhs = mt[r] - m[r] - log(l[r]);
          const double crit = lhs - log_threshold(tau, (double)(r0 + r + 1));
          if (crit > mu) mu = crit;
          if (crit >= 0.0) kept = 1;
        }
      }
      if (keep) keep[(size_t)i * nb + j] = (uint8_t)kept;
      if (margin) margin[(size_t)i * nb + j] = mu;
      if (!kept) continue; /* skipped: m, l, O untouched, V not read */

      /* retained tile: standard online-softmax update ([R2]) */
      for (int r = 0; r < R; ++r) {
        const int row = r0 + r;
        const int c1 = imin((j + 1) * T, row + 1);
        const double mnew = mt[r] > m[r] ? mt[r] : m[r];
        const double alpha = (m[r] == NEG_INF) ? 0.0 : exp(m[r] - mnew);
        double *a = acc + (size_t)r * d;
        for (int k = 0; k < d; ++k) a[k] *= alpha;
        double lsum = l[r] * alpha;
        for (int c = c0; c < c1; ++c) {
          const double p = exp(s[(size_t)r * T + (c - c0)] - mnew);
          lsum += p;
          const double *vc = V + (size_t)c * d;
          for (int k = 0; k < d; ++k) a[k] += p * vc[k];
        }
        l[r] = lsum;
        m[r] = mnew;
      }
    }
    /* epilogue: O = acc / l, LSE = m + ln l ([R2]) */
    for (int r = 0; r < R; ++r) {
      const int row = r0 + r;
      for (int k = 0; k < d; ++k) O[(size_t)row * d + k] = acc[(size_t)r * d + k] / l[r];
      LSE[row] = m[r] + log(l[r]);
    }
    free(m); free(l); free(mt); free(acc); free(s);
  }
  return 0;
}

/*
 * Forward of a prefill chunk appended to a KV cache (one (batch, head)
 * slice): Lq new queries after Lk - Lq cached keys, so query row r sits at
 * position off + r (off = Lk - Lq) and its legal keys are 0 .. off + r, with
 * Lq,r = off + r + 1 in the threshold ([R1], [R3]). Query blocks are the
 * chunk's own 128-row blocks; key tiles are aligned to them: key tile k
 * covers positions off + T (k - koff) .. + T - 1, koff = ceil(off / T), so
 * query block i's diagonal tile is k = i + koff and tile 0 may start below
 * position 0 (those keys do not exist). Traversal k = i + koff down to 0
 * ([R2]); the diagonal tile is always kept.
 * Q: [Lq][d]; K, V: [Lk][d]. O: [Lq][d], LSE: [Lq].
 * keep, margin (may be NULL): [nbq][nbq + koff], entry (i, k).
 */
int mala_oracle_fwd_chunk(const double *Q, const double *K, const double *V, int Lq,
                          int Lk, int d, int T, double scale, double tau, double *O,
                          double *LSE, uint8_t *keep, double *margin) {
  if (Lq <= 0) return 0;
  const int off = Lk - Lq;
  const int nbq = (Lq + T - 1) / T, koff = (off + T - 1) / T, nkt = nbq + koff;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i = nbq - 1; i >= 0; --i) {
    const int r0 = i * T, R = imin(Lq, (i + 1) * T) - r0;
    double *m = malloc(sizeof(double) * R);
    double *l = malloc(sizeof(double) * R);
    double *mt = malloc(sizeof(double) * R);
    double *acc = calloc((size_t)R * d, sizeof(double));
    double *s = malloc(sizeof(double) * (size_t)R * T);
    for (int r = 0; r < R; ++r) { m[r] = NEG_INF; l[r] = 0.0; }
    for (int k = i + koff; k >= 0; --k) {
      const int p0 = off + T * (k - koff); /* position of the tile's first key */
      for (int r = 0; r < R; ++r) {
        const int pos = off + r0 + r;
        double mx = NEG_INF;
        for (int c = 0; c < T; ++c) {
          const int kp = p0 + c;
          double v = NEG_INF;
          if (kp >= 0 && kp <= pos) v = scale * dot(Q + (size_t)(r0 + r) * d, K + (size_t)kp * d, d);
          s[(size_t)r * T + c] = v;
          if (v > mx) mx = v;
        }
        mt[r] = mx;
      }
      int kept;
      double mu = NEG_INF;
      if (k == i + koff || tau <= 0.0) {
        kept = 1;
        mu = INFINITY;
      } else {
        kept = 0;
        for (int r = 0; r < R; ++r) {
          const double lhs = mt[r] - m[r] - log(l[r]);
          const double crit = lhs - log_threshold(tau, (double)(off + r0 + r + 1));
          if (crit > mu) mu = crit;
          if (crit >= 0.0) kept = 1;
        }
      }
      if (keep) keep[(size_t)i * nkt + k] = (uint8_t)kept;
      if (margin) margin[(size_t)i * nkt + k] = mu;
      if (!kept) continue;
      for (int r = 0; r < R; ++r) {
        if (mt[r] == NEG_INF) continue; /* no legal key of this row in the tile */
        const double mnew = mt[r] > m[r] ? mt[r] : m[r];
        const double alpha = (m[r] == NEG_INF) ? 0.0 : exp(m[r] - mnew);
        double *a = acc + (size_t)r * d;
        for (int e = 0; e < d; ++e) a[e] *= alpha;
        double lsum = l[r] * alpha;
        for (int c = 0; c < T; ++c) {
          const double sv = s[(size_t)r * T + c];
          if (sv == NEG_INF) continue;
          const double pr = exp(sv - mnew);
          lsum += pr;
          const double *vc = V + (size_t)(p0 + c) * d;
          for (int e = 0; e < d; ++e) a[e] += pr * vc[e];
        }
        l[r] = lsum;
        m[r] = mnew;
      }
    }
    for (int r = 0; r < R; ++r) {
      for (int e = 0; e < d; ++e) O[(size_t)(r0 + r) * d + e] = acc[(size_t)r * d + e] / l[r];
      LSE[r0 + r] = m[r] + log(l[r]);
    }
    free(m); free(l); free(mt); free(acc); free(s);
  }
  return 0;
}

/* Backward tile test ([R3]): keep iff some valid row has
 * max_c s_rc - LSE_r >= ln tau - ln Lq. Returns the keep flag; *mu gets the
 * max over rows of that difference. s must hold the tile's scores. */
static int bwd_tile_test(const double *s, int T, int r0, int R, int c0, int j,
                         int i, const double *LSE, double tau, int force_first,
                         double *mu_out) {
  if (force_first && j == i) { *mu_out = INFINITY; return 1; }
  if (tau <= 0.0) { *mu_out = INFINITY; return 1; }
  double mu = NEG_INF;
  int kept = 0;
  for (int r = 0; r < R; ++r) {
    const int row = r0 + r;
    const int c1 = imin((j + 1) * T, row + 1);
    double mx = NEG_INF;
    for (int c = c0; c < c1; ++c) {
      const double v = s[(size_t)r * T + (c - c0)];
      if (v > mx) mx = v;
    }
    const double crit = (mx - LSE[row]) - log_threshold(tau, (double)(row + 1));
    if (crit > mu) mu = crit;
    if (crit >= 0.0) kept = 1;
  }
  *mu_out = mu;
  return kept;
}

static void tile_scores(const double *Q, const double *K, int d, int T,
                        double scale, int r0, int R, int c0, int j, double *s) {
  for (int r = 0; r < R; ++r) {
    const int row = r0 + r;
    const int c1 = imin((j + 1) * T, row + 1);
    for (int c = c0; c < c1; ++c)
      s[(size_t)r * T + (c - c0)] = scale * dot(Q + (size_t)row * d, K + (size_t)c * d, d);
  }
}

/*
 * Backward of one (batch, head) slice ([R3]).
 * Inputs: Q, K, V, O, dO [L][d]; LSE [L] (the forward's final log-normalizer).
 * dQ is computed for the query blocks listed in qblocks[nq] (rows of other
 * blocks untouched); dK, dV for the key blocks in kblocks[nk]. The caller
 * zero-fills outputs.
 * keep (may be NULL): [nb][nb], written for (i, j) pairs visited by the dQ
 * pass (every j <= i of the listed query blocks) and by the dK/dV pass.
 * margin (may be NULL): same indexing, max over rows of
 * (max_c s - LSE) - (ln tau - ln Lq).
 */
int mala_oracle_bwd(const double *Q, const double *K, const double *V,
                    const double *O, const double *dO, const double *LSE,
                    int L, int d, int T, double scale, double tau,
                    int force_first, const int *qblocks, int nq,
                    const int *kblocks, int nk, double *dQ, double *dK,
                    double *dV, uint8_t *keep, double *margin) {
  if (L <= 0) return 0;
  const int nb = (L + T - 1) / T;
  double *D = malloc(sizeof(double) * L);
  for (int r = 0; r < L; ++r) D[r] = dot(dO + (size_t)r * d, O + (size_t)r * d, d);

  /* dQ pass: query block i, every legal key block j <= i */
#pragma omp parallel for schedule(dynamic, 1)
  for (int n = 0; n < nq; ++n) {
    const int i = qblocks[n];
    const int r0 = i * T, R = imin(L, (i + 1) * T) - r0;
    double *s = malloc(sizeof(double) * (size_t)R * T);
    for (int j = i; j >= 0; --j) {
      const int c0 = j * T;
      tile_scores(Q, K, d, T, scale, r0, R, c0, j, s);
      double mu;
      const int kept = bwd_tile_test(s, T, r0, R, c0, j, i, LSE, tau, force_first, &mu);
      if (keep) keep[(size_t)i * nb + j] = (uint8_t)kept;
      if (margin) margin[(size_t)i * nb + j] = mu;
      if (!kept) continue;
      for (int r = 0; r < R; ++r) {
        const int row = r0 + r;
        const int c1 = imin((j + 1) * T, row + 1);
        for (int c = c0; c < c1; ++c) {
          const double p = exp(s[(size_t)r * T + (c - c0)] - LSE[row]);
          const double dp = dot(dO + (size_t)row * d, V + (size_t)c * d, d);
          const double ds = p * (dp - D[row]);
          for (int k = 0; k < d; ++k) dQ[(size_t)row * d + k] += scale * ds * K[(size_t)c * d + k];
        }
      }
    }
    free(s);
  }

  /* dK / dV pass: key block j, every query block i >= j */
#pragma omp parallel for schedule(dynamic, 1)
  for (int n = 0; n < nk; ++n) {
    const int j = kblocks[n];
    const int c0 = j * T;
    double *s = malloc(sizeof(double) * (size_t)T * T);
    for (int i = j; i < nb; ++i) {
      const int r0 = i * T, R = imin(L, (i + 1) * T) - r0;
      tile_scores(Q, K, d, T, scale, r0, R, c0, j, s);
      double mu;
      const int kept = bwd_tile_test(s, T, r0, R, c0, j, i, LSE, tau, force_first, &mu);
      if (keep) keep[(size_t)i * nb + j] = (uint8_t)kept;
      if (margin) margin[(size_t)i * nb + j] = mu;
      if (!kept) continue;
      for (int r = 0; r < R; ++r) {
        const int row = r0 + r;
        const int c1 = imin((j + 1) * T, row + 1);
        for (int c = c0; c < c1; ++c) {
          const double p = exp(s[(size_t)r * T + (c - c0)] - LSE[row]);
          const double dp = dot(dO + (size_t)row * d, V + (size_t)c * d, d);
          const double ds = p * (dp - D[row]);
          for (int k = 0; k < d; ++k) {
            dV[(size_t)c * d + k] += p * dO[(size_t)row * d + k];
            dK[(size_t)c * d + k] += scale * ds * Q[(size_t)row * d + k];
          }
        }
      }
    }
    free(s);
  }
  free(D);
  return 0;
}

/*
 * Decode step for one batch entry ([R5] one rule for prefill and decode).
 * q: [Hq][d] (one new token per query head); Kc, Vc: [Hkv][Lc][d], the cache
 * including the current token, so Lq = Lc for every head.
 * Tiles of T keys aligned from position 0, visited newest first; the first
 * visited tile is always kept. per_head = 0: the rows of a tile are the
 * G = Hq/Hkv query heads sharing KV head g (the tile test is "all rows below");
 * per_head = 1: every query head decides alone.
 * o: [Hq][d]. keep (may be NULL): [Hq or Hkv][nt] bytes. margin likewise.
 */
int mala_oracle_decode(const double *q, const double *Kc, const double *Vc,
                       int Hq, int Hkv, int Lc, int d, int T, double scale,
                       double tau, int per_head, double *o, uint8_t *keep,
                       double *margin) {
  if (Lc <= 0) return 0;
  const int G = Hq / Hkv;
  const int nt = (Lc + T - 1) / T;
  const int rows = per_head ? 1 : G;
  const int units = per_head ? Hq : Hkv;
  const double lthr = log_threshold(tau, (double)Lc);
#pragma omp parallel for schedule(dynamic, 1)
  for (int unit = 0; unit < units; ++unit) {
    const int g = per_head ? unit / G : unit;
    const int h0 = per_head ? unit : g * G;
    const double *Kg = Kc + (size_t)g * Lc * d;
    const double *Vg = Vc + (size_t)g * Lc * d;
    double *m = malloc(sizeof(double) * rows), *l = malloc(sizeof(double) * rows);
    double *mt = malloc(sizeof(double) * rows);
    double *acc = calloc((size_t)rows * d, sizeof(double));
    double *s = malloc(sizeof(double) * (size_t)rows * T);
    for (int r = 0; r < rows; ++r) { m[r] = NEG_INF; l[r] = 0.0; }
    for (int t = nt - 1; t >= 0; --t) {
      const int c0 = t * T, c1 = imin(Lc, (t + 1) * T);
      for (int r = 0; r < rows; ++r) {
        double mx = NEG_INF;
        for (int c = c0; c < c1; ++c) {
          const double v = scale * dot(q + (size_t)(h0 + r) * d, Kg + (size_t)c * d, d);
          s[(size_t)r * T + (c - c0)] = v;
          if (v > mx) mx = v;
        }
        mt[r] = mx;
      }
      int kept;
      double mu = NEG_INF;
      if (t == nt - 1 || tau <= 0.0) {
        kept = 1;
        mu = INFINITY;
      } else {
        kept = 0;
        for (int r = 0; r < rows; ++r) {
          const double crit = (mt[r] - m[r] - log(l[r])) - lthr;
          if (crit > mu) mu = crit;
          if (crit >= 0.0) kept = 1;
        }
      }
      if (keep) keep[(size_t)unit * nt + t] = (uint8_t)kept;
      if (margin) margin[(size_t)unit * nt + t] = mu;
      if (!kept) continue;
      for (int r = 0; r < rows; ++r) {
        const double mnew = mt[r] > m[r] ? mt[r] : m[r];
        const double alpha = (m[r] == NEG_INF) ? 0.0 : exp(m[r] - mnew);
        double *a = acc + (size_t)r * d;
        for (int k = 0; k < d; ++k) a[k] *= alpha;
        double lsum = l[r] * alpha;
        for (int c = c0; c < c1; ++c) {
          const double p = exp(s[(size_t)r * T + (c - c0)] - mnew);
          lsum += p;
          for (int k = 0; k < d; ++k) a[k] += p * Vg[(size_t)c * d + k];
        }
        l[r] = lsum;
        m[r] = mnew;
      }
    }
    for (int r = 0; r < rows; ++r)
      for (int k = 0; k < d; ++k) o[(size_t)(h0 + r) * d + k] = acc[(size_t)r * d + k] / l[r];
    free(m); free(l); free(mt); free(acc); free(s);
  }
  return 0;
}

/*
 * Textbook causal softmax attention (FullAttn) for one slice: the tau -> 0
 * limit of both passes ([R5]) and the reference for omitted mass and output
 * error. O [L][d], LSE [L].
 */
int mala_oracle_dense_fwd(const double *Q, const double *K, const double *V,
                          int L, int d, double scale, double *O, double *LSE) {
#pragma omp parallel for schedule(dynamic, 16)
  for (int r = 0; r < L; ++r) {
    double *s = malloc(sizeof(double) * (size_t)(r + 1));
    double mx = NEG_INF;
    for (int c = 0; c <= r; ++c) {
      s[c] = scale * dot(Q + (size_t)r * d, K + (size_t)c * d, d);
      if (s[c] > mx) mx = s[c];
    }
    double z = 0.0;
    for (int c = 0; c <= r; ++c) z += exp(s[c] - mx);
    for (int k = 0; k < d; ++k) {
      double a = 0.0;
      for (int c = 0; c <= r; ++c) a += exp(s[c] - mx) * V[(size_t)c * d + k];
      O[(size_t)r * d + k] = a / z;
    }
    LSE[r] = mx + log(z);
    free(s);
  }
  return 0;
}

/* Gradients of textbook causal softmax attention, dQ/dK/dV [L][d] zeroed by
 * the caller. P = softmax(S), dV = P^T dO, dP = dO V^T,
 * dS = P o (dP - rowsum(P o dP)), dQ = scale dS K, dK = scale dS^T Q. */
int mala_oracle_dense_bwd(const double *Q, const double *K, const double *V,
                          const double *dO, int L, int d, double scale,
                          double *dQ, double *dK, double *dV) {
  double *P = calloc((size_t)L * L, sizeof(double));
  double *dS = calloc((size_t)L * L, sizeof(double));
#pragma omp parallel for schedule(dynamic, 16)
  for (int r = 0; r < L; ++r) {
    double mx = NEG_INF;
    double *pr = P + (size_t)r * L;
    for (int c = 0; c <= r; ++c) {
      pr[c] = scale * dot(Q + (size_t)r * d, K + (size_t)c * d, d);
      if (pr[c] > mx) mx = pr[c];
    }
    double z = 0.0;
    for (int c = 0; c <= r; ++c) { pr[c] = exp(pr[c] - mx); z += pr[c]; }
    for (int c = 0; c <= r; ++c) pr[c] /= z;
    double *dsr = dS + (size_t)r * L;
    double rs = 0.0;
    for (int c = 0; c <= r; ++c) {
      dsr[c] = dot(dO + (size_t)r * d, V + (size_t)c * d, d); /* dP */
      rs += pr[c] * dsr[c];
    }
    for (int c = 0; c <= r; ++c) dsr[c] = pr[c] * (dsr[c] - rs);
    for (int k = 0; k < d; ++k) {
      double a = 0.0;
      for (int c = 0; c <= r; ++c) a += dsr[c] * K[(size_t)c * d + k];
      dQ[(size_t)r * d + k] = scale * a;
    }
  }
#pragma omp parallel for schedule(dynamic, 16)
  for (int c = 0; c < L; ++c) {
    for (int k = 0; k < d; ++k) {
      double av = 0.0, ak = 0.0;
      for (int r = c; r < L; ++r) {
        av += P[(size_t)r * L + c] * dO[(size_t)r * d + k];
        ak += dS[(size_t)r * L + c] * Q[(size_t)r * d + k];
      }
      dV[(size_t)c * d + k] = av;
      dK[(size_t)c * d + k] = scale * ak;
    }
  }
  free(P); free(dS);
  return 0;
}

/*
 * Omitted dense mass per query row ([R4] Proposition 1 quantity):
 * 1 - sum over keys in kept tiles of exp(s_rc - LSE_dense_r).
 * keep: [nb][nb] bytes (query block, key block). mass_out: [L].
 */
int mala_oracle_omitted_mass(const double *Q, const double *K, int L, int d,
                             int T, double scale, const uint8_t *keep,
                             const double *LSE_dense, double *mass_out) {
  const int nb = (L + T - 1) / T;
#pragma omp parallel for schedule(dynamic, 16)
  for (int r = 0; r < L; ++r) {
    const int i = r / T;
    double kept_mass = 0.0;
    for (int c = 0; c <= r; ++c) {
      if (!keep[(size_t)i * nb + c / T]) continue;
      kept_mass += exp(scale * dot(Q + (size_t)r * d, K + (size_t)c * d, d) - LSE_dense[r]);
    }
    mass_out[r] = 1.0 - kept_mass;
  }
  return 0;
}
