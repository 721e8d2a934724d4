/*
 * fp64 CPU oracle for block-causal softmax attention and its forward-mode JVP.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file; only the tests, the package's smoke check and the benchmark's CPU
 * baseline use it. It shares no code, header or table with the CUDA library.
 *
 * What it computes (Causal-rCM, App. B "FlashAttention-2 JVP kernel with custom
 * mask", eq. 42-45; the symbols there are lost in the page text, so they are
 * restored here from standard calculus):
 *   s_j   = scale * <q_i, k_j>                               (eq. 42)
 *   ts_j  = scale * (<tq_i, k_j> + <q_i, tk_j>)              (eq. 43)
 *   keys outside the mask take no part and carry no tangent  (text after eq. 43)
 *   p_j   = exp(s_j - m) / sum_l exp(s_l - m),  m = max_j s_j
 *   O_i   = sum_j p_j v_j
 *   mu    = sum_j p_j ts_j
 *   tO_i  = sum_j p_j (ts_j - mu) v_j + sum_j p_j tv_j      (eq. 44)
 *   LSE_i = m + ln sum_j exp(s_j - m),   tLSE_i = mu
 * Every sum runs over the keys row i may attend to. There is no tiling, no online
 * softmax and no reordering: two plain passes per row, in double precision.
 *
 * The mask (section 3.1.1 "Teacher forcing", eq. 8; Table 2 legend; section 4
 * chunk modes c1-1 / c3-3; section 3.2 Cosmos 3 super-token causality): tokens
 * are grouped into frames of T tokens and frames into chunks of c frames.
 *   tf_layout = 0: token t belongs to chunk t / (c*T); a query sees every key of
 *                  its own chunk and of all earlier chunks.
 *   tf_layout = 1: the sequence is [clean copy | noisy copy], each F*T tokens.
 *                  A clean query sees clean keys of its own and earlier chunks.
 *                  A noisy query of chunk j sees clean keys of chunks < j and the
 *                  noisy keys of its own chunk j. Clean queries see no noisy key.
 *
 * Inputs may be given as fp64, fp32 or bf16 bit patterns; every element is
 * widened to double exactly before use, so the oracle sees the same values as
 * the GPU.
 *
 * Parity status: every function here is pinned by tests (finite differences,
 * linearity, exact special cases, torch library cross-checks, brute-force mask
 * counts); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F64 = 0, ORACLE_F32 = 1, ORACLE_BF16 = 2 };

static double load_elem(const void *base, int dtype, int64_t idx) {
  if (dtype == ORACLE_F64) return ((const double *)base)[idx];
  if (dtype == ORACLE_F32) return (double)((const float *)base)[idx];
  /* bf16: the 16 stored bits are the top half of an IEEE binary32 */
  uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Chunk membership of token t, written from the definitions above. */
int oracle_visible(int64_t T, int64_t c, int64_t F, int tf, int64_t qi, int64_t kj) {
  int64_t G = c * T;       /* tokens per chunk */
  int64_t L = F * T;       /* tokens per copy of the video */
  if (!tf) {
    if (qi < 0 || kj < 0 || qi >= L || kj >= L) return 0;
    return (kj / G) <= (qi / G);
  }
  if (qi < 0 || kj < 0 || qi >= 2 * L || kj >= 2 * L) return 0;
  int q_noisy = qi >= L, k_noisy = kj >= L;
  int64_t q_chunk = (q_noisy ? qi - L : qi) / G;
  int64_t k_chunk = (k_noisy ? kj - L : kj) / G;
  if (!q_noisy) return !k_noisy && k_chunk <= q_chunk;
  if (!k_noisy) return k_chunk < q_chunk;
  return k_chunk == q_chunk;
}

/* Number of visible (query, key) pairs of one head, by brute force. */
int64_t oracle_visible_pairs(int64_t T, int64_t c, int64_t F, int tf) {
  int64_t N = F * T * (tf ? 2 : 1);
  int64_t total = 0;
#pragma omp parallel for reduction(+ : total) schedule(dynamic, 64)
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j < N; ++j) total += oracle_visible(T, c, F, tf, i, j);
  return total;
}

/*
 * Forward + JVP for a list of rows.
 *   q..tv   : [B*H, N, D] row-major in `dtype`.
 *   rows    : flat row ids bh*N + i, nrows of them.
 *   o, to   : [nrows, D] double.  lse, tlse : [nrows] double.
 * A row that sees no key gets O = tO = 0, LSE = -inf, tLSE = 0.
 * Returns 0, or -1 on a bad argument.
 */
int oracle_attn_fwd_jvp_rows(const void *q, const void *k, const void *v,
                             const void *tq, const void *tk, const void *tv,
                             int dtype, int64_t BH, int64_t N, int64_t D, double scale,
                             int64_t T, int64_t c, int64_t F, int tf,
                             const int64_t *rows, int64_t nrows,
                             double *o, double *to, double *lse, double *tlse,
                             int nthreads) {
  if (D <= 0 || N <= 0 || BH <= 0 || nrows < 0) return -1;
  if (N != F * T * (tf ? 2 : 1)) return -1;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= BH * N) return -1;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
  int bad = 0;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *ts = (double *)malloc(sizeof(double) * (size_t)N);
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    double *qi = (double *)malloc(sizeof(double) * (size_t)D);
    double *tqi = (double *)malloc(sizeof(double) * (size_t)D);
    if (!s || !ts || !keys || !qi || !tqi) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t r = 0; r < nrows; ++r) {
        int64_t bh = rows[r] / N, i = rows[r] % N;
        int64_t head = bh * N * D;
        for (int64_t d = 0; d < D; ++d) {
          qi[d] = load_elem(q, dtype, head + i * D + d);
          tqi[d] = load_elem(tq, dtype, head + i * D + d);
        }
        /* the keys this row may attend to */
        int64_t nk = 0;
        for (int64_t j = 0; j < N; ++j)
          if (oracle_visible(T, c, F, tf, i, j)) keys[nk++] = j;
        double *orow = o + r * D, *torow = to + r * D;
        for (int64_t d = 0; d < D; ++d) orow[d] = torow[d] = 0.0;
        if (nk == 0) {
          lse[r] = -INFINITY;
          tlse[r] = 0.0;
          continue;
        }
        /* pass 1: scores, score tangents and the row max */
        double m = -INFINITY;
        for (int64_t a = 0; a < nk; ++a) {
          int64_t kb = head + keys[a] * D;
          double dot = 0.0, tdot = 0.0;
          for (int64_t d = 0; d < D; ++d) {
            double kd = load_elem(k, dtype, kb + d);
            dot += qi[d] * kd;
            tdot += tqi[d] * kd + qi[d] * load_elem(tk, dtype, kb + d);
          }
          s[a] = scale * dot;
          ts[a] = scale * tdot;
          if (s[a] > m) m = s[a];
        }
        /* pass 2: normaliser, probabilities and mu = <P, tS> */
        double Z = 0.0;
        for (int64_t a = 0; a < nk; ++a) {
          s[a] = exp(s[a] - m); /* s now holds the unnormalised weight */
          Z += s[a];
        }
        double mu = 0.0;
        for (int64_t a = 0; a < nk; ++a) {
          s[a] /= Z; /* s now holds p_j */
          mu += s[a] * ts[a];
        }
        /* outputs: O = sum p v ;  tO = sum p (ts - mu) v + sum p tv */
        for (int64_t a = 0; a < nk; ++a) {
          int64_t vb = head + keys[a] * D;
          double p = s[a], pd = s[a] * (ts[a] - mu);
          for (int64_t d = 0; d < D; ++d) {
            double vd = load_elem(v, dtype, vb + d);
            orow[d] += p * vd;
            torow[d] += pd * vd + p * load_elem(tv, dtype, vb + d);
          }
        }
        lse[r] = m + log(Z);
        tlse[r] = mu;
      }
    }
    free(s);
    free(ts);
    free(keys);
    free(qi);
    free(tqi);
  }
  return bad ? -1 : 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
