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

/*
 * Layer prologue in primal-tangent form (Causal-rCM section 3.2.2, "JVP FSDP2":
 * every layer takes and returns a (primal, tangent) pair). For query and key:
 *   y  = g * x / r,            r = sqrt(mean_C(x^2) + eps)            (RMSNorm)
 *   ty = g * (tx / r - x * mean_C(x * tx) / r^3)                      (its JVP)
 * followed by the rotary embedding of interleaved pairs (2i, 2i+1) of each head,
 *   (a, b) -> (a cos t - b sin t, a sin t + b cos t),  t = theta[n][i],
 * which is linear and so rotates the tangent the same way. Values and their
 * tangents are only re-laid out: [B, N, H*D] -> [B, H, N, D].
 * The normalisation runs over the whole token (C = H*D, per_head = 0) or over
 * each head (C = D, per_head = 1).
 *   x*, t*  : [B, N, H*D] in `dtype` (F64 / F32 / BF16 codes as above)
 *   gq, gk  : [H*D] double;  cosv, sinv : [N, D/2] double
 *   outputs : [B, H, N, D] double each (q, k, v, tq, tk, tv)
 */
int oracle_qk_norm_rope_jvp(const void *xq, const void *xk, const void *xv, const void *txq,
                            const void *txk, const void *txv, int dtype, const double *gq,
                            const double *gk, const double *cosv, const double *sinv, int64_t B,
                            int64_t N, int64_t H, int64_t D, double eps, int per_head, double *q,
                            double *k, double *v, double *tq, double *tk, double *tv) {
  if (B <= 0 || N <= 0 || H <= 0 || D <= 0 || (D % 2) || eps < 0) return -1;
  const int64_t C = H * D;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t b = 0; b < B; ++b)
    for (int64_t n = 0; n < N; ++n) {
      const int64_t in_row = (b * N + n) * C;
      for (int which = 0; which < 3; ++which) {
        const void *x = which == 0 ? xq : which == 1 ? xk : xv;
        const void *tx = which == 0 ? txq : which == 1 ? txk : txv;
        double *y = which == 0 ? q : which == 1 ? k : v;
        double *ty = which == 0 ? tq : which == 1 ? tk : tv;
        const double *g = which == 0 ? gq : gk;
        for (int64_t h = 0; h < H; ++h) {
          /* normalisation statistics over the token or over this head */
          double r = 1.0, m_xtx = 0.0;
          if (which < 2) {
            int64_t lo = per_head ? h * D : 0, len = per_head ? D : C;
            double ss = 0.0, sxt = 0.0;
            for (int64_t c = lo; c < lo + len; ++c) {
              double xc = load_elem(x, dtype, in_row + c);
              ss += xc * xc;
              sxt += xc * load_elem(tx, dtype, in_row + c);
            }
            r = sqrt(ss / (double)len + eps);
            m_xtx = sxt / (double)len;
          }
          const int64_t out_row = ((b * H + h) * N + n) * D;
          for (int64_t d = 0; d < D; d += 2) {
            double a = load_elem(x, dtype, in_row + h * D + d);
            double bb = load_elem(x, dtype, in_row + h * D + d + 1);
            double ta = load_elem(tx, dtype, in_row + h * D + d);
            double tb = load_elem(tx, dtype, in_row + h * D + d + 1);
            if (which < 2) {
              double ga = g[h * D + d], gb = g[h * D + d + 1];
              double na = ga * a / r, nb = gb * bb / r;
              double tna = ga * (ta / r - a * m_xtx / (r * r * r));
              double tnb = gb * (tb / r - bb * m_xtx / (r * r * r));
              double cs = cosv[n * (D / 2) + d / 2], sn = sinv[n * (D / 2) + d / 2];
              a = na * cs - nb * sn;
              bb = na * sn + nb * cs;
              ta = tna * cs - tnb * sn;
              tb = tna * sn + tnb * cs;
            }
            y[out_row + d] = a;
            y[out_row + d + 1] = bb;
            ty[out_row + d] = ta;
            ty[out_row + d + 1] = tb;
          }
        }
      }
    }
  return 0;
}

/*
 * Backward of the primal masked attention (the student's gradient step in
 * TF-sCM; the JVP branch itself is stop-gradient). For one head, with
 * P_ij = softmax_j(scale <q_i, k_j>) over the visible keys and dO the gradient of
 * the output O = P V:
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = <dO_i, v_j>
 *   Delta_i = sum_j P_ij dP_ij            (equals <dO_i, O_i>)
 *   dS_ij = P_ij (dP_ij - Delta_i)
 *   dQ_i  = scale sum_j dS_ij k_j
 *   dK_j  = scale sum_i dS_ij q_i
 * The oracle recomputes P from q and k (it does not take an LSE), two passes per
 * row, fp64, and accumulates dK and dV row by row (each thread owns one head).
 *   q, k, v, dout : [BH, N, D] in `dtype`;  dq, dk, dv : [BH, N, D] double
 *   delta         : [BH, N] double (Delta_i), may be NULL
 */
int oracle_attn_bwd(const void *q, const void *k, const void *v, const void *dout, int dtype,
                    int64_t BH, int64_t N, int64_t D, double scale, int64_t T, int64_t c,
                    int64_t F, int tf, double *dq, double *dk, double *dv, double *delta) {
  if (D <= 0 || N <= 0 || BH <= 0) return -1;
  if (N != F * T * (tf ? 2 : 1)) return -1;
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < BH; ++bh) {
    const int64_t head = bh * N * D;
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double *dp = (double *)malloc(sizeof(double) * (size_t)N);
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    if (!p || !dp || !keys) {
#pragma omp atomic write
      bad = 1;
    } else {
      for (int64_t x = 0; x < N * D; ++x) dq[head + x] = dk[head + x] = dv[head + x] = 0.0;
      for (int64_t i = 0; i < N; ++i) {
        int64_t nk = 0;
        for (int64_t j = 0; j < N; ++j)
          if (oracle_visible(T, c, F, tf, i, j)) keys[nk++] = j;
        if (nk == 0) {
          if (delta) delta[bh * N + i] = 0.0;
          continue;
        }
        double m = -INFINITY;
        for (int64_t a = 0; a < nk; ++a) {
          double s = 0.0, t = 0.0;
          for (int64_t d = 0; d < D; ++d) {
            s += load_elem(q, dtype, head + i * D + d) * load_elem(k, dtype, head + keys[a] * D + d);
            t += load_elem(dout, dtype, head + i * D + d) * load_elem(v, dtype, head + keys[a] * D + d);
          }
          p[a] = scale * s;
          dp[a] = t;
          if (p[a] > m) m = p[a];
        }
        double Z = 0.0;
        for (int64_t a = 0; a < nk; ++a) {
          p[a] = exp(p[a] - m);
          Z += p[a];
        }
        double dl = 0.0;
        for (int64_t a = 0; a < nk; ++a) {
          p[a] /= Z;
          dl += p[a] * dp[a];
        }
        if (delta) delta[bh * N + i] = dl;
        for (int64_t a = 0; a < nk; ++a) {
          const int64_t j = keys[a];
          const double ds = p[a] * (dp[a] - dl);
          for (int64_t d = 0; d < D; ++d) {
            dv[head + j * D + d] += p[a] * load_elem(dout, dtype, head + i * D + d);
            dq[head + i * D + d] += scale * ds * load_elem(k, dtype, head + j * D + d);
            dk[head + j * D + d] += scale * ds * load_elem(q, dtype, head + i * D + d);
          }
        }
      }
    }
    free(p);
    free(dp);
    free(keys);
  }
  return bad ? -1 : 0;
}

/*
 * dQ and Delta of selected query rows (the same definitions as oracle_attn_bwd,
 * restricted to rows). Row i needs only its own softmax:
 *   p_j = exp(s_j - m) / Z over the keys row i sees,  dp_j = <dO_i, v_j>,
 *   Delta_i = sum_j p_j dp_j,  dQ_i = scale sum_j p_j (dp_j - Delta_i) k_j.
 * So a few hundred rows of a full-size problem cost a few hundred row passes,
 * not the whole N x N backward.
 *   q, k, v, dout : [BH, N, D] in `dtype`;  rows : flat ids bh*N + i
 *   dq            : [nrows, D] double;  delta : [nrows] double
 */
int oracle_attn_bwd_dq_rows(const void *q, const void *k, const void *v, const void *dout, int dtype,
                            int64_t BH, int64_t N, int64_t D, double scale, int64_t T, int64_t c,
                            int64_t F, int tf, const int64_t *rows, int64_t nrows, double *dq,
                            double *delta) {
  if (D <= 0 || N <= 0 || BH <= 0 || nrows < 0) return -1;
  if (N != F * T * (tf ? 2 : 1)) return -1;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= BH * N) return -1;
  int bad = 0;
#pragma omp parallel
  {
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double *dp = (double *)malloc(sizeof(double) * (size_t)N);
    int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
    if (!p || !dp || !keys) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for schedule(dynamic, 1)
      for (int64_t r = 0; r < nrows; ++r) {
        const int64_t bh = rows[r] / N, i = rows[r] % N, head = bh * N * D;
        double *dqrow = dq + r * D;
        for (int64_t d = 0; d < D; ++d) dqrow[d] = 0.0;
        int64_t nk = 0;
        for (int64_t j = 0; j < N; ++j)
          if (oracle_visible(T, c, F, tf, i, j)) keys[nk++] = j;
        if (nk == 0) {
          delta[r] = 0.0;
          continue;
        }
        double m = -INFINITY;
        for (int64_t a = 0; a < nk; ++a) {
          double s = 0.0, t = 0.0;
          for (int64_t d = 0; d < D; ++d) {
            s += load_elem(q, dtype, head + i * D + d) * load_elem(k, dtype, head + keys[a] * D + d);
            t += load_elem(dout, dtype, head + i * D + d) * load_elem(v, dtype, head + keys[a] * D + d);
          }
          p[a] = scale * s;
          dp[a] = t;
          if (p[a] > m) m = p[a];
        }
        double Z = 0.0;
        for (int64_t a = 0; a < nk; ++a) {
          p[a] = exp(p[a] - m);
          Z += p[a];
        }
        double dl = 0.0;
        for (int64_t a = 0; a < nk; ++a) {
          p[a] /= Z;
          dl += p[a] * dp[a];
        }
        delta[r] = dl;
        for (int64_t a = 0; a < nk; ++a) {
          const double ds = p[a] * (dp[a] - dl);
          for (int64_t d = 0; d < D; ++d)
            dqrow[d] += scale * ds * load_elem(k, dtype, head + keys[a] * D + d);
        }
      }
    }
    free(p);
    free(dp);
    free(keys);
  }
  return bad ? -1 : 0;
}
