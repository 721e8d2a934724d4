// Closed-form block-causal mask geometry and tile schedule, usable on host and
// device.
//
// The mask is the teacher-forcing / block-causal family of the Causal-rCM paper
// (section 3.1.1, eq. 8; Table 2 legend; section 4 chunk modes). Appendix B
// represents such masks as a short list of query groups, each with a few
// allowed key ranges, and streams only those ranges; the same schedule serves
// the primal and the tangent. Here that list is not stored: every row's key
// ranges and every query tile's key-tile ranges follow from four integers.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define CAJ_HD __host__ __device__ __forceinline__
#else
#define CAJ_HD inline
#endif

namespace caj {

struct MaskGeom {
  int32_t G;   // tokens per chunk (frames_per_chunk * tokens_per_frame)
  int32_t L;   // tokens of one copy of the video (n_frames * tokens_per_frame)
  int32_t N;   // sequence length (L, or 2L for the teacher-forcing layout)
  int32_t tf;  // 1 = [clean | noisy] teacher-forcing layout
};

// Keys visible to query `q`: [a0, b0) U [a1, b1), both possibly empty.
//   plain / clean query in chunk j: [0, (j+1) G)
//   noisy query in chunk j:         [0, j G) U [L + j G, L + (j+1) G)
CAJ_HD void row_key_ranges(const MaskGeom &m, int32_t q, int32_t &a0, int32_t &b0,
                           int32_t &a1, int32_t &b1) {
  if (!m.tf || q < m.L) {
    a0 = 0;
    b0 = (q / m.G + 1) * m.G;
    a1 = b1 = 0;
  } else {
    int32_t j = (q - m.L) / m.G;
    a0 = 0;
    b0 = j * m.G;
    a1 = m.L + j * m.G;
    b1 = a1 + m.G;
  }
}

// Key tiles of width bn that query rows [q0, q1) touch, as up to two ascending
// disjoint tile ranges [t0, t1) U [t2, t3). Returns the number of tiles.
CAJ_HD int32_t qtile_key_tiles(const MaskGeom &m, int32_t q0, int32_t q1, int32_t bn,
                               int32_t &t0, int32_t &t1, int32_t &t2, int32_t &t3) {
  // Union of the rows' ranges: one prefix [0, pre) plus, for noisy rows, one
  // band [lo, hi) inside the noisy copy.
  int32_t pre = 0, lo = 0, hi = 0;
  const int32_t clean_end = m.tf ? m.L : m.N;
  if (q0 < clean_end) {
    int32_t last = (q1 < clean_end ? q1 : clean_end) - 1;
    pre = (last / m.G + 1) * m.G;
  }
  if (m.tf && q1 > m.L) {
    int32_t first = q0 > m.L ? q0 : m.L;
    int32_t j0 = (first - m.L) / m.G, j1 = (q1 - 1 - m.L) / m.G;
    int32_t noisy_pre = j1 * m.G;  // the last noisy row's clean history is the widest
    if (noisy_pre > pre) pre = noisy_pre;
    lo = m.L + j0 * m.G;
    hi = m.L + (j1 + 1) * m.G;
  }
  t0 = 0;
  t1 = (pre + bn - 1) / bn;
  if (hi > lo) {
    t2 = lo / bn;
    t3 = (hi + bn - 1) / bn;
    if (t2 <= t1) {  // the prefix and the band share or touch a tile: merge
      if (t3 > t1) t1 = t3;
      t2 = t3 = t1;
    }
  } else {
    t2 = t3 = t1;
  }
  if (t1 == 0) {  // no prefix (noisy rows of chunk 0 only): the band alone
    t0 = t2;
    t1 = t3;
    t2 = t3 = t1;
  }
  return (t1 - t0) + (t3 - t2);
}

// Queries that may attend to key `k` (the transposed mask), as up to two
// intervals [a0, b0) U [a1, b1):
//   plain layout, key in chunk j:     [j G, N)
//   clean key in chunk j (TF layout): clean queries [j G, L) and noisy queries
//                                     of later chunks [L + (j+1) G, 2L)
//   noisy key in chunk j (TF layout): the noisy queries of chunk j
CAJ_HD void key_query_ranges(const MaskGeom &m, int32_t k, int32_t &a0, int32_t &b0, int32_t &a1,
                             int32_t &b1) {
  if (!m.tf) {
    a0 = (k / m.G) * m.G;
    b0 = m.N;
    a1 = b1 = 0;
  } else if (k < m.L) {
    const int32_t j = k / m.G;
    a0 = j * m.G;
    b0 = m.L;
    a1 = m.L + (j + 1) * m.G;
    b1 = 2 * m.L;
    if (a1 >= b1) a1 = b1 = 0;
  } else {
    const int32_t j = (k - m.L) / m.G;
    a0 = m.L + j * m.G;
    b0 = a0 + m.G;
    a1 = b1 = 0;
  }
}

// Query tiles of height bq that some key of [k0, k1) is visible to, as up to
// three ascending disjoint tile ranges t[0..5] ([t0,t1) U [t2,t3) U [t4,t5)).
// Returns the number of tiles.
CAJ_HD int32_t ktile_query_tiles(const MaskGeom &m, int32_t k0, int32_t k1, int32_t bq,
                                 int32_t (&t)[6]) {
  // Query intervals of the union: the first key of each part has the widest.
  int32_t lo[3], hi[3], n = 0;
  if (!m.tf) {
    lo[n] = (k0 / m.G) * m.G;
    hi[n++] = m.N;
  } else {
    if (k0 < m.L) {  // clean keys: the earliest chunk sees the most queries
      const int32_t j = k0 / m.G;
      lo[n] = j * m.G;
      hi[n++] = m.L;
      if (m.L + (j + 1) * m.G < 2 * m.L) {
        lo[n] = m.L + (j + 1) * m.G;
        hi[n++] = 2 * m.L;
      }
    }
    if (k1 > m.L) {  // noisy keys: queries of the noisy chunks they span
      const int32_t first = k0 > m.L ? k0 : m.L;
      const int32_t e0 = (first - m.L) / m.G, e1 = (k1 - 1 - m.L) / m.G;
      lo[n] = m.L + e0 * m.G;
      hi[n++] = m.L + (e1 + 1) * m.G;
    }
  }
  // sort the (at most three) intervals by start, then merge in tile units
  for (int32_t a = 0; a < n; ++a)
    for (int32_t b = a + 1; b < n; ++b)
      if (lo[b] < lo[a]) {
        int32_t x = lo[a]; lo[a] = lo[b]; lo[b] = x;
        x = hi[a]; hi[a] = hi[b]; hi[b] = x;
      }
  int32_t r = 0;
  for (int32_t a = 0; a < n; ++a) {
    const int32_t s = lo[a] / bq, e = (hi[a] + bq - 1) / bq;
    if (r > 0 && s <= t[2 * r - 1]) {
      if (e > t[2 * r - 1]) t[2 * r - 1] = e;
    } else {
      t[2 * r] = s;
      t[2 * r + 1] = e;
      ++r;
    }
  }
  int32_t total = 0;
  for (int32_t a = 0; a < r; ++a) total += t[2 * a + 1] - t[2 * a];
  for (int32_t a = r; a < 3; ++a) t[2 * a] = t[2 * a + 1] = (r ? t[2 * r - 1] : 0);
  return total;
}

// Visible (query, key) pairs of one head: n chunks of G tokens; chunk j of the
// plain layout sees j+1 chunks (G^2 n(n+1)/2 in all); the teacher-forcing
// layout adds the same count again for the noisy copy.
CAJ_HD int64_t visible_pairs(const MaskGeom &m) {
  int64_t n = m.L / m.G, G = m.G;
  int64_t half = G * G * n * (n + 1) / 2;
  return m.tf ? 2 * half : half;
}

}  // namespace caj
