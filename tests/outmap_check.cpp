// Host check of the attention kernels' output map (caj::slice_row in
// csrc/kernels.h), built and run by test_outmap_cpu.py. For every shape it
// emulates the P launches of P-way Ulysses context parallelism (launch r holds
// heads [r H/P, (r+1) H/P) over the whole sequence) and checks that each
// (head, row) lands in slice q / (N/P) at the expected row of that slice's
// [B, H, N/P, D] (or [B, N/P, H, D]) buffer and [B, H, N/P] statistics, in bounds,
// with every row of every slice written exactly once. The one-slice map must
// give the addressing of a single call (caj::out_row, head-major and
// token-major).
#include <cstdio>
#include <vector>

#include "kernels.h"

int main() {
  long bad = 0;
  for (int B : {1, 2})
    for (int H : {2, 4, 8, 12})
      for (int P : {1, 2, 3, 4, 8})
        for (int N : {64, 600, 720, 800})
          for (int tm : {0, 1}) {
            if (H % P || N % P) continue;
            const int Hp = H / P, Ls = N / P;
            const size_t lim = size_t(B) * H * Ls;
            std::vector<int> rows(P * lim, 0), stats(P * lim, 0);
            for (int r0 = 0; r0 < P; ++r0) {
              caj::OutMap m{};
              m.shards = P; m.shard_len = Ls; m.heads = Hp;
              m.head_base = r0 * Hp; m.heads_total = H; m.token_major = tm;
              for (int bh = 0; bh < B * Hp; ++bh)
                for (int q = 0; q < N; ++q) {
                  const caj::OutRow d = caj::slice_row(m, bh, q);
                  if (d.shard < 0 || d.shard >= P || d.row >= lim || d.stat >= lim) { ++bad; continue; }
                  const int b = bh / Hp, h = r0 * Hp + bh % Hp, ql = q % Ls;
                  const size_t st = (size_t(b) * H + h) * Ls + ql;
                  const size_t rw = tm ? (size_t(b) * Ls + ql) * H + h : st;
                  if (d.shard != q / Ls || d.stat != st || d.row != rw) ++bad;
                  ++rows[d.shard * lim + d.row];
                  ++stats[d.shard * lim + d.stat];
                }
            }
            for (size_t i = 0; i < rows.size(); ++i) bad += (rows[i] != 1) + (stats[i] != 1);
          }
  for (int B : {1, 3})
    for (int H : {2, 5})
      for (int N : {64, 130}) {
        caj::OutMap m{};
        m.shards = 1; m.shard_len = N; m.heads = H; m.heads_total = H;
        for (int bh = 0; bh < B * H; ++bh)
          for (int q = 0; q < N; ++q) {
            const int D = 64;
            caj::OutRow d = caj::slice_row(m, bh, q);
            bad += d.shard != 0 || d.stat != size_t(bh) * N + q || d.row != d.stat;
            bad += d.row * D != caj::out_row(bh, q, N, 0, D);
            m.token_major = 1;
            d = caj::slice_row(m, bh, q);
            m.token_major = 0;
            bad += d.row != (size_t(bh / H) * N + q) * H + bh % H;
            bad += d.row * D != caj::out_row(bh, q, N, H, D);
          }
      }
  std::printf("mismatches %ld\n", bad);
  return bad != 0;
}
