// Host check of the GEMM work-unit walk (kd_unitwalk.h): for every cluster of
// every launch shape below, the division-free walk must visit exactly the
// units cid, cid + ncl, ... with the coordinates and K ranges that the direct
// computation gives.  Prints "ok" and exits 0, or names the first mismatch.
#include <cstdio>

#include "kd_unitwalk.h"

static int check(int m_tiles2, int n_tiles, int m_fastest, int k_blocks, int k_split, int ncl) {
  const int units = m_tiles2 * n_tiles * k_split;
  for (int cid = 0; cid < ncl; ++cid) {
    kd::UnitWalk w;
    kd::walk_begin(w, m_tiles2, n_tiles, m_fastest, k_blocks, k_split, cid, ncl);
    int expect_u = cid;
    for (; w.u < units; kd::walk_next(w)) {
      int s, m, n;
      kd::unit_coords_direct(m_tiles2, n_tiles, m_fastest, w.u, s, m, n);
      const int kb0 = kd::split_first_kblock(k_blocks, k_split, s);
      const int kb1 = kd::split_first_kblock(k_blocks, k_split, s + 1);
      if (w.u != expect_u || w.split != s || w.mb2 != m || w.nb != n || w.kb0 != kb0 ||
          w.kb1 != kb1 || s >= k_split || m >= m_tiles2 || n >= n_tiles || kb1 <= kb0) {
        std::printf("mismatch: m_tiles2=%d n_tiles=%d m_fastest=%d k_blocks=%d k_split=%d ncl=%d "
                    "cid=%d u=%d (walk: u=%d split=%d mb2=%d nb=%d kb=[%d,%d); direct: split=%d "
                    "mb2=%d nb=%d kb=[%d,%d))\n",
                    m_tiles2, n_tiles, m_fastest, k_blocks, k_split, ncl, cid, expect_u, w.u,
                    w.split, w.mb2, w.nb, w.kb0, w.kb1, s, m, n, kb0, kb1);
        return 1;
      }
      expect_u += ncl;
    }
    if (expect_u < units) {
      std::printf("walk stopped early: cid=%d at u=%d of %d\n", cid, expect_u, units);
      return 1;
    }
  }
  return 0;
}

int main() {
  // the launch shapes of the 32K head (chunk 2048): forward / dz, dH, dW
  if (check(8, 512, 1, 64, 1, 74) || check(8, 16, 1, 2048, 4, 74) || check(512, 16, 0, 64, 1, 74))
    return 1;
  // the large vocabulary (d = 2880 -> 12 column tiles, V = 201088 -> 786 tiles)
  if (check(8, 786, 1, 45, 1, 74) || check(8, 12, 1, 3142, 4, 74) || check(786, 12, 0, 64, 1, 74))
    return 1;
  // every small shape, split count and cluster count up to the unit count
  for (int mt = 1; mt <= 9; ++mt)
    for (int nt = 1; nt <= 11; ++nt)
      for (int mf = 0; mf <= 1; ++mf)
        for (int ks = 1; ks <= 4; ++ks)
          for (int kbl = ks; kbl <= ks + 6; kbl += 3) {
            const int units = mt * nt * ks;
            for (int ncl = 1; ncl <= units && ncl <= 80; ++ncl)
              if (check(mt, nt, mf, kbl, ks, ncl)) return 1;
          }
  std::printf("ok\n");
  return 0;
}
