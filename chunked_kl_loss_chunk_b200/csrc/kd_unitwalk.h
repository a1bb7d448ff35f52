// kd_unitwalk.h -- the sequence of work units one cluster of a persistent GEMM
// grid takes, walked without integer division.
//
// A GEMM launch is a list of units u = 0 .. units-1, each one (K range
// `split`, tile row block mb2, tile column block nb).  Unit u lies in split
// u / per_split (per_split = m_tiles2 * n_tiles); inside it, position
// t = u mod per_split is laid out with the row block varying fastest
// (m_fastest) or the column block varying fastest.  Cluster cid takes units
// cid, cid + ncl, cid + 2 ncl, ...
//
// Finding a unit's coordinates from u costs three integer divisions, and the
// split's K range a 64-bit one.  The MMA-issuing thread pays for them between
// two units while the tensor pipe drains, so they are paid once, at the first
// unit.  After that, each step adds ncl, split once into the raster's two
// digits, with one carry, and the split's K range is recomputed only when
// the split changes.
//
// This header compiles for the device (nvcc) and for the host, so the walk
// can be checked against the direct computation on a CPU.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define KD_HD __host__ __device__ __forceinline__
#else
#define KD_HD inline
#endif

namespace kd {

// Direct coordinates of unit u.
KD_HD void unit_coords_direct(int m_tiles2, int n_tiles, int m_fastest, int u, int& split,
                              int& mb2, int& nb) {
  const int per_split = m_tiles2 * n_tiles;
  split = u / per_split;
  const int t = u - split * per_split;
  mb2 = m_fastest ? t % m_tiles2 : t / n_tiles;
  nb = m_fastest ? t / m_tiles2 : t % n_tiles;
}

// First K block of split s of k_split even ranges over k_blocks blocks.
KD_HD int split_first_kblock(int k_blocks, int k_split, int s) {
  return static_cast<int>((static_cast<int64_t>(s) * k_blocks) / k_split);
}

struct UnitWalk {
  int u, split, mb2, nb;   // the current unit
  int kb0, kb1;            // its K blocks [kb0, kb1)
  int f, s;                // raster digits of u within its split: fast, slow
  int fast_n, slow_n;      // their extents
  int df, ds;              // ncl as raster digits
  int stride;              // ncl
  int m_fastest, k_blocks, k_split;
};

KD_HD void walk_set_coords(UnitWalk& w) {
  w.mb2 = w.m_fastest ? w.f : w.s;
  w.nb = w.m_fastest ? w.s : w.f;
}

// The walk of cluster cid among ncl clusters.
KD_HD void walk_begin(UnitWalk& w, int m_tiles2, int n_tiles, int m_fastest, int k_blocks,
                      int k_split, int cid, int ncl) {
  w.m_fastest = m_fastest;
  w.k_blocks = k_blocks;
  w.k_split = k_split;
  w.stride = ncl;
  w.fast_n = m_fastest ? m_tiles2 : n_tiles;
  w.slow_n = m_fastest ? n_tiles : m_tiles2;
  w.df = ncl % w.fast_n;
  w.ds = ncl / w.fast_n;
  w.u = cid;
  unit_coords_direct(m_tiles2, n_tiles, m_fastest, cid, w.split, w.mb2, w.nb);
  w.f = m_fastest ? w.mb2 : w.nb;
  w.s = m_fastest ? w.nb : w.mb2;
  w.kb0 = split_first_kblock(k_blocks, k_split, w.split);
  w.kb1 = split_first_kblock(k_blocks, k_split, w.split + 1);
}

// Advance to the cluster's next unit (u += ncl).
KD_HD void walk_next(UnitWalk& w) {
  w.u += w.stride;
  w.f += w.df;
  w.s += w.ds;
  if (w.f >= w.fast_n) {
    w.f -= w.fast_n;
    ++w.s;
  }
  if (w.s >= w.slow_n) {
    do {
      w.s -= w.slow_n;
      ++w.split;
    } while (w.s >= w.slow_n);
    w.kb0 = split_first_kblock(w.k_blocks, w.k_split, w.split);
    w.kb1 = split_first_kblock(w.k_blocks, w.k_split, w.split + 1);
  }
  walk_set_coords(w);
}

}  // namespace kd
