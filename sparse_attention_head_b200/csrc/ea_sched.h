// ea_sched.h — work decomposition of the fused hybrid attention kernel.
//
// Shared by the device kernel and the host-side inspection entry points, so
// the CPU tests see exactly the schedule the GPU runs.
//
// Elastic Attention blog §3 ("Fused Kernel"): the routing bits enter the
// kernel as metadata and a per-thread-block branch lets one launch run FA
// heads and SA heads together.  Here the branch is taken per work unit:
//
//   unit  = (mode, b, h, pair): query rows [256*pair, 256*pair + 256) of one
//           head, split in two 128-row slots that share every K/V tile load.
//   tiles = the 128-key KV tiles the unit visits.  FA: 0..last.  SA: the sink
//           tiles [0, ceil(S/128)) and the window tiles [lo, last], where lo
//           is the tile of the first row's window start.
//   order = longest first: FA units longer than any SA unit (largest pair
//           first), then every SA unit, then the remaining FA units; inside
//           one pair index the heads of one kv group are adjacent, so their
//           K/V tiles are reused from L2.
//   deal  = rank r goes to CTA c in a snake: round k = r / G covers ranks
//           [kG, kG+G) left to right when k is even, right to left when odd.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define EA_HD __host__ __device__ __forceinline__
#else
#define EA_HD static inline
#endif

#define EA_BM 128          // query rows per slot
#define EA_BN 128          // keys per KV tile
#define EA_UNIT_ROWS 256   // query rows per unit (two slots)
#define EA_MAX_ENTRIES 4096

struct EaShape {
  int N, S, W;
  int P;        // units per head: ceil(N / 256)
  int nT;       // KV tiles per head: ceil(N / 128)
  int sa_cap;   // upper bound of an SA unit's tile count
  int pA;       // FA units with pair >= pA are longer than sa_cap
};

EA_HD int ea_cdiv(int a, int b) { return (a + b - 1) / b; }
EA_HD int ea_min(int a, int b) { return a < b ? a : b; }
EA_HD int ea_max(int a, int b) { return a > b ? a : b; }

EA_HD EaShape ea_make_shape(int N, int S, int W) {
  EaShape s;
  s.N = N; s.S = S; s.W = W;
  s.P = ea_cdiv(N, EA_UNIT_ROWS);
  s.nT = ea_cdiv(N, EA_BN);
  // An interior SA unit visits ceil(S/128) sink tiles and at most
  // 2 + ceil((W-1)/128) window tiles.
  s.sa_cap = ea_cdiv(S, EA_BN) + 2 + ea_cdiv(W - 1, EA_BN);
  // FA unit of pair p visits min(2p + 2, nT) tiles; it is "long" when that
  // exceeds sa_cap, i.e. p >= pA.
  // 2p + 2 > sa_cap  <=>  p >= floor(sa_cap / 2)
  s.pA = ea_min(s.sa_cap / 2, s.P);
  return s;
}

// Unit rank -> (sparse, entry index within its list, pair).
EA_HD void ea_unit_of_rank(const EaShape& s, int nFA, int nSA, int r,
                           int* sparse, int* e, int* pair) {
  int nA = nFA * (s.P - s.pA);
  if (r < nA) {
    *sparse = 0; *pair = s.P - 1 - r / nFA; *e = r % nFA; return;
  }
  r -= nA;
  int nB = nSA * s.P;
  if (r < nB) {
    *sparse = 1; *pair = s.P - 1 - r / nSA; *e = r % nSA; return;
  }
  r -= nB;
  *sparse = 0; *pair = s.pA - 1 - r / nFA; *e = r % nFA;
}

EA_HD int ea_num_units(const EaShape& s, int nFA, int nSA) {
  return (nFA + nSA) * s.P;
}

// k-th rank dealt to CTA c of G (or -1 past the end).
EA_HD int ea_rank_for(int k, int c, int G, int total) {
  int r = k * G + ((k & 1) ? (G - 1 - c) : c);
  return r < total ? r : -1;
}

// Tile list of one unit: [0, a) then [lo, last].
struct EaUnitTiles {
  int r0;        // first query row of slot 0
  int nslots;    // 1 or 2 valid slots
  int a, lo, last, n;
};

EA_HD EaUnitTiles ea_unit_tiles(const EaShape& s, int sparse, int pair) {
  EaUnitTiles t;
  t.r0 = pair * EA_UNIT_ROWS;
  t.nslots = (t.r0 + EA_BM < s.N) ? 2 : 1;
  int imax = ea_min(t.r0 + EA_BM * t.nslots - 1, s.N - 1);
  t.last = imax / EA_BN;
  if (!sparse) {
    t.a = 0; t.lo = 0;
  } else {
    t.lo = ea_max(0, t.r0 - s.W + 1) / EA_BN;
    t.a = ea_min(ea_min(ea_cdiv(s.S, EA_BN), t.lo), t.last + 1);
  }
  t.n = t.a + (t.last - t.lo + 1);
  return t;
}

EA_HD int ea_tile_at(const EaUnitTiles& t, int i) {
  return i < t.a ? i : t.lo + (i - t.a);
}

// Code of (slot, tile): 0 = no visible pair, 1 = all pairs visible,
// 2 = needs the element mask.  Rows past N count as rows of the slot; their
// outputs are never stored.
EA_HD int ea_tile_code(const EaShape& s, const EaUnitTiles& t, int sparse,
                       int slot, int tile) {
  if (slot >= t.nslots) return 0;
  int r0 = t.r0 + slot * EA_BM;
  int imax = ea_min(r0 + EA_BM - 1, s.N - 1);
  int c0 = tile * EA_BN;
  bool any = (c0 <= imax) &&
             (!sparse || c0 < s.S || (r0 - (c0 + EA_BN - 1)) < s.W);
  if (!any) return 0;
  bool full = (c0 + EA_BN - 1 <= r0) &&
              (!sparse || (c0 + EA_BN - 1) < s.S || (r0 + EA_BM - 1 - c0) < s.W);
  return full ? 1 : 2;
}
