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
//   order = longest first: FA units longer than any SA unit, then every SA
//           unit, then the remaining FA units, each run pair descending; at
//           one pair the entries go in list order, so the heads of one kv
//           group are adjacent and their K/V tiles are reused from L2.  For
//           long sequences (one kv head's K and V at least half the L2) the
//           long FA units instead go kv group by kv group (a sequence's kv
//           head and the query heads that read it): the CTAs running at any
//           moment then stream one or two groups' prefixes, which L2 holds.
//           Sequences of a batch may differ in length (EaSeqView).
//   deal  = dynamic: a CTA's producer warp takes the next rank from a
//           global ticket counter as it starts a unit, so no CTA waits on a
//           static share, and the units running at any moment stay adjacent
//           in the order.  The producer alone runs the cursor below and hands
//           each unit, decoded, to the other roles.
//   Measured at 256K tokens (32 query, 8 kv heads, d = 128, 24 of 32 heads
//   SA; one B200): dealt statically in a snake, the CTAs drifted apart and
//   DRAM reads were ~70x one pass over q, k, v; dealt dynamically, ~44x;
//   with the long FA units by kv group as well, ~1.4x and 8% less time.  At
//   192K tokens by group was 4% faster; at 16K-64K tokens by pair was as fast
//   or faster (up to 7%).
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

// Batches of sequences of different lengths (packed varlen batches; a
// padded batch is the case where every length is the same).  Sequences are
// viewed sorted by unit count, longest first (ties by index), and every entry
// list (FA entries, then SA entries) is grouped by sorted sequence, heads in
// order inside a sequence.  The units at pair p are then the entries of the
// sequences that have more than p units: a prefix of each list.
#define EA_MAX_SEQS 1024

struct EaSeqView {
  int nseq;                // sequences
  const int16_t* P;        // [nseq] unit count of the k-th sorted sequence, non-increasing
  const int32_t* prefFA;   // [nseq + 1] FA entries of sorted positions < k
  const int32_t* prefSA;   // [nseq + 1] SA entries of sorted positions < k
  int Pmax;                // P[0] (0 for an empty batch)
  int pA;                  // FA units with pair >= pA are longer than any SA unit
};

// pA for a batch: an interior SA unit visits at most sa_cap tiles; FA unit
// of pair p visits min(2p + 2, its tile count), longer than sa_cap when
// p >= floor(sa_cap / 2).
EA_HD int ea_split_pair(int S, int W, int Pmax) {
  const int sa_cap = ea_cdiv(S, EA_BN) + 2 + ea_cdiv(W - 1, EA_BN);
  return ea_min(sa_cap / 2, Pmax);
}

// K and V elements of one kv head (of the longest sequence, in whole units)
// from which the long FA units go kv group by kv group: 2 * 131072 * 128,
// 64 MB of bf16 K and V, half the L2.
#define EA_GROUP_MAJOR_ELEMS (1ll << 25)

EA_HD bool ea_group_major(int Pmax, int d) {
  return 2ll * Pmax * EA_UNIT_ROWS * d >= EA_GROUP_MAJOR_ELEMS;
}

// Order (longest first): FA units with pair >= pA, then every SA unit (pair
// descending), then the FA units with pair < pA (pair descending); inside
// one (phase, pair), entries in list order.  The long FA units go pair
// descending the same way, or, group-major, kv group by kv group: the
// groups in (sorted sequence, kv head) order, a group's units pair
// descending, its heads in order inside a pair.  A group's FA entries are a
// contiguous run of the FA list (grouped by sorted sequence, heads
// increasing).  A cursor walks the order; ranks must be asked in increasing
// order.
struct EaCursor {
  int phase;   // 0: long FA, 1: SA, 2: short FA, 3: past the end
  int p;       // pair
  int base;    // rank of the first unit at (phase, p), or of the group
  int cnt;     // units at (phase, p), or of the group
  int m;       // sorted sequences with more than p units
  // phase 0, group-major
  int gm;      // 1: the long FA units go kv group by kv group
  int Hq, G, Hkv;
  int k, hk;   // the group: sorted sequence position, kv head
  int fa0, nf; // its FA entries: list positions [fa0, fa0 + nf)
  int fa_end;  // scan position in the sequence's FA run
};

EA_HD int ea_phase_top(const EaSeqView& v, int phase) {
  return phase == 2 ? v.pA - 1 : v.Pmax - 1;
}
EA_HD int ea_phase_bottom(const EaSeqView& v, int phase) { return phase == 0 ? v.pA : 0; }

EA_HD void ea_cursor_settle(EaCursor& c, const EaSeqView& v) {
  while (c.phase < 3 && c.p < ea_phase_bottom(v, c.phase)) {
    ++c.phase;
    c.p = ea_phase_top(v, c.phase);
    c.m = 0;
  }
  if (c.phase >= 3) {
    c.cnt = 0;
    return;
  }
  while (c.m < v.nseq && v.P[c.m] > c.p) ++c.m;
  c.cnt = (c.phase == 1 ? v.prefSA : v.prefFA)[c.m];
}

// Group-major phase 0: the next kv group with long FA units, or phase 1.
template <class T>
EA_HD void ea_cursor_next_group(EaCursor& c, const EaSeqView& v, const T* ent) {
  for (;;) {
    if (++c.hk >= c.Hkv) {
      c.hk = 0;
      ++c.k;
    }
    if (c.k >= v.nseq) {
      c.phase = 1;
      c.p = ea_phase_top(v, 1);
      c.m = 0;
      ea_cursor_settle(c, v);
      return;
    }
    if (c.hk == 0) c.fa_end = v.prefFA[c.k];   // a new sequence: its FA run
    int a = c.fa_end;
    const int e = v.prefFA[c.k + 1];
    while (a < e && (static_cast<int>(ent[a]) % c.Hq) / c.G < c.hk) ++a;
    int b = a;
    while (b < e && (static_cast<int>(ent[b]) % c.Hq) / c.G == c.hk) ++b;
    c.fa0 = a;
    c.nf = b - a;
    c.fa_end = b;
    c.cnt = c.nf * ea_max(v.P[c.k] - v.pA, 0);
    if (c.cnt > 0) return;
  }
}

// ent: the entry lists (FA entries, then SA entries), read by the
// group-major walk only.
template <class T>
EA_HD void ea_cursor_init(EaCursor& c, const EaSeqView& v, const T* ent, int Hq, int Hkv,
                          bool group_major) {
  c.phase = 0;
  c.p = ea_phase_top(v, 0);
  c.base = 0;
  c.m = 0;
  c.gm = group_major ? 1 : 0;
  c.Hq = Hq;
  c.Hkv = Hkv;
  c.G = Hq / Hkv;
  c.k = 0;
  c.hk = -1;
  c.fa0 = c.nf = c.fa_end = 0;
  if (c.gm && v.nseq > 0 && v.pA < v.Pmax) {
    ea_cursor_next_group(c, v, ent);
  } else {
    ea_cursor_settle(c, v);
  }
}

// Unit of rank r: (sparse, entry index within its list, pair); false past
// the end.
template <class T>
EA_HD bool ea_cursor_seek(EaCursor& c, const EaSeqView& v, const T* ent, int r, int* sparse,
                          int* e, int* pair) {
  while (c.phase < 3 && r >= c.base + c.cnt) {
    c.base += c.cnt;
    if (c.phase == 0 && c.gm) {
      ea_cursor_next_group(c, v, ent);
    } else {
      --c.p;
      ea_cursor_settle(c, v);
    }
  }
  if (c.phase >= 3) return false;
  const int u = r - c.base;
  if (c.phase == 0 && c.gm) {
    *sparse = 0;
    *e = c.fa0 + u % c.nf;
    *pair = v.P[c.k] - 1 - u / c.nf;
    return true;
  }
  *sparse = c.phase == 1;
  *e = u;
  *pair = c.p;
  return true;
}

EA_HD int ea_total_units(const EaSeqView& v) {
  int total = 0;
  for (int k = 0; k < v.nseq; ++k)
    total += v.P[k] * ((v.prefFA[k + 1] - v.prefFA[k]) + (v.prefSA[k + 1] - v.prefSA[k]));
  return total;
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
