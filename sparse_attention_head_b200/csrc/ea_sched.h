// ea_sched.h — work decomposition of the fused hybrid attention kernel.
//
// Shared by the device kernel and the host-side inspection entry points, so
// the CPU tests see exactly the schedule the GPU runs.
//
// Elastic Attention blog §3 ("Fused Kernel"): the routing bits enter the
// kernel as metadata and a per-thread-block branch lets one launch run FA
// heads and SA heads together.  Here the branch is taken per work unit, and
// a unit's two 128-row query slots share every K/V tile the unit loads:
//
//   unit  = two slots.  A paired unit holds two query heads of one kv group
//           with the same route, at the same 128 rows [128 m, 128 m + 128)
//           (grouped-query attention: both heads read the same K/V tiles, so
//           each tile in shared memory serves two heads).  A kv group's heads
//           of one mode are taken two by two in head order; an odd one out
//           (and every head when a group has more than 32) runs as a single
//           unit: one head, rows [256 p, 256 p + 256), slot 1 the upper half.
//   level = m: a paired unit's block; 2p + 1 for a single unit of pair p.
//           A unit's K/V tile count grows with its level.
//   tiles = the 128-key KV tiles the unit visits.  FA: 0..last.  SA: the sink
//           tiles [0, ceil(S/128)) and the window tiles [lo, last], where lo
//           is the tile of the unit's first row's window start.
//   order = longest first: FA units longer than any SA unit, then every SA
//           unit, then the remaining FA units, each run level descending; at
//           one level the paired units, then the single units, entries in
//           list order, so the heads of one kv group are adjacent and their
//           K/V tiles are reused from L2.  For long sequences (one kv head's K
//           and V at least half the L2) the long FA units instead go kv group
//           by kv group (a sequence's kv head and the query heads that read
//           it): the CTAs running at any moment then stream one or two
//           groups' prefixes, which L2 holds.  Sequences of a batch may
//           differ in length (EaSeqView).
//   deal  = dynamic: a CTA's producer warp takes the next rank from a
//           global ticket counter as it starts a unit, so no CTA waits on a
//           static share, and the units running at any moment stay adjacent
//           in the order.  The producer alone runs the cursor below and hands
//           each unit, decoded, to the other roles.
//   Measured at 256K tokens (32 query, 8 kv heads, d = 128, 24 of 32 heads
//   SA; one B200): dealt statically in a snake, the CTAs drifted apart and
//   DRAM reads were ~70x one pass over q, k, v; dealt dynamically, ~44x;
//   with the long FA units by kv group as well, ~1.7x and 8% less time.  At
//   192K tokens by group was 4% faster; at 16K-64K tokens by level was as
//   fast or faster (up to 7%).
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define EA_HD __host__ __device__ __forceinline__
#else
#define EA_HD static inline
#endif

#define EA_BM 128          // query rows per slot
#define EA_BN 128          // keys per KV tile
#define EA_UNIT_ROWS 256   // query rows of a single-head unit (two slots)
#define EA_MAX_ENTRIES 4096
#define EA_MAX_PAIR_GROUP 32   // kv groups of more query heads run single units only

struct EaShape {
  int N, S, W;
  int P;        // single units per head: ceil(N / 256)
  int nT;       // 128-row blocks and KV tiles per head: ceil(N / 128)
};

EA_HD int ea_cdiv(int a, int b) { return (a + b - 1) / b; }
EA_HD int ea_min(int a, int b) { return a < b ? a : b; }
EA_HD int ea_max(int a, int b) { return a > b ? a : b; }

EA_HD EaShape ea_make_shape(int N, int S, int W) {
  EaShape s;
  s.N = N; s.S = S; s.W = W;
  s.P = ea_cdiv(N, EA_UNIT_ROWS);
  s.nT = ea_cdiv(N, EA_BN);
  return s;
}

// An SA unit visits at most ceil(S/128) sink tiles and 2 + ceil((W-1)/128)
// window tiles; an FA unit at level m visits up to m + 1 tiles, so the FA
// units of level >= mA are longer than any SA unit.
EA_HD int ea_long_level(int S, int W) {
  return ea_cdiv(S, EA_BN) + 2 + ea_cdiv(W - 1, EA_BN);
}

// Batches of sequences of different lengths (packed varlen batches; a
// padded batch is the case where every length is the same).  Sequences are
// viewed sorted by block count nT, longest first (ties by index), so nT and
// P = ceil(nT / 2) are both non-increasing.  The entry array holds heads
// (index b * Hq + h) in four runs: FA paired, FA single, SA paired, SA
// single; a paired entry is two consecutive heads.  Each run is grouped by
// sorted sequence, kv groups in order, heads increasing.  The units at level
// m are then, per run, the entries of a prefix of the sorted sequences.
#define EA_MAX_SEQS 1024

struct EaSeqView {
  int nseq;                // sequences
  const int16_t* nT;       // [nseq] blocks of the k-th sorted sequence, non-increasing
  const int16_t* P;        // [nseq] ceil(nT / 2)
  const int16_t* pref[4];  // [nseq + 1] entries of run j from sorted positions < k
  int run0[4];             // first head position of run j in the entry array
  int Pmax;                // P[0] (0 for an empty batch)
  int mA;                  // first long FA level
};

// Run j's prefix counts and first head position (selected with constant
// indices, so a device view's arrays stay in registers).
EA_HD const int16_t* ea_pref(const EaSeqView& v, int j) {
  return j == 0 ? v.pref[0] : j == 1 ? v.pref[1] : j == 2 ? v.pref[2] : v.pref[3];
}
EA_HD int ea_run0(const EaSeqView& v, int j) {
  return j == 0 ? v.run0[0] : j == 1 ? v.run0[1] : j == 2 ? v.run0[2] : v.run0[3];
}

EA_HD int ea_total_units(const EaSeqView& v) {
  int total = 0;
  for (int k = 0; k < v.nseq; ++k) {
    const int np = (v.pref[0][k + 1] - v.pref[0][k]) + (v.pref[2][k + 1] - v.pref[2][k]);
    const int ns = (v.pref[1][k + 1] - v.pref[1][k]) + (v.pref[3][k + 1] - v.pref[3][k]);
    total += np * v.nT[k] + ns * v.P[k];
  }
  return total;
}

// K and V elements of one kv head (of the longest sequence, in whole single
// units) from which the long FA units go kv group by kv group: 2 * 131072 *
// 128, 64 MB of bf16 K and V, half the L2.
#define EA_GROUP_MAJOR_ELEMS (1ll << 25)

EA_HD bool ea_group_major(int Pmax, int d) {
  return 2ll * Pmax * EA_UNIT_ROWS * d >= EA_GROUP_MAJOR_ELEMS;
}

// A unit as the cursor yields it.
struct EaUnitRef {
  int sparse;   // 0 FA, 1 SA
  int paired;   // 1: two heads at one block; 0: one head at a pair of blocks
  int pos;      // head position in the entry array (a paired unit: pos, pos + 1)
  int level;    // m
};

// Order (longest first): FA units of level >= mA, then every SA unit, then
// the FA units of level < mA, each run level descending; at one level the
// paired units, then the single units (single units sit at odd levels only),
// entries in list order.  The long FA units go level by level the same way,
// or, group-major, kv group by kv group: the groups in (sorted sequence, kv
// head) order, a group's units level descending, at one level its paired
// units, then its single unit.  A cursor walks the order; ranks must be
// asked in increasing order.
struct EaCursor {
  int phase;    // 0: long FA, 1: SA, 2: short FA, 3: past the end
  int m;        // level
  int base;     // rank of the first unit at the level
  int np, ns;   // paired and single units at the level
  int kp, ks;   // sorted sequences with nT > m, with 2 P > m
  // phase 0, group-major: the scope is one kv group
  int gm;       // 1: the long FA units go kv group by kv group
  int Hq, G, Hkv;
  int k, hk;    // the group: sorted sequence position, kv head
  int gp0, gnp; // its paired FA entries: run 0 entries [gp0, gp0 + gnp)
  int gs0, gns; // its single FA entries: run 1 entries [gs0, gs0 + gns)
  int gend_p, gend_s;   // scan positions in the sequence's runs
};

EA_HD int ea_phase_top(const EaSeqView& v, int phase) {
  const int top = 2 * v.Pmax - 1;
  return phase == 2 ? ea_min(v.mA - 1, top) : top;
}
EA_HD int ea_phase_bottom(const EaSeqView& v, int phase) { return phase == 0 ? v.mA : 0; }

EA_HD void ea_cursor_settle(EaCursor& c, const EaSeqView& v) {
  while (c.phase < 3 && c.m < ea_phase_bottom(v, c.phase)) {
    ++c.phase;
    c.m = ea_phase_top(v, c.phase);
    c.kp = c.ks = 0;
  }
  if (c.phase >= 3) {
    c.np = c.ns = 0;
    return;
  }
  // m only falls inside a phase: the prefixes only grow
  while (c.kp < v.nseq && v.nT[c.kp] > c.m) ++c.kp;
  while (c.ks < v.nseq && 2 * v.P[c.ks] > c.m) ++c.ks;
  const int jp = c.phase == 1 ? 2 : 0;
  c.np = ea_pref(v, jp)[c.kp];
  c.ns = (c.m & 1) ? ea_pref(v, jp + 1)[c.ks] : 0;
}

// Group-major phase 0: the current group's units at level m.
EA_HD void ea_cursor_group_level(EaCursor& c, const EaSeqView& v) {
  c.np = c.m < v.nT[c.k] ? c.gnp : 0;
  c.ns = (c.m & 1) ? c.gns : 0;
}

// Kv group of the head at position pos of the entry array.
template <class T>
EA_HD int ea_group_of(const EaCursor& c, const T* ent, int pos) {
  return (static_cast<int>(ent[pos]) % c.Hq) / c.G;
}

// Group-major phase 0: the next kv group with long FA units (at its top
// level), or the SA phase.
template <class T>
EA_HD void ea_cursor_next_group(EaCursor& c, const EaSeqView& v, const T* ent) {
  for (;;) {
    if (++c.hk >= c.Hkv) {
      c.hk = 0;
      ++c.k;
    }
    if (c.k >= v.nseq) {
      c.phase = 1;
      c.m = ea_phase_top(v, 1);
      c.kp = c.ks = 0;
      ea_cursor_settle(c, v);
      return;
    }
    if (c.hk == 0) {   // a new sequence: its runs
      c.gend_p = v.pref[0][c.k];
      c.gend_s = v.pref[1][c.k];
    }
    int a = c.gend_p, e = v.pref[0][c.k + 1];
    while (a < e && ea_group_of(c, ent, v.run0[0] + 2 * a) < c.hk) ++a;
    int b = a;
    while (b < e && ea_group_of(c, ent, v.run0[0] + 2 * b) == c.hk) ++b;
    c.gp0 = a;
    c.gnp = b - a;
    c.gend_p = b;
    a = c.gend_s;
    e = v.pref[1][c.k + 1];
    while (a < e && ea_group_of(c, ent, v.run0[1] + a) < c.hk) ++a;
    b = a;
    while (b < e && ea_group_of(c, ent, v.run0[1] + b) == c.hk) ++b;
    c.gs0 = a;
    c.gns = b - a;
    c.gend_s = b;
    for (c.m = 2 * v.P[c.k] - 1; c.m >= v.mA; --c.m) {
      ea_cursor_group_level(c, v);
      if (c.np + c.ns > 0) return;
    }
  }
}

// ent: the entry array, read by the group-major walk only.
template <class T>
EA_HD void ea_cursor_init(EaCursor& c, const EaSeqView& v, const T* ent, int Hq, int Hkv,
                          bool group_major) {
  c.phase = 0;
  c.m = ea_phase_top(v, 0);
  c.base = 0;
  c.kp = c.ks = 0;
  c.gm = group_major ? 1 : 0;
  c.Hq = Hq;
  c.Hkv = Hkv;
  c.G = Hq / Hkv;
  c.k = 0;
  c.hk = -1;
  c.gp0 = c.gnp = c.gs0 = c.gns = c.gend_p = c.gend_s = 0;
  if (c.gm && v.nseq > 0) {
    ea_cursor_next_group(c, v, ent);
  } else {
    ea_cursor_settle(c, v);
  }
}

// Unit of rank r; false past the end.
template <class T>
EA_HD bool ea_cursor_seek(EaCursor& c, const EaSeqView& v, const T* ent, int r, EaUnitRef* u) {
  while (c.phase < 3 && r >= c.base + c.np + c.ns) {
    c.base += c.np + c.ns;
    if (c.phase == 0 && c.gm) {
      for (;;) {
        if (--c.m < v.mA) {
          ea_cursor_next_group(c, v, ent);
          break;
        }
        ea_cursor_group_level(c, v);
        if (c.np + c.ns > 0) break;
      }
    } else {
      --c.m;
      ea_cursor_settle(c, v);
    }
  }
  if (c.phase >= 3) return false;
  const int i = r - c.base;
  const bool group = c.phase == 0 && c.gm;
  const int jp = c.phase == 1 ? 2 : 0;
  u->sparse = c.phase == 1;
  u->level = c.m;
  if (i < c.np) {
    u->paired = 1;
    u->pos = ea_run0(v, jp) + 2 * ((group ? c.gp0 : 0) + i);
  } else {
    u->paired = 0;
    u->pos = ea_run0(v, jp + 1) + (group ? c.gs0 : 0) + (i - c.np);
  }
  return true;
}

// Rows and tile list of one unit: slot s holds rows [r0 + s * rstep, +128);
// the tiles are [0, a) then [lo, last].
struct EaUnitTiles {
  int r0;        // first query row of slot 0
  int rstep;     // 0: both slots at r0 (two heads); 128: slot 1 is the next block
  int nslots;    // 1 or 2 valid slots
  int a, lo, last, n;
};

EA_HD EaUnitTiles ea_unit_tiles(const EaShape& s, int sparse, int paired, int level) {
  EaUnitTiles t;
  int imax;
  if (paired) {
    t.r0 = level * EA_BM;
    t.rstep = 0;
    t.nslots = 2;
    imax = ea_min(t.r0 + EA_BM - 1, s.N - 1);
  } else {
    t.r0 = (level >> 1) * EA_UNIT_ROWS;
    t.rstep = EA_BM;
    t.nslots = (t.r0 + EA_BM < s.N) ? 2 : 1;
    imax = ea_min(t.r0 + EA_BM * t.nslots - 1, s.N - 1);
  }
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
  int r0 = t.r0 + slot * t.rstep;
  int imax = ea_min(r0 + EA_BM - 1, s.N - 1);
  int c0 = tile * EA_BN;
  bool any = (c0 <= imax) &&
             (!sparse || c0 < s.S || (r0 - (c0 + EA_BN - 1)) < s.W);
  if (!any) return 0;
  bool full = (c0 + EA_BN - 1 <= r0) &&
              (!sparse || (c0 + EA_BN - 1) < s.S || (r0 + EA_BM - 1 - c0) < s.W);
  return full ? 1 : 2;
}
