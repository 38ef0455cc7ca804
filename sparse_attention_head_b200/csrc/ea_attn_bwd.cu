// ea_attn_bwd.cu — backward pass of the hybrid FA/SA attention (training).
//
// Elastic Attention blog §2.1 (training trick): the router is trained with a
// Gumbel-Softmax straight-through estimator, so the attention of the mode a
// head routes to receives the output gradient dO and must return dQ, dK, dV.
// With P = softmax(scale q k^T | visible) per head (FA: causal; SA: sink S +
// window W), L = sum(dO * O):
//   D_i = sum_c dO_ic O_ic,  dP = dO V^T,  dS = P * (dP - D),
//   dV = P^T dO,  dK = scale dS^T Q,  dQ = scale dS K,
// a kv head's dK, dV summed over its query heads (GQA).  P is recomputed from
// the forward's log-sum-exp: P = 2^(s * scale * log2e - lse * log2e).
//
// Four launches on the caller's stream:
//   1. ea_bwd_rowdot_kernel: D = rowsum(dO * O), fp32 (HBM-bound);
//   2. ea_bwd_sched_kernel: the units of the two kernels below sorted by
//      cost and assigned to CTAs (longest first; for dK/dV each to the
//      least-loaded CTA), as per-CTA lists in the workspace;
//   3. ea_bwd_dkdv_kernel: unit = (b, kv head, 128-key tile j).  K_j and V_j
//      stay in shared memory; the steps visit (query head of the group,
//      128-query tile i) pairs that see tile j.  Per step the tensor cores
//      compute S^T = K_j Q_i^T and dP^T = V_j dO_i^T into TMEM, eight warps
//      (two column halves of four) turn them into P^T and dS^T (bf16, back
//      into TMEM), and dV += P^T dO_i, dK += dS^T Q_i accumulate in TMEM (A
//      from TMEM).  The elementwise work runs in two phases (P from S while
//      dP is computed; dS from dP while dV and the next S are), so the
//      tensor pipe and the elementwise warps overlap.
//   4. ea_bwd_dq_kernel: unit = (b, head, 128-query tile i); the steps visit
//      the key tiles the forward visits: S = Q_i K_j^T, dP = dO_i V_j^T, dS,
//      dQ += dS K_j.
// Both are persistent (one CTA per SM), with a TMA producer warp, one MMA
// issuing thread and eight elementwise warps; every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ea.h"
#include "ea_internal.h"
#include "ea_math.cuh"
#include "ea_ptx.cuh"
#include "ea_sched.h"
#include "ea_tmem.cuh"

namespace ea {

// D[row] = sum_c dO[row][c] * O[row][c] over rows of [rows][d] (d = 128):
// 16 lanes per row with 16-byte loads (two rows per warp step), the 16
// partial sums reduced by xor shuffles in a fixed order.  Rows are visited as
// (b*Hq + h, q) over q < npad: for q < N the kernel writes D to dvec and, for
// the dK/dV kernel's bulk copies, -D to vd_pad and -lse * log2(e) to vl_pad;
// the padding (q >= N) gets zeros there.
__global__ void ea_bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ dout,
                                     const __nv_bfloat16* __restrict__ out,
                                     const float* __restrict__ lse, int bh_count, int N, int npad,
                                     int d, float* __restrict__ dvec, float* __restrict__ vl_pad,
                                     float* __restrict__ vd_pad) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long prow = t >> 4;                   // padded row: bh * npad + q
  const int c0 = static_cast<int>(t & 15) * 8;
  const bool in_range = prow < static_cast<long long>(bh_count) * npad;
  const int bh = in_range ? static_cast<int>(prow / npad) : 0;
  const int q = in_range ? static_cast<int>(prow % npad) : 0;
  const bool valid = in_range && q < N;
  const size_t row = static_cast<size_t>(bh) * N + q;
  float s = 0.f;
  if (valid) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(dout + row * d + c0));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(out + row * d + c0));
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      s = fmaf(__uint_as_float(wa[j] << 16), __uint_as_float(wb[j] << 16), s);
      s = fmaf(__uint_as_float(wa[j] & 0xffff0000u), __uint_as_float(wb[j] & 0xffff0000u), s);
    }
  }
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if ((t & 15) == 0 && in_range) {
    if (valid) {
      dvec[row] = s;
      vd_pad[prow] = -s;
      vl_pad[prow] = -lse[row] * 1.4426950408889634f;
    } else {
      vd_pad[prow] = 0.f;
      vl_pad[prow] = 0.f;
    }
  }
}

// Shared-memory plan of both backward kernels (d = 128).  The streamed
// operands come in two rings: tile 0 (kDkDv: Q_i; else K_j) is read by a
// step's first score product and, one phase later, by its last accumulating
// product, and the next step's first score product needs the next tile 0
// while the current one is still in use, so its ring has three slots; tile 1
// (kDkDv: dO_i; else V_j) is needed later in the step and has two.  The small
// data (per-step vectors, step descriptors, barriers) comes first and the
// tiles start 1024-aligned after it, which fills the 227 KB exactly; the
// kernel requires a 1024-aligned dynamic shared-memory base (checked).
struct BwdCfg {
  static constexpr int D = 128;
  static constexpr int kThreads = 320;           // warps 0-7 elementwise, 8 producer, 9 MMA
  static constexpr int kBlockBytes = 128 * 128;  // 128 rows x 64 bf16 (one SW128 column block)
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kStages0 = 3;             // ring of streamed tile 0
  static constexpr int kStages1 = 2;             // ring of streamed tile 1
  // kDkDv: -lse * log2e of the step's 128 query rows per tile-0 slot, and -D
  // per tile-1 slot (f32)
  static constexpr int kOffVec0 = 0;
  static constexpr int kOffVec1 = kOffVec0 + kStages0 * 128 * 4;
  static constexpr int kOffStep = kOffVec1 + kStages1 * 128 * 4;  // descriptors per tile-0 slot
  static constexpr int kOffBar = kOffStep + kStages0 * 32;
  // res_full, res_empty, full0[kStages0], empty0[kStages0], full1[kStages1],
  // empty1[kStages1], s_full, dp_full, p_full, ds_full, acc_done, acc_empty,
  // drain
  static constexpr int kNumBars = 2 + 2 * kStages0 + 2 * kStages1 + 7;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;    // tmem base, abort flag
  static constexpr int kOffTiles = 3072;
  static constexpr int kOffRes = kOffTiles;                  // 2 resident tiles
  static constexpr int kOffSt0 = kOffRes + 2 * kTileBytes;
  static constexpr int kOffSt1 = kOffSt0 + kStages0 * kTileBytes;
  static constexpr int kSmem = kOffSt1 + kStages1 * kTileBytes;
  static constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 128, 0, 0);  // both K-major
  static constexpr uint32_t kIdescTS = idesc_bf16_f32(128, D, 0, 1);    // B MN-major
  // of every 8 pairs of exponentials in the P phase, this many go to the
  // FMA-pipe polynomial instead of the MUFU
  static constexpr int kEmuPairs = 2;
  static_assert(kOffMisc + 64 <= kOffTiles, "small data overlaps the tiles");
  static_assert(kOffTiles % 1024 == 0, "tiles must be 1024-aligned");
  static_assert(kSmem <= 232448, "shared memory per CTA");
};

// Query tiles that see key tile jt for a head of mode sa: [jt, last].  FA:
// every later query; SA: every later query while the tile holds sink keys,
// else the queries within the window of the tile's first key.
__device__ __forceinline__ int bwd_last_query_tile(int jt, bool sa, int nT, int sink, int window) {
  if (!sa || jt * EA_BN < sink) return nT - 1;
  return min(nT - 1, (jt * EA_BN + EA_BN - 1 + window - 1) / EA_BM);
}

// Key tiles query tile it visits (as the forward): [0, a) then [lo, it].
__device__ __forceinline__ void bwd_key_tiles(int it, bool sa, int sink, int window, int* a,
                                              int* lo) {
  if (!sa) {
    *a = 0;
    *lo = 0;
    return;
  }
  *lo = max(0, it * EA_BM - window + 1) / EA_BN;
  *a = min(ea_cdiv(sink, EA_BN), *lo);
}

// Is key k visible from query q (global indices) for a head of mode sa?
__device__ __forceinline__ bool bwd_visible(int q, int k, int N, bool sa, int sink, int window) {
  return q < N && k <= q && (!sa || k < sink || q - k < window);
}

// Step descriptor of a stage, written by the producer before it arms the
// stage's full barrier.
struct BwdStep {
  int b, h, it, jt;   // batch row, query head, query tile, key tile
  int sa;             // head routes to SA
  int first, last;    // first / last step of the unit
  int full;           // every (query, key) pair of the block is visible
};

// Every pair of (query tile it, key tile jt) visible, for a head of mode sa?
__device__ __forceinline__ bool bwd_block_full(int it, int jt, int N, bool sa, int sink,
                                               int window) {
  const int q0 = it * EA_BM, q1 = q0 + EA_BM - 1, k0 = jt * EA_BN, k1 = k0 + EA_BN - 1;
  if (!(k1 <= q0 && q1 < N)) return false;
  return !sa || k1 < sink || q1 - k0 < window;
}



// ---------------------------------------------------------------- phases
// P phase of one thread's 64 columns (col0 ..): pr = 2^(s * sl2 + nl) on
// visible pairs and 0 elsewhere, and pk = the same as packed bf16 pairs.
// kDkDv: nl per column from vl (-lse * log2e of the column's query); else
// the row's own nl_row.  Visible columns c (0..127 within the tile): c in
// [lo_a, hi_a] and (c < sink_c or c >= win_c); kFull: every column.
template <bool kDkDv, bool kFull>
__device__ __forceinline__ void bwd_phase_p(uint32_t taddr, const float* vl, float nl_row,
                                            int col0, float sl2, int lo_a, int hi_a, int sink_c,
                                            int win_c, float (&pr)[64], uint32_t (&pk)[32]) {
  // visible columns col0 + lc (lc < 64) as 64 bits: lc in [lo_a, hi_a] and
  // (lc < sink_c or lc >= win_c), shifted by col0
  uint32_t vm[2] = {0xffffffffu, 0xffffffffu};
  if (!kFull) {
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int base = col0 + 32 * w;
      vm[w] = bits_below(hi_a + 1 - base) & ~bits_below(lo_a - base) &
              (bits_below(sink_c - base) | ~bits_below(win_c - base));
    }
  }
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    uint32_t sr[32];
    tmem_ld32_wait(taddr + 32 * ch, sr);
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      const int j = 16 * ch + jj;
      const int c = col0 + 2 * j;
      float x0, x1;
      if (kDkDv) {
        const float2 l2 = *reinterpret_cast<const float2*>(vl + c);
        x0 = l2.x;
        x1 = l2.y;
      } else {
        x0 = x1 = nl_row;
      }
      fma2_acc(x0, x1, __uint_as_float(sr[2 * jj]), __uint_as_float(sr[2 * jj + 1]), sl2, sl2);
      if ((j & 7) < BwdCfg::kEmuPairs) {
        exp2_poly2(x0, x1);
      } else {
        x0 = ex2_approx(x0);
        x1 = ex2_approx(x1);
      }
      if (!kFull) {
        // local column 2 j (and 2 j + 1) of this thread's 64: word ch, bits 2 jj, 2 jj + 1
        x0 = ((vm[ch] >> (2 * jj)) & 1u) ? x0 : 0.f;
        x1 = ((vm[ch] >> (2 * jj + 1)) & 1u) ? x1 : 0.f;
      }
      pr[2 * j] = x0;
      pr[2 * j + 1] = x1;
      pk[j] = pack_bf16x2(x0, x1);
    }
  }
}

// ---------------------------------------------------------------- units
// kDkDv: unit (b, kv head, key tile); else unit (b, head, query tile).  The
// index u enumerates them; the order in which CTAs run them is the
// schedule's (ea_bwd_sched_kernel below).
template <bool kDkDv>
__device__ __forceinline__ void bwd_unit_of(const BwdArgs& a, int u, int* b, int* hx, int* tile) {
  const int nT = ea_cdiv(a.N, EA_BN);
  if (kDkDv) {
    const int per = a.B * a.Hkv;
    *tile = u / per;
    *b = (u % per) / a.Hkv;
    *hx = (u % per) % a.Hkv;
  } else {
    const int per = a.B * a.Hq;
    *tile = nT - 1 - u / per;
    *b = (u % per) / a.Hq;
    *hx = (u % per) % a.Hq;
  }
}

// ---------------------------------------------------------------- schedule
// A unit's cost in steps (plus one for its fixed work: resident loads and
// the accumulator read-out).  kDkDv: the query tiles of the group's heads
// that see the key tile; else the key tiles the query tile visits.
template <bool kDkDv>
__device__ __forceinline__ int bwd_unit_cost(const BwdArgs& a, const uint8_t* mask, int u) {
  int b, hx, tile;
  bwd_unit_of<kDkDv>(a, u, &b, &hx, &tile);
  const int nT = ea_cdiv(a.N, EA_BN);
  if (kDkDv) {
    const int G = a.Hq / a.Hkv;
    int c = 1;
    for (int g = 0; g < G; ++g) {
      const bool sa = mask[b * a.Hq + hx * G + g] != 0;
      c += bwd_last_query_tile(tile, sa, nT, a.sink, a.window) - tile + 1;
    }
    return c;
  }
  int a0, lo;
  bwd_key_tiles(tile, mask[b * a.Hq + hx] != 0, a.sink, a.window, &a0, &lo);
  return 1 + a0 + (tile - lo + 1);
}

constexpr int kSchedBins = 4096;

// Per-CTA unit lists of one backward kernel, longest units first.  One CTA
// of 1024 threads per kernel (blockIdx.x 0: dK/dV, 1: dQ):
//   1. units are counted by cost bin (cost >> shift, so every bin index is
//      below kSchedBins) and sorted by decreasing bin, ties by unit index;
//   2. dK/dV: each unit in that order goes to the least-loaded CTA (ties to
//      the lowest index), since a few key tiles carry far more steps than
//      the rest; dQ: the sorted units are dealt in a snake, which already
//      balances its many similar units;
//   3. each CTA's units are listed in sorted order.
// Every step is deterministic: the sort's scatter and the dK/dV assignment
// and lists run in order on one warp, and the dQ lists are closed forms, so
// the schedule is the same on every run.  Results do not depend on it: a
// unit owns its output tile.
template <bool kDkDv>
__device__ void bwd_schedule(const BwdArgs& a, int grid, int* hist, long long* load,
                             uint8_t* mask, int& shift_s) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nT = ea_cdiv(a.N, EA_BN);
  const int units = a.B * (kDkDv ? a.Hkv : a.Hq) * nT;
  int* offs = kDkDv ? a.offs_kv : a.offs_q;
  int* list = kDkDv ? a.list_kv : a.list_q;
  int* sorted = kDkDv ? a.sorted_kv : a.sorted_q;
  int* cta = kDkDv ? a.cta_kv : a.cta_q;
  const int max_cost = 1 + (kDkDv ? a.Hq / a.Hkv : 1) * nT;
  if (tid == 0) {
    int sh = 0;
    while ((max_cost >> sh) >= kSchedBins) ++sh;
    shift_s = sh;
  }
  for (int i = tid; i < kSchedBins; i += blockDim.x) hist[i] = 0;
  for (int i = tid; i < kBwdMaxGrid; i += blockDim.x) load[i] = 0;
  for (int i = tid; i < a.B * a.Hq; i += blockDim.x) mask[i] = a.mask[i];
  __syncthreads();
  const int shift = shift_s;
  const unsigned lt = (1u << lane) - 1u;
  // counts per bin; lanes of a warp that share a bin add once (most units
  // of a mask share a handful of costs)
  for (int base = warp * 32; base < units; base += blockDim.x) {
    const int u = base + lane;
    const int bin = u < units ? bwd_unit_cost<kDkDv>(a, mask, u) >> shift : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, bin);
    if (u < units && (peers & lt) == 0) atomicAdd(&hist[bin], __popc(peers));
  }
  __syncthreads();
  // hist[bin] becomes the first sorted position of the bin, bins in
  // decreasing order: each thread sums four consecutive bins from the top,
  // a block scan of the thread sums gives each group's start
  {
    static_assert(kSchedBins == 4 * 1024, "four bins per thread of the 1024");
    int* wsum = reinterpret_cast<int*>(load);   // 32 warp totals (load is reset below)
    int v[4], t = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[i] = hist[kSchedBins - 1 - (4 * tid + i)];
      t += v[i];
    }
    int incl = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = wsum[lane], wi = w;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wi, off);
        if (lane >= off) wi += y;
      }
      wsum[lane] = wi - w;                      // exclusive over warps
    }
    __syncthreads();
    int run = wsum[warp] + incl - t;            // exclusive start of this thread's four bins
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hist[kSchedBins - 1 - (4 * tid + i)] = run;
      run += v[i];
    }
    __syncthreads();
    for (int i = tid; i < kBwdMaxGrid; i += blockDim.x) load[i] = 0;
    __syncthreads();
  }
  if (warp == 0) {
    // stable scatter by bin
    for (int base = 0; base < units; base += 32) {
      const int u = base + lane;
      const int bin = u < units ? bwd_unit_cost<kDkDv>(a, mask, u) >> shift : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      const int pos = u < units ? hist[bin] + __popc(peers & lt) : 0;
      __syncwarp();
      if (u < units) {
        sorted[pos] = u;
        if ((peers & lt) == 0) hist[bin] += __popc(peers);
      }
      __syncwarp();
    }
  }
  if (!kDkDv) {
    // dQ: the sorted units dealt in a snake.  Rank r = k * grid + j goes to
    // CTA j (k even) or grid - 1 - j (k odd), at position k of its list; a
    // CTA's list has units / grid entries, plus one if the last, partial
    // round reaches it, so the offsets and positions are closed forms.
    __syncthreads();
    const int F = units / grid, R = units % grid;
    auto first = [&](int c) {
      int extra = 0;
      if (R > 0) extra = (F & 1) == 0 ? min(c, R) : max(0, c - (grid - R));
      return c * F + extra;
    };
    for (int c = tid; c <= grid; c += blockDim.x) offs[c] = first(c);
    for (int r = tid; r < units; r += blockDim.x) {
      const int k = r / grid, j = r % grid;
      const int c = (k & 1) ? grid - 1 - j : j;
      list[first(c) + k] = sorted[r];
    }
    return;
  }
  if (warp == 0) {
    // dK/dV: each unit in sorted order to the least-loaded CTA (ties to the
    // lowest index).  Lane l keeps the loads of CTAs l, l + 32, ... in
    // registers (grid <= 32 * kPer) and the warp takes their minimum with
    // reductions.  Loads stay below 2^31 (units * max_cost); past that, or
    // for a larger grid, the units are dealt in a snake instead.
    constexpr int kPer = 8;
    const bool greedy = grid <= 32 * kPer &&
                        static_cast<long long>(units) * max_cost < (1ll << 31);
    // Packed keys (load << 8 | CTA) when every load stays below 2^24: the
    // key minimum is then the least load with the lowest index, one
    // reduction per unit.
    const bool packed = greedy && static_cast<long long>(units) * max_cost < (1ll << 24);
    unsigned ld[kPer];
#pragma unroll
    for (int m = 0; m < kPer; ++m)
      ld[m] = (m * 32 + lane < grid) ? (packed ? static_cast<unsigned>(m * 32 + lane) : 0u)
                                     : 0xffffffffu;
    for (int base = 0; base < units; base += 32) {
      const int mine = base + lane < units ? bwd_unit_cost<kDkDv>(a, mask, sorted[base + lane]) : 0;
      if (!greedy) {
        const int r = base + lane;
        if (r < units) {
          const int k = r / grid, j = r % grid;
          cta[r] = (k & 1) ? grid - 1 - j : j;
        }
        continue;
      }
      unsigned mywin = 0;   // lane j keeps the CTA of unit base + j
      for (int j = 0; j < 32 && base + j < units; ++j) {
        const unsigned c = static_cast<unsigned>(__shfl_sync(0xffffffffu, mine, j));
        unsigned win;
        if (packed) {
          const unsigned m01 = min(ld[0], ld[1]), m23 = min(ld[2], ld[3]);
          const unsigned m45 = min(ld[4], ld[5]), m67 = min(ld[6], ld[7]);
          const unsigned key = __reduce_min_sync(0xffffffffu, min(min(m01, m23), min(m45, m67)));
          win = key & 0xffu;
          // branch-free: only the winning slot adds
#pragma unroll
          for (int m = 0; m < kPer; ++m)
            ld[m] += (static_cast<unsigned>(m * 32 + lane) == win) ? (c << 8) : 0u;
        } else {
          unsigned best = ld[0];
          int bm = 0;
#pragma unroll
          for (int m = 1; m < kPer; ++m)
            if (ld[m] < best) {
              best = ld[m];
              bm = m;
            }
          const unsigned wmin = __reduce_min_sync(0xffffffffu, best);
          // CTA index of this lane's minimum (lane + 32 m); the smallest
          // index among the lanes that hold the warp minimum wins
          const unsigned idx =
              (best == wmin) ? static_cast<unsigned>(bm * 32 + lane) : 0xffffffffu;
          win = __reduce_min_sync(0xffffffffu, idx);
          if (static_cast<int>(win & 31) == lane) {
#pragma unroll
            for (int m = 0; m < kPer; ++m)
              if (m == static_cast<int>(win >> 5)) ld[m] += c;
          }
        }
        mywin = (lane == j) ? win : mywin;
      }
      if (base + lane < units) cta[base + lane] = static_cast<int>(mywin);
    }
    __syncwarp();
    // per-CTA counts, offsets, then the lists in sorted order
    for (int i = lane; i < grid; i += 32) load[i] = 0;
    __syncwarp();
    for (int base = 0; base < units; base += 32) {
      const int r = base + lane;
      const int c = r < units ? cta[r] : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, c);
      if (r < units && (peers & lt) == 0) load[c] += __popc(peers);
      __syncwarp();
    }
    if (lane == 0) {
      int run = 0;
      for (int i = 0; i < grid; ++i) {
        offs[i] = run;
        const int n = static_cast<int>(load[i]);
        load[i] = run;
        run += n;
      }
      offs[grid] = run;
    }
    __syncwarp();
    for (int base = 0; base < units; base += 32) {
      const int r = base + lane;
      const int c = r < units ? cta[r] : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, c);
      const int pos = r < units ? static_cast<int>(load[c]) + __popc(peers & lt) : 0;
      __syncwarp();
      if (r < units) {
        list[pos] = sorted[r];
        if ((peers & lt) == 0) load[c] += __popc(peers);
      }
      __syncwarp();
    }
  }
}

__global__ void __launch_bounds__(1024, 1) ea_bwd_sched_kernel(const __grid_constant__ BwdArgs a,
                                                               int grid_kv, int grid_q) {
  __shared__ int hist[kSchedBins];
  __shared__ long long load[kBwdMaxGrid];
  __shared__ uint8_t mask[EA_MAX_ENTRIES];
  __shared__ int shift_s;
  if (blockIdx.x == 0)
    bwd_schedule<true>(a, grid_kv, hist, load, mask, shift_s);
  else
    bwd_schedule<false>(a, grid_q, hist, load, mask, shift_s);
}

size_t bwd_sched_ints(int B, int Hq, int Hkv, int N) {
  const size_t nT = static_cast<size_t>(ea_cdiv(N, EA_BN));
  const size_t units_kv = static_cast<size_t>(B) * Hkv * nT;
  const size_t units_q = static_cast<size_t>(B) * Hq * nT;
  return 2 * (kBwdMaxGrid + 1) + 3 * (units_kv + units_q);
}

// One backward kernel per flavour (see the file comment):
//   kDkDv: resident K_j, V_j; streamed Q_i, dO_i; TMEM S^T [0,128),
//          dP^T [128,256), dV [256,384), dK [384,512).
//   else:  resident Q_i, dO_i; streamed K_j, V_j; TMEM S [0,128),
//          dP [128,256), dQ [256,384).
// Warps 0-7 elementwise (row group w % 4 = TMEM lanes 32 (w % 4), column
// half w / 4), warp 8 producer (lane 0 issues the copies; for kDkDv all its
// lanes stage the step's -lse * log2e and -D in shared memory), warp 9 the
// MMA issuing thread.
template <bool kDkDv>
__global__ void __launch_bounds__(BwdCfg::kThreads, 1) ea_bwd_attn_kernel(
    const __grid_constant__ BwdArgs args) {
  using C = BwdCfg;
  constexpr int D = C::D;
  constexpr float kLog2e = 1.4426950408889634f;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the plan fills the 227 KB with no room to align the base: require it
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicCAS(args.status, EA_OK, EA_ERR_UNSUPPORTED);
    return;
  }
  uint8_t* smem = smem_raw;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  const uint32_t bar0 = smem_u32(bar);
  const uint32_t b_res_full = bar0, b_res_empty = bar0 + 8;
  const uint32_t b_full0 = bar0 + 16, b_empty0 = b_full0 + 8 * C::kStages0;
  const uint32_t b_full1 = b_empty0 + 8 * C::kStages0, b_empty1 = b_full1 + 8 * C::kStages1;
  const uint32_t b_s_full = b_empty1 + 8 * C::kStages1, b_dp_full = b_s_full + 8;
  const uint32_t b_p_full = b_s_full + 16, b_ds_full = b_s_full + 24;
  const uint32_t b_acc_done = b_s_full + 32, b_acc_empty = b_s_full + 40;
  const uint32_t b_drain = b_s_full + 48;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  BwdStep* steps = reinterpret_cast<BwdStep*>(smem + C::kOffStep);
  float* vec0 = reinterpret_cast<float*>(smem + C::kOffVec0);
  float* vec1 = reinterpret_cast<float*>(smem + C::kOffVec1);
  const int G = args.Hq / args.Hkv;
  const int nT = ea_cdiv(args.N, EA_BN);
  // this CTA's units, longest first (ea_bwd_sched_kernel)
  const int* uoffs = kDkDv ? args.offs_kv : args.offs_q;
  const int* ulist = kDkDv ? args.list_kv : args.list_q;
  const uint64_t tlim = args.timeout_ns;
  int* status = args.status;

  if (threadIdx.x == 0) {
    // arrival counts: one (producer arrive or MMA commit) except p_full,
    // ds_full and acc_empty (all 256 elementwise threads)
    for (int i = 0; i < C::kNumBars; ++i) {
      const uint32_t a = bar0 + 8 * i;
      mbar_init(bar + i, (a == b_p_full || a == b_ds_full || a == b_acc_empty) ? 256 : 1);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 8) {
    // ============================================================ producer
    uint32_t pos = 0, nu = 0, armed0 = 0, armed1 = 0;
    bool ok = true;
    for (int kk = uoffs[blockIdx.x], kend = uoffs[blockIdx.x + 1]; kk < kend && ok; ++kk) {
      const int u = ulist[kk];
      int b, hx, tile;
      bwd_unit_of<kDkDv>(args, u, &b, &hx, &tile);
      if (nu > 0) {
        if (lane == 0)
          ok = mbar_wait(b_res_empty, (nu - 1) & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
      }
      if (lane == 0) {
        // resident operands: K_j, V_j (kDkDv) or Q_i, dO_i
        mbar_arrive_expect_tx(b_res_full, 2 * C::kTileBytes);
        const CUtensorMap* m0 = kDkDv ? &args.tm_k : &args.tm_q;
        const CUtensorMap* m1 = kDkDv ? &args.tm_v : &args.tm_do;
        const int z = kDkDv ? b * args.Hkv + hx : b * args.Hq + hx;
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(smem_u32(smem + C::kOffRes) + c * C::kBlockBytes, m0, b_res_full, c * 64,
                      tile * EA_BM, z);
          tma_load_3d(smem_u32(smem + C::kOffRes + C::kTileBytes) + c * C::kBlockBytes, m1,
                      b_res_full, c * 64, tile * EA_BM, z);
        }
      }
      ++nu;
      // steps of the unit
      const int ng = kDkDv ? G : 1;
      for (int g = 0; g < ng && ok; ++g) {
        const int h = kDkDv ? hx * G + g : hx;
        const bool sa = args.mask[b * args.Hq + h] != 0;
        int n, a = 0, lo = 0;
        if (kDkDv) {
          n = bwd_last_query_tile(tile, sa, nT, args.sink, args.window) - tile + 1;
        } else {
          bwd_key_tiles(tile, sa, args.sink, args.window, &a, &lo);
          n = a + (tile - lo + 1);
        }
        for (int i = 0; i < n && ok; ++i) {
          const int it = kDkDv ? tile + i : tile;
          const int jt = kDkDv ? tile : (i < a ? i : lo + (i - a));
          const int row = (kDkDv ? it : jt) * EA_BM;
          const uint32_t s0 = pos % C::kStages0, s1 = pos % C::kStages1;
          // tile 0 (Q_i or K_j), its -lse vector and the step descriptor
          if (pos >= C::kStages0) {
            if (lane == 0)
              ok = mbar_wait(b_empty0 + 8 * s0, ((pos / C::kStages0) - 1) & 1, s_abort, status,
                             tlim, EA_ERR_TIMEOUT);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
          }
          if (lane == 0) {
            BwdStep& st = steps[s0];
            st.b = b; st.h = h; st.it = it; st.jt = jt; st.sa = sa;
            st.first = (g == 0 && i == 0);
            st.last = (g == ng - 1 && i == n - 1);
            st.full = bwd_block_full(it, jt, args.N, sa, args.sink, args.window);
            mbar_arrive_expect_tx(b_full0 + 8 * s0, C::kTileBytes + (kDkDv ? 512u : 0u));
            ++armed0;
            if (kDkDv)   // the query tile's -lse * log2e: one 512-byte copy
              bulk_load(smem_u32(vec0 + s0 * 128),
                        args.vl_pad + (static_cast<size_t>(b) * args.Hq + h) * args.npad +
                            it * EA_BM,
                        512, b_full0 + 8 * s0);
            const uint32_t dst = smem_u32(smem + C::kOffSt0) + s0 * C::kTileBytes;
            const CUtensorMap* m = kDkDv ? &args.tm_q : &args.tm_k;
            const int z = kDkDv ? b * args.Hq + h : b * args.Hkv + h / G;
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(dst + c * C::kBlockBytes, m, b_full0 + 8 * s0, c * 64, row, z);
          }
          // tile 1 (dO_i or V_j) and its -D vector
          if (pos >= C::kStages1) {
            if (lane == 0)
              ok = mbar_wait(b_empty1 + 8 * s1, ((pos / C::kStages1) - 1) & 1, s_abort, status,
                             tlim, EA_ERR_TIMEOUT);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
          }
          if (lane == 0) {
            mbar_arrive_expect_tx(b_full1 + 8 * s1, C::kTileBytes + (kDkDv ? 512u : 0u));
            ++armed1;
            if (kDkDv)   // the query tile's -D
              bulk_load(smem_u32(vec1 + s1 * 128),
                        args.vd_pad + (static_cast<size_t>(b) * args.Hq + h) * args.npad +
                            it * EA_BM,
                        512, b_full1 + 8 * s1);
            const uint32_t dst = smem_u32(smem + C::kOffSt1) + s1 * C::kTileBytes;
            const CUtensorMap* m = kDkDv ? &args.tm_do : &args.tm_v;
            const int z = kDkDv ? b * args.Hq + h : b * args.Hkv + h / G;
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(dst + c * C::kBlockBytes, m, b_full1 + 8 * s1, c * 64, row, z);
          }
          ++pos;
        }
      }
    }
    if (lane == 0) {
      // every copy issued must land before the CTA exits
      const uint32_t n0 = armed0 < C::kStages0 ? armed0 : C::kStages0;
      for (uint32_t p = armed0 - n0; p < armed0; ++p)
        mbar_wait_drain(b_full0 + 8 * (p % C::kStages0), (p / C::kStages0) & 1, 200000000ull);
      const uint32_t n1 = armed1 < C::kStages1 ? armed1 : C::kStages1;
      for (uint32_t p = armed1 - n1; p < armed1; ++p)
        mbar_wait_drain(b_full1 + 8 * (p % C::kStages1), (p / C::kStages1) & 1, 200000000ull);
      if (nu > 0) mbar_wait_drain(b_res_full, (nu - 1) & 1, 200000000ull);
    }
  } else if (warp == 9) {
    // ============================================================ MMA issuer
    // Per step n, the score products and the two phases of the elementwise
    // warps interleave:
    //   [E: P from S(n)]    while dP(n) runs
    //   dV += P^T dO (kDkDv), then S(n + 1)   while E computes dS from dP(n)
    //   dK += dS^T Q (or dQ += dS K), then dP(n + 1)   while E computes P(n + 1)
    // so the tensor pipe and the elementwise warps work at the same time.
    // tcgen05.mma from one thread executes in issue order, so a score
    // product overwrites the columns the accumulating product before it read.
    // The whole warp runs this loop and the elected lane's MMAs and commits
    // take effect (warp-uniform descriptors and counters; the fused forward
    // runs 5% faster this way than from a lane-0 branch).
    {
      const uint32_t leader = elect_one();
      const uint32_t res = smem_u32(smem + C::kOffRes);
      // K-major views (the score products) and MN-major views (the B operand
      // of the accumulating products)
      const uint64_t d_res_k = smem_desc_sw128(res, 16, 1024);
      const uint64_t d_st0_k = smem_desc_sw128(smem_u32(smem + C::kOffSt0), 16, 1024);
      const uint64_t d_st1_k = smem_desc_sw128(smem_u32(smem + C::kOffSt1), 16, 1024);
      const uint64_t d_st0_mn = smem_desc_sw128(smem_u32(smem + C::kOffSt0), C::kBlockBytes, 1024);
      const uint64_t d_st1_mn = smem_desc_sw128(smem_u32(smem + C::kOffSt1), C::kBlockBytes, 1024);
      // which = 0: kDkDv S^T = K Q^T, else S = Q K^T (TMEM columns 0-127),
      // resident tile 0 against tile 0 of step p; which = 1: kDkDv
      // dP^T = V dO^T, else dP = dO V^T (columns 128-255), tiles 1
      auto scores = [&](uint32_t p, int which) {
        const uint64_t a = d_res_k + ((which * C::kTileBytes) >> 4);
        const uint64_t b = which ? d_st1_k + (((p % C::kStages1) * C::kTileBytes) >> 4)
                                 : d_st0_k + (((p % C::kStages0) * C::kTileBytes) >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::kBlockBytes + (k & 3) * 32) >> 4;
          mma_ss_w(leader, tmem + 128 * which, a + off, b + off, C::kIdescSS, k > 0 ? 1u : 0u);
        }
      };
      auto wait_full = [&](int which, uint32_t p) {
        return which ? mbar_wait(b_full1 + 8 * (p % C::kStages1), (p / C::kStages1) & 1, s_abort,
                                 status, tlim, EA_ERR_TIMEOUT)
                     : mbar_wait(b_full0 + 8 * (p % C::kStages0), (p / C::kStages0) & 1, s_abort,
                                 status, tlim, EA_ERR_TIMEOUT);
      };
      uint32_t pos = 0, nu = 0, nsteps = 0;
      bool ok = true;
      for (int kk = uoffs[blockIdx.x], kend = uoffs[blockIdx.x + 1]; kk < kend && ok; ++kk) {
        if (!(ok = mbar_wait(b_res_full, nu & 1, s_abort, status, tlim, EA_ERR_TIMEOUT))) break;
        const uint32_t unit = nu++;
        if (!(ok = wait_full(0, pos))) break;
        scores(pos, 0);
        mma_commit_w(leader, b_s_full);
        if (!(ok = wait_full(1, pos))) break;
        scores(pos, 1);
        mma_commit_w(leader, b_dp_full);
        bool last = false, first = true;
        while (!last && ok) {
          const uint32_t s0 = pos % C::kStages0, s1 = pos % C::kStages1;
          last = steps[s0].last != 0;
          // the previous unit's accumulators must have been read out
          if (first && unit > 0 &&
              !(ok = mbar_wait(b_acc_empty, (unit - 1) & 1, s_abort, status, tlim,
                               EA_ERR_TIMEOUT)))
            break;
          const uint64_t m0 = d_st0_mn + ((s0 * C::kTileBytes) >> 4);
          const uint64_t m1 = d_st1_mn + ((s1 * C::kTileBytes) >> 4);
          // P done (kDkDv: as bf16 P^T at the start of each column half's
          // columns) and S read
          if (!(ok = mbar_wait(b_p_full, nsteps & 1, s_abort, status, tlim, EA_ERR_TIMEOUT)))
            break;
          tc_fence_after();
          if (kDkDv) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_ts_w(leader, tmem + 256, tmem + 64 * (k >> 2) + 8 * (k & 3), m1 + ((k * 2048) >> 4),
                     C::kIdescTS, (!first || k > 0) ? 1u : 0u);            // dV += P^T dO
          }
          // (TMA-written tiles need no tcgen05 fence: the mbarrier completes
          // the copy for the tensor cores' reads)
          if (!last) {
            if (!(ok = wait_full(0, pos + 1))) break;
            scores(pos + 1, 0);
            mma_commit_w(leader, b_s_full);
          }
          // dS (bf16 at the start of each column half's dP columns)
          if (!(ok = mbar_wait(b_ds_full, nsteps & 1, s_abort, status, tlim, EA_ERR_TIMEOUT)))
            break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ts_w(leader, tmem + (kDkDv ? 384 : 256), tmem + 128 + 64 * (k >> 2) + 8 * (k & 3),
                   m0 + ((k * 2048) >> 4), C::kIdescTS,
                   (!first || k > 0) ? 1u : 0u);           // dK += dS^T Q  /  dQ += dS K
          // the step's tiles (and, read by the elementwise warps before
          // ds_full, its vectors) are free once these products complete
          mma_commit_w(leader, b_empty0 + 8 * s0);
          mma_commit_w(leader, b_empty1 + 8 * s1);
          if (!last) {
            if (!(ok = wait_full(1, pos + 1))) break;
            scores(pos + 1, 1);
            mma_commit_w(leader, b_dp_full);
          }
          ++nsteps;
          first = false;
          ++pos;
        }
        if (!ok) break;
        mma_commit_w(leader, b_acc_done);
        mma_commit_w(leader, b_res_empty);
      }
      // drain: wait for every MMA the elected lane issued
      mma_commit_w(leader, b_drain);
      mbar_wait_drain(b_drain, 0, 200000000ull);
    }
  } else {
    // ============================================================ elementwise
    const int rg = warp & 3, half = warp >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(rg * 32) << 16;
    const int t = rg * 32 + lane;        // tile row: key (kDkDv) or query
    const int col0 = half * 64;          // this warp's 64 columns
    const float sl2 = args.scale_log2;
    uint32_t pos = 0, nsteps = 0, nu = 0;
    bool ok = true;
    for (int kk = uoffs[blockIdx.x], kend = uoffs[blockIdx.x + 1]; kk < kend && ok; ++kk) {
      const int u = ulist[kk];
      int b, hx, tile;
      bwd_unit_of<kDkDv>(args, u, &b, &hx, &tile);
      const int row = tile * EA_BM + t;
      // dQ rows: the row's own -lse * log2e and -D
      float nl_row = 0.f, nd_row = 0.f;
      if (!kDkDv && row < args.N) {
        const size_t ri = (static_cast<size_t>(b) * args.Hq + hx) * args.N + row;
        nl_row = -args.lse[ri] * kLog2e;
        nd_row = -args.dvec[ri];
      }
      bool last = false;
      while (!last) {
        const uint32_t s0 = pos % C::kStages0, s1 = pos % C::kStages1;
        ok = mbar_wait(b_full0 + 8 * s0, (pos / C::kStages0) & 1, s_abort, status, tlim,
                       EA_ERR_TIMEOUT);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const BwdStep st = steps[s0];
        last = st.last != 0;
        const uint32_t par = nsteps & 1;
        ok = mbar_wait(b_s_full, par, s_abort, status, tlim, EA_ERR_TIMEOUT);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        // visible columns of this row as ranges (branch-free per element):
        // kDkDv (row = key k, column c = query q0 + c): c in [lo_a, hi_a];
        // else (row = query q, column c = key k0 + c): c in [0, hi_a] and
        // (c < sink_c or c >= win_c)
        int lo_a = 0, hi_a = 127, sink_c = 1 << 20, win_c = -(1 << 20);
        if (!st.full) {
          const bool sa = st.sa != 0;
          if (kDkDv) {
            const int k = row, q0 = st.it * EA_BM;
            lo_a = k - q0;                                   // q >= k
            hi_a = args.N - 1 - q0;                          // q < N
            if (k >= args.N) hi_a = -1;
            if (sa && k >= args.sink) hi_a = min(hi_a, k + args.window - 1 - q0);   // q - k < W
          } else {
            const int q = row, k0 = st.jt * EA_BN;
            hi_a = (q < args.N) ? q - k0 : -1;               // k <= q (< N)
            if (sa) {
              sink_c = args.sink - k0;                       // k < S
              win_c = q - args.window + 1 - k0;              // q - k < W
            }
          }
        }
        // phase 1: P kept in registers (and, kDkDv, bf16 P^T at the start of
        // this half's S columns, all of which this thread has read)
        float pr[64];
        {
          uint32_t pk[32];
          const float* vl = vec0 + s0 * 128;
          if (st.full)
            bwd_phase_p<kDkDv, true>(tmem + lane_off + col0, vl, nl_row, col0, sl2, lo_a, hi_a,
                                     sink_c, win_c, pr, pk);
          else
            bwd_phase_p<kDkDv, false>(tmem + lane_off + col0, vl, nl_row, col0, sl2, lo_a, hi_a,
                                      sink_c, win_c, pr, pk);
          if (kDkDv) {
            tmem_st32(tmem + lane_off + col0, pk);
            tmem_wait_st();
          }
        }
        tc_fence_before();
        mbar_arrive(b_p_full);
        // phase 2: dS = P (dP - D), bf16 at the start of this half's dP columns
        if (kDkDv) {   // the step's -D vector comes with tile 1
          ok = mbar_wait(b_full1 + 8 * s1, (pos / C::kStages1) & 1, s_abort, status, tlim,
                         EA_ERR_TIMEOUT);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        ++pos;
        ++nsteps;
        ok = mbar_wait(b_dp_full, par, s_abort, status, tlim, EA_ERR_TIMEOUT);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        {
          uint32_t ds[32];
          const float* vd = vec1 + s1 * 128;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            uint32_t dr[32];
            tmem_ld32_wait(tmem + lane_off + 128 + col0 + 32 * ch, dr);
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int j = 16 * ch + jj;
              const int c = col0 + 2 * j;
              float t0, t1;
              if (kDkDv) {
                const float2 d2 = *reinterpret_cast<const float2*>(vd + c);
                t0 = d2.x; t1 = d2.y;
              } else {
                t0 = t1 = nd_row;
              }
              add2_acc(t0, t1, __uint_as_float(dr[2 * jj]), __uint_as_float(dr[2 * jj + 1]));
              float e0 = 0.f, e1 = 0.f;
              fma2_acc(e0, e1, pr[2 * j], pr[2 * j + 1], t0, t1);   // dS = P (dP - D)
              ds[j] = pack_bf16x2(e0, e1);
            }
          }
          tmem_st32(tmem + lane_off + 128 + col0, ds);
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(b_ds_full);
      }
      if (!ok) break;
      // epilogue
      ok = mbar_wait(b_acc_done, nu & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++nu;
      tc_fence_after();
      if (kDkDv) {
        // half 0: dV rows; half 1: scale * dK rows (128 channels each)
        __nv_bfloat16* dst = (half ? args.dk : args.dv) +
                             ((static_cast<size_t>(b) * args.Hkv + hx) * args.N + row) * D;
        const float mul = half ? args.scale : 1.f;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          uint32_t r[64];
          tmem_ld64_wait(tmem + lane_off + 256 + half * 128 + part * 64, r);
          if (row < args.N) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + part * 64);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              uint32_t w[4];
#pragma unroll
              for (int j = 0; j < 4; ++j)
                w[j] = pack_bf16x2(__uint_as_float(r[8 * q4 + 2 * j]) * mul,
                                   __uint_as_float(r[8 * q4 + 2 * j + 1]) * mul);
              d4[q4] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      } else {
        // channel half of scale * dQ
        uint32_t r[64];
        tmem_ld64_wait(tmem + lane_off + 256 + half * 64, r);
        if (row < args.N) {
          __nv_bfloat16* dst =
              args.dq + ((static_cast<size_t>(b) * args.Hq + hx) * args.N + row) * D + half * 64;
          uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              w[j] = pack_bf16x2(__uint_as_float(r[8 * q4 + 2 * j]) * args.scale,
                                 __uint_as_float(r[8 * q4 + 2 * j + 1]) * args.scale);
            d4[q4] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(b_acc_empty);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

static int g_bwd_configured[64] = {0};

cudaError_t launch_backward(const BwdArgs& a, const void* dout, const void* out, float* dvec,
                            float* vl_pad, float* vd_pad, int grid_sms, cudaStream_t stream) {
  const long long prows = static_cast<long long>(a.B) * a.Hq * a.npad;
  ea_bwd_rowdot_kernel<<<static_cast<unsigned>((prows + 15) / 16), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(out), a.lse,
      a.B * a.Hq, a.N, a.npad, BwdCfg::D, dvec, vl_pad, vd_pad);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  int dev = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if (dev >= 64 || !g_bwd_configured[dev]) {
    if ((err = cudaFuncSetAttribute(ea_bwd_attn_kernel<true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    BwdCfg::kSmem)) != cudaSuccess)
      return err;
    if ((err = cudaFuncSetAttribute(ea_bwd_attn_kernel<false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    BwdCfg::kSmem)) != cudaSuccess)
      return err;
    if (dev < 64) g_bwd_configured[dev] = 1;
  }
  const int nT = ea_cdiv(a.N, EA_BN);
  const int units_kv = a.B * a.Hkv * nT, units_q = a.B * a.Hq * nT;
  const int sms = grid_sms < kBwdMaxGrid ? grid_sms : kBwdMaxGrid;
  const int grid_kv = units_kv < sms ? units_kv : sms;
  const int grid_q = units_q < sms ? units_q : sms;
  ea_bwd_sched_kernel<<<2, 1024, 0, stream>>>(a, grid_kv, grid_q);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  ea_bwd_attn_kernel<true><<<grid_kv, BwdCfg::kThreads, BwdCfg::kSmem, stream>>>(a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  ea_bwd_attn_kernel<false><<<grid_q, BwdCfg::kThreads, BwdCfg::kSmem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ea
