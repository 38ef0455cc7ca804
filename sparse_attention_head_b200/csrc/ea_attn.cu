// ea_attn.cu — fused hybrid FA/SA causal prefill attention for sm_100a.
//
// Elastic Attention blog (bxzpzcl.cn) §3 "Fused Kernel": the per-head routing
// decision is passed to the kernel as metadata, and one launch serves the
// heads routed to Full Attention and those routed to Sparse Attention.  The
// sparse pattern is streaming attention (S sink keys plus a causal window of
// W keys including the diagonal); full heads are plain causal attention.
//
// Design (one persistent CTA per SM, 12 warps = 3 warpgroups):
//   warps 0-3  softmax/correction/epilogue of query slot 0 (a paired unit:
//              head h0, rows r0..r0+127; a single unit: rows r0..r0+127)
//   warps 4-7  the same for slot 1 (head h1 at the same rows; a single unit:
//              rows r0+128..r0+255 of the one head)
//   warp  8    TMA producer: takes the unit tickets, walks the schedule and
//              hands each unit on through a shared-memory ring; loads the
//              Q slots once per unit, then K and V tiles of the unit's tile
//              list through a ring of shared-memory stages
//   warp  9    tcgen05 issuer (the whole warp runs the loop, the elected
//              lane issues): S_s = Q_s K^T into TMEM, then O_s += P_s V with
//              P read from TMEM (P overwrites S in place)
//   warps 10-11 idle (they complete the third warpgroup)
// Registers: launched at 168 per thread (384 x 168 = 64512); the third
// warpgroup drops to 120 and the two softmax warpgroups rise to 192
// (2 x 128 x 192 + 128 x 120 = 64512).
// TMEM (512 columns): S0 [0,128)  S1 [128,256)  O0 [256,256+d)  O1 [384,384+d).
// The MMA order per tile i is PV0(i), S0(i+1), PV1(i), S1(i+1), so one
// slot's softmax overlaps the other slot's tensor-core work.
//
// Softmax runs one query row per thread in fp32 on the log2 scale.  The row
// reference max is only moved when a tile's max exceeds it by more than 8
// (2^8 headroom in fp32/bf16), so most tiles need no O rescale; the final
// O / l uses the same reference, so the result is unchanged.  The row sum l
// adds the fp32 probabilities, except on the masked tiles of slots holding a
// row that sees fewer than 128 keys: there it adds the bf16-rounded ones
// (those the P.V product sees), so such rows' weights sum to one exactly.
//
// Every wait is bounded: on timeout the kernel records EA_ERR_TIMEOUT in the
// status word, every role leaves its loop, in-flight copies and MMAs are
// drained with bounded waits, TMEM is freed and the CTA exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ea.h"
#include "ea_internal.h"
#include "ea_math.cuh"
#include "ea_ptx.cuh"
#include "ea_router_dev.cuh"
#include "ea_sched.h"
#include "ea_tmem.cuh"

namespace ea {

// Of every 8 exp2 pairs of a score row, this many run as a polynomial on the
// FMA pipe instead of the MUFU (the two units then share the work).
constexpr int kEmuPairs = 0;
// The same for the FP8 variant, per 8 groups of four scores: its MUFU pipe
// also carries the e4m3 conversions.
constexpr int kEmuQuadsFp8 = 2;

// kFp8: q, k as e4m3 rows of d bytes; v transposed (d rows of keys); both
// products of kind::f8f6f4 with P rounded to e4m3 (d = 128 only).
template <int D, bool kFp8 = false>
struct AttnCfg {
  static constexpr int kThreads = 384;
  static constexpr uint32_t kRegsSoftmax = 192;
  static constexpr uint32_t kRegsOther = 120;
  static constexpr int kElem = kFp8 ? 1 : 2;                // bytes per value
  static constexpr int kBlockBytes = 128 * 128;             // 128 rows x 128 bytes
  static constexpr int kBlockElems = 128 / kElem;           // values per 128-byte row
  static constexpr int kDBlocks = D * kElem / 128;          // 128-byte column blocks
  static constexpr int kTileBytes = 128 * D * kElem;        // one Q slot / K / V tile
  static constexpr int kStages = (kTileBytes == 32768) ? 4 : 8;
  static constexpr int kKSteps = D * kElem / 32;            // S product: 32 bytes of K each
  static constexpr int kPVSteps = 128 * kElem / 32;         // P.V product: 32 bytes of keys each
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  // q_full, q_empty, drain, kv_full[kStages], kv_empty[kStages],
  // s_full[2], p_full[2], o_done[2], o_empty[2], p_half[2],
  // unit_full[kUnitRing], unit_empty[kUnitRing]
  static constexpr int kUnitRing = 4;                       // units the producer runs ahead
  static constexpr int kNumBars = 3 + 2 * kStages + 10 + 2 * kUnitRing;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;   // tmem base, abort, counts
  static constexpr int kOffUnit = kOffMisc + 64;            // the unit ring: {rank, word, head}
  static constexpr int kOffEnt = kOffUnit + 64;
  // sequence tables: token offset and length by index; order, block count and
  // pair count by sorted position; the four entry runs' prefix counts by
  // sorted position
  static constexpr int kOffTok = kOffEnt + EA_MAX_ENTRIES * 2;
  static constexpr int kOffLen = kOffTok + EA_MAX_SEQS * 4;
  static constexpr int kPrefLen = EA_MAX_SEQS + 2;          // int16 entries, even
  static constexpr int kOffPref = kOffLen + EA_MAX_SEQS * 4;
  static constexpr int kOffOrder = kOffPref + 4 * kPrefLen * 2;
  static constexpr int kOffP = kOffOrder + EA_MAX_SEQS * 2;
  static constexpr int kOffNT = kOffP + EA_MAX_SEQS * 2;
  static constexpr int kSmem = kOffNT + EA_MAX_SEQS * 2 + 1024;  // + alignment slack
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static constexpr uint32_t kIdescS =
      kFp8 ? idesc_e4m3_f32(128, 128) : idesc_bf16_f32(128, 128, 0, 0);
  // bf16: V [keys][d] is an MN-major B; e4m3: V^T [d][keys] is K-major
  static constexpr uint32_t kIdescPV =
      kFp8 ? idesc_e4m3_f32(128, D) : idesc_bf16_f32(128, D, 0, 1);
  static_assert(!kFp8 || D == 128, "the FP8 variant is built for d = 128");
};

// Shared-memory addresses (32-bit) of the kernel's mbarriers; the arrays
// (kv_full, kv_empty, s_full, ...) are consecutive 8-byte barriers.
struct Bars {
  uint32_t q_full;
  uint32_t q_empty;
  uint32_t drain;
  uint32_t kv_full;
  uint32_t kv_empty;
  uint32_t s_full;
  uint32_t p_full;
  uint32_t o_done;
  uint32_t o_empty;
  uint32_t p_half;
  uint32_t unit_full;
  uint32_t unit_empty;
};

// Route bit of entry idx, read through the coherent path: in a routed launch
// other CTAs wrote it earlier in the same launch.  Out of range: 0.
__device__ __forceinline__ uint8_t ld_mask(const uint8_t* mask, int idx) {
  return idx >= 0 ? *reinterpret_cast<const volatile uint8_t*>(mask + idx) : 0;
}

// Does the launch's shard run query head h of sequence b (its kv group
// selected, and the head itself when a head selection is given)?
__device__ __forceinline__ bool in_shard(const AttnArgs& args, int b, int h) {
  return (args.group_sel == nullptr ||
          args.group_sel[b * args.Hkv + h / (args.Hq / args.Hkv)] != 0) &&
         (args.head_sel == nullptr || args.head_sel[b * args.Hq + h] != 0);
}

// This CTA takes no more tickets (its producer has stopped, or never
// started); the last CTA of the launch to get here resets the dispatch
// counters for the next launch on this workspace.
__device__ __forceinline__ void release_dispatch(const AttnArgs& args) {
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(args.done_ctas, 1u) == gridDim.x - 1) {
      atomicExch(args.ticket, 0u);
      atomicExch(args.done_ctas, 0u);
    }
  }
}

// Grid barrier of the routed prologue.  Every CTA arrives once per phase;
// the last arrival resets the count and advances the generation, which the
// others wait for (no reset between launches is needed).  Bounded: returns
// false, with EA_ERR_TIMEOUT in the status word, if the others do not arrive
// in time.  Needs every CTA resident at once (a cooperative launch).
__device__ bool grid_sync(const AttnArgs& args, volatile int* s_flag, int phase) {
  __syncthreads();
#ifdef EA_TEST_HOOKS
  // test build only: CTA 0 leaves without arriving, so the others time out
  if (phase == args.debug_skip_grid_sync && blockIdx.x == 0) return false;
#else
  (void)phase;
#endif
  if (threadIdx.x == 0) {
    volatile unsigned int* gen = args.bar_gen;
    const unsigned int g = *gen;
    __threadfence();
    const unsigned int arrived = atomicAdd(args.bar_count, 1u) + 1u;
    bool ok = true;
    if (arrived == gridDim.x) {
      atomicExch(args.bar_count, 0u);
      __threadfence();
      atomicAdd(args.bar_gen, 1u);
    } else {
      const uint64_t t0 = global_ns();
      for (uint32_t it = 0; *gen == g; ++it) {
        if ((it & 63) == 63 && global_ns() - t0 > args.timeout_ns) {
          atomicCAS(args.status, 0, EA_ERR_TIMEOUT);
          ok = false;
          break;
        }
      }
    }
    __threadfence();
    *s_flag = ok ? 1 : 0;
  }
  __syncthreads();
  return *s_flag != 0;
}

// The Attention Router inside the attention launch (EA blog §2.1), with the
// standalone router kernels' arithmetic: pooling items (split, kv head, b)
// by threads 0..255 exactly as ea_router_pool_kernel, x as
// ea_router_reduce_kernel, then one warp per output of each MLP layer.  The
// phases meet at grid barriers; the mask is complete before any CTA builds
// its unit list.  Shared memory is free before the pipeline starts, so the
// Q region holds the pooling reduction.
template <int D>
__device__ bool routed_prologue(const AttnArgs& args, uint8_t* smem, volatile int* s_flag) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int B = args.B, Hkv = args.Hkv, ns = args.nsplit, hidden = args.hidden;
  const int in_dim = Hkv * D;
  float* partials = args.partials;
  float* xbuf = partials + static_cast<size_t>(B) * Hkv * ns * D;
  float* hbuf = xbuf + static_cast<size_t>(B) * in_dim;
  if (tid < kPoolThreads) {
    float* red = reinterpret_cast<float*>(smem);
    const int items = ns * Hkv * B;
    for (int it = blockIdx.x; it < items; it += gridDim.x) {
      const int split = it % ns, hk = (it / ns) % Hkv, b = it / (ns * Hkv);
      router_pool_item<D>(static_cast<const __nv_bfloat16*>(args.k_raw), args.cu_seqlens, args.N,
                          args.total, Hkv, b, hk, split, ns, partials, red, tid, 1);
    }
  }
  if (!grid_sync(args, s_flag, 0)) return false;
  for (int i = blockIdx.x * blockDim.x + tid; i < B * in_dim; i += gridDim.x * blockDim.x)
    xbuf[i] = router_x(partials, args.cu_seqlens, Hkv, args.N, args.total, D, ns, i / in_dim,
                       i % in_dim);
  if (!grid_sync(args, s_flag, 1)) return false;
  const int nw = blockDim.x / 32;
  for (int o = blockIdx.x * nw + warp; o < B * hidden; o += gridDim.x * nw) {
    const int b = o / hidden, oo = o % hidden;
    const float v = router_warp_dot(xbuf + static_cast<size_t>(b) * in_dim, in_dim, args.w1,
                                    args.b1, oo, lane);
    if (lane == 0) hbuf[static_cast<size_t>(b) * hidden + oo] = fmaxf(v, 0.f);
  }
  if (!grid_sync(args, s_flag, 2)) return false;
  for (int o = blockIdx.x * nw + warp; o < B * args.Hq; o += gridDim.x * nw) {
    const int b = o / args.Hq, oo = o % args.Hq;
    const float v = router_warp_dot(hbuf + static_cast<size_t>(b) * hidden, hidden, args.w2,
                                    args.b2, oo, lane);
    if (lane == 0) {
      if (args.logits) args.logits[o] = v;
      args.mask_out[o] = (v > args.threshold) ? 1 : 0;
    }
  }
  return grid_sync(args, s_flag, 3);
}

// One row's probabilities p = 2^(x * sl2 - msub) over keys [32 C0, 32 C1)
// of a 128-key tile:
// packed FMA, then exp2 on the MUFU for most pairs and on the FMA pipe for
// kEmuPairs of every 8 pairs; P is stored to TMEM as bf16 pairs (columns
// [0, 64) of the row's score columns) and acc gathers the row sum.  The sum
// adds the bf16-rounded values the P.V product sees when kRoundedSum, else
// the fp32 values, each within 2^-9 of its rounding (unpacking the rounded
// values costs 128 instructions per row and tile: 4-8% of the launch when
// every tile pays it).
template <bool kRoundedSum, int C0, int C1>
__device__ __forceinline__ void softmax_p_bf16(const float (&x)[128], float sl2, float msub,
                                               uint32_t tS, float (&acc)[8]) {
#pragma unroll
  for (int c = C0; c < C1; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float p0, p1;
      fma2_sc(p0, p1, x[c * 32 + 2 * j], x[c * 32 + 2 * j + 1], sl2, -msub);
      if ((j & 7) < kEmuPairs) {
        exp2_poly2(p0, p1);
      } else {
        p0 = ex2_approx(p0);
        p1 = ex2_approx(p1);
      }
      pk[j] = pack_bf16x2(p0, p1);
      if (kRoundedSum)
        add2_acc(acc[2 * (j & 3)], acc[2 * (j & 3) + 1], __uint_as_float(pk[j] << 16),
                 __uint_as_float(pk[j] & 0xffff0000u));
      else
        add2_acc(acc[2 * (j & 3)], acc[2 * (j & 3) + 1], p0, p1);
    }
    tmem_st16(tS + c * 16, pk);
  }
}

// kTrace: the per-unit trace (its own instantiation, so the others carry none
// of its code or registers)
template <int D, bool kRouted, bool kFp8 = false, bool kTrace = false>
__global__ void __launch_bounds__(384, 1) ea_hybrid_attn_kernel(const __grid_constant__ AttnArgs args) {
  using C = AttnCfg<D, kFp8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  if constexpr (kRouted) {
    if (!routed_prologue<D>(args, smem, reinterpret_cast<volatile int*>(smem + C::kOffMisc + 16))) {
      release_dispatch(args);
      return;   // a grid barrier timed out; nothing is allocated or in flight yet
    }
  }

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sKV = smem + C::kOffKV;
  uint64_t* bar_base = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  Bars bars;
  {
    const uint32_t b0 = smem_u32(bar_base);
    bars.q_full = b0;
    bars.q_empty = b0 + 8;
    bars.drain = b0 + 16;
    bars.kv_full = b0 + 24;
    bars.kv_empty = bars.kv_full + 8 * C::kStages;
    bars.s_full = bars.kv_empty + 8 * C::kStages;
    bars.p_full = bars.s_full + 16;
    bars.o_done = bars.p_full + 16;
    bars.o_empty = bars.o_done + 16;
    bars.p_half = bars.o_empty + 16;
    bars.unit_full = bars.p_half + 16;
    bars.unit_empty = bars.unit_full + 8 * C::kUnitRing;
  }
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  // per-unit trace times of softmax warp 0 lane 0 (unit start, first S ready,
  // last P handed over): kept in shared memory, off the softmax registers
  uint64_t* s_trace_ts = reinterpret_cast<uint64_t*>(smem + C::kOffMisc + 32);
  uint16_t* s_ent = reinterpret_cast<uint16_t*>(smem + C::kOffEnt);
  volatile int* s_unit = reinterpret_cast<volatile int*>(smem + C::kOffUnit);


  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    // bar_base layout: q_full, q_empty, drain, kv_full[kStages],
    // kv_empty[kStages], s_full[2], p_full[2], o_done[2], o_empty[2],
    // p_half[2], unit_full[kUnitRing], unit_empty[kUnitRing]
    mbar_init(bar_base + 0, 1);                        // q_full: producer
    mbar_init(bar_base + 1, 1);                        // q_empty: MMA issuer
    mbar_init(bar_base + 2, 1);                        // drain: MMA issuer
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(bar_base + 3 + i, 1);                  // kv_full: producer
      mbar_init(bar_base + 3 + C::kStages + i, 1);     // kv_empty: MMA issuer
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_base + 3 + 2 * C::kStages + s, 1);        // s_full
      mbar_init(bar_base + 3 + 2 * C::kStages + 2 + s, 128);  // p_full
      mbar_init(bar_base + 3 + 2 * C::kStages + 4 + s, 1);    // o_done
      mbar_init(bar_base + 3 + 2 * C::kStages + 6 + s, 128);  // o_empty
      mbar_init(bar_base + 3 + 2 * C::kStages + 8 + s, 128);  // p_half
    }
    for (int u = 0; u < C::kUnitRing; ++u) {
      mbar_init(bar_base + 3 + 2 * C::kStages + 10 + u, 1);   // unit_full: producer
      // unit_empty: the MMA warp's elected lane and lane 0 of the 8 softmax warps
      mbar_init(bar_base + 3 + 2 * C::kStages + 10 + C::kUnitRing + u, 9);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&args.tm_q);
    tma_prefetch_desc(&args.tm_k);
    tma_prefetch_desc(&args.tm_v);
  }
  if (warp == 9) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  // Sequence tables.  Lengths and token offsets by sequence index: a padded
  // batch has every length N; a packed batch reads cu_seqlens, and an
  // inconsistent one (cu[0] != 0, decreasing, or cu[B] != T) runs no unit
  // and records EA_ERR_INVALID_ARG.
  int32_t* s_tok = reinterpret_cast<int32_t*>(smem + C::kOffTok);
  int32_t* s_len = reinterpret_cast<int32_t*>(smem + C::kOffLen);
  int16_t* s_pref = reinterpret_cast<int16_t*>(smem + C::kOffPref);   // [4][kPrefLen]
  int16_t* s_order = reinterpret_cast<int16_t*>(smem + C::kOffOrder);
  int16_t* s_P = reinterpret_cast<int16_t*>(smem + C::kOffP);
  int16_t* s_nT = reinterpret_cast<int16_t*>(smem + C::kOffNT);
  const bool packed = args.cu_seqlens != nullptr;
  if (packed) {
    bool good = true;
    for (int b = threadIdx.x; b < args.B; b += blockDim.x) {
      const int t0 = args.cu_seqlens[b], t1 = args.cu_seqlens[b + 1];
      good = good && t1 >= t0 && t0 >= 0 && t1 <= args.total;
      s_tok[b] = t0;
      s_len[b] = t1 - t0;
    }
    if (threadIdx.x == 0)
      good = good && args.cu_seqlens[0] == 0 && args.cu_seqlens[args.B] == args.total;
    if (!__syncthreads_and(good)) {
      for (int b = threadIdx.x; b < args.B; b += blockDim.x) s_len[b] = 0;
      if (threadIdx.x == 0 && blockIdx.x == 0) atomicCAS(args.status, 0, EA_ERR_INVALID_ARG);
    }
  } else {
    for (int b = threadIdx.x; b < args.B; b += blockDim.x) {
      s_tok[b] = 0;
      s_len[b] = args.N;
    }
  }
  __syncthreads();
  // Sorted order: by block count, longest first, ties by index (a padded
  // batch keeps the identity order).
  for (int b = threadIdx.x; b < args.B; b += blockDim.x) {
    const int nb = ea_cdiv(s_len[b], EA_BN);
    int rank = b;
    if (packed) {
      rank = 0;
      for (int o = 0; o < args.B; ++o) {
        const int no = ea_cdiv(s_len[o], EA_BN);
        rank += (no > nb) || (no == nb && o < b);
      }
    }
    s_order[rank] = static_cast<int16_t>(b);
    s_nT[rank] = static_cast<int16_t>(nb);
    s_P[rank] = static_cast<int16_t>(ea_cdiv(nb, 2));
  }
  __syncthreads();
  // Entry runs (FA paired, FA single, SA paired, SA single), filtered by
  // args.select and the shard, each grouped by sorted sequence, kv groups in
  // order, heads increasing; a kv group's heads of one mode are paired two
  // by two, an odd one out is single (all single when a group has more than
  // EA_MAX_PAIR_GROUP heads).  Warp 0 builds them with ballots in two passes:
  // the prefix counts, then the heads at their positions.
  if (warp == 0) {
    const int Gq = args.Hq / args.Hkv;
    const bool pairing = Gq <= EA_MAX_PAIR_GROUP;
    // a chunk of lanes covers whole kv groups when pairing
    const int chunk = pairing ? (32 / Gq) * Gq : 32;
    const int gl = pairing ? (lane / Gq) * Gq : 0;
    const unsigned gmask =
        pairing ? ((Gq == 32 ? 0xffffffffu : ((1u << Gq) - 1u)) << gl) : 0u;
    const unsigned below = (1u << lane) - 1u;
    int run0[4] = {0, 0, 0, 0};
    for (int pass = 0; pass < 2; ++pass) {
      int cnt[4] = {0, 0, 0, 0};   // heads written to each run so far
      for (int k = 0; k < args.B; ++k) {
        const int b = s_order[k];
#pragma unroll
        for (int mode = 0; mode < 2; ++mode) {
          if (pass == 0 && lane == 0) {
            s_pref[(2 * mode) * C::kPrefLen + k] = static_cast<int16_t>(cnt[2 * mode] / 2);
            s_pref[(2 * mode + 1) * C::kPrefLen + k] = static_cast<int16_t>(cnt[2 * mode + 1]);
          }
          for (int h0 = 0; h0 < args.Hq; h0 += chunk) {
            const int h = h0 + lane;
            const int idx = b * args.Hq + h;
            const bool ok = lane < chunk && h < args.Hq &&
                            (args.both || (ld_mask(args.mask, idx) != 0) == (mode == 1)) &&
                            args.select != (mode == 1 ? EA_SELECT_FA : EA_SELECT_SA) &&
                            in_shard(args, b, h);
            const unsigned bits = __ballot_sync(0xffffffffu, ok);
            const int rank = __popc(bits & gmask & below);
            const int n = __popc(bits & gmask);
            const bool pr = ok && pairing && rank < (n & ~1);
            const unsigned pbits = __ballot_sync(0xffffffffu, pr);
            const unsigned sbits = __ballot_sync(0xffffffffu, ok && !pr);
            if (pass == 1 && ok) {
              const int pos = pr ? run0[2 * mode] + cnt[2 * mode] + __popc(pbits & below)
                                 : run0[2 * mode + 1] + cnt[2 * mode + 1] + __popc(sbits & below);
              s_ent[pos] = static_cast<uint16_t>(idx);
            }
            cnt[2 * mode] += __popc(pbits);
            cnt[2 * mode + 1] += __popc(sbits);
          }
        }
      }
      if (pass == 0) {
        if (lane == 0)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            s_pref[j * C::kPrefLen + args.B] = static_cast<int16_t>(j % 2 == 0 ? cnt[j] / 2 : cnt[j]);
        run0[1] = cnt[0];
        run0[2] = run0[1] + cnt[1];
        run0[3] = run0[2] + cnt[2];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = *s_tmem;
  EaSeqView view;
  view.nseq = args.B;
  view.nT = s_nT;
  view.P = s_P;
#pragma unroll
  for (int j = 0; j < 4; ++j) view.pref[j] = s_pref + j * C::kPrefLen;
  view.run0[0] = 0;
  view.run0[1] = 2 * view.pref[0][args.B];
  view.run0[2] = view.run0[1] + view.pref[1][args.B];
  view.run0[3] = view.run0[2] + 2 * view.pref[2][args.B];
  view.Pmax = args.B > 0 ? s_P[0] : 0;
  view.mA = ea_long_level(args.sink, args.window);
  const int total = ea_total_units(view);
  const int G = args.Hq / args.Hkv;
  const uint64_t tlim = args.timeout_ns;
  int* status = args.status;

  static_assert(2 * 128 * C::kRegsSoftmax + 128 * C::kRegsOther <= 384 * 168,
                "register split exceeds the launch budget");
  if (warp >= 8) {
    regs_dec<C::kRegsOther>();
    if (warp == 8) {
    // ============================================================ producer
    if (lane == 0) {
      uint32_t kv_pos = 0;
      uint32_t n_units = 0;
      bool ok = true;
      EaCursor cur;
      ea_cursor_init(cur, view, s_ent, args.Hq, args.Hkv, ea_group_major(view.Pmax, D));
      // Tickets come one unit ahead: the counter's reply (a global atomic, up
      // to microseconds under the launch's memory traffic) returns while this
      // unit's loads are issued, instead of delaying the next unit's Q load.
      unsigned int next_ticket = atomicAdd(args.ticket, 1u);
      for (int kk = 0; ok; ++kk) {
        // the next unit, published to the MMA and softmax warps through the
        // unit ring
        const int us = kk % C::kUnitRing;
        if (kk >= C::kUnitRing) {
          ok = mbar_wait(bars.unit_empty + 8 * us, ((kk / C::kUnitRing) - 1) & 1, s_abort, status,
                         tlim, EA_ERR_TIMEOUT);
          if (!ok) break;
        }
        const unsigned int ticket = next_ticket;
        const int r = ticket < static_cast<unsigned int>(total) ? static_cast<int>(ticket) : -1;
        EaUnitRef u = {0, 0, 0, 0};
        if (r >= 0) ea_cursor_seek(cur, view, s_ent, r, &u);
        const int idx = r >= 0 ? static_cast<int>(s_ent[u.pos]) : 0;
        const int idx1 = (r >= 0 && u.paired) ? static_cast<int>(s_ent[u.pos + 1]) : idx;
        // Only this thread runs the cursor: the other roles read the unit
        // decoded, {rank, level << 14 | paired << 13 | sparse << 12 | head
        // of slot 0, head of slot 1} (a head index is below 4096, a level
        // below 65536).
        s_unit[4 * us] = r;
        s_unit[4 * us + 1] = (u.level << 14) | (u.paired << 13) | (u.sparse << 12) | idx;
        s_unit[4 * us + 2] = idx1;
        mbar_arrive(bars.unit_full + 8 * us);
        if (r < 0) break;
        next_ticket = atomicAdd(args.ticket, 1u);
        const int sparse = u.sparse;
        const int b = idx / args.Hq, h = idx % args.Hq;
        // tensor coordinates: padded batch (row, head index b*H + h); packed
        // batch (token, head); both heads of a paired unit read kv head h / G
        const int tok = s_tok[b];
        const int kvz = packed ? h / G : b * args.Hkv + h / G;
        const EaShape shape = ea_make_shape(s_len[b], args.sink, args.window);
        const EaUnitTiles ut = ea_unit_tiles(shape, sparse, u.paired, u.level);
        if (n_units > 0) {
          ok = mbar_wait(bars.q_empty, (n_units - 1) & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(bars.q_full, ut.nslots * C::kTileBytes);
        for (int s = 0; s < ut.nslots; ++s) {
          const int qidx = s ? idx1 : idx;
          const int qz = packed ? qidx % args.Hq : qidx;
          for (int c = 0; c < C::kDBlocks; ++c)
            tma_load_3d(smem_u32(sQ) + s * C::kTileBytes + c * C::kBlockBytes, &args.tm_q, bars.q_full,
                        c * C::kBlockElems, tok + ut.r0 + s * ut.rstep, qz);
        }
        ++n_units;
        for (int i = 0; i < ut.n && ok; ++i) {
          const int t = ea_tile_at(ut, i);
          for (int which = 0; which < 2; ++which) {
            const uint32_t st = kv_pos % C::kStages;
            if (kv_pos >= static_cast<uint32_t>(C::kStages)) {
              ok = mbar_wait(bars.kv_empty + 8 * st, ((kv_pos / C::kStages) - 1) & 1, s_abort, status,
                             tlim, EA_ERR_TIMEOUT);
              if (!ok) break;
            }
#ifdef EA_TEST_HOOKS
            if (static_cast<int>(kv_pos) == args.debug_drop_kv_pos) {
              ++kv_pos;           // test build only: this copy never happens
              continue;
            }
#endif
            mbar_arrive_expect_tx(bars.kv_full + 8 * st, C::kTileBytes);
            const CUtensorMap* map = which ? &args.tm_v : &args.tm_k;
            if (kFp8 && which) {
              // V^T: the tile's 128 keys along the row, all d rows
              tma_load_3d(smem_u32(sKV) + st * C::kTileBytes, map, bars.kv_full + 8 * st,
                          tok + t * EA_BN, 0, kvz);
            } else {
              for (int c = 0; c < C::kDBlocks; ++c)
                tma_load_3d(smem_u32(sKV) + st * C::kTileBytes + c * C::kBlockBytes, map,
                            bars.kv_full + 8 * st, c * C::kBlockElems, tok + t * EA_BN, kvz);
            }
            ++kv_pos;
          }
        }
      }
      // Drain: every copy this thread issued must land before the CTA exits.
      const uint32_t nst = kv_pos < static_cast<uint32_t>(C::kStages) ? kv_pos : C::kStages;
      for (uint32_t p = kv_pos - nst; p < kv_pos; ++p)
        mbar_wait_drain(bars.kv_full + 8 * (p % C::kStages), (p / C::kStages) & 1, 200000000ull);
      if (n_units > 0) mbar_wait_drain(bars.q_full, (n_units - 1) & 1, 200000000ull);
    }
    __syncwarp();
    } else if (warp == 9) {
    // ============================================================ MMA issuer
    // Both slots' MMAs go out in the order PV0(i), S0(i+1), PV1(i), S1(i+1):
    // each group of eight MMAs is contiguous, and the tensor pipe always has
    // the other slot's group queued while a softmax runs.  The whole warp
    // runs this loop (its waits, tile lists and descriptors are warp-uniform
    // values) and the elected lane's tcgen05.mma / commit take effect: issued
    // from one lane inside a lane-0 branch, the same loop ran 5% slower on
    // every workload.  Only the MMAs and the waits they need are on this
    // path (K/V waits come from the async proxy and need no tcgen05 fence;
    // only P handoffs do).
    {
      const uint32_t leader = elect_one();
      uint32_t kv_pos = 0;
      uint32_t n_units = 0;
      uint32_t p_cnt[2] = {0, 0};
      uint32_t u_cnt[2] = {0, 0};
      bool ok = true;
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t kv_base = smem_u32(sKV);
      // Descriptors are built once; K steps add their byte offset >> 4 to the
      // 14-bit start-address field (all of shared memory is below 256 KB, so
      // the field never overflows).
      const uint64_t dq = smem_desc_sw128(q_base, 16, 1024);
      const uint64_t dkv_k = smem_desc_sw128(kv_base, 16, 1024);
      const uint64_t dkv_v = smem_desc_sw128(kv_base, C::kBlockBytes, 1024);
      auto issue_s = [&](int s, uint32_t st) {
        const uint64_t a0 = dq + ((s * C::kTileBytes) >> 4);
        const uint64_t b0 = dkv_k + ((st * C::kTileBytes) >> 4);
#pragma unroll
        for (int k = 0; k < C::kKSteps; ++k) {
          const uint32_t off = ((k >> 2) * C::kBlockBytes + (k & 3) * 32) >> 4;
          if (kFp8)
            mma_ss_f8_w(leader, tmem + s * 128, a0 + off, b0 + off, C::kIdescS, k > 0 ? 1u : 0u);
          else
            mma_ss_w(leader, tmem + s * 128, a0 + off, b0 + off, C::kIdescS, k > 0 ? 1u : 0u);
        }
      };
      // P from TMEM (32 bytes of keys = 8 columns per K step); B: bf16 V
      // MN-major (16 key rows per step), or e4m3 V^T K-major (32 key bytes)
      auto issue_pv = [&](int s, uint32_t st, bool acc, int k0, int k1) {
#pragma unroll
        for (int k = k0; k < k1; ++k) {
          if (kFp8)
            mma_ts_f8_w(leader, tmem + 256 + s * 128, tmem + s * 128 + k * 8,
                      dkv_k + ((st * C::kTileBytes + k * 32) >> 4), C::kIdescPV,
                      (acc || k > 0) ? 1u : 0u);
          else
            mma_ts_w(leader, tmem + 256 + s * 128, tmem + s * 128 + k * 8,
                   dkv_v + ((st * C::kTileBytes + k * 2048) >> 4), C::kIdescPV,
                   (acc || k > 0) ? 1u : 0u);
        }
      };
      for (int kk = 0; ok; ++kk) {
        const int us = kk % C::kUnitRing;
        ok = mbar_wait(bars.unit_full + 8 * us, (kk / C::kUnitRing) & 1, s_abort, status, tlim,
                       EA_ERR_TIMEOUT);
        if (!ok) break;
        const int r = s_unit[4 * us];
        const int word = s_unit[4 * us + 1];
        __syncwarp();
        if (leader) mbar_arrive(bars.unit_empty + 8 * us);
        if (r < 0) break;
        const int sparse = (word >> 12) & 1, idx = word & 4095;
        const EaShape shape = ea_make_shape(s_len[idx / args.Hq], args.sink, args.window);
        const EaUnitTiles ut = ea_unit_tiles(shape, sparse, (word >> 13) & 1, word >> 14);

        ok = mbar_wait(bars.q_full, n_units & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
        if (!ok) break;
        ++n_units;

        // K of the first tile, then S for every slot that sees it.
        {
          const uint32_t st = kv_pos % C::kStages;
          ok = mbar_wait(bars.kv_full + 8 * st, (kv_pos / C::kStages) & 1, s_abort, status, tlim,
                         EA_ERR_TIMEOUT);
          if (!ok) break;
          const int t0 = ea_tile_at(ut, 0);
          for (int s = 0; s < 2; ++s)
            if (ea_tile_code(shape, ut, sparse, s, t0)) {
              issue_s(s, st);
              mma_commit_w(leader, bars.s_full + 8 * s);
            }
          mma_commit_w(leader, bars.kv_empty + 8 * st);
        }
        bool first_pv[2] = {true, true};
        for (int i = 0; i < ut.n && ok; ++i) {
          const uint32_t vpos = kv_pos + 2 * i + 1;
          const uint32_t vst = vpos % C::kStages;
          ok = mbar_wait(bars.kv_full + 8 * vst, (vpos / C::kStages) & 1, s_abort, status, tlim,
                         EA_ERR_TIMEOUT);
          if (!ok) break;
          const bool has_next = i + 1 < ut.n;
          uint32_t kst = 0;
          if (has_next) {
            const uint32_t kpos = kv_pos + 2 * (i + 1);
            kst = kpos % C::kStages;
            ok = mbar_wait(bars.kv_full + 8 * kst, (kpos / C::kStages) & 1, s_abort, status,
                           tlim, EA_ERR_TIMEOUT);
            if (!ok) break;
          }
          const int t = ea_tile_at(ut, i);
          const int tn = has_next ? ea_tile_at(ut, i + 1) : 0;
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            if (ea_tile_code(shape, ut, sparse, s, t)) {
              ok = mbar_wait(bars.p_half + 8 * s, p_cnt[s] & 1, s_abort, status, tlim,
                             EA_ERR_TIMEOUT);
              if (!ok) break;
              if (first_pv[s]) {
                if (u_cnt[s] > 0) {
                  ok = mbar_wait(bars.o_empty + 8 * s, (u_cnt[s] - 1) & 1, s_abort, status, tlim,
                                 EA_ERR_TIMEOUT);
                  if (!ok) break;
                }
                ++u_cnt[s];
              }
              // P.V over the first 64 keys as soon as their P is stored,
              // the rest when the whole P is
              tc_fence_after();
              issue_pv(s, vst, !first_pv[s], 0, C::kPVSteps / 2);
              ok = mbar_wait(bars.p_full + 8 * s, p_cnt[s] & 1, s_abort, status, tlim,
                             EA_ERR_TIMEOUT);
              if (!ok) break;
              ++p_cnt[s];
              tc_fence_after();
              issue_pv(s, vst, true, C::kPVSteps / 2, C::kPVSteps);
              first_pv[s] = false;
              mma_commit_w(leader, bars.o_done + 8 * s);
            }
            if (has_next && ea_tile_code(shape, ut, sparse, s, tn)) {
              issue_s(s, kst);
              mma_commit_w(leader, bars.s_full + 8 * s);
            }
          }
          if (!ok) break;
          mma_commit_w(leader, bars.kv_empty + 8 * vst);
          if (has_next) mma_commit_w(leader, bars.kv_empty + 8 * kst);
        }
        if (!ok) break;
        mma_commit_w(leader, bars.q_empty);
        kv_pos += 2 * ut.n;
      }
      // Drain: wait for every MMA the elected lane issued.
      mma_commit_w(leader, bars.drain);
      mbar_wait_drain(bars.drain, 0, 200000000ull);
    }
    __syncwarp();
    }
  } else {
    regs_inc<C::kRegsSoftmax>();
    // ============================================================ softmax
    const int slot = warp >> 2;
    const int wq = warp & 3;
    const int row_local = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + slot * 128;
    const uint32_t tO = tmem + lane_off + 256 + slot * 128;
    uint32_t s_cnt = 0;
    uint32_t pv_cnt = 0;
    bool ok = true;
    for (int kk = 0; ok; ++kk) {
      const int us = kk % C::kUnitRing;
      ok = mbar_wait(bars.unit_full + 8 * us, (kk / C::kUnitRing) & 1, s_abort, status, tlim,
                     EA_ERR_TIMEOUT);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int r = s_unit[4 * us];
      const int word = s_unit[4 * us + 1];
      const int idx1 = s_unit[4 * us + 2];
      __syncwarp();
      if (lane == 0) mbar_arrive(bars.unit_empty + 8 * us);
      if (r < 0) break;
      const int sparse = (word >> 12) & 1;
      const int idx = slot ? idx1 : (word & 4095);   // this slot's head
      const int seq = idx / args.Hq;
      const int seq_len = s_len[seq];
      const EaShape shape = ea_make_shape(seq_len, args.sink, args.window);
      const EaUnitTiles ut = ea_unit_tiles(shape, sparse, (word >> 13) & 1, word >> 14);
      if (slot >= ut.nslots) continue;
      const bool tracing = kTrace && warp == 0 && lane == 0;
      if (tracing) {
        s_trace_ts[0] = global_ns();
        s_trace_ts[1] = 0;
        s_trace_ts[2] = 0;
      }
      const int row = ut.r0 + slot * ut.rstep + row_local;   // global query row
      // does some row of this slot see fewer than 128 keys?  (the count of
      // visible keys grows with the row, so the slot's first row decides)
      const int r0s = ut.r0 + slot * ut.rstep;
      const int keys0 = sparse ? ea_min(r0s + 1, args.window) +
                                     ea_min(args.sink, ea_max(0, r0s - args.window + 1))
                               : r0s + 1;
      const bool few_keys = keys0 < 128;
      // FP8: the scores carry the q and k dequantization scales
      const int kvh = seq * args.Hkv + (idx % args.Hq) / G;
      const float sl2 = kFp8 ? args.scale_log2 * args.q_scale[idx] * args.k_scale[kvh]
                             : args.scale_log2;
      float m_ref = -INFINITY;
      float l = 0.f;
      bool has_o = false;
      for (int i = 0; i < ut.n; ++i) {
        const int t = ea_tile_at(ut, i);
        const int code = ea_tile_code(shape, ut, sparse, slot, t);
        if (!code) continue;
        ok = mbar_wait(bars.s_full + 8 * slot, s_cnt & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++s_cnt;
        if (tracing && s_trace_ts[1] == 0) s_trace_ts[1] = global_ns();   // first S ready
        tc_fence_after();
        float x[128];
        {
          uint32_t raw[128];
          tmem_ld128_wait(tS, raw);
#pragma unroll
          for (int j = 0; j < 128; ++j) x[j] = __uint_as_float(raw[j]);
        }
        if (code == 2) {
          const int c0 = t * EA_BN;
          // visible key j (local): j <= row - c0, and for SA also
          // (j < sink - c0 || j >= row - window + 1 - c0); built as a
          // 128-bit mask, four words of intervals, then one bit test per key
          const int lim = row - c0;
          const int sink_hi = sparse ? args.sink - c0 : 1 << 30;
          const int win_lo = sparse ? row - args.window + 1 - c0 : -(1 << 30);
          uint32_t vm[4];
#pragma unroll
          for (int w = 0; w < 4; ++w)
            vm[w] = bits_below(lim + 1 - 32 * w) &
                    (bits_below(sink_hi - 32 * w) | ~bits_below(win_lo - 32 * w));
#pragma unroll
          for (int j = 0; j < 128; ++j)
            if (!((vm[j >> 5] >> (j & 31)) & 1u)) x[j] = -INFINITY;
        }
        // row max: eight independent chains of three-input max over x[8..119],
        // the last eight columns, then a tree
        float mk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mk[k] = x[k];
#pragma unroll
        for (int j = 8; j < 120; j += 16) {
#pragma unroll
          for (int k = 0; k < 8; ++k) mk[k] = max3f(mk[k], x[j + k], x[j + 8 + k]);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) mk[k] = fmaxf(mk[k], x[120 + k]);
        const float mx = max3f(max3f(mk[0], mk[1], mk[2]), max3f(mk[3], mk[4], mk[5]),
                               fmaxf(mk[6], mk[7]));
        const float m_tile = mx * sl2;
        bool rescale = false;
        float alpha = 1.f;
        if (m_tile > m_ref + 8.f) {
          alpha = ex2_approx(m_ref - m_tile);
          rescale = has_o && (m_ref != -INFINITY);
          l *= alpha;
          m_ref = m_tile;
        }
        const float msub = (m_ref == -INFINITY) ? 0.f : m_ref;
        // p = 2^(s * scale * log2e - m)
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.f;
        if constexpr (kFp8) {
          // e4m3 P, four keys per column (32 columns); the row sum adds the
          // unrounded values
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float p0, p1, p2, p3;
            fma2_sc(p0, p1, x[4 * j], x[4 * j + 1], sl2, -msub);
            fma2_sc(p2, p3, x[4 * j + 2], x[4 * j + 3], sl2, -msub);
            if ((j & 7) < kEmuQuadsFp8) {
              exp2_poly2(p0, p1);
              exp2_poly2(p2, p3);
            } else {
              p0 = ex2_approx(p0);
              p1 = ex2_approx(p1);
              p2 = ex2_approx(p2);
              p3 = ex2_approx(p3);
            }
            pk[j] = pack_e4m3x4(p0, p1, p2, p3);
            add2_acc(acc[2 * (j & 3)], acc[2 * (j & 3) + 1], p0 + p2, p1 + p3);
          }
          tmem_st32(tS, pk);
        } else {
          // a tile with masked pairs (code 2) holds every key of the rows
          // that see fewer than 128 keys; in a slot that has such rows the
          // row sum adds the bf16-rounded probabilities there, so their
          // weights sum to one exactly (a one-key row gives v itself)
          if (code == 2 && few_keys)
            softmax_p_bf16<true, 0, 2>(x, sl2, msub, tS, acc);
          else
            softmax_p_bf16<false, 0, 2>(x, sl2, msub, tS, acc);
        }
        // O is rescaled (rarely) before the first half of P is handed over,
        // so the first half's P.V product accumulates onto the rescaled O;
        // the previous P.V is complete, since this tile's S product followed
        // it on the same issuing thread
        if (__any_sync(0xffffffffu, rescale)) {
          ok = mbar_wait(bars.o_done + 8 * slot, (pv_cnt - 1) & 1, s_abort, status, tlim,
                         EA_ERR_TIMEOUT);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          const float a = rescale ? alpha : 1.f;
#pragma unroll
          for (int h = 0; h < D / 64; ++h) {
            uint32_t o[64];
            tmem_ld64_wait(tO + h * 64, o);
#pragma unroll
            for (int j = 0; j < 64; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * a);
            tmem_st64(tO + h * 64, o);
          }
        }
        // the first 64 keys' P: the issuer starts their P.V while the
        // second half is computed
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bars.p_half + 8 * slot);
        if constexpr (!kFp8) {
          if (code == 2 && few_keys)
            softmax_p_bf16<true, 2, 4>(x, sl2, msub, tS, acc);
          else
            softmax_p_bf16<false, 2, 4>(x, sl2, msub, tS, acc);
        }
        l += ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bars.p_full + 8 * slot);
        ++pv_cnt;
        has_o = true;
      }
      if (!ok) break;
      if (tracing) s_trace_ts[2] = global_ns();   // the unit's last P is handed over
      // Epilogue: O / l -> bf16 -> out[b, h, row, :].
      ok = mbar_wait(bars.o_done + 8 * slot, (pv_cnt - 1) & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float inv_l = kFp8 ? args.v_scale[kvh] / l : 1.f / l;
      // a training forward's other mode goes to out_other, without lse
      const bool chosen = !args.both || (sparse != 0) == (ld_mask(args.mask, idx) != 0);
      if (chosen && args.lse != nullptr && !packed && row < seq_len)   // for the backward
        args.lse[static_cast<size_t>(idx) * args.N + row] = (m_ref + __log2f(l)) * 0.6931471805599453f;
      // out row: padded [B][Hq][N][d]; packed [T][Hq][d]
      const size_t orow_index =
          packed ? (static_cast<size_t>(s_tok[seq] + row) * args.Hq + idx % args.Hq)
                 : (static_cast<size_t>(idx) * args.N + row);
      __nv_bfloat16* orow =
          reinterpret_cast<__nv_bfloat16*>(chosen ? args.out : args.out_other) + orow_index * D;
      // 32-byte stores when the output base is 32-byte aligned (every row
      // starts a multiple of 2 d bytes after it), else 16-byte ones
      const bool st32 =
          (reinterpret_cast<uintptr_t>(chosen ? args.out : args.out_other) & 31u) == 0;
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        uint32_t o[64];
        tmem_ld64_wait(tO + h * 64, o);
        if (row < seq_len) {
          uint32_t w[32];
#pragma unroll
          for (int j = 0; j < 32; ++j)
            w[j] = pack_bf16x2(__uint_as_float(o[2 * j]) * inv_l,
                               __uint_as_float(o[2 * j + 1]) * inv_l);
          if (st32) {
#pragma unroll
            for (int q = 0; q < 4; ++q) st_global_v8(orow + h * 64 + 16 * q, &w[8 * q]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow + h * 64);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bars.o_empty + 8 * slot);
      if (tracing) {
        // slot 0's rows are stored: the unit's record (the end stamped before
        // the record's slot is taken, so the atomic's round trip is not in it)
        const unsigned long long t_end = global_ns();
        const unsigned long long k = atomicAdd(args.trace, 1ull);
        if (k < static_cast<unsigned long long>(args.trace_max)) {
          unsigned long long* rec = args.trace + 8 + 6 * k;
          rec[0] = s_trace_ts[0];
          rec[1] = s_trace_ts[1];
          rec[2] = s_trace_ts[2];
          rec[3] = t_end;
          rec[4] = (static_cast<unsigned long long>(blockIdx.x) << 48) |
                   (static_cast<unsigned long long>(word >> 14) << 32) | static_cast<unsigned>(r);
          rec[5] = (static_cast<unsigned long long>(sparse) << 62) |
                   (static_cast<unsigned long long>(word & 4095) << 44) |
                   (static_cast<unsigned long long>(idx1) << 32) | static_cast<unsigned>(ut.n);
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  release_dispatch(args);
}

int attn_smem_bytes(int D) {
  return D == 128 ? AttnCfg<128>::kSmem : AttnCfg<64>::kSmem;
}

template <int D, bool kRouted, bool kFp8 = false, bool kTrace = false>
static cudaError_t launch_d(const AttnArgs& args_in, int grid, cudaStream_t stream) {
  const int smem = AttnCfg<D, kFp8>::kSmem;
  // the dispatch counters sit in the caller's status block (status word at
  // 0, the routed prologue's grid barrier at 64 and 128)
  AttnArgs args = args_in;
  args.ticket = reinterpret_cast<unsigned int*>(reinterpret_cast<char*>(args.status) + 192);
  args.done_ctas = reinterpret_cast<unsigned int*>(reinterpret_cast<char*>(args.status) + 224);
  static int configured[64] = {0};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev >= 64 || !configured[dev]) {
    err = cudaFuncSetAttribute(ea_hybrid_attn_kernel<D, kRouted, kFp8, kTrace>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    if (dev < 64) configured[dev] = 1;
  }
  if (!kRouted) {
    ea_hybrid_attn_kernel<D, false, kFp8, kTrace><<<grid, AttnCfg<D, kFp8>::kThreads, smem, stream>>>(args);
    return cudaGetLastError();
  }
  // every CTA must be resident at once: the runtime refuses a cooperative
  // launch that cannot be
  void* params[] = {const_cast<AttnArgs*>(&args)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(ea_hybrid_attn_kernel<D, true>),
                                     dim3(grid), dim3(AttnCfg<D>::kThreads), params, smem, stream);
}

cudaError_t launch_attn(int D, const AttnArgs& args, int grid, cudaStream_t stream) {
  const bool trace = args.trace != nullptr;
  if (D == 128)
    return trace ? launch_d<128, false, false, true>(args, grid, stream)
                 : launch_d<128, false>(args, grid, stream);
  if (D == 64)
    return trace ? launch_d<64, false, false, true>(args, grid, stream)
                 : launch_d<64, false>(args, grid, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_fp8(const AttnArgs& args, int grid, cudaStream_t stream) {
  return launch_d<128, false, true>(args, grid, stream);
}

cudaError_t launch_attn_routed(int D, const AttnArgs& args, int grid, cudaStream_t stream) {
  if (D == 128) return launch_d<128, true>(args, grid, stream);
  if (D == 64) return launch_d<64, true>(args, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ea
