// ea_decode.cu — one decode step of hybrid FA/SA attention with a per-head
// KV-cache policy.
//
// Elastic Attention blog (bxzpzcl.cn) §3: fusing the two modes lowers memory
// use as well as time.  In decode that saving is the cache: a head routed to
// Sparse Attention only ever reads its S sink keys and its last W keys, so a
// kv head whose query heads are all SA keeps a compact cache of S + W rows
// (sinks fixed, the rest a ring of W slots), while a kv head with at least one
// FA query head keeps every position.  The query at position t sees exactly
// the keys prefill row t sees (FA: 0..t; SA: sink + window).
//
// Step, two launches on the caller's stream:
//   1. append: the new k, v of every (b, kv head) go to their cache slot;
//   2. attention: one persistent CTA per SM walks the (kv group, 512-key
//      chunk) items that hold visible keys.  A producer warp streams each
//      item's cache rows into shared memory with bulk copies (a group's
//      visible keys are at most four contiguous row runs of its cache:
//      sinks, window, and the two sides of the ring wrap); eight consumer
//      warps read every row once for all G query heads of the group, keep an
//      fp32 online softmax per head and write one partial (o, max, sum) per
//      item and head to the workspace;
//      the CTA that completes a group's last item merges the group's partials
//      in chunk order and writes the bf16 output.
// The step is HBM-bound: its work is one read of every visible cache row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ea.h"
#include "ea_internal.h"
#include "ea_math.cuh"
#include "ea_ptx.cuh"

namespace ea {

constexpr int kDecChunk = 512;           // smallest work item (keys): bounds the partials

struct DecodeArgs {
  const __nv_bfloat16* q;      // [B][Hq][d]
  const __nv_bfloat16* k_new;  // [B][Hkv][d]
  const __nv_bfloat16* v_new;
  const int32_t* pos;          // [B]
  const uint8_t* mask;         // [B][Hq]
  const int32_t* cache_slot;   // [B][Hkv]: >= 0 full cache index, < 0 compact -(i)-1
  __nv_bfloat16* k_full;       // [n_full][max_len][d]
  __nv_bfloat16* v_full;
  __nv_bfloat16* k_sa;         // [n_sa][sink + window][d]
  __nv_bfloat16* v_sa;
  __nv_bfloat16* out;          // [B][Hq][d]
  float* part;                 // [B][Hq][nsplit][d + 2]: o, max, sum
  int* counters;               // [B][Hkv][2]: segments of each virtual group finished this step
  int* status;
  int B, Hq, Hkv, d, sink, window, max_len, nsplit, n_full, n_sa;
  float scale_log2;
  unsigned long long timeout_ns;   // bound of every barrier wait
};

__device__ __forceinline__ int dec_compact_slot(int p, int sink, int window) {
  return p < sink ? p : sink + (p - sink) % window;
}

// Visible positions of the kv group at query position t, as [0, a) then
// [lo, t]: every position for a group with an FA query head (or a full
// cache), else the sink and window positions.
__device__ __forceinline__ void dec_group_keys(bool all_sparse, int t, int sink, int window,
                                               int* a, int* lo) {
  if (!all_sparse) {
    *a = 0;
    *lo = 0;
  } else {
    *lo = max(0, t - window + 1);
    *a = min(sink, *lo);
  }
}

// A (b, kv head) whose cache slot or position lies outside its cache is
// neither written nor read.
__device__ __forceinline__ bool dec_slot_ok(const DecodeArgs& a, int slot, int t) {
  if (t < 0) return false;
  if (slot >= 0) return slot < a.n_full && t < a.max_len;
  return -slot - 1 < a.n_sa;
}

__global__ void ea_decode_append_kernel(DecodeArgs args) {
  const int b = blockIdx.y, hk = blockIdx.x;
  const int t = args.pos[b];
  const int slot = args.cache_slot[b * args.Hkv + hk];
  if (threadIdx.x < 2) args.counters[2 * (b * args.Hkv + hk) + threadIdx.x] = 0;
  if (!dec_slot_ok(args, slot, t)) {
    if (threadIdx.x == 0) atomicCAS(args.status, 0, EA_ERR_INVALID_ARG);
    // no work item reads or writes this group: its outputs are zero
    const int G = args.Hq / args.Hkv;
    __nv_bfloat16* o = args.out + (static_cast<size_t>(b) * args.Hq + hk * G) * args.d;
    for (int i = threadIdx.x; i < G * args.d; i += blockDim.x) o[i] = __float2bfloat16_rn(0.f);
    return;
  }
  if (slot < 0 && threadIdx.x == 0) {   // a compact cache behind an FA query head
    const int G = args.Hq / args.Hkv;
    for (int g = 0; g < G; ++g)
      if (args.mask[b * args.Hq + hk * G + g] == 0) {
        atomicCAS(args.status, 0, EA_ERR_INVALID_ARG);
        break;
      }
  }
  __nv_bfloat16* kd;
  __nv_bfloat16* vd;
  size_t row;
  if (slot >= 0) {
    kd = args.k_full;
    vd = args.v_full;
    row = static_cast<size_t>(slot) * args.max_len + t;
  } else {
    kd = args.k_sa;
    vd = args.v_sa;
    row = static_cast<size_t>(-slot - 1) * (args.sink + args.window) +
          dec_compact_slot(t, args.sink, args.window);
  }
  const size_t src = (static_cast<size_t>(b) * args.Hkv + hk) * args.d;
  for (int c = threadIdx.x; c < args.d / 8; c += blockDim.x) {
    reinterpret_cast<uint4*>(kd + row * args.d)[c] =
        reinterpret_cast<const uint4*>(args.k_new + src)[c];
    reinterpret_cast<uint4*>(vd + row * args.d)[c] =
        reinterpret_cast<const uint4*>(args.v_new + src)[c];
  }
}

// Keys and query heads of virtual group (b, hk, part) at this step.  A kv
// group whose query heads are all FA or all SA (or that sits on a compact
// cache) is one virtual group, part 0.  A group on a full cache with both
// kinds of heads is two: part 0 = its FA heads over every position 0..t,
// part 1 = its SA heads over the sink and window positions.  Every head of a
// virtual group sees exactly the group's key list, so nothing is masked
// inside a list and no SA head spends work on keys it does not see.
struct DecVGroup {
  int t, slot, a, lo, nvis;   // keys: [0, a) then [lo, t]; nvis of them (0: empty part)
  bool compact;
  uint32_t heads;             // bit g: query head hk * G + g belongs to this part
};

__device__ __forceinline__ DecVGroup dec_vgroup(const DecodeArgs& args, int b, int hk, int part,
                                                int G) {
  DecVGroup v;
  v.t = args.pos[b];
  v.slot = args.cache_slot[b * args.Hkv + hk];
  v.compact = v.slot < 0;
  uint32_t sparse = 0;
  for (int i = 0; i < G; ++i)
    sparse |= static_cast<uint32_t>(args.mask[b * args.Hq + hk * G + i] != 0) << i;
  const uint32_t all = (1u << G) - 1u;
  const bool split = sparse != 0 && sparse != all && !v.compact;
  bool sa_keys;
  if (!split) {
    v.heads = part == 0 ? all : 0u;
    sa_keys = sparse == all || v.compact;
  } else {
    v.heads = part == 0 ? (all & ~sparse) : sparse;
    sa_keys = part == 1;
  }
  dec_group_keys(sa_keys, v.t, args.sink, args.window, &v.a, &v.lo);
  v.nvis = (v.heads != 0 && dec_slot_ok(args, v.slot, v.t)) ? v.a + (v.t - v.lo + 1) : 0;
  return v;
}

// One stage of a segment, written by the producer before it arms the stage's
// full barrier.  n < 0 ends the stream.
struct DecDesc {
  int n;               // key rows in the stage
  int first, last;     // first / last stage of the segment
  int b, hk, vg;       // batch row, kv head, virtual group (2 * (b * Hkv + hk) + part)
  int seg, nseg;       // this CTA's segment of the virtual group, and its segment count
  uint32_t heads;      // query heads of the virtual group (bit g: head hk * G + g)
  int pad[7];
};

// Balanced contiguous split of `total` items over `grid` CTAs: CTA c owns
// [dec_range_begin(c), dec_range_begin(c + 1)).
__device__ __forceinline__ int dec_range_begin(int c, int total, int grid) {
  const int q = total / grid, r = total % grid;
  return c * q + min(c, r);
}
// The CTA whose range holds item i.
__device__ __forceinline__ int dec_cta_of(int i, int total, int grid) {
  const int q = total / grid, r = total % grid;
  const int big = r * (q + 1);
  return i < big ? i / (q + 1) : r + (i - big) / q;
}

// Consumer warps: 3 warpgroups for G <= 2 (q and o of a lane take at most
// 16 + 16 register pairs), 2 for G = 4 and 8 (32 + 32 pairs: 16 channels x 4
// heads, 8 channels x 8 heads); 3 warpgroups at 8 channels per lane measured
// slower for G = 4 (one more shuffle level per key).  The last warpgroup is
// the producer.  Register split (setmaxnreg) against the launch's 65536:
//   G <= 2:   512 threads launched at 128: 128 * 32 + 384 * 160 = 65536
//   G = 4, 8: 384 threads launched at 168: 128 * 56 + 256 * 224 = 64512
template <int G>
struct DecWarps {
  static constexpr int kConsumers = (G <= 2) ? 12 : 8;
  static constexpr int kThreads = (kConsumers + 4) * 32;
  static constexpr int kLaunchRegs = (G <= 2) ? 128 : 168;
  static constexpr int kRegsProducer = (G <= 2) ? 32 : 56;
  static constexpr int kRegsConsumer = (G <= 2) ? 160 : 224;
  static_assert(128 * kRegsProducer + kConsumers * 32 * kRegsConsumer <= kThreads * kLaunchRegs,
                "register split exceeds the launch's registers");
  static_assert(kThreads * kLaunchRegs <= 65536, "launch registers");
};
constexpr int kDecMaxGroups = 4096;        // B * Hkv
constexpr float kDecNegBig = -1.0e30f;     // running max before the first key
constexpr float kDecRescale = 8.0f;        // rescale only when the max grows by > 2^8

template <int D, int G>
struct DecLayout {
  static constexpr int kCW = DecWarps<G>::kConsumers;
  static constexpr int kDPL = (G == 8) ? 8 : 16;     // channels per lane
  static constexpr int kLPR = D / kDPL;              // lanes per key row
  static constexpr int kChunks = kDPL / 8;           // 16-byte chunks per lane
  static constexpr int kP = kDPL / 2;                // channel pairs per lane
  static constexpr int kRGW = 32 / kLPR;             // row groups per warp
  static constexpr int kNG = kCW * kRGW;
  static constexpr int kRowBytes = D * 2;
  static constexpr int kStageRows = kNG * ((kDPL == 8) ? 4 : 2);   // rows per group: 4 or 2
  static constexpr int kChunkRows = (kCW == 12) ? 576 : 512;  // keys per work item
  static constexpr int kRPS = kStageRows / kNG;      // rows per group per stage
  static constexpr int kRB = (G == 8) ? 2 : kRPS;    // rows per batch (registers)
  static constexpr int kStages = (kCW == 12) ? 3 : 4;
  static constexpr int kKV = kStageRows * kRowBytes;
  static constexpr int kQ = G * D * 2;
  static constexpr int off_k = 0;
  static constexpr int off_v = off_k + kStages * kKV;
  static constexpr int off_q = off_v + kStages * kKV;
  static constexpr int off_desc = off_q + kStages * kQ;
  static constexpr int off_full = off_desc + kStages * static_cast<int>(sizeof(DecDesc));
  static constexpr int off_empty = off_full + kStages * 8;
  static constexpr int off_flag = off_empty + kStages * 8;    // abort flag, last-segment flag
  static constexpr int off_mo = off_flag + 16;
  static constexpr int off_ml = off_mo + kCW * G * D * 4;
  static constexpr int off_table = off_ml + kCW * G * 2 * 4;
  // item table: one entry per virtual group (two per kv group) plus one
  static constexpr int bytes(int ngroups) { return off_table + (2 * ngroups + 1) * 4; }
  static_assert(bytes(kDecMaxGroups) <= 232448, "shared memory per CTA");
  static_assert(kStageRows % kNG == 0 && kRPS >= 1 && kRPS % kRB == 0, "stage rows");
  static_assert(kChunkRows % kStageRows == 0 && kChunkRows >= kDecChunk, "chunk rows");
  static_assert(sizeof(DecDesc) == 64, "descriptor size");
  static_assert(off_full % 8 == 0 && off_q % 16 == 0 && kKV % 16 == 0, "alignment");
};

template <int kCW>
__device__ __forceinline__ void named_bar_consumers() {
  asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
}

// Packed f32x2 values held in one 64-bit register pair (low word = first
// element), so the paired FMA needs no moves.
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
  uint64_t r;
  asm("{\n\t.reg .b32 lo, hi;\n\t"
      "shl.b32 lo, %1, 16;\n\t"
      "and.b32 hi, %1, 0xffff0000;\n\t"
      "mov.b64 %0, {lo, hi};\n\t}"
      : "=l"(r) : "r"(w));
  return r;
}
__device__ __forceinline__ void ffma2(uint64_t& c, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(c) : "l"(a), "l"(b));
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t pack2(float x, float y) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t a, float& x, float& y) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x), "=f"(y) : "l"(a));
}

// One stage of a virtual group whose NA query heads sit in slots 0..NA-1 of
// the state arrays.  Every row of the stage is a key all NA heads see; rows
// at and past n (a partial last stage) hold stale bytes and are skipped.
// Per batch of rows: the NA dot products of each row (kLPR lanes, reduced by
// interleaved shuffles), one running-max update (rescale only when the max
// grows by more than 2^8), then P.V.
template <class L, int G, int NA>
__device__ __forceinline__ void dec_stage(int n, const uint8_t* ks, const uint8_t* vs, int rg,
                                          int cl, const uint64_t (&q2)[G][L::kP],
                                          uint64_t (&o2)[G][L::kP], float (&m)[G],
                                          float (&l)[G]) {
  const bool full = n == L::kStageRows;
#pragma unroll
  for (int kb = 0; kb < L::kRPS; kb += L::kRB) {
    uint4 kr[L::kRB][L::kChunks], vr[L::kRB][L::kChunks];
    bool valid[L::kRB];
#pragma unroll
    for (int kk = 0; kk < L::kRB; ++kk) {
      const int r = rg + (kb + kk) * L::kNG;
      valid[kk] = full || r < n;
#pragma unroll
      for (int i = 0; i < L::kChunks; ++i) {
        const int off = r * L::kRowBytes + (cl + i * L::kLPR) * 16;
        kr[kk][i] = *reinterpret_cast<const uint4*>(ks + off);
        vr[kk][i] = *reinterpret_cast<const uint4*>(vs + off);
      }
    }
    if (!full) {
      // never multiply stale bytes
#pragma unroll
      for (int kk = 0; kk < L::kRB; ++kk)
#pragma unroll
        for (int i = 0; i < L::kChunks; ++i)
          if (!valid[kk]) vr[kk][i] = make_uint4(0, 0, 0, 0);
    }
    float sc[L::kRB][NA];
#pragma unroll
    for (int kk = 0; kk < L::kRB; ++kk) {
      uint64_t acc[NA];
#pragma unroll
      for (int h = 0; h < NA; ++h) acc[h] = 0ull;
#pragma unroll
      for (int i = 0; i < L::kChunks; ++i) {
        const uint32_t w[4] = {kr[kk][i].x, kr[kk][i].y, kr[kk][i].z, kr[kk][i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint64_t k2 = bf16x2_to_f32x2(w[e]);
#pragma unroll
          for (int h = 0; h < NA; ++h) ffma2(acc[h], q2[h][i * 4 + e], k2);
        }
      }
#pragma unroll
      for (int h = 0; h < NA; ++h) {
        float x, y;
        unpack2(acc[h], x, y);
        sc[kk][h] = x + y;
      }
    }
#pragma unroll
    for (int off = L::kLPR / 2; off > 0; off >>= 1)
#pragma unroll
      for (int kk = 0; kk < L::kRB; ++kk)
#pragma unroll
        for (int h = 0; h < NA; ++h) sc[kk][h] += __shfl_xor_sync(0xffffffffu, sc[kk][h], off);
    if (!full) {
#pragma unroll
      for (int kk = 0; kk < L::kRB; ++kk)
#pragma unroll
        for (int h = 0; h < NA; ++h) sc[kk][h] = valid[kk] ? sc[kk][h] : -INFINITY;
    }
    // one branch per batch: rescale every head whose max grew by > 2^8
    float mx[NA];
    bool grow = false;
#pragma unroll
    for (int h = 0; h < NA; ++h) {
      mx[h] = sc[0][h];
#pragma unroll
      for (int kk = 1; kk < L::kRB; ++kk) mx[h] = fmaxf(mx[h], sc[kk][h]);
      grow = grow || mx[h] > m[h] + kDecRescale;
    }
    if (grow) {
#pragma unroll
      for (int h = 0; h < NA; ++h) {
        const bool up = mx[h] > m[h] + kDecRescale;
        const float alpha = up ? ex2_approx(m[h] - mx[h]) : 1.0f;
        m[h] = up ? mx[h] : m[h];
        l[h] *= alpha;
        const uint64_t a2 = pack2(alpha, alpha);
#pragma unroll
        for (int e = 0; e < L::kP; ++e) o2[h][e] = fmul2(o2[h][e], a2);
      }
    }
#pragma unroll
    for (int kk = 0; kk < L::kRB; ++kk) {
      uint64_t p2[NA];
#pragma unroll
      for (int h = 0; h < NA; ++h) {
        const float pr = ex2_approx(sc[kk][h] - m[h]);
        l[h] += pr;
        p2[h] = pack2(pr, pr);
      }
#pragma unroll
      for (int i = 0; i < L::kChunks; ++i) {
        const uint32_t w[4] = {vr[kk][i].x, vr[kk][i].y, vr[kk][i].z, vr[kk][i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint64_t v2 = bf16x2_to_f32x2(w[e]);
#pragma unroll
          for (int h = 0; h < NA; ++h) ffma2(o2[h][i * 4 + e], p2[h], v2);
        }
      }
    }
  }
}

// Run the stage body compiled for exactly `nact` heads (1 <= nact <= NA).
// One body per head count: padding a smaller head set up to a larger body
// measured slower on mixed groups than the extra code costs.
template <class L, int G, int NA>
__device__ __forceinline__ void dec_stage_dispatch(int nact, int n, const uint8_t* ks,
                                                   const uint8_t* vs, int rg, int cl,
                                                   const uint64_t (&q2)[G][L::kP],
                                                   uint64_t (&o2)[G][L::kP], float (&m)[G],
                                                   float (&l)[G]) {
  if (NA == 1 || nact == NA) {
    dec_stage<L, G, NA>(n, ks, vs, rg, cl, q2, o2, m, l);
    return;
  }
  if constexpr (NA > 1) dec_stage_dispatch<L, G, NA - 1>(nact, n, ks, vs, rg, cl, q2, o2, m, l);
}


// Persistent split-K decode attention.  Work item = (virtual group, chunk of
// its key list) with at least one key, ordered by virtual group then chunk;
// CTA c owns one contiguous, balanced range of items, so a virtual group's
// chunks fall in one or a few consecutive CTAs (its segments).  The producer
// warp builds the item table, then streams its items' cache rows (contiguous
// runs: sinks, window, ring wrap) and, once per segment, the group's query
// rows into a ring of stages with bulk copies.  The consumer warps take a
// stage: every key row is read by kLPR lanes for all the virtual group's
// heads (a body compiled per head count), and an fp32 online softmax is kept
// per row group and head across the whole segment.  The segment's last stage
// merges the row groups and writes one partial (o, max, sum) per query head;
// the CTA that completes a virtual group's last segment merges its partials
// in segment order and writes the bf16 output.
template <int D, int G>
__global__ void __launch_bounds__(DecWarps<G>::kThreads, 1) ea_decode_attn_kernel(DecodeArgs args) {
  using L = DecLayout<D, G>;
  using W = DecWarps<G>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);
  DecDesc* desc = reinterpret_cast<DecDesc*>(smem + L::off_desc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::off_flag);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::off_flag + 4);
  int* table = reinterpret_cast<int*>(smem + L::off_table);
  const uint32_t full0 = sbase + L::off_full, empty0 = sbase + L::off_empty;
  const int ngroups = args.B * args.Hkv;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full0 + 8 * s) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty0 + 8 * s),
                   "n"(L::kCW) : "memory");
    }
    *abort_flag = 0;
    *last_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp >= L::kCW) {
    regs_dec<W::kRegsProducer>();
    if (warp != L::kCW) return;
    // ---------------- producer: item table (exclusive prefix of chunk counts)
    const int nvg = 2 * ngroups;   // virtual groups: (b, hk, part)
    int carry = 0;
    for (int base = 0; base < nvg; base += 32) {
      const int gi = base + lane;
      int cnt = 0;
      if (gi < nvg) {
        const DecVGroup g = dec_vgroup(args, (gi / 2) / args.Hkv, (gi / 2) % args.Hkv, gi % 2, G);
        cnt = (g.nvis + L::kChunkRows - 1) / L::kChunkRows;
      }
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (gi < nvg) table[gi + 1] = carry + incl;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) table[0] = 0;
    __syncwarp();
    if (lane != 0) return;

    // ---------------- producer: stream the stages
    const int total = table[nvg];
    const int grid = gridDim.x, cta = blockIdx.x;
    const int i0 = dec_range_begin(cta, total, grid), i1 = dec_range_begin(cta + 1, total, grid);
    int u = 0;                 // stage uses issued
    int gi = 0;
    bool ok = true;
    for (int it = i0; it < i1 && ok; ++it) {
      while (table[gi + 1] <= it) ++gi;
      const int b = (gi / 2) / args.Hkv, hk = (gi / 2) % args.Hkv;
      const int chunk = it - table[gi];
      const bool seg_first = it == i0 || chunk == 0;
      const bool seg_last = it == i1 - 1 || it == table[gi + 1] - 1;
      const int cta_first = dec_cta_of(table[gi], total, grid);
      const int seg = cta - cta_first;
      const int nseg = dec_cta_of(table[gi + 1] - 1, total, grid) - cta_first + 1;
      const DecVGroup g = dec_vgroup(args, b, hk, gi % 2, G);
      const __nv_bfloat16* kbase;
      const __nv_bfloat16* vbase;
      if (g.compact) {
        const size_t c = static_cast<size_t>(-g.slot - 1) * (args.sink + args.window);
        kbase = args.k_sa + c * D;
        vbase = args.v_sa + c * D;
      } else {
        const size_t c = static_cast<size_t>(g.slot) * args.max_len;
        kbase = args.k_full + c * D;
        vbase = args.v_full + c * D;
      }
      const int j0 = chunk * L::kChunkRows, j1 = min(g.nvis, j0 + L::kChunkRows);
      for (int js = j0; js < j1; js += L::kStageRows) {
        const int slot = u % L::kStages, round = u / L::kStages;
        if (round > 0 && !mbar_wait(empty0 + 8 * slot, (round - 1) & 1, abort_flag, args.status,
                                    args.timeout_ns, EA_ERR_TIMEOUT)) {
          ok = false;
          break;
        }
        const int n = min(L::kStageRows, j1 - js);
        DecDesc& d = desc[slot];
        d.n = n; d.b = b; d.hk = hk; d.vg = gi;
        d.seg = seg; d.nseg = nseg;
        const bool first = seg_first && js == j0;
        d.first = first; d.last = seg_last && js + L::kStageRows >= j1;
        d.heads = g.heads;
        const uint32_t bar = full0 + 8 * slot;
        mbar_arrive_expect_tx(bar, 2u * n * L::kRowBytes + (first ? L::kQ : 0));
        const uint32_t kdst = sbase + L::off_k + slot * L::kKV;
        const uint32_t vdst = sbase + L::off_v + slot * L::kKV;
        for (int j = js; j < js + n;) {
          int crow, run;
          if (j < g.a) {                       // sink keys: rows 0.. of either cache
            crow = j;
            run = min(js + n, g.a) - j;
          } else {
            const int p = g.lo + (j - g.a);
            if (!g.compact) {
              crow = p;
              run = js + n - j;
            } else if (p < args.sink) {
              crow = p;
              run = min(js + n - j, args.sink - p);
            } else {                           // ring: stop at the wrap
              const int r = (p - args.sink) % args.window;
              crow = args.sink + r;
              run = min(js + n - j, args.window - r);
            }
          }
          const uint32_t off = static_cast<uint32_t>(j - js) * L::kRowBytes;
          bulk_load(kdst + off, kbase + static_cast<size_t>(crow) * D, run * L::kRowBytes, bar);
          bulk_load(vdst + off, vbase + static_cast<size_t>(crow) * D, run * L::kRowBytes, bar);
          j += run;
        }
        if (first)
          bulk_load(sbase + L::off_q + slot * L::kQ,
                    args.q + (static_cast<size_t>(b) * args.Hq + hk * G) * D, L::kQ, bar);
        ++u;
      }
    }
    if (ok) {
      // end of stream
      const int slot = u % L::kStages, round = u / L::kStages;
      if (round == 0 || mbar_wait(empty0 + 8 * slot, (round - 1) & 1, abort_flag, args.status,
                                  args.timeout_ns, EA_ERR_TIMEOUT)) {
        desc[slot].n = -1;
        mbar_arrive(full0 + 8 * slot);
        return;
      }
    }
    // aborted: let the copies in flight land before the CTA exits
    for (int v = max(0, u - L::kStages); v < u; ++v)
      mbar_wait_drain(full0 + 8 * (v % L::kStages), (v / L::kStages) & 1, args.timeout_ns);
    return;
  }

  // ---------------- consumers
  regs_inc<W::kRegsConsumer>();
  constexpr int kP = L::kP;
  const int sub = lane / L::kLPR, cl = lane % L::kLPR;
  const int rg = warp * L::kRGW + sub;
  // state of the segment's heads, packed: slot k holds the k-th head of the
  // virtual group (the k-th set bit of its head mask)
  uint64_t q2[G][kP], o2[G][kP];
  float m[G], l[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = kDecNegBig;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < kP; ++e) { o2[g][e] = 0ull; q2[g][e] = 0ull; }
  }
  int nact = G;
  uint32_t heads = (1u << G) - 1u;
  const uint64_t scale2 = pack2(args.scale_log2, args.scale_log2);
  for (int u = 0;; ++u) {
    const int slot = u % L::kStages, round = u / L::kStages;
    if (!mbar_wait(full0 + 8 * slot, round & 1, abort_flag, args.status, args.timeout_ns,
                   EA_ERR_TIMEOUT))
      break;
    const DecDesc d = desc[slot];
    if (d.n < 0) break;
    if (d.first) {
      heads = d.heads;
      nact = __popc(heads);
      const uint8_t* qs = smem + L::off_q + slot * L::kQ;
#pragma unroll
      for (int k = 0; k < G; ++k) {
#pragma unroll
        for (int e = 0; e < kP; ++e) q2[k][e] = 0ull;   // slots past nact are never read
        if (k < nact) {
          const int g = __fns(heads, 0, k + 1);
#pragma unroll
          for (int i = 0; i < L::kChunks; ++i) {
            const uint4 raw =
                *reinterpret_cast<const uint4*>(qs + (g * D + (cl + i * L::kLPR) * 8) * 2);
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) q2[k][i * 4 + e] = fmul2(bf16x2_to_f32x2(w[e]), scale2);
          }
        }
        m[k] = kDecNegBig;
        l[k] = 0.f;
#pragma unroll
        for (int e = 0; e < kP; ++e) o2[k][e] = 0ull;
      }
    }
    dec_stage_dispatch<L, G, G>(nact, d.n, smem + L::off_k + slot * L::kKV,
                                smem + L::off_v + slot * L::kKV, rg, cl, q2, o2, m, l);
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * slot);

    if (d.last) {
      // merge the row groups of this warp (lanes cl, cl + kLPR, ...); slots
      // past nact hold zeros and merge to zeros
#pragma unroll
      for (int off = L::kLPR; off < 32; off <<= 1) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float mo = __shfl_xor_sync(0xffffffffu, m[g], off);
          const float lo_ = __shfl_xor_sync(0xffffffffu, l[g], off);
          const float mn = fmaxf(m[g], mo);
          const float as = ex2_approx(m[g] - mn), ao = ex2_approx(mo - mn);
          l[g] = l[g] * as + lo_ * ao;
#pragma unroll
          for (int e = 0; e < kP; ++e) {
            float x, y;
            unpack2(o2[g][e], x, y);
            const float ox = __shfl_xor_sync(0xffffffffu, x, off);
            const float oy = __shfl_xor_sync(0xffffffffu, y, off);
            o2[g][e] = pack2(x * as + ox * ao, y * as + oy * ao);
          }
          m[g] = mn;
        }
      }
      float* s_mo = reinterpret_cast<float*>(smem + L::off_mo);
      float* s_ml = reinterpret_cast<float*>(smem + L::off_ml);
      if (sub == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
          for (int i = 0; i < L::kChunks; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float x, y;
              unpack2(o2[g][i * 4 + e], x, y);
              float* dst = s_mo + (warp * G + g) * D + (cl + i * L::kLPR) * 8 + 2 * e;
              dst[0] = x;
              dst[1] = y;
            }
          if (cl == 0) {
            s_ml[(warp * G + g) * 2] = m[g];
            s_ml[(warp * G + g) * 2 + 1] = l[g];
          }
        }
      }
      named_bar_consumers<L::kCW>();
      const int hq0 = d.b * args.Hq + d.hk * G;
      for (int idx = threadIdx.x; idx < nact * (D + 2); idx += L::kCW * 32) {
        const int k = idx / (D + 2), c = idx % (D + 2);
        const int g = __fns(heads, 0, k + 1);
        float mx = kDecNegBig;
#pragma unroll
        for (int w = 0; w < L::kCW; ++w) mx = fmaxf(mx, s_ml[(w * G + k) * 2]);
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < L::kCW; ++w) {
          const float sw = ex2_approx(s_ml[(w * G + k) * 2] - mx);
          const float x = c < D ? s_mo[(w * G + k) * D + c] : s_ml[(w * G + k) * 2 + 1];
          acc += x * sw;
        }
        float* pb = args.part + ((static_cast<size_t>(hq0 + g)) * args.nsplit + d.seg) * (D + 2);
        pb[c] = (c == D) ? mx : acc;
      }
      // publish the partial; the CTA that completes the virtual group merges it
      __threadfence();
      named_bar_consumers<L::kCW>();
      if (threadIdx.x == 0) {
        const int prev = atomicAdd(args.counters + d.vg, 1);
        *last_flag = prev == d.nseg - 1;
        __threadfence();
      }
      named_bar_consumers<L::kCW>();
      if (*last_flag) {
        for (int idx = threadIdx.x; idx < nact * D; idx += L::kCW * 32) {
          const int g = __fns(heads, 0, idx / D + 1), c = idx % D;
          const float* pb = args.part + static_cast<size_t>(hq0 + g) * args.nsplit * (D + 2);
          float mx = kDecNegBig;
          for (int sp = 0; sp < d.nseg; ++sp)
            mx = fmaxf(mx, __ldcg(pb + static_cast<size_t>(sp) * (D + 2) + D));
          float acc = 0.f, sum = 0.f;
          for (int sp = 0; sp < d.nseg; ++sp) {
            const float* ps = pb + static_cast<size_t>(sp) * (D + 2);
            const float w = ex2_approx(__ldcg(ps + D) - mx);
            acc += __ldcg(ps + c) * w;
            sum += __ldcg(ps + D + 1) * w;
          }
          args.out[static_cast<size_t>(hq0 + g) * D + c] =
              __float2bfloat16_rn(sum > 0.f ? acc / sum : 0.f);
        }
      }
      // reset for the next segment (also done when its first stage arrives)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = kDecNegBig;
        l[g] = 0.f;
#pragma unroll
        for (int e = 0; e < kP; ++e) o2[g][e] = 0ull;
      }
    }
  }
}

int decode_num_splits(int max_len) { return (max_len + kDecChunk - 1) / kDecChunk; }

template <int D, int G>
static cudaError_t launch_attn_dec_g(const DecodeArgs& a, cudaStream_t stream) {
  using L = DecLayout<D, G>;
  static int configured[64] = {0};   // per device: the attribute is per context
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev >= 64 || !configured[dev]) {
    err = cudaFuncSetAttribute(ea_decode_attn_kernel<D, G>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               L::bytes(kDecMaxGroups));
    if (err != cudaSuccess) return err;
    if (dev < 64) configured[dev] = 1;
  }
  const int grid = device_sms();
  if (grid <= 0) return cudaErrorInvalidDevice;
  ea_decode_attn_kernel<D, G><<<grid, DecWarps<G>::kThreads, L::bytes(a.B * a.Hkv), stream>>>(a);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_attn_dec(const DecodeArgs& a, int G, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_attn_dec_g<D, 1>(a, stream);
    case 2: return launch_attn_dec_g<D, 2>(a, stream);
    case 4: return launch_attn_dec_g<D, 4>(a, stream);
    case 8: return launch_attn_dec_g<D, 8>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  ea_decode_append_kernel<<<dim3(a.Hkv, a.B), 32, 0, stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int G = a.Hq / a.Hkv;
  return a.d == 128 ? launch_attn_dec<128>(a, G, stream) : launch_attn_dec<64>(a, G, stream);
}

}  // namespace ea

// ------------------------------------------------------------------ C ABI
namespace {
bool dec_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace: status word (256 B), per-group item counters (rounded up to
// 256 B), then the partials.
size_t dec_counter_bytes(const ea_decode_params* p) {
  const size_t n = 2 * static_cast<size_t>(p->B) * p->Hkv * sizeof(int);
  return (n + 255) / 256 * 256;
}

ea_status check_decode(const ea_decode_params* p) {
  if (!p) return EA_ERR_INVALID_ARG;
  if (p->B <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->d <= 0 || p->max_len <= 0)
    return EA_ERR_INVALID_ARG;
  if (p->sink < 0 || p->window < 1 || p->Hq % p->Hkv != 0) return EA_ERR_INVALID_ARG;
  if (!(p->softmax_scale <= 0.f) && !(p->softmax_scale > 0.f)) return EA_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return EA_ERR_UNSUPPORTED;
  const int G = p->Hq / p->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return EA_ERR_UNSUPPORTED;
  if (p->max_len >= (1 << 30)) return EA_ERR_UNSUPPORTED;
  if (p->n_full < 0 || p->n_sa < 0 || p->n_full + p->n_sa <= 0) return EA_ERR_INVALID_ARG;
  if (static_cast<long long>(p->B) * p->Hkv > ea::kDecMaxGroups) return EA_ERR_UNSUPPORTED;
  return EA_OK;
}
}  // namespace

extern "C" {

size_t ea_decode_workspace_size(const ea_decode_params* p) {
  if (check_decode(p) != EA_OK) return 0;
  const size_t ns = ea::decode_num_splits(p->max_len > p->sink + p->window
                                              ? p->max_len : p->sink + p->window);
  return 256 + dec_counter_bytes(p) + static_cast<size_t>(p->B) * p->Hq * ns * (p->d + 2) * sizeof(float);
}

int ea_decode_kv_policy(const uint8_t* mask, int B, int Hq, int Hkv, int32_t* cache_slot,
                        int* n_full, int* n_sa) {
  if (!mask || !cache_slot || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return -1;
  const int G = Hq / Hkv;
  int nf = 0, ns = 0;
  for (int b = 0; b < B; ++b)
    for (int hk = 0; hk < Hkv; ++hk) {
      bool all_sa = true;
      for (int g = 0; g < G; ++g) all_sa = all_sa && mask[b * Hq + hk * G + g] != 0;
      cache_slot[b * Hkv + hk] = all_sa ? -(ns++) - 1 : nf++;
    }
  if (n_full) *n_full = nf;
  if (n_sa) *n_sa = ns;
  return 0;
}

ea_status ea_hybrid_attn_decode(const void* q, const void* k_new, const void* v_new,
                                const int32_t* pos, const uint8_t* route_mask,
                                const int32_t* cache_slot, void* k_full, void* v_full,
                                void* k_sa, void* v_sa, const ea_decode_params* p, void* out,
                                void* workspace, size_t workspace_bytes, void* stream) {
  ea_status st = check_decode(p);
  if (st != EA_OK) return st;
  if (!q || !k_new || !v_new || !pos || !route_mask || !cache_slot || !out)
    return EA_ERR_INVALID_ARG;
  if (p->n_full > 0 && (!k_full || !v_full)) return EA_ERR_INVALID_ARG;
  if (p->n_sa > 0 && (!k_sa || !v_sa)) return EA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k_new, v_new, out};
  for (const void* ptr : ptrs)
    if (!dec_aligned16(ptr)) return EA_ERR_MISALIGNED;
  if ((k_full && !dec_aligned16(k_full)) || (v_full && !dec_aligned16(v_full)) ||
      (k_sa && !dec_aligned16(k_sa)) || (v_sa && !dec_aligned16(v_sa)))
    return EA_ERR_MISALIGNED;
  const size_t need = ea_decode_workspace_size(p);
  if (!workspace || workspace_bytes < need) return EA_ERR_WORKSPACE;
  if (!dec_aligned16(workspace)) return EA_ERR_MISALIGNED;
  ea::DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k_new = static_cast<const __nv_bfloat16*>(k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(v_new);
  a.pos = pos;
  a.mask = route_mask;
  a.cache_slot = cache_slot;
  a.k_full = static_cast<__nv_bfloat16*>(k_full);
  a.v_full = static_cast<__nv_bfloat16*>(v_full);
  a.k_sa = static_cast<__nv_bfloat16*>(k_sa);
  a.v_sa = static_cast<__nv_bfloat16*>(v_sa);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.status = static_cast<int*>(workspace);
  a.counters = reinterpret_cast<int*>(static_cast<char*>(workspace) + 256);
  a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + 256 + dec_counter_bytes(p));
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.d = p->d;
  a.sink = p->sink;
  a.window = p->window;
  a.max_len = p->max_len;
  a.n_full = p->n_full;
  a.n_sa = p->n_sa;
  a.nsplit = ea::decode_num_splits(p->max_len > p->sink + p->window ? p->max_len
                                                                     : p->sink + p->window);
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(static_cast<float>(p->d));
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = ea::wait_timeout_ns();
  cudaError_t err = ea::launch_decode(a, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

}  // extern "C"
