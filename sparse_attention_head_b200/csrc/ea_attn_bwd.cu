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
// Three launches on the caller's stream:
//   1. ea_bwd_rowdot_kernel: D = rowsum(dO * O), fp32 (HBM-bound);
//   2. ea_bwd_dkdv_kernel: unit = (b, kv head, 128-key tile j).  K_j and V_j
//      stay in shared memory; the steps visit (query head of the group,
//      128-query tile i) pairs that see tile j.  Per step the tensor cores
//      compute S^T = K_j Q_i^T and dP^T = V_j dO_i^T into TMEM, four warps
//      turn them into P^T and dS^T (bf16, back into TMEM), and
//      dV += P^T dO_i, dK += dS^T Q_i accumulate in TMEM (A from TMEM).
//   3. ea_bwd_dq_kernel: unit = (b, head, 128-query tile i); the steps visit
//      the key tiles the forward visits: S = Q_i K_j^T, dP = dO_i V_j^T, dS,
//      dQ += dS K_j.
// Both are persistent (one CTA per SM), with a TMA producer warp, one MMA
// issuing thread and four elementwise warps; every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ea.h"
#include "ea_internal.h"
#include "ea_ptx.cuh"
#include "ea_sched.h"
#include "ea_tmem.cuh"

namespace ea {

// D[row] = sum_c dO[row][c] * O[row][c] over rows of [rows][d]; one warp per
// row, fixed shuffle order.
__global__ void ea_bwd_rowdot_kernel(const __nv_bfloat16* __restrict__ dout,
                                     const __nv_bfloat16* __restrict__ out, int rows, int d,
                                     float* __restrict__ dvec) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const __nv_bfloat16* a = dout + static_cast<size_t>(warp) * d;
  const __nv_bfloat16* b = out + static_cast<size_t>(warp) * d;
  float s = 0.f;
  for (int c = lane * 2; c < d; c += 64) {
    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(a + c));
    const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(b + c));
    s = fmaf(x.x, y.x, s);
    s = fmaf(x.y, y.y, s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) dvec[warp] = s;
}

// Shared-memory plan of both backward kernels (d = 128): two resident tiles
// (the unit's own operands) and a ring of two stages of two streamed tiles.
struct BwdCfg {
  static constexpr int D = 128;
  static constexpr int kThreads = 192;           // warps 0-3 elementwise, 4 producer, 5 MMA
  static constexpr int kBlockBytes = 128 * 128;  // 128 rows x 64 bf16 (one SW128 column block)
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr int kStages = 2;
  static constexpr int kOffRes = 0;                          // 2 resident tiles
  static constexpr int kOffStage = 2 * kTileBytes;           // kStages x 2 streamed tiles
  // per stage: lse * log2e and D of the step's 128 query rows (f32)
  static constexpr int kOffVec = kOffStage + kStages * 2 * kTileBytes;
  static constexpr int kOffStep = kOffVec + kStages * 2 * 128 * 4;   // step descriptors, 32 B each
  static constexpr int kOffBar = kOffStep + kStages * 32;
  // res_full, res_empty, st_full[2], st_empty[2], s_full, p_full, acc_done, acc_empty, drain,
  // vec_full[2] (the elementwise threads' lse / D rows of a stage)
  static constexpr int kNumBars = 2 + 3 * kStages + 5;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;    // tmem base, abort flag
  static constexpr int kSmem = kOffMisc + 64 + 1024;         // + alignment slack
  static constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 128, 0, 0);  // both K-major
  static constexpr uint32_t kIdescTS = idesc_bf16_f32(128, D, 0, 1);    // B MN-major
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
  int pad;
};



// ---------------------------------------------------------------- dK, dV
template <bool kDkDv>
__device__ __forceinline__ void bwd_unit_of(const BwdArgs& a, int u, int* b, int* hx, int* tile) {
  const int nT = ea_cdiv(a.N, EA_BN);
  if (kDkDv) {   // (b, kv head, key tile): key tile 0 (the most queries) first
    const int per = a.B * a.Hkv;
    *tile = u / per;
    *b = (u % per) / a.Hkv;
    *hx = (u % per) % a.Hkv;
  } else {       // (b, head, query tile): the last query tile (the most keys) first
    const int per = a.B * a.Hq;
    *tile = nT - 1 - u / per;
    *b = (u % per) / a.Hq;
    *hx = (u % per) % a.Hq;
  }
}

__global__ void __launch_bounds__(BwdCfg::kThreads, 1) ea_bwd_dkdv_kernel(
    const __grid_constant__ BwdArgs args) {
  using C = BwdCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  const uint32_t bar0 = smem_u32(bar);
  const uint32_t b_res_full = bar0, b_res_empty = bar0 + 8;
  const uint32_t b_st_full = bar0 + 16, b_st_empty = bar0 + 16 + 8 * C::kStages;
  const uint32_t b_s_full = bar0 + 16 + 16 * C::kStages, b_p_full = b_s_full + 8;
  const uint32_t b_acc_done = b_s_full + 16, b_acc_empty = b_s_full + 24;
  const uint32_t b_drain = b_s_full + 32;
  const uint32_t b_vec = b_s_full + 40;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  BwdStep* steps = reinterpret_cast<BwdStep*>(smem + C::kOffStep);
  float* vec = reinterpret_cast<float*>(smem + C::kOffVec);
  const int G = args.Hq / args.Hkv;
  const int nT = ea_cdiv(args.N, EA_BN);
  const int units = args.B * args.Hkv * nT;
  const uint64_t tlim = args.timeout_ns;
  int* status = args.status;

  if (threadIdx.x == 0) {
    mbar_init(bar + 0, 1);     // res_full: producer
    mbar_init(bar + 1, 1);     // res_empty: MMA commit
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(bar + 2 + i, 1);                 // st_full: producer
      mbar_init(bar + 2 + C::kStages + i, 1);    // st_empty: MMA commit
    }
    mbar_init(bar + 2 + 2 * C::kStages, 1);      // s_full: MMA commit
    mbar_init(bar + 3 + 2 * C::kStages, 128);    // p_full: elementwise threads
    mbar_init(bar + 4 + 2 * C::kStages, 1);      // acc_done: MMA commit
    mbar_init(bar + 5 + 2 * C::kStages, 128);    // acc_empty: elementwise threads
    mbar_init(bar + 6 + 2 * C::kStages, 1);      // drain: MMA commit
    for (int i = 0; i < C::kStages; ++i)
      mbar_init(bar + 7 + 2 * C::kStages + i, 128);   // vec_full: elementwise threads
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 4) {
    // ============================================================ producer
    if (lane == 0) {
      uint32_t pos = 0, nu = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int b, hk, jt;
        bwd_unit_of<true>(args, u, &b, &hk, &jt);
        if (nu > 0 && !(ok = mbar_wait(b_res_empty, (nu - 1) & 1, s_abort, status, tlim,
                                       EA_ERR_TIMEOUT)))
          break;
        mbar_arrive_expect_tx(b_res_full, 2 * C::kTileBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(smem_u32(smem + C::kOffRes) + c * C::kBlockBytes, &args.tm_k, b_res_full,
                      c * 64, jt * EA_BN, b * args.Hkv + hk);
          tma_load_3d(smem_u32(smem + C::kOffRes + C::kTileBytes) + c * C::kBlockBytes,
                      &args.tm_v, b_res_full, c * 64, jt * EA_BN, b * args.Hkv + hk);
        }
        ++nu;
        // steps: query heads of the group, then the query tiles that see jt
        int last_g = -1, last_it = 0;
        for (int g = 0; g < G; ++g) {
          const bool sa = args.mask[b * args.Hq + hk * G + g] != 0;
          last_g = g;
          last_it = bwd_last_query_tile(jt, sa, nT, args.sink, args.window);
        }
        for (int g = 0; g < G && ok; ++g) {
          const int h = hk * G + g;
          const bool sa = args.mask[b * args.Hq + h] != 0;
          const int it_last = bwd_last_query_tile(jt, sa, nT, args.sink, args.window);
          for (int it = jt; it <= it_last; ++it) {
            const uint32_t slot = pos % C::kStages;
            if (pos >= C::kStages &&
                !(ok = mbar_wait(b_st_empty + 8 * slot, ((pos / C::kStages) - 1) & 1, s_abort,
                                 status, tlim, EA_ERR_TIMEOUT)))
              break;
            BwdStep& st = steps[slot];
            st.b = b; st.h = h; st.it = it; st.jt = jt; st.sa = sa;
            st.first = (g == 0 && it == jt);
            st.last = (g == last_g && it == last_it);
            mbar_arrive_expect_tx(b_st_full + 8 * slot, 2 * C::kTileBytes);
            const uint32_t dst = smem_u32(smem + C::kOffStage) + slot * 2 * C::kTileBytes;
            for (int c = 0; c < D / 64; ++c) {
              tma_load_3d(dst + c * C::kBlockBytes, &args.tm_q, b_st_full + 8 * slot, c * 64,
                          it * EA_BM, b * args.Hq + h);
              tma_load_3d(dst + C::kTileBytes + c * C::kBlockBytes, &args.tm_do,
                          b_st_full + 8 * slot, c * 64, it * EA_BM, b * args.Hq + h);
            }
            ++pos;
          }
        }
      }
      // every copy issued must land before the CTA exits
      const uint32_t n = pos < C::kStages ? pos : C::kStages;
      for (uint32_t p = pos - n; p < pos; ++p)
        mbar_wait_drain(b_st_full + 8 * (p % C::kStages), (p / C::kStages) & 1, 200000000ull);
      if (nu > 0) mbar_wait_drain(b_res_full, (nu - 1) & 1, 200000000ull);
    }
  } else if (warp == 5) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      const uint32_t res = smem_u32(smem + C::kOffRes);
      const uint32_t stg = smem_u32(smem + C::kOffStage);
      // K-major (S^T, dP^T operands) and MN-major (dV, dK B operands) views
      const uint64_t d_res_k = smem_desc_sw128(res, 16, 1024);
      const uint64_t d_stg_k = smem_desc_sw128(stg, 16, 1024);
      const uint64_t d_stg_mn = smem_desc_sw128(stg, C::kBlockBytes, 1024);
      uint32_t pos = 0, nu = 0, nsteps = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        if (!(ok = mbar_wait(b_res_full, nu & 1, s_abort, status, tlim, EA_ERR_TIMEOUT))) break;
        if (nu > 0 && !(ok = mbar_wait(b_acc_empty, (nu - 1) & 1, s_abort, status, tlim,
                                       EA_ERR_TIMEOUT)))
          break;
        tc_fence_after();
        ++nu;
        bool last = false;
        bool first = true;
        while (!last && ok) {
          const uint32_t slot = pos % C::kStages;
          if (!(ok = mbar_wait(b_st_full + 8 * slot, (pos / C::kStages) & 1, s_abort, status,
                               tlim, EA_ERR_TIMEOUT)))
            break;
          last = steps[slot].last != 0;
          const uint64_t q_k = d_stg_k + ((slot * 2 * C::kTileBytes) >> 4);
          const uint64_t do_k = q_k + (C::kTileBytes >> 4);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {   // S^T = K Q^T, dP^T = V dO^T
            const uint32_t off = ((k >> 2) * C::kBlockBytes + (k & 3) * 32) >> 4;
            mma_ss(tmem, d_res_k + off, q_k + off, C::kIdescSS, k > 0 ? 1u : 0u);
            mma_ss(tmem + 128, d_res_k + (C::kTileBytes >> 4) + off, do_k + off, C::kIdescSS,
                   k > 0 ? 1u : 0u);
          }
          mma_commit(b_s_full);
          if (!(ok = mbar_wait(b_p_full, nsteps & 1, s_abort, status, tlim, EA_ERR_TIMEOUT)))
            break;
          ++nsteps;
          tc_fence_after();
          const uint64_t q_mn = d_stg_mn + ((slot * 2 * C::kTileBytes) >> 4);
          const uint64_t do_mn = q_mn + (C::kTileBytes >> 4);
#pragma unroll
          for (int k = 0; k < EA_BM / 16; ++k) {   // dV += P^T dO, dK += dS^T Q
            const uint32_t acc = (!first || k > 0) ? 1u : 0u;
            mma_ts(tmem + 256, tmem + k * 8, do_mn + ((k * 2048) >> 4), C::kIdescTS, acc);
            mma_ts(tmem + 384, tmem + 128 + k * 8, q_mn + ((k * 2048) >> 4), C::kIdescTS, acc);
          }
          first = false;
          mma_commit(b_st_empty + 8 * slot);
          ++pos;
        }
        if (!ok) break;
        mma_commit(b_acc_done);
        mma_commit(b_res_empty);
      }
      // drain: wait for every MMA this thread issued
      mma_commit(b_drain);
      mbar_wait_drain(b_drain, 0, 200000000ull);
    }
  } else {
    // ============================================================ elementwise
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int t = warp * 32 + lane;                 // key row within the tile
    uint32_t pos = 0, nsteps = 0, nu = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int b, hk, jt;
      bwd_unit_of<true>(args, u, &b, &hk, &jt);
      const int key = jt * EA_BN + t;
      bool last = false;
      while (!last) {
        const uint32_t slot = pos % C::kStages;
        ok = mbar_wait(b_st_full + 8 * slot, (pos / C::kStages) & 1, s_abort, status, tlim,
                       EA_ERR_TIMEOUT);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const BwdStep st = steps[slot];
        last = st.last != 0;
        const uint32_t use = pos / C::kStages;
        ++pos;
        // this step's lse * log2e and D of the 128 query rows (one per
        // thread), shared through the stage's vec_full barrier (bounded)
        float* vl = vec + slot * 256;
        float* vd = vl + 128;
        {
          const int q = st.it * EA_BM + t;
          const size_t r = (static_cast<size_t>(st.b) * args.Hq + st.h) * args.N + q;
          vl[t] = q < args.N ? args.lse[r] * 1.4426950408889634f : 0.f;
          vd[t] = q < args.N ? args.dvec[r] : 0.f;
        }
        mbar_arrive(b_vec + 8 * slot);
        ok = mbar_wait(b_vec + 8 * slot, use & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ok = mbar_wait(b_s_full, nsteps & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++nsteps;
        tc_fence_after();
        const bool sa = st.sa != 0;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t sr[64], dr[64];
          tmem_ld64_wait(tmem + lane_off + half * 64, sr);
          tmem_ld64_wait(tmem + lane_off + 128 + half * 64, dr);
          uint32_t pp[32], ds[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float p2[2], d2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = half * 64 + 2 * j + e;
              const int q = st.it * EA_BM + c;
              const bool vis = key < args.N &&
                               bwd_visible(q, key, args.N, sa, args.sink, args.window);
              const float p = vis ? ex2_approx(__uint_as_float(sr[2 * j + e]) * args.scale_log2 -
                                               vl[c])
                                  : 0.f;
              p2[e] = p;
              d2[e] = p * (__uint_as_float(dr[2 * j + e]) - vd[c]);
            }
            pp[j] = pack_bf16x2(p2[0], p2[1]);
            ds[j] = pack_bf16x2(d2[0], d2[1]);
          }
          tmem_st32(tmem + lane_off + half * 32, pp);
          tmem_st32(tmem + lane_off + 128 + half * 32, ds);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(b_p_full);
      }
      if (!ok) break;
      // epilogue: dV and scale * dK rows of this key tile
      ok = mbar_wait(b_acc_done, nu & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++nu;
      tc_fence_after();
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* dst = (which ? args.dk : args.dv) +
                             ((static_cast<size_t>(b) * args.Hkv + hk) * args.N + key) * D;
        const float mul = which ? args.scale : 1.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[64];
          tmem_ld64_wait(tmem + lane_off + 256 + which * 128 + half * 64, r);
          if (key < args.N) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + half * 64);
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
      }
      tc_fence_before();
      mbar_arrive(b_acc_empty);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dQ
__global__ void __launch_bounds__(BwdCfg::kThreads, 1) ea_bwd_dq_kernel(
    const __grid_constant__ BwdArgs args) {
  using C = BwdCfg;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  const uint32_t bar0 = smem_u32(bar);
  const uint32_t b_res_full = bar0, b_res_empty = bar0 + 8;
  const uint32_t b_st_full = bar0 + 16, b_st_empty = bar0 + 16 + 8 * C::kStages;
  const uint32_t b_s_full = bar0 + 16 + 16 * C::kStages, b_p_full = b_s_full + 8;
  const uint32_t b_acc_done = b_s_full + 16, b_acc_empty = b_s_full + 24;
  const uint32_t b_drain = b_s_full + 32;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  BwdStep* steps = reinterpret_cast<BwdStep*>(smem + C::kOffStep);
  const int G = args.Hq / args.Hkv;
  const int nT = ea_cdiv(args.N, EA_BN);
  const int units = args.B * args.Hq * nT;
  const uint64_t tlim = args.timeout_ns;
  int* status = args.status;

  if (threadIdx.x == 0) {
    mbar_init(bar + 0, 1);
    mbar_init(bar + 1, 1);
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(bar + 2 + i, 1);
      mbar_init(bar + 2 + C::kStages + i, 1);
    }
    mbar_init(bar + 2 + 2 * C::kStages, 1);      // s_full
    mbar_init(bar + 3 + 2 * C::kStages, 128);    // p_full
    mbar_init(bar + 4 + 2 * C::kStages, 1);      // acc_done
    mbar_init(bar + 5 + 2 * C::kStages, 128);    // acc_empty
    mbar_init(bar + 6 + 2 * C::kStages, 1);      // drain
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 4) {
    // ============================================================ producer
    if (lane == 0) {
      uint32_t pos = 0, nu = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int b, h, it;
        bwd_unit_of<false>(args, u, &b, &h, &it);
        const bool sa = args.mask[b * args.Hq + h] != 0;
        int a, lo;
        bwd_key_tiles(it, sa, args.sink, args.window, &a, &lo);
        const int n = a + (it - lo + 1);
        if (nu > 0 && !(ok = mbar_wait(b_res_empty, (nu - 1) & 1, s_abort, status, tlim,
                                       EA_ERR_TIMEOUT)))
          break;
        mbar_arrive_expect_tx(b_res_full, 2 * C::kTileBytes);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(smem_u32(smem + C::kOffRes) + c * C::kBlockBytes, &args.tm_q, b_res_full,
                      c * 64, it * EA_BM, b * args.Hq + h);
          tma_load_3d(smem_u32(smem + C::kOffRes + C::kTileBytes) + c * C::kBlockBytes,
                      &args.tm_do, b_res_full, c * 64, it * EA_BM, b * args.Hq + h);
        }
        ++nu;
        for (int i = 0; i < n && ok; ++i) {
          const int jt = i < a ? i : lo + (i - a);
          const uint32_t slot = pos % C::kStages;
          if (pos >= C::kStages &&
              !(ok = mbar_wait(b_st_empty + 8 * slot, ((pos / C::kStages) - 1) & 1, s_abort,
                               status, tlim, EA_ERR_TIMEOUT)))
            break;
          BwdStep& st = steps[slot];
          st.b = b; st.h = h; st.it = it; st.jt = jt; st.sa = sa;
          st.first = i == 0;
          st.last = i == n - 1;
          mbar_arrive_expect_tx(b_st_full + 8 * slot, 2 * C::kTileBytes);
          const uint32_t dst = smem_u32(smem + C::kOffStage) + slot * 2 * C::kTileBytes;
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(dst + c * C::kBlockBytes, &args.tm_k, b_st_full + 8 * slot, c * 64,
                        jt * EA_BN, b * args.Hkv + h / G);
            tma_load_3d(dst + C::kTileBytes + c * C::kBlockBytes, &args.tm_v,
                        b_st_full + 8 * slot, c * 64, jt * EA_BN, b * args.Hkv + h / G);
          }
          ++pos;
        }
      }
      const uint32_t n = pos < C::kStages ? pos : C::kStages;
      for (uint32_t p = pos - n; p < pos; ++p)
        mbar_wait_drain(b_st_full + 8 * (p % C::kStages), (p / C::kStages) & 1, 200000000ull);
      if (nu > 0) mbar_wait_drain(b_res_full, (nu - 1) & 1, 200000000ull);
    }
  } else if (warp == 5) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      const uint32_t res = smem_u32(smem + C::kOffRes);
      const uint32_t stg = smem_u32(smem + C::kOffStage);
      const uint64_t d_res_k = smem_desc_sw128(res, 16, 1024);
      const uint64_t d_stg_k = smem_desc_sw128(stg, 16, 1024);
      const uint64_t d_stg_mn = smem_desc_sw128(stg, C::kBlockBytes, 1024);
      uint32_t pos = 0, nu = 0, nsteps = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        if (!(ok = mbar_wait(b_res_full, nu & 1, s_abort, status, tlim, EA_ERR_TIMEOUT))) break;
        if (nu > 0 && !(ok = mbar_wait(b_acc_empty, (nu - 1) & 1, s_abort, status, tlim,
                                       EA_ERR_TIMEOUT)))
          break;
        tc_fence_after();
        ++nu;
        bool last = false, first = true;
        while (!last && ok) {
          const uint32_t slot = pos % C::kStages;
          if (!(ok = mbar_wait(b_st_full + 8 * slot, (pos / C::kStages) & 1, s_abort, status,
                               tlim, EA_ERR_TIMEOUT)))
            break;
          last = steps[slot].last != 0;
          const uint64_t k_k = d_stg_k + ((slot * 2 * C::kTileBytes) >> 4);
          const uint64_t v_k = k_k + (C::kTileBytes >> 4);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {   // S = Q K^T, dP = dO V^T
            const uint32_t off = ((k >> 2) * C::kBlockBytes + (k & 3) * 32) >> 4;
            mma_ss(tmem, d_res_k + off, k_k + off, C::kIdescSS, k > 0 ? 1u : 0u);
            mma_ss(tmem + 128, d_res_k + (C::kTileBytes >> 4) + off, v_k + off, C::kIdescSS,
                   k > 0 ? 1u : 0u);
          }
          mma_commit(b_s_full);
          if (!(ok = mbar_wait(b_p_full, nsteps & 1, s_abort, status, tlim, EA_ERR_TIMEOUT)))
            break;
          ++nsteps;
          tc_fence_after();
          const uint64_t k_mn = d_stg_mn + ((slot * 2 * C::kTileBytes) >> 4);
#pragma unroll
          for (int k = 0; k < EA_BN / 16; ++k)   // dQ += dS K
            mma_ts(tmem + 256, tmem + 128 + k * 8, k_mn + ((k * 2048) >> 4), C::kIdescTS,
                   (!first || k > 0) ? 1u : 0u);
          first = false;
          mma_commit(b_st_empty + 8 * slot);
          ++pos;
        }
        if (!ok) break;
        mma_commit(b_acc_done);
        mma_commit(b_res_empty);
      }
      mma_commit(b_drain);
      mbar_wait_drain(b_drain, 0, 200000000ull);
    }
  } else {
    // ============================================================ elementwise
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int t = warp * 32 + lane;                 // query row within the tile
    uint32_t pos = 0, nsteps = 0, nu = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int b, h, it;
      bwd_unit_of<false>(args, u, &b, &h, &it);
      const int q = it * EA_BM + t;
      const size_t r = (static_cast<size_t>(b) * args.Hq + h) * args.N + q;
      const float lse2 = q < args.N ? args.lse[r] * 1.4426950408889634f : 0.f;
      const float dq_d = q < args.N ? args.dvec[r] : 0.f;
      bool last = false;
      while (!last) {
        const uint32_t slot = pos % C::kStages;
        ok = mbar_wait(b_st_full + 8 * slot, (pos / C::kStages) & 1, s_abort, status, tlim,
                       EA_ERR_TIMEOUT);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const BwdStep st = steps[slot];
        last = st.last != 0;
        ++pos;
        ok = mbar_wait(b_s_full, nsteps & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++nsteps;
        tc_fence_after();
        const bool sa = st.sa != 0;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t sr[64], dr[64];
          tmem_ld64_wait(tmem + lane_off + half * 64, sr);
          tmem_ld64_wait(tmem + lane_off + 128 + half * 64, dr);
          uint32_t ds[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float d2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int key = st.jt * EA_BN + half * 64 + 2 * j + e;
              const bool vis = bwd_visible(q, key, args.N, sa, args.sink, args.window);
              const float p = vis ? ex2_approx(__uint_as_float(sr[2 * j + e]) * args.scale_log2 -
                                               lse2)
                                  : 0.f;
              d2[e] = p * (__uint_as_float(dr[2 * j + e]) - dq_d);
            }
            ds[j] = pack_bf16x2(d2[0], d2[1]);
          }
          tmem_st32(tmem + lane_off + 128 + half * 32, ds);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(b_p_full);
      }
      if (!ok) break;
      ok = mbar_wait(b_acc_done, nu & 1, s_abort, status, tlim, EA_ERR_TIMEOUT);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ++nu;
      tc_fence_after();
      __nv_bfloat16* dst = args.dq + r * D;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t rr[64];
        tmem_ld64_wait(tmem + lane_off + 256 + half * 64, rr);
        if (q < args.N) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + half * 64);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              w[j] = pack_bf16x2(__uint_as_float(rr[8 * q4 + 2 * j]) * args.scale,
                                 __uint_as_float(rr[8 * q4 + 2 * j + 1]) * args.scale);
            d4[q4] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(b_acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

static int g_bwd_configured[64] = {0};

cudaError_t launch_backward(const BwdArgs& a, const void* dout, const void* out, float* dvec,
                            int grid_sms, cudaStream_t stream) {
  const int rows = a.B * a.Hq * a.N;
  ea_bwd_rowdot_kernel<<<(rows + 7) / 8, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(out), rows,
      BwdCfg::D, dvec);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  int dev = 0;
  if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
  if (dev >= 64 || !g_bwd_configured[dev]) {
    if ((err = cudaFuncSetAttribute(ea_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    BwdCfg::kSmem)) != cudaSuccess)
      return err;
    if ((err = cudaFuncSetAttribute(ea_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    BwdCfg::kSmem)) != cudaSuccess)
      return err;
    if (dev < 64) g_bwd_configured[dev] = 1;
  }
  const int nT = ea_cdiv(a.N, EA_BN);
  const int units_kv = a.B * a.Hkv * nT, units_q = a.B * a.Hq * nT;
  ea_bwd_dkdv_kernel<<<units_kv < grid_sms ? units_kv : grid_sms, BwdCfg::kThreads, BwdCfg::kSmem,
                       stream>>>(a);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  ea_bwd_dq_kernel<<<units_q < grid_sms ? units_q : grid_sms, BwdCfg::kThreads, BwdCfg::kSmem,
                     stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ea
