// ea_router_dev.cuh — device bodies of the Attention Router shared by the
// standalone router kernels and the attention kernel's routed prologue, so
// both compute the same bits.
//
// Elastic Attention blog §2.1 "Attention Router": the layer's Key hidden
// states go through a simple MLP that emits one routing signal per head.
// Pooled input x[b] = mean of sequence b's key rows (flattened kv head,
// channel); h = ReLU(W1 x + b1); z = W2 h + b2; route r = z > threshold.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace ea {

constexpr int kPoolThreads = 256;   // threads that pool one item

// Rows of (b, kv head): padded K [B][Hkv][N][d] (cu == nullptr) or packed K
// [T][Hkv][d] with sequence b at tokens [cu[b], cu[b + 1]).  A packed range
// outside [0, T] (inconsistent offsets) pools nothing.
__device__ __forceinline__ int router_seq_rows(const int32_t* cu, int N, int total, int b,
                                               int* t0) {
  if (!cu) {
    *t0 = 0;
    return N;
  }
  const int a = cu[b], e = cu[b + 1];
  *t0 = a;
  return (a >= 0 && e >= a && e <= total) ? e - a : 0;
}

// Barrier among the kPoolThreads threads 0..255 (named barrier `id`).
__device__ __forceinline__ void pool_bar(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kPoolThreads) : "memory");
}

// One pooling item (split, hk, b) by threads 0..255: the fp32 sum of the
// item's chunk of rows, 8 channels per thread with 16-byte loads, row groups
// reduced in a fixed order into partials[b][hk][split][D].  red: shared
// [kPoolThreads / (D / 8)][D] floats.
template <int D>
__device__ __forceinline__ void router_pool_item(const __nv_bfloat16* __restrict__ k,
                                                 const int32_t* __restrict__ cu, int N, int total,
                                                 int Hkv, int b, int hk, int split, int nsplit,
                                                 float* __restrict__ partials, float* red,
                                                 int tid, int bar_id) {
  constexpr int TPR = D / 8;                 // threads per row (8 channels each)
  constexpr int RPI = kPoolThreads / TPR;    // rows per iteration
  const int cg = tid % TPR;
  const int rs = tid / TPR;
  int t0;
  const int len = router_seq_rows(cu, N, total, b, &t0);
  const int chunk = (len + nsplit - 1) / nsplit;
  const int n0 = split * chunk;
  const int n1 = min(len, n0 + chunk);
  // padded: plane (b, hk) of N rows of D; packed: token rows of Hkv * D
  const size_t row_stride = cu ? static_cast<size_t>(Hkv) * D : static_cast<size_t>(D);
  const __nv_bfloat16* base =
      (cu ? k + (static_cast<size_t>(t0) * Hkv + hk) * D
          : k + (static_cast<size_t>(b) * Hkv + hk) * N * D) + cg * 8;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  int n = n0 + rs;
#pragma unroll 4
  for (; n < n1; n += RPI) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(n) * row_stride));
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(p[j]);
      acc[2 * j] += f.x;
      acc[2 * j + 1] += f.y;
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[rs * D + cg * 8 + j] = acc[j];
  pool_bar(bar_id);
  for (int c = tid; c < D; c += kPoolThreads) {
    float s = 0.f;
    for (int r = 0; r < RPI; ++r) s += red[r * D + c];
    partials[((static_cast<size_t>(b) * Hkv + hk) * nsplit + split) * D + c] = s;
  }
  pool_bar(bar_id);   // red is reused by the next item
}

// x[b][j], j = hk * d + c: the partials summed in split order, divided by the
// sequence's row count (zero for an empty sequence).  partials and x may have
// been written earlier in the same launch, so they are read through the
// coherent path (no __restrict__, no read-only cache).
__device__ __forceinline__ float router_x(const float* partials,
                                          const int32_t* __restrict__ cu, int Hkv, int N,
                                          int total, int d, int nsplit, int b, int j) {
  const int hk = j / d, c = j % d;
  int t0;
  const int len = router_seq_rows(cu, N, total, b, &t0);
  const float* p = partials + (static_cast<size_t>(b) * Hkv + hk) * nsplit * d + c;
  // the partials are added in split order; the loads of 16 splits are issued
  // before their adds, so their L2 latencies overlap instead of queueing
  float s = 0.f;
  int sp = 0;
  for (; sp + 16 <= nsplit; sp += 16) {
    float v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = __ldcg(p + static_cast<size_t>(sp + u) * d);
#pragma unroll
    for (int u = 0; u < 16; ++u) s += v[u];
  }
  for (; sp < nsplit; ++sp) s += __ldcg(p + static_cast<size_t>(sp) * d);
  return len > 0 ? s * (1.0f / static_cast<float>(len)) : 0.f;
}

// One warp computes y = act(W[o] . x[b] + bias[o]): float4 over the input
// (lane j, j + 32, ...), lanes reduced by xor shuffles in a fixed order.
// Returns the pre-activation value on every lane.
__device__ __forceinline__ float router_warp_dot(const float* x, int in_dim,
                                                 const float* __restrict__ w,
                                                 const float* __restrict__ bias, int o,
                                                 int lane) {
  const float4* wr = reinterpret_cast<const float4*>(w + static_cast<size_t>(o) * in_dim);
  const float4* xr = reinterpret_cast<const float4*>(x);
  float acc = 0.f;
#pragma unroll 4
  for (int j = lane; j < in_dim / 4; j += 32) {
    const float4 wv = __ldg(wr + j);
    const float4 xv = __ldcg(xr + j);
    acc = fmaf(wv.x, xv.x, acc);
    acc = fmaf(wv.y, xv.y, acc);
    acc = fmaf(wv.z, xv.z, acc);
    acc = fmaf(wv.w, xv.w, acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  return acc + bias[o];
}

}  // namespace ea
