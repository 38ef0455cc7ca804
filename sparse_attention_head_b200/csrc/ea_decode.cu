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
// Step, all on the caller's stream:
//   1. append: the new k, v of every (b, kv head) go to their cache slot;
//   2. attention: CTA (split, kv head, b) reads one chunk of the group's
//      visible keys once for all G query heads (16 lanes per key row, 16-byte
//      loads), keeps an fp32 online softmax per head and writes a partial
//      (max, sum, o) to the workspace;
//   3. combine: the partials of each (b, query head) are merged in split
//      order and written as bf16.
// The step is HBM-bound: its work is one read of every visible cache row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "ea.h"
#include "ea_internal.h"

namespace ea {

constexpr int kDecThreads = 256;         // 8 warps, 16 key rows in flight per step
constexpr int kDecChunk = 512;           // visible keys per CTA (at most)

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
  int* status;
  int B, Hq, Hkv, d, sink, window, max_len, nsplit, n_full, n_sa;
  float scale_log2;
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
  if (!dec_slot_ok(args, slot, t)) {
    if (threadIdx.x == 0) atomicCAS(args.status, 0, EA_ERR_INVALID_ARG);
    return;
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

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads) ea_decode_attn_kernel(DecodeArgs args) {
  constexpr int kLanesPerRow = D / 8;                 // 16 (d=128) or 8 (d=64)
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;     // 2 or 4
  constexpr int kWarps = kDecThreads / 32;
  constexpr int kRowsPerStep = kWarps * kRowsPerWarp;
  constexpr int kGroups = kDecThreads / kLanesPerRow; // independent softmax states
  __shared__ float s_q[G][D];
  __shared__ float s_m[kGroups][G];
  __shared__ float s_l[kGroups][G];
  __shared__ float s_o[G][D];
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int t = args.pos[b];
  const int slot = args.cache_slot[b * args.Hkv + hk];
  const bool compact = slot < 0;
  bool all_sparse = true;
  bool head_sparse[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    head_sparse[g] = args.mask[b * args.Hq + hk * G + g] != 0;
    all_sparse = all_sparse && head_sparse[g];
  }
  if (compact && !all_sparse && threadIdx.x == 0 && split == 0)
    atomicCAS(args.status, 0, EA_ERR_INVALID_ARG);   // an FA head on a compact cache
  int a, lo;
  dec_group_keys(all_sparse || compact, t, args.sink, args.window, &a, &lo);
  const int nvis = dec_slot_ok(args, slot, t) ? a + (t - lo + 1) : 0;
  const int k0 = split * kDecChunk;
  const int k1 = min(nvis, k0 + kDecChunk);

  for (int i = threadIdx.x; i < G * D; i += kDecThreads) {
    const int g = i / D, c = i % D;
    s_q[g][c] = __bfloat162float(
                    args.q[(static_cast<size_t>(b) * args.Hq + hk * G + g) * D + c]) *
                args.scale_log2;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / kLanesPerRow;                // key row within the warp step
  const int cl = lane % kLanesPerRow;                 // 8-channel column block
  const int grp = warp * kRowsPerWarp + sub;          // softmax state index
  const __nv_bfloat16* kbase;
  const __nv_bfloat16* vbase;
  if (nvis == 0) {   // nothing to read; the pointers are never used
    kbase = vbase = nullptr;
  } else if (compact) {
    const size_t c = static_cast<size_t>(-slot - 1) * (args.sink + args.window);
    kbase = args.k_sa + c * D;
    vbase = args.v_sa + c * D;
  } else {
    const size_t c = static_cast<size_t>(slot) * args.max_len;
    kbase = args.k_full + c * D;
    vbase = args.v_full + c * D;
  }
  float qv[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) qv[g][e] = s_q[g][cl * 8 + e];

  float m[G], l[G], o[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[g][e] = 0.f;
  }
  // warp-uniform loop (the shuffles below need every lane); rows past the
  // chunk are loaded as zeros and skipped
  for (int jb = k0 + warp * kRowsPerWarp; jb < k1; jb += kRowsPerStep) {
    const int j = jb + sub;
    const bool valid = j < k1;
    const int p = !valid ? 0 : (j < a ? j : lo + (j - a));     // key position
    const int crow = compact ? dec_compact_slot(p, args.sink, args.window) : p;
    uint4 kraw = make_uint4(0, 0, 0, 0), vraw = make_uint4(0, 0, 0, 0);
    if (valid) {
      kraw = __ldg(reinterpret_cast<const uint4*>(kbase + static_cast<size_t>(crow) * D) + cl);
      vraw = __ldg(reinterpret_cast<const uint4*>(vbase + static_cast<size_t>(crow) * D) + cl);
    }
    const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kraw);
    const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vraw);
    float kf[8], vf[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 kk = __bfloat1622float2(k2[e]);
      const float2 vv = __bfloat1622float2(v2[e]);
      kf[2 * e] = kk.x; kf[2 * e + 1] = kk.y;
      vf[2 * e] = vv.x; vf[2 * e + 1] = vv.y;
    }
    const bool in_sa = p < args.sink || t - p < args.window;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) s = fmaf(qv[g][e], kf[e], s);
#pragma unroll
      for (int off = kLanesPerRow / 2; off > 0; off >>= 1)
        s += __shfl_xor_sync(0xffffffffu, s, off);
      if (!valid || (head_sparse[g] && !in_sa)) continue;   // not a key of this head
      const float mn = fmaxf(m[g], s);
      const float alpha = exp2f(m[g] - mn);
      const float pr = exp2f(s - mn);
      l[g] = l[g] * alpha + pr;
#pragma unroll
      for (int e = 0; e < 8; ++e) o[g][e] = fmaf(o[g][e], alpha, pr * vf[e]);
      m[g] = mn;
    }
  }
  // merge the kGroups softmax states of this CTA, then write the partial
  if (cl == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      s_m[grp][g] = m[g];
      s_l[grp][g] = l[g];
    }
  }
  for (int i = threadIdx.x; i < G * D; i += kDecThreads) (&s_o[0][0])[i] = 0.f;
  __syncthreads();
  float mg[G], sc[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float mm = -INFINITY;
    for (int r = 0; r < kGroups; ++r) mm = fmaxf(mm, s_m[r][g]);
    mg[g] = mm;
    sc[g] = (m[g] == -INFINITY) ? 0.f : exp2f(m[g] - mm);
  }
  // fixed-order merge of the o rows: one group at a time
  for (int r = 0; r < kGroups; ++r) {
    if (grp == r) {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e) s_o[g][cl * 8 + e] += o[g][e] * sc[g];
    }
    __syncthreads();
  }
  float* pb = args.part + ((static_cast<size_t>(b) * args.Hq + hk * G) * args.nsplit + split) *
                              (D + 2);
  for (int i = threadIdx.x; i < G * D; i += kDecThreads) {
    const int g = i / D, c = i % D;
    pb[static_cast<size_t>(g) * args.nsplit * (D + 2) + c] = s_o[g][c];
  }
  if (threadIdx.x < G) {
    const int g = threadIdx.x;
    float ls = 0.f;
    for (int r = 0; r < kGroups; ++r)
      ls += (s_m[r][g] == -INFINITY) ? 0.f : s_l[r][g] * exp2f(s_m[r][g] - mg[g]);
    pb[static_cast<size_t>(g) * args.nsplit * (D + 2) + D] = mg[g];
    pb[static_cast<size_t>(g) * args.nsplit * (D + 2) + D + 1] = ls;
  }
}

__global__ void ea_decode_combine_kernel(DecodeArgs args) {
  const int hq = blockIdx.x, b = blockIdx.y;
  const int D = args.d;
  const float* pb = args.part + (static_cast<size_t>(b) * args.Hq + hq) * args.nsplit * (D + 2);
  float mm = -INFINITY;
  for (int s = 0; s < args.nsplit; ++s) mm = fmaxf(mm, pb[static_cast<size_t>(s) * (D + 2) + D]);
  float ls = 0.f;
  for (int s = 0; s < args.nsplit; ++s) {
    const float ms = pb[static_cast<size_t>(s) * (D + 2) + D];
    if (ms != -INFINITY) ls += pb[static_cast<size_t>(s) * (D + 2) + D + 1] * exp2f(ms - mm);
  }
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < args.nsplit; ++s) {
      const float ms = pb[static_cast<size_t>(s) * (D + 2) + D];
      if (ms != -INFINITY) acc += pb[static_cast<size_t>(s) * (D + 2) + c] * exp2f(ms - mm);
    }
    // no visible key (a rejected slot or position): zero output
    args.out[(static_cast<size_t>(b) * args.Hq + hq) * D + c] =
        __float2bfloat16_rn(ls > 0.f ? acc / ls : 0.f);
  }
}

int decode_num_splits(int max_len) { return (max_len + kDecChunk - 1) / kDecChunk; }

template <int D>
static cudaError_t launch_attn_dec(const DecodeArgs& a, int G, cudaStream_t stream) {
  dim3 grid(a.nsplit, a.Hkv, a.B);
  switch (G) {
    case 1: ea_decode_attn_kernel<D, 1><<<grid, kDecThreads, 0, stream>>>(a); break;
    case 2: ea_decode_attn_kernel<D, 2><<<grid, kDecThreads, 0, stream>>>(a); break;
    case 4: ea_decode_attn_kernel<D, 4><<<grid, kDecThreads, 0, stream>>>(a); break;
    case 8: ea_decode_attn_kernel<D, 8><<<grid, kDecThreads, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  ea_decode_append_kernel<<<dim3(a.Hkv, a.B), 32, 0, stream>>>(a);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int G = a.Hq / a.Hkv;
  err = a.d == 128 ? launch_attn_dec<128>(a, G, stream) : launch_attn_dec<64>(a, G, stream);
  if (err != cudaSuccess) return err;
  ea_decode_combine_kernel<<<dim3(a.Hq, a.B), 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ea

// ------------------------------------------------------------------ C ABI
namespace {
bool dec_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
  return EA_OK;
}
}  // namespace

extern "C" {

size_t ea_decode_workspace_size(const ea_decode_params* p) {
  if (check_decode(p) != EA_OK) return 0;
  const size_t ns = ea::decode_num_splits(p->max_len > p->sink + p->window
                                              ? p->max_len : p->sink + p->window);
  return 256 + static_cast<size_t>(p->B) * p->Hq * ns * (p->d + 2) * sizeof(float);
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
  a.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + 256);
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
  cudaError_t err = ea::launch_decode(a, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

}  // extern "C"
