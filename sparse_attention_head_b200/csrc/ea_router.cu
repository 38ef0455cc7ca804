// ea_router.cu — Attention Router: mean-pool the key states, a two-layer MLP,
// and the hard routing decision per head.
//
// Elastic Attention blog (bxzpzcl.cn) §2.1 "Attention Router": the router
// takes the layer's Key hidden states; a simple MLP produces a routing signal
// r for every head; r = 0 selects Full Attention and r = 1 Sparse Attention.
// §2.2 sizes it at 0.27M parameters per layer for an 8B model, which is
// 1024 -> 256 -> 32 with biases.  Training draws Gumbel noise with a
// straight-through estimator (§2.1); at inference the decision is the hard
// threshold below.
//
// Kernel 1 (HBM-bound): CTA (split, kv head, batch) sums its chunk of rows
//   into fp32, 8 channels per thread with 16-byte loads, and reduces the
//   row groups in a fixed order into partials[b][hk][split][d].
// Kernel 2: one CTA per batch row sums the partials in split order, divides
//   by N, runs h = ReLU(W1 x + b1) and z = W2 h + b2 with one warp per output
//   (fixed shuffle order), writes z and the mask z > threshold.
// Both kernels are deterministic: the same inputs give the same bits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "ea.h"
#include "ea_internal.h"

namespace ea {

constexpr int kPoolThreads = 256;
constexpr int kMlpThreads = 256;

template <int D>
__global__ void __launch_bounds__(kPoolThreads) ea_router_pool_kernel(
    const __nv_bfloat16* __restrict__ k, int N, int nsplit, int chunk,
    float* __restrict__ partials) {
  constexpr int TPR = D / 8;                 // threads per row (8 channels each)
  constexpr int RPI = kPoolThreads / TPR;    // rows per iteration
  __shared__ float red[RPI][D];
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int Hkv = gridDim.y;
  const int cg = threadIdx.x % TPR;
  const int rs = threadIdx.x / TPR;
  const int n0 = split * chunk;
  const int n1 = min(N, n0 + chunk);
  const __nv_bfloat16* base = k + (static_cast<size_t>(b) * Hkv + hk) * N * D + cg * 8;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  int n = n0 + rs;
#pragma unroll 4
  for (; n < n1; n += RPI) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(n) * D));
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(p[j]);
      acc[2 * j] += f.x;
      acc[2 * j + 1] += f.y;
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) red[rs][cg * 8 + j] = acc[j];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kPoolThreads) {
    float s = 0.f;
    for (int r = 0; r < RPI; ++r) s += red[r][c];
    partials[((static_cast<size_t>(b) * Hkv + hk) * nsplit + split) * D + c] = s;
  }
}

__global__ void __launch_bounds__(kMlpThreads) ea_router_mlp_kernel(
    const float* __restrict__ partials, int Hkv, int N, int d, int nsplit,
    const float* __restrict__ w1, const float* __restrict__ b1, int hidden,
    const float* __restrict__ w2, const float* __restrict__ b2, int Hq, float threshold,
    uint8_t* __restrict__ mask, float* __restrict__ logits) {
  extern __shared__ float sm[];
  const int in_dim = Hkv * d;
  float* x = sm;                 // [in_dim]
  float* h = sm + in_dim;        // [hidden]
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = kMlpThreads / 32;
  const float inv_n = 1.0f / static_cast<float>(N);
  for (int j = threadIdx.x; j < in_dim; j += kMlpThreads) {
    const int hk = j / d, c = j % d;
    const float* p = partials + (static_cast<size_t>(b) * Hkv + hk) * nsplit * d + c;
    float s = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) s += p[static_cast<size_t>(sp) * d];
    x[j] = s * inv_n;
  }
  __syncthreads();
  // layer 1: one warp per hidden unit, float4 over the input
  for (int o = warp; o < hidden; o += nwarps) {
    const float4* wr = reinterpret_cast<const float4*>(w1 + static_cast<size_t>(o) * in_dim);
    float acc = 0.f;
    for (int j = lane; j < in_dim / 4; j += 32) {
      const float4 w = __ldg(wr + j);
      acc = fmaf(w.x, x[4 * j], acc);
      acc = fmaf(w.y, x[4 * j + 1], acc);
      acc = fmaf(w.z, x[4 * j + 2], acc);
      acc = fmaf(w.w, x[4 * j + 3], acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) h[o] = fmaxf(acc + b1[o], 0.f);
  }
  __syncthreads();
  // layer 2: one warp per head
  for (int q = warp; q < Hq; q += nwarps) {
    const float4* wr = reinterpret_cast<const float4*>(w2 + static_cast<size_t>(q) * hidden);
    float acc = 0.f;
    for (int j = lane; j < hidden / 4; j += 32) {
      const float4 w = __ldg(wr + j);
      acc = fmaf(w.x, h[4 * j], acc);
      acc = fmaf(w.y, h[4 * j + 1], acc);
      acc = fmaf(w.z, h[4 * j + 2], acc);
      acc = fmaf(w.w, h[4 * j + 3], acc);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      const float z = acc + b2[q];
      mask[static_cast<size_t>(b) * Hq + q] = (z > threshold) ? 1 : 0;
      if (logits) logits[static_cast<size_t>(b) * Hq + q] = z;
    }
  }
}

int router_num_splits(int B, int Hkv, int N) {
  // about four CTAs per SM on a 148-SM part, at least 64 rows per CTA
  const int target = 592;
  int per = (target + B * Hkv - 1) / (B * Hkv);
  const int max_split = (N + 63) / 64;
  if (per > max_split) per = max_split;
  if (per < 1) per = 1;
  return per;
}

cudaError_t launch_router(const void* k, int B, int Hkv, int N, int d, const float* w1,
                          const float* b1, int hidden, const float* w2, const float* b2,
                          int Hq, float threshold, uint8_t* mask, float* logits,
                          float* partials, int nsplit, cudaStream_t stream) {
  const int chunk = (N + nsplit - 1) / nsplit;
  dim3 grid(nsplit, Hkv, B);
  if (d == 128)
    ea_router_pool_kernel<128><<<grid, kPoolThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), N, nsplit, chunk, partials);
  else
    ea_router_pool_kernel<64><<<grid, kPoolThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), N, nsplit, chunk, partials);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t smem = static_cast<size_t>(Hkv * d + hidden) * sizeof(float);
  static int configured[64] = {0};
  int dev = 0;
  err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (smem > 48 * 1024 && dev < 64 && !configured[dev]) {
    err = cudaFuncSetAttribute(ea_router_mlp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (8192 + 4096) * static_cast<int>(sizeof(float)));
    if (err != cudaSuccess) return err;
    configured[dev] = 1;
  }
  ea_router_mlp_kernel<<<B, kMlpThreads, smem, stream>>>(partials, Hkv, N, d, nsplit, w1, b1,
                                                         hidden, w2, b2, Hq, threshold, mask,
                                                         logits);
  return cudaGetLastError();
}

}  // namespace ea

// ---------------------------------------------------------------------------
// ea_router_decide_noalloc: the router for callers that cannot allocate.
//
// The pooling partial sums go to a fixed array that lives in this library's
// device image instead of a caller-supplied workspace.  Host code must not
// pass the array's name to a kernel: on the host it only stands for the
// symbol, not a device address.  The device address is looked up once per
// device with cudaGetSymbolAddress while that device is current.
namespace {

constexpr int kNoallocMaxDevices = 64;
static __device__ __align__(256) unsigned char g_router_noalloc_scratch[EA_ROUTER_NOALLOC_MAX_BYTES];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoallocMaxDevices] = {nullptr};

// Device address of this device's scratch array, or nullptr on failure.
void* noalloc_scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_router_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" ea_status ea_router_decide_noalloc(const void* k, int B, int Hkv, int N, int d,
                                              const float* w1, const float* b1, int hidden,
                                              const float* w2, const float* b2, int Hq,
                                              float threshold, uint8_t* route_mask,
                                              float* logits_out, void* stream) {
  const size_t need = ea_router_workspace_size(B, Hkv, N, d);
  if (need > EA_ROUTER_NOALLOC_MAX_BYTES) return EA_ERR_SCRATCH_LIMIT;
  if (need == 0) return ea_router_decide(k, B, Hkv, N, d, w1, b1, hidden, w2, b2, Hq, threshold,
                                         route_mask, logits_out, nullptr, 0, stream);
  void* scratch = noalloc_scratch_for_current_device();
  if (!scratch) return EA_ERR_CUDA;
  return ea_router_decide(k, B, Hkv, N, d, w1, b1, hidden, w2, b2, Hq, threshold, route_mask,
                          logits_out, scratch, EA_ROUTER_NOALLOC_MAX_BYTES, stream);
}
