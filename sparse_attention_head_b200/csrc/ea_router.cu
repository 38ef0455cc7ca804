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
// Kernel 2 sums the partials in split order and divides by the sequence's
//   row count (x; a packed batch pools each sequence's own tokens); kernels 3
//   and 4 run h = ReLU(W1 x + b1) and z = W2 h + b2 with one warp per output
//   spread over many CTAs (fixed shuffle order), and write z and the mask
//   z > threshold.  All kernels are deterministic: same inputs, same bits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "ea.h"
#include "ea_internal.h"
#include "ea_router_dev.cuh"

namespace ea {

constexpr int kMlpThreads = 256;

template <int D>
__global__ void __launch_bounds__(kPoolThreads) ea_router_pool_kernel(
    const __nv_bfloat16* __restrict__ k, const int32_t* __restrict__ cu, int N, int total,
    int nsplit, float* __restrict__ partials) {
  __shared__ float red[(kPoolThreads / (D / 8)) * D];
  router_pool_item<D>(k, cu, N, total, gridDim.y, blockIdx.z, blockIdx.y, blockIdx.x, nsplit,
                      partials, red, threadIdx.x, 1);
}

// x[b][j] for one channel per thread.
__global__ void ea_router_reduce_kernel(const float* __restrict__ partials,
                                        const int32_t* __restrict__ cu, int Hkv, int N, int total,
                                        int d, int nsplit, float* __restrict__ x) {
  const int b = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;   // j = hk * d + c
  if (j >= Hkv * d) return;
  x[static_cast<size_t>(b) * Hkv * d + j] = router_x(partials, cu, Hkv, N, total, d, nsplit, b, j);
}

// One warp per output: y[b][o] = act(W[o] . x[b] + bias[o]).  For the last
// layer the output is the logit z, and the route bit z > threshold is
// written too.
template <bool kLast>
__global__ void __launch_bounds__(kMlpThreads) ea_router_layer_kernel(
    const float* __restrict__ x, int in_dim, const float* __restrict__ w,
    const float* __restrict__ bias, int out_dim, float* __restrict__ y, float threshold,
    uint8_t* __restrict__ mask) {
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * (kMlpThreads / 32) + warp;
  if (o >= out_dim) return;
  const float v = router_warp_dot(x + static_cast<size_t>(b) * in_dim, in_dim, w, bias, o, lane);
  if (lane == 0) {
    if (kLast) {
      if (y) y[static_cast<size_t>(b) * out_dim + o] = v;
      mask[static_cast<size_t>(b) * out_dim + o] = (v > threshold) ? 1 : 0;
    } else {
      y[static_cast<size_t>(b) * out_dim + o] = fmaxf(v, 0.f);
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

size_t router_workspace_bytes(int B, int Hkv, int N, int d, int hidden) {
  const int ns = router_num_splits(B, Hkv, N);
  const size_t parts = static_cast<size_t>(B) * Hkv * ns * d;
  const size_t x = static_cast<size_t>(B) * Hkv * d;
  const size_t h = static_cast<size_t>(B) * hidden;
  return (parts + x + h) * sizeof(float);
}

cudaError_t launch_router(const void* k, const int32_t* cu, int B, int Hkv, int N, int total,
                          int d, const float* w1, const float* b1, int hidden, const float* w2,
                          const float* b2, int Hq, float threshold, uint8_t* mask, float* logits,
                          float* partials, int nsplit, cudaStream_t stream) {
  const int in_dim = Hkv * d;
  float* xbuf = partials + static_cast<size_t>(B) * Hkv * nsplit * d;
  float* hbuf = xbuf + static_cast<size_t>(B) * in_dim;
  dim3 grid(nsplit, Hkv, B);
  if (d == 128)
    ea_router_pool_kernel<128><<<grid, kPoolThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), cu, N, total, nsplit, partials);
  else
    ea_router_pool_kernel<64><<<grid, kPoolThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), cu, N, total, nsplit, partials);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  ea_router_reduce_kernel<<<dim3((in_dim + 255) / 256, B), 256, 0, stream>>>(
      partials, cu, Hkv, N, total, d, nsplit, xbuf);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  constexpr int kWarps = kMlpThreads / 32;
  ea_router_layer_kernel<false><<<dim3((hidden + kWarps - 1) / kWarps, B), kMlpThreads, 0,
                                  stream>>>(xbuf, in_dim, w1, b1, hidden, hbuf, 0.f, nullptr);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  ea_router_layer_kernel<true><<<dim3((Hq + kWarps - 1) / kWarps, B), kMlpThreads, 0,
                                 stream>>>(hbuf, hidden, w2, b2, Hq, logits, threshold, mask);
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
