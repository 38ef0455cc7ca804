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

namespace ea {

constexpr int kPoolThreads = 256;
constexpr int kMlpThreads = 256;

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

template <int D>
__global__ void __launch_bounds__(kPoolThreads) ea_router_pool_kernel(
    const __nv_bfloat16* __restrict__ k, const int32_t* __restrict__ cu, int N, int total,
    int nsplit, float* __restrict__ partials) {
  constexpr int TPR = D / 8;                 // threads per row (8 channels each)
  constexpr int RPI = kPoolThreads / TPR;    // rows per iteration
  __shared__ float red[RPI][D];
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int Hkv = gridDim.y;
  const int cg = threadIdx.x % TPR;
  const int rs = threadIdx.x / TPR;
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
  for (int j = 0; j < 8; ++j) red[rs][cg * 8 + j] = acc[j];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kPoolThreads) {
    float s = 0.f;
    for (int r = 0; r < RPI; ++r) s += red[r][c];
    partials[((static_cast<size_t>(b) * Hkv + hk) * nsplit + split) * D + c] = s;
  }
}

// x[b][hk*d + c] = (sum over splits, in split order) / rows of sequence b
// (zero for an empty sequence); one thread per channel.
__global__ void ea_router_reduce_kernel(const float* __restrict__ partials,
                                        const int32_t* __restrict__ cu, int Hkv, int N, int total,
                                        int d, int nsplit, float* __restrict__ x) {
  const int b = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;   // j = hk * d + c
  if (j >= Hkv * d) return;
  const int hk = j / d, c = j % d;
  int t0;
  const int len = router_seq_rows(cu, N, total, b, &t0);
  const float* p = partials + (static_cast<size_t>(b) * Hkv + hk) * nsplit * d + c;
  float s = 0.f;
  for (int sp = 0; sp < nsplit; ++sp) s += p[static_cast<size_t>(sp) * d];
  x[static_cast<size_t>(b) * Hkv * d + j] = len > 0 ? s * (1.0f / static_cast<float>(len)) : 0.f;
}

// One warp per output: y[b][o] = act(W[o] . x[b] + bias[o]), float4 over the
// input, lanes reduced in a fixed shuffle order.  For the last layer the
// output is the logit z, and the route bit z > threshold is written too.
template <bool kLast>
__global__ void __launch_bounds__(kMlpThreads) ea_router_layer_kernel(
    const float* __restrict__ x, int in_dim, const float* __restrict__ w,
    const float* __restrict__ bias, int out_dim, float* __restrict__ y, float threshold,
    uint8_t* __restrict__ mask) {
  const int b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o = blockIdx.x * (kMlpThreads / 32) + warp;
  if (o >= out_dim) return;
  const float4* wr = reinterpret_cast<const float4*>(w + static_cast<size_t>(o) * in_dim);
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(b) * in_dim);
  float acc = 0.f;
#pragma unroll 4
  for (int j = lane; j < in_dim / 4; j += 32) {
    const float4 wv = __ldg(wr + j);
    const float4 xv = xr[j];
    acc = fmaf(wv.x, xv.x, acc);
    acc = fmaf(wv.y, xv.y, acc);
    acc = fmaf(wv.z, xv.z, acc);
    acc = fmaf(wv.w, xv.w, acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    const float v = acc + bias[o];
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
