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

#include <math.h>
#include <mutex>

#include "ea.h"
#include "ea_internal.h"
#include "ea_ptx.cuh"
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

// The same pooling items for rows row0 + blockIdx.y of the flattened (batch,
// kv head) index of a padded K (one shard's rows), with the whole problem's
// split count.
template <int D>
__global__ void __launch_bounds__(kPoolThreads) ea_router_pool_rows_kernel(
    const __nv_bfloat16* __restrict__ k, int N, int Hkv, int row0, int nsplit,
    float* __restrict__ partials) {
  __shared__ float red[(kPoolThreads / (D / 8)) * D];
  const int r = row0 + static_cast<int>(blockIdx.y);
  router_pool_item<D>(k, nullptr, N, 0, Hkv, r / Hkv, r % Hkv, blockIdx.x, nsplit, partials, red,
                      threadIdx.x, 1);
}

// x of those rows, [nrows][d] (one channel per thread).
__global__ void ea_router_reduce_rows_kernel(const float* __restrict__ partials, int Hkv, int N,
                                             int d, int nsplit, int row0, int nrows,
                                             float* __restrict__ x_out) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;   // (row - row0) * d + c
  if (e >= nrows * d) return;
  const int r = row0 + e / d;
  x_out[e] = router_x(partials, nullptr, Hkv, N, 0, d, nsplit, r / Hkv, (r % Hkv) * d + e % d);
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

// ---------------------------------------------------------------- training
// Gumbel-Softmax straight-through routing (EA blog §2.1, training trick),
// with the caller's Gumbel noise g0, g1 [B][Hq] and temperature tau:
//   r_soft = sigmoid((z + g1 - g0) / tau), r_hard = [z + g1 - g0 > 0].
__global__ void ea_ste_gumbel_kernel(const float* __restrict__ z, const float* __restrict__ g0,
                                     const float* __restrict__ g1, float tau, int n,
                                     uint8_t* __restrict__ r_hard, float* __restrict__ r_soft) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float u = z[i] + g1[i] - g0[i];
  if (r_hard) r_hard[i] = u > 0.f ? 1 : 0;
  if (r_soft) r_soft[i] = 1.f / (1.f + expf(-u / tau));
}

// dr partials: CTA (b*Hq + h, split) sums dO * (O_SA - O_FA) over its rows,
// from out (the head's chosen mode) and out_other (its other mode): the sum
// of dO * (out_other - out), negated where the head chose SA (mask nonzero;
// mask == nullptr: every head chose FA).
constexpr int kDrThreads = 256;
__global__ void __launch_bounds__(kDrThreads) ea_ste_dr_kernel(
    const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out,
    const __nv_bfloat16* __restrict__ out_other, const uint8_t* __restrict__ mask, int N, int d,
    int nsplit, float* __restrict__ part) {
  __shared__ float red[kDrThreads / 32];
  const int bh = blockIdx.x, split = blockIdx.y;
  const size_t len = static_cast<size_t>(N) * d;
  const size_t chunk = (len / 8 + nsplit - 1) / nsplit * 8;   // whole 8-element groups
  const size_t e0 = split * chunk, e1 = min(len, e0 + chunk);
  const size_t base = static_cast<size_t>(bh) * len;
  float acc = 0.f;
  for (size_t e = e0 + threadIdx.x * 8; e < e1; e += kDrThreads * 8) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(dout + base + e));
    const uint4 f = __ldg(reinterpret_cast<const uint4*>(out + base + e));
    const uint4 sx = __ldg(reinterpret_cast<const uint4*>(out_other + base + e));
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* f2 = reinterpret_cast<const __nv_bfloat162*>(&f);
    const __nv_bfloat162* s2 = reinterpret_cast<const __nv_bfloat162*>(&sx);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 av = __bfloat1622float2(a2[j]), fv = __bfloat1622float2(f2[j]),
                   sv = __bfloat1622float2(s2[j]);
      acc = fmaf(av.x, sv.x - fv.x, acc);
      acc = fmaf(av.y, sv.y - fv.y, acc);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < kDrThreads / 32; ++w) t += red[w];
    part[static_cast<size_t>(bh) * nsplit + split] = (mask && mask[bh]) ? -t : t;
  }
}

// dr (summed in split order) and dz = dr * r (1 - r) / tau per (b, h).
__global__ void ea_ste_dz_kernel(const float* __restrict__ part, int nsplit,
                                 const float* __restrict__ z, const float* __restrict__ g0,
                                 const float* __restrict__ g1, float tau, int n,
                                 float* __restrict__ dr, float* __restrict__ dz) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float t = 0.f;
  for (int s = 0; s < nsplit; ++s) t += part[static_cast<size_t>(i) * nsplit + s];
  const float r = 1.f / (1.f + expf(-(z[i] + g1[i] - g0[i]) / tau));
  if (dr) dr[i] = t;
  dz[i] = t * r * (1.f - r) / tau;
}

// dW2[o][j] = sum_b dz[b][o] h[b][j] (j < hidden); db2[o] = sum_b dz[b][o] (j == hidden).
__global__ void ea_ste_w2_kernel(const float* __restrict__ dz, const float* __restrict__ h, int B,
                                 int Hq, int hidden, float* __restrict__ dw2,
                                 float* __restrict__ db2) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= Hq * (hidden + 1)) return;
  const int o = i / (hidden + 1), j = i % (hidden + 1);
  float t = 0.f;
  for (int b = 0; b < B; ++b)
    t = fmaf(dz[b * Hq + o], j < hidden ? h[static_cast<size_t>(b) * hidden + j] : 1.f, t);
  if (j < hidden) dw2[static_cast<size_t>(o) * hidden + j] = t;
  else db2[o] = t;
}

// dpre[b][j] = [h > 0] * sum_o dz[b][o] W2[o][j]  (h = ReLU(pre): h > 0 iff pre > 0).
__global__ void ea_ste_dpre_kernel(const float* __restrict__ dz, const float* __restrict__ w2,
                                   const float* __restrict__ h, int B, int Hq, int hidden,
                                   float* __restrict__ dpre) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * hidden) return;
  const int b = i / hidden, j = i % hidden;
  float t = 0.f;
  for (int o = 0; o < Hq; ++o) t = fmaf(dz[b * Hq + o], w2[static_cast<size_t>(o) * hidden + j], t);
  dpre[i] = h[i] > 0.f ? t : 0.f;
}

// dW1[j][c] = sum_b dpre[b][j] x[b][c] (c < in_dim); db1[j] = sum_b dpre[b][j] (c == in_dim).
__global__ void ea_ste_w1_kernel(const float* __restrict__ dpre, const float* __restrict__ x,
                                 int B, int hidden, int in_dim, float* __restrict__ dw1,
                                 float* __restrict__ db1) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<size_t>(hidden) * (in_dim + 1)) return;
  const int j = static_cast<int>(i / (in_dim + 1)), c = static_cast<int>(i % (in_dim + 1));
  float t = 0.f;
  for (int b = 0; b < B; ++b)
    t = fmaf(dpre[static_cast<size_t>(b) * hidden + j],
             c < in_dim ? x[static_cast<size_t>(b) * in_dim + c] : 1.f, t);
  if (c < in_dim) dw1[static_cast<size_t>(j) * in_dim + c] = t;
  else db1[j] = t;
}

// dk_pool[b][c] = (sum_j dpre[b][j] W1[j][c]) / N: the keys' gradient through
// the mean pooling, the same at every position of (b, c's kv head).
__global__ void ea_ste_dx_kernel(const float* __restrict__ dpre, const float* __restrict__ w1,
                                 int B, int hidden, int in_dim, int N,
                                 float* __restrict__ dk_pool) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * in_dim) return;
  const int b = i / in_dim, c = i % in_dim;
  float t = 0.f;
  for (int j = 0; j < hidden; ++j)
    t = fmaf(dpre[static_cast<size_t>(b) * hidden + j], w1[static_cast<size_t>(j) * in_dim + c], t);
  dk_pool[i] = t / static_cast<float>(N);
}

// dk[b][hk][n][c] += dk_pool[b][hk * d + c] for every position n (bf16 in
// place): CTA (position chunk, b * Hkv + hk), thread per 8 channels of a row
// (16-byte loads and stores), the plane's d pooled values in registers.
constexpr int kDkAddThreads = 256;
__global__ void __launch_bounds__(kDkAddThreads) ea_ste_dk_add_kernel(
    const float* __restrict__ dk_pool, int N, int d, int rows_per_cta,
    __nv_bfloat16* __restrict__ dk) {
  const int bh = blockIdx.y;
  const int tpr = d / 8;                          // threads per row
  const int c0 = (threadIdx.x % tpr) * 8;
  float add[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) add[j] = dk_pool[static_cast<size_t>(bh) * d + c0 + j];
  const int n0 = blockIdx.x * rows_per_cta;
  const int n1 = min(N, n0 + rows_per_cta);
  __nv_bfloat16* plane = dk + static_cast<size_t>(bh) * N * d;
  for (int n = n0 + threadIdx.x / tpr; n < n1; n += kDkAddThreads / tpr) {
    uint4* ptr = reinterpret_cast<uint4*>(plane + static_cast<size_t>(n) * d + c0);
    uint4 v = *ptr;
    uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16) + add[2 * j];
      const float hi = __uint_as_float(w[j] & 0xffff0000u) + add[2 * j + 1];
      w[j] = pack_bf16x2(lo, hi);
    }
    *ptr = v;
  }
}

int ste_dr_splits(int B, int Hq) {
  int per = (592 + B * Hq - 1) / (B * Hq);
  return per < 1 ? 1 : (per > 64 ? 64 : per);
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

cudaError_t launch_router_pool_rows(const void* k, int B, int Hkv, int N, int d, int row0,
                                    int nrows, float* partials, float* x_out,
                                    cudaStream_t stream) {
  const int nsplit = router_num_splits(B, Hkv, N);
  dim3 grid(nsplit, nrows);
  if (d == 128)
    ea_router_pool_rows_kernel<128><<<grid, kPoolThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), N, Hkv, row0, nsplit, partials);
  else
    ea_router_pool_rows_kernel<64><<<grid, kPoolThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), N, Hkv, row0, nsplit, partials);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  ea_router_reduce_rows_kernel<<<(nrows * d + 255) / 256, 256, 0, stream>>>(
      partials, Hkv, N, d, nsplit, row0, nrows, x_out);
  return cudaGetLastError();
}

cudaError_t launch_router_mlp(const float* x, int B, int in_dim, const float* w1,
                              const float* b1, int hidden, const float* w2, const float* b2,
                              int Hq, float threshold, uint8_t* mask, float* logits, float* hbuf,
                              cudaStream_t stream) {
  constexpr int kWarps = kMlpThreads / 32;
  ea_router_layer_kernel<false><<<dim3((hidden + kWarps - 1) / kWarps, B), kMlpThreads, 0,
                                  stream>>>(x, in_dim, w1, b1, hidden, hbuf, 0.f, nullptr);
  cudaError_t err = cudaGetLastError();
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

// Device address of device dev's copy of the scratch array, or nullptr on
// failure.  dev must be the current device: the symbol lookup uses it.
void* noalloc_scratch_for_device(int dev) {
  if (dev < 0 || dev >= kNoallocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_router_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

// True if p is device memory of device dev (the only memory the router's
// kernels may be given).
bool on_device(const void* p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();   // an unknown pointer leaves no sticky error
    return false;
  }
  return a.type == cudaMemoryTypeDevice && a.device == dev;
}

}  // namespace

namespace ea {
void router_noalloc_forget() {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  for (int i = 0; i < kNoallocMaxDevices; ++i) g_noalloc_ptr[i] = nullptr;
}
}  // namespace ea

extern "C" ea_status ea_router_decide_noalloc(const void* k, int B, int Hkv, int N, int d,
                                              const float* w1, const float* b1, int hidden,
                                              const float* w2, const float* b2, int Hq,
                                              float threshold, uint8_t* route_mask,
                                              float* logits_out, void* stream) {
  // the same checks, in the same order, as ea_router_decide; the scratch
  // limit only after them
  const ea_status chk = ea::router_check_args(k, B, Hkv, N, d, w1, b1, hidden, w2, b2, Hq,
                                              threshold, route_mask);
  if (chk != EA_OK) return chk;
  const size_t need = ea_router_workspace_size(B, Hkv, N, d);
  if (need > EA_ROUTER_NOALLOC_MAX_BYTES) return EA_ERR_SCRATCH_LIMIT;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return EA_ERR_CUDA;
  // the scratch is the current device's copy: the keys and the outputs must
  // live there too
  if (!on_device(k, dev) || !on_device(w1, dev) || !on_device(b1, dev) || !on_device(w2, dev) ||
      !on_device(b2, dev) || !on_device(route_mask, dev) ||
      (logits_out && !on_device(logits_out, dev)))
    return EA_ERR_INVALID_ARG;
  void* scratch = noalloc_scratch_for_device(dev);
  if (!scratch) return EA_ERR_CUDA;
  return ea_router_decide(k, B, Hkv, N, d, w1, b1, hidden, w2, b2, Hq, threshold, route_mask,
                          logits_out, scratch, EA_ROUTER_NOALLOC_MAX_BYTES, stream);
}

// ---------------------------------------------------------------------------
// Training launches (Gumbel-Softmax straight-through routing, EA blog §2.1).
namespace ea {
namespace {
size_t align256(size_t n) { return (n + 255) / 256 * 256; }
}  // namespace

size_t router_gumbel_workspace_bytes(int B, int Hkv, int N, int d, int hidden, int Hq) {
  return align256(router_workspace_bytes(B, Hkv, N, d, hidden)) +
         align256(static_cast<size_t>(B) * Hq * 4) + align256(static_cast<size_t>(B) * Hq);
}

cudaError_t launch_router_gumbel(const void* k, int B, int Hkv, int N, int d, const float* w1,
                                 const float* b1, int hidden, const float* w2, const float* b2,
                                 int Hq, const float* g0, const float* g1, float tau,
                                 uint8_t* route_mask, float* r_soft, float* logits_out,
                                 void* workspace, cudaStream_t s) {
  char* ws = static_cast<char*>(workspace);
  const size_t n = static_cast<size_t>(B) * Hq;
  size_t off = align256(router_workspace_bytes(B, Hkv, N, d, hidden));
  float* z = logits_out ? logits_out : reinterpret_cast<float*>(ws + off);
  off += align256(n * 4);
  uint8_t* scratch_mask = reinterpret_cast<uint8_t*>(ws + off);
  cudaError_t err = launch_router(k, nullptr, B, Hkv, N, 0, d, w1, b1, hidden, w2, b2, Hq, 0.f,
                                  scratch_mask, z, reinterpret_cast<float*>(ws),
                                  router_num_splits(B, Hkv, N), s);
  if (err != cudaSuccess) return err;
  ea_ste_gumbel_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
      z, g0, g1, tau, static_cast<int>(n), route_mask, r_soft);
  return cudaGetLastError();
}

size_t router_ste_workspace_bytes(int B, int Hkv, int N, int d, int hidden, int Hq) {
  const size_t n = static_cast<size_t>(B) * Hq;
  return align256(router_workspace_bytes(B, Hkv, N, d, hidden)) +  // partials, x, h
         align256(n * 4) +                                          // z
         align256(n) +                                              // mask (unused)
         align256(n * ste_dr_splits(B, Hq) * 4) +                   // dr partials
         align256(n * 4) +                                          // dz
         align256(static_cast<size_t>(B) * hidden * 4) +            // dpre
         align256(static_cast<size_t>(B) * Hkv * d * 4);            // dk_pool
}

cudaError_t launch_router_ste(const void* k, int B, int Hkv, int N, int d, const float* w1,
                              const float* b1, int hidden, const float* w2, const float* b2,
                              int Hq, const float* g0, const float* g1, float tau,
                              const void* dout, const void* out, const void* out_other,
                              const uint8_t* route_mask, float* dr_out, float* dw1, float* db1,
                              float* dw2, float* db2, float* dk_pool_out, void* dk_accum,
                              void* workspace, cudaStream_t s) {
  const size_t n = static_cast<size_t>(B) * Hq;
  const int nsd = ste_dr_splits(B, Hq);
  const int ns = router_num_splits(B, Hkv, N);
  const int in_dim = Hkv * d;
  char* ws = static_cast<char*>(workspace);
  float* partials = reinterpret_cast<float*>(ws);
  const float* x = partials + static_cast<size_t>(B) * Hkv * ns * d;
  const float* h = x + static_cast<size_t>(B) * in_dim;
  size_t off = align256(router_workspace_bytes(B, Hkv, N, d, hidden));
  float* z = reinterpret_cast<float*>(ws + off);       off += align256(n * 4);
  uint8_t* mask = reinterpret_cast<uint8_t*>(ws + off); off += align256(n);
  float* drp = reinterpret_cast<float*>(ws + off);     off += align256(n * nsd * 4);
  float* dz = reinterpret_cast<float*>(ws + off);      off += align256(n * 4);
  float* dpre = reinterpret_cast<float*>(ws + off);
  off += align256(static_cast<size_t>(B) * hidden * 4);
  float* dkp = dk_pool_out ? dk_pool_out : reinterpret_cast<float*>(ws + off);
  // forward recompute: x, h and z exactly as the router computes them
  cudaError_t err = launch_router(k, nullptr, B, Hkv, N, 0, d, w1, b1, hidden, w2, b2, Hq, 0.f,
                                  mask, z, partials, ns, s);
  if (err != cudaSuccess) return err;
  ea_ste_dr_kernel<<<dim3(static_cast<unsigned>(n), nsd), kDrThreads, 0, s>>>(
      static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(out),
      static_cast<const __nv_bfloat16*>(out_other), route_mask, N, d, nsd, drp);
  ea_ste_dz_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(
      drp, nsd, z, g0, g1, tau, static_cast<int>(n), dr_out, dz);
  ea_ste_w2_kernel<<<(Hq * (hidden + 1) + 255) / 256, 256, 0, s>>>(dz, h, B, Hq, hidden, dw2,
                                                                   db2);
  ea_ste_dpre_kernel<<<(B * hidden + 255) / 256, 256, 0, s>>>(dz, w2, h, B, Hq, hidden, dpre);
  const size_t nw1 = static_cast<size_t>(hidden) * (in_dim + 1);
  ea_ste_w1_kernel<<<static_cast<unsigned>((nw1 + 255) / 256), 256, 0, s>>>(dpre, x, B, hidden,
                                                                            in_dim, dw1, db1);
  ea_ste_dx_kernel<<<(B * in_dim + 255) / 256, 256, 0, s>>>(dpre, w1, B, hidden, in_dim, N, dkp);
  if (dk_accum) {
    // about four CTAs per SM over all planes, whole rows per CTA
    const int planes = B * Hkv;
    int chunks = (592 + planes - 1) / planes;
    if (chunks > N) chunks = N;
    const int rows = (N + chunks - 1) / chunks;
    ea_ste_dk_add_kernel<<<dim3((N + rows - 1) / rows, planes), kDkAddThreads, 0, s>>>(
        dkp, N, d, rows, static_cast<__nv_bfloat16*>(dk_accum));
  }
  return cudaGetLastError();
}

}  // namespace ea
