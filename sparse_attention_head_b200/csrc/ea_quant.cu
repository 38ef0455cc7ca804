// ea_quant.cu — bf16 -> e4m3 quantization of attention inputs for the FP8
// variant of the fused kernel.
//
// Per (batch, head): amax = max |x| over the head's N x d values, then
// inv = 448 / amax and scale = amax / 448 in IEEE fp32 (1 and 1 for an
// all-zero head), and every value becomes e4m3(fp32(x * inv)), rounded to
// nearest even and saturated to +-448 (448 is e4m3's largest finite value).
// Layouts: BHSD codes [B][H][N][d], or, for V, the transposed codes
// [B][H][d][Npad] with Npad = N rounded up to a multiple of 16 (the P.V
// product then reads V with the keys as its contiguous K dimension); the
// padding positions are written as zero.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ea.h"
#include "ea_internal.h"
#include "ea_ptx.cuh"

namespace ea {

namespace {

constexpr int kAmaxThreads = 256;
constexpr int kQuantThreads = 256;
constexpr float kE4m3Max = 448.0f;

// Per-head fp32 reciprocal and scale from the amax bits (non-negative floats
// order as their bit patterns, so the amax was reduced with atomicMax).
__device__ __forceinline__ void head_inv_scale(uint32_t amax_bits, float* inv, float* scale) {
  const float amax = __uint_as_float(amax_bits);
  if (amax > 0.f) {
    *inv = __fdiv_rn(kE4m3Max, amax);
    *scale = __fdiv_rn(amax, kE4m3Max);
  } else {
    *inv = 1.f;
    *scale = 1.f;
  }
}

}  // namespace

// amax_bits[bh] = max(amax_bits[bh], bits of max |x| over CTA (split, bh)'s
// chunk of the head's `len` values (8 per thread step, 16-byte loads).
__global__ void __launch_bounds__(kAmaxThreads) ea_fp8_amax_kernel(
    const __nv_bfloat16* __restrict__ x, size_t len, int nsplit, uint32_t* __restrict__ amax_bits) {
  __shared__ uint32_t red[kAmaxThreads / 32];
  const int bh = blockIdx.y, split = blockIdx.x;
  const size_t chunk = (len / 8 + nsplit - 1) / nsplit * 8;
  const size_t e0 = split * chunk, e1 = min(len, e0 + chunk);
  const __nv_bfloat16* base = x + static_cast<size_t>(bh) * len;
  uint32_t m = 0;
  for (size_t e = e0 + threadIdx.x * 8; e < e1; e += kAmaxThreads * 8) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + e));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // |bf16| as the upper half of an fp32 bit pattern (sign cleared)
      m = max(m, (w[j] << 16) & 0x7fffffffu);
      m = max(m, w[j] & 0x7fff0000u);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int w = 0; w < kAmaxThreads / 32; ++w) t = max(t, red[w]);
    atomicMax(amax_bits + bh, t);
  }
}

// BHSD codes: thread per 8 consecutive values of one head (len % 8 == 0).
__global__ void __launch_bounds__(kQuantThreads) ea_fp8_quant_kernel(
    const __nv_bfloat16* __restrict__ x, size_t len, int heads,
    const uint32_t* __restrict__ amax_bits, uint8_t* __restrict__ codes,
    float* __restrict__ scale_out) {
  const size_t i = (static_cast<size_t>(blockIdx.x) * kQuantThreads + threadIdx.x) * 8;
  const size_t total = len * heads;
  if (i >= total) return;
  const int bh = static_cast<int>(i / len);
  float inv, scale;
  head_inv_scale(amax_bits[bh], &inv, &scale);
  if (i % len == 0) scale_out[bh] = scale;
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + i));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float f[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = __uint_as_float(w[j] << 16) * inv;
    f[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u) * inv;
  }
  uint2 o;
  o.x = pack_e4m3x4(f[0], f[1], f[2], f[3]);
  o.y = pack_e4m3x4(f[4], f[5], f[6], f[7]);
  *reinterpret_cast<uint2*>(codes + i) = o;
}

// Transposed codes [bh][c][Npad] (d = 128): CTA (position tile of 64, bh)
// stages x[n0 .. n0 + 63][0 .. 127] in shared memory, then thread c writes
// row c's 64 position bytes.  Positions >= N become zero.
__global__ void __launch_bounds__(128) ea_fp8_quant_t_kernel(
    const __nv_bfloat16* __restrict__ x, int N, int npad, const uint32_t* __restrict__ amax_bits,
    uint8_t* __restrict__ codes, float* __restrict__ scale_out) {
  constexpr int D = 128, TN = 64;
  __shared__ float tile[TN][D + 1];
  const int bh = blockIdx.y, n0 = blockIdx.x * TN;
  float inv, scale;
  head_inv_scale(amax_bits[bh], &inv, &scale);
  if (blockIdx.x == 0 && threadIdx.x == 0) scale_out[bh] = scale;
  const __nv_bfloat16* xb = x + static_cast<size_t>(bh) * N * D;
  // each thread loads 8 channels of 8 rows (16-byte loads, coalesced per row)
  for (int r = threadIdx.x / 16; r < TN; r += 128 / 16) {
    const int n = n0 + r, c0 = (threadIdx.x % 16) * 8;
    float f[8];
    if (n < N) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(xb + static_cast<size_t>(n) * D + c0));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        f[2 * j] = __uint_as_float(w[j] << 16) * inv;
        f[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u) * inv;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = 0.f;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) tile[r][c0 + j] = f[j];
  }
  __syncthreads();
  const int c = threadIdx.x;
  uint8_t* row = codes + (static_cast<size_t>(bh) * D + c) * npad + n0;
  const int nvalid = min(TN, npad - n0);      // bytes of this row inside [0, npad)
#pragma unroll
  for (int g = 0; g < TN / 16; ++g) {
    if (16 * g >= nvalid) break;
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = 16 * g + 4 * q;
      ow[q] = pack_e4m3x4(tile[r][c], tile[r + 1][c], tile[r + 2][c], tile[r + 3][c]);
    }
    *reinterpret_cast<uint4*>(row + 16 * g) = o;
  }
}

int fp8_npad(int N) { return (N + 15) / 16 * 16; }

size_t fp8_quant_workspace_bytes(int heads) {
  return (static_cast<size_t>(heads) * 4 + 255) / 256 * 256;
}

cudaError_t launch_fp8_quant(const void* x, int heads, int N, int d, int transpose, void* codes,
                             float* scale, void* workspace, cudaStream_t stream) {
  uint32_t* amax = static_cast<uint32_t*>(workspace);
  cudaError_t err = cudaMemsetAsync(amax, 0, static_cast<size_t>(heads) * 4, stream);
  if (err != cudaSuccess) return err;
  const size_t len = static_cast<size_t>(N) * d;
  // about four CTAs per SM across all heads, at least 64 KB of input each
  int nsplit = (592 + heads - 1) / heads;
  const int cap = static_cast<int>((len * 2 + 65535) / 65536);
  if (nsplit > cap) nsplit = cap;
  if (nsplit < 1) nsplit = 1;
  ea_fp8_amax_kernel<<<dim3(nsplit, heads), kAmaxThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), len, nsplit, amax);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  if (!transpose) {
    const size_t groups = len * heads / 8;
    ea_fp8_quant_kernel<<<static_cast<unsigned>((groups + kQuantThreads - 1) / kQuantThreads),
                          kQuantThreads, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), len,
                                                      heads, amax, static_cast<uint8_t*>(codes),
                                                      scale);
  } else {
    const int npad = fp8_npad(N);
    ea_fp8_quant_t_kernel<<<dim3((npad + 63) / 64, heads), 128, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), N, npad, amax, static_cast<uint8_t*>(codes), scale);
  }
  return cudaGetLastError();
}

}  // namespace ea
