/* A plain C99 caller of libea.so: the C ABI used with no Python and no torch.
 *
 * Seeded inputs (a 32-bit LCG; bf16 by truncation of the float bits) go to
 * the device with the CUDA runtime; the router decides the mask from k, the
 * fused prefill computes out; q, k, v, the router weights, the mask and out
 * are written to a file for the test to check against the oracle.
 *
 *   ea_c_smoke <output file>      exit status 0 on success
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "ea.h"

enum { B = 1, HQ = 4, HKV = 2, N = 300, D = 64, SINK = 8, WINDOW = 100, HIDDEN = 32 };

static uint32_t lcg_state = 12345u;
static float uniform_pm1(void) {   /* in [-1, 1) */
  lcg_state = lcg_state * 1664525u + 1013904223u;
  return (float)(lcg_state >> 8) / 8388608.0f - 1.0f;
}
static uint16_t to_bf16(float x) {  /* round toward zero: exact on the device */
  uint32_t u;
  memcpy(&u, &x, 4);
  return (uint16_t)(u >> 16);
}

#define CK(call)                                                          \
  do {                                                                    \
    cudaError_t e_ = (call);                                              \
    if (e_ != cudaSuccess) {                                              \
      fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));         \
      return 2;                                                           \
    }                                                                     \
  } while (0)
#define EA(call)                                                          \
  do {                                                                    \
    int s_ = (call);                                                      \
    if (s_ != EA_OK) {                                                    \
      fprintf(stderr, "%s: %s\n", #call, ea_status_string(s_));           \
      return 3;                                                           \
    }                                                                     \
  } while (0)

int main(int argc, char** argv) {
  if (argc != 2) return 1;
  const size_t nq = (size_t)B * HQ * N * D, nkv = (size_t)B * HKV * N * D;
  uint16_t* hq = malloc(nq * 2);
  uint16_t* hk = malloc(nkv * 2);
  uint16_t* hv = malloc(nkv * 2);
  uint16_t* hout = malloc(nq * 2);
  float* w1 = malloc(sizeof(float) * HIDDEN * HKV * D);
  float b1[HIDDEN], w2[HQ * HIDDEN], b2[HQ];
  uint8_t mask[B * HQ];
  size_t i;
  for (i = 0; i < nq; ++i) hq[i] = to_bf16(2.0f * uniform_pm1());
  /* keys with a per-channel offset, so the pooled vector is O(1) */
  for (i = 0; i < nkv; ++i) hk[i] = to_bf16(uniform_pm1() + ((i % D) % 3 == 0 ? 1.0f : -0.5f));
  for (i = 0; i < nkv; ++i) hv[i] = to_bf16(2.0f * uniform_pm1());
  for (i = 0; i < (size_t)HIDDEN * HKV * D; ++i) w1[i] = 0.1f * uniform_pm1();
  for (i = 0; i < HIDDEN; ++i) b1[i] = 0.05f * uniform_pm1();
  for (i = 0; i < (size_t)HQ * HIDDEN; ++i) w2[i] = uniform_pm1();
  /* biases far from the threshold: heads 1 and 2 sparse, whatever the data term */
  b2[0] = -5.0f; b2[1] = 5.0f; b2[2] = 5.0f; b2[3] = -5.0f;

  void *dq, *dk, *dv, *dout, *dmask, *dw1, *db1, *dw2, *db2, *rws, *aws;
  CK(cudaMalloc(&dq, nq * 2));
  CK(cudaMalloc(&dk, nkv * 2));
  CK(cudaMalloc(&dv, nkv * 2));
  CK(cudaMalloc(&dout, nq * 2));
  CK(cudaMalloc(&dmask, B * HQ));
  CK(cudaMalloc(&dw1, sizeof(float) * HIDDEN * HKV * D));
  CK(cudaMalloc(&db1, sizeof b1));
  CK(cudaMalloc(&dw2, sizeof w2));
  CK(cudaMalloc(&db2, sizeof b2));
  CK(cudaMemcpy(dq, hq, nq * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dk, hk, nkv * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dv, hv, nkv * 2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dw1, w1, sizeof(float) * HIDDEN * HKV * D, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(db1, b1, sizeof b1, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(dw2, w2, sizeof w2, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(db2, b2, sizeof b2, cudaMemcpyHostToDevice));

  const size_t rbytes = ea_router_workspace_size(B, HKV, N, D);
  ea_attn_params p;
  memset(&p, 0, sizeof p);
  p.B = B; p.Hq = HQ; p.Hkv = HKV; p.N = N; p.d = D;
  p.sink = SINK; p.window = WINDOW; p.softmax_scale = 0.0f; p.select = EA_SELECT_ALL;
  const size_t abytes = ea_hybrid_attn_workspace_size(&p);
  if (rbytes == 0 || abytes == 0) return 4;
  CK(cudaMalloc(&rws, rbytes));
  CK(cudaMalloc(&aws, abytes));
  CK(cudaMemset(aws, 0, abytes));

  EA(ea_router_decide(dk, B, HKV, N, D, (const float*)dw1, (const float*)db1, HIDDEN,
                      (const float*)dw2, (const float*)db2, HQ, 0.0f, (uint8_t*)dmask, NULL,
                      rws, rbytes, NULL));
  EA(ea_hybrid_attn_prefill(dq, dk, dv, (const uint8_t*)dmask, &p, dout, aws, abytes, NULL));
  int dev_status = -1;
  EA(ea_get_device_status(aws, NULL, &dev_status));
  if (dev_status != EA_OK) return 5;
  CK(cudaMemcpy(hout, dout, nq * 2, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(mask, dmask, B * HQ, cudaMemcpyDeviceToHost));

  FILE* f = fopen(argv[1], "wb");
  if (!f) return 6;
  const int32_t dims[9] = {B, HQ, HKV, N, D, SINK, WINDOW, HIDDEN, ea_version()};
  fwrite(dims, sizeof dims, 1, f);
  fwrite(hq, 2, nq, f);
  fwrite(hk, 2, nkv, f);
  fwrite(hv, 2, nkv, f);
  fwrite(w1, sizeof(float), (size_t)HIDDEN * HKV * D, f);
  fwrite(b1, sizeof b1, 1, f);
  fwrite(w2, sizeof w2, 1, f);
  fwrite(b2, sizeof b2, 1, f);
  fwrite(mask, 1, B * HQ, f);
  fwrite(hout, 2, nq, f);
  fclose(f);
  printf("ea_c_smoke ok: mask %d %d %d %d\n", mask[0], mask[1], mask[2], mask[3]);
  return 0;
}
