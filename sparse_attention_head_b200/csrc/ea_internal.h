// ea_internal.h — declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ea.h"

namespace ea {

// Arguments of the fused hybrid attention kernel.  The tensor maps describe
// q [B*Hq][N][d], k and v [B*Hkv][N][d] (bf16, inner dim d), or for a packed
// batch q as (d, T, Hq) and k, v as (d, T, Hkv) over [T][heads][d] memory,
// all with a 64 x 128 x 1 box and 128-byte swizzle.
struct alignas(64) AttnArgs {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  const uint8_t* mask;      // [B*Hq], nonzero = sparse
  void* out;                // bf16 [B][Hq][N][d], or [T][Hq][d] for a packed batch
  int* status;              // device status word
  // Packed batch (nullptr: padded BHSD of length N): sequence b holds tokens
  // [cu_seqlens[b], cu_seqlens[b + 1]) of q [T][Hq][d], k, v [T][Hkv][d].
  const int32_t* cu_seqlens;
  int total;                // T, tokens of a packed batch
  float* lse;               // optional [B][Hq][N]: natural log-sum-exp of each row (padded only)
  // Training forward (padded only): every head runs in both modes; the mode
  // the mask chooses goes to `out` (and `lse`), the other one to out_other.
  void* out_other;
  int both;
  // FP8 variant (q, k e4m3 BHSD, v e4m3 transposed [B*Hkv][d][Npad]): the
  // per-(batch, head) dequantization scales of q, k and v.
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  int B, Hq, Hkv, N;
  int sink, window;
  float scale_log2;         // softmax scale * log2(e)
  int select;               // ea_select
  unsigned long long timeout_ns;
  // Failure-detection test hooks, compiled only into the library built with
  // EA_TEST_HOOKS (-1 = off; the release library never sets them): the
  // producer skips the copy of K/V ring position debug_drop_kv_pos, so the
  // kernel's bounded wait for it runs out; CTA 0 of a routed launch leaves
  // without arriving at grid barrier number debug_skip_grid_sync, so the
  // other CTAs' bounded barrier waits run out.
  int debug_drop_kv_pos;
  int debug_skip_grid_sync;
  // Shard of the launch (nullptr = every head): [B*Hkv], nonzero where the
  // query heads of (batch, kv head) run; the others' output rows are not
  // written.
  const uint8_t* group_sel;
  // The same by query head (nullptr = every head): [B*Hq], nonzero where
  // head (batch, h) runs.
  const uint8_t* head_sel;
  // Dynamic unit dispatch, inside the caller's 256-byte status block: the
  // launch's ticket counter and the count of CTAs done taking tickets (the
  // last one resets both to zero for the next launch).  Set by the launcher.
  unsigned int* ticket;
  unsigned int* done_ctas;
  // Per-unit trace (nullptr = off): trace[0] counts records; record i sits
  // at trace[8 + 6 i] .. +5 = {start, first S ready, last P handed over,
  // end (ns), CTA << 48 | level << 32 | rank, sparse << 62 | head of slot 0
  // << 44 | head of slot 1 << 32 | KV tiles}; records past trace_max are
  // counted, not kept.
  unsigned long long* trace;
  int trace_max;
  // Routed launch only: the router runs in the kernel's prologue (pool,
  // x, MLP layer 1, layer 2 + threshold, separated by grid barriers) and
  // writes the route mask (`mask` above points at the same buffer).
  const void* k_raw;        // the key tensor as the router reads it
  const float* w1;
  const float* b1;
  const float* w2;
  const float* b2;
  int hidden;
  float threshold;
  uint8_t* mask_out;
  float* logits;            // may be nullptr
  float* partials;          // router scratch: partials, then x, then h
  int nsplit;
  unsigned int* bar_count;  // grid barrier: arrivals of the current phase
  unsigned int* bar_gen;    //               and its generation
};

// Arguments of the tcgen05 backward kernels (padded BHSD, d = 128).
struct BwdArgs {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;   // (d, N, B*heads) boxes of 64 x 128 x 1
  const float* lse;                      // [B][Hq][N] natural log-sum-exp
  const float* dvec;                     // [B][Hq][N] rowsum(dO * O) (computed first)
  // The dK/dV kernel's per-step vectors, written with dvec: for query q of
  // (b, h), row b * Hq + h of [B*Hq][npad] (npad = 128 * ceil(N / 128)):
  // -lse * log2(e) and -D, zero for q >= N.  Each 128-query tile's vector is
  // one 512-byte bulk copy.
  const float* vl_pad;
  const float* vd_pad;
  int npad;
  const uint8_t* mask;                   // [B][Hq]
  __nv_bfloat16* dq;                     // [B][Hq][N][d]
  __nv_bfloat16* dk;                     // [B][Hkv][N][d]
  __nv_bfloat16* dv;
  int* status;
  int B, Hq, Hkv, N, sink, window;
  float scale, scale_log2;
  unsigned long long timeout_ns;
  // Unit lists of the two kernels (written by ea_bwd_sched_kernel): CTA c
  // runs units list[offs[c]] .. list[offs[c + 1] - 1] in that order.  sorted
  // and cta are the schedule's scratch (one int per unit each).
  int* offs_kv;
  int* list_kv;
  int* sorted_kv;
  int* cta_kv;
  int* offs_q;
  int* list_q;
  int* sorted_q;
  int* cta_q;
};
// Upper bound of the CTAs a backward kernel is launched with.
constexpr int kBwdMaxGrid = 1024;
// Ints of backward workspace the unit lists need, after D.
size_t bwd_sched_ints(int B, int Hq, int Hkv, int N);
// D = rowsum(dO * O) into dvec (and the padded vectors vl_pad, vd_pad), then
// the dK/dV and dQ kernels.
cudaError_t launch_backward(const BwdArgs& a, const void* dout, const void* out, float* dvec,
                            float* vl_pad, float* vd_pad, int grid_sms, cudaStream_t stream);

// SM count of the current device (cached per device); 0 on error.
int device_sms();
// Bound of every device-side wait, from EA_WAIT_TIMEOUT_MS (default 2 s).
unsigned long long wait_timeout_ns();

// Dynamic shared memory the kernel for head dim D needs.
int attn_smem_bytes(int D);

// Launch the fused kernel (D in {64, 128}) with `grid` CTAs.
cudaError_t launch_attn(int D, const AttnArgs& args, int grid, cudaStream_t stream);
// The routed kernel (router in the prologue), as a cooperative launch: all
// CTAs resident at once (they meet at grid barriers), or an error.
cudaError_t launch_attn_routed(int D, const AttnArgs& args, int grid, cudaStream_t stream);
// The FP8 variant of the fused kernel (d = 128, not routed).
cudaError_t launch_attn_fp8(const AttnArgs& args, int grid, cudaStream_t stream);

// bf16 -> e4m3 per-head quantization (x: [heads][N][d], d = 128): codes
// [heads][N][d], or transposed [heads][d][fp8_npad(N)]; scale [heads].
int fp8_npad(int N);
size_t fp8_quant_workspace_bytes(int heads);
cudaError_t launch_fp8_quant(const void* x, int heads, int N, int d, int transpose, void* codes,
                             float* scale, void* workspace, cudaStream_t stream);

// Router: pooled partial sums, then the MLP and the threshold.
// The argument checks of ea_router_decide (status codes as its header states).
ea_status router_check_args(const void* k, int B, int Hkv, int N, int d, const float* w1,
                            const float* b1, int hidden, const float* w2, const float* b2,
                            int Hq, float threshold, const uint8_t* route_mask);
// Forget the device addresses of the fixed router scratch array (they are
// looked up again on the next call that needs them).
void router_noalloc_forget();
int router_num_splits(int B, int Hkv, int N);
size_t router_workspace_bytes(int B, int Hkv, int N, int d, int hidden);
// Pooled rows [row0, row0 + nrows) of the flattened (batch, kv head) index of
// a padded K [B][Hkv][N][d] into x_out [nrows][d], with the split count of the
// whole problem (so the bits equal those launch_router computes).
cudaError_t launch_router_pool_rows(const void* k, int B, int Hkv, int N, int d, int row0,
                                    int nrows, float* partials, float* x_out,
                                    cudaStream_t stream);
// The router's two MLP layers and threshold on a pooled x [B][in_dim];
// hbuf holds B * hidden floats.
cudaError_t launch_router_mlp(const float* x, int B, int in_dim, const float* w1,
                              const float* b1, int hidden, const float* w2, const float* b2,
                              int Hq, float threshold, uint8_t* mask, float* logits, float* hbuf,
                              cudaStream_t stream);
// cu == nullptr: padded K [B][Hkv][N][d]; else packed K [total][Hkv][d] with
// sequence b at tokens [cu[b], cu[b + 1]).
cudaError_t launch_router(const void* k, const int32_t* cu, int B, int Hkv, int N, int total,
                          int d, const float* w1, const float* b1, int hidden, const float* w2,
                          const float* b2, int Hq, float threshold, uint8_t* mask, float* logits,
                          float* partials, int nsplit, cudaStream_t stream);

// Router training: the Gumbel-Softmax decision and the straight-through
// gradients.  Workspace layouts are fixed by the *_workspace_bytes sizes.
size_t router_gumbel_workspace_bytes(int B, int Hkv, int N, int d, int hidden, int Hq);
cudaError_t launch_router_gumbel(const void* k, int B, int Hkv, int N, int d, const float* w1,
                                 const float* b1, int hidden, const float* w2, const float* b2,
                                 int Hq, const float* g0, const float* g1, float tau,
                                 uint8_t* route_mask, float* r_soft, float* logits_out,
                                 void* workspace, cudaStream_t s);
size_t router_ste_workspace_bytes(int B, int Hkv, int N, int d, int hidden, int Hq);
cudaError_t launch_router_ste(const void* k, int B, int Hkv, int N, int d, const float* w1,
                              const float* b1, int hidden, const float* w2, const float* b2,
                              int Hq, const float* g0, const float* g1, float tau,
                              const void* dout, const void* out, const void* out_other,
                              const uint8_t* route_mask, float* dr_out, float* dw1, float* db1,
                              float* dw2, float* db2, float* dk_pool_out, void* dk_accum,
                              void* workspace, cudaStream_t s);

}  // namespace ea
