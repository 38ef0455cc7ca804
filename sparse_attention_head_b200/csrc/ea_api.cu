// ea_api.cu — the C ABI of libea.so: argument checks, TMA descriptor
// encoding and kernel launches.  See include/ea.h for the contract.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "ea.h"
#include "ea_internal.h"
#include "ea_sched.h"

namespace ea {

constexpr int kMaxSmDevices = 64;
// Widest router hidden layer the workspaces are sized for.
constexpr int kRouterMaxHidden = 4096;

int device_sms() {
  static int sms[kMaxSmDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < kMaxSmDevices && sms[dev]) return sms[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < kMaxSmDevices) sms[dev] = n;
  return n;
}

unsigned long long wait_timeout_ns() {
  static unsigned long long ns = 0;
  static std::once_flag once;
  std::call_once(once, [] {
    double ms = 2000.0;
    if (const char* e = getenv("EA_WAIT_TIMEOUT_MS")) {
      double v = atof(e);
      if (v > 0) ms = v;
    }
    ns = static_cast<unsigned long long>(ms * 1e6);
  });
  return ns;
}

// Argument checks of ea_router_decide, shared with the entry point that
// uses the library's fixed scratch array (same codes for the same arguments).
ea_status router_check_args(const void* k, int B, int Hkv, int N, int d, const float* w1,
                            const float* b1, int hidden, const float* w2, const float* b2,
                            int Hq, float threshold, const uint8_t* route_mask) {
  if (!k || !w1 || !b1 || !w2 || !b2 || !route_mask) return EA_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || N <= 0 || d <= 0 || hidden <= 0 || Hq <= 0)
    return EA_ERR_INVALID_ARG;
  if (threshold != threshold) return EA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return EA_ERR_UNSUPPORTED;
  if (Hkv * d > 8192 || hidden > kRouterMaxHidden || Hq > 1024) return EA_ERR_UNSUPPORTED;
  if ((Hkv * d) % 4 != 0 || hidden % 4 != 0) return EA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(k) & 15u) || (reinterpret_cast<uintptr_t>(w1) & 15u) ||
      (reinterpret_cast<uintptr_t>(w2) & 15u))
    return EA_ERR_MISALIGNED;
  return EA_OK;
}

}  // namespace ea

namespace {

using ea::device_sms;
using ea::kRouterMaxHidden;
using ea::wait_timeout_ns;


bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Unit counts per sequence are 16-bit in the kernel's tables.
constexpr int kMaxSeqLen = 32767 * EA_UNIT_ROWS;

// Validates the attention params; EA_OK if the kernels can run them.
ea_status check_params(const ea_attn_params* p) {
  if (!p) return EA_ERR_INVALID_ARG;
  if (p->B <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->N <= 0 || p->d <= 0)
    return EA_ERR_INVALID_ARG;
  if (p->sink < 0 || p->window < 1) return EA_ERR_INVALID_ARG;
  if (p->select < EA_SELECT_ALL || p->select > EA_SELECT_SA) return EA_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return EA_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return EA_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->B) * p->Hq > EA_MAX_ENTRIES) return EA_ERR_UNSUPPORTED;
  if (p->B > EA_MAX_SEQS) return EA_ERR_UNSUPPORTED;
  if (p->N > kMaxSeqLen) return EA_ERR_UNSUPPORTED;
  if (!(p->softmax_scale <= 0.f) && !(p->softmax_scale > 0.f)) return EA_ERR_INVALID_ARG;  // NaN
  return EA_OK;
}

// Validates packed-batch params the same way.
ea_status check_varlen(const ea_varlen_params* p) {
  if (!p) return EA_ERR_INVALID_ARG;
  if (p->B <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->total < 0 || p->max_seqlen < 0 || p->d <= 0)
    return EA_ERR_INVALID_ARG;
  if (p->sink < 0 || p->window < 1) return EA_ERR_INVALID_ARG;
  if (p->select < EA_SELECT_ALL || p->select > EA_SELECT_SA) return EA_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return EA_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return EA_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->B) * p->Hq > EA_MAX_ENTRIES) return EA_ERR_UNSUPPORTED;
  if (p->B > EA_MAX_SEQS) return EA_ERR_UNSUPPORTED;
  if (p->max_seqlen > kMaxSeqLen) return EA_ERR_UNSUPPORTED;
  if (!(p->softmax_scale <= 0.f) && !(p->softmax_scale > 0.f)) return EA_ERR_INVALID_ARG;  // NaN
  return EA_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 [rows3][n][d] tensor, box 64 x 128 x 1, 128-byte swizzle, OOB -> 0.
bool encode_bhsd(CUtensorMap* m, const void* ptr, int d, int n, int rows3) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                        static_cast<cuuint64_t>(rows3)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(d) * 2 * static_cast<cuuint64_t>(n)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// e4m3 bytes as a 3-D tensor (inner, rows, planes) with the given row and
// plane strides in bytes; box 128 x 128 x 1 (128-byte rows), 128-byte swizzle.
bool encode_u8(CUtensorMap* m, const void* ptr, int inner, int rows, int planes,
               uint64_t row_stride, uint64_t plane_stride) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(planes)};
  cuuint64_t strides[2] = {row_stride, plane_stride};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Packed [T][heads][d] memory as a (d, T, heads) tensor: tokens step by
// heads * d elements, heads by d; the same 64 x 128 x 1 box.
bool encode_packed(CUtensorMap* m, const void* ptr, int d, int total, int heads) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(total),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(heads) * static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Host copy of the kernel's sequence tables (EaSeqView): the schedule views
// build exactly what the kernel's prologue builds.
struct HostSched {
  std::vector<int16_t> nT, P;
  std::vector<int16_t> pref[4];
  std::vector<int> ent, len;
  EaSeqView view;
};

// The entry runs of one mode for sorted sequence b: per kv group, the
// group's selected heads two by two (paired), an odd one out single; every
// head single when a group has more than EA_MAX_PAIR_GROUP heads.
static void host_entries(const uint8_t* mask, int b, int Hq, int Hkv, int select, int mode,
                         std::vector<int>& paired, std::vector<int>& single) {
  const int G = Hq / Hkv;
  for (int hk = 0; hk < Hkv; ++hk) {
    std::vector<int> heads;
    for (int g = 0; g < G; ++g) {
      const int idx = b * Hq + hk * G + g;
      const bool sa = mask[idx] != 0;
      if (sa == (mode == 1) && select != (mode == 1 ? EA_SELECT_FA : EA_SELECT_SA))
        heads.push_back(idx);
    }
    const int n = static_cast<int>(heads.size());
    const int npair = G <= EA_MAX_PAIR_GROUP ? n / 2 : 0;
    for (int i = 0; i < 2 * npair; ++i) paired.push_back(heads[i]);
    for (int i = 2 * npair; i < n; ++i) single.push_back(heads[i]);
  }
}

void build_host_sched(const uint8_t* mask, int B, int Hq, int Hkv, int select, const int* lens,
                      int S, int W, HostSched& h) {
  std::vector<int> order(B), nb(B);
  for (int b = 0; b < B; ++b) {
    order[b] = b;
    nb[b] = ea_cdiv(lens[b], EA_BN);
  }
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return nb[x] > nb[y]; });
  h.len.assign(lens, lens + B);
  h.nT.resize(B);
  h.P.resize(B);
  std::vector<int> runs[4];
  for (int j = 0; j < 4; ++j) h.pref[j].assign(B + 1, 0);
  for (int k = 0; k < B; ++k) {
    h.nT[k] = static_cast<int16_t>(nb[order[k]]);
    h.P[k] = static_cast<int16_t>(ea_cdiv(nb[order[k]], 2));
    for (int mode = 0; mode < 2; ++mode) {
      h.pref[2 * mode][k] = static_cast<int16_t>(runs[2 * mode].size() / 2);
      h.pref[2 * mode + 1][k] = static_cast<int16_t>(runs[2 * mode + 1].size());
      host_entries(mask, order[k], Hq, Hkv, select, mode, runs[2 * mode], runs[2 * mode + 1]);
    }
  }
  h.ent.clear();
  for (int j = 0; j < 4; ++j) {
    h.pref[j][B] = static_cast<int16_t>(j % 2 == 0 ? runs[j].size() / 2 : runs[j].size());
    h.view.run0[j] = static_cast<int>(h.ent.size());
    h.ent.insert(h.ent.end(), runs[j].begin(), runs[j].end());
    h.view.pref[j] = h.pref[j].data();
  }
  h.view.nseq = B;
  h.view.nT = h.nT.data();
  h.view.P = h.P.data();
  h.view.Pmax = B > 0 ? h.P[0] : 0;
  h.view.mA = ea_long_level(S, W);
}

// Units of a schedule in rank order: {sparse, b, h0, h1, row0, n_kv_tiles}.
// A paired unit (h1 != h0) holds rows [row0, row0 + 128) of both heads; a
// single unit (h1 == h0) rows [row0, row0 + 256) of one head.
int list_units(const HostSched& h, int Hq, int Hkv, int d, int S, int W, int32_t* units_out,
               int max_units) {
  const int total = ea_total_units(h.view);
  if (units_out) {
    EaCursor cur;
    ea_cursor_init(cur, h.view, h.ent.data(), Hq, Hkv, ea_group_major(h.view.Pmax, d));
    for (int r = 0; r < total && r < max_units; ++r) {
      EaUnitRef u;
      if (!ea_cursor_seek(cur, h.view, h.ent.data(), r, &u)) break;
      const int idx = h.ent[u.pos];
      const int idx1 = u.paired ? h.ent[u.pos + 1] : idx;
      const EaShape sh = ea_make_shape(h.len[idx / Hq], S, W);
      const EaUnitTiles ut = ea_unit_tiles(sh, u.sparse, u.paired, u.level);
      int32_t* o = units_out + 6 * r;
      o[0] = u.sparse;
      o[1] = idx / Hq;
      o[2] = idx % Hq;
      o[3] = idx1 % Hq;
      o[4] = ut.r0;
      o[5] = ut.n;
    }
  }
  return total;
}

#ifdef EA_TEST_HOOKS
// Failure-injection hooks of the test build (libea_testhooks.so), read once
// per process: EA_DEBUG_DROP_KV_POS=<n> makes the attention producer skip
// K/V ring position n of every CTA; EA_DEBUG_SKIP_GRID_SYNC=<n> makes CTA 0
// of a routed launch leave without arriving at grid barrier n (0-3).  Each
// makes a bounded device wait run out.  The release library has neither.
int debug_env(const char* name) {
  const char* e = getenv(name);
  return e ? atoi(e) : -1;
}
int debug_drop_kv_pos() {
  static const int pos = debug_env("EA_DEBUG_DROP_KV_POS");
  return pos;
}
int debug_skip_grid_sync() {
  static const int phase = debug_env("EA_DEBUG_SKIP_GRID_SYNC");
  return phase;
}
#else
int debug_drop_kv_pos() { return -1; }
int debug_skip_grid_sync() { return -1; }
#endif

constexpr size_t kAttnWorkspace = 256;

}  // namespace

extern "C" {

const char* ea_status_string(int status) {
  switch (status) {
    case EA_OK: return "ok";
    case EA_ERR_INVALID_ARG: return "invalid argument";
    case EA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case EA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case EA_ERR_CUDA: return "CUDA call failed";
    case EA_ERR_TIMEOUT: return "device wait timed out";
    case EA_ERR_WORKSPACE: return "workspace missing or too small";
    case EA_ERR_SCRATCH_LIMIT: return "problem exceeds the fixed scratch of the no-allocation entry point";
    default: return "unknown status";
  }
}

int ea_version(void) { return (1 << 16) | 0; }

// ------------------------------------------------------------------ router
// Pooled partial sums, the pooled vector x and the hidden activations h (sized
// for the largest supported hidden width, so the size does not depend on it).
size_t ea_router_workspace_size(int B, int Hkv, int N, int d) {
  if (B <= 0 || Hkv <= 0 || N <= 0 || (d != 64 && d != 128)) return 0;
  return ea::router_workspace_bytes(B, Hkv, N, d, kRouterMaxHidden);
}

ea_status ea_router_decide(const void* k, int B, int Hkv, int N, int d, const float* w1,
                           const float* b1, int hidden, const float* w2, const float* b2,
                           int Hq, float threshold, uint8_t* route_mask, float* logits_out,
                           void* workspace, size_t workspace_bytes, void* stream) {
  const ea_status chk = ea::router_check_args(k, B, Hkv, N, d, w1, b1, hidden, w2, b2, Hq,
                                              threshold, route_mask);
  if (chk != EA_OK) return chk;
  const size_t need = ea_router_workspace_size(B, Hkv, N, d);
  if (!workspace || workspace_bytes < need) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  const int ns = ea::router_num_splits(B, Hkv, N);
  cudaError_t err = ea::launch_router(k, nullptr, B, Hkv, N, 0, d, w1, b1, hidden, w2, b2, Hq,
                                      threshold, route_mask, logits_out,
                                      static_cast<float*>(workspace), ns,
                                      static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

ea_status ea_router_pool_rows(const void* k, int B, int Hkv, int N, int d, int row0, int nrows,
                             float* x_out, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (!k || !x_out) return EA_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || N <= 0 || d <= 0) return EA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return EA_ERR_UNSUPPORTED;
  if (Hkv * d > 8192) return EA_ERR_UNSUPPORTED;
  if (row0 < 0 || nrows < 0 || static_cast<long long>(row0) + nrows >
                                   static_cast<long long>(B) * Hkv)
    return EA_ERR_INVALID_ARG;
  if (!aligned16(k)) return EA_ERR_MISALIGNED;
  const size_t need = ea_router_workspace_size(B, Hkv, N, d);
  if (!workspace || workspace_bytes < need) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  if (nrows == 0) return EA_OK;
  cudaError_t err = ea::launch_router_pool_rows(k, B, Hkv, N, d, row0, nrows,
                                                static_cast<float*>(workspace), x_out,
                                                static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

size_t ea_router_mlp_workspace_size(int B, int hidden) {
  if (B <= 0 || hidden <= 0 || hidden > kRouterMaxHidden) return 0;
  return static_cast<size_t>(B) * hidden * sizeof(float);
}

ea_status ea_router_mlp(const float* x, int B, int in_dim, const float* w1, const float* b1,
                        int hidden, const float* w2, const float* b2, int Hq, float threshold,
                        uint8_t* route_mask, float* logits_out, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (!x || !w1 || !b1 || !w2 || !b2 || !route_mask) return EA_ERR_INVALID_ARG;
  if (B <= 0 || in_dim <= 0 || hidden <= 0 || Hq <= 0) return EA_ERR_INVALID_ARG;
  if (threshold != threshold) return EA_ERR_INVALID_ARG;
  if (in_dim > 8192 || hidden > kRouterMaxHidden || Hq > 1024) return EA_ERR_UNSUPPORTED;
  if (in_dim % 4 != 0 || hidden % 4 != 0) return EA_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(w2)) return EA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < ea_router_mlp_workspace_size(B, hidden))
    return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  cudaError_t err = ea::launch_router_mlp(x, B, in_dim, w1, b1, hidden, w2, b2, Hq, threshold,
                                          route_mask, logits_out, static_cast<float*>(workspace),
                                          static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

size_t ea_router_varlen_workspace_size(int B, int Hkv, int max_seqlen, int d) {
  if (B <= 0 || Hkv <= 0 || max_seqlen < 0 || (d != 64 && d != 128)) return 0;
  return ea::router_workspace_bytes(B, Hkv, max_seqlen > 0 ? max_seqlen : 1, d,
                                    kRouterMaxHidden);
}

ea_status ea_router_decide_varlen(const void* k, const int32_t* cu_seqlens, int B, int Hkv,
                                  int total, int max_seqlen, int d, const float* w1,
                                  const float* b1, int hidden, const float* w2, const float* b2,
                                  int Hq, float threshold, uint8_t* route_mask, float* logits_out,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (!k || !cu_seqlens || !w1 || !b1 || !w2 || !b2 || !route_mask) return EA_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || total < 0 || max_seqlen < 0 || d <= 0 || hidden <= 0 || Hq <= 0)
    return EA_ERR_INVALID_ARG;
  if (threshold != threshold) return EA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return EA_ERR_UNSUPPORTED;
  if (Hkv * d > 8192 || hidden > kRouterMaxHidden || Hq > 1024) return EA_ERR_UNSUPPORTED;
  if ((Hkv * d) % 4 != 0 || hidden % 4 != 0) return EA_ERR_UNSUPPORTED;
  if (!aligned16(k) || !aligned16(w1) || !aligned16(w2)) return EA_ERR_MISALIGNED;
  const size_t need = ea_router_varlen_workspace_size(B, Hkv, max_seqlen, d);
  if (!workspace || workspace_bytes < need) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  const int ns = ea::router_num_splits(B, Hkv, max_seqlen > 0 ? max_seqlen : 1);
  cudaError_t err = ea::launch_router(k, cu_seqlens, B, Hkv, 0, total, d, w1, b1, hidden, w2, b2,
                                      Hq, threshold, route_mask, logits_out,
                                      static_cast<float*>(workspace), ns,
                                      static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

// Checks shared by the router training entry points (the router's own limits
// plus the Gumbel noise and a positive temperature).
static ea_status check_router_train(const void* k, int B, int Hkv, int N, int d, const float* w1,
                                    const float* b1, int hidden, const float* w2,
                                    const float* b2, int Hq, const float* g0, const float* g1,
                                    float tau) {
  if (!k || !w1 || !b1 || !w2 || !b2 || !g0 || !g1) return EA_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || N <= 0 || d <= 0 || hidden <= 0 || Hq <= 0) return EA_ERR_INVALID_ARG;
  if (!(tau > 0.f) || tau == INFINITY) return EA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return EA_ERR_UNSUPPORTED;
  if (Hkv * d > 8192 || hidden > kRouterMaxHidden || Hq > 1024 || B > EA_MAX_SEQS)
    return EA_ERR_UNSUPPORTED;
  if (hidden % 4 != 0) return EA_ERR_UNSUPPORTED;
  if (!aligned16(k) || !aligned16(w1) || !aligned16(w2)) return EA_ERR_MISALIGNED;
  return EA_OK;
}

size_t ea_router_gumbel_workspace_size(int B, int Hkv, int N, int d, int hidden, int Hq) {
  if (B <= 0 || Hkv <= 0 || N <= 0 || hidden <= 0 || Hq <= 0 || (d != 64 && d != 128)) return 0;
  return ea::router_gumbel_workspace_bytes(B, Hkv, N, d, hidden, Hq);
}

ea_status ea_router_decide_gumbel(const void* k, int B, int Hkv, int N, int d, const float* w1,
                                  const float* b1, int hidden, const float* w2, const float* b2,
                                  int Hq, const float* g0, const float* g1, float tau,
                                  uint8_t* route_mask, float* r_soft_out, float* logits_out,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  if (!route_mask) return EA_ERR_INVALID_ARG;
  const ea_status st = check_router_train(k, B, Hkv, N, d, w1, b1, hidden, w2, b2, Hq, g0, g1, tau);
  if (st != EA_OK) return st;
  if (!workspace || workspace_bytes < ea_router_gumbel_workspace_size(B, Hkv, N, d, hidden, Hq))
    return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  const cudaError_t err = ea::launch_router_gumbel(k, B, Hkv, N, d, w1, b1, hidden, w2, b2, Hq,
                                                   g0, g1, tau, route_mask, r_soft_out,
                                                   logits_out, workspace,
                                                   static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

size_t ea_router_ste_backward_workspace_size(int B, int Hkv, int N, int d, int hidden, int Hq) {
  if (B <= 0 || Hkv <= 0 || N <= 0 || hidden <= 0 || Hq <= 0 || (d != 64 && d != 128)) return 0;
  return ea::router_ste_workspace_bytes(B, Hkv, N, d, hidden, Hq);
}

ea_status ea_router_ste_backward(const void* k, int B, int Hkv, int N, int d, const float* w1,
                                 const float* b1, int hidden, const float* w2, const float* b2,
                                 int Hq, const float* g0, const float* g1, float tau,
                                 const void* dout, const void* out, const void* out_other,
                                 const uint8_t* route_mask, float* dr_out, float* dw1,
                                 float* db1, float* dw2, float* db2,
                                 float* dk_pool_out, void* dk_accum, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!dout || !out || !out_other || !dw1 || !db1 || !dw2 || !db2) return EA_ERR_INVALID_ARG;
  const ea_status st = check_router_train(k, B, Hkv, N, d, w1, b1, hidden, w2, b2, Hq, g0, g1, tau);
  if (st != EA_OK) return st;
  if (N > kMaxSeqLen || static_cast<long long>(B) * Hkv > 65535) return EA_ERR_UNSUPPORTED;
  if (!aligned16(dout) || !aligned16(out) || !aligned16(out_other)) return EA_ERR_MISALIGNED;
  if (dk_accum && !aligned16(dk_accum)) return EA_ERR_MISALIGNED;
  if (!workspace ||
      workspace_bytes < ea_router_ste_backward_workspace_size(B, Hkv, N, d, hidden, Hq))
    return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  const cudaError_t err = ea::launch_router_ste(
      k, B, Hkv, N, d, w1, b1, hidden, w2, b2, Hq, g0, g1, tau, dout, out, out_other, route_mask,
      dr_out, dw1, db1, dw2, db2, dk_pool_out, dk_accum, workspace,
      static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

// ------------------------------------------------------------------ attention
size_t ea_hybrid_attn_workspace_size(const ea_attn_params* p) {
  return check_params(p) == EA_OK ? kAttnWorkspace : 0;
}

int ea_attn_grid_size(const ea_attn_params* p, int num_sms) {
  if (check_params(p) != EA_OK || num_sms <= 0) return 0;
  const long long units =
      static_cast<long long>(p->B) * p->Hq * ((p->N + EA_UNIT_ROWS - 1) / EA_UNIT_ROWS);
  return static_cast<int>(units < num_sms ? units : num_sms);
}

static ea_status prefill_impl(const void* q, const void* k, const void* v,
                              const uint8_t* route_mask, const ea_attn_params* p, void* out,
                              void* workspace, size_t workspace_bytes,
                              unsigned long long* trace, int trace_max, void* stream,
                              const uint8_t* group_sel = nullptr,
                              const uint8_t* head_sel = nullptr) {
  ea_status st = check_params(p);
  if (st != EA_OK) return st;
  if (!q || !k || !v || !route_mask || !out) return EA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return EA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < kAttnWorkspace) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;

  ea::AttnArgs args = {};
  if (!encode_bhsd(&args.tm_q, q, p->d, p->N, p->B * p->Hq) ||
      !encode_bhsd(&args.tm_k, k, p->d, p->N, p->B * p->Hkv) ||
      !encode_bhsd(&args.tm_v, v, p->d, p->N, p->B * p->Hkv))
    return EA_ERR_CUDA;
  args.mask = route_mask;
  args.out = out;
  args.status = static_cast<int*>(workspace);
  args.cu_seqlens = nullptr;
  args.total = 0;
  args.B = p->B;
  args.Hq = p->Hq;
  args.Hkv = p->Hkv;
  args.N = p->N;
  args.sink = p->sink;
  args.window = p->window;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(static_cast<float>(p->d));
  args.scale_log2 = scale * 1.4426950408889634f;
  args.select = p->select;
  args.timeout_ns = wait_timeout_ns();
  args.debug_drop_kv_pos = debug_drop_kv_pos();
  args.debug_skip_grid_sync = debug_skip_grid_sync();
  args.trace = trace;
  args.trace_max = trace_max;
  args.group_sel = group_sel;
  args.head_sel = head_sel;

  const int sms = device_sms();
  if (sms <= 0) return EA_ERR_CUDA;
  const int grid = ea_attn_grid_size(p, sms);
  cudaError_t err = ea::launch_attn(p->d, args, grid, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

ea_status ea_hybrid_attn_prefill(const void* q, const void* k, const void* v,
                                 const uint8_t* route_mask, const ea_attn_params* p, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return prefill_impl(q, k, v, route_mask, p, out, workspace, workspace_bytes, nullptr, 0,
                      stream);
}

ea_status ea_hybrid_attn_prefill_groups(const void* q, const void* k, const void* v,
                                       const uint8_t* route_mask, const uint8_t* group_sel,
                                       const ea_attn_params* p, void* out, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  if (!group_sel) return EA_ERR_INVALID_ARG;
  return prefill_impl(q, k, v, route_mask, p, out, workspace, workspace_bytes, nullptr, 0, stream,
                      group_sel);
}

ea_status ea_hybrid_attn_prefill_heads(const void* q, const void* k, const void* v,
                                      const uint8_t* route_mask, const uint8_t* head_sel,
                                      const ea_attn_params* p, void* out, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!head_sel) return EA_ERR_INVALID_ARG;
  return prefill_impl(q, k, v, route_mask, p, out, workspace, workspace_bytes, nullptr, 0, stream,
                      nullptr, head_sel);
}

ea_status ea_hybrid_attn_prefill_traced(const void* q, const void* k, const void* v,
                                        const uint8_t* route_mask, const ea_attn_params* p,
                                        void* out, void* workspace, size_t workspace_bytes,
                                        unsigned long long* trace, int trace_records,
                                        void* stream) {
  if (!trace || trace_records < 0) return EA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(trace) & 7u) != 0) return EA_ERR_MISALIGNED;
  return prefill_impl(q, k, v, route_mask, p, out, workspace, workspace_bytes, trace,
                      trace_records, stream);
}

// Forward of a training step (padded BHSD): the chosen mode with its
// log-sum-exp, and, when out_other is given, every head's other mode too, in
// the same launch.
static ea_status prefill_train(const void* q, const void* k, const void* v,
                               const uint8_t* route_mask, const ea_attn_params* p, void* out,
                               float* lse, void* out_other, void* workspace,
                               size_t workspace_bytes, void* stream) {
  ea_status st = check_params(p);
  if (st != EA_OK) return st;
  if (!q || !k || !v || !route_mask || !out || !lse) return EA_ERR_INVALID_ARG;
  if (out_other && p->select != EA_SELECT_ALL) return EA_ERR_INVALID_ARG;
  if (out_other && 2LL * p->B * p->Hq > EA_MAX_ENTRIES) return EA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (out_other && !aligned16(out_other)))
    return EA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < kAttnWorkspace) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  ea::AttnArgs args = {};
  if (!encode_bhsd(&args.tm_q, q, p->d, p->N, p->B * p->Hq) ||
      !encode_bhsd(&args.tm_k, k, p->d, p->N, p->B * p->Hkv) ||
      !encode_bhsd(&args.tm_v, v, p->d, p->N, p->B * p->Hkv))
    return EA_ERR_CUDA;
  args.mask = route_mask;
  args.out = out;
  args.lse = lse;
  args.out_other = out_other;
  args.both = out_other != nullptr;
  args.status = static_cast<int*>(workspace);
  args.B = p->B;
  args.Hq = p->Hq;
  args.Hkv = p->Hkv;
  args.N = p->N;
  args.sink = p->sink;
  args.window = p->window;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(static_cast<float>(p->d));
  args.scale_log2 = scale * 1.4426950408889634f;
  args.select = p->select;
  args.timeout_ns = wait_timeout_ns();
  args.debug_drop_kv_pos = debug_drop_kv_pos();
  args.debug_skip_grid_sync = debug_skip_grid_sync();
  const int sms = device_sms();
  if (sms <= 0) return EA_ERR_CUDA;
  int grid = ea_attn_grid_size(p, sms);
  if (args.both) grid = std::min(sms, 2 * grid);
  cudaError_t err = ea::launch_attn(p->d, args, grid, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

ea_status ea_hybrid_attn_prefill_lse(const void* q, const void* k, const void* v,
                                     const uint8_t* route_mask, const ea_attn_params* p,
                                     void* out, float* lse, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  return prefill_train(q, k, v, route_mask, p, out, lse, nullptr, workspace, workspace_bytes,
                       stream);
}

ea_status ea_hybrid_attn_prefill_train(const void* q, const void* k, const void* v,
                                       const uint8_t* route_mask, const ea_attn_params* p,
                                       void* out, float* lse, void* out_other, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  if (!out_other) return EA_ERR_INVALID_ARG;
  return prefill_train(q, k, v, route_mask, p, out, lse, out_other, workspace, workspace_bytes,
                       stream);
}

// ---------------------------------------------------------------- FP8
int ea_fp8_vt_stride(int N) { return N > 0 ? ea::fp8_npad(N) : 0; }

size_t ea_quantize_fp8_workspace_size(int heads) {
  return heads > 0 ? ea::fp8_quant_workspace_bytes(heads) : 0;
}

ea_status ea_quantize_fp8(const void* x, int heads, int N, int d, int transpose, void* codes,
                          float* scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !codes || !scale || heads <= 0 || N <= 0 || d <= 0) return EA_ERR_INVALID_ARG;
  if (transpose != 0 && transpose != 1) return EA_ERR_INVALID_ARG;
  if (d != 128) return EA_ERR_UNSUPPORTED;
  if (N > kMaxSeqLen || static_cast<long long>(heads) > 65535) return EA_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(codes)) return EA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < ea_quantize_fp8_workspace_size(heads))
    return EA_ERR_WORKSPACE;
  const cudaError_t err = ea::launch_fp8_quant(x, heads, N, d, transpose, codes, scale, workspace,
                                               static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

ea_status ea_hybrid_attn_prefill_fp8(const void* q8, const void* k8, const void* vt8,
                                     const float* q_scale, const float* k_scale,
                                     const float* v_scale, const uint8_t* route_mask,
                                     const ea_attn_params* p, void* out, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  ea_status st = check_params(p);
  if (st != EA_OK) return st;
  if (!q8 || !k8 || !vt8 || !q_scale || !k_scale || !v_scale || !route_mask || !out)
    return EA_ERR_INVALID_ARG;
  if (p->d != 128) return EA_ERR_UNSUPPORTED;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(vt8) || !aligned16(out))
    return EA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < kAttnWorkspace) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  const uint64_t npad = static_cast<uint64_t>(ea::fp8_npad(p->N));
  const uint64_t d = static_cast<uint64_t>(p->d);
  ea::AttnArgs args = {};
  if (!encode_u8(&args.tm_q, q8, p->d, p->N, p->B * p->Hq, d, d * p->N) ||
      !encode_u8(&args.tm_k, k8, p->d, p->N, p->B * p->Hkv, d, d * p->N) ||
      !encode_u8(&args.tm_v, vt8, p->N, p->d, p->B * p->Hkv, npad, npad * d))
    return EA_ERR_CUDA;
  args.mask = route_mask;
  args.out = out;
  args.q_scale = q_scale;
  args.k_scale = k_scale;
  args.v_scale = v_scale;
  args.status = static_cast<int*>(workspace);
  args.B = p->B;
  args.Hq = p->Hq;
  args.Hkv = p->Hkv;
  args.N = p->N;
  args.sink = p->sink;
  args.window = p->window;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(static_cast<float>(p->d));
  args.scale_log2 = scale * 1.4426950408889634f;
  args.select = p->select;
  args.timeout_ns = wait_timeout_ns();
  args.debug_drop_kv_pos = -1;
  args.debug_skip_grid_sync = -1;
  const int sms = device_sms();
  if (sms <= 0) return EA_ERR_CUDA;
  const cudaError_t err = ea::launch_attn_fp8(args, ea_attn_grid_size(p, sms),
                                              static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

// Backward workspace: status block; D [B*Hq*N]; the dK/dV kernel's padded
// vectors -lse*log2e and -D [B*Hq][npad] each; the schedule's unit lists.
size_t bwd_pad_rows(const ea_attn_params* p) {
  return static_cast<size_t>(p->B) * p->Hq * ((p->N + EA_BN - 1) / EA_BN) * EA_BN;
}

size_t ea_hybrid_attn_backward_workspace_size(const ea_attn_params* p) {
  if (check_params(p) != EA_OK || p->d != 128) return 0;
  const size_t rows = static_cast<size_t>(p->B) * p->Hq * p->N;
  return kAttnWorkspace + (rows * sizeof(float) + 255) / 256 * 256 +
         2 * bwd_pad_rows(p) * sizeof(float) +
         ea::bwd_sched_ints(p->B, p->Hq, p->Hkv, p->N) * sizeof(int);
}

ea_status ea_hybrid_attn_backward(const void* q, const void* k, const void* v, const void* out,
                                  const void* dout, const float* lse, const uint8_t* route_mask,
                                  const ea_attn_params* p, void* dq, void* dk, void* dv,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  ea_status st = check_params(p);
  if (st != EA_OK) return st;
  if (p->d != 128 || p->select != EA_SELECT_ALL) return EA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out || !dout || !lse || !route_mask || !dq || !dk || !dv)
    return EA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, out, dout, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return EA_ERR_MISALIGNED;
  const size_t need = ea_hybrid_attn_backward_workspace_size(p);
  if (!workspace || workspace_bytes < need) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  ea::BwdArgs a = {};
  if (!encode_bhsd(&a.tm_q, q, p->d, p->N, p->B * p->Hq) ||
      !encode_bhsd(&a.tm_k, k, p->d, p->N, p->B * p->Hkv) ||
      !encode_bhsd(&a.tm_v, v, p->d, p->N, p->B * p->Hkv) ||
      !encode_bhsd(&a.tm_do, dout, p->d, p->N, p->B * p->Hq))
    return EA_ERR_CUDA;
  float* dvec = reinterpret_cast<float*>(static_cast<char*>(workspace) + kAttnWorkspace);
  const size_t rows = static_cast<size_t>(p->B) * p->Hq * p->N;
  // the padded vectors after D (512-byte aligned: every tile's vector is one
  // aligned bulk copy), then the schedule's unit lists
  float* vl_pad = reinterpret_cast<float*>(static_cast<char*>(workspace) + kAttnWorkspace +
                                           (rows * sizeof(float) + 255) / 256 * 256);
  float* vd_pad = vl_pad + bwd_pad_rows(p);
  {
    int* w = reinterpret_cast<int*>(vd_pad + bwd_pad_rows(p));
    const size_t nT = static_cast<size_t>((p->N + EA_BN - 1) / EA_BN);
    const size_t ukv = static_cast<size_t>(p->B) * p->Hkv * nT;
    const size_t uq = static_cast<size_t>(p->B) * p->Hq * nT;
    a.offs_kv = w;
    a.offs_q = w + (ea::kBwdMaxGrid + 1);
    w += 2 * (ea::kBwdMaxGrid + 1);
    a.list_kv = w;
    a.sorted_kv = w + ukv;
    a.cta_kv = w + 2 * ukv;
    w += 3 * ukv;
    a.list_q = w;
    a.sorted_q = w + uq;
    a.cta_q = w + 2 * uq;
  }
  a.lse = lse;
  a.dvec = dvec;
  a.vl_pad = vl_pad;
  a.vd_pad = vd_pad;
  a.npad = static_cast<int>(((p->N + EA_BN - 1) / EA_BN) * EA_BN);
  a.mask = route_mask;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.status = static_cast<int*>(workspace);
  a.B = p->B;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.N = p->N;
  a.sink = p->sink;
  a.window = p->window;
  a.scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(static_cast<float>(p->d));
  a.scale_log2 = a.scale * 1.4426950408889634f;
  a.timeout_ns = wait_timeout_ns();
  const int sms = device_sms();
  if (sms <= 0) return EA_ERR_CUDA;
  cudaError_t err = ea::launch_backward(a, dout, out, dvec, vl_pad, vd_pad, sms,
                                        static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

ea_status ea_get_device_status(void* workspace, void* stream, int* status_out) {
  if (!workspace || !status_out) return EA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return EA_ERR_CUDA;
  if (cudaMemcpy(&host, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return EA_ERR_CUDA;
  // an error clears the whole 256-byte status block: the status word and the
  // routed launch's grid-barrier words (left mid-phase by a timeout)
  if (host != 0 && cudaMemset(workspace, 0, kAttnWorkspace) != cudaSuccess) return EA_ERR_CUDA;
  *status_out = host;
  return EA_OK;
}

size_t ea_hybrid_attn_varlen_workspace_size(const ea_varlen_params* p) {
  return check_varlen(p) == EA_OK ? kAttnWorkspace : 0;
}

ea_status ea_hybrid_attn_prefill_varlen(const void* q, const void* k, const void* v,
                                        const int32_t* cu_seqlens, const uint8_t* route_mask,
                                        const ea_varlen_params* p, void* out, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  ea_status st = check_varlen(p);
  if (st != EA_OK) return st;
  if (!q || !k || !v || !cu_seqlens || !route_mask || !out) return EA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return EA_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < kAttnWorkspace) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  if (p->total == 0 || p->max_seqlen == 0) return EA_OK;   // no token: nothing to run

  ea::AttnArgs args = {};
  if (!encode_packed(&args.tm_q, q, p->d, p->total, p->Hq) ||
      !encode_packed(&args.tm_k, k, p->d, p->total, p->Hkv) ||
      !encode_packed(&args.tm_v, v, p->d, p->total, p->Hkv))
    return EA_ERR_CUDA;
  args.mask = route_mask;
  args.out = out;
  args.status = static_cast<int*>(workspace);
  args.cu_seqlens = cu_seqlens;
  args.total = p->total;
  args.B = p->B;
  args.Hq = p->Hq;
  args.Hkv = p->Hkv;
  args.N = p->max_seqlen;
  args.sink = p->sink;
  args.window = p->window;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(static_cast<float>(p->d));
  args.scale_log2 = scale * 1.4426950408889634f;
  args.select = p->select;
  args.timeout_ns = wait_timeout_ns();
  args.debug_drop_kv_pos = debug_drop_kv_pos();
  args.debug_skip_grid_sync = debug_skip_grid_sync();

  const int sms = device_sms();
  if (sms <= 0) return EA_ERR_CUDA;
  const long long units = static_cast<long long>(p->B) * p->Hq *
                          ((p->max_seqlen + EA_UNIT_ROWS - 1) / EA_UNIT_ROWS);
  const int grid = static_cast<int>(units < sms ? units : sms);
  cudaError_t err = ea::launch_attn(p->d, args, grid, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

// ------------------------------------------------------------------ routed launches
namespace {

// Router argument checks shared by the routed entry points.
ea_status check_router_args(const void* w1, const void* b1, const void* w2, const void* b2,
                            const uint8_t* mask_out, int Hkv, int d, int hidden, int Hq,
                            float threshold) {
  if (!w1 || !b1 || !w2 || !b2 || !mask_out) return EA_ERR_INVALID_ARG;
  if (hidden <= 0 || threshold != threshold) return EA_ERR_INVALID_ARG;
  if (Hkv * d > 8192 || hidden > kRouterMaxHidden || Hq > 1024) return EA_ERR_UNSUPPORTED;
  if ((Hkv * d) % 4 != 0 || hidden % 4 != 0) return EA_ERR_UNSUPPORTED;
  if (!aligned16(w1) || !aligned16(w2)) return EA_ERR_MISALIGNED;
  return EA_OK;
}

// Router fields of a routed launch; scratch after the 256-byte status block,
// grid-barrier words inside it.
void set_router_args(ea::AttnArgs& a, const void* k, const float* w1, const float* b1,
                     int hidden, const float* w2, const float* b2, float threshold,
                     uint8_t* mask_out, float* logits, void* workspace, int nsplit) {
  a.k_raw = k;
  a.w1 = w1;
  a.b1 = b1;
  a.w2 = w2;
  a.b2 = b2;
  a.hidden = hidden;
  a.threshold = threshold;
  a.mask_out = mask_out;
  a.mask = mask_out;
  a.logits = logits;
  a.nsplit = nsplit;
  char* ws = static_cast<char*>(workspace);
  a.bar_count = reinterpret_cast<unsigned int*>(ws + 64);
  a.bar_gen = reinterpret_cast<unsigned int*>(ws + 128);
  a.partials = reinterpret_cast<float*>(ws + kAttnWorkspace);
}

}  // namespace

size_t ea_hybrid_attn_routed_workspace_size(const ea_attn_params* p, int hidden) {
  if (check_params(p) != EA_OK || hidden <= 0 || hidden > kRouterMaxHidden) return 0;
  return kAttnWorkspace + ea::router_workspace_bytes(p->B, p->Hkv, p->N, p->d, hidden);
}

ea_status ea_hybrid_attn_prefill_routed(const void* q, const void* k, const void* v,
                                        const float* w1, const float* b1, int hidden,
                                        const float* w2, const float* b2, float threshold,
                                        uint8_t* route_mask, float* logits_out,
                                        const ea_attn_params* p, void* out, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  ea_status st = check_params(p);
  if (st != EA_OK) return st;
  if (!q || !k || !v || !out) return EA_ERR_INVALID_ARG;
  st = check_router_args(w1, b1, w2, b2, route_mask, p->Hkv, p->d, hidden, p->Hq, threshold);
  if (st != EA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return EA_ERR_MISALIGNED;
  const size_t need = ea_hybrid_attn_routed_workspace_size(p, hidden);
  if (!workspace || workspace_bytes < need) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;

  ea::AttnArgs args = {};
  if (!encode_bhsd(&args.tm_q, q, p->d, p->N, p->B * p->Hq) ||
      !encode_bhsd(&args.tm_k, k, p->d, p->N, p->B * p->Hkv) ||
      !encode_bhsd(&args.tm_v, v, p->d, p->N, p->B * p->Hkv))
    return EA_ERR_CUDA;
  args.out = out;
  args.status = static_cast<int*>(workspace);
  args.cu_seqlens = nullptr;
  args.total = 0;
  args.B = p->B;
  args.Hq = p->Hq;
  args.Hkv = p->Hkv;
  args.N = p->N;
  args.sink = p->sink;
  args.window = p->window;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(static_cast<float>(p->d));
  args.scale_log2 = scale * 1.4426950408889634f;
  args.select = p->select;
  args.timeout_ns = wait_timeout_ns();
  args.debug_drop_kv_pos = debug_drop_kv_pos();
  args.debug_skip_grid_sync = debug_skip_grid_sync();
  set_router_args(args, k, w1, b1, hidden, w2, b2, threshold, route_mask, logits_out, workspace,
                  ea::router_num_splits(p->B, p->Hkv, p->N));
  const int sms = device_sms();
  if (sms <= 0) return EA_ERR_CUDA;
  cudaError_t err = ea::launch_attn_routed(p->d, args, sms, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

size_t ea_hybrid_attn_varlen_routed_workspace_size(const ea_varlen_params* p, int hidden) {
  if (check_varlen(p) != EA_OK || hidden <= 0 || hidden > kRouterMaxHidden) return 0;
  return kAttnWorkspace +
         ea::router_workspace_bytes(p->B, p->Hkv, p->max_seqlen > 0 ? p->max_seqlen : 1, p->d,
                                    hidden);
}

ea_status ea_hybrid_attn_prefill_varlen_routed(const void* q, const void* k, const void* v,
                                               const int32_t* cu_seqlens, const float* w1,
                                               const float* b1, int hidden, const float* w2,
                                               const float* b2, float threshold,
                                               uint8_t* route_mask, float* logits_out,
                                               const ea_varlen_params* p, void* out,
                                               void* workspace, size_t workspace_bytes,
                                               void* stream) {
  ea_status st = check_varlen(p);
  if (st != EA_OK) return st;
  if (!q || !k || !v || !cu_seqlens || !out) return EA_ERR_INVALID_ARG;
  st = check_router_args(w1, b1, w2, b2, route_mask, p->Hkv, p->d, hidden, p->Hq, threshold);
  if (st != EA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return EA_ERR_MISALIGNED;
  const size_t need = ea_hybrid_attn_varlen_routed_workspace_size(p, hidden);
  if (!workspace || workspace_bytes < need) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;
  if (p->total == 0) return EA_ERR_UNSUPPORTED;   // the tensor maps need a token

  ea::AttnArgs args = {};
  if (!encode_packed(&args.tm_q, q, p->d, p->total, p->Hq) ||
      !encode_packed(&args.tm_k, k, p->d, p->total, p->Hkv) ||
      !encode_packed(&args.tm_v, v, p->d, p->total, p->Hkv))
    return EA_ERR_CUDA;
  args.out = out;
  args.status = static_cast<int*>(workspace);
  args.cu_seqlens = cu_seqlens;
  args.total = p->total;
  args.B = p->B;
  args.Hq = p->Hq;
  args.Hkv = p->Hkv;
  args.N = p->max_seqlen;
  args.sink = p->sink;
  args.window = p->window;
  const float scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(static_cast<float>(p->d));
  args.scale_log2 = scale * 1.4426950408889634f;
  args.select = p->select;
  args.timeout_ns = wait_timeout_ns();
  args.debug_drop_kv_pos = debug_drop_kv_pos();
  args.debug_skip_grid_sync = debug_skip_grid_sync();
  set_router_args(args, k, w1, b1, hidden, w2, b2, threshold, route_mask, logits_out, workspace,
                  ea::router_num_splits(p->B, p->Hkv, p->max_seqlen > 0 ? p->max_seqlen : 1));
  const int sms = device_sms();
  if (sms <= 0) return EA_ERR_CUDA;
  cudaError_t err = ea::launch_attn_routed(p->d, args, sms, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? EA_OK : EA_ERR_CUDA;
}

// ------------------------------------------------------------------ schedule view
int ea_schedule_units(const uint8_t* mask, const ea_attn_params* p, int32_t* units_out,
                      int max_units) {
  if (!mask || check_params(p) != EA_OK) return -1;
  std::vector<int> lens(p->B, p->N);
  HostSched h;
  build_host_sched(mask, p->B, p->Hq, p->Hkv, p->select, lens.data(), p->sink, p->window, h);
  return list_units(h, p->Hq, p->Hkv, p->d, p->sink, p->window, units_out, max_units);
}

int ea_schedule_units_varlen(const uint8_t* mask, const ea_varlen_params* p,
                             const int32_t* cu_seqlens_host, int32_t* units_out, int max_units) {
  if (!mask || !cu_seqlens_host || check_varlen(p) != EA_OK) return -1;
  if (cu_seqlens_host[0] != 0 || cu_seqlens_host[p->B] != p->total) return -1;
  std::vector<int> lens(p->B);
  for (int b = 0; b < p->B; ++b) {
    lens[b] = cu_seqlens_host[b + 1] - cu_seqlens_host[b];
    if (lens[b] < 0) return -1;
  }
  HostSched h;
  build_host_sched(mask, p->B, p->Hq, p->Hkv, p->select, lens.data(), p->sink, p->window, h);
  return list_units(h, p->Hq, p->Hkv, p->d, p->sink, p->window, units_out, max_units);
}

int ea_schedule_unit_tiles(const uint8_t* mask, const ea_attn_params* p, int rank,
                           int32_t* tiles_out, int32_t* codes_out, int max_tiles) {
  if (!mask || check_params(p) != EA_OK) return -1;
  std::vector<int> lens(p->B, p->N);
  HostSched h;
  build_host_sched(mask, p->B, p->Hq, p->Hkv, p->select, lens.data(), p->sink, p->window, h);
  const int total = ea_total_units(h.view);
  if (rank < 0 || rank >= total) return -1;
  EaCursor cur;
  ea_cursor_init(cur, h.view, h.ent.data(), p->Hq, p->Hkv, ea_group_major(h.view.Pmax, p->d));
  EaUnitRef u;
  if (!ea_cursor_seek(cur, h.view, h.ent.data(), rank, &u)) return -1;
  const EaShape sh = ea_make_shape(p->N, p->sink, p->window);
  const EaUnitTiles ut = ea_unit_tiles(sh, u.sparse, u.paired, u.level);
  for (int i = 0; i < ut.n && i < max_tiles; ++i) {
    const int t = ea_tile_at(ut, i);
    if (tiles_out) tiles_out[i] = t;
    if (codes_out) {
      codes_out[2 * i] = ea_tile_code(sh, ut, u.sparse, 0, t);
      codes_out[2 * i + 1] = ea_tile_code(sh, ut, u.sparse, 1, t);
    }
  }
  return ut.n;
}


// ------------------------------------------------------------------ host buffers
namespace {

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Device workspace of ea_hybrid_attn_prefill_host: the attention status block,
// then the route mask, the router's scratch and device copies of q, k, v, out.
struct HostLayout {
  size_t mask, router, q, k, v, out, total;
  size_t q_bytes, kv_bytes;
};

HostLayout host_layout(const ea_attn_params* p, int hidden) {
  HostLayout L;
  const size_t head = static_cast<size_t>(p->N) * p->d * 2;
  L.q_bytes = head * p->B * p->Hq;
  L.kv_bytes = head * p->B * p->Hkv;
  size_t off = kAttnWorkspace;
  L.mask = off;
  off += up256(static_cast<size_t>(p->B) * p->Hq);
  L.router = off;
  if (hidden > 0) off += up256(ea::router_workspace_bytes(p->B, p->Hkv, p->N, p->d, kRouterMaxHidden));
  L.q = off;
  off += up256(L.q_bytes);
  L.k = off;
  off += up256(L.kv_bytes);
  L.v = off;
  off += up256(L.kv_bytes);
  L.out = off;
  off += up256(L.q_bytes);
  L.total = off;
  return L;
}

// Kv heads per chunk: the caller's choice, or about eight chunks in all.
int host_chunk(const ea_attn_params* p, int kv_heads_per_chunk) {
  int c = kv_heads_per_chunk;
  if (c <= 0) c = (p->B * p->Hkv + 7) / 8;
  return std::max(1, std::min(c, p->Hkv));
}

// The two copy streams (upload, download) of each device, created
// non-blocking on first use and kept until ea_shutdown or the process exits.
cudaStream_t g_up[ea::kMaxSmDevices] = {};
cudaStream_t g_down[ea::kMaxSmDevices] = {};
std::mutex g_stream_mu;

bool host_copy_streams(cudaStream_t* up, cudaStream_t* down) {
  cudaStream_t* s_up = g_up;
  cudaStream_t* s_down = g_down;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= ea::kMaxSmDevices) return false;
  std::lock_guard<std::mutex> lock(g_stream_mu);
  if (!s_up[dev]) {
    cudaStream_t a = nullptr, b = nullptr;
    if (cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking) != cudaSuccess) return false;
    if (cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking) != cudaSuccess) {
      cudaStreamDestroy(a);
      return false;
    }
    s_up[dev] = a;
    s_down[dev] = b;
  }
  *up = s_up[dev];
  *down = s_down[dev];
  return true;
}

// Events of one call, destroyed when the call returns (a recorded event may
// be destroyed before it completes; its resources are released afterwards).
struct CallEvents {
  std::vector<cudaEvent_t> ev;
  ~CallEvents() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
  }
  cudaEvent_t make() {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    ev.push_back(e);
    return e;
  }
};

}  // namespace

ea_status ea_shutdown(void) {
  ea::router_noalloc_forget();
  std::lock_guard<std::mutex> lock(g_stream_mu);
  int cur = -1;
  bool any = false;
  ea_status st = EA_OK;
  for (int dev = 0; dev < ea::kMaxSmDevices; ++dev) {
    if (!g_up[dev]) continue;
    if (!any) {
      if (cudaGetDevice(&cur) != cudaSuccess) return EA_ERR_CUDA;
      any = true;
    }
    // a stream's work finishes before it is destroyed
    if (cudaSetDevice(dev) != cudaSuccess || cudaStreamSynchronize(g_up[dev]) != cudaSuccess ||
        cudaStreamSynchronize(g_down[dev]) != cudaSuccess ||
        cudaStreamDestroy(g_up[dev]) != cudaSuccess ||
        cudaStreamDestroy(g_down[dev]) != cudaSuccess)
      st = EA_ERR_CUDA;
    g_up[dev] = nullptr;
    g_down[dev] = nullptr;
  }
  if (any && cudaSetDevice(cur) != cudaSuccess) st = EA_ERR_CUDA;
  return st;
}

size_t ea_hybrid_attn_host_workspace_size(const ea_attn_params* p, int hidden) {
  if (check_params(p) != EA_OK || hidden < 0 || hidden > kRouterMaxHidden) return 0;
  return host_layout(p, hidden).total;
}

int ea_hybrid_attn_host_chunks(const ea_attn_params* p, int kv_heads_per_chunk) {
  if (check_params(p) != EA_OK || kv_heads_per_chunk < 0) return 0;
  const int c = host_chunk(p, kv_heads_per_chunk);
  return p->B * ((p->Hkv + c - 1) / c);
}

ea_status ea_hybrid_attn_prefill_host(const void* q_host, const void* k_host,
                                      const void* v_host, const uint8_t* route_mask_host,
                                      const float* w1, const float* b1, int hidden,
                                      const float* w2, const float* b2, float threshold,
                                      const ea_attn_params* p, void* out_host,
                                      uint8_t* route_mask_out_host, int kv_heads_per_chunk,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  ea_status st = check_params(p);
  if (st != EA_OK) return st;
  if (!q_host || !k_host || !v_host || !out_host || kv_heads_per_chunk < 0)
    return EA_ERR_INVALID_ARG;
  if (p->select != EA_SELECT_ALL) return EA_ERR_INVALID_ARG;
  const bool routed = w1 != nullptr;
  if (!routed && !route_mask_host) return EA_ERR_INVALID_ARG;
  if (!workspace) return EA_ERR_WORKSPACE;
  const HostLayout L = host_layout(p, routed ? 1 : 0);
  char* ws = static_cast<char*>(workspace);
  uint8_t* dmask = reinterpret_cast<uint8_t*>(ws + L.mask);
  if (routed) {
    st = check_router_args(w1, b1, w2, b2, dmask, p->Hkv, p->d, hidden, p->Hq, threshold);
    if (st != EA_OK) return st;
  }
  if (workspace_bytes < L.total) return EA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return EA_ERR_MISALIGNED;

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaStream_t up = nullptr, down = nullptr;
  if (!host_copy_streams(&up, &down)) return EA_ERR_CUDA;
  char* dq = ws + L.q;
  char* dk = ws + L.k;
  char* dv = ws + L.v;
  char* dout = ws + L.out;
  const char* hq = static_cast<const char*>(q_host);
  const char* hv = static_cast<const char*>(v_host);
  char* hout = static_cast<char*>(out_host);
  const size_t head = static_cast<size_t>(p->N) * p->d * 2;
  const int G = p->Hq / p->Hkv;
  const int c = host_chunk(p, kv_heads_per_chunk);
  const size_t mask_bytes = static_cast<size_t>(p->B) * p->Hq;

  CallEvents E;
  cudaEvent_t ev_start = E.make(), ev_k = E.make();
  if (!ev_start || !ev_k) return EA_ERR_CUDA;
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  // The copies start after the work already on the caller's stream (the
  // device buffers may still be read by an earlier call).
  if (!ok(cudaEventRecord(ev_start, cs)) || !ok(cudaStreamWaitEvent(up, ev_start, 0)) ||
      !ok(cudaStreamWaitEvent(down, ev_start, 0)))
    return EA_ERR_CUDA;
  // k (all of it: the router pools every kv head) and the caller's mask first.
  if (!ok(cudaMemcpyAsync(dk, k_host, L.kv_bytes, cudaMemcpyHostToDevice, up))) return EA_ERR_CUDA;
  if (!routed &&
      !ok(cudaMemcpyAsync(dmask, route_mask_host, mask_bytes, cudaMemcpyHostToDevice, up)))
    return EA_ERR_CUDA;
  if (!ok(cudaEventRecord(ev_k, up)) || !ok(cudaStreamWaitEvent(cs, ev_k, 0))) return EA_ERR_CUDA;
  if (routed) {
    st = ea_router_decide(dk, p->B, p->Hkv, p->N, p->d, w1, b1, hidden, w2, b2, p->Hq,
                          threshold, dmask, nullptr, ws + L.router, L.q - L.router, cs);
    if (st != EA_OK) return st;
  }
  if (route_mask_out_host) {
    cudaEvent_t ev_mask = E.make();
    if (!ev_mask || !ok(cudaEventRecord(ev_mask, cs)) || !ok(cudaStreamWaitEvent(down, ev_mask, 0)) ||
        !ok(cudaMemcpyAsync(route_mask_out_host, dmask, mask_bytes, cudaMemcpyDeviceToHost, down)))
      return EA_ERR_CUDA;
  }
  // Chunks of c kv heads (and their G*c query heads) of one batch element:
  // upload q and v, attend, download out.
  for (int b = 0; b < p->B; ++b) {
    for (int g0 = 0; g0 < p->Hkv; g0 += c) {
      const int gc = std::min(c, p->Hkv - g0);
      const size_t qoff = (static_cast<size_t>(b) * p->Hq + static_cast<size_t>(g0) * G) * head;
      const size_t kvoff = (static_cast<size_t>(b) * p->Hkv + g0) * head;
      const size_t qlen = static_cast<size_t>(gc) * G * head;
      const size_t kvlen = static_cast<size_t>(gc) * head;
      cudaEvent_t ev_in = E.make(), ev_done = E.make();
      if (!ev_in || !ev_done) return EA_ERR_CUDA;
      if (!ok(cudaMemcpyAsync(dq + qoff, hq + qoff, qlen, cudaMemcpyHostToDevice, up)) ||
          !ok(cudaMemcpyAsync(dv + kvoff, hv + kvoff, kvlen, cudaMemcpyHostToDevice, up)) ||
          !ok(cudaEventRecord(ev_in, up)) || !ok(cudaStreamWaitEvent(cs, ev_in, 0)))
        return EA_ERR_CUDA;
      ea_attn_params sub = *p;
      sub.B = 1;
      sub.Hq = gc * G;
      sub.Hkv = gc;
      st = ea_hybrid_attn_prefill(dq + qoff, dk + kvoff, dv + kvoff,
                                  dmask + static_cast<size_t>(b) * p->Hq + g0 * G, &sub,
                                  dout + qoff, workspace, kAttnWorkspace, cs);
      if (st != EA_OK) return st;
      if (!ok(cudaEventRecord(ev_done, cs)) || !ok(cudaStreamWaitEvent(down, ev_done, 0)) ||
          !ok(cudaMemcpyAsync(hout + qoff, dout + qoff, qlen, cudaMemcpyDeviceToHost, down)))
        return EA_ERR_CUDA;
    }
  }
  // Work enqueued on the caller's stream later runs after the last download.
  cudaEvent_t ev_end = E.make();
  if (!ev_end || !ok(cudaEventRecord(ev_end, down)) || !ok(cudaStreamWaitEvent(cs, ev_end, 0)))
    return EA_ERR_CUDA;
  return EA_OK;
}

}  // extern "C"
