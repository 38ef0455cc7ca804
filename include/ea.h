/*
 * ea.h — C ABI of the Elastic Attention prefill library (libea.so), sm_100a.
 *
 * The method (Elastic Attention blog, bxzpzcl.cn, §2.1 "Attention Router" and
 * §3 "Fused Kernel"): a light router reads the layer's key states and emits,
 * for every head, a routing bit r; r = 0 sends the head to Full Attention
 * (causal softmax attention over all earlier tokens), r = 1 to Sparse
 * Attention (here: S sink tokens plus a causal local window of W tokens).
 * The routing bits are passed to one fused kernel as metadata, and that one
 * launch computes the FA heads and the SA heads together.
 *
 * Conventions shared by every entry point
 *  - Tensors are dense, contiguous, row-major, in BHSD order:
 *      q, out : bf16 [B][Hq][N][d]      k, v : bf16 [B][Hkv][N][d]
 *    Query head h reads kv head h / (Hq / Hkv).
 *  - Every data pointer is a DEVICE pointer owned by the caller (the
 *    *_host arguments of ea_hybrid_attn_prefill_host are the exception); the
 *    library never allocates, frees or keeps device memory of its own.
 *    Parameter structs are HOST pointers, read before the call returns.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *    enqueued on it; no entry point synchronises except ea_get_device_status.
 *  - Argument errors are returned synchronously, before anything is
 *    enqueued.  Launch failures return EA_ERR_CUDA.  A device-side wait that
 *    runs out (EA_ERR_TIMEOUT) is recorded in a device status word and read
 *    back with ea_get_device_status.
 *  - Calls on different streams may run concurrently as long as each has its
 *    own workspace and output buffers.
 *  - ea_router_decide, ea_hybrid_attn_prefill and ea_hybrid_attn_decode may
 *    be captured into a CUDA graph once each has run eagerly on the device
 *    (the first call sets the kernels' shared-memory attributes); replays
 *    read the captured buffers' current contents.
 */
#ifndef EA_H_
#define EA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ea_status {
  EA_OK = 0,
  EA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, bad enum   */
  EA_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels handle   */
  EA_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned            */
  EA_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed           */
  EA_ERR_TIMEOUT = 5,       /* a device-side wait ran out (see status)     */
  EA_ERR_WORKSPACE = 6,     /* workspace missing or smaller than required  */
  EA_ERR_SCRATCH_LIMIT = 7  /* too large for ea_router_decide_noalloc's
                               fixed scratch (EA_ROUTER_NOALLOC_MAX_BYTES)  */
} ea_status;

/* Which heads one attention call computes.  EA_SELECT_ALL is the fused
 * single launch; EA_SELECT_FA / EA_SELECT_SA compute only the heads routed
 * to that mode (two such calls form the split "serial dispatch" pass that
 * the Elastic Attention blog, §3, contrasts with the fused kernel). */
typedef enum ea_select {
  EA_SELECT_ALL = 0,
  EA_SELECT_FA = 1,
  EA_SELECT_SA = 2
} ea_select;

/* Static string for a status code (never NULL). */
const char* ea_status_string(int status);

/* Library ABI version, (major << 16) | minor. */
int ea_version(void);

/* ------------------------------------------------------------------------
 * Attention Router (Elastic Attention blog §2.1: the router takes the key
 * hidden states and a simple MLP emits one routing signal per head; r = 0 is
 * Full Attention, r = 1 is Sparse Attention; §2.2: 0.27M parameters per
 * layer for an 8B model = 1024 -> 256 -> 32 with biases).
 *
 *   x[b]          = (1/N) * sum_n K[b, :, n, :]   flattened (kv_head, channel)
 *   h             = ReLU(W1 x + b1)              W1: [hidden][Hkv*d], b1: [hidden]
 *   z[b, :]       = W2 h + b2                    W2: [Hq][hidden],    b2: [Hq]
 *   route_mask[b, j] = (z[b, j] > threshold) ? 1 : 0     (a tie routes to FA)
 *
 * k          : device bf16 [B][Hkv][N][d].
 * w1,b1,w2,b2: device fp32, row-major (out x in), 16-byte aligned;
 *              Hkv*d and hidden must be multiples of 4.
 * route_mask : device uint8 [B][Hq], written (1 = sparse, 0 = full).
 * logits_out : device fp32 [B][Hq] or NULL; receives z when non-NULL.
 * workspace  : device scratch of at least ea_router_workspace_size(...)
 *              bytes (pooled partial sums, the pooled vector and the hidden
 *              activations), 16-byte aligned; its contents need no
 *              initialisation and are overwritten.
 * Limits: d in {64, 128}; Hkv*d <= 8192; hidden <= 4096; Hq <= 1024.
 * Pooling sums in fp32 in a fixed order (bit-reproducible run to run).
 * ---------------------------------------------------------------------- */
size_t ea_router_workspace_size(int B, int Hkv, int N, int d);

ea_status ea_router_decide(const void* k, int B, int Hkv, int N, int d,
                           const float* w1, const float* b1, int hidden,
                           const float* w2, const float* b2, int Hq,
                           float threshold, uint8_t* route_mask,
                           float* logits_out, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Router of a packed variable-length batch: the same pooling, MLP and
 * threshold, where sequence b's router input is the mean of ITS OWN key rows
 * (the method routes per input, EA blog §2.1).
 * k          : device bf16 [total][Hkv][d], 16-byte aligned.
 * cu_seqlens : device int32 [B+1] (as for ea_hybrid_attn_prefill_varlen).
 *              An empty sequence pools to zero (its routing comes from the
 *              biases alone); a sequence whose range is not inside [0, total]
 *              pools nothing (zero) and is never read.
 * max_seqlen : host bound of every length (sizes the workspace and split).
 * workspace  : >= ea_router_varlen_workspace_size(B, Hkv, max_seqlen, d).
 * Other arguments, limits and determinism as for ea_router_decide. */
size_t ea_router_varlen_workspace_size(int B, int Hkv, int max_seqlen, int d);

ea_status ea_router_decide_varlen(const void* k, const int32_t* cu_seqlens, int B, int Hkv,
                                  int total, int max_seqlen, int d, const float* w1,
                                  const float* b1, int hidden, const float* w2,
                                  const float* b2, int Hq, float threshold,
                                  uint8_t* route_mask, float* logits_out, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * ea_router_decide without a caller-supplied workspace.
 *
 * The pages have no counterpart: this entry point exists for callers that
 * cannot allocate device memory at the point they route a layer — code that
 * runs inside a host framework which owns all device memory and forbids its
 * plug-ins to call cudaMalloc, or a serving loop that must not allocate
 * after warm-up because cudaMalloc/cudaFree can synchronise the device and
 * take the allocator's locks.
 *
 * Same inputs, outputs and result bits as ea_router_decide.  The pooling
 * scratch lives in a fixed device array inside libea.so, of
 * EA_ROUTER_NOALLOC_MAX_BYTES bytes, which every GPU that loads the library
 * keeps until the process exits.  A problem whose scratch need,
 * ea_router_workspace_size(B, Hkv, N, d), exceeds that size is rejected with
 * EA_ERR_SCRATCH_LIMIT before anything is enqueued.
 *
 * Arguments are checked exactly as ea_router_decide checks them, with the
 * same codes; only then is the scratch need compared with the limit.  The
 * scratch used is the CURRENT device's copy of the array, so k, the weights,
 * route_mask and logits_out must be device memory of the current device
 * (EA_ERR_INVALID_ARG otherwise), and `stream` must belong to that device.
 *
 * The first call on a device looks up that device's copy of the array (a
 * runtime symbol query, no allocation), so make the first call on each
 * device before any stream capture.  The entry point never calls cudaMalloc,
 * cudaFree or any allocating routine.  A device reset invalidates the
 * looked-up address: call ea_shutdown before resetting a device.
 *
 * All calls on one device share the array: two calls whose work overlaps on
 * the GPU (different streams, no ordering between them) race on it and give
 * undefined results.  A CUDA graph captured from this call uses the same
 * array, so its replays must be ordered with each other, with the replays of
 * any other such graph and with eager calls, in the same way.  Calls ordered
 * on one stream are safe; each call overwrites every scratch value it reads,
 * so stale contents never matter.
 * ---------------------------------------------------------------------- */
#define EA_ROUTER_NOALLOC_MAX_BYTES (1u << 20)

ea_status ea_router_decide_noalloc(const void* k, int B, int Hkv, int N, int d,
                                   const float* w1, const float* b1, int hidden,
                                   const float* w2, const float* b2, int Hq,
                                   float threshold, uint8_t* route_mask,
                                   float* logits_out, void* stream);

/* ------------------------------------------------------------------------
 * Fused hybrid prefill attention (Elastic Attention blog §3: the routing
 * decision enters the kernel as metadata and one launch serves the FA heads
 * and the SA heads together; §2.1 "结果融合": each head's result lands in
 * its own slot of the output, which is the concatenation).
 *
 * For each (b, h) with r = route_mask[b*Hq + h] and kv head hk = h / (Hq/Hkv):
 *   visible(i, j) = j <= i                                  if r == 0 (FA)
 *                 = j <= i && (j < sink || i - j < window)  if r == 1 (SA)
 *   out[b,h,i,:] = sum_j softmax_j(scale * q[b,h,i,:].k[b,hk,j,:] | visible) v[b,hk,j,:]
 * with scale = softmax_scale > 0 ? softmax_scale : 1/sqrt(d).
 * Square causal prefill: query i and key i are the same position.
 *
 * Arithmetic: bf16 operands on the tensor cores, fp32 scores, fp32 online
 * softmax, P rounded to bf16 for the P.V product, fp32 accumulation, output
 * rounded to bf16 (round to nearest even).
 * ---------------------------------------------------------------------- */
typedef struct ea_attn_params {
  int B, Hq, Hkv, N, d;
  int sink;              /* S >= 0 sink tokens seen by SA heads             */
  int window;            /* W >= 1, the local window including the diagonal */
  float softmax_scale;   /* <= 0 selects 1/sqrt(d)                          */
  int select;            /* ea_select                                       */
} ea_attn_params;

/* Bytes of workspace ea_hybrid_attn_prefill needs (a status word and the
 * schedule's scratch); 0 if p is invalid. */
size_t ea_hybrid_attn_workspace_size(const ea_attn_params* p);

/* q, k, v   : device bf16, BHSD as above, 16-byte aligned.
 * route_mask: device uint8 [B][Hq], 0 = FA, 1 = SA (any nonzero is SA).
 * p         : host pointer.
 * out       : device bf16 [B][Hq][N][d]; rows of heads not selected by
 *             p->select are left untouched.
 * workspace : device, >= ea_hybrid_attn_workspace_size(p) bytes, ZEROED
 *             once before its first use.  Its first 256 bytes are the status
 *             block: the kernel writes a nonzero error code into its status
 *             word, and keeps its dispatch counters (CTAs take work units
 *             from a global counter) at bytes 192-231, back at zero when the
 *             launch ends.  ea_get_device_status reads the status word and,
 *             after an error, clears the whole block.  Launches that may
 *             run at the same time need separate workspaces.
 * Limits: d in {64, 128}; Hq % Hkv == 0; B <= 1024; B*Hq <= 4096;
 * N <= 32767 * 256.
 */
ea_status ea_hybrid_attn_prefill(const void* q, const void* k, const void* v,
                                 const uint8_t* route_mask,
                                 const ea_attn_params* p, void* out,
                                 void* workspace, size_t workspace_bytes,
                                 void* stream);

/* ------------------------------------------------------------------------
 * Head-sharded multi-GPU prefill (one process per GPU).  The path splits
 * into independent (batch, kv group) problems, so the work is sharded over
 * (b, kv head) pairs; the only exchange is the router's pooled vector, which
 * needs the keys of every kv head of a batch row (Elastic Attention blog
 * §2.1: the router reads the layer's Key hidden states).  Per layer, on
 * every rank:
 *   1. ea_router_pool_rows pools the rank's rows of the flattened (b, kv
 *      head) index into its slice of x;
 *   2. the caller all-gathers the slices (NCCL) into x [B][Hkv*d];
 *   3. ea_router_mlp runs the router's MLP and threshold on x (every rank
 *      gets the same mask);
 *   4. ea_hybrid_attn_prefill_groups computes the (b, kv head) groups the
 *      rank was assigned (a balanced assignment by the mask's per-group
 *      cost), writing only those heads' output rows.
 * Steps 1 + 3 give the bits of ea_router_decide, and step 4 over the union
 * of the ranks' groups the bits of ea_hybrid_attn_prefill.
 * ---------------------------------------------------------------------- */

/* Pools the key rows of flattened (b, kv head) indices [row0, row0 + nrows)
 * of a padded K (device bf16 [B][Hkv][N][d], 16-byte aligned), row r being
 * (b = r / Hkv, hk = r % Hkv): x_out (device fp32 [nrows][d]) receives
 * mean over n of K[b][hk][n][:], with the pooling kernels and split count
 * ea_router_decide uses for the whole [B][Hkv] problem, so every value has
 * its bits.  workspace: >= ea_router_workspace_size(B, Hkv, N, d) bytes.
 * Errors: EA_ERR_INVALID_ARG for NULL pointers or a row range outside
 * [0, B*Hkv); otherwise as ea_router_decide.  nrows = 0 enqueues nothing. */
ea_status ea_router_pool_rows(const void* k, int B, int Hkv, int N, int d, int row0, int nrows,
                             float* x_out, void* workspace, size_t workspace_bytes,
                             void* stream);

/* Bytes of workspace ea_router_mlp needs (B * hidden fp32); 0 if invalid. */
size_t ea_router_mlp_workspace_size(int B, int hidden);

/* The router's MLP and decision on a pooled x (device fp32 [B][in_dim],
 * in_dim = Hkv * d, 16-byte aligned): z = W2 ReLU(W1 x + b1) + b2 and
 * route_mask = z > threshold, with the kernels of ea_router_decide (same
 * bits for the same x).  Weights, outputs and limits as ea_router_decide. */
ea_status ea_router_mlp(const float* x, int B, int in_dim, const float* w1, const float* b1,
                        int hidden, const float* w2, const float* b2, int Hq, float threshold,
                        uint8_t* route_mask, float* logits_out, void* workspace,
                        size_t workspace_bytes, void* stream);

/* ea_hybrid_attn_prefill restricted to a shard: group_sel (device uint8
 * [B][Hkv], required) marks the (b, kv head) groups whose query heads run;
 * the output rows of the other heads are left untouched.  Each head's rows
 * have the bits the unrestricted call gives them.  Other arguments, limits
 * and errors as ea_hybrid_attn_prefill (NULL group_sel: EA_ERR_INVALID_ARG). */
ea_status ea_hybrid_attn_prefill_groups(const void* q, const void* k, const void* v,
                                        const uint8_t* route_mask, const uint8_t* group_sel,
                                        const ea_attn_params* p, void* out, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* The same restricted by query head: head_sel (device uint8 [B][Hq]) is
 * nonzero where head (b, h) runs.  For a shard that splits a kv group whose
 * heads cost more than a rank's share: the ranks holding its heads each read
 * the group's K and V.  Each head's rows have the bits of the unrestricted
 * call; the other heads' rows are left untouched.  NULL head_sel:
 * EA_ERR_INVALID_ARG; otherwise as ea_hybrid_attn_prefill. */
ea_status ea_hybrid_attn_prefill_heads(const void* q, const void* k, const void* v,
                                       const uint8_t* route_mask, const uint8_t* head_sel,
                                       const ea_attn_params* p, void* out, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the device status word kept
 * in `workspace` (an attention workspace).  *status_out receives EA_OK or
 * the error a kernel recorded (EA_ERR_TIMEOUT when a bounded device wait ran
 * out).  Returns EA_ERR_CUDA if the synchronisation or the copy fails. */
ea_status ea_get_device_status(void* workspace, void* stream, int* status_out);

/* Forward for training: ea_hybrid_attn_prefill plus the natural log-sum-exp
 * of every row, lse (device fp32 [B][Hq][N]) = log sum_j exp(scale q_i.k_j)
 * over the row's visible keys; the backward reads it. */
ea_status ea_hybrid_attn_prefill_lse(const void* q, const void* k, const void* v,
                                     const uint8_t* route_mask, const ea_attn_params* p,
                                     void* out, float* lse, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* ea_hybrid_attn_prefill with a per-unit trace, for load-balance
 * measurements (the results are those of the untraced call, bit for bit).
 * It launches a kernel instantiation of its own, the untraced kernel plus the
 * trace stores, so ea_hybrid_attn_prefill carries none of that code.
 * trace: device
 * uint64 [8 + 6 * trace_records], 8-byte aligned, ZEROED by the caller before
 * the call.  trace[0] receives the number of work units the launch ran; the
 * first trace_records units, in completion order, each leave six values at
 * trace[8 + 6 i], times on the device's global timer in ns, all seen by the
 * unit's first query slot: its start, the moment its first score tile was
 * ready, the moment it handed over its last probabilities, its end (its rows
 * stored); then (CTA index << 48) | (level << 32) | schedule rank, and
 * (1 if SA << 62) | (head of slot 0 << 44) | (head of slot 1 << 32) | its KV
 * tile count, a head given as b * Hq + h (the two equal for a single unit;
 * the level is a paired unit's 128-row block, 2p + 1 for a single unit of
 * 256-row pair p).  Errors as for ea_hybrid_attn_prefill, plus EA_ERR_INVALID_ARG
 * for a NULL trace or negative trace_records and EA_ERR_MISALIGNED for a trace
 * that is not 8-byte aligned. */
ea_status ea_hybrid_attn_prefill_traced(const void* q, const void* k, const void* v,
                                        const uint8_t* route_mask, const ea_attn_params* p,
                                        void* out, void* workspace, size_t workspace_bytes,
                                        unsigned long long* trace, int trace_records,
                                        void* stream);

/* Forward of a training step: every head in BOTH modes, in one launch.  The
 * mode route_mask chooses goes to out, with its log-sum-exp in lse (as
 * ea_hybrid_attn_prefill_lse); the other mode to out_other (device bf16
 * [B][Hq][N][d]).  The straight-through router gradient needs both
 * (ea_router_ste_backward); only the chosen mode receives an attention
 * gradient, since the hard route is 0 or 1.  Requires p->select ==
 * EA_SELECT_ALL and 2*B*Hq <= 4096. */
ea_status ea_hybrid_attn_prefill_train(const void* q, const void* k, const void* v,
                                       const uint8_t* route_mask, const ea_attn_params* p,
                                       void* out, float* lse, void* out_other, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Backward pass (training; EA blog §2.1: the router is trained through a
 * Gumbel-Softmax straight-through estimator, so the attention of each head's
 * mode receives the output gradient).  With P the forward's softmax of a head
 * (its own mode) and L = sum(dout * out):
 *   dV = P^T dO, dP = dO V^T, D_i = sum_c dO_ic O_ic, dS = P * (dP - D),
 *   dQ = scale dS K, dK = scale dS^T Q,
 * dK and dV of a kv head summed over its query heads.
 * q, k, v, out, dout : device bf16, padded BHSD (out and dout [B][Hq][N][d]).
 * lse        : the forward's log-sum-exp (ea_hybrid_attn_prefill_lse).
 * route_mask : the forward's mask.
 * dq         : device bf16 [B][Hq][N][d]; dk, dv: [B][Hkv][N][d]; written.
 * workspace  : >= ea_hybrid_attn_backward_workspace_size(p) bytes, zeroed
 *              once; status word, then D (fp32 [B][Hq][N]), then the two
 *              kernels' work schedules (per-CTA unit lists, rebuilt by every
 *              call from route_mask).
 * Arithmetic: bf16 tensor-core operands (P and dS rounded to bf16), fp32
 * accumulation, bf16 results.  Limits: d = 128, p->select == EA_SELECT_ALL,
 * plus those of ea_hybrid_attn_prefill. */
size_t ea_hybrid_attn_backward_workspace_size(const ea_attn_params* p);

ea_status ea_hybrid_attn_backward(const void* q, const void* k, const void* v, const void* out,
                                  const void* dout, const float* lse, const uint8_t* route_mask,
                                  const ea_attn_params* p, void* dq, void* dk, void* dv,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * FP8 (e4m3) variant of the fused attention.  Not on the pages: the same
 * attention (FA causal, SA sink + window, one launch) over inputs stored as
 * e4m3 bytes with one fp32 dequantization scale per (batch, head); what it
 * computes is the attention of code * scale.  e4m3: 1 sign, 4 exponent bits
 * (bias 7), 3 mantissa bits, largest finite 448, subnormals m * 2^-9.
 *
 * ea_quantize_fp8: x device bf16 [heads][N][d] (heads = B * H, d = 128).
 *   Per head, amax = max |x|, scale[h] = amax / 448 and every value becomes
 *   e4m3(x * (448 / amax)) (fp32 arithmetic, round to nearest even,
 *   saturating); an all-zero head gets scale 1.  transpose = 0 writes codes
 *   [heads][N][d]; transpose = 1 writes [heads][d][ea_fp8_vt_stride(N)] (the
 *   layout the attention reads V in; positions >= N are zero).  scale: device
 *   fp32 [heads].  workspace >= ea_quantize_fp8_workspace_size(heads) bytes
 *   (per-head amax, reset by the call).  Deterministic (max is order-free).
 *
 * ea_hybrid_attn_prefill_fp8: q8 [B][Hq][N][128], k8 [B][Hkv][N][128] and
 *   vt8 [B][Hkv][128][ea_fp8_vt_stride(N)] e4m3 codes (as ea_quantize_fp8
 *   writes them), q_scale [B*Hq], k_scale and v_scale [B*Hkv] fp32, all device;
 *   out bf16 [B][Hq][N][128].  Both products run on the tensor cores as
 *   e4m3 x e4m3 -> fp32; the probabilities are rounded to e4m3 for the P.V
 *   product (the row sum is not), so results are within the e4m3 rounding of
 *   P of the exact attention of the dequantized inputs.  Params, mask,
 *   workspace and status as for ea_hybrid_attn_prefill; d must be 128; padded
 *   batches only.
 * ---------------------------------------------------------------------- */
int ea_fp8_vt_stride(int N);

size_t ea_quantize_fp8_workspace_size(int heads);

ea_status ea_quantize_fp8(const void* x, int heads, int N, int d, int transpose, void* codes,
                          float* scale, void* workspace, size_t workspace_bytes, void* stream);

ea_status ea_hybrid_attn_prefill_fp8(const void* q8, const void* k8, const void* vt8,
                                     const float* q_scale, const float* k_scale,
                                     const float* v_scale, const uint8_t* route_mask,
                                     const ea_attn_params* p, void* out, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Router training (EA blog §2.1, training trick: the binary routing is made
 * differentiable with Gumbel-Softmax and a straight-through estimator).
 *
 * Reading: the two-way Gumbel-Softmax over (FA, SA) with logits (0, z) and
 * the caller's Gumbel noise g0 (FA), g1 (SA), device fp32 [B][Hq], gives
 *   r_soft = sigmoid((z + g1 - g0) / tau),   r_hard = [z + g1 - g0 > 0];
 * the forward runs r_hard (out = r_hard O_SA + (1 - r_hard) O_FA) and the
 * backward takes the gradient of r_soft.  The noise is an input so that the
 * caller owns the random stream (g = -log(-log U), U uniform in (0, 1)).
 *
 * ea_router_decide_gumbel: the router's pooling and MLP (bit-identical z to
 * ea_router_decide), then route_mask = r_hard (device uint8 [B][Hq]);
 * r_soft_out and logits_out (device fp32 [B][Hq]) are optional (NULL).
 * workspace >= ea_router_gumbel_workspace_size(...), 16-byte aligned.
 *
 * ea_router_ste_backward: dout, out, out_other device bf16 [B][Hq][N][d]:
 * the layer output's gradient, each head's output in the mode route_mask
 * chose and in its other mode (as ea_hybrid_attn_prefill_train writes them);
 * route_mask == NULL reads as every head having chosen FA, so that out and
 * out_other are then O_FA and O_SA.  With O_SA - O_FA taken from them,
 *   dr[b,h]  = sum_{n,c} dout * (O_SA - O_FA)          (dL/dr_hard)
 *   dz       = dr * r_soft (1 - r_soft) / tau
 * then back through z = W2 ReLU(W1 x + b1) + b2 and the mean pooling:
 *   dw2 [Hq][hidden], db2 [Hq], dw1 [hidden][Hkv*d], db1 [hidden] (device
 *   fp32, written, summed over the batch); dr_out (device fp32 [B][Hq],
 *   optional); dk_pool_out (device fp32 [B][Hkv*d], optional) = dx / N, the
 *   gradient every key position of (b, kv head) receives through the pool;
 *   dk_accum (device bf16 [B][Hkv][N][d], optional) gets dk_pool added in
 *   place (the attention backward's dk plus the router's share).
 * The forward is recomputed from k (no saved activations).  Gradients are
 * summed in fp32 in a fixed order (bit-reproducible run to run).
 * workspace >= ea_router_ste_backward_workspace_size(...), 16-byte aligned.
 * Limits: those of ea_router_decide, B <= 1024, N <= 32767*256 and
 * B * Hkv <= 65535 (backward); dk_accum 16-byte aligned;
 * tau finite and > 0 (else EA_ERR_INVALID_ARG).
 * ---------------------------------------------------------------------- */
size_t ea_router_gumbel_workspace_size(int B, int Hkv, int N, int d, int hidden, int Hq);

ea_status ea_router_decide_gumbel(const void* k, int B, int Hkv, int N, int d,
                                  const float* w1, const float* b1, int hidden,
                                  const float* w2, const float* b2, int Hq,
                                  const float* g0, const float* g1, float tau,
                                  uint8_t* route_mask, float* r_soft_out, float* logits_out,
                                  void* workspace, size_t workspace_bytes, void* stream);

size_t ea_router_ste_backward_workspace_size(int B, int Hkv, int N, int d, int hidden, int Hq);

ea_status ea_router_ste_backward(const void* k, int B, int Hkv, int N, int d,
                                 const float* w1, const float* b1, int hidden,
                                 const float* w2, const float* b2, int Hq,
                                 const float* g0, const float* g1, float tau,
                                 const void* dout, const void* out, const void* out_other,
                                 const uint8_t* route_mask, float* dr_out, float* dw1,
                                 float* db1, float* dw2, float* db2, float* dk_pool_out,
                                 void* dk_accum, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* ------------------------------------------------------------------------
 * Packed variable-length batch (the same attention; not on the pages, which
 * route per input, EA blog §2.1: every sequence is its own square causal
 * prefill).  Sequence b holds tokens [cu_seqlens[b], cu_seqlens[b+1]) of the
 * packed tensors; positions restart at 0 in every sequence, and a sequence
 * sees only its own tokens.
 *
 * q, out   : device bf16 [T][Hq][d] (token-major, then head, then channel).
 * k, v     : device bf16 [T][Hkv][d].  All 16-byte aligned.
 * cu_seqlens: device int32 [B+1], cu[0] = 0, non-decreasing, cu[B] = T.  An
 *             inconsistent array runs nothing and records EA_ERR_INVALID_ARG
 *             in the status word.  Empty sequences are allowed.
 * route_mask: device uint8 [B][Hq], as for ea_hybrid_attn_prefill.
 * p->max_seqlen bounds every length (it sizes the grid only).
 * Workspace as for ea_hybrid_attn_prefill (ea_hybrid_attn_varlen_workspace_size).
 * Limits: d in {64, 128}; Hq % Hkv == 0; B <= 1024; B*Hq <= 4096;
 * max_seqlen <= 32767 * 256; T < 2^31.
 * ---------------------------------------------------------------------- */
typedef struct ea_varlen_params {
  int B, Hq, Hkv;
  int total;             /* T = cu_seqlens[B]                               */
  int max_seqlen;        /* >= every cu_seqlens[b+1] - cu_seqlens[b]        */
  int d;
  int sink, window;
  float softmax_scale;   /* <= 0 selects 1/sqrt(d)                          */
  int select;            /* ea_select                                       */
} ea_varlen_params;

size_t ea_hybrid_attn_varlen_workspace_size(const ea_varlen_params* p);

ea_status ea_hybrid_attn_prefill_varlen(const void* q, const void* k, const void* v,
                                        const int32_t* cu_seqlens, const uint8_t* route_mask,
                                        const ea_varlen_params* p, void* out, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Router and attention in ONE launch (the router runs in the attention
 * kernel's prologue, so a routed prefill layer is a single launch).  Same
 * results, bit for bit, as ea_router_decide (ea_router_decide_varlen)
 * followed by ea_hybrid_attn_prefill (ea_hybrid_attn_prefill_varlen): the
 * prologue pools, reduces and runs both MLP layers with the router kernels'
 * arithmetic, and its phases meet at grid barriers.  The launch is
 * cooperative: every CTA is resident at once or the call returns EA_ERR_CUDA.
 *
 * Arguments: the attention call's, plus the router's (w1, b1, hidden, w2, b2,
 * threshold as for ea_router_decide).  route_mask (device uint8 [B][Hq]) is
 * WRITTEN with the decisions and logits_out (device fp32 [B][Hq] or NULL)
 * with z.  workspace: >= the *_routed_workspace_size bytes, zeroed once
 * before first use; its first 256 bytes hold the status word and the grid
 * barrier, the rest the router's scratch.  A barrier that waits past
 * EA_WAIT_TIMEOUT_MS records EA_ERR_TIMEOUT and the launch ends without
 * running attention; ea_get_device_status then clears those 256 bytes.
 * Packed batches need T > 0. */
size_t ea_hybrid_attn_routed_workspace_size(const ea_attn_params* p, int hidden);

ea_status ea_hybrid_attn_prefill_routed(const void* q, const void* k, const void* v,
                                        const float* w1, const float* b1, int hidden,
                                        const float* w2, const float* b2, float threshold,
                                        uint8_t* route_mask, float* logits_out,
                                        const ea_attn_params* p, void* out, void* workspace,
                                        size_t workspace_bytes, void* stream);

size_t ea_hybrid_attn_varlen_routed_workspace_size(const ea_varlen_params* p, int hidden);

ea_status ea_hybrid_attn_prefill_varlen_routed(const void* q, const void* k, const void* v,
                                               const int32_t* cu_seqlens, const float* w1,
                                               const float* b1, int hidden, const float* w2,
                                               const float* b2, float threshold,
                                               uint8_t* route_mask, float* logits_out,
                                               const ea_varlen_params* p, void* out,
                                               void* workspace, size_t workspace_bytes,
                                               void* stream);

/* Host view of the packed batch's schedule, like ea_schedule_units below:
 * cu_seqlens_host is a HOST int32 [B+1] copy; units_out rows are
 * {sparse, b, h0, h1, row0, n_kv_tiles}.  Returns the unit count or -1. */
int ea_schedule_units_varlen(const uint8_t* mask, const ea_varlen_params* p,
                             const int32_t* cu_seqlens_host, int32_t* units_out, int max_units);

/* ------------------------------------------------------------------------
 * Decode step with a per-head KV-cache policy.
 *
 * Elastic Attention blog §3: the fused treatment of FA and SA heads lowers
 * memory use as well as time.  In decode the saving is the cache: a head
 * routed to SA only reads its S sink keys and its last W keys, so a kv head
 * whose query heads are ALL routed SA keeps a compact cache of S + W rows;
 * any other kv head keeps every position.  The query at position t sees the
 * keys prefill row t sees (FA: 0..t; SA: j < S or t - j < W).
 *
 * Caches (caller-owned, device, bf16, d contiguous):
 *   full    k_full, v_full [n_full][max_len][d]   row p holds position p
 *   compact k_sa,   v_sa   [n_sa][sink+window][d] position p < S at row p,
 *                                                 p >= S at S + (p - S) % W
 * cache_slot[b*Hkv + hk] (device int32) picks a kv head's cache: c >= 0 is
 * full cache c, c < 0 is compact cache -c-1.  A compact cache may back only
 * a kv head whose query heads are all SA (ea_decode_kv_policy builds such an
 * assignment); otherwise the step records EA_ERR_INVALID_ARG in the status
 * word and FA heads of that group see only sink + window keys.  A slot
 * outside its pool, pos[b] < 0, or pos[b] >= max_len on a full cache also
 * records EA_ERR_INVALID_ARG: that (b, kv head) is neither written nor read
 * and its outputs are zero.
 *
 * One step, per sequence b: the new k_new, v_new [B][Hkv][d] are written at
 * position pos[b] (device int32 [B]; 0 <= pos[b] < max_len for full caches),
 * then every query head attends: out[b, h, :] (bf16 [B][Hq][d]) from
 * q [B][Hq][d].  Sequences may sit at different positions.  fp32 softmax
 * and accumulation; the partial results of the split key range live in the
 * workspace (ea_decode_workspace_size bytes, zeroed once: its first word is
 * the status word read by ea_get_device_status).
 * ---------------------------------------------------------------------- */
typedef struct ea_decode_params {
  int B, Hq, Hkv, d;
  int sink, window;
  int max_len;           /* positions a full cache holds                 */
  float softmax_scale;   /* <= 0 selects 1/sqrt(d)                       */
  int n_full, n_sa;      /* caches in each pool; every cache_slot entry
                            must name one of them                        */
} ea_decode_params;

size_t ea_decode_workspace_size(const ea_decode_params* p);

ea_status ea_hybrid_attn_decode(const void* q, const void* k_new, const void* v_new,
                                const int32_t* pos, const uint8_t* route_mask,
                                const int32_t* cache_slot, void* k_full, void* v_full,
                                void* k_sa, void* v_sa, const ea_decode_params* p,
                                void* out, void* workspace, size_t workspace_bytes,
                                void* stream);

/* Host helper: from a host route mask [B][Hq], assign every (b, kv head) a
 * full cache (some query head is FA) or a compact cache (all are SA):
 * cache_slot (host int32 [B][Hkv]) gets the encoding above, numbered in
 * (b, hk) order; *n_full and *n_sa receive the pool sizes.  Returns 0, or -1
 * on invalid arguments. */
int ea_decode_kv_policy(const uint8_t* mask, int B, int Hq, int Hkv, int32_t* cache_slot,
                        int* n_full, int* n_sa);

/* ------------------------------------------------------------------------
 * Prefill from HOST buffers, transfers overlapped with the attention.
 *
 * The pages move no data between host and device; this entry point serves a
 * caller whose q, k, v live in host memory (and who wants out back there).
 * It runs the same method as ea_router_decide followed by
 * ea_hybrid_attn_prefill (Elastic Attention blog §2.1 router, §3 fused
 * kernel) on device copies of the inputs, with bit-identical results, but
 * splits the transfers so that most of them overlap the compute:
 *   1. k (all of it: the router pools every kv head) and, without a router,
 *      the caller's mask are uploaded; the router runs on k.
 *   2. The heads are walked in chunks of c kv heads (with their c*Hq/Hkv
 *      query heads) of one batch element: the chunk's q and v are uploaded,
 *      its attention runs (ea_hybrid_attn_prefill on that head range), and
 *      its rows of out are downloaded, so one chunk's upload and another's
 *      download overlap a third chunk's attention.
 *
 * q_host, k_host, v_host : HOST bf16 BHSD.  Pinned memory (cudaHostAlloc or
 *             cudaHostRegister) is needed for the copies to overlap anything;
 *             pageable memory gives the same results without the overlap.
 * route_mask_host : HOST uint8 [B][Hq] (0 = FA, nonzero = SA) when w1 is
 *             NULL; ignored when the router runs.
 * w1, b1, hidden, w2, b2, threshold : the router as for ea_router_decide
 *             (DEVICE pointers: weights stay resident), or w1 = NULL to use
 *             route_mask_host.
 * p         : host pointer; p->select must be EA_SELECT_ALL.
 * out_host  : HOST bf16 [B][Hq][N][d] (pinned for the overlap).
 * route_mask_out_host : HOST uint8 [B][Hq] that receives the mask used, or
 *             NULL.
 * kv_heads_per_chunk : c in 1..Hkv (larger values are clamped to Hkv), or 0
 *             for about eight chunks in all (ea_hybrid_attn_host_chunks
 *             gives the count).
 * workspace : DEVICE, >= ea_hybrid_attn_host_workspace_size(p, hidden)
 *             bytes (hidden = 0 without a router), 16-byte aligned, ZEROED
 *             once before its first use.  Its first 256 bytes are the
 *             attention status block, read by ea_get_device_status(workspace,
 *             ...); the rest holds the device mask, the router's scratch and
 *             device copies of q, k, v and out.
 * stream    : the call's work starts after the work already enqueued on
 *             `stream`, and work enqueued on `stream` afterwards starts after
 *             all of it, the last download included: synchronise `stream`
 *             before reading out_host.  The copies themselves run on two
 *             non-blocking streams that the library creates per device on
 *             first use and keeps until the process exits.  The call never
 *             synchronises.
 * Argument errors are returned before anything is enqueued; a CUDA failure
 * part way returns EA_ERR_CUDA with earlier chunks already enqueued.  Limits:
 * those of ea_hybrid_attn_prefill (and of ea_router_decide with a router).
 * Two calls in flight at once need separate workspaces and host buffers.
 * ---------------------------------------------------------------------- */
size_t ea_hybrid_attn_host_workspace_size(const ea_attn_params* p, int hidden);

/* Releases what the library holds between calls: the copy streams of
 * ea_hybrid_attn_prefill_host, on every device that created them (after the
 * work already on them finishes; the current device is restored).  Call it
 * with no library call in flight; a later host-buffer call creates the
 * streams again.  Nothing else is held: every other buffer is the caller's,
 * and ea_router_decide_noalloc's fixed scratch is static device memory that
 * lives until the process exits (ea_shutdown only forgets the device
 * addresses it looked up for it, so the next call looks them up again: call
 * ea_shutdown before resetting a device).  EA_OK, or EA_ERR_CUDA if a CUDA
 * call failed (the streams are forgotten either way). */
ea_status ea_shutdown(void);

/* Number of chunks (kernel launches) a call with these arguments makes; 0
 * if p is invalid or kv_heads_per_chunk < 0. */
int ea_hybrid_attn_host_chunks(const ea_attn_params* p, int kv_heads_per_chunk);

ea_status ea_hybrid_attn_prefill_host(const void* q_host, const void* k_host,
                                      const void* v_host, const uint8_t* route_mask_host,
                                      const float* w1, const float* b1, int hidden,
                                      const float* w2, const float* b2, float threshold,
                                      const ea_attn_params* p, void* out_host,
                                      uint8_t* route_mask_out_host, int kv_heads_per_chunk,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Host-side view of the fused kernel's work schedule, for inspection and
 * tests (no GPU needed).  A unit is two 128-row query slots run by one CTA
 * over the same K/V tiles: a paired unit holds rows [row0, row0 + 128) of
 * two query heads h0 != h1 of one kv group with the same route (the group's
 * heads of that mode two by two, in head order); a single unit holds rows
 * [row0, row0 + 256) of one head h0 (= h1), an odd one out of its group.
 * Units are ordered longest first; a CTA takes the next unit of that order
 * from a global counter whenever it starts one (the order is fixed, the CTA
 * that runs a unit is not).
 *
 * mask        : host uint8 [B][Hq].
 * units_out   : host int32 [max_units][6] = {sparse, b, h0, h1, row0,
 *               n_kv_tiles} in schedule rank order (may be NULL to only
 *               count).
 * Returns the number of units (>= 0), or -1 on invalid arguments.
 * ---------------------------------------------------------------------- */
int ea_schedule_units(const uint8_t* mask, const ea_attn_params* p,
                      int32_t* units_out, int max_units);

/* The KV tiles (128 keys each) unit `rank` visits, in visiting order, and
 * per tile and query slot (slot 0: head h0 at rows row0..row0+127; slot 1:
 * head h1 at the same rows, or, single, head h0 at the next 128) a code: 0 = skipped, 1 = every pair visible, 2 = needs the element
 * mask.  tiles_out: host int32 [max_tiles]; codes_out: host int32
 * [max_tiles][2].  Returns the tile count, or -1 on invalid arguments. */
int ea_schedule_unit_tiles(const uint8_t* mask, const ea_attn_params* p,
                           int rank, int32_t* tiles_out, int32_t* codes_out,
                           int max_tiles);

/* Number of CTAs the fused kernel launches for these params when the device
 * has `num_sms` SMs: min(num_sms, B*Hq*ceil(N/256)); 0 if p is invalid.  CTAs
 * left without units by the mask exit at once. */
int ea_attn_grid_size(const ea_attn_params* p, int num_sms);

#ifdef __cplusplus
}
#endif

#endif /* EA_H_ */
