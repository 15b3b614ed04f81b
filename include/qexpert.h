/*
 * qexpert.h -- C ABI of the B200 (sm_100a) quantized MoE expert step.
 *
 * The operation is the per-token MoE expert step of LLM decode as the
 * Flash-MoE pages describe it:
 *   lilting.ch, "Flash-MoE: running a 397B-parameter model on a 48 GB
 *   MacBook", sections "Model architecture" (512 experts per layer, 4 active
 *   per token), "Core technique: SSD expert streaming" (about 6.75 MB per
 *   4-bit expert) and "Metal Compute Shaders" (4-bit and 2-bit dequant
 *   matrix-vector products, two-pass RMS normalisation, MoE combine as a
 *   weighted sum, and the fma(nibble, scale*x, bias*x) dequant rewrite);
 *   tomo3141592653.github.io summary "Running a 400B-parameter LLM on iPhone
 *   17 Pro", section "Hybrid quantisation" (MLX-style 4-bit quantisation);
 *   nzkcom.pages.dev "flash-moe-romance-vs-utility", table of adopted
 *   optimisations (hot experts at 4 bits, cold ones at 2 bits).
 *
 * For one token x (hidden size H) and one layer:
 *   xn   = x / sqrt(mean(x^2) + eps) * gamma                 (RMSNorm)
 *   l_e  = W_r[e,:] . xn + offset_e            e = 0..E-1    (router)
 *   idx  = the K largest l_e, ties to the lower index         (top-K)
 *   w_k  = exp(l_idx_k - l_max) / sum_j exp(l_idx_j - l_max)  (renormalised softmax)
 *   g,u  = deq(W_gate) xn, deq(W_up) xn       [I]            (dequant-matvec)
 *   h    = silu(g) * u                                        (SwiGLU)
 *   y_k  = deq(W_down) h                      [H]
 *   out  = sum_k w_k y_k (+ x if a residual is requested)     (combine)
 * with deq(W)[r,c] = q[r,c] * scale[r, c/64] + bias[r, c/64].
 *
 * ---------------------------------------------------------------------
 * Packed matrix layout (qe_qmat), R rows x C columns, bits b in {4, 2}:
 *   wq     uint32 [R, C*b/32], row-major; field j of a word (bits
 *          [b*j, b*j+b), low bits first) is column word*32/b + j.
 *   scales bf16 bit patterns (uint16) [R, C/64], row-major.
 *   biases bf16 bit patterns (uint16) [R, C/64], row-major.
 * An expert is gate [I, H], up [I, H], down [H, I].
 *
 * Conventions for every entry point:
 *   - Pointers named dev_* or documented as device memory are device
 *     pointers owned by the caller; the library never frees them.  Unless a
 *     function says otherwise the library allocates nothing.
 *   - Device pointers must be aligned to their element size; router_w rows
 *     and every packed-weight, scale and bias pointer of an expert descriptor
 *     must be 16-byte aligned, and the workspace 256-byte aligned.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream) and
 *     launch only kernels, so they can be captured into a CUDA graph, except
 *     where a function says it synchronises.
 *   - Every function returns QE_OK (0) or a negative status; the thread-local
 *     message of the last failure is qe_last_error().  Argument errors are
 *     reported before anything is launched.  Errors found on the device
 *     (a bounded wait that gave up, a bad expert descriptor) are recorded in
 *     the workspace and returned by qe_workspace_status().
 *   - Shapes: H % 64 == 0, I % 64 == 0, group == 64, 1 <= K <= 16, K <= E,
 *     E <= 1024, H <= 8192, I <= 8192.
 *   - Activations entering the dequant-matvecs must satisfy |v| < 2^90.
 */
#ifndef QEXPERT_H
#define QEXPERT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define QE_API __attribute__((visibility("default")))
#else
#define QE_API
#endif

/* A CUDA stream (cudaStream_t). */
typedef struct CUstream_st* qe_stream_t;

/* Status codes. */
#define QE_OK 0
#define QE_ERR_INVALID_ARG (-1) /* bad pointer, shape or descriptor       */
#define QE_ERR_UNSUPPORTED (-2) /* valid but not supported here            */
#define QE_ERR_CUDA (-3)        /* a CUDA runtime call failed              */
#define QE_ERR_TIMEOUT (-4)     /* a bounded device-side wait gave up      */
#define QE_ERR_OOM (-5)         /* host or device allocation failed        */

/* Activation dtypes. */
#define QE_F32 0
#define QE_BF16 1

/* One packed matrix (device pointers). */
typedef struct {
  const uint32_t* wq;
  const uint16_t* scales;
  const uint16_t* biases;
  int32_t bits; /* 4 or 2 */
  int32_t reserved;
} qe_qmat;

/* One expert: gate [I,H], up [I,H], down [H,I]. */
typedef struct {
  qe_qmat gate, up, down;
} qe_expert;

/* Layer shape. group must be 64. */
typedef struct {
  int32_t hidden;    /* H */
  int32_t n_experts; /* E */
  int32_t top_k;     /* K */
  int32_t inter;     /* I: expert intermediate size */
  int32_t group;     /* quantisation group along the input axis: 64 */
  float eps;         /* RMSNorm epsilon */
} qe_cfg;

/* The weights of one MoE layer.  router_w fp32 [E,H] device; logit_offset
 * fp32 [E] device or NULL (added to the logits before top-K and softmax);
 * gamma fp32 [H] device or NULL (meaning 1); experts: device array of E
 * descriptors. */
typedef struct {
  const float* router_w;
  const float* logit_offset;
  const float* gamma;
  const qe_expert* experts;
} qe_layer;

/* Message of the calling thread's last failure ("" if none). */
QE_API const char* qe_last_error(void);

/* Library version string. */
QE_API const char* qe_version(void);

/* ------------------------------------------------------------------ pool */

/* Bytes of one expert in the standard pool layout at `bits` (4 or 2):
 * gate, up and down packed words, then their scales and biases, every
 * segment 256-byte aligned.  Returns 0 for an invalid shape. */
QE_API size_t qe_expert_bytes(const qe_cfg* cfg, int bits);

/* Fill `table_out` (HOST array of n descriptors) for n experts stored back to
 * back from dev_base (device, 256-byte aligned) in the standard layout, with
 * stride qe_expert_bytes(cfg, bits).  Byte offsets of expert 0's segments are
 * written to seg_offsets[9] if not NULL, in the order gate wq, up wq, down wq,
 * gate scales, gate biases, up scales, up biases, down scales, down biases. */
QE_API int qe_pool_table(const qe_cfg* cfg, void* dev_base, int bits, int n, qe_expert* table_out,
                  size_t* seg_offsets);

/* ------------------------------------------------------------- workspace */

/* Bytes of device workspace the calls below need for T tokens. */
QE_API size_t qe_workspace_bytes(const qe_cfg* cfg, int T);

/* Zero a workspace (device).  Call once after allocating it.  After a call
 * that reported QE_ERR_TIMEOUT the workspace stays usable: the single-token
 * kernel tags what it publishes with a launch epoch kept in the workspace,
 * so nothing a timed-out launch left behind is mistaken for new data. */
QE_API int qe_workspace_init(void* dev_ws, size_t ws_bytes, qe_stream_t stream);

/* Synchronise `stream`, then return (and clear) the status the device wrote
 * into the workspace: QE_OK, QE_ERR_TIMEOUT or QE_ERR_INVALID_ARG. */
QE_API int qe_workspace_status(void* dev_ws, qe_stream_t stream);

/* Time budget of every bounded device-side wait, in nanoseconds (default
 * 200 ms).  Applies to launches made after the call. */
QE_API void qe_set_wait_budget_ns(uint64_t ns);

/* ----------------------------------------------------------- entry points */

/* RMSNorm + router + softmax + top-K for T tokens (sections "Model
 * architecture" and "Metal Compute Shaders" above).
 *   x          [T,H] device, fp32 (x_dtype QE_F32) or bf16 bits (QE_BF16)
 *   gamma      [H] device or NULL; router_w [E,H] fp32 device;
 *   logit_offset [E] device or NULL
 *   xn         [T,H] fp32 device output (may be NULL)
 *   topk_idx   [T,K] int32 device output, descending logit order
 *   topk_w     [T,K] fp32 device output, sums to 1 per token
 * The norm and the router are evaluated in double precision, so the chosen
 * experts are those of an fp64 evaluation up to summation order. */
QE_API int moe_route(const qe_cfg* cfg, const void* x, int x_dtype, const float* gamma,
              const float* router_w, const float* logit_offset, int T, float* xn,
              int32_t* topk_idx, float* topk_w, void* dev_ws, size_t ws_bytes,
              qe_stream_t stream);

/* Expert FFN for T tokens x K selected experts, 4-bit experts only:
 *   y[t,k,:] = deq(down_e) (silu(deq(gate_e) xn[t]) * deq(up_e) xn[t]),
 *   e = topk_idx[t,k]  (section "Metal Compute Shaders": 4-bit matvec).
 *   experts  device table [E] (each selected descriptor must have bits 4)
 *   xn [T,H] fp32 device; topk_idx [T,K] int32 device; y [T,K,H] fp32 device.
 * A selected descriptor with other bits, a NULL pointer or a misaligned
 * pointer leaves its y rows untouched and records QE_ERR_INVALID_ARG. */
QE_API int moe_expert_ffn_q4(const qe_cfg* cfg, const qe_expert* experts, const float* xn,
                      const int32_t* topk_idx, int T, float* y, void* dev_ws, size_t ws_bytes,
                      qe_stream_t stream);

/* Same with 2-bit experts (section "Metal Compute Shaders": 2-bit matvec). */
QE_API int moe_expert_ffn_q2(const qe_cfg* cfg, const qe_expert* experts, const float* xn,
                      const int32_t* topk_idx, int T, float* y, void* dev_ws, size_t ws_bytes,
                      qe_stream_t stream);

/* Same with each expert's own bits (4 or 2), for tiered pools. */
QE_API int moe_expert_ffn_mixed(const qe_cfg* cfg, const qe_expert* experts, const float* xn,
                         const int32_t* topk_idx, int T, float* y, void* dev_ws, size_t ws_bytes,
                         qe_stream_t stream);

/* Weighted combine (section "Metal Compute Shaders": MoE combine):
 *   out[t,:] = sum_k w[t,k] * y[t,k,:]  (+ residual[t,:] if not NULL),
 * k summed in ascending order.  y [T,K,H], w [T,K], residual/out [T,H]; all
 * fp32 device.  out may alias residual. */
QE_API int moe_combine(const float* y, const float* w, const float* residual, int T, int K, int H,
                float* out, qe_stream_t stream);

/* The whole layer step: out[t] = combine(expert FFNs of route(x[t]))
 * (+ x[t] if add_residual).  x [T,H] device fp32 or bf16 (x_dtype); out
 * [T,H] fp32 device (must not alias x); topk_idx/topk_w [T,K] device outputs
 * or NULL.  For T == 1 this is one persistent kernel covering the router,
 * the K experts and the combine; it keeps each SM's share of the K selected
 * experts resident in shared memory, so it takes hidden <= 4096, inter <=
 * 1024 and n_experts <= 8 x the SM count whose share fits, with x 16-byte
 * aligned (8 for bf16) and gamma 16-byte aligned.  Other single tokens take
 * the batched path.  For T > 1
 * the tokens are one batch: assignments are grouped per expert, and each
 * selected expert's weights are read once per pass over up to 4 of its
 * tokens. */
QE_API int moe_layer_step(const qe_cfg* cfg, const qe_layer* layer, const void* x, int x_dtype, int T,
                   float* out, int add_residual, int32_t* topk_idx, float* topk_w, void* dev_ws,
                   size_t ws_bytes, qe_stream_t stream);

/* moe_layer_step on host buffers: x_host [T,H] (fp32 or bf16 bits, page-
 * locked for the copy to run asynchronously) is copied into the workspace,
 * the layer step runs on `stream` (the fused kernel for T == 1, the batched
 * path otherwise), the result is copied to out_host [T,H] fp32, and the call
 * returns after synchronising `stream`.  Routing is not returned.  The
 * workspace is the one qe_workspace_bytes(cfg, T) sizes. */
QE_API int moe_layer_step_host(const qe_cfg* cfg, const qe_layer* layer, const void* x_host, int x_dtype, int T,
                               float* out_host, int add_residual, void* dev_ws, size_t ws_bytes, qe_stream_t stream);

/* The single-token layer step of moe_layer_step (T == 1, fused kernel) for
 * callers that cannot allocate device memory: a plugin whose host engine
 * hands it only input and output buffers, or code running beside an
 * allocator that has already reserved the GPU's memory for itself.  The
 * paper has no counterpart of this call; it only changes where the scratch
 * lives.
 *
 * Instead of a workspace it uses a fixed scratch array built into the
 * library (172,288 bytes, 256-byte aligned), which every GPU that loads the
 * library holds until the process exits.  It calls no allocation routine.
 *   x       [1,H] device, fp32 or bf16 bits (x_dtype); out [1,H] fp32
 *           device (must not alias x); topk_idx/topk_w [1,K] device outputs
 *           or NULL, as in moe_layer_step.
 *   dev_status  int32 device output or NULL: after the step it holds the
 *           device-side status of this call (QE_OK, QE_ERR_TIMEOUT or
 *           QE_ERR_INVALID_ARG), read by the caller after synchronising.
 * Limits: top_k * inter <= 16384, plus the single-token kernel's own: hidden
 * <= 4096, inter <= 1024, n_experts <= 8 x the SM count, the experts' share
 * of one SM within its shared memory, x 16-byte aligned (8 for bf16) and
 * gamma 16-byte aligned.  Anything else is rejected before anything is
 * launched: QE_ERR_INVALID_ARG for top_k * inter and the alignment,
 * QE_ERR_UNSUPPORTED for the rest.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it per device
 * ordinal, for the device's primary context (the one the CUDA runtime uses);
 * do not call it under another driver-API context of the same device.  Make
 * that first call before any stream capture.  Every call clears the array's
 * error word on `stream` before its kernel; the launch epoch kept in the
 * array advances with every call, so a call after one that timed out needs
 * no re-initialisation.  All calls on a device share the array and
 * its contents outlive the call: two calls whose work overlaps on the GPU
 * (other streams, other threads) race and give wrong results; order them
 * on one stream or with events. */
QE_API int moe_layer_step_noalloc(const qe_cfg* cfg, const qe_layer* layer, const void* x, int x_dtype,
                                  float* out, int add_residual, int32_t* topk_idx, float* topk_w,
                                  int32_t* dev_status, qe_stream_t stream);

/* ----------------------------------------------------------------- tiers */

/* Two-tier expert residency (lilting.ch "Flash-MoE", sections "Core
 * technique: SSD expert streaming" and "Trust the OS": experts are streamed
 * from slow storage on demand through a cache; nzkcom.pages.dev
 * "flash-moe-romance-vs-utility", adopted optimisations: hot experts at 4
 * bits, cold experts at 2 bits).  Hot experts stay resident in HBM (the
 * caller's descriptors); cold experts live in page-locked host memory mapped
 * into the device's address space and are copied on demand into a pool of
 * HBM slots with least-recently-used replacement.  The replacement state (the
 * slot map, last-use stamps, counters) lives on the device and is updated by
 * kernels in stream order, so no call waits for the host: a tiered layer step
 * is a fixed sequence of kernel launches and can be captured in a CUDA graph.
 * All calls on one tier must be ordered on the device (one stream, or
 * streams ordered with events).  qe_tier_create is the one call of this
 * library that allocates device memory (the slot pool and its state). */
typedef struct qe_tier qe_tier;

typedef struct {
  qe_cfg cfg;
  int32_t n_layers;
  int32_t cold_bits;   /* bits of every cold expert: 2 or 4 */
  int32_t max_tokens;  /* most tokens one call routes */
  int32_t reserved;
  /* HOST array [n_layers * n_experts]: for a cold expert (l, e), entry
   * l*E+e is the base of its qe_expert_bytes(cfg, cold_bits) bytes in the
   * standard pool layout, in page-locked host memory that the device can
   * read (cudaHostAlloc, or cudaHostRegister with cudaHostRegisterMapped),
   * 16-byte aligned; NULL marks a hot expert.  The array is copied; the
   * memory it points to must outlive the tier. */
  const void* const* cold_host;
  size_t cache_bytes;  /* HBM for cold-expert slots: floor(cache_bytes / expert bytes) slots */
} qe_tier_desc;

/* Create a tier on the current device.  QE_ERR_OOM if the slot pool cannot
 * be allocated; QE_ERR_INVALID_ARG if a cold expert is not 16-byte aligned
 * or not device-readable page-locked memory.  Synchronous. */
QE_API int qe_tier_create(const qe_tier_desc* desc, qe_tier** out);

/* Make the experts host_idx[0..n) (HOST array, indices into layer `layer`)
 * usable from dev_table (device, E descriptors of that layer), on `stream`:
 * for each distinct cold expert, in call order, a hit reuses its slot and a
 * miss takes the least recently used slot not needed by this call; then the
 * misses are copied in from host memory by a kernel and every cold expert's
 * descriptor is written into dev_table.  Hot entries of dev_table are left
 * as they are.  The indices are checked on the host first: QE_ERR_INVALID_ARG
 * for one out of range, QE_ERR_OOM if the call needs more distinct cold
 * experts than there are slots; a refused call changes nothing. */
QE_API int qe_tier_resolve(qe_tier* t, int layer, const int32_t* host_idx, int n, qe_expert* dev_table,
                           qe_stream_t stream);

/* The layer step with tiered experts, all on `stream` with no host
 * synchronisation: routing (as moe_route), the resolve of the routed experts
 * into layer->experts on the device (as qe_tier_resolve), the copy of the
 * misses, then the expert FFNs and the combine (+ x if add_residual): the
 * single-token kernel with this routing for T = 1, moe_layer_step's batched
 * path otherwise.  Arguments as moe_layer_step; T <= max_tokens, and
 * QE_ERR_OOM before any launch if T * top_k exceeds the number of slots (the
 * routing, unknown to the host, could need that many cold experts). */
QE_API int qe_tier_layer_step(qe_tier* t, int layer, const qe_layer* layer_w, const void* x, int x_dtype, int T,
                              float* out, int add_residual, int32_t* topk_idx, float* topk_w, void* dev_ws,
                              size_t ws_bytes, qe_stream_t stream);

/* Counters since creation: distinct cold experts found in the cache (hits),
 * copied in (misses), and bytes copied host->device.  Synchronises the
 * device first (the counters live there).  Returns the first error a resolve
 * met on the device, if any (QE_ERR_INVALID_ARG for an index out of range,
 * QE_ERR_OOM), after filling the counters. */
QE_API int qe_tier_stats(const qe_tier* t, uint64_t* hits, uint64_t* misses, uint64_t* h2d_bytes);

/* Number of HBM slots of the tier (0 for NULL). */
QE_API int qe_tier_slots(const qe_tier* t);

/* Synchronise the device, then free everything the tier allocated.  NULL is
 * a no-op. */
QE_API void qe_tier_destroy(qe_tier* t);

/* Test hook: make CTA `cta` of the next fused single-token launches skip
 * publishing its router logits (-1 disables).  Every CTA's bounded wait for
 * those logits then gives up and the workspace reports QE_ERR_TIMEOUT. */
QE_API void qe_test_skip_arrival(int cta);

/* Test hook, host only (no GPU involved): the single-token kernel's plan for
 * CTA `cta` of a grid of `sms` CTAs with `smem_optin` bytes of shared memory
 * per block, computed by the functions the kernel itself uses.  bits[K]: the
 * bits of the K selected experts; seg[K*9]: their segment addresses in
 * qe_pool_table's order (any 16-byte aligned values).  Writes geom[64] (the
 * geometry; geom[21] = copies, geom[22] = reads, geom[23] = first gate/up
 * row, geom[24 + b] = the bytes mbarrier b is armed with), copies[n][4] =
 * {shared-memory offset, source address, bytes, mbarrier} and reads[n][6] =
 * {kind, expert, a, b, shared-memory offset,
 * bytes} (kind 0 gate/up word, a = 2*pair + up, b = 32-column chunk; 1
 * gate/up scale or bias, a = 4*pair + segment, b = group; 2 down word, a =
 * owned row, b = chunk; 3 down scale or bias, a = 2*row + segment, b =
 * group).  Returns QE_ERR_UNSUPPORTED for a shape the kernel does not take
 * and QE_ERR_INVALID_ARG if the arrays are too small. */
QE_API int qe_fused_plan_probe(int H, int E, int K, int I, int sms, int smem_optin, int cta, const int* bits,
                               const uint64_t* seg, int* geom, long long* copies, int max_copies, long long* reads,
                               int max_reads);

/* Tracing: while dev_buf (device, uint64 [SMs][16]) is set, every fused
 * single-token launch writes globaltimer stamps (ns) of its phases per CTA:
 * 0 start, 1 router dot products done, 2 all logits received, 3 top-K done,
 * 4 expert copies issued, 5 first row pair landed, 6 gate/up done, 7 all of
 * h received and staged, 8 down rows done, 9 end, 10 experts and weights
 * known (before their descriptors are read), 11 warp 0 has the last
 * expert's gate/up rows, 12 warp 0 has its down rows, 13 all of h
 * received, 14 every thread has its logits, 15 warp 0 done with its top-K
 * rounds.  Slots a CTA does not
 * reach keep their old value.  NULL disables tracing. */
QE_API void qe_trace_fused(void* dev_buf);

/* ---------------------------------------------------------------------
 * GatedDeltaNet decode step (the linear-attention recurrence of 45 of the
 * model's 60 layers): lilting.ch, "Flash-MoE: running a 397B-parameter model
 * on a 48 GB MacBook", section "GatedDeltaNet acceleration" (64 heads x
 * 128x128 state matrices updated per token with the BLAS calls scal, gemv
 * and ger); tomo3141592653.github.io summary "Running a 400B-parameter LLM
 * on iPhone 17 Pro", section "GatedDeltaNet" (a fixed O(1) state).  The pages
 * print no formula; the recurrence is read as the gated delta rule, per head
 *   S <- alpha S;  u = S k;  S <- S + beta (v - u) k^T;  o = S q,
 * i.e. S' = alpha S (I - beta k k^T) + beta v k^T and o = S' q.
 *
 *   state  device fp32 [n_heads][dv][dk], row-major (row i is value
 *          component i); updated in place.  16-byte aligned.
 *   q, k   device fp32 [n_heads][dk]; 16-byte aligned.  (Unit-length keys
 *          keep the recurrence non-expansive; nothing here requires it.)
 *   v      device fp32 [n_heads][dv].
 *   alpha, beta  device fp32 [n_heads]: decay and write strength per head.
 *   out    device fp32 [n_heads][dv]: o of every head.  Must not overlap any
 *          input.
 * n_heads counts independent heads (a batch of sequences is n_seq * heads
 * heads).  Shapes: n_heads >= 0 (0 launches nothing), dv >= 1, 4 <= dk <= 512,
 * dk % 4 == 0; anything else returns QE_ERR_INVALID_ARG before any launch,
 * as do NULL, misaligned or overlapping pointers.  Asynchronous on `stream`,
 * one kernel launch, graph-capturable; the launch may overlap the tail of the
 * previous kernel in the stream but reads nothing before that kernel has
 * finished.  The arithmetic is fp32 (the pages use single-precision BLAS). */
QE_API int gdn_decode_step(int n_heads, int dk, int dv, float* state, const float* q, const float* k,
                           const float* v, const float* alpha, const float* beta, float* out, qe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QEXPERT_H */
