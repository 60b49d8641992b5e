/*
 * fmoe.h — C ABI of the B200 (sm_100a) routed-expert MoE layer library (libfmoe.so).
 *
 * The library computes, per token, the routed-expert forward of one sparse
 * Mixture-of-Experts layer as the Flash-MoE pages describe it:
 *
 *   logits = W_r x (+ b)                      router matvec  (tinai-dev README,
 *                                             "Pipeline mỗi lớp": routing on the GPU)
 *   top-K of softmax(logits), renormalised    (same page: softmax + topK routing;
 *                                             intelliparadigm.com §2.1 router snippet)
 *   for each selected expert k and the shared expert s:
 *     W = scale * code + bias  (4- or 2-bit codes, one bf16 (scale, bias) per
 *                               64-element group)       (hotdry.top "量化策略",
 *                                                        juejin.cn "Metal 着色器")
 *     h = silu(W_g x) * (W_u x); o = W_d h               (hotdry.top "Metal GPU管线":
 *                                                        fused SwiGLU)
 *   y = resid + sum_k w_k o_k + sigmoid(g_s . x) o_s     (hotdry.top "Metal GPU管线":
 *                                                        fused combine + residual +
 *                                                        sigmoid-gated shared expert)
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device, owned by the
 *     caller and borrowed (weights and workspace for the layer's lifetime, inputs and
 *     outputs for the call).  bf16 values are passed as uint16_t bit patterns.
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy default stream.
 *   - Forward entry points are asynchronous: they validate on the host, enqueue kernels
 *     on `stream` and return.  They allocate nothing, copy nothing between host and
 *     device and do not synchronise.
 *   - Host-detectable problems (bad config, NULL or misaligned pointer, missing
 *     workspace) return an error status before anything is enqueued.  Problems found
 *     on the device (an expert index out of range, a bounded wait that ran out) set a
 *     sticky error word in the layer's workspace; while it is set, further forward
 *     calls on that layer do no work.  fmoe_layer_get_error() reads and clears it.
 *   - Calls on one layer must be ordered (one stream, or streams ordered by events):
 *     they share the layer's workspace.
 *   - No CPU fallback exists: without a usable sm_100 device, fmoe_layer_create fails.
 */
#ifndef FMOE_H
#define FMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FMOE_OK = 0,
  FMOE_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or config value        */
  FMOE_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels are built for    */
  FMOE_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed         */
  FMOE_ERR_NO_WORKSPACE = 4,  /* workspace missing or smaller than required          */
  FMOE_ERR_DEVICE = 5,        /* fmoe_layer_get_error found a device-side error      */
  FMOE_ERR_SCRATCH_LIMIT = 6  /* fmoe_layer_forward_noalloc: layer needs more scratch */
} fmoe_status;

/* Device-side error bits reported by fmoe_layer_get_error(). */
#define FMOE_DEVERR_BARRIER_TIMEOUT 0x1u  /* a grid-wide wait ran past its time limit  */
#define FMOE_DEVERR_COPY_TIMEOUT    0x2u  /* a wait for a bulk copy ran past the limit */
#define FMOE_DEVERR_BAD_EXPERT      0x4u  /* fmoe_expert_forward got idx out of range  */
#define FMOE_DEVERR_PLAN            0x8u  /* a batched launch's work split overran the
                                             limits its plan was checked against     */

/* Layer geometry.  hidden (H) and inter (I) are multiples of 64; bits is 4 or 2;
 * 1 <= top_k (K) <= n_experts (E); has_shared and has_router_bias are 0 or 1. */
typedef struct {
  int hidden;
  int inter;
  int n_experts;
  int top_k;
  int bits;
  int has_shared;
  int has_router_bias;
} fmoe_config;

/* Weights, all device pointers.
 *
 * experts: (n_experts + has_shared) packed expert records back to back, routed experts
 *   0..E-1 first and the shared expert last; base 256-byte aligned; each record is
 *   fmoe_record_bytes(H, I, bits) bytes.  One record holds four regions, each starting
 *   at a multiple of 256 bytes from the record start:
 *     GU_Q : for r in 0..I-1: gate code row r (H*bits/8 bytes), then up code row r
 *     GU_SB: for r in 0..I-1: gate (scale,bias) row r (H/64 uint32), then up row r
 *     D_Q  : for j in 0..H-1: down code row j (I*bits/8 bytes)
 *     D_SB : for j in 0..H-1: down (scale,bias) row j (I/64 uint32)
 *   A code row is little-endian uint32 words holding 32/bits codes each; code c of a
 *   word occupies bits [bits*c, bits*c + bits) and is the weight of column
 *   32/bits * word + c.  A (scale,bias) uint32 holds the bf16 scale in its low half and
 *   the bf16 bias in its high half and covers 64 consecutive columns of its row.
 *   Dequantised weight: W[r][c] = scale[r][c/64] * code[r][c] + bias[r][c/64].
 *   (Format of the expert records: 8 nibbles / 16 crumbs per uint32 and bf16 scale
 *   and bias per 64-group; 7,077,888 bytes per 4-bit expert at H=4096, I=1024 — the
 *   "~6.75MB per expert" of hotdry.top "MoE稀疏架构".)
 * router: fp32 [E][H] row-major, 16-byte aligned.
 * router_bias: fp32 [E] added to the logits, or NULL when has_router_bias == 0.
 * shared_gate: fp32 [H], 16-byte aligned, or NULL when has_shared == 0. */
typedef struct {
  const void* experts;
  const float* router;
  const float* router_bias;
  const float* shared_gate;
} fmoe_weights;

typedef struct fmoe_layer* fmoe_layer_t;

/* Bytes of one packed expert record (0 if H or I is not a positive multiple of 64 or
 * bits is not 2 or 4). */
size_t fmoe_record_bytes(int hidden, int inter, int bits);

/* Device workspace bytes a layer with this config needs (0 for an invalid config). */
size_t fmoe_workspace_bytes(const fmoe_config* cfg);

/* Validates cfg and the weight pointers and creates a layer handle on the current
 * device.  The handle keeps copies of cfg and the pointers (not the data).  Errors:
 * INVALID_ARG (NULL/misaligned pointers, bad values), UNSUPPORTED (shapes whose
 * working set does not fit the kernels' shared-memory plan), CUDA (no sm_100 device). */
fmoe_status fmoe_layer_create(const fmoe_config* cfg, const fmoe_weights* w, fmoe_layer_t* out);

/* Releases the handle (host memory only).  NULL is accepted. */
fmoe_status fmoe_layer_destroy(fmoe_layer_t layer);

/* Attaches a caller-owned device workspace of at least fmoe_workspace_bytes() bytes,
 * 256-byte aligned, and zeroes it (synchronously).  Must precede forward calls. */
fmoe_status fmoe_layer_set_workspace(fmoe_layer_t layer, void* dev_ptr, size_t bytes);

/* Routing only.  x: bf16 [T][H] (16-byte aligned).  Writes idx int32 [T][K] (experts
 * in descending router probability, ties to the lower index), w fp32 [T][K] (the K
 * probabilities renormalised to sum to 1) and, if shared_sigma != NULL and the layer
 * has a shared expert, fp32 [T] sigmoid(g_s . x).  T == 0 is a no-op. */
fmoe_status fmoe_route(fmoe_layer_t layer, const uint16_t* x, int T, int32_t* idx, float* w,
                       float* shared_sigma, void* stream);

/* Experts and combine for given routing: y[t] = resid[t] + sum_k w[t][k] o_{idx[t][k]}(x[t])
 * + shared_sigma[t] o_s(x[t]).  x, resid, y: bf16 [T][H], 16-byte aligned; y may alias
 * resid but not x.  idx int32 [T][K], w fp32 [T][K], shared_sigma fp32 [T] (ignored
 * without a shared expert).  An idx outside [0, E) sets FMOE_DEVERR_BAD_EXPERT and
 * that token's y is not written. */
fmoe_status fmoe_expert_forward(fmoe_layer_t layer, const uint16_t* x, const uint16_t* resid, int T,
                                const int32_t* idx, const float* w, const float* shared_sigma,
                                uint16_t* y, void* stream);

/* The whole layer: routing, experts and combine, one token after another:
 * y[t] = resid[t] + sum_k w_k o_k(x[t]) + sigma o_s(x[t]).  resid may equal x; y may
 * alias resid but not x.
 * Range: the dequantising dot products scale each chunk of 32 (4-bit) or 64 (2-bit)
 * activations by a power of two chosen from the chunk's largest magnitude, so their
 * products stay exact for activations x (and hidden values h = silu(W_g x)(W_u x))
 * from about 2^-103 to 2^105 in magnitude whatever their spread; h and the outputs must
 * fit fp32 (and y bf16), which bounds useful inputs well inside that range. */
fmoe_status fmoe_layer_forward(fmoe_layer_t layer, const uint16_t* x, const uint16_t* resid, int T,
                               uint16_t* y, void* stream);

/* RMS normalisation with unit gain (hotdry.top "Metal GPU管线": two-pass RMSNorm, a
 * sum of squares then the scaling): out[t] = bf16(h[t] / sqrt(mean(h[t]^2) + eps)),
 * computed in double and rounded once.  h, out: bf16 [T][H], may alias. */
fmoe_status fmoe_rmsnorm(const uint16_t* h, uint16_t* out, int T, int H, double eps, void* stream);

/* One pre-norm block of a layer stack, with the normalisation fused into the layer
 * kernel: n[t] = bf16(h[t] / sqrt(mean(h[t]^2) + eps)) (as fmoe_rmsnorm computes it),
 * then h_out[t] = h[t] + sum_k w_k o_k(n[t]) + sigma o_s(n[t]), routing on n[t], rounded
 * once to bf16.  (hotdry.top "Metal GPU管线": RMSNorm, routing, experts and the combine
 * with the residual run as one deferred sequence per layer; the stacks of the pages
 * keep attention, which this library replaces by the normalisation and residual
 * alone.)  h, h_out: bf16 [T][H], 16-byte aligned; h_out may alias h (in place).
 * T == 0 is a no-op. */
fmoe_status fmoe_block_forward(fmoe_layer_t layer, const uint16_t* h, int T, double eps, uint16_t* h_out,
                               void* stream);

/* ---- Batched decode: T tokens per call, grouped by expert --------------------------
 * The same per-token results as the single-token entry points (routing identical bit
 * for bit; outputs within the same tolerance of the fp64 definition), computed in
 * another order: the T*K (token, slot) pairs are grouped by expert, so each active
 * expert's weights stream from HBM once for all of its tokens.  The pages decode one
 * token at a time; grouping several tokens' pairs by expert is this library's
 * addition for batched decode.  Each (token, expert) output is the same quantity as
 * on the single-token path; the grouped matvecs compute it on the tensor cores (codes
 * entered as exact bf16 1 + c/2^b, exact products, fp32 sums folded with the scale
 * and bias once per 64-column group).
 * Launch sequence per call: router (fp64, all tokens in one pass over the router),
 * top-K per token plus the grouping, grouped gate/up + SwiGLU, grouped down, combine
 * (plus the small-tile kernels before each grouped phase, or a staging kernel before
 * gate/up on the tcgen05 kernels, when those are selected; see
 * fmoe_layer_batched_kind). */

/* Bytes of the batched-path workspace for up to max_tokens (1..64) tokens per call (0
 * for an invalid config or max_tokens).  With the environment variable
 * FMOE_GROUPED_TCGEN05 = "1" at the time of the call it includes the tcgen05 kernels'
 * activation tiles (shapes they take only; see fmoe_layer_batched_kind); a workspace
 * sized without them runs the mma.sync kernels. */
size_t fmoe_batch_workspace_bytes(const fmoe_config* cfg, int max_tokens);

/* Attaches a caller-owned device workspace for the batched entry points (separate from
 * the single-token workspace), 256-byte aligned, of at least
 * fmoe_batch_workspace_bytes(cfg, max_tokens) bytes, and zeroes it (synchronously).
 * Errors: INVALID_ARG, NO_WORKSPACE (too small), UNSUPPORTED (shapes the batched
 * kernels' shared-memory plan cannot hold), CUDA. */
fmoe_status fmoe_layer_set_batch_workspace(fmoe_layer_t layer, void* dev_ptr, size_t bytes, int max_tokens);

/* Which kernels run the batched path's grouped matvecs:
 *   1 = the default: the mma.sync tensor-core kernels for every tile;
 *   3 = tiles of at most 2 pairs on CUDA-core dequantising matvecs (the single-token
 *       path's dot), larger tiles on the mma.sync kernels: taken when the environment
 *       variable FMOE_GROUPED_SMALL is "1" when the workspace is attached and their
 *       shared memory fits;
 *   2 = the tcgen05 kernels (A = dequantised codes in tensor memory, TMA-staged codes),
 *       taken when FMOE_GROUPED_TCGEN05 is "1" at attach time, hidden and inter are
 *       multiples of 256 (4-bit) or 512 (2-bit) and the expert records admit TMA
 *       tensor maps (it takes precedence over FMOE_GROUPED_SMALL);
 *   0 = no batch workspace attached or layer NULL.
 * All compute the same per-(pair, row) sums to within fp32 rounding. */
int fmoe_layer_batched_kind(fmoe_layer_t layer);

/* Routing of T <= max_tokens tokens in one batched pass: idx int32 [T][K], w fp32 [T][K],
 * shared_sigma fp32 [T] (may be NULL), as fmoe_route computes them. */
fmoe_status fmoe_route_batched(fmoe_layer_t layer, const uint16_t* x, int T, int32_t* idx, float* w,
                               float* shared_sigma, void* stream);

/* The whole layer for T <= max_tokens tokens, grouped by expert:
 * y[t] = resid[t] + sum_k w_k o_k(x[t]) + sigma o_s(x[t]).  x, resid, y: bf16 [T][H],
 * 16-byte aligned; y may alias x or resid. */
fmoe_status fmoe_layer_forward_batched(fmoe_layer_t layer, const uint16_t* x, const uint16_t* resid, int T,
                                       uint16_t* y, void* stream);

/* fmoe_block_forward for T <= max_tokens tokens on the batched path: the normalised
 * input n = bf16(h / sqrt(mean(h^2) + eps)) is written to the batch workspace, then
 * h_out = h + MoE(n).  h_out may alias h. */
fmoe_status fmoe_block_forward_batched(fmoe_layer_t layer, const uint16_t* h, int T, double eps, uint16_t* h_out,
                                       void* stream);

/* A stack of layers applied as pre-norm blocks, h <- h + MoE_l(RMSNorm(h)) for
 * l = 0 .. n_layers-1.  The stack keeps the layer handles (not owned: they must outlive
 * it, with their workspaces attached) and eps.  All layers must have the same hidden
 * size and live on the same device. */
typedef struct fmoe_stack* fmoe_stack_t;

/* Creates a stack over layers[0 .. n_layers-1].  Errors: INVALID_ARG (NULL handles,
 * n_layers < 1, eps < 0, mixed hidden sizes or devices), NO_WORKSPACE (a layer without
 * workspace).  Host memory only. */
fmoe_status fmoe_stack_create(const fmoe_layer_t* layers, int n_layers, double eps, fmoe_stack_t* out);

/* Releases the stack handle (not the layers).  NULL is accepted. */
fmoe_status fmoe_stack_destroy(fmoe_stack_t stack);

/* Decode through the whole stack, in place, on h bf16 [T][H] (16-byte aligned).
 * batch == 1: token after token, each through every block (one fmoe_block_forward
 * launch per layer and token) before the next starts.  batch > 1: steps of `batch`
 * tokens (the last step may be shorter), each step through every block on the batched
 * path (fmoe_block_forward_batched; every layer needs a batch workspace with
 * max_tokens >= batch, else NO_WORKSPACE).  Asynchronous on `stream`; capturable. */
fmoe_status fmoe_stack_forward(fmoe_stack_t stack, uint16_t* h, int T, int batch, void* stream);

/* An instantiated CUDA graph of the launches fmoe_stack_forward(stack, h, T, batch)
 * makes (the pages' deferred per-layer command buffer plays this role).  The graph captures the pointer h and the layers' weights
 * and workspaces: they must stay valid and unmoved while the graph lives. */
typedef struct fmoe_graph* fmoe_graph_t;

/* Captures and instantiates the graph (on a private stream, with the stack's device
 * current; nothing is executed).  Errors: INVALID_ARG, CUDA. */
fmoe_status fmoe_stack_graph_create(fmoe_stack_t stack, uint16_t* h, int T, int batch, fmoe_graph_t* out);

/* Replays the graph on `stream` (asynchronous). */
fmoe_status fmoe_graph_launch(fmoe_graph_t graph, void* stream);

/* Destroys the graph.  NULL is accepted. */
fmoe_status fmoe_graph_destroy(fmoe_graph_t graph);

/* Synchronises the device, returns the layer's device error bits in *device_error
 * (0 if none) and clears them (and the layer's barrier state).  Returns FMOE_OK when no
 * error was set, FMOE_ERR_DEVICE when one was.  A layer without any workspace that has
 * run fmoe_layer_forward_noalloc reports the bits of the last fmoe_layer_forward_noalloc
 * call on its device (whatever layer made it: the calls share one array) and clears
 * them; call it with that device current. */
fmoe_status fmoe_layer_get_error(fmoe_layer_t layer, uint32_t* device_error);

/* Upper bound, in nanoseconds, of every device-side wait of this layer (grid-wide
 * exchanges of partial results, bulk-copy completion).  Default 2e9 (2 s).  A wait that exceeds it sets an
 * error bit and the kernel returns. */
fmoe_status fmoe_layer_set_wait_limit(fmoe_layer_t layer, uint64_t nanoseconds);

/* Test hook for the failure path: when cta >= 0, thread block `cta` of the next forward
 * calls returns before it publishes anything, so the other blocks' bounded wait for
 * its partial results runs out and FMOE_DEVERR_BARRIER_TIMEOUT is set.  -1 (default)
 * disables it. */
fmoe_status fmoe_layer_debug_hold_block(fmoe_layer_t layer, int cta);

/* Diagnostic hook: when dev_buf != NULL (a device buffer of fmoe_layer_grid_size() * 32
 * uint64), every block of the following forward calls records its phase boundaries
 * while it processes token `token` of a call: %globaltimer (ns) in dev_buf[block*32 + i]
 * and the SM clock counter in dev_buf[block*32 + 16 + i], for i = 0 start, 1 activations
 * staged, 2 router rows done, 3 top-K start (the shared expert's gate/up done), 4 top-K
 * done, 5 gate/up done, 6 h rows of all blocks visible, 7 h staged, 8 down rows done,
 * 9 token done, 10 router logits of all blocks visible, 11 expert ranks start, 12 expert
 * ranks done, 14 first batch of h loaded, 15 h loaded.  NULL (default) disables it. */
fmoe_status fmoe_layer_debug_timeline(fmoe_layer_t layer, uint64_t* dev_buf, int token);

/* Number of thread blocks one forward launch uses (one per SM of the device). */
int fmoe_layer_grid_size(fmoe_layer_t layer);

/* ---- GatedDeltaNet step (the linear-attention layers beside the MoE) ---------------
 * One token of `heads` GatedDeltaNet heads, in place on the state:
 *   S_h <- alpha_h S_h;  u = S_h k_h;  S_h <- S_h + beta_h (v_h - u) k_h^T;  o_h = S_h q_h
 * (hotdry.top "Metal GPU管线", linear-attention paragraph: the pages run a scaling,
 * matrix-vector products and a rank-1 update with BLAS on 64 heads x 128 x 128; the
 * composition is GatedDeltaNet's gated delta rule).  All fp32 device pointers:
 * state [heads][dv][dk] row-major (updated in place), q, k [heads][dk], v [heads][dv],
 * alpha, beta [heads], o [heads][dv].  state, q and k 16-byte aligned; 4 <= dk <= 512,
 * dk a multiple of 4; dv >= 1.  heads == 0 is a no-op.  Asynchronous on `stream`.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
fmoe_status fmoe_gdn_step(float* state, const float* q, const float* k, const float* v, const float* alpha,
                          const float* beta, float* o, int heads, int dk, int dv, void* stream);

/* ---- Host-memory expert tier ------------------------------------------------------
 * A layer whose routed experts do not all stay in HBM: their records live in host
 * memory and a cache of `slots` records in HBM holds the experts used most recently
 * (least recently used evicted).  The Flash-MoE pages keep the experts on SSD and read
 * the selected ones per token (hotdry.top "SSD流式加载": parallel pread of the K
 * experts, the OS page cache as the only cache); here the slow tier is host memory
 * over the host link and the cache is explicit, in HBM.
 *
 * Per call (T tokens): the routing runs on the GPU (router in HBM, as fmoe_route), the
 * indices come back to the host, every expert not in the cache is copied host -> device
 * into a free or least-recently-used slot, and the experts run on the cache with the
 * routing remapped to slots (as fmoe_expert_forward).  The outputs equal
 * fmoe_layer_forward's bit for bit (the same kernels on byte-identical records).
 *
 * Ownership: host_experts (E routed records, format as fmoe_weights.experts) is
 * caller-owned host memory, pinned (cudaHostRegister or cudaMallocHost) for
 * asynchronous copies; the router, its bias and the shared gate are device memory;
 * dev_buf is a caller-owned device buffer of fmoe_tier_buffer_bytes() bytes (256-byte
 * aligned) holding the cache, the shared expert's record (copied in at creation from
 * `shared_record`, a device or host pointer to one record) and the workspaces.  The
 * tier keeps pointers, not copies.  Calls on one tier must be serialised by the
 * caller.  Errors: INVALID_ARG, UNSUPPORTED (slots < top_k * max_tokens, or shapes the
 * kernels cannot hold), CUDA. */
typedef struct fmoe_tier* fmoe_tier_t;

/* Device bytes of a tier's buffer (cache of `slots` records, the shared record, the
 * two layers' workspaces and the routing buffers for max_tokens tokens); 0 if invalid. */
size_t fmoe_tier_buffer_bytes(const fmoe_config* cfg, int slots, int max_tokens);

fmoe_status fmoe_tier_create(const fmoe_config* cfg, const void* host_experts, const void* shared_record,
                             const float* router, const float* router_bias, const float* shared_gate,
                             void* dev_buf, size_t buf_bytes, int slots, int max_tokens, fmoe_tier_t* out);

/* y = resid + sum_k w_k o_k(x) + sigma o_s(x) for T <= max_tokens tokens, as
 * fmoe_layer_forward.  Synchronises `stream` once (the routing is read back to place
 * the experts); the expert copies and the expert kernel are then enqueued on `stream`. */
fmoe_status fmoe_tier_forward(fmoe_tier_t tier, const uint16_t* x, const uint16_t* resid, int T, uint16_t* y,
                              void* stream);

/* Counters since creation: expert lookups that hit the cache, those that missed (each
 * miss copies one record host -> device) and the bytes copied. */
fmoe_status fmoe_tier_stats(fmoe_tier_t tier, uint64_t* hits, uint64_t* misses, uint64_t* bytes_h2d);

/* Device error bits of the tier's two layers (as fmoe_layer_get_error). */
fmoe_status fmoe_tier_get_error(fmoe_tier_t tier, uint32_t* device_error);

/* Releases the tier (host memory only).  NULL is accepted. */
fmoe_status fmoe_tier_destroy(fmoe_tier_t tier);

/* Size in bytes of the fixed device scratch array of fmoe_layer_forward_noalloc. */
#define FMOE_NOALLOC_SCRATCH_BYTES (128 * 1024)

/* fmoe_layer_forward without any allocation, for callers that cannot allocate device
 * memory themselves -- code running where cudaMalloc is unavailable or forbidden
 * (inside a captured region that must not allocate, a host framework that owns all
 * device memory, a tiny runtime without an allocator) -- and so cannot provide the
 * workspace fmoe_layer_set_workspace expects.  The pages describing the method have
 * no counterpart of this entry point: it exists for such callers only.
 *
 * Same arguments and results as fmoe_layer_forward; the layer needs no workspace.
 * The scratch lives in one file-scope device array of FMOE_NOALLOC_SCRATCH_BYTES
 * (128 KiB), which every GPU that loads the library keeps until the process exits.
 * A layer whose fmoe_workspace_bytes() exceed that size is rejected with
 * FMOE_ERR_SCRATCH_LIMIT before anything is enqueued.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress, with that device
 * current), so make that first call before any stream capture.  That address is cached
 * per device for the life of the process: after cudaDeviceReset() on a device the
 * cached address belongs to the destroyed context, and the library must not be used on
 * that device again.  Each call first clears the array's control words (an
 * asynchronous memset on `stream`, no allocation) and nothing else allocates or frees
 * memory.  All calls, on all layers and streams, share the one array: calls that
 * overlap on the GPU race and must be ordered by the caller.  Device-side error bits of
 * a call land in the array's error word; fmoe_layer_get_error on a layer without
 * workspace reads and clears them, and the next call clears them too. */
fmoe_status fmoe_layer_forward_noalloc(fmoe_layer_t layer, const uint16_t* x, const uint16_t* resid, int T,
                                       uint16_t* y, void* stream);

/* Human-readable name of a status value. */
const char* fmoe_status_string(fmoe_status status);

#ifdef __cplusplus
}
#endif

#endif /* FMOE_H */
