/*
 * moe.h -- C ABI of the B200 (sm_100a) int4 routed-expert MoE decode layer.
 *
 * The layer (one decode step of a GLM-5.2 / DeepSeek-V3 style MoE block):
 *   1. router GEMV:   logit[e] = sum_h W_g[e][h] * x[h]
 *   2. noaux_tc:      s = sigmoid(logit), s' = s + e_score_correction_bias;
 *                     group score = sum of the two largest s' of each of
 *                     n_group groups; keep topk_group groups; top_k largest
 *                     s' inside them (ties to the lower index);
 *                     w_j = routed_scaling_factor * s_j / sum_j s_j
 *   3. gather:        the top_k selected int4 experts
 *   4. expert FFN:    h = silu(W_gate x) * (W_up x); y_e = W_down h
 *   5. combine:       y = sum_j w_j * y_{e_j} + y_shared
 * Sources: "LightLX" page, section "How it works" (256 experts per layer, a
 * router picks 8 per token, noaux_tc sigmoid router, resident shared
 * experts); colibri summary ("Show HN: run GLM 5.2 on a slow computer"),
 * section "Principales fonctionnalites implementees" (DeepSeek-V3 sigmoid
 * router with noaux_tc, routed_scaling_factor, shared expert; int4
 * dequant-on-use kernels; batch-union MoE; per-layer LRU expert cache).
 *
 * int4 format (the layer's spec): symmetric two's-complement codes in
 * [-8, 7], two per byte, byte j of a row holding input 2j in its low nibble
 * and 2j+1 in its high nibble; one fp16 scale per group_size (= 32)
 * consecutive inputs of a row.  Weight value = code * scale.
 *
 * Conventions for every call:
 *  - Pointers named *_dev are device memory; *_host are host memory.
 *    Sizes are element counts unless named *_bytes.
 *  - All compute calls are asynchronous on the given stream (a cudaStream_t
 *    passed as void*; NULL = the legacy default stream).  The returned status
 *    covers argument checks and launch errors only; faults of the kernels
 *    themselves surface at the next synchronising call (moe_ws_check).
 *  - No call throws; moe_last_error() gives a text for the last failure of
 *    the calling thread.
 *  - The caller owns x, y, idx, w and the workspace; the library owns what
 *    moe_layer_create / moe_cache_create allocate.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer */
  MOE_ERR_CUDA = 2,         /* a CUDA runtime call failed */
  MOE_ERR_OOM = 3,          /* an allocation failed or would not fit */
  MOE_ERR_TIMEOUT = 4,      /* a bounded wait ran out (host or device) */
  MOE_ERR_UNSUPPORTED = 5,  /* shape outside what the kernels handle */
  MOE_ERR_DEVICE = 6        /* a kernel reported an error in the workspace */
} moe_status;

/* Layer shape.  Supported: hidden / 32 and inter / 32 each 2, 4, 8, 16 or a
 * multiple of 32 up to 256 (GLM-5.2: hidden 6144, inter 2048); group_size
 * 32; n_experts <= 1024 divisible by n_group; n_experts / n_group <= 32;
 * n_group <= 32; top_k <= 32; topk_group * (n_experts / n_group) >= top_k;
 * n_shared 0 or 1.  Other shapes return MOE_ERR_UNSUPPORTED. */
typedef struct {
  int32_t hidden;
  int32_t inter;
  int32_t n_experts;
  int32_t n_shared;
  int32_t top_k;
  int32_t n_group;
  int32_t topk_group;
  int32_t group_size;
  float routed_scaling_factor;
} moe_config;

/* One expert in the canonical layout, every pointer 16-byte aligned:
 *   q_gate, q_up  uint8 [inter][hidden/2]       packed int4 codes
 *   s_gate, s_up  fp16  [inter][hidden/32]      scales
 *   q_down        uint8 [hidden][inter/2]
 *   s_down        fp16  [hidden][inter/32]
 * Bytes per expert: 3*hidden*inter/2 + 3*hidden*inter/16. */
typedef struct {
  const uint8_t* q_gate;
  const uint8_t* q_up;
  const uint16_t* s_gate;
  const uint16_t* s_up;
  const uint8_t* q_down;
  const uint16_t* s_down;
} moe_expert;

typedef struct moe_layer moe_layer;

/* ---- layers ---------------------------------------------------------- */

/* Create a layer VIEW over caller-owned device tensors (nothing is copied):
 *   w_router_dev fp32 [n_experts][hidden], bias_dev fp32 [n_experts],
 *   experts_host[n_experts] (host array of device pointers), shared_host
 *   (host pointer to one moe_expert of device pointers; NULL iff
 *   n_shared == 0).
 * The device tensors must stay alive and unchanged until moe_layer_destroy.
 * Allocates a small device pointer table (about 48 bytes per expert) on the
 * current device.  Errors: INVALID_ARG (null / misaligned / host memory where
 * device memory is required), UNSUPPORTED (shape), OOM, CUDA. */
moe_status moe_layer_create(const moe_config* cfg, const float* w_router_dev,
                            const float* bias_dev,
                            const moe_expert* experts_host,
                            const moe_expert* shared_host, moe_layer** out);
void moe_layer_destroy(moe_layer* layer);

/* Repoint routed expert e of a layer at other device tensors (used by the
 * expert cache).  Enqueued on stream, so kernels already enqueued on that
 * stream still see the old pointers. */
moe_status moe_layer_set_expert(moe_layer* layer, int e,
                                const moe_expert* expert_host, void* stream);

/* Adaptive expert top-p of a layer (colibri summary, "Telechargement et
 * execution du modele": the --topp option, adaptive expert top-p, fewer
 * expert bytes read; the pages give no formula, so the rule here is this
 * library's reading): of the top_k experts the router selects, keep the
 * fewest, taken in descending weight (ties: the lower id first), whose
 * weights add up to at least p * routed_scaling_factor, and normalise the
 * kept weights again over the kept experts.  Routes then carry the kept ids
 * ascending followed by -1 (weight 0) for each dropped slot; -1 entries are
 * skipped by moe_expert_ffn, and a dropped expert's bytes are not read.
 * p >= 1 turns it off (the default); p must be > 0.  Applies to every call
 * that routes (moe_route, moe_layer_forward, the residual and stack calls).
 * Not thread-safe against calls on the same layer. */
moe_status moe_layer_set_top_p(moe_layer* layer, float p);

/* ---- workspace --------------------------------------------------------- */

/* Bytes of device workspace a call with T tokens needs.  The workspace must
 * be 256-byte aligned and zero-filled before its first use, and the caller
 * must not write it between calls (moe_ws_check aside): the fused kernel
 * leaves its counters zero after every call but keeps a call count and the
 * router score records, tagged with that count, from call to call, in a
 * region that no other call writes.  A workspace sized for T tokens serves
 * every call with T or fewer tokens, one-token and batched calls mixed.  One
 * workspace must not be used by two calls that can run at the same time. */
size_t moe_workspace_bytes(const moe_config* cfg, int T);

/* Synchronise the stream, then read the device error word of a workspace.
 * Returns MOE_OK, or MOE_ERR_DEVICE / MOE_ERR_TIMEOUT when a kernel reported
 * a problem (the error word is then cleared), or MOE_ERR_CUDA. */
moe_status moe_ws_check(void* ws_dev, size_t ws_bytes, void* stream);

/* ---- the hot path ------------------------------------------------------ */

/* Pointer rules for moe_route, moe_expert_ffn, moe_layer_forward,
 * moe_layer_forward_noalloc, moe_layer_forward_residual and moe_stack_forward:
 * all buffers are device memory of the current device; x / y / x_next buffers start on a 16-byte boundary; idx,
 * w, scores, xn_out and status buffers on a 4-byte boundary.  A NULL (where
 * not nullable), host or misaligned pointer returns MOE_ERR_INVALID_ARG
 * before anything is launched. */

/* Steps 1-2 for T tokens.  x_dev bf16 [T][hidden]; idx_dev int32 [T][top_k]
 * (ascending expert ids); w_dev fp32 [T][top_k]; scores_dev fp32
 * [T][n_experts] = sigmoid scores s (nullable, for inspection).
 * 1 <= T <= 64. */
moe_status moe_route(const moe_layer* layer, const void* x_dev, int T,
                     int32_t* idx_dev, float* w_dev, float* scores_dev,
                     void* ws_dev, size_t ws_bytes, void* stream);

/* Steps 3-5 for T tokens with given routes: y_dev fp32 [T][hidden] =
 * sum_j w[t][j] * FFN_{idx[t][j]}(x_t) + FFN_shared(x_t).  Expert ids must be
 * in [0, n_experts), or -1 for a slot dropped by top-p (skipped); any other
 * id sets the workspace error word and its term is skipped.  1 <= T <= 64. */
moe_status moe_expert_ffn(const moe_layer* layer, const void* x_dev, int T,
                          const int32_t* idx_dev, const float* w_dev,
                          float* y_dev, void* ws_dev, size_t ws_bytes,
                          void* stream);

/* moe_expert_ffn for a subset of the slots, so that the experts of a token
 * can run in several calls (a streamed cache runs the resident experts first
 * and each copied one once its copy is done: colibri summary, "Principales
 * fonctionnalites implementees", the next expert block read while another is
 * multiplied).  slot_mask bit j (j < top_k) runs routed slot j of every
 * token, bit top_k the shared expert; the partial outputs of the other slots
 * in the workspace are left as they are.  combine != 0 then writes y from the
 * partial outputs of every slot -- those of this call and of earlier calls on
 * the same workspace with the same x, idx and T -- in the fixed slot order,
 * so that calls covering every slot once give y bitwise equal to one
 * moe_expert_ffn call.  combine == 0 leaves y unwritten.  Other arguments
 * and errors as moe_expert_ffn. */
moe_status moe_expert_ffn_part(const moe_layer* layer, const void* x_dev, int T,
                               const int32_t* idx_dev, const float* w_dev,
                               float* y_dev, uint64_t slot_mask, int combine,
                               void* ws_dev, size_t ws_bytes, void* stream);

/* Steps 1-5 for T tokens.  idx_out_dev / w_out_dev nullable.  T == 1 runs the
 * single fused persistent decode kernel; T > 1 runs the batched path, which
 * reads every distinct selected expert once for all tokens routed to it.
 * 1 <= T <= 64.
 * The fused kernel (T == 1 here, moe_layer_forward_residual,
 * moe_stack_forward, moe_layer_forward_noalloc) needs the whole device: one
 * CTA on every SM at once, launched cooperatively.  When SMs are held by
 * other work the launch fails (MOE_ERR_CUDA) instead of waiting. */
moe_status moe_layer_forward(const moe_layer* layer, const void* x_dev, int T,
                             float* y_dev, int32_t* idx_out_dev,
                             float* w_out_dev, void* ws_dev, size_t ws_bytes,
                             void* stream);

/* moe_layer_forward for one token (T = 1) without a caller workspace, so
 * that the call allocates no device memory: its scratch is a fixed
 * 512 KiB array in the library's device image (one per device), and the
 * call makes no cudaMalloc, cudaFree or other allocating call.  The pages
 * have no counterpart to this entry point; it exists for callers that may
 * not allocate (for example while another component owns the allocator).
 *   x_dev bf16 [hidden]; y_dev fp32 [hidden]; idx_out_dev int32 [top_k] and
 *   w_out_dev fp32 [top_k] nullable, as in moe_layer_forward.
 *   status_out_dev (nullable) uint32: after the kernel, the device error word
 *   of this call (0 = none; 1 = expert id out of range, 2 = a device-side
 *   wait ran out), written on `stream`.
 * Results are bitwise those of moe_layer_forward(layer, x_dev, 1, ...).
 * Shapes whose one-token workspace, moe_workspace_bytes(cfg, 1), exceeds
 * 512 KiB are refused with MOE_ERR_UNSUPPORTED.  The current device must be
 * the layer's.  Each call first clears the array's error word on `stream`,
 * then runs the same kernels as moe_layer_forward.
 * The first call on each device resolves the array's address
 * (cudaGetSymbolAddress, which may load the module), zero-fills the array's
 * control words on `stream` and sets the decode kernel's shared-memory
 * attribute: make it before any stream capture.
 * All calls on one device share the one array: calls that can overlap on
 * the device (different streams, or host threads without ordering between
 * them) race on it and give undefined results; calls on one stream are
 * ordered and safe. */
moe_status moe_layer_forward_noalloc(const moe_layer* layer, const void* x_dev,
                                     float* y_dev, int32_t* idx_out_dev,
                                     float* w_out_dev, uint32_t* status_out_dev,
                                     void* stream);

/* ---- stacked layers (pre-norm residual stream) --------------------------- */

/* One decoder MoE step on an fp32 residual stream (the reading of a stack of
 * layers: RMSNorm with unit gain before each MoE block, as in the upstream
 * model -- "LightLX", "How it works": RMSNorm):
 *   x_next = x + MoE(bf16(x / sqrt(mean(x^2) + norm_eps)))
 * x_dev, x_next_dev fp32 [hidden], distinct, 16-byte aligned.  xn_out_dev
 * (nullable, 4-byte aligned) receives
 * the bf16 normalised input the experts saw.  One token (T = 1); the shape
 * must be one the fused decode kernel covers (MOE_ERR_UNSUPPORTED otherwise).
 * The workspace is that of moe_workspace_bytes(cfg, 1). */
moe_status moe_layer_forward_residual(const moe_layer* layer, const float* x_dev,
                                      float* x_next_dev, uint16_t* xn_out_dev,
                                      int32_t* idx_out_dev, float* w_out_dev,
                                      float norm_eps, void* ws_dev,
                                      size_t ws_bytes, void* stream);

/* n_layers residual steps in order, one token: layers[l] maps x_l to
 * x_{l+1}; x_in_dev = x_0, x_out_dev = x_{n_layers}; x_tmp_dev is a third
 * fp32 [hidden] buffer (unused for one layer).  idx_out_dev (nullable)
 * int32 [n_layers][top_k].  All launches are enqueued on stream (capturable
 * into a CUDA graph). */
moe_status moe_stack_forward(const moe_layer* const* layers, int n_layers,
                             const float* x_in_dev, float* x_out_dev,
                             float* x_tmp_dev, int32_t* idx_out_dev,
                             float norm_eps, void* ws_dev, size_t ws_bytes,
                             void* stream);

/* ---- host-streamed experts: per-layer LRU cache in HBM ------------------ */
/* colibri summary ("Show HN: run GLM 5.2 on a slow computer"), section
 * "Execution d'un MoE basee sur le streaming disque": a per-layer LRU cache
 * of routed experts in front of a larger store; "Principales fonctionnalites
 * implementees": the next expert block is read while another is multiplied.
 * Here the store is pinned host memory and the cache is HBM. */
typedef struct moe_cache moe_cache;

/* host_experts: host array [n_layers][n_experts] of moe_expert whose six
 * pointers are pinned host memory (cudaHostAlloc / registered), caller-owned,
 * alive until moe_cache_destroy.  Allocates n_layers * slots_per_layer expert
 * slots in HBM (MOE_ERR_OOM if they do not fit) and a copy stream.
 * top_k <= slots_per_layer <= n_experts. */
moe_status moe_cache_create(const moe_config* cfg, int n_layers,
                            int slots_per_layer,
                            const moe_expert* host_experts, moe_cache** out);
void moe_cache_destroy(moe_cache* cache);

/* The layer view of `layer` (created on first call, owned by the cache):
 * router weight / bias and the shared expert are resident device tensors as
 * in moe_layer_create; routed entries point into the cache's slots and are
 * valid for the ids of the latest moe_cache_acquire of that layer. */
moe_status moe_cache_layer(moe_cache* cache, int layer,
                           const float* w_router_dev, const float* bias_dev,
                           const moe_expert* shared_host, moe_layer** view);

/* Make experts ids_host[0..n) (ascending, distinct) of `layer` resident:
 * LRU bookkeeping on the host; every miss is copied host -> slot with
 * cudaMemcpyAsync on the cache's copy stream (after the layer's last
 * release event, so no slot still in use is overwritten; if the layer was
 * acquired again with no release in between, after everything enqueued on
 * compute_stream so far); compute_stream then waits for the copies and the
 * layer view's pointer table is updated on it.  Replacement: hits are
 * touched in ascending id order, then each miss in ascending id order takes
 * the lowest empty slot, else the least recently used slot not holding one
 * of ids.  n <= slots_per_layer, n <= 32.
 * Transactional: the replacement state, the counters and the pointer table
 * change only when every copy was enqueued.  On a failed enqueue the call
 * returns MOE_ERR_CUDA and the layer keeps its previous state, except that
 * the slots its copies may have reached are marked empty (so a later
 * acquire reloads rather than trusts them). */
moe_status moe_cache_acquire(moe_cache* cache, int layer,
                             const int32_t* ids_host, int n,
                             void* compute_stream);
/* moe_cache_acquire with one completion per copied expert instead of one
 * for the call: the replacement, counters, usage log and the pointer-table
 * update on compute_stream are those of moe_cache_acquire, but compute_stream
 * does not wait for the copies.  missed_host[j] (n int32, caller-owned) is
 * set to 1 when ids_host[j] was copied by this call, else 0; before compute
 * on compute_stream reads a copied expert, the caller calls
 * moe_cache_wait_expert for it (a hit needs no wait: this call makes
 * compute_stream wait for any copy of a hit's slot still pending), so the
 * resident experts can run while the copies are on the link.
 * Transactional and with the limits of moe_cache_acquire. */
moe_status moe_cache_acquire_split(moe_cache* cache, int layer,
                                   const int32_t* ids_host, int n,
                                   void* compute_stream, int32_t* missed_host);
/* Make compute_stream wait until the copy that loaded `expert` into
 * `layer`'s cache is done (MOE_ERR_INVALID_ARG if the expert is not in the
 * cache). */
moe_status moe_cache_wait_expert(moe_cache* cache, int layer, int expert,
                                 void* compute_stream);
/* One token of `layer` through the cache, the resident experts first:
 * moe_cache_acquire_split of the token's top_k ids (ids_host, ascending,
 * distinct; the same ids as idx_dev, which the kernels read), then
 * moe_expert_ffn_part of the hits and the shared expert at once, then, for
 * each copied expert in slot order, moe_cache_wait_expert and its own
 * moe_expert_ffn_part; the last call combines.  y_dev is bitwise that of
 * moe_expert_ffn on the resident layer.  x_dev bf16 [1][hidden], idx_dev
 * int32 [1][top_k], w_dev fp32 [1][top_k], y_dev fp32 [1][hidden], a
 * workspace of moe_workspace_bytes(cfg, 1).  n_copied (nullable): how many
 * experts were copied.  Errors as the calls it makes; on an error after the
 * acquire the caller still releases the layer. */
moe_status moe_cache_expert_ffn(moe_cache* cache, int layer, const void* x_dev,
                                const int32_t* ids_host, const int32_t* idx_dev,
                                const float* w_dev, float* y_dev, void* ws_dev,
                                size_t ws_bytes, void* stream, int* n_copied);
/* Hot-store (colibri summary, "Learning cache et attentes selon le
 * materiel": routed experts are logged and the most used are pinned at
 * start-up).  Makes ids_host[0..n) (ascending, distinct) the pinned set of
 * `layer`: each is made resident as by moe_cache_acquire (copies on the copy
 * stream, compute_stream waits for them, the pointer table is updated on
 * it) and its slot is never chosen as a victim afterwards; the previously
 * pinned experts not in ids become ordinary LRU entries.  n = 0 unpins all.
 * 0 <= n <= slots_per_layer - top_k.  Counts its bytes in
 * bytes_h2d but not as hits, misses or usage.  Transactional like
 * moe_cache_acquire.  With p experts pinned, an acquire takes at most
 * slots_per_layer - p ids. */
moe_status moe_cache_pin(moe_cache* cache, int layer, const int32_t* ids_host,
                         int n, void* compute_stream);
/* The usage log of `layer`: counts_host[e] (n_experts entries, caller-owned
 * host memory) = how many committed moe_cache_acquire calls of the layer
 * named expert e.  The ranking a caller pins by is its own choice. */
moe_status moe_cache_usage(const moe_cache* cache, int layer,
                           uint64_t* counts_host);
/* Mark the end of the compute that reads `layer`'s slots on compute_stream. */
moe_status moe_cache_release(moe_cache* cache, int layer, void* compute_stream);
/* Cumulative counters of a layer (any pointer nullable). */
moe_status moe_cache_stats(const moe_cache* cache, int layer, uint64_t* hits,
                           uint64_t* misses, uint64_t* bytes_h2d);
/* Wait for the cache's copy stream. */
moe_status moe_cache_sync(moe_cache* cache);
/* Wait at most timeout_ms for the cache's copy stream, polling it from the
 * host (cudaStreamQuery): MOE_OK when every enqueued copy has finished,
 * MOE_ERR_TIMEOUT when the deadline passes first (the copies go on; a later
 * wait can succeed), MOE_ERR_CUDA if the stream reports an error. */
moe_status moe_cache_wait(moe_cache* cache, int timeout_ms);

/* The cache's replacement rule run on the host over a trace [T][n_layers][k]
 * of ascending ids (no GPU needed): per-layer hits and misses after T calls
 * with `capacity` slots, all empty at the start. */
moe_status moe_lru_replay(int n_layers, int n_experts, int capacity, int k,
                          int T, const int32_t* trace, uint64_t* hits,
                          uint64_t* misses);
/* moe_lru_replay with the hot-store: before the first call, experts
 * pinned[l][0..n_pinned) (ascending) of each layer l are loaded and pinned
 * as by moe_cache_pin (their loads are not counted); n_pinned <= capacity -
 * k. */
moe_status moe_lru_replay_pinned(int n_layers, int n_experts, int capacity,
                                 int k, int T, const int32_t* trace,
                                 int n_pinned, const int32_t* pinned,
                                 uint64_t* hits, uint64_t* misses);

/* ---- diagnostics ------------------------------------------------------- */

/* One dequantising int4 GEMV with the layer kernels' group dot product:
 * y_dev[r] = sum_c q[r][c] * fp16(s[r][c / 32]) * x_dev[c] for r < rows.
 * q_dev uint8 [rows][cols/2] (16-byte aligned, packing as in moe_expert),
 * s_dev fp16 [rows][cols/32], x_dev fp32 [cols] (16-byte aligned), y_dev
 * fp32 [rows].  cols follows the rule for hidden in moe_config.  For checks
 * of the packing and the scale indexing (x = a unit vector returns one
 * dequantised column). */
moe_status moe_debug_gemv_int4(const uint8_t* q_dev, const uint16_t* s_dev,
                               int rows, int cols, const float* x_dev,
                               float* y_dev, void* stream);

/* Host-side fault injection for tests of the error paths (nothing is
 * injected unless armed; one armed fault at a time, process-wide):
 *   MOE_FAULT_CACHE_ALLOC  the n-th later device allocation of
 *                          moe_cache_create fails (as cudaErrorMemoryAllocation)
 *   MOE_FAULT_CACHE_COPY   the n-th later host -> device copy enqueue of
 *                          moe_cache_acquire fails (as cudaErrorInvalidValue)
 *   MOE_FAULT_CACHE_STALL  the next moe_cache_acquire that copies holds its
 *                          copy stream for n ms first (a host function)
 *   MOE_FAULT_NONE         disarm
 * No GPU work is faulted: the failures are return codes the library makes
 * up on the host. */
typedef enum {
  MOE_FAULT_NONE = 0,
  MOE_FAULT_CACHE_ALLOC = 1,
  MOE_FAULT_CACHE_COPY = 2,
  MOE_FAULT_CACHE_STALL = 3
} moe_fault;
moe_status moe_debug_inject_fault(int kind, int n);

const char* moe_status_string(moe_status s);
/* Text of the last failure on the calling thread ("" if none). */
const char* moe_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
