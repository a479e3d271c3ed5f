/*
 * duolm.h -- C ABI of the DuoLM multi-item-scoring (MIS) ranker on B200.
 *
 * The library scores the K candidates of each request with a Qwen3-style
 * ranker: request tokens are embedded through a virtual-id lookup, the shared
 * prefix of each request is computed once, every candidate branch attends to
 * that prefix and to itself only (tree mask, unified logical position), and a
 * shared linear head reads one score per candidate.  Sources:
 *   DuoLM summary page (paper.rainbus.top, "DuoLM:基于语言模型的快速高效个性化推荐框架"),
 *   sections 核心方法 (ranker and score head s = w^T h), 方法步骤详情 steps 3-5
 *   (FP16 item table addressed by virtual id V + i; shared prefix prefilled
 *   once; candidate j sees only the prefix and itself at logical position L_q;
 *   scores in input order; CUDA Graph replay), 研究动机 (s^MIS = s),
 *   未来方向 (3) (history appended within a session adds only its own K/V:
 *   the prefix KV store and duolm_prepare_cached).  The request compiler
 *   (duolm_compile) builds the token sequences of step 3 from item ids and
 *   feedback on the host.
 *
 * Conventions for every call:
 *   - Return 0 on success, a negative DUOLM_E_* code on failure; the text of
 *     the last failure is in duolm_last_error(ctx).
 *   - Pointers documented as "host" are read (or written) only during the
 *     call and stay owned by the caller.  The library owns all device memory
 *     it allocates and frees it in duolm_destroy.
 *   - A context is bound to one device and one CUDA stream and is not
 *     thread-safe: use one context per stream.
 *   - Calls that return results to host memory synchronise the context's
 *     stream before returning.
 */
#ifndef DUOLM_H
#define DUOLM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DUOLM_OK 0
#define DUOLM_E_ARG (-1)       /* null pointer, bad size, bad mode or descriptor */
#define DUOLM_E_ID (-2)        /* a token id is negative or >= vocab + table rows */
#define DUOLM_E_OFFSETS (-3)   /* offsets do not start at 0 or are not non-decreasing */
#define DUOLM_E_EMPTY (-4)     /* a request with L = 0 or K = 0, or branch_len < 1 */
#define DUOLM_E_CAPACITY (-5)  /* batch larger than the reserved capacity */
#define DUOLM_E_CUDA (-6)      /* a CUDA runtime call failed (text in last_error) */
#define DUOLM_E_DEVICE (-7)    /* a kernel raised the device error flag */
#define DUOLM_E_STATE (-8)     /* call out of order (no table loaded, nothing prepared) */

#define DUOLM_DTYPE_FP32 0     /* fp32 weights, fp32 arithmetic everywhere */
#define DUOLM_DTYPE_BF16 1     /* bf16 weights; fp16 tensor-core operands, fp32 accumulate */

#define DUOLM_MODE_MIS 0          /* shared prefix + tree-masked branches */
#define DUOLM_MODE_INDEPENDENT 1  /* every candidate as its own full sequence */

typedef struct duolm_ctx duolm_ctx;

/* Ranker shape.  Requirements: d % 8 == 0 and d <= 2048; n_q_heads % n_kv_heads
 * == 0; head_dim even.  FP32 models: head_dim % 32 == 0 and head_dim <= 256.
 * BF16 models: head_dim == 128, d % 256 == 0, ffn % 128 == 0,
 * n_q_heads / n_kv_heads in {1, 2, 4}, n_q_heads + 2 * n_kv_heads even.
 * Violations fail with DUOLM_E_ARG. */
typedef struct {
    int n_layers, d, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
    float rope_theta, rms_eps;
    int dtype; /* DUOLM_DTYPE_* */
} duolm_model_desc;

/* Number of weight tensors duolm_model_load expects: 1 + 11 * n_layers + 2. */
int duolm_weight_count(const duolm_model_desc *desc);

/*
 * Create a context on `device` and copy the ranker weights to it.
 * host_weights: duolm_weight_count(desc) host pointers, each to a row-major
 *   tensor of the descriptor's dtype (uint16 bfloat16 bit patterns for BF16,
 *   float for FP32), in this order:
 *     embed [vocab][d];
 *     per layer: attn_norm [d], wq [n_q_heads*head_dim][d],
 *       wk [n_kv_heads*head_dim][d], wv [n_kv_heads*head_dim][d],
 *       q_norm [head_dim], k_norm [head_dim], wo [d][n_q_heads*head_dim],
 *       mlp_norm [d], w_gate [ffn][d], w_up [ffn][d], w_down [d][ffn];
 *     final_norm [d], head [d].
 *   Matrices are [out_features][in_features].
 * cuda_stream: a cudaStream_t to run on, or NULL for a stream owned by the
 *   context.
 * For BF16 weights each matrix is stored on the device as FP16 times a
 * power-of-two scale chosen per matrix so that every bfloat16 value converts
 * exactly; a matrix that cannot be converted exactly fails with DUOLM_E_ARG.
 * On success *out holds the context; on failure *out is NULL.
 */
int duolm_model_load(const duolm_model_desc *desc, const void *const *host_weights, int device,
                     void *cuda_stream, duolm_ctx **out);

/*
 * Replace the virtual-id item table D with host FP16 rows (uint16 IEEE
 * binary16 bit patterns), row-major [n_items][d].  Ranker id vocab + i then
 * reads row i (DuoLM summary page, 方法步骤详情 step 3).  Synchronous.
 */
int duolm_vid_table_load(duolm_ctx *ctx, const uint16_t *fp16_rows, int64_t n_items);

/*
 * Build the item table on the device from raw encoder outputs through the
 * continuous interface z_i = e^gamma * rho * a_i / RMS(a_i), RMS without
 * epsilon, computed in fp64 and rounded to FP16 to nearest even (DuoLM
 * summary page, 前置知识 "连续输入接口" and 核心方法).
 * a_rows: host float [n_items][d].  Synchronous.
 */
int duolm_vid_table_build(duolm_ctx *ctx, const float *a_rows, int64_t n_items, double gamma,
                          double rho);

/* Reference scale rho of the interface estimated from the loaded embedding:
 * the mean over vocabulary rows of each row's RMS, in fp64.  Synchronous. */
int duolm_embedding_rho(duolm_ctx *ctx, double *rho_out);

/*
 * Reserve device workspace for batches of up to max_tokens packed tokens,
 * max_requests requests and max_candidates candidates (after expansion:
 * independent mode turns each candidate into a request of one candidate).
 * Optional: duolm_prepare grows the workspace on demand, which frees and
 * reallocates device memory and re-captures the CUDA graph.
 */
int duolm_reserve(duolm_ctx *ctx, int64_t max_tokens, int64_t max_requests, int64_t max_candidates);

/*
 * Validate and stage one batch.  Request q has prefix
 * prefix_ids[prefix_offsets[q] .. prefix_offsets[q+1]) (L_q >= 1 tokens) and
 * candidates cand_offsets[q] .. cand_offsets[q+1]) (K_q >= 1); candidate c
 * has branch tokens branch_ids[c*branch_len .. (c+1)*branch_len), the last of
 * which is scored.  All pointers are host; offsets have n_requests + 1
 * entries and start at 0.  mode is DUOLM_MODE_*.
 * The packed layout, position ids and attention work list are built on the
 * host and copied to the device on the context stream (asynchronously: the
 * host buffers may be reused as soon as the call returns).
 * In independent mode the batch must fit the reserved capacity after
 * expansion (K_q * (L_q + b) tokens per request); otherwise DUOLM_E_CAPACITY.
 */
int duolm_prepare(duolm_ctx *ctx, int n_requests, const int32_t *prefix_ids,
                  const int64_t *prefix_offsets, const int32_t *branch_ids,
                  const int64_t *cand_offsets, int branch_len, int mode);

/*
 * Prefix KV reuse (incremental history append; DuoLM summary page, 未来方向
 * (3): when new history items arrive only their vectors and K/V are added).
 * A causal prefix's K/V at every layer depend only on the tokens before
 * them, so a request can start from the K/V an earlier call computed for
 * the first c tokens of its prefix and run only the tokens after them; its
 * scores are those of the whole sequence.
 *
 * duolm_kv_store_reserve: allocate the store, n_slots slots of slot_tokens
 * token rows (K and V of every layer and KV head; 2 * n_layers * n_kv_heads
 * * head_dim * element size bytes per row: 112 KB for the Qwen3-0.6B
 * shape in fp16).  Frees any previous store and its contents (every slot
 * length back to 0), drops the prepared batch and the CUDA graph;
 * n_slots = 0 frees the store.  Synchronous.  DUOLM_E_ARG for negative
 * sizes or slot_tokens above the position limit (32,768), DUOLM_E_CAPACITY
 * above 2^31 rows per layer, DUOLM_E_CUDA when the memory is not there.
 */
int duolm_kv_store_reserve(duolm_ctx *ctx, int n_slots, int slot_tokens);

/* Tokens whose K/V slot `slot` holds (DUOLM_E_ARG for a bad slot). */
int duolm_kv_slot_length(const duolm_ctx *ctx, int slot);

/*
 * duolm_prepare in multi-item mode with per-request prefix reuse.  For
 * request q (host arrays of n_requests entries):
 *   slot[q] = -1: as in duolm_prepare (cached[q] and keep[q] must be 0);
 *   slot[q] = s >= 0: the first cached[q] tokens of the request's prefix
 *     are the first cached[q] tokens slot s holds (cached[q] <= the slot's
 *     length); prefix_ids holds only the L_q tokens after them (L_q may be 0
 *     when cached[q] > 0: new candidates for an unchanged prefix), at
 *     positions cached[q] .. cached[q] + L_q - 1, and the branches sit at
 *     position cached[q] + L_q.  The first keep[q] (0 <= keep[q] <= L_q) of
 *     the new tokens are appended to the slot: once the batch has run, the
 *     slot holds cached[q] + keep[q] tokens (keep[q] = 0 leaves it as it
 *     is).  A trailing header is usually left out of keep so that the next
 *     call can append history before it.
 * A slot that a request of the batch appends to may not be used by any
 * other request of the same batch.  Errors as duolm_prepare, plus
 * DUOLM_E_STATE (no store reserved, or cached[q] above the slot's length),
 * DUOLM_E_ARG (bad slot, cached, keep or sharing), DUOLM_E_CAPACITY
 * (cached[q] + keep[q] above slot_tokens).
 */
int duolm_prepare_cached(duolm_ctx *ctx, int n_requests, const int32_t *prefix_ids,
                         const int64_t *prefix_offsets, const int32_t *branch_ids,
                         const int64_t *cand_offsets, int branch_len, const int32_t *slot,
                         const int32_t *cached, const int32_t *keep);

/* duolm_prepare_cached + duolm_execute + scores to the host + duolm_sync. */
int duolm_score_cached(duolm_ctx *ctx, int n_requests, const int32_t *prefix_ids,
                       const int64_t *prefix_offsets, const int32_t *branch_ids,
                       const int64_t *cand_offsets, int branch_len, const int32_t *slot,
                       const int32_t *cached, const int32_t *keep, float *scores_out);

/*
 * Run the ranker on the prepared batch, asynchronously on the context
 * stream.  Scores (fp32, one per candidate, input order) land in the device
 * buffer returned by duolm_scores_device.  Uses the CUDA graph unless
 * disabled with duolm_set_graph(ctx, 0).
 */
int duolm_execute(duolm_ctx *ctx);

/* Device pointer to the scores of the last duolm_execute ([n_candidates] fp32). */
const float *duolm_scores_device(const duolm_ctx *ctx);

/* Synchronise the context stream and check the device error flag. */
int duolm_sync(duolm_ctx *ctx);

/*
 * One whole call: prepare + execute + copy the scores to host memory
 * (scores_out: host float [cand_offsets[n_requests]]) + synchronise.  This is
 * the request-level operation of the DuoLM summary page (paper.rainbus.top),
 * 方法步骤详情 step 4: the K candidates of a request are packed behind its
 * shared prefix, the prefix is prefilled once, each candidate sees only the
 * prefix and its own branch at the unified logical positions, and the K
 * scores s = w^T h come back in input order.  Arguments as duolm_prepare;
 * scores_out is caller-owned host memory, written before the call returns.
 * Errors as duolm_prepare and duolm_execute, plus DUOLM_E_DEVICE when a
 * kernel raised the device error flag.
 */
int duolm_score(duolm_ctx *ctx, int n_requests, const int32_t *prefix_ids,
                const int64_t *prefix_offsets, const int32_t *branch_ids,
                const int64_t *cand_offsets, int branch_len, int mode, float *scores_out);

/* Launch through a captured CUDA graph (1, default) or kernel by kernel (0). */
int duolm_set_graph(duolm_ctx *ctx, int enabled);

/* Programmatic dependent launch between the pass's kernels (1, default):
 * each kernel after the first may be scheduled while its predecessor
 * finishes and runs its prologue (barrier set-up, tensor-memory allocation)
 * before waiting for the predecessor's results; 0 launches every kernel
 * after its predecessor has completed.  Results are the same either way. */
int duolm_set_pdl(duolm_ctx *ctx, int enabled);

/* Number of kernel launches one duolm_execute issues for the prepared batch
 * (graph nodes when the graph is used). */
int64_t duolm_launches_per_execute(const duolm_ctx *ctx);

/* Text of the last failure on this context ("" if none).  Valid until the
 * next call on the context.  With ctx == NULL: the reason the calling
 * thread's last context-free call (duolm_model_load, duolm_compile) failed. */
const char *duolm_last_error(const duolm_ctx *ctx);

/* Free every device resource of the context (NULL is ignored). */
void duolm_destroy(duolm_ctx *ctx);

/* Template text of one ranker prompt format (see duolm_compile). */
typedef struct {
  int32_t vocab;                 /* V: the VID of table row i is V + i */
  int32_t marker;                /* token before each history item's VIDs */
  int32_t m;                     /* table rows per item (1: one vector per item) */
  const int32_t *instr;          /* instruction tokens at the start of every prefix */
  int32_t n_instr;
  const int32_t *header;         /* tokens after the history, ending the prefix */
  int32_t n_header;
  const int32_t *branch_header;  /* tokens before a candidate's VIDs in its branch */
  int32_t n_branch_header;
} duolm_template;

/*
 * duolm_compile -- build the packed layout of duolm_prepare / duolm_score
 * from request records, on several host threads (DuoLM summary page,
 * 方法步骤详情 step 3: requests carry item ids and feedback, the runtime
 * builds the token sequence; the pages name this input compilation as the
 * host bottleneck at high request rates).  Needs no context and no GPU.
 * Request r's prefix is
 *   instr, then for each of its history items h: marker, the VIDs
 *   V + h m .. V + h m + m - 1, the feedback tokens of h; then header;
 * its candidates c each get a branch of branch_len = n_branch_header + m
 * tokens: branch_header, then the VIDs V + c m .. V + c m + m - 1.
 *   hist_items [hist_offsets[n_requests]] (int64), hist_offsets [n_requests + 1];
 *   feedback [feedback_offsets[H]] (int32 tokens < V), feedback_offsets
 *     [H + 1] with H = hist_offsets[n_requests] (one entry per history item);
 *   cand_items [cand_offsets[n_requests]], cand_offsets [n_requests + 1]
 *     (every request has at least one candidate);
 *   n_items: table items (ids must be < n_items); n_threads > 0: that many
 *     worker threads (at most n_requests and the host's hardware threads),
 *     <= 0: one per 256K output tokens, at most the host's hardware threads.
 * Output (caller-owned host arrays): prefix_ids [prefix_capacity] and
 * prefix_offsets [n_requests + 1]; branch_ids [branch_capacity], candidate
 * c's branch at c * branch_len (the candidate offsets are cand_offsets).
 * Returns DUOLM_E_ARG (null pointers, bad template), DUOLM_E_OFFSETS,
 * DUOLM_E_EMPTY (a request without candidates), DUOLM_E_ID (an item, token
 * or template id out of range; the outputs are then incomplete),
 * DUOLM_E_CAPACITY (an output array too small; nothing written but
 * prefix_offsets).  duolm_last_error(NULL) holds the reason.
 */
int duolm_compile(const duolm_template *tpl, int n_requests, const int64_t *hist_items,
                  const int64_t *hist_offsets, const int32_t *feedback, const int64_t *feedback_offsets,
                  const int64_t *cand_items, const int64_t *cand_offsets, int64_t n_items, int n_threads,
                  int32_t *prefix_ids, int64_t prefix_capacity, int64_t *prefix_offsets, int32_t *branch_ids,
                  int64_t branch_capacity);

/*
 * duolm_compile for requests that continue a prefix in the KV store
 * (incremental history append, see duolm_prepare_cached).  hist_cached[r]
 * (host, n_requests entries): -1 for a request that does not use the store
 * (compiled whole; cached_out 0, keep_out 0); h >= 0 when its slot holds the
 * instruction and its first h history items (h = 0: the slot is empty).
 * Only the rest is compiled: for h > 0 the prefix is history items h.. and
 * the header, for h = 0 the instruction, every history item and the header.
 * cached_out[r] receives the tokens the slot holds (the instruction and the
 * first h items; 0 for h = 0), keep_out[r] the new prefix tokens to append
 * (everything but the header), both ready for duolm_prepare_cached.
 * Errors as duolm_compile (on DUOLM_E_CAPACITY cached_out and keep_out are
 * not written either); DUOLM_E_ARG also for h outside -1..items.
 */
int duolm_compile_append(const duolm_template *tpl, int n_requests, const int64_t *hist_items,
                         const int64_t *hist_offsets, const int32_t *feedback,
                         const int64_t *feedback_offsets, const int64_t *cand_items,
                         const int64_t *cand_offsets, int64_t n_items, int n_threads,
                         const int32_t *hist_cached, int32_t *prefix_ids, int64_t prefix_capacity,
                         int64_t *prefix_offsets, int32_t *branch_ids, int64_t branch_capacity,
                         int32_t *cached_out, int32_t *keep_out);

/*
 * duolm_gather -- the hot path's first step alone: the virtual-id gather of
 * the ranker's inputs (DuoLM summary page, 方法步骤详情 step 3: an id below
 * the vocabulary V reads the embedding, id V + i reads row i of the FP16 item
 * table) with what the gather writes for the first layer's norm, for n ids
 * already in device memory.  Lets the gather be measured on its own (for
 * example over millions of lookups of a large table) and checked row by row.
 *   ids:  device int32 [n], each in [0, V + n_items); read only.  An id out of
 *         range raises the device error flag (reported by the next
 *         duolm_sync as DUOLM_E_DEVICE) and its row is written as zeros.
 *   x:    device float [n][d]: the gathered rows (fp32; the fp16 table and
 *         bf16 embedding values are exact in fp32).
 *   xg:   device uint16 [n][d]: fp16 bit patterns of x times the first
 *         layer's attention-norm gain.
 *   ssp:  device float [n][d / 64]: per row, slot 0 holds the sum of x^2 and
 *         the other slots 0.
 * All buffers belong to the caller.  The work is queued on the context's
 * stream and the call returns without waiting (duolm_sync waits and checks
 * the error flag).  Returns DUOLM_E_ARG for n < 0, n > INT32_MAX or a null
 * pointer with n > 0; DUOLM_E_STATE for an fp32 model (its gather normalises
 * in place instead).
 */
int duolm_gather(duolm_ctx *ctx, const int32_t *ids, int64_t n, float *x, uint16_t *xg, float *ssp);

/* Largest vocabulary duolm_embedding_rho_static accepts (rows of its
 * built-in scratch array: 2 MB of fp64, held by every GPU that loads the
 * library until the process exits). */
#define DUOLM_RHO_STATIC_MAX_ROWS 262144

/*
 * duolm_embedding_rho_static -- the reference scale rho of duolm_embedding_rho
 * (mean over embedding rows of each row's RMS, fp64) for callers that must
 * not allocate device memory.  The paper has no counterpart: it is a
 * deployment aid.  Some callers cannot call cudaMalloc: a serving process
 * that has already carved all of the GPU's memory into its own pools gets an
 * out-of-memory failure or a fragmented pool from a fresh allocation, and a
 * latency-critical loop cannot afford an allocation that may wait for the
 * whole device.  This entry point allocates nothing: its per-row scratch is a
 * fixed array of DUOLM_RHO_STATIC_MAX_ROWS doubles built into the library.
 *   embed:  device pointer to the embedding, [vocab][d] row-major, uint16
 *           bfloat16 bit patterns (dtype DUOLM_DTYPE_BF16) or float
 *           (DUOLM_DTYPE_FP32); read only.
 *   rho_out: device pointer to one double; written by the call.
 *   cuda_stream: the cudaStream_t to launch on (NULL: the default stream).
 * The call only enqueues work on the stream of the current device and
 * returns; rho_out is valid once that stream has reached it.  Outside stream
 * capture every call looks up the scratch array's device address with the
 * device current (so a reset device or a new context is followed); while the
 * stream is being captured the address from the last call outside capture
 * on that device is used, so make the first call on each device before any
 * stream capture (DUOLM_E_STATE otherwise).  Every element of the scratch a
 * call reads is first written by the same call, so nothing needs clearing,
 * but all calls in the process share the one array: calls whose work
 * overlaps on the GPU (different streams, no ordering between them) race and
 * may return wrong results.  A CUDA error left pending by earlier work is
 * reported (DUOLM_E_CUDA) before anything is enqueued.  Returns 0;
 * DUOLM_E_ARG for a null pointer, d < 1 or a bad dtype; DUOLM_E_CAPACITY when
 * vocab is < 1 or above DUOLM_RHO_STATIC_MAX_ROWS; DUOLM_E_CUDA when the
 * address lookup or a launch fails; the reason in duolm_last_error(NULL).
 */
int duolm_embedding_rho_static(const void *embed, int dtype, int64_t vocab, int d, double *rho_out,
                               void *cuda_stream);

/* ---- introspection (tests) --------------------------------------------- */

/* Packed layout of the prepared batch as the device holds it: n_tokens,
 * and per token its ranker id and position id (host int32 [n_tokens] each;
 * either may be NULL).  Synchronous. */
int duolm_debug_layout(duolm_ctx *ctx, int64_t *n_tokens, int32_t *ids_out, int32_t *pos_out);

/* Evaluate, on the device, the attention kernels' visibility predicate for
 * every (query token, key token) pair of request q of the prepared batch:
 * out is host uint8 [T_q][T_q], T_q = L_q + K_q * b.  Synchronous. */
int duolm_debug_mask(duolm_ctx *ctx, int request, uint8_t *out);

/* Run the embedding and the first n_layers layers of the prepared batch and
 * copy the fp32 residual stream out (host float [n_tokens][d]).  n_layers = 0
 * gives the looked-up rows.  Synchronous. */
int duolm_debug_residual(duolm_ctx *ctx, int n_layers, float *x_out);

/*
 * The attention work list duolm_prepare builds on the tensor-core path, for
 * a batch described by its request sizes alone (host only, no context, no
 * GPU).  Request r has a whole prefix of L[r] tokens, cached[r] of them from
 * the prefix KV store, and K[r] candidates of branch_len tokens.  Writes
 * items [cap_items][4] = {request, KV head, kind (1: whole candidate
 * branches from branch row `row`; 0: prefix rows from `row`), row} and
 * cta_off [n_ctas + 1] (CTA c runs items cta_off[c] .. cta_off[c+1] - 1).
 * Returns the item count, DUOLM_E_CAPACITY when above cap_items, DUOLM_E_ARG.
 */
int64_t duolm_debug_attention_plan(int n_requests, const int32_t *L, const int32_t *K,
                                   const int32_t *cached, int branch_len, int n_kv_heads,
                                   int rows_per_item, int n_ctas, int32_t *items, int64_t cap_items,
                                   int32_t *cta_off);

/* Copy the device item table out (host uint16 [n_items][d]).  Synchronous. */
int duolm_debug_table(duolm_ctx *ctx, uint16_t *out, int64_t n_items);

/* Bytes the last duolm_prepare / duolm_prepare_cached copied host ->
 * device (the packed plan and the per-request cached-prefix records). */
int64_t duolm_plan_bytes(const duolm_ctx *ctx);

/*
 * One projection of layer `layer` through the tensor-core GEMM alone
 * (BF16 models only): out = a * W^T with W = wqkv (which 0, [qd+2kd][d]),
 * wo (1, [d][qd]), gate/up (2, [2*ffn][d], rows in 128-row blocks alternating
 * gate and up) or w_down (3, [d][ffn]); which + 4 computes the same product
 * as four K-slices summed by the split-K reduction small batches use for the
 * O and down projections.  a: host uint16 fp16 bit patterns
 * [n_tokens][K] where n_tokens is the prepared batch's token count; out: host
 * float [n_tokens][N].  Overwrites the batch's activations.  Synchronous.
 */
int duolm_debug_gemm(duolm_ctx *ctx, int layer, int which, const uint16_t *a, float *out);

/*
 * Failure-detection self test: launch one kernel that waits on an mbarrier
 * nothing ever arrives on, through the same bounded wait the GEMM kernels
 * use.  The wait gives up after its time limit (2 s), records
 * "wait-timeout" in the device status word and returns; the call then
 * returns DUOLM_E_DEVICE and the context stays usable.
 */
int duolm_debug_wait_timeout(duolm_ctx *ctx);

/* Kernel classes of duolm_profile. */
#define DUOLM_PROF_EMBED 0
#define DUOLM_PROF_GEMM_QKV 1
#define DUOLM_PROF_ATTENTION 2
#define DUOLM_PROF_GEMM_O 3
#define DUOLM_PROF_RMSNORM 4
#define DUOLM_PROF_GEMM_GATE_UP 5
#define DUOLM_PROF_GEMM_DOWN 6
#define DUOLM_PROF_HEAD 7
#define DUOLM_PROF_KV_APPEND 8
#define DUOLM_PROF_N 9

/*
 * Run the prepared batch n_steps times kernel by kernel with a CUDA event
 * after every launch, and return per kernel class the summed device time in
 * ms (ms_out[DUOLM_PROF_N]) and the number of launches (count_out).
 * Synchronous; the scores of the last step are left as by duolm_execute.
 */
int duolm_profile(duolm_ctx *ctx, int n_steps, double *ms_out, int64_t *count_out);

#ifdef __cplusplus
}
#endif
#endif /* DUOLM_H */
