/*
 * moe_route.h -- C ABI of the B200 (sm_100a) MoE routing library.
 *
 * The library computes, on one GPU, the Mixture-of-Experts routing hot path
 * described by these pages (cited by title and section):
 *   [TE]  Implementation:NVIDIA TransformerEngine Fused Router
 *   [TRT] flashinfer.fused_moe.trtllm_gen_routing
 *   [NKI] RMSNorm Router Top-K A2AV Kernel API Reference
 *   [LMD] Implementation:InternLM Lmdeploy Gemm MoeUtils
 *   [MAX] max.nn.moe.SigmoidTopKRouter
 *
 * Conventions for every entry point:
 *   - Buffers are caller-owned.  Pointers named as device pointers must point
 *     to device memory of the current CUDA device; the library never
 *     allocates, frees or synchronises (except moe_status, which reads one
 *     word back).  Tensors are row-major with the last dimension contiguous.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call is asynchronous and stream-ordered.
 *   - Arguments are validated before any launch; a failed check returns a
 *     negative MOE_ERR_* code and launches nothing.  MOE_ERR_CUDA reports a
 *     launch failure (cudaGetLastError after the launch).
 *   - Every device-side wait (on a kernel's own bulk copies or tensor-core
 *     operations) is bounded; on expiry the kernel records
 *     MOE_ERR_DEVICE_TIMEOUT in the status word at the start of its
 *     workspace and returns, leaving outputs undefined.  Read it with
 *     moe_status().  No kernel waits on another thread block.
 *   - A workspace must be zero-filled once before its first use
 *     (moe_workspace_init or any memset); the library leaves it consistent
 *     for the next call.  One workspace serves one stream at a time: calls
 *     that may overlap on the GPU need separate workspaces.
 *   - Inputs must be finite (no NaN or Inf logits or hidden states) unless an
 *     entry point states otherwise (moe_aux_scores).
 */
#ifndef MOE_ROUTE_H
#define MOE_ROUTE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)    /* an argument breaks a documented constraint */
#define MOE_ERR_UNSUPPORTED (-2)    /* valid per the pages but outside this build's limits */
#define MOE_ERR_WORKSPACE (-3)      /* workspace missing or smaller than required */
#define MOE_ERR_CUDA (-4)           /* a CUDA runtime call or launch failed */
#define MOE_ERR_DEVICE_TIMEOUT (-5) /* a bounded device-side wait expired (status word) */
#define MOE_ERR_DEVICE_BOUNDS (-6)  /* a kernel's own bounds check skipped an out-of-range index
                                       (status word; indicates a library bug; outputs undefined) */

/* ---- element types and score functions ---- */
#define MOE_F32 0
#define MOE_BF16 1
#define MOE_SOFTMAX 0
#define MOE_SIGMOID 1

/* Limits of this build. */
#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOPK 32

/*
 * Parameters of one routing call.  Field meanings follow [TE: Signature,
 * I/O Contract], [TRT: Parameters] and [MAX: steps 1-4].
 */
typedef struct moe_route_params {
  int32_t num_tokens;          /* T >= 0 */
  int32_t num_experts;         /* E, 1..MOE_MAX_EXPERTS */
  int32_t top_k;               /* k, 1..min(E, MOE_MAX_TOPK) [TE: topk; TRT: top_k] */
  int32_t score_fn;            /* MOE_SOFTMAX | MOE_SIGMOID [TE: score_function] */
  int32_t softmax_before_topk; /* 1: score, then top-k on score (+bias) [TE: use_pre_softmax];
                                  0: top-k on logit (+bias), then the score function over the
                                  k selected (softmax over the k, or sigmoid each) */
  int32_t n_group;             /* grouped routing; n_group <= 1 or topk_group == 0 disables
                                  [TRT: n_group, topk_group; TE: num_groups, group_topk] */
  int32_t topk_group;          /* groups kept per token */
  int32_t group_score_topn;    /* a group's score = sum of its top-n keys; 1 or 2 */
  int32_t renormalize;         /* selected weights divided by their sum [TRT: norm_topk_prob;
                                  MAX: norm_topk_prob] */
  float scaling_factor;        /* weights times this [TRT: routed_scaling_factor; TE:
                                  scaling_factor] */
  int32_t tile_tokens_dim;     /* power of two, 1..4096 [TRT: tile_tokens_dim] */
  int32_t logits_dtype;        /* MOE_F32 | MOE_BF16 [TRT: routing_logits] */
  int32_t bias_dtype;          /* MOE_F32 | MOE_BF16 [TRT: routing_bias] */
  int32_t weights_dtype;       /* MOE_F32 | MOE_BF16 [TRT: Notes, topk_weights dtype] */
  int32_t local_expert_offset; /* expert-parallel shard: the experts [local_expert_offset,   */
  int32_t local_num_experts;   /* local_expert_offset + local_num_experts) are local; 0 (with
                                  offset 0) = all E [TRT: local_expert_offset, local_num_experts].
                                  Selection and weights stay global; counts, offsets, slots and
                                  tiles cover the local experts only (tile_expert = local index,
                                  global expert = it + local_expert_offset [TRT: Notes]); a
                                  selection of another shard's expert gets
                                  expanded_to_permuted = -1 */
  int32_t num_fused_shared_experts; /* S >= 0 [TRT: num_fused_shared_experts -- extra fused
                                  shared-expert slots appended per token].  Each token's S slots
                                  follow its k routed ones: expert E + s, weight 1.0 (outside
                                  selection, renormalisation and scaling); every token selects
                                  every shared expert; the shared experts are local on every
                                  shard, after its routed experts (local index L + s).  The
                                  outputs then hold k + S slots per token and L + S local
                                  experts; E + S <= MOE_MAX_EXPERTS, k + S <= MOE_MAX_TOPK */
} moe_route_params;

/* Human-readable name of a status code (static string). */
const char* moe_error_string(int code);

/* Zero-fill `bytes` of workspace on `stream` (what a workspace needs once). */
int moe_workspace_init(void* ws, size_t bytes, void* stream);

/*
 * Read and optionally clear the status word at the start of a workspace.
 * Synchronises `stream`.  *status receives MOE_OK or MOE_ERR_DEVICE_TIMEOUT.
 */
int moe_status(void* ws, void* stream, int32_t* status, int clear);

/*
 * Upper bounds for the permutation outputs of moe_route:
 *   max_padded = T*k' + min(E + S, T*k') * (tile - 1)   (rows of permuted_to_token;
 *                k' = k + S slots per token, S fused shared experts)
 *   max_tiles  = max_padded / tile                (entries of the tile tables)
 * [TRT: tile_tokens_dim -- each expert's rows are padded to the tile].
 */
int moe_route_capacity(const moe_route_params* p, int64_t* max_padded, int64_t* max_tiles);

/* Workspace bytes moe_route needs on the current device for these parameters. */
int moe_route_workspace_bytes(const moe_route_params* p, size_t* bytes);

/*
 * moe_route -- expert selection, routing weights and permutation bookkeeping
 * [TE: Description, fused_topk_with_score_function; TRT: standalone routing
 * (expert selection + permutation), Returns, Notes; MAX: steps 2-4; LMD:
 * invokeMoeGate_V2].
 *
 * Per token t:
 *   score   s_e = softmax(logits_t)_e, sigmoid(logit_te), or the logit itself
 *                 when softmax_before_topk == 0; computed in fp32
 *   key     s_e + bias_e (bias only selects; NULL = no bias)
 *   groups  (optional) experts in n_group contiguous groups; group score =
 *           sum of its group_score_topn largest keys; the topk_group best
 *           groups (ties -> lower group) stay selectable
 *   top-k   the k largest keys, ties -> lower expert index; slot order =
 *           descending key
 *   weight  w_j = v_j / sum(v) * scale (renormalize) or v_j * scale, where v_j
 *           is the selected expert's unbiased score (softmax_before_topk == 0:
 *           the score function applied to the k selected logits)
 * Bookkeeping over all T*k selections (token-major order), for the local
 * experts e = local_expert_offset + le, le < L = local_num_experts (all E
 * when local_num_experts == 0):
 *   expert_counts[le]         rows routed to e
 *   padded_offsets[le]        exclusive prefix of ceil(count/tile)*tile; [L] = P
 *   expanded_to_permuted[i]   row of selection i = t*k + j in the expert-
 *                             contiguous padded layout; rows of one expert
 *                             follow token order; -1 when the selected
 *                             expert is not local
 *   permuted_to_token[p]      source token of row p, -1 on padding rows (p < P)
 *   tile_expert[c]            local expert le of tile c (rows c*tile ..
 *                             c*tile+tile-1)
 *   tile_mn_limit[c]          exclusive end of tile c's valid rows
 *   totals[0] = P (total_num_padded_tokens), totals[1] = P / tile
 *                             (num_non_exiting_ctas); device-resident, so a
 *                             consumer sized for the capacity can exit early
 * Entries of permuted_to_token at or past P, and of the tile tables at or past
 * P/tile, are not written.
 *
 * Device pointers (caller-owned):
 *   logits [T,E] (logits_dtype), bias [E] (bias_dtype) or NULL,
 *   topk_ids [T,k] int32, topk_weights [T,k] (weights_dtype),
 *   expert_counts [L], padded_offsets [L+1], expanded_to_permuted [T*k],
 *   permuted_to_token [max_padded], tile_expert [max_tiles],
 *   tile_mn_limit [max_tiles], totals [2] -- all int32,
 *   ws [ws_bytes] from moe_route_workspace_bytes (zero-filled before first use).
 * Two launches chained by programmatic dependent launch: a selection kernel
 * (one block per contiguous token segment) writes ids and weights, a count
 * table row per segment and each selection's rank in its segment; a
 * bookkeeping kernel turns them into slots, offsets and tile tables.  The
 * bias is read before waiting on the preceding kernel: a preceding kernel that
 * lets its dependents start early must not write it (the logits are read after
 * the wait).  The sigmoid fast path (E = 8 * {8, 16, 32} bf16 or {8, 16} fp32
 * logits, 16-byte aligned, k <= 8, ungrouped or 8 groups with 2 * topk_group
 * >= k) chooses candidates with an approximate key whose error bound is
 * checked exhaustively by the test suite, and computes every key that can
 * decide the result with the stated fp32 formula.
 * Errors: MOE_ERR_INVALID_ARG (sizes, k > E, tile not a power of two, groups
 * not dividing E, k > topk_group * E / n_group, a local expert range outside
 * [0, E), NULL outputs),
 * MOE_ERR_UNSUPPORTED (E or k past the build limits, a group layout the
 * kernels do not map: with groups, a lane holds v in {2,3,4,5,6,8,12,16,24,32}
 * experts (the least with 32v >= E) and a group must span a power of two of
 * whole lanes or a lane whole groups; k + S past the slot limit or E + S past
 * the expert limit), MOE_ERR_WORKSPACE (ws smaller than
 * moe_route_workspace_bytes), MOE_ERR_CUDA (a launch failed).  Device-side
 * errors (MOE_ERR_DEVICE_TIMEOUT from a bounded wait on a bulk copy) are not
 * returned here: they are recorded in the status word at the start of ws and
 * read with moe_status.
 */
int moe_route(const moe_route_params* p, const void* logits, const void* bias, int32_t* topk_ids,
              void* topk_weights, int32_t* expert_counts, int32_t* padded_offsets,
              int32_t* expanded_to_permuted, int32_t* permuted_to_token, int32_t* tile_expert,
              int32_t* tile_mn_limit, int32_t* totals, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_route_no_alloc -- moe_route for callers that cannot allocate device
 * memory: serving runtimes whose memory manager owns the whole GPU and forbids
 * allocations outside its pool, plugin or custom-op interfaces that provide
 * inputs and outputs but no workspace, plain C callers without a device
 * allocator, and latency-critical paths that cannot pay for cudaMalloc.  (The
 * pages have no counterpart; this is an interface convenience.)
 *
 * Same arguments, results and errors as moe_route, without ws/ws_bytes: the
 * workspace is a library-owned __device__ array of 512 KB that every GPU loading
 * the library holds until the process exits.  Calls needing more (the workspace
 * grows with E and the SM count; moe_route_workspace_bytes reports it) return
 * MOE_ERR_WORKSPACE.  The first call on a device (or the first
 * moe_route_no_alloc_status) does the set-up: it looks up the array's device
 * address (cudaGetSymbolAddress) and zero-fills its 64-byte header on `stream`;
 * make that first call before any stream capture.  A failed set-up returns
 * MOE_ERR_CUDA and is tried again by the next call.  All calls share the one
 * array: calls that may overlap on the GPU (different streams, or several host
 * threads) race and must be serialised by the caller.  The call allocates no
 * device memory.  Device-side status (a bounds check) lands in the array's
 * status word, which later calls keep (sticky, first error wins): read it with
 * moe_route_no_alloc_status.
 */
int moe_route_no_alloc(const moe_route_params* p, const void* logits, const void* bias, int32_t* topk_ids,
                       void* topk_weights, int32_t* expert_counts, int32_t* padded_offsets,
                       int32_t* expanded_to_permuted, int32_t* permuted_to_token, int32_t* tile_expert,
                       int32_t* tile_mn_limit, int32_t* totals, void* stream);

/*
 * moe_route_no_alloc_status -- read the status word of moe_route_no_alloc's
 * library-owned workspace on the current device (MOE_OK or the first
 * MOE_ERR_DEVICE_* recorded since it was last cleared).  Synchronises
 * `stream`; clear != 0 resets it to MOE_OK.  (No counterpart on the pages.)
 */
int moe_route_no_alloc_status(void* stream, int32_t* status, int clear);

/* Workspace bytes of the aux-loss entry points (scores, loss forward). */
int moe_aux_workspace_bytes(int32_t num_tokens, int32_t num_experts, size_t* bytes);

/*
 * moe_aux_scores -- scores and routing map for the load-balancing loss
 * [TE: Description, fused_compute_score_for_moe_aux_loss; Signature].
 *   probs [T,E] fp32      = softmax(logits_t) (MOE_SIGMOID: sigmoid / row sum)
 *   routing_map [T,E] u8  = 1 at the token's k largest probs (ties -> lower e)
 *   tokens_per_expert [E] = column sums of routing_map (int32)
 * logits [T,E] fp32.  All pointers device, caller-owned; ws as above.
 * A logit of -inf (a masked expert) gives a zero prob; a row whose score sum
 * is not finite (a NaN or +inf logit) still marks exactly k experts (probs
 * undefined).
 */
int moe_aux_scores(int32_t T, int32_t E, int32_t k, int32_t score_fn, const float* logits,
                   float* probs, uint8_t* routing_map, int32_t* tokens_per_expert, void* ws,
                   size_t ws_bytes, void* stream);

/*
 * moe_aux_loss_fwd -- load-balancing loss [TE: Description, fused_moe_aux_loss;
 * Signature (probs, tokens_per_expert, total_num_tokens, num_experts, topk,
 * coeff)]:
 *   loss = coeff * E / (T_total * k) * sum_e ( sum_t probs[t,e] ) * tpe[e]
 * probs [T_rows,E] fp32, tokens_per_expert [E] int32, loss: one fp32 on the
 * device.  Deterministic (fixed reduction order).
 */
int moe_aux_loss_fwd(int32_t T_rows, int32_t T_total, int32_t E, int32_t k, float coeff,
                     const float* probs, const int32_t* tokens_per_expert, float* loss, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * moe_route_weights_bwd -- backward of the routed weights [TE: Description,
 * FusedTopkScoreFunction / fused_topk_with_score_function, forward and
 * backward]: dL/dlogits [T,E] fp32 given dL/dweights [T,k] fp32 for the
 * selection topk_ids [T,k] that moe_route returned with the same params
 * (score_fn, softmax_before_topk, renormalize, scaling_factor; logits in
 * logits_dtype).  The selection, the groups and the bias carry no gradient.
 * With v_j the score of slot j (sigmoid of its logit; its softmax probability
 * over all E; or the softmax over the k selected logits when top-k comes
 * first), w_j = scale*v_j (/ sum_i v_i when renormalising):
 *   gv_i = scale*gw_i, or scale/S*(gw_i - sum_j gw_j v_j / S) with S = sum v
 *   sigmoid:       grad[e_j] = gv_j * v_j * (1 - v_j)
 *   softmax first: grad[e]   = p_e * (gv at e - sum_j v_j gv_j), every e
 *   top-k first:   grad[e_j] = v_j * (gv_j - sum_i v_i gv_i)
 * and 0 elsewhere.  k <= 32.  ws (optional, >= 64 bytes) receives
 * MOE_ERR_DEVICE_BOUNDS for an id outside [0, E).  Returns
 * MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED for bad parameters.
 */
int moe_route_weights_bwd(const moe_route_params* p, const void* logits, const int32_t* topk_ids,
                          const float* grad_weights, float* grad_logits, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_aux_scores_bwd -- backward of the aux scores [TE: Description,
 * fused_compute_score_for_moe_aux_loss, forward and backward]: given the
 * upstream gradient with respect to the softmax probs,
 *   grad_logits[t,e] = p[t,e] * (grad_probs[t,e] - sum_j p[t,j] grad_probs[t,j])
 * probs, grad_probs, grad_logits [T,E] fp32 (probs as moe_aux_scores wrote
 * them).  score_fn MOE_SIGMOID returns MOE_ERR_UNSUPPORTED: the sigmoid scores
 * normalised by their row sum need that sum, which the probs do not carry
 * (moe_aux_scores_bwd_logits computes it from the logits).
 * No workspace; returns MOE_ERR_INVALID_ARG for bad sizes or null pointers.
 */
int moe_aux_scores_bwd(int32_t T, int32_t E, int32_t score_fn, const float* probs, const float* grad_probs,
                       float* grad_logits, void* stream);

/*
 * moe_aux_scores_bwd_logits -- backward of the aux scores from the logits
 * [TE: Description, fused_compute_score_for_moe_aux_loss, forward and
 * backward; I/O Contract, score_function "softmax" or "sigmoid"]: the scores
 * are recomputed from the logits as moe_aux_scores computes them, so the
 * sigmoid scores (divided by their row sum) have a backward too:
 *   softmax: p = softmax(x);             grad = p * (g - sum_e p_e g_e)
 *   sigmoid: s = sigmoid(x), S = sum s;  grad = s (1 - s) / S * (g - sum_e p_e g_e)
 * logits, grad_probs (dL/dprobs), grad_logits [T,E] fp32, device,
 * caller-owned; rows may start anywhere (16-byte vectors when aligned).
 * No workspace.  Returns MOE_ERR_INVALID_ARG for bad sizes, an unknown
 * score_fn or null pointers; MOE_ERR_UNSUPPORTED for E > MOE_MAX_EXPERTS.
 */
int moe_aux_scores_bwd_logits(int32_t T, int32_t E, int32_t score_fn, const float* logits,
                              const float* grad_probs, float* grad_logits, void* stream);

/*
 * moe_aux_loss_bwd -- gradient of the loss [TE: Description, forward and
 * backward].  With C = coeff * E / (T_total * k) and g = *grad_loss (device):
 *   grad_probs[t,e]  = g * C * tpe[e]                       (optional, may be NULL)
 *   grad_logits[t,e] = p[t,e] * (grad_probs[t,e] - sum_j p[t,j] grad_probs[t,j])
 *                      (softmax backward; optional, may be NULL)
 * tokens_per_expert is treated as a constant.  No workspace.
 */
int moe_aux_loss_bwd(int32_t T_rows, int32_t T_total, int32_t E, int32_t k, float coeff,
                     const float* grad_loss, const float* probs, const int32_t* tokens_per_expert,
                     float* grad_probs, float* grad_logits, void* stream);

/*
 * moe_dispatch -- gather token rows into the expert-contiguous padded buffer
 * [LMD: invokeMoeDispatch].
 *   out[expanded_to_permuted[t*k+j], :] = hidden[t, :]
 *   out[p, :] = 0 for padding rows p < P (permuted_to_token[p] == -1)
 * Rows at or past P (= totals[0], read on the device) are not written.  Slots
 * whose expanded_to_permuted is negative (another expert-parallel shard's
 * selection) are skipped, and a token with no slot here is not read.
 * hidden [T,H], out [max_padded,H] (dtype MOE_BF16 or MOE_F32),
 * expanded_to_permuted [T*k], permuted_to_token [max_padded], totals [2]: the
 * outputs of moe_route.  H * element size must be a multiple of 16 bytes and
 * hidden/out 16-byte aligned.
 */
int moe_dispatch(int32_t T, int32_t H, int32_t k, int32_t dtype, const void* hidden,
                 const int32_t* expanded_to_permuted, const int32_t* permuted_to_token,
                 const int32_t* totals, int64_t max_padded, void* out, void* stream);

/*
 * moe_combine -- weighted sum of each token's k expert rows back in token
 * order [LMD: invokeMoeCombine, routing scales]:
 *   out[t, :] = round( sum_j w[t,j] * expert_out[expanded_to_permuted[t*k+j], :] )
 * accumulated in fp32 in slot order, stored in `dtype` (bf16: round to
 * nearest even).  Slots whose expanded_to_permuted is negative (another
 * expert-parallel shard's selection) are skipped: they add nothing here.
 * expert_out [max_padded,H], out [T,H] (dtype MOE_BF16 or MOE_F32), weights
 * [T,k] (weights_dtype).  Padding rows of expert_out are never read.  A slot
 * whose expanded_to_permuted is max_padded or more (a stale or mismatched map)
 * is skipped, and when ws (optional, >= 64 bytes, zero-filled before first use)
 * is given MOE_ERR_DEVICE_BOUNDS is recorded in its status word (moe_status).
 * H * element size must be a multiple of 16 bytes and rows 16-byte aligned.
 */
int moe_combine(int32_t T, int32_t H, int32_t k, int32_t dtype, const void* expert_out, int64_t max_padded,
                const int32_t* expanded_to_permuted, const void* weights, int32_t weights_dtype,
                void* out, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_ep_regroup -- the receiving side of an expert-parallel all-to-all-v
 * dispatch (direction 0) and the sending side of its return (direction 1)
 * [NKI: Background -- the router top-k feeds the all-to-all-v MoE dispatch
 * path; TRT: Parameters local_expert_offset / local_num_experts, Returns --
 * the tile-padded expert-contiguous layout; LMD: invokeMoeDispatch /
 * invokeMoeCombine].
 * A world of `world` ranks; this rank owns `local_experts` experts.
 * counts [world][local_experts] int32 (device): rows rank s sends for local
 * expert e.  recv [n_recv, H] holds them ordered by source rank, then expert,
 * then the source's token order, n_recv = sum of counts (what every rank's
 * route over all experts with tile 1, followed by moe_dispatch, sends to this
 * rank).  Direction 0 writes padded [max_padded, H]: the rows ordered by local
 * expert, then source rank, then token, each expert padded to `tile` rows
 * (padding rows zero) -- exactly the layout moe_route gives this rank's
 * experts for all ranks' tokens concatenated in rank order -- and
 * padded_offsets [local_experts + 1], totals [2] (P, P / tile) and
 * padded_to_recv [max_padded] (receive row of each padded row, -1 on padding;
 * rows >= P untouched).  Direction 1 reads padded (the expert outputs in that
 * layout) and writes recv (receive order), for the return all-to-all-v; the
 * offsets, totals and padded_to_recv arguments are ignored.
 * dtype MOE_BF16 | MOE_F32; H * element size a multiple of 16 bytes; recv and
 * padded 16-byte aligned; tile a power of two <= 4096; world * local_experts
 * <= 8192.  If the counts disagree with n_recv, or the padded rows exceed
 * max_padded, nothing is moved and ws (optional, >= 64 bytes) records
 * MOE_ERR_DEVICE_BOUNDS.  Reads the counts after waiting on the preceding
 * kernel (programmatic dependent launch).
 */
int moe_ep_regroup(int32_t world, int32_t local_experts, int32_t H, int32_t dtype, int32_t tile, const int32_t* counts,
                   int32_t direction, void* recv, int64_t n_recv, void* padded, int64_t max_padded,
                   int32_t* padded_offsets, int32_t* totals, int32_t* padded_to_recv, void* ws, size_t ws_bytes,
                   void* stream);

/*
 * Workspace bytes of moe_rmsnorm_router_topk (header and the fp32 partial
 * logits of the K-split projection; depends on T, H and E).  The workspace
 * must be zero before its first use (moe_workspace_init).
 */
int moe_rmsnorm_router_topk_workspace_bytes(int32_t T, int32_t H, int32_t E, size_t* bytes);

/*
 * moe_rmsnorm_router_topk -- fused RMSNorm + router projection + top-k for
 * small decode batches [NKI: Background; Parameters; Returns; Notes].
 *   out_norm[t,h] = bf16( x[t,h] / sqrt(mean_h x[t,h]^2 + eps) * gamma[h] )
 *   logit[t,e]    = sum_h out_norm[t,h] * W[h,e] + bias[e]   (fp32 accumulate,
 *                   tensor cores)
 *   ids[t,:]      = top-k on the raw logits, ties -> lower expert (ACT2:
 *                   activation after top-k)
 *   affinities    = bf16(sigmoid(logit)) at the selected experts (MOE_SOFTMAX:
 *                   softmax over the k selected logits), 0 elsewhere
 * hidden [T,H], gamma [H], W [H,E], bias [E] or NULL, out_norm [T,H],
 * affinities [T,E] -- bf16; ids [T,k] int32; debug_logits [T,E] fp32 or NULL
 * (receives the logits when given).  T <= 128 and H % 128 == 0 [NKI: Notes];
 * this build also needs E % 16 == 0, E <= 1024 and H <= 32768, and every
 * pointer 16-byte aligned.  Three launches chained by programmatic dependent
 * launch: a row-parallel RMSNorm writing out_norm; the projection split over
 * K-slices (one CTA per token group x 64 experts x slice, all resident at
 * once) writing fp32 partial logits to the workspace; a block per token that
 * adds the partials in slice order and takes the top-k.  Each launch reads
 * W, gamma and bias before waiting on its predecessor: a preceding kernel
 * that lets dependents start early must not write them.  Device-side waits
 * are bounded and a wait that gives up leaves MOE_ERR_DEVICE_TIMEOUT in the
 * workspace status word (outputs are then left unwritten).
 * Returns MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE for
 * bad arguments, MOE_ERR_CUDA when the launch fails.  Calls sharing one
 * workspace must not overlap in time.
 */
int moe_rmsnorm_router_topk(int32_t T, int32_t H, int32_t E, int32_t k, float eps, int32_t act,
                            const void* hidden, const void* gamma, const void* W, const void* bias,
                            void* out_norm, int32_t* ids, void* affinities, float* debug_logits,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * Test hook for the bounded waits of the kernels (a wait on a shared-memory
 * barrier, as the kernels wait on their bulk copies): one thread arms a
 * barrier and waits on it for at most timeout_ns.  With never_complete != 0
 * the barrier expects bytes that never arrive, so the wait gives up and the
 * status word of ws (64 bytes) must read MOE_ERR_DEVICE_TIMEOUT afterwards;
 * with 0 it completes at once.  The kernel returns normally either way.
 */
int moe_debug_wait_timeout(int32_t never_complete, int64_t timeout_ns, void* ws, size_t ws_bytes, void* stream);

/*
 * Test hook for the sigmoid fast path of moe_route: for each i writes
 *   err[i]   = proxy(x[i], b[i]) - (sigmoid(x[i]) + b[i])
 *   delta[i] = the error bound the fast path assumes for a block whose
 *              largest |0.5 + bias| is |0.5 + b[i]|
 * where proxy(x, b) = 0.5 * tanh.approx(x / 2) + (0.5 + b) in packed f16 (x
 * rounded to f16, the tanh and the fused multiply-add in f16) is the
 * approximate key that chooses candidates, and sigmoid(x) + b = 1 / (1 +
 * exp(-x)) + b in fp32 is the exact key.  f32_logits selects the bound for
 * fp32 logits (whose rounding to f16 adds to the error).  moe_route assumes
 * |err| <= delta; the tests check |err| <= delta / 2.  x, b, err, delta are
 * device arrays of n floats.
 */
int moe_debug_sigmoid_proxy_error(const float* x, const float* b, int64_t n, int32_t f32_logits, float* err,
                                  float* delta, void* stream);

/*
 * Test hook for the division the aux-scores kernel uses in place of one IEEE
 * division per entry: a / b from the reciprocal 1/b (one IEEE division per
 * row) and two fused-multiply-add corrections (Markstein's method), within
 * its range (a >= 2^-60, 2^-20 <= b <= 2^20).  Counts, into *mismatches
 * (device uint32, zeroed by the caller), the pairs in range whose result
 * differs in any bit from the IEEE quotient a[i] / b[i]; pairs out of range
 * are skipped.  a, b: n device floats.  MOE_ERR_INVALID_ARG for null
 * pointers with n > 0.
 */
int moe_debug_div_check(const float* a, const float* b, int64_t n, uint32_t* mismatches, void* stream);

/*
 * Test hook for moe_route_no_alloc_status: records `code` (negative) in the
 * status word of the no-alloc workspace on the current device, as a kernel's
 * bounds check would (first error wins), without running a route.
 */
int moe_debug_no_alloc_record(int32_t code, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ROUTE_H */
