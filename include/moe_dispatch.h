/*
 * moe_dispatch.h -- C ABI of the B200 (sm_100a) MoE router-and-dispatch library
 * (libmoe_dispatch.so).
 *
 * The path, in call order on one CUDA stream:
 *   moe_gate_gemm  -> fp32 gate logits = x . W^T on tcgen05 tensor cores
 *   moe_route      -> score, selection-only bias, group limit, top-k with a
 *                     per-token k, weights (renormalise, route_scale)
 *   moe_hash_route -> (side path) expert ids looked up by token id
 *   moe_dispatch   -> per-expert counts, offsets, stable expert-major order
 *   moe_permute    -> hidden rows copied into expert-contiguous order
 *   moe_combine    -> weighted fp32 sum of expert outputs back in token order,
 *                     plus an optional shared expert
 *
 * Further entry points on the same buffers:
 *   moe_gate_route            gate GEMM with the route in its epilogue
 *   moe_route_grouped         per-group candidates, then a global top-k
 *   moe_dispatch_limited      dispatch with a per-expert capacity and expert
 *                             blocks padded for tiled expert GEMMs
 *   moe_expert_gate_up / moe_expert_down
 *                             the routed experts' SwiGLU FFN (grouped GEMMs)
 *   moe_ep_layout / moe_ep_permute / moe_ep_combine
 *                             expert-parallel exchange over peer memory
 *   moe_dispatch_static       dispatch without a caller workspace
 *   moe_permute_bounded / moe_combine_bounded
 *                             permute / combine with dest_pos bounds-checked
 *   moe_wait_probe            diagnostic for the bounded-wait timeout path
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers into memory the caller owns; the
 *     library never allocates, frees or synchronises, and launches only on the
 *     given stream.  Calls are asynchronous: outputs are ready when the stream
 *     reaches them.
 *   - Row-major layouts, no padding between rows.  bf16 tensors are passed as
 *     moe_bf16_t (the raw 16-bit pattern).
 *   - Host-side validation is synchronous: a bad argument returns a status and
 *     launches nothing.  T = 0 is a valid no-op returning MOE_OK.
 *   - d_status (where present, nullable) is a device int32 the caller zeroes;
 *     kernels record the first device-side problem there (out-of-range id or
 *     token, NaN logit, a wait that timed out) and never trap.  Read it after
 *     the stream has synchronised.
 *   - A failed launch returns MOE_ERR_CUDA after clearing the CUDA error.
 *   - The library keeps no state between calls and is re-entrant.
 *
 * Sources, by page title and section:
 *   "DeepSeek-V3.2-Exp - Select experts" (Explanation; gate-forward code
 *     excerpt): fp32 gate linear, softmax/sigmoid, selection-only bias, group
 *     limit, top-k, weights from unbiased scores, renormalise, route_scale.
 *   "Crate ferrox_moe" (Functions; Structs RoutingDecision, MoeLayerConfig;
 *     Enums GatingFunction): sqrt-softplus and gpt-oss scoring, norm_topk_prob,
 *     route_hash, combine_expert_outputs.
 *   "Feature Request: dynamic number of experts (hyperparam per request)": k
 *     chosen per request from the same ranking.
 *   "I modelli MoE open hanno router opposti": shared experts, hash-routed
 *     first layers, expert counts and k of the model families.
 */
#ifndef MOE_DISPATCH_H
#define MOE_DISPATCH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; declared here so this header needs no CUDA
 * headers.  NULL means the legacy default stream. */
typedef struct CUstream_st *moe_stream_t;

/* bf16 storage: the upper 16 bits of an IEEE binary32. */
typedef uint16_t moe_bf16_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* host validation failed; nothing launched */
    MOE_ERR_UNSUPPORTED = 2,  /* valid but outside this build's limits */
    MOE_ERR_CUDA = 3,         /* a CUDA call or launch failed */
    MOE_ERR_DEVICE_INDEX = 4, /* (d_status) id/token/k out of range seen on device */
    MOE_ERR_TIMEOUT = 5,      /* (d_status) a bounded device wait gave up */
    MOE_ERR_NAN_LOGIT = 6     /* (d_status) NaN logit seen; row still routed */
} moe_status;

/* Scoring functions.  "Crate ferrox_moe", Enums: GatingFunction. */
typedef enum {
    MOE_SCORE_SOFTMAX = 0,       /* softmax over all E, then top-k */
    MOE_SCORE_SIGMOID = 1,       /* 1/(1+exp(-l)) per expert */
    MOE_SCORE_SQRT_SOFTPLUS = 2, /* sqrt(log(1+exp(l))) per expert */
    MOE_SCORE_TOPK_SOFTMAX = 3   /* gpt-oss: top-k on logits, softmax over those k */
} moe_score_fn;

/* Static per-layer routing configuration ("Crate ferrox_moe", MoeLayerConfig;
 * the gate's constructor fields in "DeepSeek-V3.2-Exp - Select experts"). */
typedef struct {
    int32_t num_experts;  /* E: 1..512 */
    int32_t k_max;        /* slots per token: 0..min(E, 32); per-token k <= k_max */
    int32_t score;        /* moe_score_fn */
    int32_t n_groups;     /* contiguous expert groups; 1 = no group limit; <= 32 */
    int32_t topk_groups;  /* groups kept when n_groups > 1 */
    int32_t group_topn;   /* group score = sum of its group_topn best keys: 1 (amax) or 2 */
    int32_t renormalize;  /* nonzero: divide the selected weights by their sum */
    float route_scale;    /* multiplies every weight (after renormalisation) */
} moe_route_params;

/* Human-readable name of a status code (static string). */
const char *moe_status_string(moe_status s);

/*
 * moe_gate_gemm -- gate logits ("DeepSeek-V3.2-Exp - Select experts", gate
 * forward: the linear layer computed in fp32).
 *   logits[t][e] = sum_i x[t][i] * w[e][i]
 * x      [T][d] bf16, w [E][d] bf16 (both K-major), logits [T][E] fp32 out.
 * Products are exact in fp32 and accumulate in fp32 on tcgen05 tensor cores.
 * Limits: 1 <= E <= 512, d >= 8 and d % 8 == 0 (16-byte rows), x, w 16-byte
 * aligned, T * E < 2^31.  d_status (nullable) receives MOE_ERR_TIMEOUT if a
 * pipeline wait exceeds its bound (it never should).
 */
moe_status moe_gate_gemm(const moe_bf16_t *x, const moe_bf16_t *w, float *logits, int64_t T,
                         int32_t d, int32_t E, int32_t *d_status, moe_stream_t stream);

/*
 * moe_route -- scoring, selection and weights, one fused pass per token row.
 * ("DeepSeek-V3.2-Exp - Select experts": Explanation and gate forward;
 *  "Crate ferrox_moe": route_top_k_*; "Feature Request: dynamic number of
 *  experts": per-request k.)
 *   score s_e from the logit; selection key = s_e + bias[e] (bias nullable);
 *   if n_groups > 1: group score = sum of the group_topn largest keys of each
 *   contiguous group of E/n_groups experts, keep the topk_groups best groups;
 *   take the k_t largest keys of kept experts (k_t = k_per_token[t], or k_max
 *   if k_per_token is NULL), in descending key order, equal keys -> lower id;
 *   weight = unbiased s_e (gpt-oss: softmax over the k_t selected logits),
 *   divided by their sum if renormalize, times route_scale.
 * logits [T][E] fp32, 16-byte aligned; bias [E] fp32 or NULL; k_per_token [T]
 * int32 or NULL.
 * Out: topk_ids [T][k_max] int32 (-1 in slots >= k_t), topk_w [T][k_max] fp32
 * (0 in those slots).
 * Validation: E % n_groups == 0, k_max <= topk_groups * E / n_groups,
 * group_topn in {1, 2} and <= E / n_groups.  On the device a k_per_token value
 * outside [0, k_max] is clamped and reported as MOE_ERR_DEVICE_INDEX; a NaN
 * logit ranks below every number and is reported as MOE_ERR_NAN_LOGIT.
 */
moe_status moe_route(const float *logits, const float *bias, const int32_t *k_per_token,
                     const moe_route_params *params, int64_t T, int32_t *topk_ids,
                     float *topk_w, int32_t *d_status, moe_stream_t stream);

/*
 * moe_route_grouped -- grouped top-k ("Crate ferrox_moe", Functions,
 * route_top_k_grouped): the E experts form params->n_groups contiguous
 * groups; each group keeps its k_per_group best experts by score (the same
 * score function as moe_route), and of those candidates the params->k_max best
 * are selected, in descending score order, ties to the lower id.  Weights as
 * moe_route (score of the expert, renormalize, route_scale; gpt-oss: softmax
 * over the selected logits).  No bias and no per-token k: the page gives the
 * rule without them.  params->topk_groups and group_topn are ignored.
 * logits [T][E] fp32 (4-byte aligned); topk_ids, topk_w [T][k_max].
 * Limits: E <= 512, E % n_groups == 0, 1 <= k_per_group <= E/n_groups,
 * k_max <= min(32, n_groups * k_per_group).  NaN logits rank lowest and report
 * MOE_ERR_NAN_LOGIT.
 */
moe_status moe_route_grouped(const float *logits, const moe_route_params *params,
                             int32_t k_per_group, int64_t T, int32_t *topk_ids, float *topk_w,
                             int32_t *d_status, moe_stream_t stream);

/*
 * moe_gate_route -- moe_gate_gemm and moe_route in one kernel (the gate linear
 * and the router are one function in "DeepSeek-V3.2-Exp - Select experts",
 * gate forward).  Same inputs, outputs and status rules as the two calls in a
 * row, except that the logits are written only if `logits` is non-NULL: each
 * token's row of logits is routed straight from the tensor-core accumulator.
 * Selected ids are the same as moe_route's on the same logits; weights agree
 * to rounding.  Limits: k_max <= 16 (else MOE_ERR_UNSUPPORTED), plus those of
 * both calls.
 */
moe_status moe_gate_route(const moe_bf16_t *x, const moe_bf16_t *w, const float *bias,
                          const int32_t *k_per_token, const moe_route_params *params, int64_t T,
                          int32_t d, int32_t *topk_ids, float *topk_w, float *logits,
                          int32_t *d_status, moe_stream_t stream);

/*
 * moe_hash_route -- expert ids from a token-id table ("Crate ferrox_moe",
 * route_hash: the DeepSeek-V4 hash layers look the ids up by token id; no
 * bias, no selection).
 *   topk_ids[t][j] = tid2eid[token_ids[t]][j]  (a repeated id keeps both slots)
 * tid2eid [vocab][k] int32, row-major (ggml's [k, vocab]); k <= 32.
 * Weights: with logits [T][E] given, the score (params->score) of each looked-up
 * expert, then renormalize / route_scale as in moe_route; with logits NULL,
 * route_scale / k per slot.  params->num_experts = E; other fields of params
 * besides score, renormalize and route_scale are ignored.
 * A token id outside [0, vocab) empties its row (ids -1, weights 0); a table
 * entry outside [0, E) empties its slot; both report MOE_ERR_DEVICE_INDEX.
 */
moe_status moe_hash_route(const int32_t *token_ids, const int32_t *tid2eid, int32_t vocab,
                          int32_t k, const float *logits, const moe_route_params *params,
                          int64_t T, int32_t *topk_ids, float *topk_w, int32_t *d_status,
                          moe_stream_t stream);

/*
 * moe_dispatch_workspace_size -- bytes of device scratch moe_dispatch needs for
 * T tokens, k_max slots and E experts (depends only on T*k_max and E; never
 * more than 606,208 bytes: at most 296 segments of E rounded up to 4 int32).
 */
moe_status moe_dispatch_workspace_size(int64_t T, int32_t k_max, int32_t E, size_t *bytes);

/*
 * moe_dispatch -- histogram, exclusive scan and stable scatter of the
 * assignments into expert-contiguous order (the dispatch step that makes
 * "only the selected experts process the input" concrete).
 *   counts[e]   = number of slots with id e;
 *   offsets[0]  = 0, offsets[e+1] = offsets[e] + counts[e]  (offsets[E] = N);
 *   walking slots in flat order a = t*k_max + j (slots with id -1 skipped),
 *   pos = offsets[e] + number of earlier slots with the same e;
 *   sorted_token[pos] = t, dest_pos[a] = pos (-1 for empty slots).
 * topk_ids [T][k_max]; counts [E]; offsets [E+1]; sorted_token capacity
 * T*k_max (the first N entries are written); dest_pos [T][k_max].
 * workspace: ws_bytes >= moe_dispatch_workspace_size(), 256-byte aligned; its
 * contents need no initialisation.  T*k_max < 2^31.  An id outside [-1, E) is
 * treated as empty and reported as MOE_ERR_DEVICE_INDEX.
 */
moe_status moe_dispatch(const int32_t *topk_ids, int64_t T, int32_t k_max, int32_t E,
                        int32_t *counts, int32_t *offsets, int32_t *sorted_token,
                        int32_t *dest_pos, void *workspace, size_t ws_bytes, int32_t *d_status,
                        moe_stream_t stream);

/*
 * moe_dispatch_limited_rows -- rows that sorted_token (and the permuted xs)
 * must hold for moe_dispatch_limited with these sizes:
 *   min(T*k_max, E*capacity) + E*(pad - 1)   (capacity 0: T*k_max + E*(pad-1)).
 * capacity >= 0, 1 <= pad <= 4096; MOE_ERR_UNSUPPORTED when the bound reaches 2^31.
 */
moe_status moe_dispatch_limited_rows(int64_t T, int32_t k_max, int32_t E, int32_t capacity,
                                     int32_t pad, int64_t *rows);

/*
 * moe_dispatch_limited -- moe_dispatch with a per-expert capacity and expert
 * blocks padded for a tiled expert GEMM.  The capacity is the Switch-style
 * top-1 limit the open-MoE router survey lists among the router levers ("I
 * modelli MoE open hanno router opposti"); the pages give no formula, and the
 * reading here is: expert e keeps the first `capacity` of its slots in flat
 * order a = t*k_max + j and drops the others.  capacity 0 keeps every slot.
 *   counts[e]   = number of slots with id e (the demand, before the cut);
 *   kept[e]     = min(counts[e], capacity);
 *   offsets[0]  = 0, offsets[e+1] = offsets[e] + kept[e] rounded up to a
 *                 multiple of pad;
 *   a kept slot of rank r (earlier slots with the same e) gets
 *   pos = offsets[e] + r, sorted_token[pos] = t, dest_pos[a] = pos;
 *   a dropped or empty slot gets dest_pos[a] = -1;
 *   sorted_token[offsets[e] + kept[e] .. offsets[e+1]) = -1 (padding rows);
 *   *dropped (nullable) = sum over e of counts[e] - kept[e].
 * sorted_rows: capacity of sorted_token, >= moe_dispatch_limited_rows().
 * capacity 0 with pad 1 gives exactly moe_dispatch's outputs.  moe_permute and
 * moe_combine take the dest_pos as they are (dropped slots are skipped; the
 * padding rows of xs are not written).  Workspace, alignment, device-error
 * and stream rules as moe_dispatch.
 */
moe_status moe_dispatch_limited(const int32_t *topk_ids, int64_t T, int32_t k_max, int32_t E,
                                int32_t capacity, int32_t pad, int32_t *counts, int32_t *offsets,
                                int32_t *sorted_token, int64_t sorted_rows, int32_t *dest_pos,
                                int32_t *dropped, void *workspace, size_t ws_bytes,
                                int32_t *d_status, moe_stream_t stream);

/*
 * moe_dispatch_static -- moe_dispatch without a caller-provided workspace.
 * (No counterpart in the source pages: this entry point exists for callers that
 * cannot allocate device memory, e.g. a plugin running inside a host framework
 * that owns every device allocation, or code that must avoid the implicit
 * device synchronisation of cudaMalloc.)
 * Same arguments, outputs and status rules as moe_dispatch, minus workspace and
 * ws_bytes.  Its scratch is a 606,208-byte array inside the library (the most
 * moe_dispatch_workspace_size() returns for any size it accepts: 296 segments
 * x 512 experts x 4 bytes), held by every GPU that loads the library until the
 * process exits; so every size moe_dispatch accepts fits, and the sizes it
 * refuses (T*k_max >= 2^31) are refused here the same way, with nothing
 * launched.  The library allocates and frees nothing here either.
 * The scratch array's device address is looked up (cudaGetSymbolAddress) by
 * the first call in each CUDA context and cached under that context's unique
 * id, so a context destroyed and created again (e.g. after cudaDeviceReset) is
 * looked up afresh; that first call may create the device's primary context,
 * so make it before any stream capture.  Each device's context has its own
 * copy of the array.  All calls share the one array: two calls whose work overlaps on
 * the GPU (different streams, or different host threads) race and give wrong
 * results; serialise them.  The array keeps the last call's contents, but no
 * call depends on them: everything a call reads from it, it wrote first.
 */
moe_status moe_dispatch_static(const int32_t *topk_ids, int64_t T, int32_t k_max, int32_t E,
                               int32_t *counts, int32_t *offsets, int32_t *sorted_token,
                               int32_t *dest_pos, int32_t *d_status, moe_stream_t stream);

/*
 * moe_permute -- xs[dest_pos[t][j]] = x[t] for every slot with dest_pos >= 0
 * (a bit-exact row copy into expert-contiguous order).  Token-major: each row
 * of x is read once and written to its k_t destinations.
 * x [T][d] bf16; dest_pos [T][k_max] from moe_dispatch; xs [N][d] bf16.
 * d % 8 == 0; x and xs 16-byte aligned.
 */
moe_status moe_permute(const moe_bf16_t *x, const int32_t *dest_pos, int64_t T, int32_t k_max,
                       int32_t d, moe_bf16_t *xs, moe_stream_t stream);

/*
 * moe_combine -- weighted sum of expert outputs back in token order
 * ("Crate ferrox_moe", combine_expert_outputs: routed plus shared).
 *   out[t] = bf16_rne( sum_{j: dest_pos[t][j] >= 0} topk_w[t][j] * y[dest_pos[t][j]]
 *                      + shared[t] )
 * accumulated in fp32 in slot order j = 0, 1, ..., the shared expert (unit
 * weight, nullable) added last.
 * y [N][d] bf16 (expert outputs in expert-contiguous order); topk_w,
 * dest_pos [T][k_max]; shared [T][d] bf16 or NULL; out [T][d] bf16.
 * d % 8 == 0; y, shared, out 16-byte aligned.
 */
moe_status moe_combine(const moe_bf16_t *y, const float *topk_w, const int32_t *dest_pos,
                       const moe_bf16_t *shared, int64_t T, int32_t k_max, int32_t d,
                       moe_bf16_t *out, moe_stream_t stream);

/*
 * moe_permute_bounded / moe_combine_bounded -- moe_permute and moe_combine
 * with every dest_pos checked against the rows the caller's buffer holds
 * (xs_rows for permute, y_rows for combine): a value outside [-1, rows) is
 * skipped (no row is read or written for that slot) and reported in
 * *d_status (nullable) as MOE_ERR_DEVICE_INDEX.  Otherwise the same
 * arguments, results and limits as the plain calls.  The plain calls trust
 * dest_pos as moe_dispatch wrote it; in a library built with MOE_CHECKED
 * they check it as well, against T * k_max rows (the most a dispatch of T
 * tokens fills; use these bounded calls for padded layouts, whose
 * moe_dispatch_limited_rows can exceed that), and skip without reporting,
 * having no status argument.  (The pages' combine, "Crate ferrox_moe",
 * combine_expert_outputs, has no index to check: these exist for callers
 * that pass dest_pos from elsewhere.)
 */
moe_status moe_permute_bounded(const moe_bf16_t *x, const int32_t *dest_pos, int64_t T,
                               int32_t k_max, int32_t d, moe_bf16_t *xs, int64_t xs_rows,
                               int32_t *d_status, moe_stream_t stream);
moe_status moe_combine_bounded(const moe_bf16_t *y, const float *topk_w, const int32_t *dest_pos,
                               const moe_bf16_t *shared, int64_t T, int32_t k_max, int32_t d,
                               int64_t y_rows, moe_bf16_t *out, int32_t *d_status,
                               moe_stream_t stream);

/*
 * moe_wait_probe -- diagnostic (no counterpart in the pages): one warp runs the
 * library's bounded mbarrier wait against a barrier that nothing completes,
 * with a limit of limit_ns nanoseconds (1 ns .. 1 s).  The wait gives up,
 * *d_status receives MOE_ERR_TIMEOUT (first error wins) and *d_outcome
 * (nullable) 2 (1 would mean the barrier completed).  Lets a test exercise the
 * timeout path every kernel's waits take, with no fault and no hang.
 */
moe_status moe_wait_probe(uint64_t limit_ns, int32_t *d_status, int32_t *d_outcome,
                          moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Expert-parallel exchange.  In multi-GPU expert parallelism every router
 * choice becomes all-to-all traffic ("I modelli MoE open hanno router
 * opposti", closing paragraphs); here that traffic is the permute's stores and
 * the combine's loads themselves, made over peer memory (NVLink) with plain
 * 16-byte accesses.  G ranks, expert e on rank e / (E/G).
 * Receive layout of rank d (the pages fix none; this is the plain reading):
 * its experts in ascending order; inside one expert the rows of source rank 0,
 * then 1, ...; inside one source, that rank's slots in flat order.
 * Per step on every rank: moe_dispatch (local) -> all-gather of counts ->
 * moe_ep_layout -> moe_ep_permute -> barrier -> experts on the receive buffer
 * -> barrier -> moe_ep_combine.  The all-gather and the barriers are the
 * caller's collectives (e.g. NCCL); nothing here waits on another GPU.
 * ------------------------------------------------------------------------ */

/*
 * moe_ep_layout -- owner rank and receive row of every slot of this rank.
 *   all_counts [G][E]: every rank's moe_dispatch counts (gathered);
 *   topk_ids, dest_pos [T][k_max], offsets [E+1]: this rank's moe_dispatch
 *   inputs and outputs;
 *   dest_rank[a] = e / (E/G);  dest_row[a] = row of slot a on that rank
 *   (both -1 for an empty slot);
 *   recv_offsets [E/G + 1]: this rank's receive blocks, recv_offsets[le] =
 *   first row of its local expert le, recv_offsets[E/G] = rows it receives.
 * 1 <= G <= 64, 0 <= rank < G, E <= 512, E % G == 0.  A slot whose dest_pos
 * disagrees with offsets/all_counts, or an id outside [-1, E), gets -1/-1
 * and reports MOE_ERR_DEVICE_INDEX.
 */
moe_status moe_ep_layout(const int32_t *all_counts, const int32_t *topk_ids,
                         const int32_t *dest_pos, const int32_t *offsets, int32_t G, int32_t rank,
                         int64_t T, int32_t k_max, int32_t E, int32_t *dest_rank,
                         int32_t *dest_row, int32_t *recv_offsets, int32_t *d_status,
                         moe_stream_t stream);

/*
 * moe_ep_permute -- recv_r[dest_row[t][j]] = x[t] with r = dest_rank[t][j]:
 * each row of x is read once and stored to its owners' receive buffers.
 * peer_recv: DEVICE array of G pointers, entry r = rank r's receive buffer
 * ([recv_capacity][d] bf16, 16-byte aligned) as mapped in this process (its
 * own buffer for r == this rank).  A (rank, row) outside [0,G) x
 * [0,recv_capacity), or a null/unaligned entry, skips the slot and reports
 * MOE_ERR_DEVICE_INDEX.  The receivers must not be using their buffers while
 * this runs, and read them only after every sender's call has completed.
 */
moe_status moe_ep_permute(const moe_bf16_t *x, const int32_t *dest_rank, const int32_t *dest_row,
                          moe_bf16_t *const *peer_recv, int32_t G, int64_t recv_capacity,
                          int64_t T, int32_t k_max, int32_t d, int32_t *d_status,
                          moe_stream_t stream);

/*
 * moe_ep_combine -- moe_combine whose expert rows live on their owners:
 *   out[t] = bf16_rne( sum_j topk_w[t][j] * y_r[dest_row[t][j]] + shared[t] ),
 *   r = dest_rank[t][j]; fp32 in slot order, shared added last.
 * peer_y: DEVICE array of G pointers to the ranks' expert outputs
 * ([recv_capacity][d] bf16, in receive layout).  Bounds and status as
 * moe_ep_permute.  The owners' outputs must be complete before this runs.
 */
moe_status moe_ep_combine(moe_bf16_t *const *peer_y, const int32_t *dest_rank,
                          const int32_t *dest_row, const float *topk_w, const moe_bf16_t *shared,
                          int32_t G, int64_t recv_capacity, int64_t T, int32_t k_max, int32_t d,
                          moe_bf16_t *out, int32_t *d_status, moe_stream_t stream);

/* ------------------------------------------------------------------------
 * Routed experts' FFN over the expert-ordered rows ("Crate ferrox_moe",
 * Functions: run_expert, run_expert_oai, swiglu_oai; Constants:
 * SWIGLU_OAI_ALPHA = 1.702, SWIGLU_OAI_LIMIT = 7.0).  Two grouped GEMMs on
 * tcgen05 tensor cores; row r belongs to the expert e whose block
 * [offsets[e], offsets[e+1]) holds it, and the blocks must start on multiples
 * of 128 rows (moe_dispatch_limited with pad = 128 writes such offsets; rows
 * of a block past the expert's own tokens are padding and give padding).
 * The page names the clamped SwiGLU and its constants but not its formula;
 * the reading here is the published gpt-oss one:
 *   MOE_ACT_SWIGLU:     act(g, u) = g * sigmoid(g) * u
 *   MOE_ACT_SWIGLU_OAI: g' = min(g, 7), u' = clamp(u, -7, 7),
 *                       act(g, u) = g' * sigmoid(1.702 * g') * (u' + 1)
 * ------------------------------------------------------------------------ */
typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_SWIGLU_OAI = 1 } moe_activation;

/*
 * moe_expert_gate_up -- h[r] = bf16( act(xs[r] . W1[e]^T + b1[e],
 *                                        xs[r] . W3[e]^T + b3[e]) )
 * xs [rows][d] bf16; w1, w3 [E][F][d] bf16 (row f of expert e is the weight
 * vector of output feature f, K-major); b1, b3 [E][F] fp32 or NULL;
 * h [rows][F] bf16.  fp32 accumulation, activation in fp32, one rounding.
 * d, F multiples of 16; E <= 4096; rows/128 <= 65535; xs, w1, w3, h 16-byte
 * aligned.  Offsets not 128-aligned, or offsets[E] > rows, report
 * MOE_ERR_DEVICE_INDEX and leave the affected tiles unwritten.
 */
moe_status moe_expert_gate_up(const moe_bf16_t *xs, const int32_t *offsets, const moe_bf16_t *w1,
                              const moe_bf16_t *w3, const float *b1, const float *b3, int32_t E,
                              int32_t d, int32_t F, int64_t rows, int32_t act, moe_bf16_t *h,
                              int32_t *d_status, moe_stream_t stream);

/*
 * moe_expert_down -- y[r] = bf16( h[r] . W2[e]^T + b2[e] )
 * h [rows][F] bf16; w2 [E][d][F] bf16; b2 [E][d] fp32 or NULL; y [rows][d]
 * bf16 (the expert outputs moe_combine reads).  Limits and status as
 * moe_expert_gate_up.
 */
moe_status moe_expert_down(const moe_bf16_t *h, const int32_t *offsets, const moe_bf16_t *w2,
                           const float *b2, int32_t E, int32_t d, int32_t F, int64_t rows,
                           moe_bf16_t *y, int32_t *d_status, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DISPATCH_H */
