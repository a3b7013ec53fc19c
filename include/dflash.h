/*
 * dflash.h — C ABI of the DFlash draft-proposal library for NVIDIA B200 (sm_100a).
 *
 * The library implements the data-parallel hot path of DFlash block-diffusion
 * speculative decoding as described in "DFlash Speculative Decoding in the vLLM
 * Neuron Framework" (AWS Neuron design doc) and the two pull requests
 * "[Feat][Spec Decode] DFlash" (vLLM #36847) and "Dflash: Block Diffusion
 * Speculative Decoding" (QEfficient #995):
 *
 *   dflash_inject_context  — §"Context KV Injection (Precompute)": concat'd target
 *                            aux states -> fc -> hidden_norm -> all layers' K/V
 *                            (k_norm + RoPE on keys) -> paged-cache scatter.
 *   dflash_propose         — §"Draft Block Construction", §"DFlash Draft Model
 *                            Architecture": [bonus, mask, ..., mask] block, non-causal
 *                            Qwen3-style decoder stack over the injected context,
 *                            aliased target LM head, greedy argmax -> K drafts.
 *   dflash_verify_greedy   — §"Component Overview" (greedy rejection sampler):
 *                            longest prefix of drafts matching the target's argmax,
 *                            plus one bonus token; rejected slots are -1
 *                            (§"Async Rejection and Position Correction").
 *   dflash_paged_slots     — §"Paged KV Integration" (_paged_slots helper).
 *   dflash_prepare_proposal_inputs — §"Async Rejection and Position Correction"
 *                            (_correct_target_positions_for_async, _current_seq_lens),
 *                            §"Paged KV Integration", §"Draft Block Construction".
 *   dflash_spec_step, dflash_step_graph_* — the four calls above as one step with
 *                            nothing from the host between them, eager or as one
 *                            CUDA graph owned by the library.
 *   dflash_create_vocab_shard, dflash_propose_keys, dflash_finalize_draft_keys —
 *                            §"DFlashQwen3ForCausalLM": the aliased LM head split over
 *                            the vocabulary across tensor-parallel ranks, combined
 *                            by one all-reduce MAX of 8 bytes per draft row.
 *
 * Conventions for every call
 *   - All tensor arguments are DEVICE pointers unless stated otherwise; bf16 means
 *     IEEE bfloat16 stored as uint16.  Row-major, densely packed.
 *   - `stream` is a cudaStream_t passed as void*.  Calls only enqueue work on it:
 *     no call synchronizes the stream, and no call other than dflash_create* and
 *     dflash_step_graph_create (the graph and its capture stream) allocates
 *     memory.  Work may be captured into a CUDA graph.
 *   - The caller owns every buffer it passes; the handle owns only the packed
 *     weight copies and small tables it builds in dflash_create.
 *   - Shape and argument errors are detected on the host before any launch and
 *     returned as a negative dflash_status; nothing is enqueued in that case.
 *   - Conditions that can only be seen on the device (a page id outside the pool,
 *     a position past the block table or the RoPE table, a token id outside the
 *     vocabulary, a pipeline wait that ran out) never trap: the kernel skips the
 *     access and sets a bit in the handle's device error word, which
 *     dflash_check_device_errors() reads and clears.
 *   - A handle may be used by one stream at a time (calls on one handle must not
 *     overlap on the GPU).
 */
#ifndef DFLASH_H_
#define DFLASH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DFLASH_OK = 0,
  DFLASH_ERR_INVALID_ARG = -1,       /* null pointer, negative size, inconsistent arguments */
  DFLASH_ERR_CUDA = -2,              /* a CUDA runtime/driver call or a launch failed        */
  DFLASH_ERR_WORKSPACE = -3,         /* workspace smaller than the *_workspace_bytes value   */
  DFLASH_ERR_UNSUPPORTED_SHAPE = -4, /* geometry outside what the kernels are built for       */
  DFLASH_ERR_DEVICE_BOUNDS = -5,     /* returned by dflash_check_device_errors (see above)    */
  DFLASH_ERR_UNIMPLEMENTED = -6,
  DFLASH_ERR_DEVICE_TIMEOUT = -7,    /* returned by dflash_check_device_errors                */
  DFLASH_ERR_RANGE = -8,             /* weights outside the fp16 range the path stores them in */
  DFLASH_ERR_EXCHANGE = -9           /* the caller's all-reduce hook reported a failure        */
} dflash_status;

/* Device error bits reported by dflash_check_device_errors(). */
#define DFLASH_DEVERR_TIMEOUT   0x1u  /* a bounded pipeline wait gave up                        */
#define DFLASH_DEVERR_SLOT      0x2u  /* slot / page id outside the KV pool                     */
#define DFLASH_DEVERR_TABLE     0x4u  /* position // page_size past the block-table row width   */
#define DFLASH_DEVERR_TOKEN     0x8u  /* bonus token id outside [0, vocab)                      */
#define DFLASH_DEVERR_POSITION  0x10u /* position outside [0, max_position) of the RoPE table   */
#define DFLASH_DEVERR_INPUT     0x20u /* malformed proposal-preparation input (see below)       */

/* Draft-model geometry.  block_size / mask_token_id / target_layer_ids are the
 * fields of the pages' DFlashConfig; the rest is the Qwen3 layer shape.
 * Supported: head_dim in {64, 128}; hidden, n_q_heads*head_dim, intermediate and
 * n_target_layers*hidden multiples of 64; vocab a multiple of 32;
 * n_q_heads % n_kv_heads == 0 with block_size*(n_q_heads/n_kv_heads) <= 128;
 * 2 <= block_size <= 64; n_layers <= 64; page_size == 16. */
typedef struct dflash_config {
  int hidden;
  int n_layers;
  int n_q_heads;
  int n_kv_heads;
  int head_dim;
  int intermediate;
  int vocab;
  int n_target_layers;            /* number of tapped target layers (T)                   */
  const int* target_layer_ids;    /* HOST array [n_target_layers], concat order; recorded */
                                  /* for validation only (may be NULL)                    */
  int block_size;                 /* bs; the call proposes K = bs - 1 drafts              */
  int mask_token_id;
  int page_size;                  /* tokens per KV page (16)                              */
  float rms_eps;
  float rope_theta;
  int max_position;               /* RoPE table covers positions [0, max_position)        */
} dflash_config;

/* Draft weights: DEVICE pointers, bf16, row-major [out_features, in_features].
 * Per-layer entries are HOST arrays of n_layers device pointers.
 *   fc_w [H, T*H]   hidden_norm_w [H]   embed [V, H]   lm_head [V, H]   final_norm_w [H]
 *   in_norm_w/post_norm_w [H]   wq [Hq*d, H]   wk, wv [Hkv*d, H]   wo [H, Hq*d]
 *   q_norm_w, k_norm_w [d]      w_gate, w_up [I, H]   w_down [H, I]
 * Every weight of a GEMM is copied by dflash_create into a tile-contiguous
 * layout (each 256-row x 64-column tile one contiguous 32 KB chunk, so that the
 * weight stream reads whole chunks).  Storage precision of the path: the
 * projections whose inputs are bounded by construction (RMSNorm outputs,
 * attention outputs) run with fp16 operands, so the copies of wq|wk|wv
 * (stacked), w_gate|w_up (interleaved in 16-row blocks), the stacked per-layer
 * [wk; wv], wo and lm_head are fp16 (bf16 -> fp16 is exact in fp16's normal
 * range); fc_w and w_down stay bf16.  Those source buffers may be freed after
 * dflash_create returns.  The norm weights and the embedding (the target's
 * aliased table) are used in place: those pointers must stay valid and
 * unchanged for the lifetime of the handle.  The GEMM weight pointers must be
 * 16-byte aligned (DFLASH_ERR_INVALID_ARG otherwise). */
typedef struct dflash_weights {
  const void* fc_w;
  const void* hidden_norm_w;
  const void* embed;
  const void* lm_head;
  const void* final_norm_w;
  const void* const* in_norm_w;
  const void* const* post_norm_w;
  const void* const* wq;
  const void* const* wk;
  const void* const* wv;
  const void* const* wo;
  const void* const* q_norm_w;
  const void* const* k_norm_w;
  const void* const* w_gate;
  const void* const* w_up;
  const void* const* w_down;
} dflash_weights;

typedef struct dflash_handle dflash_handle;

/* Validates the geometry, makes `device` current, packs the weights and builds
 * the RoPE table (cos/sin of pos * theta^(-2i/d), evaluated in double precision
 * on the device).  Synchronizes the device once at the end.  On success *out
 * receives the handle; on failure *out is NULL and nothing is leaked.
 * Range of the fp16 storage (DFLASH_ERR_RANGE otherwise): every weight copied
 * to fp16 (wq, wk, wv, wo, w_gate, w_up, lm_head) has |w| <= 65504 and at most
 * 1% of the nonzero ones lie below 2^-14 (where fp16 keeps them only as
 * subnormals); the norm weights whose RMSNorm outputs are stored in fp16
 * (hidden_norm_w, in_norm_w, post_norm_w, final_norm_w) have
 * sqrt(hidden) * max|w| <= 65504, the bound of those outputs. */
dflash_status dflash_create(const dflash_config* cfg, const dflash_weights* w,
                            int device, dflash_handle** out);

/* A handle whose LM head holds only the vocabulary rows [vocab_start,
 * vocab_start + vocab_count): one rank's shard of the tensor-parallel LM head
 * (§"DFlashQwen3ForCausalLM": the aliased head is a column-parallel linear
 * over the vocabulary; every rank runs the rest of the draft in full).
 * w->lm_head points at that shard, [vocab_count, H] bf16; w->embed stays the
 * whole [vocab, H] table; cfg->vocab is the whole vocabulary.  vocab_start and
 * vocab_count must be multiples of 32 (DFLASH_ERR_UNSUPPORTED_SHAPE), with
 * vocab_count >= 1 and vocab_start + vocab_count <= vocab (DFLASH_ERR_INVALID_ARG).
 * A shard handle proposes through dflash_propose_keys (dflash_propose and
 * dflash_spec_step reject it: a shard's own argmax is not a draft); the
 * whole-vocabulary shard (0, vocab) is what dflash_create builds. */
dflash_status dflash_create_vocab_shard(const dflash_config* cfg, const dflash_weights* w,
                                        int device, int vocab_start, int vocab_count,
                                        dflash_handle** out);

/* Tensor-parallel rank tp_rank of tp_size (§"Context KV Injection": each rank
 * projects and stores "this rank's KV heads only"; §"DFlashQwen3ForCausalLM":
 * the aliased LM head is a column-parallel linear over the vocabulary).  The
 * handle holds rank r's slice of the draft: kv heads [r Hkv/S, (r+1) Hkv/S)
 * with their query heads (each kv head keeps its query group), MLP features
 * [r I/S, (r+1) I/S), the matching columns of Wo and W_down (row-parallel:
 * each rank forms a partial sum of the layer's O and down outputs), and the
 * LM-head vocabulary rows [vocab_start, vocab_start + vocab_count).  fc,
 * hidden_norm, the norms and the embedding are replicated.  cfg and w describe
 * the WHOLE model (every rank passes the same); the slices are copied out of
 * w.  Requires n_kv_heads % tp_size == 0 and intermediate % (64 tp_size) == 0
 * (DFLASH_ERR_UNSUPPORTED_SHAPE), 0 <= tp_rank < tp_size and the vocabulary
 * rules of dflash_create_vocab_shard.  The handle's KV pools hold its own kv
 * heads only ([num_pages, n_kv_heads / tp_size, page_size, head_dim]):
 * dflash_inject_context on it projects and writes those heads; it proposes
 * through dflash_propose_tp.  tp_size 1 gives a whole-model handle. */
dflash_status dflash_create_tp_shard(const dflash_config* cfg, const dflash_weights* w,
                                     int device, int tp_rank, int tp_size, int vocab_start,
                                     int vocab_count, dflash_handle** out);

/* Frees everything the handle owns.  The caller must make sure no work that
 * uses the handle is still pending.  NULL is a no-op. */
void dflash_destroy(dflash_handle* h);

/* Workspace (device memory, >= 256-byte aligned, contents need not be
 * initialised) needed by dflash_inject_context for up to `max_rows` rows. */
size_t dflash_inject_workspace_bytes(const dflash_handle* h, int max_rows);

/* Workspace needed by dflash_propose for a batch of up to `max_batch` requests
 * with block tables `max_pages_per_seq` entries wide. */
size_t dflash_propose_workspace_bytes(const dflash_handle* h, int max_batch,
                                      int max_pages_per_seq);

/* Diagnostics: byte offset, inside the workspace of a dflash_propose /
 * dflash_propose_keys call with this B and max_pages_per_seq, of the rows that
 * call hands to the LM head: [B * K, hidden] fp16, row b * K + i the
 * final-RMSNormed hidden state of block slot 1 + i of request b
 * (§"DFlashQwen3ForCausalLM": the kept rows of compute_draft_tokens).  Valid
 * after the call until the workspace is reused, so that the LM head's greedy
 * pick can be checked on exactly the rows it saw.  (size_t)-1 for a NULL
 * handle or non-positive sizes. */
size_t dflash_propose_final_rows_offset(const dflash_handle* h, int B, int max_pages_per_seq);

/* Workspace needed by dflash_verify_greedy for [B, K+1, V] target logits. */
size_t dflash_verify_workspace_bytes(int B, int K, int V);

/* Maximum number of partial keys (request x target row x vocabulary chunk)
 * that dflash_verify_greedy_noalloc can hold: 8192 (64 KiB of device memory). */
#define DFLASH_VERIFY_NOALLOC_MAX_PARTIALS 8192

/* The same greedy verification as dflash_verify_greedy, for callers that cannot
 * allocate device memory for a workspace: an embedding runtime that reserved
 * all device memory for its own pool, a plugin that only receives its input
 * and output buffers, or a latency-critical loop where cudaMalloc/cudaFree
 * would synchronize the device.  (The pages have no counterpart of this call;
 * it is an addition of this library.)
 * Arguments, outputs and results are exactly those of dflash_verify_greedy,
 * without the workspace.  Its scratch is a fixed 64 KiB array inside this
 * library's device memory, present on every device that loads the library
 * until the process exits; the call allocates nothing.
 *   - The first call on a device looks up that array's device address (with
 *     the device current) and caches it with the id of the device's current
 *     context; make that first call before any stream capture.  After a device
 *     reset (a new context) the next call looks the address up again.
 *   - Every call shares the one array and leaves its last contents behind.
 *     Calls that overlap on the GPU (e.g. on two streams at once) race on it
 *     and give wrong results; order them on one stream.
 *   - Batches needing more than DFLASH_VERIFY_NOALLOC_MAX_PARTIALS partial keys
 *     are rejected with DFLASH_ERR_WORKSPACE before any launch (every batch up
 *     to 512 requests with K = 15 fits). */
dflash_status dflash_verify_greedy_noalloc(const int32_t* drafts, const float* target_logits,
                                           int B, int K, int V, int32_t* out_tokens,
                                           int32_t* num_accepted, int32_t* bonus,
                                           void* stream);

/* _paged_slots (§"Paged KV Integration"), exactly as the page writes it:
 *   page_no = min(positions[i] / page_size, max_pages_per_seq - 1)
 *   slots[i] = block_table[req_ids[i] * max_pages_per_seq + page_no] * page_size
 *              + positions[i] % page_size
 * positions, req_ids: [n] int64 (>= 0); block_table: [*, max_pages_per_seq] int32;
 * slots: [n] int64 out.  Note the clamp: a position past the table aliases the
 * row's last page.  A negative position yields slot -1 (a padding row).
 * req_ids must index existing block-table rows.  n == 0 is a no-op. */
dflash_status dflash_paged_slots(const int64_t* positions, const int64_t* req_ids,
                                 int n, const int32_t* block_table,
                                 int max_pages_per_seq, int page_size,
                                 int64_t* slots, void* stream);

/* Proposal-input preparation on the device, with the async rejection
 * correction (§"Async Rejection and Position Correction", §"Paged KV
 * Integration", §"Draft Block Construction"), so that a whole speculative step
 * (verify -> prepare -> inject -> propose) runs on one stream with no host
 * round trip.  In the pages' order:
 *   1. request of target row r: the b with last_token_indices[b-1] < r <=
 *      last_token_indices[b]; rows past last_token_indices[B-1] are trailing
 *      padding;
 *   2. prev_rejected[b] = (1 + prev_num_draft[b]) - #{j : prev_sampled[b][j] != -1
 *      and prev_sampled[b][j] < vocab}; positions_out[r] = target_positions[r]
 *      - prev_rejected[req(r)] (prev_sampled == NULL: no previous step, no
 *      correction);
 *   3. seq_lens_out[b] = positions_out[last_token_indices[b]] + 1 - cur_rejected[b],
 *      cur_rejected[b] = (1 + cur_num_draft[b]) - #valid(cur_sampled[b]);
 *   4. bonus_out[b] = the last valid entry of cur_sampled[b];
 *   5. slot_mapping_out[r] = the _paged_slots formula at (positions_out[r],
 *      req(r)) (with the page's clamp); -1 for padding rows (their position is
 *      copied unchanged).
 * Inputs (device): target_positions [n] int64; last_token_indices [B] int32,
 * strictly increasing, < n; cur_sampled [B, cur_width] int32 (the rejection
 * sampler's output of this step, -1 padded, e.g. out_tokens of
 * dflash_verify_greedy); cur_num_draft [B] int32; prev_sampled
 * [B, prev_width] int32 and prev_num_draft [B] int32, both NULL or both set;
 * block_table [B, max_pages_per_seq] int32.  Outputs (device, caller-owned):
 * positions_out, slot_mapping_out [n] int64; seq_lens_out, bonus_out [B]
 * int32 — ready for dflash_inject_context (positions, slots) and
 * dflash_propose (bonus_tokens, seq_lens).
 * Host errors (DFLASH_ERR_INVALID_ARG) before any launch: n < 0, B < 0,
 * widths < 1, page_size < 1, vocab < 1, a missing pointer (the per-request
 * ones and the block table may be NULL only when B == 0: every row is then
 * padding), prev_sampled / prev_num_draft given alone.  Device errors set DFLASH_DEVERR_INPUT in
 * *device_error (a device word, nullable) and skip the value: indices not
 * strictly increasing or past n, a request with no valid sampler output
 * (bonus_out = -1), a corrected position < 0 (slot -1).  One launch; B == 0
 * and n == 0 are no-ops. */
dflash_status dflash_prepare_proposal_inputs(
    const int64_t* target_positions, int n, const int32_t* last_token_indices, int B,
    const int32_t* cur_sampled, int cur_width, const int32_t* cur_num_draft,
    const int32_t* prev_sampled, int prev_width, const int32_t* prev_num_draft,
    const int32_t* block_table, int max_pages_per_seq, int page_size, int vocab,
    int64_t* positions_out, int64_t* slot_mapping_out, int32_t* seq_lens_out,
    int32_t* bonus_out, unsigned* device_error, void* stream);

/* precompute_and_store_context_kv (§"Context KV Injection (Precompute)"):
 *   ctx = hidden_norm(fc(aux))                       [n, H]
 *   for every layer l and kv head h:
 *     k = RoPE(k_norm_l(Wk_l,h ctx), positions)      written to k_cache[l]
 *     v = Wv_l,h ctx                                 written to v_cache[l]
 * at slot_mapping (slot s -> page s / page_size, offset s % page_size).
 *   aux          [n, T*H] bf16, the target's tapped states concatenated in
 *                target_layer_ids order
 *   positions    [n] int64 absolute positions (RoPE), 0 <= pos < max_position
 *   slot_mapping [n] int64; a negative slot marks a padding row, skipped
 *   k_cache, v_cache: HOST arrays of n_layers device pointers, each pool
 *                [num_pages, n_kv_heads, page_size, head_dim] bf16
 * n == 0 is a no-op.  Needs dflash_inject_workspace_bytes(h, n) of workspace. */
dflash_status dflash_inject_context(dflash_handle* h, const void* aux,
                                    const int64_t* positions,
                                    const int64_t* slot_mapping, int n,
                                    void* const* k_cache, void* const* v_cache,
                                    int num_pages, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* One draft proposal for B requests (DFlashQwen3ForCausalLM.forward after
 * injection).  Request b's block is [bonus_tokens[b], mask, ..., mask] at
 * positions seq_lens[b] + [0, bs); every block query attends (non-causally) to
 * the request's keys [0, seq_lens[b] + bs): its injected context and its whole
 * block.  The block's own K/V are written to the cache at those positions
 * (they are scratch until the next injection overwrites them).
 *   bonus_tokens  [B] int32        seq_lens [B] int32 (context tokens injected)
 *   block_table   [B, max_pages_per_seq] int32; must cover seq_len + bs - 1
 *   draft_tokens  [B, K] int32 out (K = bs - 1), greedy argmax of the LM head on
 *                 block slots 1..bs-1 (ties -> lowest id; NaN counts as -inf)
 *   block_tokens  [B, bs] int32 out, cat(bonus, drafts); may be NULL
 *   logits_out    [B*K, V] fp32 out (debug); may be NULL
 * B == 0 is a no-op; B > 65535 (requests per attention launch) or B * bs > 2^24 is
 * DFLASH_ERR_UNSUPPORTED_SHAPE.  Needs dflash_propose_workspace_bytes(h, B, max_pages_per_seq). */
dflash_status dflash_propose(dflash_handle* h, const int32_t* bonus_tokens,
                             const int32_t* seq_lens, const int32_t* block_table,
                             int B, int max_pages_per_seq, void* const* k_cache,
                             void* const* v_cache, int num_pages,
                             int32_t* draft_tokens, int32_t* block_tokens,
                             float* logits_out, void* workspace,
                             size_t workspace_bytes, void* stream);

/* The proposal of dflash_propose up to the LM head's greedy pick, over this
 * handle's vocabulary rows, exported for a cross-rank exchange instead of
 * turned into drafts:
 *   draft_keys [B, K] int64 out: for draft row (b, i) the key
 *     ((ordered bits of the row's largest logit) << 32 | (2^32 - 1 - its
 *     vocabulary id)) with bit 63 flipped, where the ordered bits of a float
 *     sort like the float (-0 as +0, NaN as -inf).  The signed int64 maximum of
 *     the keys of all shards (an all-reduce MAX, 8 bytes per row) is the key
 *     of the whole vocabulary's greedy pick, ties -> lowest id.
 *   logits_out [B*K, vocab_count] fp32 out (debug; this shard's columns);
 *     may be NULL.
 * Everything else (arguments, workspace, errors) as dflash_propose; a
 * whole-vocabulary handle works too.  Then dflash_finalize_draft_keys. */
dflash_status dflash_propose_keys(dflash_handle* h, const int32_t* bonus_tokens,
                                  const int32_t* seq_lens, const int32_t* block_table, int B,
                                  int max_pages_per_seq, void* const* k_cache,
                                  void* const* v_cache, int num_pages, int64_t* draft_keys,
                                  float* logits_out, void* workspace, size_t workspace_bytes,
                                  void* stream);

/* The exchange of a tensor-parallel proposal: sum `count` fp32 values at the
 * DEVICE pointer `data` element-wise over every rank of the group, in place
 * (an all-reduce SUM, e.g. ncclAllReduce with ncclSum), ordered after the work
 * already enqueued on `stream` and before the work enqueued after the call
 * returns (the library enqueues its next kernels on `stream` right after).
 * `user` is passed through.  Return 0 on success. */
typedef int (*dflash_allreduce_fn)(float* data, size_t count, void* stream, void* user);

/* dflash_propose_keys on a tensor-parallel shard (dflash_create_tp_shard):
 * every layer runs on this rank's heads and MLP features; after the O
 * projection and after the down projection the rank's partial sums (the
 * [B * block_size, hidden] fp32 rows, in the workspace) go through
 * `exchange`, and the summed rows are added to the replicated residual
 * stream.  Every rank of the group must make the same call (same B, block
 * tables, bonus tokens and sequence lengths; each with its own KV pools of its
 * kv heads).  Output: this rank's vocabulary shard's greedy-pick keys, as
 * dflash_propose_keys; an all-reduce MAX of them over the ranks, then
 * dflash_finalize_draft_keys, gives the drafts.  DFLASH_ERR_INVALID_ARG for a
 * whole-model handle or a NULL exchange; DFLASH_ERR_EXCHANGE if the hook
 * returns non-zero (the kernels enqueued before it stay enqueued). */
dflash_status dflash_propose_tp(dflash_handle* h, const int32_t* bonus_tokens,
                                const int32_t* seq_lens, const int32_t* block_table, int B,
                                int max_pages_per_seq, void* const* k_cache,
                                void* const* v_cache, int num_pages, int64_t* draft_keys,
                                float* logits_out, void* workspace, size_t workspace_bytes,
                                void* stream, dflash_allreduce_fn exchange, void* user);

/* Drafts from the exchanged keys of dflash_propose_keys: draft_tokens [B, K]
 * int32 = the vocabulary id in each key; block_tokens [B, block_size] int32
 * (nullable) = cat(bonus_tokens[b], drafts[b]).  A key that names no id below
 * `vocab` (no shard wrote the row) gives -1 and sets DFLASH_DEVERR_INPUT in
 * *device_error (nullable).  Host errors: B < 0, block_size < 2, vocab < 1, a
 * missing pointer.  One launch on the device of `stream`; B == 0 is a no-op. */
dflash_status dflash_finalize_draft_keys(const int64_t* draft_keys, const int32_t* bonus_tokens,
                                         int B, int block_size, int vocab,
                                         int32_t* draft_tokens, int32_t* block_tokens,
                                         unsigned* device_error, void* stream);

/* Greedy verification.  target_logits row j (j = 0..K) of request b is the
 * target's prediction after block slot j (slot 0 = previous bonus token,
 * slot j = drafts[b][j-1]).  With t_j = argmax_v target_logits[b][j][v] (fp32
 * compare, ties -> lowest index, NaN counts as -inf):
 *   n = largest m <= K with drafts[b][i] == t_i for all i < m
 *   out_tokens[b] = [drafts[b][0..n-1], t_n, -1, ..., -1]   ([B, K+1] int32)
 *   num_accepted[b] = n, bonus[b] = t_n                      ([B] int32 each)
 * drafts [B, K] int32; target_logits [B, K+1, V] fp32.  Bit-exact by construction.
 * B == 0 is a no-op; B * (K + 1) > 2^30 rows is DFLASH_ERR_UNSUPPORTED_SHAPE.
 * Needs dflash_verify_workspace_bytes(B, K, V). */
dflash_status dflash_verify_greedy(const int32_t* drafts, const float* target_logits,
                                   int B, int K, int V, int32_t* out_tokens,
                                   int32_t* num_accepted, int32_t* bonus,
                                   void* workspace, size_t workspace_bytes,
                                   void* stream);

/* ---- the whole speculative step ------------------------------------------ */

/* Buffers of one speculative-decoding step (dflash_spec_step).  Device
 * pointers, caller-owned; K = block_size - 1, V = vocab, n target rows.
 * Inputs:
 *   prev_drafts        [B, K] int32   the drafts the target has just scored
 *   target_logits      [B, K+1, V] fp32  the target's predictions after each
 *                      verified slot (as for dflash_verify_greedy)
 *   target_positions   [n] int64      optimistic positions of the target rows
 *   last_token_indices [B] int32      last target row of each request
 *   num_draft          [B] int32      drafts verified this step per request
 *                      (cur_num_draft of dflash_prepare_proposal_inputs)
 *   prev_sampled       [B, prev_width] int32 and prev_num_draft [B] int32: the
 *                      previous step's sampler output, both NULL on a first step
 *   aux                [n, T*H] bf16  the target's tapped states of the rows
 *   block_table        [B, max_pages_per_seq] int32
 *   k_cache, v_cache   HOST arrays of n_layers device pointers (paged pools of
 *                      num_pages pages, as for dflash_inject_context)
 * Outputs:
 *   out_tokens [B, K+1], num_accepted [B]     verification (the accepted
 *                                             tokens of this step)
 *   positions, slot_mapping [n] int64         corrected rows of the injection
 *   seq_lens, bonus [B] int32                 the new block's start and first token
 *   draft_tokens [B, K], block_tokens [B, bs] (nullable) the next proposal
 *   device_error (device word)                input errors seen by the
 *                                             preparation (DFLASH_DEVERR_INPUT);
 *                                             NULL: the handle's error word
 *                                             (dflash_check_device_errors) */
typedef struct dflash_step_io {
  int B;
  int n;
  const int32_t* prev_drafts;
  const float* target_logits;
  const int64_t* target_positions;
  const int32_t* last_token_indices;
  const int32_t* num_draft;
  const int32_t* prev_sampled;
  int prev_width;
  const int32_t* prev_num_draft;
  const void* aux;
  const int32_t* block_table;
  int max_pages_per_seq;
  void* const* k_cache;
  void* const* v_cache;
  int num_pages;
  int32_t* out_tokens;
  int32_t* num_accepted;
  int64_t* positions;
  int64_t* slot_mapping;
  int32_t* seq_lens;
  int32_t* bonus;
  int32_t* draft_tokens;
  int32_t* block_tokens;
  unsigned* device_error;
} dflash_step_io;

/* Workspace needed by dflash_spec_step (and dflash_step_graph_create) for B
 * requests, n target rows and block tables max_pages_per_seq wide: the
 * verification's, the injection's and the proposal's workspaces side by side
 * (256-byte aligned pieces).  0 for invalid sizes. */
size_t dflash_spec_step_workspace_bytes(const dflash_handle* h, int B, int n,
                                        int max_pages_per_seq);

/* One whole speculative step with no host round trip (§"Async Rejection and
 * Position Correction": with the proposal inputs prepared on the device the
 * step needs nothing from the host between its stages):
 *   1. dflash_verify_greedy(prev_drafts, target_logits) -> out_tokens,
 *      num_accepted (its bonus is written to `bonus`, then rewritten by 2.
 *      with the same value: the last valid entry of out_tokens);
 *   2. dflash_prepare_proposal_inputs(target_positions, last_token_indices,
 *      cur_sampled = out_tokens (width K+1), num_draft, prev_sampled,
 *      prev_num_draft) -> positions, slot_mapping, seq_lens, bonus;
 *   3. dflash_inject_context over the n target rows (padding rows, slot -1,
 *      are skipped);
 *   4. dflash_propose(bonus, seq_lens) -> draft_tokens, block_tokens.
 * Every argument is checked on the host before the first launch (the checks
 * of the four calls, plus n >= B when B > 0); B == 0 is a no-op.  The calls
 * only enqueue work on `stream`, so the step may be captured into a CUDA graph
 * (dflash_step_graph_create does that). */
dflash_status dflash_spec_step(dflash_handle* h, const dflash_step_io* io, void* workspace,
                               size_t workspace_bytes, void* stream);

/* A speculative step captured once into a CUDA graph owned by the library
 * (every launch of dflash_spec_step with PDL edges kept), replayed by
 * dflash_step_graph_launch on any stream of the handle's device.  The graph
 * holds the pointers of `io` and `workspace` (and the handle's weights): the
 * caller rewrites the inputs in place between launches and keeps every buffer
 * alive until dflash_step_graph_destroy.  Feeding a step's drafts to the next
 * step as prev_drafts means two graphs over two buffer sets, or a copy.
 * create: the same host checks as dflash_spec_step (DFLASH_ERR_INVALID_ARG as
 * well while launch profiling is enabled on the handle), captured on a stream
 * of the handle's device; nothing runs until the first launch.  Errors:
 * DFLASH_ERR_CUDA if capture or instantiation fails (e.g. a capture already
 * open on the calling thread).  B == 0 gives a graph whose launches do
 * nothing. */
typedef struct dflash_step_graph dflash_step_graph;
dflash_status dflash_step_graph_create(dflash_handle* h, const dflash_step_io* io,
                                       void* workspace, size_t workspace_bytes,
                                       dflash_step_graph** out);
dflash_status dflash_step_graph_launch(dflash_step_graph* g, void* stream);
/* NULL is a no-op; the caller makes sure no launch of the graph is pending. */
void dflash_step_graph_destroy(dflash_step_graph* g);

/* ---- component entry points (each runs one kernel family of the path) ---- */

/* out[m, n] = sum_k A[m, k] * W[n, k] in fp32 — the tcgen05 GEMM that every
 * projection of the path runs on, with a plain fp32 store as its epilogue.
 *   A [M, K] bf16, W [N, K] bf16 (row-major), out [M, N] fp32.
 * K must be a multiple of 64 and N a multiple of 32.  M == 0 is a no-op.
 * Needs dflash_linear_workspace_bytes(h, M, N, K) of workspace. */
size_t dflash_linear_workspace_bytes(const dflash_handle* h, int M, int N, int K);
dflash_status dflash_linear(dflash_handle* h, const void* A, const void* W, int M, int N,
                            int K, float* out, void* workspace, size_t workspace_bytes,
                            void* stream);
/* Same with the launch plan chosen by the caller: tile width block_n in
 * {32, 64, 128, 256}; `splits` = 1 schedules whole tiles, n >= 2 schedules
 * stream-K with ceil(K/64 / n) k-blocks per CTA (<= K/64); 0 for either means
 * "as the automatic plan".  Stream-K needs 2 * CTAs * min(M,128) * block_n * 4
 * bytes of workspace, CTAs <= tiles * n + 1 (dflash_linear_workspace_bytes
 * covers only the automatic plan). */
dflash_status dflash_linear_ex(dflash_handle* h, const void* A, const void* W, int M, int N,
                               int K, float* out, int block_n, int splits, void* workspace,
                               size_t workspace_bytes, void* stream);

/* One layer of non-causal block attention (§"What is DFlash": every block query
 * attends to the injected context and the whole block), on a layer's caches:
 *   q [B*bs, n_q_heads, head_dim] bf16 (block rows in request order)
 *   o [B*bs, n_q_heads*head_dim] fp16 out (as the proposal path stores it)
 * Request b attends to its logical keys [0, seq_lens[b] + bs), located through
 * block_table exactly as in dflash_propose; scale 1/sqrt(head_dim).
 * B > 65535 is DFLASH_ERR_UNSUPPORTED_SHAPE.
 * Needs dflash_attention_workspace_bytes(h, B, max_pages_per_seq). */
size_t dflash_attention_workspace_bytes(const dflash_handle* h, int B, int max_pages_per_seq);
dflash_status dflash_block_attention(dflash_handle* h, const void* q, const int32_t* seq_lens,
                                     const int32_t* block_table, int B, int max_pages_per_seq,
                                     const void* k_cache, const void* v_cache, int num_pages,
                                     void* o, void* workspace, size_t workspace_bytes,
                                     void* stream);

/* The attention launch plan that a proposal with this geometry uses
 * (diagnostics; host only, no device needed): kv groups of bs * G query rows
 * (G = query heads per kv head), block tables of W pages of P keys, on
 * `num_sms` SMs.  forced_ring: 0 (the planner's choice), 2 or 6 as
 * DFLASH_ATTN_STAGES forces it (the one-CTA-per-tile kernel with that ring);
 * flags: bit 0 the opt-in cluster combine, bit 1 the opt-in persistent
 * kernel, bit 2 32-key tiles for the two-CTA kernel (DFLASH_ATTN_TILE=32).
 * Without bits 0-1 or a forced ring, head_dim 128 takes the two-CTA-per-SM
 * kernel with P V transposed (64-key tiles in a two-deep ring; with bit 2,
 * 32-key tiles in a four-deep ring),
 * its splits sized for 8 CTAs per SM.  Written to *out;
 * DFLASH_ERR_INVALID_ARG for a non-positive size or a NULL out. */
typedef struct dflash_attention_plan {
  int tcgen05;        /* 1: the tcgen05 kernel (bs * G <= 64), 0: the mma.sync kernel */
  int keys_per_tile;  /* tcgen05 kernels: 32, 64 or 128 */
  int ring_depth;     /* tcgen05 kernels: K/V tiles in flight per CTA (2, 4 or 6) */
  int ctas_per_sm;    /* tcgen05 kernels: 2 for the two-CTA kernels, else 1 */
  int chunk_keys;     /* keys per split */
  int max_splits;     /* splits of the longest request */
  int cluster;        /* splits combined inside a thread-block cluster */
  int persistent;     /* persistent CTAs walking the items */
  int transposed_pv;  /* head_dim 128 default: two CTAs per SM, O^T = V^T P^T (M = 128) */
} dflash_attention_plan;
dflash_status dflash_plan_attention_info(int B, int n_kv_heads, int max_pages_per_seq,
                                         int page_size, int block_size, int q_per_kv,
                                         int head_dim, int num_sms, int forced_ring, int flags,
                                         dflash_attention_plan* out);

/* The GEMM launch plan the library takes for D[M, N] = A[M, K] W[N, K]^T
 * with an epilogue that groups `group` output columns (32, 64 or 128), host
 * only (no device, no allocation).  On a device the library queries how many
 * thread-block clusters fit at once; here those capacities are parameters:
 * clusters of S CTAs for the few-row cluster split-K are taken as
 * num_sms / S, and pair_split_cap is the number of four-CTA clusters of the
 * split-K pair kernel that fit (0: never split).  K must be a multiple of 64.
 * DFLASH_ERR_INVALID_ARG for sizes out of range. */
typedef struct dflash_gemm_plan {
  int pair;           /* 1: CTA pairs (tcgen05.mma.cta_group::2), 0: one SM per tile */
  int tile_m;         /* rows of a tile (256 for pairs, 128 otherwise) */
  int tile_n;         /* columns of a tile */
  int k_splits;       /* pairs: K split over this many pairs; one SM: cluster split-K size */
  int stream_k;       /* one SM: (tile, k-block) iterations dealt in equal ranges */
  int staged;         /* one SM: the few-row staged epilogue (M <= 32) */
  int tiles;          /* output tiles */
  int grid;           /* CTAs launched (pairs: an upper bound before the occupancy query) */
} dflash_gemm_plan;
dflash_status dflash_plan_gemm_info(int M, int N, int K, int group, int num_sms,
                                    int pair_split_cap, dflash_gemm_plan* out);

/* ---- a small causal target model on the device ---------------------------
 *
 * DFlash reads the target model's auxiliary hidden states (§"Target Auxiliary
 * Hidden State Extraction"): the target captures the residual stream BEFORE
 * the requested layers and returns the captured states concatenated, one
 * [n, n_capture * hidden] tensor per forward, the input of
 * dflash_inject_context.  The draft checkpoint's target_layer_ids name the
 * state AFTER layer i (HuggingFace output hidden-state ids), so the runner
 * asks the target for layer i + 1 (the page's "crucial off-by-one").
 *
 * dflash_target_* is a small Qwen3-style causal LM with that capture
 * interface (the same layer as the draft's, with causal attention and an
 * un-aliased final norm + LM head), so that the whole speculative loop —
 * target forward, greedy verification, injection, proposal — runs on the
 * device and can be checked against plain greedy decoding of the same target.
 * It is built for exact reproducibility, not speed: fp32 weights and
 * activations, and every output element reduced in one fixed order that does
 * not depend on how many rows a call processes, so a token at a position gets
 * bit-identical logits whether decoded alone or inside a block.  One sequence
 * per instance; its K/V cache ([n_layers][max_len][n_kv_heads][head_dim] fp32)
 * is owned by the instance. */

/* capture_layers[i] = target_layer_ids[i] + 1 (host arrays of n entries); each
 * id must lie in [0, target_n_layers - 1] (DFLASH_ERR_INVALID_ARG otherwise):
 * capture layer target_n_layers is the last layer's output, before the final
 * norm. */
dflash_status dflash_aux_capture_layers(const int* target_layer_ids, int n, int target_n_layers,
                                        int* capture_layers);

typedef struct dflash_target_config {
  int hidden;
  int n_layers;
  int n_q_heads;
  int n_kv_heads;
  int head_dim;                /* a multiple of 32, <= 128 */
  int intermediate;
  int vocab;
  float rms_eps;
  float rope_theta;
  int max_len;                 /* the sequence's positions [0, max_len) */
  int n_capture;               /* captured states per row (may be 0) */
  const int* capture_layers;   /* HOST [n_capture]: pre-layer index in [0, n_layers] */
} dflash_target_config;

/* DEVICE pointers, fp32, row-major [out, in]; per-layer entries are HOST arrays
 * of n_layers device pointers; all used in place except wq|wk|wv and
 * w_gate|w_up, which the instance stacks into copies of its own.
 *   embed, lm_head [vocab, hidden]; final_norm_w, in_norm_w, post_norm_w [hidden];
 *   wq [Hq*d, hidden]; wk, wv [Hkv*d, hidden]; wo [hidden, Hq*d];
 *   q_norm_w, k_norm_w [d]; w_gate, w_up [I, hidden]; w_down [hidden, I] */
typedef struct dflash_target_weights {
  const float* embed;
  const float* final_norm_w;
  const float* lm_head;
  const float* const* in_norm_w;
  const float* const* post_norm_w;
  const float* const* wq;
  const float* const* wk;
  const float* const* wv;
  const float* const* wo;
  const float* const* q_norm_w;
  const float* const* k_norm_w;
  const float* const* w_gate;
  const float* const* w_up;
  const float* const* w_down;
} dflash_target_weights;

typedef struct dflash_target dflash_target;

/* Allocates the instance (weight copies, K/V cache, error word) on `device`
 * and synchronizes it.  DFLASH_ERR_INVALID_ARG for missing pointers or sizes,
 * a capture layer outside [0, n_layers]; DFLASH_ERR_UNSUPPORTED_SHAPE for a
 * head_dim that is not a multiple of 32 up to 128, or n_q_heads not a multiple
 * of n_kv_heads. */
dflash_status dflash_target_create(const dflash_target_config* cfg,
                                   const dflash_target_weights* w, int device,
                                   dflash_target** out);
void dflash_target_destroy(dflash_target* t);
size_t dflash_target_workspace_bytes(const dflash_target* t, int n);

/* Forward of tokens[0..n) (DEVICE int32) at positions [start_pos, start_pos + n)
 * of the instance's sequence: writes their K/V into the cache, attends
 * causally over [0, position], and writes
 *   logits [n, vocab] fp32 (DEVICE): the prediction after each token;
 *   aux [n, n_capture * hidden] bf16 (DEVICE; may be NULL when n_capture == 0):
 *     row r, slot k = the residual state of token r before layer
 *     capture_layers[k] (the embedding for 0, the last layer's output for
 *     n_layers).
 * Positions at or past start_pos + n of the cache are untouched (stale rows of
 * rejected tokens are overwritten by the next forward that covers them).
 * Host errors: start_pos < 0 or start_pos + n > max_len, missing pointers
 * (DFLASH_ERR_INVALID_ARG), a workspace below dflash_target_workspace_bytes
 * (DFLASH_ERR_WORKSPACE).  A token outside [0, vocab) embeds as zeros and sets
 * DFLASH_DEVERR_TOKEN (dflash_target_check_device_errors). */
dflash_status dflash_target_forward(dflash_target* t, const int32_t* tokens, int n, int start_pos,
                                    float* logits, void* aux, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* Synchronizes the device, reads and clears the instance's device error word. */
dflash_status dflash_target_check_device_errors(dflash_target* t, unsigned* bits);

/* ---- launch accounting and per-launch timing (diagnostics) ---- */

/* Kernel families launched by the calls above (ids for dflash_profile_read). */
enum {
  DFLASH_KERNEL_EMBED_NORM = 0,      /* block build + embedding + first RMSNorm       */
  DFLASH_KERNEL_GEMM_QKV = 1,        /* QKV GEMM + q/k norm + RoPE + block K/V write  */
  DFLASH_KERNEL_ATTENTION = 2,       /* non-causal paged block attention             */
  DFLASH_KERNEL_ATTN_COMBINE = 3,    /* split-KV merge                               */
  DFLASH_KERNEL_GEMM_O = 4,          /* O projection + residual                      */
  DFLASH_KERNEL_RMSNORM = 5,         /* row RMSNorms (post-attn, next input, final, hidden_norm) */
  DFLASH_KERNEL_GEMM_GATE_UP = 6,    /* gate/up GEMM + SwiGLU                        */
  DFLASH_KERNEL_GEMM_DOWN = 7,       /* down projection + residual                   */
  DFLASH_KERNEL_GEMM_LM_HEAD = 8,    /* LM head + fused greedy argmax                */
  DFLASH_KERNEL_ARGMAX_FINALIZE = 9, /* draft / block token write-out                */
  DFLASH_KERNEL_GEMM_FC = 10,        /* fc over the tapped states                    */
  DFLASH_KERNEL_GEMM_KV_INJECT = 11, /* all layers' K/V + k_norm + RoPE + scatter    */
  DFLASH_KERNEL_LINEAR = 12,         /* dflash_linear / dflash_linear_ex             */
  DFLASH_KERNEL_GEMM_MLP = 13,       /* few rows: gate/up + SwiGLU + down + residual, one launch */
  DFLASH_KERNEL_KINDS = 14
};

/* Number of kernel launches the handle's calls have issued so far (launches
 * captured into a CUDA graph are counted once, at capture). */
unsigned long long dflash_launch_count(const dflash_handle* h);

/* Static name of a kernel family id, or NULL. */
const char* dflash_kernel_name(int kind);

/* While enabled, each launch of the handle's calls (up to max_launches of them
 * until the next read) is bracketed by two CUDA events recorded on the call's
 * stream.  dflash_profile_read synchronizes the device, returns per family k <
 * n_kinds the number of recorded launches and their summed event time (ms),
 * and restarts the recording.  Enabling allocates the events (a set-up call,
 * not for use inside stream capture). */
dflash_status dflash_profile_enable(dflash_handle* h, int max_launches);
dflash_status dflash_profile_read(dflash_handle* h, int n_kinds, int* launches,
                                  double* total_ms);
dflash_status dflash_profile_disable(dflash_handle* h);

/* Synchronizes the device, reads and clears the handle's device error word.
 * Returns DFLASH_OK if it was zero, DFLASH_ERR_DEVICE_TIMEOUT if the timeout bit
 * was set, DFLASH_ERR_DEVICE_BOUNDS otherwise; *bits (may be NULL) receives the
 * raw DFLASH_DEVERR_* mask.  (verify and paged_slots take no handle and have
 * no device-detected error conditions.) */
dflash_status dflash_check_device_errors(dflash_handle* h, unsigned* bits);

/* Diagnostics.  Every bounded wait of the library's kernels (pipeline
 * barriers, cross-CTA arrival counters) gives up after `cycles` SM clock
 * cycles on `device`, sets DFLASH_DEVERR_TIMEOUT and lets its kernel wind down
 * (default 4e9 cycles, about 2 s).  One value per device for the whole
 * process; set it only while no kernel of the library runs on the device
 * (the call synchronizes with the device).  DFLASH_ERR_INVALID_ARG for
 * cycles <= 0. */
dflash_status dflash_set_wait_limit(int device, long long cycles);

/* Diagnostics: enqueues one kernel on `stream` whose single bounded wait can
 * never complete (an mbarrier that nothing arrives on), so that it runs out
 * after the device's wait limit and sets DFLASH_DEVERR_TIMEOUT in the handle's
 * error word; dflash_check_device_errors then returns
 * DFLASH_ERR_DEVICE_TIMEOUT.  Nothing faults or traps and the context stays
 * usable; the handle's next calls run normally once the bit is read. */
dflash_status dflash_selftest_wait_timeout(dflash_handle* h, void* stream);

/* Static, human-readable name of a status code. */
const char* dflash_status_string(dflash_status s);

/* Library build identification (static string). */
const char* dflash_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DFLASH_H_ */
