/*
 * pp.h - C ABI of libpp, exact softmax attention over a preference-packed sequence on B200 (sm_100a).
 *
 * Problem (pages: "Preference Packing: Efficient Preference Optimization for LLMs", abstract and method digest;
 * "prefix_grouper_utils.py", section 1 building position ids, section 2 building the grouper, and the
 * prefix-sharing diagram; "PackInfer: Compute- and I/O-Efficient Attention for Batched LLM Inference", abstract):
 * a batch of G groups is packed into one flat sequence of T tokens. Group g stores its prompt prefix P_g once,
 * followed by its k_g responses S_g1..S_gk. A prefix token attends causally within the prefix; a token of S_i
 * attends to the whole prefix and causally within S_i, never to a sibling response or to another group. Position
 * ids run 0..P_g-1 on the prefix and restart at P_g for every response.
 *
 * Conventions for every call
 *   - Ownership: the caller owns all memory. The library allocates nothing on the device or the host (apart from a
 *     few small static tables of its own); every buffer is passed in as a raw pointer with its size.
 *   - Pointers: "_d" names and every tensor argument are DEVICE pointers on the current CUDA device, except where a
 *     comment says host. Tensors are dense and row-major:
 *       Q, O, dO, dQ: [T, Hq, d]; K, V, dK, dV: [T, Hkv, d]; LSE: [Hq, T] fp32; pos ids: int32 [T].
 *     The packed order is group by group: prefix, then the responses in order.
 *   - Asynchrony: every call only enqueues work on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *     returns without synchronising, except pp_get_status().
 *   - Errors: arguments are validated on the host before anything is enqueued; an invalid argument returns
 *     PP_ERR_INVALID_ARG (or PP_ERR_UNSUPPORTED / PP_ERR_WORKSPACE) and enqueues nothing. A failed launch returns
 *     PP_ERR_CUDA. Problems only the device can see (inconsistent descriptors, a bounded wait that ran out) set a
 *     device error word that pp_get_status() reads. pp_last_error() returns a message for the calling thread.
 *   - Limits: T < 2^31 - 256; d in {64, 128}; Hq % Hkv == 0; Hq <= 256.
 */
#ifndef PP_H_
#define PP_H_

#include <stdint.h>

#if defined(__GNUC__)
#define PP_API __attribute__((visibility("default")))
#else
#define PP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PP_OK = 0,
    PP_ERR_INVALID_ARG = -1,   /* host-side validation failed; nothing was enqueued */
    PP_ERR_UNSUPPORTED = -2,   /* valid but unsupported combination (e.g. backward in fp32) */
    PP_ERR_CUDA = -3,          /* a CUDA runtime/driver call failed */
    PP_ERR_DEVICE_TIMEOUT = -4,/* a kernel's bounded wait ran out (reported by pp_get_status) */
    PP_ERR_WORKSPACE = -5,     /* a buffer is smaller than the size the library asked for */
    PP_ERR_DEVICE_INPUT = -6   /* the device found inconsistent descriptors (reported by pp_get_status) */
} pp_status;

typedef enum { PP_BF16 = 0, PP_FP32 = 1 } pp_dtype;

/* One group's descriptor ("prefix_grouper_utils.py" section 1: each group carries its prefix length and its
 * responses' lengths). The response lengths themselves are the segments of cu_seqlens. */
typedef struct {
    int32_t prefix_len;    /* P_g >= 0 */
    int32_t num_suffixes;  /* k_g >= 0 */
} pp_group_desc;

/* Which pass a workspace size is asked for. */
enum { PP_PASS_FWD = 0, PP_PASS_BWD = 1 };

/* ---------------------------------------------------------------------------------------------------------------
 * pp_meta_bounds (host only, no device work)
 * Upper bound on the bytes of the metadata buffer that pp_build_meta fills, from the sizes alone.
 *   num_groups G >= 1, num_segments = sum_g (1 + k_g), total_tokens T >= 0, num_heads_q / num_heads_kv as for the
 *   attention calls. *meta_bytes (host pointer) receives the size. Errors: PP_ERR_INVALID_ARG.
 */
PP_API pp_status pp_meta_bounds(int32_t num_groups, int32_t num_segments, int64_t total_tokens, int32_t num_heads_q,
                         int32_t num_heads_kv, int64_t *meta_bytes);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_build_meta: group descriptors + segment boundaries -> grouped position ids and the tile schedule.
 * ("prefix_grouper_utils.py" section 1 for the position ids; "PackInfer" abstract for building the attention work
 * directly over the packed query-key regions and balancing it across thread blocks.)
 *   groups_d      device pp_group_desc[num_groups]
 *   cu_seqlens_d  device int32[num_segments + 1]: packed segment boundaries in the packed order (for each group its
 *                 prefix, then each response); zero-length segments allowed. cu[0] must be 0, cu[nseg] must be T,
 *                 and num_segments must equal sum_g (1 + k_g); a violation found on the device sets
 *                 PP_ERR_DEVICE_INPUT (pp_get_status) and leaves the outputs undefined.
 *   pos_ids_d     device int32[T] out: position ids (prefix 0..P-1, every response restarts at P).
 *   meta_d        device buffer out, meta_bytes >= the pp_meta_bounds value, 256-byte aligned. Its content is
 *                 private to the library (read it only through the calls below); it holds the per-token segment
 *                 table, the forward query tiles (128 rows, aligned to each group's start) in cost order, and the
 *                 backward key/value tiles (128 rows) split into work chunks in cost order.
 * The buffers must stay alive and unchanged while attention calls that use them are in flight.
 */
PP_API pp_status pp_build_meta(const pp_group_desc *groups_d, int32_t num_groups, const int32_t *cu_seqlens_d,
                        int32_t num_segments, int64_t total_tokens, int32_t num_heads_q, int32_t num_heads_kv,
                        int32_t *pos_ids_d, void *meta_d, int64_t meta_bytes, void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_meta_tiles: expand the schedule in meta_d into explicit tiles, for checking and inspection.
 *   which = PP_PASS_FWD: query tiles of 128 rows x key tiles of 128 rows; PP_PASS_BWD: key tiles of 128 rows x
 *   query tiles of 128 rows. Both are aligned to each group's start. Writes one int32 triple
 *   (q_row0, kv_row0, class) per non-empty tile into tiles_d (device int32[3 * capacity]), class 1 = every pair in
 *   the tile allowed (FULL), 2 = some allowed (PARTIAL); fully masked tiles are never listed. *count_d (device
 *   int32) receives the number of tiles (possibly > capacity; only the first `capacity` are written). The order is
 *   unspecified. The classification is the same device code the attention kernels use.
 */
PP_API pp_status pp_meta_tiles(const void *meta_d, int32_t which, int32_t *tiles_d, int64_t capacity, int32_t *count_d,
                        void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_meta_schedule: the work lists the attention kernels execute, in their stored order, for checking.
 * ("PackInfer" abstract: attention work over the packed query-key regions, ordered to balance the thread blocks.)
 *   which = PP_PASS_FWD: the forward query tiles in cost order (the order pp_attn_fwd and the dQ half of
 *   pp_attn_bwd walk them); one record per key tile a query tile visits. which = PP_PASS_BWD: the backward work
 *   chunks (key tile x a range of its query tiles) in their stored order; one record per query tile of a chunk.
 *   Each record is five int32 (item, q_row0, kv_row0, class, split): item = position of the query tile (fwd) or of
 *   the chunk (bwd) in its list; class 1 = FULL, 2 = PARTIAL; split = 1 if the chunk's key tile is split over
 *   several chunks (its dK/dV partials are added in fp32), else 0 (always 0 for fwd). records_d: device
 *   int32[5 * capacity]; *count_d (device int32) receives the number of records (only the first `capacity` are
 *   written). The order of the records is unspecified; their item fields give the stored order.
 */
PP_API pp_status pp_meta_schedule(const void *meta_d, int32_t which, int32_t *records_d, int64_t capacity,
                                  int32_t *count_d, void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_rope: rotary embedding at the grouped position ids, in place on q and k (v untouched).
 * Rotate-half form with base theta: for m < d/2, w_m = theta^(-2m/d), a = pos * w_m,
 *   y_m = x_m cos a - x_{m+d/2} sin a,  y_{m+d/2} = x_{m+d/2} cos a + x_m sin a
 * (the pages give the positions, "prefix_grouper_utils.py" section 1, but not the variant; rotate-half is the
 * reading taken). inverse != 0 rotates by -a, which maps gradients of the rotated tensors back.
 *   q: [T, hq, d], k: [T, hkv, d] (either may be NULL to skip it), dt = PP_BF16 or PP_FP32 storage; the angle is
 *   formed in fp64 and the rotation in fp32, rounded to nearest even on store. theta > 0 (0 means 10000).
 */
PP_API pp_status pp_rope(void *q, void *k, const int32_t *pos_ids_d, int64_t T, int32_t hq, int32_t hkv, int32_t d,
                  float theta, pp_dtype dt, int32_t inverse, void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_workspace_bytes (host only): scratch bytes pp_attn_fwd (which = PP_PASS_FWD) or pp_attn_bwd
 * (PP_PASS_BWD) needs for these sizes. *bytes (host pointer) receives it.
 */
PP_API pp_status pp_workspace_bytes(int32_t which, int64_t T, int32_t hq, int32_t hkv, int32_t d, int64_t *bytes);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_bwd_ds_bytes (host only): extra backward workspace, beyond pp_workspace_bytes(PP_PASS_BWD, ...), that lets
 * pp_attn_bwd keep one dS tile (128 keys x 128 queries, bf16, 32 KiB) per backward step and form dq from them
 * instead of recomputing the scores. A step is (key tile of 128 rows, query tile of 128 rows that attends it, q
 * head), for every kv head; the count follows the mask (same descriptors as pp_build_meta). groups_host,
 * cu_host: host copies of the descriptors and segment bounds; *bytes (host) receives 1024 + steps * 32768.
 * Returns PP_ERR_INVALID_ARG for descriptors that disagree with the segments or segment bounds that decrease.
 */
PP_API pp_status pp_bwd_ds_bytes(const pp_group_desc *groups_host, int32_t G, const int32_t *cu_host,
                                 int32_t nseg, int32_t hq, int32_t hkv, int64_t *bytes);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_attn_fwd: O and the per-row log-sum-exp of exact packed attention.
 *   s_ij = softmax_scale * q_i . k_j over the allowed keys j of row i (q head h reads kv head h / (hq/hkv));
 *   lse_i = ln sum_j exp(s_ij) (natural log of the scaled scores); o_i = sum_j exp(s_ij - lse_i) v_j.
 *   q, k, v: inputs as above in dtype dt (PP_BF16: tcgen05 tensor-core path, fp32 accumulation;
 *   PP_FP32: fp32 CUDA-core path, meant for small checks). o: [T, hq, d] out in dt; lse: [hq, T] fp32 out.
 *   softmax_scale 0 means 1/sqrt(d). meta_d from pp_build_meta with the same T, hq, hkv.
 *   workspace: device scratch of ws_bytes >= pp_workspace_bytes(PP_PASS_FWD, ...), 256-byte aligned; contents
 *   need not be initialised. Rows of fully masked positions do not exist (every row attends at least itself).
 */
PP_API pp_status pp_attn_fwd(const void *q, const void *k, const void *v, const void *meta_d, int64_t T, int32_t hq,
                      int32_t hkv, int32_t d, float softmax_scale, pp_dtype dt, void *o, float *lse,
                      void *workspace, int64_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_attn_bwd: gradients of sum(O * dO) with respect to q, k and v (bf16 only).
 *   D_i = dO_i . o_i; p_ij = exp(s_ij - lse_i); dS_ij = p_ij (dO_i . v_j - D_i);
 *   dq_i = scale sum_j dS_ij k_j; dk_j = scale sum_h sum_i dS_ij q_i; dv_j = sum_h sum_i p_ij dO_i
 *   (sums over the q heads h that share kv head j's head). q, k, v, o, lse: the forward's inputs and outputs;
 *   dout: [T, hq, d]. dq, dk, dv: outputs in bf16 with the shapes of q, k, v (fully overwritten).
 *   workspace: ws_bytes >= pp_workspace_bytes(PP_PASS_BWD, ...), 256-byte aligned, contents need not be
 *   initialised. It holds (-lse/scale, -D) per row and q head, and fp32 dK/dV for the prefix key tiles, which are
 *   attended by every response of their group and so are split into chunks whose partials are added there (fp32
 *   reduction adds, one per element and chunk) before conversion to bf16. Each row tile of dq is produced by exactly
 *   one CTA (no reduction). If ws_bytes also covers pp_bwd_ds_bytes(...) for the batch, the dK/dV kernel keeps
 *   every step's dS tile after the base workspace and dq is formed from them (the fast path); otherwise the dq
 *   kernel recomputes the tile's scores and dP. The choice is made on the device from the batch's step count, so
 *   either size is valid. A batch of T tokens that could exceed 2^31 - 1 steps per kv head (about 4.2 M tokens at
 *   hq/hkv = 4) always takes the recompute path. The result is deterministic except for the order of the dK/dV adds.
 */
PP_API pp_status pp_attn_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
                      const void *dout, const void *meta_d, int64_t T, int32_t hq, int32_t hkv, int32_t d,
                      float softmax_scale, void *dq, void *dk, void *dv, void *workspace, int64_t ws_bytes,
                      void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_attn_bwd_noalloc: pp_attn_bwd for callers that cannot allocate device memory.
 * (The paper has no counterpart; this is a convenience of the library.)
 * Some callers cannot call cudaMalloc or ask anyone for a scratch buffer: a plugin or custom op handed only its
 * input and output pointers by a host framework whose caching allocator owns the device memory, or code that must
 * not allocate at that point. This entry point takes the same arguments as pp_attn_bwd minus the workspace, and
 * uses instead a scratch array compiled into the library (a file-scope __device__ array of
 * PP_NOALLOC_SCRATCH_BYTES = 64 MiB; every GPU that loads libpp holds it until the process exits). It calls no
 * allocator at all.
 *   Limit: the scratch a call needs (pp_workspace_bytes(PP_PASS_BWD, T, hq, hkv, d)) must fit in 64 MiB, e.g.
 *   T <= about 7,600 tokens at 32/8 heads and d = 128; a larger call returns PP_ERR_WORKSPACE and enqueues nothing.
 *   Set-up: the first call on each device looks up the array's device address (cudaGetSymbolAddress) with that
 *   device current; make that first call before any stream capture.
 *   Sharing: every call on a device uses the same array, which keeps the last call's contents; the call clears the
 *   parts that must start at zero itself. Calls that overlap on the GPU (other streams, other host threads) race
 *   on the array: serialise them.
 */
#define PP_NOALLOC_SCRATCH_BYTES (64ll << 20)
PP_API pp_status pp_attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const float *lse,
                              const void *dout, const void *meta_d, int64_t T, int32_t hq, int32_t hkv, int32_t d,
                              float softmax_scale, void *dq, void *dk, void *dv, void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_decode_attn: one decoding step of every response over a group-contiguous KV cache.
 * The cache holds the packed layout of pp_build_meta (each group's prefix rows, then each response's rows), the
 * newest token of each response last. Each response has one query (its newest token), which attends to its group's
 * prefix and its own rows, the packed mask at the response's last row ("PackInfer" abstract: group-contiguous KV
 * and attention over packed query-key regions; "Preference Packing": the prompt is shared by its responses).
 * A prefix chunk is read from HBM once per group and serves all of the group's responses (flash-decoding in
 * 128-key chunks on the tensor cores: the chunk's queries, every response that sees it times the r q heads of a kv
 * head, form the rows of S = Q K^T and O = P V; fp32 partials are combined per query). hq / hkv <= 128.
 *   q: [n_resp, hq, d] bf16, n_resp = num_segments - num_groups (responses in packed order). k_cache, v_cache:
 *   [T, hkv, d] bf16. groups_d, cu_d: the device descriptors and segment bounds of the cache (as for
 *   pp_build_meta; every response of nonzero length has its query's K/V as its last row). d = 128.
 *   o: [n_resp, hq, d] bf16; lse: [hq, n_resp] fp32 (natural log); a response with no keys gets 0 and -inf.
 *   workspace: ws_bytes >= pp_decode_workspace_bytes for the same descriptors, 256-byte aligned. Descriptors that
 *   disagree with T, num_segments or the sized workspace set PP_ERR_DEVICE_INPUT and yield NaN outputs.
 */
PP_API pp_status pp_decode_workspace_bytes(const pp_group_desc *groups_host, int32_t num_groups,
                                           const int32_t *cu_seqlens_host, int32_t num_segments, int32_t num_heads_q,
                                           int64_t *bytes);
PP_API pp_status pp_decode_attn(const void *q, const void *k_cache, const void *v_cache, const pp_group_desc *groups_d,
                                int32_t num_groups, const int32_t *cu_seqlens_d, int32_t num_segments, int64_t T,
                                int32_t hq, int32_t hkv, int32_t d, float softmax_scale, void *o, float *lse,
                                void *workspace, int64_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_pack_batch: pack an ungrouped micro-batch on the device ("prefix_grouper_utils.py" section 2, building the
 * grouper from a micro-batch). Consecutive samples with equal uids form a group (a uid that reappears later starts a
 * new group); the group's prefix is the valid prompt tokens of its first sample; the packed sequence is, group by
 * group, the prefix followed by each sample's valid response tokens, in order, without padding.
 *   prompts int32 [bs, Lp] and prompt_mask uint8 [bs, Lp]; responses int32 [bs, Lr] and response_mask uint8 [bs, Lr]
 *   (nonzero mask = valid token; padding may be on either side); uids int64 [bs]. 0 <= bs <= 8192.
 *   Outputs: packed_ids int32 [capacity >= bs * (Lp + Lr)] (first T written); groups pp_group_desc [bs] (first G
 *   written: prefix_len, num_suffixes = group size); cu_seqlens int32 [2 * bs + 1] (first nseg + 1 written: each
 *   group's prefix, then each response, empty segments kept; the layout pp_build_meta takes); sample_offsets
 *   int32 [bs, 2] = (packed offset of the sample's prompt if it heads its group, else -1; packed offset of its
 *   response); counts int32 [3] = {G, nseg = G + bs, T}. All device pointers; nothing is allocated.
 *   The counts are device values: a caller reads them (a synchronising copy) to size and call pp_build_meta.
 *   Errors: PP_ERR_INVALID_ARG (sizes, NULL pointers, capacity), PP_ERR_UNSUPPORTED (bs > 8192).
 */
PP_API pp_status pp_pack_batch(const int32_t *prompts, const uint8_t *prompt_mask, int32_t Lp, const int32_t *responses,
                               const uint8_t *response_mask, int32_t Lr, const int64_t *uids, int32_t bs,
                               int32_t *packed_ids, int64_t capacity, pp_group_desc *groups, int32_t *cu_seqlens,
                               int32_t *sample_offsets, int32_t *counts, void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_response_logprobs: log-probability of every response token under the packed logits (the read-out of
 * "prefix_grouper_utils.py" section 3: split_output(logits, include_prefix_last=1) puts the group's last prefix row
 * in front of each response's rows, the last row of each block is dropped, the rows are divided by the temperature,
 * and the log-softmax is read at each completion token).
 *   On the packed layout: the token at response row y is predicted by row y - 1, except a response's first token,
 *   which is predicted by its group's last prefix row (o_g + P_g - 1). out[y] = x[src, id_y] / temperature -
 *   ln sum_v exp(x[src, v] / temperature), computed in fp32 with one pass over the row.
 *   logits: [T, V] row-major, dt PP_BF16 or PP_FP32, aligned to its element size (rows need not be 16-byte
 *   aligned). token_ids: int32 [T], the packed input ids. meta_d from pp_build_meta for the same groups.
 *   temperature > 0. out: fp32 [T]; prefix rows, and a response's first token in a group with P_g = 0 (no row
 *   predicts it), get 0. All pointers are device pointers; nothing is allocated.
 *   A token id outside [0, V) writes NaN at its row and sets PP_ERR_DEVICE_INPUT (reported by pp_get_status).
 */
PP_API pp_status pp_response_logprobs(const void *logits, pp_dtype dt, int64_t V, const int32_t *token_ids,
                                      const void *meta_d, int64_t T, float temperature, float *out, void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_plan_batches (host only): plan training batches of packed preference groups ("Preference Packing" abstract and
 * method digest: packing combined with batch sorting, batch size following the lengths). A group costs its packed
 * length group_tokens[g] (P_g + sum of its response lengths). With sort_by_length != 0 the groups are taken longest
 * first (stable: ties keep their input order), otherwise in input order; batches are filled greedily in that order
 * up to token_capacity tokens; a group longer than the capacity forms a batch of its own.
 *   group_tokens: int64 [num_groups] (host, >= 0). order: int32 [num_groups] out, the groups in batch order.
 *   batch_of_group: int32 [num_groups] out. *num_batches out. token_capacity >= 1.
 *   Errors: PP_ERR_INVALID_ARG (no message is recorded for this call; it touches no device state).
 */
PP_API pp_status pp_plan_batches(const int64_t *group_tokens, int32_t num_groups, int64_t token_capacity,
                                 int32_t sort_by_length, int32_t *order, int32_t *batch_of_group, int32_t *num_batches);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_selftest_bounded_wait: exercise the error channel of the kernels' bounded waits without a fault.
 * (The pages have no counterpart; this checks the library's failure detection.) Every mbarrier wait in the attention
 * kernels gives up after a time limit (2 s), records PP_ERR_DEVICE_TIMEOUT in the device error word and returns, so
 * a stuck pipeline ends with an error status instead of a hung GPU. This call launches one small kernel whose single
 * wait, with the same wait code and the given limit, is on an mbarrier that nothing arrives on; it issues no copy and
 * no MMA, so nothing is in flight when the wait gives up. The next pp_get_status() returns PP_ERR_DEVICE_TIMEOUT
 * (and clears the word); the context stays usable.
 *   limit_ns in [1e3, 2e9]. waited_ns_d: device uint64 out, the time the wait took before it gave up (0 if it
 *   completed, which cannot happen here). Errors: PP_ERR_INVALID_ARG.
 */
PP_API pp_status pp_selftest_bounded_wait(int64_t limit_ns, unsigned long long *waited_ns_d, void *stream);

/* ---------------------------------------------------------------------------------------------------------------
 * pp_get_status: synchronises `stream`, then reads and clears this device's error word. Returns PP_OK,
 * PP_ERR_DEVICE_TIMEOUT, PP_ERR_DEVICE_INPUT or PP_ERR_CUDA (a sticky CUDA error is reported as such).
 */
PP_API pp_status pp_get_status(void *stream);

/* Message describing the last failure seen by the calling thread ("" if none). Valid until its next call. */
PP_API const char *pp_last_error(void);

/* Library version string. */
PP_API const char *pp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PP_H_ */
