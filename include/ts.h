/*
 * ts.h -- C ABI of libts, the B200 (sm_100a) TokenSelect decode-step library.
 *
 * TokenSelect picks, at every decode step and for every sequence, a small set
 * of critical cached tokens and runs attention over those tokens only.  The
 * method (TokenSelect GitHub README, section "Key Takeaways"; GrooveSquid
 * summary of the TokenSelect paper, medium-difficulty summary):
 *   1. criticality of each cached token, per query head, is the Query-Key dot
 *      product                                             -> ts_score
 *   2. per-head soft voting: each head's criticality is normalised by a
 *      softmax over the tokens and the heads' results are summed -> ts_score
 *   3. the highest-voted tokens, plus fixed sink and local windows, are
 *      selected                                             -> ts_select
 *   4. Selection Cache: when consecutive queries are similar the previous
 *      selection is reused                                  -> ts_selcache
 *   5. attention over the selected tokens                   -> ts_sparse_attn
 *
 * Conventions (every call):
 *   - All pointers named *_dev or documented as "device" are CUDA device
 *     memory owned by the caller.  libts never allocates device memory, keeps
 *     no device state between calls except inside the caller's workspace, and
 *     never synchronises the stream except in ts_get_device_status.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and target the current CUDA device.  Argument errors are
 *     detected on the host and returned before anything is launched; launch
 *     failures return TS_ERR_CUDA.  ts_last_error() describes the last error
 *     of the calling thread.
 *   - bf16 tensors are IEEE bfloat16 bit patterns.  There is no CPU fallback:
 *     every result is computed by sm_100a kernels.
 *   - A workspace must not be used by two calls that can run concurrently.
 */
#ifndef TS_H_
#define TS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define TS_API __attribute__((visibility("default")))
#else
#define TS_API
#endif

typedef enum {
    TS_OK = 0,
    TS_ERR_INVALID_ARG = 1,     /* bad shape, pointer, alignment or value      */
    TS_ERR_UNSUPPORTED = 2,     /* valid but outside what the kernels support  */
    TS_ERR_WORKSPACE = 3,       /* workspace missing or smaller than required  */
    TS_ERR_CUDA = 4,            /* a CUDA runtime/driver call failed           */
    TS_ERR_DEVICE_TIMEOUT = 5   /* a bounded device-side wait gave up          */
} ts_status_t;

/*
 * One layer's KV cache for a (possibly ragged) batch, in token-major "NHD"
 * layout: element (token t, kv head g, channel c) of K is at
 *   k + t*stride_tok + g*stride_head + c        (in bf16 elements)
 * where t runs over the concatenated tokens of all sequences; sequence b owns
 * tokens [seq_offsets[b], seq_offsets[b+1]).  V has the same layout and
 * strides.  Query head h reads kv head h / (h_q / h_kv) (contiguous GQA
 * groups).
 *
 *   batch              >= 1 sequences
 *   h_q, h_kv          query / kv heads; h_q % h_kv == 0;
 *                      supported: h_kv in {1,2,4,8}, h_q/h_kv <= 16
 *   head_dim           64 or 128
 *   seq_offsets_dev    device int64 [batch+1], non-decreasing, [0] == 0
 *   seq_offsets_host   host copy of the same (used for sizing and checks;
 *                      must match seq_offsets_dev)
 *   k, v               device bf16, 16-byte aligned
 *   stride_tok,        in elements; multiples of 8; stride_head >= head_dim,
 *   stride_head        stride_tok >= (h_kv-1)*stride_head + head_dim
 *   scale              softmax scale; 0 selects 1/sqrt(head_dim)
 *   capacity           0, or (batch 1 only) the number of tokens the K and V
 *                      buffers hold, >= the current length: the cache can
 *                      then grow on the device (ts_append_kv).  Workspace
 *                      sizes, launch shapes and the tensor map follow the
 *                      capacity and every kernel takes the current length
 *                      from seq_offsets_dev, so one workspace and one
 *                      captured graph serve every length up to it.
 *   page_size          0 (the layout above), or the tokens per page of a
 *                      paged cache: then k and v are a pool of pool_pages
 *                      pages of page_size token rows each (row r of the pool
 *                      at k + r*stride_tok, same strides), and token i of
 *                      sequence b sits in pool row
 *                        page_table[b*page_table_stride + i/page_size]
 *                          * page_size + i % page_size.
 *                      seq_offsets still give the sequences' lengths and lay
 *                      out the votes; ids stay sequence-local.  Supported:
 *                      page_size a power of two in [8, 4096] (a scoring stage
 *                      of 128/h_kv tokens that spans several pages is loaded
 *                      one page and kv head at a time); capacity 0.
 *   page_table_dev     device int32 [batch * page_table_stride], the block
 *                      table; entries of pages a sequence uses must be in
 *                      [0, pool_pages): a page outside it reads as zero keys
 *                      in the scoring and is left out of the attention (no
 *                      access outside the pool; the results are not defined)
 *   page_table_stride  entries per sequence, >= the pages of the longest
 *   pool_pages         pages in the pool
 */
typedef struct ts_kv {
    int32_t batch, h_q, h_kv, head_dim;
    const int64_t *seq_offsets_dev;
    const int64_t *seq_offsets_host;
    const void *k;
    const void *v;
    int64_t stride_tok, stride_head;
    float scale;
    int64_t capacity;
    int32_t page_size, page_table_stride;
    int64_t pool_pages;
    const int32_t *page_table_dev;
} ts_kv_t;

/*
 * Workspace bytes needed by ts_score, ts_select and ts_sparse_attn for this
 * cache shape and a selection of k top tokens plus n_sink + n_local window
 * tokens (capacity k + n_sink + n_local).  The size depends on the current
 * device's SM count.  Returns 0 when the arguments are invalid.
 */
TS_API size_t ts_workspace_bytes(const ts_kv_t *kv, int32_t k, int32_t n_sink, int32_t n_local);

/*
 * Zero a workspace (the status word and the selection counters and
 * histogram).  Call once after allocating a workspace, before its first use,
 * on the stream that will use it.  The library returns every counter to zero
 * itself at the end of each call, so a workspace needs no re-initialisation
 * between calls (only after a call that reported an error).
 */
TS_API ts_status_t ts_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * Selection Cache decision (TokenSelect README, "Key Takeaways", Selection
 * Cache: consecutive similar queries share one token selection).
 * For each sequence b, over the flattened h_q*head_dim query vector:
 *   cos_b    = <q_b, q_prev_b> / (|q_b| |q_prev_b|)     (float64 accumulation)
 *              with cos_b = 0 when either vector is zero (no direction)
 *   reuse[b] = !first_step && cos_b >= threshold
 * then q_prev_b <- q_b.  (A zero query therefore reuses only when
 * threshold <= 0.)
 *   q          device bf16 [batch, h_q, head_dim] contiguous
 *   q_prev     device bf16, same shape; caller-owned state, overwritten
 *   reuse      device int32 [batch], written (0/1)
 *   cos_out    device float64 [batch] or NULL; receives cos_b (0 on the first step)
 */
TS_API ts_status_t ts_selcache(const void *q, void *q_prev, int32_t *reuse, double *cos_out,
                        int32_t first_step, int32_t batch, int32_t h_q, int32_t head_dim,
                        double threshold, void *stream);

/*
 * Soft vote (TokenSelect README, "Key Takeaways": per-head Q.K criticality,
 * per-head softmax over tokens, summed over heads).  For every sequence b with
 * reuse[b] == 0 and every token i in [0, n_b):
 *   s[h,i] = scale * q[b,h,:] . K[b,i,h/G,:]
 *   L[b,h] = log sum_i exp(s[h,i])
 *   votes[seq_offsets[b] + i] = sum_h exp(s[h,i] - L[b,h])
 * so the votes of a sequence sum to h_q.  Sequences with reuse[b] != 0 are
 * skipped (their votes are left as they were).
 *   q          device bf16 [batch, h_q, head_dim] contiguous, 16-byte aligned
 *   reuse      device int32 [batch] or NULL (NULL: score every sequence)
 *   votes      device float32 [seq_offsets[batch]] (a cache with a capacity:
 *              [capacity]), written
 * The float32 votes carry a relative error of a few 1e-7.
 */
TS_API ts_status_t ts_score(const ts_kv_t *kv, const void *q, const int32_t *reuse, float *votes,
                     void *ws, size_t ws_bytes, void *stream);

/*
 * The two phases of ts_score, callable separately (ts_score == ts_score_logits
 * followed by ts_score_vote on the same stream and workspace):
 *   ts_score_logits  per-head logits s[h,i] and log-normalisers L[b,h] into
 *                    the workspace (one streaming pass over K)
 *   ts_score_vote    votes from the workspace's logits and L
 * Arguments as for ts_score.  The workspace carries the intermediate results
 * from the first call to the second.
 */
TS_API ts_status_t ts_score_logits(const ts_kv_t *kv, const void *q, const int32_t *reuse,
                                   void *ws, size_t ws_bytes, void *stream);
TS_API ts_status_t ts_score_vote(const ts_kv_t *kv, const int32_t *reuse, float *votes,
                                 void *ws, size_t ws_bytes, void *stream);

/*
 * The soft vote of ts_score (same definition, arguments, workspace and
 * errors) from one cooperative kernel instead of two passes: the kv heads are
 * scored a few at a time (as many as keep one pass's logits within 32 MB of
 * L2), and each pass's normalisers and votes are taken while the next pass
 * streams K, with the logit lines dropped from L2 once read.  The votes equal
 * ts_score's up to rounding (a few 1e-7 relative: the normalisers are merged
 * in another order).  The kernel needs every CTA of its grid resident (one
 * per SM); it synchronises them with counters in the workspace's control
 * block, which it returns to zero.  ts_score and ts_decode_step use the
 * two-pass kernels, which are faster on B200 at every workload measured.
 */
TS_API ts_status_t ts_score_fused(const ts_kv_t *kv, const void *q, const int32_t *reuse, float *votes,
                                  void *ws, size_t ws_bytes, void *stream);

/*
 * Token selection (TokenSelect README summary: a small number of critical KV
 * tokens take part in attention).  For every sequence b with reuse[b] == 0:
 *   sink  = [0, s')         s' = min(n_sink, n_b)
 *   local = [l0, n_b)       l0 = max(n_b - n_local, s')
 *   T     = the min(k, l0 - s') tokens of [s', l0) with the largest votes,
 *           equal votes going to the lower token id
 *   ids[b, 0:count[b]] = sink U T U local in ascending order (sequence-local
 *   0-based ids), ids[b, count[b]:] = -1.
 * Sequences with reuse[b] != 0 keep their previous ids and count, unless
 * their length changed since those were written (a growing cache, see
 * ts_append_kv): then the previous top-k part, the ids of the old row inside
 * both the old and the new candidate ranges, is kept and the sink and local
 * windows are those of the new length.
 *   votes      device float32 [seq_offsets[batch]] (non-negative, finite)
 *   ids        device int32 [batch, k + n_sink + n_local]
 *   count      device int32 [batch]
 *   ws         workspace (ts_workspace_bytes), shared with ts_score
 * Sequences may hold at most 4194304 tokens.
 */
TS_API ts_status_t ts_select(const ts_kv_t *kv, const float *votes, int32_t k, int32_t n_sink,
                      int32_t n_local, const int32_t *reuse, int32_t *ids, int32_t *count,
                      void *ws, size_t ws_bytes, void *stream);

/*
 * Attention over the selected tokens:
 *   out[b,h,:] = sum_j softmax_j(scale * q[b,h,:] . K[b,ids_j,h/G,:]) * V[b,ids_j,h/G,:]
 * over j < count[b] (count[b] == 0 gives zeros).
 *   ids        device int32 [batch, ids_capacity], ids in [0, n_b)
 *   count      device int32 [batch], 0 <= count[b] <= ids_capacity
 *   out        device float32 [batch, h_q, head_dim], 16-byte aligned, written
 * ids_capacity (= k + n_sink + n_local) is at most 16384.  Ids outside
 * [0, n_b) are skipped.
 */
TS_API ts_status_t ts_sparse_attn(const ts_kv_t *kv, const void *q, const int32_t *ids,
                           const int32_t *count, int32_t ids_capacity, float *out,
                           void *ws, size_t ws_bytes, void *stream);

/*
 * ts_sparse_attn for callers that cannot allocate device memory.  The paper
 * has no counterpart: this is a deployment variant of the same attention.
 * Some hosts own every byte of device memory through their own pool and let
 * no library call cudaMalloc or take a workspace after start-up, or run under
 * a memory budget fixed when the process initialises.  This call therefore
 * takes no workspace and allocates nothing: its scratch (the split-K
 * partials) is a 4 MiB array built into the library, which every GPU that
 * loads the library holds until the process exits.
 *   - Arguments, results and errors as for ts_sparse_attn.  Shapes whose
 *     scratch would exceed 4 MiB (B * h_kv * splits * (h_q/h_kv) * (d+4) * 4
 *     bytes, splits = ceil(ids_capacity / 64)) are rejected with
 *     TS_ERR_UNSUPPORTED before anything is launched.
 *   - The first call on each device looks the array up (cudaGetSymbolAddress
 *     with that device current).  Under CUDA's lazy module loading (the
 *     default) the 4 MiB are committed on a device only when the library's
 *     code first loads there, at that first call or at the first call of any
 *     other entry point.  A caller whose memory budget is fixed at start-up
 *     should therefore make one call per device at start-up, before it takes
 *     its budget and before any stream capture.  A device reset ends the
 *     context the address belongs to; the next call looks it up again.
 *   - Every call shares the one array, which keeps the last call's
 *     contents: calls that can overlap on the GPU (on different streams, or
 *     from different threads) race with each other.  Nothing in it has to
 *     start at zero: a call writes every partial it reads before reading it.
 */
TS_API ts_status_t ts_sparse_attn_noalloc(const ts_kv_t *kv, const void *q, const int32_t *ids,
                                          const int32_t *count, int32_t ids_capacity, float *out,
                                          void *stream);

/*
 * One whole decode step of one layer: ts_selcache, ts_score, ts_select and
 * ts_sparse_attn in that order on `stream`, with the same arguments and the
 * same results as the four calls (selection capacity k + n_sink + n_local, the
 * ids row length; bit for bit).  Fewer kernels run: the vote pass also builds
 * the selection's first-level vote histogram, which ts_select otherwise builds
 * in a kernel of its own (ts_decode_step_kernels gives the count).  Every
 * argument is checked before the first launch.
 *   With TS_REUSE_SKIP=1 in the environment, a call under stream capture
 *   with the selection cache able to reuse (first_step 0, threshold <= 1)
 *   captures the scoring and selection kernels into the body of a
 *   conditional graph node that the cosine kernel switches off when every
 *   sequence reuses: such a replayed step runs 3 kernels (the cosine test
 *   and the two attention kernels) instead of 9.  The results are the same
 *   either way.  The body is captured on a stream the library creates once
 *   per context.  Off by default: the node's edges cannot use programmatic
 *   launch, which on B200 costs more than the skipped kernels save.
 *   reuse      device int32 [batch], required: written by the selection cache
 *              and read by every later phase (sequences that reuse keep their
 *              previous ids and count; their votes are left as they were)
 *   q          16-byte aligned; out 16-byte aligned; ws as ts_workspace_bytes
 */
TS_API ts_status_t ts_decode_step(const ts_kv_t *kv, const void *q, void *q_prev, int32_t *reuse,
                                  double *cos_out, int32_t first_step, double threshold, int32_t k,
                                  int32_t n_sink, int32_t n_local, float *votes, int32_t *ids,
                                  int32_t *count, float *out, void *ws, size_t ws_bytes, void *stream);

/*
 * Append one token to a growing cache (capacity mode, batch 1), entirely on
 * the device: the token's K and V rows go to position n = seq_offsets_dev[1]
 * and seq_offsets_dev[1] becomes n + 1, so a captured graph can append step
 * after step.  With the selection cache on, a later step that reuses its
 * selection keeps the previous top-k part and takes the sink and local
 * windows of the new length (TokenSelect README, "Key Takeaways", Selection
 * Cache).
 *   kv            the cache, capacity > 0
 *   seq_offsets   kv->seq_offsets_dev, writable
 *   k_cache, v_cache   kv->k and kv->v, writable
 *   k_new, v_new  device bf16 [h_kv][head_dim] each, contiguous, 16-byte aligned
 *   ws            a workspace of this cache: appending to a full cache
 *                 writes nothing and records the error in its status word
 *                 (ts_get_device_status then returns TS_ERR_INVALID_ARG)
 * The host copy kv->seq_offsets_host is not read here and not updated.
 */
TS_API ts_status_t ts_append_kv(const ts_kv_t *kv, int64_t *seq_offsets, void *k_cache, void *v_cache,
                                const void *k_new, const void *v_new, void *ws, size_t ws_bytes, void *stream);

/*
 * Number of kernels one ts_decode_step call on this cache launches (for
 * launch accounting and profiling), or -1 with ts_last_error set when the
 * cache description or the selection sizes are invalid.  Host only; touches
 * no device memory.
 */
TS_API int32_t ts_decode_step_kernels(const ts_kv_t *kv, int32_t k, int32_t n_sink, int32_t n_local);

/*
 * Read and clear the device status word of a workspace (synchronises the
 * stream).  Returns TS_ERR_DEVICE_TIMEOUT when a kernel's bounded wait gave
 * up since the last read, TS_ERR_INVALID_ARG when ts_append_kv found the
 * cache full, TS_OK otherwise.  *site_out (may be NULL) receives a code
 * naming the wait or the call.  After TS_ERR_DEVICE_TIMEOUT the results of
 * every call since the last TS_OK read are void, and so are the workspace's
 * contents: re-initialise it (ts_workspace_init) before reuse.
 */
TS_API ts_status_t ts_get_device_status(void *ws, size_t ws_bytes, uint32_t *site_out, void *stream);

/*
 * Self-test of the bounded-wait path: launches one block that waits on a
 * shared-memory barrier nobody arrives at, giving up after spin_limit polls;
 * the give-up is recorded in the workspace status word (read it with
 * ts_get_device_status).  Nothing else is touched.
 */
TS_API ts_status_t ts_selftest_expire_wait(void *ws, size_t ws_bytes, uint32_t spin_limit, void *stream);

/*
 * ---------------------------------------------------------------------------
 * Token-axis split of one sequence across ranks.  Each rank holds a
 * contiguous shard [t, t + n_loc) of one sequence's tokens as a batch-1
 * cache of its own (kv, without capacity) and runs the step's phases on it;
 * three small exchanges, which the caller performs (e.g. NCCL all-gathers
 * over NVLink), join them into exactly the single-sequence step:
 *   1. ts_score_normalisers -> all-gather L -> ts_merge_normalisers ->
 *      ts_score_vote_normalised: the votes of the shard's tokens under the
 *      whole sequence's per-head softmax (TokenSelect README, "Key
 *      Takeaways": the per-head softmax is over every cached token);
 *   2. ts_select_candidates -> all-gather keys -> ts_select_merge: the whole
 *      sequence's top-k (ties to the lower token id) with its sink and local
 *      windows, as this shard's rows;
 *   3. ts_sparse_attn_lse -> all-gather out and lse -> ts_merge_attention:
 *      the attention over every selected token.
 * Token ids in the shard's rows are shard-local (id + t is the sequence
 * id); the keys carry sequence ids.
 * ---------------------------------------------------------------------------
 */

/* Score pass A and the normaliser merge on the shard (ts_score_logits), the
 * merge writing L_out[b][h] = log sum_i exp(s[h][i]) over the shard's tokens
 * (float64, device [batch][h_q]): every entry -inf when the shard holds no
 * token; in a batch of several sequences, the rows of a sequence that
 * reuses (reuse[b] != 0) or is empty are left as they were.  The
 * workspace's own normalisers are not written. */
TS_API ts_status_t ts_score_normalisers(const ts_kv_t *kv, const void *q, const int32_t *reuse, double *L_out,
                                        void *ws, size_t ws_bytes, void *stream);

/* Score pass B with given normalisers: votes[i] = sum_h exp(s[h][i] - L_in[b][h])
 * for the logits of the last ts_score_normalisers / ts_score_logits call on
 * this workspace (L_in: device float64 [batch][h_q], read in place by the
 * kernel). */
TS_API ts_status_t ts_score_vote_normalised(const ts_kv_t *kv, const int32_t *reuse, const double *L_in,
                                            float *votes, void *ws, size_t ws_bytes, void *stream);

/* L_out[i] = log sum_r exp(L_parts[r][i]) for i < count, r < parts (float64,
 * device; -inf parts contribute nothing). */
TS_API ts_status_t ts_merge_normalisers(const double *L_parts, int32_t parts, int64_t count, double *L_out,
                                        void *stream);

/*
 * The shard's best min(k, its candidates) candidates of the sequence's top-k
 * (candidates [s', l0) of the whole sequence as in ts_select, n_global its
 * length, shard_offset = t) as keys: keys_out[j] = (vote bits << 32) |
 * (2^32 - 1 - sequence id), ascending by id, 0 after them (device uint64
 * [k]).  ids and count (device, k + n_sink + n_local entries) are scratch
 * here: they hold the shard's own selection.  A larger key is a larger vote,
 * or the lower id of two equal votes.
 */
TS_API ts_status_t ts_select_candidates(const ts_kv_t *kv, const float *votes, int32_t k, int32_t n_sink,
                                        int32_t n_local, int64_t shard_offset, int64_t n_global, int32_t *ids,
                                        int32_t *count, uint64_t *keys_out, void *ws, size_t ws_bytes,
                                        void *stream);

/*
 * The sequence's selection, this shard's part: T = the k-th largest key of
 * keys_all (device uint64 [parts][k], every shard's ts_select_candidates
 * output, this one's at `rank`), or every key when there are at most k;
 *   ids = [0, s_loc) U (this shard's keys >= T, as shard-local ids) U
 *         [n_loc - l_loc, n_loc), ascending, -1 after count,
 * s_loc and l_loc the shard's parts of the sequence's sink and local
 * windows.  ids: device int32 [k + n_sink + n_local]; count: int32 [1].
 */
TS_API ts_status_t ts_select_merge(const ts_kv_t *kv, const uint64_t *keys_all, int32_t parts, int32_t rank,
                                   int32_t k, int32_t n_sink, int32_t n_local, int64_t shard_offset,
                                   int64_t n_global, int32_t *ids, int32_t *count, void *stream);

/* ts_sparse_attn, also writing lse_out[b][h] = log sum_j exp(scale * q_h . K[ids[j]])
 * over the selected tokens (device float32 [batch][h_q]; -inf when none). */
TS_API ts_status_t ts_sparse_attn_lse(const ts_kv_t *kv, const void *q, const int32_t *ids, const int32_t *count,
                                      int32_t ids_capacity, float *out, float *lse_out, void *ws,
                                      size_t ws_bytes, void *stream);

/* out[i][c] = sum_r w_r out_parts[r][i][c], w_r = exp(lse_parts[r][i] - LSE_i),
 * LSE_i = log sum_r exp(lse_parts[r][i]) (rows i < rows, c < head_dim; 0
 * where every part is -inf).  Device float32 throughout. */
TS_API ts_status_t ts_merge_attention(const float *out_parts, const float *lse_parts, int32_t parts, int64_t rows,
                                      int32_t head_dim, float *out, void *stream);

/*
 * ---------------------------------------------------------------------------
 * Page-level comparator after Quest (Bohrium page for "Quest: Query-Aware
 * Sparsity for Efficient Long-Context LLM Inference", arXiv 2406.10774:
 * Abstract; Method Overview, item 4).  Each page of P consecutive tokens of a
 * sequence keeps the element-wise minimum and maximum of its keys; a query
 * bounds every key of the page from above with them; the Top-K pages by that
 * bound are attended.  The selection has the same form as ts_select's (one
 * ascending id row per sequence with the sink and local windows), so
 * ts_sparse_attn attends over it unchanged.
 *
 * Pages: page j of sequence b holds its tokens [j*P, min((j+1)*P, n_b)), the
 * last one possibly short; P is a power of two in [1, 4096].  The metadata
 * and the scores have ts_quest_rows() rows; page j of sequence b is row
 * (seq_offsets[b] / P) + b + j (at most one unused row per sequence; rows
 * not holding a page are never written or read).  A cache with a capacity
 * is laid out for the capacity; a paged KV cache (page_size != 0) is read
 * through its block table, its page size independent of P.
 * ---------------------------------------------------------------------------
 */

/* Rows of the page metadata and scores of this cache for page size P,
 * floor(n_total / P) + batch rounded up to a multiple of 4 (n_total: the
 * capacity of a growing cache), or -1 with ts_last_error set when kv or P
 * is invalid.  Host only. */
TS_API int64_t ts_quest_rows(const ts_kv_t *kv, int32_t page_size);

/*
 * Page metadata [Quest, Abstract: the minimal and maximal key values of each
 * page]: kmin[row][g][c] and kmax[row][g][c] = the minimum and maximum over
 * the page's tokens of K[token][g][c].
 *   kmin, kmax   device bf16 [ts_quest_rows][h_kv][head_dim] each, 16-byte
 *                aligned (caller-owned); only the rows of pages are written
 * Reads K once.
 */
TS_API ts_status_t ts_quest_metadata(const ts_kv_t *kv, int32_t page_size, void *kmin, void *kmax, void *stream);

/*
 * Page metadata of the newest tokens only: the rows of every page that holds
 * one of a sequence's last last_tokens tokens are recomputed from all the
 * page's tokens, as ts_quest_metadata computes them; every other row is left
 * as it is.  The current lengths are read from seq_offsets_dev on the
 * device, so after ts_append_kv (one token: last_tokens = 1) the call
 * updates the page that took the token, also inside a captured graph.
 *   last_tokens  >= 1 (a value above a sequence's length covers all of it)
 *   kmin, kmax   as for ts_quest_metadata, holding the other pages' rows
 * Reads at most (floor(last_tokens / P) + 2) * P tokens of K per sequence.
 */
TS_API ts_status_t ts_quest_metadata_update(const ts_kv_t *kv, int32_t page_size, int64_t last_tokens, void *kmin,
                                            void *kmax, void *stream);

/*
 * Page scores [Quest, Method Overview (4)]: with scale as in ts_score and
 * kv head g(h) = h / (h_q / h_kv),
 *   score[row of page j] = sum_h scale * sum_c max(q[h][c] * kmin[j][g(h)][c],
 *                                                  q[h][c] * kmax[j][g(h)][c]),
 * the per-head upper bound of the scaled logit over the page's min/max box,
 * summed over the query heads (one selection serves all heads).  fp32,
 * computed as one dot product per page of [kmax | kmin] with the query's
 * head-summed positive and negative parts.
 *   q            device bf16 [batch][h_q][head_dim], contiguous, 16-byte aligned
 *   kmin, kmax   from ts_quest_metadata
 *   scores       device fp32 [ts_quest_rows] (caller-owned), 16-byte aligned;
 *                only the rows of pages are written
 */
TS_API ts_status_t ts_quest_score(const ts_kv_t *kv, const void *q, int32_t page_size, const void *kmin,
                                  const void *kmax, float *scores, void *stream);

/*
 * Page selection with the token windows of ts_select: sink [0, s'),
 * s' = min(n_sink, n); local [l0, n), l0 = max(n - n_local, s'); a page is a
 * candidate when it holds a token of [s', l0).  The Top-K pages are the first
 * min(floor(k / P), candidates) candidate pages by (score descending, page
 * ascending) [Quest, Abstract: only the Top-K critical pages are loaded];
 *   ids[b] = ascending [0, s') U (tokens of the chosen pages in [s', l0)) U [l0, n),
 * count[b] = their number (at most s' + k + (n - l0)); ids[b][count..) = -1.
 *   scores      from ts_quest_score (all ts_quest_rows entries readable)
 *   ids         device int32 [batch][k + n_sink + n_local]; count int32 [batch]
 * One cluster of 8 CTAs per sequence (the pages split among them); no
 * workspace.  The usual case (at most 2048 chosen pages, at most 2048 pages
 * tied in the threshold's bin) reads the scores three times; heavy ties or
 * larger budgets take a general path on one CTA that reads them five times.
 */
TS_API ts_status_t ts_quest_select(const ts_kv_t *kv, const float *scores, int32_t page_size, int32_t k,
                                   int32_t n_sink, int32_t n_local, int32_t *ids, int32_t *count, void *stream);

TS_API const char *ts_status_string(ts_status_t status);

/* Human-readable description of the calling thread's last error ("" if none). */
TS_API const char *ts_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TS_H_ */
