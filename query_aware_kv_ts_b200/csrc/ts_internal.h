// Host-side internals of libts: workspace layout, per-launch plans and the
// launchers each kernel file provides to api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/ts.h"

namespace ts {

constexpr int kMaxBatch = 1024;        // sequences per call (shared-memory tables)
constexpr int kScoreRows = 128;                 // K rows per stage (h_kv heads x T tokens): the MMA's M
constexpr int kScoreEpiWarps = 8;               // two per TMEM lane quarter (each half of the heads)
constexpr int kScoreThreads = (kScoreEpiWarps + 2) * 32;   // + TMA producer warp + MMA warp
constexpr int kScoreMaxStages = 12;
constexpr int kScoreAccBufs = 4;                // TMEM accumulators in flight
constexpr size_t kScoreDynSmemBudget = 212 * 1024;   // + the kernel's ~13 KB of static shared memory
constexpr size_t kFusedDynSmemBudget = 224 * 1024;   // + the fused kernel's ~2 KB of static shared memory
constexpr int kVoteThreads = 256;
constexpr int kSelectThreads = 256;
constexpr int kSelectTokensPerCta = 2048;     // candidates per selection range
constexpr int kMaxSelectRanges = 2048;        // ranges per sequence: n <= 4M candidates
constexpr int kAttnThreads = 256;
constexpr int kAttnRows = 64;         // selected rows per attention CTA (one split)
constexpr int kMaxCapacity = 16384;   // k + sink + local
constexpr int kFusedRows = 128;       // K rows per stage of the fused scoring kernel (HS heads x T tokens)
constexpr size_t kFusedPassLogitsBytes = size_t(32) << 20;   // logits one fused-scoring pass may keep in L2

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch with programmatic stream serialization (the kernel's prologue may
// overlap the previous kernel in the stream; see pdl_wait) and, when
// cluster > 1, a thread-block cluster of that many CTAs along x.
// Programmatic dependent launch is on unless the environment sets TS_NO_PDL=1.
bool pdl_enabled();

template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster,
                      Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = (unsigned)cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Cooperative launch (every CTA of the grid resident at once, as a kernel
// with grid-wide barriers needs), with programmatic stream serialization
// unless TS_NO_PDL=1.
template <typename... KArgs, typename... Args>
cudaError_t launch_coop(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    attr[n].id = cudaLaunchAttributeCooperative;
    attr[n].val.cooperative = 1;
    ++n;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)n;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Control-block words (the first 256 bytes of every workspace, zeroed by
// ts_workspace_init): [0] status, [1] site; [8, 9] the reuse-skip counters of
// the cosine kernel; [16, 16 + passes) the fused scoring kernel's per-pass
// arrival counters, [24] its finished-CTA count.
constexpr int kCtrlFusedBarrier = 16;

// Everything derived from the cache shape that the kernels and the workspace
// layout need.  Built identically by every entry point.
struct Plan {
    int B, Hq, Hkv, G, D;
    int64_t n_total;         // seq_offsets[B]
    int64_t n_max;           // longest sequence
    bool paged;              // k, v are a pool of pages (block table in kv->page_table_dev)
    int page_shift;          // log2(page_size) when paged
    int64_t kv_rows;         // token rows of k and v: n_total, the capacity, or the pool's rows
    float scale;
    int sms;
    // score pass A
    int tile_tokens;         // T: tokens per pipeline stage
    int box_tokens;          // tokens of one TMA box of K: T, or a shorter page of a paged cache
    int box_heads;           // kv heads of one TMA box of K: h_kv, or 1 for 8-token pages shorter than T
    int stage_bytes;
    int64_t max_chunks;      // sum_b ceil(n_b / T)
    int score_grid;          // <= 256
    int score_partials_per_slot;   // R: epilogue warps of pass A that see one kv head
    int64_t ld_logits;       // logits row stride: n_total rounded up to 4
    // fused scoring (HS kv heads of T = 128 / HS tokens per stage)
    int fused_hs;            // kv heads per pass (4, 2 or 1; divides h_kv)
    int fused_t;             // tokens per chunk
    int fused_gp;            // staged query rows per kv head (4, 8 or 16)
    int fused_n;             // MMA N: max(16, HS * GP)
    int64_t fused_chunks;    // sum_b ceil(n_b / T)
    int fused_grid;          // min(SMs, fused_chunks)
    int64_t fused_ld;        // its logits row stride: fused_chunks * T
    // selection
    int sel_ranges;          // ranges of kSelectTokensPerCta candidates per sequence (grid x)
    // attention
    int capacity;            // ids row length (k + sink + local)
    int attn_splits;
    // workspace layout (byte offsets)
    size_t off_ctrl, off_chunk_table, off_L, off_partials, off_logits, off_sel_hist, off_sel_cand,
        off_sel_inb1, off_sel_bin, off_sel_above, off_sel_range_off, off_sel_thr, off_sel_mode, off_sel_prev_n,
        off_vacc, off_attn_part,
        total_bytes;
};

// Fill `p` from the cache description (capacity < 0: attention part not
// needed).  Returns TS_OK or an error with ts_last_error set.
ts_status_t make_plan(const ts_kv_t *kv, int capacity, Plan *p);

void set_error(const char *fmt, ...);

// The calling thread's current CUDA context (a driver handle), or nullptr when
// none is current or the driver entry point is unavailable.  Per-device state
// the library caches (kernel attributes, symbol addresses) is keyed by it, so
// that a device reset, which ends the context, makes the cache look again.
void *current_context();

// Raise `kernel`'s dynamic shared-memory limit to `bytes` on the current
// context, once per (kernel, context); thread-safe.
cudaError_t ensure_dyn_smem(const void *kernel, int bytes);

// Launchers (return cudaGetLastError() of the launch).
// One token appended at seq_offsets[1] (batch 1); ctrl[0] = 2 when full.
cudaError_t launch_append(int64_t *seq_offsets, void *k_cache, void *v_cache, const void *k_new, const void *v_new,
                          int64_t stride_tok, int64_t stride_head, int Hkv, int D, int64_t capacity, uint32_t *ctrl,
                          cudaStream_t st);

// In a graph replay the cosine kernel can switch off the conditional node
// that holds the scoring and selection kernels: the last of its blocks sets
// the node's condition to 0 when every sequence reuses its selection.
// counters: two words of the workspace control block (zero between steps).
constexpr int kCtrlSkipCounters = 8;   // control-block words 8, 9
struct SelcacheSkip {
    cudaGraphConditionalHandle handle = 0;
    uint32_t *counters = nullptr;
    int enabled = 0;
};
cudaError_t launch_selcache(const void *q, void *q_prev, int32_t *reuse, double *cos_out, int first_step,
                            int B, int len, double theta, cudaStream_t st, const SelcacheSkip *skip = nullptr);

// seq_off_host: the host copy of the offsets (prefetch hints before the
// dependency wait; the device copy decides the work).
// page_table, page_table_stride: the block table of a paged cache (p.paged).
// L_out: where the normaliser merge writes L (null: the workspace).
cudaError_t launch_score(const Plan &p, const CUtensorMap &kmap, const void *q, const int64_t *seq_off,
                         const int64_t *seq_off_host, const int32_t *reuse, uint8_t *ws, cudaStream_t st,
                         const int32_t *page_table = nullptr, int page_table_stride = 0, double *L_out = nullptr);

// Selection parameters, for the vote pass that also builds the selection's
// level-1 histogram.
struct SelectWindow {
    int k, n_sink, n_local;
};

// L_in: the normalisers to use instead of the workspace's (null: the workspace's)
cudaError_t launch_vote(const Plan &p, const int64_t *seq_off, const int32_t *reuse, float *votes, uint8_t *ws,
                        cudaStream_t st, const SelectWindow *hist_window = nullptr, const double *L_in = nullptr);

// Logits, normalisers and votes in one cooperative kernel, one kv-head group
// at a time (kmap_head: boxes of {64 channels, 128 tokens, 1 head}); with a
// window it also builds the selection's level-1 histogram.
cudaError_t launch_score_fused(const Plan &p, const CUtensorMap &kmap_head, const void *q, const int64_t *seq_off,
                               const int64_t *seq_off_host, const int32_t *reuse, float *votes, uint8_t *ws,
                               cudaStream_t st, const SelectWindow *hist_window = nullptr);

// hist_ready: the level-1 histogram was already built by the vote pass.
cudaError_t launch_select(const Plan &p, const int64_t *seq_off, const float *votes, int k, int n_sink,
                          int n_local, const int32_t *reuse, int32_t *ids, int32_t *count, uint8_t *ws,
                          cudaStream_t st, bool hist_ready = false);

// lse (or null): [B][Hq] natural log-sum-exp of each head's scaled logits
// over the selected tokens (-inf when none), for joining shards.
cudaError_t launch_attn(const Plan &p, const ts_kv_t *kv, const void *q, const int32_t *ids,
                        const int32_t *count, float *out, uint8_t *ws, cudaStream_t st, float *lse = nullptr);

// Attention with its scratch in a fixed device array instead of a workspace
// (sets the error message itself).
ts_status_t launch_attn_noalloc(const Plan &p, const ts_kv_t *kv, const void *q, const int32_t *ids,
                                const int32_t *count, float *out, cudaStream_t st);

cudaError_t launch_selftest_wait(uint32_t *ctrl, uint32_t spin_limit, cudaStream_t st);

// Token-axis split of one sequence (split.cu): the joins' arithmetic.
cudaError_t launch_merge_normalisers(const double *L_parts, int parts, int64_t count, double *L_out,
                                     cudaStream_t st);
cudaError_t launch_candidate_keys(const float *votes, const int32_t *ids, const int32_t *count, int s_loc, int l_loc,
                                  int64_t shard_offset, int kcap, unsigned long long *keys, cudaStream_t st);
cudaError_t launch_select_merge(const unsigned long long *keys, int parts, int kcap, int k, int rank, int s_loc,
                                int l_loc, int64_t n_loc, int64_t shard_offset, int cap, int32_t *ids,
                                int32_t *count, cudaStream_t st);
cudaError_t launch_merge_attention(const float *o_parts, const float *lse_parts, int parts, int64_t rows, int d,
                                   float *out, cudaStream_t st);

// Page-level comparator (quest.cu): rows of the page metadata and scores,
// page j of sequence b at row (seq_offsets[b] >> log2 P) + b + j.
int64_t quest_rows(const Plan &p, int page_size);
// last_tokens > 0: only the pages holding the sequences' last last_tokens tokens
cudaError_t launch_quest_meta(const Plan &p, const ts_kv_t *kv, int page_size, void *kmin, void *kmax,
                              cudaStream_t st, int64_t last_tokens = 0);
cudaError_t launch_quest_score(const Plan &p, const ts_kv_t *kv, const void *q, int page_size, const void *kmin,
                               const void *kmax, float *scores, cudaStream_t st);
cudaError_t launch_quest_select(const Plan &p, const ts_kv_t *kv, const float *scores, int page_size, int k,
                                int n_sink, int n_local, int32_t *ids, int32_t *count, cudaStream_t st);

}  // namespace ts
