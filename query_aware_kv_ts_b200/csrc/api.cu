// libts C ABI: argument validation, workspace layout, TMA descriptor set-up
// and kernel launches.  No CPU fallback: every result comes from a kernel.
#include <cudaTypedefs.h>

#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {

namespace {
thread_local std::string g_last_error;

int device_sms()
{
    static std::mutex mu;
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        cached[dev] = sms;
    }
    return cached[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

ts_status_t cuda_fail(cudaError_t e, const char *what)
{
    set_error("%s: %s", what, cudaGetErrorString(e));
    return TS_ERR_CUDA;
}
}  // namespace

void *current_context()
{
    using GetCurrent = CUresult (*)(CUcontext *);
    static std::once_flag once;
    static GetCurrent fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<GetCurrent>(p);
    });
    CUcontext ctx = nullptr;
    if (fn == nullptr || fn(&ctx) != CUDA_SUCCESS)
        return nullptr;
    return ctx;
}

cudaError_t ensure_dyn_smem(const void *kernel, int bytes)
{
    struct Done {
        const void *kernel;
        void *ctx;
        int bytes;
    };
    static std::mutex mu;
    static std::vector<Done> done;
    // (no context yet: the attribute is set on every call)
    void *ctx = current_context();
    std::lock_guard<std::mutex> lock(mu);
    for (const Done &d : done)
        if (d.kernel == kernel && d.ctx == ctx && ctx != nullptr && d.bytes >= bytes)
            return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess)
        return e;
    if (ctx != nullptr) {
        for (Done &d : done)
            if (d.kernel == kernel && d.ctx == ctx) {
                d.bytes = bytes;
                return cudaSuccess;
            }
        done.push_back({kernel, ctx, bytes});
    }
    return cudaSuccess;
}

// Captured into a graph, ts_decode_step can put its scoring and selection
// kernels in a conditional node that the cosine kernel switches off when
// every sequence reuses its selection.  Off unless the environment sets
// TS_REUSE_SKIP=1 (read at every call): measured on B200, the two edges a
// conditional node forces to full serialisation (no programmatic launch
// into or out of it) cost more than the early-exiting kernels it skips.
static bool reuse_skip_enabled()
{
    const char *e = getenv("TS_REUSE_SKIP");
    return e != nullptr && e[0] == '1';
}

// A non-blocking stream of the current context on which the body of a
// conditional graph node is captured (the caller's stream is capturing the
// enclosing graph).  Created at the first use in a context, kept for the
// process's lifetime.
static cudaError_t body_stream(cudaStream_t *out)
{
    static std::mutex mu;
    static std::vector<std::pair<void *, cudaStream_t>> streams;
    void *ctx = current_context();
    std::lock_guard<std::mutex> lock(mu);
    for (const auto &e : streams)
        if (e.first == ctx && ctx != nullptr) {
            *out = e.second;
            return cudaSuccess;
        }
    cudaStream_t st = nullptr;
    const cudaError_t e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
    if (e != cudaSuccess)
        return e;
    streams.push_back({ctx, st});
    *out = st;
    return cudaSuccess;
}

bool pdl_enabled()
{
    static const bool on = [] {
        const char *e = getenv("TS_NO_PDL");
        return !(e != nullptr && e[0] == '1');
    }();
    return on;
}

void set_error(const char *fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
}

ts_status_t make_plan(const ts_kv_t *kv, int capacity, Plan *p)
{
    if (kv == nullptr) {
        set_error("kv is NULL");
        return TS_ERR_INVALID_ARG;
    }
    if (kv->batch < 1 || kv->h_q < 1 || kv->h_kv < 1) {
        set_error("batch, h_q and h_kv must be >= 1 (got %d, %d, %d)", kv->batch, kv->h_q, kv->h_kv);
        return TS_ERR_INVALID_ARG;
    }
    if (kv->h_q % kv->h_kv != 0) {
        set_error("h_q (%d) must be a multiple of h_kv (%d)", kv->h_q, kv->h_kv);
        return TS_ERR_INVALID_ARG;
    }
    if (kv->head_dim != 64 && kv->head_dim != 128) {
        set_error("head_dim must be 64 or 128 (got %d)", kv->head_dim);
        return TS_ERR_UNSUPPORTED;
    }
    const int G = kv->h_q / kv->h_kv;
    if (!(kv->h_kv == 1 || kv->h_kv == 2 || kv->h_kv == 4 || kv->h_kv == 8) || G > 16) {
        set_error("supported: h_kv in {1,2,4,8} and h_q/h_kv <= 16 (got h_kv %d, group %d)", kv->h_kv, G);
        return TS_ERR_UNSUPPORTED;
    }
    if (kv->batch > kMaxBatch) {
        set_error("batch %d exceeds the supported maximum %d", kv->batch, kMaxBatch);
        return TS_ERR_UNSUPPORTED;
    }
    if (kv->seq_offsets_dev == nullptr || kv->seq_offsets_host == nullptr) {
        set_error("seq_offsets_dev and seq_offsets_host are required");
        return TS_ERR_INVALID_ARG;
    }
    if (kv->k == nullptr || kv->v == nullptr) {
        set_error("k and v are required");
        return TS_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(kv->k) | reinterpret_cast<uintptr_t>(kv->v)) & 15u) {
        set_error("k and v must be 16-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    const int D = kv->head_dim;
    if (kv->stride_tok % 8 != 0 || kv->stride_head % 8 != 0 || kv->stride_head < D ||
        kv->stride_tok < (int64_t)(kv->h_kv - 1) * kv->stride_head + D) {
        set_error("strides (tok %lld, head %lld) must be multiples of 8 with stride_head >= head_dim and "
                  "stride_tok >= (h_kv-1)*stride_head + head_dim",
                  (long long)kv->stride_tok, (long long)kv->stride_head);
        return TS_ERR_INVALID_ARG;
    }
    if (!isfinite(kv->scale)) {
        set_error("scale must be finite");
        return TS_ERR_INVALID_ARG;
    }
    const int64_t *off = kv->seq_offsets_host;
    if (off[0] != 0) {
        set_error("seq_offsets[0] must be 0");
        return TS_ERR_INVALID_ARG;
    }
    int64_t n_max = 0;
    for (int b = 0; b < kv->batch; ++b) {
        const int64_t n = off[b + 1] - off[b];
        if (n < 0) {
            set_error("seq_offsets must be non-decreasing (sequence %d)", b);
            return TS_ERR_INVALID_ARG;
        }
        n_max = n > n_max ? n : n_max;
    }
    int64_t n_total = off[kv->batch];
    if (kv->capacity < 0) {
        set_error("capacity must be >= 0");
        return TS_ERR_INVALID_ARG;
    }
    if (kv->capacity > 0) {
        // a growing cache: sizes for its largest length, work from the device offsets
        if (kv->batch != 1) {
            set_error("a cache with a capacity must hold one sequence (batch %d)", kv->batch);
            return TS_ERR_UNSUPPORTED;
        }
        if (kv->capacity < n_total) {
            set_error("capacity %lld is below the current length %lld", (long long)kv->capacity,
                      (long long)n_total);
            return TS_ERR_INVALID_ARG;
        }
        n_total = n_max = kv->capacity;
    }
    if (n_total >= (int64_t(1) << 31)) {
        set_error("total tokens %lld must be below 2^31", (long long)n_total);
        return TS_ERR_UNSUPPORTED;
    }
    // a paged cache: k and v are a pool of pages, a block table maps pages
    p->paged = kv->page_size != 0;
    p->kv_rows = n_total;
    if (p->paged) {
        const int64_t ps = kv->page_size;
        if (ps < 8 || (ps & (ps - 1)) != 0 || ps > 4096) {
            set_error("page_size %lld must be a power of two in [8, 4096]", (long long)ps);
            return TS_ERR_UNSUPPORTED;
        }
        if (kv->capacity != 0) {
            set_error("a paged cache cannot also have a capacity");
            return TS_ERR_UNSUPPORTED;
        }
        if (kv->page_table_dev == nullptr || kv->pool_pages < 1 || kv->page_table_stride < 1) {
            set_error("a paged cache needs page_table_dev, pool_pages >= 1 and page_table_stride >= 1");
            return TS_ERR_INVALID_ARG;
        }
        if ((n_max + ps - 1) / ps > kv->page_table_stride) {
            set_error("page_table_stride %d is below the %lld pages of the longest sequence", kv->page_table_stride,
                      (long long)((n_max + ps - 1) / ps));
            return TS_ERR_INVALID_ARG;
        }
        if (kv->pool_pages * ps >= (int64_t(1) << 31)) {
            set_error("the pool's %lld rows must be below 2^31", (long long)(kv->pool_pages * ps));
            return TS_ERR_UNSUPPORTED;
        }
        p->kv_rows = kv->pool_pages * ps;
        int shift = 0;
        while ((int64_t(1) << shift) < ps)
            ++shift;
        p->page_shift = shift;
    } else {
        p->page_shift = 0;
    }
    if (n_max > (int64_t)kMaxSelectRanges * kSelectTokensPerCta) {
        set_error("sequence length %lld exceeds the supported maximum %lld", (long long)n_max,
                  (long long)kMaxSelectRanges * kSelectTokensPerCta);
        return TS_ERR_UNSUPPORTED;
    }
    const int sms = device_sms();
    if (sms <= 0) {
        set_error("no CUDA device");
        return TS_ERR_CUDA;
    }

    p->B = kv->batch;
    p->Hq = kv->h_q;
    p->Hkv = kv->h_kv;
    p->G = G;
    p->D = D;
    p->n_total = n_total;
    p->n_max = n_max;
    p->scale = kv->scale != 0.0f ? kv->scale : (float)(1.0 / sqrt((double)D));
    p->sms = sms;
    p->tile_tokens = kScoreRows / kv->h_kv;          // one stage = 128 K rows (h_kv heads x T tokens)
    // pages shorter than a stage's T tokens: one TMA box {64, page, h_kv} per
    // page (the stage's rows then go page by page), or for 8-token pages one
    // box {64, 8, 1} per page and kv head (rows head by head as usual)
    p->box_tokens = (p->paged && (1 << p->page_shift) < p->tile_tokens) ? (1 << p->page_shift) : p->tile_tokens;
    p->box_heads = (p->box_tokens < p->tile_tokens && p->box_tokens < 16) ? 1 : kv->h_kv;
    p->stage_bytes = kScoreRows * D * 2;
    int64_t chunks = 0;
    for (int b = 0; b < kv->batch; ++b) {
        const int64_t n = kv->capacity > 0 ? n_total : off[b + 1] - off[b];
        chunks += (n + p->tile_tokens - 1) / p->tile_tokens;
    }
    p->max_chunks = chunks;
    const int grid_cap = sms < 256 ? sms : 256;
    p->score_grid = (int)(chunks < grid_cap ? chunks : grid_cap);
    {
        // two stage parities x the pieces of up to 32 tokens (one lane
        // quarter's rows of one kv head) that a chunk of T = 128 / h_kv
        // tokens of a head is cut into: blocks of EBT tokens of a head, EBT
        // = T, or the page size when a paged stage goes page by page
        const int ebt = p->box_heads > 1 ? p->box_tokens : p->tile_tokens;
        const int span = ebt < 32 ? ebt : 32;
        p->score_partials_per_slot = 2 * (p->tile_tokens / span);
    }
    p->ld_logits = (n_total + 3) / 4 * 4;
    {
        // fused scoring: HS kv heads per pass, the largest of 4, 2, 1 that
        // divides h_kv and whose logits (HS * G * n_total * 4 bytes) fit the
        // L2 share a pass may keep; GP rows per kv head in the staged queries
        // (HS * GP >= 8 keeps every pass's first row on a 1024-byte atom)
        int hs = 4;
        while (hs > 1 && (kv->h_kv % hs != 0 || (double)hs * G * (double)n_total * 4.0 > (double)kFusedPassLogitsBytes))
            hs >>= 1;
        int gp = 4;
        while (gp < G || hs * gp < 8)
            gp <<= 1;
        p->fused_hs = hs;
        p->fused_gp = gp;
        p->fused_t = kFusedRows / hs;
        p->fused_n = hs * gp < 16 ? 16 : hs * gp;
        int64_t fc = 0;
        for (int b = 0; b < kv->batch; ++b) {
            const int64_t n = kv->capacity > 0 ? n_total : off[b + 1] - off[b];   // a growing cache: its capacity
            fc += (n + p->fused_t - 1) / p->fused_t;
        }
        p->fused_chunks = fc;
        p->fused_grid = (int)(fc < grid_cap ? fc : grid_cap);
        p->fused_ld = fc * p->fused_t;
    }
    p->sel_ranges = (int)((n_max + kSelectTokensPerCta - 1) / kSelectTokensPerCta) + 1;
    p->capacity = capacity;
    if (capacity > kMaxCapacity) {
        set_error("k + n_sink + n_local = %d exceeds the supported maximum %d", capacity, kMaxCapacity);
        return TS_ERR_UNSUPPORTED;
    }
    // every attention CTA takes at most kAttnRows selected rows
    p->attn_splits = capacity > 0 ? (capacity + kAttnRows - 1) / kAttnRows : 0;

    // small per-call tables first (they share a few pages), then the arrays
    // that grow with the cache, then the attention partials
    size_t o = 0;
    p->off_ctrl = o;
    o += 256;
    // everything above is the control block that ts_workspace_init zeroes
    const size_t nt1 = (size_t)(n_total > 0 ? n_total : 1);
    p->off_chunk_table = o;
    o = align_up(o + sizeof(int32_t) * (p->B + 1), 256);
    p->off_L = o;
    o = align_up(o + sizeof(double) * p->B * p->Hq, 256);
    p->off_partials = o;
    {
        // the two-phase pass A keeps R partials per (CTA, sequence) slot and
        // head, the fused kernel one
        const size_t two_phase = (size_t)(p->score_grid + p->B) * p->score_partials_per_slot;
        const size_t fused = (size_t)(p->fused_grid + p->B);
        o = align_up(o + sizeof(float) * 2 * (two_phase > fused ? two_phase : fused) * p->Hq, 256);
    }
    p->off_sel_inb1 = o;
    o = align_up(o + sizeof(uint32_t) * (size_t)p->B * p->sel_ranges, 256);
    p->off_sel_bin = o;
    o = align_up(o + sizeof(uint32_t) * 2 * (size_t)p->B, 256);
    p->off_sel_above = o;
    o = align_up(o + sizeof(uint32_t) * (size_t)p->B * p->sel_ranges, 256);
    p->off_sel_range_off = o;
    o = align_up(o + sizeof(uint32_t) * (size_t)p->B * p->sel_ranges, 256);
    p->off_sel_thr = o;
    o = align_up(o + sizeof(uint64_t) * (size_t)p->B, 256);
    p->off_sel_mode = o;
    o = align_up(o + sizeof(int32_t) * (size_t)p->B, 256);
    p->off_sel_prev_n = o;   // length + 1 at the previous selection (0: none yet)
    o = align_up(o + sizeof(int64_t) * (size_t)p->B, 256);
    p->off_sel_hist = o;
    o = align_up(o + sizeof(uint32_t) * 4096 * (size_t)p->B, 256);
    p->off_logits = o;
    {
        // two-phase rows of ld_logits tokens; fused rows of fused_ld (chunk-padded)
        const int64_t ld = p->ld_logits > p->fused_ld ? p->ld_logits : p->fused_ld;
        o = align_up(o + sizeof(float) * (size_t)p->Hq * (size_t)(ld > 0 ? ld : 4), 256);
    }
    // the fused scoring's running votes between passes, chunk-aligned like
    // its logits (16-byte aligned lines for bulk copies)
    p->off_vacc = o;
    o = align_up(o + sizeof(float) * (size_t)(p->fused_ld > 0 ? p->fused_ld : 4), 256);
    p->off_sel_cand = o;
    o = align_up(o + 8 * nt1, 256);
    // last: the only part whose size depends on the selection capacity, so
    // every offset above is the same for every entry point
    p->off_attn_part = o;
    if (capacity > 0)
        o = align_up(o + sizeof(float) * (size_t)p->B * p->Hkv * p->attn_splits * p->G * (D + 4), 256);
    p->total_bytes = o;
    return TS_OK;
}

static ts_status_t check_ws(const Plan &p, void *ws, size_t ws_bytes)
{
    if (ws == nullptr) {
        set_error("workspace is NULL");
        return TS_ERR_WORKSPACE;
    }
    if (reinterpret_cast<uintptr_t>(ws) & 255u) {
        set_error("workspace must be 256-byte aligned");
        return TS_ERR_WORKSPACE;
    }
    if (ws_bytes < p.total_bytes) {
        set_error("workspace too small: %zu bytes given, %zu needed", ws_bytes, p.total_bytes);
        return TS_ERR_WORKSPACE;
    }
    return TS_OK;
}

// K as a 3-D tensor (channels, tokens, kv heads) for TMA.  fused: boxes of
// {64, T, HS} (the fused scoring kernel, HS kv heads of T = 128 / HS tokens
// per stage); else {64, T, h_kv} (the two-phase pass A, every head of
// T = 128 / h_kv tokens per stage), or for a paged cache whose pages are
// shorter than T {64, page, h_kv} (one box per page) or, for 8-token pages,
// {64, 8, 1} (one box per page and kv head).
static ts_status_t encode_kmap(const Plan &p, const ts_kv_t *kv, CUtensorMap *map, bool fused = false)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr) {
        set_error("cuTensorMapEncodeTiled is not available from the driver");
        return TS_ERR_CUDA;
    }
    // dims (innermost first): channels, tokens, kv heads
    cuuint64_t dims[3] = {(cuuint64_t)p.D, (cuuint64_t)p.kv_rows, (cuuint64_t)p.Hkv};
    cuuint64_t strides[2] = {(cuuint64_t)kv->stride_tok * 2, (cuuint64_t)kv->stride_head * 2};
    cuuint32_t box[3] = {64u, fused ? (cuuint32_t)p.fused_t : (cuuint32_t)p.box_tokens,
                         fused ? (cuuint32_t)p.fused_hs : (cuuint32_t)p.box_heads};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(kv->k), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d)", (int)r);
        return TS_ERR_CUDA;
    }
    return TS_OK;
}

}  // namespace ts

using namespace ts;

extern "C" {

size_t ts_workspace_bytes(const ts_kv_t *kv, int32_t k, int32_t n_sink, int32_t n_local)
{
    if (k < 0 || n_sink < 0 || n_local < 0)
        return 0;
    Plan p;
    if (make_plan(kv, k + n_sink + n_local, &p) != TS_OK)
        return 0;
    return p.total_bytes;
}

ts_status_t ts_workspace_init(void *ws, size_t ws_bytes, void *stream)
{
    if (ws == nullptr || ws_bytes < 256) {
        set_error("workspace is NULL or smaller than its control block");
        return TS_ERR_WORKSPACE;
    }
    // The whole workspace starts at zero: the status word, and the selection
    // histogram and list counters, which the library returns to zero itself
    // after every use.
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "ts_workspace_init");
}

ts_status_t ts_selcache(const void *q, void *q_prev, int32_t *reuse, double *cos_out, int32_t first_step,
                        int32_t batch, int32_t h_q, int32_t head_dim, double threshold, void *stream)
{
    if (q == nullptr || q_prev == nullptr || reuse == nullptr) {
        set_error("q, q_prev and reuse are required");
        return TS_ERR_INVALID_ARG;
    }
    if (batch < 1 || h_q < 1 || (head_dim != 64 && head_dim != 128)) {
        set_error("bad shape (batch %d, h_q %d, head_dim %d)", batch, h_q, head_dim);
        return TS_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(q_prev)) & 3u) {
        set_error("q and q_prev must be 4-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    if (isnan(threshold)) {
        set_error("threshold is NaN");
        return TS_ERR_INVALID_ARG;
    }
    cudaError_t e = launch_selcache(q, q_prev, reuse, cos_out, first_step != 0, batch, h_q * head_dim, threshold,
                                    static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "ts_selcache launch");
}

static ts_status_t score_prologue(const ts_kv_t *kv, void *ws, size_t ws_bytes, Plan *p)
{
    ts_status_t s = make_plan(kv, -1, p);
    if (s != TS_OK)
        return s;
    // the score phases need everything up to the attention partials
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < p->off_attn_part) {
        set_error("workspace missing, misaligned or too small (%zu < %zu)", ws_bytes, p->off_attn_part);
        return TS_ERR_WORKSPACE;
    }
    return TS_OK;
}

// Pass A and the normaliser merge, the merge writing L to L_out (null: the
// workspace, where pass B reads it).
static ts_status_t score_logits_to(const ts_kv_t *kv, const void *q, const int32_t *reuse, void *ws,
                                   size_t ws_bytes, void *stream, double *L_out)
{
    Plan p;
    ts_status_t s = score_prologue(kv, ws, ws_bytes, &p);
    if (s != TS_OK)
        return s;
    if (q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15u)) {
        set_error("q is required and must be 16-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    if (p.n_total == 0)
        return TS_OK;
    CUtensorMap kmap;
    s = encode_kmap(p, kv, &kmap);
    if (s != TS_OK)
        return s;
    cudaError_t e = launch_score(p, kmap, q, kv->seq_offsets_dev, kv->seq_offsets_host, reuse, static_cast<uint8_t *>(ws),
                                 static_cast<cudaStream_t>(stream), kv->page_table_dev, kv->page_table_stride, L_out);
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "score pass A launch");
}

ts_status_t ts_score_logits(const ts_kv_t *kv, const void *q, const int32_t *reuse, void *ws, size_t ws_bytes,
                            void *stream)
{
    return score_logits_to(kv, q, reuse, ws, ws_bytes, stream, nullptr);
}

ts_status_t ts_score_vote(const ts_kv_t *kv, const int32_t *reuse, float *votes, void *ws, size_t ws_bytes,
                          void *stream)
{
    Plan p;
    ts_status_t s = score_prologue(kv, ws, ws_bytes, &p);
    if (s != TS_OK)
        return s;
    if (votes == nullptr) {
        set_error("votes is required");
        return TS_ERR_INVALID_ARG;
    }
    if (p.n_total == 0)
        return TS_OK;
    cudaError_t e = launch_vote(p, kv->seq_offsets_dev, reuse, votes, static_cast<uint8_t *>(ws),
                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "score pass B launch");
}

ts_status_t ts_score(const ts_kv_t *kv, const void *q, const int32_t *reuse, float *votes, void *ws,
                     size_t ws_bytes, void *stream)
{
    if (votes == nullptr) {
        set_error("votes is required");
        return TS_ERR_INVALID_ARG;
    }
    ts_status_t s = ts_score_logits(kv, q, reuse, ws, ws_bytes, stream);
    if (s != TS_OK)
        return s;
    return ts_score_vote(kv, reuse, votes, ws, ws_bytes, stream);
}

ts_status_t ts_score_fused(const ts_kv_t *kv, const void *q, const int32_t *reuse, float *votes, void *ws,
                           size_t ws_bytes, void *stream)
{
    Plan p;
    ts_status_t s = score_prologue(kv, ws, ws_bytes, &p);
    if (s != TS_OK)
        return s;
    if (p.paged) {
        set_error("ts_score_fused takes packed caches only (use ts_score for a paged cache)");
        return TS_ERR_UNSUPPORTED;
    }
    if (votes == nullptr) {
        set_error("votes is required");
        return TS_ERR_INVALID_ARG;
    }
    if (q == nullptr || (reinterpret_cast<uintptr_t>(q) & 15u)) {
        set_error("q is required and must be 16-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    if (p.n_total == 0)
        return TS_OK;
    CUtensorMap kmap;
    s = encode_kmap(p, kv, &kmap, true);
    if (s != TS_OK)
        return s;
    cudaError_t e = launch_score_fused(p, kmap, q, kv->seq_offsets_dev, kv->seq_offsets_host, reuse, votes,
                                      static_cast<uint8_t *>(ws), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "fused scoring launch");
}

ts_status_t ts_select(const ts_kv_t *kv, const float *votes, int32_t k, int32_t n_sink, int32_t n_local,
                      const int32_t *reuse, int32_t *ids, int32_t *count, void *ws, size_t ws_bytes, void *stream)
{
    if (k < 0 || n_sink < 0 || n_local < 0 || (int64_t)k + n_sink + n_local > (int64_t(1) << 30)) {
        set_error("k, n_sink, n_local must be non-negative with a sum below 2^30");
        return TS_ERR_INVALID_ARG;
    }
    Plan p;
    ts_status_t s = make_plan(kv, k + n_sink + n_local, &p);
    if (s != TS_OK)
        return s;
    if (votes == nullptr || ids == nullptr || count == nullptr) {
        set_error("votes, ids and count are required");
        return TS_ERR_INVALID_ARG;
    }
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < p.off_attn_part) {
        set_error("workspace missing, misaligned or too small (%zu < %zu)", ws_bytes, p.off_attn_part);
        return TS_ERR_WORKSPACE;
    }
    cudaError_t e = launch_select(p, kv->seq_offsets_dev, votes, k, n_sink, n_local, reuse, ids, count,
                                  static_cast<uint8_t *>(ws), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "select launch");
}

ts_status_t ts_sparse_attn(const ts_kv_t *kv, const void *q, const int32_t *ids, const int32_t *count,
                           int32_t ids_capacity, float *out, void *ws, size_t ws_bytes, void *stream)
{
    if (ids_capacity < 1) {
        set_error("ids_capacity must be >= 1");
        return TS_ERR_INVALID_ARG;
    }
    Plan p;
    ts_status_t s = make_plan(kv, ids_capacity, &p);
    if (s != TS_OK)
        return s;
    if (q == nullptr || ids == nullptr || count == nullptr || out == nullptr) {
        set_error("q, ids, count and out are required");
        return TS_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15u) {
        set_error("q and out must be 16-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    s = check_ws(p, ws, ws_bytes);
    if (s != TS_OK)
        return s;
    cudaError_t e = launch_attn(p, kv, q, ids, count, out, static_cast<uint8_t *>(ws),
                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "sparse attention launch");
}

ts_status_t ts_sparse_attn_noalloc(const ts_kv_t *kv, const void *q, const int32_t *ids, const int32_t *count,
                                   int32_t ids_capacity, float *out, void *stream)
{
    if (ids_capacity < 1) {
        set_error("ids_capacity must be >= 1");
        return TS_ERR_INVALID_ARG;
    }
    Plan p;
    ts_status_t s = make_plan(kv, ids_capacity, &p);
    if (s != TS_OK)
        return s;
    if (q == nullptr || ids == nullptr || count == nullptr || out == nullptr) {
        set_error("q, ids, count and out are required");
        return TS_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15u) {
        set_error("q and out must be 16-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    return launch_attn_noalloc(p, kv, q, ids, count, out, static_cast<cudaStream_t>(stream));
}

// ts_decode_step under stream capture with the selection cache able to
// reuse: cosine test -> IF (condition) { scoring, selection } -> attention.  The condition is 1 at every launch of the graph; the cosine
// kernel sets it to 0 when every sequence reuses, and the body then does not
// run at all (its kernels would only have read the flags and returned).
static ts_status_t decode_step_graph(const Plan &p, const CUtensorMap &kmap, const ts_kv_t *kv, const void *q,
                                     void *q_prev, int32_t *reuse, double *cos_out, double threshold, int32_t k,
                                     int32_t n_sink, int32_t n_local, float *votes, int32_t *ids, int32_t *count,
                                     float *out, uint8_t *w, cudaStream_t st, cudaGraph_t graph)
{
    cudaGraphConditionalHandle handle;
    cudaError_t e = cudaGraphConditionalHandleCreate(&handle, graph, 1u, cudaGraphCondAssignDefault);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: conditional handle");
    SelcacheSkip skip = {};
    skip.handle = handle;
    skip.counters = reinterpret_cast<uint32_t *>(w + p.off_ctrl) + kCtrlSkipCounters;
    skip.enabled = 1;
    e = launch_selcache(q, q_prev, reuse, cos_out, 0, p.B, p.Hq * p.D, threshold, st, &skip);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: selection cache launch");
    cudaStreamCaptureStatus cap;
    const cudaGraphNode_t *deps = nullptr;
    size_t ndeps = 0;
    e = cudaStreamGetCaptureInfo(st, &cap, nullptr, &graph, &deps, &ndeps);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: capture dependencies");
    cudaGraphNodeParams np = {};
    np.type = cudaGraphNodeTypeConditional;
    np.conditional.handle = handle;
    np.conditional.type = cudaGraphCondTypeIf;
    np.conditional.size = 1;
    cudaGraphNode_t cond_node;
    e = cudaGraphAddNode(&cond_node, graph, deps, ndeps, &np);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: conditional node");
    cudaGraph_t body = np.conditional.phGraph_out[0];
    cudaStream_t side;
    e = body_stream(&side);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: body capture stream");
    e = cudaStreamBeginCaptureToGraph(side, body, nullptr, nullptr, 0, cudaStreamCaptureModeRelaxed);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: body capture");
    const SelectWindow win = {k, n_sink, n_local};
    cudaError_t le = launch_score(p, kmap, q, kv->seq_offsets_dev, kv->seq_offsets_host, reuse, w, side,
                                  kv->page_table_dev, kv->page_table_stride);
    if (le == cudaSuccess)
        le = launch_vote(p, kv->seq_offsets_dev, reuse, votes, w, side, &win);
    if (le == cudaSuccess)
        le = launch_select(p, kv->seq_offsets_dev, votes, k, n_sink, n_local, reuse, ids, count, w, side, true);
    cudaGraph_t captured = nullptr;
    e = cudaStreamEndCapture(side, &captured);
    if (le != cudaSuccess)
        return cuda_fail(le, "ts_decode_step: conditional body launch");
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: body capture end");
    e = cudaStreamUpdateCaptureDependencies(st, &cond_node, 1, cudaStreamSetCaptureDependencies);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: capture dependencies");
    e = launch_attn(p, kv, q, ids, count, out, w, st);
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "ts_decode_step: sparse attention launch");
}

ts_status_t ts_decode_step(const ts_kv_t *kv, const void *q, void *q_prev, int32_t *reuse, double *cos_out,
                           int32_t first_step, double threshold, int32_t k, int32_t n_sink, int32_t n_local,
                           float *votes, int32_t *ids, int32_t *count, float *out, void *ws, size_t ws_bytes,
                           void *stream)
{
    // every argument is checked before the first launch
    if (k < 0 || n_sink < 0 || n_local < 0 || (int64_t)k + n_sink + n_local > (int64_t(1) << 30) ||
        k + n_sink + n_local < 1) {
        set_error("k, n_sink, n_local must be non-negative with a sum in [1, 2^30)");
        return TS_ERR_INVALID_ARG;
    }
    Plan p;
    ts_status_t s = make_plan(kv, k + n_sink + n_local, &p);
    if (s != TS_OK)
        return s;
    if (q == nullptr || q_prev == nullptr || reuse == nullptr || votes == nullptr || ids == nullptr ||
        count == nullptr || out == nullptr) {
        set_error("q, q_prev, reuse, votes, ids, count and out are required");
        return TS_ERR_INVALID_ARG;
    }
    if (((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15u) ||
        (reinterpret_cast<uintptr_t>(q_prev) & 3u)) {
        set_error("q and out must be 16-byte aligned, q_prev 4-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    if (isnan(threshold)) {
        set_error("threshold is NaN");
        return TS_ERR_INVALID_ARG;
    }
    s = check_ws(p, ws, ws_bytes);
    if (s != TS_OK)
        return s;
    CUtensorMap kmap;
    if (p.n_total > 0) {
        s = encode_kmap(p, kv, &kmap);
        if (s != TS_OK)
            return s;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint8_t *w = static_cast<uint8_t *>(ws);
    // captured into a graph with the selection cache able to reuse: scoring
    // and selection go into a conditional node the cosine kernel can switch off
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaGraph_t graph = nullptr;
    cudaError_t e = cudaStreamGetCaptureInfo(st, &cap, nullptr, &graph, nullptr, nullptr);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: capture query");
    const bool can_reuse = first_step == 0 && threshold <= 1.0 + 1e-6;
    if (cap == cudaStreamCaptureStatusActive && can_reuse && p.n_total > 0 && reuse_skip_enabled())
        return decode_step_graph(p, kmap, kv, q, q_prev, reuse, cos_out, threshold, k, n_sink, n_local, votes, ids,
                                 count, out, w, st, graph);
    e = launch_selcache(q, q_prev, reuse, cos_out, first_step != 0, p.B, p.Hq * p.D, threshold, st);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: selection cache launch");
    if (p.n_total > 0) {
        e = launch_score(p, kmap, q, kv->seq_offsets_dev, kv->seq_offsets_host, reuse, w, st, kv->page_table_dev,
                         kv->page_table_stride);
        if (e != cudaSuccess)
            return cuda_fail(e, "ts_decode_step: score pass A launch");
        const SelectWindow win = {k, n_sink, n_local};
        e = launch_vote(p, kv->seq_offsets_dev, reuse, votes, w, st, &win);
        if (e != cudaSuccess)
            return cuda_fail(e, "ts_decode_step: score pass B launch");
    }
    e = launch_select(p, kv->seq_offsets_dev, votes, k, n_sink, n_local, reuse, ids, count, w, st, true);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_decode_step: select launch");
    e = launch_attn(p, kv, q, ids, count, out, w, st);
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "ts_decode_step: sparse attention launch");
}

int32_t ts_decode_step_kernels(const ts_kv_t *kv, int32_t k, int32_t n_sink, int32_t n_local)
{
    if (k < 0 || n_sink < 0 || n_local < 0 || (int64_t)k + n_sink + n_local > (int64_t(1) << 30) ||
        k + n_sink + n_local < 1) {
        set_error("k, n_sink, n_local must be non-negative with a sum in [1, 2^30)");
        return -1;
    }
    Plan p;
    if (make_plan(kv, k + n_sink + n_local, &p) != TS_OK)
        return -1;
    // selection cache; score pass A, normaliser merge, vote pass (with the
    // selection histogram); collect, resolve, write; attention split, merge
    return 1 + (p.n_total > 0 ? 3 : 0) + 3 + 2;
}

ts_status_t ts_get_device_status(void *ws, size_t ws_bytes, uint32_t *site_out, void *stream)
{
    if (ws == nullptr || ws_bytes < 256) {
        set_error("workspace is NULL or too small");
        return TS_ERR_WORKSPACE;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t h[2] = {0u, 0u};
    cudaError_t e = cudaMemcpyAsync(h, ws, sizeof h, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(ws, 0, sizeof h, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    if (e != cudaSuccess)
        return cuda_fail(e, "ts_get_device_status");
    if (site_out)
        *site_out = h[1];
    if (h[0] == 2u) {
        set_error("ts_append_kv found the cache full");
        return TS_ERR_INVALID_ARG;
    }
    if (h[0] != 0u) {
        set_error("a device-side wait gave up (site %u)", h[1]);
        return TS_ERR_DEVICE_TIMEOUT;
    }
    return TS_OK;
}

ts_status_t ts_append_kv(const ts_kv_t *kv, int64_t *seq_offsets, void *k_cache, void *v_cache, const void *k_new,
                         const void *v_new, void *ws, size_t ws_bytes, void *stream)
{
    if (kv == nullptr || kv->capacity <= 0) {
        set_error("ts_append_kv needs a cache with a capacity");
        return TS_ERR_INVALID_ARG;
    }
    if (seq_offsets != kv->seq_offsets_dev || k_cache != kv->k || v_cache != kv->v) {
        set_error("seq_offsets, k_cache and v_cache must be the cache's own device arrays");
        return TS_ERR_INVALID_ARG;
    }
    if (k_new == nullptr || v_new == nullptr ||
        ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & 15u)) {
        set_error("k_new and v_new must be 16-byte aligned device rows");
        return TS_ERR_INVALID_ARG;
    }
    if (ws == nullptr || ws_bytes < 256) {
        set_error("workspace is NULL or smaller than its control block");
        return TS_ERR_WORKSPACE;
    }
    Plan p;
    const ts_status_t s = make_plan(kv, -1, &p);
    if (s != TS_OK)
        return s;
    cudaError_t e = launch_append(seq_offsets, k_cache, v_cache, k_new, v_new, kv->stride_tok, kv->stride_head,
                                  p.Hkv, p.D, kv->capacity, reinterpret_cast<uint32_t *>(ws),
                                  static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "ts_append_kv");
}

ts_status_t ts_selftest_expire_wait(void *ws, size_t ws_bytes, uint32_t spin_limit, void *stream)
{
    if (ws == nullptr || ws_bytes < 256) {
        set_error("workspace is NULL or too small");
        return TS_ERR_WORKSPACE;
    }
    if (spin_limit == 0 || spin_limit > (1u << 20)) {
        set_error("spin_limit must be in [1, 2^20]");
        return TS_ERR_INVALID_ARG;
    }
    cudaError_t e = launch_selftest_wait(static_cast<uint32_t *>(ws), spin_limit, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "selftest launch");
}

// ---------------------------------------------------------------------------
// Token-axis split of one sequence across ranks
// ---------------------------------------------------------------------------

ts_status_t ts_score_normalisers(const ts_kv_t *kv, const void *q, const int32_t *reuse, double *L_out, void *ws,
                                 size_t ws_bytes, void *stream)
{
    if (L_out == nullptr) {
        set_error("L_out is required");
        return TS_ERR_INVALID_ARG;
    }
    // the merge writes L_out itself (no copy between kernels: the chain keeps
    // its programmatic launches)
    ts_status_t s = score_logits_to(kv, q, reuse, ws, ws_bytes, stream, L_out);
    if (s != TS_OK)
        return s;
    Plan p;
    s = make_plan(kv, -1, &p);
    if (s != TS_OK)
        return s;
    if (p.n_total != 0)
        return TS_OK;
    // nothing scored: every L is -inf (a merge of no parts)
    cudaError_t e = launch_merge_normalisers(nullptr, 0, (int64_t)p.B * p.Hq, L_out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "normalisers launch");
}

ts_status_t ts_score_vote_normalised(const ts_kv_t *kv, const int32_t *reuse, const double *L_in, float *votes,
                                     void *ws, size_t ws_bytes, void *stream)
{
    Plan p;
    ts_status_t s = score_prologue(kv, ws, ws_bytes, &p);
    if (s != TS_OK)
        return s;
    if (votes == nullptr || L_in == nullptr) {
        set_error("votes and L_in are required");
        return TS_ERR_INVALID_ARG;
    }
    if (p.n_total == 0)
        return TS_OK;
    cudaError_t e = launch_vote(p, kv->seq_offsets_dev, reuse, votes, static_cast<uint8_t *>(ws),
                                static_cast<cudaStream_t>(stream), nullptr, L_in);
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "score pass B launch");
}

ts_status_t ts_merge_normalisers(const double *L_parts, int32_t parts, int64_t count, double *L_out, void *stream)
{
    if (L_parts == nullptr || L_out == nullptr || parts < 1 || count < 0) {
        set_error("L_parts and L_out are required, parts >= 1, count >= 0");
        return TS_ERR_INVALID_ARG;
    }
    cudaError_t e = launch_merge_normalisers(L_parts, parts, count, L_out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "normaliser merge launch");
}

// The shard's share of the sequence's windows: sink [0, s') and local window
// [l0, n) of the whole sequence, intersected with [t, t + n_loc), as counts
// of the shard's first and last tokens.
static ts_status_t shard_windows(const ts_kv_t *kv, int32_t n_sink, int32_t n_local, int64_t t, int64_t n_global,
                                 int64_t *n_loc, int *s_loc, int *l_loc)
{
    if (kv == nullptr || kv->batch != 1 || kv->seq_offsets_host == nullptr || kv->capacity != 0) {
        set_error("a shard is one sequence (batch 1, no capacity)");
        return TS_ERR_INVALID_ARG;
    }
    *n_loc = kv->seq_offsets_host[1] - kv->seq_offsets_host[0];
    if (t < 0 || *n_loc < 0 || t + *n_loc > n_global || n_global >= (int64_t(1) << 31)) {
        set_error("shard [%lld, %lld) must lie in the sequence [0, %lld), below 2^31 tokens", (long long)t,
                  (long long)(t + *n_loc), (long long)n_global);
        return TS_ERR_INVALID_ARG;
    }
    const int64_t s = n_sink < n_global ? n_sink : n_global;
    const int64_t l0 = n_global - n_local > s ? n_global - n_local : s;
    int64_t a = (s < t + *n_loc ? s : t + *n_loc) - t;
    int64_t c = t + *n_loc - (l0 > t ? l0 : t);
    *s_loc = (int)(a < 0 ? 0 : a);
    *l_loc = (int)(c < 0 ? 0 : c);
    return TS_OK;
}

ts_status_t ts_select_candidates(const ts_kv_t *kv, const float *votes, int32_t k, int32_t n_sink, int32_t n_local,
                                 int64_t shard_offset, int64_t n_global, int32_t *ids, int32_t *count,
                                 uint64_t *keys_out, void *ws, size_t ws_bytes, void *stream)
{
    if (k < 1 || n_sink < 0 || n_local < 0 || (int64_t)k + n_sink + n_local > kMaxCapacity) {
        set_error("k >= 1, n_sink, n_local >= 0, k + n_sink + n_local <= %d", kMaxCapacity);
        return TS_ERR_INVALID_ARG;
    }
    int64_t n_loc;
    int s_loc, l_loc;
    ts_status_t s = shard_windows(kv, n_sink, n_local, shard_offset, n_global, &n_loc, &s_loc, &l_loc);
    if (s != TS_OK)
        return s;
    if (votes == nullptr || ids == nullptr || count == nullptr || keys_out == nullptr) {
        set_error("votes, ids, count and keys_out are required");
        return TS_ERR_INVALID_ARG;
    }
    s = ts_select(kv, votes, k, s_loc, l_loc, nullptr, ids, count, ws, ws_bytes, stream);
    if (s != TS_OK)
        return s;
    cudaError_t e = launch_candidate_keys(votes, ids, count, s_loc, l_loc, shard_offset, k,
                                          reinterpret_cast<unsigned long long *>(keys_out),
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "candidate keys launch");
}

ts_status_t ts_select_merge(const ts_kv_t *kv, const uint64_t *keys_all, int32_t parts, int32_t rank, int32_t k,
                            int32_t n_sink, int32_t n_local, int64_t shard_offset, int64_t n_global, int32_t *ids,
                            int32_t *count, void *stream)
{
    if (k < 1 || n_sink < 0 || n_local < 0 || (int64_t)k + n_sink + n_local > kMaxCapacity || parts < 1 ||
        rank < 0 || rank >= parts || (int64_t)parts * k > (int64_t(1) << 30)) {
        set_error("k >= 1, 0 <= rank < parts, k + n_sink + n_local <= %d", kMaxCapacity);
        return TS_ERR_INVALID_ARG;
    }
    int64_t n_loc;
    int s_loc, l_loc;
    ts_status_t s = shard_windows(kv, n_sink, n_local, shard_offset, n_global, &n_loc, &s_loc, &l_loc);
    if (s != TS_OK)
        return s;
    if (keys_all == nullptr || ids == nullptr || count == nullptr) {
        set_error("keys_all, ids and count are required");
        return TS_ERR_INVALID_ARG;
    }
    cudaError_t e = launch_select_merge(reinterpret_cast<const unsigned long long *>(keys_all), parts, k, k, rank,
                                        s_loc, l_loc, n_loc, shard_offset, k + n_sink + n_local, ids, count,
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "selection merge launch");
}

ts_status_t ts_sparse_attn_lse(const ts_kv_t *kv, const void *q, const int32_t *ids, const int32_t *count,
                               int32_t ids_capacity, float *out, float *lse_out, void *ws, size_t ws_bytes,
                               void *stream)
{
    if (ids_capacity < 1) {
        set_error("ids_capacity must be >= 1");
        return TS_ERR_INVALID_ARG;
    }
    Plan p;
    ts_status_t s = make_plan(kv, ids_capacity, &p);
    if (s != TS_OK)
        return s;
    if (q == nullptr || ids == nullptr || count == nullptr || out == nullptr || lse_out == nullptr) {
        set_error("q, ids, count, out and lse_out are required");
        return TS_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15u) {
        set_error("q and out must be 16-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    s = check_ws(p, ws, ws_bytes);
    if (s != TS_OK)
        return s;
    cudaError_t e = launch_attn(p, kv, q, ids, count, out, static_cast<uint8_t *>(ws),
                                static_cast<cudaStream_t>(stream), lse_out);
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "sparse attention launch");
}

ts_status_t ts_merge_attention(const float *out_parts, const float *lse_parts, int32_t parts, int64_t rows,
                               int32_t head_dim, float *out, void *stream)
{
    if (out_parts == nullptr || lse_parts == nullptr || out == nullptr || parts < 1 || rows < 0 || head_dim < 1) {
        set_error("out_parts, lse_parts and out are required, parts >= 1, rows >= 0, head_dim >= 1");
        return TS_ERR_INVALID_ARG;
    }
    cudaError_t e = launch_merge_attention(out_parts, lse_parts, parts, rows, head_dim, out,
                                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "attention merge launch");
}

// ---------------------------------------------------------------------------
// Page-level comparator
// ---------------------------------------------------------------------------

static ts_status_t quest_prologue(const ts_kv_t *kv, int32_t page_size, int capacity, Plan *p)
{
    if (page_size < 1 || page_size > 4096 || (page_size & (page_size - 1)) != 0) {
        set_error("page_size %d must be a power of two in [1, 4096]", page_size);
        return TS_ERR_INVALID_ARG;
    }
    return make_plan(kv, capacity, p);
}

int64_t ts_quest_rows(const ts_kv_t *kv, int32_t page_size)
{
    Plan p;
    if (quest_prologue(kv, page_size, 1, &p) != TS_OK)
        return -1;
    return quest_rows(p, page_size);
}

ts_status_t ts_quest_metadata(const ts_kv_t *kv, int32_t page_size, void *kmin, void *kmax, void *stream)
{
    Plan p;
    ts_status_t s = quest_prologue(kv, page_size, 1, &p);
    if (s != TS_OK)
        return s;
    if (kmin == nullptr || kmax == nullptr ||
        ((reinterpret_cast<uintptr_t>(kmin) | reinterpret_cast<uintptr_t>(kmax)) & 15u)) {
        set_error("kmin and kmax are required and must be 16-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    cudaError_t e = launch_quest_meta(p, kv, page_size, kmin, kmax, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "quest metadata launch");
}

ts_status_t ts_quest_metadata_update(const ts_kv_t *kv, int32_t page_size, int64_t last_tokens, void *kmin,
                                     void *kmax, void *stream)
{
    if (last_tokens < 1) {
        set_error("last_tokens %lld must be at least 1", (long long)last_tokens);
        return TS_ERR_INVALID_ARG;
    }
    Plan p;
    ts_status_t s = quest_prologue(kv, page_size, 1, &p);
    if (s != TS_OK)
        return s;
    if (kmin == nullptr || kmax == nullptr ||
        ((reinterpret_cast<uintptr_t>(kmin) | reinterpret_cast<uintptr_t>(kmax)) & 15u)) {
        set_error("kmin and kmax are required and must be 16-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    cudaError_t e =
        launch_quest_meta(p, kv, page_size, kmin, kmax, static_cast<cudaStream_t>(stream), last_tokens);
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "quest metadata update launch");
}

ts_status_t ts_quest_score(const ts_kv_t *kv, const void *q, int32_t page_size, const void *kmin, const void *kmax,
                           float *scores, void *stream)
{
    Plan p;
    ts_status_t s = quest_prologue(kv, page_size, 1, &p);
    if (s != TS_OK)
        return s;
    if (q == nullptr || kmin == nullptr || kmax == nullptr || scores == nullptr ||
        ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(kmin) | reinterpret_cast<uintptr_t>(kmax) |
          reinterpret_cast<uintptr_t>(scores)) & 15u)) {
        set_error("q, kmin, kmax and scores are required and 16-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    cudaError_t e = launch_quest_score(p, kv, q, page_size, kmin, kmax, scores, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "quest score launch");
}

ts_status_t ts_quest_select(const ts_kv_t *kv, const float *scores, int32_t page_size, int32_t k, int32_t n_sink,
                            int32_t n_local, int32_t *ids, int32_t *count, void *stream)
{
    if (k < 0 || n_sink < 0 || n_local < 0) {
        set_error("k, n_sink and n_local must be >= 0");
        return TS_ERR_INVALID_ARG;
    }
    Plan p;
    ts_status_t s = quest_prologue(kv, page_size, k + n_sink + n_local, &p);
    if (s != TS_OK)
        return s;
    if (scores == nullptr || ids == nullptr || count == nullptr || (reinterpret_cast<uintptr_t>(scores) & 15u)) {
        set_error("scores, ids and count are required; scores 16-byte aligned");
        return TS_ERR_INVALID_ARG;
    }
    cudaError_t e = launch_quest_select(p, kv, scores, page_size, k, n_sink, n_local, ids, count,
                                        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TS_OK : cuda_fail(e, "quest select launch");
}

const char *ts_status_string(ts_status_t status)
{
    switch (status) {
    case TS_OK: return "TS_OK";
    case TS_ERR_INVALID_ARG: return "TS_ERR_INVALID_ARG";
    case TS_ERR_UNSUPPORTED: return "TS_ERR_UNSUPPORTED";
    case TS_ERR_WORKSPACE: return "TS_ERR_WORKSPACE";
    case TS_ERR_CUDA: return "TS_ERR_CUDA";
    case TS_ERR_DEVICE_TIMEOUT: return "TS_ERR_DEVICE_TIMEOUT";
    }
    return "TS_ERR_UNKNOWN";
}

const char *ts_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
