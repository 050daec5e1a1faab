// Score pass A: per-head criticality logits over the whole K cache and the
// per-head softmax normalisers (TokenSelect README, "Key Takeaways": per-head
// Q.K criticality; per-head soft voting normalises each head by a softmax
// over the tokens).
//
// For every active sequence b, KV head g and query head h = g*G + j:
//   s[h, i] = scale * q[b, h, :] . K[b, i, g, :]        (fp32 accumulation)
// written to the logits workspace [h_q][ld], and
//   L[b, h] = log sum_i exp(s[h, i])                   (score_merge below)
//
// Design (B200):
//  * One CTA per SM, persistent.  The active sequences' tokens are cut into
//    chunks of T = 128 / h_kv tokens, so that a chunk holds 128 K rows (h_kv
//    heads x T tokens, one pipeline stage).  Several sequences: CTA j takes
//    the contiguous, balanced chunk range [j*C/grid, (j+1)*C/grid); one
//    sequence: the chunks are dealt round-robin (CTA j: j, j + grid, ...), so
//    every SM reads from every part of the cache.
//  * Warp 8 streams K with 3-D TMA boxes {64 channels, T tokens, h_kv heads}
//    (128-byte swizzle, L2 evict-first) into a ring of stages guarded by
//    mbarriers.  Before waiting for the previous kernel in the stream it
//    already asks L2 for its first tiles.
//  * Warp 9 owns the tensor cores: it allocates TMEM, writes the sequence's
//    queries into shared memory in the same swizzled K-major layout (row
//    g*GP + j = query head g*G + j, rows j >= G zero; GP = 4, 8 or 16), and one
//    lane issues, per stage, the tcgen05.mma chain
//        D[128 x N] = Kstage[128 x d] . Q[N x d]^T,   N = h_kv * GP,
//    d/16 instructions of K = 16 into one of four TMEM accumulators, then
//    commits to the stage's "empty" barrier (the ring slot is free once the
//    MMAs have read it) and to the accumulator's "full" barrier.  Row g*T + t
//    of D holds token t's logits against every query head; the columns
//    g*GP .. g*GP+G-1 are the ones of its own group.
//  * Warps 0-7 are the epilogue: thread i of warps w and w+4 owns TMEM lane
//    32w + i, i.e. one (kv head, token) row; warp w takes the even stages and
//    warp w+4 the odd ones (two warps per TMEM lane quarter hide the load and
//    exp latencies for any group size).  A thread loads its group's G
//    columns with tcgen05.ld, frees the accumulator, scales, stores the
//    logits (a warp writes 32 consecutive tokens of a head: coalesced) and
//    keeps an online (max, sum exp) per head; when the CTA leaves a sequence
//    each warp reduces these over its lanes (integer max of order-preserving
//    keys, a fixed shuffle tree: deterministic) and writes them, with no
//    barrier, as its own partial of each head: entry r of slot j + b (CTA j,
//    sequence b), R entries per slot.  The slot is unique: along the chunk
//    order neither j nor b decreases and one of them grows at every new
//    (CTA, sequence) segment.  No fences, atomics or waits on other CTAs;
//    every wait on a barrier is bounded.
//  * score_merge (one warp per sequence and head) folds the partials of the
//    CTAs that cover the sequence (j0..j1; every CTA with chunks for one
//    sequence) into L[b, h]: fp32 terms exp(m - M) <= 1 summed in float64.
#include "score_common.cuh"
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

constexpr int kMaxPrefetchTiles = 6;
constexpr int kProducerWarp = kScoreEpiWarps;       // 8
constexpr int kMmaWarp = kScoreEpiWarps + 1;        // 9

struct ScoreArgs {
    const __nv_bfloat16 *q;   // [B, Hq, D]
    const int64_t *seq_off;   // [B + 1]
    const int32_t *reuse;     // [B] or null
    float *logits;            // [Hq][ld]
    int64_t ld;
    float2 *partials;         // [Hq][S][R] (max, sum exp(x - max)) at slot CTA + sequence, entry per warp
    int S;                    // segment slots per head: grid + B
    int R;                    // partials per segment slot: epilogue warps that see one head
    int32_t *chunk_table;     // [B + 1] first active chunk of each sequence (for score_merge)
    uint32_t *ctrl;           // status word
    int B, Hq, Hkv, G;
    int T;                    // tokens per chunk / stage
    int stage_bytes;
    int nstages;              // ring depth
    int64_t pf_off[33];       // B <= 32: the host copy of the offsets, for the prefetch hints only
    uint32_t tmem_cols;       // TMEM columns allocated (power of 2 >= 4 * N)
    float scale;
    // paged cache (page_table != null): token i of sequence b is pool row
    // page_table[b * pt_stride + (i >> page_shift)] << page_shift | (i & (page - 1))
    const int32_t *page_table;
    int pt_stride;
    int page_shift;
    int64_t pool_pages;
    int box_tokens;           // BT: tokens of one TMA box: T, or the page size when pages are shorter than T
    int box_heads;            // kv heads of one TMA box: h_kv, or 1 (one box per page and kv head)
};

struct __align__(16) ScoreShared {
    uint64_t full[kScoreMaxStages];
    uint64_t empty[kScoreMaxStages];
    uint64_t acc_full[kScoreAccBufs];
    uint64_t acc_empty[kScoreAccBufs];
    uint64_t mma_done;        // every MMA issued so far has completed
    int64_t off[kMaxBatch + 1];
    int32_t chunk_start[kMaxBatch + 1];
    uint32_t tmem_base;
    int32_t pf_start[32];     // all-active chunk table of the prefetch hints (B <= 32)
    int64_t pf_off[32];       // and the sequence offsets it was built from
};

__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap *map, int32_t x, int32_t y, int32_t z)
{
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// chunk_start[b] (b <= B): first chunk of sequence b, leaving out sequences
// that reuse their selection when use_reuse is set.  Every thread calls it.
__device__ __forceinline__ void build_chunk_table(ScoreShared &sh, const int32_t *reuse, int B, int T, int warp,
                                                  int lane, bool use_reuse)
{
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        const int64_t n = sh.off[b + 1] - sh.off[b];
        const bool active = !use_reuse || reuse == nullptr || reuse[b] == 0;
        sh.chunk_start[b + 1] = (active && n > 0) ? (int32_t)((n + T - 1) / T) : 0;
    }
    __syncthreads();
    if (warp == 0) {
        int32_t run = 0;
        for (int base = 0; base < B; base += 32) {
            const int b = base + lane;
            int32_t x = (b < B) ? sh.chunk_start[b + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o)
                    x += y;
            }
            if (b < B)
                sh.chunk_start[b + 1] = run + x;
            run += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0)
            sh.chunk_start[0] = 0;
    }
    __syncthreads();
}

// B <= 32: lane b < B computes c0 = first chunk of sequence b and c1 = one past
// its last (sequences with reuse set, when reuse is given, have no chunks),
// with one round trip for the offsets and flags and a warp scan.
__device__ __forceinline__ void warp_chunk_scan(const int64_t *seq_off, const int32_t *reuse, int B, int T,
                                                int lane, int32_t &c0, int32_t &c1, int64_t &o0, int64_t &o1)
{
    int32_t x = 0;
    o0 = o1 = 0;
    if (lane < B) {
        o0 = __ldcg(seq_off + lane);
        o1 = __ldcg(seq_off + lane + 1);
        const int64_t n = o1 - o0;
        const bool active = reuse == nullptr || __ldcg(reuse + lane) == 0;
        x = (active && n > 0) ? (int32_t)((n + T - 1) / T) : 0;
    }
    int32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    c0 = incl - x;
    c1 = incl;
}

// The queries of sequence b as the UMMA B operand: N = h_kv*GP rows of d
// channels, bf16, K-major with the 128-byte swizzle (64-channel halves of
// N * 128 bytes).  Whole warp.
// MMA N: one GP-row block per kv head, at least 16 (the M = 128 shapes need
// N to be a multiple of 16).
template <int GP>
__host__ __device__ constexpr int score_mma_n(int Hkv)
{
    return Hkv * GP < 16 ? 16 : Hkv * GP;
}

template <int D, int GP>
__device__ __forceinline__ void stage_queries(uint8_t *qs, const __nv_bfloat16 *qb, int G, int Hkv, int lane)
{
    const int N = score_mma_n<GP>(Hkv);
    constexpr int kChunks = D / 8;           // 16-byte chunks per row
    constexpr int kBatch = 8;
    for (int c0 = lane; c0 < N * kChunks; c0 += 32 * kBatch) {
        uint4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int c = c0 + u * 32;
            const int n = c / kChunks, cc = c - n * kChunks;
            const int g = n / GP, j = n - g * GP;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (c < N * kChunks && g < Hkv && j < G)   // rows past the last head stay zero
                v[u] = __ldg(reinterpret_cast<const uint4 *>(qb + (int64_t)(g * G + j) * D) + cc);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int c = c0 + u * 32;
            if (c < N * kChunks) {
                const int n = c / kChunks, cc = c - n * kChunks;
                const int half = cc >> 3, ci = cc & 7;
                *reinterpret_cast<uint4 *>(qs + (size_t)half * N * 128 + n * 128 + ((ci ^ (n & 7)) << 4)) = v[u];
            }
        }
    }
}

// End of a (CTA, sequence) segment in the epilogue: reduce each head's
// (max, sum exp) over the lanes of this warp that hold it (one integer max
// reduction, one exp2 per lane, a fixed shuffle tree of adds: deterministic)
// and write it as this warp's partial of the head.  A (CTA, sequence) segment
// owns R partial slots per head, one per epilogue warp that sees the head
// (two stage parities x the lane quarters the head spans); score_merge folds
// them.  No barrier: the warps of the CTA never wait for each other here.
// (m, z) are consumed: on return they hold the warp's (max, sum) per head.
template <int GP>
__device__ __forceinline__ void score_flush(float (&m)[GP], float (&z)[GP], int G, int span, int lane, int slot,
                                            int g, float2 *partials, int64_t stride, int64_t slot_base)
{
    const uint32_t grp = span == 32 ? 0xffffffffu : (lane < 16 ? 0x0000ffffu : 0xffff0000u);
#pragma unroll
    for (int j = 0; j < GP; ++j) {
        const float M = float_from_order_key(__reduce_max_sync(grp, float_order_key(m[j])));
        z[j] = (m[j] == -INFINITY) ? 0.0f : z[j] * exp2f((m[j] - M) * kLog2e);
        m[j] = M;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        if (o < span) {
#pragma unroll
            for (int j = 0; j < GP; ++j)
                z[j] += __shfl_xor_sync(0xffffffffu, z[j], o);
        }
    if ((lane % span) == 0) {
#pragma unroll
        for (int j = 0; j < GP; ++j)
            if (j < G)
                partials[(int64_t)(g * G + j) * stride + slot_base + slot] = make_float2(m[j], z[j]);
    }
}

template <int D, int GP>
__global__ void __launch_bounds__(kScoreThreads, 1)
score_pass_a(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ ScoreArgs a)
{
    extern __shared__ uint8_t dyn_smem[];
    __shared__ ScoreShared sh;
    uint8_t *stages = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    const int NS = a.nstages;
    uint8_t *qs = stages + (size_t)NS * a.stage_bytes;      // 1024-byte aligned: stages are multiples of 16 KB

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = a.B;
    const int T = a.T;
    const int Hkv = a.Hkv;
    const int N = score_mma_n<GP>(Hkv);

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int s = 0; s < kScoreAccBufs; ++s) {
            mbar_init(&sh.acc_full[s], 1);
            mbar_init(&sh.acc_empty[s], kScoreEpiWarps / 2);   // the four warps of that stage parity
        }
        mbar_init(&sh.mma_done, 1);
        mbar_fence_init();
    }
    if (warp == kMmaWarp)
        tmem_alloc(&sh.tmem_base, a.tmem_cols);
    // ---- before the previous kernel has finished: only L2 prefetch hints,
    //      computed as if every sequence were active (a wrong guess costs
    //      nothing but bandwidth; the data itself is read after the wait) -----
    const int npf = NS < kMaxPrefetchTiles ? NS : kMaxPrefetchTiles;
    if (a.page_table != nullptr) {
        // a paged cache: no host copy of the block table, so no early hints
        if (warp == kProducerWarp && lane == 0)
            tma_prefetch_desc(&kmap);
    } else if (B <= 32) {
        if (warp == kProducerWarp) {
            if (lane == 0)
                tma_prefetch_desc(&kmap);
            // all-active chunk table from the host offsets (kernel parameters:
            // no memory round trip before the wait)
            int32_t x = 0;
            int64_t o0 = 0;
            if (lane < B) {
                o0 = a.pf_off[lane];
                const int64_t n = a.pf_off[lane + 1] - o0;
                x = n > 0 ? (int32_t)((n + T - 1) / T) : 0;
            }
            int32_t c1 = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, c1, o);
                if (lane >= o)
                    c1 += y;
            }
            const int32_t c0 = c1 - x;
            if (lane < B) {
                sh.pf_start[lane] = c0;
                sh.pf_off[lane] = o0;
            }
            const int32_t total = __shfl_sync(0xffffffffu, c1, B - 1);
            __syncwarp();
            if (lane == 0) {
                const bool il = B == 1;
                const int32_t v0 = il ? (int32_t)blockIdx.x : chunk_split(blockIdx.x, total, gridDim.x);
                const int32_t v1 = il ? total : chunk_split(blockIdx.x + 1, total, gridDim.x);
                const int32_t vs = il ? (int32_t)gridDim.x : 1;
                int b = 0;
                for (int32_t v = v0; v < v1 && v < v0 + npf * vs; v += vs) {
                    while (b + 1 < B && sh.pf_start[b + 1] <= v)
                        ++b;
                    const int64_t t0 = sh.pf_off[b] + (int64_t)(v - sh.pf_start[b]) * T;
#pragma unroll
                    for (int x = 0; x < D / 64; ++x)
                        tma_prefetch_l2_3d(&kmap, x * 64, (int32_t)t0, 0);
                }
            }
        }
    } else {
        for (int b = tid; b <= B; b += blockDim.x)
            sh.off[b] = __ldcg(a.seq_off + b);
        __syncthreads();
        build_chunk_table(sh, a.reuse, B, T, warp, lane, false);
        if (warp == kProducerWarp && lane == 0) {
            tma_prefetch_desc(&kmap);
            const int32_t total = sh.chunk_start[B];
            const int32_t v0 = chunk_split(blockIdx.x, total, gridDim.x);
            const int32_t v1 = chunk_split(blockIdx.x + 1, total, gridDim.x);
            for (int32_t v = v0; v < v1 && v < v0 + npf; ++v) {
                const int b = upper_seq(sh.chunk_start, B, v);
                const int64_t t0 = sh.off[b] + (int64_t)(v - sh.chunk_start[b]) * T;
#pragma unroll
                for (int x = 0; x < D / 64; ++x)
                    tma_prefetch_l2_3d(&kmap, x * 64, (int32_t)t0, 0);
            }
        }
    }
    pdl_wait();
    pdl_launch_dependents();

    // ---- the real chunk table (reuse flags come from the previous kernel);
    //      the offsets are re-read too, in case a caller's kernel wrote them;
    //      offsets and flags are loaded together: one round trip -------------
    tmem_fence_before();
    if (B <= 32) {
        if (warp == 0) {
            int32_t c0, c1;
            int64_t o0, o1;
            warp_chunk_scan(a.seq_off, a.reuse, B, T, lane, c0, c1, o0, o1);
            if (lane < B) {
                sh.chunk_start[lane] = c0;
                sh.off[lane] = o0;
            }
            if (lane == B - 1) {
                sh.chunk_start[B] = c1;
                sh.off[B] = o1;
            }
        }
        __syncthreads();
    } else {
        __syncthreads();
        for (int b = tid; b < B; b += blockDim.x) {
            const int64_t o0 = __ldcg(a.seq_off + b), o1 = __ldcg(a.seq_off + b + 1);
            const bool active = a.reuse == nullptr || __ldcg(a.reuse + b) == 0;
            sh.off[b] = o0;
            if (b == B - 1)
                sh.off[B] = o1;
            const int64_t n = o1 - o0;
            sh.chunk_start[b + 1] = (active && n > 0) ? (int32_t)((n + T - 1) / T) : 0;
        }
        __syncthreads();
        if (warp == 0) {
            int32_t run = 0;
            for (int base = 0; base < B; base += 32) {
                const int b = base + lane;
                int32_t x = (b < B) ? sh.chunk_start[b + 1] : 0;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o)
                        x += y;
                }
                if (b < B)
                    sh.chunk_start[b + 1] = run + x;
                run += __shfl_sync(0xffffffffu, x, 31);
            }
            if (lane == 0)
                sh.chunk_start[0] = 0;
        }
        __syncthreads();
    }
    tmem_fence_after();
    if (blockIdx.x == 0)
        for (int b = tid; b <= B; b += blockDim.x)
            a.chunk_table[b] = sh.chunk_start[b];
    const int32_t total = sh.chunk_start[B];
    // chunks of this CTA: v_begin, v_begin + v_step, ... < v_end.  A single
    // sequence is dealt round-robin (CTA j: j, j + grid, ...), so every SM
    // reads from every part of the cache; several sequences keep contiguous
    // ranges [j*C/grid, (j+1)*C/grid) (one segment per CTA and sequence).
    const bool interleave = B == 1;
    const int32_t v_begin = interleave ? (int32_t)blockIdx.x : chunk_split(blockIdx.x, total, gridDim.x);
    const int32_t v_end = interleave ? total : chunk_split(blockIdx.x + 1, total, gridDim.x);
    const int32_t v_step = interleave ? (int32_t)gridDim.x : 1;
    const uint32_t tmem = sh.tmem_base;
    const int half_bytes = kScoreRows * 128;   // one 64-channel box

    if (warp == kProducerWarp) {
        // ================= TMA producer ====================================
        // The whole warp walks the chunks.  A warp-wide lookup finds the K
        // row of every page of the next 32 / npp chunks, one page per lane
        // (the block table of a paged cache costs one round trip per
        // lookup), and lane 0 issues the loads.  npp = 1 unless a paged
        // cache's pages are shorter than a chunk; then each page of the chunk
        // arrives as one box {64, page, h_kv} (the epilogue reads the rows
        // page by page), or, for 8-token pages, as one box {64, 8, 1} per kv
        // head placed where the chunk's single box {64, T, h_kv} would have
        // put those rows.
        const uint64_t pol = l2_policy_evict_first();
        const int BT = a.box_tokens;                     // tokens of one box
        const int npp = T / BT;                          // boxes along the tokens of a chunk (power of 2, <= 16)
        const int cpb = 32 / npp;                        // chunks per lookup
        const int64_t oob_row = a.pool_pages << a.page_shift;   // past the pool: reads zeros
        uint32_t it = 0;
        int32_t my_row = 0;
        bool stop = false;
        for (int32_t v = v_begin; v < v_end && !stop; v += v_step, ++it) {
            const int jb = (int)(it % (uint32_t)cpb);
            if (jb == 0) {
                const int32_t vl = v + (lane / npp) * v_step;
                const int p = lane % npp;
                my_row = 0;
                if (vl < v_end) {
                    const int bl = upper_seq(sh.chunk_start, B, vl);
                    // first token of this lane's box in its sequence
                    const int64_t i0 = (int64_t)(vl - sh.chunk_start[bl]) * T + (int64_t)p * BT;
                    if (a.page_table == nullptr) {
                        my_row = (int32_t)(sh.off[bl] + i0);
                    } else if (i0 >= sh.off[bl + 1] - sh.off[bl]) {
                        my_row = (int32_t)oob_row;       // a page past the sequence's end: never looked up
                    } else {
                        // a box lies in one page (BT = min(T, page), both powers of two); an
                        // entry outside the pool reads past the pool's rows: zero keys
                        const int32_t pg = __ldcg(a.page_table + (int64_t)bl * a.pt_stride + (i0 >> a.page_shift));
                        my_row = (pg >= 0 && pg < a.pool_pages)
                                     ? (int32_t)(((int64_t)pg << a.page_shift) + (i0 & ((1 << a.page_shift) - 1)))
                                     : (int32_t)oob_row;
                    }
                }
            }
            const int s = it % NS;
            bool ok = true;
            if (lane == 0) {
                if (it >= (uint32_t)NS) {
                    const uint32_t par = ((it / NS) - 1) & 1;
                    if (!mbar_wait_bounded(&sh.empty[s], par, kSpinLimit)) {
                        report_timeout(a.ctrl, kSiteScoreEmpty);
                        // nothing is issued after this (the MMA warp times out
                        // on full[] too); before leaving, wait (bounded) for the
                        // tiles already in flight: the last NS issued stages
                        for (uint32_t j = it > (uint32_t)NS ? it - NS : 0u; j < it; ++j)
                            (void)mbar_wait_bounded(&sh.full[j % NS], (j / NS) & 1, kSpinLimit);
                        ok = false;
                    }
                }
                if (ok)
                    mbar_arrive_expect_tx(&sh.full[s], (uint32_t)a.stage_bytes);
            }
            stop = !__shfl_sync(0xffffffffu, ok ? 1 : 0, 0);
            if (stop)
                break;
            uint8_t *dst = stages + (size_t)s * a.stage_bytes;
            for (int p = 0; p < npp; ++p) {
                const int32_t row = __shfl_sync(0xffffffffu, my_row, jb * npp + p);
                if (lane == 0) {
                    if (a.box_heads == a.Hkv) {
#pragma unroll
                        for (int x = 0; x < D / 64; ++x)
                            tma_load_3d(dst + x * half_bytes + p * a.Hkv * BT * 128, &kmap, &sh.full[s], x * 64, row,
                                        0, pol);
                    } else {
#pragma unroll
                        for (int x = 0; x < D / 64; ++x)
                            for (int g = 0; g < a.Hkv; ++g)
                                tma_load_3d(dst + x * half_bytes + (g * T + p * BT) * 128, &kmap, &sh.full[s],
                                            x * 64, row, g, pol);
                    }
                }
            }
        }
        return;   // takes no part in the final barrier
    }

    if (warp == kMmaWarp) {
        // ================= tensor cores: queries, MMA chain ===============
        constexpr uint32_t kIdescM = 128;
        const uint32_t idesc = umma_idesc_bf16_f32(kIdescM, N);
        int cur_b = -1;
        bool dead = false;
        uint32_t done_par = 0;
        uint32_t it = 0;
        for (int32_t v = v_begin; v < v_end && !dead; v += v_step, ++it) {
            const int b = upper_seq(sh.chunk_start, B, v);
            if (b != cur_b) {
                if (cur_b >= 0) {   // the old queries may still be read by MMAs in flight
                    if (lane == 0)
                        umma_commit(&sh.mma_done);
                    __syncwarp();
                    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&sh.mma_done, done_par, kSpinLimit));
                    done_par ^= 1u;
                    if (!ok) {
                        if (lane == 0)
                            report_timeout(a.ctrl, kSiteScoreMma);
                        dead = true;
                        break;
                    }
                }
                stage_queries<D, GP>(qs, a.q + (int64_t)b * a.Hq * D, a.G, Hkv, lane);
                fence_proxy_async_smem();
                __syncwarp();
                cur_b = b;
            }
            const int s = it % NS;
            const uint32_t par = (it / NS) & 1;
            const int buf = it % kScoreAccBufs;
            bool ok = true;
            if (lane == 0) {
                ok = mbar_wait_bounded(&sh.full[s], par, kSpinLimit);
                if (ok && it >= (uint32_t)kScoreAccBufs)
                    ok = mbar_wait_bounded(&sh.acc_empty[buf], ((it / kScoreAccBufs) - 1) & 1, kSpinLimit);
                if (ok) {
                    tmem_fence_after();
                    const uint32_t a_base = smem_u32(stages + (size_t)s * a.stage_bytes);
                    const uint32_t b_base = smem_u32(qs);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t koff = (uint32_t)((ks & 3) * 32);
                        const uint64_t ad = umma_desc_sw128(a_base + (uint32_t)((ks >> 2) * half_bytes) + koff);
                        const uint64_t bd = umma_desc_sw128(b_base + (uint32_t)((ks >> 2) * N * 128) + koff);
                        umma_bf16(tmem + (uint32_t)(buf * N), ad, bd, idesc, ks > 0);
                    }
                    umma_commit(&sh.empty[s]);        // the ring slot is free once these MMAs have read it
                    umma_commit(&sh.acc_full[buf]);   // the accumulator is ready for the epilogue
                } else {
                    report_timeout(a.ctrl, kSiteScoreMma);
                }
            }
            dead = !__shfl_sync(0xffffffffu, ok ? 1 : 0, 0);
            __syncwarp();
        }
        // every MMA this warp issued has completed before TMEM is released
        if (it > 0) {
            if (lane == 0)
                umma_commit(&sh.mma_done);
            __syncwarp();
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&sh.mma_done, done_par, kSpinLimit))) {
                if (lane == 0)
                    report_timeout(a.ctrl, kSiteScoreMma);
                // one more bounded wait before TMEM is released under MMAs
                // that may still be running (the step's results are void)
                (void)mbar_wait_bounded(&sh.mma_done, done_par, kSpinLimit);
            }
        }
    } else {
        // ================= epilogue: warps 0-3, one TMEM lane each =========
        const int quarter = warp & 3, hs = warp >> 2;
        // Row r of a stage holds kv head g, token t of the chunk.  The rows
        // come in blocks of EBT tokens of one head, the h_kv blocks of a
        // page side by side, then the next page: EBT = T (one block per
        // head) unless a paged cache's pages are shorter than T and were
        // loaded as one box of every kv head per page.
        const int EBT = a.box_heads > 1 ? a.box_tokens : T;
        const int PB = a.Hkv * EBT;                // rows of one page of blocks
        const int r = quarter * 32 + lane;         // accumulator row
        const int g = (r % PB) / EBT;              // kv head
        const int t = (r / PB) * EBT + r % EBT;    // token within the chunk
        const int g_lo = ((quarter * 32) % PB) / EBT;   // first kv head of this warp's rows
        const int span = EBT < 32 ? EBT : 32;      // lanes of this warp with the same head
        // this warp's partial slot for head g: the two stage parities x the
        // span-token pieces of the chunk (the piece of this warp's first row
        // of head g)
        const int slot = hs * (T / span) + ((r - lane % span) / PB * EBT + (r - lane % span) % EBT) / span;
        const int G = a.G;
        const float scale = a.scale;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        float m[GP], z[GP];
        int cur_b = -1;
        bool dead = false;
        uint32_t it = 0;

        auto flush_segment = [&]() {
            score_flush<GP>(m, z, G, span, lane, slot, g, a.partials, (int64_t)a.S * a.R,
                            ((int64_t)blockIdx.x + cur_b) * a.R);
        };

        for (int32_t v = v_begin; v < v_end; v += v_step, ++it) {
            const int b = upper_seq(sh.chunk_start, B, v);
            if (b != cur_b) {
                if (cur_b >= 0)
                    flush_segment();
                cur_b = b;
#pragma unroll
                for (int j = 0; j < GP; ++j) {
                    m[j] = -INFINITY;
                    z[j] = 0.0f;
                }
            }
            if (dead || (int)(it & 1u) != hs)
                continue;                          // the other warp of this lane quarter takes it
            const int buf = it % kScoreAccBufs;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&sh.acc_full[buf], (it / kScoreAccBufs) & 1, kSpinLimit))) {
                if (lane == 0)
                    report_timeout(a.ctrl, kSiteScoreAcc);
                dead = true;
                continue;
            }
            tmem_fence_after();
            uint32_t raw[GP], raw2[GP];
            const uint32_t taddr = lane_base + (uint32_t)(buf * N + g_lo * GP);
            tmem_ld_32x32b<GP>(taddr, raw);
            if (span < 32)
                tmem_ld_32x32b<GP>(taddr + GP, raw2);   // two heads per lane quarter
            tmem_wait_ld();
            tmem_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&sh.acc_empty[buf]);
            const bool second = g != g_lo;           // only with two heads per lane quarter
            const int64_t tok = sh.off[b] + (int64_t)(v - sh.chunk_start[b]) * T + t;
            if (tok < sh.off[b + 1]) {
#pragma unroll
                for (int j = 0; j < GP; ++j) {
                    if (j < G) {
                        const float x = __uint_as_float(second ? raw2[j] : raw[j]) * scale;
                        a.logits[(int64_t)(g * G + j) * a.ld + tok] = x;
                        online_push(m[j], z[j], x);
                    }
                }
            }
        }
        if (cur_b >= 0)
            flush_segment();
    }
    // epilogue and MMA warps: every accumulator has been read and every MMA
    // has completed before the MMA warp frees TMEM
    tmem_fence_before();
    named_bar_sync(2, (kScoreEpiWarps + 1) * 32);
    tmem_fence_after();
    if (warp == kMmaWarp)
        tmem_dealloc(tmem, a.tmem_cols);
}

// L[b, h] from the partials of sequence b (one warp per sequence and head).
// CTA j of pass A covers chunks [j*total/grid, (j+1)*total/grid); the CTAs
// that cover the sequence's chunks [cs, ce) are j0 = owner(cs) ..
// j1 = owner(ce-1), owner(v) = ((v+1)*grid - 1) / total, and CTA j wrote the
// R partials of its segment at slot j + b.  The table entries and every
// partial the sequence could own are loaded together (one round trip);
// entries of CTAs outside j0..j1, or without chunks, are dropped.  fp32
// terms exp(m - M) <= 1 summed in float64 in a fixed order.
template <int R>
__global__ void __launch_bounds__(32)
score_merge(const float2 *partials, int S, const int32_t *chunk_table, double *L, int B, int Hq, int grid_a)
{
    pdl_wait();
    pdl_launch_dependents();
    const int h = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x;
    constexpr int kPer = 8 * R;   // grid_a * R <= 256 * R entries over 32 lanes
    const int n = grid_a * R;
    const int32_t cs = __ldcg(chunk_table + b), ce = __ldcg(chunk_table + b + 1), total = __ldcg(chunk_table + B);
    const float2 *row = partials + ((int64_t)h * S + b) * R;
    float2 pv[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        pv[i] = e < n ? __ldcg(row + e) : make_float2(-INFINITY, 0.0f);
    }
    if (cs == ce)
        return;   // reused or empty sequence: its L is not needed
    const int j0 = (int)(((int64_t)(cs + 1) * grid_a - 1) / total);
    const int j1 = (int)(((int64_t)ce * grid_a - 1) / total);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        const int j = e / R;   // R is a power of 2: a shift
        bool keep;
        if (B == 1) {   // round-robin chunks: CTA j has some iff j < total
            keep = e < n && j < total;
        } else {
            keep = e < n && j >= j0 && j <= j1;
            if (keep && total < grid_a)   // some CTAs had no chunks and wrote nothing
                keep = chunk_split(j, total, grid_a) < chunk_split(j + 1, total, grid_a);
        }
        if (!keep)
            pv[i] = make_float2(-INFINITY, 0.0f);
    }
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
        M = fmaxf(M, pv[i].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    double Z = 0.0;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
        if (pv[i].y > 0.0f)
            Z += (double)(pv[i].y * exp2f((pv[i].x - M) * kLog2e));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        Z += __shfl_xor_sync(0xffffffffu, Z, o);
    if (lane == 0)
        L[(int64_t)b * Hq + h] = (double)M + log(Z);
}

template <int D, int GP>
cudaError_t launch_score_t(const Plan &p, const CUtensorMap &kmap, ScoreArgs args, cudaStream_t st)
{
    const int N = score_mma_n<GP>(p.Hkv);
    const size_t q_bytes = (size_t)N * D * 2;
    int ns = (int)((kScoreDynSmemBudget - q_bytes) / (size_t)p.stage_bytes);
    ns = ns < kScoreMaxStages ? ns : kScoreMaxStages;
    args.nstages = ns;
    uint32_t cols = 32;
    while (cols < (uint32_t)(kScoreAccBufs * N))
        cols <<= 1;
    args.tmem_cols = cols;
    const size_t dyn = (size_t)ns * p.stage_bytes + q_bytes + 1024;
    cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void *>(score_pass_a<D, GP>),
                                    (int)(kScoreDynSmemBudget + 1024));
    if (e != cudaSuccess)
        return e;
    return launch_ex(score_pass_a<D, GP>, dim3((unsigned)p.score_grid), dim3(kScoreThreads), dyn, st, 1, kmap,
                     args);
}

}  // namespace

cudaError_t launch_score(const Plan &p, const CUtensorMap &kmap, const void *q, const int64_t *seq_off,
                         const int64_t *seq_off_host, const int32_t *reuse, uint8_t *ws, cudaStream_t st,
                         const int32_t *page_table, int page_table_stride, double *L_out)
{
    ScoreArgs a;
    for (int b = 0; b <= 32; ++b)
        a.pf_off[b] = (p.B <= 32 && b <= p.B) ? seq_off_host[b] : 0;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.seq_off = seq_off;
    a.reuse = reuse;
    a.logits = reinterpret_cast<float *>(ws + p.off_logits);
    a.ld = p.ld_logits;
    a.partials = reinterpret_cast<float2 *>(ws + p.off_partials);
    a.S = p.score_grid + p.B;
    a.R = p.score_partials_per_slot;
    a.chunk_table = reinterpret_cast<int32_t *>(ws + p.off_chunk_table);
    a.ctrl = reinterpret_cast<uint32_t *>(ws + p.off_ctrl);
    a.B = p.B;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.T = p.tile_tokens;
    a.stage_bytes = p.stage_bytes;
    a.scale = p.scale;
    a.page_table = p.paged ? page_table : nullptr;
    a.pt_stride = p.paged ? page_table_stride : 0;
    a.page_shift = p.page_shift;
    a.pool_pages = p.paged ? p.kv_rows >> p.page_shift : 0;
    a.box_tokens = p.box_tokens;
    a.box_heads = p.box_heads;
    cudaError_t e;
    // GP: columns per kv head in the MMA's N (the smallest of 4, 8, 16 that
    // holds the group); a small N keeps the query tile small and leaves
    // shared memory to the K ring
    if (p.D == 128)
        e = p.G <= 4 ? launch_score_t<128, 4>(p, kmap, a, st)
                     : (p.G <= 8 ? launch_score_t<128, 8>(p, kmap, a, st) : launch_score_t<128, 16>(p, kmap, a, st));
    else
        e = p.G <= 4 ? launch_score_t<64, 4>(p, kmap, a, st)
                     : (p.G <= 8 ? launch_score_t<64, 8>(p, kmap, a, st) : launch_score_t<64, 16>(p, kmap, a, st));
    if (e != cudaSuccess)
        return e;
    const float2 *parts = reinterpret_cast<const float2 *>(ws + p.off_partials);
    const int32_t *table = reinterpret_cast<const int32_t *>(ws + p.off_chunk_table);
    double *Lp = L_out != nullptr ? L_out : reinterpret_cast<double *>(ws + p.off_L);
    const dim3 mgrid((unsigned)p.Hq, (unsigned)p.B);
    const int S = p.score_grid + p.B;
    switch (p.score_partials_per_slot) {
    case 2:
        return launch_ex(score_merge<2>, mgrid, dim3(32), 0, st, 1, parts, S, table, Lp, p.B, p.Hq, p.score_grid);
    case 4:
        return launch_ex(score_merge<4>, mgrid, dim3(32), 0, st, 1, parts, S, table, Lp, p.B, p.Hq, p.score_grid);
    default:
        return launch_ex(score_merge<8>, mgrid, dim3(32), 0, st, 1, parts, S, table, Lp, p.B, p.Hq, p.score_grid);
    }
}

}  // namespace ts
