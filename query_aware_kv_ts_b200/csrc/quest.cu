// Page-level comparator after Quest (Bohrium page for "Quest: Query-Aware
// Sparsity for Efficient Long-Context LLM Inference", arXiv 2406.10774:
// Abstract; Method Overview, item 4): each page of P tokens keeps the
// element-wise minimum and maximum of its keys; a query bounds every key of
// the page from above through those two vectors; the Top-K pages by that
// bound are attended.  Here one selection serves all heads of a sequence,
// so a page's score is the per-head bound summed over the query heads, and
// the chosen pages' tokens join the sink and local windows of the
// token-level selection, in the same id rows that ts_sparse_attn reads.
//
// Layout: page j of sequence b (tokens [j*P, min((j+1)*P, n_b))) has row
// (seq_offsets[b] >> log2 P) + b + j of the metadata and of the scores;
// every kernel finds it from the offsets alone (no prefix sum), at the cost
// of at most one unused row per sequence.
//
// All three kernels move little data per unit of work and are HBM- or
// latency-bound, so they run on the CUDA cores: the metadata pass reads K
// once (one warp per page, 16-byte loads, bf16x2 min / max); the score pass
// reads the metadata once and folds the sum over heads into one dot product
// per page (below); the selection is one CTA per sequence doing a radix
// select over the pages' order keys.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "score_common.cuh"
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {

namespace {

constexpr int kQuestWarps = 8;              // pages handled together by one CTA of the metadata / score passes
constexpr int kQuestSelThreads = 1024;      // one CTA per sequence
constexpr int kQuestSelBins = 2048;         // radix digits of 11, 11 and 10 bits

struct QuestKV {
    const __nv_bfloat16 *k;
    const int64_t *seq_off;      // device offsets [B+1]
    int64_t st, sh;              // token and head strides (elements)
    const int32_t *page_table;   // paged KV cache: block table [B][pt_stride], else null
    int pt_stride, kv_page_shift;
    int64_t pool_pages;
    int Hkv, D;
    int P_shift;                 // log2 of the comparator's page size
};

// K row of token i of sequence b, or -1 when a paged cache's entry lies
// outside the pool.
__device__ __forceinline__ int64_t token_row(const QuestKV &a, int b, int64_t off0, int64_t i)
{
    if (a.page_table == nullptr)
        return off0 + i;
    const int32_t pg = __ldg(a.page_table + (int64_t)b * a.pt_stride + (i >> a.kv_page_shift));
    if (pg < 0 || pg >= a.pool_pages)
        return -1;
    return ((int64_t)pg << a.kv_page_shift) + (i & ((int64_t(1) << a.kv_page_shift) - 1));
}

__device__ __forceinline__ uint4 bf16x8_min(uint4 x, uint4 y)
{
    uint4 r;
    const __nv_bfloat162 *a = reinterpret_cast<const __nv_bfloat162 *>(&x);
    const __nv_bfloat162 *c = reinterpret_cast<const __nv_bfloat162 *>(&y);
    __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(&r);
#pragma unroll
    for (int e = 0; e < 4; ++e)
        o[e] = __hmin2(a[e], c[e]);
    return r;
}

__device__ __forceinline__ uint4 bf16x8_max(uint4 x, uint4 y)
{
    uint4 r;
    const __nv_bfloat162 *a = reinterpret_cast<const __nv_bfloat162 *>(&x);
    const __nv_bfloat162 *c = reinterpret_cast<const __nv_bfloat162 *>(&y);
    __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(&r);
#pragma unroll
    for (int e = 0; e < 4; ++e)
        o[e] = __hmax2(a[e], c[e]);
    return r;
}

// ---------------------------------------------------------------------------
// Page metadata: one warp per page.  Lane l owns the 16-byte chunks l,
// l + 32, ... (CH of them) of the h_kv * d channels of a token row; the
// warp's lanes look up the rows of 32 tokens at a time and walk them, U
// tokens' loads in flight.  last_tokens > 0: only the pages holding one of
// the sequence's last last_tokens tokens (its current length read here, so
// that the update follows appends made on the device), each recomputed
// from all its tokens.
// ---------------------------------------------------------------------------
template <int CH>
__global__ void __launch_bounds__(kQuestWarps * 32)
quest_meta(const QuestKV a, __nv_bfloat16 *kmin, __nv_bfloat16 *kmax, int64_t last_tokens)
{
    constexpr int U = 8 / CH;
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t off0 = a.seq_off[b];
    const int64_t n = a.seq_off[b + 1] - off0;
    const int64_t j_first = last_tokens > 0 ? max((int64_t)0, n - last_tokens) >> a.P_shift : 0;
    const int64_t j = j_first + (int64_t)blockIdx.x * kQuestWarps + warp;   // page of the sequence
    const int64_t t0 = j << a.P_shift;
    if (t0 >= n)
        return;
    const int64_t t1 = min(t0 + (int64_t(1) << a.P_shift), n);
    const int E8 = (a.Hkv * a.D) >> 3;                             // 16-byte chunks per token row
    int64_t coff[CH];
    bool cval[CH];
    uint4 lo[CH], hi[CH];
#pragma unroll
    for (int x = 0; x < CH; ++x) {
        const int q = lane + 32 * x;
        cval[x] = q < E8;
        const int e = (q << 3) % (a.Hkv * a.D);
        coff[x] = (int64_t)(e / a.D) * a.sh + (e % a.D);
        lo[x] = make_uint4(0x7f807f80u, 0x7f807f80u, 0x7f807f80u, 0x7f807f80u);   // +inf
        hi[x] = make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);   // -inf
    }
    for (int64_t tb = t0; tb < t1; tb += 32) {
        const int cnt = (int)min((int64_t)32, t1 - tb);
        const int64_t my_row = lane < cnt ? token_row(a, b, off0, tb + lane) : -1;
        for (int i = 0; i < cnt; i += U) {
            uint4 v[U][CH];
            bool ok[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t row = __shfl_sync(0xffffffffu, my_row, (i + u) & 31);
                ok[u] = i + u < cnt && row >= 0;
#pragma unroll
                for (int x = 0; x < CH; ++x)
                    if (ok[u] && cval[x])
                        v[u][x] = __ldcs(reinterpret_cast<const uint4 *>(a.k + row * a.st + coff[x]));
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int x = 0; x < CH; ++x)
                    if (ok[u] && cval[x]) {
                        lo[x] = bf16x8_min(lo[x], v[u][x]);
                        hi[x] = bf16x8_max(hi[x], v[u][x]);
                    }
        }
    }
    const int64_t out = (((a.seq_off[b] >> a.P_shift) + b + j) * (int64_t)(a.Hkv * a.D));
#pragma unroll
    for (int x = 0; x < CH; ++x)
        if (cval[x]) {
            const int q = lane + 32 * x;
            *reinterpret_cast<uint4 *>(kmin + out + q * 8) = lo[x];
            *reinterpret_cast<uint4 *>(kmax + out + q * 8) = hi[x];
        }
}

// ---------------------------------------------------------------------------
// Page scores.  For query head h of kv head g the bound of the page is
//   scale * sum_c max(q_h[c] kmin[g][c], q_h[c] kmax[g][c])
//     = scale * sum_c (max(q_h[c], 0) kmax[g][c] + min(q_h[c], 0) kmin[g][c]),
// so the sum over the G heads of group g is one dot product of the page's
// [kmax | kmin] row with the sequence's weights
//   A[g][c] = scale * sum_h max(q_h[c], 0),  Bw[g][c] = scale * sum_h min(q_h[c], 0)
// (fp32), which each lane keeps for its own channels.  One warp per U pages
// (U pages' loads in flight), a shuffle sum per page.
// ---------------------------------------------------------------------------
template <int CH>
__global__ void __launch_bounds__(kQuestWarps * 32)
quest_score(const int64_t *seq_off, const __nv_bfloat16 *q, const __nv_bfloat16 *kmin, const __nv_bfloat16 *kmax,
            float *scores, int Hq, int Hkv, int D, int P_shift, float scale)
{
    constexpr int U = 4 / CH > 0 ? 4 / CH : 1;   // pages per batch: 8 16-byte loads per lane
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t off0 = seq_off[b];
    const int64_t n = seq_off[b + 1] - off0;
    const int64_t pages = (n + (int64_t(1) << P_shift) - 1) >> P_shift;
    const int64_t wid = (int64_t)blockIdx.x * kQuestWarps + warp;
    const int64_t wstride = (int64_t)gridDim.x * kQuestWarps * U;
    if (wid * U >= pages)
        return;
    const int E = Hkv * D, E8 = E >> 3, G = Hq / Hkv;
    float wA[CH][8], wB[CH][8];
#pragma unroll
    for (int x = 0; x < CH; ++x) {
        const int qc = lane + 32 * x;
#pragma unroll
        for (int e = 0; e < 8; ++e)
            wA[x][e] = wB[x][e] = 0.0f;
        if (qc < E8) {
            const int g = (qc * 8) / D, c = (qc * 8) % D;
            for (int jh = 0; jh < G; ++jh) {
                const uint4 qv = __ldg(reinterpret_cast<const uint4 *>(q + ((int64_t)b * Hq + g * G + jh) * D + c));
                const __nv_bfloat16 *qe = reinterpret_cast<const __nv_bfloat16 *>(&qv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float f = __bfloat162float(qe[e]);
                    wA[x][e] += fmaxf(f, 0.0f);
                    wB[x][e] += fminf(f, 0.0f);
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                wA[x][e] *= scale;
                wB[x][e] *= scale;
            }
        }
    }
    const int64_t row0 = (off0 >> P_shift) + b;
    uint4 mn[U][CH], mx[U][CH];
    auto load = [&](int64_t j0) {
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int x = 0; x < CH; ++x) {
                const int qc = lane + 32 * x;
                if (j0 + u < pages && qc < E8) {
                    const int64_t o = (row0 + j0 + u) * E + qc * 8;
                    mn[u][x] = __ldcs(reinterpret_cast<const uint4 *>(kmin + o));
                    mx[u][x] = __ldcs(reinterpret_cast<const uint4 *>(kmax + o));
                }
            }
    };
    int64_t j0 = wid * U;
    load(j0);
    while (j0 < pages) {
        // the batch's dot products, then the next batch's loads go out
        // before the shuffle sums and the stores
        float acc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            acc[u] = 0.0f;
#pragma unroll
            for (int x = 0; x < CH; ++x) {
                const int qc = lane + 32 * x;
                if (j0 + u < pages && qc < E8) {
                    const __nv_bfloat16 *lo = reinterpret_cast<const __nv_bfloat16 *>(&mn[u][x]);
                    const __nv_bfloat16 *hi = reinterpret_cast<const __nv_bfloat16 *>(&mx[u][x]);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        acc[u] = fmaf(wA[x][e], __bfloat162float(hi[e]), acc[u]);
                        acc[u] = fmaf(wB[x][e], __bfloat162float(lo[e]), acc[u]);
                    }
                }
            }
        }
        const int64_t jn = j0 + wstride;
        if (jn < pages)
            load(jn);
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
            if (lane == 0 && j0 + u < pages)
                scores[row0 + j0 + u] = acc[u];
        }
        j0 = jn;
    }
}

// ---------------------------------------------------------------------------
// Page selection: one CTA per sequence.
// ---------------------------------------------------------------------------

// Exclusive prefix sum of one value per thread over the CTA (thread order);
// returns the thread's prefix and leaves the total in *total.
__device__ __forceinline__ uint32_t cta_exclusive_scan(uint32_t v, uint32_t *warp_sums, uint32_t *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o)
            x += y;
    }
    if (lane == 31)
        warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < nw ? warp_sums[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o)
                s += y;
        }
        warp_sums[lane] = s;   // inclusive over warps
    }
    __syncthreads();
    const uint32_t before = (warp > 0 ? warp_sums[warp - 1] : 0u) + x - v;
    *total = warp_sums[nw - 1];
    __syncthreads();           // warp_sums is reused by the next scan
    return before;
}

// Ascending unsigned key of a score: larger score, larger key; -0 and +0
// are the same score (equal scores go to the lower page).
__device__ __forceinline__ uint32_t score_key(float s)
{
    return (uint32_t)float_order_key(s == 0.0f ? 0.0f : s) ^ 0x80000000u;
}

// Calls f(c, key) for this thread's candidates c = tid, tid + blockDim.x, ...
// < nc, with kQSelBatch loads in flight.
constexpr int kQSelBatch = 8;
template <typename F>
__device__ __forceinline__ void for_each_key(const float *sc, int64_t nc, F f)
{
    for (int64_t c0 = threadIdx.x; c0 < nc; c0 += (int64_t)kQSelBatch * blockDim.x) {
        float v[kQSelBatch];
#pragma unroll
        for (int u = 0; u < kQSelBatch; ++u) {
            const int64_t c = c0 + (int64_t)u * blockDim.x;
            v[u] = c < nc ? __ldcg(sc + c) : 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kQSelBatch; ++u) {
            const int64_t c = c0 + (int64_t)u * blockDim.x;
            if (c < nc)
                f(c, score_key(v[u]));
        }
    }
}

// The page selection, one cluster of kQSelCluster CTAs of 1024 threads per
// sequence.  Candidate pages [jlo, jlo + nc) are those holding a token of
// [s_end, l0); `take` of them are chosen.
//
// Fast path (at most 2048 pages to choose, the usual case): each CTA of the
// cluster takes an equal slice of the candidates.  Their keys' min and max
// (combined through distributed shared memory) span 2048 equal bins (equal
// bins in key space spread a concentrated score distribution over many
// bins, so the histograms' shared atomics rarely collide); the slices'
// histograms are summed by rank 0, which finds the threshold bin; each CTA
// then appends its sure winners (a higher bin) and its threshold-bin pages
// to rank 0's shared memory, where rank 0 decides the rest by counting ranks:
// the bucket's pages by (key desc, page asc), the chosen pages by page for
// their token positions.  Three coalesced passes over the scores, spread
// over the cluster's SMs (one SM's issue rate bounded a single-CTA version).
// General path (more than 2048 pages to choose, or more than 2048 tied in
// the threshold bin): rank 0 alone runs a three-digit radix select over all
// 32 key bits and two passes in page order over a contiguous range per
// thread.  Every cross-CTA access lies between cluster barriers, and no CTA
// leaves while another may still read its shared memory.
constexpr int kQSelCluster = 8;
constexpr int kQSelList = 2048;     // chosen pages the fast path holds
constexpr int kQSelBucket = 2048;   // pages of the threshold bin it holds

__global__ void __launch_bounds__(kQuestSelThreads)
quest_select(const float *scores, const int64_t *seq_off, int P_shift, int k, int n_sink, int n_local, int cap,
             int32_t *ids, int32_t *count)
{
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    const int C = (int)cl.num_blocks(), rank = (int)cl.block_rank();
    __shared__ uint32_t hist[kQuestSelBins];
    __shared__ uint32_t warp_sums[32];
    __shared__ uint32_t warp_lo[32], warp_hi[32];
    __shared__ uint32_t s_kmin, s_kmax, s_gmin, s_gmax, s_digit, s_above, s_nlist, s_nbucket;
    __shared__ uint32_t s_dec_digit, s_dec_above, s_dec_over;   // rank 0's decision, read by every rank
    __shared__ int32_t list[kQSelList];
    __shared__ uint32_t bkey[kQSelBucket];
    __shared__ int32_t bidx[kQSelBucket];
    __shared__ uint32_t spos[kQSelList];
    pdl_wait();   // the scores come from the previous kernel (launched with programmatic serialization)
    pdl_launch_dependents();
    const int b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t off0 = seq_off[b];
    const int64_t n = seq_off[b + 1] - off0;
    const float *sc = scores + (off0 >> P_shift) + b;   // page j's score at sc[j]
    int32_t *row = ids + (int64_t)b * cap;
    const int64_t P = int64_t(1) << P_shift;
    const int64_t s_end = n_sink < n ? n_sink : n;
    const int64_t l0 = n - n_local > s_end ? n - n_local : s_end;
    const int64_t jlo = s_end >> P_shift;
    const int64_t nc = s_end < l0 ? ((l0 + P - 1) >> P_shift) - jlo : 0;
    const int64_t kp = (int64_t)k >> P_shift;
    const int64_t take = kp < nc ? kp : nc;
    auto page_lo = [&](int64_t j) { return (j << P_shift) > s_end ? (j << P_shift) : s_end; };
    auto page_hi = [&](int64_t j) { return ((j + 1) << P_shift) < l0 ? ((j + 1) << P_shift) : l0; };

    // general path: rank 0 alone (every decision that leads here is the same
    // in every rank, and the other ranks have left or no longer touch rank
    // 0's radix state)
    auto general = [&]() -> uint32_t {
        uint32_t prefix = 0u, pmask = 0u, above = 0u;
        for (int pass = 0; pass < 3; ++pass) {
            const int psh = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
            const uint32_t pdm = pass == 2 ? 1023u : 2047u;
            for (int i = tid; i < kQuestSelBins; i += blockDim.x)
                hist[i] = 0u;
            __syncthreads();
            for_each_key(sc + jlo, nc, [&](int64_t, uint32_t key) {
                if ((key & pmask) == prefix)
                    atomicAdd(&hist[(key >> psh) & pdm], 1u);
            });
            __syncthreads();
            const int top = (int)pdm;
            const int d1 = top - 2 * tid, d2 = d1 - 1;
            const uint32_t h1 = d1 >= 0 ? hist[d1] : 0u, h2 = d2 >= 0 ? hist[d2] : 0u;
            uint32_t tot;
            const uint32_t before = above + cta_exclusive_scan(h1 + h2, warp_sums, &tot);
            if (d1 >= 0 && before < (uint32_t)take && before + h1 >= (uint32_t)take) {
                s_digit = (uint32_t)d1;
                s_above = before;
            } else if (d2 >= 0 && before + h1 < (uint32_t)take && before + h1 + h2 >= (uint32_t)take) {
                s_digit = (uint32_t)d2;
                s_above = before + h1;
            }
            __syncthreads();
            prefix |= s_digit << psh;
            pmask |= pdm << psh;
            above = s_above;
            __syncthreads();
        }
        const uint32_t T = prefix, need = (uint32_t)take - above;
        const int64_t R = (nc + blockDim.x - 1) / blockDim.x;
        const int64_t c0 = (int64_t)tid * R, c1 = c0 + R < nc ? c0 + R : nc;
        uint32_t eq = 0u;
        for (int64_t c = c0; c < c1; ++c)
            eq += score_key(sc[jlo + c]) == T ? 1u : 0u;
        uint32_t unused;
        const uint32_t eq_rank = cta_exclusive_scan(eq, warp_sums, &unused);
        uint32_t ntok = 0u;
        {
            uint32_t rk = eq_rank;
            for (int64_t c = c0; c < c1; ++c) {
                const uint32_t key = score_key(sc[jlo + c]);
                if (key > T || (key == T && rk++ < need))
                    ntok += (uint32_t)(page_hi(jlo + c) - page_lo(jlo + c));
            }
        }
        uint32_t tt;
        uint32_t pos = (uint32_t)s_end + cta_exclusive_scan(ntok, warp_sums, &tt);
        {
            uint32_t rk = eq_rank;
            for (int64_t c = c0; c < c1; ++c) {
                const uint32_t key = score_key(sc[jlo + c]);
                if (key > T || (key == T && rk++ < need))
                    for (int64_t i = page_lo(jlo + c); i < page_hi(jlo + c); ++i)
                        row[pos++] = (int32_t)i;
            }
        }
        return tt;
    };

    uint32_t total_tok = 0u;
    if (take == nc) {
        if (rank != 0)
            return;
        // every candidate page (or none): every token of [s_end, l0)
        total_tok = nc > 0 ? (uint32_t)(l0 - s_end) : 0u;
        for (int64_t i = s_end + tid; i < s_end + total_tok; i += blockDim.x)
            row[i] = (int32_t)i;
    } else if (take > 0 && take > kQSelList) {
        if (rank != 0)
            return;
        total_tok = general();
    } else if (take > 0) {
        // this rank's slice of the candidates
        const int64_t c_lo = nc * rank / C, c_hi = nc * (rank + 1) / C;
        // pass 1: the slice's smallest and largest key
        uint32_t lo = 0xffffffffu, hi = 0u;
        for_each_key(sc + jlo + c_lo, c_hi - c_lo, [&](int64_t, uint32_t key) {
            lo = key < lo ? key : lo;
            hi = key > hi ? key : hi;
        });
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint32_t a2 = __shfl_xor_sync(0xffffffffu, lo, o), b2 = __shfl_xor_sync(0xffffffffu, hi, o);
            lo = a2 < lo ? a2 : lo;
            hi = b2 > hi ? b2 : hi;
        }
        if (lane == 0) {
            warp_lo[warp] = lo;
            warp_hi[warp] = hi;
        }
        for (int i = tid; i < kQuestSelBins; i += blockDim.x)
            hist[i] = 0u;
        __syncthreads();
        if (warp == 0) {
            lo = warp_lo[lane];
            hi = warp_hi[lane];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const uint32_t a2 = __shfl_xor_sync(0xffffffffu, lo, o), b2 = __shfl_xor_sync(0xffffffffu, hi, o);
                lo = a2 < lo ? a2 : lo;
                hi = b2 > hi ? b2 : hi;
            }
            if (lane == 0) {
                s_kmin = lo;
                s_kmax = hi;
            }
        }
        cl.sync();   // 1: every slice's min and max
        if (tid == 0) {
            uint32_t gl = 0xffffffffu, gh = 0u;
            for (int r = 0; r < C; ++r) {
                const uint32_t rl = *cl.map_shared_rank(&s_kmin, r), rh = *cl.map_shared_rank(&s_kmax, r);
                gl = rl < gl ? rl : gl;
                gh = rh > gh ? rh : gh;
            }
            s_gmin = gl;
            s_gmax = gh;
        }
        __syncthreads();
        // digit of a key: its place among 2048 equal bins over [kmin, kmax]
        // of all the keys (a monotone map: a higher digit is a larger key)
        const uint32_t kbase = s_gmin;
        const float kscale = (float)kQuestSelBins / ((float)(s_gmax - s_gmin) + 1.0f);
        auto digit_of = [&](uint32_t key) {
            const uint32_t d = (uint32_t)((float)(key - kbase) * kscale);
            return d < (uint32_t)(kQuestSelBins - 1) ? d : (uint32_t)(kQuestSelBins - 1);
        };
        // pass 2: the slice's histogram
        for_each_key(sc + jlo + c_lo, c_hi - c_lo, [&](int64_t, uint32_t key) { atomicAdd(&hist[digit_of(key)], 1u); });
        cl.sync();   // 2: every slice's histogram
        if (rank == 0) {
            // the threshold bin of the summed histograms (digits in descending
            // order, two per thread; each thread sums and keeps its own two)
            const int d1 = kQuestSelBins - 1 - 2 * tid, d2 = d1 - 1;
            uint32_t h1 = 0u, h2 = 0u;
            for (int r = 0; r < C; ++r) {
                const uint32_t *rh = cl.map_shared_rank(hist, r);
                h1 += rh[d1];
                h2 += rh[d2];
            }
            uint32_t tot;
            const uint32_t before = cta_exclusive_scan(h1 + h2, warp_sums, &tot);
            if (before < (uint32_t)take && before + h1 >= (uint32_t)take) {
                s_dec_digit = (uint32_t)d1;
                s_dec_above = before;
                s_dec_over = h1 > (uint32_t)kQSelBucket ? 1u : 0u;
            } else if (before + h1 < (uint32_t)take && before + h1 + h2 >= (uint32_t)take) {
                s_dec_digit = (uint32_t)d2;
                s_dec_above = before + h1;
                s_dec_over = h2 > (uint32_t)kQSelBucket ? 1u : 0u;
            }
            if (tid == 0) {
                s_nlist = 0u;
                s_nbucket = 0u;
            }
        }
        cl.sync();   // 3: rank 0's decision; nobody reads another rank's histogram any more
        const uint32_t digit = *cl.map_shared_rank(&s_dec_digit, 0);
        const uint32_t above = *cl.map_shared_rank(&s_dec_above, 0);
        const uint32_t over = *cl.map_shared_rank(&s_dec_over, 0);
        if (over != 0u) {
            if (rank != 0)
                return;
            total_tok = general();
        } else {
            // pass 3: the slice's sure winners and threshold-bin pages, into rank 0
            uint32_t *r_nlist = cl.map_shared_rank(&s_nlist, 0);
            uint32_t *r_nbucket = cl.map_shared_rank(&s_nbucket, 0);
            int32_t *r_list = cl.map_shared_rank(list, 0);
            uint32_t *r_bkey = cl.map_shared_rank(bkey, 0);
            int32_t *r_bidx = cl.map_shared_rank(bidx, 0);
            for_each_key(sc + jlo + c_lo, c_hi - c_lo, [&](int64_t c, uint32_t key) {
                const uint32_t d = digit_of(key);
                if (d > digit) {
                    r_list[atomicAdd(r_nlist, 1u)] = (int32_t)(c_lo + c);
                } else if (d == digit) {
                    const uint32_t slot = atomicAdd(r_nbucket, 1u);
                    r_bkey[slot] = key;
                    r_bidx[slot] = (int32_t)(c_lo + c);
                }
            });
            cl.sync();   // 4: every slice's pages are in rank 0
            if (rank != 0)
                return;
            // the bucket, ranked by (key desc, page asc): the first take - above join the list
            const uint32_t nb = s_nbucket, need = (uint32_t)take - above;
            for (uint32_t e = tid; e < nb; e += blockDim.x) {
                const uint32_t ke = bkey[e];
                const int32_t ie = bidx[e];
                uint32_t rk = 0u;
                for (uint32_t f = 0; f < nb; ++f)
                    rk += (bkey[f] > ke || (bkey[f] == ke && bidx[f] < ie)) ? 1u : 0u;
                if (rk < need)
                    list[above + rk] = ie;
            }
            __syncthreads();
            // the chosen pages in page order: rank by counting, token counts by rank
            const uint32_t nl = (uint32_t)take;
            constexpr int kPer = kQSelList / kQuestSelThreads;
            int32_t my_page[kPer];
            uint32_t my_rank[kPer];
#pragma unroll
            for (int r = 0; r < kPer; ++r) {
                const uint32_t e = tid + r * blockDim.x;
                my_page[r] = -1;
                my_rank[r] = 0u;
                if (e < nl) {
                    const int32_t pe = list[e];
                    uint32_t rk = 0u;
                    for (uint32_t f = 0; f < nl; ++f)
                        rk += list[f] < pe ? 1u : 0u;
                    my_page[r] = pe;
                    my_rank[r] = rk;
                    spos[rk] = (uint32_t)(page_hi(jlo + pe) - page_lo(jlo + pe));
                }
            }
            __syncthreads();
            // exclusive positions over the ranks, two entries per thread
            const uint32_t a0 = 2 * tid < nl ? spos[2 * tid] : 0u;
            const uint32_t a1 = 2 * tid + 1 < nl ? spos[2 * tid + 1] : 0u;
            const uint32_t before = cta_exclusive_scan(a0 + a1, warp_sums, &total_tok);
            if (2 * tid < nl)
                spos[2 * tid] = before;
            if (2 * tid + 1 < nl)
                spos[2 * tid + 1] = before + a0;
            __syncthreads();
#pragma unroll
            for (int r = 0; r < kPer; ++r)
                if (my_page[r] >= 0) {
                    const int64_t j = jlo + my_page[r];
                    uint32_t pos = (uint32_t)s_end + spos[my_rank[r]];
                    for (int64_t i = page_lo(j); i < page_hi(j); ++i)
                        row[pos++] = (int32_t)i;
                }
        }
    } else if (rank != 0) {
        return;   // nothing to choose: rank 0 writes the windows
    }
    // (rank 0) the windows, the count and the padding
    const int64_t m = s_end + total_tok + (n - l0);
    for (int64_t i = tid; i < s_end; i += blockDim.x)
        row[i] = (int32_t)i;
    for (int64_t i = l0 + tid; i < n; i += blockDim.x)
        row[s_end + total_tok + (i - l0)] = (int32_t)i;
    for (int64_t i = m + tid; i < cap; i += blockDim.x)
        row[i] = -1;
    if (tid == 0)
        count[b] = (int32_t)m;
}

int log2_exact(int x)
{
    int s = 0;
    while ((1 << s) < x)
        ++s;
    return s;
}

QuestKV make_quest_kv(const Plan &p, const ts_kv_t *kv, int page_size)
{
    QuestKV a;
    a.k = static_cast<const __nv_bfloat16 *>(kv->k);
    a.seq_off = kv->seq_offsets_dev;
    a.st = kv->stride_tok;
    a.sh = kv->stride_head;
    a.page_table = p.paged ? kv->page_table_dev : nullptr;
    a.pt_stride = p.paged ? kv->page_table_stride : 0;
    a.kv_page_shift = p.page_shift;
    a.pool_pages = p.paged ? p.kv_rows >> p.page_shift : 0;
    a.Hkv = p.Hkv;
    a.D = p.D;
    a.P_shift = log2_exact(page_size);
    return a;
}

// 16-byte chunks of a token row per lane: 1, 2 or 4 (h_kv * d in 64 .. 1024)
int chunks_per_lane(const Plan &p)
{
    const int e8 = p.Hkv * p.D / 8;
    return e8 <= 32 ? 1 : (e8 <= 64 ? 2 : 4);
}

}  // namespace

int64_t quest_rows(const Plan &p, int page_size)
{
    // sum over b of ceil(n_b / P) <= floor(n_total / P) + B (n_total: the
    // capacity of a growing cache), rounded up to a multiple of 4 so that the
    // selection may read the scores as aligned groups of four
    return (p.n_total / page_size + p.B + 3) / 4 * 4;
}

cudaError_t launch_quest_meta(const Plan &p, const ts_kv_t *kv, int page_size, void *kmin, void *kmax,
                              cudaStream_t st, int64_t last_tokens)
{
    const QuestKV a = make_quest_kv(p, kv, page_size);
    int64_t max_pages = (p.n_max + page_size - 1) / page_size;
    if (last_tokens > 0)   // the last t tokens span at most floor(t / P) + 2 pages
        max_pages = min(max_pages, last_tokens / page_size + 2);
    const dim3 grid((unsigned)((max_pages + kQuestWarps - 1) / kQuestWarps), (unsigned)p.B);
    if (max_pages == 0)
        return cudaSuccess;
    __nv_bfloat16 *lo = static_cast<__nv_bfloat16 *>(kmin), *hi = static_cast<__nv_bfloat16 *>(kmax);
    switch (chunks_per_lane(p)) {
    case 1:
        quest_meta<1><<<grid, kQuestWarps * 32, 0, st>>>(a, lo, hi, last_tokens);
        break;
    case 2:
        quest_meta<2><<<grid, kQuestWarps * 32, 0, st>>>(a, lo, hi, last_tokens);
        break;
    default:
        quest_meta<4><<<grid, kQuestWarps * 32, 0, st>>>(a, lo, hi, last_tokens);
        break;
    }
    return cudaGetLastError();
}

cudaError_t launch_quest_score(const Plan &p, const ts_kv_t *kv, const void *q, int page_size, const void *kmin,
                               const void *kmax, float *scores, cudaStream_t st)
{
    const int ch = chunks_per_lane(p);
    const int u = 4 / ch > 0 ? 4 / ch : 1;
    const int64_t max_pages = (p.n_max + page_size - 1) / page_size;
    if (max_pages == 0)
        return cudaSuccess;
    // persistent warps: two resident CTAs per SM over the batch (about 110
    // registers a thread), each warp walking its pages with a stride (its
    // query weights built once)
    const int64_t per_cta = (int64_t)kQuestWarps * u;
    int64_t gx = (max_pages + per_cta - 1) / per_cta;
    const int64_t cap_x = (2 * (int64_t)p.sms + p.B - 1) / p.B;
    gx = gx < cap_x ? gx : (cap_x > 0 ? cap_x : 1);
    const dim3 grid((unsigned)gx, (unsigned)p.B);
    const __nv_bfloat16 *qq = static_cast<const __nv_bfloat16 *>(q);
    const __nv_bfloat16 *lo = static_cast<const __nv_bfloat16 *>(kmin), *hi = static_cast<const __nv_bfloat16 *>(kmax);
    const int ps = log2_exact(page_size);
    switch (ch) {
    case 1:
        quest_score<1><<<grid, kQuestWarps * 32, 0, st>>>(kv->seq_offsets_dev, qq, lo, hi, scores, p.Hq, p.Hkv, p.D,
                                                         ps, p.scale);
        break;
    case 2:
        quest_score<2><<<grid, kQuestWarps * 32, 0, st>>>(kv->seq_offsets_dev, qq, lo, hi, scores, p.Hq, p.Hkv, p.D,
                                                         ps, p.scale);
        break;
    default:
        quest_score<4><<<grid, kQuestWarps * 32, 0, st>>>(kv->seq_offsets_dev, qq, lo, hi, scores, p.Hq, p.Hkv, p.D,
                                                         ps, p.scale);
        break;
    }
    return cudaGetLastError();
}

cudaError_t launch_quest_select(const Plan &p, const ts_kv_t *kv, const float *scores, int page_size, int k,
                                int n_sink, int n_local, int32_t *ids, int32_t *count, cudaStream_t st)
{
    // one cluster of kQSelCluster CTAs per sequence
    return launch_ex(quest_select, dim3(kQSelCluster, (unsigned)p.B), dim3(kQuestSelThreads), 0, st, kQSelCluster,
                     scores, kv->seq_offsets_dev, log2_exact(page_size), k, n_sink, n_local, k + n_sink + n_local, ids,
                     count);
}

}  // namespace ts
