// Fused scoring: per-head logits, softmax normalisers and soft votes of one
// layer-step in one persistent kernel, a few kv heads at a time (TokenSelect
// README, "Key Takeaways": per-head Q.K criticality, per-head softmax over
// the tokens, summed over the heads as the soft vote).
//
// For every active sequence b, kv head g and query head h = g*G + j:
//   s[h, i] = scale * q[b, h, :] . K[b, i, g, :]        (fp32 accumulation)
//   L[b, h] = log sum_i exp(s[h, i])
//   v[i]    = sum_h exp(s[h, i] - L[b, h])              (heads in order)
//
// Why a few kv heads at a time.  The vote needs every head's normaliser,
// which needs every token's logit, so the logits must be kept until the
// whole cache has been scored.  Scored all at once they are h_q * n * 4 bytes
// (117 MB at 28 heads x 1M tokens), more than L2 keeps beside the K stream:
// they go to DRAM and come back.  The kernel therefore scores HS kv heads per
// pass (h_kv / HS passes), HS chosen on the host so that one pass's logits
// (HS * G * n * 4 bytes; 29 MB at 1M tokens with HS = 1) stay in L2 until
// their votes are taken; each logit line is discarded from L2 once read, so
// dead data is not written back.  Short caches take every head in one pass.
//
// Design (B200).  One CTA per SM, cooperative launch (the grid barriers below
// need every CTA resident):
//  * The active sequences' tokens are cut into chunks of T = 128 / HS tokens
//    (a chunk never spans two sequences); a pipeline stage holds one chunk of
//    HS kv heads (128 K rows).  Every pass uses the same chunks and CTA j the
//    same ones: B == 1 round-robin (j, j + P, ...), so that every SM reads
//    from every part of the cache; B > 1 the balanced contiguous range
//    [j*C/P, (j+1)*C/P).  Logits live at logits[h][c*T + t] for active chunk
//    c: 32 consecutive tokens of a head are one 128-byte line.
//  * Warp 8 streams K with 3-D TMA boxes {64 channels, T tokens, HS heads}
//    (128-byte swizzle, L2 evict-first) into a ring of stages, pass after
//    pass.
//  * Warp 9 owns the tensor cores: it stages the sequence's queries in shared
//    memory (K-major, 128-byte swizzle; row g*GP + j = query head g*G + j,
//    zero for j >= G and for the padding rows after the last head) and one
//    lane issues per stage D[128 x N] = Kstage[128 x d] . Q_p[N x d]^T, Q_p
//    the N = max(16, HS*GP) rows of the pass's heads (tcgen05.mma kind::f16,
//    bf16 in, fp32 accumulator in one of four TMEM buffers).  Row hh*T + t of
//    D is token t of the pass's kv head hh; its columns hh*GP + j (j < G) are
//    that token's logits.
//  * Warps 0-7 (two per TMEM lane quarter, alternate stages; a quarter's 32
//    rows are 32 tokens of one head) read a token's G logits, store them, and
//    keep an online (max, sum exp) per head.  At the end of a (CTA, sequence,
//    pass) segment the eight warps reduce theirs (integer max of order-
//    preserving keys, fixed shuffle tree) and combine them through shared
//    memory in a fixed order into one partial per head at slot j + b
//    (unique: along the chunk order neither j nor b decreases).  When the CTA
//    has finished pass p one thread publishes it: a fence, then an add to the
//    pass's arrival counter.
//  * Warps 10-15 take the votes of pass p once every CTA has published it
//    (bounded spin on the counter): per segment they merge the partials of
//    the CTAs that cover the sequence into L[b, h] (fp32 terms exp(m - M) <= 1
//    summed in float64), then for each of the CTA's tokens add the pass's
//    HS*G terms exp_exact_arg(s, L) to the token's vote in head order (the
//    running vote is kept in the output array between passes), and discard
//    the logit lines they read.  L2 latency under the K stream is several
//    microseconds, so a vote thread keeps the next 24 loads in flight while
//    it sums the previous 24, and a segment's first loads are issued before
//    its normalisers are merged.  Pass p's votes overlap the K stream of pass p+1; the
//    last pass's votes are the tail of the kernel and the epilogue warps join
//    them.  With a histogram buffer (the one-call decode step) the last pass
//    also builds the selection's level-1 histogram of the candidates' votes
//    (top 12 bits; warp-aggregated shared-memory counts per sequence, then
//    added to the sequence's global histogram).  The vote workers synchronise
//    on shared-memory mbarriers (exact arrival counts).
//  * Dependents are released once the first grid barrier has passed (every
//    CTA resident), so that an early-launched next kernel cannot take the SM
//    space a CTA of this grid still needs.  The last CTA to finish resets
//    the counters for the next call.
// Every wait is bounded: a wait that gives up records its site in the status
// word, stops this role's work (the step's results are void) and still meets
// the CTA's own barriers, so the kernel always ends.
#include "score_common.cuh"
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

constexpr int kFEpiWarps = 8;
constexpr int kFProducerWarp = 8;
constexpr int kFMmaWarp = 9;
constexpr int kFVoteWarp0 = 10;
constexpr int kFVoteWarps = 6;
// 16 warps: four per SM sub-partition, whose register file (16K registers)
// then gives each thread 128
constexpr int kFThreads = (kFEpiWarps + 2 + kFVoteWarps) * 32;   // 512
constexpr int kFMaxRing = 8;      // line slots per vote worker warp
constexpr size_t kFVoteRingBytes = 24 * 1024;   // the vote warps' rings together (in flight during the K stream)
constexpr int kFRows = 128;       // K rows per stage (HS heads x T tokens): the MMA's M
constexpr int kFAccBufs = 4;
constexpr int kFMaxStages = 8;
constexpr int kFMaxPrefetch = 6;
constexpr int kFMaxPassHeads = 64;   // HS * G <= 4 * 16

// named barriers (0 is __syncthreads); the vote workers synchronise on
// mbarriers instead (exact arrival counts across warps of different roles)
constexpr uint32_t kBarTmem = 2;  // epilogue + MMA warps: every TMEM read done
constexpr uint32_t kBarEpi = 3;   // the eight epilogue warps

struct FusedArgs {
    const __nv_bfloat16 *q;   // [B, Hq, D]
    const int64_t *seq_off;   // [B + 1]
    const int32_t *reuse;     // [B] or null
    float *logits;            // [Hq][ld]: token t of active chunk c at c*T + t
    int64_t ld;
    float2 *partials;         // [Hq][S]: (max, sum exp(x - max)) of (CTA j, sequence b) at slot j + b
    int S;                    // grid + B
    float *votes;             // [n_total]
    float *vacc;              // [ld]: running votes between passes, chunk-aligned like the logits
    uint32_t *hist;           // [B][4096] level-1 selection histogram, or null
    int k, n_sink, n_local;   // the selection's window (histogram candidates)
    uint32_t *bar;            // [passes] arrival counters, [8] finished CTAs
    uint32_t *ctrl;           // status word
    int B, Hq, Hkv, G;
    int HS;                   // kv heads per pass
    int T;                    // tokens per chunk: 128 / HS
    int N;                    // MMA N: max(16, HS * GP)
    int stage_bytes;
    int nstages;
    int qrows;                // staged query rows: Hkv * GP + (N - HS * GP)
    uint32_t tmem_cols;
    uint32_t off_q, off_hist, off_tab;   // dynamic shared-memory offsets from the aligned base
    uint32_t off_vring;       // the vote warps' line rings
    uint32_t slot_bytes;      // one line slot: (HS*G + 1) rows of 32 floats
    int ring_v, ring_e;       // slots per vote warp; per epilogue warp in the last pass (in the K ring's space)
    int64_t pf_off[33];       // B <= 32: host copy of the offsets (prefetch hints only)
    float scale;
};

struct __align__(16) FusedShared {
    uint64_t full[kFMaxStages];
    uint64_t empty[kFMaxStages];
    uint64_t acc_full[kFAccBufs];
    uint64_t acc_empty[kFAccBufs];
    uint64_t mma_done;
    uint64_t vote_bar;            // the vote warps (arrivals: one per warp)
    uint64_t tail_bar;            // epilogue + vote warps, for the last pass
    uint32_t tmem_base;
    int32_t vote_ok;              // the vote warps' grid-barrier wait for their pass succeeded
    int32_t tail_ok;              // epilogue warp 0's wait for the last pass succeeded
    uint64_t ring_full[kFEpiWarps + kFVoteWarps][kFMaxRing];   // a worker warp's line slot has landed
    float2 seg[kFEpiWarps][16];   // epilogue warps' (max, sum) per head at a segment end
    float Lhi[kFMaxPassHeads], Llo[kFMaxPassHeads];   // L of the current segment's heads (hi + lo)
    int32_t pf_start[32];
    int64_t pf_off[32];
};

__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap *map, int32_t x, int32_t y, int32_t z)
{
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Drop a 128-byte L2 line without writing it back (its data is dead).
__device__ __forceinline__ void l2_discard_line(const void *p)
{
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// The sequence's queries as the UMMA B operand: qrows rows of D channels,
// bf16, K-major with the 128-byte swizzle (64-channel halves of qrows * 128
// bytes); row g*GP + j holds query head g*G + j, the others are zero.
template <int D, int GP>
__device__ __forceinline__ void stage_queries_fused(uint8_t *qs, const __nv_bfloat16 *qb, int G, int Hkv, int qrows,
                                                    int lane)
{
    constexpr int kChunks = D / 8;   // 16-byte chunks per row
    constexpr int kBatch = 8;
    const int total = qrows * kChunks;
    for (int c0 = lane; c0 < total; c0 += 32 * kBatch) {
        uint4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int c = c0 + u * 32;
            const int n = c / kChunks, cc = c - n * kChunks;
            const int g = n / GP, j = n - g * GP;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (c < total && g < Hkv && j < G)
                v[u] = __ldg(reinterpret_cast<const uint4 *>(qb + (int64_t)(g * G + j) * D) + cc);
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int c = c0 + u * 32;
            if (c < total) {
                const int n = c / kChunks, cc = c - n * kChunks;
                const int half = cc >> 3, ci = cc & 7;
                *reinterpret_cast<uint4 *>(qs + (size_t)half * qrows * 128 + n * 128 + ((ci ^ (n & 7)) << 4)) = v[u];
            }
        }
    }
}

// End of a (CTA, sequence, pass) segment in the epilogue: each warp reduces
// its lanes' (max, sum) per head, then thread e < HS*G of the epilogue
// combines, in a fixed order, the warps whose rows hold kv head hh = e / G
// (head j = e % G) and writes the segment's partial of query head
// (p*HS + hh)*G + j.  All eight epilogue warps call it; (m, z) are consumed.
template <int GP>
__device__ __forceinline__ void fused_flush(FusedShared &sh, float (&m)[GP], float (&z)[GP], const FusedArgs &a,
                                            int lane, int warp, int p, int64_t slot)
{
#pragma unroll
    for (int j = 0; j < GP; ++j) {
        const float M = float_from_order_key(__reduce_max_sync(0xffffffffu, float_order_key(m[j])));
        z[j] = (m[j] == -INFINITY) ? 0.0f : z[j] * exp2f((m[j] - M) * kLog2e);
        m[j] = M;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int j = 0; j < GP; ++j)
            z[j] += __shfl_xor_sync(0xffffffffu, z[j], o);
    if (lane == 0)
#pragma unroll
        for (int j = 0; j < GP; ++j)
            if (j < a.G)
                sh.seg[warp][j] = make_float2(m[j], z[j]);
    named_bar_sync(kBarEpi, kFEpiWarps * 32);
    const int e = warp * 32 + lane;
    if (e < a.HS * a.G) {
        const int hh = e / a.G, j = e - hh * a.G;
        const int qpt = a.T / 32;   // lane quarters per kv head
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kFEpiWarps; ++w)
            if ((w & 3) / qpt == hh)
                M = fmaxf(M, sh.seg[w][j].x);
        float Z = 0.0f;
        if (M != -INFINITY)
#pragma unroll
            for (int w = 0; w < kFEpiWarps; ++w) {
                const float2 s2 = sh.seg[w][j];
                if ((w & 3) / qpt == hh && s2.x != -INFINITY)
                    Z += s2.y * exp2f((s2.x - M) * kLog2e);
            }
        a.partials[(int64_t)((p * a.HS + hh) * a.G + j) * a.S + slot] = make_float2(M, Z);
    }
    named_bar_sync(kBarEpi, kFEpiWarps * 32);
}

// The chunks of CTA j: begin, begin + step, ... < end.
struct ChunkRange {
    int32_t begin, end, step;
};

__device__ __forceinline__ ChunkRange cta_chunks(int B, int32_t total)
{
    ChunkRange r;
    if (B == 1) {
        r.begin = (int32_t)blockIdx.x;
        r.end = total;
        r.step = (int32_t)gridDim.x;
    } else {
        r.begin = chunk_split(blockIdx.x, total, gridDim.x);
        r.end = chunk_split(blockIdx.x + 1, total, gridDim.x);
        r.step = 1;
    }
    return r;
}

// Wait until every CTA has published pass p (one thread), bounded.
__device__ __forceinline__ bool wait_pass(const FusedArgs &a, int p)
{
    const uint32_t want = gridDim.x;
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (ld_acquire_gpu(a.bar + p) >= want) {
            __threadfence();
            return true;
        }
        __nanosleep(i < 64 ? 32 : 256);
    }
    report_timeout(a.ctrl, kSiteFusedGrid);
    return false;
}

// A CTA-local barrier over a set of whole warps: lane 0 of each warp arrives
// on an mbarrier initialised with the set's warp count, every thread waits
// for the phase (bounded).  Exact arrival counts, whatever each warp did
// before; `phase` is the caller's running parity.
__device__ __forceinline__ bool warpset_sync(uint64_t *bar, uint32_t &phase, uint32_t *ctrl)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
        mbar_arrive(bar);
    const bool ok = mbar_wait_bounded(bar, phase, kSpinLimit);
    phase ^= 1u;
    if (!ok && (threadIdx.x & 31) == 0)
        report_timeout(ctrl, kSiteFusedCta);
    __syncwarp();
    return ok;
}

// A worker warp's ring of line slots.  A line is 32 consecutive tokens of
// one chunk; its slot holds row 0 = the tokens' running votes (pass > 0) and
// row 1 + e = their logits of the pass's head e, each row 128 bytes, brought
// in with bulk asynchronous copies (completion on the slot's mbarrier), so
// that the loads of several lines are in flight without holding registers.
struct LineRing {
    uint8_t *slots;      // ring x slot_bytes
    uint64_t *full;      // one mbarrier per slot (arrival count 1)
    int ring;
    uint32_t phase;      // bit r: parity of slot r's next completion
};

// The line geometry of a segment: line l is sub-line l % (T/32) of the
// segment's chunk l / (T/32).
struct SegLines {
    const float *lg0;       // logits of the pass's first head
    int32_t s_off, s_end;   // the sequence's tokens (n_total < 2^31)
    int32_t cs_b;           // its first chunk
    int32_t vseg, step;     // the segment's chunks: vseg, vseg + step, ...
    int32_t nlines;
    int HG, spc;            // heads of the pass; sub-lines per chunk (T / 32)
};

__device__ __forceinline__ void line_pos(const FusedArgs &a, const SegLines &sl, int32_t l, int32_t &tok0,
                                         int32_t &col0)
{
    const int32_t kk = l / sl.spc, sub = l - kk * sl.spc;
    const int32_t c = sl.vseg + kk * sl.step;
    tok0 = sl.s_off + (c - sl.cs_b) * a.T + sub * 32;
    col0 = c * a.T + sub * 32;
}

// Lane 0: bring line l of the segment into slot r.
__device__ __forceinline__ void line_issue(const FusedArgs &a, const SegLines &sl, LineRing &rg, int r, int32_t l,
                                           int p)
{
    int32_t tok0, col0;
    line_pos(a, sl, l, tok0, col0);
    uint8_t *dst = rg.slots + (size_t)r * a.slot_bytes;
    const uint32_t rows = (uint32_t)sl.HG + (p > 0 ? 1u : 0u);
    mbar_arrive_expect_tx(&rg.full[r], rows * 128u);
    if (p > 0)
        bulk_copy_g2s(dst, a.vacc + col0, 128u, &rg.full[r]);
    for (int e = 0; e < sl.HG; ++e)
        bulk_copy_g2s(dst + (size_t)(e + 1) * 128, sl.lg0 + (int64_t)e * a.ld + col0, 128u, &rg.full[r]);
}

// The votes of pass p for this CTA's tokens, by `nw` worker warps (worker
// index wid) that synchronise on `bar` (phase: the caller's running parity);
// each warp runs its lines through its own ring.  Every worker calls it, in
// the same order; ok = the pass's grid barrier was passed.
template <bool HIST>
__device__ void fused_vote_pass(const FusedArgs &a, FusedShared &sh, const int64_t *off, const int32_t *cs,
                                uint32_t *hist_s, int p, int wid, int nw, uint64_t *bar, uint32_t &phase,
                                LineRing &rg, bool last, bool ok, int32_t total)
{
    const int nthr = nw * 32;
    const int lane = threadIdx.x & 31;
    const int tid = wid * 32 + lane;
    const int B = a.B;
    const int HG = a.HS * a.G;
    const ChunkRange cr = cta_chunks(B, total);
    const int P = (int)gridDim.x;
    const int npass = a.Hkv / a.HS;
    float *vout_base = (p + 1 < npass) ? a.vacc : nullptr;   // running votes, or the output on the last pass
    int32_t v = cr.begin;
    while (v < cr.end) {
        const int b = upper_seq(cs, B, v);
        // this segment: the CTA's chunks of sequence b, from v on
        const int32_t ce = min(cs[b + 1], cr.end);
        const int32_t nseg = (ce - v + cr.step - 1) / cr.step;
        SegLines sl;
        sl.lg0 = a.logits + (int64_t)p * HG * a.ld;
        sl.s_off = (int32_t)off[b];
        sl.s_end = (int32_t)off[b + 1];
        sl.cs_b = cs[b];
        sl.vseg = v;
        sl.step = cr.step;
        sl.spc = a.T / 32;
        sl.nlines = nseg * sl.spc;
        sl.HG = HG;
        warpset_sync(bar, phase, a.ctrl);   // the previous segment's readers of Lhi / Llo are done
        // this warp's lines: wid, wid + nw, ...; the first ring-full are
        // requested now, before the normalisers are merged
        const int32_t nmine = sl.nlines > wid ? (sl.nlines - wid + nw - 1) / nw : 0;
        if (ok && lane == 0) {
            fence_proxy_async_global();   // the pass's logits and running votes, written by this CTA's threads
            for (int r = 0; r < rg.ring && r < nmine; ++r)
                line_issue(a, sl, rg, r, wid + r * nw, p);
        }
        // ---- L[b, h] for the pass's heads from the partials of every CTA
        //      that covers sequence b (each warp's heads loaded together) -------
        if (ok) {
            const int32_t c0 = cs[b], c1 = cs[b + 1];
            int j0, j1;
            if (B == 1) {
                j0 = 0;
                j1 = min(total, P) - 1;
            } else {
                j0 = (int)(((int64_t)(c0 + 1) * P - 1) / total);
                j1 = (int)(((int64_t)c1 * P - 1) / total);
            }
            for (int e0 = wid; e0 < HG; e0 += 2 * nw) {
                float2 pv[2][8];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int e = e0 + r * nw;
                    const float2 *row_p = a.partials + (int64_t)(p * HG + e) * a.S + b;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int jj = j0 + lane + 32 * i;
                        bool keep = e < HG && jj <= j1;
                        if (keep && B > 1 && total < P)   // CTAs without chunks wrote nothing
                            keep = chunk_split(jj, total, P) < chunk_split(jj + 1, total, P);
                        pv[r][i] = keep ? __ldcg(row_p + jj) : make_float2(-INFINITY, 0.0f);
                    }
                }
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int e = e0 + r * nw;
                    float M = -INFINITY;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        M = fmaxf(M, pv[r][i].x);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
                    double Z = 0.0;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        if (pv[r][i].y > 0.0f)
                            Z += (double)(pv[r][i].y * exp2f((pv[r][i].x - M) * kLog2e));
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        Z += __shfl_xor_sync(0xffffffffu, Z, o);
                    if (lane == 0 && e < HG) {
                        const double L = (double)M + log(Z);
                        const float hi = (float)L;
                        sh.Lhi[e] = hi;
                        sh.Llo[e] = (float)(L - (double)hi);
                    }
                }
            }
        }
        warpset_sync(bar, phase, a.ctrl);
        // ---- the votes of the segment's tokens --------------------------------
        // histogram candidates [s', l0) of the sequence, when the selection
        // ranks some but not all of them
        bool hist_on = false;
        int32_t cand_lo = 0, cand_hi = 0;
        if (HIST && last) {
            const int32_t n = sl.s_end - sl.s_off;
            const int32_t se = min(a.n_sink, n);
            const int32_t l0 = max(n - a.n_local, se);
            const int32_t keff = min(a.k, l0 - se);
            hist_on = !(keff == 0 || keff == l0 - se);
            cand_lo = se;
            cand_hi = l0;
        }
        if (ok) {
            for (int32_t i = 0; i < nmine; ++i) {
                const int r = i % rg.ring;
                const int32_t l = wid + i * nw;
                const bool landed = mbar_wait_bounded(&rg.full[r], (rg.phase >> r) & 1u, kSpinLimit);
                rg.phase ^= 1u << r;
                if (!landed && lane == 0)
                    report_timeout(a.ctrl, kSiteFusedCta);
                const float *row = reinterpret_cast<const float *>(rg.slots + (size_t)r * a.slot_bytes);
                int32_t tok0, col0;
                line_pos(a, sl, l, tok0, col0);
                const int32_t tok = tok0 + lane;
                float acc = p > 0 ? row[lane] : 0.0f;
                for (int e = 0; e < HG; ++e)
                    acc += exp_exact_arg(row[(e + 1) * 32 + lane], sh.Lhi[e], sh.Llo[e]);
                const bool valid = tok < sl.s_end;
                if (valid) {
                    if (vout_base != nullptr)
                        vout_base[col0 + lane] = acc;
                    else
                        a.votes[tok] = acc;
                }
                if (HIST && hist_on) {
                    const int32_t li = tok - sl.s_off;
                    const bool cand = valid && li >= cand_lo && li < cand_hi;
                    const uint32_t bin = cand ? (__float_as_uint(acc) >> 20) : 0xffffffffu;
                    const uint32_t peers = __match_any_sync(0xffffffffu, bin);
                    if (cand && lane == __ffs(peers) - 1)
                        atomicAdd(&hist_s[bin], (uint32_t)__popc(peers));
                }
                // the slot is read (every lane's values are in registers): drop
                // the line's logits from L2 and reuse the slot for a later line
                __syncwarp();
                for (int e = lane; e < HG; e += 32)
                    l2_discard_line(sl.lg0 + (int64_t)e * a.ld + col0);
                if (lane == 0 && i + rg.ring < nmine) {
                    fence_proxy_async_smem();
                    line_issue(a, sl, rg, r, l + rg.ring * nw, p);
                }
            }
        }
        if (HIST && last) {
            warpset_sync(bar, phase, a.ctrl);   // every candidate of the segment counted
            uint32_t *gh = a.hist + (size_t)b * 4096;
            for (int i = tid; i < 4096; i += nthr) {
                const uint32_t c = hist_s[i];
                if (c != 0u) {
                    if (hist_on && ok)
                        atomicAdd(&gh[i], c);
                    hist_s[i] = 0u;
                }
            }
        }
        v = v + nseg * cr.step;
    }
}

template <int D, int GP, bool HIST>
__global__ void __launch_bounds__(kFThreads, 1)
score_fused(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ FusedArgs a)
{
    extern __shared__ uint8_t dyn_smem[];
    __shared__ FusedShared sh;
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = base;
    uint8_t *qs = base + a.off_q;
    uint32_t *hist_s = reinterpret_cast<uint32_t *>(base + a.off_hist);
    int64_t *off = reinterpret_cast<int64_t *>(base + a.off_tab);
    int32_t *cs = reinterpret_cast<int32_t *>(base + a.off_tab + 8 * (a.B + 1));
    const int NS = a.nstages;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = a.B;
    const int HS = a.HS;
    const int T = a.T;
    const int G = a.G;
    const int npass = a.Hkv / HS;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int s = 0; s < kFAccBufs; ++s) {
            mbar_init(&sh.acc_full[s], 1);
            mbar_init(&sh.acc_empty[s], kFEpiWarps / 2);   // the four warps of that stage parity
        }
        mbar_init(&sh.mma_done, 1);
        mbar_init(&sh.vote_bar, kFVoteWarps);
        mbar_init(&sh.tail_bar, kFEpiWarps + kFVoteWarps);
        for (int w = 0; w < kFEpiWarps + kFVoteWarps; ++w)
            for (int r = 0; r < kFMaxRing; ++r)
                mbar_init(&sh.ring_full[w][r], 1);
        mbar_fence_init();
    }
    if (warp == kFMmaWarp)
        tmem_alloc(&sh.tmem_base, a.tmem_cols);
    if (HIST && warp >= kFVoteWarp0)
        for (int i = tid - kFVoteWarp0 * 32; i < 4096; i += kFVoteWarps * 32)
            hist_s[i] = 0u;
    // ---- before the previous kernel has finished: L2 prefetch hints for the
    //      first tiles of pass 0, as if every sequence were active (a wrong
    //      guess costs bandwidth only) ---------------------------------------
    if (B <= 32 && warp == kFProducerWarp) {
        if (lane == 0)
            tma_prefetch_desc(&kmap);
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
        if (lane < B) {
            sh.pf_start[lane] = c1 - x;
            sh.pf_off[lane] = o0;
        }
        const int32_t total = __shfl_sync(0xffffffffu, c1, B - 1);
        __syncwarp();
        if (lane == 0 && total > 0) {
            const ChunkRange cr = cta_chunks(B, total);
            int b = 0, nfetch = 0;
            for (int32_t v = cr.begin; v < cr.end && nfetch < min(NS, kFMaxPrefetch); v += cr.step, ++nfetch) {
                while (b + 1 < B && sh.pf_start[b + 1] <= v)
                    ++b;
                const int64_t t0 = sh.pf_off[b] + (int64_t)(v - sh.pf_start[b]) * T;
#pragma unroll
                for (int xx = 0; xx < D / 64; ++xx)
                    tma_prefetch_l2_3d(&kmap, xx * 64, (int32_t)t0, 0);
            }
        }
        __syncwarp();
    }
    pdl_wait();

    // ---- the chunk table of the active sequences (one round trip for the
    //      offsets and the reuse flags) --------------------------------------
    tmem_fence_before();
    for (int b = tid; b < B; b += blockDim.x) {
        const int64_t o0 = __ldcg(a.seq_off + b), o1 = __ldcg(a.seq_off + b + 1);
        const bool active = a.reuse == nullptr || __ldcg(a.reuse + b) == 0;
        off[b] = o0;
        if (b == B - 1)
            off[B] = o1;
        const int64_t n = o1 - o0;
        cs[b + 1] = (active && n > 0) ? (int32_t)((n + T - 1) / T) : 0;
    }
    __syncthreads();
    if (warp == 0) {
        int32_t run = 0;
        for (int b0 = 0; b0 < B; b0 += 32) {
            const int b = b0 + lane;
            int32_t x = (b < B) ? cs[b + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o)
                    x += y;
            }
            if (b < B)
                cs[b + 1] = run + x;
            run += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0)
            cs[0] = 0;
    }
    __syncthreads();
    tmem_fence_after();
    const int32_t total = cs[B];
    const uint32_t tmem = sh.tmem_base;
    if (total == 0) {   // every sequence reuses its selection (or is empty)
        if (warp == kFMmaWarp)
            tmem_dealloc(tmem, a.tmem_cols);
        return;
    }
    const ChunkRange cr = cta_chunks(B, total);
    const int32_t nmy = cr.end > cr.begin ? (cr.end - cr.begin + cr.step - 1) / cr.step : 0;
    constexpr int kHalfBytes = kFRows * 128;   // one 64-channel box

    if (warp == kFProducerWarp) {
        // ================= TMA producer: one elected lane ==================
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            uint32_t it = 0;
            bool stop = false;
            for (int p = 0; p < npass && !stop; ++p) {
                int b = 0;
                for (int32_t r = 0; r < nmy; ++r, ++it) {
                    const int32_t v = cr.begin + r * cr.step;
                    while (b + 1 < B && cs[b + 1] <= v)
                        ++b;
                    const int64_t t0 = off[b] + (int64_t)(v - cs[b]) * T;
                    const int s = it % NS;
                    if (it >= (uint32_t)NS) {
                        if (!mbar_wait_bounded(&sh.empty[s], ((it / NS) - 1) & 1, kSpinLimit)) {
                            report_timeout(a.ctrl, kSiteScoreEmpty);
                            // wait (bounded) for the tiles already in flight
                            for (uint32_t j = it > (uint32_t)NS ? it - NS : 0u; j < it; ++j)
                                (void)mbar_wait_bounded(&sh.full[j % NS], (j / NS) & 1, kSpinLimit);
                            stop = true;
                            break;
                        }
                    }
                    mbar_arrive_expect_tx(&sh.full[s], (uint32_t)a.stage_bytes);
#pragma unroll
                    for (int x = 0; x < D / 64; ++x)
                        tma_load_3d(stages + (size_t)s * a.stage_bytes + x * kHalfBytes, &kmap, &sh.full[s], x * 64,
                                    (int32_t)t0, p * HS, pol);
                }
            }
        }
        return;   // takes no part in the later barriers
    }

    if (warp == kFMmaWarp) {
        // ================= tensor cores ====================================
        const uint32_t idesc = umma_idesc_bf16_f32(kFRows, a.N);
        int cur_b = -1;
        bool dead = false;
        uint32_t done_par = 0;
        uint32_t it = 0;
        for (int p = 0; p < npass && !dead; ++p) {
            int b = 0;
            for (int32_t r = 0; r < nmy && !dead; ++r, ++it) {
                const int32_t v = cr.begin + r * cr.step;
                while (b + 1 < B && cs[b + 1] <= v)
                    ++b;
                if (b != cur_b) {
                    if (it > 0) {   // the old queries may still be read by MMAs in flight
                        if (lane == 0)
                            umma_commit(&sh.mma_done);
                        __syncwarp();
                        const bool ok =
                            __all_sync(0xffffffffu, mbar_wait_bounded(&sh.mma_done, done_par, kSpinLimit));
                        done_par ^= 1u;
                        if (!ok) {
                            if (lane == 0)
                                report_timeout(a.ctrl, kSiteScoreMma);
                            dead = true;
                            break;
                        }
                    }
                    stage_queries_fused<D, GP>(qs, a.q + (int64_t)b * a.Hq * D, G, a.Hkv, a.qrows, lane);
                    fence_proxy_async_smem();
                    __syncwarp();
                    cur_b = b;
                }
                const int s = it % NS;
                const uint32_t par = (it / NS) & 1;
                const int buf = it % kFAccBufs;
                bool ok = true;
                if (lane == 0) {
                    ok = mbar_wait_bounded(&sh.full[s], par, kSpinLimit);
                    if (ok && it >= (uint32_t)kFAccBufs)
                        ok = mbar_wait_bounded(&sh.acc_empty[buf], ((it / kFAccBufs) - 1) & 1, kSpinLimit);
                    if (ok) {
                        tmem_fence_after();
                        const uint32_t a_base = smem_u32(stages + (size_t)s * a.stage_bytes);
                        const uint32_t b_base = smem_u32(qs) + (uint32_t)(p * HS * GP * 128);
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t koff = (uint32_t)((ks & 3) * 32);
                            const uint64_t ad = umma_desc_sw128(a_base + (uint32_t)((ks >> 2) * kHalfBytes) + koff);
                            const uint64_t bd =
                                umma_desc_sw128(b_base + (uint32_t)((ks >> 2) * a.qrows * 128) + koff);
                            umma_bf16(tmem + (uint32_t)(buf * a.N), ad, bd, idesc, ks > 0);
                        }
                        umma_commit(&sh.empty[s]);
                        umma_commit(&sh.acc_full[buf]);
                    } else {
                        report_timeout(a.ctrl, kSiteScoreMma);
                    }
                }
                dead = !__shfl_sync(0xffffffffu, ok ? 1 : 0, 0);
                __syncwarp();
            }
        }
        if (it > 0) {
            if (lane == 0)
                umma_commit(&sh.mma_done);
            __syncwarp();
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(&sh.mma_done, done_par, kSpinLimit))) {
                if (lane == 0)
                    report_timeout(a.ctrl, kSiteScoreMma);
                (void)mbar_wait_bounded(&sh.mma_done, done_par, kSpinLimit);
            }
        }
        tmem_fence_before();
        named_bar_sync(kBarTmem, (kFEpiWarps + 1) * 32);
        tmem_fence_after();
        tmem_dealloc(tmem, a.tmem_cols);
        return;
    }

    LineRing tail_ring;   // this worker warp's line slots for the last pass's votes
    if (warp < kFEpiWarps) {
        // ================= epilogue: logits and segment partials ===========
        const int quarter = warp & 3, hs = warp >> 2;
        const int hh = quarter / (T / 32);               // the pass's kv head of this lane quarter
        const int t_row = quarter * 32 + lane - hh * T;  // token within the chunk
        const float scale = a.scale;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        float m[GP], z[GP];
        bool dead = false;
        uint32_t it = 0;
        for (int p = 0; p < npass; ++p) {
            int cur_b = -1;
            int b = 0;
            float *lg_pass = a.logits + (int64_t)(p * HS + hh) * G * a.ld;
            for (int32_t r = 0; r < nmy; ++r, ++it) {
                const int32_t v = cr.begin + r * cr.step;
                while (b + 1 < B && cs[b + 1] <= v)
                    ++b;
                if (b != cur_b) {
                    if (cur_b >= 0)
                        fused_flush<GP>(sh, m, z, a, lane, warp, p, (int64_t)blockIdx.x + cur_b);
                    cur_b = b;
#pragma unroll
                    for (int j = 0; j < GP; ++j) {
                        m[j] = -INFINITY;
                        z[j] = 0.0f;
                    }
                }
                if (dead || (int)(it & 1u) != hs)
                    continue;   // the other warp of this lane quarter takes it
                const int buf = it % kFAccBufs;
                if (!__all_sync(0xffffffffu,
                                mbar_wait_bounded(&sh.acc_full[buf], (it / kFAccBufs) & 1, kSpinLimit))) {
                    if (lane == 0)
                        report_timeout(a.ctrl, kSiteScoreAcc);
                    dead = true;
                    continue;
                }
                tmem_fence_after();
                uint32_t raw[GP];
                tmem_ld_32x32b<GP>(lane_base + (uint32_t)(buf * a.N + hh * GP), raw);
                tmem_wait_ld();
                tmem_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&sh.acc_empty[buf]);
                const int64_t tok = off[b] + (int64_t)(v - cs[b]) * T + t_row;
                if (tok < off[b + 1]) {
                    float *lg = lg_pass + (int64_t)v * T + t_row;
#pragma unroll
                    for (int j = 0; j < GP; ++j) {
                        if (j < G) {
                            const float x = __uint_as_float(raw[j]) * scale;
                            lg[(int64_t)j * a.ld] = x;
                            online_push(m[j], z[j], x);
                        }
                    }
                }
            }
            if (cur_b >= 0)
                fused_flush<GP>(sh, m, z, a, lane, warp, p, (int64_t)blockIdx.x + cur_b);
            // pass p done in this CTA: publish it (the flush's barrier has
            // ordered every epilogue warp's stores before this)
            if (warp == 0 && lane == 0) {
                __threadfence();
                atomicAdd(a.bar + p, 1u);
            }
        }
        // every TMEM read done: the MMA warp may free TMEM (and every stage
        // has been consumed: the ring's space now holds these warps' line
        // slots for the last pass's votes)
        tmem_fence_before();
        named_bar_sync(kBarTmem, (kFEpiWarps + 1) * 32);
        tail_ring.slots = stages + (size_t)warp * a.ring_e * a.slot_bytes;
        tail_ring.full = sh.ring_full[warp];
        tail_ring.ring = a.ring_e;
        tail_ring.phase = 0;
        // ---- then help with the last pass's votes ------------------------------
        if (warp == 0 && lane == 0) {
            const bool ok = wait_pass(a, npass - 1);
            sh.tail_ok = ok ? 1 : 0;
            if (npass == 1 && ok)
                pdl_launch_dependents();
        }
    } else {
        // ================= vote warps ======================================
        const int wid = warp - kFVoteWarp0;
        uint32_t phase = 0;
        LineRing rg;
        rg.slots = base + a.off_vring + (size_t)wid * a.ring_v * a.slot_bytes;
        rg.full = sh.ring_full[kFEpiWarps + wid];
        rg.ring = a.ring_v;
        rg.phase = 0;
        for (int p = 0; p + 1 < npass; ++p) {
            if (wid == 0 && lane == 0) {
                const bool ok = wait_pass(a, p);
                sh.vote_ok = ok ? 1 : 0;
                if (p == 0 && ok)
                    pdl_launch_dependents();
            }
            warpset_sync(&sh.vote_bar, phase, a.ctrl);
            const bool ok = sh.vote_ok != 0;
            warpset_sync(&sh.vote_bar, phase, a.ctrl);   // vote_ok is read before it is rewritten
            fused_vote_pass<HIST>(a, sh, off, cs, hist_s, p, wid, kFVoteWarps, &sh.vote_bar, phase, rg, false, ok,
                                  total);
        }
        tail_ring = rg;
    }
    // ---- the last pass's votes: epilogue warps (workers 0-7) and vote warps
    //      (workers 8-13); epilogue warp 0 has waited for the pass ------------
    uint32_t tphase = 0;
    warpset_sync(&sh.tail_bar, tphase, a.ctrl);
    const bool ok = sh.tail_ok != 0;
    const int wid = warp < kFEpiWarps ? warp : warp - 2;
    fused_vote_pass<HIST>(a, sh, off, cs, hist_s, npass - 1, wid, kFEpiWarps + kFVoteWarps, &sh.tail_bar, tphase,
                          tail_ring, true, ok, total);
    warpset_sync(&sh.tail_bar, tphase, a.ctrl);
    if (tid == 0 && ok) {
        // every CTA that got here has passed every grid barrier: the last one
        // resets the counters for the next call
        __threadfence();
        if (atomicAdd(a.bar + 8, 1u) == gridDim.x - 1) {
            for (int p = 0; p < npass; ++p)
                atomicExch(a.bar + p, 0u);
            atomicExch(a.bar + 8, 0u);
        }
    }
}

template <int D, int GP, bool HIST>
cudaError_t launch_fused_t(const Plan &p, const CUtensorMap &kmap, FusedArgs args, cudaStream_t st)
{
    // dynamic shared memory: stages | queries | histogram | offsets | chunk table
    const int qrows = p.Hkv * GP + (p.fused_n - p.fused_hs * GP);
    const uint32_t q_bytes = (uint32_t)(qrows * D * 2);
    const uint32_t hist_bytes = HIST ? 4096u * 4u : 0u;
    const uint32_t tab_bytes = (uint32_t)(8 * (p.B + 1) + 4 * (p.B + 1));
    // the vote warps' line rings: about kFVoteRingBytes, 1 to kFMaxRing slots each
    const uint32_t slot_bytes = (uint32_t)(p.fused_hs * p.G + 1) * 128u;
    int ring_v = (int)(kFVoteRingBytes / ((size_t)kFVoteWarps * slot_bytes));
    ring_v = ring_v < 1 ? 1 : (ring_v > kFMaxRing ? kFMaxRing : ring_v);
    const uint32_t vring_bytes = (uint32_t)(kFVoteWarps * ring_v) * slot_bytes;
    const size_t fixed = (size_t)q_bytes + hist_bytes + vring_bytes + tab_bytes + 1024;
    int ns = (int)((kFusedDynSmemBudget - fixed) / (size_t)args.stage_bytes);
    ns = ns < kFMaxStages ? ns : kFMaxStages;
    if (ns < 2)
        return cudaErrorInvalidConfiguration;
    // the epilogue warps' rings for the last pass live in the stages' space
    int ring_e = (int)(((size_t)ns * args.stage_bytes) / ((size_t)kFEpiWarps * slot_bytes));
    ring_e = ring_e < 1 ? 1 : (ring_e > kFMaxRing ? kFMaxRing : ring_e);
    if ((size_t)kFEpiWarps * ring_e * slot_bytes > (size_t)ns * args.stage_bytes)
        return cudaErrorInvalidConfiguration;
    args.nstages = ns;
    args.qrows = qrows;
    args.slot_bytes = slot_bytes;
    args.ring_v = ring_v;
    args.ring_e = ring_e;
    args.off_q = (uint32_t)(ns * args.stage_bytes);
    args.off_hist = args.off_q + q_bytes;
    args.off_vring = args.off_hist + hist_bytes;
    args.off_tab = args.off_vring + vring_bytes;
    uint32_t cols = 32;
    while (cols < (uint32_t)(kFAccBufs * p.fused_n))
        cols <<= 1;
    args.tmem_cols = cols;
    const size_t dyn = (size_t)args.off_tab + tab_bytes + 1024;
    cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void *>(score_fused<D, GP, HIST>), (int)kFusedDynSmemBudget);
    if (e != cudaSuccess)
        return e;
    return launch_coop(score_fused<D, GP, HIST>, dim3((unsigned)p.fused_grid), dim3(kFThreads), dyn, st, kmap,
                       args);
}

template <int D, bool HIST>
cudaError_t launch_fused_gp(const Plan &p, const CUtensorMap &kmap, const FusedArgs &a, cudaStream_t st)
{
    switch (p.fused_gp) {
    case 4: return launch_fused_t<D, 4, HIST>(p, kmap, a, st);
    case 8: return launch_fused_t<D, 8, HIST>(p, kmap, a, st);
    default: return launch_fused_t<D, 16, HIST>(p, kmap, a, st);
    }
}

}  // namespace

cudaError_t launch_score_fused(const Plan &p, const CUtensorMap &kmap_pass, const void *q, const int64_t *seq_off,
                               const int64_t *seq_off_host, const int32_t *reuse, float *votes, uint8_t *ws,
                               cudaStream_t st, const SelectWindow *hist_window)
{
    FusedArgs a;
    for (int b = 0; b <= 32; ++b)
        a.pf_off[b] = (p.B <= 32 && b <= p.B) ? seq_off_host[b] : 0;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.seq_off = seq_off;
    a.reuse = reuse;
    a.logits = reinterpret_cast<float *>(ws + p.off_logits);
    a.ld = p.fused_ld;
    a.partials = reinterpret_cast<float2 *>(ws + p.off_partials);
    a.S = p.fused_grid + p.B;
    a.votes = votes;
    a.vacc = reinterpret_cast<float *>(ws + p.off_vacc);
    a.hist = hist_window != nullptr ? reinterpret_cast<uint32_t *>(ws + p.off_sel_hist) : nullptr;
    a.k = hist_window != nullptr ? hist_window->k : 0;
    a.n_sink = hist_window != nullptr ? hist_window->n_sink : 0;
    a.n_local = hist_window != nullptr ? hist_window->n_local : 0;
    a.bar = reinterpret_cast<uint32_t *>(ws + p.off_ctrl) + kCtrlFusedBarrier;
    a.ctrl = reinterpret_cast<uint32_t *>(ws + p.off_ctrl);
    a.B = p.B;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.HS = p.fused_hs;
    a.T = p.fused_t;
    a.N = p.fused_n;
    a.stage_bytes = kFRows * p.D * 2;
    a.scale = p.scale;
    if (hist_window != nullptr)
        return p.D == 128 ? launch_fused_gp<128, true>(p, kmap_pass, a, st) : launch_fused_gp<64, true>(p, kmap_pass, a, st);
    return p.D == 128 ? launch_fused_gp<128, false>(p, kmap_pass, a, st) : launch_fused_gp<64, false>(p, kmap_pass, a, st);
}

}  // namespace ts
