// Token selection: top-k by soft vote plus the sink and local windows
// (TokenSelect README summary: a small number of critical KV tokens take part
// in attention; the vote ordering with ties to the lower token id).
//
// Order.  Candidate token i of a sequence gets the 64-bit key
//   key(i) = (bits(v_i) << 32) | (0xffffffff - i)
// Votes are non-negative fp32, so their bit patterns order like the values,
// and the low word makes equal votes order by ascending id: the top k keys
// are exactly the top k tokens with ties to the lower id, and "token i is
// selected" is key(i) >= T, T the k-th largest key.
//
// Four short kernels spread over the whole GPU (grid: ranges of kTPC
// candidates x sequences), except the per-sequence resolve step:
//  S0 sel_hist     histogram of the top 12 vote bits of the candidates
//                  (shared-memory histogram per range, then global atomics)
//  S2 sel_collect  every range finds the bin b1 that holds the k-th largest
//                  vote, counts its candidates above b1 and inside b1, and
//                  writes the ones inside b1 to its own slots of the
//                  candidate list (no atomics: slots [r*2048, r*2048 + count))
//  S3 sel_resolve  one CTA per sequence: exact radix select of T among the
//                  (few) b1 candidates, 8-bit digits over the 52 key bits
//                  below b1 until at most 32 keys share the prefix, then one
//                  warp ranks those directly; range offsets = each range's
//                  candidates above b1 plus its b1 candidates >= T,
//                  prefix-summed; clears the histogram for the next call
//  S4 sel_write    every range writes its selected ids in ascending order at
//                  its offset (one block scan); range 0 also writes the sink
//                  and local windows, the count and the -1 padding
// No kernel waits on another CTA: the four steps are ordered by the stream.
// The one-call decode step builds S0's histogram inside the vote pass and
// starts at S2.  Every kernel fetches what it needs in at most two round trips
// (the loads that do not depend on one another are issued together).
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

constexpr int NT = kSelectThreads;          // 256
constexpr int kWarps = NT / 32;
constexpr int kTPC = kSelectTokensPerCta;   // candidates per range (per CTA)
constexpr int kPer = kTPC / NT;             // candidates per thread
constexpr int kResolveSmem = 2560;          // b1 candidates kept in shared memory by S3

struct SelArgs {
    const uint32_t *votes;     // fp32 vote bits [n_total]
    const int64_t *seq_off;
    const int32_t *reuse;
    int32_t *ids;              // [B][cap]
    int32_t *count;            // [B]
    uint32_t *hist;            // [B][4096]
    uint2 *cand;               // [n_total] (vote bits, token id); range r of sequence b at seq_off[b] + r*2048
    uint32_t *inb1;            // [B][rps] candidates inside bin b1, per range
    uint2 *bin;                // [B] (b1, candidates above b1), written by S2
    uint32_t *above;           // [B][rps] candidates above bin b1, per range
    uint32_t *range_off;       // [B][rps] output offset of each range within the top-k part
    unsigned long long *thr;   // [B] threshold key T
    int32_t *mode;             // [B] 0: none, 1: keys >= T, 2: every candidate
    int64_t *prev_n;           // [B] sequence length + 1 when its row was last written (0: never)
    int k, n_sink, n_local, cap, B, rps;
};

struct Window {
    int64_t off, n, s_end, l0, nc, keff;
};

__device__ __forceinline__ Window make_window(const SelArgs &a, int64_t off, int64_t end)
{
    Window w;
    w.off = off;
    w.n = end - off;
    w.s_end = min((int64_t)a.n_sink, w.n);
    w.l0 = max(w.n - (int64_t)a.n_local, w.s_end);
    w.nc = w.l0 - w.s_end;
    w.keff = min((int64_t)a.k, w.nc);
    return w;
}

__device__ __forceinline__ unsigned long long make_key(uint32_t vbits, int64_t id)
{
    return ((unsigned long long)vbits << 32) | (unsigned long long)(0xffffffffu - (uint32_t)id);
}

// The 4096-bin histogram of a sequence: loads into registers (issued
// together), then the copy to shared memory.
constexpr int kHistPer = 4096 / NT;
__device__ __forceinline__ void load_hist_regs(uint32_t (&v)[kHistPer], const uint32_t *gh)
{
#pragma unroll
    for (int u = 0; u < kHistPer; ++u)
        v[u] = __ldcg(gh + u * NT + threadIdx.x);
}
__device__ __forceinline__ void store_hist(uint32_t *h, const uint32_t (&v)[kHistPer])
{
#pragma unroll
    for (int u = 0; u < kHistPer; ++u)
        h[u * NT + threadIdx.x] = v[u];
}

// Exclusive scan over the block of one value per thread (all threads call):
// warp scans, one barrier, then every warp scans the warp totals itself.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t x, uint32_t *tmp, uint32_t &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    if (lane == 31)
        tmp[warp] = incl;
    __syncthreads();
    const uint32_t w = lane < kWarps ? tmp[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < kWarps; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o)
            wi += y;
    }
    const uint32_t before = __shfl_sync(0xffffffffu, wi - w, warp);
    total = __shfl_sync(0xffffffffu, wi, kWarps - 1);
    __syncthreads();   // tmp is rewritten by the next scan
    return before + incl - x;
}

// In the 4096-bin histogram (bin 4095 on top), the bin holding the need-th key
// counted from the top, and the keys above it.  Thread t owns the 16
// consecutive bins 4095-16t .. 4080-16t, kept in registers.  All threads call.
__device__ __forceinline__ void bin_from_top(const uint32_t *h, int64_t need, uint32_t *tmp, uint32_t *bc,
                                             uint32_t &bin, uint32_t &above)
{
    constexpr int kNb = 4096, kOwn = kNb / NT;
    const int top = kNb - 1 - threadIdx.x * kOwn;
    uint32_t c[kOwn];
    uint32_t local = 0;
#pragma unroll
    for (int i = 0; i < kOwn; ++i) {
        c[i] = h[top - i];
        local += c[i];
    }
    uint32_t tot;
    const uint32_t ex = block_excl_scan(local, tmp, tot);
    if ((int64_t)ex < need && (int64_t)ex + local >= need) {
        int64_t cum = ex;
        uint32_t found = 0, at = 0;
        bool done = false;
#pragma unroll
        for (int i = 0; i < kOwn; ++i) {
            if (!done && cum + c[i] >= need) {
                found = (uint32_t)(top - i);
                at = (uint32_t)cum;
                done = true;
            }
            cum += c[i];
        }
        bc[0] = found;
        bc[1] = at;
    }
    __syncthreads();
    bin = bc[0];
    above = bc[1];
}

// ---------------------------------------------------------------------------
// S0: level-1 histogram (top 12 bits) of the candidates
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(NT)
sel_hist(const SelArgs a)
{
    __shared__ uint32_t h[4096];
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.y, r = blockIdx.x;
    const int32_t re = a.reuse != nullptr ? __ldcg(a.reuse + b) : 0;
    const int64_t off = __ldcg(a.seq_off + b), end = __ldcg(a.seq_off + b + 1);
    for (int i = threadIdx.x; i < 4096; i += NT)
        h[i] = 0u;
    if (re != 0)
        return;
    const Window w = make_window(a, off, end);
    const int64_t lo = w.s_end + (int64_t)r * kTPC;
    if (w.keff == 0 || w.keff == w.nc || lo >= w.l0)
        return;
    const int64_t hi = min(lo + kTPC, w.l0);
    const uint32_t *vb = a.votes + w.off;
    uint32_t kk[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int64_t i = lo + u * NT + threadIdx.x;
        kk[u] = i < hi ? __ldcg(vb + i) : 0u;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int64_t i = lo + u * NT + threadIdx.x;
        const uint32_t bin = i < hi ? (kk[u] >> 20) : 0xffffffffu;
        // one atomic for the warp's most common bin, one per lane for the others
        const uint32_t act = __ballot_sync(0xffffffffu, bin != 0xffffffffu);
        if (act) {
            const int leader = __ffs(act) - 1;
            const uint32_t lb = __shfl_sync(0xffffffffu, bin, leader);
            const uint32_t same = __ballot_sync(0xffffffffu, bin == lb);
            if (lane == leader)
                atomicAdd(&h[lb], (uint32_t)__popc(same));
            else if (bin != 0xffffffffu && bin != lb)
                atomicAdd(&h[bin], 1u);
        }
    }
    __syncthreads();
    uint32_t *gh = a.hist + (size_t)b * 4096;
    for (int i = threadIdx.x; i < 4096; i += NT)
        if (h[i] != 0u)
            atomicAdd(&gh[i], h[i]);
}

// ---------------------------------------------------------------------------
// S2: bin b1 of the k-th largest vote; count above it, list the keys in it
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(NT)
sel_collect(const SelArgs a)
{
    __shared__ uint32_t h[4096];
    __shared__ uint32_t tmp[kWarps + 1];
    __shared__ uint32_t bc[2];
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.y, r = blockIdx.x;
    // round trip 1: flag, bounds and the sequence's histogram
    const int32_t re = a.reuse != nullptr ? __ldcg(a.reuse + b) : 0;
    const int64_t off = __ldcg(a.seq_off + b), end = __ldcg(a.seq_off + b + 1);
    uint32_t hv[kHistPer];
    load_hist_regs(hv, a.hist + (size_t)b * 4096);
    if (re != 0)
        return;
    const Window w = make_window(a, off, end);
    const int64_t lo = w.s_end + (int64_t)r * kTPC;
    if (w.keff == 0 || w.keff == w.nc || lo >= w.l0)
        return;
    const int64_t hi = min(lo + kTPC, w.l0);
    // round trip 2: the range's votes
    const uint32_t *vb = a.votes + w.off;
    uint32_t kk[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int64_t i = lo + u * NT + threadIdx.x;
        kk[u] = i < hi ? __ldcg(vb + i) : 0u;
    }
    store_hist(h, hv);
    __syncthreads();
    uint32_t b1, above_b1;
    bin_from_top(h, w.keff, tmp, bc, b1, above_b1);
    if (r == 0 && threadIdx.x == 0)
        a.bin[b] = make_uint2(b1, above_b1);   // every range finds the same b1

    uint32_t mine_above = 0, mine_in = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int64_t i = lo + u * NT + threadIdx.x;
        const bool valid = i < hi;
        const uint32_t bin = kk[u] >> 20;
        mine_above += (valid && bin > b1) ? 1u : 0u;
        mine_in += (valid && bin == b1) ? 1u : 0u;
    }
    // one scan of both counts (each total <= 2048, so the low field never carries)
    uint32_t tot;
    const uint32_t ex = block_excl_scan((mine_above << 16) | mine_in, tmp, tot);
    uint2 *cl = a.cand + w.off + (lo - w.s_end);
    uint32_t pos = ex & 0xffffu;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int64_t i = lo + u * NT + threadIdx.x;
        if (i < hi && (kk[u] >> 20) == b1)
            cl[pos++] = make_uint2(kk[u], (uint32_t)i);
    }
    if (threadIdx.x == 0) {
        a.above[(size_t)b * a.rps + r] = tot >> 16;
        a.inb1[(size_t)b * a.rps + r] = tot & 0xffffu;
    }
}

// ---------------------------------------------------------------------------
// S3: exact threshold among the b1 candidates; per-range offsets
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(NT)
sel_resolve(const SelArgs a)
{
    constexpr int kAbovePer = kMaxSelectRanges / NT;   // per-range counts held per thread
    __shared__ uint32_t h[NT];                         // one digit's histogram (<= 256 bins)
    __shared__ uint32_t tmp[kWarps + 1];
    __shared__ uint32_t bc[3];
    __shared__ unsigned long long keys[kResolveSmem];
    __shared__ uint32_t rcnt[kMaxSelectRanges];
    __shared__ unsigned long long s_list[32];
    __shared__ uint32_t s_nlist;
    __shared__ unsigned long long s_T;
    __shared__ uint32_t s_rstart[kMaxSelectRanges + 1];   // first list index of each range
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.x;
    // round trip 1: flag, bounds, b1 with the count above it, and the
    // per-range counts above and inside b1
    const int32_t re = a.reuse != nullptr ? __ldcg(a.reuse + b) : 0;
    const int64_t off = __ldcg(a.seq_off + b), end = __ldcg(a.seq_off + b + 1);
    const uint2 bn = __ldcg(&a.bin[b]);
    uint32_t ab[kAbovePer], ib[kAbovePer];
#pragma unroll
    for (int u = 0; u < kAbovePer; ++u) {
        const int r = u * NT + threadIdx.x;
        ab[u] = r < a.rps ? __ldcg(&a.above[(size_t)b * a.rps + r]) : 0u;
        ib[u] = r < a.rps ? __ldcg(&a.inb1[(size_t)b * a.rps + r]) : 0u;
    }
    if (re != 0)
        return;
    const Window w = make_window(a, off, end);
    const int nranges = (int)((w.nc + kTPC - 1) / kTPC);
    if (w.keff == 0 || w.keff == w.nc) {
        if (threadIdx.x == 0) {
            a.mode[b] = w.keff == 0 ? 0 : 2;
            a.thr[b] = 0ull;
        }
        // every candidate selected: range r starts at r * kTPC
        for (int r = threadIdx.x; r < nranges; r += NT)
            a.range_off[(size_t)b * a.rps + r] = w.keff == 0 ? 0u : (uint32_t)((int64_t)r * kTPC);
        return;
    }
    uint32_t *gh = a.hist + (size_t)b * 4096;
    for (int i = threadIdx.x; i < 4096; i += NT)
        gh[i] = 0u;                                  // ready for the next call
    // list index of each range's first b1 candidate
    uint32_t m = 0;
#pragma unroll
    for (int u = 0; u < kAbovePer; ++u) {
        if (u * NT >= nranges)
            break;
        const int r = u * NT + threadIdx.x;
        uint32_t tot;
        const uint32_t ex = block_excl_scan(r < nranges ? ib[u] : 0u, tmp, tot);
        if (r < nranges)
            s_rstart[r] = m + ex;
        m += tot;
    }
    if (threadIdx.x == 0) {
        s_rstart[nranges] = m;
        s_nlist = 0u;
    }
    __syncthreads();
    // candidate j of the list: range r with s_rstart[r] <= j < s_rstart[r+1]
    const uint2 *cl = a.cand + w.off;
    auto addr_of = [&](uint32_t j) -> const uint2 * {
        int lo_r = 0, hi_r = nranges;
        while (hi_r - lo_r > 1) {
            const int mid = (lo_r + hi_r) >> 1;
            if (s_rstart[mid] <= j)
                lo_r = mid;
            else
                hi_r = mid;
        }
        return cl + (int64_t)lo_r * kTPC + (j - s_rstart[lo_r]);
    };
    // round trip 2: the b1 candidates
    const bool in_smem = m <= (uint32_t)kResolveSmem;
    if (in_smem) {
        constexpr int kBatch = 10;                   // kResolveSmem / NT
        for (uint32_t j0 = threadIdx.x; j0 < m; j0 += kBatch * NT) {
            uint2 c[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u)
                c[u] = j0 + u * NT < m ? __ldcg(addr_of(j0 + u * NT)) : make_uint2(0u, 0u);
#pragma unroll
            for (int u = 0; u < kBatch; ++u)
                if (j0 + u * NT < m)
                    keys[j0 + u * NT] = make_key(c[u].x, c[u].y);
        }
    }
    __syncthreads();
    auto key_at = [&](uint32_t j) -> unsigned long long {
        if (in_smem)
            return keys[j];
        const uint2 c = __ldcg(addr_of(j));
        return make_key(c.x, c.y);
    };

    // radix select of the need-th largest key among the m candidates: they
    // share the top 12 bits (b1); 8-bit digits over bits 51..4, then 3..0,
    // while more than 32 keys share the prefix found so far
    int64_t need = (int64_t)w.keff - bn.y;
    unsigned long long prefix = (unsigned long long)bn.x << 52;
    unsigned long long pmask = 0xfffull << 52;
    uint32_t alive = m;
    for (int shift = 44; alive > 32u && shift >= -4; shift -= 8) {
        const int sh = shift < 0 ? 0 : shift;
        const int nb = shift < 0 ? 16 : 256;
        h[threadIdx.x] = 0u;
        __syncthreads();
        for (uint32_t j = threadIdx.x; j < m; j += NT) {
            const unsigned long long key = key_at(j);
            if ((key & pmask) == prefix)
                atomicAdd(&h[(uint32_t)(key >> sh) & (uint32_t)(nb - 1)], 1u);
        }
        __syncthreads();
        const int t = threadIdx.x;
        const uint32_t c = t < nb ? h[nb - 1 - t] : 0u;
        uint32_t tot;
        const uint32_t ex = block_excl_scan(c, tmp, tot);
        if (t < nb && (int64_t)ex < need && (int64_t)(ex + c) >= need) {
            bc[0] = (uint32_t)(nb - 1 - t);
            bc[1] = ex;
            bc[2] = c;
        }
        __syncthreads();
        const uint32_t dig = bc[0];
        need -= bc[1];
        alive = bc[2];
        __syncthreads();
        prefix |= (unsigned long long)dig << sh;
        pmask |= (unsigned long long)(nb - 1) << sh;
    }
    unsigned long long T;
    if (pmask == ~0ull) {
        T = prefix;   // every bit resolved: the one key left
    } else {
        // at most 32 keys share the prefix (keys are distinct): list them and
        // let one warp rank them against each other
        for (uint32_t j = threadIdx.x; j < m; j += NT) {
            const unsigned long long key = key_at(j);
            if ((key & pmask) == prefix) {
                const uint32_t pos = atomicAdd(&s_nlist, 1u);
                if (pos < 32u)
                    s_list[pos] = key;
            }
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            const uint32_t c = min(s_nlist, 32u);
            const unsigned long long mine = lane < (int)c ? s_list[lane] : 0ull;
            uint32_t rank = 0;
#pragma unroll
            for (int l = 0; l < 32; ++l) {
                const unsigned long long o = __shfl_sync(0xffffffffu, mine, l);
                rank += (l < (int)c && o > mine) ? 1u : 0u;
            }
            if (lane < (int)c && (int64_t)rank == need - 1)
                s_T = mine;
        }
        __syncthreads();
        T = s_T;
    }

    // per-range counts of selected b1 candidates, then range offsets
    for (int r = threadIdx.x; r < nranges; r += NT)
        rcnt[r] = 0u;
    __syncthreads();
    for (uint32_t j = threadIdx.x; j < m; j += NT) {
        const unsigned long long key = key_at(j);
        if (key >= T) {
            const uint32_t id = 0xffffffffu - (uint32_t)(key & 0xffffffffull);
            atomicAdd(&rcnt[(id - (uint32_t)w.s_end) / kTPC], 1u);
        }
    }
    __syncthreads();
    uint32_t run = 0;
#pragma unroll
    for (int u = 0; u < kAbovePer; ++u) {
        if (u * NT >= nranges)
            break;
        const int r = u * NT + threadIdx.x;
        const uint32_t c = r < nranges ? ab[u] + rcnt[r] : 0u;
        uint32_t tot;
        const uint32_t ex = block_excl_scan(c, tmp, tot);
        if (r < nranges)
            a.range_off[(size_t)b * a.rps + r] = run + ex;
        run += tot;
    }
    if (threadIdx.x == 0) {
        a.thr[b] = T;
        a.mode[b] = 1;
    }
}

// ---------------------------------------------------------------------------
// S4: ordered write of the selected ids; windows, count and padding
// ---------------------------------------------------------------------------
// A sequence that reuses its selection keeps its row unless its length
// changed since the row was written (a cache that grows between decode
// steps).  Then the row becomes: the sink window of the new length, the kept
// top-k part (the old row's ids inside both the old and the new candidate
// ranges), the local window of the new length, -1 padding; the count follows.
// The old row is ascending, so the kept ids are one contiguous run of it; they
// are staged in the sequence's candidate-list slots (unused in a reused step)
// before the row is rewritten in place.  One block, all threads.
__device__ void rewrite_reused_row(const SelArgs &a, int b, int64_t off, int64_t end)
{
    __shared__ uint32_t s_cnt[2];
    const int64_t n_new = end - off;
    const int64_t pn = __ldcg(&a.prev_n[b]);
    if (pn == 0 || pn - 1 == n_new) {   // unknown or unchanged length: the row stays
        if (threadIdx.x == 0)
            a.prev_n[b] = n_new + 1;
        return;
    }
    const Window wo = make_window(a, off, off + (pn - 1));
    const Window wn = make_window(a, off, end);
    int32_t *row = a.ids + (int64_t)b * a.cap;
    const int m_old = max(0, min(__ldcg(a.count + b), a.cap));
    const int64_t lo_id = max(wo.s_end, wn.s_end), hi_id = min(wo.l0, wn.l0);
    if (threadIdx.x < 2)
        s_cnt[threadIdx.x] = 0u;
    __syncthreads();
    uint32_t below_lo = 0, below_hi = 0;
    for (int j = threadIdx.x; j < m_old; j += NT) {
        const int32_t id = __ldcg(row + j);
        below_lo += (id < lo_id) ? 1u : 0u;
        below_hi += (id < hi_id) ? 1u : 0u;
    }
    atomicAdd(&s_cnt[0], below_lo);
    atomicAdd(&s_cnt[1], below_hi);
    __syncthreads();
    const int j0 = (int)s_cnt[0];
    const int nt = hi_id > lo_id ? min((int)s_cnt[1] - j0, a.k) : 0;   // at most the top-k part
    uint32_t *stage = reinterpret_cast<uint32_t *>(a.cand + off);   // n_new >= nt slots of 8 bytes
    for (int t = threadIdx.x; t < nt; t += NT)
        stage[t] = (uint32_t)__ldcg(row + j0 + t);
    __syncthreads();
    const int64_t m_new = wn.s_end + nt + (wn.n - wn.l0);
    for (int64_t i = threadIdx.x; i < wn.s_end; i += NT)
        row[i] = (int32_t)i;
    for (int t = threadIdx.x; t < nt; t += NT)
        row[wn.s_end + t] = (int32_t)__ldcg(stage + t);
    for (int64_t j = threadIdx.x; j < wn.n - wn.l0; j += NT)
        row[wn.s_end + nt + j] = (int32_t)(wn.l0 + j);
    for (int64_t j = m_new + threadIdx.x; j < a.cap; j += NT)
        row[j] = -1;
    if (threadIdx.x == 0) {
        a.count[b] = (int32_t)m_new;
        a.prev_n[b] = n_new + 1;
    }
}

__global__ void __launch_bounds__(NT)
sel_write(const SelArgs a)
{
    __shared__ uint32_t tmp[kWarps + 1];
    __shared__ __align__(16) uint32_t sv[kTPC];
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.y, r = blockIdx.x;
    // round trip 1: flag, bounds, mode, threshold and this range's offset
    const int32_t re = a.reuse != nullptr ? __ldcg(a.reuse + b) : 0;
    const int64_t off = __ldcg(a.seq_off + b), end = __ldcg(a.seq_off + b + 1);
    const int md = __ldcg(&a.mode[b]);
    const unsigned long long T = __ldcg(&a.thr[b]);
    const uint32_t base = r < a.rps ? __ldcg(&a.range_off[(size_t)b * a.rps + r]) : 0u;
    if (re != 0) {
        if (r == 0)
            rewrite_reused_row(a, b, off, end);   // the previous row, with the windows of a grown cache
        return;
    }
    const Window w = make_window(a, off, end);
    int32_t *idrow = a.ids + (int64_t)b * a.cap;
    if (r == 0) {
        if (threadIdx.x == 0)
            a.prev_n[b] = w.n + 1;
        const int64_t mcount = w.s_end + w.keff + (w.n - w.l0);
        for (int64_t i = threadIdx.x; i < w.s_end; i += NT)
            idrow[i] = (int32_t)i;
        for (int64_t j = threadIdx.x; j < w.n - w.l0; j += NT)
            idrow[w.s_end + w.keff + j] = (int32_t)(w.l0 + j);
        for (int64_t j = mcount + threadIdx.x; j < a.cap; j += NT)
            idrow[j] = -1;
        if (threadIdx.x == 0)
            a.count[b] = (int32_t)mcount;
    }
    const int64_t lo = w.s_end + (int64_t)r * kTPC;
    if (lo >= w.l0 || md == 0)
        return;
    const int64_t hi = min(lo + kTPC, w.l0);
    // round trip 2: the range's votes, loaded coalesced and regrouped through
    // shared memory so that each thread owns kPer consecutive candidates
    const uint32_t *vb = a.votes + w.off;
    {
        uint32_t v[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int64_t i = lo + u * NT + threadIdx.x;
            v[u] = i < hi ? __ldcg(vb + i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u)
            sv[u * NT + threadIdx.x] = v[u];
    }
    __syncthreads();
    const int64_t t0 = lo + (int64_t)threadIdx.x * kPer;
    const uint4 va = *reinterpret_cast<const uint4 *>(sv + threadIdx.x * kPer);
    const uint4 vc = *reinterpret_cast<const uint4 *>(sv + threadIdx.x * kPer + 4);
    const uint32_t mv[kPer] = {va.x, va.y, va.z, va.w, vc.x, vc.y, vc.z, vc.w};
    bool f[kPer];
    uint32_t cnt = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int64_t i = t0 + u;
        f[u] = i < hi && (md == 2 || make_key(mv[u], i) >= T);
        cnt += f[u] ? 1u : 0u;
    }
    uint32_t tot;
    uint32_t pos = block_excl_scan(cnt, tmp, tot);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        if (f[u]) {
            const int64_t at = w.s_end + (int64_t)base + pos;
            if (at < w.s_end + w.keff)   // never past the top-k part of the row
                idrow[at] = (int32_t)(t0 + u);
            ++pos;
        }
    }
}

}  // namespace

cudaError_t launch_select(const Plan &p, const int64_t *seq_off, const float *votes, int k, int n_sink,
                          int n_local, const int32_t *reuse, int32_t *ids, int32_t *count, uint8_t *ws,
                          cudaStream_t st, bool hist_ready)
{
    SelArgs a;
    a.votes = reinterpret_cast<const uint32_t *>(votes);
    a.seq_off = seq_off;
    a.reuse = reuse;
    a.ids = ids;
    a.count = count;
    a.hist = reinterpret_cast<uint32_t *>(ws + p.off_sel_hist);
    a.cand = reinterpret_cast<uint2 *>(ws + p.off_sel_cand);
    a.inb1 = reinterpret_cast<uint32_t *>(ws + p.off_sel_inb1);
    a.bin = reinterpret_cast<uint2 *>(ws + p.off_sel_bin);
    a.above = reinterpret_cast<uint32_t *>(ws + p.off_sel_above);
    a.range_off = reinterpret_cast<uint32_t *>(ws + p.off_sel_range_off);
    a.thr = reinterpret_cast<unsigned long long *>(ws + p.off_sel_thr);
    a.mode = reinterpret_cast<int32_t *>(ws + p.off_sel_mode);
    a.prev_n = reinterpret_cast<int64_t *>(ws + p.off_sel_prev_n);
    a.k = k;
    a.n_sink = n_sink;
    a.n_local = n_local;
    a.cap = k + n_sink + n_local;
    a.B = p.B;
    a.rps = p.sel_ranges;
    const dim3 grid((unsigned)p.sel_ranges, (unsigned)p.B);
    cudaError_t e = hist_ready ? cudaSuccess : launch_ex(sel_hist, grid, dim3(NT), 0, st, 1, a);
    if (e == cudaSuccess)
        e = launch_ex(sel_collect, grid, dim3(NT), 0, st, 1, a);
    if (e == cudaSuccess)
        e = launch_ex(sel_resolve, dim3((unsigned)p.B), dim3(NT), 0, st, 1, a);
    if (e == cudaSuccess)
        e = launch_ex(sel_write, grid, dim3(NT), 0, st, 1, a);
    return e;
}

}  // namespace ts
