// Token selection: top-k by soft vote plus the sink and local windows
// (TokenSelect README summary: a small number of critical KV tokens take part
// in attention; the vote ordering with ties to the lower token id).
//
// One thread-block cluster (8 CTAs, 1024 threads each) per sequence.  The
// candidates [s', l0) are split into 8 contiguous ranges, one per CTA.
//
// Exact radix select of the k-th largest vote.  Votes are non-negative fp32,
// so their bit patterns order like the values.  Three digit levels
// (bits 31..20, 19..8, 7..0): each CTA builds a shared-memory histogram of
// its range (restricted to keys matching the digits found so far), the
// cluster reduces it through distributed shared memory (CTA r owns bin slice
// r), and every CTA locates the bin holding the k-th largest key.  After three
// levels the k-th largest key vk is known exactly, together with r = the
// number of tokens equal to vk that belong to the top k (the lowest-id ties).
//
// Ordered compaction: token i of the candidates is selected iff
// key(i) > vk, or key(i) == vk and fewer than r ties precede it.  Per-CTA
// counts exchanged over the cluster give each CTA its output offset; a
// block-wide scan places ids in ascending order.  CTA 0 writes the sink and
// local windows and the count; the tail of the id row is padded with -1.
// Cluster barriers are hardware barriers: there is no software spin here.
#include <cooperative_groups.h>

#include "ts_device.cuh"
#include "ts_internal.h"

namespace cg = cooperative_groups;

namespace ts {
namespace {

constexpr int CS = kSelectClusterSize;
constexpr int NT = kSelectThreads;
constexpr int kWarps = NT / 32;

struct SelectArgs {
    const uint32_t *votes;   // fp32 vote bits [n_total]
    const int64_t *seq_off;
    const int32_t *reuse;
    int32_t *ids;            // [B][cap]
    int32_t *count;          // [B]
    int k, n_sink, n_local, cap;
};

struct SelectShared {
    uint32_t hist[4096];
    uint32_t red[4096 / CS];      // this CTA's cluster-reduced bin slice
    uint32_t rev[4096 / CS];      // copy of the slice holding the target
    uint32_t warp_tmp[kWarps + 1];
    uint32_t slice_total;
    uint32_t cnt[2];              // this CTA's (above, ties)
    uint32_t bcast[4];
};

// Exclusive scan over the block of one value per thread; returns the
// exclusive prefix and sets `total`.  Every thread of the block must call it.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t x, uint32_t *warp_tmp, uint32_t &total)
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
        warp_tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t w = (lane < kWarps) ? warp_tmp[lane] : 0u;
        uint32_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o)
                wi += y;
        }
        if (lane < kWarps)
            warp_tmp[lane] = wi - w;
        if (lane == kWarps - 1)
            warp_tmp[kWarps] = wi;
    }
    __syncthreads();
    const uint32_t excl = warp_tmp[warp] + incl - x;
    total = warp_tmp[kWarps];
    __syncthreads();
    return excl;
}

// Sum over the block; every thread gets the result.
__device__ __forceinline__ uint32_t block_sum(uint32_t x, uint32_t *warp_tmp)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        x += __shfl_xor_sync(0xffffffffu, x, o);
    if ((threadIdx.x & 31) == 0)
        warp_tmp[threadIdx.x >> 5] = x;
    __syncthreads();
    uint32_t t = 0;
    for (int w = 0; w < kWarps; ++w)
        t += warp_tmp[w];
    __syncthreads();
    return t;
}

__global__ void __cluster_dims__(CS, 1, 1) __launch_bounds__(NT, 1)
select_kernel(const SelectArgs a)
{
    __shared__ SelectShared sh;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int b = blockIdx.x / CS;
    const int tid = threadIdx.x;

    if (a.reuse != nullptr && a.reuse[b] != 0)
        return;   // whole cluster: the previous ids stay

    const int64_t off = a.seq_off[b];
    const int64_t n = a.seq_off[b + 1] - off;
    const int64_t s_end = min((int64_t)a.n_sink, n);
    const int64_t l0 = max(n - (int64_t)a.n_local, s_end);
    const int64_t nc = l0 - s_end;
    const int64_t keff = min((int64_t)a.k, nc);
    const uint32_t *vb = a.votes + off;
    const int64_t my_lo = s_end + nc * rank / CS;
    const int64_t my_hi = s_end + nc * (rank + 1) / CS;
    int32_t *idrow = a.ids + (int64_t)b * a.cap;

    // mode 0: radix select, 1: every candidate, 2: none
    const int mode = (keff == nc) ? 1 : (keff == 0 ? 2 : 0);
    uint32_t vk = 0;
    int64_t r_ties = 0;
    uint32_t my_above = 0, my_ties = 0;   // this CTA's keys > vk and == vk

    if (mode == 0) {
        uint32_t prefix = 0, pmask = 0;
        int64_t need = keff;
#pragma unroll 1
        for (int level = 0; level < 3; ++level) {
            const int shift = level == 0 ? 20 : (level == 1 ? 8 : 0);
            const int bins = level == 2 ? 256 : 4096;
            const int W = bins / CS;
            for (int i = tid; i < bins; i += NT)
                sh.hist[i] = 0u;
            __syncthreads();
            for (int64_t i = my_lo + tid; i < my_hi; i += NT) {
                const uint32_t key = __ldcg(vb + i);
                if ((key & pmask) == prefix)
                    atomicAdd(&sh.hist[(key >> shift) & (uint32_t)(bins - 1)], 1u);
            }
            __syncthreads();
            cluster.sync();
            // reduce my slice of bins over the cluster
            uint32_t part = 0;
            for (int j = tid; j < W; j += NT) {
                uint32_t s = 0;
#pragma unroll
                for (int q = 0; q < CS; ++q)
                    s += cluster.map_shared_rank(sh.hist, q)[rank * W + j];
                sh.red[j] = s;
                part += s;
            }
            part = block_sum(part, sh.warp_tmp);
            if (tid == 0)
                sh.slice_total = part;
            cluster.sync();
            // which slice (from the top) holds the need-th largest key?
            if (tid == 0) {
                int64_t cum = 0;
                int sel = 0;
                for (int q = CS - 1; q >= 0; --q) {
                    const uint32_t t = *cluster.map_shared_rank(&sh.slice_total, q);
                    if (cum + (int64_t)t >= need) {
                        sel = q;
                        break;
                    }
                    cum += t;
                }
                sh.bcast[0] = (uint32_t)sel;
                sh.bcast[1] = (uint32_t)cum;
            }
            __syncthreads();
            const int sel = (int)sh.bcast[0];
            const int64_t cum_slices = (int64_t)sh.bcast[1];
            // copy that slice reversed (top bin first) and scan it
            for (int j = tid; j < W; j += NT)
                sh.rev[j] = cluster.map_shared_rank(sh.red, sel)[W - 1 - j];
            __syncthreads();
            const uint32_t c = (tid < W) ? sh.rev[tid] : 0u;
            uint32_t tot;
            const uint32_t ex = block_excl_scan(c, sh.warp_tmp, tot);
            const int64_t before = cum_slices + (int64_t)ex;
            if (tid < W && before < need && before + (int64_t)c >= need) {
                sh.bcast[2] = (uint32_t)(sel * W + (W - 1 - tid));
                sh.bcast[3] = (uint32_t)ex + (uint32_t)cum_slices;
            }
            __syncthreads();
            const uint32_t bin = sh.bcast[2];
            need -= (int64_t)sh.bcast[3];
            prefix |= bin << shift;
            pmask |= (uint32_t)(bins - 1) << shift;
            // my own keys above the chosen bin (and, at the last level, equal to it)
            uint32_t mine = 0;
            for (int j = (int)bin + 1 + tid; j < bins; j += NT)
                mine += sh.hist[j];
            my_above += block_sum(mine, sh.warp_tmp);
            if (level == 2)
                my_ties = sh.hist[bin];
            cluster.sync();   // others are done reading my hist / red / slice_total
        }
        vk = prefix;
        r_ties = need;
    }

    // ---- counts per CTA --------------------------------------------------
    if (mode == 1)
        my_above = (uint32_t)(my_hi - my_lo);
    if (tid == 0) {
        sh.cnt[0] = my_above;
        sh.cnt[1] = my_ties;
    }
    cluster.sync();
    if (tid == 0) {
        int64_t tie_before = 0, sel_before = 0, tb = 0;
        for (int q = 0; q < rank; ++q) {
            const uint32_t *cq = cluster.map_shared_rank(sh.cnt, q);
            const int64_t ca = cq[0], ct = cq[1];
            const int64_t take = max((int64_t)0, min(r_ties - tb, ct));
            sel_before += ca + take;
            tb += ct;
        }
        tie_before = tb;
        sh.bcast[0] = (uint32_t)tie_before;
        sh.bcast[1] = (uint32_t)sel_before;
    }
    cluster.sync();   // every remote read of cnt is done
    const int64_t tie_before = (int64_t)sh.bcast[0];
    const int64_t sel_before = (int64_t)sh.bcast[1];

    // ---- ordered compaction of my range -----------------------------------
    if (mode != 2) {
        int64_t run_ties = 0, run_sel = 0;
        for (int64_t base = my_lo; base < my_hi; base += NT) {
            const int64_t i = base + tid;
            bool is_tie = false, flag = false;
            if (i < my_hi) {
                if (mode == 1) {
                    flag = true;
                } else {
                    const uint32_t key = __ldcg(vb + i);
                    flag = key > vk;
                    is_tie = key == vk;
                }
            }
            if (mode == 0) {
                uint32_t tot;
                const uint32_t ex = block_excl_scan((uint32_t)is_tie, sh.warp_tmp, tot);
                if (is_tie && tie_before + run_ties + (int64_t)ex < r_ties)
                    flag = true;
                run_ties += (int64_t)tot;
            }
            uint32_t tot2;
            const uint32_t pos = block_excl_scan((uint32_t)flag, sh.warp_tmp, tot2);
            const int64_t at = s_end + sel_before + run_sel + (int64_t)pos;
            if (flag && at < s_end + keff)      // never past the top-k part of the row
                idrow[at] = (int32_t)i;
            run_sel += (int64_t)tot2;
        }
    }

    // ---- windows, count and padding (CTA 0) --------------------------------
    if (rank == 0) {
        const int64_t m = s_end + keff + (n - l0);
        for (int64_t i = tid; i < s_end; i += NT)
            idrow[i] = (int32_t)i;
        for (int64_t j = tid; j < n - l0; j += NT)
            idrow[s_end + keff + j] = (int32_t)(l0 + j);
        for (int64_t j = m + tid; j < a.cap; j += NT)
            idrow[j] = -1;
        if (tid == 0)
            a.count[b] = (int32_t)m;
    }
}

}  // namespace

cudaError_t launch_select(const Plan &p, const int64_t *seq_off, const float *votes, int k, int n_sink,
                          int n_local, const int32_t *reuse, int32_t *ids, int32_t *count, cudaStream_t st)
{
    SelectArgs a;
    a.votes = reinterpret_cast<const uint32_t *>(votes);
    a.seq_off = seq_off;
    a.reuse = reuse;
    a.ids = ids;
    a.count = count;
    a.k = k;
    a.n_sink = n_sink;
    a.n_local = n_local;
    a.cap = k + n_sink + n_local;
    select_kernel<<<p.B * CS, NT, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ts
