// Token-axis split of one sequence across ranks: each rank holds a contiguous
// shard [t_r, t_r + n_r) of the sequence's tokens and runs the decode step's
// phases on it; three small exchanges join them (the collectives themselves
// are the caller's, e.g. NCCL all-gathers):
//   1. each head's log-normaliser: the shards' L_h^r are combined by
//      log-sum-exp into the sequence's L_h (the soft vote's softmax is over
//      all n tokens, TokenSelect README, "Key Takeaways" (2));
//   2. the top-k: each rank's k best candidates, as keys (vote bits, global
//      id) ordered by vote and then by lower id, are gathered; the k-th
//      largest of all of them is the sequence's threshold, and each rank
//      keeps its own candidates at or above it;
//   3. the attention: each rank attends over its own selected tokens and
//      reports each head's output and log-sum-exp; the outputs are combined
//      with weights exp(lse_r - LSE).
// These kernels are the arithmetic of the joins; the phases themselves are
// the single-GPU kernels run on the shard.
#include <math.h>

#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {

namespace {

constexpr int kJoinThreads = 256;
constexpr int kSelMergeThreads = 1024;
constexpr int kSelMergeBins = 2048;   // 11-bit digits of the 64-bit keys
constexpr int kSelMergeBatch = 8;     // keys a thread loads per round trip

// L = log(sum_r exp(L_r)) per entry, in float64 (an entry of -inf is a shard
// with no tokens).
__global__ void __launch_bounds__(kJoinThreads)
merge_normalisers(const double *L_parts, int parts, int64_t count, double *L_out)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= count)
        return;
    double M = -INFINITY;
    for (int r = 0; r < parts; ++r)
        M = fmax(M, L_parts[(int64_t)r * count + i]);
    if (M == -INFINITY) {
        L_out[i] = -INFINITY;
        return;
    }
    double z = 0.0;
    for (int r = 0; r < parts; ++r)
        z += exp(L_parts[(int64_t)r * count + i] - M);
    L_out[i] = M + log(z);
}

// The rank's top-k candidates as keys: ids[s_loc, s_loc + t) of its row are
// its chosen candidates (ascending), t = count - s_loc - l_loc; key = (vote
// bits << 32) | (2^32 - 1 - global id), so that a larger key is a larger
// vote, or the lower id of two equal votes; 0 pads the list to kcap.
__global__ void __launch_bounds__(kJoinThreads)
candidate_keys(const float *votes, const int32_t *ids, const int32_t *count, int s_loc, int l_loc,
               int64_t shard_offset, int kcap, unsigned long long *keys)
{
    const int t = max(0, __ldcg(count) - s_loc - l_loc);
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < kcap; j += gridDim.x * blockDim.x) {
        unsigned long long key = 0ull;
        if (j < t) {
            const int32_t id = __ldcg(ids + s_loc + j);
            const uint32_t vb = __float_as_uint(__ldcg(votes + id));
            key = ((unsigned long long)vb << 32) | (unsigned long long)(0xffffffffu - (uint32_t)(shard_offset + id));
        }
        keys[j] = key;
    }
}

__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_sums, uint32_t *total)
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
        warp_sums[lane] = s;
    }
    __syncthreads();
    const uint32_t before = (warp > 0 ? warp_sums[warp - 1] : 0u) + x - v;
    *total = warp_sums[nw - 1];
    __syncthreads();
    return before;
}

// The sequence's threshold and this rank's row.  keys: [parts][kcap] (every
// rank's list, this rank's at `rank`, ascending by id); k: the sequence's
// budget.  T: a key such that exactly k keys are >= T (a radix select over
// the 64-bit keys, six digits at most), or 1 when there are at most k nonzero
// keys (every one is chosen).  The
// row: the shard's sink part [0, s_loc), its own keys >= T (as shard-local
// ids, ascending), its local-window part [n_loc - l_loc, n_loc); -1 after.
__global__ void __launch_bounds__(kSelMergeThreads)
select_merge(const unsigned long long *keys, int parts, int kcap, int k, int rank, int s_loc, int l_loc,
             int64_t n_loc, int64_t shard_offset, int cap, int32_t *ids, int32_t *count)
{
    __shared__ uint32_t hist[kSelMergeBins];
    __shared__ uint32_t warp_sums[32];
    __shared__ uint32_t s_digit, s_above, s_bin, s_nonzero;
    const int tid = threadIdx.x;
    const int64_t total = (int64_t)parts * kcap;
    for (int i = tid; i < kSelMergeBins; i += blockDim.x)
        hist[i] = 0u;
    if (tid == 0)
        s_nonzero = 0u;
    __syncthreads();
    unsigned long long prefix = 0ull, pmask = 0ull;
    uint32_t nz = 0u;
    // Histogram of the digit (key >> sh) & dmask of the nonzero keys under the
    // current prefix, counting the nonzero keys too when asked.  The keys are
    // read in trips of kSelMergeBatch independent loads per thread (one memory
    // round trip per trip, not per key), with the same loop bounds for the
    // whole block (the warp-wide match needs every lane); a warp adds each
    // distinct digit once with its multiplicity: the high digits of the top
    // candidates' votes fall into a few bins, on which one shared atomic per
    // lane would serialise.
    auto histogram = [&](int sh, uint32_t dmask, bool count_nonzero) {
        const int64_t per_trip = (int64_t)blockDim.x * kSelMergeBatch;
        for (int64_t base = 0; base < total; base += per_trip) {
            unsigned long long kk[kSelMergeBatch];
#pragma unroll
            for (int u = 0; u < kSelMergeBatch; ++u) {
                const int64_t i = base + (int64_t)u * blockDim.x + tid;
                kk[u] = i < total ? __ldcg(keys + i) : 0ull;
            }
#pragma unroll
            for (int u = 0; u < kSelMergeBatch; ++u) {
                if (count_nonzero)
                    nz += kk[u] != 0ull ? 1u : 0u;
                const bool take = kk[u] != 0ull && (kk[u] & pmask) == prefix;
                const uint32_t bin = take ? (uint32_t)(kk[u] >> sh) & dmask : 0xffffffffu;
                const unsigned grp = __match_any_sync(0xffffffffu, bin);
                if (take && __ffs(grp) - 1 == (int)(tid & 31))
                    atomicAdd(&hist[bin], (uint32_t)__popc(grp));
            }
        }
    };
    // the first digit's histogram in the same trips as the count
    histogram(53, 0x7ffu, true);
    nz = __reduce_add_sync(0xffffffffu, nz);
    if ((tid & 31) == 0)
        atomicAdd(&s_nonzero, nz);
    __syncthreads();
    const uint32_t real = s_nonzero;
    unsigned long long T = 1ull;   // at most k keys: every nonzero key
    if (real > (uint32_t)k && k > 0) {
        // the k-th largest key lies among the nonzero ones: digits from the
        // top, until the chosen digit's bin holds exactly the keys still
        // needed (then every key under the prefix is chosen and the prefix
        // with its lower bits 0 is the threshold), at the latest at the last
        // digit (keys are distinct: its bin holds the k-th key alone)
        uint32_t above = 0u;
        for (int pass = 0; pass < 6; ++pass) {
            const int sh = pass < 5 ? 53 - 11 * pass : 0;
            const int width = pass < 5 ? 11 : 9;
            const uint32_t dmask = (1u << width) - 1u;
            if (pass > 0) {
                for (int i = tid; i < kSelMergeBins; i += blockDim.x)
                    hist[i] = 0u;
                __syncthreads();
                histogram(sh, dmask, false);
                __syncthreads();
            }
            const int top = (int)dmask;
            const int d1 = top - 2 * tid, d2 = d1 - 1;
            const uint32_t h1 = d1 >= 0 ? hist[d1] : 0u, h2 = d2 >= 0 ? hist[d2] : 0u;
            uint32_t tot;
            const uint32_t before = above + block_exclusive_scan(h1 + h2, warp_sums, &tot);
            if (d1 >= 0 && before < (uint32_t)k && before + h1 >= (uint32_t)k) {
                s_digit = (uint32_t)d1;
                s_above = before;
                s_bin = h1;
            } else if (d2 >= 0 && before + h1 < (uint32_t)k && before + h1 + h2 >= (uint32_t)k) {
                s_digit = (uint32_t)d2;
                s_above = before + h1;
                s_bin = h2;
            }
            __syncthreads();
            prefix |= (unsigned long long)s_digit << sh;
            pmask |= (unsigned long long)dmask << sh;
            above = s_above;
            const bool whole_bin = s_above + s_bin == (uint32_t)k;
            __syncthreads();
            if (whole_bin)
                break;
        }
        T = prefix;   // exactly k keys are >= T
    } else if (k == 0) {
        T = ~0ull;    // nothing chosen (no key reaches it: the id field is never all ones)
    }
    // this rank's keys >= T, in order: contiguous ranges per thread
    const unsigned long long *own = keys + (int64_t)rank * kcap;
    const int per = (kcap + blockDim.x - 1) / blockDim.x;
    const int c0 = tid * per, c1 = min(c0 + per, kcap);
    uint32_t mine = 0u;
    for (int c = c0; c < c1; ++c) {
        const unsigned long long key = __ldcg(own + c);
        mine += (key != 0ull && key >= T) ? 1u : 0u;
    }
    uint32_t chosen;
    uint32_t pos = (uint32_t)s_loc + block_exclusive_scan(mine, warp_sums, &chosen);
    for (int c = c0; c < c1; ++c) {
        const unsigned long long key = __ldcg(own + c);
        if (key != 0ull && key >= T) {
            const uint32_t gid = 0xffffffffu - (uint32_t)(key & 0xffffffffull);
            ids[pos++] = (int32_t)((int64_t)gid - shard_offset);
        }
    }
    const int64_t m = s_loc + (int64_t)chosen + l_loc;
    for (int64_t i = tid; i < s_loc; i += blockDim.x)
        ids[i] = (int32_t)i;
    for (int64_t i = tid; i < l_loc; i += blockDim.x)
        ids[s_loc + chosen + i] = (int32_t)(n_loc - l_loc + i);
    for (int64_t i = m + tid; i < cap; i += blockDim.x)
        ids[i] = -1;
    if (tid == 0)
        *count = (int32_t)m;
}

// out = sum_r exp(lse_r - LSE) * o_r, LSE = log(sum_r exp(lse_r)), per (row,
// channel); rows with every lse -inf (no selected token anywhere) are 0.
__global__ void __launch_bounds__(kJoinThreads)
merge_attention(const float *o_parts, const float *lse_parts, int parts, int64_t rows, int d, float *out)
{
    const int64_t row = blockIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < parts; ++r)
        M = fmaxf(M, lse_parts[(int64_t)r * rows + row]);
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float acc = 0.0f, z = 0.0f;
        if (M != -INFINITY) {
            for (int r = 0; r < parts; ++r) {
                const float l = lse_parts[(int64_t)r * rows + row];
                if (l == -INFINITY)
                    continue;
                const float w = expf(l - M);
                z += w;
                acc = fmaf(w, o_parts[((int64_t)r * rows + row) * d + c], acc);
            }
        }
        out[row * d + c] = z > 0.0f ? acc / z : 0.0f;
    }
}

}  // namespace

cudaError_t launch_merge_normalisers(const double *L_parts, int parts, int64_t count, double *L_out, cudaStream_t st)
{
    if (count <= 0)
        return cudaSuccess;
    merge_normalisers<<<(unsigned)((count + kJoinThreads - 1) / kJoinThreads), kJoinThreads, 0, st>>>(
        L_parts, parts, count, L_out);
    return cudaGetLastError();
}

cudaError_t launch_candidate_keys(const float *votes, const int32_t *ids, const int32_t *count, int s_loc, int l_loc,
                                  int64_t shard_offset, int kcap, unsigned long long *keys, cudaStream_t st)
{
    const int blocks = (kcap + kJoinThreads - 1) / kJoinThreads;
    candidate_keys<<<blocks > 0 ? blocks : 1, kJoinThreads, 0, st>>>(votes, ids, count, s_loc, l_loc, shard_offset,
                                                                    kcap, keys);
    return cudaGetLastError();
}

cudaError_t launch_select_merge(const unsigned long long *keys, int parts, int kcap, int k, int rank, int s_loc,
                                int l_loc, int64_t n_loc, int64_t shard_offset, int cap, int32_t *ids,
                                int32_t *count, cudaStream_t st)
{
    select_merge<<<1, kSelMergeThreads, 0, st>>>(keys, parts, kcap, k, rank, s_loc, l_loc, n_loc, shard_offset, cap,
                                                ids, count);
    return cudaGetLastError();
}

cudaError_t launch_merge_attention(const float *o_parts, const float *lse_parts, int parts, int64_t rows, int d,
                                   float *out, cudaStream_t st)
{
    if (rows <= 0)
        return cudaSuccess;
    merge_attention<<<(unsigned)rows, 128, 0, st>>>(o_parts, lse_parts, parts, rows, d, out);
    return cudaGetLastError();
}

}  // namespace ts
