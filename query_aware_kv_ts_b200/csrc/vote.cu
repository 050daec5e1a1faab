// Score pass B: the soft vote (TokenSelect README, "Key Takeaways": per-head
// criticality normalised by softmax and summed over all heads).
//   votes[i] = sum_h exp(s[h, i] - L[b, h])
// reading the logits written by pass A (L2-resident for moderate n) and the
// float64 log-normalisers L.
//
// Precision: s - L is formed exactly as an unevaluated float pair (two-sum of
// s and the high part of L, minus L's low part), and exp(hi + lo) is taken as
// expf(hi) * (1 + lo) (one fma) with |lo| < 2^-18, so the only rounding left is that of
// expf itself (a few 1e-8 relative).  A plain fp32 subtraction would lose up
// to half an ulp of |s - L| (~1e-6 for |s - L| ~ 20), which is larger than the
// vote band inside which the selection is allowed to differ.
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

struct VoteArgs {
    const float *logits;   // [Hq][ld]
    int64_t ld;
    const double *L;       // [B][Hq]
    const int64_t *seq_off;
    const int32_t *reuse;
    float *votes;
    int B, Hq;
};

constexpr int kMaxHeadsVote = 256;

__global__ void __launch_bounds__(kVoteThreads)
vote_pass_b(const VoteArgs a)
{
    __shared__ int64_t s_off[kMaxBatch + 1];
    __shared__ int32_t s_start[kMaxBatch + 1];
    __shared__ float s_hi[kMaxHeadsVote], s_lo[kMaxHeadsVote];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int B = a.B;
    for (int b = tid; b <= B; b += blockDim.x)
        s_off[b] = a.seq_off[b];
    __syncthreads();
    for (int b = tid; b < B; b += blockDim.x) {
        const int64_t n = s_off[b + 1] - s_off[b];
        const bool active = (a.reuse == nullptr) || (a.reuse[b] == 0);
        s_start[b + 1] = active ? (int32_t)((n + kVoteTokensPerBlock - 1) / kVoteTokensPerBlock) : 0;
    }
    __syncthreads();
    if (warp == 0) {
        int32_t run = 0;
        for (int base = 0; base < B; base += 32) {
            const int b = base + lane;
            int32_t x = (b < B) ? s_start[b + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o)
                    x += y;
            }
            if (b < B)
                s_start[b + 1] = run + x;
            run += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0)
            s_start[0] = 0;
    }
    __syncthreads();
    const int32_t v = blockIdx.x;
    if (v >= s_start[B])
        return;
    const int b = upper_seq(s_start, B, v);
    for (int h = tid; h < a.Hq; h += blockDim.x) {
        const double L = a.L[(int64_t)b * a.Hq + h];
        const float hi = (float)L;
        s_hi[h] = hi;
        s_lo[h] = (float)(L - (double)hi);
    }
    __syncthreads();

    const int64_t base = s_off[b] + (int64_t)(v - s_start[b]) * kVoteTokensPerBlock;
    const int64_t end = min(base + kVoteTokensPerBlock, s_off[b + 1]);
    constexpr int kPer = kVoteTokensPerBlock / kVoteThreads;
    float acc[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j)
        acc[j] = 0.0f;
    for (int h = 0; h < a.Hq; ++h) {
        const float Lhi = s_hi[h], Llo = s_lo[h];
        const float *row = a.logits + (int64_t)h * a.ld;
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int64_t i = base + tid + j * kVoteThreads;
            if (i < end) {
                const float s = __ldcg(row + i);
                // two-sum: t + e == s - Lhi exactly
                const float t = s - Lhi;
                const float bp = t - s;
                const float e = (s - (t - bp)) + (-Lhi - bp);
                const float lo = e - Llo;
                const float et = expf(t);
                acc[j] += fmaf(et, lo, et);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int64_t i = base + tid + j * kVoteThreads;
        if (i < end)
            a.votes[i] = acc[j];
    }
}

}  // namespace

cudaError_t launch_vote(const Plan &p, const int64_t *seq_off, const int32_t *reuse, float *votes, uint8_t *ws,
                        cudaStream_t st)
{
    if (p.max_vote_blocks <= 0)
        return cudaSuccess;
    VoteArgs a;
    a.logits = reinterpret_cast<const float *>(ws + p.off_logits);
    a.ld = p.n_total;
    a.L = reinterpret_cast<const double *>(ws + p.off_L);
    a.seq_off = seq_off;
    a.reuse = reuse;
    a.votes = votes;
    a.B = p.B;
    a.Hq = p.Hq;
    vote_pass_b<<<(unsigned)p.max_vote_blocks, kVoteThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ts
