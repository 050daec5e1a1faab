// Selection Cache decision (TokenSelect README, "Key Takeaways": consecutive
// similar queries share one token selection; GrooveSquid summary: the
// Selection Cache lowers the selection frequency).
// One block per sequence: float64 cosine of the flattened h_q*d query against
// the previous step's query (0 when either vector is zero), reuse = !first &&
// cos >= threshold, then the current query replaces the previous one.  Each
// thread overwrites exactly the q_prev elements it read, so no barrier is
// needed between read and write.
// Replayed from a CUDA graph, the kernel can also switch off the graph's
// scoring and selection (a conditional node) for a step in which every
// sequence reuses its selection: those kernels would only read the flags and
// return.
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

constexpr int kSelcacheThreads = 256;

__global__ void __launch_bounds__(kSelcacheThreads)
selcache_kernel(const uint32_t *__restrict__ q, uint32_t *__restrict__ q_prev, int32_t *reuse, double *cos_out, int first_step,
                int len_pairs, double theta, const SelcacheSkip skip)
{
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.x;
    const uint32_t *__restrict__ qb = q + (int64_t)b * len_pairs;
    uint32_t *__restrict__ pb = q_prev + (int64_t)b * len_pairs;
    // Loads are issued in batches before any store, so that a thread waits
    // on memory once per batch instead of once per element.
    double ab = 0.0, aa = 0.0, bb = 0.0;
    constexpr int kBatch = 8;
    for (int i0 = threadIdx.x; i0 < len_pairs; i0 += kBatch * kSelcacheThreads) {
        uint32_t xs[kBatch], ys[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * kSelcacheThreads;
            xs[u] = i < len_pairs ? __ldcg(qb + i) : 0u;
            ys[u] = i < len_pairs ? __ldcg(pb + i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const double x0 = bf16_lo(xs[u]), x1 = bf16_hi(xs[u]);
            const double y0 = bf16_lo(ys[u]), y1 = bf16_hi(ys[u]);
            ab += x0 * y0 + x1 * y1;
            aa += x0 * x0 + x1 * x1;
            bb += y0 * y0 + y1 * y1;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * kSelcacheThreads;
            if (i < len_pairs)
                pb[i] = xs[u];
        }
    }
    __shared__ double red[3][kSelcacheThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ab += __shfl_xor_sync(0xffffffffu, ab, o);
        aa += __shfl_xor_sync(0xffffffffu, aa, o);
        bb += __shfl_xor_sync(0xffffffffu, bb, o);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red[0][warp] = ab;
        red[1][warp] = aa;
        red[2][warp] = bb;
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int kW = kSelcacheThreads / 32;
        double sab = lane < kW ? red[0][lane] : 0.0;
        double saa = lane < kW ? red[1][lane] : 0.0;
        double sbb = lane < kW ? red[2][lane] : 0.0;
#pragma unroll
        for (int o = kW / 2; o > 0; o >>= 1) {
            sab += __shfl_xor_sync(0xffffffffu, sab, o);
            saa += __shfl_xor_sync(0xffffffffu, saa, o);
            sbb += __shfl_xor_sync(0xffffffffu, sbb, o);
        }
        if (lane != 0)
            return;
        double c = 0.0;
        int r = 0;
        if (!first_step) {
            c = (saa > 0.0 && sbb > 0.0) ? sab / (sqrt(saa) * sqrt(sbb)) : 0.0;
            r = (c >= theta) ? 1 : 0;
        }
        reuse[b] = r;
        if (cos_out)
            cos_out[b] = c;
        if (skip.enabled) {
            // the last block to finish has seen every sequence's decision:
            // when all of them reuse, the graph's scoring and selection are
            // switched off for this replay
            atomicAdd(&skip.counters[0], (uint32_t)r);
            __threadfence();
            if (atomicAdd(&skip.counters[1], 1u) == gridDim.x - 1) {
                __threadfence();
                if (atomicAdd(&skip.counters[0], 0u) == gridDim.x)
                    cudaGraphSetConditional(skip.handle, 0u);
                atomicExch(&skip.counters[0], 0u);   // zero again for the next replay
                atomicExch(&skip.counters[1], 0u);
            }
        }
    }
}

}  // namespace

cudaError_t launch_selcache(const void *q, void *q_prev, int32_t *reuse, double *cos_out, int first_step, int B,
                            int len, double theta, cudaStream_t st, const SelcacheSkip *skip)
{
    SelcacheSkip sk = {};
    if (skip != nullptr)
        sk = *skip;
    return launch_ex(selcache_kernel, dim3((unsigned)B), dim3(kSelcacheThreads), 0, st, 1,
                     static_cast<const uint32_t *>(q), static_cast<uint32_t *>(q_prev), reuse, cos_out, first_step,
                     len / 2, theta, sk);
}

}  // namespace ts
