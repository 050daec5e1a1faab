// Selection Cache decision (TokenSelect README, "Key Takeaways": consecutive
// similar queries share one token selection; GrooveSquid summary: the
// Selection Cache lowers the selection frequency).
// One block per sequence: float64 cosine of the flattened h_q*d query against
// the previous step's query, reuse = !first && cos >= threshold, then the
// current query replaces the previous one.  Each thread overwrites exactly the
// q_prev elements it read, so no barrier is needed between read and write.
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

constexpr int kSelcacheThreads = 256;

__global__ void __launch_bounds__(kSelcacheThreads)
selcache_kernel(const uint32_t *q, uint32_t *q_prev, int32_t *reuse, double *cos_out, int first_step,
                int len_pairs, double theta)
{
    const int b = blockIdx.x;
    const uint32_t *qb = q + (int64_t)b * len_pairs;
    uint32_t *pb = q_prev + (int64_t)b * len_pairs;
    double ab = 0.0, aa = 0.0, bb = 0.0;
    for (int i = threadIdx.x; i < len_pairs; i += blockDim.x) {
        const uint32_t x = qb[i];
        const uint32_t y = pb[i];
        const double x0 = bf16_lo(x), x1 = bf16_hi(x);
        const double y0 = bf16_lo(y), y1 = bf16_hi(y);
        ab += x0 * y0 + x1 * y1;
        aa += x0 * x0 + x1 * x1;
        bb += y0 * y0 + y1 * y1;
        pb[i] = x;
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
    if (threadIdx.x == 0) {
        double sab = 0.0, saa = 0.0, sbb = 0.0;
        for (int w = 0; w < kSelcacheThreads / 32; ++w) {
            sab += red[0][w];
            saa += red[1][w];
            sbb += red[2][w];
        }
        double c = 0.0;
        int r = 0;
        if (!first_step) {
            c = (saa > 0.0 && sbb > 0.0) ? sab / (sqrt(saa) * sqrt(sbb)) : 0.0;
            r = (c >= theta) ? 1 : 0;
        }
        reuse[b] = r;
        if (cos_out)
            cos_out[b] = c;
    }
}

}  // namespace

cudaError_t launch_selcache(const void *q, void *q_prev, int32_t *reuse, double *cos_out, int first_step, int B,
                            int len, double theta, cudaStream_t st)
{
    selcache_kernel<<<B, kSelcacheThreads, 0, st>>>(static_cast<const uint32_t *>(q),
                                                    static_cast<uint32_t *>(q_prev), reuse, cos_out, first_step,
                                                    len / 2, theta);
    return cudaGetLastError();
}

}  // namespace ts
