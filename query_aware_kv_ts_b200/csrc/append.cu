// Appending one token to a growing cache (batch 1, capacity mode): the new
// token's K and V rows are copied to position n = seq_offsets[1] and
// seq_offsets[1] becomes n + 1, all on the device, so that a captured graph
// can append step after step (a decode loop; TokenSelect README, "Key
// Takeaways": the Selection Cache serves consecutive decode steps).
// One block: every thread reads n, copies its 16-byte pieces of both rows,
// and after a barrier one thread publishes the new length.  A full cache
// (n >= capacity) writes nothing and sets the workspace status word to 2.
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads)
append_kernel(int64_t *seq_offsets, __nv_bfloat16 *k_cache, __nv_bfloat16 *v_cache, const uint4 *k_new,
              const uint4 *v_new, int64_t stride_tok, int64_t stride_head, int Hkv, int D, int64_t capacity,
              uint32_t *ctrl)
{
    pdl_wait();   // the previous step's kernels read the offsets and the rows
    const int64_t n = __ldcg(seq_offsets + 1);
    if (n < 0 || n >= capacity) {
        if (threadIdx.x == 0 && atomicCAS(&ctrl[0], 0u, 2u) == 0u)
            atomicExch(&ctrl[1], 0u);
        pdl_launch_dependents();
        return;
    }
    const int per_row = D / 8;   // 16-byte pieces of one head's row
    for (int i = threadIdx.x; i < 2 * Hkv * per_row; i += blockDim.x) {
        const bool isv = i >= Hkv * per_row;
        const int j = isv ? i - Hkv * per_row : i;
        const int g = j / per_row, c = j - g * per_row;
        __nv_bfloat16 *dst = (isv ? v_cache : k_cache) + n * stride_tok + (int64_t)g * stride_head + c * 8;
        *reinterpret_cast<uint4 *>(dst) = (isv ? v_new : k_new)[j];
    }
    __syncthreads();   // every thread has read n before it changes
    if (threadIdx.x == 0)
        seq_offsets[1] = n + 1;
    pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_append(int64_t *seq_offsets, void *k_cache, void *v_cache, const void *k_new, const void *v_new,
                          int64_t stride_tok, int64_t stride_head, int Hkv, int D, int64_t capacity, uint32_t *ctrl,
                          cudaStream_t st)
{
    return launch_ex(append_kernel, dim3(1), dim3(kAppendThreads), 0, st, 1, seq_offsets,
                     static_cast<__nv_bfloat16 *>(k_cache), static_cast<__nv_bfloat16 *>(v_cache),
                     static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), stride_tok, stride_head,
                     Hkv, D, capacity, ctrl);
}

}  // namespace ts
