// Attention over the selected tokens (TokenSelect README summary: a small
// number of critical KV cache tokens take part in the attention calculation).
//   out[b, h, :] = sum_j softmax_j(scale * q_h . K[ids_j, g]) * V[ids_j, g]
//
// Split-K decode attention: grid (splits, h_kv, B).  Each CTA takes a slice of
// one sequence's selected ids for one KV head g and serves all G query heads
// of g from the same gathered K/V rows, so each selected row is read from HBM
// once.  Warps take rows round-robin; a lane holds d/32 channels of the row,
// the G dot products are finished with warp butterflies, and every warp keeps
// an online softmax (max, sum, weighted V) per head.  The CTA merges its warps
// and writes one partial per (split, head); the CTA that completes the last
// split of (b, g) (atomic ticket, no waiting) merges the splits into out.
#include <mutex>

#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kAttnWarps = kAttnThreads / 32;

struct AttnArgs {
    const __nv_bfloat16 *k, *v;
    int64_t st, sh;
    const __nv_bfloat16 *q;
    const int64_t *seq_off;
    const int32_t *ids;
    const int32_t *count;
    int cap;
    float *out;
    float *part;        // [B][Hkv][splits][G][D + 2]
    uint32_t *tickets;  // [B][Hkv]
    int B, Hq, Hkv, G, splits;
    float scale_log2;   // scale * log2(e): logits in base-2 units
};

template <int CPL>
struct RowLoad;
template <>
struct RowLoad<4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&f)[4])
    {
        const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
        f[0] = bf16_lo(w.x);
        f[1] = bf16_hi(w.x);
        f[2] = bf16_lo(w.y);
        f[3] = bf16_hi(w.y);
    }
};
template <>
struct RowLoad<2> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&f)[2])
    {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(p));
        f[0] = bf16_lo(w);
        f[1] = bf16_hi(w);
    }
};

template <int D, int GM>
__global__ void __launch_bounds__(kAttnThreads)
attn_split(const AttnArgs a)
{
    constexpr int CPL = D / 32;
    __shared__ float s_m[kAttnWarps][GM], s_l[kAttnWarps][GM];
    __shared__ float s_acc[kAttnWarps][GM][D];
    __shared__ int s_last;

    const int sp = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = a.G;
    int m_b = a.count[b];
    m_b = max(0, min(m_b, a.cap));
    const int lo = (int)((int64_t)m_b * sp / a.splits);
    const int hi = (int)((int64_t)m_b * (sp + 1) / a.splits);
    const int64_t off = a.seq_off[b];
    const int64_t n_b = a.seq_off[b + 1] - off;

    float qf[GM][CPL];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        if (h < G) {
            float t[CPL];
            RowLoad<CPL>::load(a.q + ((int64_t)b * a.Hq + g * G + h) * D + lane * CPL, t);
#pragma unroll
            for (int c = 0; c < CPL; ++c)
                qf[h][c] = t[c];
        } else {
#pragma unroll
            for (int c = 0; c < CPL; ++c)
                qf[h][c] = 0.0f;
        }
    }
    float mr[GM], lr[GM], acc[GM][CPL];
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        mr[h] = -INFINITY;
        lr[h] = 0.0f;
#pragma unroll
        for (int c = 0; c < CPL; ++c)
            acc[h][c] = 0.0f;
    }

    const int32_t *idrow = a.ids + (int64_t)b * a.cap;
    const __nv_bfloat16 *kb = a.k + (int64_t)g * a.sh + lane * CPL;
    const __nv_bfloat16 *vb = a.v + (int64_t)g * a.sh + lane * CPL;
    for (int j = lo + warp; j < hi; j += kAttnWarps) {
        const int32_t id = __ldg(idrow + j);
        if (id < 0 || (int64_t)id >= n_b)
            continue;                       // outside the sequence: ignored, never read
        const int64_t tok = off + id;
        float kf[CPL], vf[CPL];
        RowLoad<CPL>::load(kb + tok * a.st, kf);
        RowLoad<CPL>::load(vb + tok * a.st, vf);
#pragma unroll
        for (int h = 0; h < GM; ++h) {
            if (h < G) {
                float d = 0.0f;
#pragma unroll
                for (int c = 0; c < CPL; ++c)
                    d = fmaf(qf[h][c], kf[c], d);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    d += __shfl_xor_sync(0xffffffffu, d, o);
                const float s = d * a.scale_log2;
                const float mn = fmaxf(mr[h], s);
                const float corr = exp2f(mr[h] - mn);
                const float p = exp2f(s - mn);
                lr[h] = lr[h] * corr + p;
#pragma unroll
                for (int c = 0; c < CPL; ++c)
                    acc[h][c] = fmaf(acc[h][c], corr, p * vf[c]);
                mr[h] = mn;
            }
        }
    }

    // ---- merge the warps of this CTA ---------------------------------------
#pragma unroll
    for (int h = 0; h < GM; ++h) {
        if (h < G) {
            if (lane == 0) {
                s_m[warp][h] = mr[h];
                s_l[warp][h] = lr[h];
            }
#pragma unroll
            for (int c = 0; c < CPL; ++c)
                s_acc[warp][h][lane * CPL + c] = acc[h][c];
        }
    }
    __syncthreads();
    const int stride = D + 2;
    float *mypart = a.part + (((int64_t)b * a.Hkv + g) * a.splits + sp) * (int64_t)(G * stride);
    for (int idx = threadIdx.x; idx < G * D; idx += kAttnThreads) {
        const int h = idx / D, c = idx - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kAttnWarps; ++w)
            M = fmaxf(M, s_m[w][h]);
        float A = 0.0f, Lsum = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kAttnWarps; ++w) {
                if (s_m[w][h] != -INFINITY) {
                    const float e = exp2f(s_m[w][h] - M);
                    A = fmaf(s_acc[w][h][c], e, A);
                    Lsum = fmaf(s_l[w][h], e, Lsum);
                }
            }
        }
        mypart[h * stride + c] = A;
        if (c == 0) {
            mypart[h * stride + D] = M;
            mypart[h * stride + D + 1] = Lsum;
        }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t t = atomicAdd(&a.tickets[b * a.Hkv + g], 1u);
        s_last = (t == (uint32_t)a.splits - 1) ? 1 : 0;
    }
    __syncthreads();
    if (!s_last)
        return;

    // ---- last split of (b, g): merge the splits ---------------------------
    __threadfence();
    const float *parts = a.part + ((int64_t)b * a.Hkv + g) * a.splits * (int64_t)(G * stride);
    for (int idx = threadIdx.x; idx < G * D; idx += kAttnThreads) {
        const int h = idx / D, c = idx - h * D;
        float M = -INFINITY;
        for (int q = 0; q < a.splits; ++q)
            M = fmaxf(M, __ldcg(parts + (int64_t)q * G * stride + h * stride + D));
        float A = 0.0f, Lsum = 0.0f;
        if (M != -INFINITY) {
            for (int q = 0; q < a.splits; ++q) {
                const float *pq = parts + (int64_t)q * G * stride + h * stride;
                const float mq = __ldcg(pq + D);
                if (mq != -INFINITY) {
                    const float e = exp2f(mq - M);
                    A = fmaf(__ldcg(pq + c), e, A);
                    Lsum = fmaf(__ldcg(pq + D + 1), e, Lsum);
                }
            }
        }
        a.out[((int64_t)b * a.Hq + g * G + h) * D + c] = (Lsum > 0.0f) ? A / Lsum : 0.0f;
    }
    if (threadIdx.x == 0)
        a.tickets[b * a.Hkv + g] = 0u;
}

template <int D, int GM>
cudaError_t launch_attn_t(const Plan &p, const AttnArgs &a, cudaStream_t st)
{
    dim3 grid((unsigned)p.attn_splits, (unsigned)p.Hkv, (unsigned)p.B);
    attn_split<D, GM><<<grid, kAttnThreads, 0, st>>>(a);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free variant (ts_sparse_attn_noalloc)
// ---------------------------------------------------------------------------
// Some callers cannot hand this library any device memory: runtimes that own
// every byte of device memory through their own pool and let no library call
// cudaMalloc or take a workspace after start-up, and deployments whose memory
// budget is fixed when the process initialises.  For them the split-K
// partials and the per-(sequence, kv head) tickets live in this file-scope
// array instead of a caller workspace.  Every GPU that loads the library holds
// it until the process exits; all calls share it (and it keeps the last call's
// contents), so calls that can overlap on the GPU race with each other.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) uint8_t g_attn_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array for the current device, looked up once per
// device (with that device current) and cached.
static uint8_t *noalloc_scratch_ptr(ts_status_t *status)
{
    static std::mutex mu;
    static uint8_t *ptrs[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        set_error("ts_sparse_attn_noalloc: no usable current device");
        *status = TS_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (ptrs[dev] == nullptr) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_attn_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            set_error("ts_sparse_attn_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
            *status = TS_ERR_CUDA;
            return nullptr;
        }
        ptrs[dev] = static_cast<uint8_t *>(ptr);
    }
    *status = TS_OK;
    return ptrs[dev];
}

}  // namespace

ts_status_t launch_attn_noalloc(const Plan &p, const ts_kv_t *kv, const void *q, const int32_t *ids,
                                const int32_t *count, float *out, cudaStream_t st)
{
    const size_t ticket_bytes = align_up(sizeof(uint32_t) * (size_t)p.B * p.Hkv, 256);
    const size_t part_bytes = sizeof(float) * (size_t)p.B * p.Hkv * p.attn_splits * p.G * (p.D + 2);
    if (ticket_bytes + part_bytes > kNoAllocScratchBytes) {
        set_error("ts_sparse_attn_noalloc: this shape needs %zu bytes of scratch, more than the fixed %zu; "
                  "use ts_sparse_attn with a workspace",
                  ticket_bytes + part_bytes, kNoAllocScratchBytes);
        return TS_ERR_UNSUPPORTED;
    }
    ts_status_t status;
    uint8_t *scratch = noalloc_scratch_ptr(&status);
    if (scratch == nullptr)
        return status;
    // the tickets must start at zero whatever an earlier call left behind
    cudaError_t e = cudaMemsetAsync(scratch, 0, ticket_bytes, st);
    if (e != cudaSuccess) {
        set_error("ts_sparse_attn_noalloc: clearing the tickets failed: %s", cudaGetErrorString(e));
        return TS_ERR_CUDA;
    }
    AttnArgs a;
    a.k = static_cast<const __nv_bfloat16 *>(kv->k);
    a.v = static_cast<const __nv_bfloat16 *>(kv->v);
    a.st = kv->stride_tok;
    a.sh = kv->stride_head;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.seq_off = kv->seq_offsets_dev;
    a.ids = ids;
    a.count = count;
    a.cap = p.capacity;
    a.out = out;
    a.tickets = reinterpret_cast<uint32_t *>(scratch);
    a.part = reinterpret_cast<float *>(scratch + ticket_bytes);
    a.B = p.B;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.splits = p.attn_splits;
    a.scale_log2 = p.scale * kLog2e;
    if (p.D == 128)
        e = p.G <= 8 ? launch_attn_t<128, 8>(p, a, st) : launch_attn_t<128, 16>(p, a, st);
    else
        e = p.G <= 8 ? launch_attn_t<64, 8>(p, a, st) : launch_attn_t<64, 16>(p, a, st);
    if (e != cudaSuccess) {
        set_error("ts_sparse_attn_noalloc launch: %s", cudaGetErrorString(e));
        return TS_ERR_CUDA;
    }
    return TS_OK;
}

cudaError_t launch_attn(const Plan &p, const ts_kv_t *kv, const void *q, const int32_t *ids, const int32_t *count,
                        float *out, uint8_t *ws, cudaStream_t st)
{
    AttnArgs a;
    a.k = static_cast<const __nv_bfloat16 *>(kv->k);
    a.v = static_cast<const __nv_bfloat16 *>(kv->v);
    a.st = kv->stride_tok;
    a.sh = kv->stride_head;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.seq_off = kv->seq_offsets_dev;
    a.ids = ids;
    a.count = count;
    a.cap = p.capacity;
    a.out = out;
    a.part = reinterpret_cast<float *>(ws + p.off_attn_part);
    a.tickets = reinterpret_cast<uint32_t *>(ws + p.off_attn_tickets);
    a.B = p.B;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.splits = p.attn_splits;
    a.scale_log2 = p.scale * kLog2e;
    if (p.D == 128)
        return p.G <= 8 ? launch_attn_t<128, 8>(p, a, st) : launch_attn_t<128, 16>(p, a, st);
    return p.G <= 8 ? launch_attn_t<64, 8>(p, a, st) : launch_attn_t<64, 16>(p, a, st);
}

}  // namespace ts
