// Attention over the selected tokens (TokenSelect README summary: a small
// number of critical KV cache tokens take part in the attention calculation).
//   out[b, h, :] = sum_j softmax_j(scale * q_h . K[ids_j, g]) * V[ids_j, g]
//
// Split-K decode attention: grid (splits, h_kv, B), 256 threads, at most 64
// selected rows per CTA (small splits spread the gather over many SMs: a
// block's load phase costs about 10-16 ns per KB it loads).  Each CTA:
//  1. gathers its K and V rows into shared memory with coalesced 16-byte
//     asynchronous copies (every row of the CTA in flight at once);
//  2. computes the logits of the G query heads of kv head g on tensor cores
//     (m16n8k16 bf16 -> fp32: rows as M, heads as N, channels as K; the Q
//     fragments stay in registers);
//  3. takes the softmax of each head over its rows (warp reductions);
//  4. computes O^T = V^T P^T on tensor cores: V^T fragments come from the
//     row-major V tile with transposed ldmatrix, and P is split into a bf16
//     high part and a bf16 remainder (two products) so that the weights keep
//     ~16 significant bits instead of bf16's 8;
//  5. writes (max, sum, weighted V) per head as its partial.
// attn_merge (one block per (b, query head), launched right after) folds the
// splits: a thread owns 4 output channels and every NG-th split, loads all of
// them at once, and the NG split groups are combined through shared memory.
// Each selected K/V row is read from HBM once for all G heads of its group.
#include <stdlib.h>

#include <mutex>

#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2f = 0.693147180559945309f;   // ln 2
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int R = kAttnRows;

struct AttnArgs {
    const __nv_bfloat16 *k, *v;
    int64_t st, sh;
    const __nv_bfloat16 *q;
    const int64_t *seq_off;
    const int32_t *ids;
    const int32_t *count;
    int cap;
    float *out;
    float *part;        // [B][Hkv][splits][G][D + 4]: D weighted-V sums, then (max, sum)
    int B, Hq, Hkv, G, splits;
    float scale_log2;   // scale * log2(e): logits in base-2 units
    float *lse;         // or null: [B][Hq] natural log-sum-exp of each head's scaled logits
    // paged cache (page_table != null): token i of sequence b is pool row
    // page_table[b * pt_stride + (i >> page_shift)] << page_shift | (i & (page - 1))
    const int32_t *page_table;
    int pt_stride, page_shift;
    int64_t pool_pages;
};

// Dynamic shared memory of attn_split: K and V tiles, the logits, then the
// tensor-core path's bf16 weight halves, or the CUDA-core path's fp32 queries.
template <int D, int NB, bool TC>
constexpr size_t attn_smem_bytes()
{
    return (size_t)2 * R * (D * 2 + 16) + (size_t)R * NB * 8 * 4 +
           (TC ? (size_t)2 * NB * 8 * R * 2 : (size_t)NB * 8 * D * 4);
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float x)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// TC: logits and weighted sums on tensor cores (mma.sync, P split into a
// bf16 head and remainder); otherwise on the CUDA cores in fp32 (one warp per
// row for the logits, lanes splitting the channels; one thread per channel
// pair and head for the weighted sums).
template <int D, int NB, bool TC>
__global__ void __launch_bounds__(kAttnThreads)
attn_split(const AttnArgs a)
{
    constexpr int GM = NB * 8;
    constexpr int RS = D * 2 + 16;          // shared-memory row stride: conflict-free ldmatrix
    constexpr int PS = D + 4;               // partial row: D sums, max, sum, 2 pad (16-byte rows)
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *sK = smem;
    uint8_t *sV = sK + R * RS;
    float *sS = reinterpret_cast<float *>(sV + R * RS);          // [R][GM] logits (base 2), then weights (CUDA cores)
    uint16_t *sPh = reinterpret_cast<uint16_t *>(sS + R * GM);   // [GM][R] weights, bf16 high part (tensor cores)
    uint16_t *sPl = sPh + GM * R;                                 // [GM][R] bf16 remainder (tensor cores)
    float *sQ = sS + R * GM;                                      // [GM][D] fp32 queries (CUDA cores)
    __shared__ float s_m[GM], s_l[GM];
    __shared__ int32_t s_id[R];
    __shared__ int32_t s_row[R];   // the id's K / V row (its pool row in a paged cache)
    __shared__ uint8_t s_valid[R];

    pdl_wait();                 // ids and count come from the selection kernel
    pdl_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int G = a.G;
    // splits cut the id row's capacity, not its count, so the ids can be
    // fetched in the same round trip as the count
    const int lo = (int)((int64_t)a.cap * sp / a.splits);
    const int hi_cap = (int)((int64_t)a.cap * (sp + 1) / a.splits);
    const int32_t id_pref = (threadIdx.x < (unsigned)(hi_cap - lo))
                                ? __ldcg(a.ids + (int64_t)b * a.cap + lo + threadIdx.x) : -1;
    int m_b = __ldcg(a.count + b);
    m_b = max(0, min(m_b, a.cap));
    const int nrows = max(0, min(min(hi_cap, m_b) - lo, R));
    const int64_t off = a.seq_off[b];
    const int64_t n_b = a.seq_off[b + 1] - off;
    const int r0 = lane >> 2, c0 = (lane & 3) * 2;

    // ---- 1. gather: ids to shared memory, then every K and V row of the split
    //         with coalesced 16-byte async copies (CPR consecutive threads per row)
    if (tid < R) {
        int32_t id = -1;
        if (tid < nrows) {
            id = id_pref;
            if (id < 0 || (int64_t)id >= n_b)
                id = -1;                            // ids outside the sequence are ignored
        }
        int32_t row = (int32_t)(off + id);
        if (id >= 0 && a.page_table != nullptr) {
            // one more round trip in a paged cache: the id's page
            const int32_t pg = __ldcg(a.page_table + (int64_t)b * a.pt_stride + (id >> a.page_shift));
            if (pg >= 0 && pg < a.pool_pages)
                row = (pg << a.page_shift) | (id & ((1 << a.page_shift) - 1));
            else
                id = -1;                            // a page outside the pool: left out
        }
        s_id[tid] = id;
        s_row[tid] = row;
        s_valid[tid] = id >= 0 ? 1 : 0;
    }
    __syncthreads();
    {
        constexpr int CPR = D * 2 / 16;             // 16-byte chunks per row
        for (int idx = tid; idx < 2 * R * CPR; idx += kAttnThreads) {
            const int row = idx / CPR, chunk = idx - row * CPR;
            const bool isV = row >= R;
            const int r = isV ? row - R : row;
            uint8_t *dst = (isV ? sV : sK) + r * RS + chunk * 16;
            const int32_t id = s_id[r];
            if (id >= 0) {
                const __nv_bfloat16 *src = (isV ? a.v : a.k) + (int64_t)s_row[r] * a.st + (int64_t)g * a.sh;
                cp_async_16(dst, reinterpret_cast<const uint8_t *>(src) + chunk * 16);
            } else if (isV) {
                *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);   // P is 0 there; V must be finite
            }
        }
    }

    uint32_t bq[TC ? D / 16 : 1][NB][2];
    if constexpr (TC) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int j = nb * 8 + r0;
                if (j < G) {
                    const uint32_t *qp = reinterpret_cast<const uint32_t *>(
                        a.q + ((int64_t)b * a.Hq + g * G + j) * D + ks * 16 + c0);
                    bq[ks][nb][0] = __ldg(qp);
                    bq[ks][nb][1] = __ldg(qp + 4);
                } else {
                    bq[ks][nb][0] = 0u;
                    bq[ks][nb][1] = 0u;
                }
            }
    } else {
        // the G queries as fp32 in shared memory (rows j >= G stay unread)
        for (int i = tid; i < G * D / 2; i += kAttnThreads) {
            const int j = i / (D / 2), c = 2 * (i - j * (D / 2));
            const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(a.q + ((int64_t)b * a.Hq + g * G + j) * D + c));
            sQ[j * D + c] = bf16_lo(w);
            sQ[j * D + c + 1] = bf16_hi(w);
        }
    }
    cp_async_wait_all();
    __syncthreads();

    // ---- 2. logits S = Q K^T (base-2 units) ----------------------------------
    if constexpr (!TC) {
        // one warp per row: lane l takes channels [l*D/32, (l+1)*D/32) of every
        // head, then a butterfly sum leaves each head's dot product in every lane
        constexpr int CPL = D / 32;
        for (int r = warp; r < R; r += kAttnWarps) {
            const bool rv = r < nrows && s_valid[r];
            float kf[CPL];
            if constexpr (CPL == 4) {
                const uint2 w = *reinterpret_cast<const uint2 *>(sK + r * RS + lane * 8);
                kf[0] = bf16_lo(w.x);
                kf[1] = bf16_hi(w.x);
                kf[2] = bf16_lo(w.y);
                kf[3] = bf16_hi(w.y);
            } else {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(sK + r * RS + lane * 4);
                kf[0] = bf16_lo(w);
                kf[1] = bf16_hi(w);
            }
            float mine = -INFINITY;
#pragma unroll
            for (int j = 0; j < GM; ++j) {
                if (j < G) {
                    float d = 0.0f;
#pragma unroll
                    for (int i = 0; i < CPL; ++i)
                        d = fmaf(kf[i], sQ[j * D + lane * CPL + i], d);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        d += __shfl_xor_sync(0xffffffffu, d, o);
                    if (lane == j)
                        mine = d;
                }
            }
            if (lane < GM)
                sS[r * GM + lane] = (rv && lane < G) ? mine * a.scale_log2 : -INFINITY;
        }
    }
    const int nmb = TC ? (nrows + 15) / 16 : 0;
    for (int mb = warp; mb < nmb; mb += kAttnWarps) {
        float acc[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int e = 0; e < 4; ++e)
                acc[nb][e] = 0.0f;
        const int trow = mb * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const uint32_t row_addr = smem_u32(sK + trow * RS) + (uint32_t)((lane >> 4) * 16);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(a0, a1, a2, a3, row_addr + ks * 32);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
                mma_16816(acc[nb], a0, a1, a2, a3, bq[ks][nb][0], bq[ks][nb][1]);
        }
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const int r = mb * 16 + r0 + rr * 8;
            const bool rv = r < nrows && s_valid[r];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    const int j = nb * 8 + c0 + cc;
                    sS[r * GM + j] = (rv && j < G) ? acc[nb][rr * 2 + cc] * a.scale_log2 : -INFINITY;
                }
        }
    }
    __syncthreads();

    // ---- 3. softmax of each head over this split's rows ---------------------
    for (int h = warp; h < GM; h += kAttnWarps) {
        float x[R / 32];
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < R / 32; ++i) {
            const int r = lane + 32 * i;
            x[i] = (r < nrows && h < G) ? sS[r * GM + h] : -INFINITY;
            mx = fmaxf(mx, x[i]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float sum = 0.0f;
#pragma unroll
        for (int i = 0; i < R / 32; ++i) {
            const int r = lane + 32 * i;
            const float p = (mx == -INFINITY) ? 0.0f : exp2f(x[i] - mx);
            sum += p;
            if constexpr (TC) {
                const uint16_t hb = bf16_bits_rn(p);
                sPh[h * R + r] = hb;
                sPl[h * R + r] = bf16_bits_rn(p - __uint_as_float((uint32_t)hb << 16));
            } else {
                sS[r * GM + h] = p;   // the weight replaces its logit (read above by this lane)
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
            s_m[h] = mx;
            s_l[h] = sum;
        }
    }
    __syncthreads();

    const int64_t GS = (int64_t)G * PS;
    float *mypart = a.part + (((int64_t)b * a.Hkv + g) * a.splits + sp) * GS;
    if constexpr (!TC) {
        // ---- 4'. O = P^T V on the CUDA cores: thread = (channel pair, heads
        //          hg, hg + NH, ...); a warp shares its heads (weights broadcast)
        constexpr int CP = D / 2;                    // channel pairs
        constexpr int NH = kAttnThreads / CP;        // head groups
        constexpr int HPT = (GM + NH - 1) / NH;      // heads per thread (at most)
        const int cp = tid % CP, hg = tid / CP;
        float o2[HPT][2];
#pragma unroll
        for (int u = 0; u < HPT; ++u)
            o2[u][0] = o2[u][1] = 0.0f;
        for (int r = 0; r < nrows; ++r) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(sV + r * RS + cp * 4);
            const float v0 = bf16_lo(w), v1 = bf16_hi(w);
#pragma unroll
            for (int u = 0; u < HPT; ++u) {
                const int h = hg + u * NH;
                if (h < G) {
                    const float pw = sS[r * GM + h];
                    o2[u][0] = fmaf(pw, v0, o2[u][0]);
                    o2[u][1] = fmaf(pw, v1, o2[u][1]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < HPT; ++u) {
            const int h = hg + u * NH;
            if (h < G)
                *reinterpret_cast<float2 *>(mypart + h * PS + 2 * cp) = make_float2(o2[u][0], o2[u][1]);
        }
    } else {
        // ---- 4. O^T = V^T P^T: warp w owns channels [16w, 16w + 16) --------------
        float o[NB][4];
    #pragma unroll
        for (int nb = 0; nb < NB; ++nb)
    #pragma unroll
            for (int e = 0; e < 4; ++e)
                o[nb][e] = 0.0f;
        if (warp < D / 16) {
            const int cw = warp * 16;
            const int nks = (nrows + 15) / 16;
            for (int ks = 0; ks < nks; ++ks) {
                const int rb = ks * 16;
                const uint32_t addr = smem_u32(sV + (rb + (lane & 7) + ((lane >> 4) & 1) * 8) * RS) +
                                      (uint32_t)((cw + ((lane >> 3) & 1) * 8) * 2);
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4_trans(a0, a1, a2, a3, addr);
    #pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const int h = nb * 8 + r0;
                    const int rr = rb + c0;
                    const uint32_t bh0 = *reinterpret_cast<const uint32_t *>(sPh + h * R + rr);
                    const uint32_t bh1 = *reinterpret_cast<const uint32_t *>(sPh + h * R + rr + 8);
                    const uint32_t bl0 = *reinterpret_cast<const uint32_t *>(sPl + h * R + rr);
                    const uint32_t bl1 = *reinterpret_cast<const uint32_t *>(sPl + h * R + rr + 8);
                    mma_16816(o[nb], a0, a1, a2, a3, bh0, bh1);
                    mma_16816(o[nb], a0, a1, a2, a3, bl0, bl1);
                }
            }
        }

        // ---- 5. this split's partial ---------------------------------------------
        if (warp < D / 16) {
    #pragma unroll
            for (int nb = 0; nb < NB; ++nb)
    #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int ch = warp * 16 + r0 + (e >= 2 ? 8 : 0);
                    const int h = nb * 8 + c0 + (e & 1);
                    if (h < G)
                        mypart[h * PS + ch] = o[nb][e];
                }
        }
    }
    if (tid < G) {
        mypart[tid * PS + D] = s_m[tid];
        mypart[tid * PS + D + 1] = s_l[tid];
    }
}

// out[b, h, :] for query head h = g*G + j from the splits of (b, g).  Thread
// (sg, c): output channels 4c..4c+3 of every split s = sg (mod NG), all loaded
// in one round trip (kMergeBatch splits per thread per trip); the NG groups'
// (max, sum, weighted sums) are then combined through shared memory.
constexpr int kMergeBatch = 8;
template <int D>
__global__ void __launch_bounds__(kAttnThreads)
attn_merge(const AttnArgs a)
{
    constexpr int PS = D + 4;
    constexpr int CQ = D / 4;                    // channel quads
    constexpr int NG = kAttnThreads / CQ;        // split groups
    __shared__ float4 s_acc[NG][CQ];
    __shared__ float2 s_ml[NG][CQ];
    pdl_wait();
    pdl_launch_dependents();
    const int h = blockIdx.x, b = blockIdx.y;
    const int G = a.G;
    const int g = h / G, j = h - g * G;
    const int c = threadIdx.x % CQ, sg = threadIdx.x / CQ;
    const int64_t GS = (int64_t)G * PS;
    const float *parts = a.part + ((int64_t)b * a.Hkv + g) * a.splits * GS + (int64_t)j * PS;
    float M = -INFINITY, L = 0.0f;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int s0 = sg; s0 < a.splits; s0 += kMergeBatch * NG) {
        float4 v4[kMergeBatch];
        float2 ml[kMergeBatch];
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {
            const int sp = s0 + i * NG;
            if (sp < a.splits) {
                const float *pq = parts + (int64_t)sp * GS;
                v4[i] = __ldcg(reinterpret_cast<const float4 *>(pq + 4 * c));
                ml[i] = __ldcg(reinterpret_cast<const float2 *>(pq + D));
            } else {
                v4[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                ml[i] = make_float2(-INFINITY, 0.0f);
            }
        }
        float Mb = M;
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i)
            Mb = fmaxf(Mb, ml[i].x);
        if (Mb == -INFINITY)
            continue;
        const float r = (M == -INFINITY) ? 0.0f : exp2f(M - Mb);
        L *= r;
        acc.x *= r;
        acc.y *= r;
        acc.z *= r;
        acc.w *= r;
#pragma unroll
        for (int i = 0; i < kMergeBatch; ++i) {
            if (ml[i].x != -INFINITY) {
                const float w = exp2f(ml[i].x - Mb);
                L = fmaf(ml[i].y, w, L);
                acc.x = fmaf(w, v4[i].x, acc.x);
                acc.y = fmaf(w, v4[i].y, acc.y);
                acc.z = fmaf(w, v4[i].z, acc.z);
                acc.w = fmaf(w, v4[i].w, acc.w);
            }
        }
        M = Mb;
    }
    s_acc[sg][c] = acc;
    s_ml[sg][c] = make_float2(M, L);
    __syncthreads();
    if (sg != 0)
        return;
    float Mt = -INFINITY;
#pragma unroll
    for (int q = 0; q < NG; ++q)
        Mt = fmaxf(Mt, s_ml[q][c].x);
    float Lt = 0.0f;
    float4 o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (Mt != -INFINITY) {
#pragma unroll
        for (int q = 0; q < NG; ++q) {
            const float2 mlq = s_ml[q][c];
            if (mlq.x != -INFINITY) {
                const float w = exp2f(mlq.x - Mt);
                const float4 aq = s_acc[q][c];
                Lt = fmaf(mlq.y, w, Lt);
                o.x = fmaf(w, aq.x, o.x);
                o.y = fmaf(w, aq.y, o.y);
                o.z = fmaf(w, aq.z, o.z);
                o.w = fmaf(w, aq.w, o.w);
            }
        }
    }
    const float inv = Lt > 0.0f ? 1.0f / Lt : 0.0f;
    *reinterpret_cast<float4 *>(a.out + ((int64_t)b * a.Hq + h) * D + 4 * c) =
        make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    if (a.lse != nullptr && c == 0)   // (max and sum are the same in every channel quad)
        a.lse[(int64_t)b * a.Hq + h] = Lt > 0.0f ? (Mt + log2f(Lt)) * kLn2f : -INFINITY;
}

template <int D, int NB, bool TC>
cudaError_t launch_attn_t(const Plan &p, const AttnArgs &a, cudaStream_t st)
{
    constexpr size_t smem = attn_smem_bytes<D, NB, TC>();
    cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void *>(attn_split<D, NB, TC>), (int)smem);
    if (e != cudaSuccess)
        return e;
    dim3 grid((unsigned)p.attn_splits, (unsigned)p.Hkv, (unsigned)p.B);
    e = launch_ex(attn_split<D, NB, TC>, grid, dim3(kAttnThreads), smem, st, 1, a);
    if (e != cudaSuccess)
        return e;
    return launch_ex(attn_merge<D>, dim3((unsigned)p.Hq, (unsigned)p.B), dim3(kAttnThreads), 0, st, 1, a);
}

// The logits and weighted sums run on the CUDA cores when the environment
// sets TS_ATTN_CUDA_CORES=1 (read at every call; for comparing the two), on
// the tensor cores otherwise.
static bool attn_cuda_cores()
{
    const char *e = getenv("TS_ATTN_CUDA_CORES");
    return e != nullptr && e[0] == '1';
}

cudaError_t launch_attn_any(const Plan &p, const AttnArgs &a, cudaStream_t st)
{
    if (attn_cuda_cores()) {
        if (p.D == 128)
            return p.G <= 8 ? launch_attn_t<128, 1, false>(p, a, st) : launch_attn_t<128, 2, false>(p, a, st);
        return p.G <= 8 ? launch_attn_t<64, 1, false>(p, a, st) : launch_attn_t<64, 2, false>(p, a, st);
    }
    if (p.D == 128)
        return p.G <= 8 ? launch_attn_t<128, 1, true>(p, a, st) : launch_attn_t<128, 2, true>(p, a, st);
    return p.G <= 8 ? launch_attn_t<64, 1, true>(p, a, st) : launch_attn_t<64, 2, true>(p, a, st);
}

AttnArgs make_args(const Plan &p, const ts_kv_t *kv, const void *q, const int32_t *ids, const int32_t *count,
                   float *out)
{
    AttnArgs a;
    a.lse = nullptr;
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
    a.part = nullptr;
    a.B = p.B;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.splits = p.attn_splits;
    a.scale_log2 = p.scale * kLog2e;
    a.page_table = p.paged ? kv->page_table_dev : nullptr;
    a.pt_stride = p.paged ? kv->page_table_stride : 0;
    a.page_shift = p.page_shift;
    a.pool_pages = p.paged ? p.kv_rows >> p.page_shift : 0;
    return a;
}

// ---------------------------------------------------------------------------
// Allocation-free variant (ts_sparse_attn_noalloc)
// ---------------------------------------------------------------------------
// Some callers cannot hand this library any device memory: runtimes that own
// every byte of device memory through their own pool and let no library call
// cudaMalloc or take a workspace after start-up, and deployments whose memory
// budget is fixed when the process initialises.  For them the split-K
// partials live in this file-scope array instead of a caller workspace.  Every GPU that loads the library holds
// it until the process exits; all calls share it (and it keeps the last call's
// contents), so calls that can overlap on the GPU race with each other.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) uint8_t g_attn_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array for the current device, looked up once per
// device (with that device current) and cached together with the context it
// belongs to: after a device reset the device has a new context, in which the
// library's module (and the array) is loaded afresh, and the address is
// looked up again.
static uint8_t *noalloc_scratch_ptr(ts_status_t *status)
{
    static std::mutex mu;
    static uint8_t *ptrs[64] = {nullptr};
    static void *ctxs[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        set_error("ts_sparse_attn_noalloc: no usable current device");
        *status = TS_ERR_CUDA;
        return nullptr;
    }
    void *ctx = current_context();
    std::lock_guard<std::mutex> lock(mu);
    if (ptrs[dev] == nullptr || ctxs[dev] != ctx || ctx == nullptr) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_attn_noalloc_scratch);
        if (e != cudaSuccess || ptr == nullptr) {
            set_error("ts_sparse_attn_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
            *status = TS_ERR_CUDA;
            return nullptr;
        }
        ptrs[dev] = static_cast<uint8_t *>(ptr);
        ctxs[dev] = current_context();
    }
    *status = TS_OK;
    return ptrs[dev];
}

}  // namespace

ts_status_t launch_attn_noalloc(const Plan &p, const ts_kv_t *kv, const void *q, const int32_t *ids,
                                const int32_t *count, float *out, cudaStream_t st)
{
    const size_t part_bytes = sizeof(float) * (size_t)p.B * p.Hkv * p.attn_splits * p.G * (p.D + 4);
    if (part_bytes > kNoAllocScratchBytes) {
        set_error("ts_sparse_attn_noalloc: this shape needs %zu bytes of scratch, more than the fixed %zu; "
                  "use ts_sparse_attn with a workspace",
                  part_bytes, kNoAllocScratchBytes);
        return TS_ERR_UNSUPPORTED;
    }
    ts_status_t status;
    uint8_t *scratch = noalloc_scratch_ptr(&status);
    if (scratch == nullptr)
        return status;
    // every partial the merge reads is written by the same call first, so
    // nothing in the array has to start at zero
    AttnArgs a = make_args(p, kv, q, ids, count, out);
    a.part = reinterpret_cast<float *>(scratch);
    cudaError_t e = launch_attn_any(p, a, st);
    if (e != cudaSuccess) {
        set_error("ts_sparse_attn_noalloc launch: %s", cudaGetErrorString(e));
        return TS_ERR_CUDA;
    }
    return TS_OK;
}

cudaError_t launch_attn(const Plan &p, const ts_kv_t *kv, const void *q, const int32_t *ids, const int32_t *count,
                        float *out, uint8_t *ws, cudaStream_t st, float *lse)
{
    AttnArgs a = make_args(p, kv, q, ids, count, out);
    a.part = reinterpret_cast<float *>(ws + p.off_attn_part);
    a.lse = lse;
    return launch_attn_any(p, a, st);
}

}  // namespace ts
