// Score pass A: per-head criticality logits over the whole K cache and the
// per-head softmax normalisers (TokenSelect README, "Key Takeaways": per-head
// Q.K criticality; per-head soft voting normalises each head by a softmax
// over the tokens).
//
// For every active sequence b, KV head g and query head h = g*G + j:
//   s[h, i] = scale * q[b, h, :] . K[b, i, g, :]        (fp32 accumulation)
// written to the logits workspace [h_q][ld], and
//   L[b, h] = log sum_i exp(s[h, i])                   (score_merge below)
//
// Design (B200):
//  * One CTA per SM, persistent.  The active sequences' tokens are cut into
//    chunks of T tokens (one pipeline stage, 32 KB of K); CTA j takes the
//    contiguous, balanced chunk range [j*C/grid, (j+1)*C/grid), so a CTA
//    spans one or two sequences and the load is balanced to one chunk.
//  * A producer warp streams K with 3-D TMA boxes {64 channels, T tokens,
//    h_kv heads} (128-byte swizzle, L2 evict-first) into a 6-stage ring of
//    32 KB stages guarded by mbarriers.  Before waiting for the previous
//    kernel in the stream it already asks L2 for its first tiles, so the
//    first DRAM round trip overlaps that kernel.
//  * Eight consumer warps each own one KV head g and a share of the 16-token
//    row blocks of a stage.  The G query heads of g are the N dimension of a
//    bf16 m16n8k16 tensor-core tile (N = 8 covers G <= 8; two tiles for
//    G <= 16), K rows the M dimension, the head dimension K: the Q fragments
//    live in registers; K fragments come from shared memory with ldmatrix
//    (conflict-free thanks to the swizzle).
//  * The epilogue scales, stores the logits and keeps an online
//    (max, sum exp) per head and thread over the CTA's chunks of a sequence;
//    when the CTA leaves the sequence these are reduced over the CTA and
//    written as one partial of head h at slot j + b (CTA j, sequence b).  The
//    slot is unique: along the chunk order neither j nor b decreases and one
//    of them grows at every new (CTA, sequence) segment.  No fences, atomics
//    or waits on other CTAs.
//  * score_merge (one warp per sequence and head) folds the partials of
//    CTAs j0..j1, the CTAs that cover the sequence, into L[b, h]: fp32 terms
//    exp(m - M) <= 1 summed in float64.
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kPrefetchTiles = kScoreStages;

struct ScoreArgs {
    const __nv_bfloat16 *q;   // [B, Hq, D]
    const int64_t *seq_off;   // [B + 1]
    const int32_t *reuse;     // [B] or null
    float *logits;            // [Hq][ld]
    int64_t ld;
    float2 *partials;         // [Hq][S] (max, sum exp(x - max)) at slot CTA + sequence
    int S;                    // slots per head: grid + B
    int32_t *chunk_table;     // [B + 1] first active chunk of each sequence (for score_merge)
    uint32_t *ctrl;           // status word
    int B, Hq, Hkv, G;
    int T;                    // tokens per chunk / stage
    int stage_bytes;
    float scale;
};

struct __align__(16) ScoreShared {
    uint64_t full[kScoreStages];
    uint64_t empty[kScoreStages];
    int64_t off[kMaxBatch + 1];
    int32_t chunk_start[kMaxBatch + 1];
    float2 red[kScoreConsumerWarps][16];
    int32_t pf_start[32];     // all-active chunk table of the prefetch hints (B <= 32)
    int64_t pf_off[32];       // and the sequence offsets it was built from
};

__device__ __forceinline__ void online_push(float &m, float &z, float x)
{
    if (x > m) {
        z = z * exp2f((m - x) * kLog2e) + 1.0f;
        m = x;
    } else {
        z += exp2f((x - m) * kLog2e);
    }
}

__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap *map, int32_t x, int32_t y, int32_t z)
{
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// chunk_start[b] (b <= B): first chunk of sequence b, leaving out sequences
// that reuse their selection when use_reuse is set.  Every thread calls it.
__device__ __forceinline__ void build_chunk_table(ScoreShared &sh, const int32_t *reuse, int B, int T, int warp,
                                                  int lane, bool use_reuse)
{
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        const int64_t n = sh.off[b + 1] - sh.off[b];
        const bool active = !use_reuse || reuse == nullptr || reuse[b] == 0;
        sh.chunk_start[b + 1] = (active && n > 0) ? (int32_t)((n + T - 1) / T) : 0;
    }
    __syncthreads();
    if (warp == 0) {
        int32_t run = 0;
        for (int base = 0; base < B; base += 32) {
            const int b = base + lane;
            int32_t x = (b < B) ? sh.chunk_start[b + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o)
                    x += y;
            }
            if (b < B)
                sh.chunk_start[b + 1] = run + x;
            run += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0)
            sh.chunk_start[0] = 0;
    }
    __syncthreads();
}

// B <= 32: lane b < B computes c0 = first chunk of sequence b and c1 = one past
// its last (sequences with reuse set, when reuse is given, have no chunks),
// with one round trip for the offsets and flags and a warp scan.
__device__ __forceinline__ void warp_chunk_scan(const int64_t *seq_off, const int32_t *reuse, int B, int T,
                                                int lane, int32_t &c0, int32_t &c1, int64_t &o0, int64_t &o1)
{
    int32_t x = 0;
    o0 = o1 = 0;
    if (lane < B) {
        o0 = __ldcg(seq_off + lane);
        o1 = __ldcg(seq_off + lane + 1);
        const int64_t n = o1 - o0;
        const bool active = reuse == nullptr || __ldcg(reuse + lane) == 0;
        x = (active && n > 0) ? (int32_t)((n + T - 1) / T) : 0;
    }
    int32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += y;
    }
    c0 = incl - x;
    c1 = incl;
}

template <int D, int NB>
__global__ void __launch_bounds__(kScoreThreads, 1)
score_pass_a(const __grid_constant__ CUtensorMap kmap, const ScoreArgs a)
{
    extern __shared__ uint8_t dyn_smem[];
    __shared__ ScoreShared sh;
    uint8_t *stages = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = a.B;
    const int T = a.T;

    if (tid == 0) {
        for (int s = 0; s < kScoreStages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], kScoreConsumerWarps);
        }
        mbar_fence_init();
    }
    // ---- before the previous kernel has finished: only L2 prefetch hints,
    //      computed as if every sequence were active (a wrong guess costs
    //      nothing but bandwidth; the data itself is read after the wait) -----
    if (B <= 32) {
        if (warp == kScoreConsumerWarps) {
            if (lane == 0)
                tma_prefetch_desc(&kmap);
            int32_t c0, c1;
            int64_t o0, o1;
            warp_chunk_scan(a.seq_off, nullptr, B, T, lane, c0, c1, o0, o1);
            if (lane < B) {
                sh.pf_start[lane] = c0;
                sh.pf_off[lane] = o0;
            }
            const int32_t total = __shfl_sync(0xffffffffu, c1, B - 1);
            __syncwarp();
            if (lane == 0) {
                const int32_t v0 = (int32_t)((int64_t)blockIdx.x * total / gridDim.x);
                const int32_t v1 = (int32_t)((int64_t)(blockIdx.x + 1) * total / gridDim.x);
                int b = 0;
                for (int32_t v = v0; v < v1 && v < v0 + kPrefetchTiles; ++v) {
                    while (b + 1 < B && sh.pf_start[b + 1] <= v)
                        ++b;
                    const int64_t t0 = sh.pf_off[b] + (int64_t)(v - sh.pf_start[b]) * T;
#pragma unroll
                    for (int x = 0; x < D / 64; ++x)
                        tma_prefetch_l2_3d(&kmap, x * 64, (int32_t)t0, 0);
                }
            }
        }
    } else {
        for (int b = tid; b <= B; b += blockDim.x)
            sh.off[b] = __ldcg(a.seq_off + b);
        __syncthreads();
        build_chunk_table(sh, a.reuse, B, T, warp, lane, false);
        if (warp == kScoreConsumerWarps && lane == 0) {
            tma_prefetch_desc(&kmap);
            const int32_t total = sh.chunk_start[B];
            const int32_t v0 = (int32_t)((int64_t)blockIdx.x * total / gridDim.x);
            const int32_t v1 = (int32_t)((int64_t)(blockIdx.x + 1) * total / gridDim.x);
            for (int32_t v = v0; v < v1 && v < v0 + kPrefetchTiles; ++v) {
                const int b = upper_seq(sh.chunk_start, B, v);
                const int64_t t0 = sh.off[b] + (int64_t)(v - sh.chunk_start[b]) * T;
#pragma unroll
                for (int x = 0; x < D / 64; ++x)
                    tma_prefetch_l2_3d(&kmap, x * 64, (int32_t)t0, 0);
            }
        }
    }
    pdl_wait();
    pdl_launch_dependents();

    // ---- the real chunk table (reuse flags come from the previous kernel);
    //      the offsets are re-read too, in case a caller's kernel wrote them;
    //      offsets and flags are loaded together: one round trip -------------
    if (B <= 32) {
        if (warp == 0) {
            int32_t c0, c1;
            int64_t o0, o1;
            warp_chunk_scan(a.seq_off, a.reuse, B, T, lane, c0, c1, o0, o1);
            if (lane < B) {
                sh.chunk_start[lane] = c0;
                sh.off[lane] = o0;
            }
            if (lane == B - 1) {
                sh.chunk_start[B] = c1;
                sh.off[B] = o1;
            }
        }
        __syncthreads();
    } else {
        __syncthreads();
        for (int b = tid; b < B; b += blockDim.x) {
            const int64_t o0 = __ldcg(a.seq_off + b), o1 = __ldcg(a.seq_off + b + 1);
            const bool active = a.reuse == nullptr || __ldcg(a.reuse + b) == 0;
            sh.off[b] = o0;
            if (b == B - 1)
                sh.off[B] = o1;
            const int64_t n = o1 - o0;
            sh.chunk_start[b + 1] = (active && n > 0) ? (int32_t)((n + T - 1) / T) : 0;
        }
        __syncthreads();
        if (warp == 0) {
            int32_t run = 0;
            for (int base = 0; base < B; base += 32) {
                const int b = base + lane;
                int32_t x = (b < B) ? sh.chunk_start[b + 1] : 0;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o)
                        x += y;
                }
                if (b < B)
                    sh.chunk_start[b + 1] = run + x;
                run += __shfl_sync(0xffffffffu, x, 31);
            }
            if (lane == 0)
                sh.chunk_start[0] = 0;
        }
        __syncthreads();
    }
    if (blockIdx.x == 0)
        for (int b = tid; b <= B; b += blockDim.x)
            a.chunk_table[b] = sh.chunk_start[b];
    const int32_t total = sh.chunk_start[B];
    const int32_t v_begin = (int32_t)((int64_t)blockIdx.x * total / gridDim.x);
    const int32_t v_end = (int32_t)((int64_t)(blockIdx.x + 1) * total / gridDim.x);
    const int Hkv = a.Hkv;
    const int half_bytes = T * Hkv * 128;   // one 64-channel box

    if (warp == kScoreConsumerWarps) {
        // ================= producer: one elected lane issues TMA ==========
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            uint32_t it = 0;
            for (int32_t v = v_begin; v < v_end; ++v, ++it) {
                const int b = upper_seq(sh.chunk_start, B, v);
                const int64_t t0 = sh.off[b] + (int64_t)(v - sh.chunk_start[b]) * T;
                const int s = it % kScoreStages;
                if (it >= kScoreStages) {
                    const uint32_t par = ((it / kScoreStages) - 1) & 1;
                    if (!mbar_wait_bounded(&sh.empty[s], par, kSpinLimit)) {
                        report_timeout(a.ctrl, kSiteScoreEmpty);
                        break;   // nothing issued after this: the consumers time out on full[] too
                    }
                }
                mbar_arrive_expect_tx(&sh.full[s], (uint32_t)a.stage_bytes);
#pragma unroll
                for (int x = 0; x < D / 64; ++x)
                    tma_load_3d(stages + (size_t)s * a.stage_bytes + x * half_bytes, &kmap, &sh.full[s], x * 64,
                                (int32_t)t0, 0, pol);
            }
        }
        return;
    }

    // ===================== consumers (warps 0..7) =========================
    const int ctid = tid;                       // 0..255
    const int g = warp % Hkv;
    const int wsub = warp / Hkv;
    const int nsub = kScoreConsumerWarps / Hkv;
    const int mblocks = T / 16;
    const int G = a.G;
    const int r0 = lane >> 2;
    const int c0 = (lane & 3) * 2;
    const float scale = a.scale;

    uint32_t bq[D / 16][NB][2];
    float m[NB][2], z[NB][2];
    int cur_b = -1;
    uint32_t it = 0;
    bool dead = false;

    // Close this CTA's run of chunks of a sequence: reduce (max, sum) per head
    // over the CTA and publish one partial per head at slot blockIdx.x + cur_b.
    auto flush_segment = [&]() {
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) {
                    const float m2 = __shfl_xor_sync(0xffffffffu, m[nb][cc], o);
                    const float z2 = __shfl_xor_sync(0xffffffffu, z[nb][cc], o);
                    lse_merge(m[nb][cc], z[nb][cc], m2, z2);
                }
                if (lane < 4)
                    sh.red[warp][nb * 8 + c0 + cc] = make_float2(m[nb][cc], z[nb][cc]);
            }
        named_bar_sync(1, kScoreConsumerWarps * 32);
        for (int h = ctid; h < a.Hq; h += kScoreConsumerWarps * 32) {
            const int gh = h / G, j = h - gh * G;
            float M = -INFINITY, Z = 0.0f;
            for (int w2 = gh; w2 < kScoreConsumerWarps; w2 += Hkv)
                lse_merge(M, Z, sh.red[w2][j].x, sh.red[w2][j].y);
            a.partials[(int64_t)h * a.S + blockIdx.x + cur_b] = make_float2(M, Z);
        }
        named_bar_sync(1, kScoreConsumerWarps * 32);   // sh.red is rewritten by the next flush
    };

    for (int32_t v = v_begin; v < v_end; ++v, ++it) {
        const int b = upper_seq(sh.chunk_start, B, v);
        const int64_t t0 = sh.off[b] + (int64_t)(v - sh.chunk_start[b]) * T;
        const int64_t hi = sh.off[b + 1];

        if (b != cur_b) {
            if (cur_b >= 0)
                flush_segment();
            cur_b = b;
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
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    m[nb][cc] = -INFINITY;
                    z[nb][cc] = 0.0f;
                }
        }

        const int s = it % kScoreStages;
        const uint32_t par = (it / kScoreStages) & 1;
        if (!dead && !mbar_wait_bounded(&sh.full[s], par, kSpinLimit)) {
            report_timeout(a.ctrl, kSiteScoreFull);
            dead = true;
        }
        if (!dead) {
            const uint32_t stage_base = smem_u32(stages + (size_t)s * a.stage_bytes);
            for (int mb = wsub; mb < mblocks; mb += nsub) {
                float acc[NB][4];
#pragma unroll
                for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        acc[nb][e] = 0.0f;
                const int trow = mb * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const uint32_t row_addr = stage_base + (uint32_t)((g * T + trow) * 128);
                const int swz = trow & 7;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int chunk = (ks & 3) * 2 + (lane >> 4);
                    const uint32_t addr =
                        row_addr + (uint32_t)((ks >> 2) * half_bytes) + (uint32_t)((chunk ^ swz) << 4);
                    uint32_t a0, a1, a2, a3;
                    ldmatrix_x4(a0, a1, a2, a3, addr);
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
                        mma_16816(acc[nb], a0, a1, a2, a3, bq[ks][nb][0], bq[ks][nb][1]);
                }
                // epilogue: rows r0 and r0 + 8 of this block, columns c0, c0 + 1
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int64_t tok = t0 + mb * 16 + r0 + rr * 8;
                    if (tok < hi) {
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                            for (int cc = 0; cc < 2; ++cc) {
                                const int j = nb * 8 + c0 + cc;
                                if (j < G) {
                                    const float x = acc[nb][rr * 2 + cc] * scale;
                                    a.logits[(int64_t)(g * G + j) * a.ld + tok] = x;
                                    online_push(m[nb][cc], z[nb][cc], x);
                                }
                            }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&sh.empty[s]);
    }
    if (cur_b >= 0)
        flush_segment();
}

// L[b, h] from the partials of sequence b (one warp per sequence and head).
// CTA j of pass A covers chunks [j*total/grid, (j+1)*total/grid); the CTAs that
// cover the sequence's chunks [cs, ce) are j0 = owner(cs) .. j1 = owner(ce-1),
// owner(v) = ((v+1)*grid - 1) / total, and CTA j wrote at slot j + b.  The
// table entries and every slot the sequence could own are loaded together (one
// round trip); slots outside j0..j1, or of CTAs without chunks, are dropped.
__global__ void __launch_bounds__(32)
score_merge(const float2 *partials, int S, const int32_t *chunk_table, double *L, int B, int Hq, int grid_a)
{
    pdl_wait();
    pdl_launch_dependents();
    const int h = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x;
    constexpr int kPer = 8;   // grid_a <= 256
    const int32_t cs = __ldcg(chunk_table + b), ce = __ldcg(chunk_table + b + 1), total = __ldcg(chunk_table + B);
    const float2 *row = partials + (int64_t)h * S + b;
    float2 pv[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int j = lane + 32 * i;
        pv[i] = j < grid_a ? __ldcg(row + j) : make_float2(-INFINITY, 0.0f);
    }
    if (cs == ce)
        return;   // reused or empty sequence: its L is not needed
    const int j0 = (int)(((int64_t)(cs + 1) * grid_a - 1) / total);
    const int j1 = (int)(((int64_t)ce * grid_a - 1) / total);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int j = lane + 32 * i;
        bool keep = j >= j0 && j <= j1;
        if (keep && total < grid_a)   // some CTAs had no chunks and wrote nothing
            keep = (int64_t)j * total / grid_a < (int64_t)(j + 1) * total / grid_a;
        if (!keep)
            pv[i] = make_float2(-INFINITY, 0.0f);
    }
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
        M = fmaxf(M, pv[i].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    double Z = 0.0;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
        if (pv[i].y > 0.0f)
            Z += (double)(pv[i].y * exp2f((pv[i].x - M) * kLog2e));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        Z += __shfl_xor_sync(0xffffffffu, Z, o);
    if (lane == 0)
        L[(int64_t)b * Hq + h] = (double)M + log(Z);
}

template <int D, int NB>
cudaError_t launch_score_t(const Plan &p, const CUtensorMap &kmap, const ScoreArgs &args, cudaStream_t st)
{
    const size_t dyn = (size_t)kScoreStages * p.stage_bytes + 1024;
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(score_pass_a<D, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)dyn);
        if (e != cudaSuccess)
            return e;
        configured_dev = dev;
    }
    return launch_ex(score_pass_a<D, NB>, dim3((unsigned)p.score_grid), dim3(kScoreThreads), dyn, st, 1, kmap,
                     args);
}

}  // namespace

cudaError_t launch_score(const Plan &p, const CUtensorMap &kmap, const void *q, const int64_t *seq_off,
                         const int32_t *reuse, uint8_t *ws, cudaStream_t st)
{
    ScoreArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.seq_off = seq_off;
    a.reuse = reuse;
    a.logits = reinterpret_cast<float *>(ws + p.off_logits);
    a.ld = p.ld_logits;
    a.partials = reinterpret_cast<float2 *>(ws + p.off_partials);
    a.S = p.score_grid + p.B;
    a.chunk_table = reinterpret_cast<int32_t *>(ws + p.off_chunk_table);
    a.ctrl = reinterpret_cast<uint32_t *>(ws + p.off_ctrl);
    a.B = p.B;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.T = p.tile_tokens;
    a.stage_bytes = p.stage_bytes;
    a.scale = p.scale;
    cudaError_t e;
    if (p.D == 128)
        e = p.G <= 8 ? launch_score_t<128, 1>(p, kmap, a, st) : launch_score_t<128, 2>(p, kmap, a, st);
    else
        e = p.G <= 8 ? launch_score_t<64, 1>(p, kmap, a, st) : launch_score_t<64, 2>(p, kmap, a, st);
    if (e != cudaSuccess)
        return e;
    return launch_ex(score_merge, dim3((unsigned)p.Hq, (unsigned)p.B), dim3(32), 0, st, 1,
                     reinterpret_cast<const float2 *>(ws + p.off_partials), p.score_grid + p.B,
                     reinterpret_cast<const int32_t *>(ws + p.off_chunk_table),
                     reinterpret_cast<double *>(ws + p.off_L), p.B, p.Hq, p.score_grid);
}

}  // namespace ts
