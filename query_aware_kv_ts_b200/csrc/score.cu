// Score pass A: per-head criticality logits over the whole K cache and the
// per-head softmax normalisers (TokenSelect README, "Key Takeaways": per-head
// Q.K criticality; per-head soft voting normalises each head by a softmax
// over the tokens).
//
// For every active sequence b, KV head g and query head h = g*G + j:
//   s[h, i] = scale * q[b, h, :] . K[b, i, g, :]        (fp32 accumulation)
// written to the logits workspace [h_q][n_total], and
//   L[b, h] = log sum_i exp(s[h, i])                   (float64 merge)
//
// Design (B200):
//  * One CTA per SM, persistent over single-stage chunks of T tokens of the
//    active sequences, dealt round-robin so that all CTAs sweep K together
//    and the load is balanced to within one chunk.  A producer warp streams K with 3-D TMA boxes
//    {64 channels, T tokens, h_kv heads} (128-byte swizzle, L2 evict-first)
//    into a 6-stage ring of ~32 KB stages guarded by mbarriers.
//  * Eight consumer warps each own one KV head g and a share of the 16-token
//    row blocks of a stage.  The G query heads of g are the N dimension of a
//    bf16 m16n8k16 tensor-core tile (N = 8 covers G <= 8; two tiles for
//    G <= 16), K rows the M dimension, the head dimension K: the Q fragments
//    live in registers for the whole chunk; K fragments come from shared
//    memory with ldmatrix (conflict-free thanks to the swizzle).
//  * The epilogue scales, stores the logits and keeps an online
//    (max, sum exp) per head and thread over all of the CTA's chunks of a
//    sequence; when the CTA leaves the sequence these are reduced over the
//    CTA and written as one partial per (CTA, sequence, head).
//  * The CTA that finishes the last chunk of a sequence (atomic ticket, no
//    waiting) merges that sequence's partials in float64 into L[b, :].
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

struct ScoreArgs {
    const __nv_bfloat16 *q;   // [B, Hq, D]
    const int64_t *seq_off;   // [B + 1]
    const int32_t *reuse;     // [B] or null
    float *logits;            // [Hq][ld]
    int64_t ld;
    float2 *partials;         // [max_chunks][Hq] (max, sum exp(x - max))
    uint32_t *tickets;        // [B]
    double *L;                // [B][Hq]
    uint32_t *ctrl;
    int B, Hq, Hkv, G;
    int T;                    // tokens per stage
    int stage_bytes;
    int64_t chunk_tokens;
    float scale;
};

struct __align__(16) ScoreShared {
    uint64_t full[kScoreStages];
    uint64_t empty[kScoreStages];
    int64_t off[kMaxBatch + 1];
    int32_t chunk_start[kMaxBatch + 1];
    float2 red[kScoreConsumerWarps][16];
    int32_t abort;
    int32_t last;
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

    // ---- sequence table: chunk_start[b] = first chunk of sequence b -------
    for (int b = tid; b <= B; b += blockDim.x)
        sh.off[b] = a.seq_off[b];
    if (tid == 0) {
        for (int s = 0; s < kScoreStages; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], kScoreConsumerWarps);
        }
        sh.abort = 0;
        mbar_fence_init();
    }
    __syncthreads();
    for (int b = tid; b < B; b += blockDim.x) {
        int64_t n = sh.off[b + 1] - sh.off[b];
        bool active = (a.reuse == nullptr) || (a.reuse[b] == 0);
        sh.chunk_start[b + 1] = (active && n > 0) ? (int32_t)((n + a.chunk_tokens - 1) / a.chunk_tokens) : 0;
    }
    __syncthreads();
    if (warp == 0) {
        int32_t run = 0;
        for (int base = 0; base < B; base += 32) {
            int b = base + lane;
            int32_t x = (b < B) ? sh.chunk_start[b + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int32_t y = __shfl_up_sync(0xffffffffu, x, o);
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
    const int32_t total_chunks = sh.chunk_start[B];
    const int T = a.T;
    const int Hkv = a.Hkv;
    const int half_bytes = T * Hkv * 128;   // one 64-channel box

    if (warp == kScoreConsumerWarps) {
        // ================= producer: one elected lane issues TMA ==========
        if (lane == 0) {
            tma_prefetch_desc(&kmap);
            const uint64_t pol = l2_policy_evict_first();
            uint32_t it = 0;
            for (int32_t v = blockIdx.x; v < total_chunks; v += gridDim.x) {
                const int b = upper_seq(sh.chunk_start, B, v);
                const int64_t lo = sh.off[b] + (int64_t)(v - sh.chunk_start[b]) * a.chunk_tokens;
                const int64_t hi = min(lo + a.chunk_tokens, sh.off[b + 1]);
                for (int64_t t0 = lo; t0 < hi; t0 += T, ++it) {
                    const int s = it % kScoreStages;
                    if (it >= kScoreStages) {
                        const uint32_t par = ((it / kScoreStages) - 1) & 1;
                        if (*(volatile int32_t *)&sh.abort ||
                            !mbar_wait_bounded(&sh.empty[s], par, kSpinLimit)) {
                            if (!*(volatile int32_t *)&sh.abort)
                                report_timeout(a.ctrl, kSiteScoreEmpty);
                            *(volatile int32_t *)&sh.abort = 1;
                            continue;
                        }
                    }
                    mbar_arrive_expect_tx(&sh.full[s], (uint32_t)a.stage_bytes);
#pragma unroll
                    for (int x = 0; x < D / 64; ++x)
                        tma_load_3d(stages + (size_t)s * a.stage_bytes + x * half_bytes, &kmap, &sh.full[s],
                                    x * 64, (int32_t)t0, 0, pol);
                }
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
    int32_t seg_first = 0, seg_count = 0;
    uint32_t it = 0;

    // Close this CTA's run of chunks of sequence sb: reduce (max, sum) per
    // head over the CTA, publish one partial at slot seg_first, and let the
    // CTA that completes the sequence's last chunk merge its partials.
    auto flush_segment = [&](int sb) {
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
            a.partials[(int64_t)seg_first * a.Hq + h] = make_float2(M, Z);
        }
        __threadfence();
        named_bar_sync(1, kScoreConsumerWarps * 32);
        if (ctid == 0) {
            const uint32_t nch = (uint32_t)(sh.chunk_start[sb + 1] - sh.chunk_start[sb]);
            const uint32_t t = atomicAdd(&a.tickets[sb], (uint32_t)seg_count);
            sh.last = (t + (uint32_t)seg_count == nch) ? 1 : 0;
        }
        named_bar_sync(1, kScoreConsumerWarps * 32);
        if (sh.last) {
            // Every CTA that took chunks of sb wrote its partial at the slot of
            // its first chunk there: slots [cs, cs + min(nc, gridDim.x)).
            __threadfence();
            const int32_t cs = sh.chunk_start[sb];
            const int32_t nslots = min(sh.chunk_start[sb + 1] - cs, (int32_t)gridDim.x);
            for (int h = warp; h < a.Hq; h += kScoreConsumerWarps) {
                float M = -INFINITY;
                for (int c = lane; c < nslots; c += 32)
                    M = fmaxf(M, __ldcg(&a.partials[(int64_t)(cs + c) * a.Hq + h]).x);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
                double Z = 0.0;
                for (int c = lane; c < nslots; c += 32) {
                    const float2 p = __ldcg(&a.partials[(int64_t)(cs + c) * a.Hq + h]);
                    if (p.y > 0.0f)
                        Z += (double)p.y * exp((double)p.x - (double)M);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    Z += __shfl_xor_sync(0xffffffffu, Z, o);
                if (lane == 0)
                    a.L[(int64_t)sb * a.Hq + h] = (double)M + log(Z);
            }
            if (ctid == 0)
                a.tickets[sb] = 0u;
        }
        named_bar_sync(1, kScoreConsumerWarps * 32);
    };

    for (int32_t v = blockIdx.x; v < total_chunks; v += gridDim.x) {
        const int b = upper_seq(sh.chunk_start, B, v);
        const int64_t lo = sh.off[b] + (int64_t)(v - sh.chunk_start[b]) * a.chunk_tokens;
        const int64_t hi = min(lo + a.chunk_tokens, sh.off[b + 1]);

        if (b != cur_b) {
            if (cur_b >= 0)
                flush_segment(cur_b);
            cur_b = b;
            seg_first = v;
            seg_count = 0;
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
        ++seg_count;

        for (int64_t t0 = lo; t0 < hi; t0 += T, ++it) {
            const int s = it % kScoreStages;
            const uint32_t par = (it / kScoreStages) & 1;
            bool ok = !*(volatile int32_t *)&sh.abort;
            if (ok && !mbar_wait_bounded(&sh.full[s], par, kSpinLimit)) {
                report_timeout(a.ctrl, kSiteScoreFull);
                *(volatile int32_t *)&sh.abort = 1;
                ok = false;
            }
            if (ok) {
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
                        const uint32_t addr = row_addr + (uint32_t)((ks >> 2) * half_bytes) +
                                              (uint32_t)((chunk ^ swz) << 4);
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
    }
    if (cur_b >= 0)
        flush_segment(cur_b);
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
    score_pass_a<D, NB><<<p.score_grid, kScoreThreads, dyn, st>>>(kmap, args);
    return cudaGetLastError();
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
    a.ld = p.n_total;
    a.partials = reinterpret_cast<float2 *>(ws + p.off_partials);
    a.tickets = reinterpret_cast<uint32_t *>(ws + p.off_score_tickets);
    a.L = reinterpret_cast<double *>(ws + p.off_L);
    a.ctrl = reinterpret_cast<uint32_t *>(ws + p.off_ctrl);
    a.B = p.B;
    a.Hq = p.Hq;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.T = p.tile_tokens;
    a.stage_bytes = p.stage_bytes;
    a.chunk_tokens = p.chunk_tokens;
    a.scale = p.scale;
    if (p.D == 128)
        return p.G <= 8 ? launch_score_t<128, 1>(p, kmap, a, st) : launch_score_t<128, 2>(p, kmap, a, st);
    return p.G <= 8 ? launch_score_t<64, 1>(p, kmap, a, st) : launch_score_t<64, 2>(p, kmap, a, st);
}

}  // namespace ts
