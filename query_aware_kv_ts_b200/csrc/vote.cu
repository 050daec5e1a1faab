// Score pass B: the soft vote (TokenSelect README, "Key Takeaways": per-head
// criticality normalised by softmax and summed over all heads).
//   votes[i] = sum_h exp(s[h, i] - L[b, h])
// reading the logits written by pass A (L2-resident for moderate n) and the
// float64 log-normalisers L.
//
// Precision: each term is exp_exact_arg (score_common.cuh): s - L formed
// exactly, the base-2 exponent carried as a head/tail pair, so the only
// rounding left is the hardware 2^x (a few 1e-8 relative) and the sum over
// heads.
//
// Work split: grid (groups / threads, B).  Long sequences: a thread takes 4
// consecutive tokens aligned to 4 in the logits rows (row stride padded to 4),
// so each head's logits arrive as one 16-byte load, the next 4 heads' loads in
// flight while 4 heads are computed; short
// sequences: four lanes per token, each summing every fourth head (the exp
// chains are latency-bound: more warps per token hide them), then two shuffles.
// The reuse flag, the sequence bounds and the normalisers L are fetched in one
// round trip, the logits in the next.
//
// With a histogram buffer (the one-call decode step) the pass also builds the
// selection's level-1 histogram of its candidates' votes (top 12 bits of the
// fp32 pattern, the bins the selection starts from): a shared-memory
// histogram per block, merged into the sequence's global one with atomics.
#include "score_common.cuh"
#include "ts_device.cuh"
#include "ts_internal.h"

namespace ts {
namespace {

struct VoteArgs {
    const float *logits;   // [Hq][ld], ld % 4 == 0
    int64_t ld;
    const double *L;       // [B][Hq]
    const int64_t *seq_off;
    const int32_t *reuse;
    float *votes;
    uint32_t *hist;        // [B][4096] level-1 selection histogram, or null
    int k, n_sink, n_local;
    int B, Hq;
};

constexpr int kMaxHeadsVote = 256;
constexpr int kHeadBatch = 8;

// Blackwell's packed fp32 instructions: two lanes per instruction, each lane
// rounded exactly as the scalar IEEE operation.  The low half is the first
// element (the lower address when loaded from memory).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// exp_exact_arg of two tokens at once: the same operations in the same
// order, lane by lane (u is carried negated, -u = t * -log2e_hi exactly),
// so each lane's result is bit-identical to the scalar function's.
struct PackedL {
    uint64_t hi, nhi, lo;   // (L_hi, L_hi), (-L_hi, -L_hi), (L_lo, L_lo)
};
__device__ __forceinline__ uint64_t exp_exact_arg2(uint64_t s, const PackedL &L)
{
    const uint64_t kHi2 = f2_pack(kLog2eHi, kLog2eHi), kNHi2 = f2_pack(-kLog2eHi, -kLog2eHi);
    const uint64_t kLo2 = f2_pack(kLog2eLo, kLog2eLo), kLn22 = f2_pack(kLn2, kLn2);
    const uint64_t t = f2_sub(s, L.hi);
    const uint64_t bp = f2_sub(t, s);
    const uint64_t e = f2_add(f2_sub(s, f2_sub(t, bp)), f2_sub(L.nhi, bp));
    const uint64_t d = f2_sub(e, L.lo);
    const uint64_t nu = f2_mul(t, kNHi2);
    const uint64_t u_lo = f2_add(f2_fma(t, kHi2, nu), f2_fma(t, kLo2, f2_mul(d, kHi2)));
    float nu0, nu1;
    f2_unpack(nu, nu0, nu1);
    const uint64_t p = f2_pack(exp2f(-nu0), exp2f(-nu1));
    return f2_fma(p, f2_mul(u_lo, kLn22), p);
}

template <int TPT, bool HIST>
__global__ void __launch_bounds__(kVoteThreads, 4)
vote_pass_b(const VoteArgs a)
{
    __shared__ float s_hi[kMaxHeadsVote], s_lo[kMaxHeadsVote];
    __shared__ PackedL s_pl[TPT == 4 ? kMaxHeadsVote : 1];
    __shared__ uint32_t s_hist[HIST ? 4096 : 1];
    __shared__ uint16_t s_used[HIST ? 1024 : 1];   // bins this block touched (<= its tokens)
    __shared__ uint32_t s_nused;
    __shared__ int64_t s_bounds[2];
    __shared__ int32_t s_reuse;
    const int tid = threadIdx.x;
    const int nt = blockDim.x;
    if (HIST) {
        for (int i = tid; i < 4096; i += nt)
            s_hist[i] = 0u;
        if (tid == 0)
            s_nused = 0u;
    }
    pdl_wait();
    pdl_launch_dependents();
    const int b = blockIdx.y;
    // one round trip: flag, bounds and normalisers (h_q <= 2 * blockDim), each
    // word loaded by one thread of the block and shared (hundreds of blocks
    // read the same words)
    if (tid == 0) {
        s_reuse = a.reuse != nullptr ? __ldcg(a.reuse + b) : 0;
        s_bounds[0] = __ldcg(a.seq_off + b);
        s_bounds[1] = __ldcg(a.seq_off + b + 1);
    }
    double Lv[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int h = tid + u * nt;
        Lv[u] = h < a.Hq ? __ldcg(a.L + (int64_t)b * a.Hq + h) : 0.0;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int h = tid + u * nt;
        if (h < a.Hq) {
            const float hi = (float)Lv[u];
            const float lo = (float)(Lv[u] - (double)hi);
            s_hi[h] = hi;
            s_lo[h] = lo;
            if (TPT == 4)
                s_pl[TPT == 4 ? h : 0] = PackedL{f2_pack(hi, hi), f2_pack(-hi, -hi), f2_pack(lo, lo)};
        }
    }
    __syncthreads();
    if (s_reuse != 0)
        return;
    const int64_t off = s_bounds[0];
    const int64_t end = s_bounds[1];
    // TPT == 4: thread = 4 consecutive tokens; TPT == 1: 4 lanes per token
    const int tpb = TPT == 1 ? nt / 4 : nt * TPT;                  // tokens per block
    const int q4 = TPT == 1 ? (tid & 3) : 0;
    const int64_t base = off & ~int64_t(TPT - 1);                  // first aligned group of the sequence
    const int64_t i0 = base + (int64_t)blockIdx.x * tpb + (TPT == 1 ? (tid >> 2) : (int64_t)tid * TPT);
    if (base + (int64_t)blockIdx.x * tpb >= end)
        return;   // the whole block is past this sequence
    float acc[TPT];
#pragma unroll
    for (int j = 0; j < TPT; ++j)
        acc[j] = 0.0f;
    if (i0 < end) {
        if constexpr (TPT == 4) {
            // software-pipelined over batches of kPipe heads: the next batch's
            // loads are in flight while this one is computed; tokens in pairs
            // on the packed fp32 pipes (a 16-byte load is two packed pairs)
            constexpr int kPipe = 4;
            const ulonglong2 *lg = reinterpret_cast<const ulonglong2 *>(a.logits + i0);
            const int64_t ld4 = a.ld / 4;
            const ulonglong2 zero = make_ulonglong2(0ull, 0ull);
            ulonglong2 cur[kPipe], nxt[kPipe];
            uint64_t acc01 = 0ull, acc23 = 0ull;   // +0.0f in both halves
#pragma unroll
            for (int u = 0; u < kPipe; ++u)
                cur[u] = u < a.Hq ? __ldcg(lg + (int64_t)u * ld4) : zero;
            for (int h0 = 0; h0 < a.Hq; h0 += kPipe) {
#pragma unroll
                for (int u = 0; u < kPipe; ++u) {
                    const int h = h0 + kPipe + u;
                    nxt[u] = h < a.Hq ? __ldcg(lg + (int64_t)h * ld4) : zero;
                }
#pragma unroll
                for (int u = 0; u < kPipe; ++u) {
                    if (h0 + u < a.Hq) {
                        const PackedL L = s_pl[h0 + u];
                        acc01 = f2_add(acc01, exp_exact_arg2(cur[u].x, L));
                        acc23 = f2_add(acc23, exp_exact_arg2(cur[u].y, L));
                    }
                }
#pragma unroll
                for (int u = 0; u < kPipe; ++u)
                    cur[u] = nxt[u];
            }
            f2_unpack(acc01, acc[0], acc[1]);
            f2_unpack(acc23, acc[2], acc[3]);
        } else {
            // four lanes per token, each summing every fourth head
            for (int h0 = q4; h0 < a.Hq; h0 += 4 * kHeadBatch) {
                float sv[kHeadBatch];
#pragma unroll
                for (int u = 0; u < kHeadBatch; ++u)
                    if (h0 + 4 * u < a.Hq)
                        sv[u] = __ldcg(a.logits + (int64_t)(h0 + 4 * u) * a.ld + i0);
#pragma unroll
                for (int u = 0; u < kHeadBatch; ++u)
                    if (h0 + 4 * u < a.Hq)
                        acc[0] += exp_exact_arg(sv[u], s_hi[h0 + 4 * u], s_lo[h0 + 4 * u]);
            }
        }
    }
    if constexpr (TPT == 1) {
        acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
        acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 2);
    }
    if (i0 < end && (TPT > 1 || q4 == 0)) {
#pragma unroll
        for (int j = 0; j < TPT; ++j) {
            const int64_t i = i0 + j;
            if (i >= off && i < end)
                a.votes[i] = acc[j];
        }
    }
    if constexpr (HIST) {
        // candidates [s', l0) of the sequence; nothing to rank when the
        // selection takes none or all of them (block-uniform)
        const int64_t n = end - off;
        const int64_t s_end = min((int64_t)a.n_sink, n);
        const int64_t l0 = max(n - (int64_t)a.n_local, s_end);
        const int64_t keff = min((int64_t)a.k, l0 - s_end);
        if (keff == 0 || keff == l0 - s_end)
            return;
        const int lane = tid & 31;
#pragma unroll
        for (int j = 0; j < TPT; ++j) {
            const int64_t li = i0 + j - off;   // sequence-local id
            const bool cand = i0 < end && li >= s_end && li < l0 && q4 == 0;
            const uint32_t bin = cand ? (__float_as_uint(acc[j]) >> 20) : 0xffffffffu;
            // one atomic for the warp's first bin, one per lane for the others;
            // whoever finds a bin empty lists it
            const uint32_t act = __ballot_sync(0xffffffffu, cand);
            if (act) {
                const int leader = __ffs(act) - 1;
                const uint32_t lb = __shfl_sync(0xffffffffu, bin, leader);
                const uint32_t same = __ballot_sync(0xffffffffu, bin == lb);
                uint32_t mine = 0xffffffffu;
                if (lane == leader)
                    mine = lb;
                else if (cand && bin != lb)
                    mine = bin;
                if (mine != 0xffffffffu) {
                    const uint32_t add = (lane == leader) ? (uint32_t)__popc(same) : 1u;
                    if (atomicAdd(&s_hist[mine], add) == 0u)
                        s_used[atomicAdd(&s_nused, 1u)] = (uint16_t)mine;
                }
            }
        }
        __syncthreads();
        uint32_t *gh = a.hist + (size_t)b * 4096;
        const uint32_t nused = s_nused;
        for (uint32_t u = tid; u < nused; u += nt) {
            const uint32_t bin = s_used[u];
            atomicAdd(&gh[bin], s_hist[bin]);
        }
    }
}

}  // namespace

cudaError_t launch_vote(const Plan &p, const int64_t *seq_off, const int32_t *reuse, float *votes, uint8_t *ws,
                        cudaStream_t st, const SelectWindow *hist_window, const double *L_in)
{
    if (p.n_max <= 0)
        return cudaSuccess;
    VoteArgs a;
    a.logits = reinterpret_cast<const float *>(ws + p.off_logits);
    a.ld = p.ld_logits;
    a.L = L_in != nullptr ? L_in : reinterpret_cast<const double *>(ws + p.off_L);
    a.seq_off = seq_off;
    a.reuse = reuse;
    a.votes = votes;
    a.hist = hist_window != nullptr ? reinterpret_cast<uint32_t *>(ws + p.off_sel_hist) : nullptr;
    a.k = hist_window != nullptr ? hist_window->k : 0;
    a.n_sink = hist_window != nullptr ? hist_window->n_sink : 0;
    a.n_local = hist_window != nullptr ? hist_window->n_local : 0;
    a.B = p.B;
    a.Hq = p.Hq;
    // long sequences: 4 tokens per thread (16-byte loads, 256 threads);
    // short ones: 64 tokens per 256-thread block, four lanes per token
    if (p.n_total > 262144) {
        const int64_t groups = (p.n_max + 3) / 4 + 1;
        const unsigned gx = (unsigned)((groups + kVoteThreads - 1) / kVoteThreads);
        if (a.hist != nullptr)
            return launch_ex(vote_pass_b<4, true>, dim3(gx, (unsigned)p.B), dim3(kVoteThreads), 0, st, 1, a);
        return launch_ex(vote_pass_b<4, false>, dim3(gx, (unsigned)p.B), dim3(kVoteThreads), 0, st, 1, a);
    }
    const int nt = kVoteThreads;                 // 64 tokens x 4 lanes
    const unsigned gx = (unsigned)((p.n_max + nt / 4) / (nt / 4));
    if (a.hist != nullptr)
        return launch_ex(vote_pass_b<1, true>, dim3(gx, (unsigned)p.B), dim3(nt), 0, st, 1, a);
    return launch_ex(vote_pass_b<1, false>, dim3(gx, (unsigned)p.B), dim3(nt), 0, st, 1, a);
}

}  // namespace ts
