// CPU emulation of the page-level comparator's selection (quest_select in
// query_aware_kv_ts_b200/csrc/quest.cu), for tests/test_quest_select_cpu.py.
//
// The kernel's own source is compiled for the host: one cluster of C CTAs
// of 1024 threads per sequence, as C * 1024 std::threads; __syncthreads is a
// barrier over a CTA's threads, cluster.sync() one over the cluster's, the
// warp intrinsics exchanges through a per-warp barrier, and every __shared__
// declaration (rewritten by the test into an emu_shared call) gets storage
// of its own per CTA, which map_shared_rank maps into another CTA's.
//
//   quest_select_emu IN OUT: IN holds int64 {B, log2 P, k, n_sink, n_local,
//   rows}, int64 seq_offsets[B + 1], float scores[rows]; OUT receives int32
//   ids[B][k + n_sink + n_local] and int32 count[B].
#include <atomic>
#include <barrier>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <thread>
#include <vector>

struct dim3 {
    unsigned x = 1, y = 1, z = 1;
};
static thread_local dim3 threadIdx;
static thread_local dim3 blockIdx;
static thread_local int t_cta;   // rank of the thread's CTA in its cluster
static dim3 blockDim{1024, 1, 1};
static int g_cluster = 8;
static std::vector<std::barrier<> *> g_cta_barrier;    // [cluster]
static std::barrier<> *g_cluster_barrier;
static std::vector<std::barrier<> *> g_warp_barrier;   // [cluster * 32]
static uint32_t g_lane_word[64][32][32];

#define __global__
#define __device__
#define __forceinline__ inline
#define __launch_bounds__(x)
#define __restrict__

// per-CTA shared storage: (CTA, declaration) -> block
struct Block {
    char *base;
    size_t bytes;
};
static std::mutex g_mu;
static std::map<std::pair<int, int>, Block> g_blocks;
template <typename T> static T *emu_shared(int decl, size_t count)
{
    std::lock_guard<std::mutex> lock(g_mu);
    const auto key = std::make_pair(t_cta, decl);
    auto it = g_blocks.find(key);
    if (it == g_blocks.end()) {
        char *p = static_cast<char *>(calloc(count * sizeof(T), 1));
        g_blocks[key] = Block{p, count * sizeof(T)};
        return reinterpret_cast<T *>(p);
    }
    return reinterpret_cast<T *>(it->second.base);
}
static void free_shared()
{
    for (auto &kv : g_blocks)
        free(kv.second.base);
    g_blocks.clear();
}

static void __syncthreads() { g_cta_barrier[t_cta]->arrive_and_wait(); }
namespace cooperative_groups {
struct cluster_group {
    unsigned num_blocks() const { return (unsigned)g_cluster; }
    unsigned block_rank() const { return (unsigned)t_cta; }
    void sync() const { g_cluster_barrier->arrive_and_wait(); }
    template <typename T> T *map_shared_rank(T *p, int r) const
    {
        std::lock_guard<std::mutex> lock(g_mu);
        for (auto &kv : g_blocks) {
            if (kv.first.first != t_cta)
                continue;
            char *b = kv.second.base;
            if (reinterpret_cast<char *>(p) >= b && reinterpret_cast<char *>(p) < b + kv.second.bytes) {
                auto jt = g_blocks.find(std::make_pair(r, kv.first.second));
                if (jt == g_blocks.end()) {
                    std::fprintf(stderr, "map_shared_rank: CTA %d has not declared block %d yet\n", r,
                                 kv.first.second);
                    std::abort();
                }
                return reinterpret_cast<T *>(jt->second.base + (reinterpret_cast<char *>(p) - b));
            }
        }
        std::fprintf(stderr, "map_shared_rank: not a shared-memory pointer of this CTA\n");
        std::abort();
    }
};
static cluster_group this_cluster() { return cluster_group(); }
}  // namespace cooperative_groups

template <typename F>
static uint32_t warp_exchange(uint32_t v, F read)
{
    const int w = t_cta * 32 + (int)(threadIdx.x >> 5), l = (int)(threadIdx.x & 31);
    uint32_t *words = g_lane_word[t_cta][threadIdx.x >> 5];
    g_warp_barrier[w]->arrive_and_wait();
    words[l] = v;
    g_warp_barrier[w]->arrive_and_wait();
    const uint32_t r = read(words, l);
    g_warp_barrier[w]->arrive_and_wait();
    return r;
}
static uint32_t __shfl_up_sync(unsigned, uint32_t v, int o)
{
    return warp_exchange(v, [&](const uint32_t *x, int l) { return l >= o ? x[l - o] : v; });
}
static uint32_t __shfl_xor_sync(unsigned, uint32_t v, int o)
{
    return warp_exchange(v, [&](const uint32_t *x, int l) { return x[l ^ o]; });
}
static uint32_t atomicAdd(uint32_t *p, uint32_t v) { return std::atomic_ref<uint32_t>(*p).fetch_add(v); }
static float __ldcg(const float *p) { return *p; }
static int __float_as_int(float x)
{
    int b;
    std::memcpy(&b, &x, 4);
    return b;
}
static void pdl_wait() {}
static void pdl_launch_dependents() {}

#include "order_key.inc"
#include "constants.inc"
#include "select.inc"

int main(int argc, char **argv)
{
    if (argc < 3)
        return 2;
    FILE *f = std::fopen(argv[1], "rb");
    if (f == nullptr)
        return 2;
    int64_t hdr[6];
    if (std::fread(hdr, 8, 6, f) != 6)
        return 2;
    const int B = (int)hdr[0], P_shift = (int)hdr[1], k = (int)hdr[2], s = (int)hdr[3], l = (int)hdr[4];
    const int64_t rows = hdr[5];
    std::vector<int64_t> off(B + 1);
    std::vector<float> scores(rows);
    if (std::fread(off.data(), 8, B + 1, f) != (size_t)(B + 1) || std::fread(scores.data(), 4, rows, f) != (size_t)rows)
        return 2;
    std::fclose(f);
    g_cluster = kQSelCluster;
    const int cap = k + s + l;
    std::vector<int32_t> ids((size_t)B * cap, -7), count(B, -7);
    for (int c = 0; c < g_cluster; ++c)
        g_cta_barrier.push_back(new std::barrier<>(1024));
    for (int w = 0; w < g_cluster * 32; ++w)
        g_warp_barrier.push_back(new std::barrier<>(32));
    for (int b = 0; b < B; ++b) {   // one cluster per sequence, one after another
        g_cluster_barrier = new std::barrier<>(g_cluster * 1024);
        std::vector<std::thread> threads;
        for (int c = 0; c < g_cluster; ++c)
            for (int t = 0; t < 1024; ++t)
                threads.emplace_back([&, c, t, b]() {
                    t_cta = c;
                    threadIdx.x = (unsigned)t;
                    blockIdx.x = (unsigned)c;
                    blockIdx.y = (unsigned)b;
                    quest_select(scores.data(), off.data(), P_shift, k, s, l, cap, ids.data(), count.data());
                });
        for (auto &th : threads)
            th.join();
        delete g_cluster_barrier;
        free_shared();
    }
    FILE *o = std::fopen(argv[2], "wb");
    if (o == nullptr)
        return 2;
    std::fwrite(ids.data(), 4, ids.size(), o);
    std::fwrite(count.data(), 4, count.size(), o);
    std::fclose(o);
    std::printf("ok\n");
    return 0;
}
