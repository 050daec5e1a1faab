// CPU emulation of the token split's key merge (select_merge in
// query_aware_kv_ts_b200/csrc/split.cu), for tests/test_split_key_merge_cpu.py.
//
// The kernel's own source is compiled for the host: its one CTA of 1024
// threads runs as 1024 std::threads, __syncthreads is a barrier over all of
// them, and each warp intrinsic is an exchange through a per-warp barrier.
// The test writes the kernel's constants (constants.inc) and its source
// (kernel.inc) next to this file's build; every key set below is merged for
// the first and the last rank and the row is compared with the one a sort
// of all the keys gives.  Prints "<cases> cases, <failures> failures".
#include <algorithm>
#include <atomic>
#include <barrier>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <random>
#include <thread>
#include <vector>

struct dim3 {
    unsigned x = 1, y = 1, z = 1;
};
static thread_local dim3 threadIdx;
static dim3 blockDim{1024, 1, 1};
static std::barrier<> *g_block;
static std::barrier<> *g_warp[32];
static uint32_t g_lane_word[32][32];

#define __global__
#define __device__
#define __forceinline__ inline
#define __launch_bounds__(x)
#define __shared__ static

static void __syncthreads() { g_block->arrive_and_wait(); }
static int warp_of() { return (int)(threadIdx.x >> 5); }
static int lane_of() { return (int)(threadIdx.x & 31); }

// every lane publishes v, then reads what the warp published
template <typename F>
static uint32_t warp_exchange(uint32_t v, F read)
{
    const int w = warp_of();
    g_warp[w]->arrive_and_wait();
    g_lane_word[w][lane_of()] = v;
    g_warp[w]->arrive_and_wait();
    const uint32_t r = read(g_lane_word[w]);
    g_warp[w]->arrive_and_wait();
    return r;
}
static uint32_t __shfl_up_sync(unsigned, uint32_t v, int o)
{
    const int l = lane_of();
    return warp_exchange(v, [&](const uint32_t *x) { return l >= o ? x[l - o] : v; });
}
static unsigned __match_any_sync(unsigned, uint32_t v)
{
    return warp_exchange(v, [&](const uint32_t *x) {
        unsigned m = 0;
        for (int l = 0; l < 32; ++l)
            m |= (x[l] == v ? 1u : 0u) << l;
        return m;
    });
}
static uint32_t __reduce_add_sync(unsigned, uint32_t v)
{
    return warp_exchange(v, [&](const uint32_t *x) {
        uint32_t s = 0;
        for (int l = 0; l < 32; ++l)
            s += x[l];
        return s;
    });
}
static int __ffs(unsigned m) { return m ? __builtin_ctz(m) + 1 : 0; }
static int __popc(unsigned m) { return __builtin_popcount(m); }
static uint32_t atomicAdd(uint32_t *p, uint32_t v) { return std::atomic_ref<uint32_t>(*p).fetch_add(v); }
static unsigned long long __ldcg(const unsigned long long *p) { return *p; }
using std::min;

#include "constants.inc"
#include "kernel.inc"

struct KeySet {
    int parts, kcap, k;
    uint64_t vote_values;   // votes drawn from this many values (<= 2: votes of 0 and 1)
    int padding;            // zero keys at the end of every odd rank's list
};

int main()
{
    g_block = new std::barrier<>(1024);
    for (auto &w : g_warp)
        w = new std::barrier<>(32);
    const std::vector<KeySet> sets = {
        {8, 256, 256, 1u << 20, 0},  // few ties
        {8, 256, 256, 50, 0},        // many equal votes: the threshold inside a tie
        {4, 300, 300, 3, 100},       // three vote values, padded ranks
        {2, 100, 100, 1000, 60},
        {3, 500, 499, 7, 0},
        {8, 512, 1, 1u << 30, 0},    // k = 1
        {4, 200, 150, 1, 50},        // every vote +0: only the ids decide
        {2, 300, 250, 2, 200},       // votes of 0 and 1 among padding
        {8, 64, 0, 10, 0},           // k = 0: nothing chosen
        {1, 64, 64, 2, 0},           // one rank
        {2, 100, 100, 10, 100},      // no more real keys than k: all of them
        {2, 100, 100, 10, 99},       // one real key more than k
    };
    std::mt19937_64 rng(7);
    int cases = 0, failures = 0;
    for (const KeySet &c : sets) {
        ++cases;
        const int64_t total = (int64_t)c.parts * c.kcap;
        std::vector<unsigned long long> keys(total, 0ull);
        uint32_t gid = 0;
        for (int r = 0; r < c.parts; ++r) {
            const int real = c.kcap - (r % 2 ? c.padding : 0);
            for (int j = 0; j < real; ++j) {
                gid += 1 + (uint32_t)(rng() % 3);   // ascending sequence ids
                const float v = c.vote_values <= 2 ? (float)(rng() % c.vote_values)
                                                   : 1.0f + (float)(rng() % c.vote_values) / 64.0f;
                uint32_t vb;
                std::memcpy(&vb, &v, 4);
                keys[(int64_t)r * c.kcap + j] = ((unsigned long long)vb << 32) | (0xffffffffu - gid);
            }
        }
        std::vector<unsigned long long> sorted;
        for (unsigned long long x : keys)
            if (x)
                sorted.push_back(x);
        std::sort(sorted.rbegin(), sorted.rend());
        const unsigned long long T =
            c.k == 0 ? ~0ull : ((int64_t)sorted.size() > c.k ? sorted[c.k - 1] : 1ull);
        for (int rank = 0; rank < c.parts; rank += std::max(1, c.parts - 1)) {
            const int s_loc = 2, l_loc = 3, cap = c.kcap + s_loc + l_loc;
            const int64_t n_loc = int64_t(1) << 26;
            std::vector<int32_t> ids(cap, -7);
            int32_t count = -7;
            std::vector<std::thread> threads;
            for (int t = 0; t < 1024; ++t)
                threads.emplace_back([&, t]() {
                    threadIdx.x = (unsigned)t;
                    select_merge(keys.data(), c.parts, c.kcap, c.k, rank, s_loc, l_loc, n_loc, 0, cap, ids.data(),
                                 &count);
                });
            for (auto &th : threads)
                th.join();
            std::vector<int32_t> want;
            for (int i = 0; i < s_loc; ++i)
                want.push_back(i);
            for (int j = 0; j < c.kcap; ++j) {
                const unsigned long long x = keys[(int64_t)rank * c.kcap + j];
                if (x && x >= T)
                    want.push_back((int32_t)(0xffffffffu - (uint32_t)(x & 0xffffffffull)));
            }
            for (int i = 0; i < l_loc; ++i)
                want.push_back((int32_t)(n_loc - l_loc + i));
            bool ok = count == (int32_t)want.size();
            for (size_t i = 0; ok && i < want.size(); ++i)
                ok = ids[i] == want[i];
            for (int i = (int)want.size(); ok && i < cap; ++i)
                ok = ids[i] == -1;
            if (!ok) {
                ++failures;
                std::printf("FAIL parts=%d kcap=%d k=%d values=%llu padding=%d rank=%d: count %d, want %zu\n",
                            c.parts, c.kcap, c.k, (unsigned long long)c.vote_values, c.padding, rank, count,
                            want.size());
            }
        }
    }
    std::printf("%d cases, %d failures\n", cases, failures);
    return failures != 0;
}
