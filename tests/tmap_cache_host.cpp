// Host build of the library's tensor-map cache (causal_attention_sdpa_b200/csrc/tmap_cache.h) for
// the CPU tests, with a fake 128-byte "tensor map" whose bytes are a function of the key and a
// counter of encoder calls, so the tests can see hits, misses, replacement and failed encodes.
#include <thread>
#include <vector>

#include "tmap_cache.h"

namespace {
struct FakeMap {
    long long w[16];
};
gpt_attn::TmapCache<FakeMap, 4> g_cache;   // four slots, so replacement is easy to reach
int g_encodes = 0;
bool g_fail = false;

bool fake_encode(const gpt_attn::TmapKey& k, FakeMap* m) {
    if (g_fail) return false;
    ++g_encodes;
    for (int i = 0; i < 16; ++i)
        m->w[i] = (long long)k.base * 31 + k.kind * 7 + k.d0 * 5 + k.d1 * 3 + k.d2 + k.d3 * 11 + k.s1 * 13 +
                  k.s2 * 17 + k.s3 * 19 + i;
    return true;
}
}  // namespace

extern "C" {
// Looks the key up; writes the map's first word to *word.  Returns 1 on success.
int tc_get(long long base, int kind, int d0, int d1, int d2, long long* word) {
    gpt_attn::TmapKey k{(uintptr_t)base, kind, d0, d1, d2, 1, (long long)d0, (long long)d0 * d1, (long long)d0 * d1 * d2};
    FakeMap m;
    if (!g_cache.get(k, &m, fake_encode)) return 0;
    *word = m.w[0];
    return 1;
}
long long tc_expected_word(long long base, int kind, int d0, int d1, int d2) {
    const long long s1 = d0, s2 = (long long)d0 * d1, s3 = s2 * d2;
    return base * 31 + kind * 7 + d0 * 5 + d1 * 3 + d2 + 11 + s1 * 13 + s2 * 17 + s3 * 19;
}
// A key that differs from tc_get's only in one stride (fields: 0 token, 1 head, 2 batch).
int tc_get_stride(long long base, int which, long long delta, long long* word) {
    gpt_attn::TmapKey k{(uintptr_t)base, 1, 64, 128, 2, 1, 64, 64 * 128, 64 * 128 * 2};
    if (which == 0) k.s1 += delta;
    if (which == 1) k.s2 += delta;
    if (which == 2) k.s3 += delta;
    FakeMap m;
    if (!g_cache.get(k, &m, fake_encode)) return 0;
    *word = m.w[0];
    return 1;
}
int tc_encodes() { return g_encodes; }
void tc_set_fail(int f) { g_fail = f != 0; }
void tc_stats(long long* h, long long* m, int* u) { g_cache.stats(h, m, u); }
void tc_clear() {
    g_cache.clear();
    g_encodes = 0;
}
// Several host threads looking up the same few keys at once; returns the number of wrong values.
int tc_threads(int n_threads, int iters) {
    std::vector<std::thread> ts;
    std::vector<int> bad(n_threads, 0);
    for (int t = 0; t < n_threads; ++t)
        ts.emplace_back([t, iters, &bad] {
            for (int i = 0; i < iters; ++i) {
                const long long base = 4096 * (1 + (i + t) % 3);
                long long w = 0;
                if (!tc_get(base, 1, 64, 1024, 12, &w) || w != tc_expected_word(base, 1, 64, 1024, 12)) ++bad[t];
            }
        });
    for (auto& th : ts) th.join();
    int s = 0;
    for (int b : bad) s += b;
    return s;
}
}
