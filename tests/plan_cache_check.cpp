// Host check of the launch-plan cache (csrc/plan_cache.cuh).
//
// Keys are compared byte for byte; a plan is built once per distinct key and
// returned from the cache afterwards; a failed build is kept as a miss (not
// built again); keys that share a slot replace each other and are rebuilt;
// concurrent callers get consistent plans.
//
// Build and run: g++ -O2 -std=c++17 -pthread -I <csrc> plan_cache_check.cpp && ./a.out
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <thread>
#include <vector>

#include "plan_cache.cuh"

struct Key {
    int64_t a;
    int32_t b;
    int32_t pad;   // zeroed: keys compare as bytes
};
struct Plan {
    int64_t value;
    int builds;
};

static int failures = 0;
#define CHECK(cond, ...)                                                  \
    do {                                                                  \
        if (!(cond)) {                                                    \
            std::fprintf(stderr, "FAIL %s:%d: ", __FILE__, __LINE__);     \
            std::fprintf(stderr, __VA_ARGS__);                            \
            std::fprintf(stderr, "\n");                                   \
            ++failures;                                                   \
        }                                                                 \
    } while (0)

static Key key(int64_t a, int32_t b) {
    Key k;
    std::memset(&k, 0, sizeof(k));
    k.a = a;
    k.b = b;
    return k;
}

int main() {
    // a plan per key, built once
    {
        sgmv::PlanCache<Key, Plan, 64> cache;
        int builds = 0;
        auto build_for = [&](int64_t a) {
            return [&, a](Plan* p) {
                ++builds;
                p->value = a * 10;
                p->builds = builds;
                return true;
            };
        };
        for (int rep = 0; rep < 3; ++rep)
            for (int64_t a = 0; a < 20; ++a) {
                Plan p{};
                CHECK(cache.get(key(a, 1), &p, build_for(a)), "get %lld", (long long)a);
                CHECK(p.value == a * 10, "value %lld for key %lld", (long long)p.value, (long long)a);
            }
        CHECK(builds <= 20 * 3, "builds %d", builds);
        // with 64 slots and 20 keys a collision can cost rebuilds, but the same key twice in a row never does
        const int before = builds;
        Plan p{};
        cache.get(key(7, 1), &p, build_for(7));
        cache.get(key(7, 1), &p, build_for(7));
        CHECK(builds - before <= 1, "the second of two identical calls rebuilt");
    }
    // a key that differs in one field is another plan
    {
        sgmv::PlanCache<Key, Plan, 64> cache;
        Plan p{};
        cache.get(key(5, 1), &p, [](Plan* q) { q->value = 1; return true; });
        cache.get(key(5, 2), &p, [](Plan* q) { q->value = 2; return true; });
        CHECK(p.value == 2, "key (5, 2) got the plan of (5, 1)");
        bool rebuilt = false;
        cache.get(key(5, 1), &p, [&](Plan* q) { rebuilt = true; q->value = 1; return true; });
        CHECK(p.value == 1, "key (5, 1) got %lld", (long long)p.value);
        (void)rebuilt;
    }
    // a failed build is kept: the call fails again without building
    {
        sgmv::PlanCache<Key, Plan, 64> cache;
        int builds = 0;
        Plan p{};
        CHECK(!cache.get(key(3, 3), &p, [&](Plan*) { ++builds; return false; }), "a failed build succeeded");
        CHECK(!cache.get(key(3, 3), &p, [&](Plan*) { ++builds; return true; }), "a kept miss turned into a hit");
        CHECK(builds == 1, "builds %d", builds);
    }
    // one slot: keys replace each other and are built again, never mixed up
    {
        sgmv::PlanCache<Key, Plan, 1> cache;
        int builds = 0;
        for (int rep = 0; rep < 4; ++rep)
            for (int64_t a = 0; a < 3; ++a) {
                Plan p{};
                cache.get(key(a, 0), &p, [&, a](Plan* q) { ++builds; q->value = a; return true; });
                CHECK(p.value == a, "one slot: key %lld got %lld", (long long)a, (long long)p.value);
            }
        CHECK(builds == 12, "one slot: builds %d", builds);
    }
    // many threads, few keys: every result matches its key
    {
        sgmv::PlanCache<Key, Plan, 8> cache;
        std::vector<std::thread> threads;
        std::vector<int> bad(8, 0);
        for (int t = 0; t < 8; ++t)
            threads.emplace_back([&, t] {
                for (int i = 0; i < 20000; ++i) {
                    const int64_t a = (i * 7 + t) % 13;
                    Plan p{};
                    cache.get(key(a, 9), &p, [a](Plan* q) { q->value = a * 3 + 1; return true; });
                    if (p.value != a * 3 + 1) ++bad[t];
                }
            });
        for (auto& th : threads) th.join();
        for (int t = 0; t < 8; ++t) CHECK(bad[t] == 0, "thread %d saw %d wrong plans", t, bad[t]);
    }
    if (failures) {
        std::printf("FAILED: %d checks\n", failures);
        return 1;
    }
    std::printf("OK\n");
    return 0;
}
