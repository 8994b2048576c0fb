// Host-only check of fa::PerDevice (csrc/per_device.h), driven with fake device
// indices: compiled and run by tests/test_per_device.py. Prints "ok" and exits 0
// when every check holds; otherwise prints the failed check and exits 1.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "per_device.h"

static int failures = 0;
#define CHECK(cond)                                              \
    do {                                                         \
        if (!(cond)) {                                           \
            std::printf("FAILED line %d: %s\n", __LINE__, #cond); \
            ++failures;                                          \
        }                                                        \
    } while (0)

int main() {
    // Each device gets its own value, made once; later reads return it.
    {
        fa::PerDevice<long> cache;
        int made[fa::kMaxDevices] = {};
        for (int round = 0; round < 3; ++round)
            for (int dev = 0; dev < fa::kMaxDevices; ++dev) {
                long v = -1;
                const bool ok = cache.get(dev, [&](long& out) { ++made[dev]; out = 1000 + dev; return true; }, &v);
                CHECK(ok);
                CHECK(v == 1000 + dev);
            }
        for (int dev = 0; dev < fa::kMaxDevices; ++dev) CHECK(made[dev] == 1);
    }
    // Device 1's value is not device 0's: the case of an address looked up on
    // whichever device was current first.
    {
        fa::PerDevice<const void*> addr;
        static int word0 = 0, word1 = 0;
        const void* a0 = nullptr;
        const void* a1 = nullptr;
        CHECK(addr.get(0, [](const void*& p) { p = &word0; return true; }, &a0));
        CHECK(addr.get(1, [](const void*& p) { p = &word1; return true; }, &a1));
        CHECK(a0 == &word0 && a1 == &word1 && a0 != a1);
        const void* again = nullptr;
        CHECK(addr.get(0, [](const void*& p) { p = nullptr; return true; }, &again));
        CHECK(again == &word0);
    }
    // A failed set-up is not cached: the next call tries again; the output is
    // left as it was on failure.
    {
        fa::PerDevice<int> cache;
        int tries = 0, v = 7;
        CHECK(!cache.get(3, [&](int&) { ++tries; return false; }, &v));
        CHECK(v == 7);
        CHECK(cache.get(3, [&](int& out) { ++tries; out = 42; return true; }, &v));
        CHECK(v == 42 && tries == 2);
        CHECK(cache.get(3, [&](int& out) { ++tries; out = 0; return true; }, &v));
        CHECK(v == 42 && tries == 2);
    }
    // Device indices outside [0, kMaxDevices) are refused without calling make.
    {
        fa::PerDevice<int> cache;
        int calls = 0, v = 5;
        CHECK(!cache.get(-1, [&](int& out) { ++calls; out = 1; return true; }, &v));
        CHECK(!cache.get(fa::kMaxDevices, [&](int& out) { ++calls; out = 1; return true; }, &v));
        CHECK(calls == 0 && v == 5);
    }
    // Many host threads asking for the same devices at once: make runs exactly
    // once per device and everyone sees its value.
    {
        fa::PerDevice<int> cache;
        std::atomic<int> made[fa::kMaxDevices];
        for (auto& m : made) m = 0;
        std::atomic<int> wrong{0};
        std::vector<std::thread> pool;
        for (int t = 0; t < 8; ++t)
            pool.emplace_back([&, t] {
                for (int i = 0; i < 4 * fa::kMaxDevices; ++i) {
                    const int dev = (i * 7 + t) % fa::kMaxDevices;
                    int v = -1;
                    const bool ok = cache.get(dev, [&](int& out) { made[dev]++; out = 3 * dev + 1; return true; }, &v);
                    if (!ok || v != 3 * dev + 1) wrong++;
                }
            });
        for (auto& th : pool) th.join();
        CHECK(wrong.load() == 0);
        for (int dev = 0; dev < fa::kMaxDevices; ++dev) CHECK(made[dev].load() == 1);
    }
    if (failures == 0) std::printf("ok\n");
    return failures == 0 ? 0 : 1;
}
