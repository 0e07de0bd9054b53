// Host-only test of PerDeviceMemo (fp8_math_b200/csrc/devcache.h), the table
// behind the library's per-device setup: the dynamic shared-memory attribute
// of each GEMM kernel and the occupancy of each quantize kernel.  No GPU:
// "devices" and "kernels" are plain integers and addresses.  Exit status 0
// when every check holds; the first failed check is printed.
#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

#include "devcache.h"

static int failures = 0;
#define CHECK(c)                                                   \
    do {                                                           \
        if (!(c)) {                                                \
            std::printf("check failed, line %d: %s\n", __LINE__, #c); \
            failures++;                                            \
        }                                                          \
    } while (0)

int main() {
    static int kern[6];  // distinct keys
    const void *k0 = &kern[0], *k1 = &kern[1];

    {  // one computation per (key, device); values stay per device
        bsq::PerDeviceMemo<64> m;
        int calls = 0;
        auto value_for = [&](int dev) { return [&calls, dev] { calls++; return 100 + dev; }; };
        auto ok = [](int) { return true; };
        CHECK(m.get(k0, 0, value_for(0), ok) == 100);
        CHECK(m.get(k0, 1, value_for(1), ok) == 101);
        CHECK(m.get(k0, 0, value_for(7), ok) == 100);  // cached: not recomputed
        CHECK(m.get(k0, 1, value_for(7), ok) == 101);
        CHECK(m.get(k1, 0, value_for(2), ok) == 102);  // another key on device 0
        CHECK(calls == 3);
        CHECK(m.size() == 3);
    }
    {  // a failed computation is not kept: the next call tries again
        bsq::PerDeviceMemo<64> m;
        int calls = 0;
        auto ok = [](int v) { return v >= 0; };
        CHECK(m.get(k0, 3, [&] { calls++; return -1; }, ok) == -1);
        CHECK(m.get(k0, 3, [&] { calls++; return 5; }, ok) == 5);
        CHECK(m.get(k0, 3, [&] { calls++; return 9; }, ok) == 5);
        CHECK(calls == 2);
    }
    {  // a full table still answers, uncached
        bsq::PerDeviceMemo<2> m;
        int calls = 0;
        auto ok = [](int) { return true; };
        for (int d = 0; d < 4; d++) m.get(k0, d, [&, d] { calls++; return d; }, ok);
        CHECK(m.size() == 2);
        CHECK(m.get(k0, 3, [&] { calls++; return 3; }, ok) == 3);
        CHECK(calls == 5);
    }
    {  // concurrent first calls from many threads on 4 devices x 6 keys: each
       // pair computed exactly once, every thread sees its device's value
        bsq::PerDeviceMemo<64> m;
        std::atomic<int> calls{0}, wrong{0};
        std::vector<std::thread> ts;
        for (int t = 0; t < 16; t++)
            ts.emplace_back([&, t] {
                for (int rep = 0; rep < 200; rep++)
                    for (int k = 0; k < 6; k++) {
                        const int dev = (t + rep + k) & 3;
                        const int v = m.get(
                            &kern[k], dev, [&, k, dev] { calls++; return 10 * k + dev; }, [](int) { return true; });
                        if (v != 10 * k + dev) wrong++;
                    }
            });
        for (auto &th : ts) th.join();
        CHECK(calls.load() == 24);
        CHECK(wrong.load() == 0);
        CHECK(m.size() == 24);
    }
    if (failures == 0) std::printf("ok\n");
    return failures == 0 ? 0 : 1;
}
