// Host-side check of the per-device launch caches (no CUDA): grants and cached values are
// kept per device index, a device's grant only grows, the setter runs once per device and
// size increase, and concurrent threads leave each device with the largest grant asked.
// Prints "ok" and exits 0, or prints the first failed check and exits 1.
#include <cstdio>
#include <mutex>
#include <thread>
#include <vector>

#include "launch_cache.h"

#define CHECK(c)                                                       \
    do {                                                               \
        if (!(c)) {                                                    \
            std::printf("FAILED line %d: %s\n", __LINE__, #c);         \
            return 1;                                                  \
        }                                                              \
    } while (0)

int main() {
    using rmsk::PerDevice;
    using rmsk::SmemGrant;
    {
        SmemGrant g;
        std::vector<std::pair<int, int>> calls;  // (device, bytes) passed to the setter
        int cur = 0;
        auto set = [&](int b) { calls.push_back({cur, b}); return 0; };
        cur = 0;
        CHECK(g.grant(0, 100000, set) == 0);
        CHECK(calls.size() == 1 && calls[0].second == 100000);
        CHECK(g.grant(0, 60000, set) == 0);  // smaller: nothing to set on device 0
        CHECK(calls.size() == 1);
        cur = 1;
        CHECK(g.grant(1, 60000, set) == 0);  // device 1 has its own limit
        CHECK(calls.size() == 2 && calls[1].first == 1 && calls[1].second == 60000);
        cur = 0;
        CHECK(g.grant(0, 200000, set) == 0);  // larger: set again on device 0
        CHECK(calls.size() == 3 && calls[2].second == 200000);
        CHECK(g.granted(0) == 200000 && g.granted(1) == 60000 && g.granted(2) == 0);
        // a failing setter leaves the grant unchanged and returns its code
        CHECK(g.grant(2, 5000, [](int) { return 7; }) == 7);
        CHECK(g.granted(2) == 0);
        // devices beyond the table are not cached: the setter runs every time
        int n = 0;
        auto count = [&](int) { ++n; return 0; };
        g.grant(rmsk::kMaxDevices, 10, count);
        g.grant(rmsk::kMaxDevices, 10, count);
        CHECK(n == 2);
    }
    {
        PerDevice<3> c;
        int runs = 0;
        CHECK(c.get(0, 0, [&] { ++runs; return 4; }) == 4);
        CHECK(c.get(0, 0, [&] { ++runs; return 9; }) == 4);  // cached
        CHECK(c.get(1, 0, [&] { ++runs; return 9; }) == 9);  // other device
        CHECK(c.get(0, 2, [&] { ++runs; return 2; }) == 2);  // other key
        CHECK(runs == 3);
        CHECK(c.get(0, 1, [&] { ++runs; return -1; }) == -1);  // failures are not stored
        CHECK(c.get(0, 1, [&] { ++runs; return 5; }) == 5);
        CHECK(runs == 5);
        CHECK(c.get(0, 3, [&] { ++runs; return 6; }) == 6);  // key out of range: uncached
        CHECK(c.get(0, 3, [&] { ++runs; return 6; }) == 6);
        CHECK(runs == 7);
    }
    {
        // many threads, two devices: the final grant is the largest asked on each device, and
        // the grants each device saw through its setter only ever grew
        SmemGrant g;
        std::vector<int> seen[2];
        std::mutex mu;
        std::vector<std::thread> ts;
        for (int t = 0; t < 16; ++t)
            ts.emplace_back([&, t] {
                for (int i = 0; i < 2000; ++i) {
                    const int dev = (t + i) & 1;
                    const int bytes = 1000 + ((t * 7919 + i * 104729) % 200000);
                    g.grant(dev, bytes, [&](int b) {
                        std::lock_guard<std::mutex> l(mu);
                        seen[dev].push_back(b);
                        return 0;
                    });
                }
            });
        for (auto& th : ts) th.join();
        int most[2] = {0, 0};
        for (int t = 0; t < 16; ++t)
            for (int i = 0; i < 2000; ++i) {
                const int dev = (t + i) & 1;
                const int bytes = 1000 + ((t * 7919 + i * 104729) % 200000);
                if (bytes > most[dev]) most[dev] = bytes;
            }
        for (int d = 0; d < 2; ++d) {
            CHECK(g.granted(d) == most[d]);
            for (size_t k = 1; k < seen[d].size(); ++k) CHECK(seen[d][k] > seen[d][k - 1]);
        }
    }
    std::printf("ok\n");
    return 0;
}
