// Host-side check of the per-device shared-memory limit cache (lb_attr_cache.h): devices are kept apart, the
// record only grows, a failed raise leaves it as it was, and racing threads end with the largest request
// raised on every device, each device's limit never lowered.
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <thread>
#include <vector>

#include "lb_attr_cache.h"

#define CHECK(c)                                                                  \
    do {                                                                          \
        if (!(c)) {                                                               \
            std::fprintf(stderr, "check failed line %d: %s\n", __LINE__, #c);     \
            std::exit(1);                                                         \
        }                                                                         \
    } while (0)

static int kernel_a, kernel_b;   // stand-ins for two kernels' addresses

int main()
{
    lb::AttrCache c;
    int calls = 0;
    auto ok = [&](long) { ++calls; return 0; };
    CHECK(c.ensure(0, &kernel_a, 1000, ok) == 0 && calls == 1);
    CHECK(c.ensure(0, &kernel_a, 800, ok) == 0 && calls == 1);        // already enough on device 0
    CHECK(c.ensure(1, &kernel_a, 800, ok) == 0 && calls == 2);        // device 1 is raised on its own
    CHECK(c.ensure(0, &kernel_b, 800, ok) == 0 && calls == 3);        // and every kernel on its own
    CHECK(c.ensure(0, &kernel_a, 2000, ok) == 0 && calls == 4);
    CHECK(c.raised(0, &kernel_a) == 2000 && c.raised(1, &kernel_a) == 800);
    // a failed raise returns the error and leaves the record alone
    CHECK(c.ensure(1, &kernel_a, 5000, [](long) { return 7; }) == 7);
    CHECK(c.raised(1, &kernel_a) == 800);

    // racing threads on four devices: the setter sees only increasing values per device
    lb::AttrCache r;
    std::atomic<long> last[4];
    std::atomic<int> bad{0};
    for (auto &x : last) x = 0;
    std::vector<std::thread> ts;
    for (int t = 0; t < 8; ++t)
        ts.emplace_back([&, t]() {
            for (int i = 0; i < 2000; ++i) {
                const int dev = (i + t) & 3;
                const long want = 1 + (i * 7919 + t * 104729) % 50000;
                r.ensure(dev, &kernel_a, want, [&](long b) {
                    if (b <= last[dev].load()) ++bad;
                    last[dev] = b;
                    return 0;
                });
                if (r.raised(dev, &kernel_a) < want) ++bad;
            }
        });
    for (auto &th : ts) th.join();
    CHECK(bad == 0);
    for (int d = 0; d < 4; ++d) CHECK(r.raised(d, &kernel_a) == last[d].load());
    std::printf("attr cache ok\n");
    return 0;
}
