// Per-device record of the dynamic shared-memory limit raised for each kernel.
//
// CUDA keeps a kernel's maximum dynamic shared memory per device context, so a
// process that drives several GPUs, or several host threads making their
// first calls at once, must raise it per device and must not race on the
// record.  This cache is keyed by (device, kernel), locked, and grow-only: the
// setter runs only when a larger limit than any raised so far on that device
// is needed, and the record is updated only after the setter succeeded.
// Plain C++ (no CUDA types), so that its logic is tested on the host.
#pragma once

#include <map>
#include <mutex>
#include <utility>

namespace lb {

class AttrCache {
public:
    // Ensures the limit of `fn` on `device` is at least `bytes`; `set(bytes)` raises it and returns 0 on
    // success (its error code otherwise, returned unchanged; the record is then left as it was).
    template <typename Setter>
    int ensure(int device, const void *fn, long bytes, Setter &&set)
    {
        std::lock_guard<std::mutex> lock(mu_);
        long &have = raised_[std::make_pair(device, fn)];
        if (bytes <= have) return 0;
        const int e = set(bytes);
        if (e == 0) have = bytes;
        return e;
    }
    long raised(int device, const void *fn)
    {
        std::lock_guard<std::mutex> lock(mu_);
        auto it = raised_.find(std::make_pair(device, fn));
        return it == raised_.end() ? 0 : it->second;
    }

private:
    std::mutex mu_;
    std::map<std::pair<int, const void *>, long> raised_;
};

}  // namespace lb
