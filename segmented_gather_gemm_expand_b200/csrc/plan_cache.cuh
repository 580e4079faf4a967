// Host cache of launch plans.
//
// A plan of the tensor-core kernels holds TMA tensor maps; encoding one costs
// about a microsecond of host time, and a call needs up to ten.  A serving loop
// calls again and again with the same buffers and shapes, so plans are kept,
// keyed by every byte of a key struct the caller fills (every field of the
// call's problem, the device, its SM count and any forced choice).  A call the
// kernel cannot take is kept too, as a miss.  The cache is direct-mapped by an
// FNV-1a hash of the key; a collision replaces the slot.  Lookups and stores
// hold a mutex; the plan is built outside it.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>

namespace sgmv {

template <class Key, class Plan, int SLOTS = 64>
class PlanCache {
public:
    // The plan for key: a stored one, else build(out) (a bool-returning
    // callable that fills *out), which is then stored.  The key must be
    // fully written, padding included (memset it before filling the fields),
    // since keys compare as bytes.
    template <class Build>
    bool get(const Key& key, Plan* out, Build&& build) {
        Slot& slot = slots_[hash(key) % SLOTS];
        {
            std::lock_guard<std::mutex> lk(mu_);
            if (slot.used && std::memcmp(&slot.key, &key, sizeof(Key)) == 0) {
                if (slot.ok) *out = slot.plan;
                return slot.ok;
            }
        }
        const bool ok = build(out);
        std::lock_guard<std::mutex> lk(mu_);
        slot.used = true;
        slot.ok = ok;
        slot.key = key;
        if (ok) slot.plan = *out;
        return ok;
    }

private:
    struct Slot {
        bool used = false, ok = false;
        Key key;
        Plan plan;
    };
    static uint64_t hash(const Key& key) {
        const unsigned char* b = reinterpret_cast<const unsigned char*>(&key);
        uint64_t h = 1469598103934665603ull;
        for (size_t i = 0; i < sizeof(Key); ++i) h = (h ^ b[i]) * 1099511628211ull;
        return h;
    }
    Slot slots_[SLOTS];
    std::mutex mu_;
};

}  // namespace sgmv
