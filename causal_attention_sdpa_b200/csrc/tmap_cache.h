// Host-side cache of encoded TMA tensor maps.
//
// A tensor map (CUtensorMap, 128 bytes) is a pure function of its key: the
// tensor's base address, element type, extents and strides, the box and the
// swizzle.  Encoding one costs a driver call; every forward call needs four
// and every backward call up to seven, so repeated calls on the same buffers
// (a training loop, a benchmark) look them up here instead.  Because the
// value depends on nothing but the key, a hit is always correct, even when a
// buffer was freed and another one allocated at the same address.
//
// The cache is a fixed table of kSlots entries with round-robin replacement,
// guarded by a mutex (the library may be called from several host threads).
// It is written against an encoder functor so that host tests can check it
// with a fake encoder and no GPU.
#pragma once

#include <stdint.h>
#include <string.h>

#include <mutex>

namespace gpt_attn {

enum class TmapKind : int {
    kBf16Box64x128 = 1,    // bf16 4-D (D, T, H, B) with strides, 64-column x 128-row boxes, 128-byte swizzle
    kF32Box32x128 = 2,     // fp32 3-D (D, T, B*H) contiguous, 32-column x 128-row boxes, 128-byte swizzle
};

struct TmapKey {
    uintptr_t base;
    int kind;
    int d0, d1, d2, d3;    // extents, innermost first: D, T, H, B (fp32 maps: D, T, B*H, 1)
    long long s1, s2, s3;  // element strides of dimensions 1..3 (token, head, batch)
    bool operator==(const TmapKey& o) const {
        return base == o.base && kind == o.kind && d0 == o.d0 && d1 == o.d1 && d2 == o.d2 && d3 == o.d3 &&
               s1 == o.s1 && s2 == o.s2 && s3 == o.s3;
    }
};

// Value is a trivially copyable 128-byte map (CUtensorMap in the library, a
// plain struct in the host tests).
template <typename Value, int kSlots = 64>
class TmapCache {
public:
    // Returns true and fills `out` on a hit or a successful encode; returns false
    // (and caches nothing) if `encode(key, &value)` fails.
    template <typename Encode>
    bool get(const TmapKey& key, Value* out, Encode&& encode) {
        {
            std::lock_guard<std::mutex> lk(mu_);
            for (int i = 0; i < used_; ++i) {
                if (keys_[i] == key) {
                    memcpy(out, &vals_[i], sizeof(Value));
                    ++hits_;
                    return true;
                }
            }
        }
        Value v;
        if (!encode(key, &v)) return false;
        std::lock_guard<std::mutex> lk(mu_);
        ++misses_;
        int slot;
        if (used_ < kSlots) {
            slot = used_++;
        } else {
            slot = next_;
            next_ = (next_ + 1) % kSlots;
        }
        keys_[slot] = key;
        memcpy(&vals_[slot], &v, sizeof(Value));
        memcpy(out, &v, sizeof(Value));
        return true;
    }

    void stats(long long* hits, long long* misses, int* used) {
        std::lock_guard<std::mutex> lk(mu_);
        *hits = hits_;
        *misses = misses_;
        *used = used_;
    }

    void clear() {
        std::lock_guard<std::mutex> lk(mu_);
        used_ = next_ = 0;
        hits_ = misses_ = 0;
    }

private:
    std::mutex mu_;
    TmapKey keys_[kSlots];
    Value vals_[kSlots];
    int used_ = 0;
    int next_ = 0;
    long long hits_ = 0, misses_ = 0;
};

}  // namespace gpt_attn
