// dg_map_cache.h -- cache of encoded TMA tensor maps.
//
// A tensor map (CUtensorMap) is a pure function of the arguments of cuTensorMapEncodeTiled:
// element type, rank, base address, sizes, strides, box, element strides, interleave, swizzle,
// L2 promotion and out-of-bounds fill.  Encoding costs host time on every GEMM call (two to four
// maps per call), while a serving loop calls the same GEMMs on the same buffers again and again.
// The cache keys an entry on ALL of those arguments, compared byte for byte, so a hit returns
// exactly the map the driver would encode: there is no staleness to manage (a freed and
// re-allocated buffer at the same address with the same layout is described by the same map).
// Direct-mapped, kSlots entries, one mutex; a colliding key simply replaces the entry.
#pragma once

#include <cuda.h>

#include <cstdint>
#include <cstring>
#include <mutex>

namespace dg {

struct TensorMapKey {
    uint64_t base;
    uint64_t dims[5];
    uint64_t strides[4];
    uint32_t box[5];
    uint32_t estr[5];
    int32_t dtype, rank, interleave, swizzle, l2, oob;
};

// Fills `k` from encode arguments; every byte (padding included) is defined, so keys compare
// with memcmp.
inline void make_map_key(TensorMapKey &k, CUtensorMapDataType dt, uint32_t rank, const void *base,
                         const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box,
                         const cuuint32_t *estr, CUtensorMapInterleave il, CUtensorMapSwizzle sw,
                         CUtensorMapL2promotion l2, CUtensorMapFloatOOBfill oob)
{
    std::memset(&k, 0, sizeof(k));
    k.base = reinterpret_cast<uint64_t>(base);
    for (uint32_t i = 0; i < rank && i < 5; ++i) {
        k.dims[i] = dims[i];
        k.box[i] = box[i];
        k.estr[i] = estr[i];
        if (i + 1 < rank && i < 4)
            k.strides[i] = strides[i];
    }
    k.dtype = static_cast<int32_t>(dt);
    k.rank = static_cast<int32_t>(rank);
    k.interleave = static_cast<int32_t>(il);
    k.swizzle = static_cast<int32_t>(sw);
    k.l2 = static_cast<int32_t>(l2);
    k.oob = static_cast<int32_t>(oob);
}

class TensorMapCache {
public:
    static constexpr int kSlots = 1024;

    // Returns the cached map for `k`, or calls encode(out) and caches its result on success.
    template <class Encode>
    CUresult get(const TensorMapKey &k, CUtensorMap *out, Encode encode)
    {
        const uint32_t slot = static_cast<uint32_t>(hash(k) % kSlots);
        {
            std::lock_guard<std::mutex> lock(mu_);
            if (enabled_) {
                const Entry &e = entries_[slot];
                if (e.valid && std::memcmp(&e.key, &k, sizeof(k)) == 0) {
                    *out = e.map;
                    ++hits_;
                    return CUDA_SUCCESS;
                }
            }
        }
        const CUresult r = encode(out);
        if (r == CUDA_SUCCESS) {
            std::lock_guard<std::mutex> lock(mu_);
            ++misses_;
            if (enabled_) {
                Entry &e = entries_[slot];
                e.valid = true;
                std::memcpy(&e.key, &k, sizeof(k));
                e.map = *out;
            }
        }
        return r;
    }

    // Turns the cache on or off (off also drops every entry); returns the previous state.
    bool set_enabled(bool on)
    {
        std::lock_guard<std::mutex> lock(mu_);
        const bool prev = enabled_;
        enabled_ = on;
        if (!on)
            for (Entry &e : entries_)
                e.valid = false;
        return prev;
    }

    void stats(unsigned long long &hits, unsigned long long &misses)
    {
        std::lock_guard<std::mutex> lock(mu_);
        hits = hits_;
        misses = misses_;
    }

private:
    struct Entry {
        bool valid = false;
        TensorMapKey key;
        CUtensorMap map;
    };

    // FNV-1a over the key's bytes
    static uint64_t hash(const TensorMapKey &k)
    {
        const unsigned char *p = reinterpret_cast<const unsigned char *>(&k);
        uint64_t h = 1469598103934665603ull;
        for (size_t i = 0; i < sizeof(k); ++i) {
            h ^= p[i];
            h *= 1099511628211ull;
        }
        return h;
    }

    std::mutex mu_;
    bool enabled_ = true;
    unsigned long long hits_ = 0, misses_ = 0;
    Entry entries_[kSlots];
};

}  // namespace dg
