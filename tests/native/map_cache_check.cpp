// Host-only check of the tensor-map cache (dg_map_cache.h) with a fake encoder: a hit returns
// the bytes the encoder produced for the same arguments, any differing argument misses,
// colliding keys evict correctly, turning the cache off drops entries, and concurrent callers
// always receive the map of their own arguments.  Exit status 0 = all checks passed.
#include <cstdio>
#include <cstring>
#include <thread>
#include <vector>

#include "dg_map_cache.h"

static int g_encodes = 0;
static int g_failures = 0;

#define CHECK(c)                                                            \
    do {                                                                    \
        if (!(c)) {                                                         \
            std::fprintf(stderr, "check failed: %s (line %d)\n", #c, __LINE__); \
            ++g_failures;                                                   \
        }                                                                   \
    } while (0)

// The fake map: its first bytes are a digest of the key's words and then its base address,
// enough to tell maps of different keys apart.
static void fake_fill(const dg::TensorMapKey &k, CUtensorMap *out)
{
    std::memset(out, 0, sizeof(*out));
    uint64_t words[sizeof(k) / 8];
    std::memcpy(words, &k, sizeof(words));
    uint64_t acc = 0;
    for (uint64_t w : words)
        acc = acc * 31 + w;
    std::memcpy(out, &acc, sizeof(acc));
    std::memcpy(reinterpret_cast<char *>(out) + 8, &k.base, sizeof(k.base));
}

struct Args {
    uint64_t base;
    cuuint64_t dims[3];
    cuuint64_t strides[2];
    cuuint32_t box[3];
    CUtensorMapSwizzle sw;
};

static dg::TensorMapKey key_of(const Args &a)
{
    cuuint32_t estr[3] = {1, 1, 1};
    dg::TensorMapKey k;
    dg::make_map_key(k, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, reinterpret_cast<void *>(a.base), a.dims,
                     a.strides, a.box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, a.sw,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return k;
}

static CUtensorMap lookup(dg::TensorMapCache &c, const Args &a)
{
    const dg::TensorMapKey k = key_of(a);
    CUtensorMap m;
    CUresult r = c.get(k, &m, [&](CUtensorMap *out) {
        ++g_encodes;
        fake_fill(k, out);
        return CUDA_SUCCESS;
    });
    CHECK(r == CUDA_SUCCESS);
    return m;
}

static bool same(const CUtensorMap &x, const CUtensorMap &y)
{
    return std::memcmp(&x, &y, sizeof(x)) == 0;
}

int main()
{
    static dg::TensorMapCache cache;
    Args a{0x10000, {7168, 4096, 1}, {7168, 7168ull * 4096}, {128, 128, 1}, CU_TENSOR_MAP_SWIZZLE_128B};

    // a repeat hits and returns the same bytes
    CUtensorMap m1 = lookup(cache, a);
    CUtensorMap m2 = lookup(cache, a);
    CHECK(g_encodes == 1);
    CHECK(same(m1, m2));

    // every argument matters
    Args b = a;
    b.base += 256;
    lookup(cache, b);
    Args c = a;
    c.dims[1] = 4095;
    lookup(cache, c);
    Args d = a;
    d.box[1] = 64;
    lookup(cache, d);
    Args e = a;
    e.sw = CU_TENSOR_MAP_SWIZZLE_64B;
    lookup(cache, e);
    Args f = a;
    f.strides[1] += 16;
    lookup(cache, f);
    CHECK(g_encodes == 6);
    CHECK(!same(lookup(cache, b), m1));

    // unused trailing dimensions do not leak into the key
    cuuint64_t dims5[5] = {1, 2, 3, 99, 99}, str5[4] = {16, 32, 77, 77};
    cuuint32_t box5[5] = {1, 1, 1, 55, 55}, es5[5] = {1, 1, 1, 9, 9};
    dg::TensorMapKey k1, k2;
    dg::make_map_key(k1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, nullptr, dims5, str5, box5, es5,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    dims5[3] = 0;
    str5[2] = 0;
    box5[3] = 0;
    es5[3] = 0;
    dg::make_map_key(k2, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, nullptr, dims5, str5, box5, es5,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    CHECK(std::memcmp(&k1, &k2, sizeof(k1)) == 0);

    // many more keys than slots: every lookup still returns the map of its own key
    std::vector<Args> many;
    for (int i = 0; i < 3 * dg::TensorMapCache::kSlots; ++i) {
        Args x = a;
        x.base = 0x100000 + 512ull * i;
        many.push_back(x);
    }
    for (const Args &x : many) {
        CUtensorMap m = lookup(cache, x);
        CUtensorMap ref;
        fake_fill(key_of(x), &ref);
        CHECK(same(m, ref));
    }
    for (const Args &x : many) {
        CUtensorMap m = lookup(cache, x);
        CUtensorMap ref;
        fake_fill(key_of(x), &ref);
        CHECK(same(m, ref));
    }

    // off: every lookup encodes; on again: a repeat hits
    CHECK(cache.set_enabled(false) == true);
    int before = g_encodes;
    lookup(cache, a);
    lookup(cache, a);
    CHECK(g_encodes == before + 2);
    CHECK(cache.set_enabled(true) == false);
    lookup(cache, a);
    before = g_encodes;
    lookup(cache, a);
    CHECK(g_encodes == before);

    // concurrent callers receive the map of their own arguments
    std::vector<std::thread> ts;
    int bad[4] = {0, 0, 0, 0};
    for (int t = 0; t < 4; ++t) {
        ts.emplace_back([&, t]() {
            for (int i = 0; i < 2000; ++i) {
                Args x = a;
                x.base = 0x200000 + 1024ull * ((i * 7 + t) % 300);
                const dg::TensorMapKey k = key_of(x);
                CUtensorMap m;
                cache.get(k, &m, [&](CUtensorMap *out) {
                    fake_fill(k, out);
                    return CUDA_SUCCESS;
                });
                CUtensorMap ref;
                fake_fill(k, &ref);
                if (!same(m, ref))
                    ++bad[t];
            }
        });
    }
    for (auto &th : ts)
        th.join();
    CHECK(bad[0] + bad[1] + bad[2] + bad[3] == 0);

    // a failed encode is not cached
    Args z = a;
    z.base = 0xdead00;
    const dg::TensorMapKey kz = key_of(z);
    CUtensorMap mz;
    CHECK(cache.get(kz, &mz, [](CUtensorMap *) { return CUDA_ERROR_INVALID_VALUE; }) ==
          CUDA_ERROR_INVALID_VALUE);
    int calls = 0;
    cache.get(kz, &mz, [&](CUtensorMap *out) {
        ++calls;
        fake_fill(kz, out);
        return CUDA_SUCCESS;
    });
    CHECK(calls == 1);

    unsigned long long hits = 0, misses = 0;
    cache.stats(hits, misses);
    CHECK(hits > 0 && misses > 0);
    if (g_failures == 0)
        std::printf("map cache: all checks passed (%llu hits, %llu misses)\n", hits, misses);
    return g_failures == 0 ? 0 : 1;
}
