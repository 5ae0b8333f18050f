// Host check of the tensor-map cache (tmap_cache.h) with a fake encoder that counts its
// calls and writes a pattern derived from the key into the map: a repeated key must be
// served without encoding and return the map made for it; different pointers, shapes,
// boxes or devices must be encoded; the least recently used entry is the one evicted;
// a failed encode stores nothing; concurrent lookups stay consistent. Prints "ok <n>".
#include "tmap_cache.h"

#include <atomic>
#include <cstdio>
#include <thread>
#include <vector>

using namespace sq;

static std::atomic<long> g_encodes{0};

static CUresult fake_encode(const TmapKey& k, CUtensorMap* out) {
  ++g_encodes;
  std::memset(out, 0, sizeof(*out));
  const uint64_t h = tmap_key_hash(k);
  std::memcpy(out, &h, sizeof(h));
  std::memcpy(reinterpret_cast<char*>(out) + 8, &k.base, sizeof(k.base));
  return CUDA_SUCCESS;
}

static bool map_is_for(const CUtensorMap& m, const TmapKey& k) {
  CUtensorMap want;
  fake_encode(k, &want);
  --g_encodes;
  return std::memcmp(&m, &want, sizeof(m)) == 0;
}

static TmapKey key(int dev, uint64_t base, uint64_t rows, uint32_t box_b) {
  const uint64_t dims[5] = {128, 20, 11, 1, rows};
  const uint64_t strides[4] = {256, 10240, 225280, 256};
  const uint32_t box[5] = {64, 20, box_b, 1, 1};
  return make_tmap_key(dev, 10, 3, 5, reinterpret_cast<const void*>(base), dims, strides, box);
}

static int fail(const char* what) {
  std::printf("FAIL %s\n", what);
  return 1;
}

int main() {
  long checks = 0;
  {
    TmapCache<4> c;
    CUtensorMap m;
    const TmapKey a = key(0, 0x1000, 654720, 6);
    auto enc = [&](const TmapKey& k) { return [&k](CUtensorMap* o) { return fake_encode(k, o); }; };
    if (c.get(a, &m, enc(a)) != CUDA_SUCCESS || g_encodes != 1 || !map_is_for(m, a)) return fail("first get");
    if (c.get(a, &m, enc(a)) != CUDA_SUCCESS || g_encodes != 1 || !map_is_for(m, a)) return fail("repeat is a hit");
    // every field of the key matters
    const TmapKey variants[4] = {key(0, 0x2000, 654720, 6), key(0, 0x1000, 327360, 6), key(0, 0x1000, 654720, 5),
                                 key(1, 0x1000, 654720, 6)};
    for (const TmapKey& v : variants) {
      const long before = g_encodes;
      if (c.get(v, &m, enc(v)) != CUDA_SUCCESS || g_encodes != before + 1 || !map_is_for(m, v))
        return fail("distinct key encoded");
      ++checks;
    }
    // table of 4: the five keys above overflowed it once; `a` was the least recently used
    long before = g_encodes;
    c.get(a, &m, enc(a));
    if (g_encodes != before + 1 || !map_is_for(m, a)) return fail("least recently used evicted");
    before = g_encodes;
    c.get(variants[3], &m, enc(variants[3]));  // most recent before `a`: still present
    if (g_encodes != before || !map_is_for(m, variants[3])) return fail("recent entry kept");
    unsigned long long hits = 0, misses = 0;
    c.stats(&hits, &misses);
    if (hits != 2 || misses != 6) return fail("counters");
    // a failed encode stores nothing and is retried next time
    const TmapKey bad = key(0, 0x9000, 654720, 6);
    if (c.get(bad, &m, [](CUtensorMap*) { return CUDA_ERROR_INVALID_VALUE; }) != CUDA_ERROR_INVALID_VALUE)
      return fail("error passed on");
    before = g_encodes;
    if (c.get(bad, &m, enc(bad)) != CUDA_SUCCESS || g_encodes != before + 1) return fail("failure not cached");
    checks += 8;
  }
  {
    // many threads, 32 keys over a table of 16: every returned map is the one for its key
    TmapCache<16> c;
    std::atomic<int> bad{0};
    std::vector<std::thread> ts;
    for (int t = 0; t < 8; ++t)
      ts.emplace_back([&, t] {
        uint64_t s = 0x9e3779b97f4a7c15ull * (t + 1);
        for (int i = 0; i < 20000; ++i) {
          s = s * 6364136223846793005ull + 1442695040888963407ull;
          const TmapKey k = key(int(s >> 62), 0x1000 + ((s >> 40) & 7) * 0x1000, 654720, 6);
          CUtensorMap m;
          if (c.get(k, &m, [&k](CUtensorMap* o) { return fake_encode(k, o); }) != CUDA_SUCCESS || !map_is_for(m, k))
            ++bad;
        }
      });
    for (auto& th : ts) th.join();
    unsigned long long hits = 0, misses = 0;
    c.stats(&hits, &misses);
    if (bad != 0) return fail("concurrent maps");
    if (hits + misses != 8ull * 20000) return fail("concurrent counters");
    checks += 160000;
  }
  std::printf("ok %ld\n", checks);
  return 0;
}
