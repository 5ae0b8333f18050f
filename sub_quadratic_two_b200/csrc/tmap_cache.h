// tmap_cache.h - host-side cache of encoded TMA tensor maps.
//
// A forward call needs eight tensor maps and a backward call eight more; each is a
// driver call (cuTensorMapEncodeTiled) of a few microseconds on the host. A map depends
// only on the arguments of that call (base address, extents, strides, box, element type
// and swizzle) and on the device, so a call that repeats the pointers and shape of an
// earlier one can reuse its maps. The cache is a fixed table of N entries keyed on
// exactly those arguments, shared by all host threads under one mutex, and evicts the
// least recently used entry. A key never goes stale: if memory is freed and another
// buffer of the same shape is allocated at the same address, the map it holds is the
// map that address and shape encode.
#pragma once

#include <cuda.h>

#include <cstdint>
#include <cstring>
#include <mutex>

namespace sq {

struct TmapKey {
  int device;
  int dtype;    // CUtensorMapDataType
  int swizzle;  // CUtensorMapSwizzle
  int rank;
  uint64_t base;
  uint64_t dims[5];
  uint64_t strides[4];
  uint32_t box[5];
  uint32_t pad;  // keeps the struct free of implicit padding (compared bytewise)
};

inline TmapKey make_tmap_key(int device, int dtype, int swizzle, int rank, const void* base, const uint64_t* dims,
                             const uint64_t* strides, const uint32_t* box) {
  TmapKey k;
  std::memset(&k, 0, sizeof(k));
  k.device = device;
  k.dtype = dtype;
  k.swizzle = swizzle;
  k.rank = rank;
  k.base = reinterpret_cast<uint64_t>(base);
  for (int i = 0; i < rank && i < 5; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
    if (i < 4 && i + 1 < rank) k.strides[i] = strides[i];
  }
  return k;
}

// A 64-bit hash of the key's words (multiply and xor-shift per word): a cheap first
// comparison before the full one.
inline uint64_t tmap_key_hash(const TmapKey& k) {
  static_assert(sizeof(TmapKey) % 8 == 0, "key is hashed as 64-bit words");
  uint64_t w[sizeof(TmapKey) / 8];
  std::memcpy(w, &k, sizeof(k));
  uint64_t h = 0x9e3779b97f4a7c15ull;
  for (size_t i = 0; i < sizeof(TmapKey) / 8; ++i) {
    h = (h ^ w[i]) * 0xff51afd7ed558ccdull;
    h ^= h >> 32;
  }
  return h;
}

template <int N>
class TmapCache {
 public:
  // The map for `key`: copied from the table, or made by enc(CUtensorMap*) -> CUresult
  // (called without the lock held) and stored. A failed encode stores nothing.
  template <typename Enc>
  CUresult get(const TmapKey& key, CUtensorMap* out, Enc&& enc) {
    const uint64_t h = tmap_key_hash(key);
    {
      std::lock_guard<std::mutex> lock(mu_);
      for (int i = 0; i < used_; ++i) {
        if (slots_[i].hash == h && std::memcmp(&slots_[i].key, &key, sizeof(key)) == 0) {
          slots_[i].stamp = ++clock_;
          *out = slots_[i].map;
          ++hits_;
          return CUDA_SUCCESS;
        }
      }
    }
    CUtensorMap m;
    const CUresult r = enc(&m);
    if (r != CUDA_SUCCESS) return r;
    std::lock_guard<std::mutex> lock(mu_);
    ++misses_;
    int slot = -1;
    for (int i = 0; i < used_ && slot < 0; ++i)  // another thread may have stored it meanwhile
      if (slots_[i].hash == h && std::memcmp(&slots_[i].key, &key, sizeof(key)) == 0) slot = i;
    if (slot < 0) {
      if (used_ < N) {
        slot = used_++;
      } else {
        slot = 0;
        for (int i = 1; i < N; ++i)
          if (slots_[i].stamp < slots_[slot].stamp) slot = i;
      }
    }
    slots_[slot].key = key;
    slots_[slot].hash = h;
    slots_[slot].map = m;
    slots_[slot].stamp = ++clock_;
    *out = m;
    return CUDA_SUCCESS;
  }

  void stats(unsigned long long* hits, unsigned long long* misses) {
    std::lock_guard<std::mutex> lock(mu_);
    if (hits != nullptr) *hits = hits_;
    if (misses != nullptr) *misses = misses_;
  }

 private:
  struct Slot {
    TmapKey key;
    uint64_t hash;
    uint64_t stamp;
    CUtensorMap map;
  };
  Slot slots_[N];
  int used_ = 0;
  uint64_t clock_ = 0;
  unsigned long long hits_ = 0, misses_ = 0;
  std::mutex mu_;
};

}  // namespace sq
