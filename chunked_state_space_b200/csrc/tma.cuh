// Host-side creation of TMA tensor maps (cuTensorMapEncodeTiled, fetched
// from the driver through the runtime so that libssd does not link libcuda).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <unordered_map>

namespace ssd {
namespace tma {

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// Tiled map over a bf16 tensor of `rank` dims (innermost first); strides in
// bytes for dims 1..rank-1; box in elements.  128-byte swizzle by default.
inline bool encode(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank, const uint64_t* dims,
                   const uint64_t* strides_bytes, const uint32_t* box,
                   CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), (const cuuint64_t*)dims,
                  (const cuuint64_t*)strides_bytes, (const cuuint32_t*)box, (const cuuint32_t*)es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline bool encode_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                        const uint64_t* strides_bytes, const uint32_t* box,
                        CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box, sw);
}

// encode_bf16 for rank-4 maps with the default swizzle, remembered by their
// arguments: a map depends only on them, so a caller that launches on the same
// buffers again (a layer stack, a benchmark loop) skips the driver call.  The
// table is bounded (cleared when full) and guarded by a mutex.
struct MapKey {
  const void* base;
  uint64_t dims[4], strides[3];
  uint32_t box[4];
  bool operator==(const MapKey& o) const {
    return base == o.base && memcmp(dims, o.dims, sizeof(dims)) == 0 && memcmp(strides, o.strides, sizeof(strides)) == 0 &&
           memcmp(box, o.box, sizeof(box)) == 0;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    uint64_t h = 1469598103934665603ull;
    auto mix = [&](uint64_t v) { h = (h ^ v) * 1099511628211ull; };
    mix((uint64_t)(uintptr_t)k.base);
    for (uint64_t v : k.dims) mix(v);
    for (uint64_t v : k.strides) mix(v);
    for (uint32_t v : k.box) mix(v);
    return (size_t)h;
  }
};

inline bool encode_bf16_4d_cached(CUtensorMap* map, const void* base, const uint64_t* dims,
                                  const uint64_t* strides_bytes, const uint32_t* box) {
  static std::mutex mu;
  static std::unordered_map<MapKey, CUtensorMap, MapKeyHash> table;
  MapKey key;
  key.base = base;
  memcpy(key.dims, dims, sizeof(key.dims));
  memcpy(key.strides, strides_bytes, sizeof(key.strides));
  memcpy(key.box, box, sizeof(key.box));
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = table.find(key);
    if (it != table.end()) {
      *map = it->second;
      return true;
    }
  }
  if (!encode_bf16(map, base, 4, dims, strides_bytes, box)) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (table.size() >= 65536) table.clear();
  table.emplace(key, *map);
  return true;
}

}  // namespace tma
}  // namespace ssd
