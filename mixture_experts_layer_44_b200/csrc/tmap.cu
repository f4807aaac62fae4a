// Tensor-map encoding through the driver entry point, with a small cache.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "tmap.cuh"

namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_uncached(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int rank,
                     const cuuint64_t* dims, const cuuint64_t* strides_bytes,
                     const cuuint32_t* box) {
  auto fn = get_encode();
  if (!fn) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, dt, rank, const_cast<void*>(base), dims,
                  strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Small cache of encoded tensor maps: a layer called again on the same
// buffers reuses its descriptors instead of encoding four per call.  The map
// depends only on the key (device, base, rank, dims, strides, box).
struct MapKey {
  int dev, rank, dtype;
  const void* base;
  cuuint64_t dims[3], strides[2];
  cuuint32_t box[3];
};

}  // namespace

namespace moe_host {

namespace {

bool encode_cached(CUtensorMap* m, CUtensorMapDataType dt, const void* base, int rank,
                   const cuuint64_t* dims, const cuuint64_t* strides_bytes,
                   const cuuint32_t* box) {
  constexpr int kSlots = 64;
  static std::mutex mu;
  static MapKey keys[kSlots];
  static CUtensorMap maps[kSlots];
  static int used = 0, next = 0;
  MapKey k;
  std::memset(&k, 0, sizeof(k));
  cudaGetDevice(&k.dev);
  k.rank = rank;
  k.dtype = static_cast<int>(dt);
  k.base = base;
  for (int i = 0; i < rank; ++i) {
    k.dims[i] = dims[i];
    k.box[i] = box[i];
    if (i + 1 < rank) k.strides[i] = strides_bytes[i];
  }
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (std::memcmp(&keys[i], &k, sizeof(k)) == 0) {
      *m = maps[i];
      return true;
    }
  if (!encode_uncached(m, dt, base, rank, dims, strides_bytes, box)) return false;
  const int slot = used < kSlots ? used++ : (next++ % kSlots);
  keys[slot] = k;
  maps[slot] = *m;
  return true;
}

}  // namespace

bool encode_bf16_sw128(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                       const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  return encode_cached(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box);
}

bool encode_f16_sw128(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                      const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  return encode_cached(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base, rank, dims, strides_bytes, box);
}

bool encode_f32_sw128(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                      const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  return encode_cached(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, rank, dims, strides_bytes, box);
}

}  // namespace moe_host
