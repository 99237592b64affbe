// Host-side TMA tensor-map encoding through the driver entry point (no link
// against libcuda): a 3-D view [dim2][dim1][dim0] of a contiguous bf16 array.
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"

namespace nsa {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int device_sm_count() {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cache[dev] = sms;
  return sms;
}

cudaError_t ensure_dyn_smem(const void* func, int bytes) {
  struct Entry {
    const void* f;
    int dev, bytes;
  };
  static std::mutex mu;
  static Entry done[256];
  static int ndone = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // The lock is held across the attribute call, so no caller can see the
  // kernel as prepared before the limit is raised.
  std::lock_guard<std::mutex> lk(mu);
  for (int i = 0; i < ndone; ++i)
    if (done[i].f == func && done[i].dev == dev && done[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  for (int i = 0; i < ndone; ++i)
    if (done[i].f == func && done[i].dev == dev) {
      done[i].bytes = bytes;
      return cudaSuccess;
    }
  if (ndone < 256) done[ndone++] = Entry{func, dev, bytes};
  return cudaSuccess;
}

namespace {
struct MapKey {
  const void* base;
  uint64_t d0, d1, d2;
  uint32_t b0, b1, b2;
  bool swz;
  int dev;
  bool operator==(const MapKey& o) const {
    return base == o.base && d0 == o.d0 && d1 == o.d1 && d2 == o.d2 && b0 == o.b0 &&
           b1 == o.b1 && b2 == o.b2 && swz == o.swz && dev == o.dev;
  }
};
constexpr int kMapCache = 32;
MapKey g_keys[kMapCache];
CUtensorMap g_maps[kMapCache];
int g_next = 0;
std::mutex g_mu;
}  // namespace

// Encoded maps are cached (keyed by address, shape, box and device): encoding
// costs a driver call, and a decode step reuses the same buffers every call.
bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t dim0, uint64_t dim1,
                       uint64_t dim2, uint32_t box0, uint32_t box1, uint32_t box2, bool swizzle128) {
  int dev = 0;
  cudaGetDevice(&dev);
  const MapKey key{base, dim0, dim1, dim2, box0, box1, box2, swizzle128, dev};
  {
    std::lock_guard<std::mutex> lk(g_mu);
    for (int i = 0; i < kMapCache; ++i)
      if (g_keys[i] == key) {
        *m = g_maps[i];
        return true;
      }
  }
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {dim0, dim1, dim2};
  cuuint64_t strides[2] = {dim0 * 2, dim0 * dim1 * 2};   // bytes, dims 1 and 2
  cuuint32_t box[3] = {box0, box1, box2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  g_keys[g_next] = key;
  g_maps[g_next] = *m;
  g_next = (g_next + 1) % kMapCache;
  return true;
}

}  // namespace nsa
