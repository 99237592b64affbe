// nsa_decode_noalloc: the decode entry point for callers that cannot allocate
// device memory, with its scratch in a static device array of this module.
#include <cstdio>
#include <mutex>

#include "internal.h"

namespace nsa {
namespace {

// Scratch of the no-allocation decode. Every GPU that loads this module holds
// it until the process exits; decode needs about 39 MB for 32 sequences of
// 65536 tokens with 4 KV heads.
constexpr size_t kNoAllocScratchBytes = 64ull << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch on the current device. In host code the
// array's name only stands for the symbol, so the address is looked up once
// per device, with that device current, and cached.
nsa_status scratch_address(void** out) {
  static std::mutex mu;
  static void* cache[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 128) {
    set_last_error(NSA_ERR_CUDA, "cudaGetDevice failed");
    return NSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      char msg[160];
      snprintf(msg, sizeof(msg), "cudaGetSymbolAddress(static decode scratch): %s",
               cudaGetErrorString(e));
      set_last_error(NSA_ERR_CUDA, msg);
      return NSA_ERR_CUDA;
    }
    cache[dev] = p;
  }
  *out = cache[dev];
  return NSA_OK;
}

}  // namespace
}  // namespace nsa

using namespace nsa;

extern "C" nsa_status nsa_decode_noalloc(const nsa_params* p, const void* q, const void* k_cache,
                                         const void* v_cache, const int32_t* seq_lens,
                                         const void* k_cmp, const void* v_cmp,
                                         const float* w_gate, void* out, int32_t* sel_idx,
                                         void* stream) {
  size_t need = 0;
  nsa_status st = nsa_workspace_size(p, NSA_OP_DECODE, &need);
  if (st != NSA_OK) return st;
  if (need > kNoAllocScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "decode needs %zu bytes of scratch but the static scratch holds %zu; "
             "use nsa_decode with a caller workspace",
             need, kNoAllocScratchBytes);
    set_last_error(NSA_ERR_UNSUPPORTED, msg);
    return NSA_ERR_UNSUPPORTED;
  }
  void* ws = nullptr;
  if (need > 0) {
    st = scratch_address(&ws);
    if (st != NSA_OK) return st;
  }
  return nsa_decode(p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, w_gate, out, sel_idx, ws,
                    need > 0 ? kNoAllocScratchBytes : 0, stream);
}
