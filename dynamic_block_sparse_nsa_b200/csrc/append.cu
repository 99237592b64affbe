// Streaming decode: one new token per sequence goes into the KV caches, and
// every s tokens a new compressed block becomes complete (lchairun NSA
// article: decode reads the compressed cache and the selected / recent tokens;
// EP94 notes section five: compressed block i covers tokens [i s, i s + l - 1]).
//
// The block written here is computed exactly as nsa_compress_kv computes it
// (fp64 products and sum over j = 0 .. l - 1 in that order, one rounding), so a
// cache grown token by token equals the compression of the whole sequence.
#include "device_common.cuh"
#include "internal.h"

namespace nsa {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) append_kernel(const T* __restrict__ k_new,
                                                     const T* __restrict__ v_new,
                                                     const int32_t* __restrict__ pos,
                                                     T* __restrict__ kc_, T* __restrict__ vc_,
                                                     const float* __restrict__ w,
                                                     T* __restrict__ k_cmp, T* __restrict__ v_cmp,
                                                     unsigned* err, int T_, int Hkv, int d, int l,
                                                     int s, int Nc) {
  const int b = blockIdx.y;
  const long row = (long)Hkv * d;
  const int p = pos[b];
  if (p < 0 || p >= T_) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(err, kErrAppendPos);
    return;
  }
  const bool closes = p + 1 >= l && (p + 1 - l) % s == 0;  // block i = (p + 1 - l) / s completes
  const int i = closes ? (p + 1 - l) / s : -1;
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < row;
       e += (long)gridDim.x * blockDim.x) {
    const T kn = k_new[(long)b * row + e], vn = v_new[(long)b * row + e];
    T* kd = kc_ + ((long)b * T_ + p) * row + e;
    T* vd = vc_ + ((long)b * T_ + p) * row + e;
    *kd = kn;
    *vd = vn;
    if (i >= 0 && i < Nc) {
      const T* ks = kc_ + ((long)b * T_ + (long)i * s) * row + e;
      const T* vs = vc_ + ((long)b * T_ + (long)i * s) * row + e;
      double ak = 0.0, av = 0.0;
      for (int j = 0; j < l; ++j) {
        const double wj = (double)__ldg(w + j);
        // the last token of the block is the one this thread just wrote
        ak = fma(wj, to_f64(j == l - 1 ? kn : ks[(long)j * row]), ak);
        av = fma(wj, to_f64(j == l - 1 ? vn : vs[(long)j * row]), av);
      }
      k_cmp[((long)b * Nc + i) * row + e] = round_store_f64<T>(ak);
      v_cmp[((long)b * Nc + i) * row + e] = round_store_f64<T>(av);
    }
  }
}

}  // namespace

cudaError_t launch_append(const nsa_params& p, const void* k_new, const void* v_new,
                          const int32_t* pos, void* k_cache, void* v_cache, const float* w,
                          void* k_cmp, void* v_cmp, unsigned* err, cudaStream_t stream) {
  const int Nc = nsa_num_cmp_blocks(p.T, p.cmp_block, p.cmp_stride);
  const long row = (long)p.Hkv * p.d;
  dim3 grid((unsigned)((row + 255) / 256), (unsigned)p.B);
  TraceScope trace("append_kv", stream);
  if (p.dtype == NSA_DTYPE_BF16)
    append_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        (const __nv_bfloat16*)k_new, (const __nv_bfloat16*)v_new, pos, (__nv_bfloat16*)k_cache,
        (__nv_bfloat16*)v_cache, w, (__nv_bfloat16*)k_cmp, (__nv_bfloat16*)v_cmp, err, p.T, p.Hkv,
        p.d, p.cmp_block, p.cmp_stride, Nc);
  else
    append_kernel<float><<<grid, 256, 0, stream>>>(
        (const float*)k_new, (const float*)v_new, pos, (float*)k_cache, (float*)v_cache, w,
        (float*)k_cmp, (float*)v_cmp, err, p.T, p.Hkv, p.d, p.cmp_block, p.cmp_stride, Nc);
  return cudaGetLastError();
}

}  // namespace nsa
