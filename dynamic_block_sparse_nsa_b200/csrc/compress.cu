// Token compression (EP94 notes §五 branch one; lchairun.cn NSA article,
// compression paragraph): each compressed block i of the keys (and, with the
// same weights, of the values) is the weighted sum of l consecutive tokens
// starting at i*s:
//     k_cmp[b,i,g,:] = sum_{j<l} w[j] * k[b, i*s + j, g, :]
//
// Bandwidth-bound: each token is read about l/s times, mostly from L2. The
// sum runs in fp64 (each product of a bf16/fp32 input and an fp32 weight is
// exact in fp64) and is rounded once to the storage type, so the stored
// block is the correctly rounded exact sum.
#include "device_common.cuh"
#include "internal.h"

namespace nsa {

template <typename T, int VEC>
__global__ void __launch_bounds__(256) compress_kernel(const T* __restrict__ k,
                                                       const T* __restrict__ v,
                                                       const float* __restrict__ w,
                                                       T* __restrict__ kc, T* __restrict__ vc,
                                                       int B, int T_, int Hkv, int d, int l,
                                                       int s, int Nc) {
  const long row = (long)Hkv * d;          // elements per token
  const long per_seq_out = (long)Nc * row;
  const long total = (long)B * per_seq_out / VEC;
  for (long idx = blockIdx.x * (long)blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const long o = idx * VEC;                // flat output index
    const int b = (int)(o / per_seq_out);
    const long r = o - (long)b * per_seq_out;
    const int i = (int)(r / row);
    const long ge = r - (long)i * row;       // g * d + e
    const T* ks = k + ((long)b * T_ + (long)i * s) * row + ge;
    const T* vs = v + ((long)b * T_ + (long)i * s) * row + ge;
    double ak[VEC], av[VEC];
#pragma unroll
    for (int u = 0; u < VEC; ++u) ak[u] = av[u] = 0.0;
    for (int j = 0; j < l; ++j) {
      const double wj = (double)__ldg(w + j);
#pragma unroll
      for (int u = 0; u < VEC; ++u) {
        ak[u] = fma(wj, to_f64(ks[(long)j * row + u]), ak[u]);
        av[u] = fma(wj, to_f64(vs[(long)j * row + u]), av[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
      kc[o + u] = round_store_f64<T>(ak[u]);
      vc[o + u] = round_store_f64<T>(av[u]);
    }
  }
}

cudaError_t launch_compress(const nsa_params& p, const void* k, const void* v, const float* w,
                            void* kc, void* vc, cudaStream_t stream) {
  const int Nc = nsa_num_cmp_blocks(p.T, p.cmp_block, p.cmp_stride);
  if (Nc == 0 || p.B == 0) return cudaSuccess;
  const long total = (long)p.B * Nc * p.Hkv * p.d;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  constexpr int kThreads = 256;
  TraceScope trace("compress_kv", stream);
  if (p.dtype == NSA_DTYPE_BF16) {
    constexpr int VEC = 2;
    long blocks = (total / VEC + kThreads - 1) / kThreads;
    if (blocks > (long)sms * 16) blocks = (long)sms * 16;
    compress_kernel<__nv_bfloat16, VEC><<<(unsigned)blocks, kThreads, 0, stream>>>(
        (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, w, (__nv_bfloat16*)kc,
        (__nv_bfloat16*)vc, p.B, p.T, p.Hkv, p.d, p.cmp_block, p.cmp_stride, Nc);
  } else {
    long blocks = (total + kThreads - 1) / kThreads;
    if (blocks > (long)sms * 16) blocks = (long)sms * 16;
    compress_kernel<float, 1><<<(unsigned)blocks, kThreads, 0, stream>>>(
        (const float*)k, (const float*)v, w, (float*)kc, (float*)vc, p.B, p.T, p.Hkv, p.d,
        p.cmp_block, p.cmp_stride, Nc);
  }
  return cudaGetLastError();
}

}  // namespace nsa
