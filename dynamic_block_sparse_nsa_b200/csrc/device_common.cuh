// Device helpers shared by the kernels: element loads/stores, the fp64 ->
// storage rounding of compressed blocks, and warp reductions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace nsa {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ double to_f64(float x) { return (double)x; }
__device__ __forceinline__ double to_f64(__nv_bfloat16 x) { return (double)__bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Round an fp64 value once to the storage type, to nearest with ties to even.
// For bf16 this is done directly from fp64 (not through fp32, which would round
// twice): x is scaled so that the bf16 quantum of its binade becomes 1, rounded
// to an integer with rint (ties-to-even), and scaled back. The result has at
// most 8 significant bits, so the final conversion through fp32 is exact.
template <typename T> __device__ __forceinline__ T round_store_f64(double x);
template <> __device__ __forceinline__ float round_store_f64<float>(double x) {
  return __double2float_rn(x);
}
template <> __device__ __forceinline__ __nv_bfloat16 round_store_f64<__nv_bfloat16>(double x) {
  if (x == 0.0 || !isfinite(x)) return __float2bfloat16_rn((float)x);
  int e;
  frexp(x, &e);                 // |x| = f * 2^e, 0.5 <= f < 1
  int q = e - 8;                // quantum of 8-significant-bit values here
  if (q < -133) q = -133;       // bf16 subnormal quantum
  double r = ldexp(rint(ldexp(x, -q)), q);
  // Largest finite bf16 is (2 - 2^-7) * 2^127; anything rounded beyond is inf.
  if (fabs(r) > 3.3895313892515355e38) r = copysign(__longlong_as_double(0x7ff0000000000000LL), x);
  return __float2bfloat16_rn((float)r);   // exact: r is a bf16 value
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Top-selection order: a higher score wins; equal scores go to the lower index.
__device__ __forceinline__ bool sel_better(float sa, int ja, float sb, int jb) {
  return sa > sb || (sa == sb && ja < jb);
}

}  // namespace nsa
