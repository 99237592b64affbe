// Quest-style block selection for the tensor-core prefill (EP94 notes §八: the
// selection ablation compares NSA's compressed-branch scores with a Quest-style
// heuristic block score; the Quest bound is taken for it): for selection block
// j of KV head g and query row t, with kmin / kmax the element-wise minimum and
// maximum of the block's keys up to t,
//     score(t, g, j) = sum over the group's heads h of sum_e max(q_he kmin_e, q_he kmax_e).
// Since max(q kmin, q kmax) = max(q, 0) kmax + min(q, 0) kmin, the sum over the
// heads moves inside: with P_e = sum_h max(q_he, 0) and N_e = sum_h min(q_he, 0),
//     score(t, g, j) = P . kmax_j + N . kmin_j,
// one dot product of length 2d per (token, group, block) against a per-block
// table. Three kernels for the prefill:
//   quest_bounds  kmax, kmin of every full selection block (bf16: the extremes
//                 of bf16 keys are bf16 values), [B, nblk, Hkv, 2, d];
//   quest_scores  per 64-token chunk (one selection block of queries) and KV
//                 head: P and N of its tokens, the dot products with the table
//                 rows of the earlier blocks as an fp32 CUDA-core GEMM tile, and
//                 the chunk's own block from the running extremes of its keys
//                 up to each token; [B, T, Hkv, pitch] fp32;
//   quest_select  a warp per (token, KV head): block 0 and the n - 1 best
//                 others (ties to the lower index), ascending, -1 padded.
// and, for decode, the same table kept beside the KV cache: block_bounds
// builds it from a cache, append_bounds folds in each appended token (the
// decode's scores are in the decode kernels).
#include <cuda_bf16.h>

#include <cstdint>

#include "device_common.cuh"
#include "internal.h"

namespace nsa {
namespace {

constexpr int QD = 128;          // head dimension of the tensor-core prefill
constexpr int QG = 16;           // query heads per KV head
constexpr int QB = 64;           // selection block = tokens per scores chunk
constexpr int QK = 2 * QD;       // dot-product length: [P | N] . [kmax | kmin]
constexpr int QPITCH = QB + 4;   // shared row pitch (floats): 16-byte rows, few bank conflicts
constexpr int QThreads = 256;

__global__ void __launch_bounds__(QD) quest_bounds_kernel(const __nv_bfloat16* __restrict__ k,
                                                          __nv_bfloat16* __restrict__ bounds,
                                                          int T, int Hkv, int nfull) {
  const int j = blockIdx.x, g = blockIdx.y, b = blockIdx.z, e = threadIdx.x;
  if (j >= nfull) return;
  const __nv_bfloat16* src = k + (((size_t)b * T + (size_t)j * QB) * Hkv + g) * QD + e;
  float mx = -INFINITY, mn = INFINITY;
#pragma unroll 8
  for (int u = 0; u < QB; ++u) {
    const float x = __bfloat162float(src[(size_t)u * Hkv * QD]);
    mx = fmaxf(mx, x);
    mn = fminf(mn, x);
  }
  __nv_bfloat16* dst = bounds + (((size_t)b * nfull + j) * Hkv + g) * 2 * QD;
  dst[e] = __float2bfloat16_rn(mx);       // exact: an element of the block
  dst[QD + e] = __float2bfloat16_rn(mn);
}

struct QuestScoreArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* bounds;  // [B, nfull, Hkv, 2, d]
  float* scores;                // [B, T, Hkv, pitch]
  int T, Hq, Hkv, nfull, pitch;
};

// One CTA per (64-token chunk c, KV head, sequence). Its tokens all sit in
// selection block c, so their candidates are blocks 0 .. c.
__global__ void __launch_bounds__(QThreads) quest_scores_kernel(const QuestScoreArgs a) {
  extern __shared__ __align__(16) float qsm[];
  float* pn = qsm;                  // [QK][QPITCH]: P (k < d) and N (k >= d) per token
  float* tb = pn + QK * QPITCH;     // [QK][QPITCH]: kmax / kmin per table row
  __shared__ float red[QB][4];
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = c * QB;
  const int ntok = min(QB, a.T - t0);

  // P and N of each token: sums over the group's heads of the positive and the
  // negative parts of the raw query
  for (int idx = tid; idx < QB * QD; idx += QThreads) {
    const int tok = idx / QD, e = idx % QD;
    float P = 0.f, N = 0.f;
    if (tok < ntok) {
      const __nv_bfloat16* qr = a.q + (((size_t)b * a.T + t0 + tok) * a.Hq + g * QG) * QD + e;
#pragma unroll
      for (int h = 0; h < QG; ++h) {
        const float x = __bfloat162float(qr[h * QD]);
        P += fmaxf(x, 0.f);
        N += fminf(x, 0.f);
      }
    }
    pn[e * QPITCH + tok] = P;
    pn[(QD + e) * QPITCH + tok] = N;
  }
  __syncthreads();

  // earlier blocks 0 .. c-1, 64 table rows at a time: a 4 x 4 register tile of
  // (token, block) dot products per thread
  const int ty = tid >> 4, tx = tid & 15;
  float* srow0 = a.scores + (((size_t)b * a.T + t0) * a.Hkv + g) * a.pitch;
  const size_t tstride = (size_t)a.Hkv * a.pitch;  // between consecutive tokens
  for (int j0 = 0; j0 < c; j0 += QB) {
    const int nj = min(QB, c - j0);
    for (int idx = tid; idx < QB * QK; idx += QThreads) {
      const int jj = idx / QK, kk = idx % QK;
      float x = 0.f;
      if (jj < nj)
        x = __bfloat162float(
            a.bounds[(((size_t)b * a.nfull + j0 + jj) * a.Hkv + g) * QK + kk]);
      tb[kk * QPITCH + jj] = x;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) acc[i][jj] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < QK; ++kk) {
      const float4 av = *reinterpret_cast<const float4*>(pn + kk * QPITCH + ty * 4);
      const float4 bv = *reinterpret_cast<const float4*>(tb + kk * QPITCH + tx * 4);
      const float ar[4] = {av.x, av.y, av.z, av.w};
      const float br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(ar[i], br[jj], acc[i][jj]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tok = ty * 4 + i;
      if (tok >= ntok) continue;
      float* dst = srow0 + tok * tstride + j0 + tx * 4;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        if (tx * 4 + jj < nj) dst[jj] = acc[i][jj];
    }
    __syncthreads();  // tb is refilled next
  }

  // block c itself: for token t0 + i the extremes of keys t0 .. t0 + i. Thread
  // e < d keeps the running extremes of dimension e; each token's sum over e is
  // reduced per warp, then over the four warps.
  if (warp < 4) {
    const int e = tid;
    const __nv_bfloat16* kr = a.k + (((size_t)b * a.T + t0) * a.Hkv + g) * QD + e;
    float mx = -INFINITY, mn = INFINITY;
    for (int i = 0; i < ntok; ++i) {
      const float x = __bfloat162float(kr[(size_t)i * a.Hkv * QD]);
      mx = fmaxf(mx, x);
      mn = fminf(mn, x);
      float v = fmaf(pn[e * QPITCH + i], mx, pn[(QD + e) * QPITCH + i] * mn);
      v = warp_sum(v);
      if (lane == 0) red[i][warp] = v;
    }
  }
  __syncthreads();
  if (tid < ntok) {
    const float v = (red[tid][0] + red[tid][1]) + (red[tid][2] + red[tid][3]);
    srow0[tid * tstride + c] = v;
  }
}

// Order-preserving 32-bit image of a float (-0 taken as +0): larger floats map
// to larger unsigned values.
__device__ __forceinline__ unsigned ordered_bits(float x) {
  const unsigned u = __float_as_uint(x + 0.f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct QuestSelArgs {
  float* scores;        // [B, T, Hkv, pitch]
  int32_t* sel;         // [B, T, Hkv, n]
  int B, T, Hkv, n, pitch;
};

// A warp per (sequence, token, KV head). The candidate key is (ordered score
// bits, ~index): unique, ordered by score and then by the lower index. Each
// lane keeps its best key; per round the warp maximum goes by two redux.sync
// and its owner rescans its share.
__global__ void __launch_bounds__(256) quest_select_kernel(const QuestSelArgs a) {
  const long long wid = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long U = (long long)a.B * a.T * a.Hkv;
  if (wid >= U) return;
  const long long bt = wid / a.Hkv;  // (sequence, token); wid % Hkv is the KV head
  const int t = (int)(bt % a.T);
  const int ncand = t / QB + 1;
  int32_t* dst = a.sel + (size_t)wid * a.n;
  if (ncand <= a.n) {
    for (int i = lane; i < a.n; i += 32) dst[i] = i < ncand ? i : -1;
    return;
  }
  float* sc = a.scores + (size_t)wid * a.pitch;  // workspace: a taken block becomes -inf
  auto rescan = [&](unsigned& bh, unsigned& bl) {
    bh = 0u;
    bl = 0u;
    for (int j = 1 + lane; j < ncand; j += 32) {
      const unsigned kh = ordered_bits(sc[j]), kl = ~(unsigned)j;
      if (kh > bh || (kh == bh && kl > bl)) {
        bh = kh;
        bl = kl;
      }
    }
  };
  unsigned bh, bl;
  rescan(bh, bl);
  int mine = lane == 0 ? 0 : 0x7fffffff;  // lane 0: block 0; lane r: the r-th pick
  for (int r = 1; r < a.n; ++r) {
    const unsigned mh = __reduce_max_sync(0xffffffffu, bh);
    const unsigned ml = __reduce_max_sync(0xffffffffu, bh == mh ? bl : 0u);
    const int pick = (int)~ml;
    if (lane == r) mine = pick;
    if (bh == mh && bl == ml) {
      // the owner drops it (finite scores remain above -inf: n - 1 < ncand - 1)
      sc[pick] = -INFINITY;
      rescan(bh, bl);
    }
  }
  int rank = 0;
  for (int o = 0; o < 32; ++o) rank += (__shfl_sync(0xffffffffu, mine, o) < mine) ? 1 : 0;
  if (lane < a.n) dst[rank] = mine;
}

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

// Keys' block extremes beside a KV cache (decode): block j of sequence b and
// KV head g covers keys [j bs, min(j bs + bs, len_b)); blocks at or past the
// length are left alone. One thread per head-dimension element.
template <typename T>
__global__ void block_bounds_kernel(const T* __restrict__ k, const int32_t* __restrict__ lens,
                                    T* __restrict__ bounds, int T_, int Hkv, int d, int bs,
                                    int nblk, unsigned* err) {
  const int j = blockIdx.x, g = blockIdx.y, b = blockIdx.z, e = threadIdx.x;
  const int L = __ldg(lens + b);
  if (L < 1 || L > T_) {
    if (j == 0 && g == 0 && e == 0) atomicOr(err, kErrSeqLen);
    return;
  }
  const int u0 = j * bs;
  if (u0 >= L) return;
  const int u1 = min(u0 + bs, L);
  const T* src = k + (((size_t)b * T_ + u0) * Hkv + g) * d + e;
  float mx = -INFINITY, mn = INFINITY;
  for (int u = u0; u < u1; ++u) {
    const float x = to_f32(src[(size_t)(u - u0) * Hkv * d]);
    mx = fmaxf(mx, x);
    mn = fminf(mn, x);
  }
  T* dst = bounds + (((size_t)b * nblk + j) * Hkv + g) * 2 * d;
  dst[e] = from_f32<T>(mx);  // exact: an element of the block
  dst[d + e] = from_f32<T>(mn);
}

// One appended token per sequence at pos[b]: its block's extremes take it in
// (the first token of a block starts them).
template <typename T>
__global__ void append_bounds_kernel(const T* __restrict__ k_new, const int32_t* __restrict__ pos,
                                     T* __restrict__ bounds, int T_, int Hkv, int d, int bs,
                                     int nblk, unsigned* err) {
  const int g = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
  const int P = __ldg(pos + b);
  if (P < 0 || P >= T_) {
    if (g == 0 && e == 0) atomicOr(err, kErrAppendPos);
    return;
  }
  const T xv = k_new[((size_t)b * Hkv + g) * d + e];
  T* dst = bounds + (((size_t)b * nblk + P / bs) * Hkv + g) * 2 * d;
  if (P % bs == 0) {
    dst[e] = xv;
    dst[d + e] = xv;
  } else {
    const float x = to_f32(xv);
    if (x > to_f32(dst[e])) dst[e] = xv;
    if (x < to_f32(dst[d + e])) dst[d + e] = xv;
  }
}

}  // namespace

cudaError_t launch_block_bounds(const nsa_params& p, const void* k, const int32_t* seq_lens,
                                void* kbounds, unsigned* err, cudaStream_t stream) {
  const int nblk = (p.T + p.sel_block - 1) / p.sel_block;
  const dim3 grid(nblk, p.Hkv, p.B);
  TraceScope trace("block_bounds", stream);
  if (p.dtype == NSA_DTYPE_BF16)
    block_bounds_kernel<__nv_bfloat16><<<grid, p.d, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), seq_lens, static_cast<__nv_bfloat16*>(kbounds), p.T,
        p.Hkv, p.d, p.sel_block, nblk, err);
  else
    block_bounds_kernel<float><<<grid, p.d, 0, stream>>>(static_cast<const float*>(k), seq_lens,
                                                        static_cast<float*>(kbounds), p.T, p.Hkv,
                                                        p.d, p.sel_block, nblk, err);
  return cudaGetLastError();
}

cudaError_t launch_append_bounds(const nsa_params& p, const void* k_new, const int32_t* pos,
                                 void* kbounds, unsigned* err, cudaStream_t stream) {
  const int nblk = (p.T + p.sel_block - 1) / p.sel_block;
  const dim3 grid(p.Hkv, p.B);
  TraceScope trace("append_bounds", stream);
  if (p.dtype == NSA_DTYPE_BF16)
    append_bounds_kernel<__nv_bfloat16><<<grid, p.d, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k_new), pos, static_cast<__nv_bfloat16*>(kbounds), p.T,
        p.Hkv, p.d, p.sel_block, nblk, err);
  else
    append_bounds_kernel<float><<<grid, p.d, 0, stream>>>(static_cast<const float*>(k_new), pos,
                                                         static_cast<float*>(kbounds), p.T, p.Hkv,
                                                         p.d, p.sel_block, nblk, err);
  return cudaGetLastError();
}


bool quest_tc_supported(const nsa_params& p) {
  const int nblk = (p.T + QB - 1) / QB;
  return p.d == QD && p.Hq == QG * p.Hkv && p.sel_block == QB && p.top_n <= 32 && nblk <= 4096;
}

size_t quest_ws_bytes(const nsa_params& p) {
  const int nblk = (p.T + QB - 1) / QB;
  const int nfull = p.T / QB;
  const int pitch = (nblk + 3) & ~3;
  return al256((size_t)p.B * nfull * p.Hkv * QK * 2) + al256((size_t)p.B * p.T * p.Hkv * pitch * 4);
}

cudaError_t launch_quest_select(const nsa_params& p, const void* q, const void* k, int32_t* sel,
                                void* ws, cudaStream_t stream) {
  const int nblk = (p.T + QB - 1) / QB;
  const int nfull = p.T / QB;
  const int pitch = (nblk + 3) & ~3;
  unsigned char* w = static_cast<unsigned char*>(ws);
  __nv_bfloat16* bounds = reinterpret_cast<__nv_bfloat16*>(w);
  w += al256((size_t)p.B * nfull * p.Hkv * QK * 2);
  float* scores = reinterpret_cast<float*>(w);
  cudaError_t e;
  if (nfull > 0) {
    TraceScope trace("quest_bounds", stream);
    quest_bounds_kernel<<<dim3(nfull, p.Hkv, p.B), QD, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), bounds, p.T, p.Hkv, nfull);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    QuestScoreArgs a{static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                     bounds, scores, p.T, p.Hq, p.Hkv, nfull, pitch};
    const int smem = 2 * QK * QPITCH * 4;
    if ((e = ensure_dyn_smem((const void*)quest_scores_kernel, smem)) != cudaSuccess) return e;
    TraceScope trace("quest_scores", stream);
    quest_scores_kernel<<<dim3(nblk, p.Hkv, p.B), QThreads, smem, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    QuestSelArgs a{scores, sel, p.B, p.T, p.Hkv, p.top_n, pitch};
    const long long U = (long long)p.B * p.T * p.Hkv;
    TraceScope trace("quest_select", stream);
    quest_select_kernel<<<(unsigned)((U + 7) / 8), 256, 0, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace nsa
