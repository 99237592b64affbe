// Generic CUDA-core path: one CTA per (query row, KV head) computes the whole
// NSA forward of the G query heads of that GQA group, and one CTA per (query
// row, head) the MoBA forward. Any head dim, group size and dtype the ABI
// accepts runs here; the tensor-core kernels cover the large bf16 shapes.
//
// NSA row (EP94 notes §五, §六; lchairun.cn NSA article):
//   1. compressed branch, pass 1: log-sum-exp of the scaled logits over the
//      visible compressed blocks (block i visible when i*s + l - 1 <= t);
//   2. pass 2: normalised probabilities p, o_cmp = p V~, and the block score of
//      each selection block j = sum over the group's heads of the p mass on the
//      compressed blocks that overlap j;
//   3. top-n: block 0 kept, the n-1 best others (ties to the lower index);
//      with sel_mode 1 the scores are the Quest-style block bound instead;
//   4. selected branch: softmax over the tokens of the chosen blocks up to t;
//   5. window branch: softmax over [max(0, t-w+1), t];
//   6. gates g = sigmoid(q . Wg) (or fixed), out = g0 o_cmp + g1 o_slc + g2 o_win.
// Keys are staged through shared memory in chunks of kCH rows; every K/V row is
// loaded once per CTA and used by all G heads (the group-shared read of §六).
#include <climits>

#include "device_common.cuh"
#include "internal.h"

namespace nsa {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kCH = 64;

struct Ctx {
  int G, d;
  float scale;
  float* qs;      // [G][d]
  float* oacc;    // [G][d]
  float* outacc;  // [G][d]
  float* Ks;      // [kCH][d + 1]
  float* Vs;      // [kCH][d]
  float* z;       // [G][kCH]
  float* ptot;    // [kCH]
  float* mh;      // [G]   running max, then lse
  float* sh;      // [G]   running sum
  float* fac;     // [G]   rescale factor of the last chunk
  float* gate;    // [G][3]
  float* scores;  // [nblk]
  float* red_s;   // [kWarps]
  int* red_j;     // [kWarps]
  int* sel;       // [n]
  int* misc;      // [4]
};

// Shared-memory size in floats/ints for a group of G heads of dim d.
__host__ __device__ inline size_t ctx_bytes(int G, int d, int nblk, int nsel) {
  size_t f = 3 * (size_t)G * d + (size_t)kCH * (d + 1) + (size_t)kCH * d + (size_t)G * kCH + kCH +
             6 * (size_t)G + nblk + kWarps;
  size_t i = kWarps + nsel + 4;
  return (f + i) * 4;
}

__device__ inline Ctx carve(float* sm, int G, int d, int nblk, float scale) {
  Ctx c;
  c.G = G;
  c.d = d;
  c.scale = scale;
  float* p = sm;
  c.qs = p; p += G * d;
  c.oacc = p; p += G * d;
  c.outacc = p; p += G * d;
  c.Ks = p; p += kCH * (d + 1);
  c.Vs = p; p += kCH * d;
  c.z = p; p += G * kCH;
  c.ptot = p; p += kCH;
  c.mh = p; p += G;
  c.sh = p; p += G;
  c.fac = p; p += G;
  c.gate = p; p += 3 * G;
  c.scores = p; p += nblk;
  c.red_s = p; p += kWarps;
  int* ip = reinterpret_cast<int*>(p);
  c.red_j = ip; ip += kWarps;
  c.misc = ip; ip += 4;
  c.sel = ip;
  return c;
}

// Copy rows r0 .. r0+nk-1 (row stride `stride` elements) into dst (pitch floats).
template <typename T>
__device__ inline void stage_rows(float* dst, int pitch, const T* base, long stride, int r0,
                                  int nk, int d) {
  for (int x = threadIdx.x; x < nk * d; x += kThreads) {
    const int c = x / d, e = x - c * d;
    dst[c * pitch + e] = to_f32(base[(long)(r0 + c) * stride + e]);
  }
}

// z[h][c] = scale * q_h . K_c for the nk staged keys.
__device__ inline void logits(const Ctx& c, int nk) {
  for (int x = threadIdx.x; x < c.G * kCH; x += kThreads) {
    const int h = x / kCH, col = x - h * kCH;
    if (col < nk) {
      const float* kr = c.Ks + col * (c.d + 1);
      const float* qh = c.qs + h * c.d;
      float acc = 0.f;
      for (int e = 0; e < c.d; ++e) acc = fmaf(qh[e], kr[e], acc);
      c.z[h * kCH + col] = acc * c.scale;
    }
  }
}

// Online-softmax step for each head: z -> exp(z - m_new), running max/sum
// updated, fac[h] = exp(m_old - m_new).
__device__ inline void online_step(const Ctx& c, int nk) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int h = warp; h < c.G; h += kWarps) {
    float* zh = c.z + h * kCH;
    float cm = -INFINITY;
    for (int col = lane; col < nk; col += 32) cm = fmaxf(cm, zh[col]);
    cm = warp_max(cm);
    const float mold = c.mh[h];
    const float mnew = fmaxf(mold, cm);
    const float f = expf(mold - mnew);
    float ps = 0.f;
    for (int col = lane; col < nk; col += 32) {
      const float pv = expf(zh[col] - mnew);
      zh[col] = pv;
      ps += pv;
    }
    ps = warp_sum(ps);
    __syncwarp();
    if (lane == 0) {
      c.mh[h] = mnew;
      c.sh[h] = c.sh[h] * f + ps;
      c.fac[h] = f;
    }
  }
}

// oacc[h][e] (* fac[h] if rescale) += sum_c z[h][c] * V[c][e].
__device__ inline void accumulate_pv(const Ctx& c, int nk, bool rescale) {
  for (int x = threadIdx.x; x < c.G * c.d; x += kThreads) {
    const int h = x / c.d, e = x - h * c.d;
    float acc = rescale ? c.oacc[x] * c.fac[h] : c.oacc[x];
    const float* ph = c.z + h * kCH;
    for (int col = 0; col < nk; ++col) acc = fmaf(ph[col], c.Vs[col * c.d + e], acc);
    c.oacc[x] = acc;
  }
}

// Online softmax attention of all G heads over the key range [r0, r1] of
// (kbase, vbase); accumulates into oacc / mh / sh (caller initialises them).
template <typename T>
__device__ inline void attend_range(const Ctx& c, const T* kbase, const T* vbase, long stride,
                                    int r0, int r1) {
  for (int c0 = r0; c0 <= r1; c0 += kCH) {
    const int nk = min(kCH, r1 - c0 + 1);
    stage_rows(c.Ks, c.d + 1, kbase, stride, c0, nk, c.d);
    stage_rows(c.Vs, c.d, vbase, stride, c0, nk, c.d);
    __syncthreads();
    logits(c, nk);
    __syncthreads();
    online_step(c, nk);
    __syncthreads();
    accumulate_pv(c, nk, true);
    __syncthreads();
  }
}

__device__ inline void reset_branch(const Ctx& c) {
  for (int x = threadIdx.x; x < c.G * c.d; x += kThreads) c.oacc[x] = 0.f;
  for (int h = threadIdx.x; h < c.G; h += kThreads) {
    c.mh[h] = -INFINITY;
    c.sh[h] = 0.f;
  }
}

// outacc += gate[:, which] * oacc / sh (a branch with no keys adds nothing).
__device__ inline void add_branch(const Ctx& c, int which, bool normalise) {
  for (int x = threadIdx.x; x < c.G * c.d; x += kThreads) {
    const int h = x / c.d;
    const float s = normalise ? c.sh[h] : 1.f;
    if (s > 0.f) c.outacc[x] = fmaf(c.gate[h * 3 + which], c.oacc[x] / s, c.outacc[x]);
  }
}

// Top selection over scores[lo, ncand): keeps `forced` (>= 0) plus the best
// `want` others by (score desc, index asc); writes sel[0..) ascending and
// returns the count. Taken entries of scores are overwritten with -inf and
// -inf entries are never picked.
__device__ inline int select_top(const Ctx& c, int lo, int ncand, int forced, int want) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int ns = 0;
  if (forced >= 0) {
    if (threadIdx.x == 0) c.sel[0] = forced;
    ns = 1;
  }
  for (int r = 0; r < want; ++r) {
    float bs = -INFINITY;
    int bj = INT_MAX;
    for (int j = lo + threadIdx.x; j < ncand; j += kThreads) {
      const float sj = c.scores[j];
      if (sj != -INFINITY && sel_better(sj, j, bs, bj)) {
        bs = sj;
        bj = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (sel_better(os, oj, bs, bj)) {
        bs = os;
        bj = oj;
      }
    }
    if (lane == 0) {
      c.red_s[warp] = bs;
      c.red_j[warp] = bj;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float s0 = c.red_s[0];
      int j0 = c.red_j[0];
      for (int w = 1; w < kWarps; ++w)
        if (sel_better(c.red_s[w], c.red_j[w], s0, j0)) {
          s0 = c.red_s[w];
          j0 = c.red_j[w];
        }
      c.sel[ns + r] = j0;
      c.scores[j0] = -INFINITY;
    }
    __syncthreads();
  }
  ns += want;
  if (threadIdx.x == 0) {
    for (int a = 1; a < ns; ++a) {  // insertion sort, ascending
      const int x = c.sel[a];
      int p = a - 1;
      while (p >= 0 && c.sel[p] > x) {
        c.sel[p + 1] = c.sel[p];
        --p;
      }
      c.sel[p + 1] = x;
    }
  }
  __syncthreads();
  return ns;
}

// Adaptive selection over scores[0, ncand) (lchairun NSA article, adaptive
// sparsification): block 0, then the best others by (score desc, index asc)
// until the chosen scores reach top_p times the sum over all candidates, at
// most n blocks. Sums in fp64. Writes sel[0..) ascending; returns the count.
__device__ inline int select_top_p(const Ctx& c, int ncand, int n, float top_p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ double tot_s, cum_s;
  __shared__ int stop_s;
  double part = 0.0;
  for (int j = threadIdx.x; j < ncand; j += kThreads) part += (double)c.scores[j];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  __shared__ double wpart[kWarps];
  if (lane == 0) wpart[warp] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kWarps; ++w) t += wpart[w];
    tot_s = t;
    cum_s = (double)c.scores[0];
    c.sel[0] = 0;
    c.scores[0] = -INFINITY;
    stop_s = (1 >= n || 1 >= ncand || cum_s >= (double)top_p * t) ? 1 : 0;
  }
  __syncthreads();
  int ns = 1;
  while (!stop_s) {
    float bs = -INFINITY;
    int bj = INT_MAX;
    for (int j = 1 + threadIdx.x; j < ncand; j += kThreads) {
      const float sj = c.scores[j];
      if (sj != -INFINITY && sel_better(sj, j, bs, bj)) {
        bs = sj;
        bj = j;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      if (sel_better(os, oj, bs, bj)) {
        bs = os;
        bj = oj;
      }
    }
    if (lane == 0) {
      c.red_s[warp] = bs;
      c.red_j[warp] = bj;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float s0 = c.red_s[0];
      int j0 = c.red_j[0];
      for (int w = 1; w < kWarps; ++w)
        if (sel_better(c.red_s[w], c.red_j[w], s0, j0)) {
          s0 = c.red_s[w];
          j0 = c.red_j[w];
        }
      c.sel[ns] = j0;
      cum_s += (double)s0;
      c.scores[j0] = -INFINITY;
      stop_s = (ns + 1 >= n || ns + 1 >= ncand || cum_s >= (double)top_p * tot_s) ? 1 : 0;
    }
    __syncthreads();
    ++ns;
  }
  if (threadIdx.x == 0) {
    for (int x = 1; x < ns; ++x) {  // insertion sort, ascending
      const int v = c.sel[x];
      int q = x - 1;
      while (q >= 0 && c.sel[q] > v) {
        c.sel[q + 1] = c.sel[q];
        --q;
      }
      c.sel[q + 1] = v;
    }
  }
  __syncthreads();
  return ns;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) nsa_rows_kernel(NsaRowArgs a) {
  extern __shared__ float sm[];
  const int G = a.Hq / a.Hkv, d = a.d;
  const int g = blockIdx.y, b = blockIdx.z;
  const long tok = (long)a.Hkv * d;
  const int nblk = (a.T + a.bs - 1) / a.bs;
  Ctx c = carve(sm, G, d, nblk, a.scale);

  int t;
  const T* qrow;
  T* orow;
  int32_t* selrow = nullptr;
  if (a.decode) {
    const int len = a.seq_lens[b];
    qrow = (const T*)a.q + ((long)b * a.Hq + (long)g * G) * d;
    orow = (T*)a.out + ((long)b * a.Hq + (long)g * G) * d;
    if (a.sel_idx) selrow = a.sel_idx + ((long)b * a.Hkv + g) * a.n;
    if (len < 1 || len > a.T) {
      for (int x = threadIdx.x; x < G * d; x += kThreads) orow[x] = from_f32<T>(0.f);
      if (selrow)
        for (int x = threadIdx.x; x < a.n; x += kThreads) selrow[x] = -1;
      if (threadIdx.x == 0) atomicOr(a.err, kErrSeqLen);
      return;
    }
    t = len - 1;
  } else {
    t = blockIdx.x;
    qrow = (const T*)a.q + (((long)b * a.T + t) * a.Hq + (long)g * G) * d;
    orow = (T*)a.out + (((long)b * a.T + t) * a.Hq + (long)g * G) * d;
    if (a.sel_idx) selrow = a.sel_idx + (((long)b * a.T + t) * a.Hkv + g) * a.n;
  }
  const T* kb = (const T*)a.k + (long)b * a.T * tok + (long)g * d;
  const T* vb = (const T*)a.v + (long)b * a.T * tok + (long)g * d;
  const T* kcb = (const T*)a.kc + (long)b * a.Nc * tok + (long)g * d;
  const T* vcb = (const T*)a.vc + (long)b * a.Nc * tok + (long)g * d;

  for (int x = threadIdx.x; x < G * d; x += kThreads) {
    c.qs[x] = to_f32(qrow[x]);
    c.outacc[x] = 0.f;
  }
  __syncthreads();
  // Gates (EP94 notes §五 gating): per head and branch, from the raw query.
  for (int x = threadIdx.x; x < G * 3; x += kThreads) {
    const int h = x / 3, br = x - h * 3;
    float gv;
    if (a.gate_mode == 1) {
      gv = a.fixed_gates[br];
    } else {
      float dot = 0.f;
      for (int e = 0; e < d; ++e) dot = fmaf(c.qs[h * d + e], a.w_gate[e * 3 + br], dot);
      gv = 1.f / (1.f + expf(-dot));
    }
    c.gate[x] = gv;
  }

  // ---- compressed branch and block scores ----
  int nvis = 0;
  if (t + 1 >= a.l) nvis = min(a.Nc, (t + 1 - a.l) / a.s + 1);
  const int ncand = t / a.bs + 1;
  for (int j = threadIdx.x; j < ncand; j += kThreads) c.scores[j] = 0.f;
  reset_branch(c);
  __syncthreads();
  if (nvis > 0) {
    // pass 1: lse per head
    for (int c0 = 0; c0 < nvis; c0 += kCH) {
      const int nk = min(kCH, nvis - c0);
      stage_rows(c.Ks, d + 1, kcb, tok, c0, nk, d);
      __syncthreads();
      logits(c, nk);
      __syncthreads();
      online_step(c, nk);
      __syncthreads();
    }
    for (int h = threadIdx.x; h < G; h += kThreads) c.mh[h] = c.mh[h] + logf(c.sh[h]);
    __syncthreads();
    // pass 2: normalised p, o_cmp and block scores
    for (int c0 = 0; c0 < nvis; c0 += kCH) {
      const int nk = min(kCH, nvis - c0);
      stage_rows(c.Ks, d + 1, kcb, tok, c0, nk, d);
      stage_rows(c.Vs, d, vcb, tok, c0, nk, d);
      __syncthreads();
      logits(c, nk);
      __syncthreads();
      for (int x = threadIdx.x; x < G * kCH; x += kThreads) {
        const int h = x / kCH, col = x - h * kCH;
        if (col < nk) c.z[x] = expf(c.z[x] - c.mh[h]);
      }
      __syncthreads();
      accumulate_pv(c, nk, false);
      for (int col = threadIdx.x; col < nk; col += kThreads) {
        float s = 0.f;
        for (int h = 0; h < G; ++h) s += c.z[h * kCH + col];
        c.ptot[col] = s;
      }
      __syncthreads();
      // Selection block j collects the compressed blocks i with
      // [i*s, i*s + l - 1] intersecting [j*bs, j*bs + bs - 1].
      const int jlo = (c0 * a.s) / a.bs;
      const int jhi = min(ncand - 1, ((c0 + nk - 1) * a.s + a.l - 1) / a.bs);
      for (int j = jlo + threadIdx.x; j <= jhi; j += kThreads) {
        const int num = j * a.bs - a.l + 1;
        int ilo = num <= 0 ? 0 : (num + a.s - 1) / a.s;
        int ihi = (j * a.bs + a.bs - 1) / a.s;
        ilo = max(ilo, c0);
        ihi = min(ihi, c0 + nk - 1);
        float s = 0.f;
        for (int i = ilo; i <= ihi; ++i) s += c.ptot[i - c0];
        c.scores[j] += s;
      }
      __syncthreads();
    }
    add_branch(c, 0, false);
  }
  __syncthreads();

  // ---- Quest-style block bound (sel_mode 1; EP94 notes §八, the selection
  // ablation): per block j the element-wise min / max of its keys up to t and
  // the sum over the group's heads of sum_e max(q_e kmin_e, q_e kmax_e); it
  // replaces the compressed-branch scores as the selection's ranking. ----
  if (a.sel_mode == 1) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int j = warp; j < ncand; j += kWarps) {
      const int u1 = min(j * a.bs + a.bs - 1, t);
      float acc = 0.f;
      for (int e = lane; e < d; e += 32) {
        float mn = INFINITY, mx = -INFINITY;
        for (int u = j * a.bs; u <= u1; ++u) {
          const float x = to_f32(kb[(long)u * tok + e]);
          mn = fminf(mn, x);
          mx = fmaxf(mx, x);
        }
        for (int h = 0; h < G; ++h) {
          const float qe = c.qs[h * d + e];
          acc += fmaxf(qe * mn, qe * mx);
        }
      }
      acc = warp_sum(acc);
      if (lane == 0) c.scores[j] = acc;
    }
    __syncthreads();
  }

  // ---- top-n selection (block 0 forced) ----
  int ns;
  if (a.top_p > 0.f) {
    ns = select_top_p(c, ncand, a.n, a.top_p);
  } else if (ncand <= a.n) {
    for (int j = threadIdx.x; j < ncand; j += kThreads) c.sel[j] = j;
    __syncthreads();
    ns = ncand;
  } else {
    if (threadIdx.x == 0) c.scores[0] = -INFINITY;
    __syncthreads();
    ns = select_top(c, 1, ncand, 0, a.n - 1);
  }
  if (selrow)
    for (int x = threadIdx.x; x < a.n; x += kThreads) selrow[x] = x < ns ? c.sel[x] : -1;

  // ---- selected branch ----
  reset_branch(c);
  __syncthreads();
  for (int q = 0; q < ns; ++q) {
    const int j = c.sel[q];
    attend_range(c, kb, vb, tok, j * a.bs, min(j * a.bs + a.bs - 1, t));
  }
  add_branch(c, 1, true);
  __syncthreads();

  // ---- sliding window ----
  reset_branch(c);
  __syncthreads();
  attend_range(c, kb, vb, tok, max(0, t - a.w + 1), t);
  add_branch(c, 2, true);
  __syncthreads();

  for (int x = threadIdx.x; x < G * d; x += kThreads) orow[x] = from_f32<T>(c.outacc[x]);
}

// ---------------------------------------------------------------------------
// MoBA (EP94 notes §九/§十; LateTalk ep.103)
// ---------------------------------------------------------------------------

// kbar[b, j, g, :] = mean of the m keys of block j, accumulated in fp64.
template <typename T>
__global__ void __launch_bounds__(256) moba_block_mean_kernel(const T* __restrict__ k,
                                                              float* __restrict__ kbar, int B,
                                                              int T_, int Hkv, int d, int m) {
  const int nfull = T_ / m;
  const long row = (long)Hkv * d;
  const long total = (long)B * nfull * row;
  for (long o = blockIdx.x * (long)blockDim.x + threadIdx.x; o < total;
       o += (long)gridDim.x * blockDim.x) {
    const int b = (int)(o / ((long)nfull * row));
    const long r = o - (long)b * nfull * row;
    const int j = (int)(r / row);
    const long ge = r - (long)j * row;
    const T* src = k + ((long)b * T_ + (long)j * m) * row + ge;
    double acc = 0.0;
    for (int u = 0; u < m; ++u) acc += to_f64(src[(long)u * row]);
    kbar[o] = (float)(acc / m);
  }
}

// The same for bf16 keys with d a multiple of 8: each thread sums 8 adjacent
// dimensions (16-byte loads, eight fp64 accumulators, eight rows' loads in
// flight), so the kernel streams the keys at HBM rate.
__global__ void __launch_bounds__(256) moba_block_mean8_kernel(const __nv_bfloat16* __restrict__ k,
                                                               float* __restrict__ kbar, int B,
                                                               int T_, int Hkv, int d, int m) {
  const int nfull = T_ / m;
  const long row = (long)Hkv * d;
  const long total8 = (long)B * nfull * row / 8;
  for (long o8 = blockIdx.x * (long)blockDim.x + threadIdx.x; o8 < total8;
       o8 += (long)gridDim.x * blockDim.x) {
    const long o = o8 * 8;
    const int b = (int)(o / ((long)nfull * row));
    const long r = o - (long)b * nfull * row;
    const int j = (int)(r / row);
    const long ge = r - (long)j * row;
    const __nv_bfloat16* src = k + ((long)b * T_ + (long)j * m) * row + ge;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 8
    for (int u = 0; u < m; ++u) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (long)u * row));
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        acc[2 * e] += (double)f.x;
        acc[2 * e + 1] += (double)f.y;
      }
    }
    float4 lo, hi;
    lo.x = (float)(acc[0] / m);
    lo.y = (float)(acc[1] / m);
    lo.z = (float)(acc[2] / m);
    lo.w = (float)(acc[3] / m);
    hi.x = (float)(acc[4] / m);
    hi.y = (float)(acc[5] / m);
    hi.z = (float)(acc[6] / m);
    hi.w = (float)(acc[7] / m);
    reinterpret_cast<float4*>(kbar + o)[0] = lo;
    reinterpret_cast<float4*>(kbar + o)[1] = hi;
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads) moba_rows_kernel(MobaArgs a) {
  extern __shared__ float sm[];
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = a.Hq / a.Hkv, g = h / G, d = a.d, m = a.m;
  const long tok = (long)a.Hkv * d;
  const int nblk = (a.T + m - 1) / m, nfull = a.T / m;
  Ctx c = carve(sm, 1, d, nblk, a.scale);
  const T* qrow = (const T*)a.q + (((long)b * a.T + t) * a.Hq + h) * d;
  T* orow = (T*)a.out + (((long)b * a.T + t) * a.Hq + h) * d;
  for (int e = threadIdx.x; e < d; e += kThreads) c.qs[e] = to_f32(qrow[e]);
  __syncthreads();
  const int own = t / m;
  // Gate scores of the earlier blocks: q . mean(K_block).
  const float* kbb = a.kbar + (long)b * nfull * tok + (long)g * d;
  for (int j = threadIdx.x; j < own; j += kThreads) {
    const float* kr = kbb + (long)j * tok;
    float acc = 0.f;
    for (int e = 0; e < d; ++e) acc = fmaf(c.qs[e], kr[e], acc);
    c.scores[j] = acc;
  }
  __syncthreads();
  int ns;
  if (own <= a.topk - 1) {
    for (int j = threadIdx.x; j <= own; j += kThreads) c.sel[j] = j;
    __syncthreads();
    ns = own + 1;
  } else {
    ns = select_top(c, 0, own, own, a.topk - 1);
  }
  if (a.sel_idx) {
    int32_t* srow = a.sel_idx + (((long)b * a.T + t) * a.Hq + h) * a.topk;
    for (int x = threadIdx.x; x < a.topk; x += kThreads) srow[x] = x < ns ? c.sel[x] : -1;
  }
  reset_branch(c);
  __syncthreads();
  const T* kb = (const T*)a.k + (long)b * a.T * tok + (long)g * d;
  const T* vb = (const T*)a.v + (long)b * a.T * tok + (long)g * d;
  for (int q = 0; q < ns; ++q) {
    const int j = c.sel[q];
    attend_range(c, kb, vb, tok, j * m, min(j * m + m - 1, t));
  }
  for (int e = threadIdx.x; e < d; e += kThreads) orow[e] = from_f32<T>(c.oacc[e] / c.sh[0]);
}

int device_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

size_t nsa_rows_simt_smem(const NsaRowArgs& a) {
  const int G = a.Hq / a.Hkv;
  const int nblk = (a.T + a.bs - 1) / a.bs;
  return ctx_bytes(G, a.d, nblk, a.n);
}

cudaError_t launch_nsa_rows_simt(const NsaRowArgs& a, cudaStream_t stream) {
  const size_t smem = nsa_rows_simt_smem(a);
  dim3 grid(a.decode ? 1 : a.T, a.Hkv, a.B);
  TraceScope trace("nsa_rows_simt", stream);
  if (a.dtype == NSA_DTYPE_BF16) {
    auto kern = nsa_rows_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kThreads, smem, stream>>>(a);
  } else {
    auto kern = nsa_rows_kernel<float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kThreads, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

size_t moba_simt_smem(const MobaArgs& a) {
  const int nblk = (a.T + a.m - 1) / a.m;
  return ctx_bytes(1, a.d, nblk, a.topk);
}

cudaError_t launch_moba_block_mean(const MobaArgs& a, cudaStream_t stream) {
  const int nfull = a.T / a.m;
  const long total = (long)a.B * nfull * a.Hkv * a.d;
  if (total > 0) {
    long blocks = (total + 255) / 256;
    const long cap = (long)device_sms() * 16;
    if (blocks > cap) blocks = cap;
    TraceScope trace("moba_block_mean", stream);
    const bool vec = a.dtype == NSA_DTYPE_BF16 && a.d % 8 == 0 &&
                     reinterpret_cast<uintptr_t>(a.k) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(a.kbar) % 16 == 0;
    if (vec) {
      const long b8 = (total / 8 + 255) / 256;
      moba_block_mean8_kernel<<<(unsigned)(b8 < cap ? b8 : cap), 256, 0, stream>>>(
          (const __nv_bfloat16*)a.k, a.kbar, a.B, a.T, a.Hkv, a.d, a.m);
    } else if (a.dtype == NSA_DTYPE_BF16)
      moba_block_mean_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, stream>>>(
          (const __nv_bfloat16*)a.k, a.kbar, a.B, a.T, a.Hkv, a.d, a.m);
    else
      moba_block_mean_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(
          (const float*)a.k, a.kbar, a.B, a.T, a.Hkv, a.d, a.m);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_moba_simt(const MobaArgs& a, cudaStream_t stream) {
  cudaError_t e = launch_moba_block_mean(a, stream);
  if (e != cudaSuccess) return e;
  const size_t smem = moba_simt_smem(a);
  dim3 grid(a.T, a.Hq, a.B);
  TraceScope trace("moba_rows_simt", stream);
  if (a.dtype == NSA_DTYPE_BF16) {
    auto kern = moba_rows_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kThreads, smem, stream>>>(a);
  } else {
    auto kern = moba_rows_kernel<float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kThreads, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

// Failure-path hook: poll *flag at most max_iters times; on giving up, set the
// timeout bit of the error word and return (no trap, no endless loop).
__global__ void bounded_wait_kernel(const volatile int32_t* flag, int max_iters, unsigned* err) {
  if (threadIdx.x != 0) return;
  for (int i = 0; i < max_iters; ++i) {
    if (*flag != 0) return;
    __nanosleep(1000);
  }
  atomicOr(err, kErrTimeout);
}

cudaError_t launch_bounded_wait(const int32_t* flag, int max_iters, unsigned* err,
                                cudaStream_t stream) {
  TraceScope trace("bounded_wait", stream);
  bounded_wait_kernel<<<1, 32, 0, stream>>>(flag, max_iters, err);
  return cudaGetLastError();
}

}  // namespace nsa
