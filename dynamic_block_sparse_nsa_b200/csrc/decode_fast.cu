// NSA single-token decode, bf16, head dim 128, 16 query heads per KV head
// (the GQA group fills the 16 rows of one m16n8k16 tensor-core tile), selection
// blocks of 64 tokens.
//
// Decode moves the group's one shared KV subset and is bound by HBM bytes
// (EP94 notes §六; lchairun.cn NSA article, decode paragraph). Four kernels:
//
//  dec_cmp_partial  stream kernel over the compressed keys (see below); also
//                   writes, per 64-key tile and head, the running max it used
//                   and the exp-sums of its keys per overlapped selection
//                   block, because block scores need probabilities normalised
//                   by the final lse, which is known only at the end.
//  dec_select       one CTA per (sequence, KV head): merges the partials into
//                   lse and o_cmp, rescales the tile records into block scores
//                   summed over the group's heads, keeps block 0 plus the top
//                   n-1 others (ties to the lower index), computes the gates.
//  dec_sel_win      stream kernel over the selected blocks, then the window.
//  dec_combine      one CTA per unit: out = g0 o_cmp + g1 o_slc + g2 o_win.
//
// Stream kernel: persistent, one CTA per SM, 1 TMA producer warp + 4 consumer
// warps. The global sequence of 64-key tiles (sequence-major, then KV head,
// then tile) is split evenly over the CTAs. K and V halves of each tile go
// through a ring of 16 KB slots (128B-swizzled TMA boxes, L2 evict-first),
// each slot released as soon as it has been read. Consumer warps take tiles
// round-robin and keep online-softmax partials (m, l, O); at every segment
// boundary (unit, or unit and branch) the four warps merge their partials and
// write one per (CTA, segment), slot = cta + segment.
// Softmax runs in the log2 domain: z2 = (q . k) * scale * log2(e).
#include <algorithm>
#include <climits>

#include "device_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace nsa {
namespace {

constexpr int G = 16;                       // query heads per KV head
constexpr int D = 128;                      // head dim
constexpr int TK = 64;                      // keys per tile
constexpr int NCW = 4;                      // consumer warps
constexpr int SLOTS = 12;                   // ring of half-tiles (K or V)
constexpr int HALF_BYTES = TK * 64 * 2;     // 64 rows x 64 dims of bf16 (one TMA box)
constexpr int SLOT_BYTES = 2 * HALF_BYTES;  // 64 keys x 128 dims
constexpr int PART = 2 * G + G * D;         // m[16], l[16], o[16][128]
constexpr int MERGE_FLOATS = NCW * PART;
constexpr int SCR_PITCH = TK + 2;  // even: float2 stores stay aligned
constexpr uint64_t kWaitNs = 2000000000ull;

enum { MODE_CMP = 0, MODE_SW = 1 };

__device__ __forceinline__ int n_visible(int L, int l, int s, int Nc) {
  if (L < l) return 0;
  return min(Nc, (L - l) / s + 1);
}

__device__ __forceinline__ bool len_ok(int L, const DecFastArgs& a) { return L >= 1 && L <= a.T; }

// Selected blocks of a row at position L-1: all candidates when there are at
// most n, else exactly n.
__device__ __forceinline__ int n_selected(int L, const DecFastArgs& a) {
  return min(a.n, (L - 1) / a.bs + 1);
}

template <int MODE>
__device__ __forceinline__ int unit_tiles(int L, const DecFastArgs& a) {
  if (!len_ok(L, a)) return 0;
  if (MODE == MODE_CMP) return (n_visible(L, a.l, a.s, a.Nc) + TK - 1) / TK;
  const int wlen = min(a.w, L);
  return n_selected(L, a) + (wlen + TK - 1) / TK;
}

// ---------------------------------------------------------------------------
// consumer math (one warp: 16 heads x 64 keys)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void load_q_frags(uint32_t (&qa)[8][4], const __nv_bfloat16* q,
                                             int lane) {
  const uint32_t* qw = reinterpret_cast<const uint32_t*>(q);
  const int r0 = lane >> 2, c = (lane & 3) * 2;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    qa[ks][0] = __ldg(qw + (r0 * D + ks * 16 + c) / 2);
    qa[ks][1] = __ldg(qw + ((r0 + 8) * D + ks * 16 + c) / 2);
    qa[ks][2] = __ldg(qw + (r0 * D + ks * 16 + 8 + c) / 2);
    qa[ks][3] = __ldg(qw + ((r0 + 8) * D + ks * 16 + 8 + c) / 2);
  }
}

// S[16 x 64] = Q K^T over a swizzled 64-key tile.
__device__ __forceinline__ void qk_tile(float (&s)[8][4], const uint32_t (&qa)[8][4],
                                        uint32_t kbase, int lane) {
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
  const int mi = lane >> 3, r = lane & 7;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      const int key = (2 * np + (mi >> 1)) * 8 + r;
      const int chunk = 2 * ks + (mi & 1);
      const uint32_t addr =
          kbase + (chunk >> 3) * HALF_BYTES + key * 128 + (((chunk & 7) ^ (key & 7)) << 4);
      uint32_t b0, b1, b2, b3;
      ptx::ldsm_x4(addr, b0, b1, b2, b3);
      ptx::mma_16816(s[2 * np], qa[ks], b0, b1);
      ptx::mma_16816(s[2 * np + 1], qa[ks], b2, b3);
    }
  }
}

// O[16 x 128] += P[16 x 64] V over a swizzled 64-key tile.
__device__ __forceinline__ void pv_tile(float (&o)[16][4], const float (&p)[8][4], uint32_t vbase,
                                        int lane) {
  const int mi = lane >> 3, r = lane & 7;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t a[4];
    a[0] = ptx::pack_bf16(p[2 * kk][0], p[2 * kk][1]);
    a[1] = ptx::pack_bf16(p[2 * kk][2], p[2 * kk][3]);
    a[2] = ptx::pack_bf16(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = ptx::pack_bf16(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {
      const int key = kk * 16 + (mi & 1) * 8 + r;
      const int chunk = 2 * dp + (mi >> 1);
      const uint32_t addr =
          vbase + (chunk >> 3) * HALF_BYTES + key * 128 + (((chunk & 7) ^ (key & 7)) << 4);
      uint32_t b0, b1, b2, b3;
      ptx::ldsm_x4_t(addr, b0, b1, b2, b3);
      ptx::mma_16816(o[2 * dp], a, b0, b1);
      ptx::mma_16816(o[2 * dp + 1], a, b2, b3);
    }
  }
}

__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// Online-softmax step over one 64-key tile: mask keys >= nvalid, scale to the
// log2 domain, update running max/sum of rows r0 = lane/4 and r1 = r0 + 8,
// rescale O, and turn s into p = exp2(z - m_new).
__device__ __forceinline__ void softmax_step(float (&s)[8][4], float (&o)[16][4], float& m0,
                                             float& m1, float& l0, float& l1, int nvalid,
                                             float scale_log2, int lane) {
  const int c = (lane & 3) * 2;
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const bool ok = nt * 8 + c + e < nvalid;
      s[nt][e] = ok ? s[nt][e] * scale_log2 : -INFINITY;
      s[nt][2 + e] = ok ? s[nt][2 + e] * scale_log2 : -INFINITY;
      mx0 = fmaxf(mx0, s[nt][e]);
      mx1 = fmaxf(mx1, s[nt][2 + e]);
    }
  mx0 = quad_max(mx0);
  mx1 = quad_max(mx1);
  const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
  const float c0 = mn0 == -INFINITY ? 1.f : exp2f(m0 - mn0);
  const float c1 = mn1 == -INFINITY ? 1.f : exp2f(m1 - mn1);
  float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      s[nt][e] = mn0 == -INFINITY ? 0.f : exp2f(s[nt][e] - mn0);
      s[nt][2 + e] = mn1 == -INFINITY ? 0.f : exp2f(s[nt][2 + e] - mn1);
      sum0 += s[nt][e];
      sum1 += s[nt][2 + e];
    }
  sum0 = quad_sum(sum0);
  sum1 = quad_sum(sum1);
  l0 = l0 * c0 + sum0;
  l1 = l1 * c1 + sum1;
  m0 = mn0;
  m1 = mn1;
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    o[dt][0] *= c0;
    o[dt][1] *= c0;
    o[dt][2] *= c1;
    o[dt][3] *= c1;
  }
}

__device__ __forceinline__ void write_warp_partial(float* mrg, int w, int lane, float m0, float m1,
                                                   float l0, float l1, const float (&o)[16][4]) {
  float* pw = mrg + w * PART;
  const int r0 = lane >> 2, c = (lane & 3) * 2;
  if ((lane & 3) == 0) {
    pw[r0] = m0;
    pw[r0 + 8] = m1;
    pw[G + r0] = l0;
    pw[G + r0 + 8] = l1;
  }
  float* po = pw + 2 * G;
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    *reinterpret_cast<float2*>(po + r0 * D + dt * 8 + c) = make_float2(o[dt][0], o[dt][1]);
    *reinterpret_cast<float2*>(po + (r0 + 8) * D + dt * 8 + c) = make_float2(o[dt][2], o[dt][3]);
  }
}

// 128 consumer threads combine the NCW warp partials into dst.
__device__ __forceinline__ void merge_warps_to(float* dst, const float* mrg, int tid) {
  const int h = tid >> 3, e0 = (tid & 7) * 16;
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < NCW; ++w) M = fmaxf(M, mrg[w * PART + h]);
  float f[NCW], L = 0.f;
#pragma unroll
  for (int w = 0; w < NCW; ++w) {
    const float mw = mrg[w * PART + h];
    f[w] = (M == -INFINITY || mw == -INFINITY) ? 0.f : exp2f(mw - M);
    L += f[w] * mrg[w * PART + G + h];
  }
  if ((tid & 7) == 0) {
    dst[h] = M;
    dst[G + h] = L;
  }
#pragma unroll
  for (int e = e0; e < e0 + 16; e += 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
      const float4 v = *reinterpret_cast<const float4*>(mrg + w * PART + 2 * G + h * D + e);
      acc.x += f[w] * v.x;
      acc.y += f[w] * v.y;
      acc.z += f[w] * v.z;
      acc.w += f[w] * v.w;
    }
    *reinterpret_cast<float4*>(dst + 2 * G + h * D + e) = acc;
  }
}

// ---------------------------------------------------------------------------
// global tile order and its even split over CTAs
// ---------------------------------------------------------------------------

struct Plan {
  long long t0, t1;
  int b, g, tile, ntiles;
};

template <int MODE>
struct Walker {
  int b, g, tile, ntiles;
  __device__ void advance(const DecFastArgs& a) {
    if (++tile < ntiles) return;
    tile = 0;
    if (++g < a.Hkv) return;
    g = 0;
    do {
      ++b;
      ntiles = b < a.B ? unit_tiles<MODE>(a.seq_lens[b], a) : 1;
    } while (ntiles == 0);
  }
};

template <int MODE>
__device__ long long total_tiles_warp(const DecFastArgs& a, int lane) {
  long long total = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    long long tb = b < a.B ? (long long)unit_tiles<MODE>(a.seq_lens[b], a) * a.Hkv : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tb += __shfl_xor_sync(0xffffffffu, tb, o);
    total += tb;
  }
  return total;
}

template <int MODE>
__device__ void make_plan(const DecFastArgs& a, Plan* plan, int lane) {
  const long long total = total_tiles_warp<MODE>(a, lane);
  const long long c = blockIdx.x, grid = gridDim.x;
  const long long t0 = total * c / grid, t1 = total * (c + 1) / grid;
  if (lane == 0) {
    plan->t0 = t0;
    plan->t1 = t1;
    plan->b = plan->g = plan->tile = 0;
    plan->ntiles = 1;
    if (t1 > t0) {
      long long acc = 0;
      for (int b = 0; b < a.B; ++b) {
        const int nt = unit_tiles<MODE>(a.seq_lens[b], a);
        const long long span = (long long)nt * a.Hkv;
        if (t0 < acc + span) {
          const long long off = t0 - acc;
          plan->b = b;
          plan->g = (int)(off / nt);
          plan->tile = (int)(off % nt);
          plan->ntiles = nt;
          break;
        }
        acc += span;
      }
    }
  }
}

// CTA (of `grid`) whose share of `total` tiles holds global tile `tile`.
__device__ __forceinline__ int owner_cta(long long tile, long long total, long long grid) {
  long long cc = tile * grid / total;
  while (cc > 0 && total * cc / grid > tile) --cc;
  while (cc + 1 < grid && total * (cc + 1) / grid <= tile) ++cc;
  return (int)cc;
}

// ---------------------------------------------------------------------------
// the stream kernel
// ---------------------------------------------------------------------------

template <int MODE>
struct TileSrc {
  int row;      // TMA row (outer coordinate)
  int nvalid;   // valid keys in the tile
};

template <int MODE>
__device__ __forceinline__ TileSrc<MODE> tile_source(const DecFastArgs& a, int b, int g, int tile) {
  TileSrc<MODE> ts;
  const int L = a.seq_lens[b];
  if (MODE == MODE_CMP) {
    ts.row = b * a.Nc + tile * TK;
    ts.nvalid = min(TK, n_visible(L, a.l, a.s, a.Nc) - tile * TK);
  } else {
    const int t = L - 1, ns = n_selected(L, a);
    int start;
    if (tile < ns) {
      start = a.sel[(long)(b * a.Hkv + g) * a.n + tile] * a.bs;
    } else {
      start = t - min(a.w, L) + 1 + (tile - ns) * TK;
    }
    ts.row = b * a.T + start;
    ts.nvalid = min(TK, t - start + 1);
  }
  return ts;
}

template <int MODE>
__device__ __forceinline__ int segment_of(const DecFastArgs& a, int b, int g, int tile) {
  const int u = b * a.Hkv + g;
  if (MODE == MODE_CMP) return u;
  return 2 * u + (tile >= n_selected(a.seq_lens[b], a) ? 1 : 0);
}

template <int MODE>
__global__ void __launch_bounds__(160, 1)
    dec_stream_kernel(const __grid_constant__ DecFastArgs a, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* slots = smem;
  float* mrg = reinterpret_cast<float*>(smem + SLOTS * SLOT_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(mrg + MERGE_FLOATS);
  uint64_t* empty = full + SLOTS;
  Plan* plan = reinterpret_cast<Plan*>(empty + SLOTS);
  int* abort_flag = reinterpret_cast<int*>(plan + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == NCW) {
    make_plan<MODE>(a, plan, lane);
    if (lane == 0) {
      for (int i = 0; i < SLOTS; ++i) {
        ptx::mbar_init(&full[i], 1);
        ptx::mbar_init(&empty[i], 1);
      }
      *abort_flag = 0;
      ptx::fence_mbar_init();
      ptx::prefetch_tmap(&tk);
      ptx::prefetch_tmap(&tv);
    }
  }
  __syncthreads();
  const long long ntl = plan->t1 - plan->t0;
  if (ntl <= 0) return;
  float* part = MODE == MODE_CMP ? a.part1 : a.part3;

  if (warp == NCW) {
    // ---------------- producer: half-tile i = 2k (K) or 2k+1 (V) ----------------
    if (lane == 0) {
      const uint64_t pol = ptx::policy_evict_first();
      Walker<MODE> wk{plan->b, plan->g, plan->tile, plan->ntiles};
      long long i = 0;
      TileSrc<MODE> ts{};
      for (; i < 2 * ntl; ++i) {
        const int sl = (int)(i % SLOTS);
        const long long use = i / SLOTS;
        if (use > 0 && !ptx::mbar_wait(&empty[sl], (uint32_t)((use - 1) & 1), kWaitNs)) {
          atomicOr(a.err, kErrTimeout);
          atomicExch(abort_flag, 1);
        }
        if (*(volatile int*)abort_flag) break;
        const bool isv = i & 1;
        if (!isv) ts = tile_source<MODE>(a, wk.b, wk.g, wk.tile);
        unsigned char* dst = slots + sl * SLOT_BYTES;
        const CUtensorMap* m = isv ? &tv : &tk;
        ptx::mbar_arrive_expect_tx(&full[sl], SLOT_BYTES);
        ptx::tma_load_3d(dst, m, &full[sl], 0, wk.g, ts.row, pol);
        ptx::tma_load_3d(dst + HALF_BYTES, m, &full[sl], 64, wk.g, ts.row, pol);
        if (isv) wk.advance(a);
      }
      // every issued load must have landed before the CTA exits
      const long long issued = i;
      for (int sl = 0; sl < SLOTS && sl < issued; ++sl) {
        const long long last_use = (issued - 1 - sl) / SLOTS;
        if (!ptx::mbar_wait(&full[sl], (uint32_t)(last_use & 1), kWaitNs))
          atomicOr(a.err, kErrTimeout);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int tid = threadIdx.x;
  float* scr = mrg + warp * (G * SCR_PITCH);
  Walker<MODE> wk{plan->b, plan->g, plan->tile, plan->ntiles};
  int cur_seg = segment_of<MODE>(a, wk.b, wk.g, wk.tile);
  int cur_b = wk.b, cur_g = wk.g;
  uint32_t qa[8][4];
  const __nv_bfloat16* qbase = reinterpret_cast<const __nv_bfloat16*>(a.q);
  load_q_frags(qa, qbase + ((long)cur_b * a.Hq + cur_g * G) * D, lane);
  float o[16][4];
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int r0 = lane >> 2, c = (lane & 3) * 2;

  auto flush = [&](int seg) {
    ptx::named_bar_sync(1, NCW * 32);
    write_warp_partial(mrg, warp, lane, m0, m1, l0, l1, o);
    ptx::named_bar_sync(1, NCW * 32);
    merge_warps_to(part + (long)(blockIdx.x + seg) * PART, mrg, tid);
    ptx::named_bar_sync(1, NCW * 32);
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
  };

  for (long long k = 0; k < ntl; ++k) {
    const int seg = segment_of<MODE>(a, wk.b, wk.g, wk.tile);
    if (seg != cur_seg) {
      flush(cur_seg);
      cur_seg = seg;
      if (wk.b != cur_b || wk.g != cur_g) {
        cur_b = wk.b;
        cur_g = wk.g;
        load_q_frags(qa, qbase + ((long)cur_b * a.Hq + cur_g * G) * D, lane);
      }
    }
    if ((int)(k % NCW) == warp) {
      const int slk = (int)((2 * k) % SLOTS), slv = (int)((2 * k + 1) % SLOTS);
      const uint32_t pk = (uint32_t)(((2 * k) / SLOTS) & 1);
      const uint32_t pv = (uint32_t)(((2 * k + 1) / SLOTS) & 1);
      const TileSrc<MODE> ts = tile_source<MODE>(a, wk.b, wk.g, wk.tile);
      bool ok = !*(volatile int*)abort_flag;
      if (ok && !ptx::mbar_wait(&full[slk], pk, kWaitNs)) {
        if (lane == 0) {
          atomicOr(a.err, kErrTimeout);
          atomicExch(abort_flag, 1);
        }
        ok = false;
      }
      float s[8][4];
      if (ok) qk_tile(s, qa, ptx::smem_u32(slots + slk * SLOT_BYTES), lane);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[slk]);
      if (ok) {
        softmax_step(s, o, m0, m1, l0, l1, ts.nvalid, a.scale_log2, lane);
        if (MODE == MODE_CMP) {
          // tile record: running max per head, and exp-sums per overlapped block
#pragma unroll
          for (int nt = 0; nt < 8; ++nt) {
            *reinterpret_cast<float2*>(scr + r0 * SCR_PITCH + nt * 8 + c) =
                make_float2(s[nt][0], s[nt][1]);
            *reinterpret_cast<float2*>(scr + (r0 + 8) * SCR_PITCH + nt * 8 + c) =
                make_float2(s[nt][2], s[nt][3]);
          }
          __syncwarp();
          const int u = wk.b * a.Hkv + wk.g;
          float* rec = a.trec + ((long)u * a.tiles_max + wk.tile) * (G * (1 + a.nbt));
          if ((lane & 3) == 0) {
            rec[r0] = m0;
            rec[r0 + 8] = m1;
          }
          for (int x = lane; x < G * a.nbt; x += 32) {
            const int jl = x >> 4, h = x & 15;
            const int lo = a.klo[jl], hi = min((int)a.khi[jl], ts.nvalid - 1);
            float acc = 0.f;
            for (int kk = lo; kk <= hi; ++kk) acc += scr[h * SCR_PITCH + kk];
            rec[G + x] = acc;  // [1 + jl][h]
          }
          __syncwarp();
        }
      }
      if (ok && !ptx::mbar_wait(&full[slv], pv, kWaitNs)) {
        if (lane == 0) {
          atomicOr(a.err, kErrTimeout);
          atomicExch(abort_flag, 1);
        }
        ok = false;
      }
      if (ok) pv_tile(o, s, ptx::smem_u32(slots + slv * SLOT_BYTES), lane);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[slv]);
    }
    wk.advance(a);
  }
  flush(cur_seg);
}

// ---------------------------------------------------------------------------
// dec_select
// ---------------------------------------------------------------------------

constexpr int SEL_THREADS = 256;

__global__ void __launch_bounds__(SEL_THREADS) dec_select_kernel(const __grid_constant__ DecFastArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int u = blockIdx.x, b = u / a.Hkv, g = u - b * a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nblk = (a.T + a.bs - 1) / a.bs;
  long long* red_ll = reinterpret_cast<long long*>(sm);  // [16]
  float* lse2 = sm + 32;                  // [16]
  float* gate = lse2 + G;                 // [16][3]
  float* fac = gate + 3 * G;              // [tiles_max][16]
  float* scores = fac + a.tiles_max * G;  // [nblk]
  float* red_s = scores + nblk;           // [8]
  int* red_j = reinterpret_cast<int*>(red_s + 8);
  int* sel = red_j + 8;                   // [n]
  __shared__ int c_first, c_last;

  const int L = a.seq_lens[b];
  float* oacc = a.oacc + (long)u * G * D;
  if (!len_ok(L, a)) {
    for (int x = tid; x < G * D; x += SEL_THREADS)
      reinterpret_cast<__nv_bfloat16*>(a.out)[((long)b * a.Hq + g * G) * D + x] =
          __float2bfloat16_rn(0.f);
    if (a.sel_out)
      for (int x = tid; x < a.n; x += SEL_THREADS) a.sel_out[(long)u * a.n + x] = -1;
    if (tid == 0) atomicOr(a.err, kErrSeqLen);
    return;
  }
  const int t = L - 1;
  const int nvis = n_visible(L, a.l, a.s, a.Nc);
  const int ncand = t / a.bs + 1;
  const int tiles_u = (nvis + TK - 1) / TK;
  const __nv_bfloat16* qg =
      reinterpret_cast<const __nv_bfloat16*>(a.q) + ((long)b * a.Hq + g * G) * D;

  // gates (EP94 notes §五 gating): one warp per (head, branch) dot product
  for (int x = warp; x < 3 * G; x += SEL_THREADS / 32) {
    const int h = x / 3, br = x - h * 3;
    float gv;
    if (a.gate_mode == 1) {
      gv = a.fixed_gates[br];
    } else {
      float dot = 0.f;
      for (int e = lane; e < D; e += 32)
        dot = fmaf(__bfloat162float(qg[h * D + e]), __ldg(a.w_gate + e * 3 + br), dot);
      dot = warp_sum(dot);
      gv = 1.f / (1.f + expf(-dot));
    }
    if (lane == 0) {
      gate[x] = gv;
      a.gates[(long)u * 3 * G + x] = gv;
    }
  }
  for (int j = tid; j < ncand; j += SEL_THREADS) scores[j] = 0.f;

  if (nvis > 0) {
    long long before = 0, total = 0;
    for (int bb = tid; bb < a.B; bb += SEL_THREADS) {
      const long long nt = (long long)unit_tiles<MODE_CMP>(a.seq_lens[bb], a) * a.Hkv;
      total += nt;
      if (bb < b) before += nt;
    }
    for (int o = 16; o > 0; o >>= 1) {
      total += __shfl_xor_sync(0xffffffffu, total, o);
      before += __shfl_xor_sync(0xffffffffu, before, o);
    }
    if (lane == 0) {
      red_ll[2 * warp] = total;
      red_ll[2 * warp + 1] = before;
    }
    __syncthreads();
    if (tid == 0) {
      long long T0 = 0, P0 = 0;
      for (int w = 0; w < SEL_THREADS / 32; ++w) {
        T0 += red_ll[2 * w];
        P0 += red_ll[2 * w + 1];
      }
      const long long Pu = P0 + (long long)g * tiles_u;
      c_first = owner_cta(Pu, T0, a.grid1);
      c_last = owner_cta(Pu + tiles_u - 1, T0, a.grid1);
    }
    __syncthreads();
    if (tid < G) {
      float M = -INFINITY;
      for (int cc = c_first; cc <= c_last; ++cc)
        M = fmaxf(M, a.part1[(long)(cc + u) * PART + tid]);
      float Ls = 0.f;
      for (int cc = c_first; cc <= c_last; ++cc) {
        const float* pp = a.part1 + (long)(cc + u) * PART;
        Ls += exp2f(pp[tid] - M) * pp[G + tid];
      }
      lse2[tid] = M + log2f(Ls);
    }
    __syncthreads();
    for (int x = tid; x < G * D; x += SEL_THREADS) {
      const int h = x / D;
      float acc = 0.f;
      for (int cc = c_first; cc <= c_last; ++cc) {
        const float* pp = a.part1 + (long)(cc + u) * PART;
        acc += exp2f(pp[h] - lse2[h]) * pp[2 * G + x];
      }
      oacc[x] = gate[h * 3] * acc;
    }
    const float* rec = a.trec + (long)u * a.tiles_max * (G * (1 + a.nbt));
    for (int x = tid; x < tiles_u * G; x += SEL_THREADS) {
      const int tau = x / G, h = x - tau * G;
      fac[x] = exp2f(rec[(long)tau * G * (1 + a.nbt) + h] - lse2[h]);
    }
    __syncthreads();
    // block j gets its record entries from tile j / R and, for its first
    // compressed key, possibly the tile before (R = blocks per tile start)
    const int R = (TK * a.s) / a.bs;
    for (int j = tid; j < ncand; j += SEL_THREADS) {
      float acc = 0.f;
      const int tau_hi = min(j / R, tiles_u - 1);
      const int tau_lo = max(0, (j - a.nbt + R) / R);
      for (int tau = tau_lo; tau <= tau_hi; ++tau) {
        const int jl = j - tau * R;
        if (jl < 0 || jl >= a.nbt) continue;
        const float4* rt = reinterpret_cast<const float4*>(
            rec + (long)tau * G * (1 + a.nbt) + G * (1 + jl));
        const float* f = fac + tau * G;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float4 v = __ldg(rt + q4);
          acc += f[4 * q4] * v.x;
          acc += f[4 * q4 + 1] * v.y;
          acc += f[4 * q4 + 2] * v.z;
          acc += f[4 * q4 + 3] * v.w;
        }
      }
      scores[j] = acc;
    }
  } else {
    for (int x = tid; x < G * D; x += SEL_THREADS) oacc[x] = 0.f;
  }
  __syncthreads();

  // top-n: block 0 kept, the best n-1 others (ties to the lower index)
  int ns;
  if (ncand <= a.n) {
    for (int j = tid; j < ncand; j += SEL_THREADS) sel[j] = j;
    ns = ncand;
  } else {
    if (tid == 0) sel[0] = 0;
    for (int r = 1; r < a.n; ++r) {
      float bs = -INFINITY;
      int bj = INT_MAX;
      for (int j = 1 + tid; j < ncand; j += SEL_THREADS) {
        const float sj = scores[j];
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
        red_s[warp] = bs;
        red_j[warp] = bj;
      }
      __syncthreads();
      if (warp == 0) {
        float s0 = lane < SEL_THREADS / 32 ? red_s[lane] : -INFINITY;
        int j0 = lane < SEL_THREADS / 32 ? red_j[lane] : INT_MAX;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) {
          const float os = __shfl_xor_sync(0xffffffffu, s0, o);
          const int oj = __shfl_xor_sync(0xffffffffu, j0, o);
          if (sel_better(os, oj, s0, j0)) {
            s0 = os;
            j0 = oj;
          }
        }
        if (lane == 0) {
          sel[r] = j0;
          scores[j0] = -INFINITY;
        }
      }
      __syncthreads();
    }
    if (tid == 0) {
      for (int x = 1; x < a.n; ++x) {
        const int v = sel[x];
        int p = x - 1;
        while (p >= 0 && sel[p] > v) {
          sel[p + 1] = sel[p];
          --p;
        }
        sel[p + 1] = v;
      }
    }
    ns = a.n;
  }
  __syncthreads();
  for (int x = tid; x < a.n; x += SEL_THREADS) {
    const int v = x < ns ? sel[x] : -1;
    a.sel[(long)u * a.n + x] = v;
    if (a.sel_out) a.sel_out[(long)u * a.n + x] = v;
  }
}

// ---------------------------------------------------------------------------
// dec_combine
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(128) dec_combine_kernel(const __grid_constant__ DecFastArgs a) {
  const int u = blockIdx.x, b = u / a.Hkv, g = u - b * a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ long long red[8];
  __shared__ int crange[4];
  const int L = a.seq_lens[b];
  if (!len_ok(L, a)) return;  // output zeroed by dec_select
  const int ns = n_selected(L, a);
  const int nw = (min(a.w, L) + TK - 1) / TK;
  long long total = 0, before = 0;
  for (int bb = tid; bb < a.B; bb += 128) {
    const long long nt = (long long)unit_tiles<MODE_SW>(a.seq_lens[bb], a) * a.Hkv;
    total += nt;
    if (bb < b) before += nt;
  }
  for (int o = 16; o > 0; o >>= 1) {
    total += __shfl_xor_sync(0xffffffffu, total, o);
    before += __shfl_xor_sync(0xffffffffu, before, o);
  }
  if (lane == 0) {
    red[2 * warp] = total;
    red[2 * warp + 1] = before;
  }
  __syncthreads();
  if (tid == 0) {
    long long T0 = 0, P0 = 0;
    for (int w = 0; w < 4; ++w) {
      T0 += red[2 * w];
      P0 += red[2 * w + 1];
    }
    const long long Pu = P0 + (long long)g * (ns + nw);
    crange[0] = owner_cta(Pu, T0, a.grid3);
    crange[1] = owner_cta(Pu + ns - 1, T0, a.grid3);
    crange[2] = owner_cta(Pu + ns, T0, a.grid3);
    crange[3] = owner_cta(Pu + ns + nw - 1, T0, a.grid3);
  }
  __syncthreads();
  const int h = tid >> 3, e0 = (tid & 7) * 16;
  float res[16];
  const float* oc = a.oacc + (long)u * G * D + h * D + e0;
#pragma unroll
  for (int e = 0; e < 16; ++e) res[e] = oc[e];
#pragma unroll
  for (int br = 0; br < 2; ++br) {
    const int seg = 2 * u + br;
    const int c0 = crange[2 * br], c1 = crange[2 * br + 1];
    float M = -INFINITY;
    for (int cc = c0; cc <= c1; ++cc) M = fmaxf(M, a.part3[(long)(cc + seg) * PART + h]);
    float Ls = 0.f;
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.f;
    for (int cc = c0; cc <= c1; ++cc) {
      const float* pp = a.part3 + (long)(cc + seg) * PART;
      const float mm = pp[h];
      const float f = mm == -INFINITY ? 0.f : exp2f(mm - M);
      Ls += f * pp[G + h];
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] += f * pp[2 * G + h * D + e0 + e];
    }
    const float gs = a.gates[(long)u * 3 * G + h * 3 + 1 + br] / Ls;
#pragma unroll
    for (int e = 0; e < 16; ++e) res[e] += gs * acc[e];
  }
  __nv_bfloat16* orow =
      reinterpret_cast<__nv_bfloat16*>(a.out) + ((long)b * a.Hq + g * G + h) * D + e0;
#pragma unroll
  for (int e = 0; e < 16; e += 2)
    *reinterpret_cast<__nv_bfloat162*>(orow + e) = __floats2bfloat162_rn(res[e], res[e + 1]);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  size_t part1, trec, oacc, gates, sel, part3, total;
};

WsLayout ws_layout(const DecFastArgs& a) {
  WsLayout w{};
  const size_t units = (size_t)a.B * a.Hkv;
  size_t off = 0;
  w.part1 = off; off = align256(off + (size_t)(a.grid1 + units) * PART * 4);
  w.trec = off; off = align256(off + units * a.tiles_max * G * (1 + a.nbt) * 4);
  w.oacc = off; off = align256(off + units * G * D * 4);
  w.gates = off; off = align256(off + units * 3 * G * 4);
  w.sel = off; off = align256(off + units * a.n * 4);
  w.part3 = off; off = align256(off + (size_t)(a.grid3 + 2 * units) * PART * 4);
  w.total = off;
  return w;
}

DecFastArgs base_args(const nsa_params& p) {
  DecFastArgs a{};
  a.B = p.B;
  a.T = p.T;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.l = p.cmp_block;
  a.s = p.cmp_stride;
  a.bs = p.sel_block;
  a.n = p.top_n;
  a.w = p.window;
  a.Nc = nsa_num_cmp_blocks(p.T, p.cmp_block, p.cmp_stride);
  a.nbt = (63 * a.s + a.l - 1) / a.bs + 2;
  a.tiles_max = (a.Nc + TK - 1) / TK;
  for (int jl = 0; jl < a.nbt && jl < kDecMaxNbt; ++jl) {
    // keys of a 64-key tile (relative index) overlapping its jl-th block
    const int num = jl * a.bs - a.l + 1;
    const int lo = num <= 0 ? 0 : (num + a.s - 1) / a.s;
    const int hi = std::min(TK - 1, (jl * a.bs + a.bs - 1) / a.s);
    a.klo[jl] = (int8_t)std::min(lo, 127);
    a.khi[jl] = (int8_t)hi;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  a.grid1 = sms;
  a.grid3 = sms;
  const float scale = p.softmax_scale != 0.f ? p.softmax_scale : 1.f / sqrtf((float)p.d);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.gate_mode = p.gate_mode;
  for (int i = 0; i < 3; ++i) a.fixed_gates[i] = p.fixed_gates[i];
  return a;
}

constexpr size_t kStreamSmem =
    1024 + SLOTS * SLOT_BYTES + MERGE_FLOATS * 4 + 2 * SLOTS * 8 + sizeof(Plan) + 16;

}  // namespace

bool decode_fast_eligible(const nsa_params& p) {
  if (!(p.dtype == NSA_DTYPE_BF16 && p.d == D && p.Hq == G * p.Hkv && p.sel_block == TK &&
        p.top_n <= 256 && p.T >= 1))
    return false;
  // 64-key compressed tiles must start on selection-block boundaries
  if ((TK * p.cmp_stride) % p.sel_block != 0) return false;
  const int nbt = (63 * p.cmp_stride + p.cmp_block - 1) / p.sel_block + 2;
  return nbt <= kDecMaxNbt;
}

size_t decode_fast_ws_bytes(const nsa_params& p) {
  if (!decode_fast_eligible(p)) return 0;
  return ws_layout(base_args(p)).total;
}

cudaError_t launch_decode_fast(const nsa_params& p, const void* q, const void* k, const void* v,
                               const int32_t* seq_lens, const void* kc, const void* vc,
                               const float* w_gate, void* out, int32_t* sel_out, void* ws,
                               unsigned* err, cudaStream_t stream) {
  DecFastArgs a = base_args(p);
  const WsLayout L = ws_layout(a);
  char* w = static_cast<char*>(ws);
  a.q = q;
  a.seq_lens = seq_lens;
  a.w_gate = w_gate;
  a.out = out;
  a.sel_out = sel_out;
  a.err = err;
  a.part1 = reinterpret_cast<float*>(w + L.part1);
  a.trec = reinterpret_cast<float*>(w + L.trec);
  a.oacc = reinterpret_cast<float*>(w + L.oacc);
  a.gates = reinterpret_cast<float*>(w + L.gates);
  a.sel = reinterpret_cast<int*>(w + L.sel);
  a.part3 = reinterpret_cast<float*>(w + L.part3);

  CUtensorMap tkc, tvc, tk, tv;
  const uint64_t rows = (uint64_t)p.B * p.T;
  bool okm = true;
  if (a.Nc > 0) {
    const uint64_t rows_c = (uint64_t)p.B * a.Nc;
    okm &= make_tmap_bf16_3d(&tkc, kc, D, p.Hkv, rows_c, 64, 1, TK, true);
    okm &= make_tmap_bf16_3d(&tvc, vc, D, p.Hkv, rows_c, 64, 1, TK, true);
  }
  okm &= make_tmap_bf16_3d(&tk, k, D, p.Hkv, rows, 64, 1, TK, true);
  okm &= make_tmap_bf16_3d(&tv, v, D, p.Hkv, rows, 64, 1, TK, true);
  if (!okm) return cudaErrorInvalidValue;

  cudaError_t e;
  if (a.Nc > 0) {
    TraceScope trace("dec_cmp_partial", stream);
    cudaFuncSetAttribute(dec_stream_kernel<MODE_CMP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kStreamSmem);
    dec_stream_kernel<MODE_CMP><<<a.grid1, 160, kStreamSmem, stream>>>(a, tkc, tvc);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const int nblk = (p.T + p.sel_block - 1) / p.sel_block;
    const size_t smem = (size_t)(32 + G + 3 * G + a.tiles_max * G + nblk + 8) * 4 + 8 * 4 +
                        (size_t)a.n * 4 + 16;
    TraceScope trace("dec_select", stream);
    cudaFuncSetAttribute(dec_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dec_select_kernel<<<p.B * p.Hkv, SEL_THREADS, smem, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    TraceScope trace("dec_sel_win", stream);
    cudaFuncSetAttribute(dec_stream_kernel<MODE_SW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kStreamSmem);
    dec_stream_kernel<MODE_SW><<<a.grid3, 160, kStreamSmem, stream>>>(a, tk, tv);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    TraceScope trace("dec_combine", stream);
    dec_combine_kernel<<<p.B * p.Hkv, 128, 0, stream>>>(a);
    return cudaGetLastError();
  }
}

}  // namespace nsa
