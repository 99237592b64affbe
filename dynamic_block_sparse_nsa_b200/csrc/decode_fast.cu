// NSA single-token decode, bf16, head dim 128, 16 query heads per KV head
// (the GQA group fills the 16 rows of one m16n8k16 tensor-core tile).
//
// Decode moves the group's one shared KV subset and is bound by HBM bytes
// (EP94 notes §六; lchairun.cn NSA article, decode paragraph). Three kernels:
//
//  dec_cmp_partial  persistent, one CTA per SM, 1 TMA producer warp + 4
//                   consumer warps. The (sequence, KV head, 64-key tile) space
//                   of the compressed keys is split evenly over the CTAs; each
//                   CTA streams its range through a 5-stage mbarrier pipeline
//                   (128B-swizzled TMA boxes, L2 evict-first) and keeps online
//                   softmax partials (m, l, O) per unit segment. Because block
//                   scores need probabilities normalised by the final lse, each
//                   tile also records, per head, the running max it used and
//                   the exp-sums of its keys per overlapped selection block.
//  dec_select       one CTA per (sequence, KV head): merges the partials into
//                   lse and o_cmp, rescales the tile records into block scores
//                   summed over the group's heads, keeps block 0 plus the top
//                   n-1 others (ties to the lower index), computes the gates.
//  dec_sel_win      one CTA per 128-key item of the selected blocks or the
//                   window: TMA load, tile softmax, partial; the last CTA of a
//                   unit merges the partials and writes out = g0 o_cmp + g1
//                   o_slc + g2 o_win.
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
constexpr int STAGES = 5;
constexpr int HALF_BYTES = TK * 64 * 2;     // 64 rows x 64 dims of bf16 (one TMA box)
constexpr int TILE_BYTES = 2 * HALF_BYTES;  // 64 keys x 128 dims
constexpr int STAGE_BYTES = 2 * TILE_BYTES; // K~ tile + V~ tile
constexpr int PART = 2 * G + G * D;         // m[16], l[16], o[16][128]
constexpr int MERGE_FLOATS = NCW * (2 * G + G * D);
constexpr int SCR_PITCH = TK + 1;
constexpr uint64_t kWaitNs = 2000000000ull;

__device__ __forceinline__ int n_visible(int L, int l, int s, int Nc) {
  if (L < l) return 0;
  return min(Nc, (L - l) / s + 1);
}

__device__ __forceinline__ int tiles_of(int L, const DecFastArgs& a) {
  if (L < 1 || L > a.T) return 0;
  return (n_visible(L, a.l, a.s, a.Nc) + TK - 1) / TK;
}

// ---------------------------------------------------------------------------
// shared pieces of the consumer math
// ---------------------------------------------------------------------------

// A fragments of the 16 x 128 query block of unit (b, g), loaded from global.
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

// S[16 x 8*NT] = Q K^T for keys [key0, key0 + 8*NT) of a swizzled tile.
template <int NT>
__device__ __forceinline__ void qk_tile(float (&s)[NT][4], const uint32_t (&qa)[8][4],
                                        uint32_t kbase, int key0, int lane) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
  const int mi = lane >> 3, r = lane & 7;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      const int key = key0 + (2 * np + (mi >> 1)) * 8 + r;
      const int chunk = 2 * ks + (mi & 1);
      const uint32_t addr =
          kbase + (chunk >> 3) * HALF_BYTES + key * 128 + ((((chunk & 7) ^ (key & 7))) << 4);
      uint32_t b0, b1, b2, b3;
      ptx::ldsm_x4(addr, b0, b1, b2, b3);
      ptx::mma_16816(s[2 * np], qa[ks], b0, b1);
      ptx::mma_16816(s[2 * np + 1], qa[ks], b2, b3);
    }
  }
}

// O[16 x 128] += P[16 x 16*KS] V for keys [key0, key0 + 16*KS) of a swizzled tile.
template <int KS>
__device__ __forceinline__ void pv_tile(float (&o)[16][4], const float (&p)[2 * KS][4],
                                        uint32_t vbase, int key0, int lane) {
  const int mi = lane >> 3, r = lane & 7;
#pragma unroll
  for (int kk = 0; kk < KS; ++kk) {
    uint32_t a[4];
    a[0] = ptx::pack_bf16(p[2 * kk][0], p[2 * kk][1]);
    a[1] = ptx::pack_bf16(p[2 * kk][2], p[2 * kk][3]);
    a[2] = ptx::pack_bf16(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = ptx::pack_bf16(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {
      const int key = key0 + kk * 16 + (mi & 1) * 8 + r;
      const int chunk = 2 * dp + (mi >> 1);
      const uint32_t addr =
          vbase + (chunk >> 3) * HALF_BYTES + key * 128 + ((((chunk & 7) ^ (key & 7))) << 4);
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

// Softmax step over NT n-tiles (8 keys each): mask keys >= nvalid, scale to
// the log2 domain, update the running max / sum of rows r0 and r1, rescale O,
// turn s into p = exp2(z - m).
template <int NT>
__device__ __forceinline__ void softmax_step(float (&s)[NT][4], float (&o)[16][4], float& m0,
                                             float& m1, float& l0, float& l1, int nvalid,
                                             float scale_log2, int lane) {
  const int c = (lane & 3) * 2;
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
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
  for (int nt = 0; nt < NT; ++nt)
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

// Merge the per-warp partials (in `mrg`: [NCW][m 16 | l 16 | o 16x128]) of
// the nthreads consumer threads into one partial written to dst.
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
    po[r0 * D + dt * 8 + c] = o[dt][0];
    po[r0 * D + dt * 8 + c + 1] = o[dt][1];
    po[(r0 + 8) * D + dt * 8 + c] = o[dt][2];
    po[(r0 + 8) * D + dt * 8 + c + 1] = o[dt][3];
  }
}

// 128 threads combine NCW warp partials into dst (m, l, unnormalised o).
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
#pragma unroll 4
  for (int e = e0; e < e0 + 16; ++e) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < NCW; ++w) acc += f[w] * mrg[w * PART + 2 * G + h * D + e];
    dst[2 * G + h * D + e] = acc;
  }
}

// ---------------------------------------------------------------------------
// dec_cmp_partial
// ---------------------------------------------------------------------------

struct Plan {
  long long t0, t1;   // global tile range of this CTA
  int b, g, tile, ntiles;
};

// Per-warp walk of the global tile order (sequence-major, then KV head, then
// tile). All warps advance their own copy identically.
struct Walker {
  int b, g, tile, ntiles;
  __device__ void advance(const DecFastArgs& a) {
    if (++tile < ntiles) return;
    tile = 0;
    if (++g < a.Hkv) return;
    g = 0;
    do {
      ++b;
      ntiles = b < a.B ? tiles_of(a.seq_lens[b], a) : 1;
    } while (ntiles == 0);
  }
};

__device__ void make_plan(const DecFastArgs& a, Plan* plan, int lane) {
  // total tiles and this CTA's even share
  long long total = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    long long tb = b < a.B ? (long long)tiles_of(a.seq_lens[b], a) * a.Hkv : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tb += __shfl_xor_sync(0xffffffffu, tb, o);
    total += tb;
  }
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
        const int nt = tiles_of(a.seq_lens[b], a);
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

__global__ void __launch_bounds__(160, 1)
    dec_cmp_partial_kernel(const __grid_constant__ DecFastArgs a,
                           const __grid_constant__ CUtensorMap tkc,
                           const __grid_constant__ CUtensorMap tvc) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* stages = smem;
  float* mrg = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);  // merge area / scratch
  uint64_t* full = reinterpret_cast<uint64_t*>(mrg + MERGE_FLOATS);
  uint64_t* empty = full + STAGES;
  Plan* plan = reinterpret_cast<Plan*>(empty + STAGES);
  int* abort_flag = reinterpret_cast<int*>(plan + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == NCW) {
    make_plan(a, plan, lane);
    if (lane == 0) {
      for (int i = 0; i < STAGES; ++i) {
        ptx::mbar_init(&full[i], 1);
        ptx::mbar_init(&empty[i], 1);
      }
      *abort_flag = 0;
      ptx::fence_mbar_init();
      ptx::prefetch_tmap(&tkc);
      ptx::prefetch_tmap(&tvc);
    }
  }
  __syncthreads();
  const long long ntl = plan->t1 - plan->t0;
  if (ntl <= 0) return;

  if (warp == NCW) {
    // ---------------- producer ----------------
    if (lane == 0) {
      const uint64_t pol = ptx::policy_evict_first();
      Walker wk{plan->b, plan->g, plan->tile, plan->ntiles};
      long long k = 0;
      for (; k < ntl; ++k) {
        const int st = (int)(k % STAGES);
        const long long use = k / STAGES;
        if (use > 0 && !ptx::mbar_wait(&empty[st], (uint32_t)((use - 1) & 1), kWaitNs)) {
          atomicOr(a.err, kErrTimeout);
          atomicExch(abort_flag, 1);
        }
        if (*(volatile int*)abort_flag) break;
        unsigned char* dk = stages + st * STAGE_BYTES;
        unsigned char* dv = dk + TILE_BYTES;
        const int row = wk.b * a.Nc + wk.tile * TK;
        ptx::mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
        ptx::tma_load_3d(dk, &tkc, &full[st], 0, wk.g, row, pol);
        ptx::tma_load_3d(dk + HALF_BYTES, &tkc, &full[st], 64, wk.g, row, pol);
        ptx::tma_load_3d(dv, &tvc, &full[st], 0, wk.g, row, pol);
        ptx::tma_load_3d(dv + HALF_BYTES, &tvc, &full[st], 64, wk.g, row, pol);
        wk.advance(a);
      }
      // Drain: every issued load must have landed before the CTA exits.
      const long long issued = k;
      for (int st = 0; st < STAGES && st < issued; ++st) {
        const long long last_use = (issued - 1 - st) / STAGES;
        if (!ptx::mbar_wait(&full[st], (uint32_t)(last_use & 1), kWaitNs))
          atomicOr(a.err, kErrTimeout);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int tid = threadIdx.x;  // 0..127
  float* scr = mrg + warp * (G * SCR_PITCH);  // per-warp probability scratch
  Walker wk{plan->b, plan->g, plan->tile, plan->ntiles};
  int cur_b = wk.b, cur_g = wk.g;
  uint32_t qa[8][4];
  const __nv_bfloat16* qbase = reinterpret_cast<const __nv_bfloat16*>(a.q);
  load_q_frags(qa, qbase + ((long)cur_b * a.Hq + cur_g * G) * D, lane);
  float o[16][4];
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int r0 = lane >> 2, c = (lane & 3) * 2;
  const int nbt = a.nbt;

  auto flush = [&](int fb, int fg) {
    ptx::named_bar_sync(1, NCW * 32);
    write_warp_partial(mrg, warp, lane, m0, m1, l0, l1, o);
    ptx::named_bar_sync(1, NCW * 32);
    const int u = fb * a.Hkv + fg;
    merge_warps_to(a.part1 + (long)(blockIdx.x + u) * PART, mrg, tid);
    ptx::named_bar_sync(1, NCW * 32);
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
  };

  for (long long k = 0; k < ntl; ++k) {
    if (wk.b != cur_b || wk.g != cur_g) {
      flush(cur_b, cur_g);
      cur_b = wk.b;
      cur_g = wk.g;
      load_q_frags(qa, qbase + ((long)cur_b * a.Hq + cur_g * G) * D, lane);
    }
    if ((int)(k % NCW) == warp) {
      const int st = (int)(k % STAGES);
      const uint32_t parity = (uint32_t)((k / STAGES) & 1);
      bool ok = !*(volatile int*)abort_flag;
      if (ok && !ptx::mbar_wait(&full[st], parity, kWaitNs)) {
        if (lane == 0) {
          atomicOr(a.err, kErrTimeout);
          atomicExch(abort_flag, 1);
        }
        ok = false;
      }
      if (ok) {
        const int L = a.seq_lens[wk.b];
        const int nvis = n_visible(L, a.l, a.s, a.Nc);
        const int i0 = wk.tile * TK;
        const int nvalid = min(TK, nvis - i0);
        const uint32_t kb = ptx::smem_u32(stages + st * STAGE_BYTES);
        float s[8][4];
        qk_tile<8>(s, qa, kb, 0, lane);
        softmax_step<8>(s, o, m0, m1, l0, l1, nvalid, a.scale_log2, lane);
        // per-tile block-score record: running max + exp-sums per selection block
        __syncwarp();
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          scr[r0 * SCR_PITCH + nt * 8 + c] = s[nt][0];
          scr[r0 * SCR_PITCH + nt * 8 + c + 1] = s[nt][1];
          scr[(r0 + 8) * SCR_PITCH + nt * 8 + c] = s[nt][2];
          scr[(r0 + 8) * SCR_PITCH + nt * 8 + c + 1] = s[nt][3];
        }
        __syncwarp();
        const int u = wk.b * a.Hkv + wk.g;
        float* rec = a.trec + ((long)u * a.tiles_max + wk.tile) * (G * (1 + nbt));
        if ((lane & 3) == 0) {
          rec[r0 * (1 + nbt)] = m0;
          rec[(r0 + 8) * (1 + nbt)] = m1;
        }
        const int jbase = (i0 * a.s) / a.bs;
        for (int x = lane; x < G * nbt; x += 32) {
          const int h = x / nbt, jl = x - h * nbt;
          const int j = jbase + jl;
          const int num = j * a.bs - a.l + 1;
          int ilo = num <= 0 ? 0 : (num + a.s - 1) / a.s;
          int ihi = (j * a.bs + a.bs - 1) / a.s;
          ilo = max(ilo, i0);
          ihi = min(ihi, i0 + nvalid - 1);
          float acc = 0.f;
          for (int i = ilo; i <= ihi; ++i) acc += scr[h * SCR_PITCH + (i - i0)];
          rec[h * (1 + nbt) + 1 + jl] = acc;
        }
        pv_tile<4>(o, s, kb + TILE_BYTES, 0, lane);
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[st]);
    }
    wk.advance(a);
  }
  flush(cur_b, cur_g);
}

// ---------------------------------------------------------------------------
// dec_select
// ---------------------------------------------------------------------------

constexpr int SEL_THREADS = 256;

__global__ void __launch_bounds__(SEL_THREADS) dec_select_kernel(const __grid_constant__ DecFastArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int u = blockIdx.x, b = u / a.Hkv, g = u - b * a.Hkv;
  const int tid = threadIdx.x;
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
  if (L < 1 || L > a.T) {
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

  // gates (EP94 notes §五 gating)
  if (tid < 3 * G) {
    const int h = tid / 3, br = tid - h * 3;
    float gv;
    if (a.gate_mode == 1) {
      gv = a.fixed_gates[br];
    } else {
      float dot = 0.f;
      for (int e = 0; e < D; ++e) dot = fmaf(__bfloat162float(qg[h * D + e]), a.w_gate[e * 3 + br], dot);
      gv = 1.f / (1.f + expf(-dot));
    }
    gate[tid] = gv;
    a.gates[(long)u * 3 * G + tid] = gv;
  }
  for (int j = tid; j < ncand; j += SEL_THREADS) scores[j] = 0.f;

  if (nvis > 0) {
    // position of this unit in the global tile order and the CTAs covering it
    long long before = 0, total = 0;
    for (int bb = tid; bb < a.B; bb += SEL_THREADS) {
      const long long nt = (long long)tiles_of(a.seq_lens[bb], a) * a.Hkv;
      total += nt;
      if (bb < b) before += nt;
    }
    for (int o = 16; o > 0; o >>= 1) {
      total += __shfl_xor_sync(0xffffffffu, total, o);
      before += __shfl_xor_sync(0xffffffffu, before, o);
    }
    if ((tid & 31) == 0) {
      red_ll[2 * (tid >> 5)] = total;
      red_ll[2 * (tid >> 5) + 1] = before;
    }
    __syncthreads();
    if (tid == 0) {
      long long T0 = 0, P0 = 0;
      for (int w = 0; w < SEL_THREADS / 32; ++w) {
        T0 += red_ll[2 * w];
        P0 += red_ll[2 * w + 1];
      }
      const long long Pu = P0 + (long long)g * tiles_u;
      const long long grid = a.grid1;
      auto owner = [&](long long tile) {  // CTA whose range holds `tile`
        long long cc = tile * grid / T0;
        while (cc > 0 && T0 * cc / grid > tile) --cc;
        while (cc + 1 < grid && T0 * (cc + 1) / grid <= tile) ++cc;
        return (int)cc;
      };
      c_first = owner(Pu);
      c_last = owner(Pu + tiles_u - 1);
    }
    __syncthreads();
    // lse per head
    if (tid < G) {
      float M = -INFINITY;
      for (int cc = c_first; cc <= c_last; ++cc) M = fmaxf(M, a.part1[(long)(cc + u) * PART + tid]);
      float Ls = 0.f;
      for (int cc = c_first; cc <= c_last; ++cc) {
        const float* pp = a.part1 + (long)(cc + u) * PART;
        Ls += exp2f(pp[tid] - M) * pp[G + tid];
      }
      lse2[tid] = M + log2f(Ls);
    }
    __syncthreads();
    // o_cmp (normalised) times its gate
    for (int x = tid; x < G * D; x += SEL_THREADS) {
      const int h = x / D;
      float acc = 0.f;
      for (int cc = c_first; cc <= c_last; ++cc) {
        const float* pp = a.part1 + (long)(cc + u) * PART;
        acc += exp2f(pp[h] - lse2[h]) * pp[2 * G + x];
      }
      oacc[x] = gate[h * 3] * acc;
    }
    // tile factors exp2(m_ref - lse)
    const float* rec = a.trec + (long)u * a.tiles_max * (G * (1 + a.nbt));
    for (int x = tid; x < tiles_u * G; x += SEL_THREADS) {
      const int tau = x / G, h = x - tau * G;
      fac[x] = exp2f(rec[(long)tau * G * (1 + a.nbt) + h * (1 + a.nbt)] - lse2[h]);
    }
    __syncthreads();
    // block scores summed over the group's heads
    for (int j = tid; j < ncand; j += SEL_THREADS) {
      const int num = j * a.bs - a.l + 1;
      const int ilo = num <= 0 ? 0 : (num + a.s - 1) / a.s;
      const int ihi = min((j * a.bs + a.bs - 1) / a.s, nvis - 1);
      float acc = 0.f;
      if (ilo <= ihi) {
        for (int tau = ilo / TK; tau <= ihi / TK; ++tau) {
          const int jl = j - (tau * TK * a.s) / a.bs;
          const float* rt = rec + (long)tau * G * (1 + a.nbt);
          for (int h = 0; h < G; ++h) acc += fac[tau * G + h] * rt[h * (1 + a.nbt) + 1 + jl];
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
    const int warp = tid >> 5, lane = tid & 31;
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
      if (tid == 0) {
        float s0 = red_s[0];
        int j0 = red_j[0];
        for (int w = 1; w < SEL_THREADS / 32; ++w)
          if (sel_better(red_s[w], red_j[w], s0, j0)) {
            s0 = red_s[w];
            j0 = red_j[w];
          }
        sel[r] = j0;
        scores[j0] = -INFINITY;
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
  if (tid == 0) a.cnt3[u] = 0u;
}

// ---------------------------------------------------------------------------
// dec_sel_win
// ---------------------------------------------------------------------------

constexpr int SW_KEYS = 128;                 // keys per item (2 sub-tiles of 64)
constexpr int SW_TILE = 2 * TILE_BYTES;      // 128 keys x 128 dims

__global__ void __launch_bounds__(128)
    dec_sel_win_kernel(const __grid_constant__ DecFastArgs a, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ks_ = smem;                  // K: [2 sub-tiles][2 halves][64][64]
  unsigned char* vs_ = smem + SW_TILE;        // V
  float* mrg = reinterpret_cast<float*>(smem + 2 * SW_TILE);
  uint64_t* bar = reinterpret_cast<uint64_t*>(mrg + MERGE_FLOATS);
  __shared__ int info[8];  // nsel, isel, iwin, wstart, blk0, blk1, is_last

  const int u = blockIdx.y, item = blockIdx.x;
  const int b = u / a.Hkv, g = u - b * a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = a.seq_lens[b];
  if (L < 1 || L > a.T) return;  // reported by dec_select
  const int t = L - 1;
  if (tid == 0) {
    int nsel = 0;
    for (int x = 0; x < a.n; ++x) nsel += a.sel[(long)u * a.n + x] >= 0;
    const int wlen = min(a.w, L);
    info[0] = nsel;
    info[1] = (nsel + 1) / 2;
    info[2] = (wlen + SW_KEYS - 1) / SW_KEYS;
    info[3] = t - wlen + 1;
    const int isel = info[1];
    if (item < isel) {
      info[4] = a.sel[(long)u * a.n + 2 * item];
      info[5] = 2 * item + 1 < nsel ? a.sel[(long)u * a.n + 2 * item + 1] : -1;
    } else {
      info[4] = info[5] = -1;
    }
    ptx::mbar_init(bar, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  const int isel = info[1], iwin = info[2];
  const bool is_sel = item < isel, is_win = !is_sel && item < isel + iwin;
  // key positions of the two 64-key sub-tiles (-1: not loaded)
  int pos0[2];
  if (is_sel) {
    pos0[0] = info[4] * a.bs;
    pos0[1] = info[5] >= 0 ? info[5] * a.bs : -1;
  } else if (is_win) {
    const int p = info[3] + (item - isel) * SW_KEYS;
    pos0[0] = p;
    pos0[1] = p + TK <= t ? p + TK : -1;
  } else {
    pos0[0] = pos0[1] = -1;
  }

  bool ok = true;
  if (is_sel || is_win) {
    if (tid == 0) {
      const uint64_t pol = ptx::policy_evict_first();
      const int nsub = pos0[1] >= 0 ? 2 : 1;
      ptx::mbar_arrive_expect_tx(bar, nsub * 2 * TILE_BYTES);
      for (int st = 0; st < nsub; ++st) {
        const int row = b * a.T + pos0[st];
        unsigned char* dk = ks_ + st * TILE_BYTES;
        unsigned char* dv = vs_ + st * TILE_BYTES;
        ptx::tma_load_3d(dk, &tk, bar, 0, g, row, pol);
        ptx::tma_load_3d(dk + HALF_BYTES, &tk, bar, 64, g, row, pol);
        ptx::tma_load_3d(dv, &tv, bar, 0, g, row, pol);
        ptx::tma_load_3d(dv + HALF_BYTES, &tv, bar, 64, g, row, pol);
      }
    }
    if (!ptx::mbar_wait(bar, 0, kWaitNs)) {
      if (lane == 0) atomicOr(a.err, kErrTimeout);
      ok = false;
    }
  }

  // each warp: 32 keys of one sub-tile
  const int st = warp >> 1, kofs = (warp & 1) * 32;
  float o[16][4];
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  if (ok && pos0[st] >= 0) {
    uint32_t qa[8][4];
    load_q_frags(qa, reinterpret_cast<const __nv_bfloat16*>(a.q) + ((long)b * a.Hq + g * G) * D,
                 lane);
    const uint32_t kb = ptx::smem_u32(ks_ + st * TILE_BYTES);
    const uint32_t vb = ptx::smem_u32(vs_ + st * TILE_BYTES);
    float s[4][4];
    qk_tile<4>(s, qa, kb, kofs, lane);
    // keys past t (last selected block, window tail) are masked
    const int nvalid = min(32, t - (pos0[st] + kofs) + 1);
    softmax_step<4>(s, o, m0, m1, l0, l1, nvalid, a.scale_log2, lane);
    pv_tile<2>(o, s, vb, kofs, lane);
  }
  write_warp_partial(mrg, warp, lane, m0, m1, l0, l1, o);
  __syncthreads();
  float* dst = a.part3 + ((long)u * a.items_max + item) * PART;
  merge_warps_to(dst, mrg, tid);
  __threadfence();
  __syncthreads();
  if (tid == 0) info[6] = atomicAdd(&a.cnt3[u], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!info[6]) return;
  __threadfence();

  // last CTA of the unit: merge the selected and window partials, apply gates
  const int h = tid >> 3, e0 = (tid & 7) * 16;
  float Ms = -INFINITY, Mw = -INFINITY;
  for (int it = 0; it < isel; ++it)
    Ms = fmaxf(Ms, __ldcg(a.part3 + ((long)u * a.items_max + it) * PART + h));
  for (int it = isel; it < isel + iwin; ++it)
    Mw = fmaxf(Mw, __ldcg(a.part3 + ((long)u * a.items_max + it) * PART + h));
  float Ls = 0.f, Lw = 0.f;
  for (int it = 0; it < isel + iwin; ++it) {
    const float* pp = a.part3 + ((long)u * a.items_max + it) * PART;
    const float mm = __ldcg(pp + h);
    if (mm == -INFINITY) continue;
    if (it < isel) Ls += exp2f(mm - Ms) * __ldcg(pp + G + h);
    else Lw += exp2f(mm - Mw) * __ldcg(pp + G + h);
  }
  const float g1 = a.gates[(long)u * 3 * G + h * 3 + 1] / Ls;
  const float g2 = a.gates[(long)u * 3 * G + h * 3 + 2] / Lw;
  __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + ((long)b * a.Hq + g * G + h) * D;
  const float* oc = a.oacc + (long)u * G * D + h * D;
  for (int e = e0; e < e0 + 16; ++e) {
    float accs = 0.f, accw = 0.f;
    for (int it = 0; it < isel + iwin; ++it) {
      const float* pp = a.part3 + ((long)u * a.items_max + it) * PART;
      const float mm = __ldcg(pp + h);
      if (mm == -INFINITY) continue;
      const float ov = __ldcg(pp + 2 * G + h * D + e);
      if (it < isel) accs += exp2f(mm - Ms) * ov;
      else accw += exp2f(mm - Mw) * ov;
    }
    orow[e] = __float2bfloat16_rn(__ldcg(oc + e) + g1 * accs + g2 * accw);
  }
  if (tid == 0) a.cnt3[u] = 0u;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  size_t part1, trec, oacc, gates, sel, part3, cnt3, total;
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
  w.part3 = off; off = align256(off + units * a.items_max * PART * 4);
  w.cnt3 = off; off = align256(off + units * 4);
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
  a.items_max = (a.n + 1) / 2 + (std::min(a.w, a.T) + SW_KEYS - 1) / SW_KEYS;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  a.grid1 = sms;
  const float scale = p.softmax_scale != 0.f ? p.softmax_scale : 1.f / sqrtf((float)p.d);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.gate_mode = p.gate_mode;
  for (int i = 0; i < 3; ++i) a.fixed_gates[i] = p.fixed_gates[i];
  return a;
}

constexpr size_t kCmpSmem = 1024 + STAGES * STAGE_BYTES + MERGE_FLOATS * 4 + 2 * STAGES * 8 +
                            sizeof(Plan) + 16;
constexpr size_t kSwSmem = 1024 + 2 * SW_TILE + MERGE_FLOATS * 4 + 16;

}  // namespace

bool decode_fast_eligible(const nsa_params& p) {
  return p.dtype == NSA_DTYPE_BF16 && p.d == D && p.Hq == G * p.Hkv && p.sel_block == 64 &&
         p.top_n <= 64 && p.cmp_block <= 64 * p.cmp_stride && p.T >= 1;
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
  a.cnt3 = reinterpret_cast<unsigned*>(w + L.cnt3);

  CUtensorMap tkc, tvc, tk, tv;
  const uint64_t rows_c = (uint64_t)p.B * (a.Nc > 0 ? a.Nc : 1);
  const uint64_t rows = (uint64_t)p.B * p.T;
  bool okm = true;
  if (a.Nc > 0) {
    okm &= make_tmap_bf16_3d(&tkc, kc, D, p.Hkv, rows_c, 64, 1, TK, true);
    okm &= make_tmap_bf16_3d(&tvc, vc, D, p.Hkv, rows_c, 64, 1, TK, true);
  }
  okm &= make_tmap_bf16_3d(&tk, k, D, p.Hkv, rows, 64, 1, TK, true);
  okm &= make_tmap_bf16_3d(&tv, v, D, p.Hkv, rows, 64, 1, TK, true);
  if (!okm) return cudaErrorInvalidValue;

  if (a.Nc > 0) {
    TraceScope trace("dec_cmp_partial", stream);
    cudaFuncSetAttribute(dec_cmp_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kCmpSmem);
    dec_cmp_partial_kernel<<<a.grid1, 160, kCmpSmem, stream>>>(a, tkc, tvc);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    const int nblk = (p.T + p.sel_block - 1) / p.sel_block;
    const size_t smem = (size_t)(32 + G + 3 * G + a.tiles_max * G + nblk + 8) * 4 + 8 * 4 +
                        (size_t)a.n * 4 + 16;
    TraceScope trace("dec_select", stream);
    cudaFuncSetAttribute(dec_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dec_select_kernel<<<p.B * p.Hkv, SEL_THREADS, smem, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    TraceScope trace("dec_sel_win", stream);
    cudaFuncSetAttribute(dec_sel_win_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)kSwSmem);
    dim3 grid(a.items_max, p.B * p.Hkv);
    dec_sel_win_kernel<<<grid, 128, kSwSmem, stream>>>(a, tk, tv);
    return cudaGetLastError();
  }
}

}  // namespace nsa
