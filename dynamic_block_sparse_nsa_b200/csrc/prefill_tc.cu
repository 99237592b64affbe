// NSA causal prefill on the sm_100a tensor cores (tcgen05 MMAs with TMEM
// accumulators, operands staged by TMA), for bf16 inputs, head dimension 128
// and 16 query heads per KV head, with compression block 32 at stride 16 and
// selection block 64 (EP94 notes section five; lchairun NSA article, the three
// branches and the gate).
//
// Two kernels:
//  pf_main  one CTA per (sequence, KV head, 8 consecutive tokens): the 128 rows
//           (token, head of the group) share every K / V tile (GQA group
//           sharing, EP94 notes section six).
//           1. compressed attention over the visible compressed blocks (online
//              softmax, P kept in TMEM as the A operand of the PV MMA);
//           2. sliding-window attention over [t - w + 1, t];
//           3. the block scores: S^T = K~ Q^T is recomputed with the final
//              log-sum-exp of step 1, so each thread holds one compressed key
//              and sums its probabilities over the 16 heads of the group in
//              registers; a selection block j collects compressed blocks
//              4j-1 .. 4j+3;
//           4. top-n per token with block 0 forced (ties to the lower index);
//           5. g_cmp * o_cmp + g_win * o_win (bf16) and g_slc to the workspace.
//  pf_slc   persistent; one unit per (sequence, token, KV head): the selected
//           blocks, two per 128-key tile, give S^T = K_sel Q^T (M = 128 keys,
//           N = 16 heads); an exact softmax over all selected keys per head;
//           O^T = V_sel^T P^T; out = acc + g_slc * o_slc in bf16.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace nsa {
namespace {

constexpr int G = 16;             // query heads per KV head
constexpr int D = 128;            // head dimension
constexpr int TQ = 8;             // tokens per pf_main tile (TQ * G = 128 rows)
constexpr int KT = 128;           // keys per tile
constexpr int CL = 32, CS = 16;   // compression block and stride
constexpr int SB = 64;            // selection block
constexpr uint32_t ATOM = 16384;  // one d-half of a 128-row bf16 tile
constexpr uint32_t TILE = 32768;  // a 128 x 128 bf16 tile
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kMaxSel = 16;       // top_n bound: 8 tiles of two blocks in pf_slc
constexpr int kMainStagesMax = 4;
constexpr int kMainThreads = 320; // TMA, MMA, 8 softmax warps
constexpr int kSlcThreads = 256;  // K/V TMA, Q/acc loads, MMA, TMEM owner, 4 softmax warps
constexpr int kSlcStages = 5;     // one ring of K and V tiles, in the order the MMAs use them
constexpr uint32_t kQ16 = 4096;   // 16 rows x 128 d bf16
constexpr uint32_t kNegInf = 0xff800000u;  // bits of -inf

struct PfArgs {
  const float* w_gate;
  __nv_bfloat16* acc;  // [B, T, Hq, d]: g_cmp * o_cmp + g_win * o_win
  float* gslc;   // [B, T, Hq]
  int32_t* sel;  // [B, T, Hkv, n]
  __nv_bfloat16* out;
  unsigned* err;
  int B, T, Hq, Hkv, Nc, n, w, nblk, stages;
  float c;       // softmax scale * log2(e)
  int gate_mode;
  float fixed_gates[3];
  // Branches a fixed zero gate removes (the output is unchanged without them):
  int run_cmp;     // compressed attention (pass 1), needed for its output or the selection
  int need_sel;    // block scores and top-n (pass 3, step 4)
  int run_win;     // window attention (pass 2)
  int direct_out;  // no selected branch: pf_main writes the bf16 output itself
  float top_p;     // 0: top-n; else adaptive selection
};

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
  return (unsigned char*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

// Bounded wait that records a timeout and switches the CTA to abort mode
// (every later wait returns at once, loops run out with their fixed bounds).
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort,
                                              unsigned* err) {
  if (*abort) return false;
  if (ptx::mbar_wait(bar, parity, kWaitNs)) return true;
  *abort = 1;
  atomicOr(err, kErrTimeout);
  return false;
}

// K-major SW128 operand of a 128-row (or 16-row) tile, MMA step ks of 8.
__device__ __forceinline__ uint64_t kmaj(uint32_t base, int ks, uint32_t half_bytes) {
  return tc::sdesc(base + (ks >> 2) * half_bytes + (ks & 3) * 32, 16, 1024, tc::kSw128);
}

// MN-major SW128 operand of a [128 keys][128 d] tile (d contiguous), step ks.
__device__ __forceinline__ uint64_t mnmaj(uint32_t base, int ks) {
  return tc::sdesc(base + ks * 2048, ATOM, 1024, tc::kSw128);
}

__device__ __forceinline__ float sigmoidf(float x) { return 1.f / (1.f + __expf(-x)); }

// The three gates of query row `row` of a K-major SW128 Q tile (two d-halves
// of `half_bytes` each): sigmoid(q . Wg[:, k]) or the fixed gates.
__device__ __forceinline__ void row_gates(const PfArgs& a, const unsigned char* q,
                                          const float* wg, int row, uint32_t half_bytes,
                                          float (&gt)[3]) {
  if (a.gate_mode != 0) {
    gt[0] = a.fixed_gates[0];
    gt[1] = a.fixed_gates[1];
    gt[2] = a.fixed_gates[2];
    return;
  }
  float z0 = 0.f, z1 = 0.f, z2 = 0.f;
#pragma unroll 1
  for (int ch = 0; ch < 16; ++ch) {  // runs once per row: kept compact
    const int hf = ch >> 3, c8 = ch & 7;
    const uint4 v = *reinterpret_cast<const uint4*>(q + hf * half_bytes + row * 128 +
                                                    ((c8 ^ (row & 7)) << 4));
    const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&v);
    // Wg rows ch*8 .. ch*8+7: 24 floats, six 16-byte loads
    float w[24];
#pragma unroll
    for (int i = 0; i < 6; ++i) {
      const float4 w4 = reinterpret_cast<const float4*>(wg + ch * 24)[i];
      w[4 * i] = w4.x;
      w[4 * i + 1] = w4.y;
      w[4 * i + 2] = w4.z;
      w[4 * i + 3] = w4.w;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(e[k]);
      z0 += f.x * w[6 * k + 0] + f.y * w[6 * k + 3];
      z1 += f.x * w[6 * k + 1] + f.y * w[6 * k + 4];
      z2 += f.x * w[6 * k + 2] + f.y * w[6 * k + 5];
    }
  }
  gt[0] = sigmoidf(z0);
  gt[1] = sigmoidf(z1);
  gt[2] = sigmoidf(z2);
}

// ============================================================================
// pf_main
// ============================================================================

struct MainBars {
  uint64_t full[kMainStagesMax], empty[kMainStagesMax];
  uint64_t q_full, s_full[2], p_full[2], o_done[2], fin;
  uint32_t tmem;
  int abort;
  float xm[2][2][128];  // per tile parity, column half, row: partial row maxima
  float xl[2][2][128];  // per branch, column half, row: partial row sums
};

// TMEM columns of pf_main.
constexpr uint32_t kO1 = 0, kO2 = 128, kS0 = 256;  // S buffers at 256 and 384

// Exact top-k of the candidate blocks 1 .. ncand - 1 of one token (k < ncand
// - 1), by one warp: higher score first, the lower index among equal scores.
// Each candidate has the unique key (score bits + 1) << 32 | ~index (scores are
// sums of probabilities, >= 0; a larger key is a better block). Every lane
// keeps the four largest keys of its candidates (index = 1 + lane mod 32) in
// registers; each pick is the warp maximum of the lanes' best keys, popped
// from its lane, which rescans its candidates below the last popped key only
// once it has given up all four. dst gets block 0, then the picks in
// increasing order.
__device__ void warp_topk_lists(const float* scx, int ncand, int k, int32_t* dst, int lane) {
  auto key = [&](int jb) -> unsigned long long {
    const float v = scx[jb];
    const uint32_t kh = v < 0.f ? 0u : __float_as_uint(v) + 1u;
    return ((unsigned long long)kh << 32) | (uint32_t)~(uint32_t)jb;
  };
  unsigned long long t0 = 0, t1 = 0, t2 = 0, t3 = 0;  // 0: empty (no key is 0)
  auto fill = [&](unsigned long long below) {
    t0 = t1 = t2 = t3 = 0;
    for (int jb = 1 + lane; jb < ncand; jb += 32) {
      const unsigned long long x = key(jb);
      if (x >= below || x <= t3) continue;
      const bool g0 = x > t0, g1 = x > t1, g2 = x > t2;
      t3 = g2 ? t2 : x;
      t2 = g2 ? (g1 ? t1 : x) : t2;
      t1 = g1 ? (g0 ? t0 : x) : t1;
      t0 = g0 ? x : t0;
    }
  };
  fill(~0ull);
  int mine = lane == 0 ? 0 : 0x7fffffff;
  for (int i = 0; i < k; ++i) {
    const uint32_t hi = (uint32_t)(t0 >> 32), lo = (uint32_t)t0;
    const uint32_t mh = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t ml = __reduce_max_sync(0xffffffffu, hi == mh ? lo : 0u);
    if (lane == i + 1) mine = (int)~ml;
    if (hi == mh && lo == ml) {  // this lane's best was taken
      const unsigned long long last = t0;
      t0 = t1;
      t1 = t2;
      t2 = t3;
      t3 = 0;
      if (t0 == 0) fill(last);
    }
  }
  int rank = 0;
  for (int o = 0; o < 32; ++o) rank += (__shfl_sync(0xffffffffu, mine, o) < mine) ? 1 : 0;
  if (lane <= k) dst[rank] = mine;
}

__global__ void __launch_bounds__(kMainThreads, 1)
    pf_main_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tkc,
                   const __grid_constant__ CUtensorMap tvc, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const PfArgs a) {
  extern __shared__ unsigned char smraw[];
  unsigned char* base = align1024(smraw);
  unsigned char* sQ = base;
  unsigned char* ring = base + TILE;
  float* sc = reinterpret_cast<float*>(ring + a.stages * TILE);  // [TQ][nblk]
  float* slse = sc + TQ * a.nblk;                                  // [128]
  float* spk = slse + 128;                                          // [TQ][128]
  float* scarry = spk + TQ * KT;                                    // [TQ] (+ pad)
  float* swg = scarry + 16;                                         // [D][3]
  MainBars* bars = reinterpret_cast<MainBars*>(swg + D * 3);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.stages;
  const int ntq = (a.T + TQ - 1) / TQ;
  const int BH = a.B * a.Hkv;
  const int bg = blockIdx.x % BH;
  const int r = ntq - 1 - (int)(blockIdx.x / BH);  // longest tiles first
  const int b = bg / a.Hkv, g = bg % a.Hkv;
  const int t0 = r * TQ;
  const int tlast = min(t0 + TQ - 1, a.T - 1);
  const int nvis = tlast >= CL - 1 ? min(a.Nc, (tlast - (CL - 1)) / CS + 1) : 0;
  const int J1 = a.run_cmp ? (nvis + KT - 1) / KT : 0;  // compressed tiles (passes 1 and 3)
  const int ks0 = max(0, t0 - a.w + 1);
  const int J2 = a.run_win ? (tlast - ks0 + KT) / KT : 0;  // window tiles
  const int J3 = a.need_sel ? J1 : 0;                       // score tiles
  const int A = J1 + J2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      ptx::mbar_init(&bars->full[i], 1);
      ptx::mbar_init(&bars->empty[i], 1);
    }
    ptx::mbar_init(&bars->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->s_full[i], 1);
      ptx::mbar_init(&bars->p_full[i], 256);  // the eight softmax warps
      ptx::mbar_init(&bars->o_done[i], 1);
    }
    ptx::mbar_init(&bars->fin, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem;

  if (warp == 0) {
    // ---------------- TMA producers: lane L < S issues loads c = L (mod S) ----------------
    // (one issuing thread keeps only a few bulk copies moving; S threads in
    // parallel reach the SM's ingest rate)
    if (lane < S) {
      if (lane == 0) {
        ptx::prefetch_tmap(&tq);
        ptx::prefetch_tmap(&tkc);
        ptx::prefetch_tmap(&tvc);
        ptx::prefetch_tmap(&tk);
        ptx::prefetch_tmap(&tv);
      }
      const uint64_t keep = ptx::policy_evict_last(), once = ptx::policy_evict_first();
      if (lane == 0) {
        const int qrow = b * a.T + t0;
        ptx::mbar_arrive_expect_tx(&bars->q_full, TILE);
        ptx::tma_load_3d(sQ, &tq, &bars->q_full, 0, g * G, qrow, once);
        ptx::tma_load_3d(sQ + ATOM, &tq, &bars->q_full, 64, g * G, qrow, once);
      }
      int c = 0, mine = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* m, int z) {
        const int cc = c++;
        if (!ok || cc % S != lane) return;
        const int st = lane;
        if (cc >= S && !wait_or_abort(&bars->empty[st], (uint32_t)(((cc / S) - 1) & 1), abort,
                                      a.err)) {
          ok = false;
          return;
        }
        unsigned char* dst = ring + st * TILE;
        ptx::mbar_arrive_expect_tx(&bars->full[st], TILE);
        ptx::tma_load_3d(dst, m, &bars->full[st], 0, g, z, keep);
        ptx::tma_load_3d(dst + ATOM, m, &bars->full[st], 64, g, z, keep);
        ++mine;
      };
      auto k_of = [&](int i) {
        if (i < J1) load(&tkc, b * a.Nc + i * KT);
        else load(&tk, b * a.T + ks0 + (i - J1) * KT);
      };
      auto v_of = [&](int i) {
        if (i < J1) load(&tvc, b * a.Nc + i * KT);
        else load(&tv, b * a.T + ks0 + (i - J1) * KT);
      };
      for (int i = 0; i < A; ++i) {
        k_of(i);
        if (i >= 1) v_of(i - 1);
      }
      if (A >= 1) v_of(A - 1);
      for (int i = 0; i < J3; ++i) load(&tkc, b * a.Nc + i * KT);
      // this lane's last load must land before the CTA exits (earlier ones on
      // the same stage completed before their stage was reused)
      if (mine > 0) {
        const int last = lane + (mine - 1) * S;
        if (!ptx::mbar_wait(&bars->full[lane], (uint32_t)((last / S) & 1), kWaitNs))
          atomicOr(a.err, kErrTimeout);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t iss = tc::idesc_bf16(128, 128, false, false);
      const uint32_t its = tc::idesc_bf16(128, 128, false, true);
      const uint32_t q0 = ptx::smem_u32(sQ), r0 = ptx::smem_u32(ring);
      bool ok = wait_or_abort(&bars->q_full, 0, abort, a.err);
      tc::fence_after_sync();
      int c = 0;
      auto take = [&]() -> int {
        const int st = c % S;
        if (ok) ok = wait_or_abort(&bars->full[st], (uint32_t)((c / S) & 1), abort, a.err);
        tc::fence_after_sync();
        return st;
      };
      for (int i = 0; ok && i <= A; ++i) {
        if (i < A) {
          const int bs = i & 1;
          if (i >= 2) ok = ok && wait_or_abort(&bars->p_full[bs], (uint32_t)(((i - 2) >> 1) & 1),
                                               abort, a.err);
          const int st = take();
          if (!ok) break;
          const uint32_t kb = r0 + st * TILE;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::mma_ss(tmem + kS0 + bs * 128, kmaj(q0, ks, ATOM), kmaj(kb, ks, ATOM), iss, ks > 0);
          tc::commit(&bars->empty[st]);
          tc::commit(&bars->s_full[bs]);
          ++c;
        }
        if (i >= 1) {
          const int pj = i - 1, pb = pj & 1;
          ok = ok && wait_or_abort(&bars->p_full[pb], (uint32_t)((pj >> 1) & 1), abort, a.err);
          tc::fence_after_sync();
          const int st = take();
          if (!ok) break;
          const uint32_t vb = r0 + st * TILE;
          const uint32_t od = tmem + (pj < J1 ? kO1 : kO2);
          const bool first = (pj == 0 || pj == J1);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::mma_ts(od, tmem + kS0 + pb * 128 + ks * 8, mnmaj(vb, ks), its, (!first || ks > 0));
          tc::commit(&bars->empty[st]);
          tc::commit(&bars->o_done[pj & 1]);
          ++c;
        }
      }
      for (int jj = 0; ok && jj < J3; ++jj) {
        const int j = A + jj, bs = j & 1;
        if (j >= 2) ok = wait_or_abort(&bars->p_full[bs], (uint32_t)(((j - 2) >> 1) & 1), abort,
                                       a.err);
        const int st = take();
        if (!ok) break;
        const uint32_t kb = r0 + st * TILE;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc::mma_ss(tmem + kS0 + bs * 128, kmaj(kb, ks, ATOM), kmaj(q0, ks, ATOM), iss, ks > 0);
        tc::commit(&bars->empty[st]);
        tc::commit(&bars->s_full[bs]);
        ++c;
      }
      tc::commit(&bars->fin);
      if (!ptx::mbar_wait(&bars->fin, 0, kWaitNs)) atomicOr(a.err, kErrTimeout);
    }
  } else {
    // ---------------- softmax / scores / selection / epilogue ----------------
    // Eight warps: two per TMEM lane quarter, splitting each row's 128 columns
    // (keys in steps 1-2, query rows in step 3) into halves.
    const int sw = warp - 2;           // 0..7
    const int half = sw >> 2;          // column half
    const int qd = warp & 3;
    const int row = qd * 32 + lane;    // TMEM lane: query row in steps 1-2, key in step 3
    const int sid = half * 128 + row;  // 0..255 among the softmax threads
    const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
    const uint32_t hc = half * 64;     // this thread's first column of a 128-column tile
    const int tt = row >> 4, h = row & 15;
    const int t = min(t0 + tt, a.T - 1);
    const bool row_ok = t0 + tt < a.T;
    const int nv_t = t >= CL - 1 ? min(a.Nc, (t - (CL - 1)) / CS + 1) : 0;
    const int wlo = max(0, t - a.w + 1);
    for (int i = sid; i < TQ * a.nblk; i += 256) sc[i] = 0.f;
    if (sid < TQ) scarry[sid] = 0.f;
    if (a.gate_mode == 0)
      for (int i = sid; i < D * 3; i += 256) swg[i] = __ldg(a.w_gate + i);

    float m1 = -INFINITY, l1 = 0.f, m2 = -INFINITY, l2 = 0.f;  // l: this half's sum
    for (int j = 0; j < A; ++j) {
      const int bs = j & 1;
      wait_or_abort(&bars->s_full[bs], (uint32_t)((j >> 1) & 1), abort, a.err);
      tc::fence_after_sync();
      const bool cmp = j < J1;
      const int kb = (cmp ? j * KT : ks0 + (j - J1) * KT) + (int)hc;
      const int lo = cmp ? 0 : wlo, hi = cmp ? nv_t - 1 : t;
      uint32_t u[64];
      tc::ld64_sync(tl + kS0 + bs * 128 + hc, u);
      if (kb < lo || kb + 63 > hi) {  // these columns straddle the row's key range
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const int key = kb + e;
          if (key < lo || key > hi) u[e] = kNegInf;
        }
      }
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int e = 0; e < 64; e += 4) {
        mx0 = fmaxf(mx0, __uint_as_float(u[e]));
        mx1 = fmaxf(mx1, __uint_as_float(u[e + 1]));
        mx2 = fmaxf(mx2, __uint_as_float(u[e + 2]));
        mx3 = fmaxf(mx3, __uint_as_float(u[e + 3]));
      }
      // the row maximum over both halves (exchange buffers alternate by tile)
      bars->xm[bs][half][row] = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
      ptx::named_bar_sync(1, 256);
      const float mt = fmaxf(bars->xm[bs][0][row], bars->xm[bs][1][row]) * a.c;
      float& m = cmp ? m1 : m2;
      float& l = cmp ? l1 : l2;
      const float mn = fmaxf(m, mt);
      if (mn != -INFINITY && (m == -INFINITY || mn > m + 8.f)) {
        if (m != -INFINITY) {
          // rescale this half of the row of O once the previous PV MMA finished
          const float f = exp2f(m - mn);
          l *= f;
          wait_or_abort(&bars->o_done[(j - 1) & 1], (uint32_t)(((j - 1) >> 1) & 1), abort, a.err);
          tc::fence_after_sync();
          const uint32_t oc = tl + (cmp ? kO1 : kO2) + hc;
#pragma unroll 1
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w[16];
            tc::ld16_sync(oc + q4 * 16, w);
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * f);
            tc::st16(oc + q4 * 16, w);
          }
          tc::st_wait();
        }
        m = mn;
      }
      // p = 2^(s c - m); masked keys (-inf) give 0; a row without any valid key
      // so far keeps m = -inf and gets p = 0 through a zero offset
      const float nm = m == -INFINITY ? 0.f : -m;
      float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 2; ++q4) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ptx::ex2(fmaf(__uint_as_float(u[q4 * 32 + 2 * e]), a.c, nm));
          const float p1 = ptx::ex2(fmaf(__uint_as_float(u[q4 * 32 + 2 * e + 1]), a.c, nm));
          ls0 += p0;
          ls1 += p1;
          pk[e] = ptx::pack_bf16(p0, p1);
        }
        tc::st16(tl + kS0 + bs * 128 + half * 32 + q4 * 16, pk);
      }
      l += ls0 + ls1;
      tc::st_wait();
      tc::fence_before_sync();
      ptx::mbar_arrive(&bars->p_full[bs]);
    }
    // row sums over both halves
    bars->xl[0][half][row] = l1;
    bars->xl[1][half][row] = l2;
    ptx::named_bar_sync(1, 256);
    l1 = bars->xl[0][0][row] + bars->xl[0][1][row];
    l2 = bars->xl[1][0][row] + bars->xl[1][1][row];

    // log-sum-exp (log2 domain) of the compressed branch for step 3
    if (half == 0) slse[row] = l1 > 0.f ? -(m1 + __log2f(l1)) : -INFINITY;  // negated, for fma
    ptx::named_bar_sync(1, 256);

    // step 3: block scores; thread = compressed key `row` of each tile, tokens
    // 4 half .. 4 half + 3
    for (int jj = 0; jj < J3; ++jj) {
      const int j = A + jj, bs = j & 1;
      wait_or_abort(&bars->s_full[bs], (uint32_t)((j >> 1) & 1), abort, a.err);
      tc::fence_after_sync();
      uint32_t u[64];
      tc::ld64_sync(tl + kS0 + bs * 128 + hc, u);
      tc::fence_before_sync();
      ptx::mbar_arrive(&bars->p_full[bs]);
      const int kk = jj * KT + row;
#pragma unroll
      for (int xx = 0; xx < TQ / 2; ++xx) {
        const int x = half * (TQ / 2) + xx, tok = t0 + x;
        float acc0 = 0.f, acc1 = 0.f;
        if (tok < a.T && kk < a.Nc && kk * CS + CL - 1 <= tok) {
          const float4* nl = reinterpret_cast<const float4*>(slse + x * G);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 l4 = nl[q];
            acc0 += ptx::ex2(fmaf(__uint_as_float(u[xx * G + 4 * q]), a.c, l4.x));
            acc1 += ptx::ex2(fmaf(__uint_as_float(u[xx * G + 4 * q + 1]), a.c, l4.y));
            acc0 += ptx::ex2(fmaf(__uint_as_float(u[xx * G + 4 * q + 2]), a.c, l4.z));
            acc1 += ptx::ex2(fmaf(__uint_as_float(u[xx * G + 4 * q + 3]), a.c, l4.w));
          }
        }
        spk[x * KT + row] = acc0 + acc1;
      }
      // selection block q of this tile collects compressed keys 4q-1 .. 4q+3
      // (key 4q-1 of block 0 comes from the previous tile)
      ptx::named_bar_sync(1, 256);
      {
        const int x = sid >> 5, q = sid & 31;
        const float* px = spk + x * KT;
        const float nc = q == 31 ? px[KT - 1] : 0.f;
        const int jb = jj * (KT / 4) + q;
        const float prev = q > 0 ? px[4 * q - 1] : scarry[x];
        const float v = prev + px[4 * q] + px[4 * q + 1] + px[4 * q + 2] + px[4 * q + 3];
        if (jb < a.nblk) sc[x * a.nblk + jb] = v;
        ptx::named_bar_sync(1, 256);
        if (q == 31) {
          scarry[x] = nc;
          // the block after the last tile holds only the carried key
          if (jj == J1 - 1 && J1 * (KT / 4) < a.nblk) sc[x * a.nblk + J1 * (KT / 4)] = nc;
        }
      }
    }
    ptx::named_bar_sync(1, 256);

    // step 4: top-n of token `sw`, one warp per token. A candidate's key is
    // (score bits + 1, ~index): unique, ordered by score and then by the lower
    // index; a taken block gets key 0.
    if (a.need_sel) {
      const int x = sw, tok = t0 + x;
      if (tok < a.T) {  // warp-uniform
        const int ncand = tok / SB + 1;
        int32_t* dst = a.sel + ((size_t)(b * a.T + tok) * a.Hkv + g) * a.n;
        if (a.top_p > 0.f) {
          // adaptive: block 0, then the best others until their scores reach
          // top_p of the total over all candidates (fp64 sums), at most n
          float* scx = sc + x * a.nblk;
          double part = 0.0;
          for (int jb = lane; jb < ncand; jb += 32) part += (double)scx[jb];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
          const double goal = (double)a.top_p * part;
          double cum = (double)scx[0];
          uint32_t bh = 0, bl = 0;
          auto rescan = [&]() {
            uint32_t hh = 0, ll = 0;
            for (int jb = 1 + lane; jb < ncand; jb += 32) {
              const float vv = scx[jb];
              const uint32_t kh = vv < 0.f ? 0u : __float_as_uint(vv) + 1u;
              const uint32_t kl = ~(uint32_t)jb;
              if (kh > hh || (kh == hh && kl > ll)) {
                hh = kh;
                ll = kl;
              }
            }
            bh = hh;
            bl = ll;
          };
          rescan();
          int mine = lane == 0 ? 0 : 0x7fffffff;
          int cnt = 1;
          while (cnt < a.n && cnt < ncand && cum < goal) {  // warp-uniform
            const uint32_t mh = __reduce_max_sync(0xffffffffu, bh);
            const uint32_t ml = __reduce_max_sync(0xffffffffu, bh == mh ? bl : 0u);
            const int pick = (int)~ml;
            cum += (double)__uint_as_float(mh - 1u);
            if (lane == cnt) mine = pick;
            ++cnt;
            if (((pick - 1) & 31) == lane) {
              scx[pick] = -1.f;
              rescan();
            }
          }
          int rank = 0;
          for (int o = 0; o < 32; ++o) rank += (__shfl_sync(0xffffffffu, mine, o) < mine) ? 1 : 0;
          if (lane < cnt) dst[rank] = mine;
          for (int i = cnt + lane; i < a.n; i += 32) dst[i] = -1;
        } else if (ncand <= a.n) {
          for (int i = lane; i < a.n; i += 32) dst[i] = i < ncand ? i : -1;
        } else {
          warp_topk_lists(sc + x * a.nblk, ncand, a.n - 1, dst, lane);
        }
      }
    }

    // step 5: gated compressed + window outputs (this half's 64 columns), g_slc
    if (A >= 1)
      wait_or_abort(&bars->o_done[(A - 1) & 1], (uint32_t)(((A - 1) >> 1) & 1), abort, a.err);
    tc::fence_after_sync();
    float gt[3];
    row_gates(a, sQ, swg, row, ATOM, gt);
    const float i1 = l1 > 0.f ? gt[0] / l1 : 0.f;
    const float i2 = l2 > 0.f ? gt[2] / l2 : 0.f;
    const size_t orow = ((size_t)(b * a.T + t) * a.Hq + g * G + h) * D + hc;
    // An accumulator a branch never wrote (no visible key, or the branch
    // skipped) has l = 0, so i = 0 keeps its unwritten columns out.
#pragma unroll 1
    for (int c16 = 0; c16 < 4; ++c16) {  // runs once per row: kept compact
      uint32_t u1[16], u2[16];
      tc::ld16_sync(tl + kO1 + hc + c16 * 16, u1);
      tc::ld16_sync(tl + kO2 + hc + c16 * 16, u2);
      float o[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        o[e] = (i1 != 0.f ? __uint_as_float(u1[e]) * i1 : 0.f) +
               (i2 != 0.f ? __uint_as_float(u2[e]) * i2 : 0.f);
      if (row_ok) {
        if (a.direct_out) {
          uint4 pk[2];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int e = 0; e < 8; ++e) pw[e] = ptx::pack_bf16(o[2 * e], o[2 * e + 1]);
          uint4* dst = reinterpret_cast<uint4*>(a.out + orow + c16 * 16);
          dst[0] = pk[0];
          dst[1] = pk[1];
        } else {
          uint4 pk[2];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int e = 0; e < 8; ++e) pw[e] = ptx::pack_bf16(o[2 * e], o[2 * e + 1]);
          uint4* dst = reinterpret_cast<uint4*>(a.acc + orow + c16 * 16);
          dst[0] = pk[0];
          dst[1] = pk[1];
        }
      }
    }
    if (row_ok && !a.direct_out && half == 0)
      a.gslc[(size_t)(b * a.T + t) * a.Hq + g * G + h] = gt[1];
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ============================================================================
// pf_slc
// ============================================================================

struct SlcBars {
  uint64_t full[kSlcStages], empty[kSlcStages];
  uint64_t q_full[2], q_empty[2], s_full[2], p_full[2], o_full[2], o_free[2], fin;
  uint64_t a_full[2], a_empty[2];
  uint32_t tmem;
  int abort;
  alignas(16) float red[2][4][G];
};

constexpr uint32_t kAccBytes = G * D * 2;  // one unit's acc rows (bf16)
constexpr uint32_t kAccSlot = kAccBytes + 256;  // + its 16 gates

// TMEM columns of pf_slc: S^T of unit parity p at 128 p (8 tiles x 16 heads),
// O^T at 256 + 16 p.
constexpr uint32_t kSlcO = 256;

// Reduces v[16] (one value per head) over the 32 lanes of a warp with 16
// shuffles: each step exchanges the half of the values the partner keeps, so
// lane L ends with the reduction of head L / 2.
template <bool MAX>
__device__ __forceinline__ float xreduce16(const float (&v)[G], int lane) {
  auto op = [](float x, float y) { return MAX ? fmaxf(x, y) : x + y; };
  float w8[8], w4[4], w2[2];
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float send = b4 ? v[j] : v[j + 8];
    w8[j] = op(b4 ? v[j + 8] : v[j], __shfl_xor_sync(0xffffffffu, send, 16));
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float send = b3 ? w8[j] : w8[j + 4];
    w4[j] = op(b3 ? w8[j + 4] : w8[j], __shfl_xor_sync(0xffffffffu, send, 8));
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float send = b2 ? w4[j] : w4[j + 2];
    w2[j] = op(b2 ? w4[j + 2] : w4[j], __shfl_xor_sync(0xffffffffu, send, 4));
  }
  const float w1 = op(b1 ? w2[1] : w2[0], __shfl_xor_sync(0xffffffffu, b1 ? w2[0] : w2[1], 2));
  return op(w1, __shfl_xor_sync(0xffffffffu, w1, 1));
}

// A unit's selection row packed two block indices per word (0xffff = unused
// slot; blocks stay below 65535 for the supported T). Loaded one unit ahead so
// the latency of the global reads overlaps the current unit's work.
struct SelRow {
  uint32_t w[kMaxSel / 2];
  __device__ __forceinline__ void load(const int32_t* sl, int n) {
#pragma unroll
    for (int i = 0; i < kMaxSel / 2; ++i) {
      const int s0 = 2 * i < n ? __ldg(sl + 2 * i) : -1;
      const int s1 = 2 * i + 1 < n ? __ldg(sl + 2 * i + 1) : -1;
      w[i] = ((uint32_t)s0 & 0xffffu) | (((uint32_t)s1 & 0xffffu) << 16);
    }
  }
  __device__ __forceinline__ int blk(int i) const {  // -1 when unused
    const uint32_t x = (w[i >> 1] >> (16 * (i & 1))) & 0xffffu;
    return x == 0xffffu ? -1 : (int)x;
  }
  __device__ __forceinline__ int count() const {
    int c = 0;
#pragma unroll
    for (int i = 0; i < kMaxSel; ++i) c += blk(i) >= 0 ? 1 : 0;
    return c;
  }
};

__global__ void __launch_bounds__(kSlcThreads, 1)
    pf_slc_kernel(const __grid_constant__ CUtensorMap tq16, const __grid_constant__ CUtensorMap tk64,
                  const __grid_constant__ CUtensorMap tv64, const PfArgs a) {
  extern __shared__ unsigned char smraw[];
  unsigned char* base = align1024(smraw);
  unsigned char* ring = base;                                // kSlcStages x 32 KB
  unsigned char* sP = ring + kSlcStages * TILE;              // 32 KB: [1024 keys][16] SW32
  unsigned char* sQ = sP + 32768;                            // 2 x 4 KB
  unsigned char* sA = sQ + 2 * kQ16;                         // 2 x (acc 4 KB + gates)
  SlcBars* bars = reinterpret_cast<SlcBars*>(sA + 2 * kAccSlot);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long BT = (long long)a.B * a.T;
  const long long U = BT * a.Hkv;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlcStages; ++i) {
      ptx::mbar_init(&bars->full[i], 4);  // one arrival per issuing lane
      ptx::mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->q_full[i], 1);
      ptx::mbar_init(&bars->q_empty[i], 1);
      ptx::mbar_init(&bars->s_full[i], 1);
      ptx::mbar_init(&bars->p_full[i], 128);
      ptx::mbar_init(&bars->o_full[i], 1);
      ptx::mbar_init(&bars->o_free[i], 128);
      ptx::mbar_init(&bars->a_full[i], 1);
      ptx::mbar_init(&bars->a_empty[i], 128);
    }
    ptx::mbar_init(&bars->fin, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 3) {
    tc::tmem_alloc(&bars->tmem, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem;

  // unit u -> (g, b, t): group-major so that concurrent CTAs share one group's K/V in L2
  auto unit_of = [&](long long u, int& b, int& t, int& g) {
    g = (int)(u / BT);
    const long long bt = u % BT;
    b = (int)(bt / a.T);
    t = (int)(bt % a.T);
  };

  if (warp == 0) {
    // ---------------- TMA producer of the K / V ring ----------------
    // One ring in the order the MMA warp consumes it: the K tiles of unit k,
    // then the V tiles of unit k - 1 (whose softmax runs meanwhile), so no
    // slot waits for the other operand's stream. Lane L < 4 issues box L of
    // every tile (selected block L / 2, d-half L % 2): four issuing threads
    // keep enough bulk copies moving to reach the SM's ingest rate. A tile's
    // full barrier takes one arrival per lane.
    if (lane < 4) {
      if (lane == 0) {
        ptx::prefetch_tmap(&tk64);
        ptx::prefetch_tmap(&tv64);
      }
      const uint64_t keep = ptx::policy_evict_last();
      const int hb = lane >> 1, dh = lane & 1;
      int c = 0;
      bool ok = true;
      SelRow cur, prv, nxt;
      int pb = 0, pt = 0, pg = 0;  // unit k - 1
      auto row_of = [&](long long uu) {
        int b, t, g;
        unit_of(uu, b, t, g);
        return a.sel + ((size_t)(b * a.T + t) * a.Hkv + g) * a.n;
      };
      // the tiles of one unit's K or V, two selected blocks per tile (a
      // missing second block reads past the tensor: zero fill)
      auto tiles = [&](const CUtensorMap* m, const SelRow& sr, int b, int g) {
        const int nsel = sr.count();
        for (int i = 0; ok && i < (nsel + 1) / 2; ++i) {
          const int st = c % kSlcStages;
          if (c >= kSlcStages &&
              !wait_or_abort(&bars->empty[st], (uint32_t)(((c / kSlcStages) - 1) & 1), abort,
                             a.err)) {
            ok = false;
            break;
          }
          unsigned char* dst = ring + st * TILE + dh * ATOM + hb * (ATOM / 2);
          const int z = (2 * i + hb < nsel) ? b * a.T + SB * sr.blk(2 * i + hb) : (int)BT;
          ptx::mbar_arrive_expect_tx(&bars->full[st], ATOM / 2);
          ptx::tma_load_3d(dst, m, &bars->full[st], dh * 64, g, z, keep);
          ++c;
        }
      };
      if (blockIdx.x < U) cur.load(row_of(blockIdx.x), a.n);
      long long u = blockIdx.x;
      for (int k = 0; ok && u < U; u += gridDim.x, ++k) {
        int b, t, g;
        unit_of(u, b, t, g);
        if (u + gridDim.x < U) nxt.load(row_of(u + gridDim.x), a.n);
        tiles(&tk64, cur, b, g);
        if (k >= 1) tiles(&tv64, prv, pb, pg);
        prv = cur;
        pb = b;
        pt = t;
        pg = g;
        cur = nxt;
      }
      if (ok && u != (long long)blockIdx.x) tiles(&tv64, prv, pb, pg);
      (void)pt;
      for (int kq = max(0, c - kSlcStages); kq < c; ++kq)
        if (!ptx::mbar_wait(&bars->full[kq % kSlcStages], (uint32_t)((kq / kSlcStages) & 1),
                            kWaitNs))
          atomicOr(a.err, kErrTimeout);
    }
  } else if (warp == 1) {
    // ---------------- Q rows, acc rows and g_slc of each unit ----------------
    if (lane == 0) {
      ptx::prefetch_tmap(&tq16);
      const uint64_t once = ptx::policy_evict_first();
      int k = 0;
      bool ok = true;
      for (long long u = blockIdx.x; u < U; u += gridDim.x, ++k) {
        int b, t, g;
        unit_of(u, b, t, g);
        const int qs = k & 1;
        if (k >= 2 && !wait_or_abort(&bars->q_empty[qs], (uint32_t)(((k >> 1) - 1) & 1), abort,
                                     a.err)) {
          ok = false;
          break;
        }
        unsigned char* qd = sQ + qs * kQ16;
        ptx::mbar_arrive_expect_tx(&bars->q_full[qs], kQ16);
        ptx::tma_load_3d(qd, &tq16, &bars->q_full[qs], 0, g * G, b * a.T + t, once);
        ptx::tma_load_3d(qd + kQ16 / 2, &tq16, &bars->q_full[qs], 64, g * G, b * a.T + t, once);
        // the unit's acc rows and g_slc, for the epilogue
        if (k >= 2 && !wait_or_abort(&bars->a_empty[qs], (uint32_t)(((k >> 1) - 1) & 1), abort,
                                     a.err)) {
          ok = false;
          break;
        }
        const size_t row0 = (size_t)(b * a.T + t) * a.Hq + g * G;
        unsigned char* ad = sA + qs * kAccSlot;
        ptx::mbar_arrive_expect_tx(&bars->a_full[qs], kAccBytes + G * 4);
        ptx::bulk_load(ad, a.acc + row0 * D, kAccBytes, &bars->a_full[qs]);
        ptx::bulk_load(ad + kAccBytes, a.gslc + row0, G * 4, &bars->a_full[qs]);
      }
      (void)ok;
      for (int kq = max(0, k - 2); kq < k; ++kq) {
        if (!ptx::mbar_wait(&bars->q_full[kq & 1], (uint32_t)((kq >> 1) & 1), kWaitNs))
          atomicOr(a.err, kErrTimeout);
        if (!ptx::mbar_wait(&bars->a_full[kq & 1], (uint32_t)((kq >> 1) & 1), kWaitNs))
          atomicOr(a.err, kErrTimeout);
      }
    }
  } else if (warp == 2) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t is16 = tc::idesc_bf16(128, 16, false, false);
      const uint32_t ipv = tc::idesc_bf16(128, 16, true, true);
      const uint32_t rr = ptx::smem_u32(ring);
      const uint32_t pb0 = ptx::smem_u32(sP), qb = ptx::smem_u32(sQ);
      int c = 0, k = 0, prev_tiles = 0;
      bool ok = true;
      auto pv = [&](int kk, int ntile) {
        const int pp = kk & 1;
        ok = ok && wait_or_abort(&bars->p_full[pp], (uint32_t)((kk >> 1) & 1), abort, a.err);
        if (kk >= 2)
          ok = ok && wait_or_abort(&bars->o_free[pp], (uint32_t)(((kk >> 1) - 1) & 1), abort, a.err);
        tc::fence_after_sync();
        for (int i = 0; ok && i < ntile; ++i) {
          const int st = c % kSlcStages;
          ok = wait_or_abort(&bars->full[st], (uint32_t)((c / kSlcStages) & 1), abort, a.err);
          tc::fence_after_sync();
          if (!ok) break;
          const uint32_t vb = rr + st * TILE;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::mma_ss(tmem + kSlcO + pp * 16, mnmaj(vb, ks),
                       tc::sdesc(pb0 + i * 4096 + ks * 512, 16, 256, tc::kSw32), ipv,
                       (i > 0 || ks > 0));
          tc::commit(&bars->empty[st]);
          ++c;
        }
        tc::commit(&bars->o_full[pp]);
      };
      SelRow cur, nxt;
      auto row_of = [&](long long uu) {
        int b, t, g;
        unit_of(uu, b, t, g);
        return a.sel + ((size_t)(b * a.T + t) * a.Hkv + g) * a.n;
      };
      if (blockIdx.x < U) cur.load(row_of(blockIdx.x), a.n);
      for (long long u = blockIdx.x; ok && u < U; u += gridDim.x, ++k) {
        if (u + gridDim.x < U) nxt.load(row_of(u + gridDim.x), a.n);
        const int ntile = (cur.count() + 1) / 2;
        const int pk = k & 1;
        ok = wait_or_abort(&bars->q_full[pk], (uint32_t)((k >> 1) & 1), abort, a.err);
        tc::fence_after_sync();
        const uint32_t qd = qb + pk * kQ16;
        for (int i = 0; ok && i < ntile; ++i) {
          const int st = c % kSlcStages;
          ok = wait_or_abort(&bars->full[st], (uint32_t)((c / kSlcStages) & 1), abort, a.err);
          tc::fence_after_sync();
          if (!ok) break;
          const uint32_t kb = rr + st * TILE;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            tc::mma_ss(tmem + pk * 128 + i * 16, kmaj(kb, ks, ATOM), kmaj(qd, ks, kQ16 / 2), is16,
                       ks > 0);
          tc::commit(&bars->empty[st]);
          ++c;
        }
        tc::commit(&bars->q_empty[pk]);
        tc::commit(&bars->s_full[pk]);
        if (k >= 1 && ok) pv(k - 1, prev_tiles);
        prev_tiles = ntile;
        cur = nxt;
      }
      if (k >= 1 && ok) pv(k - 1, prev_tiles);
      tc::commit(&bars->fin);
      if (!ptx::mbar_wait(&bars->fin, 0, kWaitNs)) atomicOr(a.err, kErrTimeout);
    }
  } else if (warp >= 4) {
    // ---------------- softmax and epilogue ----------------
    const int qd = warp & 3;
    const int r = qd * 32 + lane;  // TMEM lane: key row of a tile, then d in the epilogue
    const int half = r >> 6, kr = r & (SB - 1);
    const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
    int k = 0;
    int pb = 0, pt = 0, pg = 0;
    float pl[G];
    auto epilogue = [&](int kk) {
      const int pp = kk & 1;
      uint32_t u[16];
      tc::ld16_sync(tl + kSlcO + pp * 16, u);
      wait_or_abort(&bars->a_full[pp], (uint32_t)((kk >> 1) & 1), abort, a.err);
      const __nv_bfloat16* accs = reinterpret_cast<const __nv_bfloat16*>(sA + pp * kAccSlot);
      const float* gsl = reinterpret_cast<const float*>(sA + pp * kAccSlot + kAccBytes);
      __nv_bfloat16* o = a.out + ((size_t)(pb * a.T + pt) * a.Hq + pg * G) * D + r;
#pragma unroll
      for (int hh = 0; hh < G; ++hh)
        o[hh * D] = __float2bfloat16_rn(
            fmaf(gsl[hh] / pl[hh], __uint_as_float(u[hh]), __bfloat162float(accs[hh * D + r])));
      tc::fence_before_sync();
      ptx::mbar_arrive(&bars->o_free[pp]);
      ptx::mbar_arrive(&bars->a_empty[pp]);
    };
    SelRow cur, nxt;
    auto row_of = [&](long long uu) {
      int b, t, g;
      unit_of(uu, b, t, g);
      return a.sel + ((size_t)(b * a.T + t) * a.Hkv + g) * a.n;
    };
    if (blockIdx.x < U) cur.load(row_of(blockIdx.x), a.n);
    for (long long u = blockIdx.x; u < U; u += gridDim.x, ++k) {
      int b, t, g;
      unit_of(u, b, t, g);
      if (u + gridDim.x < U) nxt.load(row_of(u + gridDim.x), a.n);
      const int nsel = cur.count();
      const int pk = k & 1;
      wait_or_abort(&bars->s_full[pk], (uint32_t)((k >> 1) & 1), abort, a.err);
      tc::fence_after_sync();
      // uu: S^T of this key lane (8 tiles x 16 heads), masked in place, then
      // the probabilities
      uint32_t uu[128];
      tc::ld128_sync(tl + pk * 128, uu);
      float mh[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) mh[hh] = -INFINITY;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int blk = cur.blk(2 * i + half);
        if (!(2 * i + half < nsel && blk * SB + kr <= t)) {
#pragma unroll
          for (int hh = 0; hh < G; ++hh) uu[i * G + hh] = kNegInf;
        }
#pragma unroll
        for (int hh = 0; hh < G; ++hh) mh[hh] = fmaxf(mh[hh], __uint_as_float(uu[i * G + hh]));
      }
      // per-head maximum over the 128 keys of the four warps, then over warps
      const float mw = xreduce16<true>(mh, lane);
      if ((lane & 1) == 0) bars->red[0][qd][lane >> 1] = mw;
      ptx::named_bar_sync(1, 128);
      float nmc[G];  // -max * c; finite, since key 0 of block 0 is always valid
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 r0 = reinterpret_cast<const float4*>(bars->red[0][0])[q];
        const float4 r1 = reinterpret_cast<const float4*>(bars->red[0][1])[q];
        const float4 r2 = reinterpret_cast<const float4*>(bars->red[0][2])[q];
        const float4 r3 = reinterpret_cast<const float4*>(bars->red[0][3])[q];
        nmc[4 * q] = -fmaxf(fmaxf(r0.x, r1.x), fmaxf(r2.x, r3.x)) * a.c;
        nmc[4 * q + 1] = -fmaxf(fmaxf(r0.y, r1.y), fmaxf(r2.y, r3.y)) * a.c;
        nmc[4 * q + 2] = -fmaxf(fmaxf(r0.z, r1.z), fmaxf(r2.z, r3.z)) * a.c;
        nmc[4 * q + 3] = -fmaxf(fmaxf(r0.w, r1.w), fmaxf(r2.w, r3.w)) * a.c;
      }
      float lh[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) lh[hh] = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float x = ptx::ex2(fmaf(__uint_as_float(uu[i * G + hh]), a.c, nmc[hh]));
          uu[i * G + hh] = __float_as_uint(x);
          lh[hh] += x;
        }
      }
      const float lw = xreduce16<false>(lh, lane);
      if ((lane & 1) == 0) bars->red[1][qd][lane >> 1] = lw;
      // P of the previous unit must have been read by its PV MMA
      if (k >= 1)
        wait_or_abort(&bars->o_full[(k - 1) & 1], (uint32_t)(((k - 1) >> 1) & 1), abort, a.err);
      tc::fence_after_sync();
      const int ntile = (nsel + 1) / 2;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i < ntile) {
          const int R = i * KT + r;
          unsigned char* rowp = sP + (R >> 3) * 256 + (R & 7) * 32;
          uint4 lo, hi;
          lo.x = ptx::pack_bf16(__uint_as_float(uu[i * G + 0]), __uint_as_float(uu[i * G + 1]));
          lo.y = ptx::pack_bf16(__uint_as_float(uu[i * G + 2]), __uint_as_float(uu[i * G + 3]));
          lo.z = ptx::pack_bf16(__uint_as_float(uu[i * G + 4]), __uint_as_float(uu[i * G + 5]));
          lo.w = ptx::pack_bf16(__uint_as_float(uu[i * G + 6]), __uint_as_float(uu[i * G + 7]));
          hi.x = ptx::pack_bf16(__uint_as_float(uu[i * G + 8]), __uint_as_float(uu[i * G + 9]));
          hi.y = ptx::pack_bf16(__uint_as_float(uu[i * G + 10]), __uint_as_float(uu[i * G + 11]));
          hi.z = ptx::pack_bf16(__uint_as_float(uu[i * G + 12]), __uint_as_float(uu[i * G + 13]));
          hi.w = ptx::pack_bf16(__uint_as_float(uu[i * G + 14]), __uint_as_float(uu[i * G + 15]));
          const bool sw = (R & 7) >= 4;  // 32-byte swizzle: rows 4..7 swap halves
          *reinterpret_cast<uint4*>(rowp + (sw ? 16 : 0)) = lo;
          *reinterpret_cast<uint4*>(rowp + (sw ? 0 : 16)) = hi;
        }
      }
      ptx::fence_proxy_async();
      tc::fence_before_sync();
      ptx::mbar_arrive(&bars->p_full[pk]);
      if (k >= 1) epilogue(k - 1);
      ptx::named_bar_sync(1, 128);  // red[1] complete; red[0] free for the next unit
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 r0 = reinterpret_cast<const float4*>(bars->red[1][0])[q];
        const float4 r1 = reinterpret_cast<const float4*>(bars->red[1][1])[q];
        const float4 r2 = reinterpret_cast<const float4*>(bars->red[1][2])[q];
        const float4 r3 = reinterpret_cast<const float4*>(bars->red[1][3])[q];
        pl[4 * q] = (r0.x + r1.x) + (r2.x + r3.x);
        pl[4 * q + 1] = (r0.y + r1.y) + (r2.y + r3.y);
        pl[4 * q + 2] = (r0.z + r1.z) + (r2.z + r3.z);
        pl[4 * q + 3] = (r0.w + r1.w) + (r2.w + r3.w);
      }
      pb = b;
      pt = t;
      pg = g;
      cur = nxt;
    }
    if (k >= 1) {
      wait_or_abort(&bars->o_full[(k - 1) & 1], (uint32_t)(((k - 1) >> 1) & 1), abort, a.err);
      tc::fence_after_sync();
      epilogue(k - 1);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 3) tc::tmem_dealloc(tmem, 512);
}

size_t main_smem(int stages, int nblk) {
  return 1024 + TILE + (size_t)stages * TILE + (size_t)TQ * nblk * 4 + 128 * 4 +
         (size_t)TQ * KT * 4 + 16 * 4 + D * 3 * 4 + sizeof(MainBars);
}

size_t slc_smem() {
  return 1024 + kSlcStages * (size_t)TILE + 32768 + 2 * kQ16 + 2 * kAccSlot +
         sizeof(SlcBars);
}

int main_stages(int nblk) {
  for (int s = kMainStagesMax; s >= 2; --s)
    if (main_smem(s, nblk) <= 227 * 1024) return s;
  return 0;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

bool prefill_tc_eligible(const nsa_params& p) {
  if (p.dtype != NSA_DTYPE_BF16 || p.d != D || p.Hkv < 1 || p.Hq != G * p.Hkv) return false;
  if (p.sel_mode == 1 && (p.top_p != 0.f || !quest_tc_supported(p))) return false;
  if (p.sel_mode != 0 && p.sel_mode != 1) return false;
  if (p.cmp_block != CL || p.cmp_stride != CS || p.sel_block != SB) return false;
  if (p.top_n < 1 || p.top_n > kMaxSel || p.window < 1) return false;
  if ((long long)p.B * p.T >= (1ll << 30)) return false;
  const int nblk = (p.T + SB - 1) / SB;
  return main_stages(nblk) >= 2;
}

size_t prefill_tc_ws_bytes(const nsa_params& p) {
  const size_t rows = (size_t)p.B * p.T * p.Hq;
  return align256(rows * D * 2) + align256(rows * 4) +
         align256((size_t)p.B * p.T * p.Hkv * p.top_n * 4) +
         (p.sel_mode == 1 ? quest_ws_bytes(p) : 0);
}

cudaError_t launch_prefill_tc(const nsa_params& p, const void* q, const void* k, const void* v,
                              const void* kc, const void* vc, const float* w_gate, void* out,
                              int32_t* sel_out, void* ws, unsigned* err, cudaStream_t stream) {
  PfArgs a{};
  const size_t rows = (size_t)p.B * p.T * p.Hq;
  unsigned char* w = static_cast<unsigned char*>(ws);
  a.acc = reinterpret_cast<__nv_bfloat16*>(w);
  w += align256(rows * D * 2);
  a.gslc = reinterpret_cast<float*>(w);
  w += align256(rows * 4);
  a.sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(w);
  w += align256((size_t)p.B * p.T * p.Hkv * p.top_n * 4);
  const bool quest = p.sel_mode == 1;  // the selection comes from the block bounds
  a.w_gate = w_gate;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.err = err;
  a.B = p.B;
  a.T = p.T;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.Nc = nsa_num_cmp_blocks(p.T, p.cmp_block, p.cmp_stride);
  a.n = p.top_n;
  a.w = p.window;
  a.nblk = (p.T + SB - 1) / SB;
  a.stages = main_stages(a.nblk);
  const float scale = p.softmax_scale > 0.f ? p.softmax_scale : 1.f / sqrtf((float)p.d);
  a.c = scale * 1.4426950408889634f;
  a.gate_mode = p.gate_mode;
  for (int i = 0; i < 3; ++i) a.fixed_gates[i] = p.fixed_gates[i];
  const bool fixed = p.gate_mode == 1;
  const bool slc_branch = !(fixed && p.fixed_gates[1] == 0.f);
  a.need_sel = !quest && (slc_branch || sel_out != nullptr);
  a.run_cmp = !(fixed && p.fixed_gates[0] == 0.f) || a.need_sel;
  a.run_win = !(fixed && p.fixed_gates[2] == 0.f);
  a.direct_out = !slc_branch;
  a.top_p = p.top_p;

  const uint64_t BT = (uint64_t)p.B * p.T;
  CUtensorMap tq, tq16, tk, tv, tk64, tv64, tkc, tvc;
  bool ok = make_tmap_bf16_3d(&tq, q, D, p.Hq, BT, 64, G, TQ, true) &&
            make_tmap_bf16_3d(&tq16, q, D, p.Hq, BT, 64, G, 1, true) &&
            make_tmap_bf16_3d(&tk, k, D, p.Hkv, BT, 64, 1, KT, true) &&
            make_tmap_bf16_3d(&tv, v, D, p.Hkv, BT, 64, 1, KT, true) &&
            make_tmap_bf16_3d(&tk64, k, D, p.Hkv, BT, 64, 1, SB, true) &&
            make_tmap_bf16_3d(&tv64, v, D, p.Hkv, BT, 64, 1, SB, true);
  if (a.Nc > 0) {
    ok = ok && make_tmap_bf16_3d(&tkc, kc, D, p.Hkv, (uint64_t)p.B * a.Nc, 64, 1, KT, true) &&
         make_tmap_bf16_3d(&tvc, vc, D, p.Hkv, (uint64_t)p.B * a.Nc, 64, 1, KT, true);
  } else {
    tkc = tk;  // never read: no compressed block is visible anywhere
    tvc = tv;
  }
  if (!ok) return cudaErrorInvalidValue;

  cudaError_t e;
  if (quest && (slc_branch || sel_out != nullptr) &&
      (e = launch_quest_select(p, q, k, a.sel, w, stream)) != cudaSuccess)
    return e;
  const size_t sm1 = main_smem(a.stages, a.nblk);
  if ((e = ensure_dyn_smem((const void*)pf_main_kernel, 227 * 1024)) != cudaSuccess) return e;
  {
    TraceScope trace("pf_cmp_win", stream);
    const long long grid = (long long)p.B * p.Hkv * ((p.T + TQ - 1) / TQ);
    pf_main_kernel<<<(unsigned)grid, kMainThreads, sm1, stream>>>(tq, tkc, tvc, tk, tv, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.direct_out) return cudaSuccess;
  const size_t sm2 = slc_smem();
  if ((e = ensure_dyn_smem((const void*)pf_slc_kernel, (int)sm2)) != cudaSuccess) return e;
  {
    TraceScope trace("pf_slc_attn", stream);
    const long long U = (long long)p.B * p.T * p.Hkv;
    const int grid = (int)std::min<long long>(U, device_sm_count());
    pf_slc_kernel<<<grid, kSlcThreads, sm2, stream>>>(tq16, tk64, tv64, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace nsa
