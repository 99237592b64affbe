// MoBA causal prefill on the sm_100a tensor cores, block-centric (EP94 notes
// sections nine and ten: mean-pooled block keys, parameter-free top-k gating,
// the query's own block always attended; LateTalk ep.103). bf16, d = 128,
// block m a multiple of 128 (m <= 2048), top_k <= 8.
//
// A query row (token t, head h) attends to its own block c = t / m over
// [c m, t] and to top_k - 1 earlier blocks chosen by q . mean(K_block). With
// independent per-row choices no two rows share much, so the work is grouped
// by key block instead of by query (the gather / re-index view of the pages):
//   moba_split each fp32 block mean split once into three bf16 parts
//              (hi + mid + lo: 24 significant bits);
//   moba_gate  scores per row at fp32 accuracy as a tcgen05 product of the
//              query tile with the parts (TMEM accumulators), the picks,
//              the selection row, and per-(head, block) pick counts;
//   moba_scan  offsets of each (sequence, head, block) bucket and of its
//              128-row tiles;
//   moba_fill  the rows of every bucket (token, slot) and each bucket tile's
//              descriptor;
//   moba_blk   per bucket tile: 128 gathered query rows against the block's m
//              keys (tcgen05, TMEM accumulators), written as a normalised
//              partial output and its log-sum-exp;
//   moba_own   per 128 consecutive tokens of one head: causal attention over
//              the own block, merged with the row's partials into the output.
// The gate and both attention kernels are persistent (one CTA per SM) and
// warp-specialised: a TMA warp, one MMA-issuing thread, and row warps; in the
// attention kernels four softmax warps hand each tile's O (double-buffered in
// TMEM) and its rows' (m, l) to four epilogue / merge warps.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace nsa {
namespace {

constexpr int D = 128;
constexpr int KT = 128;           // keys per tile, rows per query tile
constexpr uint32_t ATOM = 16384;  // one d-half of a 128-row bf16 tile
constexpr uint32_t TILE = 32768;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kMaxTopk = 8;
constexpr int kStages = 4;
constexpr int kThreads = 192;     // TMA lanes, MMA thread, 4 softmax warps
constexpr int kBlkThreads = 320;  // moba_blk: + 4 epilogue warps
constexpr uint32_t kNegInf = 0xff800000u;

struct MobaTcArgs {
  const __nv_bfloat16* q;
  const float* kbar;      // [B, nfull, Hkv, d]
  __nv_bfloat16* kparts;  // [B, Hkv, 3, gate_rows(nfull), d]: hi, mid, lo of each block mean
  __nv_bfloat16* out;
  int32_t* sel;           // [B, T, Hq, topk]
  int32_t* cnt;           // [NB] picks per bucket (b, h, j)
  int32_t* off;           // [NB] first row of each bucket in `list`
  int32_t* toff;          // [NB + 1] first tile of each bucket
  int32_t* cur;           // [NB] fill cursors
  int32_t* list;          // rows: t * 8 + slot
  int4* tdesc;            // [tiles] each 128-row bucket tile: {bucket, first row, rows, 0}
  __nv_bfloat16* po;      // [B, T, Hq, topk - 1, d] partial outputs (normalised, bf16)
  float* plse;            // [B, T, Hq, topk - 1] their log2-sum-exp
  unsigned* err;
  int B, T, Hq, Hkv, m, topk, nfull, NB;
  float c;                // softmax scale * log2(e)
};

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
  return (unsigned char*)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort,
                                              unsigned* err) {
  if (*abort) return false;
  if (ptx::mbar_wait(bar, parity, kWaitNs)) return true;
  *abort = 1;
  atomicOr(err, kErrTimeout);
  return false;
}

__device__ __forceinline__ uint64_t kmaj(uint32_t base, int ks) {
  return tc::sdesc(base + (ks >> 2) * ATOM + (ks & 3) * 32, 16, 1024, tc::kSw128);
}

__device__ __forceinline__ uint64_t mnmaj(uint32_t base, int ks) {
  return tc::sdesc(base + ks * 2048, ATOM, 1024, tc::kSw128);
}

// ============================================================================
// gate, scan, fill
// ============================================================================

// Block scores q . kbar_j on the tensor cores without losing fp32 accuracy:
// q is bf16, and each fp32 block mean is split into three bf16 parts
// (hi + mid + lo, 24 significant bits), so every product q_e * part_e is exact
// in fp32 and the tensor core sums them in fp32, like the fp32 dot product on
// CUDA cores. A work item is 128 tokens of one (sequence, head); the tokens
// share one own block (m is a multiple of 128), so they score the same past
// blocks 0 .. own - 1. Per chunk of 128 blocks the three parts are loaded
// (TMA, one part per ring stage) and S = Q [hi | mid | lo]^T accumulates in a
// 128-column TMEM buffer that the four row warps then read: thread `row`
// keeps the best top_k - 1 of its row (higher score first, ties to the lower
// block: blocks arrive in increasing order and only a strictly higher score
// displaces a kept one).
//
// The kernel is persistent, one CTA per SM: items are taken round-robin in
// order of decreasing own block (the longest first) with the heads of one
// token tile next to each other, so the CTAs running at a time read whole
// token rows of q. The TMA warp runs ahead across items (two query tiles, a
// four-stage ring of parts), the MMA warp fills four score buffers, and the
// row warps drain them.
constexpr int kGateStages = 4;
constexpr int kGateAcc = 4;   // TMEM score buffers of 128 columns
constexpr int kGateBox = 32;  // block rows per TMA box of the parts

// Rows of the parts tensor per (sequence, KV head, part): the blocks padded to
// a whole number of TMA boxes, so every box the gate loads lies in the tensor.
__host__ __device__ inline int gate_rows(int nfull) {
  return nfull < kGateBox ? kGateBox : (nfull + kGateBox - 1) / kGateBox * kGateBox;
}

struct GateBars {
  uint64_t full[kGateStages], empty[kGateStages];
  uint64_t q_full[2], q_free[2], acc_full[kGateAcc], acc_free[kGateAcc], fin;
  uint32_t tmem;
  int abort;
};

size_t gate_smem() { return 1024 + (size_t)(2 + kGateStages) * TILE + sizeof(GateBars); }

// Work item i of the gate: token tile, sequence and head.
struct GateItem {
  int t0, b, h, own, nch;
};

__device__ __forceinline__ GateItem gate_item(const MobaTcArgs& a, int i, int want) {
  const int ntq = (a.T + KT - 1) / KT, bh = i % (a.B * a.Hq);
  GateItem it;
  it.t0 = (ntq - 1 - i / (a.B * a.Hq)) * KT;
  it.b = bh / a.Hq;
  it.h = bh % a.Hq;
  it.own = it.t0 / a.m;
  // 128-block chunks to score: none when every past block is taken, or none is
  it.nch = it.own > want && want > 0 ? (it.own + KT - 1) / KT : 0;
  return it;
}

// The selection row of token t when no block is scored: every block 0 .. own
// when there are at most top_k of them, else (top_k = 1) the own block alone;
// -1 after. Each past block taken counts a row into its bucket.
__device__ void gate_emit_unscored(const MobaTcArgs& a, int b, int h, int t, int own) {
  int32_t* dst = a.sel + ((size_t)(b * a.T + t) * a.Hq + h) * a.topk;
  if (own < a.topk) {
    for (int i = 0; i < a.topk; ++i) dst[i] = i <= own ? i : -1;
    for (int j = 0; j < own; ++j) atomicAdd(a.cnt + ((size_t)b * a.Hq + h) * a.nfull + j, 1);
  } else {
    dst[0] = own;
  }
}

// The best W (score, block) of one row, in registers (W = top_k - 1 is a
// compile-time constant, so no index is dynamic), sorted by decreasing score.
// Insertion is branch-free, so the lanes of a warp never diverge: entry i
// takes the candidate if it beats entry i but not entry i - 1, entry i - 1 if
// the candidate beats that too. Strict comparisons keep the lower block first
// among equal scores (candidates arrive in increasing block order).
template <int W>
struct KeepBest {
  float s[W];
  int j[W];
  __device__ __forceinline__ KeepBest() {
#pragma unroll
    for (int i = 0; i < W; ++i) {
      s[i] = -INFINITY;
      j[i] = -1;
    }
  }
  __device__ __forceinline__ void offer(float x, int k) {
    bool gt[W];
#pragma unroll
    for (int i = 0; i < W; ++i) gt[i] = x > s[i];
#pragma unroll
    for (int i = W - 1; i > 0; --i) {
      s[i] = gt[i] ? (gt[i - 1] ? s[i - 1] : x) : s[i];
      j[i] = gt[i] ? (gt[i - 1] ? j[i - 1] : k) : j[i];
    }
    s[0] = gt[0] ? x : s[0];
    j[0] = gt[0] ? k : j[0];
  }
  // The row: the picks in increasing block order, then the own block, -1
  // after; each pick counts a row into its bucket.
  __device__ __forceinline__ void emit(const MobaTcArgs& a, int b, int h, int t, int own) {
    int v[W];
#pragma unroll
    for (int i = 0; i < W; ++i) v[i] = j[i] < 0 ? 0x7fffffff : j[i];
#pragma unroll
    for (int p = 0; p < W; ++p)
#pragma unroll
      for (int i = 0; i + 1 < W - p; ++i)
        if (v[i] > v[i + 1]) {
          const int x = v[i];
          v[i] = v[i + 1];
          v[i + 1] = x;
        }
    int n = 0;
#pragma unroll
    for (int i = 0; i < W; ++i) n += v[i] != 0x7fffffff;
    int32_t* dst = a.sel + ((size_t)(b * a.T + t) * a.Hq + h) * a.topk;
    int32_t* cnt = a.cnt + ((size_t)b * a.Hq + h) * a.nfull;
#pragma unroll
    for (int i = 0; i < W; ++i)
      if (i < n) {
        dst[i] = v[i];
        atomicAdd(cnt + v[i], 1);
      }
    for (int i = n; i < a.topk; ++i) dst[i] = i == n ? own : -1;
  }
};

// Row warps 0-3 over the CTA's items: thread = row = TMEM lane. Per chunk the
// scores of its nb blocks are read 32 columns at a time and offered in block
// order.
template <int W>
__device__ __forceinline__ void gate_rows(const MobaTcArgs& a, GateBars* bars, volatile int* abort,
                                          uint32_t tl, int row, int want) {
  const int NI = a.B * a.Hq * ((a.T + KT - 1) / KT);
  int ac = 0;
  for (int i = blockIdx.x; i < NI; i += gridDim.x) {
    const GateItem it = gate_item(a, i, want);
    const int t = it.t0 + row;
    if (it.nch == 0) {
      if (t < a.T) gate_emit_unscored(a, it.b, it.h, t, it.own);
      continue;
    }
    KeepBest<W> kb;
    for (int c = 0; c < it.nch; ++c, ++ac) {
      const int buf = ac % kGateAcc, c0 = c * KT, nb = min(KT, it.own - c0);
      if (!wait_or_abort(&bars->acc_full[buf], (uint32_t)((ac / kGateAcc) & 1), abort, a.err))
        return;
      tc::fence_after_sync();
      for (int x = 0; x < nb; x += 32) {
        uint32_t r[32];
        tc::ld32_sync(tl + buf * KT + x, r);
        if (x + 32 <= nb) {
#pragma unroll
          for (int k = 0; k < 32; ++k) kb.offer(__uint_as_float(r[k]), c0 + x + k);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (x + k < nb) kb.offer(__uint_as_float(r[k]), c0 + x + k);
        }
      }
      tc::fence_before_sync();
      ptx::mbar_arrive(&bars->acc_free[buf]);
    }
    if (t < a.T) kb.emit(a, it.b, it.h, t, it.own);
  }
}

// Warps 0-3: the rows (TMEM lane = row); warp 4 lane 0: TMA; warp 5 lane 0:
// MMAs. One CTA per SM (grid = min(items, SMs)).
__global__ void __launch_bounds__(kThreads, 1)
    moba_gate_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tp,
                     const MobaTcArgs a) {
  extern __shared__ unsigned char smraw[];
  unsigned char* base = align1024(smraw);
  unsigned char* sQ = base;  // two query tiles
  unsigned char* ring = base + 2 * TILE;
  GateBars* bars = reinterpret_cast<GateBars*>(ring + kGateStages * TILE);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int want = a.topk - 1;
  const int NI = a.B * a.Hq * ((a.T + KT - 1) / KT);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGateStages; ++i) {
      ptx::mbar_init(&bars->full[i], 1);
      ptx::mbar_init(&bars->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bars->q_full[i], 1);
      ptx::mbar_init(&bars->q_free[i], 1);
    }
    for (int i = 0; i < kGateAcc; ++i) {
      ptx::mbar_init(&bars->acc_full[i], 1);
      ptx::mbar_init(&bars->acc_free[i], KT);
    }
    ptx::mbar_init(&bars->fin, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(&bars->tmem, kGateAcc * KT);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem;

  if (warp == 4) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tq);
      ptx::prefetch_tmap(&tp);
      const uint64_t first = ptx::policy_evict_first(), keep = ptx::policy_evict_last();
      int lastq[2] = {-1, -1}, last[kGateStages];
      for (int s = 0; s < kGateStages; ++s) last[s] = -1;
      int qi = 0, st = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < NI; i += gridDim.x) {
        const GateItem it = gate_item(a, i, want);
        if (it.nch == 0) continue;
        const int qb = qi & 1;
        if (qi >= 2 &&
            !wait_or_abort(&bars->q_free[qb], (uint32_t)(((qi - 2) >> 1) & 1), abort, a.err))
          break;
        unsigned char* qd = sQ + qb * TILE;
        ptx::mbar_arrive_expect_tx(&bars->q_full[qb], TILE);
        ptx::tma_load_3d(qd, &tq, &bars->q_full[qb], 0, it.h, it.b * a.T + it.t0, first);
        ptx::tma_load_3d(qd + ATOM, &tq, &bars->q_full[qb], 64, it.h, it.b * a.T + it.t0, first);
        lastq[qb] = qi++;
        const int z = (it.b * a.Hkv + it.h / (a.Hq / a.Hkv)) * 3;
        for (int c = 0; ok && c < it.nch; ++c) {
          const int c0 = c * KT, nbox = (min(KT, it.own - c0) + kGateBox - 1) / kGateBox;
          for (int pp = 0; pp < 3; ++pp, ++st) {
            const int s = st % kGateStages;
            if (st >= kGateStages &&
                !wait_or_abort(&bars->empty[s], (uint32_t)(((st / kGateStages) - 1) & 1), abort,
                               a.err)) {
              ok = false;
              break;
            }
            unsigned char* dst = ring + s * TILE;
            ptx::mbar_arrive_expect_tx(&bars->full[s], (uint32_t)(nbox * 2 * kGateBox * 128));
            for (int x = 0; x < nbox; ++x) {
              ptx::tma_load_3d(dst + x * kGateBox * 128, &tp, &bars->full[s], 0,
                               c0 + x * kGateBox, z + pp, keep);
              ptx::tma_load_3d(dst + ATOM + x * kGateBox * 128, &tp, &bars->full[s], 64,
                               c0 + x * kGateBox, z + pp, keep);
            }
            last[s] = st;
          }
        }
      }
      // every issued load lands before the CTA can exit
      for (int s = 0; s < kGateStages; ++s)
        if (last[s] >= 0 &&
            !ptx::mbar_wait(&bars->full[s], (uint32_t)((last[s] / kGateStages) & 1), kWaitNs))
          atomicOr(a.err, kErrTimeout);
      for (int s = 0; s < 2; ++s)
        if (lastq[s] >= 0 &&
            !ptx::mbar_wait(&bars->q_full[s], (uint32_t)((lastq[s] >> 1) & 1), kWaitNs))
          atomicOr(a.err, kErrTimeout);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t r0 = ptx::smem_u32(ring);
      int qi = 0, st = 0, ac = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < NI; i += gridDim.x) {
        const GateItem it = gate_item(a, i, want);
        if (it.nch == 0) continue;
        const int qb = qi & 1;
        ok = wait_or_abort(&bars->q_full[qb], (uint32_t)((qi >> 1) & 1), abort, a.err);
        tc::fence_after_sync();
        const uint32_t q0 = ptx::smem_u32(sQ + qb * TILE);
        for (int c = 0; ok && c < it.nch; ++c, ++ac) {
          const int buf = ac % kGateAcc, nb = min(KT, it.own - c * KT);
          const uint32_t id = tc::idesc_bf16(128, (nb + 15) & ~15, false, false);
          if (ac >= kGateAcc) {
            ok = wait_or_abort(&bars->acc_free[buf], (uint32_t)(((ac / kGateAcc) - 1) & 1), abort,
                               a.err);
            tc::fence_after_sync();
          }
          for (int pp = 0; ok && pp < 3; ++pp, ++st) {
            const int s = st % kGateStages;
            ok = wait_or_abort(&bars->full[s], (uint32_t)((st / kGateStages) & 1), abort, a.err);
            if (!ok) break;
            tc::fence_after_sync();
            const uint32_t kb = r0 + s * TILE;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
              tc::mma_ss(tmem + buf * KT, kmaj(q0, ks), kmaj(kb, ks), id, (pp > 0 || ks > 0));
            tc::commit(&bars->empty[s]);
          }
          if (ok) tc::commit(&bars->acc_full[buf]);
        }
        tc::commit(&bars->q_free[qb]);
        ++qi;
      }
      tc::commit(&bars->fin);
      if (!ptx::mbar_wait(&bars->fin, 0, kWaitNs)) atomicOr(a.err, kErrTimeout);
    }
  } else {
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const int row = warp * 32 + lane;
    switch (want) {
      case 0: gate_rows<1>(a, bars, abort, tl, row, want); break;  // no item is scored
      case 1: gate_rows<1>(a, bars, abort, tl, row, want); break;
      case 2: gate_rows<2>(a, bars, abort, tl, row, want); break;
      case 3: gate_rows<3>(a, bars, abort, tl, row, want); break;
      case 4: gate_rows<4>(a, bars, abort, tl, row, want); break;
      case 5: gate_rows<5>(a, bars, abort, tl, row, want); break;
      case 6: gate_rows<6>(a, bars, abort, tl, row, want); break;
      default: gate_rows<7>(a, bars, abort, tl, row, want); break;
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, kGateAcc * KT);
}

// Each fp32 block mean once into three bf16 parts hi + mid + lo (hi = bf16(x),
// mid = bf16(x - hi), lo = bf16(x - hi - mid): 24 significant bits), so every
// product with a bf16 query element is exact in fp32. Layout
// [B, Hkv, 3, gate_rows(nfull), d]; the padding rows are zero.
__global__ void __launch_bounds__(256) moba_split_kernel(MobaTcArgs a) {
  const int nr = gate_rows(a.nfull);
  const size_t n4 = (size_t)a.B * a.Hkv * nr * (D / 4);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t rest = i / (D / 4);
    const int e = (int)(i - rest * (D / 4)) * 4;
    const int j = (int)(rest % nr);
    const size_t bg = rest / nr;
    const int b = (int)(bg / a.Hkv), g = (int)(bg % a.Hkv);
    float xs[4] = {0.f, 0.f, 0.f, 0.f};
    if (j < a.nfull) {
      const float4 x =
          reinterpret_cast<const float4*>(a.kbar + (((size_t)b * a.nfull + j) * a.Hkv + g) * D + e)[0];
      xs[0] = x.x;
      xs[1] = x.y;
      xs[2] = x.z;
      xs[3] = x.w;
    }
    __nv_bfloat16 hi[4], mid[4], lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      hi[k] = __float2bfloat16_rn(xs[k]);
      const float r1 = xs[k] - __bfloat162float(hi[k]);
      mid[k] = __float2bfloat16_rn(r1);
      lo[k] = __float2bfloat16_rn(r1 - __bfloat162float(mid[k]));
    }
    __nv_bfloat16* dst = a.kparts + (bg * 3 * nr + j) * D + e;
    *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(hi);
    *reinterpret_cast<uint2*>(dst + (size_t)nr * D) = *reinterpret_cast<const uint2*>(mid);
    *reinterpret_cast<uint2*>(dst + 2 * (size_t)nr * D) = *reinterpret_cast<const uint2*>(lo);
  }
}
// Exclusive prefix sums of the bucket counts (rows) and of their 128-row
// tiles, in one CTA.
__global__ void __launch_bounds__(1024) moba_scan_kernel(MobaTcArgs a) {
  __shared__ int wsum[2][32];
  __shared__ int carry[2];
  if (threadIdx.x == 0) carry[0] = carry[1] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < a.NB; base += 1024) {
    const int i = base + threadIdx.x;
    const int c = i < a.NB ? a.cnt[i] : 0;
    int v0 = c, v1 = (c + KT - 1) / KT;
    int x0 = v0, x1 = v1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
      if (lane >= o) {
        x0 += y0;
        x1 += y1;
      }
    }
    if (lane == 31) {
      wsum[0][warp] = x0;
      wsum[1][warp] = x1;
    }
    __syncthreads();
    if (warp == 0) {
      int s0 = wsum[0][lane], s1 = wsum[1][lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y0 = __shfl_up_sync(0xffffffffu, s0, o), y1 = __shfl_up_sync(0xffffffffu, s1, o);
        if (lane >= o) {
          s0 += y0;
          s1 += y1;
        }
      }
      wsum[0][lane] = s0;
      wsum[1][lane] = s1;
    }
    __syncthreads();
    const int pre0 = carry[0] + (warp ? wsum[0][warp - 1] : 0) + x0 - v0;
    const int pre1 = carry[1] + (warp ? wsum[1][warp - 1] : 0) + x1 - v1;
    if (i < a.NB) {
      a.off[i] = pre0;
      a.toff[i] = pre1;
      a.cur[i] = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      carry[0] += wsum[0][31];
      carry[1] += wsum[1][31];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) a.toff[a.NB] = carry[1];
}

// Rows into buckets: list[off[bucket] + k] = t * 8 + slot; and the
// descriptor of every bucket tile (one 16-byte load for moba_blk).
__global__ void moba_fill_kernel(MobaTcArgs a) {
  for (int bk = blockIdx.x * blockDim.x + threadIdx.x; bk < a.NB; bk += gridDim.x * blockDim.x)
    for (int k = a.toff[bk], r = 0; k < a.toff[bk + 1]; ++k, r += KT)
      a.tdesc[k] = make_int4(bk, a.off[bk] + r, min(KT, a.cnt[bk] - r), 0);
  const long long n = (long long)a.B * a.T * a.Hq;
  for (long long r = blockIdx.x * (long long)blockDim.x + threadIdx.x; r < n;
       r += (long long)gridDim.x * blockDim.x) {
    const int h = (int)(r % a.Hq);
    const long long bt = r / a.Hq;
    const int b = (int)(bt / a.T), t = (int)(bt % a.T);
    const int32_t* s = a.sel + r * a.topk;
    const int own = t / a.m;
    int slot = 0;
    for (int i = 0; i < a.topk; ++i) {
      const int j = s[i];
      if (j < 0 || j == own) continue;
      const int bk = (b * a.Hq + h) * a.nfull + j;
      const int pos = atomicAdd(a.cur + bk, 1);
      a.list[a.off[bk] + pos] = t * 8 + slot;
      ++slot;
    }
  }
}

// ============================================================================
// the attention kernels: shared pieces
// ============================================================================

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full[2], q_free[2], s_full[2], p_full[2], o_done[2], fin;
  uint64_t o_full[2], o_free[2], ml_full, ml_free;  // moba_blk: O per tile parity, (m, l) hand-off
  uint32_t tmem;
  int abort;
};

// TMEM: O at 0, S buffers at 128 and 256, the second O (odd tiles or items) at 384
constexpr uint32_t kO = 0, kS0 = 128, kO2 = 384;

__device__ void init_bars(Bars* bars, int q_full_count) {
  for (int i = 0; i < kStages; ++i) {
    ptx::mbar_init(&bars->full[i], 1);
    ptx::mbar_init(&bars->empty[i], 1);
  }
  for (int i = 0; i < 2; ++i) {
    ptx::mbar_init(&bars->q_full[i], q_full_count);
    ptx::mbar_init(&bars->q_free[i], 1);
    ptx::mbar_init(&bars->s_full[i], 1);
    ptx::mbar_init(&bars->p_full[i], 128);
    ptx::mbar_init(&bars->o_done[i], 1);
  }
  for (int i = 0; i < 2; ++i) {
    ptx::mbar_init(&bars->o_full[i], 1);
    ptx::mbar_init(&bars->o_free[i], 128);
  }
  ptx::mbar_init(&bars->ml_full, 128);
  ptx::mbar_init(&bars->ml_free, 128);
  ptx::mbar_init(&bars->fin, 1);
  bars->abort = 0;
  ptx::fence_mbar_init();
}

// One K or V tile (128 keys x 128 d) from lane `lane` of the producer warp:
// loads c = lane (mod kStages) go to stage `lane`.
struct Producer {
  unsigned char* ring;
  Bars* bars;
  volatile int* abort;
  unsigned* err;
  int lane, c = 0, mine = 0;
  bool ok = true;
  __device__ void load(const CUtensorMap* m, int g, int z, uint64_t pol) {
    const int cc = c++;
    if (!ok || cc % kStages != lane) return;
    if (cc >= kStages &&
        !wait_or_abort(&bars->empty[lane], (uint32_t)(((cc / kStages) - 1) & 1), abort, err)) {
      ok = false;
      return;
    }
    unsigned char* dst = ring + lane * TILE;
    ptx::mbar_arrive_expect_tx(&bars->full[lane], TILE);
    ptx::tma_load_3d(dst, m, &bars->full[lane], 0, g, z, pol);
    ptx::tma_load_3d(dst + ATOM, m, &bars->full[lane], 64, g, z, pol);
    ++mine;
  }
  __device__ void drain() {
    if (mine > 0) {
      const int last = lane + (mine - 1) * kStages;
      if (!ptx::mbar_wait(&bars->full[lane], (uint32_t)((last / kStages) & 1), kWaitNs))
        atomicOr(err, kErrTimeout);
    }
  }
};

// MMA side of query tile kt with `nk` key tiles: S_u = Q K_u^T into S buffer
// (j & 1), O += P_u V_u with P from TMEM; j and c are the running tile and
// load counters of the CTA. O of tile kt is O[kt & 1]: the tile's first PV
// waits until the epilogue of tile kt - 2 has released that buffer, and its
// last PV commits o_full[kt & 1].
struct Mma {
  Bars* bars;
  volatile int* abort;
  unsigned* err;
  uint32_t tmem, r0;
  int j = 0, c = 0;
  bool ok = true;
  __device__ int take() {
    const int st = c % kStages;
    if (ok) ok = wait_or_abort(&bars->full[st], (uint32_t)((c / kStages) & 1), abort, err);
    tc::fence_after_sync();
    return st;
  }
  __device__ void tile(uint32_t q0, int nk, int qbuf, int kt = 0) {
    const uint32_t ob = (kt & 1) ? kO2 : kO;
    const uint32_t iss = tc::idesc_bf16(128, 128, false, false);
    const uint32_t its = tc::idesc_bf16(128, 128, false, true);
    const int j0 = j;
    for (int u = 0; ok && u <= nk; ++u) {
      if (u < nk) {
        const int jj = j0 + u, bs = jj & 1;
        if (jj >= 2)
          ok = ok && wait_or_abort(&bars->p_full[bs], (uint32_t)(((jj - 2) >> 1) & 1), abort, err);
        const int st = take();
        if (!ok) break;
        const uint32_t kb = r0 + st * TILE;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc::mma_ss(tmem + kS0 + bs * 128, kmaj(q0, ks), kmaj(kb, ks), iss, ks > 0);
        tc::commit(&bars->empty[st]);
        tc::commit(&bars->s_full[bs]);
        ++c;
        if (u == nk - 1) tc::commit(&bars->q_free[qbuf]);
      }
      if (u >= 1) {
        const int pj = j0 + u - 1, pb = pj & 1;
        ok = ok && wait_or_abort(&bars->p_full[pb], (uint32_t)((pj >> 1) & 1), abort, err);
        if (u == 1 && kt >= 2)
          ok = ok && wait_or_abort(&bars->o_free[kt & 1], (uint32_t)(((kt >> 1) - 1) & 1), abort,
                                   err);
        tc::fence_after_sync();
        const int st = take();
        if (!ok) break;
        const uint32_t vb = r0 + st * TILE;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc::mma_ts(tmem + ob, tmem + kS0 + pb * 128 + ks * 8, mnmaj(vb, ks), its,
                     (u > 1 || ks > 0));
        tc::commit(&bars->empty[st]);
        tc::commit(&bars->o_done[pj & 1]);
        if (u == nk) tc::commit(&bars->o_full[kt & 1]);
        ++c;
      }
    }
    j = j0 + nk;
  }
};

// Softmax side: thread `row` of the query tile, one S tile at a time; keys at
// index >= klim are masked (the causal edge). m is kept in the log2 domain.
struct Softmax {
  Bars* bars;
  volatile int* abort;
  unsigned* err;
  uint32_t tl;
  float cs;
  int j = 0;
  uint32_t obuf = kO;  // O's TMEM column of the current tile
  // The row's nk key tiles [kb0, kb0 + 128 nk). The next tile's scores are
  // loaded from TMEM before this tile's P stores are waited for, so the two
  // TMEM latencies overlap (the next S is in the other buffer, and its QK MMA
  // never waits for this tile's P).
  __device__ void run(int nk, int kb0, int klim, float& m, float& l) {
    if (nk <= 0) return;
    uint32_t u[128];
    wait_or_abort(&bars->s_full[j & 1], (uint32_t)((j >> 1) & 1), abort, err);
    tc::fence_after_sync();
    tc::ld128_nowait(tl + kS0 + (j & 1) * 128, u);
    tc::ld_wait128(u);
    for (int t = 0; t < nk; ++t) {
      const int bs = j & 1, kb = kb0 + t * KT;
      if (kb + KT > klim) {
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (kb + e >= klim) u[e] = kNegInf;
      }
      float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
#pragma unroll
      for (int e = 0; e < 128; e += 4) {
        mx0 = fmaxf(mx0, __uint_as_float(u[e]));
        mx1 = fmaxf(mx1, __uint_as_float(u[e + 1]));
        mx2 = fmaxf(mx2, __uint_as_float(u[e + 2]));
        mx3 = fmaxf(mx3, __uint_as_float(u[e + 3]));
      }
      const float mt = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * cs;
      const float mn = fmaxf(m, mt);
      if (mn != -INFINITY && (m == -INFINITY || mn > m + 8.f)) {
        if (m != -INFINITY) {
          const float f = exp2f(m - mn);
          l *= f;
          wait_or_abort(&bars->o_done[(j - 1) & 1], (uint32_t)(((j - 1) >> 1) & 1), abort, err);
          tc::fence_after_sync();
#pragma unroll 1
          for (int q4 = 0; q4 < 8; ++q4) {
            uint32_t w[16];
            const uint32_t oc = tl + obuf + q4 * 16;
            tc::ld16_sync(oc, w);
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * f);
            tc::st16(oc, w);
          }
          tc::st_wait();
        }
        m = mn;
      }
      const float nm = m == -INFINITY ? 0.f : -m;
      float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = ptx::ex2(fmaf(__uint_as_float(u[q4 * 32 + 2 * e]), cs, nm));
          const float p1 = ptx::ex2(fmaf(__uint_as_float(u[q4 * 32 + 2 * e + 1]), cs, nm));
          ls0 += p0;
          ls1 += p1;
          pk[e] = ptx::pack_bf16(p0, p1);
        }
        tc::st16(tl + kS0 + bs * 128 + q4 * 16, pk);
      }
      l += ls0 + ls1;
      const bool more = t + 1 < nk;
      if (more) {
        wait_or_abort(&bars->s_full[(j + 1) & 1], (uint32_t)(((j + 1) >> 1) & 1), abort, err);
        tc::fence_after_sync();
        tc::ld128_nowait(tl + kS0 + ((j + 1) & 1) * 128, u);
      }
      tc::st_wait();
      tc::fence_before_sync();
      ptx::mbar_arrive(&bars->p_full[bs]);
      if (more) tc::ld_wait128(u);
      ++j;
    }
  }
};


// ============================================================================
// moba_blk: bucket tiles (gathered rows x one earlier block)
// ============================================================================

struct BlkTile {
  int b, h, j, first, nrow;  // rows list[first .. first + nrow)
};

__device__ __forceinline__ BlkTile blk_tile(const MobaTcArgs& a, int i) {
  BlkTile w;
  const int4 d = a.tdesc[i];
  const int bk = d.x, bh = bk / a.nfull;
  w.j = bk % a.nfull;
  w.h = bh % a.Hq;
  w.b = bh / a.Hq;
  w.first = d.y;
  w.nrow = d.z;
  return w;
}

__global__ void __launch_bounds__(kBlkThreads, 1)
    moba_blk_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const MobaTcArgs a) {
  extern __shared__ unsigned char smraw[];
  unsigned char* base = align1024(smraw);
  unsigned char* sQ = base;              // 2 x 32 KB
  unsigned char* ring = base + 2 * TILE;
  Bars* bars = reinterpret_cast<Bars*>(ring + kStages * TILE);
  float2* ml_s = reinterpret_cast<float2*>(bars + 1);  // [row]
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntile = a.toff[a.NB];
  const int G = a.Hq / a.Hkv;
  const int nk = a.m / KT;

  if (threadIdx.x == 0) init_bars(bars, 128);
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem;

  if (warp == 0) {
    if (lane < kStages) {
      if (lane == 0) {
        ptx::prefetch_tmap(&tk);
        ptx::prefetch_tmap(&tv);
      }
      Producer pr{ring, bars, abort, a.err, lane};
      const uint64_t keep = ptx::policy_evict_last();
      BlkTile wn = blockIdx.x < (unsigned)ntile ? blk_tile(a, blockIdx.x) : BlkTile{};
      for (int i = blockIdx.x; pr.ok && i < ntile; i += gridDim.x) {
        const BlkTile w = wn;
        if (i + (int)gridDim.x < ntile) wn = blk_tile(a, i + gridDim.x);  // in flight meanwhile
        const int g = w.h / G;
        const int z0 = w.b * a.T + w.j * a.m;
        for (int u = 0; u < nk; ++u) {
          pr.load(&tk, g, z0 + u * KT, keep);
          if (u >= 1) pr.load(&tv, g, z0 + (u - 1) * KT, keep);
        }
        pr.load(&tv, g, z0 + (nk - 1) * KT, keep);
      }
      pr.drain();
    }
  } else if (warp == 1) {
    if (lane == 0) {
      Mma mm{bars, abort, a.err, tmem, ptx::smem_u32(ring)};
      int k = 0;
      for (int i = blockIdx.x; mm.ok && i < ntile; i += gridDim.x, ++k) {
        const int qb = k & 1;
        mm.ok = wait_or_abort(&bars->q_full[qb], (uint32_t)((k >> 1) & 1), abort, a.err);
        tc::fence_after_sync();
        mm.tile(ptx::smem_u32(sQ + qb * TILE), nk, qb, k);
      }
      tc::commit(&bars->fin);
      if (!ptx::mbar_wait(&bars->fin, 0, kWaitNs)) atomicOr(a.err, kErrTimeout);
    }
  } else if (warp < 6) {
    // softmax warps: tile after tile, O of tile k in O[k & 1]; each row's
    // (m, l) goes to the epilogue warps through shared memory
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    Softmax sm{bars, abort, a.err, tmem + ((uint32_t)(qd * 32) << 16), a.c};
    int k = 0;
    for (int i = blockIdx.x; i < ntile; i += gridDim.x, ++k) {
      sm.obuf = (k & 1) ? kO2 : kO;
      float m = -INFINITY, l = 0.f;
      sm.run(nk, 0, 1 << 30, m, l);
      if (k >= 1)  // the epilogue warps have read tile k - 1's
        wait_or_abort(&bars->ml_free, (uint32_t)((k - 1) & 1), abort, a.err);
      ml_s[row] = make_float2(m, l);
      ptx::mbar_arrive(&bars->ml_full);
    }
  } else {
    // epilogue warps: the query rows of tile k + 2 are copied (cp.async, this
    // thread's row, zeros past the bucket) while tile k's normalised partial
    // outputs and log-sum-exps are written from O[k & 1], which is then
    // released to the MMA thread; the rows are handed over at the end.
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
    auto gather = [&](const BlkTile& w, int e, int kq) {
      const int qb = kq & 1;
      if (kq >= 2) wait_or_abort(&bars->q_free[qb], (uint32_t)(((kq >> 1) - 1) & 1), abort, a.err);
      unsigned char* dq = sQ + qb * TILE;
      const bool live = e >= 0;
      const __nv_bfloat16* src =
          a.q + ((size_t)(w.b * a.T + (live ? e >> 3 : 0)) * a.Hq + w.h) * D;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        ptx::cp_async16_zfill(dq + (c >> 3) * ATOM + row * 128 + (((c & 7) ^ (row & 7)) << 4),
                              src + c * 8, live ? 16u : 0u);
      ptx::cp_async_commit();
    };
    auto hand_over = [&](int kq) {
      ptx::cp_async_wait<0>();
      ptx::fence_proxy_async();
      ptx::mbar_arrive(&bars->q_full[kq & 1]);
    };
    auto entry = [&](const BlkTile& w) { return row < w.nrow ? a.list[w.first + row] : -1; };
    if (blockIdx.x < (unsigned)ntile) {
      const int G1 = gridDim.x;
      BlkTile cur = blk_tile(a, blockIdx.x);
      int ecur = entry(cur);
      gather(cur, ecur, 0);
      hand_over(0);
      BlkTile nxt{};
      int enxt = -1;
      if ((int)blockIdx.x + G1 < ntile) {
        nxt = blk_tile(a, blockIdx.x + G1);
        enxt = entry(nxt);
        gather(nxt, enxt, 1);
        hand_over(1);
      }
      int k = 0;
      for (int i = blockIdx.x; i < ntile && !*abort; i += G1, ++k) {
        const bool more2 = i + 2 * G1 < ntile;
        BlkTile n2{};
        int en2 = -1;
        if (more2) {
          n2 = blk_tile(a, i + 2 * G1);
          en2 = entry(n2);
          gather(n2, en2, k + 2);
        }
        wait_or_abort(&bars->ml_full, (uint32_t)(k & 1), abort, a.err);
        const float2 ml = ml_s[row];
        ptx::mbar_arrive(&bars->ml_free);
        wait_or_abort(&bars->o_full[k & 1], (uint32_t)((k >> 1) & 1), abort, a.err);
        tc::fence_after_sync();
        const float m = ml.x, l = ml.y;
        const bool live = ecur >= 0;
        const int e = live ? ecur : 0;
        const size_t pr =
            ((size_t)(cur.b * a.T + (e >> 3)) * a.Hq + cur.h) * (a.topk - 1) + (e & 7);
        const float il = l > 0.f ? 1.f / l : 0.f;
        const uint32_t ob = (k & 1) ? kO2 : kO;
#pragma unroll 1
        for (int c32 = 0; c32 < 4; ++c32) {
          uint32_t o[32];
          tc::ld32_sync(tl + ob + c32 * 32, o);
          if (live) {
            uint4 pk[4];
            uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
            for (int x = 0; x < 16; ++x)
              pw[x] = ptx::pack_bf16(__uint_as_float(o[2 * x]) * il,
                                     __uint_as_float(o[2 * x + 1]) * il);
            uint4* dst = reinterpret_cast<uint4*>(a.po + pr * D + c32 * 32);
#pragma unroll
            for (int x = 0; x < 4; ++x) dst[x] = pk[x];
          }
        }
        if (live) a.plse[pr] = m + __log2f(l);
        tc::fence_before_sync();
        ptx::mbar_arrive(&bars->o_free[k & 1]);
        if (more2) hand_over(k + 2);
        cur = nxt;
        ecur = enxt;
        nxt = n2;
        enxt = en2;
      }
      ptx::cp_async_wait<0>();  // no copy in flight past an abort
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ============================================================================
// moba_own: own block, causal, merged with the partials
// ============================================================================

// Work item i: 128 consecutive tokens of one (sequence, head), the heads of a
// token tile adjacent (the tiles of one block and head, which share its keys,
// run at about the same time on different SMs).
struct OwnItem {
  int b, h, t0, c0, nk;
};

__device__ __forceinline__ OwnItem own_item(const MobaTcArgs& a, int i) {
  OwnItem it;
  const int bh = i % (a.B * a.Hq);
  it.b = bh / a.Hq;
  it.h = bh % a.Hq;
  it.t0 = (i / (a.B * a.Hq)) * KT;
  const int tlast = min(it.t0 + KT - 1, a.T - 1);
  it.c0 = (it.t0 / a.m) * a.m;  // own block start (a 128-token tile never straddles blocks)
  it.nk = (tlast - it.c0) / KT + 1;
  return it;
}

// Merge of a row: its own-block output (o / l, log2-sum-exp m + log2 l, o in
// TMEM once the last PV MMA is done) with its np partials (normalised, bf16)
// and their log2-sum-exps: out = sum_i 2^(lse_i - M) o_i / sum_i 2^(lse_i - M).
__device__ __forceinline__ void merge_weights(const float* plse, int np, float m, float l,
                                              float& wown, float (&wp)[kMaxTopk], float& inv) {
  float lse[kMaxTopk];
  float M = m + __log2f(l);  // key t itself is always visible: l > 0
  const float lown = M;
#pragma unroll
  for (int s = 0; s < kMaxTopk - 1; ++s) {
    lse[s] = s < np ? plse[s] : -INFINITY;
    M = fmaxf(M, lse[s]);
  }
  wown = exp2f(lown - M) / l;
  float wsum = exp2f(lown - M);
#pragma unroll
  for (int s = 0; s < kMaxTopk - 1; ++s) {
    wp[s] = s < np ? exp2f(lse[s] - M) : 0.f;
    wsum += wp[s];
  }
  inv = 1.f / wsum;
}

__device__ __forceinline__ void store_row16(__nv_bfloat16* dst, const float (&acc)[16], float inv) {
  uint4 pk[2];
  uint32_t* pw = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
  for (int e = 0; e < 8; ++e) pw[e] = ptx::pack_bf16(acc[2 * e] * inv, acc[2 * e + 1] * inv);
  reinterpret_cast<uint4*>(dst)[0] = pk[0];
  reinterpret_cast<uint4*>(dst)[1] = pk[1];
}

__device__ __forceinline__ void add_partial(float (&acc)[16], float w, uint4 a0, uint4 a1) {
  const __nv_bfloat162* e0 = reinterpret_cast<const __nv_bfloat162*>(&a0);
  const __nv_bfloat162* e1 = reinterpret_cast<const __nv_bfloat162*>(&a1);
#pragma unroll
  for (int y = 0; y < 4; ++y) {
    const float2 f = __bfloat1622float2(e0[y]), g = __bfloat1622float2(e1[y]);
    acc[2 * y] = fmaf(w, f.x, acc[2 * y]);
    acc[2 * y + 1] = fmaf(w, f.y, acc[2 * y + 1]);
    acc[8 + 2 * y] = fmaf(w, g.x, acc[8 + 2 * y]);
    acc[8 + 2 * y + 1] = fmaf(w, g.y, acc[8 + 2 * y + 1]);
  }
}

// The hand-offs of item k to a merge warp: the row's (m, l) from the softmax
// warps (then released), and O[k & 1] once the item's last PV MMA is done.
struct OwnHandoff {
  Bars* bars;
  volatile int* abort;
  unsigned* err;
  const float2* ml_s;
  __device__ __forceinline__ float2 take_ml(int k, int row) const {
    wait_or_abort(&bars->ml_full, (uint32_t)(k & 1), abort, err);
    const float2 ml = ml_s[row];
    ptx::mbar_arrive(&bars->ml_free);
    return ml;
  }
  __device__ __forceinline__ void wait_o(int k) const {
    wait_or_abort(&bars->o_full[k & 1], (uint32_t)((k >> 1) & 1), abort, err);
    tc::fence_after_sync();
  }
  __device__ __forceinline__ void release_o(int k) const {
    tc::fence_before_sync();
    ptx::mbar_arrive(&bars->o_free[k & 1]);
  }
};

// Up to two partials (top_k <= 3): the rows' log2-sum-exps and the first
// 64 columns of both rows are loaded before the item's O is waited for, the
// second 64 columns while the first are merged (two waits for memory, off the
// softmax warps' path).
__device__ __forceinline__ void own_merge_preloaded(const MobaTcArgs& a, const OwnHandoff& hf,
                                                    uint32_t to, int k, int row, size_t prow,
                                                    int np, bool live, __nv_bfloat16* dst) {
  const uint4* s0 = reinterpret_cast<const uint4*>(a.po + prow * D);
  uint4 p0[8], p1[8];
  auto load_half = [&](int hv) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      p0[c] = np > 0 ? __ldg(s0 + 8 * hv + c) : make_uint4(0, 0, 0, 0);
      p1[c] = np > 1 ? __ldg(s0 + 16 + 8 * hv + c) : make_uint4(0, 0, 0, 0);
    }
  };
  float pl[kMaxTopk];
#pragma unroll
  for (int s = 0; s < kMaxTopk; ++s) pl[s] = s < np ? a.plse[prow + s] : -INFINITY;
  load_half(0);
  const float2 ml = hf.take_ml(k, row);
  float wown, wp[kMaxTopk], inv;
  merge_weights(pl, np, ml.x, ml.y, wown, wp, inv);
  hf.wait_o(k);
#pragma unroll 1
  for (int hv = 0; hv < 2; ++hv) {
    if (hv == 1) load_half(1);
#pragma unroll
    for (int c32 = 0; c32 < 2; ++c32) {
      uint32_t o[32];
      tc::ld32_sync(to + hv * 64 + c32 * 32, o);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int c = 2 * c32 + h2;  // 16-column chunk within the half
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = __uint_as_float(o[16 * h2 + e]) * wown;
        add_partial(acc, wp[0], p0[2 * c], p0[2 * c + 1]);
        add_partial(acc, wp[1], p1[2 * c], p1[2 * c + 1]);
        if (live) store_row16(dst + hv * 64 + c * 16, acc, inv);
      }
    }
  }
  hf.release_o(k);
}

// Any number of partials: 16 columns at a time (two chunks' loads in flight).
__device__ __forceinline__ void own_merge_chunked(const MobaTcArgs& a, const OwnHandoff& hf,
                                                  uint32_t to, int k, int row, size_t prow,
                                                  int np, bool live, __nv_bfloat16* dst) {
  if (np > 0) ptx::bulk_prefetch_l2(a.po + prow * D, (uint32_t)(np * D * 2));
  const float2 ml = hf.take_ml(k, row);
  float wown, wp[kMaxTopk], inv;
  merge_weights(a.plse + prow, np, ml.x, ml.y, wown, wp, inv);
  hf.wait_o(k);
#pragma unroll 2
  for (int c16 = 0; c16 < 8; ++c16) {
    uint32_t o[16];
    tc::ld16_sync(to + c16 * 16, o);
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = __uint_as_float(o[e]) * wown;
#pragma unroll
    for (int s = 0; s < kMaxTopk - 1; ++s) {
      if (s >= np) break;
      const uint4* ps = reinterpret_cast<const uint4*>(a.po + (prow + s) * D + c16 * 16);
      add_partial(acc, wp[s], __ldg(ps), __ldg(ps + 1));
    }
    if (live) store_row16(dst + c16 * 16, acc, inv);
  }
  hf.release_o(k);
}

// Persistent, one CTA per SM: lanes 0-3 of warp 0 load the query tiles (two
// buffers, lane 0) and the K / V tiles (a four-stage ring), warp 1 lane 0
// issues the MMAs, warps 2-5 run the softmax, warps 6-9 the merge with the
// partials, so one item's merge overlaps the next item's softmax.
__global__ void __launch_bounds__(kBlkThreads, 1)
    moba_own_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, const MobaTcArgs a) {
  extern __shared__ unsigned char smraw[];
  unsigned char* base = align1024(smraw);
  unsigned char* sQ = base;  // 2 x 32 KB
  unsigned char* ring = base + 2 * TILE;
  Bars* bars = reinterpret_cast<Bars*>(ring + kStages * TILE);
  float2* ml_s = reinterpret_cast<float2*>(bars + 1);  // [row]
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NI = a.B * a.Hq * ((a.T + KT - 1) / KT);
  const int G = a.Hq / a.Hkv;

  if (threadIdx.x == 0) init_bars(bars, 1);
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = bars->tmem;

  if (warp == 0) {
    if (lane < kStages) {
      if (lane == 0) {
        ptx::prefetch_tmap(&tq);
        ptx::prefetch_tmap(&tk);
        ptx::prefetch_tmap(&tv);
      }
      Producer pr{ring, bars, abort, a.err, lane};
      const uint64_t first = ptx::policy_evict_first(), keep = ptx::policy_evict_last();
      int kq = 0, lastq[2] = {-1, -1};
      for (int i = blockIdx.x; pr.ok && i < NI; i += gridDim.x, ++kq) {
        const OwnItem it = own_item(a, i);
        if (lane == 0) {
          const int qb = kq & 1;
          if (kq >= 2 &&
              !wait_or_abort(&bars->q_free[qb], (uint32_t)(((kq >> 1) - 1) & 1), abort, a.err)) {
            pr.ok = false;
            break;
          }
          unsigned char* qd = sQ + qb * TILE;
          ptx::mbar_arrive_expect_tx(&bars->q_full[qb], TILE);
          ptx::tma_load_3d(qd, &tq, &bars->q_full[qb], 0, it.h, it.b * a.T + it.t0, first);
          ptx::tma_load_3d(qd + ATOM, &tq, &bars->q_full[qb], 64, it.h, it.b * a.T + it.t0,
                           first);
          lastq[qb] = kq;
        }
        const int g = it.h / G, z0 = it.b * a.T + it.c0;
        for (int u = 0; u < it.nk; ++u) {
          pr.load(&tk, g, z0 + u * KT, keep);
          if (u >= 1) pr.load(&tv, g, z0 + (u - 1) * KT, keep);
        }
        pr.load(&tv, g, z0 + (it.nk - 1) * KT, keep);
      }
      pr.drain();
      if (lane == 0)  // every issued query load lands before the CTA can exit
        for (int s = 0; s < 2; ++s)
          if (lastq[s] >= 0 &&
              !ptx::mbar_wait(&bars->q_full[s], (uint32_t)((lastq[s] >> 1) & 1), kWaitNs))
            atomicOr(a.err, kErrTimeout);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      Mma mm{bars, abort, a.err, tmem, ptx::smem_u32(ring)};
      int kq = 0;
      for (int i = blockIdx.x; mm.ok && i < NI; i += gridDim.x, ++kq) {
        const OwnItem it = own_item(a, i);
        const int qb = kq & 1;
        mm.ok = wait_or_abort(&bars->q_full[qb], (uint32_t)((kq >> 1) & 1), abort, a.err);
        tc::fence_after_sync();
        mm.tile(ptx::smem_u32(sQ + qb * TILE), it.nk, qb, kq);
      }
      tc::commit(&bars->fin);
      if (!ptx::mbar_wait(&bars->fin, 0, kWaitNs)) atomicOr(a.err, kErrTimeout);
    }
  } else if (warp < 6) {
    // softmax warps: item after item, O of item k in O[k & 1]; each row's
    // (m, l) goes to the merge warps through shared memory
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    Softmax sm{bars, abort, a.err, tmem + ((uint32_t)(qd * 32) << 16), a.c};
    int k = 0;
    for (int i = blockIdx.x; i < NI; i += gridDim.x, ++k) {
      const OwnItem it = own_item(a, i);
      const int t = min(it.t0 + row, a.T - 1);
      sm.obuf = (k & 1) ? kO2 : kO;
      float m = -INFINITY, l = 0.f;
      sm.run(it.nk, it.c0, t + 1, m, l);
      if (k >= 1)  // the merge warps have read item k - 1's
        wait_or_abort(&bars->ml_free, (uint32_t)((k - 1) & 1), abort, a.err);
      ml_s[row] = make_float2(m, l);
      ptx::mbar_arrive(&bars->ml_full);
    }
  } else {
    // merge warps: item k's row, from O[k & 1] and its partials
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
    const OwnHandoff hf{bars, abort, a.err, ml_s};
    int k = 0;
    for (int i = blockIdx.x; i < NI; i += gridDim.x, ++k) {
      const OwnItem it = own_item(a, i);
      const int t = min(it.t0 + row, a.T - 1);
      const bool live = it.t0 + row < a.T;
      const int np = live ? min(a.topk - 1, t / a.m) : 0;
      const size_t prow = ((size_t)(it.b * a.T + t) * a.Hq + it.h) * (a.topk - 1);
      __nv_bfloat16* dst = a.out + ((size_t)(it.b * a.T + t) * a.Hq + it.h) * D;
      const uint32_t to = tl + ((k & 1) ? kO2 : kO);
      if (a.topk <= 3)
        own_merge_preloaded(a, hf, to, k, row, prow, np, live, dst);
      else
        own_merge_chunked(a, hf, to, k, row, prow, np, live, dst);
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

size_t attn_smem(int qbufs) { return 1024 + (size_t)(qbufs + kStages) * TILE + sizeof(Bars); }
// Both attention kernels: + the (m, l) hand-off of each row (one buffer: the
// kernels then stay within the 196 KB shared-memory configuration, which
// leaves the SM more L1)
size_t blk_smem() { return attn_smem(2) + KT * sizeof(float2); }


size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

bool moba_tc_eligible(const nsa_params& p) {
  if (p.dtype != NSA_DTYPE_BF16 || p.d != D || p.Hkv < 1 || p.Hq % p.Hkv != 0) return false;
  if (p.sel_block < KT || p.sel_block % KT != 0 || p.sel_block > 2048) return false;
  if (p.top_n < 1 || p.top_n > kMaxTopk) return false;
  return (long long)p.B * p.T * p.Hq < (1ll << 31) / D && (long long)p.B * p.T < (1ll << 30) / 8;
}

// Workspace after the block means: selection (when the caller passes none),
// bucket counts / offsets / tile offsets / cursors, the bucket rows, the
// partial outputs and their log-sum-exp, the split block means, and the
// descriptor of each bucket tile (at most one partial tile per bucket beyond
// rows / 128 full ones).
size_t moba_tc_ws_bytes(const nsa_params& p, size_t kbar_bytes) {
  const size_t rows = (size_t)p.B * p.T * p.Hq;
  const size_t NB = (size_t)p.B * p.Hq * (p.T / p.sel_block);
  const size_t np = (size_t)(p.top_n - 1);
  const size_t parts = (size_t)p.B * p.Hkv * 3 * gate_rows(p.T / p.sel_block) * D * 2;
  return align256(kbar_bytes) + align256(rows * p.top_n * 4) + 4 * align256((NB + 1) * 4) +
         align256(rows * np * 4 + 4) + align256(rows * np * D * 2 + 4) + align256(rows * np * 4 + 4) +
         align256(parts + 4) + align256((NB + rows * np / KT + 2) * 16);
}

cudaError_t launch_moba_tc(const nsa_params& p, const void* q, const void* k, const void* v,
                           void* out, int32_t* sel_out, void* ws, size_t kbar_bytes,
                           unsigned* err, cudaStream_t stream) {
  MobaTcArgs a{};
  const size_t rows = (size_t)p.B * p.T * p.Hq;
  a.B = p.B;
  a.T = p.T;
  a.Hq = p.Hq;
  a.Hkv = p.Hkv;
  a.m = p.sel_block;
  a.topk = p.top_n;
  a.nfull = p.T / p.sel_block;
  a.NB = p.B * p.Hq * a.nfull;
  const size_t np = (size_t)(p.top_n - 1);
  unsigned char* w = static_cast<unsigned char*>(ws);
  a.kbar = reinterpret_cast<const float*>(w);
  w += align256(kbar_bytes);
  int32_t* selws = reinterpret_cast<int32_t*>(w);
  w += align256(rows * p.top_n * 4);
  a.sel = sel_out ? sel_out : selws;
  a.cnt = reinterpret_cast<int32_t*>(w);
  w += align256(((size_t)a.NB + 1) * 4);
  a.off = reinterpret_cast<int32_t*>(w);
  w += align256(((size_t)a.NB + 1) * 4);
  a.toff = reinterpret_cast<int32_t*>(w);
  w += align256(((size_t)a.NB + 1) * 4);
  a.cur = reinterpret_cast<int32_t*>(w);
  w += align256(((size_t)a.NB + 1) * 4);
  a.list = reinterpret_cast<int32_t*>(w);
  w += align256(rows * np * 4 + 4);
  a.po = reinterpret_cast<__nv_bfloat16*>(w);
  w += align256(rows * np * D * 2 + 4);
  a.plse = reinterpret_cast<float*>(w);
  w += align256(rows * np * 4 + 4);
  a.kparts = reinterpret_cast<__nv_bfloat16*>(w);
  w += align256((size_t)p.B * p.Hkv * 3 * gate_rows(a.nfull) * D * 2 + 4);
  a.tdesc = reinterpret_cast<int4*>(w);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.err = err;
  const float scale = p.softmax_scale > 0.f ? p.softmax_scale : 1.f / sqrtf((float)p.d);
  a.c = scale * 1.4426950408889634f;

  const uint64_t BT = (uint64_t)p.B * p.T;
  CUtensorMap tq, tk, tv, tp;
  if (!make_tmap_bf16_3d(&tq, q, D, p.Hq, BT, 64, 1, KT, true) ||
      !make_tmap_bf16_3d(&tp, a.kparts, D, gate_rows(a.nfull), (uint64_t)p.B * p.Hkv * 3, 64,
                         kGateBox, 1, true) ||
      !make_tmap_bf16_3d(&tk, k, D, p.Hkv, BT, 64, 1, KT, true) ||
      !make_tmap_bf16_3d(&tv, v, D, p.Hkv, BT, 64, 1, KT, true))
    return cudaErrorInvalidValue;

  cudaError_t e;
  if (a.NB > 0 && (e = cudaMemsetAsync(a.cnt, 0, (size_t)a.NB * 4, stream)) != cudaSuccess) return e;
  if (a.nfull > 0) {
    TraceScope trace("moba_split", stream);
    const size_t n4 = (size_t)a.B * a.Hkv * gate_rows(a.nfull) * (D / 4);
    const int grid = (int)std::min<size_t>((n4 + 255) / 256, (size_t)device_sm_count() * 8);
    moba_split_kernel<<<grid, 256, 0, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    TraceScope trace("moba_gate", stream);
    if ((e = ensure_dyn_smem((const void*)moba_gate_kernel, (int)gate_smem())) != cudaSuccess)
      return e;
    const long long items = (long long)p.B * p.Hq * ((p.T + KT - 1) / KT);
    const int grid = (int)std::min<long long>(items, device_sm_count());
    moba_gate_kernel<<<grid, kThreads, gate_smem(), stream>>>(tq, tp, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.NB > 0 && p.top_n > 1) {
    {
      TraceScope trace("moba_scan", stream);
      moba_scan_kernel<<<1, 1024, 0, stream>>>(a);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
      TraceScope trace("moba_fill", stream);
      const long long n = (long long)rows;
      const int grid = (int)std::min<long long>((n + 255) / 256, (long long)device_sm_count() * 8);
      moba_fill_kernel<<<grid, 256, 0, stream>>>(a);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
      const size_t sm = blk_smem();
      if ((e = ensure_dyn_smem((const void*)moba_blk_kernel, (int)sm)) != cudaSuccess) return e;
      TraceScope trace("moba_blk", stream);
      moba_blk_kernel<<<device_sm_count(), kBlkThreads, sm, stream>>>(tk, tv, a);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  {
    const size_t sm = blk_smem();
    if ((e = ensure_dyn_smem((const void*)moba_own_kernel, (int)sm)) != cudaSuccess) return e;
    TraceScope trace("moba_own", stream);
    const long long items = (long long)p.B * p.Hq * ((p.T + KT - 1) / KT);
    const int grid = (int)std::min<long long>(items, device_sm_count());
    moba_own_kernel<<<grid, kBlkThreads, sm, stream>>>(tq, tk, tv, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace nsa
