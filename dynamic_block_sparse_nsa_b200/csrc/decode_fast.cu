// NSA single-token decode, bf16, head dim 128, 16 query heads per KV head
// (the GQA group fills the 16 rows of one m16n8k16 tensor-core tile), selection
// blocks of 64 tokens.
//
// Decode moves the group's one shared KV subset and is bound by HBM bytes
// (EP94 notes §六; lchairun.cn NSA article, decode paragraph). Four kernels,
// each launched to be scheduled while its predecessor drains (programmatic
// dependent launch; each waits for the predecessor's writes first):
//
//  dec_cmp_partial  stream kernel over the compressed keys (see below); also
//                   writes, per 32-key sub-tile and head, the running max it
//                   used and the exp-sums of its keys per overlapped selection
//                   block, because block scores need probabilities normalised
//                   by the final lse, which is known only at the end.
//  dec_select       one CTA per (sequence, KV head): merges the partials' (m, l)
//                   into the lse, rescales the sub-tile records into block
//                   scores summed over the group's heads, keeps block 0 plus
//                   the top n-1 others (ties to the lower index).
//  dec_sel_win      stream kernel over the selected blocks, then the window.
//  dec_combine      merges the partials of all three branches, computes the
//                   gates: out = g0 o_cmp + g1 o_slc + g2 o_win.
//
// Stream kernel: persistent, one CTA per SM, 4 pairs of consumer warps, each
// pair fed by its own TMA producer warp. The global sequence of 64-key tiles (sequence-major, then KV
// head, then tile) is split evenly over the SMs x 4 pair streams; each pair has
// a private ring of three 16 KB slots (K or V of a tile, 128B-swizzled TMA
// boxes, L2 evict-first) so no stream waits on another's slot. The two warps
// of a pair take 32 keys each of every tile and keep online-softmax partials
// (m, l, O), written once per segment they touch (segment = unit, or unit and
// branch).
// Softmax runs in the log2 domain: z2 = (q . k) * scale * log2(e).
#include <algorithm>
#include <climits>
#include <utility>

#include "device_common.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace nsa {
namespace {

constexpr int G = 16;                       // query heads per KV head
constexpr int D = 128;                      // head dim
constexpr int TK = 64;                      // keys per tile
constexpr int HALF_BYTES = TK * 64 * 2;     // 64 rows x 64 dims of bf16 (one TMA box)
constexpr int SLOT_BYTES = 2 * HALF_BYTES;  // 64 keys x 128 dims
constexpr int PART = 2 * G + G * D / 2;     // floats: m[16], l[16], then o[16][128] in bf16
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
// consumer math (one warp: 16 heads x 32 keys of a 64-key tile)
// ---------------------------------------------------------------------------

constexpr int WK = 32;  // keys per consumer warp per tile (two warps share a tile)

// S[16 x 8*NT] = Q K^T with the query block in shared memory (row r's 16-byte
// chunk c stored at chunk c ^ (r & 7)); even and odd k-steps accumulate in
// separate registers so consecutive tensor-core ops do not wait on each other.
template <int NT>
__device__ __forceinline__ void qk_tile_q(float (&s)[NT][4], uint32_t qbase, uint32_t kbase,
                                          int key0, int lane) {
  float t[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) s[nt][i] = t[nt][i] = 0.f;
  const int mi = lane >> 3, r = lane & 7;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    uint32_t qa[4];
    {
      const int row = (mi & 1) * 8 + r;
      const int chunk = 2 * ks + (mi >> 1);
      ptx::ldsm_x4(qbase + row * 256 + ((chunk ^ (row & 7)) << 4), qa[0], qa[1], qa[2], qa[3]);
    }
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      const int key = key0 + (2 * np + (mi >> 1)) * 8 + r;
      const int chunk = 2 * ks + (mi & 1);
      const uint32_t addr =
          kbase + (chunk >> 3) * HALF_BYTES + key * 128 + (((chunk & 7) ^ (key & 7)) << 4);
      uint32_t b0, b1, b2, b3;
      ptx::ldsm_x4(addr, b0, b1, b2, b3);
      if (ks & 1) {
        ptx::mma_16816(t[2 * np], qa, b0, b1);
        ptx::mma_16816(t[2 * np + 1], qa, b2, b3);
      } else {
        ptx::mma_16816(s[2 * np], qa, b0, b1);
        ptx::mma_16816(s[2 * np + 1], qa, b2, b3);
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) s[nt][i] += t[nt][i];
}

// The 16 x 128 query block of a unit into shared memory (swizzled as above);
// the two warps of a pair copy 8 rows each.
__device__ __forceinline__ void stage_q_half(unsigned char* qs, const __nv_bfloat16* q, int hw,
                                             int lane) {
  const uint4* src = reinterpret_cast<const uint4*>(q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int x = hw * 128 + i * 32 + lane;  // 16-byte chunk: row x / 16, chunk x % 16
    const int r = x >> 4, c = x & 15;
    *reinterpret_cast<uint4*>(qs + r * 256 + ((c ^ (r & 7)) << 4)) = __ldg(src + x);
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

// Online-softmax step over NT n-tiles (8 keys each): mask keys >= nvalid,
// scale to the log2 domain, update running max/sum of rows r0 = lane/4 and
// r1 = r0 + 8, rescale O, and turn s into p = exp2(z - m_new).
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

// As softmax_step, but the running max only moves when some row's tile max
// exceeds it by more than 8 (log2 units): below that, p = exp2(z - m) <= 256
// stays well inside fp32 and bf16, the normalisation by l stays exact, and the
// common case skips rescaling the accumulators.
template <int NT>
__device__ __forceinline__ void softmax_step_lazy(float (&s)[NT][4], float (&o)[16][4], float& m0,
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
  const bool grow = mx0 > m0 + 8.f || mx1 > m1 + 8.f;
  if (__any_sync(0xffffffffu, grow)) {
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float c0 = exp2f(m0 - mn0), c1 = exp2f(m1 - mn1);  // 0 when m was -inf
    l0 *= c0;
    l1 *= c1;
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      o[dt][0] *= c0;
      o[dt][1] *= c0;
      o[dt][2] *= c1;
      o[dt][3] *= c1;
    }
    m0 = mn0;
    m1 = mn1;
  }
  float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      s[nt][e] = exp2f(s[nt][e] - m0);
      s[nt][2 + e] = exp2f(s[nt][2 + e] - m1);
      sum0 += s[nt][e];
      sum1 += s[nt][2 + e];
    }
  l0 += quad_sum(sum0);
  l1 += quad_sum(sum1);
}

// Score record of a warp's 32-key compressed sub-tile straight from the
// probabilities in registers, for a compressed block of two strides and a
// selection block of four (l = 2s, bs = 4s): selection block jl of the
// sub-tile then takes keys 4jl-1 .. 4jl+3 (key -1 and keys past 31 absent),
// i.e. the 4-key group jl plus the last key of group jl-1 (blocks 8 and 9 keep
// key 31 alone and nothing). In the accumulator layout lane quad q holds keys
// 8nt + 2q, 8nt + 2q + 1 of rows r0 and r0 + 8, so a group is a lane pair and
// the extra key one shuffle away. Writes rec[h] = m (running max) and
// rec[16 (1 + jl) + h] = the block's exp-sum, as the shared-memory path does.
__device__ __forceinline__ void record_regs(float* rec, const float (&p)[4][4], float m0, float m1,
                                            int lane) {
  const int q = lane & 3, r0 = lane >> 2, base = lane & ~3;
  float* blk = rec + G;
  float prev0 = 0.f, prev1 = 0.f;  // last key of group 2nt - 1 (rows r0, r0 + 8)
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    float g0 = p[nt][0] + p[nt][1], g1 = p[nt][2] + p[nt][3];
    g0 += __shfl_xor_sync(0xffffffffu, g0, 1);  // group 2nt + q / 2
    g1 += __shfl_xor_sync(0xffffffffu, g1, 1);
    const float ea0 = __shfl_sync(0xffffffffu, p[nt][1], base | 1);  // key 8nt + 3
    const float ea1 = __shfl_sync(0xffffffffu, p[nt][3], base | 1);
    const float eb0 = __shfl_sync(0xffffffffu, p[nt][1], base | 3);  // key 8nt + 7
    const float eb1 = __shfl_sync(0xffffffffu, p[nt][3], base | 3);
    if (q == 0) {
      blk[(2 * nt) * G + r0] = g0 + prev0;
      blk[(2 * nt) * G + r0 + 8] = g1 + prev1;
    } else if (q == 2) {
      blk[(2 * nt + 1) * G + r0] = g0 + ea0;
      blk[(2 * nt + 1) * G + r0 + 8] = g1 + ea1;
    }
    prev0 = eb0;
    prev1 = eb1;
  }
  if (q == 0) {
    blk[8 * G + r0] = prev0;
    blk[8 * G + r0 + 8] = prev1;
    rec[r0] = m0;
    rec[r0 + 8] = m1;
  } else if (q == 2) {
    blk[9 * G + r0] = 0.f;
    blk[9 * G + r0 + 8] = 0.f;
  }
}

// ---------------------------------------------------------------------------
// global tile order and its even split over the pair streams
// ---------------------------------------------------------------------------

struct StreamPlan {
  int len;  // 64-key tiles of this stream
  int b, g, tile, ntiles;
};

// Walk of the global tile order (sequence-major, then KV head, then tile),
// caching the current sequence's length and selected-block count. `lens`
// points at the sequence lengths (a shared-memory copy when it fits).
template <int MODE>
struct Walker {
  int b, g, tile, ntiles, L, ns;
  __device__ void init(const DecFastArgs& a, const int* lens, const StreamPlan& p) {
    b = p.b;
    g = p.g;
    tile = p.tile;
    ntiles = p.ntiles;
    L = lens[b];
    ns = n_selected(L, a);
  }
  __device__ void advance(const DecFastArgs& a, const int* lens) {
    if (++tile < ntiles) return;
    tile = 0;
    if (++g < a.Hkv) return;
    g = 0;
    do {
      ++b;
      L = b < a.B ? lens[b] : 1;
      ntiles = b < a.B ? unit_tiles<MODE>(L, a) : 1;
    } while (ntiles == 0);
    ns = n_selected(L, a);
  }
  __device__ int segment(const DecFastArgs& a) const {
    const int u = b * a.Hkv + g;
    return MODE == MODE_CMP ? u : 2 * u + (tile >= ns ? 1 : 0);
  }
};

constexpr int LENS_CAP = 1024;  // sequence lengths kept in shared memory

// Plans of the NS streams of this CTA (computed by one warp). Stream
// v = cta * NS + i owns global tiles [total*v/V, total*(v+1)/V), where
// V = min(all streams, total) (streams v >= V are idle). `pre` is
// scratch for the per-sequence prefix of tile counts (cap entries); `lens_s`
// receives a copy of the lengths when B <= LENS_CAP.
template <int MODE, int NS>
__device__ void make_plans(const DecFastArgs& a, StreamPlan* plans, int* lens_s, long long* pre,
                           int cap, int lane) {
  const bool cached = a.B <= LENS_CAP;
  const bool use_pre = a.B + 1 <= cap;
  long long carry = 0;
  if (use_pre && lane == 0) pre[0] = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    const int L = b < a.B ? __ldg(a.seq_lens + b) : 0;
    if (cached && b < a.B) lens_s[b] = L;
    long long x = b < a.B ? (long long)unit_tiles<MODE>(L, a) * a.Hkv : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {  // inclusive warp scan
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (use_pre && b < a.B) pre[b + 1] = carry + x;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  __syncwarp();
  const long long total = carry;
  // At most one stream per tile: then every stream owns at least one tile, so
  // the streams between a segment's first and last owner all wrote partials.
  const long long V = min((long long)gridDim.x * NS, total);
  if (lane < NS) {
    const long long v = (long long)blockIdx.x * NS + lane;
    const long long t0 = v < V ? total * v / V : 0, t1 = v < V ? total * (v + 1) / V : 0;
    StreamPlan p{};
    p.len = (int)(t1 - t0);
    p.ntiles = 1;
    if (t1 > t0) {
      int b;
      long long acc;
      if (use_pre) {  // first b with pre[b + 1] > t0
        int lo = 0, hi = a.B - 1;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (pre[mid + 1] > t0) hi = mid;
          else lo = mid + 1;
        }
        b = lo;
        acc = pre[b];
      } else {
        acc = 0;
        for (b = 0; b < a.B; ++b) {
          const long long span = (long long)unit_tiles<MODE>(__ldg(a.seq_lens + b), a) * a.Hkv;
          if (t0 < acc + span) break;
          acc += span;
        }
      }
      const int nt = unit_tiles<MODE>(__ldg(a.seq_lens + b), a);
      const long long off = t0 - acc;
      p.b = b;
      p.g = (int)(off / nt);
      p.tile = (int)(off % nt);
      p.ntiles = nt;
    }
    plans[lane] = p;
  }
}

// Streams holding unit u's tiles in a stream kernel's plan, from the lengths
// alone (the split of make_plans): with `pre` the tiles of the units before u,
// `nt` its own, `total` all tiles and V the streams in use, stream v owns
// [total v / V, total (v + 1) / V), so tile x lies in stream
// ceil((x + 1) V / total) - 1.
__device__ __forceinline__ int stream_of_tile(long long x, long long V, long long total) {
  return (int)(((x + 1) * V - 1) / total);
}

// Block-wide: tiles (times Hkv) of the sequences before b and of all
// sequences, for both stream kernels. `red` holds 4 * (threads / 32) entries.
// Reads only the sequence lengths (an input of the call).
__device__ void tile_spans(const DecFastArgs& a, int b, long long (&pre)[2], long long (&total)[2],
                           long long* red) {
  long long acc[4] = {0, 0, 0, 0};
  for (int i = threadIdx.x; i < a.B; i += blockDim.x) {
    const int L = __ldg(a.seq_lens + i);
    const long long x0 = (long long)unit_tiles<MODE_CMP>(L, a) * a.Hkv;
    const long long x1 = (long long)unit_tiles<MODE_SW>(L, a) * a.Hkv;
    acc[2] += x0;
    acc[3] += x1;
    if (i < b) {
      acc[0] += x0;
      acc[1] += x1;
    }
  }
  const int nw = blockDim.x >> 5, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], o);
    if (lane == 0) red[k * nw + w] = acc[k];
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    long long v = 0;
    for (int i = 0; i < nw; ++i) v += red[k * nw + i];
    acc[k] = v;
  }
  pre[0] = acc[0];
  pre[1] = acc[1];
  total[0] = acc[2];
  total[1] = acc[3];
}

// ---------------------------------------------------------------------------
// the stream kernel
// ---------------------------------------------------------------------------

constexpr int NPAIR = 4;              // consumer warp pairs = tile streams per CTA
constexpr int PSLOTS = 3;             // ring slots per pair: K and V of a tile + one ahead
constexpr int SLOTS = NPAIR * PSLOTS;
constexpr int NCW = 2 * NPAIR;        // consumer warps
constexpr int NPW = NPAIR;            // producer warps, one per pair
constexpr int STREAM_THREADS = (NCW + NPW) * 32;
constexpr int RPITCH = WK + 2;        // record scratch pitch (floats)
constexpr int QBYTES = G * D * 2;     // query block of a pair

template <int MODE>
struct StreamCfg {
  static constexpr size_t SMEM = 1024 + (size_t)SLOTS * SLOT_BYTES + NPAIR * QBYTES +
                                 2 * SLOTS * 8 + SLOTS * 4 + NPAIR * sizeof(StreamPlan) + 64 +
                                 LENS_CAP * 4;
};

struct TileSrc {
  int row;     // TMA row (outer coordinate)
  int nvalid;  // valid keys in the 64-key tile
};

template <int MODE>
__device__ __forceinline__ TileSrc tile_source(const DecFastArgs& a, const Walker<MODE>& wk) {
  TileSrc ts;
  if (MODE == MODE_CMP) {
    ts.row = wk.b * a.Nc + wk.tile * TK;
    ts.nvalid = min(TK, n_visible(wk.L, a.l, a.s, a.Nc) - wk.tile * TK);
  } else {
    const int t = wk.L - 1;
    int start;
    bool unused = false;
    if (wk.tile < wk.ns) {
      // adaptive selection may keep fewer than n blocks: unused slots hold -1
      const int blk = __ldg(a.sel + (long)(wk.b * a.Hkv + wk.g) * a.n + wk.tile);
      unused = blk < 0;
      start = unused ? 0 : blk * a.bs;
    } else {
      start = t - min(a.w, wk.L) + 1 + (wk.tile - wk.ns) * TK;
    }
    ts.row = wk.b * a.T + start;
    ts.nvalid = unused ? 0 : min(TK, t - start + 1);
  }
  return ts;
}

// Write one warp's (m, l, unnormalised O) partial straight to global: m and l
// in fp32, O in bf16 (half the bytes the merge reads back; each partial then
// carries a relative rounding of 2^-9, the output's own precision).
__device__ __forceinline__ void store_partial(float* dst, int lane, float m0, float m1, float l0,
                                              float l1, const float (&o)[16][4]) {
  const int r0 = lane >> 2, c = (lane & 3) * 2;
  if ((lane & 3) == 0) {
    dst[r0] = m0;
    dst[r0 + 8] = m1;
    dst[G + r0] = l0;
    dst[G + r0 + 8] = l1;
  }
  __nv_bfloat16* po = reinterpret_cast<__nv_bfloat16*>(dst + 2 * G);
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) {
    *reinterpret_cast<__nv_bfloat162*>(po + r0 * D + dt * 8 + c) =
        __floats2bfloat162_rn(o[dt][0], o[dt][1]);
    *reinterpret_cast<__nv_bfloat162*>(po + (r0 + 8) * D + dt * 8 + c) =
        __floats2bfloat162_rn(o[dt][2], o[dt][3]);
  }
}

// One CTA per SM: warps 0..7 are four pairs of consumers, warps 8..11 the TMA
// producers (one per pair). Pair p streams its own range of 64-key tiles
// through its own ring of three 16 KB slots (K and V of the current tile and
// the K of the next); warp h of the pair handles keys [32h, 32h + 32) of every
// tile, with its own online softmax state, and writes its partial to slot
// 2 * (stream + segment) + h. Every consumer takes part in every phase of its
// pair's slots, so the mbarrier phase parity is always unambiguous.
template <int MODE, bool RF>
__global__ void __launch_bounds__(STREAM_THREADS, 1)
    dec_stream_kernel(const __grid_constant__ DecFastArgs a, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv) {
  using C = StreamCfg<MODE>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* slots = smem;
  unsigned char* qsm = slots + SLOTS * SLOT_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(qsm + NPAIR * QBYTES);
  uint64_t* empty = full + SLOTS;
  int* info = reinterpret_cast<int*>(empty + SLOTS);
  StreamPlan* plans = reinterpret_cast<StreamPlan*>(info + SLOTS);
  int* abort_flag = reinterpret_cast<int*>(plans + NPAIR);
  int* lens_s = abort_flag + 1;  // [LENS_CAP]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The compressed-branch kernel's predecessor is the caller's: it waits
  // before reading anything. The selected/window kernel's predecessors are
  // this library's own, which waited on the caller's writes already, so its
  // plan (from the sequence lengths, an input) is made before the wait.
  if (MODE == MODE_CMP) ptx::grid_dep_wait();
  // The next decode kernel may be scheduled as this grid's CTAs finish (this
  // grid is resident in full: one CTA per SM), so its input-only set-up
  // overlaps this grid's tail; it waits for this grid before reading its output.
  ptx::grid_dep_launch();
  if (warp == NCW) {
    // the slot ring is idle until the pipeline starts: use it as plan scratch
    make_plans<MODE, NPAIR>(a, plans, lens_s, reinterpret_cast<long long*>(slots),
                            SLOTS * SLOT_BYTES / 8, lane);
    if (lane == 0) {
      for (int i = 0; i < SLOTS; ++i) {
        ptx::mbar_init(&full[i], 1);
        ptx::mbar_init(&empty[i], 2);
      }
      *abort_flag = 0;
      ptx::fence_mbar_init();
      ptx::prefetch_tmap(&tk);
      ptx::prefetch_tmap(&tv);
    }
  }
  if (MODE != MODE_CMP) ptx::grid_dep_wait();  // the selection, and this kernel's workspace
  __syncthreads();
  const int* lens_p = a.B <= LENS_CAP ? lens_s : a.seq_lens;
  float* part = MODE == MODE_CMP ? a.part1 : a.part3;

  if (warp >= NCW) {
    // ---------------- producers: warp NCW + p fills pair p's ring ----------------
    // Lanes 0 and 1 each issue one 8 KB box of every half-tile: TMA ingest
    // grows with the number of issuing threads, and one thread for all rings
    // is slower than the HBM share of an SM.
    const int p = warp - NCW;
    if (lane >= 2) return;
    const uint64_t pol = ptx::policy_evict_first();
    const int hend = 2 * plans[p].len;
    if (hend == 0) return;
    Walker<MODE> wk;
    wk.init(a, lens_p, plans[p]);
    TileSrc ts = tile_source<MODE>(a, wk);
    int h = 0;
    for (; h < hend; ++h) {
      const int sl = p * PSLOTS + h % PSLOTS;
      const int use = h / PSLOTS;
      // both lanes wait for the slot; they go on only together
      const bool freed = use == 0 || ptx::mbar_wait(&empty[sl], (uint32_t)((use - 1) & 1), kWaitNs);
      const bool aborted = lane == 0 && *(volatile int*)abort_flag;
      const unsigned fb = __ballot_sync(0x3u, freed), ab = __ballot_sync(0x3u, aborted);
      if (fb != 0x3u) {
        if (lane == 0) {
          atomicOr(a.err, kErrTimeout);
          atomicExch(abort_flag, 1);
        }
        break;
      }
      if (ab) break;
      const bool isv = h & 1;
      if (lane == 0) {
        if (!isv) {
          // first / last stream of each segment, for the merging kernels
          const int u = wk.b * a.Hkv + wk.g;
          const int v = blockIdx.x * NPAIR + p;
          if (MODE == MODE_CMP) {
            if (wk.tile == 0) a.rng1[2 * u] = v;
            if (wk.tile == wk.ntiles - 1) a.rng1[2 * u + 1] = v;
          } else {
            if (wk.tile == 0) a.rng3[4 * u] = v;
            if (wk.tile == wk.ns - 1) a.rng3[4 * u + 1] = v;
            if (wk.tile == wk.ns) a.rng3[4 * u + 2] = v;
            if (wk.tile == wk.ntiles - 1) a.rng3[4 * u + 3] = v;
          }
        }
        info[sl] = ts.nvalid;
        ptx::mbar_arrive_expect_tx(&full[sl], SLOT_BYTES);
      }
      __syncwarp(0x3u);
      ptx::tma_load_3d(slots + sl * SLOT_BYTES + lane * HALF_BYTES, isv ? &tv : &tk, &full[sl],
                       64 * lane, wk.g, ts.row, pol);
      if (isv) {
        wk.advance(a, lens_p);
        if (h + 1 < hend) ts = tile_source<MODE>(a, wk);  // next tile, early
      }
    }
    // every issued load must have landed before the CTA exits
    if (lane == 0)
      for (int k = 0; k < PSLOTS && k < h; ++k) {
        const int last = h - 1 - ((h - 1 - k) % PSLOTS);  // last half-tile in slot k
        if (!ptx::mbar_wait(&full[p * PSLOTS + last % PSLOTS], (uint32_t)((last / PSLOTS) & 1),
                            kWaitNs))
          atomicOr(a.err, kErrTimeout);
      }
    return;
  }

  // ---------------- consumers ----------------
  const int pair = warp >> 1, hw = warp & 1;
  const int my_len = plans[pair].len;
  if (my_len <= 0) return;
  unsigned char* qs = qsm + pair * QBYTES;
  const uint32_t qbase = ptx::smem_u32(qs);
  const long long vstream = (long long)blockIdx.x * NPAIR + pair;
  Walker<MODE> wk;
  wk.init(a, lens_p, plans[pair]);
  int cur_seg = wk.segment(a);
  int cur_b = wk.b, cur_g = wk.g;
  const __nv_bfloat16* qg = reinterpret_cast<const __nv_bfloat16*>(a.q);
  stage_q_half(qs, qg + ((long)cur_b * a.Hq + cur_g * G) * D, hw, lane);
  ptx::named_bar_sync(1 + pair, 64);
  float o[16][4];
#pragma unroll
  for (int dt = 0; dt < 16; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  const int r0 = lane >> 2, c = (lane & 3) * 2;
  for (int r = 0; r < my_len; ++r) {
    const int seg = wk.segment(a);
    if (seg != cur_seg) {
      store_partial(part + (2 * (vstream + cur_seg) + hw) * PART, lane, m0, m1, l0, l1, o);
#pragma unroll
      for (int dt = 0; dt < 16; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
      cur_seg = seg;
      if (wk.b != cur_b || wk.g != cur_g) {
        cur_b = wk.b;
        cur_g = wk.g;
        ptx::named_bar_sync(1 + pair, 64);  // both warps are done with the old block
        stage_q_half(qs, qg + ((long)cur_b * a.Hq + cur_g * G) * D, hw, lane);
        ptx::named_bar_sync(1 + pair, 64);
      }
    }
    const int hk = 2 * r, hv = 2 * r + 1;
    const int slk = pair * PSLOTS + hk % PSLOTS, slv = pair * PSLOTS + hv % PSLOTS;
    bool ok = !*(volatile int*)abort_flag;
    if (ok && !ptx::mbar_wait(&full[slk], (uint32_t)((hk / PSLOTS) & 1), kWaitNs)) {
      if (lane == 0) {
        atomicOr(a.err, kErrTimeout);
        atomicExch(abort_flag, 1);
      }
      ok = false;
    }
    const int nvalid = ok ? min(WK, info[slk] - WK * hw) : 0;
    float s[4][4];
    if (nvalid > 0) qk_tile_q<4>(s, qbase, ptx::smem_u32(slots + slk * SLOT_BYTES), WK * hw, lane);
    constexpr bool early = MODE != MODE_CMP || RF;  // K slot not needed after QK
    if (early) {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[slk]);
    }
    if (nvalid > 0) {
      softmax_step_lazy<4>(s, o, m0, m1, l0, l1, nvalid, a.scale_log2, lane);
      if (MODE == MODE_CMP && RF && a.want_rec) {
        const int u = wk.b * a.Hkv + wk.g;
        record_regs(a.trec + ((long)u * a.tiles_max + 2 * wk.tile + hw) * (G * (1 + a.nbt)), s, m0,
                    m1, lane);
      } else if (MODE == MODE_CMP && a.want_rec) {
        // record of this 32-key sub-tile: running max per head, and per
        // overlapped selection block the exp-sum of its keys. Scratch: this
        // warp's own 32 key rows of the K slot (first TMA box), already read.
        __syncwarp();
        float* scr = reinterpret_cast<float*>(slots + slk * SLOT_BYTES + hw * (WK * 128));
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          *reinterpret_cast<float2*>(scr + r0 * RPITCH + nt * 8 + c) =
              make_float2(s[nt][0], s[nt][1]);
          *reinterpret_cast<float2*>(scr + (r0 + 8) * RPITCH + nt * 8 + c) =
              make_float2(s[nt][2], s[nt][3]);
        }
        __syncwarp();
        const int u = wk.b * a.Hkv + wk.g;
        float* rec = a.trec + ((long)u * a.tiles_max + 2 * wk.tile + hw) * (G * (1 + a.nbt));
        if ((lane & 3) == 0) {
          rec[r0] = m0;
          rec[r0 + 8] = m1;
        }
        for (int x = lane; x < G * a.nbt; x += 32) {
          const int jl = x >> 4, hh = x & 15;
          const int lo = a.klo[jl], hi = min((int)a.khi[jl], nvalid - 1);
          float acc = 0.f;
          for (int kk = lo; kk <= hi; ++kk) acc += scr[hh * RPITCH + kk];
          rec[G + x] = acc;  // [1 + jl][h]
        }
        ptx::fence_proxy_async();  // scratch writes before the slot's next TMA fill
      }
    }
    if (!early) {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&empty[slk]);
    }
    if (ok && !ptx::mbar_wait(&full[slv], (uint32_t)((hv / PSLOTS) & 1), kWaitNs)) {
      if (lane == 0) {
        atomicOr(a.err, kErrTimeout);
        atomicExch(abort_flag, 1);
      }
      ok = false;
    }
    if (ok && nvalid > 0) pv_tile<2>(o, s, ptx::smem_u32(slots + slv * SLOT_BYTES), WK * hw, lane);
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty[slv]);
    wk.advance(a, lens_p);
  }
  store_partial(part + (2 * (vstream + cur_seg) + hw) * PART, lane, m0, m1, l0, l1, o);
}

// ---------------------------------------------------------------------------
// dec_select
// ---------------------------------------------------------------------------

constexpr int SEL_THREADS = 512;
constexpr int SEL_WARPS = SEL_THREADS / 32;
constexpr int kRecIssuers = 8;   // threads issuing the bulk copies of the score records
constexpr int MAXSEL = 64;       // top_n bound of the fast path
constexpr int MAXCAND = 4096;    // selection blocks bound of the fast path (T <= 262144)
constexpr size_t kSelDynSmemMax = 192 * 1024;  // dec_select dynamic shared memory (+ ~18 KB static)

// Dynamic shared memory of dec_select: the unit's score records, the sort keys,
// and two per-(sub-tile, head) arrays.
__host__ __device__ inline size_t sel_dyn_smem(int T, int sel_block, int tiles_max, int nbt) {
  const int nblk = (T + sel_block - 1) / sel_block;
  int npow = 2;  // >= 2 keeps the float arrays after the keys 16-byte aligned
  while (npow < nblk) npow <<= 1;
  return (size_t)tiles_max * 16 * (1 + nbt) * 4 + (size_t)npow * 8 + 2 * (size_t)tiles_max * 16 * 4 +
         16;
}

// Sort key of a candidate block: higher score first, then the lower index.
// Scores are >= 0, so their IEEE bits order like the values; the low word is
// the inverted index. Keys are unique, so the top set is exact.
__device__ __forceinline__ unsigned long long sel_key(float score, int j) {
  return ((unsigned long long)__float_as_uint(score) << 32) | (0xffffffffu - (unsigned)j);
}

__global__ void __launch_bounds__(SEL_THREADS) dec_select_kernel(const __grid_constant__ DecFastArgs a) {
  // dynamic: records [tiles_max][16 (1 + nbt)] | keys [npow] u64 | fac [tiles_max][16]
  //          | tsum [tiles_max][16]
  extern __shared__ __align__(128) unsigned char dyn_raw[];
  __shared__ float lse2[G];
  __shared__ int sel[MAXSEL];
  __shared__ unsigned hist[256];
  __shared__ int cut_bin, cut_above, nsel_s;
  __shared__ __align__(8) uint64_t rec_bar;
  __shared__ long long span_red[4 * SEL_WARPS];

  const int u = blockIdx.x, b = u / a.Hkv, g = u - b * a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    ptx::mbar_init(&rec_bar, kRecIssuers);
    ptx::fence_mbar_init();
  }
  // the compressed-branch streams of this unit, from the lengths (before the
  // wait when the predecessor is this library's kernel, which waited on the
  // caller's writes)
  if (!a.after_cmp) ptx::grid_dep_wait();
  ptx::grid_dep_launch();  // the selected/window kernel's set-up overlaps this one
  long long pre[2], tot[2];
  tile_spans(a, b, pre, tot, span_red);
  const int L = __ldg(a.seq_lens + b);
  int v_first = 0, v_last = -1;
  {
    const int nt = unit_tiles<MODE_CMP>(L, a);
    if (nt > 0) {
      const long long V = min((long long)a.grid1, tot[0]);
      const long long T0 = pre[0] + (long long)g * nt;
      v_first = stream_of_tile(T0, V, tot[0]);
      v_last = stream_of_tile(T0 + nt - 1, V, tot[0]);
    }
  }
  ptx::grid_dep_wait();  // partials and records of dec_cmp_partial
  const int nblk = (a.T + a.bs - 1) / a.bs;
  int npow = 2;  // as in sel_dyn_smem
  while (npow < nblk) npow <<= 1;
  const int rec_floats = G * (1 + a.nbt);
  float* recs = reinterpret_cast<float*>(dyn_raw);
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(recs + (size_t)a.tiles_max * rec_floats);
  float* fac = reinterpret_cast<float*>(keys + npow);
  float* tsum = fac + (size_t)a.tiles_max * G;

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
  const int rtiles_u = (nvis + WK - 1) / WK;  // 32-key record sub-tiles
  __syncthreads();  // rec_bar initialised

  if (nvis > 0) {
    // The unit's score records, in bulk copies that land while the lse is
    // merged: kRecIssuers threads each copy a share of the sub-tiles (one
    // thread's copies alone move too few bytes at a time).
    if (tid < kRecIssuers) {
      const int r0 = rtiles_u * tid / kRecIssuers, r1 = rtiles_u * (tid + 1) / kRecIssuers;
      const uint32_t bytes = (uint32_t)(r1 - r0) * rec_floats * 4;
      ptx::mbar_arrive_expect_tx(&rec_bar, bytes);
      if (bytes > 0)
        ptx::bulk_load(recs + (size_t)r0 * rec_floats,
                       a.trec + ((long)u * a.tiles_max + r0) * rec_floats, bytes, &rec_bar);
    }
    // lse of the compressed branch per head (warp h): log2 of sum_p 2^m_p l_p
    // over the unit's partials, each lane merging a strided share first
    {
      const long long first = 2 * ((long long)v_first + u);
      const int np = 2 * (v_last - v_first + 1);
      const int h = warp;  // SEL_WARPS == G
      float M = -INFINITY, Ls = 0.f;
      for (int pp = lane; pp < np; pp += 32) {
        const float* src = a.part1 + (first + pp) * PART;
        const float m = __ldcg(src + h), l = __ldcg(src + G + h);
        if (m == -INFINITY) continue;
        const float Mn = fmaxf(M, m);
        Ls = Ls * exp2f(M - Mn) + l * exp2f(m - Mn);  // exp2f(-inf) = 0 on the first
        M = Mn;
      }
      const float Mw = warp_max(M);
      const float c = M == -INFINITY ? 0.f : Ls * exp2f(M - Mw);
      const float Lw = warp_sum(c);
      if (lane == 0) lse2[h] = Mw + log2f(Lw);
    }
    // records landed? then factors exp2(m_ref - lse) per (sub-tile, head)
    if (!ptx::mbar_wait(&rec_bar, 0, kWaitNs) && tid == 0) atomicOr(a.err, kErrTimeout);
    __syncthreads();
    for (int x = tid; x < rtiles_u * G; x += SEL_THREADS) {
      const int tau = x >> 4, h = x & 15;
      fac[x] = exp2f(recs[tau * rec_floats + h] - lse2[h]);
    }
    __syncthreads();
    // per (sub-tile, block slot): the head-weighted sum of the record. Four
    // threads share a 16-wide dot product, one float4 each, so a warp reads
    // consecutive 16-byte words of the record rows (no bank conflicts).
    {
      // item x = (tau, r = 4 jl + q4); (tau, r) advances by a fixed step
      const int per_tau = a.nbt * 4;
      const int nitems = rtiles_u * per_tau;
      const int dtau = SEL_THREADS / per_tau, dr = SEL_THREADS - dtau * per_tau;
      int tau = tid / per_tau, r = tid - tau * per_tau;
      for (int x0 = 0; x0 < nitems; x0 += SEL_THREADS) {
        const bool in = x0 + tid < nitems;  // warps stay converged for the shuffles below
        float v = 0.f;
        if (in) {
          const float4 rv = *reinterpret_cast<const float4*>(recs + tau * rec_floats + G + 4 * r);
          const float4 fv = *reinterpret_cast<const float4*>(fac + tau * G + 4 * (r & 3));
          v = rv.x * fv.x + rv.y * fv.y + rv.z * fv.z + rv.w * fv.w;
        }
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        if (in && (r & 3) == 0) tsum[tau * 16 + (r >> 2)] = v;
        tau += dtau;
        r += dr;
        if (r >= per_tau) {
          r -= per_tau;
          ++tau;
        }
      }
    }
    __syncthreads();
    // block j collects the slots of the sub-tiles whose block ranges include it
    const int rsh = a.r_shift;  // blocks between sub-tile starts = 1 << rsh
    for (int j = tid; j < ncand; j += SEL_THREADS) {
      float v = 0.f;
      const int tau_hi = min(j >> rsh, rtiles_u - 1);
      const int tau_lo = max(0, (j - a.nbt + (1 << rsh)) >> rsh);
      for (int tau = tau_lo; tau <= tau_hi; ++tau) {
        const int jl = j - (tau << rsh);
        if (jl >= 0 && jl < a.nbt) v += tsum[tau * 16 + jl];
      }
      keys[j] = sel_key(v, j);
    }
  } else {
    for (int j = tid; j < ncand; j += SEL_THREADS) keys[j] = sel_key(0.f, j);
  }
  if (tid == 0) nsel_s = 0;
  __syncthreads();

  // top-n: block 0 kept, the best n-1 others (ties to the lower index). The
  // (n-1)-th largest key among blocks 1..ncand-1 is found by radix selection
  // on 8-bit digits (keys are unique); every key at or above it is kept.
  int ns;
  if (ncand <= a.n) {
    for (int j = tid; j < ncand; j += SEL_THREADS) sel[j] = j;
    ns = ncand;
  } else if (a.n == 1) {
    if (tid == 0) sel[0] = 0;
    ns = 1;
  } else {
    int need = a.n - 1;
    unsigned long long prefix = 0ull, mask = 0ull;
    for (int shift = 56; shift >= 0; shift -= 8) {
      if (tid < 256) hist[tid] = 0u;
      __syncthreads();
      // a warp whose candidates all share the digit adds them with one atomic
      // (the leading digits are mostly equal across all candidates)
      for (int j0 = 1; j0 < ncand; j0 += SEL_THREADS) {
        const int j = j0 + tid;
        const unsigned long long k = j < ncand ? keys[j] : 0ull;
        const bool in = j < ncand && (k & mask) == prefix;
        const unsigned bin = (unsigned)((k >> shift) & 255u);
        const unsigned inset = __ballot_sync(0xffffffffu, in);
        if (inset == 0u) continue;
        const unsigned b0 = __shfl_sync(0xffffffffu, bin, __ffs(inset) - 1);
        if (__all_sync(0xffffffffu, !in || bin == b0)) {
          if (lane == 0) atomicAdd(&hist[b0], (unsigned)__popc(inset));
        } else if (in) {
          atomicAdd(&hist[bin], 1u);
        }
      }
      __syncthreads();
      if (warp == 0) {
        // lane l holds bins 255-8l .. 248-8l (descending)
        unsigned c[8], tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          c[i] = hist[255 - 8 * lane - i];
          tot += c[i];
        }
        unsigned incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const unsigned excl = incl - tot;
        const bool here = excl < (unsigned)need && (unsigned)need <= incl;
        if (here) {
          unsigned cum = excl;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (cum + c[i] >= (unsigned)need) {
              cut_bin = 255 - 8 * lane - i;
              cut_above = (int)cum;
              break;
            }
            cum += c[i];
          }
        }
      }
      __syncthreads();
      const int d = cut_bin;
      need -= cut_above;
      prefix |= (unsigned long long)d << shift;
      mask |= 255ull << shift;
      if ((int)hist[d] == need) break;  // all of bin d is kept
      __syncthreads();
    }
    // keys >= prefix are exactly the n-1 kept blocks
    for (int j = 1 + tid; j < ncand; j += SEL_THREADS)
      if (keys[j] >= prefix) sel[1 + atomicAdd(&nsel_s, 1)] = j;
    if (tid == 0) sel[0] = 0;
    __syncthreads();
    // ascending order: each entry's rank among the n kept
    if (tid < a.n) {
      const int v = sel[tid];
      int rank = 0;
      for (int k = 0; k < a.n; ++k) rank += sel[k] < v;
      hist[rank] = (unsigned)v;  // hist is free: reuse as the sorted list
    }
    __syncthreads();
    if (tid < a.n) sel[tid] = (int)hist[tid];
    ns = a.n;
  }
  __syncthreads();
  if (a.top_p > 0.f) {
    // Adaptive selection (lchairun NSA article, adaptive sparsification): the
    // top-p set is a best-first prefix of at most n blocks, so it is cut from
    // the top-n set above: block 0, then the kept blocks by key (score desc,
    // index asc) until their scores reach top_p of the total over all
    // candidates (fp64 sums).
    __shared__ double wtot[SEL_WARPS];
    __shared__ int ord[MAXSEL];
    double part = 0.0;
    for (int j = tid; j < ncand; j += SEL_THREADS)
      part += (double)__uint_as_float((unsigned)(keys[j] >> 32));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) wtot[warp] = part;
    // the kept blocks other than 0, ordered by key (descending)
    const int nk = ns - 1;
    if (tid < nk) {
      const int j = sel[1 + tid];
      const unsigned long long kj = keys[j];
      int rank = 0;
      for (int i = 0; i < nk; ++i) rank += keys[sel[1 + i]] > kj ? 1 : 0;
      ord[rank] = j;
    }
    __syncthreads();
    if (tid == 0) {
      double tot = 0.0;
      for (int w = 0; w < SEL_WARPS; ++w) tot += wtot[w];
      const double goal = (double)a.top_p * tot;
      double cum = (double)__uint_as_float((unsigned)(keys[0] >> 32));
      int m = 0;
      while (m < nk && cum < goal) {
        cum += (double)__uint_as_float((unsigned)(keys[ord[m]] >> 32));
        ++m;
      }
      nsel_s = m + 1;
    }
    __syncthreads();
    ns = nsel_s;
    // ascending: block 0 first, then ord[0 .. ns - 1) sorted
    int v = -1, rank = 0;
    if (tid < ns) {
      v = tid == 0 ? 0 : ord[tid - 1];
      for (int i = 1; i < ns; ++i) rank += ord[i - 1] < v ? 1 : 0;
      rank += tid == 0 ? 0 : 1;  // block 0 precedes every other block
    }
    __syncthreads();
    if (tid < ns) sel[rank] = v;
    __syncthreads();
  }
  for (int x = tid; x < a.n; x += SEL_THREADS) {
    const int v = x < ns ? sel[x] : -1;
    a.sel[(long)u * a.n + x] = v;
    if (a.sel_out) a.sel_out[(long)u * a.n + x] = v;
  }
}

// ---------------------------------------------------------------------------
// dec_quest_select
// ---------------------------------------------------------------------------

// Order-preserving 32-bit image of a float (-0 taken as +0).
__device__ __forceinline__ unsigned ordered_bits(float x) {
  const unsigned u = __float_as_uint(x + 0.f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Quest-style selection (EP94 notes §八, the selection ablation; the Quest
// bound): one CTA per (sequence, KV head). With P = sum over the group's heads
// of max(q, 0) and N of min(q, 0), block j scores P . kmax_j + N . kmin_j from
// the caller's block-bounds table (its entry for the block holding the query
// covers the keys so far); block 0 and the n - 1 best others are kept (ties to
// the lower index). Replaces dec_select; the compressed branch's partials are
// merged by dec_combine as usual.
__global__ void __launch_bounds__(SEL_THREADS) dec_quest_select_kernel(const __grid_constant__ DecFastArgs a) {
  __shared__ __align__(16) float pn[2 * D];
  __shared__ float qsc[MAXCAND];
  __shared__ int sel[MAXSEL];
  const int u = blockIdx.x, b = u / a.Hkv, g = u - b * a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // inputs only before the wait when the predecessor is this library's
  // kernel, which waited on the caller's writes
  if (!a.after_cmp) ptx::grid_dep_wait();
  ptx::grid_dep_launch();  // the selected/window kernel's set-up overlaps this one
  const int L = __ldg(a.seq_lens + b);
  if (tid < D) {
    const __nv_bfloat16* qg =
        reinterpret_cast<const __nv_bfloat16*>(a.q) + ((long)b * a.Hq + g * G) * D + tid;
    float P = 0.f, N = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float x = __bfloat162float(qg[h * D]);
      P += fmaxf(x, 0.f);
      N += fminf(x, 0.f);
    }
    pn[tid] = P;
    pn[D + tid] = N;
  }
  ptx::grid_dep_wait();
  if (!len_ok(L, a)) {
    for (int x = tid; x < G * D; x += SEL_THREADS)
      reinterpret_cast<__nv_bfloat16*>(a.out)[((long)b * a.Hq + g * G) * D + x] =
          __float2bfloat16_rn(0.f);
    if (a.sel_out)
      for (int x = tid; x < a.n; x += SEL_THREADS) a.sel_out[(long)u * a.n + x] = -1;
    if (tid == 0) atomicOr(a.err, kErrSeqLen);
    return;
  }
  __syncthreads();
  const int ncand = (L - 1) / a.bs + 1;
  int ns;
  if (ncand <= a.n) {
    for (int j = tid; j < ncand; j += SEL_THREADS) sel[j] = j;
    ns = ncand;
  } else {
    // warp w scores blocks w, w + 16, ...: lane l takes table elements 8l .. 8l + 7
    const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(a.kbounds);
    float pl[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) pl[i] = pn[8 * lane + i];
    for (int j = warp; j < ncand; j += SEL_WARPS) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(
                                 kb + (((size_t)b * a.nblk + j) * a.Hkv + g) * 2 * D) +
                             lane);
      const __nv_bfloat162* e2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
      float v = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(e2[i]);
        v = fmaf(pl[2 * i], f.x, v);
        v = fmaf(pl[2 * i + 1], f.y, v);
      }
      v = warp_sum(v);
      if (lane == 0) qsc[j] = v;
    }
    __syncthreads();
    if (warp == 0) {
      // top n - 1 of blocks 1 .. ncand - 1: per round the warp maximum of the
      // lanes' best (ordered score bits, ~index) keys; the owner drops it
      auto rescan = [&](unsigned& bh, unsigned& bl) {
        bh = 0u;
        bl = 0u;
        for (int j = 1 + lane; j < ncand; j += 32) {
          const unsigned kh = ordered_bits(qsc[j]), kl = ~(unsigned)j;
          if (kh > bh || (kh == bh && kl > bl)) {
            bh = kh;
            bl = kl;
          }
        }
      };
      unsigned bh, bl;
      rescan(bh, bl);
      for (int r = 1; r < a.n; ++r) {
        const unsigned mh = __reduce_max_sync(0xffffffffu, bh);
        const unsigned ml = __reduce_max_sync(0xffffffffu, bh == mh ? bl : 0u);
        const int pick = (int)~ml;
        if (lane == 0) sel[r] = pick;
        if (bh == mh && bl == ml) {
          qsc[pick] = -INFINITY;  // finite scores remain above it (n - 1 < ncand - 1)
          rescan(bh, bl);
        }
      }
      if (lane == 0) sel[0] = 0;
    }
    __syncthreads();
    // ascending order
    int v = 0, rank = 0;
    if (tid < a.n) {
      v = sel[tid];
      for (int k = 0; k < a.n; ++k) rank += sel[k] < v;
    }
    __syncthreads();
    if (tid < a.n) sel[rank] = v;
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

constexpr int CMB_HEADS = 4;                   // heads per CTA
constexpr int CMB_GROUP = CMB_HEADS * 16;      // threads per branch: 16 per head, 8 dims each
constexpr int CMB_THREADS = 3 * CMB_GROUP;     // one group per branch
constexpr int CMB_CHUNK = 8;                   // partials whose loads are in flight together

// Per thread: the online merge of partials [first, first + np) for head h,
// dims e0 .. e0 + 7: M = max m_p, Ls = sum_p 2^(m_p - M) l_p,
// run = sum_p 2^(m_p - M) o_p. Partials with m = -inf (no valid key) add nothing.
__device__ __forceinline__ void merge_thread(const float* part, long long first, int np, int h,
                                             int e0, float& M, float& Ls, float (&run)[8]) {
  for (int p0 = 0; p0 < np; p0 += CMB_CHUNK) {
    float m[CMB_CHUNK], l[CMB_CHUNK];
    uint4 o[CMB_CHUNK];
#pragma unroll
    for (int i = 0; i < CMB_CHUNK; ++i) {
      if (p0 + i < np) {
        const float* src = part + (first + p0 + i) * PART;
        m[i] = __ldcg(src + h);
        l[i] = __ldcg(src + G + h);
        o[i] = __ldcg(reinterpret_cast<const uint4*>(
            reinterpret_cast<const __nv_bfloat16*>(src + 2 * G) + h * D + e0));
      } else {
        m[i] = -INFINITY;
      }
    }
    float Mn = M;
#pragma unroll
    for (int i = 0; i < CMB_CHUNK; ++i) Mn = fmaxf(Mn, m[i]);
    if (Mn == -INFINITY) continue;
    const float r = exp2f(M - Mn);  // 0 while nothing was merged (M = -inf)
    Ls *= r;
#pragma unroll
    for (int e = 0; e < 8; ++e) run[e] *= r;
#pragma unroll
    for (int i = 0; i < CMB_CHUNK; ++i) {
      if (m[i] == -INFINITY) continue;
      const float f = exp2f(m[i] - Mn);
      Ls = fmaf(f, l[i], Ls);
      const __nv_bfloat162* ob = reinterpret_cast<const __nv_bfloat162*>(&o[i]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 v = __bfloat1622float2(ob[k]);
        run[2 * k] = fmaf(f, v.x, run[2 * k]);
        run[2 * k + 1] = fmaf(f, v.y, run[2 * k + 1]);
      }
    }
    M = Mn;
  }
}

// CTA (unit, head quarter): three thread groups merge the compressed,
// selected and window partials of four heads at once, each thread on its own
// (no block-wide steps inside the merge); the gates come from the raw query;
// out = sum over branches of g_c o_c.
__global__ void __launch_bounds__(CMB_THREADS) dec_combine_kernel(const __grid_constant__ DecFastArgs a) {
  const int u = blockIdx.x, b = u / a.Hkv, g = u - b * a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int br = tid / CMB_GROUP, hl = (tid % CMB_GROUP) >> 4, e0 = (tid & 15) * 8;
  const int h = blockIdx.y * CMB_HEADS + hl;
  __shared__ float gate_s[CMB_HEADS * 3];
  __shared__ __align__(16) float contrib[3][CMB_HEADS][D];
  __shared__ long long span_red[4 * (CMB_THREADS / 32)];
  // Before the wait (the predecessors are this library's kernels, which
  // waited on the caller's writes): the streams of this unit's three
  // branches, from the lengths, and the gates, from the query.
  long long pre[2], tot[2];
  tile_spans(a, b, pre, tot, span_red);
  const int L = __ldg(a.seq_lens + b);
  if (!len_ok(L, a)) return;  // output zeroed by dec_select (uniform over the CTA)
  int2 rg = make_int2(0, -1);
  if (br == 0) {
    const int nt = unit_tiles<MODE_CMP>(L, a);
    if (nt > 0) {
      const long long V = min((long long)a.grid1, tot[0]);
      const long long T0 = pre[0] + (long long)g * nt;
      rg = make_int2(stream_of_tile(T0, V, tot[0]), stream_of_tile(T0 + nt - 1, V, tot[0]));
    }
  } else {
    const int nt = unit_tiles<MODE_SW>(L, a), ns = n_selected(L, a);
    const long long V = min((long long)a.grid3, tot[1]);
    const long long T0 = pre[1] + (long long)g * nt;
    const long long x0 = br == 1 ? T0 : T0 + ns, x1 = br == 1 ? T0 + ns - 1 : T0 + nt - 1;
    rg = make_int2(stream_of_tile(x0, V, tot[1]), stream_of_tile(x1, V, tot[1]));
  }

  // gates (EP94 notes §五 gating): sigmoid(q_h . Wg[:, c]), a warp per dot product
  const __nv_bfloat16* qg =
      reinterpret_cast<const __nv_bfloat16*>(a.q) + ((long)b * a.Hq + g * G) * D;
  for (int x = warp; x < CMB_HEADS * 3; x += CMB_THREADS / 32) {
    const int hh = blockIdx.y * CMB_HEADS + x / 3, c = x % 3;
    float gv;
    if (a.gate_mode == 1) {
      gv = a.fixed_gates[c];
    } else {
      float dot = 0.f;
#pragma unroll
      for (int e = lane; e < D; e += 32)
        dot = fmaf(__bfloat162float(qg[hh * D + e]), __ldg(a.w_gate + e * 3 + c), dot);
      dot = warp_sum(dot);
      gv = 1.f / (1.f + expf(-dot));
    }
    if (lane == 0) gate_s[x] = gv;
  }
  ptx::grid_dep_wait();  // partials of dec_cmp_partial / dec_sel_win

  const float* part;
  long long first;
  int np;
  if (br == 0) {  // compressed branch: absent while no compressed block is complete
    part = a.part1;
    if (n_visible(L, a.l, a.s, a.Nc) > 0) {
      first = 2 * ((long long)rg.x + u);
      np = 2 * (rg.y - rg.x + 1);
    } else {
      first = 0;
      np = 0;
    }
  } else {  // selected (segment 2u), window (segment 2u + 1)
    part = a.part3;
    first = 2 * ((long long)rg.x + 2 * u + (br - 1));
    np = 2 * (rg.y - rg.x + 1);
  }
  float M = -INFINITY, Ls = 0.f, run[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) run[e] = 0.f;
  merge_thread(part, first, np, h, e0, M, Ls, run);
  __syncthreads();  // gates
  const float sc = Ls > 0.f ? gate_s[hl * 3 + br] / Ls : 0.f;
  float4* dst = reinterpret_cast<float4*>(&contrib[br][hl][e0]);
  dst[0] = make_float4(sc * run[0], sc * run[1], sc * run[2], sc * run[3]);
  dst[1] = make_float4(sc * run[4], sc * run[5], sc * run[6], sc * run[7]);
  __syncthreads();
  for (int x = tid; x < CMB_HEADS * D / 4; x += CMB_THREADS) {
    const int hh = x / (D / 4), e = (x % (D / 4)) * 4;
    const float4 c0 = *reinterpret_cast<const float4*>(&contrib[0][hh][e]);
    const float4 c1 = *reinterpret_cast<const float4*>(&contrib[1][hh][e]);
    const float4 c2 = *reinterpret_cast<const float4*>(&contrib[2][hh][e]);
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) +
                          ((long)b * a.Hq + g * G + blockIdx.y * CMB_HEADS + hh) * D + e;
    // the same branch order as the oracle: cmp, then slc, then win
    const float o0 = (c0.x + c1.x) + c2.x, o1 = (c0.y + c1.y) + c2.y;
    const float o2 = (c0.z + c1.z) + c2.z, o3 = (c0.w + c1.w) + c2.w;
    *reinterpret_cast<__nv_bfloat162*>(orow) = __floats2bfloat162_rn(o0, o1);
    *reinterpret_cast<__nv_bfloat162*>(orow + 2) = __floats2bfloat162_rn(o2, o3);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  size_t part1, trec, sel, part3, rng1, rng3, total;
};

WsLayout ws_layout(const DecFastArgs& a) {
  WsLayout w{};
  const size_t units = (size_t)a.B * a.Hkv;
  size_t off = 0;
  w.part1 = off; off = align256(off + 2 * (size_t)(a.grid1 + units) * PART * 4);
  w.trec = off; off = align256(off + units * a.tiles_max * G * (1 + a.nbt) * 4);
  w.sel = off; off = align256(off + units * a.n * 4);
  w.part3 = off; off = align256(off + 2 * (size_t)(a.grid3 + 2 * units) * PART * 4);
  w.rng1 = off; off = align256(off + units * 2 * 4);
  w.rng3 = off; off = align256(off + units * 4 * 4);
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
  a.nbt = ((WK - 1) * a.s + a.l - 1) / a.bs + 2;
  a.r_shift = 0;
  while ((1 << a.r_shift) < (WK * a.s) / a.bs) ++a.r_shift;
  a.tiles_max = (a.Nc + WK - 1) / WK;  // 32-key record sub-tiles
  for (int jl = 0; jl < a.nbt && jl < kDecMaxNbt; ++jl) {
    // keys of a 32-key sub-tile (relative index) overlapping its jl-th block
    const int num = jl * a.bs - a.l + 1;
    const int lo = num <= 0 ? 0 : (num + a.s - 1) / a.s;
    const int hi = std::min(WK - 1, (jl * a.bs + a.bs - 1) / a.s);
    a.klo[jl] = (int8_t)std::min(lo, 127);
    a.khi[jl] = (int8_t)hi;
  }
  const int sms = device_sm_count();
  a.grid1 = sms * NPAIR;  // tile streams: one per consumer pair
  a.grid3 = sms * NPAIR;
  const float scale = p.softmax_scale != 0.f ? p.softmax_scale : 1.f / sqrtf((float)p.d);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.gate_mode = p.gate_mode;
  for (int i = 0; i < 3; ++i) a.fixed_gates[i] = p.fixed_gates[i];
  a.top_p = p.top_p;
  return a;
}


// Launch with programmatic stream serialization: the grid may be scheduled
// once the previous kernel's CTAs have called grid_dep_launch (the
// compressed-branch, selection and selected/window kernels do so at their
// start). Every decode kernel calls grid_dep_wait before it reads anything an
// earlier kernel writes; before that wait it reads only the call's inputs, and
// only when its predecessor is this library's kernel (which waited on the
// caller's writes first), so the order of memory effects is that of plain
// launches.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace

namespace {
// Shapes of the fast decode kernels (either selection).
bool decode_fast_shape(const nsa_params& p) {
  if (!(p.dtype == NSA_DTYPE_BF16 && p.d == D && p.Hq == G * p.Hkv && p.sel_block == TK &&
        p.top_n <= MAXSEL && p.T >= 1 && (p.T + p.sel_block - 1) / p.sel_block <= MAXCAND))
    return false;
  // 32-key compressed sub-tiles must start on selection-block boundaries, a
  // power-of-two number of blocks apart
  if ((WK * p.cmp_stride) % p.sel_block != 0) return false;
  const int R = (WK * p.cmp_stride) / p.sel_block;
  if ((R & (R - 1)) != 0) return false;
  const int nbt = ((WK - 1) * p.cmp_stride + p.cmp_block - 1) / p.sel_block + 2;
  if (nbt > 16 || nbt > kDecMaxNbt) return false;
  // dec_select keeps a whole unit's score records in shared memory
  const int Nc = nsa_num_cmp_blocks(p.T, p.cmp_block, p.cmp_stride);
  return sel_dyn_smem(p.T, p.sel_block, (Nc + WK - 1) / WK, nbt) <= kSelDynSmemMax;
}
}  // namespace

bool decode_fast_eligible(const nsa_params& p) { return p.sel_mode == 0 && decode_fast_shape(p); }

bool decode_quest_fast_eligible(const nsa_params& p) {
  return p.sel_mode == 1 && p.top_p == 0.f && decode_fast_shape(p);
}

size_t decode_fast_ws_bytes(const nsa_params& p) {
  if (!decode_fast_eligible(p) && !decode_quest_fast_eligible(p)) return 0;
  return ws_layout(base_args(p)).total;
}

cudaError_t launch_decode_fast(const nsa_params& p, const void* q, const void* k, const void* v,
                               const int32_t* seq_lens, const void* kc, const void* vc,
                               const float* w_gate, void* out, int32_t* sel_out, void* ws,
                               unsigned* err, cudaStream_t stream, const void* kbounds) {
  DecFastArgs a = base_args(p);
  a.kbounds = kbounds;
  a.want_rec = kbounds == nullptr;
  a.nblk = (p.T + p.sel_block - 1) / p.sel_block;
  a.after_cmp = a.Nc > 0;
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
  a.sel = reinterpret_cast<int*>(w + L.sel);
  a.part3 = reinterpret_cast<float*>(w + L.part3);
  a.rng1 = reinterpret_cast<int*>(w + L.rng1);
  a.rng3 = reinterpret_cast<int*>(w + L.rng3);

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
    constexpr size_t smem = StreamCfg<MODE_CMP>::SMEM;
    // score records from registers when l = 2s and bs = 4s
    const bool rf = p.cmp_block == 2 * p.cmp_stride && p.sel_block == 4 * p.cmp_stride;
    auto kern = rf ? dec_stream_kernel<MODE_CMP, true> : dec_stream_kernel<MODE_CMP, false>;
    if ((e = ensure_dyn_smem((const void*)kern, (int)smem)) != cudaSuccess) return e;
    if ((e = launch_pdl(kern, dim3(a.grid1 / NPAIR), dim3(STREAM_THREADS), smem, stream, a, tkc,
                        tvc)) != cudaSuccess)
      return e;
  }
  if (kbounds) {
    TraceScope trace("dec_quest_select", stream);
    if ((e = launch_pdl(dec_quest_select_kernel, dim3(p.B * p.Hkv), dim3(SEL_THREADS), 0, stream,
                        a)) != cudaSuccess)
      return e;
  } else {
    const size_t smem = sel_dyn_smem(p.T, p.sel_block, a.tiles_max, a.nbt);
    TraceScope trace("dec_select", stream);
    if ((e = ensure_dyn_smem((const void*)dec_select_kernel, (int)kSelDynSmemMax)) != cudaSuccess)
      return e;
    if ((e = launch_pdl(dec_select_kernel, dim3(p.B * p.Hkv), dim3(SEL_THREADS), smem, stream,
                        a)) != cudaSuccess)
      return e;
  }
  {
    TraceScope trace("dec_sel_win", stream);
    constexpr size_t smem = StreamCfg<MODE_SW>::SMEM;
    if ((e = ensure_dyn_smem((const void*)dec_stream_kernel<MODE_SW, false>, (int)smem)) !=
        cudaSuccess)
      return e;
    if ((e = launch_pdl(dec_stream_kernel<MODE_SW, false>, dim3(a.grid3 / NPAIR),
                        dim3(STREAM_THREADS), smem, stream, a, tk, tv)) != cudaSuccess)
      return e;
  }
  {
    TraceScope trace("dec_combine", stream);
    return launch_pdl(dec_combine_kernel, dim3(p.B * p.Hkv, G / CMB_HEADS), dim3(CMB_THREADS), 0,
                      stream, a);
  }
}

}  // namespace nsa
