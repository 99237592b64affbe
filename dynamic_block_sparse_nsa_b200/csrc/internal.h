// Host-side declarations shared by the library's translation units.
// Every launcher enqueues on `stream` and returns the launch status.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "nsa.h"

namespace nsa {

// Device error word bits (read and cleared by nsa_check).
enum : unsigned {
  kErrTimeout = 1u,     // a bounded wait gave up
  kErrSeqLen = 2u,      // a decode sequence length outside [1, T]
  kErrAppendPos = 4u,   // an append position outside [0, T)
};

// Arguments of the generic (CUDA-core) NSA row kernel, used for prefill and
// decode of any supported shape and dtype.
struct NsaRowArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* kc;
  const void* vc;
  const float* w_gate;
  void* out;
  int32_t* sel_idx;
  const int32_t* seq_lens;  // decode only
  unsigned* err;
  int B, T, Hq, Hkv, d;
  int l, s, bs, n, w, Nc;
  float scale;
  int gate_mode;
  float fixed_gates[3];
  int decode;               // 0 prefill (row per token), 1 decode (row per sequence)
  nsa_dtype dtype;
  float top_p;              // 0: top-n; else adaptive selection
  int sel_mode;             // 0: compressed-branch scores; 1: Quest block bound
};

struct NsaBwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* kc;
  const void* vc;
  const float* w_cmp;
  const float* w_gate;
  const int32_t* sel;       // [B, T, Hkv, n] the forward's selected blocks
  const void* dout;
  float* dq;                // [B, T, Hq, d]
  float* dk;                // [B, T, Hkv, d]
  float* dv;
  float* dw_cmp;            // [l]
  float* dw_gate;           // [d, 3]
  float* dkc;               // workspace [B, Nc, Hkv, d]
  float* dvc;
  float* dz;                // workspace [B, T, Hq, 3]
  int B, T, Hq, Hkv, d;
  int l, s, bs, n, w, Nc;
  float scale;
  int gate_mode;
  float fixed_gates[3];
  nsa_dtype dtype;
};

// Prefill backward (generic CUDA-core path).
size_t nsa_bwd_smem(int G, int d);
size_t nsa_bwd_ws_bytes(const nsa_params& p);
cudaError_t launch_nsa_backward(NsaBwdArgs a, void* ws, cudaStream_t stream);

struct MobaArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  int32_t* sel_idx;
  float* kbar;              // workspace [B, T/m, Hkv, d] fp32
  unsigned* err;
  int B, T, Hq, Hkv, d, m, topk;
  float scale;
  nsa_dtype dtype;
};

// Arguments of the bf16 / d=128 / 16-heads-per-group decode kernels.
constexpr int kDecMaxNbt = 48;
struct DecFastArgs {
  const void* q;
  const int32_t* seq_lens;
  const float* w_gate;
  void* out;
  int32_t* sel_out;
  unsigned* err;
  int B, T, Hq, Hkv, Nc, l, s, bs, n, w;
  int nbt;        // selection blocks one 32-key compressed sub-tile can overlap (bound)
  int r_shift;    // log2 of the selection blocks between sub-tile starts
  int tiles_max;  // 64-key compressed tiles per sequence at capacity T
  int grid1;      // tile streams (CTAs x consumer pairs) of the compressed-branch kernel
  int grid3;      // tile streams of the selected/window kernel
  float scale_log2;
  int gate_mode;
  float fixed_gates[3];
  float top_p;    // 0: top-n; else adaptive selection
  int8_t klo[kDecMaxNbt], khi[kDecMaxNbt];  // per block of a tile: its key range
  float* part1;   // compressed-branch partials, slot = 2 * (stream + unit) + half
  float* trec;    // per-tile block-score records
  int* sel;       // per unit [n]
  float* part3;   // selected / window partials, slot = 2 * (stream + 2 * unit + branch) + half
  int* rng1;      // per unit: first/last stream of its compressed tiles
  int* rng3;      // per unit: first/last stream of its selected and window tiles
  const void* kbounds;  // Quest-style selection: block key extremes [B, nblk, Hkv, 2, d]; else NULL
  int want_rec;         // the compressed-branch kernel writes score records (NSA selection)
  int nblk;             // selection blocks at capacity T
  int after_cmp;        // the selection kernel follows this library's compressed-branch
                        // kernel (else the caller's work: it waits before any read)
};

bool decode_fast_eligible(const nsa_params& p);
// The same kernels with the Quest-style selection from a block-bounds table
// (nsa_decode_quest): sel_mode == 1 on the fast decode's shapes.
bool decode_quest_fast_eligible(const nsa_params& p);
size_t decode_fast_ws_bytes(const nsa_params& p);
cudaError_t launch_decode_fast(const nsa_params& p, const void* q, const void* k, const void* v,
                               const int32_t* seq_lens, const void* kc, const void* vc,
                               const float* w_gate, void* out, int32_t* sel_out, void* ws,
                               unsigned* err, cudaStream_t stream, const void* kbounds = nullptr);

// Tensor-core prefill: bf16, d = 128, 16 query heads per KV head, l = 32,
// s = 16, selection block 64, top_n <= 16.
bool prefill_tc_eligible(const nsa_params& p);
size_t prefill_tc_ws_bytes(const nsa_params& p);
cudaError_t launch_prefill_tc(const nsa_params& p, const void* q, const void* k, const void* v,
                              const void* kc, const void* vc, const float* w_gate, void* out,
                              int32_t* sel_out, void* ws, unsigned* err, cudaStream_t stream);

// Quest-style block selection (nsa_params.sel_mode = 1) for the tensor-core
// prefill: per-block key extremes, block scores, top-n into `sel`
// [B, T, Hkv, n]. Its workspace follows the prefill's own.
bool quest_tc_supported(const nsa_params& p);
// Block key extremes beside a KV cache, and their update by one appended token.
cudaError_t launch_block_bounds(const nsa_params& p, const void* k, const int32_t* seq_lens,
                                void* kbounds, unsigned* err, cudaStream_t stream);
cudaError_t launch_append_bounds(const nsa_params& p, const void* k_new, const int32_t* pos,
                                 void* kbounds, unsigned* err, cudaStream_t stream);
size_t quest_ws_bytes(const nsa_params& p);
cudaError_t launch_quest_select(const nsa_params& p, const void* q, const void* k, int32_t* sel,
                                void* ws, cudaStream_t stream);

// Kernel trace: bracket a launch with events when tracing is on.
void trace_begin(const char* name, cudaStream_t stream);
void trace_end(cudaStream_t stream);

struct TraceScope {
  cudaStream_t s;
  TraceScope(const char* name, cudaStream_t st) : s(st) { trace_begin(name, st); }
  ~TraceScope() { trace_end(s); }
};

// Record `msg` as this host thread's error detail (nsa_last_error_detail).
void set_last_error(nsa_status s, const char* msg);

// Multiprocessor count of the current device (cached per device).
int device_sm_count();

// Raises the dynamic shared-memory limit of kernel `func` to `bytes` on the
// current device (once per kernel and device; safe from several host threads:
// a caller returns only after the limit is in place).
cudaError_t ensure_dyn_smem(const void* func, int bytes);

// 3-D TMA map over a contiguous bf16 array [dim2][dim1][dim0] with a box of
// (box0, box1, box2) elements; false if the driver rejects it.
bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t dim0, uint64_t dim1,
                       uint64_t dim2, uint32_t box0, uint32_t box1, uint32_t box2, bool swizzle128);

cudaError_t launch_compress(const nsa_params& p, const void* k, const void* v, const float* w,
                            void* kc, void* vc, cudaStream_t stream);
cudaError_t launch_append(const nsa_params& p, const void* k_new, const void* v_new,
                          const int32_t* pos, void* k_cache, void* v_cache, const float* w,
                          void* k_cmp, void* v_cmp, unsigned* err, cudaStream_t stream);

// Shared-memory bytes the generic row kernel needs (0 if unsupported).
size_t nsa_rows_simt_smem(const NsaRowArgs& a);
cudaError_t launch_nsa_rows_simt(const NsaRowArgs& a, cudaStream_t stream);

size_t moba_simt_smem(const MobaArgs& a);
cudaError_t launch_moba_simt(const MobaArgs& a, cudaStream_t stream);
cudaError_t launch_moba_block_mean(const MobaArgs& a, cudaStream_t stream);

// Tensor-core MoBA: bf16, d = 128, block a multiple of 128 (<= 2048),
// top_k <= 8. Its workspace starts with the block means (kbar_bytes).
bool moba_tc_eligible(const nsa_params& p);
size_t moba_tc_ws_bytes(const nsa_params& p, size_t kbar_bytes);
cudaError_t launch_moba_tc(const nsa_params& p, const void* q, const void* k, const void* v,
                           void* out, int32_t* sel_out, void* ws, size_t kbar_bytes,
                           unsigned* err, cudaStream_t stream);

cudaError_t launch_bounded_wait(const int32_t* flag, int max_iters, unsigned* err,
                                cudaStream_t stream);

}  // namespace nsa
