// Host-side declarations shared by the library's translation units.
// Every launcher enqueues on `stream` and returns the launch status.
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "nsa.h"

namespace nsa {

// Device error word bits (read and cleared by nsa_check).
enum : unsigned {
  kErrTimeout = 1u,     // a bounded wait gave up
  kErrSeqLen = 2u,      // a decode sequence length outside [1, T]
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
};

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

// Kernel trace: bracket a launch with events when tracing is on.
void trace_begin(const char* name, cudaStream_t stream);
void trace_end(cudaStream_t stream);

struct TraceScope {
  cudaStream_t s;
  TraceScope(const char* name, cudaStream_t st) : s(st) { trace_begin(name, st); }
  ~TraceScope() { trace_end(s); }
};

cudaError_t launch_compress(const nsa_params& p, const void* k, const void* v, const float* w,
                            void* kc, void* vc, cudaStream_t stream);

// Shared-memory bytes the generic row kernel needs (0 if unsupported).
size_t nsa_rows_simt_smem(const NsaRowArgs& a);
cudaError_t launch_nsa_rows_simt(const NsaRowArgs& a, cudaStream_t stream);

size_t moba_simt_smem(const MobaArgs& a);
cudaError_t launch_moba_simt(const MobaArgs& a, cudaStream_t stream);

cudaError_t launch_bounded_wait(const int32_t* flag, int max_iters, unsigned* err,
                                cudaStream_t stream);

}  // namespace nsa
