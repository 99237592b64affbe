// C ABI of the library (declared in include/nsa.h): host-side validation,
// workspace sizing, dispatch to the kernels, and the device error word.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "internal.h"

namespace nsa {
namespace {

thread_local std::string g_detail;

nsa_status fail(nsa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_detail = buf;
  return s;
}

nsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(NSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// One error word per device; each device holds its own copy of this module.
__device__ unsigned g_err_word;

unsigned* err_word(nsa_status* st) {
  static std::mutex mu;
  static unsigned* cache[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 128) {
    *st = cuda_fail(e, "cudaGetDevice");
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!cache[dev]) {
    e = cudaGetSymbolAddress((void**)&cache[dev], g_err_word);
    if (e != cudaSuccess) {
      *st = cuda_fail(e, "cudaGetSymbolAddress(error word)");
      return nullptr;
    }
  }
  *st = NSA_OK;
  return cache[dev];
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int max_smem_optin() {
  int dev = 0, v = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return v;
}

float eff_scale(const nsa_params* p) {
  return p->softmax_scale != 0.f ? p->softmax_scale : 1.f / std::sqrt((float)p->d);
}

// Checks shared by every call.
nsa_status check_common(const nsa_params* p) {
  if (!p) return fail(NSA_ERR_INVALID_ARGUMENT, "params is NULL");
  if (p->B < 1 || p->T < 1 || p->Hq < 1 || p->Hkv < 1)
    return fail(NSA_ERR_INVALID_ARGUMENT, "B, T, Hq, Hkv must be >= 1 (got %d, %d, %d, %d)", p->B,
                p->T, p->Hq, p->Hkv);
  if (p->B > 65535 || p->Hq > 65535)
    return fail(NSA_ERR_UNSUPPORTED, "B and Hq must be <= 65535");
  if (p->Hq % p->Hkv != 0)
    return fail(NSA_ERR_INVALID_ARGUMENT, "Hq (%d) must be a multiple of Hkv (%d)", p->Hq, p->Hkv);
  if (p->d != 64 && p->d != 128)
    return fail(NSA_ERR_UNSUPPORTED, "head dim d must be 64 or 128 (got %d)", p->d);
  if (p->dtype != NSA_DTYPE_F32 && p->dtype != NSA_DTYPE_BF16)
    return fail(NSA_ERR_INVALID_ARGUMENT, "unknown dtype %d", (int)p->dtype);
  if (!std::isfinite(p->softmax_scale))
    return fail(NSA_ERR_INVALID_ARGUMENT, "softmax_scale must be finite");
  return NSA_OK;
}

nsa_status check_nsa(const nsa_params* p) {
  nsa_status s = check_common(p);
  if (s != NSA_OK) return s;
  if (p->cmp_block < 1 || p->cmp_stride < 1 || p->cmp_stride > p->cmp_block)
    return fail(NSA_ERR_INVALID_ARGUMENT, "need 1 <= cmp_stride <= cmp_block (got l=%d s=%d)",
                p->cmp_block, p->cmp_stride);
  if (p->sel_block < 1 || p->top_n < 1 || p->window < 1)
    return fail(NSA_ERR_INVALID_ARGUMENT, "sel_block, top_n, window must be >= 1");
  if (p->top_n > 1024) return fail(NSA_ERR_UNSUPPORTED, "top_n must be <= 1024");
  if (p->gate_mode != 0 && p->gate_mode != 1)
    return fail(NSA_ERR_INVALID_ARGUMENT, "gate_mode must be 0 or 1");
  if (!(p->top_p >= 0.f && p->top_p <= 1.f))
    return fail(NSA_ERR_INVALID_ARGUMENT, "top_p must be in [0, 1] (0: top-n selection)");
  if (p->sel_mode != 0 && p->sel_mode != 1)
    return fail(NSA_ERR_INVALID_ARGUMENT, "sel_mode must be 0 (compressed scores) or 1 (Quest bound)");
  if (p->sel_mode == 1 && p->top_p != 0.f)
    return fail(NSA_ERR_INVALID_ARGUMENT, "sel_mode 1 (Quest bound) needs top_p == 0");
  if (p->Hkv > 65535) return fail(NSA_ERR_UNSUPPORTED, "Hkv must be <= 65535");
  return NSA_OK;
}

NsaRowArgs row_args(const nsa_params* p) {
  NsaRowArgs a{};
  a.B = p->B;
  a.T = p->T;
  a.Hq = p->Hq;
  a.Hkv = p->Hkv;
  a.d = p->d;
  a.l = p->cmp_block;
  a.s = p->cmp_stride;
  a.bs = p->sel_block;
  a.n = p->top_n;
  a.w = p->window;
  a.Nc = nsa_num_cmp_blocks(p->T, p->cmp_block, p->cmp_stride);
  a.scale = eff_scale(p);
  a.gate_mode = p->gate_mode;
  for (int i = 0; i < 3; ++i) a.fixed_gates[i] = p->fixed_gates[i];
  a.top_p = p->top_p;
  a.sel_mode = p->sel_mode;
  a.dtype = p->dtype;
  return a;
}

size_t moba_kbar_bytes(const nsa_params* p) {
  const size_t nfull = (size_t)(p->T / p->sel_block);
  return round_up((size_t)p->B * nfull * p->Hkv * p->d * sizeof(float), 256);
}

size_t moba_ws_bytes(const nsa_params* p) {
  const size_t kb = moba_kbar_bytes(p);
  return moba_tc_eligible(*p) ? moba_tc_ws_bytes(*p, kb) : kb;
}

nsa_status check_workspace(void* ws, size_t have, size_t need) {
  if (need == 0) return NSA_OK;
  if (!ws) return fail(NSA_ERR_INVALID_ARGUMENT, "workspace is NULL but %zu bytes are needed", need);
  if ((uintptr_t)ws % 256 != 0) return fail(NSA_ERR_INVALID_ARGUMENT, "workspace must be 256-byte aligned");
  if (have < need)
    return fail(NSA_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, %zu needed", have, need);
  return NSA_OK;
}

}  // namespace

void set_last_error(nsa_status, const char* msg) { g_detail = msg ? msg : ""; }

}  // namespace nsa

using namespace nsa;

extern "C" {

int nsa_num_cmp_blocks(int T, int l, int s) {
  if (l < 1 || s < 1 || T < l) return 0;
  return (T - l) / s + 1;
}

nsa_status nsa_workspace_size(const nsa_params* p, int op, size_t* bytes) {
  g_detail.clear();
  if (!bytes) return fail(NSA_ERR_INVALID_ARGUMENT, "bytes is NULL");
  *bytes = 0;
  switch (op) {
    case NSA_OP_COMPRESS: {
      nsa_status s = check_nsa(p);
      if (s != NSA_OK) return s;
      *bytes = 0;
      return NSA_OK;
    }
    case NSA_OP_PREFILL: {
      nsa_status s = check_nsa(p);
      if (s != NSA_OK) return s;
      *bytes = prefill_tc_eligible(*p) ? prefill_tc_ws_bytes(*p) : 0;
      return NSA_OK;
    }
    case NSA_OP_DECODE: {
      nsa_status s = check_nsa(p);
      if (s != NSA_OK) return s;
      *bytes = decode_fast_ws_bytes(*p);
      return NSA_OK;
    }
    case NSA_OP_PREFILL_BACKWARD: {
      nsa_status s = check_nsa(p);
      if (s != NSA_OK) return s;
      *bytes = nsa_bwd_ws_bytes(*p);
      return NSA_OK;
    }
    case NSA_OP_MOBA_PREFILL: {
      nsa_status s = check_common(p);
      if (s != NSA_OK) return s;
      if (p->sel_block < 1) return fail(NSA_ERR_INVALID_ARGUMENT, "sel_block must be >= 1");
      *bytes = moba_ws_bytes(p);
      return NSA_OK;
    }
    default:
      return fail(NSA_ERR_INVALID_ARGUMENT, "unknown op %d", op);
  }
}

nsa_status nsa_compress_kv(const nsa_params* p, const void* k, const void* v, const float* w_cmp,
                           void* k_cmp, void* v_cmp, void* stream) {
  g_detail.clear();
  nsa_status s = check_nsa(p);
  if (s != NSA_OK) return s;
  if (nsa_num_cmp_blocks(p->T, p->cmp_block, p->cmp_stride) == 0) return NSA_OK;  // nothing to write
  if (!k || !v || !w_cmp || !k_cmp || !v_cmp)
    return fail(NSA_ERR_INVALID_ARGUMENT, "k, v, w_cmp, k_cmp, v_cmp must be non-NULL");
  cudaError_t e = launch_compress(*p, k, v, w_cmp, k_cmp, v_cmp, (cudaStream_t)stream);
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "compress launch");
}

nsa_status nsa_prefill(const nsa_params* p, const void* q, const void* k, const void* v,
                       const void* k_cmp, const void* v_cmp, const float* w_gate, void* out,
                       int32_t* sel_idx, void* workspace, size_t ws_bytes, void* stream) {
  g_detail.clear();
  nsa_status s = check_nsa(p);
  if (s != NSA_OK) return s;
  const int Nc = nsa_num_cmp_blocks(p->T, p->cmp_block, p->cmp_stride);
  if (!q || !k || !v || !out || (Nc > 0 && (!k_cmp || !v_cmp)))
    return fail(NSA_ERR_INVALID_ARGUMENT, "q, k, v, k_cmp, v_cmp, out must be non-NULL");
  if (p->gate_mode == 0 && !w_gate)
    return fail(NSA_ERR_INVALID_ARGUMENT, "w_gate must be non-NULL when gate_mode == 0");
  unsigned* err = err_word(&s);
  if (!err) return s;
  if (prefill_tc_eligible(*p)) {
    s = check_workspace(workspace, ws_bytes, prefill_tc_ws_bytes(*p));
    if (s != NSA_OK) return s;
    cudaError_t e = launch_prefill_tc(*p, q, k, v, k_cmp, v_cmp, w_gate, out, sel_idx, workspace,
                                      err, (cudaStream_t)stream);
    return e == cudaSuccess ? NSA_OK : cuda_fail(e, "prefill launch");
  }
  NsaRowArgs a = row_args(p);
  a.q = q; a.k = k; a.v = v; a.kc = k_cmp; a.vc = v_cmp;
  a.w_gate = w_gate; a.out = out; a.sel_idx = sel_idx; a.err = err; a.decode = 0;
  const size_t smem = nsa_rows_simt_smem(a);
  if (smem > (size_t)max_smem_optin())
    return fail(NSA_ERR_UNSUPPORTED, "group size %d x head dim %d needs %zu bytes of shared memory",
                p->Hq / p->Hkv, p->d, smem);
  cudaError_t e = launch_nsa_rows_simt(a, (cudaStream_t)stream);
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "prefill launch");
}

nsa_status nsa_prefill_backward(const nsa_params* p, const void* q, const void* k, const void* v,
                                const void* k_cmp, const void* v_cmp, const float* w_cmp,
                                const float* w_gate, const int32_t* sel_idx, const void* dout,
                                float* dq, float* dk, float* dv, float* dw_cmp, float* dw_gate,
                                void* workspace, size_t ws_bytes, void* stream) {
  g_detail.clear();
  nsa_status s = check_nsa(p);
  if (s != NSA_OK) return s;
  const int Nc = nsa_num_cmp_blocks(p->T, p->cmp_block, p->cmp_stride);
  if (!q || !k || !v || !w_cmp || !sel_idx || !dout || !dq || !dk || !dv || !dw_cmp ||
      (Nc > 0 && (!k_cmp || !v_cmp)))
    return fail(NSA_ERR_INVALID_ARGUMENT,
                "q, k, v, k_cmp, v_cmp, w_cmp, sel_idx, dout, dq, dk, dv, dw_cmp must be non-NULL");
  if (p->gate_mode == 0 && (!w_gate || !dw_gate))
    return fail(NSA_ERR_INVALID_ARGUMENT, "w_gate and dw_gate must be non-NULL when gate_mode == 0");
  if (p->top_n > 64) return fail(NSA_ERR_UNSUPPORTED, "the backward supports top_n <= 64");
  const size_t smem = nsa_bwd_smem(p->Hq / p->Hkv, p->d);
  if (smem > (size_t)max_smem_optin())
    return fail(NSA_ERR_UNSUPPORTED, "group size %d x head dim %d needs %zu bytes of shared memory",
                p->Hq / p->Hkv, p->d, smem);
  s = check_workspace(workspace, ws_bytes, nsa_bwd_ws_bytes(*p));
  if (s != NSA_OK) return s;
  NsaBwdArgs a{};
  a.q = q; a.k = k; a.v = v; a.kc = k_cmp; a.vc = v_cmp;
  a.w_cmp = w_cmp; a.w_gate = w_gate; a.sel = sel_idx; a.dout = dout;
  a.dq = dq; a.dk = dk; a.dv = dv; a.dw_cmp = dw_cmp; a.dw_gate = dw_gate;
  a.B = p->B; a.T = p->T; a.Hq = p->Hq; a.Hkv = p->Hkv; a.d = p->d;
  a.l = p->cmp_block; a.s = p->cmp_stride; a.bs = p->sel_block; a.n = p->top_n; a.w = p->window;
  a.Nc = Nc;
  a.scale = eff_scale(p);
  a.gate_mode = p->gate_mode;
  for (int i = 0; i < 3; ++i) a.fixed_gates[i] = p->fixed_gates[i];
  a.dtype = p->dtype;
  cudaError_t e = launch_nsa_backward(a, workspace, (cudaStream_t)stream);
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "prefill backward launch");
}

nsa_status nsa_decode(const nsa_params* p, const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* seq_lens, const void* k_cmp, const void* v_cmp,
                      const float* w_gate, void* out, int32_t* sel_idx, void* workspace,
                      size_t ws_bytes, void* stream) {
  g_detail.clear();
  nsa_status s = check_nsa(p);
  if (s != NSA_OK) return s;
  const int Nc = nsa_num_cmp_blocks(p->T, p->cmp_block, p->cmp_stride);
  if (!q || !k_cache || !v_cache || !seq_lens || !out || (Nc > 0 && (!k_cmp || !v_cmp)))
    return fail(NSA_ERR_INVALID_ARGUMENT,
                "q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, out must be non-NULL");
  if (p->gate_mode == 0 && !w_gate)
    return fail(NSA_ERR_INVALID_ARGUMENT, "w_gate must be non-NULL when gate_mode == 0");
  unsigned* err = err_word(&s);
  if (!err) return s;
  if (decode_fast_eligible(*p)) {
    s = check_workspace(workspace, ws_bytes, decode_fast_ws_bytes(*p));
    if (s != NSA_OK) return s;
    cudaError_t e = launch_decode_fast(*p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, w_gate,
                                       out, sel_idx, workspace, err, (cudaStream_t)stream);
    return e == cudaSuccess ? NSA_OK : cuda_fail(e, "decode launch");
  }
  NsaRowArgs a = row_args(p);
  a.q = q; a.k = k_cache; a.v = v_cache; a.kc = k_cmp; a.vc = v_cmp;
  a.w_gate = w_gate; a.out = out; a.sel_idx = sel_idx; a.seq_lens = seq_lens; a.err = err;
  a.decode = 1;
  const size_t smem = nsa_rows_simt_smem(a);
  if (smem > (size_t)max_smem_optin())
    return fail(NSA_ERR_UNSUPPORTED, "group size %d x head dim %d needs %zu bytes of shared memory",
                p->Hq / p->Hkv, p->d, smem);
  cudaError_t e = launch_nsa_rows_simt(a, (cudaStream_t)stream);
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "decode launch");
}

nsa_status nsa_decode_quest(const nsa_params* p, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* seq_lens, const void* k_cmp,
                            const void* v_cmp, const void* k_bounds, const float* w_gate,
                            void* out, int32_t* sel_idx, void* workspace, size_t ws_bytes,
                            void* stream) {
  g_detail.clear();
  nsa_status s = check_nsa(p);
  if (s != NSA_OK) return s;
  if (p->sel_mode != 1)
    return fail(NSA_ERR_INVALID_ARGUMENT, "nsa_decode_quest needs sel_mode == 1 (Quest bound)");
  if (!decode_quest_fast_eligible(*p))  // other shapes: the CUDA-core path reads the keys
    return nsa_decode(p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, w_gate, out, sel_idx,
                      workspace, ws_bytes, stream);
  const int Nc = nsa_num_cmp_blocks(p->T, p->cmp_block, p->cmp_stride);
  if (!q || !k_cache || !v_cache || !seq_lens || !out || !k_bounds ||
      (Nc > 0 && (!k_cmp || !v_cmp)))
    return fail(NSA_ERR_INVALID_ARGUMENT,
                "q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, k_bounds, out must be non-NULL");
  if (p->gate_mode == 0 && !w_gate)
    return fail(NSA_ERR_INVALID_ARGUMENT, "w_gate must be non-NULL when gate_mode == 0");
  unsigned* err = err_word(&s);
  if (!err) return s;
  s = check_workspace(workspace, ws_bytes, decode_fast_ws_bytes(*p));
  if (s != NSA_OK) return s;
  cudaError_t e = launch_decode_fast(*p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, w_gate, out,
                                     sel_idx, workspace, err, (cudaStream_t)stream, k_bounds);
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "decode launch");
}

nsa_status nsa_block_bounds(const nsa_params* p, const void* k_cache, const int32_t* seq_lens,
                            void* k_bounds, void* stream) {
  g_detail.clear();
  nsa_status s = check_common(p);
  if (s != NSA_OK) return s;
  if (p->sel_block < 1) return fail(NSA_ERR_INVALID_ARGUMENT, "sel_block must be >= 1");
  if (!k_cache || !seq_lens || !k_bounds)
    return fail(NSA_ERR_INVALID_ARGUMENT, "k_cache, seq_lens, k_bounds must be non-NULL");
  unsigned* err = err_word(&s);
  if (!err) return s;
  cudaError_t e = launch_block_bounds(*p, k_cache, seq_lens, k_bounds, err, (cudaStream_t)stream);
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "block bounds launch");
}

nsa_status nsa_append_bounds(const nsa_params* p, const void* k_new, const int32_t* pos,
                             void* k_bounds, void* stream) {
  g_detail.clear();
  nsa_status s = check_common(p);
  if (s != NSA_OK) return s;
  if (p->sel_block < 1) return fail(NSA_ERR_INVALID_ARGUMENT, "sel_block must be >= 1");
  if (!k_new || !pos || !k_bounds)
    return fail(NSA_ERR_INVALID_ARGUMENT, "k_new, pos, k_bounds must be non-NULL");
  unsigned* err = err_word(&s);
  if (!err) return s;
  cudaError_t e = launch_append_bounds(*p, k_new, pos, k_bounds, err, (cudaStream_t)stream);
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "append bounds launch");
}

nsa_status moba_prefill(const nsa_params* p, const void* q, const void* k, const void* v,
                        void* out, int32_t* sel_idx, void* workspace, size_t ws_bytes,
                        void* stream) {
  g_detail.clear();
  nsa_status s = check_common(p);
  if (s != NSA_OK) return s;
  if (p->sel_block < 1 || p->top_n < 1 || p->top_n > 1024)
    return fail(NSA_ERR_INVALID_ARGUMENT, "need sel_block >= 1 and 1 <= top_n <= 1024");
  if (!q || !k || !v || !out)
    return fail(NSA_ERR_INVALID_ARGUMENT, "q, k, v, out must be non-NULL");
  const size_t need = moba_ws_bytes(p);
  s = check_workspace(workspace, ws_bytes, need);
  if (s != NSA_OK) return s;
  unsigned* err = err_word(&s);
  if (!err) return s;
  MobaArgs a{};
  a.q = q; a.k = k; a.v = v; a.out = out; a.sel_idx = sel_idx; a.kbar = (float*)workspace;
  a.err = err;
  a.B = p->B; a.T = p->T; a.Hq = p->Hq; a.Hkv = p->Hkv; a.d = p->d; a.m = p->sel_block;
  a.topk = p->top_n; a.scale = eff_scale(p); a.dtype = p->dtype;
  if (moba_tc_eligible(*p)) {
    cudaError_t e = launch_moba_block_mean(a, (cudaStream_t)stream);
    if (e == cudaSuccess)
      e = launch_moba_tc(*p, q, k, v, out, sel_idx, workspace, moba_kbar_bytes(p), err,
                         (cudaStream_t)stream);
    return e == cudaSuccess ? NSA_OK : cuda_fail(e, "moba launch");
  }
  if (moba_simt_smem(a) > (size_t)max_smem_optin())
    return fail(NSA_ERR_UNSUPPORTED, "MoBA shape needs too much shared memory");
  cudaError_t e = launch_moba_simt(a, (cudaStream_t)stream);
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "moba launch");
}

nsa_status nsa_check(void* stream) {
  g_detail.clear();
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned word = 0;
  e = cudaMemcpyFromSymbol(&word, g_err_word, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  if (word) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_err_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  }
  if (word & kErrTimeout) return fail(NSA_ERR_DEVICE_TIMEOUT, "a bounded device wait gave up");
  if (word & kErrSeqLen)
    return fail(NSA_ERR_INVALID_ARGUMENT, "a decode sequence length was outside [1, T]");
  if (word & kErrAppendPos)
    return fail(NSA_ERR_INVALID_ARGUMENT, "an append position was outside [0, T)");
  return NSA_OK;
}

nsa_status nsa_append_kv(const nsa_params* p, const void* k_new, const void* v_new,
                         const int32_t* pos, void* k_cache, void* v_cache, const float* w_cmp,
                         void* k_cmp, void* v_cmp, void* stream) {
  g_detail.clear();
  nsa_status s = check_nsa(p);
  if (s != NSA_OK) return s;
  const int Nc = nsa_num_cmp_blocks(p->T, p->cmp_block, p->cmp_stride);
  if (!k_new || !v_new || !pos || !k_cache || !v_cache || (Nc > 0 && (!w_cmp || !k_cmp || !v_cmp)))
    return fail(NSA_ERR_INVALID_ARGUMENT,
                "k_new, v_new, pos, k_cache, v_cache, w_cmp, k_cmp, v_cmp must be non-NULL");
  unsigned* err = err_word(&s);
  if (!err) return s;
  cudaError_t e = launch_append(*p, k_new, v_new, pos, k_cache, v_cache, w_cmp, k_cmp, v_cmp, err,
                                (cudaStream_t)stream);
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "append launch");
}

nsa_status nsa_debug_bounded_wait(const int32_t* flag, int max_iters, void* stream) {
  g_detail.clear();
  if (!flag || max_iters < 0) return fail(NSA_ERR_INVALID_ARGUMENT, "flag NULL or max_iters < 0");
  nsa_status s;
  unsigned* err = err_word(&s);
  if (!err) return s;
  cudaError_t e = launch_bounded_wait(flag, max_iters, err, (cudaStream_t)stream);
  return e == cudaSuccess ? NSA_OK : cuda_fail(e, "bounded wait launch");
}

const char* nsa_status_string(nsa_status s) {
  switch (s) {
    case NSA_OK: return "NSA_OK";
    case NSA_ERR_INVALID_ARGUMENT: return "NSA_ERR_INVALID_ARGUMENT";
    case NSA_ERR_UNSUPPORTED: return "NSA_ERR_UNSUPPORTED";
    case NSA_ERR_WORKSPACE_TOO_SMALL: return "NSA_ERR_WORKSPACE_TOO_SMALL";
    case NSA_ERR_CUDA: return "NSA_ERR_CUDA";
    case NSA_ERR_DEVICE_TIMEOUT: return "NSA_ERR_DEVICE_TIMEOUT";
  }
  return "NSA_ERR_UNKNOWN";
}

const char* nsa_last_error_detail(void) { return g_detail.c_str(); }

}  // extern "C"
