/*
 * nsa.h -- C ABI of the B200 (sm_100a) Native Sparse Attention / MoBA
 * forward library (libnsa_b200.so).
 *
 * Operations (the sources print no equations; each operation is the plain
 * reading of their prose with the constants of the workload statement):
 *   - nsa_compress_kv: token compression, "Zhang Xiaojun EP94 notes" §五 branch
 *     one; lchairun.cn NSA article, compression paragraph.
 *   - nsa_prefill / nsa_decode: the three-branch NSA forward, EP94 notes §五
 *     (compressed, selected and sliding-window branches, gating) and §六 (GQA
 *     group-shared selection); lchairun.cn NSA article, selection, window and
 *     gate paragraphs (decode is bound by KV bytes moved).
 *   - moba_prefill: MoBA, EP94 notes §九/§十/§十六 (mean-pooled block keys,
 *     parameter-free per-head top-k, block 512, top-3); LateTalk ep.103 (the
 *     query's own block is always attended).
 *
 * Conventions for every call:
 *   - Tensors are plain device pointers, contiguous, row-major, in the layout
 *     given per argument ("bshd": [batch, tokens, heads, head_dim]). The caller
 *     allocates and owns all of them; the library never allocates or frees
 *     device memory and never synchronises, except nsa_check.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). All work is enqueued asynchronously on it.
 *   - Arguments are validated on the host before anything is launched; on an
 *     error nothing is written and a status other than NSA_OK is returned,
 *     with a message in nsa_last_error_detail().
 *   - Launch failures return NSA_ERR_CUDA. Faults found on the device (a
 *     bounded wait that gave up, a sequence length out of range) set a
 *     per-device error word that nsa_check reports.
 *   - Thread safety: calls on different streams may run concurrently; the
 *     error-detail string is thread-local.
 */
#ifndef NSA_B200_H_
#define NSA_B200_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NSA_API __attribute__((visibility("default")))
#else
#define NSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NSA_OK = 0,
  NSA_ERR_INVALID_ARGUMENT = 1, /* bad pointer, shape, size or mode          */
  NSA_ERR_UNSUPPORTED = 2,      /* valid but not implemented (e.g. head dim) */
  NSA_ERR_WORKSPACE_TOO_SMALL = 3,
  NSA_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed      */
  NSA_ERR_DEVICE_TIMEOUT = 5    /* a bounded device-side wait gave up        */
} nsa_status;

typedef enum { NSA_DTYPE_F32 = 0, NSA_DTYPE_BF16 = 1 } nsa_dtype;

/* Operation ids for nsa_workspace_size. */
typedef enum {
  NSA_OP_COMPRESS = 0,
  NSA_OP_PREFILL = 1,
  NSA_OP_DECODE = 2,
  NSA_OP_MOBA_PREFILL = 3,
  NSA_OP_PREFILL_BACKWARD = 4
} nsa_op;

/* Problem description shared by all calls.
 *   B, T       batch and tokens (prefill: every sequence has T tokens; decode:
 *              T is the KV-cache capacity, the live length comes from seq_lens;
 *              MoBA: tokens per sequence).
 *   Hq, Hkv    query heads and KV heads; Hq % Hkv == 0; query head h reads KV
 *              head h / (Hq / Hkv) (consecutive heads form a GQA group).
 *   d          head dimension: 64 or 128.
 *   cmp_block, cmp_stride   compression length l and stride s (l >= s >= 1).
 *   sel_block  selection block size (NSA: 64); MoBA block size m (512).
 *   top_n      NSA: blocks kept per (token, KV head), block 0 included;
 *              MoBA: blocks kept per (token, head), the own block included.
 *   window     sliding-window length w (>= 1).
 *   softmax_scale  0 selects 1/sqrt(d).
 *   gate_mode  0: g = sigmoid(q . Wg) per branch (Wg [d,3], order cmp, slc,
 *              win, raw unscaled q); 1: g = fixed_gates for every query.
 *   dtype      element type of q, k, v, compressed k/v and out.
 *   top_p      0: keep top_n blocks. In (0, 1]: adaptive selection (lchairun
 *              NSA article, adaptive sparsification): block 0, then the other
 *              blocks by score (ties to the lower index) up to the first prefix
 *              whose score sum reaches top_p times the sum over all candidate
 *              blocks, at most top_n blocks; unused sel_idx slots hold -1.
 *   sel_mode   block scores the NSA selection ranks: 0 the compressed-branch
 *              probability mass on each block, summed over the GQA group
 *              (EP94 notes §五); 1 the Quest-style block bound of the pages'
 *              selection ablation (EP94 notes §八): with kmin, kmax the
 *              element-wise min and max of the block's keys up to the query,
 *              sum over the group's heads of sum_e max(q_e kmin_e, q_e kmax_e).
 *              Mode 1 needs top_p == 0. Prefill (bf16, d = 128, 16 heads per
 *              KV head, selection block 64) takes it from a block-bounds
 *              table built inside the call; decode takes that table from the
 *              caller through nsa_decode_quest (nsa_decode computes the bounds
 *              from the keys, on the CUDA-core path).
 * MoBA uses B, T, Hq, Hkv, d, sel_block, top_n, softmax_scale and dtype. */
typedef struct {
  int B, T, Hq, Hkv, d;
  int cmp_block, cmp_stride;
  int sel_block, top_n, window;
  float softmax_scale;
  int gate_mode;
  float fixed_gates[3];
  nsa_dtype dtype;
  float top_p;
  int sel_mode;
} nsa_params;

/* Bytes of caller-provided device workspace `op` needs for `p` (0 is
 * possible). The workspace must be 256-byte aligned. */
NSA_API nsa_status nsa_workspace_size(const nsa_params* p, int op, size_t* bytes);

/* Number of compressed blocks for T tokens: floor((T - l) / s) + 1, or 0 when
 * T < l. Compressed block i covers tokens [i*s, i*s + l - 1]. */
NSA_API int nsa_num_cmp_blocks(int T, int cmp_block, int cmp_stride);

/* Token compression (EP94 notes §五 branch one).
 *   k, v       [B, T, Hkv, d] dtype.
 *   w_cmp      [cmp_block] fp32 weights shared by keys and values.
 *   k_cmp, v_cmp  [B, Nc, Hkv, d] dtype outputs, Nc = nsa_num_cmp_blocks(T):
 *              k_cmp[b,i,g,:] = sum_j w_cmp[j] * k[b, i*s + j, g, :]
 *              (accumulated in fp64, rounded once to dtype, nearest-even). */
NSA_API nsa_status nsa_compress_kv(const nsa_params* p, const void* k, const void* v,
                           const float* w_cmp, void* k_cmp, void* v_cmp, void* stream);

/* NSA causal prefill (EP94 notes §五, §六).
 *   q          [B, T, Hq, d]; k, v [B, T, Hkv, d]; k_cmp, v_cmp [B, Nc, Hkv, d]
 *              (from nsa_compress_kv).
 *   w_gate     [d, 3] fp32 (ignored when gate_mode == 1; may then be NULL).
 *   out        [B, T, Hq, d] dtype.
 *   sel_idx    [B, T, Hkv, top_n] int32 or NULL: the selected blocks of each
 *              (token, KV head), ascending, block 0 first, -1 padded when
 *              fewer than top_n blocks exist.
 *   workspace  device scratch of nsa_workspace_size(NSA_OP_PREFILL) bytes. */
NSA_API nsa_status nsa_prefill(const nsa_params* p, const void* q, const void* k, const void* v,
                       const void* k_cmp, const void* v_cmp, const float* w_gate, void* out,
                       int32_t* sel_idx, void* workspace, size_t ws_bytes, void* stream);

/* NSA prefill backward: gradients of L = sum(dout * out) of nsa_prefill
 * (EP94 notes §五: the compressed branch carries the gradient that trains the
 * selection; lchairun.cn NSA article, the paragraph on trainability). The
 * selected blocks are constants of the backward (the top-n choice is
 * discrete); gradients flow through the gates, the three attentions and the
 * compression, whose storage rounding is taken as the identity.
 *   q, k, v, k_cmp, v_cmp, w_gate  as passed to nsa_prefill; k_cmp, v_cmp are
 *              nsa_compress_kv(k, v, w_cmp).
 *   w_cmp      [cmp_block] fp32, the compression weights.
 *   sel_idx    [B, T, Hkv, top_n] int32: the forward's selected blocks (as
 *              nsa_prefill writes them); entries < 0, repeated, or past the
 *              row's own block are ignored.
 *   dout       [B, T, Hq, d] dtype.
 *   dq         [B, T, Hq, d] fp32 output.
 *   dk, dv     [B, T, Hkv, d] fp32 outputs (overwritten).
 *   dw_cmp     [cmp_block] fp32 output.
 *   dw_gate    [d, 3] fp32 output; zeros when gate_mode == 1 (may be NULL then).
 *   workspace  device scratch of nsa_workspace_size(NSA_OP_PREFILL_BACKWARD)
 *              bytes (caller-owned; contents need not be initialised).
 * Runs on CUDA cores in fp32; dk, dv and the compressed-branch gradients are
 * summed with atomics, so their last bits can vary between runs. top_n > 64
 * returns NSA_ERR_UNSUPPORTED. */
NSA_API nsa_status nsa_prefill_backward(const nsa_params* p, const void* q, const void* k,
                                const void* v, const void* k_cmp, const void* v_cmp,
                                const float* w_cmp, const float* w_gate, const int32_t* sel_idx,
                                const void* dout, float* dq, float* dk, float* dv, float* dw_cmp,
                                float* dw_gate, void* workspace, size_t ws_bytes, void* stream);

/* NSA single-token decode over a KV cache (EP94 notes §六; lchairun.cn NSA
 * article: decode moves the group's one shared KV subset).
 *   q          [B, Hq, d]: the query of the token at position seq_lens[b]-1.
 *   k_cache, v_cache  [B, T, Hkv, d] (T = capacity); positions < seq_lens[b]
 *              are live and include the current token.
 *   seq_lens   [B] int32 device array, 1 <= seq_lens[b] <= T (violations set
 *              the device error word and zero that sequence's output).
 *   k_cmp, v_cmp  [B, Nc(T), Hkv, d]; entries of blocks ending before
 *              seq_lens[b] are read.
 *   w_gate, out [B, Hq, d], sel_idx [B, Hkv, top_n], workspace: as prefill. */
NSA_API nsa_status nsa_decode(const nsa_params* p, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* seq_lens, const void* k_cmp,
                      const void* v_cmp, const float* w_gate, void* out, int32_t* sel_idx,
                      void* workspace, size_t ws_bytes, void* stream);

/* Streaming decode: appends one token per sequence to the caches (lchairun NSA
 * article: decode reads the compressed cache, which gains one block every s
 * tokens, plus the selected and most recent tokens; EP94 notes §五).
 *   k_new, v_new      [B, Hkv, d] dtype: the new token's keys and values.
 *   pos               [B] int32, device: where to write, the sequence's length
 *                     before the append (0 <= pos < T).
 *   k_cache, v_cache  [B, T, Hkv, d] dtype, written at [b, pos[b]].
 *   w_cmp             [cmp_block] fp32 (the weights given to nsa_compress_kv).
 *   k_cmp, v_cmp      [B, Nc, Hkv, d] dtype. When pos + 1 completes compressed
 *                     block i = (pos + 1 - l) / s (pos + 1 >= l and
 *                     (pos + 1 - l) % s == 0), entry i is written exactly as
 *                     nsa_compress_kv computes it; no other entry is touched.
 *   A position outside [0, T) writes nothing for that sequence and sets the
 *   device error word (nsa_check then returns NSA_ERR_INVALID_ARGUMENT). The
 *   caller passes seq_lens = pos + 1 to the next nsa_decode. */
NSA_API nsa_status nsa_append_kv(const nsa_params* p, const void* k_new, const void* v_new,
                                 const int32_t* pos, void* k_cache, void* v_cache,
                                 const float* w_cmp, void* k_cmp, void* v_cmp, void* stream);

/* Quest-style block bounds beside a KV cache, for nsa_decode_quest (EP94 notes
 * §八: the selection ablation's Quest-style block score).
 *   k_cache    [B, T, Hkv, d] dtype.
 *   seq_lens   [B] int32, device, 1 <= seq_lens[b] <= T.
 *   k_bounds   [B, nblk, Hkv, 2, d] dtype, nblk = ceil(T / sel_block):
 *              k_bounds[b, j, g, 0, :] is the element-wise maximum and
 *              k_bounds[b, j, g, 1, :] the minimum of the keys of selection
 *              block j among the first seq_lens[b] tokens (the block holding
 *              the last token covers the tokens so far). Entries of blocks at
 *              or past seq_lens[b] are not written. Uses B, T, Hkv, d,
 *              sel_block and dtype of p.
 *   A length outside [1, T] writes nothing for that sequence and sets the
 *   device error word (nsa_check: NSA_ERR_INVALID_ARGUMENT). */
NSA_API nsa_status nsa_block_bounds(const nsa_params* p, const void* k_cache,
                                    const int32_t* seq_lens, void* k_bounds, void* stream);

/* Keeps k_bounds current after nsa_append_kv wrote token pos[b] (0 <= pos[b]
 * < T): block pos[b] / sel_block then covers keys up to pos[b] (a block's
 * first token restarts its extremes).
 *   k_new      [B, Hkv, d] dtype (the appended keys); pos [B] int32, device. */
NSA_API nsa_status nsa_append_bounds(const nsa_params* p, const void* k_new, const int32_t* pos,
                                     void* k_bounds, void* stream);

/* NSA decode that ranks blocks by the Quest-style bound (p->sel_mode must be
 * 1; EP94 notes §八): for the query's group, sum over its heads of
 * sum_e max(q_e kmin_e, q_e kmax_e), with kmin / kmax read from k_bounds as
 * nsa_block_bounds / nsa_append_bounds keep them; block 0 and the n - 1 best
 * others (ties to the lower index) are kept, the three branches and gates are
 * nsa_decode's. Arguments as nsa_decode plus k_bounds; the workspace is
 * nsa_workspace_size(NSA_OP_DECODE). On shapes other than the bf16, d = 128,
 * 16 heads per KV head, selection block 64 fast path, the CUDA-core path
 * computes the bounds from the keys (k_bounds unused). */
NSA_API nsa_status nsa_decode_quest(const nsa_params* p, const void* q, const void* k_cache,
                                    const void* v_cache, const int32_t* seq_lens,
                                    const void* k_cmp, const void* v_cmp, const void* k_bounds,
                                    const float* w_gate, void* out, int32_t* sel_idx,
                                    void* workspace, size_t ws_bytes, void* stream);

/* nsa_decode without a workspace argument, for callers that cannot allocate
 * device memory: code that runs while a stream capture is in progress
 * (cudaMalloc is not permitted during a global-mode capture), real-time or
 * callback threads that must not block in an allocator, and hosts whose device
 * memory is owned by another runtime's pool. Nothing here states whether the
 * call itself can be captured into a graph.
 * The sources describe no such call; it has no counterpart in the method.
 *   Same arguments and results as nsa_decode, minus workspace / ws_bytes. The
 *   scratch is a static 64 MiB device array in this library, held on every GPU
 *   that loads it until the process exits. Shapes whose decode scratch
 *   (nsa_workspace_size(NSA_OP_DECODE)) exceeds 64 MiB are rejected with
 *   NSA_ERR_UNSUPPORTED before anything runs (32 sequences of 65536 tokens
 *   with 4 KV heads need about 39 MB).
 *   The first call on each device looks the scratch's address up (once, with
 *   that device current); make that first call before any stream capture.
 *   All calls share the one scratch: calls that overlap on the GPU (different
 *   streams, no ordering) race and corrupt each other's results. Nothing in
 *   it must start at zero: every call writes each scratch byte it reads.
 *   No device memory is allocated or freed, by this call or any library
 *   routine it uses. */
NSA_API nsa_status nsa_decode_noalloc(const nsa_params* p, const void* q, const void* k_cache,
                                      const void* v_cache, const int32_t* seq_lens,
                                      const void* k_cmp, const void* v_cmp, const float* w_gate,
                                      void* out, int32_t* sel_idx, void* stream);

/* MoBA causal prefill (EP94 notes §九/§十).
 *   q [B, T, Hq, d]; k, v [B, T, Hkv, d]; out [B, T, Hq, d].
 *   Block m = sel_block; each (token t, head h) keeps its own block t/m and the
 *   top_n - 1 earlier blocks by q . mean(K_block) (ties to the lower index),
 *   then one causal softmax over the kept tokens.
 *   sel_idx    [B, T, Hq, top_n] int32 or NULL (ascending, -1 padded). */
NSA_API nsa_status moba_prefill(const nsa_params* p, const void* q, const void* k, const void* v,
                        void* out, int32_t* sel_idx, void* workspace, size_t ws_bytes,
                        void* stream);

/* Synchronise `stream`, then read and clear this device's error word:
 * NSA_ERR_DEVICE_TIMEOUT if a bounded wait gave up, NSA_ERR_INVALID_ARGUMENT
 * if a kernel met an out-of-range sequence length, else NSA_OK (or
 * NSA_ERR_CUDA if the synchronisation itself failed). */
NSA_API nsa_status nsa_check(void* stream);

/* Test hook for the failure path: launches one kernel that waits for *flag
 * (device int) to become nonzero for at most max_iters polls, then sets the
 * error word and returns. Nothing sets the flag in the test, so nsa_check must
 * report NSA_ERR_DEVICE_TIMEOUT while the context stays usable. */
NSA_API nsa_status nsa_debug_bounded_wait(const int32_t* flag, int max_iters, void* stream);

/* Kernel trace (timing aid). While enabled, every kernel this library
 * launches is bracketed by two CUDA events recorded on its stream; records
 * accumulate until the next nsa_trace_enable call. Enabling clears the
 * record; at most `capacity` launches are kept (later ones are counted but
 * not timed). Events are created at enable time, so the traced region itself
 * creates none. Not for concurrent use from several host threads. */
NSA_API nsa_status nsa_trace_enable(int on, int capacity);

/* Restrict event brackets to kernels whose name starts with `prefix` (NULL or
 * "" = every kernel). Every launch is still counted. Events between kernels
 * delay the next launch slightly, so timing only the kernel of interest keeps
 * the rest of the timeline undisturbed. */
NSA_API nsa_status nsa_trace_set_filter(const char* prefix);

/* Number of launches since the trace was enabled (including untimed ones). */
NSA_API int nsa_trace_count(void);

/* Number of launches bracketed with events (see nsa_trace_set_filter). */
NSA_API int nsa_trace_timed(void);

/* Name and device duration (ms) of timed launch i (0 <= i < nsa_trace_timed();
 * synchronises on its stop event). NSA_ERR_INVALID_ARGUMENT when out of range. */
NSA_API nsa_status nsa_trace_get(int i, const char** name, float* ms);

/* Static description of a status code. */
NSA_API const char* nsa_status_string(nsa_status s);

/* Detail of the last error returned on this host thread ("" if none). */
NSA_API const char* nsa_last_error_detail(void);

#ifdef __cplusplus
}
#endif

#endif /* NSA_B200_H_ */
