/*
 * hyb_attn.h -- C ABI of the B200 (sm_100a) decode-step hybrid sparse + linear
 * attention.
 *
 * What one decode step computes, for each batch row b and KV head h (a "unit")
 * with the G = n_q_heads / n_kv_heads query heads of its group:
 *
 *   positions [0, T) of the unit's history split into            (SALSA: Training-
 *     sinks    [0, min(S, T)),                                    Consistent Sparse
 *     window   [max(S, T - W), T),                                Caching with Sink
 *     evicted  L = [S, T - W)  (empty when T <= S + W),           Preservation for
 *   L tiled into blocks j = [S + j*Bk, min(S + (j+1)*Bk, T - W))  Linearized LLMs,
 *   from position S; the newest block may be partial.             abstract)
 *
 *   block score  score_j = sum_{i in group} q'_i . mu_j + 1/2 sum_c q'_ic^2 var_jc,
 *   q' = q * scale, mu_j / var_j the block's key mean and population variance
 *   (SPLA: Block Sparse Plus Linear Attention for Long Context Modeling --
 *   abstract, and sections "Principled Block Selection via Taylor Expansion" and
 *   "Grouped Sparsity");
 *
 *   the top_k blocks by score (ties to the lower index) are attended exactly
 *   together with the sinks and the window: weight exp(s_t), s_t = q'.k_t;
 *   every other evicted token gets the first-order Taylor weight 1 + s_t (SLAKE:
 *   Softmax-Approximated Training-Free Linear Attention with KV-Cache Eviction
 *   for Long-Sequence LLMs, abstract, PTAA), computed without reading it as the
 *   global linear state (H = sum_L k v^T, zk = sum_L k, zv = sum_L v, n = |L|)
 *   minus the selected blocks' own (1 + s_t) terms (SPLA abstract, section
 *   "IO-Efficient Implementation");
 *
 *   one shared normaliser:
 *     o_i = [sum_X e^{s_t} v_t + sum_{L\sel} (1 + s_t) v_t] / [sum_X e^{s_t} + sum_{L\sel} (1 + s_t)].
 *
 * Conventions for every call:
 *   - The caller owns all device memory and every stream; the library owns only
 *     the host-side context.  Pointers are device pointers unless the name ends
 *     in _host, and must be 16-byte aligned.
 *   - Calls are asynchronous: they enqueue kernels on `stream` and return.
 *   - Return value 0 is success; a negative HYB_E* code means nothing was
 *     enqueued (except HYB_ECUDA, where a launch failed).  No exception or abort
 *     crosses the ABI.
 *   - Anomalies found on the device (non-finite output, denominator <= 0, an
 *     out-of-range block index in a caller-given selection, a timed-out wait)
 *     set bits in a device status word, read with hyb_attn_status().
 *   - Batch rows share the length T unless the context was created with
 *     per-row lengths (hyb_attn_init_rows); every row then grows by the same
 *     appends.  One context holds one layer.
 *   - Supported: head_dim 64 or 128; group size G in {1, 2, 4};
 *     batch * n_kv_heads * capacity < 2^31.
 */
#ifndef HYB_ATTN_H
#define HYB_ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes -------------------------------------------------------- */
#define HYB_OK          0
#define HYB_EINVAL     (-1)  /* bad shape, pointer, alignment or argument */
#define HYB_ECAPACITY  (-2)  /* append would pass `capacity` tokens */
#define HYB_ECUDA      (-3)  /* a CUDA call or kernel launch failed */
#define HYB_ESTATE     (-4)  /* call not valid in the current state (e.g. decode at T = 0) */
#define HYB_ENOMEM     (-5)  /* host allocation of the context failed */
#define HYB_ESCRATCH   (-6)  /* the call needs more scratch than the library's fixed device area */

/* ---- device status bits (hyb_attn_status) -------------------------------- */
#define HYB_STATUS_NONFINITE     0x1u  /* an output element was NaN or Inf */
#define HYB_STATUS_DENOMINATOR   0x2u  /* a shared normaliser was <= 0 (no clamp is applied) */
#define HYB_STATUS_BAD_SELECTION 0x4u  /* a caller-given block index was out of range (skipped) */
#define HYB_STATUS_TIMEOUT       0x8u  /* a bounded wait inside a kernel gave up */
#define HYB_STATUS_NAN_SCORE     0x10u /* a block score was NaN (ranked last) */

/* ---- failure injection for tests (hyb_attn_set_test_flags) ---------------- */
#define HYB_TEST_WITHHOLD_SCORES 0x1u  /* rank 1 of every unit's cluster does not hand its block
                                          scores to the other ranks, whose bounded wait for them
                                          then runs out (HYB_STATUS_TIMEOUT; outputs invalid) */

/* ---- configuration ------------------------------------------------------- */
typedef struct hyb_attn_config {
  int32_t batch;       /* B  >= 1 */
  int32_t n_q_heads;   /* Hq >= 1, a multiple of n_kv_heads; query head i belongs to KV head i / G */
  int32_t n_kv_heads;  /* Hkv >= 1 */
  int32_t head_dim;    /* d: 64 or 128 */
  int32_t block_size;  /* Bk >= 1: tokens per selectable block of the evicted stream */
  int32_t n_sink;      /* S >= 0: leading positions always attended exactly */
  int32_t window;      /* W >= 0: trailing positions always attended exactly */
  int32_t top_k;       /* k >= 0: blocks attended exactly per (b, KV head) */
  int64_t capacity;    /* rows per (b, KV head) in the KV cache, >= 1 */
  float   scale;       /* q' = q * scale; 0 selects 1/sqrt(head_dim) */
  /* Per-KV-head budgets (host arrays of n_kv_heads entries, read when a context
   * is created), or NULL for every head at (window, top_k): KV head h keeps
   * window head_window[h] >= window and selects head_top_k[h] <= top_k blocks.
   * `window` is then the smallest window (it sizes the statistics arrays) and
   * `top_k` the largest top-k (the row length of selection arrays, whose
   * entries past a head's own count are -1).  Both or neither; at most
   * 32 KV heads.  (SALSA abstract: sparse-cache budgets allocated per layer;
   * per head here, the same knob one level finer.) */
  const int32_t* head_window;
  const int32_t* head_top_k;
} hyb_attn_config;

/* Sizes (in elements, except where noted) of the caller-owned buffers for a
 * configuration.  max_blocks = ceil(max(0, capacity - S - W) / Bk) is the row
 * count of the block-statistics arrays per unit. */
typedef struct hyb_attn_sizes {
  int64_t kv_cache_elems;   /* B * Hkv * capacity * d   (bf16, each of K and V) */
  int64_t H_elems;          /* B * Hkv * d * d          (fp32) */
  int64_t z_elems;          /* B * Hkv * d              (fp32, each of zk and zv) */
  int64_t n_elems;          /* B * Hkv                  (fp32) */
  int64_t max_blocks;       /* ceil(max(0, capacity - S - W) / Bk) */
  int64_t stats_elems;      /* B * Hkv * max_blocks * d (fp32, each of mu and var) */
  int64_t workspace_bytes;  /* scratch the library uses between and inside calls */
} hyb_attn_sizes;

/* Caller-owned device buffers of one layer.  Layouts (row-major, unit index
 * u = b * Hkv + h):
 *   k_cache, v_cache  bf16 [B][Hkv][capacity][d]   position t of unit u at row u*capacity + t
 *   H                 fp32 [B][Hkv][d][d]          H[u][r][c] = sum_{t in L} k_t[r] v_t[c]
 *   zk, zv            fp32 [B][Hkv][d]
 *   n                 fp32 [B][Hkv]                |L| (exact up to 2^24)
 *   mu, var           fp32 [B][Hkv][max_blocks][d] key mean / population variance of block j
 *   workspace         hyb_attn_sizes.workspace_bytes bytes, 256-byte aligned; contents are
 *                     private to the library.  Contexts whose calls are serialised on one
 *                     stream may share one workspace.
 * The state arrays (H, zk, zv, n, mu, var) are written by hyb_attn_init and hold
 * the evicted tokens up to the last decode: a token that leaves the window is
 * folded in by the next decode (which reads the state anyway), or by
 * hyb_attn_sync_state.  After hyb_attn_sync_state, copying them together with
 * the caches and T is a complete checkpoint of the layer (restored with
 * hyb_attn_attach).
 * There is no separate running sum and sum of squares of the newest (open)
 * block: its mean and variance rows are updated in place, one evicted token at
 * a time (Welford's update), so the open block is an ordinary candidate row of
 * mu / var and a decode reads one layout for every block. */
typedef struct hyb_attn_buffers {
  void*  k_cache;
  void*  v_cache;
  float* H;
  float* zk;
  float* zv;
  float* n;
  float* mu;
  float* var;
  void*  workspace;
  size_t workspace_bytes;
} hyb_attn_buffers;

typedef struct hyb_attn_ctx hyb_attn_ctx;  /* opaque host-side handle, one per layer */

/* Host-only description of how one decode at length T is split into work
 * (exposed for tests and tooling; no device access). */
typedef struct hyb_attn_plan_info {
  int64_t T;
  int64_t n_blocks;          /* nb: candidate blocks at T */
  int64_t k_eff;             /* min(top_k, nb) */
  int64_t exact_tokens;      /* |sinks| + |window| + tokens of k_eff full blocks (upper bound) */
  int32_t chunks_per_unit;   /* 64-token pieces of the exact set per unit (fixed for a given T) */
  int32_t cluster_ctas;      /* CTAs per unit (one thread-block cluster); the device may use fewer */
  int32_t grid_ctas;         /* grid of the decode kernel: units * cluster_ctas */
} hyb_attn_plan_info;

/* Fill `out` with the buffer sizes of `cfg`.  Host only; never touches a GPU.
 * Returns HYB_EINVAL for an unsupported configuration. */
int hyb_attn_query_sizes(const hyb_attn_config* cfg, hyb_attn_sizes* out);

/* Workspace bytes for `cfg` (0 for an unsupported configuration).  Host only. */
size_t hyb_attn_workspace_size(const hyb_attn_config* cfg);

/* Work split of a decode at length T on a device with `n_sm` multiprocessors.
 * Host only. */
int hyb_attn_plan(const hyb_attn_config* cfg, int64_t T, int32_t n_sm, hyb_attn_plan_info* out);

/* Create a context for one layer whose caches already hold T0 tokens per unit
 * (positions [0, T0) of k_cache / v_cache), and build the state of those tokens
 * on `stream`: the linear state over L = [S, T0 - W) and the statistics of every
 * block of L, the newest possibly partial (SPLA abstract: block statistics and a
 * recurrent state of the unselected tokens).  The context records the buffer
 * pointers; the caller keeps them alive until hyb_attn_destroy.  The current
 * CUDA device must be the device owning the buffers.
 * Errors: HYB_EINVAL (cfg, pointers, alignment, T0 outside [0, capacity]),
 * HYB_ENOMEM, HYB_ECUDA.  On error *out is set to NULL. */
int hyb_attn_init(hyb_attn_ctx** out, const hyb_attn_config* cfg, const hyb_attn_buffers* buf,
                  int64_t T0, cudaStream_t stream);

/* As hyb_attn_init, with a length of its own for every batch row: row_T0 is a
 * host array of `batch` lengths in [1, capacity] (at most 128 rows), positions
 * [0, row_T0[b]) of row b's caches are its history, and each row's state is
 * built over its own evicted range.  Every later append or decode step moves
 * all rows by the same count; hyb_attn_length reports the longest row and
 * hyb_attn_row_length each one.  A decode attends, for row b, to [0, T_b) with
 * its own window, blocks and top-k.  Errors as hyb_attn_init. */
int hyb_attn_init_rows(hyb_attn_ctx** out, const hyb_attn_config* cfg, const hyb_attn_buffers* buf,
                       const int64_t* row_T0, cudaStream_t stream);

/* Create a context over buffers that already hold the synced state of a
 * history of length T -- the caches' positions [0, T) and H, zk, zv, n, mu,
 * var exactly as hyb_attn_sync_state left them (a checkpoint copied back by the
 * caller) -- without rebuilding the state, so that the next decode is
 * bit-identical to the one the checkpointed context would have made.  Resets
 * the device status word.  Errors as hyb_attn_init. */
int hyb_attn_attach(hyb_attn_ctx** out, const hyb_attn_config* cfg, const hyb_attn_buffers* buf,
                    int64_t T, cudaStream_t stream);
/* hyb_attn_attach for a checkpoint of a context with per-row lengths (row_T:
 * host array of `batch` lengths, as hyb_attn_row_length reported them). */
int hyb_attn_attach_rows(hyb_attn_ctx** out, const hyb_attn_config* cfg, const hyb_attn_buffers* buf,
                         const int64_t* row_T, cudaStream_t stream);

/* Append one token per unit: k_new, v_new bf16 [B][Hkv][d].  The token is
 * written at position T; then T += 1.  If the token at position T - W - 1
 * (after the increment) lies at or past S it has left the window: the next
 * decode (or hyb_attn_sync_state) folds it into H, zk, zv, n (a rank-1 update,
 * SPLA "Recurrence") and into the running mean / population variance of its
 * block (Welford's update), which opens a new block when the previous one is
 * full.  Any number of appends may come between decodes.  Errors: HYB_EINVAL
 * (null or misaligned pointers), HYB_ECAPACITY (T == capacity), HYB_ECUDA. */
int hyb_attn_append(hyb_attn_ctx* ctx, const void* k_new, const void* v_new, cudaStream_t stream);

/* Append n >= 1 tokens per unit in one launch (a prefill continuation):
 * k_new, v_new bf16 [B][Hkv][n][d], token j written at position T + j; then
 * T += n.  Equivalent to n calls of hyb_attn_append: every token that leaves the
 * window is folded by the next decode (or hyb_attn_sync_state) into H, zk, zv,
 * n and its block's statistics, in position order (SPLA "Recurrence"; several
 * evicted tokens make a small dense K^T V update of H).  Errors: HYB_EINVAL
 * (null or misaligned pointers, n < 1 or n > 65535), HYB_ECAPACITY
 * (T + n > capacity), HYB_ECUDA. */
int hyb_attn_append_chunk(hyb_attn_ctx* ctx, const void* k_new, const void* v_new, int32_t n,
                          cudaStream_t stream);

/* Fold every token evicted since the last decode into the state arrays, so that
 * they describe L = [S, T - W) exactly (for a checkpoint, or to read them).  A
 * no-op when nothing is pending; one launch otherwise (the dense fold pass when
 * 5 or more tokens are pending, else the decode kernel in fold-only mode).
 * Errors: HYB_EINVAL, HYB_ECUDA. */
int hyb_attn_sync_state(hyb_attn_ctx* ctx, cudaStream_t stream);

/* One decode step at the current length T for every unit:
 *   q           bf16 [B][Hq][d]  (input)
 *   out         fp32 [B][Hq][d]  (output)
 *   sel_out     int32 [B][Hkv][top_k] or NULL: the selected block indices,
 *               ascending, -1 padded when nb < top_k
 *   scores_out  fp32 [B][Hkv][max_blocks] or NULL: the block scores (entries
 *               [0, nb) of each unit are written)
 * One kernel launch: per unit a thread-block cluster scores the blocks, folds in
 * the tokens evicted since the previous decode, forms the global linear term
 * phi(q)^T state, selects the top-k, attends sinks, window and selected blocks
 * exactly (split-K over the cluster, with the selected blocks' (1 + s)
 * subtraction) and merges under the shared normaliser.  When 5 or more evicted
 * tokens are pending (a chunked append, or many appends since the last fold),
 * a dense fold pass over them is launched first (H += K^T V over the run, zk,
 * zv, n, and the touched blocks' statistics merged pairwise).
 * Errors: HYB_EINVAL (null or misaligned pointers), HYB_ESTATE (T == 0),
 * HYB_ECUDA. */
int hyb_attn_decode(hyb_attn_ctx* ctx, const void* q, float* out, int32_t* sel_out,
                    float* scores_out, cudaStream_t stream);

/* hyb_attn_decode followed by hyb_attn_append(k_new, v_new) in the same
 * launch: the decode kernel also writes the new token at row T, then
 * T += 1 -- one decode step of a generation loop.  The decode attends to
 * [0, T) as stored before the call.  Errors: those of both calls. */
int hyb_attn_decode_append(hyb_attn_ctx* ctx, const void* q, const void* k_new, const void* v_new,
                           float* out, int32_t* sel_out, float* scores_out, cudaStream_t stream);

/* n decode steps of n consecutive new tokens (speculative verification of a
 * draft of n tokens): row j decodes q[j] at length T + j -- it attends to the
 * stored history and to the chunk's tokens 0 .. j-1, with its own window, block
 * statistics, scores and top-k -- and then appends token j; T += n in all.
 * The result is that of n calls of hyb_attn_decode_append.  The rows go in
 * groups of 4 (then 2, then 1) through the multi-query kernel, one launch per
 * group: what the group's rows share (the sinks and windows, the block
 * statistics, the linear state, the blocks several rows select) is read once.
 * A group falls back to one launch per row when the context has per-row
 * lengths or per-head budgets, top_k > 32, window < rows - 1, or more blocks
 * than the kernel keeps scores for (4096 / rows per row).
 *   q       bf16 [n][B][Hq][d]     k_new, v_new  bf16 [n][B][Hkv][d]
 *   out     fp32 [n][B][Hq][d]     sel_out       int32 [n][B][Hkv][top_k] or NULL
 * Errors: HYB_EINVAL (null or misaligned pointers, n < 1), HYB_ESTATE (T == 0),
 * HYB_ECAPACITY (T + n > capacity), HYB_ECUDA.  On an error at row j, rows
 * before j have been decoded and appended. */
int hyb_attn_decode_chunk(hyb_attn_ctx* ctx, const void* q, const void* k_new, const void* v_new, int32_t n,
                          float* out, int32_t* sel_out, cudaStream_t stream);

/* As hyb_attn_decode, with the block selection given by the caller instead of
 * the top-k: sel int32 [B][Hkv][top_k], each row ascending and distinct, -1
 * entries ignored.  Indices outside [0, nb) are skipped and raise
 * HYB_STATUS_BAD_SELECTION.  Used to compare outputs for a fixed selection. */
int hyb_attn_decode_with_selection(hyb_attn_ctx* ctx, const void* q, const int32_t* sel,
                                   float* out, cudaStream_t stream);

/* Decode with strided block selection ("SPLA: Block Sparse Plus Linear
 * Attention for Long Context Modeling", table of contents: "Strided block
 * selection" -- the page gives the heading only; the reading implemented
 * here is a fixed stride of always-exact blocks): the last block of every
 * `stride` consecutive candidate blocks (index j with j % stride == stride - 1)
 * is exact, and the top-k_top blocks by the usual score among the others (ties
 * to the lower index) are added.  The union replaces the top-k as the decode's
 * selection; the rest of the decode is hyb_attn_decode's.
 *   q       bf16 [B][Hq][d], device, 16-byte aligned;  out fp32 [B][Hq][d].
 *   k_top   >= 0;  stride >= 1 (stride 1: every block; stride > nb: plain top-k).
 *   sel_out optional int32 [B][Hkv][top_k] (device): the selection, ascending,
 *           -1 padded.
 * The configuration's top_k must hold the union (nb / stride + min(k_top,
 * the other blocks)), else HYB_EINVAL; so must one length and one budget for
 * every unit (no per-row lengths, no per-head budgets).  Launches: one
 * selection launch that reads the block statistics (a block holding evictions
 * not folded yet, at most 4 tokens, is scored from its statistics with them
 * folded in registers), then the decode, which folds them into the state as
 * hyb_attn_decode does; 5 or more pending evictions are first folded by one
 * dense pass.  Scores that are NaN raise HYB_STATUS_NAN_SCORE. */
int hyb_attn_decode_strided(hyb_attn_ctx* ctx, const void* q, int32_t k_top, int32_t stride, float* out,
                            int32_t* sel_out, cudaStream_t stream);

/* One decode + append step from host memory, for callers whose inputs and
 * outputs live on the host: copies q_host (bf16 [B][Hq][d]) and k_host, v_host
 * (bf16 [B][Hkv][d]) to device staging space in the workspace, runs
 * hyb_attn_decode_append (hyb_attn_decode without k_host), and copies the fp32 output back to
 * out_host ([B][Hq][d]).  All copies are cudaMemcpyAsync on `stream`; host
 * buffers should be pinned for the copies to be asynchronous.  k_host / v_host
 * may be NULL to skip the append.  The call returns after enqueueing; the output
 * is valid once `stream` has been synchronised. */
int hyb_attn_step_host(hyb_attn_ctx* ctx, const void* q_host, const void* k_host,
                       const void* v_host, float* out_host, cudaStream_t stream);

/* A whole decode step of several layers from host memory, with one copy in and
 * one copy out: in_host holds, layer after layer, that layer's q (bf16
 * [B][Hq][d]) then k and v of the appended token (bf16 [B][Hkv][d] each);
 * out_host receives, layer after layer, the fp32 [B][Hq][d] outputs.  One
 * cudaMemcpyAsync brings every layer's input to `staging` (caller-owned device
 * memory, 256-byte aligned, at least hyb_attn_step_layers_staging_bytes), the
 * layers' decode + append launches follow back to back on `stream` (chained
 * as usual), and one cudaMemcpyAsync returns every output.  Host buffers
 * should be pinned.  The layers may have different budgets and shapes; their
 * contexts may share one workspace (the calls are serialised on `stream`).
 * Errors: HYB_EINVAL, HYB_ECAPACITY (a layer is full: nothing is enqueued),
 * HYB_ECUDA. */
size_t hyb_attn_step_layers_staging_bytes(hyb_attn_ctx* const* ctxs, int32_t n_layers);
int hyb_attn_step_layers_host(hyb_attn_ctx* const* ctxs, int32_t n_layers, const void* in_host, float* out_host,
                              void* staging, size_t staging_bytes, cudaStream_t stream);

/* Decode without any allocation, for callers that cannot allocate device
 * memory themselves: code that runs under an allocator it does not own (a
 * framework's caching pool, a plugin host, an embedded runtime) or that must
 * not call cudaMalloc/cudaFree on its hot path, where those calls synchronise
 * the device.  The pages have no counterpart for this call; it exists for the
 * library's users.
 *
 * Same arguments and result as hyb_attn_decode without scores_out, but the
 * per-call scratch (the block scores and the selection) comes from a fixed
 * device array inside the library, of HYB_NOALLOC_SCRATCH_BYTES (16 MiB) per
 * GPU, that every GPU which loads the library holds until the process exits.
 * A configuration whose decode scratch exceeds it is rejected with
 * HYB_ESCRATCH.  The call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.  Its device status bits go to the context's
 * status word, as for every other call (read with hyb_attn_status).
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  The current device must be the context's device.  All calls share
 * the one array and it keeps the last call's contents (nothing in it needs to
 * start at zero: a decode writes every score and selection entry before it
 * reads it), so calls whose work overlaps on the GPU (two streams, two
 * threads) race on the array and must be serialised by the caller.
 * Errors: HYB_EINVAL, HYB_ESTATE, HYB_ESCRATCH, HYB_ECUDA. */
#define HYB_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int hyb_attn_decode_noalloc(hyb_attn_ctx* ctx, const void* q, float* out, int32_t* sel_out, cudaStream_t stream);

/* Current length T (host mirror; no device access): the longest row's. */
int64_t hyb_attn_length(const hyb_attn_ctx* ctx);

/* Current length of batch row b (host mirror), or -1 for a bad argument. */
int64_t hyb_attn_row_length(const hyb_attn_ctx* ctx, int32_t b);

/* Copy the device status word to *flags (synchronises `stream`); with clear != 0
 * reset it to zero afterwards.  Returns HYB_OK or HYB_ECUDA.  The status word
 * lives in the context's workspace, so reading it is a device-to-host copy on
 * the caller's stream followed by a synchronisation of that stream (the word is
 * valid only once the decodes before it have finished), and `clear` lets a
 * caller poll and reset in one call. */
int hyb_attn_status(hyb_attn_ctx* ctx, uint32_t* flags, int clear, cudaStream_t stream);

/* Profiling hook: when both events are non-NULL, every later decode records
 * `begin` just before and `end` just after its kernel on the decode's stream,
 * so the caller can time one decode alone.  Pass NULL, NULL to stop. */
int hyb_attn_set_timing_events(hyb_attn_ctx* ctx, cudaEvent_t begin, cudaEvent_t end);

/* Limit, in nanoseconds, of the kernels' bounded waits for progress (a ring
 * stage, the other ranks' scores, the selection); 0 restores the default of
 * 1 s.  A wait that runs out sets HYB_STATUS_TIMEOUT and its CTA skips the
 * rest of its work; the waits that guard a CTA's exit keep the default.
 * Accepted: 0 or [1e5, 6e10].  Host only. */
int hyb_attn_set_wait_limit(hyb_attn_ctx* ctx, uint64_t ns);

/* Failure injection for tests: HYB_TEST_* flags applied to every later decode
 * (0 turns them off).  No flag faults, traps or hangs the GPU; a withheld
 * hand-off makes a bounded wait run out.  Host only. */
int hyb_attn_set_test_flags(hyb_attn_ctx* ctx, uint32_t flags);

/* Release the host context (device buffers stay with the caller). */
void hyb_attn_destroy(hyb_attn_ctx* ctx);

/* Name and description of the last CUDA error that made a call on this thread
 * return HYB_ECUDA ("cudaSuccess: no error" if none).  Host only. */
const char* hyb_attn_last_cuda_error(void);

/* Static description of a return code. */
const char* hyb_attn_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* HYB_ATTN_H */
