// Internal declarations shared by the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hyb_attn.h"

namespace hyb {

constexpr int kTile = 64;             // tokens per attention chunk (one ring stage holds K and V)
constexpr int kBoxRows = 16;          // rows per TMA box of a ragged chunk
constexpr int kMaxCluster = 16;       // CTAs per unit (thread-block cluster; above 8 is non-portable)
constexpr int kSelCache = 256;        // selection entries a CTA keeps in shared memory
constexpr int kMaxGroup = 4;          // query heads per KV head
constexpr uint64_t kWaitLimit = 1000000000ull;  // ns: a kernel-internal wait gives up after ~1 s (default)

// Per-slot layout of a split-K partial: m[4], l[4], dsel[4], pad[4], acc[4][D], nsel[4][D].
__host__ __device__ constexpr int partial_floats(int D) { return 16 + 8 * D; }

// Merge of a unit's outputs across its C CTAs: rank r merges outputs
// [e0(r), e1(r)) of the unit's G x D (e0(r) = r G D / C, rounded down).  Its
// receiving buffer holds one slot per sending rank: a header of 12 floats (per
// head: the exact part's running max and weight sum, and D_glob - D_sel;
// padded to 16) and a (exact part, N_glob - N_sel) pair per output of the slice.
__host__ __device__ constexpr int merge_slice_begin(int GD, int C, int r) { return r * GD / C; }
__host__ __device__ constexpr int merge_stride(int GD, int C) { return 16 + ((2 * ((GD + C - 1) / C) + 3) & ~3); }
__host__ __device__ constexpr int merge_floats_for(int D, int C) { return C * merge_stride(kMaxGroup * D, C); }
// the largest buffer over every cluster size
__host__ __device__ constexpr int merge_floats(int D, int C = 1) {
  return C > kMaxCluster ? 0
                         : (merge_floats_for(D, C) > merge_floats(D, C + 1) ? merge_floats_for(D, C)
                                                                               : merge_floats(D, C + 1));
}

struct Geometry {        // a decode at length T with the configuration's uniform budget (host: plan, sizes)
  int64_t T;
  int64_t nb;            // candidate blocks
  int64_t k_eff;         // min(top_k, nb)
  int64_t sink_len;      // min(S, T)
  int64_t win_start;     // max(S, T - W) (== T when T <= S)
  int64_t ev_end;        // T - W when T > S + W else S
  int32_t n_sink_chunks, n_win_chunks, chunks_per_block, n_sel_chunks, chunks_per_unit;
};

constexpr int kMaxRaggedRows = 128;   // batch rows that may have lengths of their own
constexpr int kMaxHeadBudgets = 32;   // KV heads that may have a (top_k, window) of their own

// What makes one unit's length and budget differ from another's.  Row b of the
// batch has length T - row_lag[b] (every row grows by the same appends), KV
// head h has window head_W[h] and top-k head_k[h]; uniform when the flags are 0.
struct UnitTables {
  int32_t ragged, per_head;
  int32_t row_lag[kMaxRaggedRows];
  int32_t head_W[kMaxHeadBudgets];
  int32_t head_k[kMaxHeadBudgets];
};

// One unit's geometry at the current step, derived on the device from the
// launch's T, S, W, Bk, top_k, the tables and the number of appends whose
// evictions are not yet folded (`pending`).
struct UnitGeo {
  int32_t T;             // this row's length
  int32_t W, top_k;      // this head's window and top-k
  int32_t sink_len, win_start, ev_end, nb, k_eff;
  int32_t n_sink_chunks, n_win_chunks, n_sel_chunks;
  int32_t fold_begin, fold_end;   // evicted positions not yet in the state
};

__host__ __device__ inline int32_t ev_end_at(int32_t T, int32_t S, int32_t W) { return T > S + W ? T - W : S; }

// tb == null: every unit at (T, W, top_k)
__host__ __device__ inline UnitGeo unit_geo(const UnitTables* tb, int unit, int Hkv, int32_t T, int32_t S,
                                            int32_t W, int32_t Bk, int32_t top_k, int32_t cpb, int32_t pending) {
  UnitGeo g;
  const int b = unit / Hkv, h = unit - b * Hkv;
  g.T = T - ((tb != nullptr && tb->ragged) ? tb->row_lag[b] : 0);
  g.W = (tb != nullptr && tb->per_head) ? tb->head_W[h] : W;
  g.top_k = (tb != nullptr && tb->per_head) ? tb->head_k[h] : top_k;
  g.sink_len = g.T < S ? g.T : S;
  g.win_start = g.T > S ? (g.T - g.W > S ? g.T - g.W : S) : g.T;
  g.ev_end = ev_end_at(g.T, S, g.W);
  g.nb = g.ev_end > S ? (g.ev_end - S + Bk - 1) / Bk : 0;
  g.k_eff = g.top_k < g.nb ? g.top_k : g.nb;
  g.n_sink_chunks = (g.sink_len + kTile - 1) / kTile;
  g.n_win_chunks = (g.T - g.win_start + kTile - 1) / kTile;
  g.n_sel_chunks = g.k_eff * cpb;
  g.fold_end = g.ev_end;
  g.fold_begin = ev_end_at(g.T - pending > 0 ? g.T - pending : 0, S, g.W);
  return g;
}

struct FusedParams {           // one decode (or, with q == null, the fold only) of one layer
  const __nv_bfloat16* q;       // [B][Hq][D]
  float* mu;                    // [units][max_blocks][D]  (pending evictions folded in place)
  float* var;
  float* H;                     // [units][D][D]
  float* zk;                    // [units][D]
  float* zv;
  float* n;                     // [units]
  __nv_bfloat16* k_cache;       // [units][cap][D]
  __nv_bfloat16* v_cache;
  const __nv_bfloat16* k_new;   // optional token written at each row's position T: [units][D]
  const __nv_bfloat16* v_new;
  float* scores;                // [units][max_blocks] (workspace, or the caller's buffer)
  const int32_t* sel_given;     // [units][top_k] caller's selection, or null: top-k of the scores
  int32_t* sel;                 // [units][top_k] selections that do not fit shared memory
  int32_t* sel_out;             // optional copy of the selection
  uint32_t* status;
  float* out;                   // [B][Hq][D]
  int64_t cap, max_blocks;
  int32_t T, S, W, Bk, top_k;   // T: the longest row; W, top_k: uniform budget (top_k: row stride of sel)
  int32_t pending;              // appends whose evictions are not folded yet
  int32_t chunks_per_block;
  int32_t units, Hkv, G, C;     // C: CTAs (cluster size) per unit
  int32_t mstride;              // merge: floats per sending rank's slot (merge_stride)
  int32_t mslice[kMaxCluster + 1];  // merge: rank r merges outputs [mslice[r], mslice[r + 1])
  float scale;
  uint64_t wait_ns;             // limit of every bounded wait for progress inside the kernel
  uint32_t test_flags;          // HYB_TEST_* (0 in normal use)
};

// The decode kernel's per-unit tables, a launch parameter of their own only in
// the variant for contexts that have them (the uniform variant's launches stay
// small).
template <bool kTab> struct TabArg {};
template <> struct TabArg<true> { UnitTables tb; };

struct AppendParams {       // write n tokens per unit at each row's positions [T_b, T_b + n)
  const __nv_bfloat16* k_new; // [units][n][D]
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  int64_t cap;
  int32_t T, units, Hkv, n;
  UnitTables tb;
};

struct FoldParams {         // fold every unit's pending evicted positions into the state
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  float* H; float* zk; float* zv; float* n; float* mu; float* var;
  int64_t cap, max_blocks;
  int32_t T, S, W, Bk, pending;
  int32_t units, Hkv;
  UnitTables tb;
};
// pending appends from which a decode or a state sync folds the evictions with
// fold_kernel (one dense pass) instead of inside the decode kernel
constexpr int64_t kFoldKernelMin = 5;

struct InitParams {          // the state of every unit's evicted range [S, ev_end(T_b, W_h))
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  float* H; float* zk; float* zv; float* n; float* mu; float* var;
  double* H64;                // [units][D][D] accumulators
  double* z64;                // [units][2][D]
  uint32_t* status;
  int64_t cap, max_blocks;
  int32_t T, S, W, Bk;
  int32_t units, Hkv, nb_max, ev_max;   // the largest block count and evicted length over the units
  int32_t tokens_per_cta;
  UnitTables tb;
};

// Launchers (kernels live in the .cu files); return cudaError_t of the launch.
// Decode-path launches use programmatic dependent launch; every kernel waits
// for its predecessor grid before it touches memory, so stream order holds.
// maps: K and V with 64-row boxes, then K and V with 16-row boxes.
cudaError_t launch_append(const AppendParams& p, int D, cudaStream_t s);
// stream: some unit of the launch has more than kStreamBlocks candidate blocks
// (the variant whose statistics warps keep the top-k while scoring)
constexpr int kStreamBlocks = 512;
cudaError_t launch_fused(const CUtensorMap* maps, const FusedParams& p, const UnitTables& tb, bool stream, int D,
                         cudaStream_t s);
cudaError_t prepare_fused(int D);
// clusters of c CTAs of the decode kernel the current device can hold at once (0: none)
int fused_max_clusters(int D, int c);
cudaError_t launch_init(const InitParams& p, int D, cudaStream_t s);
// The multi-query decode kernel (k_multi.cu): NR (2 or 4) consecutive new
// tokens per unit in one launch.  Requirements the host checks: uniform
// lengths and budgets, top_k <= 32, window >= NR - 1, the last row's block
// count <= multi_score_capacity(NR); p.mstride / p.mslice computed with
// multi_merge_stride over NR * G * D outputs.
int multi_rows_max();
int multi_score_capacity(int NR);
int multi_merge_stride(int NR, int GD, int C);
cudaError_t prepare_multi(int D);
int multi_max_clusters(int D, int NR, int c);
cudaError_t launch_multi(const CUtensorMap* maps, const FusedParams& p, int D, int NR, cudaStream_t s);
cudaError_t launch_fold(const FoldParams& p, int D, cudaStream_t s);
// per device, before the first launch: shared-memory size, cluster and carveout attributes
cudaError_t prepare_state(int D);

}  // namespace hyb
