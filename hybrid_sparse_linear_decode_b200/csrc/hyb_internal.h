// Internal declarations shared by the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hyb_attn.h"

namespace hyb {

constexpr int kTile = 64;             // tokens per attention chunk (one pipeline stage)
constexpr int kBoxRows = 16;          // rows per TMA box
constexpr int kStages = 3;            // attention pipeline depth per CTA
constexpr int kAttendThreads = 128;   // 4 warps; warp w takes tokens [16w, 16w+16) of a chunk
constexpr int kAttendCtasPerSm = 1;   // one per SM beside the select kernel's two
constexpr int kAttendMaxRegs = 200;   // with 2 select CTAs: 128*200 + 2*256*72 registers per SM
constexpr int kMaxAttendCtas = 1024;  // upper bound of the attention grid (sizes the workspace)
constexpr int kSelectThreads = 256;
constexpr int kSelectCtasPerSm = 2;
constexpr int kSelectMaxRegs = 72;    // 2 select CTAs + 1 attention CTA share an SM's registers
constexpr int kSelStages = 3;         // select pipeline depth per CTA
constexpr int kSelItemBytes = 16384;  // block statistics or state rows of one select work item
constexpr int kSelCache = 256;        // selection entries a CTA keeps in shared memory
constexpr int kMaxGroup = 4;          // query heads per KV head supported by the attention kernel
constexpr uint64_t kWaitLimit = 1000000000ull;  // ns: a kernel-internal wait gives up after ~1 s

// Select work items: a score item covers sel_item_blocks(D) consecutive blocks
// (their mean and variance rows), a linear item sel_item_rows(D) rows of H.
__host__ __device__ constexpr int sel_item_blocks(int D) { return kSelItemBytes / (8 * D); }
__host__ __device__ constexpr int sel_item_rows(int D) { return kSelItemBytes / (4 * D); }
__host__ __device__ constexpr int sel_lin_items(int D) { return D / sel_item_rows(D); }

// Per-slot layout of a split-K partial: m[4], l[4], dsel[4], pad[4], acc[4][D], nsel[4][D].
__host__ __device__ constexpr int partial_floats(int D) { return 16 + 8 * D; }

struct Geometry {        // everything a decode at length T needs, computed on the host
  int64_t T;
  int64_t nb;            // candidate blocks
  int64_t k_eff;         // min(top_k, nb)
  int64_t sink_len;      // min(S, T)
  int64_t win_start;     // max(S, T - W) (== T when T <= S)
  int64_t ev_end;        // T - W when T > S + W else S
  int32_t n_sink_chunks, n_win_chunks, chunks_per_block, n_sel_chunks, chunks_per_unit;
};

struct SelectParams {
  const __nv_bfloat16* q;     // [B][Hq][D]; null: fold the pending evictions only
  float* mu;                  // [units][max_blocks][D] (pending evictions folded in place)
  float* var;
  float* H;                   // [units][D][D]
  float* zk;                  // [units][D]
  float* zv;
  float* n;                   // [units]
  const __nv_bfloat16* k_cache;  // [units][cap][D]: keys / values of the pending evictions
  const __nv_bfloat16* v_cache;
  float* scores;              // [units][max_blocks]
  float* lin;                 // [units][lin_items][G][D + 1]: partial N_glob over row groups, D_glob in item 0
  uint32_t* status;
  int64_t max_blocks, cap;
  int64_t fold_begin, fold_end;  // evicted positions not yet in the state
  int32_t units, G, nb, S, Bk;
  int32_t score_items, lin_items, items_per_unit, total_items;
  float scale;
};

struct AttendParams {
  const __nv_bfloat16* q;     // [B][Hq][D]
  const float* scores;        // [units][max_blocks] block scores (select kernel)
  const int32_t* sel_given;   // [units][top_k] caller's selection, or null: top-k of the scores
  int32_t* sel;               // [units][top_k] selection rows that do not fit shared memory
  int32_t* sel_out;           // optional copy of the selection
  const float* lin;           // [units][lin_items][G][D + 1]
  float* partials;            // [units][splits][partial_floats(D)]
  uint32_t* tickets;          // [units]
  uint32_t* status;
  float* out;                 // [B][Hq][D]
  const __nv_bfloat16* k_new; // optional token appended after the decode: [units][D]
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_cache;     // written at position T when k_new is given
  __nv_bfloat16* v_cache;
  int64_t cap;                // cache rows per unit
  int64_t max_blocks;
  int32_t T, S, Bk, top_k, nb, k_eff;
  int32_t sink_len, win_start, ev_end;
  int32_t n_sink_chunks, n_win_chunks, chunks_per_block, chunks_per_unit;
  int32_t units, G, grid, lin_items;
  int32_t splits;             // CTAs per unit; CTA x works on unit x / splits
  float scale;
};

struct AppendParams {       // write one token per unit at position T
  const __nv_bfloat16* k_new; // [units][D]
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  int64_t cap, T;
  int32_t units;
};

struct InitParams {
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  float* H; float* zk; float* zv; float* n; float* mu; float* var;
  double* H64;                // [units][D][D] accumulators
  double* z64;                // [units][2][D]
  uint32_t* tickets_sel; uint32_t* tickets_att; uint32_t* status;
  int64_t cap, max_blocks;
  int64_t ev_begin, ev_end;   // evicted range [S, T0 - W)
  int32_t units, S, Bk, nb, tokens_per_cta;
};

// Launchers (kernels live in the .cu files); return cudaError_t of the launch.
// All decode-path launches use programmatic dependent launch; every kernel waits
// for its predecessor grid before it completes, so stream order still holds.
cudaError_t launch_select(const SelectParams& p, int D, int grid, cudaStream_t s);
// maps: K and V with 64-row boxes, then K and V with 16-row boxes
cudaError_t launch_attend(const CUtensorMap* maps, const AttendParams& p, int D, cudaStream_t s);
cudaError_t launch_append(const AppendParams& p, int D, cudaStream_t s);
cudaError_t launch_init(const InitParams& p, int D, cudaStream_t s);
size_t attend_smem_bytes(int D);
// per device, before the first launch: shared-memory size and carveout attributes
cudaError_t prepare_attend(int D);
cudaError_t prepare_select(int D);
cudaError_t prepare_state(int D);

}  // namespace hyb
