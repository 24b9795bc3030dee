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
constexpr int kAttendCtasPerSm = 2;
constexpr int kMaxAttendCtas = 1024;  // upper bound of the attention grid (sizes the workspace)
constexpr int kScoreBlocksPerCta = 64;
constexpr int kSelectThreads = 256;
constexpr int kSelCache = 64;         // selection entries a warp group caches in shared memory
constexpr int kMaxGroup = 4;          // query heads per KV head supported by the attention kernel
constexpr uint64_t kWaitLimit = 1000000000ull;  // ns: a kernel-internal wait gives up after ~1 s

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
  const __nv_bfloat16* q;     // [B][Hq][D]
  const float* mu;            // [units][max_blocks][D]
  const float* var;
  const float* H;             // [units][D][D]
  const float* zk;            // [units][D]
  const float* zv;
  const float* n;             // [units]
  float* scores;              // [units][max_blocks]
  int32_t* sel;               // [units][top_k]
  int32_t* sel_out;           // optional copy
  float* lin;                 // [units][G][D + 1]: N_glob[D], D_glob
  uint32_t* tickets;          // [units]
  uint32_t* status;
  int64_t max_blocks;
  int32_t units, G, nb, top_k, k_eff;
  int32_t score_ctas, lin_ctas;
  int32_t do_select;
  float scale;
};

struct AttendParams {
  const __nv_bfloat16* q;     // [B][Hq][D]
  const int32_t* sel;         // [units][top_k]
  const float* lin;           // [units][G][D + 1]
  float* partials;            // [slots][partial_floats(D)]
  uint32_t* tickets;          // [units]
  uint32_t* status;
  float* out;                 // [B][Hq][D]
  int64_t cap;                // cache rows per unit
  int32_t T, S, Bk, top_k, nb, k_eff;
  int32_t sink_len, win_start, ev_end;
  int32_t n_sink_chunks, n_win_chunks, chunks_per_block, chunks_per_unit;
  int32_t units, G, grid;
  int32_t splits;             // CTAs per unit; CTA x works on unit x / splits
  int32_t merge_only;         // no exact tokens at all: each CTA merges one unit
  float scale;
};

struct AppendParams {
  const __nv_bfloat16* k_new; // [units][D]
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  float* H; float* zk; float* zv; float* n; float* mu; float* var;
  int64_t cap, T, p;          // T before the append; p = evicted position (valid if evict)
  int64_t max_blocks;
  int32_t units, evict, blk, cnt;  // block of p and its token count after the fold
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
cudaError_t launch_select(const SelectParams& p, int D, int grid_x, cudaStream_t s);
// maps: K and V with 64-row boxes, then K and V with 16-row boxes
cudaError_t launch_attend(const CUtensorMap* maps, const AttendParams& p, int D, bool pdl, cudaStream_t s);
cudaError_t launch_append(const AppendParams& p, int D, cudaStream_t s);
cudaError_t launch_init(const InitParams& p, int D, cudaStream_t s);
size_t attend_smem_bytes(int D);
// per device, before the first launch: shared-memory size and carveout attributes
cudaError_t prepare_attend(int D);
cudaError_t prepare_select(int D);
cudaError_t prepare_state(int D);

}  // namespace hyb
