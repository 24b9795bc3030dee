// Strided block selection (a separate kernel ahead of the decode).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace hyb {

struct StridedSelParams {
  const __nv_bfloat16* q;   // [units][G][D]
  const float* mu;          // [units][max_blocks][D] block means
  const float* var;         // [units][max_blocks][D] block population variances
  const __nv_bfloat16* k_cache;  // [units][cap][D]: the keys of the pending evictions
  int32_t* sel;             // [units][width]: the selection, ascending, -1 padded
  int32_t* sel_copy;        // optional second copy of sel (the caller's), or null
  uint32_t* status;         // status word: HYB_STATUS_NAN_SCORE
  int64_t max_blocks, cap;
  // evicted positions [fold_begin, fold_end) not yet in the statistics (the
  // same for every unit): their blocks are scored from rows folded here, in
  // registers; the decode that follows folds them into the state
  int32_t S, Bk, fold_begin, fold_end;
  int32_t units, nb, G, k, stride, width;
  int32_t parts;            // CTAs (one cluster) per unit, 1..kSelMaxParts
  float scale;
};

constexpr int kSelMaxParts = 8;  // a portable cluster size

// CTAs per unit: as many as fill the device's n_sm SMs once, at most 8, each
// with at least 64 blocks.
int strided_select_parts(int nb, int units, int n_sm);
// Dynamic shared memory the kernel needs for nb candidate blocks (0: too many).
size_t strided_select_smem(int D, int nb);
cudaError_t prepare_strided_select(int D);
cudaError_t launch_strided_select(const StridedSelParams& p, int D, cudaStream_t s);

}  // namespace hyb
