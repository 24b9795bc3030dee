// Strided block selection ("SPLA: Block Sparse Plus Linear Attention for Long
// Context Modeling", table of contents: "Strided block selection"; the page
// gives the heading only).  Reading used here: a fixed stride of always-exact
// blocks -- the last block of every `stride` consecutive candidate blocks
// (j % stride == stride - 1) -- plus the top-k by the usual Taylor score among
// the other blocks (larger score first, ties to the lower index).  The union,
// ascending, is handed to the decode as its selection, so the exact part and
// the subtraction of the selected blocks' linear terms are the decode's own.
//
// One CTA per unit: the group's q' sums, the score of every candidate block
// from its mean and variance rows (one warp per block, lanes over channels),
// the top-k by repeated block-wide maxima of packed (key << 32 | ~index)
// words, the union as a bitmap, compacted in block order by one warp.  This is
// a separate launch that reads the block statistics once more; it serves a
// selection rule the pages only name, not the decode step's hot path.

#include "hyb_device.cuh"
#include "k_select.h"

namespace hyb {
namespace {

constexpr int kSelThreads = 256, kSelWarps = kSelThreads / 32;

__device__ __forceinline__ unsigned long long shfl_xor_u64s(unsigned long long v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((unsigned long long)hi << 32) | lo;
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) strided_select_kernel(const __grid_constant__ StridedSelParams p) {
  extern __shared__ __align__(16) uint8_t sel_smem[];
  float* q1 = reinterpret_cast<float*>(sel_smem);      // sum_i q'_i
  float* q2 = q1 + D;                                    // 1/2 sum_i q'_i^2
  float* sc = q2 + D;                                    // [nb] block scores
  uint32_t* bm = reinterpret_cast<uint32_t*>(sc + ((p.nb + 3) & ~3));  // [ceil(nb / 32)] selected blocks
  __shared__ unsigned long long red[kSelWarps];
  __shared__ uint32_t nan_seen;
  const int unit = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nb = p.nb, words = (nb + 31) >> 5;
  if (tid == 0) {
    pdl_wait_primary();  // the statistics and q may come from the previous grid
    nan_seen = 0u;
  }
  __syncthreads();
  pdl_allow_dependents();
  for (int c = tid; c < D; c += kSelThreads) {
    float a = 0.f, b = 0.f;
    for (int i = 0; i < p.G; ++i) {
      const float v = __bfloat162float(p.q[((int64_t)unit * p.G + i) * D + c]) * p.scale;
      a += v;
      b += 0.5f * v * v;
    }
    q1[c] = a;
    q2[c] = b;
  }
  for (int w = tid; w < words; w += kSelThreads) bm[w] = 0u;
  __syncthreads();
  // scores: q'.mu_j + 1/2 q'^2 . var_j summed over the group's heads
  for (int j = warp; j < nb; j += kSelWarps) {
    const float* mu = p.mu + ((int64_t)unit * p.max_blocks + j) * D;
    const float* var = p.var + ((int64_t)unit * p.max_blocks + j) * D;
    float acc = 0.f;
#pragma unroll
    for (int c = lane; c < D; c += 32) acc += q1[c] * mu[c] + q2[c] * var[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      sc[j] = acc;
      if (acc != acc) nan_seen = 1u;
    }
  }
  // the strided blocks are always taken
  for (int j = p.stride - 1 + tid * p.stride; j < nb; j += kSelThreads * p.stride) atomicOr(&bm[j >> 5], 1u << (j & 31));
  __syncthreads();
  // top-k among the others: k rounds of the largest packed word below the last
  const int n_fixed = nb / p.stride;
  const int kk = min(p.k, nb - n_fixed);
  unsigned long long last = ~0ull;
#pragma unroll 1
  for (int it = 0; it < kk; ++it) {
    unsigned long long best = 0ull;
    for (int j = tid; j < nb; j += kSelThreads) {
      if (j % p.stride == p.stride - 1) continue;
      const unsigned long long v = ((unsigned long long)float_key(sc[j]) << 32) | (uint32_t)~(uint32_t)j;
      if (v < last && v > best) best = v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long y = shfl_xor_u64s(best, o);
      best = y > best ? y : best;
    }
    if (lane == 0) red[warp] = best;
    __syncthreads();
    best = red[0];
#pragma unroll
    for (int w = 1; w < kSelWarps; ++w) best = red[w] > best ? red[w] : best;
    last = best;
    if (tid == 0 && best != 0ull) {  // (a candidate always remains: kk <= the other blocks)
      const int j = (int)~(uint32_t)best;
      bm[j >> 5] |= 1u << (j & 31);
    }
    __syncthreads();  // red is rewritten next round; the bitmap is complete after the last
  }
  // the union in block order, -1 padded to the row width
  if (warp == 0) {
    int32_t* row = p.sel + (int64_t)unit * p.width;
    int32_t* copy = p.sel_copy != nullptr ? p.sel_copy + (int64_t)unit * p.width : nullptr;
    int base = 0;
#pragma unroll 1
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t bits = w < words ? bm[w] : 0u;
      const int cnt = __popc(bits);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = base + incl - cnt;
      uint32_t u = bits;
      while (u) {
        const int b = __ffs(u) - 1;
        u &= u - 1u;
        if (pos < p.width) {
          row[pos] = (w << 5) + b;
          if (copy) copy[pos] = (w << 5) + b;
        }
        ++pos;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    for (int e = base + lane; e < p.width; e += 32) {
      row[e] = -1;
      if (copy) copy[e] = -1;
    }
  }
  if (tid == 0 && nan_seen) atomicOr(p.status, HYB_STATUS_NAN_SCORE);
}

}  // namespace

size_t strided_select_smem(int D, int nb) {
  const size_t bytes = (size_t)(2 * D + ((nb + 3) & ~3)) * 4 + (size_t)((nb + 31) / 32) * 4;
  return bytes <= 200 * 1024 ? bytes : 0;
}

cudaError_t prepare_strided_select(int D) {
  const void* f = D == 128 ? (const void*)strided_select_kernel<128> : (const void*)strided_select_kernel<64>;
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
}

cudaError_t launch_strided_select(const StridedSelParams& p, int D, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.units);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = strided_select_smem(D, p.nb);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (D == 128) return cudaLaunchKernelEx(&cfg, strided_select_kernel<128>, p);
  return cudaLaunchKernelEx(&cfg, strided_select_kernel<64>, p);
}

}  // namespace hyb
