// Strided block selection ("SPLA: Block Sparse Plus Linear Attention for Long
// Context Modeling", table of contents: "Strided block selection"; the page
// gives the heading only).  Reading used here: a fixed stride of always-exact
// blocks -- the last block of every `stride` consecutive candidate blocks
// (j % stride == stride - 1) -- plus the top-k by the usual Taylor score among
// the other blocks (larger score first, ties to the lower index).  The union,
// ascending, is handed to the decode as its selection, so the exact part and
// the subtraction of the selected blocks' linear terms are the decode's own.
//
// One cluster of `parts` CTAs per unit (as many as fill the SMs once, at most
// 8), each scoring a contiguous share of the blocks.  A CTA's mean and
// variance rows are prefetched into L2 before the wait for the previous grid
// (L2 is the point of coherence, so a row that grid still writes is current
// there).  Scoring: every warp takes 8 rows per step with one 16-byte load of
// the mean and one of the variance per lane (16 loads in flight per lane; the
// first step's loads are issued before the group's q' sums are formed, so the
// two round trips overlap), and reduces the 8 rows' partial sums at once.
// The scores of the non-strided blocks are stored compacted into the shared
// memory of the cluster's first CTA (c = j - (j + 1) / stride, which keeps
// block order, so ties to the lower compacted index are ties to the lower
// block); two cluster barriers bracket these stores (every CTA has started;
// every score is in place).  A block that holds evictions not yet folded into
// the statistics (the previous step's, usually one token) is scored from its
// rows folded in registers one token at a time by Welford's update, the
// decode's own fold, which the decode that follows writes back.  The first
// CTA then selects.
// Top-k: up to 32, one warp's bound-and-rank selection (the decode kernel's);
// above 32, or when too many keys tie at the bound, k rounds of block-wide
// maxima of packed (key << 32 | ~index) words.  The union is a bitmap,
// compacted in block order by one warp.  This is a separate launch that reads
// the block statistics once more; it serves a selection rule the pages only
// name, not the decode step's hot path.

#include "k_common.cuh"
#include "k_select.h"

namespace hyb {
namespace {

constexpr int kSelThreads = 512, kSelWarps = kSelThreads / 32;
constexpr int kSelSteps = 8;      // rows per lane per step (loads in flight: 2 per row)
constexpr int kSelCap = 256;      // candidates at the bound the one-warp selection ranks
constexpr int kSelMinRows = 512;  // the one-warp selection reads 512 scores when it has fewer

// every thread of every CTA of the cluster arrives, then waits (release /
// acquire: shared-memory stores into other CTAs before it are visible after it)
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive;\n\tbarrier.cluster.wait;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ unsigned long long shfl_xor_u64s(unsigned long long v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((unsigned long long)hi << 32) | lo;
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) strided_select_kernel(const __grid_constant__ StridedSelParams p) {
  constexpr int LPR = D / 4;       // lanes per row (one float4 of channels each)
  constexpr int RPW = 32 / LPR;    // rows per warp per load
  static_assert(D % 4 == 0 && 32 % LPR == 0, "a row is a whole number of 16-byte lane slices within a warp");
  constexpr int kRowsPerIter = RPW * kSelSteps;
  extern __shared__ __align__(16) uint8_t sel_smem[];
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(sel_smem);  // [kSelCap]
  float* q1 = reinterpret_cast<float*>(cand + kSelCap);                       // sum_i q'_i
  float* q2 = q1 + D;                                                           // 1/2 sum_i q'_i^2
  float* csc = q2 + D;                                      // [max(nc, 512)] scores of the non-strided blocks
  const int nb = p.nb, stride = p.stride, words = (nb + 31) >> 5;
  const int n_fixed = nb / stride, nc = nb - n_fixed;
  const int ncp = ((nc > kSelMinRows ? nc : kSelMinRows) + 3) & ~3;
  uint32_t* bm = reinterpret_cast<uint32_t*>(csc + ncp);   // [words] selected blocks
  __shared__ unsigned long long red[kSelWarps];
  __shared__ int32_t selc[32];
  __shared__ uint32_t nan_seen, warp_ok;
  const int parts = p.parts, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int unit = blockIdx.x / parts;
  const int part = parts > 1 ? (int)cluster_rank() : 0;
  const int share = (nb + parts - 1) / parts;
  const int r0 = min(nb, part * share), r1 = min(nb, r0 + share);
  const int64_t row0 = (int64_t)unit * p.max_blocks;
  if (tid == 0) {
    const int64_t first = (row0 + r0) * D * 4, bytes = (int64_t)(r1 - r0) * D * 4;
    for (int64_t o = 0; o < bytes; o += 32768) {
      const uint32_t n = (uint32_t)(bytes - o < 32768 ? bytes - o : 32768);
      bulk_prefetch_l2(reinterpret_cast<const char*>(p.mu) + first + o, n);
      bulk_prefetch_l2(reinterpret_cast<const char*>(p.var) + first + o, n);
    }
    pdl_wait_primary();  // the statistics and q may come from the previous grid
    nan_seen = 0u;
  }
  __syncthreads();
  pdl_allow_dependents();
  // scores q'.mu_j + 1/2 q'^2 . var_j summed over the group's heads
  const int sub = lane / LPR, cl = lane % LPR;
  float4 m[kSelSteps], v[kSelSteps];
  auto load_rows = [&](int j0) {
#pragma unroll
    for (int s = 0; s < kSelSteps; ++s) {
      const int j = j0 + s * RPW + sub;
      if (j < r1) {
        const int64_t off = (row0 + j) * D + 4 * cl;
        m[s] = __ldg(reinterpret_cast<const float4*>(p.mu + off));
        v[s] = __ldg(reinterpret_cast<const float4*>(p.var + off));
      } else {
        m[s] = make_float4(0.f, 0.f, 0.f, 0.f);
        v[s] = m[s];
      }
    }
  };
  int j0 = r0 + warp * kRowsPerIter;
  load_rows(j0);
  for (int c = tid; c < D; c += kSelThreads) {
    float a = 0.f, b = 0.f;
    for (int i = 0; i < p.G; ++i) {
      const float x = __bfloat162float(p.q[((int64_t)unit * p.G + i) * D + c]) * p.scale;
      a += x;
      b += 0.5f * x * x;
    }
    q1[c] = a;
    q2[c] = b;
  }
  for (int w = tid; w < words; w += kSelThreads) bm[w] = 0u;
  if (parts > 1) cluster_sync_all();  // every CTA of the cluster has started before its shared memory is written
  else __syncthreads();
  const float4 a1 = *reinterpret_cast<const float4*>(q1 + 4 * cl);
  const float4 a2 = *reinterpret_cast<const float4*>(q2 + 4 * cl);
  const uint32_t csc_first = parts > 1 ? map_rank(smem_u32(csc), 0u) : 0u;  // csc in the first CTA
  // blocks [jb0, jb1] hold evictions not yet folded (none: jb0 > jb1)
  const bool folds = p.fold_end > p.fold_begin;
  const int jb0 = folds ? (p.fold_begin - p.S) / p.Bk : 1, jb1 = folds ? (p.fold_end - 1 - p.S) / p.Bk : 0;
  bool nan = false;
  auto put = [&](int j, float sc) {  // one score: the NaN flag, and the compacted slot of a non-strided block
    nan |= sc != sc;
    if (j % stride != stride - 1) {
      const int c = j - (j + 1) / stride;
      if (part == 0) csc[c] = sc;
      else st_cluster_f32(csc_first + 4u * (uint32_t)c, sc);
    }
  };
#pragma unroll 1
  while (true) {
    float acc[kSelSteps];
#pragma unroll
    for (int s = 0; s < kSelSteps; ++s)
      acc[s] = a1.x * m[s].x + a1.y * m[s].y + a1.z * m[s].z + a1.w * m[s].w + a2.x * v[s].x + a2.y * v[s].y +
               a2.z * v[s].z + a2.w * v[s].w;
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1)
#pragma unroll
      for (int s = 0; s < kSelSteps; ++s) acc[s] += __shfl_xor_sync(0xffffffffu, acc[s], o);
    if (cl == 0) {
#pragma unroll
      for (int s = 0; s < kSelSteps; ++s) {
        const int j = j0 + s * RPW + sub;
        if (j < r1 && (j < jb0 || j > jb1)) put(j, acc[s]);
      }
    }
    j0 += kSelWarps * kRowsPerIter;
    if (j0 >= r1) break;
    load_rows(j0);
  }
  // the blocks with pending evictions in this CTA's share, one warp each
  // (lanes [0, LPR): four channels each)
#pragma unroll 1
  for (int j = max(jb0, r0) + warp; j <= min(jb1, r1 - 1); j += kSelWarps) {
    float sc = 0.f;
    if (sub == 0) {
      const int64_t bs = p.S + (int64_t)j * p.Bk;
      const int64_t t0 = bs > p.fold_begin ? bs : (int64_t)p.fold_begin;
      const int64_t t1 = bs + p.Bk < p.fold_end ? bs + p.Bk : (int64_t)p.fold_end;
      float mm[4] = {0.f, 0.f, 0.f, 0.f}, vv[4] = {0.f, 0.f, 0.f, 0.f};
      if (t0 > bs) {  // the tokens [bs, t0) are in the stored rows
        const int64_t off = (row0 + j) * D + 4 * cl;
        const float4 a = __ldg(reinterpret_cast<const float4*>(p.mu + off));
        const float4 b = __ldg(reinterpret_cast<const float4*>(p.var + off));
        mm[0] = a.x; mm[1] = a.y; mm[2] = a.z; mm[3] = a.w;
        vv[0] = b.x; vv[1] = b.y; vv[2] = b.z; vv[3] = b.w;
      }
#pragma unroll 1
      for (int64_t t = t0; t < t1; ++t) {
        const uint2 w = *reinterpret_cast<const uint2*>(p.k_cache + ((int64_t)unit * p.cap + t) * D + 4 * cl);
        const float x[4] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y)};
        const float cnt = (float)(t - bs + 1);
        const float inv = 1.f / cnt;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (t == bs) {  // the block's first token
            mm[c] = x[c];
            vv[c] = 0.f;
          } else {
            const float delta = x[c] - mm[c];
            const float m1 = mm[c] + delta * inv;
            vv[c] = (vv[c] * (cnt - 1.f) + delta * (x[c] - m1)) * inv;
            mm[c] = m1;
          }
        }
      }
      sc = a1.x * mm[0] + a1.y * mm[1] + a1.z * mm[2] + a1.w * mm[3] + a2.x * vv[0] + a2.y * vv[1] + a2.z * vv[2] +
           a2.w * vv[3];
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
    if (lane == 0) put(j, sc);
  }
  if (nan) nan_seen = 1u;
  if (parts > 1) cluster_sync_all();  // every score is in the first CTA
  else __syncthreads();
  if (tid == 0 && nan_seen) atomicOr(p.status, HYB_STATUS_NAN_SCORE);
  if (part != 0) return;
  // the strided blocks are always taken
  for (int64_t j = stride - 1 + (int64_t)tid * stride; j < nb; j += (int64_t)kSelThreads * stride)
    atomicOr(&bm[j >> 5], 1u << (j & 31));
  __syncthreads();
  // top-k among the others (compacted index c is block c + c / (stride - 1))
  const int kk = min(p.k, nc);
  if (kk == nc) {  // every other block
    for (int c = tid; c < nc; c += kSelThreads) {
      const int j = c + c / (stride - 1);
      atomicOr(&bm[j >> 5], 1u << (j & 31));
    }
  } else if (kk > 0) {
    bool ok = false;
    if (kk <= 32) {
      if (warp == 0) {
        bool wn;
        const bool r = topk_warp(csc, nc, kk, selc, nullptr, cand, kSelCap, wn);
        __syncwarp();
        if (r && lane < kk) {
          const int c = selc[lane];
          const int j = c + c / (stride - 1);
          atomicOr(&bm[j >> 5], 1u << (j & 31));
        }
        if (lane == 0) warp_ok = r ? 1u : 0u;
      }
      __syncthreads();
      ok = warp_ok != 0u;
    }
    if (!ok) {  // k rounds of the largest packed word below the last
      unsigned long long last = ~0ull;
#pragma unroll 1
      for (int it = 0; it < kk; ++it) {
        unsigned long long best = 0ull;
        for (int c = tid; c < nc; c += kSelThreads) {
          const unsigned long long w = ((unsigned long long)float_key(csc[c]) << 32) | (uint32_t)~(uint32_t)c;
          if (w < last && w > best) best = w;
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
        if (tid == 0 && best != 0ull) {  // (a candidate always remains: kk < nc)
          const int c = (int)~(uint32_t)best;
          const int j = c + c / (stride - 1);
          bm[j >> 5] |= 1u << (j & 31);
        }
        __syncthreads();  // red is rewritten next round; the bitmap is complete after the last
      }
    }
  }
  __syncthreads();
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
}

}  // namespace

int strided_select_parts(int nb, int units, int n_sm) {
  int parts = n_sm / (units > 0 ? units : 1);
  parts = parts < kSelMaxParts ? parts : kSelMaxParts;
  const int by_rows = (nb + 63) / 64;  // at least 64 blocks a CTA
  parts = parts < by_rows ? parts : by_rows;
  return parts > 1 ? parts : 1;
}

size_t strided_select_smem(int D, int nb) {
  const size_t rows = (size_t)((nb > kSelMinRows ? nb : kSelMinRows) + 3) & ~(size_t)3;
  const size_t bytes = (size_t)kSelCap * 8 + (2 * (size_t)D + rows) * 4 + (size_t)((nb + 31) / 32) * 4;
  return bytes <= 200 * 1024 ? bytes : 0;
}

cudaError_t prepare_strided_select(int D) {
  const void* f = D == 128 ? (const void*)strided_select_kernel<128> : (const void*)strided_select_kernel<64>;
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
}

cudaError_t launch_strided_select(const StridedSelParams& p, int D, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  if (p.parts < 1 || p.parts > kSelMaxParts) return cudaErrorInvalidValue;
  cfg.gridDim = dim3((unsigned)p.units * (unsigned)p.parts);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = strided_select_smem(D, p.nb);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)p.parts;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.parts > 1 ? 2 : 1;
  if (D == 128) return cudaLaunchKernelEx(&cfg, strided_select_kernel<128>, p);
  return cudaLaunchKernelEx(&cfg, strided_select_kernel<64>, p);
}

}  // namespace hyb
