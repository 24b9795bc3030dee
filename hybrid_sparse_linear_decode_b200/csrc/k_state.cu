// State kernels: the cache write of an append, the dense fold of a run of
// evicted tokens, and the build of the state of a prefilled history.  Between
// decodes the state lags the history by the tokens evicted since the last
// decode; the next decode folds those in (the fused decode kernel itself for up
// to three tokens, fold_kernel first for more).
//
// The state of a unit (batch row, KV head) covers the evicted tokens
// L = [S, T - W) -- past the sinks and out of the sliding window ("SALSA:
// Training-Consistent Sparse Caching with Sink Preservation for Linearized
// LLMs", abstract: window + sparse cache + linear-attention hidden state):
//   H = sum_L k v^T, zk = sum_L k, zv = sum_L v, n = |L|   (the recurrent state
//   of residual linear attention, "SPLA: Block Sparse Plus Linear Attention for
//   Long Context Modeling", sections "Residual Linear Attention" / "Recurrence"),
//   mu_j, var_j = mean and population variance of the keys of block
//   j = [S + j*Bk, min(S + (j+1)*Bk, T - W))   (the block statistics the
//   selection metric expands around, SPLA abstract).
#include "hyb_device.cuh"
#include "hyb_internal.h"

namespace hyb {

namespace {

// ---------------------------------------------------------------- append
// Writes n tokens per unit at rows [T, T + n) of the caches: grid (units, n),
// D/4 threads of 16 bytes.  A token's later eviction from the window is folded
// into the state by the decode after it, which reads the caches.
template <int D>
__global__ void __launch_bounds__(D / 4) append_kernel(const __grid_constant__ AppendParams p) {
  const int unit = blockIdx.x, j = blockIdx.y, tid = threadIdx.x;  // token j of the chunk
  const int32_t Tb = p.T - (p.tb.ragged ? p.tb.row_lag[unit / p.Hkv] : 0);  // this row's length
  if (tid == 0) pdl_wait_primary();  // the previous decode may still read these caches' rows
  __syncthreads();
  pdl_allow_dependents();
  const bool is_v = tid >= D / 8;
  const int e = (tid % (D / 8)) * 8;
  const __nv_bfloat16* src = (is_v ? p.v_new : p.k_new) + ((int64_t)unit * p.n + j) * D + e;
  __nv_bfloat16* dst = (is_v ? p.v_cache : p.k_cache) + ((int64_t)unit * p.cap + Tb + j) * D + e;
  *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
}

// ---------------------------------------------------------------- chunk fold
// The pending evicted positions [fb, fe) of every unit (each row's length and
// each head's window give its own range) folded into the state in one
// pass, for several pending tokens (a chunked append, or many appends between
// decodes; SPLA "Recurrence" applied to a run of tokens is a small dense
// update).  One CTA per unit: H += K^T V over the run (fp32 thread tiles of the
// D x D outer-product sum, keys / values staged through shared memory 32
// tokens at a time), zk += sum k, zv += sum v, n += count; then, per block the
// run touches, the block's mean and population variance merged with those of
// its new tokens by the pairwise combination of Chan, Golub and LeVeque
// (n = na + nb, mean = ma + d nb / n, M2 = M2a + M2b + d^2 na nb / n, with
// d = mb - ma), in fp64.  The tokens of a block folded before fb are exactly
// those before fb, as folds go in position order.
template <int D>
__global__ void __launch_bounds__(256) fold_kernel(const __grid_constant__ FoldParams p) {
  constexpr int RT = D / 16;
  __shared__ __align__(16) float ks[32][D];
  __shared__ __align__(16) float vs[32][D];
  const int unit = blockIdx.x, tid = threadIdx.x;
  const UnitGeo g = unit_geo(&p.tb, unit, p.Hkv, p.T, p.S, p.W, p.Bk, 0, 1, p.pending);
  const int64_t fb = g.fold_begin, fe = g.fold_end;
  if (tid == 0) pdl_wait_primary();  // the caches' rows and the state may come from the previous grid
  __syncthreads();
  pdl_allow_dependents();
  if (fe <= fb) return;  // nothing pending in this unit (a short row)
  const int tr = tid / 16, tc = tid % 16;
  const int64_t ub = (int64_t)unit * p.cap;
  float acc[RT][RT];
#pragma unroll
  for (int i = 0; i < RT; ++i)
#pragma unroll
    for (int j = 0; j < RT; ++j) acc[i][j] = 0.f;
  float zacc = 0.f;
  for (int64_t tt = fb; tt < fe; tt += 32) {
    const int n = (int)min((int64_t)32, fe - tt);
    for (int e = tid; e < 32 * D; e += 256) {
      const int r = e / D, c = e % D;
      float kv = 0.f, vv = 0.f;
      if (r < n) {
        kv = __bfloat162float(p.k_cache[(ub + tt + r) * D + c]);
        vv = __bfloat162float(p.v_cache[(ub + tt + r) * D + c]);
      }
      ks[r][c] = kv;
      vs[r][c] = vv;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < 32; ++r) {
      float a[RT], b[RT];
#pragma unroll
      for (int i = 0; i < RT; ++i) {
        a[i] = ks[r][tr * RT + i];
        b[i] = vs[r][tc * RT + i];
      }
#pragma unroll
      for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int j = 0; j < RT; ++j) acc[i][j] += a[i] * b[j];
    }
    if (tid < D) {
      for (int r = 0; r < n; ++r) zacc += ks[r][tid];
    } else if (tid < 2 * D) {
      for (int r = 0; r < n; ++r) zacc += vs[r][tid - D];
    }
    __syncthreads();
  }
  float* H = p.H + (int64_t)unit * D * D;
#pragma unroll
  for (int i = 0; i < RT; ++i)
#pragma unroll
    for (int j = 0; j < RT; ++j) H[(int64_t)(tr * RT + i) * D + tc * RT + j] += acc[i][j];
  if (tid < D) p.zk[(int64_t)unit * D + tid] += zacc;
  else if (tid < 2 * D) p.zv[(int64_t)unit * D + tid - D] += zacc;
  if (tid == 0) p.n[unit] += (float)(fe - fb);
  if (tid < D) {  // one channel per thread
    const __nv_bfloat16* kc = p.k_cache + ub * D + tid;
    const int64_t j0 = (fb - p.S) / p.Bk, j1 = (fe - 1 - p.S) / p.Bk;
    for (int64_t j = j0; j <= j1; ++j) {
      const int64_t bs = p.S + j * p.Bk;
      const int64_t a0 = max(bs, fb), a1 = min(bs + (int64_t)p.Bk, fe);
      const double na = (double)(a0 - bs), nb = (double)(a1 - a0);
      double sb = 0.0, qb = 0.0;
      for (int64_t t = a0; t < a1; ++t) sb += (double)__bfloat162float(kc[t * D]);
      const double mb = sb / nb;
      for (int64_t t = a0; t < a1; ++t) {
        const double d = (double)__bfloat162float(kc[t * D]) - mb;
        qb += d * d;
      }
      const int64_t so = ((int64_t)unit * p.max_blocks + j) * D + tid;
      double mu = mb, m2 = qb, nn = nb;
      if (na > 0.0) {
        const double ma = (double)p.mu[so], m2a = (double)p.var[so] * na, d = mb - ma;
        nn = na + nb;
        mu = ma + d * nb / nn;
        m2 = m2a + qb + d * d * na * nb / nn;
      }
      p.mu[so] = (float)mu;
      p.var[so] = (float)(m2 / nn);
    }
  }
}

// ---------------------------------------------------------------- init
// Every unit's evicted range is L = [S, ev_end(T_b, W_h)): its row's length
// and its head's window.
// (1) H, zk, zv over L: grid (ceil(max |L| / tokens_per_cta), units).  Each CTA
//     accumulates its token range in fp32 (thread tile RT x RT of the D x D
//     outer-product sum, keys/values staged through shared memory 32 tokens at a
//     time) and adds the result into fp64 accumulators.
template <int D>
__global__ void __launch_bounds__(256) init_linear_kernel(const __grid_constant__ InitParams p) {
  constexpr int RT = D / 16;
  __shared__ __align__(16) float ks[32][D];
  __shared__ __align__(16) float vs[32][D];
  const int unit = blockIdx.y, tid = threadIdx.x;
  const int tr = tid / 16, tc = tid % 16;
  const UnitGeo g = unit_geo(&p.tb, unit, p.Hkv, p.T, p.S, p.W, p.Bk, 0, 1, 0);
  const int64_t t0 = p.S + (int64_t)blockIdx.x * p.tokens_per_cta;
  const int64_t t1 = min(t0 + (int64_t)p.tokens_per_cta, (int64_t)g.ev_end);
  if (t0 >= t1) return;  // past this unit's evicted range
  const int64_t ub = (int64_t)unit * p.cap;
  float acc[RT][RT];
#pragma unroll
  for (int i = 0; i < RT; ++i)
#pragma unroll
    for (int j = 0; j < RT; ++j) acc[i][j] = 0.f;
  float zacc = 0.f;
  for (int64_t tt = t0; tt < t1; tt += 32) {
    const int n = (int)min((int64_t)32, t1 - tt);
    for (int e = tid; e < 32 * D; e += 256) {
      const int r = e / D, c = e % D;
      float kv = 0.f, vv = 0.f;
      if (r < n) {
        kv = __bfloat162float(p.k_cache[(ub + tt + r) * D + c]);
        vv = __bfloat162float(p.v_cache[(ub + tt + r) * D + c]);
      }
      ks[r][c] = kv;
      vs[r][c] = vv;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < 32; ++r) {
      float a[RT], b[RT];
#pragma unroll
      for (int i = 0; i < RT; ++i) {
        a[i] = ks[r][tr * RT + i];
        b[i] = vs[r][tc * RT + i];
      }
#pragma unroll
      for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int j = 0; j < RT; ++j) acc[i][j] += a[i] * b[j];
    }
    if (tid < D) {
      for (int r = 0; r < n; ++r) zacc += ks[r][tid];
    } else if (tid < 2 * D) {
      for (int r = 0; r < n; ++r) zacc += vs[r][tid - D];
    }
    __syncthreads();
  }
  double* H64 = p.H64 + (int64_t)unit * D * D;
#pragma unroll
  for (int i = 0; i < RT; ++i)
#pragma unroll
    for (int j = 0; j < RT; ++j) atomicAdd(H64 + (int64_t)(tr * RT + i) * D + tc * RT + j, (double)acc[i][j]);
  if (tid < 2 * D) atomicAdd(p.z64 + (int64_t)unit * 2 * D + tid, (double)zacc);
}

// (2) block statistics: one warp per block, two passes (mean, then the mean
//     squared deviation) in fp64.
template <int D>
__global__ void __launch_bounds__(256) init_stats_kernel(const __grid_constant__ InitParams p) {
  constexpr int CPL = D / 32;
  const int unit = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * 8 + warp;
  const UnitGeo g = unit_geo(&p.tb, unit, p.Hkv, p.T, p.S, p.W, p.Bk, 0, 1, 0);
  if (j >= g.nb) return;
  const int64_t bs = p.S + (int64_t)j * p.Bk;
  const int64_t be = min(bs + (int64_t)p.Bk, (int64_t)g.ev_end);
  const double cnt = (double)(be - bs);
  const __nv_bfloat16* kc = p.k_cache + (int64_t)unit * p.cap * D;
  double s[CPL], q[CPL];
#pragma unroll
  for (int i = 0; i < CPL; ++i) s[i] = q[i] = 0.0;
  for (int64_t t = bs; t < be; ++t)
#pragma unroll
    for (int i = 0; i < CPL; ++i) s[i] += (double)__bfloat162float(kc[t * D + lane + 32 * i]);
#pragma unroll
  for (int i = 0; i < CPL; ++i) s[i] /= cnt;
  for (int64_t t = bs; t < be; ++t)
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const double d = (double)__bfloat162float(kc[t * D + lane + 32 * i]) - s[i];
      q[i] += d * d;
    }
  const int64_t so = ((int64_t)unit * p.max_blocks + j) * D;
#pragma unroll
  for (int i = 0; i < CPL; ++i) {
    p.mu[so + lane + 32 * i] = (float)s[i];
    p.var[so + lane + 32 * i] = (float)(q[i] / cnt);
  }
}

// (3) fp64 accumulators -> fp32 state; reset the status word.
template <int D>
__global__ void __launch_bounds__(256) init_finalize_kernel(const __grid_constant__ InitParams p) {
  const int unit = blockIdx.x, tid = threadIdx.x;
  const UnitGeo g = unit_geo(&p.tb, unit, p.Hkv, p.T, p.S, p.W, p.Bk, 0, 1, 0);
  const double* H64 = p.H64 + (int64_t)unit * D * D;
  float* H = p.H + (int64_t)unit * D * D;
  for (int e = tid; e < D * D; e += 256) H[e] = (float)H64[e];
  if (tid < D) {
    p.zk[(int64_t)unit * D + tid] = (float)p.z64[(int64_t)unit * 2 * D + tid];
    p.zv[(int64_t)unit * D + tid] = (float)p.z64[(int64_t)unit * 2 * D + D + tid];
  }
  if (tid == 0) {
    p.n[unit] = (float)(g.ev_end - p.S);
    if (unit == 0) *p.status = 0u;
  }
}

}  // namespace

cudaError_t prepare_state(int D) {
  const void* fs[] = {D == 128 ? (const void*)append_kernel<128> : (const void*)append_kernel<64>,
                      D == 128 ? (const void*)fold_kernel<128> : (const void*)fold_kernel<64>,
                      D == 128 ? (const void*)init_linear_kernel<128> : (const void*)init_linear_kernel<64>,
                      D == 128 ? (const void*)init_stats_kernel<128> : (const void*)init_stats_kernel<64>,
                      D == 128 ? (const void*)init_finalize_kernel<128> : (const void*)init_finalize_kernel<64>};
  for (const void* f : fs) {
    const cudaError_t e =
        cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_fold(const FoldParams& p, int D, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.units);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (D == 128) return cudaLaunchKernelEx(&cfg, fold_kernel<128>, p);
  return cudaLaunchKernelEx(&cfg, fold_kernel<64>, p);
}

cudaError_t launch_append(const AppendParams& p, int D, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.units, p.n);
  cfg.blockDim = dim3(D / 4);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (D == 128) return cudaLaunchKernelEx(&cfg, append_kernel<128>, p);
  return cudaLaunchKernelEx(&cfg, append_kernel<64>, p);
}

cudaError_t launch_init(const InitParams& p, int D, cudaStream_t s) {
  const int64_t ev = p.ev_max;
  if (ev > 0) {
    const dim3 g1((unsigned)((ev + p.tokens_per_cta - 1) / p.tokens_per_cta), p.units);
    if (D == 128)
      init_linear_kernel<128><<<g1, 256, 0, s>>>(p);
    else
      init_linear_kernel<64><<<g1, 256, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.nb_max > 0) {
    const dim3 g2((unsigned)((p.nb_max + 7) / 8), p.units);
    if (D == 128)
      init_stats_kernel<128><<<g2, 256, 0, s>>>(p);
    else
      init_stats_kernel<64><<<g2, 256, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (D == 128)
    init_finalize_kernel<128><<<p.units, 256, 0, s>>>(p);
  else
    init_finalize_kernel<64><<<p.units, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace hyb
