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
// Writes n tokens per unit at rows [T, T + n) of the caches: grid (units,
// n / kAppendTokens<D>), 256 threads, one 16-byte piece of a key or value row
// each.  A token's later eviction from the window is folded into the state by
// the decode after it, which reads the caches.
template <int D>
constexpr int kAppendTokens = 256 / (D / 4);  // tokens per CTA (D / 4 pieces per token)
template <int D>
__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendParams p) {
  const int unit = blockIdx.x, tid = threadIdx.x;
  const int j = blockIdx.y * kAppendTokens<D> + tid / (D / 4);  // token j of the chunk
  const int32_t Tb = p.T - (p.tb.ragged ? p.tb.row_lag[unit / p.Hkv] : 0);  // this row's length
  if (tid == 0) pdl_wait_primary();  // the previous decode may still read these caches' rows
  __syncthreads();
  pdl_allow_dependents();
  if (j >= p.n) return;
  const int piece = tid % (D / 4);
  const bool is_v = piece >= D / 8;
  const int e = (piece % (D / 8)) * 8;
  const __nv_bfloat16* src = (is_v ? p.v_new : p.k_new) + ((int64_t)unit * p.n + j) * D + e;
  __nv_bfloat16* dst = (is_v ? p.v_cache : p.k_cache) + ((int64_t)unit * p.cap + Tb + j) * D + e;
  *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
}

// ---------------------------------------------------------------- chunk fold
// The pending evicted positions [fb, fe) of every unit (each row's length and
// each head's window give its own range) folded into the state in one
// pass, for several pending tokens (a chunked append, or many appends between
// decodes; SPLA "Recurrence" applied to a run of tokens is a small dense
// update).  Two CTAs per unit, CTA h taking key channels [h D/2, (h+1) D/2):
// its rows of H += K^T V (fp32 thread tiles of the outer-product sum, the tile
// held in registers from before the first token; keys and values staged
// through shared memory 32 tokens at a time, the next 32 fetched while these
// are multiplied), its channels of zk += sum k and zv += sum v, and its
// channels of the statistics of every block the run touches: the new tokens'
// mean and squared deviations as fp32 sums shifted by a value near the mean
// (the stored mean, else the block's first new key, so that the squares do not
// cancel), merged with the stored mean and population variance in fp64 by the
// pairwise combination of Chan, Golub and LeVeque (n = na + nb, mean = ma +
// d nb / n, M2 = M2a + M2b + d^2 na nb / n, with d = mb - ma).  The tokens of a block folded before fb are exactly those
// before fb, as folds go in position order.
template <int D>
__global__ void __launch_bounds__(256) fold_kernel(const __grid_constant__ FoldParams p) {
  constexpr int DH = D / 2;                           // this CTA's key channels (rows of H)
  constexpr int RR = DH / 16, RC = D / 16;            // thread tile of H: RR rows x RC columns
  constexpr int KP = DH / 8, VP = D / 8, TP = KP + VP;  // 16-byte pieces per token
  constexpr int NP = (32 * TP + 255) / 256;           // pieces per thread per 32 tokens
  __shared__ __align__(16) float ks[32][DH];
  __shared__ __align__(16) float vs[32][D];
  const int unit = blockIdx.x, half = blockIdx.y, tid = threadIdx.x;
  const UnitGeo g = unit_geo(&p.tb, unit, p.Hkv, p.T, p.S, p.W, p.Bk, 0, 1, p.pending);
  const int64_t fb = g.fold_begin, fe = g.fold_end;
  if (tid == 0) pdl_wait_primary();  // the caches' rows and the state may come from the previous grid
  __syncthreads();
  pdl_allow_dependents();
  if (fe <= fb) return;  // nothing pending in this unit (a short row)
  const int tr = tid / 16, tc = tid % 16;
  const int c0 = half * DH;
  const int64_t ub = (int64_t)unit * p.cap;
  float* Hrow = p.H + ((int64_t)unit * D + c0 + tr * RR) * D + tc * RC;
  float acc[RR][RC];
#pragma unroll
  for (int i = 0; i < RR; ++i)
#pragma unroll
    for (int j = 0; j < RC; j += 4) {
      const float4 x = *reinterpret_cast<const float4*>(Hrow + (int64_t)i * D + j);
      acc[i][j] = x.x;
      acc[i][j + 1] = x.y;
      acc[i][j + 2] = x.z;
      acc[i][j + 3] = x.w;
    }
  // statistics (threads [0, DH): key channel c0 + tid): the first block may
  // hold tokens folded before fb
  const int64_t j_first = (fb - p.S) / p.Bk, na_first = fb - (p.S + j_first * p.Bk);
  const int c = c0 + tid;
  double ma = 0.0, va = 0.0;
  if (tid < DH && na_first > 0) {
    const int64_t so = ((int64_t)unit * p.max_blocks + j_first) * D + c;
    ma = (double)p.mu[so];
    va = (double)p.var[so];
  }
  int64_t cur_j = -1, na = 0, next_bs = 0;  // the current block and the start of the next
  float shift = 0.f, s1 = 0.f, s2 = 0.f;
  int cnt = 0;
  auto flush = [&]() {
    if (cnt == 0) return;
    const int64_t so = ((int64_t)unit * p.max_blocks + cur_j) * D + c;
    const double nb = (double)cnt, mb = (double)shift + (double)s1 / nb,
                 m2b = fmax(0.0, (double)s2 - (double)s1 * (double)s1 / nb);
    double mu = mb, m2 = m2b, nn = nb;
    if (na > 0) {
      const double nad = (double)na, d = mb - ma;
      nn = nad + nb;
      mu = ma + d * nb / nn;
      m2 = va * nad + m2b + d * d * nad * nb / nn;
    }
    p.mu[so] = (float)mu;
    p.var[so] = (float)(m2 / nn);
  };
  float zacc = 0.f;
  uint4 pre[NP];
  auto fetch = [&](int64_t tt) {
    const int n = (int)min((int64_t)32, fe - tt);
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const int e = tid + q * 256, r = e / TP, x = e % TP;
      pre[q] = make_uint4(0u, 0u, 0u, 0u);
      if (e < 32 * TP && r < n) {
        const __nv_bfloat16* src = x < KP ? p.k_cache + (ub + tt + r) * D + c0 + x * 8
                                          : p.v_cache + (ub + tt + r) * D + (x - KP) * 8;
        pre[q] = __ldg(reinterpret_cast<const uint4*>(src));
      }
    }
  };
  fetch(fb);
  for (int64_t tt = fb; tt < fe; tt += 32) {
    const int n = (int)min((int64_t)32, fe - tt);
#pragma unroll
    for (int q = 0; q < NP; ++q) {  // rows past n are zero
      const int e = tid + q * 256, r = e / TP, x = e % TP;
      if (e < 32 * TP) {
        float* dst = x < KP ? &ks[r][x * 8] : &vs[r][(x - KP) * 8];
        const uint32_t w[4] = {pre[q].x, pre[q].y, pre[q].z, pre[q].w};
        *reinterpret_cast<float4*>(dst) = make_float4(bf16_lo(w[0]), bf16_hi(w[0]), bf16_lo(w[1]), bf16_hi(w[1]));
        *reinterpret_cast<float4*>(dst + 4) = make_float4(bf16_lo(w[2]), bf16_hi(w[2]), bf16_lo(w[3]), bf16_hi(w[3]));
      }
    }
    __syncthreads();
    if (tt + 32 < fe) fetch(tt + 32);
    const int n4 = (n + 3) & ~3;
#pragma unroll 4
    for (int r = 0; r < n4; ++r) {
      float a[RR], b[RC];
      if constexpr (RR == 4) {
        const float4 x = *reinterpret_cast<const float4*>(&ks[r][tr * RR]);
        a[0] = x.x;
        a[1] = x.y;
        a[2] = x.z;
        a[3] = x.w;
      } else {
#pragma unroll
        for (int i = 0; i < RR; ++i) a[i] = ks[r][tr * RR + i];
      }
#pragma unroll
      for (int j = 0; j < RC; j += 4) {
        const float4 y = *reinterpret_cast<const float4*>(&vs[r][tc * RC + j]);
        b[j] = y.x;
        b[j + 1] = y.y;
        b[j + 2] = y.z;
        b[j + 3] = y.w;
      }
#pragma unroll
      for (int i = 0; i < RR; ++i)
#pragma unroll
        for (int j = 0; j < RC; ++j) acc[i][j] += a[i] * b[j];
    }
    if (tid < DH) {
      for (int r = 0; r < n; ++r) {
        const float kf = ks[r][tid];
        zacc += kf;
        const int64_t t = tt + r;
        if (cur_j < 0 || t >= next_bs) {  // a new block: close the previous one
          flush();
          const int64_t j = (t - p.S) / p.Bk;
          next_bs = p.S + (j + 1) * p.Bk;
          cur_j = j;
          na = j == j_first ? na_first : 0;
          shift = na > 0 ? (float)ma : kf;
          s1 = s2 = 0.f;
          cnt = 0;
        }
        const float d = kf - shift;
        s1 += d;
        s2 = fmaf(d, d, s2);
        ++cnt;
      }
    } else if (tid < 2 * DH) {
      for (int r = 0; r < n; ++r) zacc += vs[r][c0 + tid - DH];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < RR; ++i)
#pragma unroll
    for (int j = 0; j < RC; j += 4)
      *reinterpret_cast<float4*>(Hrow + (int64_t)i * D + j) =
          make_float4(acc[i][j], acc[i][j + 1], acc[i][j + 2], acc[i][j + 3]);
  if (tid < DH) {
    flush();
    p.zk[(int64_t)unit * D + c] += zacc;
  } else if (tid < 2 * DH) {
    p.zv[(int64_t)unit * D + c0 + tid - DH] += zacc;
  }
  if (tid == 0 && half == 0) p.n[unit] += (float)(fe - fb);
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
  cfg.gridDim = dim3(p.units, 2);  // two CTAs per unit: halves of the key channels
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
  const int tpc = D == 128 ? kAppendTokens<128> : kAppendTokens<64>;
  cfg.gridDim = dim3(p.units, (p.n + tpc - 1) / tpc);
  cfg.blockDim = dim3(256);
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
