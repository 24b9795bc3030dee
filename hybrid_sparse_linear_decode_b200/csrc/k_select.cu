// Block scoring, top-k block selection and the global linear term of one
// decode step (one launch).
//
// Grid (score_ctas + lin_ctas, units).  A unit is one (batch row, KV head).
//
// * Score CTAs: each scores up to kScoreBlocksPerCta candidate blocks with the
//   second-order Taylor block score of "SPLA: Block Sparse Plus Linear Attention
//   for Long Context Modeling" (Abstract; "Principled Block Selection via Taylor
//   Expansion"), summed over the query heads of the KV group ("Grouped
//   Sparsity"):
//       score_j = sum_i q'_i . mu_j + 1/2 sum_i sum_c q'_ic^2 var_jc
//               = Q1 . mu_j + Q2 . var_j,   Q1 = sum_i q'_i,  Q2 = 1/2 sum_i q'_i^2,
//   i.e. two fp32 dot products per block, read with 16-byte vector loads: the
//   kernel is a single streaming pass over the block statistics.
//   The last score CTA of a unit (atomic ticket, no spinning) selects the top_k
//   blocks: a 4-pass 8-bit radix select finds the k-th largest score key, then
//   an order-preserving block-wide compaction emits every larger block plus the
//   lowest-index blocks equal to it -- ties go to the lower index and the output
//   is ascending.
// * Linear CTAs: phi(q)^T state for the global linear term of SLAKE's
//   first-order Taylor kernel (exp(s) ~ 1 + s): per query head i,
//       N_glob_i = zv + H^T q'_i,   D_glob_i = n + q'_i . zk,
//   each CTA owning 32 columns of H (coalesced row reads, fp32 accumulation).
#include "hyb_device.cuh"
#include "hyb_internal.h"

namespace hyb {

namespace {

constexpr uint32_t kFull = 0xffffffffu;

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

constexpr int kKeysInSmem = 4096;  // blocks whose keys fit the staging buffer (16 KB)

// Top-k of scores[0, nb) with ties to the lower index; writes sel[0, top_k)
// ascending, -1 padded.  Runs on one CTA of kSelectThreads threads.  The score
// keys are staged once in shared memory (when nb <= kKeysInSmem), so the radix
// passes and the compaction run at shared-memory latency.
__device__ void select_top_k(const SelectParams& p, int unit) {
  __shared__ uint32_t s_keys[kKeysInSmem];
  __shared__ uint32_t s_hist[256];
  __shared__ uint32_t s_wcnt[2][kSelectThreads / 32];
  __shared__ uint32_t s_digit, s_above;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int nwarps = kSelectThreads / 32;
  const float* sc = p.scores + (int64_t)unit * p.max_blocks;
  int32_t* sel = p.sel + (int64_t)unit * p.top_k;
  const int nb = p.nb;
  const int k = p.k_eff;

  const bool staged = nb <= kKeysInSmem;
  auto key = [&](int j) -> uint32_t { return staged ? s_keys[j] : float_key(__ldcg(sc + j)); };
  if (k >= nb) {
    for (int j = tid; j < p.top_k; j += kSelectThreads) sel[j] = j < nb ? j : -1;
  } else {
    bool nan_seen = false;
    if (staged) {
      for (int j = tid; j < nb; j += kSelectThreads) {
        const float f = __ldcg(sc + j);
        nan_seen |= (f != f);
        s_keys[j] = float_key(f);
      }
    }
    uint32_t prefix = 0, pmask = 0, need = (uint32_t)k;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = tid; i < 256; i += kSelectThreads) s_hist[i] = 0;
      __syncthreads();
      for (int j = tid; j < nb; j += kSelectThreads) {
        const uint32_t u = key(j);
        if (!staged && pass == 0 && u == 0u) nan_seen |= (__ldcg(sc + j) != __ldcg(sc + j));
        if ((u & pmask) == prefix) atomicAdd(&s_hist[(u >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        // lane l owns digits 255-8l .. 248-8l, highest first
        uint32_t cnt[8], local = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          cnt[e] = s_hist[255 - 8 * lane - e];
          local += cnt[e];
        }
        uint32_t incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_up_sync(kFull, incl, o);
          if (lane >= o) incl += v;
        }
        const uint32_t excl = incl - local;
        if (excl < need && incl >= need) {
          uint32_t c = excl;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (c + cnt[e] >= need) {
              s_digit = 255u - 8u * lane - e;
              s_above = c;
              break;
            }
            c += cnt[e];
          }
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      pmask |= 0xffu << shift;
      need -= s_above;
      __syncthreads();
    }
    if (nan_seen) atomicOr(p.status, HYB_STATUS_NAN_SCORE);
    const uint32_t tau = prefix;  // key of the k-th largest score
    // `need` blocks equal to tau are taken, lowest index first
    uint32_t taken_base = 0, eq_base = 0;
    for (int base = 0; base < nb; base += kSelectThreads) {
      const int j = base + tid;
      const uint32_t u = j < nb ? key(j) : 0u;
      const bool gt = j < nb && u > tau;
      const bool eq = j < nb && u == tau;
      const uint32_t beq = __ballot_sync(kFull, eq);
      if (lane == 0) s_wcnt[0][warp] = __popc(beq);
      __syncthreads();
      uint32_t eq_rank = eq_base + __popc(beq & lanemask_lt());
      for (int w = 0; w < warp; ++w) eq_rank += s_wcnt[0][w];
      const bool take = gt || (eq && eq_rank < need);
      const uint32_t bt = __ballot_sync(kFull, take);
      if (lane == 0) s_wcnt[1][warp] = __popc(bt);
      __syncthreads();
      uint32_t pos = taken_base + __popc(bt & lanemask_lt());
      for (int w = 0; w < warp; ++w) pos += s_wcnt[1][w];
      if (take) sel[pos] = j;
      uint32_t tt = 0, te = 0;
      for (int w = 0; w < nwarps; ++w) {
        tt += s_wcnt[1][w];
        te += s_wcnt[0][w];
      }
      taken_base += tt;
      eq_base += te;
      __syncthreads();
    }
    for (int j = k + tid; j < p.top_k; j += kSelectThreads) sel[j] = -1;
  }
  if (p.sel_out != nullptr) {
    __syncthreads();
    __threadfence_block();
    for (int j = tid; j < p.top_k; j += kSelectThreads)
      p.sel_out[(int64_t)unit * p.top_k + j] = sel[j];
  }
}

template <int D>
__device__ void score_blocks(const SelectParams& p, int unit, const float (*s_q)[D]) {
  __shared__ __align__(16) float s_q1[D];
  __shared__ __align__(16) float s_q2[D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int c = tid; c < D; c += kSelectThreads) {
    float a = 0.f, b = 0.f;
    for (int i = 0; i < p.G; ++i) {
      a += s_q[i][c];
      b += s_q[i][c] * s_q[i][c];
    }
    s_q1[c] = a;
    s_q2[c] = 0.5f * b;
  }
  __syncthreads();

  constexpr int LPB = D / 8;                  // lanes per block, 8 channels each
  constexpr int BPW = 32 / LPB;               // blocks per warp per pass
  constexpr int BPP = (kSelectThreads / 32) * BPW;  // blocks per CTA pass
  constexpr int PASSES = kScoreBlocksPerCta / BPP;
  static_assert(kScoreBlocksPerCta % BPP == 0, "blocks per CTA must be a multiple of the pass width");
  const int sub = lane / LPB, li = lane % LPB;
  const float4 qa0 = *reinterpret_cast<const float4*>(&s_q1[li * 8]);
  const float4 qa1 = *reinterpret_cast<const float4*>(&s_q1[li * 8 + 4]);
  const float4 qb0 = *reinterpret_cast<const float4*>(&s_q2[li * 8]);
  const float4 qb1 = *reinterpret_cast<const float4*>(&s_q2[li * 8 + 4]);
  const int j0 = blockIdx.x * kScoreBlocksPerCta;
  const int64_t ubase = (int64_t)unit * p.max_blocks;
  const float* mu = p.mu + ubase * D;
  const float* var = p.var + ubase * D;

  float4 m0[PASSES], m1[PASSES], v0[PASSES], v1[PASSES];
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {           // issue every load first
    const int j = j0 + ps * BPP + warp * BPW + sub;
    if (j < p.nb) {
      const float4* pm = reinterpret_cast<const float4*>(mu + (int64_t)j * D + li * 8);
      const float4* pv = reinterpret_cast<const float4*>(var + (int64_t)j * D + li * 8);
      m0[ps] = __ldg(pm);
      m1[ps] = __ldg(pm + 1);
      v0[ps] = __ldg(pv);
      v1[ps] = __ldg(pv + 1);
    } else {
      m0[ps] = m1[ps] = v0[ps] = v1[ps] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    float acc = qa0.x * m0[ps].x + qa0.y * m0[ps].y + qa0.z * m0[ps].z + qa0.w * m0[ps].w;
    acc += qa1.x * m1[ps].x + qa1.y * m1[ps].y + qa1.z * m1[ps].z + qa1.w * m1[ps].w;
    acc += qb0.x * v0[ps].x + qb0.y * v0[ps].y + qb0.z * v0[ps].z + qb0.w * v0[ps].w;
    acc += qb1.x * v1[ps].x + qb1.y * v1[ps].y + qb1.z * v1[ps].z + qb1.w * v1[ps].w;
#pragma unroll
    for (int o = LPB / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
    const int j = j0 + ps * BPP + warp * BPW + sub;
    if (li == 0 && j < p.nb) p.scores[ubase + j] = acc;
  }

  if (!p.do_select) return;
  __syncthreads();
  __shared__ int s_last;
  if (tid == 0) {
    __threadfence();  // release this CTA's scores (ordered after the barrier)
    const uint32_t prev = atomicAdd(&p.tickets[unit], 1u);
    s_last = (prev == (uint32_t)p.score_ctas - 1u);
    __threadfence();
  }
  __syncthreads();
  if (!s_last) return;
  select_top_k(p, unit);
  if (tid == 0) p.tickets[unit] = 0u;  // ready for the next decode
}

template <int D>
__device__ void linear_term(const SelectParams& p, int unit, const float (*s_q)[D]) {
  __shared__ float s_red[kSelectThreads / 32][kMaxGroup][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = kSelectThreads / 32;
  constexpr int RPW = D / NW;  // rows of H per warp
  const int cb = blockIdx.x - p.score_ctas;
  const int c = cb * 32 + lane;
  const float* H = p.H + (int64_t)unit * D * D;
  float acc[kMaxGroup] = {0.f, 0.f, 0.f, 0.f};
  float h[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) h[rr] = __ldg(H + (int64_t)(warp * RPW + rr) * D + c);
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int r = warp * RPW + rr;
#pragma unroll
    for (int i = 0; i < kMaxGroup; ++i)
      if (i < p.G) acc[i] += s_q[i][r] * h[rr];
  }
#pragma unroll
  for (int i = 0; i < kMaxGroup; ++i) s_red[warp][i][lane] = acc[i];
  __syncthreads();
  const int64_t lbase = (int64_t)unit * p.G * (D + 1);
  if (warp == 0) {
    const float zv = __ldg(p.zv + (int64_t)unit * D + c);
    for (int i = 0; i < p.G; ++i) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) s += s_red[w][i][lane];
      p.lin[lbase + (int64_t)i * (D + 1) + c] = zv + s;
    }
  } else if (warp == 1 && cb == 0) {
    const float* zk = p.zk + (int64_t)unit * D;
    for (int i = 0; i < p.G; ++i) {
      float s = 0.f;
      for (int r = lane; r < D; r += 32) s += s_q[i][r] * __ldg(zk + r);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
      if (lane == 0) p.lin[lbase + (int64_t)i * (D + 1) + D] = __ldg(p.n + unit) + s;
    }
  } else if (warp == 2 && cb == 0 && p.nb == 0 && p.sel_out != nullptr) {
    for (int j = lane; j < p.top_k; j += 32) p.sel_out[(int64_t)unit * p.top_k + j] = -1;
  }
}

template <int D>
__global__ void __launch_bounds__(kSelectThreads) select_kernel(const SelectParams p) {
  // the attention kernel may be scheduled now; it waits for this grid before
  // reading the selection and the linear term
  pdl_allow_dependents();
  __shared__ __align__(16) float s_q[kMaxGroup][D];
  const int unit = blockIdx.y;
  const __nv_bfloat16* q = p.q + (int64_t)unit * p.G * D;
  for (int e = threadIdx.x; e < p.G * D; e += kSelectThreads)
    s_q[e / D][e % D] = __bfloat162float(q[e]) * p.scale;
  __syncthreads();
  if ((int)blockIdx.x < p.score_ctas)
    score_blocks<D>(p, unit, s_q);
  else
    linear_term<D>(p, unit, s_q);
}

}  // namespace

cudaError_t prepare_select(int D) {
  // the same shared-memory carveout as the attention kernel, so the SMs need no
  // reconfiguration between the two launches of a decode
  const void* f = D == 128 ? (const void*)select_kernel<128> : (const void*)select_kernel<64>;
  return cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
}

cudaError_t launch_select(const SelectParams& p, int D, int grid_x, cudaStream_t s) {
  const dim3 grid(grid_x, p.units);
  if (D == 128)
    select_kernel<128><<<grid, kSelectThreads, 0, s>>>(p);
  else
    select_kernel<64><<<grid, kSelectThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace hyb
