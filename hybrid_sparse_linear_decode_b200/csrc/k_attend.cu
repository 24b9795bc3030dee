// Exact attention over the gathered sinks, window and selected blocks, the
// selected blocks' (1 + s) subtraction terms, and the merge under one shared
// normaliser -- one launch per decode step.
//
// Work: each unit (batch row, KV head) owns a fixed list of <= 64-token chunks
// of its exact set X (sink pieces, window pieces, then ceil(Bk/64) pieces per
// selected block).  The units' lists are concatenated and cut into `grid`
// contiguous ranges, one per CTA (split-K); every (CTA, unit) pair writes one
// partial record, and the last CTA to finish a unit (atomic ticket, no
// spinning) merges that unit's partials with the global linear term.
//
// CTA: 2 groups of 4 warps (8 warps, so two per SM sub-partition and up to 255
// registers a thread).  A 4-stage shared-memory ring is filled with TMA tensor
// loads (cp.async.bulk.tensor, 128-byte swizzle, 16-row boxes, no multicast) of
// each chunk's K and V rows; group g owns the chunks of local index i = g (mod 2)
// and hence stages g and g + 2: after its 4 warps have consumed chunk i (group
// barrier), the group's leader thread reuses the stage for chunk i + 4.  Warp w
// of a group handles tokens [16w, 16w+16) of a chunk.
//
// Per warp and 16 tokens, on the tensor cores (mma.sync m16n8k16, bf16 in, fp32
// accumulate), with the G <= 4 query heads of the KV group packed into the
// 16-row M dimension:
//   S^T = Qpad * K^T  -- rows 0-3 and 4-7 both hold q_0..q_3, rows 8-15 zero,
//                        so lanes of rows 0-3 get s for the softmax part and
//                        lanes of rows 4-7 the same s for the Taylor part;
//   O  += A * V       -- A rows 0-3: e^{s - m} (online max m per head),
//                        rows 4-7: (1 + s) on selected-block tokens, 0 otherwise,
//                        rows 8-15: the bf16 rounding remainders of rows 0-7
//                        (hi/lo split), so the weights enter at ~16-bit precision.
// So the exact part N_ex, D_ex and the subtraction terms N_sel, D_sel come out of
// the same pass over each K/V tile ("SPLA: Block Sparse Plus Linear Attention
// for Long Context Modeling", Abstract: residual = global - selected; "SLAKE",
// Abstract: first-order Taylor exp(s) ~ 1 + s).
//
// Merge of a unit (per query head, base-2 exponent m of the exact part):
//   o = (N_ex + 2^{-m} (N_glob - N_sel)) / (D_ex + 2^{-m} (D_glob - D_sel)),
// evaluated as the equal form (N_ex 2^m + ...)/(D_ex 2^m + ...) when m < 0.
#include "hyb_device.cuh"
#include "hyb_internal.h"

namespace hyb {

namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kConsumerThreads = kConsumerGroups * kWarpsPerGroup * 32;

template <int D>
struct AttendSmem {
  static constexpr int kTileBytes = kTile * D * 2;      // one of K or V for 64 tokens
  static constexpr int kBoxBytes = kBoxRows * D * 2;
  uint8_t kv[kStages][2][kTileBytes];                   // 1024-byte aligned (base aligned)
  float wpart[kConsumerGroups * kWarpsPerGroup][partial_floats(D)];
  uint64_t full[kStages];
  int4 desc[kStages];                                   // start, len, is_sel, unit
  int abort_flag;
  int last_flag;
};

// Byte offset of (row t, 16-byte chunk C) in a tile written by TMA with the
// 128-byte swizzle: 128-byte line L = t*(D/64) + C/8, chunk slot (C%8) ^ (L%8).
template <int D>
__device__ __forceinline__ uint32_t swz(int t, int C) {
  const int L = t * (D / 64) + (C >> 3);
  return (uint32_t)(L * 128 + (((C & 7) ^ (L & 7)) << 4));
}

__device__ __forceinline__ void group_sync(int grp) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "n"(kWarpsPerGroup * 32) : "memory");
}

__device__ __forceinline__ int64_t cta_of_chunk(int64_t c, int64_t total, int grid) {
  return ((c + 1) * grid - 1) / total;
}

__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Merge the partial records of `unit` written by CTAs [first, last] (slot =
// cta + unit) with the global linear term; consumer threads only.
template <int D>
__device__ void merge_unit(const AttendParams& p, int unit, int64_t first, int64_t last, int ctid) {
  constexpr int PF = partial_floats(D);
  pdl_wait_primary();  // the linear term comes from the preceding select kernel
  const int G = p.G;
  const float* lin = p.lin + (int64_t)unit * G * (D + 1);
  for (int e = ctid; e < G * D; e += kConsumerThreads) {
    const int i = e / D, d = e % D;
    float M = -INFINITY;
    for (int64_t c = first; c <= last; ++c) M = fmaxf(M, __ldcg(p.partials + (c + unit) * PF + i));
    const float Ms = (M == -INFINITY) ? 0.f : M;
    float Dex = 0.f, Nex = 0.f, Dsel = 0.f, Nsel = 0.f;
    for (int64_t c = first; c <= last; ++c) {
      const float* gp = p.partials + (c + unit) * PF;
      const float m = __ldcg(gp + i);
      const float f = (m == -INFINITY) ? 0.f : exp2f(m - Ms);
      Dex += __ldcg(gp + 4 + i) * f;
      Dsel += __ldcg(gp + 8 + i);
      Nex += __ldcg(gp + 16 + i * D + d) * f;
      Nsel += __ldcg(gp + 16 + 4 * D + i * D + d);
    }
    const float Ng = __ldcg(lin + (int64_t)i * (D + 1) + d);
    const float Dg = __ldcg(lin + (int64_t)i * (D + 1) + D);
    float num, den;
    if (Ms >= 0.f) {
      const float f = exp2f(-Ms);
      num = Nex + f * (Ng - Nsel);
      den = Dex + f * (Dg - Dsel);
    } else {
      const float f = exp2f(Ms);
      num = Nex * f + (Ng - Nsel);
      den = Dex * f + (Dg - Dsel);
    }
    const float o = num / den;
    p.out[((int64_t)unit * G + i) * D + d] = o;
    if (!(den > 0.f)) atomicOr(p.status, HYB_STATUS_DENOMINATOR);
    if (!isfinite(o)) atomicOr(p.status, HYB_STATUS_NONFINITE);
  }
}

// Hand chunk i (local index within this CTA's range) to its pipeline stage:
// write its descriptor and start the TMA loads of its K and V rows (16-row boxes;
// rows past the chunk end are read too and ignored).  Called by one thread.
template <int D>
__device__ void issue_chunk(const CUtensorMap* tmK, const CUtensorMap* tmV, const AttendParams& p,
                            AttendSmem<D>& sm, int64_t c_begin, int i, bool& waited) {
  using S = AttendSmem<D>;
  const int64_t c = c_begin + i;
  const int cpu = p.chunks_per_unit;
  const int unit = (int)(c / cpu);
  const int ci = (int)(c % cpu);
  const int stage = i % kStages;
  int start = 0, len = 0, is_sel = 0;
  if (ci < p.n_sink_chunks) {
    start = ci * kTile;
    len = min(kTile, p.sink_len - start);
  } else if (ci < p.n_sink_chunks + p.n_win_chunks) {
    start = p.win_start + (ci - p.n_sink_chunks) * kTile;
    len = min(kTile, p.T - start);
  } else {
    if (!waited) {  // the selection is written by the preceding select kernel
      pdl_wait_primary();
      waited = true;
    }
    const int s = ci - p.n_sink_chunks - p.n_win_chunks;
    const int slot = s / p.chunks_per_block, piece = s % p.chunks_per_block;
    is_sel = 1;
    const int j = slot < p.k_eff ? __ldcg(p.sel + (int64_t)unit * p.top_k + slot) : -1;
    if (j >= 0 && j < p.nb) {
      const int bs = p.S + j * p.Bk;
      const int be = min(bs + p.Bk, p.ev_end);
      start = bs + piece * kTile;
      len = max(0, min(kTile, be - start));
    } else if (j != -1) {
      atomicOr(p.status, HYB_STATUS_BAD_SELECTION);
    }
  }
  sm.desc[stage] = make_int4(start, len, is_sel, unit);
  if (len > 0) {
    const int nbox = (len + kBoxRows - 1) / kBoxRows;
    mbar_arrive_expect_tx(&sm.full[stage], (uint32_t)(nbox * S::kBoxBytes * 2));
    const int row = (int)((int64_t)unit * p.cap + start);
    const uint32_t kdst = smem_u32(sm.kv[stage][0]);
    const uint32_t vdst = smem_u32(sm.kv[stage][1]);
    for (int bx = 0; bx < nbox; ++bx) {
      tma_load_3d(kdst + bx * S::kBoxBytes, tmK, 0, 0, row + bx * kBoxRows, &sm.full[stage]);
      tma_load_3d(vdst + bx * S::kBoxBytes, tmV, 0, 0, row + bx * kBoxRows, &sm.full[stage]);
    }
  } else {
    mbar_arrive(&sm.full[stage]);
  }
}

template <int D>
__global__ void __launch_bounds__(kAttendThreads, 1)
    attend_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const AttendParams p) {
  constexpr int PF = partial_floats(D);
  constexpr int NT8 = D / 8;   // 8-column tiles of the head dimension
  constexpr int KS = D / 16;   // k-steps of the QK product
  extern __shared__ uint8_t smem_raw[];
  AttendSmem<D>& sm = *reinterpret_cast<AttendSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;

  if (p.merge_only) {  // empty exact set: output = global linear term only
    merge_unit<D>(p, cta, 0, -1, tid);
    return;
  }

  const int64_t c_begin = (int64_t)cta * p.total_chunks / p.grid;
  const int64_t c_end = (int64_t)(cta + 1) * p.total_chunks / p.grid;
  const int n_local = (int)(c_end - c_begin);

  const int grp = warp / kWarpsPerGroup;
  const int wi = warp % kWarpsPerGroup;
  const bool leader = (wi == 0 && lane == 0);
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[s], 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  bool waited = false;       // leader: has waited for the select kernel
  int next_issue = grp;      // leader: next local chunk index of this group to issue
  if (leader) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    for (; next_issue < n_local && next_issue < kStages; next_issue += kConsumerGroups)
      issue_chunk<D>(&tmK, &tmV, p, sm, c_begin, next_issue, waited);
  }

  const int g = lane >> 2, tig = lane & 3;
  const bool p_lane = g < 4;           // rows 0-3: softmax part; rows 4-7: Taylor part
  const int head = g & 3;
  const bool head_ok = head < p.G;
  const int cpu = p.chunks_per_unit;
  const int r0 = wi * 16;
  const int mi = lane >> 3, rr = lane & 7;

  int64_t c = c_begin;
  while (c < c_end) {
    const int unit = (int)(c / cpu);
    const int64_t seg_end = min(c_end, (int64_t)(unit + 1) * cpu);

    uint32_t qa[KS][2];
    {
      const uint32_t* qrow =
          reinterpret_cast<const uint32_t*>(p.q + ((int64_t)unit * p.G + (head_ok ? head : 0)) * D);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        qa[kk][0] = head_ok ? __ldg(qrow + kk * 8 + tig) : 0u;
        qa[kk][1] = head_ok ? __ldg(qrow + kk * 8 + 4 + tig) : 0u;
      }
    }
    float O[NT8][4];
#pragma unroll
    for (int n = 0; n < NT8; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f, dsel_run = 0.f;

    const int i_seg = (int)(c - c_begin);
    for (int i = i_seg + ((i_seg & 1) != grp ? 1 : 0); c_begin + i < seg_end; i += kConsumerGroups) {
      const int stage = i % kStages;
      bool ok = !*(volatile int*)&sm.abort_flag;
      if (ok && !mbar_wait_bounded(&sm.full[stage], (i / kStages) & 1, kWaitLimit)) {
        sm.abort_flag = 1;
        atomicOr(p.status, HYB_STATUS_TIMEOUT);
        ok = false;
      }
      const int4 dsc = sm.desc[stage];
      const int nvalid = ok ? min(16, dsc.y - r0) : 0;
      if (nvalid > 0) {
        const uint32_t kb = smem_u32(sm.kv[stage][0]);
        const uint32_t vb = smem_u32(sm.kv[stage][1]);
        if (nvalid < 16) {
          // rows past the chunk may hold tokens beyond T (unwritten cache rows):
          // zero their V rows so that 0-weight * garbage cannot make a NaN
          constexpr int CPR = D / 8;  // 16-byte chunks per row
          for (int e = lane; e < (16 - nvalid) * CPR; e += 32) {
            const int t = r0 + nvalid + e / CPR;
            *reinterpret_cast<uint4*>(&sm.kv[stage][1][swz<D>(t, e % CPR)]) = make_uint4(0, 0, 0, 0);
          }
          // order these generic-proxy writes before the next TMA write of the stage
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
        }
        // ---- S^T = Qpad K^T for 16 tokens (two 8-token n-tiles)
        float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + swz<D>(r0 + (mi >> 1) * 8 + rr, kk * 2 + (mi & 1)), b0, b1, b2, b3);
          mma_16816(sacc[0], qa[kk][0], 0u, qa[kk][1], 0u, b0, b1);
          mma_16816(sacc[1], qa[kk][0], 0u, qa[kk][1], 0u, b2, b3);
        }
        // ---- weights of this lane's 4 tokens: n-tile nt, element e -> token nt*8 + 2*tig + e
        float s[4], x[4];
        bool v[4];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int nt = q4 >> 1, e = q4 & 1;
          v[q4] = (nt * 8 + 2 * tig + e) < nvalid;
          s[q4] = sacc[nt][e] * p.scale;
          x[q4] = (p_lane && v[q4]) ? s[q4] * kLog2e : -INFINITY;
        }
        float tmax = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 2));
        const float m_new = fmaxf(m_run, tmax);
        const float alpha = (p_lane && m_new != -INFINITY) ? exp2f(m_run - m_new) : 1.f;
        const bool sel_tok = dsc.z != 0;
        float w[4], wsum = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          w[q4] = p_lane ? (v[q4] ? exp2f(x[q4] - m_new) : 0.f) : ((v[q4] && sel_tok) ? 1.f + s[q4] : 0.f);
          wsum += w[q4];
        }
        if (p_lane) {
          l_run = l_run * alpha + wsum;
          m_run = m_new;
        } else {
          dsel_run += wsum;
        }
        if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll
          for (int n = 0; n < NT8; ++n) {
            O[n][0] *= alpha;
            O[n][1] *= alpha;
            O[n][2] *= alpha;
            O[n][3] *= alpha;
          }
        }
        uint32_t a0, a1, a2, a3;  // rows g (hi) / g+8 (lo), tokens 0-7 / 8-15 of the k=16 step
        split_bf16(w[0], w[1], a0, a1);
        split_bf16(w[2], w[3], a2, a3);
        // ---- O += A V over 16 tokens
#pragma unroll
        for (int np = 0; np < NT8 / 2; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vb + swz<D>(r0 + (mi & 1) * 8 + rr, np * 2 + (mi >> 1)), b0, b1, b2, b3);
          mma_16816(O[2 * np], a0, a1, a2, a3, b0, b1);
          mma_16816(O[2 * np + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      group_sync(grp);  // the group is done with this stage
      if (leader && next_issue < n_local && !*(volatile int*)&sm.abort_flag) {
        issue_chunk<D>(&tmK, &tmV, p, sm, c_begin, next_issue, waited);
        next_issue += kConsumerGroups;
      }
    }

    // ---- this warp's partial -> shared memory
    {
      float l = l_run + __shfl_xor_sync(kFull, l_run, 1);
      l += __shfl_xor_sync(kFull, l, 2);
      float ds = dsel_run + __shfl_xor_sync(kFull, dsel_run, 1);
      ds += __shfl_xor_sync(kFull, ds, 2);
      float* wp = sm.wpart[warp];
      if (tig == 0) {
        if (p_lane) {
          wp[head] = m_run;
          wp[4 + head] = l;
        } else {
          wp[8 + head] = ds;
        }
      }
      float* dst = wp + 16 + (p_lane ? 0 : 4 * D) + head * D;
#pragma unroll
      for (int n = 0; n < NT8; ++n) {
        dst[n * 8 + 2 * tig] = O[n][0] + O[n][2];
        dst[n * 8 + 2 * tig + 1] = O[n][1] + O[n][3];
      }
    }
    __syncthreads();
    // ---- combine the 8 warps -> one partial record for (cta, unit)
    {
      constexpr int NW = kConsumerGroups * kWarpsPerGroup;
      float* gp = p.partials + (int64_t)(cta + unit) * PF;
      if (tid < 4) {
        float M = -INFINITY;
        for (int w = 0; w < NW; ++w) M = fmaxf(M, sm.wpart[w][tid]);
        float l = 0.f, ds = 0.f;
        for (int w = 0; w < NW; ++w) {
          const float m = sm.wpart[w][tid];
          l += (m == -INFINITY) ? 0.f : sm.wpart[w][4 + tid] * exp2f(m - M);
          ds += sm.wpart[w][8 + tid];
        }
        gp[tid] = M;
        gp[4 + tid] = l;
        gp[8 + tid] = ds;
      }
      for (int e = tid; e < 8 * D; e += kConsumerThreads) {
        float acc = 0.f;
        if (e < 4 * D) {
          const int hh = e / D;
          float M = -INFINITY;
          for (int w = 0; w < NW; ++w) M = fmaxf(M, sm.wpart[w][hh]);
          for (int w = 0; w < NW; ++w) {
            const float m = sm.wpart[w][hh];
            if (m != -INFINITY) acc += sm.wpart[w][16 + e] * exp2f(m - M);
          }
        } else {
          for (int w = 0; w < NW; ++w) acc += sm.wpart[w][16 + e];
        }
        gp[16 + e] = acc;
      }
      __threadfence();
    }
    __syncthreads();
    const int64_t first = cta_of_chunk((int64_t)unit * cpu, p.total_chunks, p.grid);
    const int64_t last = cta_of_chunk((int64_t)(unit + 1) * cpu - 1, p.total_chunks, p.grid);
    if (tid == 0) {
      const uint32_t prev = atomicAdd(&p.tickets[unit], 1u);
      sm.last_flag = (prev == (uint32_t)(last - first));
    }
    __syncthreads();
    if (sm.last_flag) {
      __threadfence();
      merge_unit<D>(p, unit, first, last, tid);
      if (tid == 0) p.tickets[unit] = 0u;
    }
    __syncthreads();
    c = seg_end;
  }
  if (leader && *(volatile int*)&sm.abort_flag) {
    // do not leave while copies into this CTA's shared memory may be in flight
    for (int i = next_issue - kConsumerGroups; i >= 0 && i >= next_issue - kStages; i -= kConsumerGroups)
      mbar_wait_bounded(&sm.full[i % kStages], (i / kStages) & 1, kWaitLimit);
  }
}

}  // namespace

size_t attend_smem_bytes(int D);

cudaError_t prepare_attend(int D) {
  const int smem = (int)attend_smem_bytes(D);
  if (D == 128) return cudaFuncSetAttribute(attend_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return cudaFuncSetAttribute(attend_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

size_t attend_smem_bytes(int D) {
  return (D == 128 ? sizeof(AttendSmem<128>) : sizeof(AttendSmem<64>)) + 1024;
}

cudaError_t launch_attend(const CUtensorMap* tmK, const CUtensorMap* tmV, const AttendParams& p, int D, bool pdl,
                          cudaStream_t s) {
  const size_t smem = attend_smem_bytes(D);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.merge_only ? p.units : p.grid);
  cfg.blockDim = dim3(kAttendThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (D == 128) return cudaLaunchKernelEx(&cfg, attend_kernel<128>, *tmK, *tmV, p);
  return cudaLaunchKernelEx(&cfg, attend_kernel<64>, *tmK, *tmV, p);
}

}  // namespace hyb
