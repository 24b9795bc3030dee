// Block scoring and the global linear term of one decode step, plus the fold
// of the evictions since the previous decode into the state (one launch).
//
// Persistent grid of kSelectCtasPerSm CTAs per SM.  The work of a decode is a
// list of equal-sized items, unit-major (a unit is one (batch row, KV head)):
// per unit, ceil(nb / R) score items of R consecutive blocks, then
// sel_lin_items(D) linear items of sel_item_rows(D) rows of H each.  CTA c
// takes the contiguous item range [c*N/grid, (c+1)*N/grid), so its data is
// one near-sequential stream; thread 0 pulls each item (the rows, and the
// unit's query heads) into a kSelStages-deep shared-memory ring with untiled
// bulk copies (cp.async.bulk, no multicast) and the CTA works from there.
//
// * Score items: the second-order Taylor block score of "SPLA: Block Sparse
//   Plus Linear Attention for Long Context Modeling" (Abstract; "Principled
//   Block Selection via Taylor Expansion"), summed over the query heads of the
//   KV group ("Grouped Sparsity"):
//       score_j = sum_i ( q'_i . mu_j + 1/2 sum_c q'_ic^2 var_jc ).
//   The top-k over these scores runs in the attention kernel, which reads them.
// * Linear items: phi(q)^T state of the global linear term of SLAKE's
//   first-order Taylor kernel (exp(s) ~ 1 + s), per query head i and row group g:
//       N_i += sum_{r in g} q'_ir H[r][:]  (+ zv in group 0),
//       D_i  = n + q'_i . zk               (group 0),
//   written as one partial per row group; the attention merge adds the groups.
// * Evictions since the previous decode (positions [fold_begin, fold_end) of
//   the evicted stream, usually one token) are folded into the rows each item
//   holds before it uses them: H += k v^T, zk += k, zv += v, n += 1 (the
//   recurrence of SPLA's residual linear attention) and Welford's running mean
//   / population variance of the token's block (B. P. Welford, Technometrics
//   4(3), 1962).  With q == null the kernel only folds (items with nothing to
//   fold load nothing).
//
// Launch chaining (programmatic dependent launch): the first kernel of a
// decode; it waits for its predecessor grid before touching memory, then lets
// the attention kernel start at once, which streams the window beside it and
// waits for this grid only before it needs the scores.
#include "hyb_device.cuh"
#include "hyb_internal.h"

namespace hyb {

namespace {

constexpr uint32_t kFull = 0xffffffffu;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& raw, float (&f)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = bf16_lo(w[e]);
    f[2 * e + 1] = bf16_hi(w[e]);
  }
}

template <int D>
struct SelectSmem {
  struct Stage {
    float data[kSelItemBytes / 4];         // mean rows then variance rows, or rows of H
    __nv_bfloat16 q[kMaxGroup * D];        // the item's query heads
  };
  Stage st[kSelStages];
  uint64_t full[kSelStages];
  int abort;
};

// ---------------------------------------------------------------- items
__device__ __forceinline__ bool item_has_fold(const SelectParams& p, int local, int R) {
  if (p.fold_end <= p.fold_begin) return false;
  if (local >= p.score_items) return true;  // every linear item folds into its rows
  const int64_t j0 = (int64_t)local * R;
  const int64_t jb0 = (p.fold_begin - p.S) / p.Bk, jb1 = (p.fold_end - 1 - p.S) / p.Bk;
  return jb1 >= j0 && jb0 < j0 + R;
}

// Start the copies of item `it` into stage `stage` (thread 0).
template <int D>
__device__ void issue_item(const SelectParams& p, SelectSmem<D>& sm, int it, int stage) {
  constexpr int R = sel_item_blocks(D), RL = sel_item_rows(D);
  const int unit = it / p.items_per_unit, local = it % p.items_per_unit;
  auto& st = sm.st[stage];
  if (p.q == nullptr && !item_has_fold(p, local, R)) {
    mbar_arrive(&sm.full[stage]);
    return;
  }
  const uint32_t qbytes = p.q ? (uint32_t)(p.G * D * 2) : 0u;
  uint32_t bytes;
  const float* src0;
  const float* src1 = nullptr;
  if (local < p.score_items) {
    const int j0 = local * R;
    const int nblk = min(R, p.nb - j0);
    bytes = (uint32_t)(nblk * D * 4);
    src0 = p.mu + ((int64_t)unit * p.max_blocks + j0) * D;
    src1 = p.var + ((int64_t)unit * p.max_blocks + j0) * D;
  } else {
    const int r0 = (local - p.score_items) * RL;
    bytes = (uint32_t)(RL * D * 4);
    src0 = p.H + ((int64_t)unit * D + r0) * D;
  }
  mbar_arrive_expect_tx(&sm.full[stage], qbytes + (src1 ? 2u : 1u) * bytes);
  if (qbytes) bulk_load(smem_u32(st.q), p.q + (int64_t)unit * p.G * D, qbytes, &sm.full[stage]);
  bulk_load(smem_u32(st.data), src0, bytes, &sm.full[stage]);
  if (src1) bulk_load(smem_u32(st.data + R * D), src1, bytes, &sm.full[stage]);
}

// Score item: R blocks, D/8 lanes per block, 8 channels per lane.
template <int D>
__device__ void score_item(const SelectParams& p, typename SelectSmem<D>::Stage& st, int unit, int local) {
  constexpr int R = sel_item_blocks(D), LPB = D / 8;
  static_assert(R * LPB == kSelectThreads, "one thread per 8 channels of a block");
  const int tid = threadIdx.x, b = tid / LPB, li = tid % LPB;
  const int j = local * R + b;
  const bool valid = j < p.nb;
  float m[8], v[8];
  {
    const float4* pm = reinterpret_cast<const float4*>(st.data + b * D + li * 8);
    const float4* pv = reinterpret_cast<const float4*>(st.data + R * D + b * D + li * 8);
    const float4 m0 = pm[0], m1 = pm[1], v0 = pv[0], v1 = pv[1];
    m[0] = m0.x; m[1] = m0.y; m[2] = m0.z; m[3] = m0.w; m[4] = m1.x; m[5] = m1.y; m[6] = m1.z; m[7] = m1.w;
    v[0] = v0.x; v[1] = v0.y; v[2] = v0.z; v[3] = v0.w; v[4] = v1.x; v[5] = v1.y; v[6] = v1.z; v[7] = v1.w;
  }
  if (valid && p.fold_end > p.fold_begin) {
    const int64_t bs = p.S + (int64_t)j * p.Bk;
    const int64_t a = max(bs, p.fold_begin), e = min(bs + p.Bk, p.fold_end);
    if (a < e) {
      for (int64_t t = a; t < e; ++t) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p.k_cache + ((int64_t)unit * p.cap + t) * D + li * 8));
        float x[8];
        bf16x8_to_f32(raw, x);
        if (t == bs) {  // the block's first token: the stored row is not read
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            m[c] = x[c];
            v[c] = 0.f;
          }
        } else {
          const float cnt = (float)(t - bs + 1);
          const float inv = 1.f / cnt;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float delta = x[c] - m[c];
            const float m1 = m[c] + delta * inv;
            v[c] = (v[c] * (cnt - 1.f) + delta * (x[c] - m1)) * inv;
            m[c] = m1;
          }
        }
      }
      float4* gm = reinterpret_cast<float4*>(p.mu + ((int64_t)unit * p.max_blocks + j) * D + li * 8);
      float4* gv = reinterpret_cast<float4*>(p.var + ((int64_t)unit * p.max_blocks + j) * D + li * 8);
      gm[0] = make_float4(m[0], m[1], m[2], m[3]);
      gm[1] = make_float4(m[4], m[5], m[6], m[7]);
      gv[0] = make_float4(v[0], v[1], v[2], v[3]);
      gv[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
  if (p.q == nullptr) return;
  float acc = 0.f;  // sum over the group's heads of q'_i . mu + 1/2 q'_i^2 . var (8 channels)
  for (int i = 0; i < p.G; ++i) {
    float f[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(st.q + i * D + li * 8), f);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float qs = f[c] * p.scale;
      acc += qs * (m[c] + 0.5f * qs * v[c]);
    }
  }
#pragma unroll
  for (int o = LPB / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
  if (li == 0 && valid) p.scores[(int64_t)unit * p.max_blocks + j] = acc;
}

// Linear item `rg`: rows [rg*RL, (rg+1)*RL) of H; thread (h, c) holds column c
// of RPT consecutive rows.
template <int D>
__device__ void lin_item(const SelectParams& p, typename SelectSmem<D>::Stage& st, int unit, int rg) {
  constexpr int RL = sel_item_rows(D), NH = kSelectThreads / D, RPT = RL / NH;
  static_assert(RPT % 8 == 0, "rows per thread come in 16-byte key loads");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = tid % D, h = tid / D;
  const int rl = h * RPT;          // first row of this thread inside the item
  const int r0 = rg * RL + rl;     // ... and inside H
  const bool fold = p.fold_end > p.fold_begin;
  if (p.q == nullptr && !fold) return;
  float hv[RPT];
#pragma unroll
  for (int rr = 0; rr < RPT; ++rr) hv[rr] = st.data[(rl + rr) * D + c];
  const bool zrow = (rg == 0 && h == 0);                     // owner of zk[c], zv[c]
  const bool nown = (rg == 0 && tid == kSelectThreads - 32);  // owner of n (writes D_glob too)
  float zkc = 0.f, zvc = 0.f, n_new = 0.f;
  if (zrow) {
    zkc = p.zk[(int64_t)unit * D + c];
    zvc = p.zv[(int64_t)unit * D + c];
  }
  if (nown) n_new = p.n[unit];
  if (fold) {
    const int64_t ub = (int64_t)unit * p.cap;
    for (int64_t t = p.fold_begin; t < p.fold_end; ++t) {
      const __nv_bfloat16* kt = p.k_cache + (ub + t) * D;
      const float vt = __bfloat162float(p.v_cache[(ub + t) * D + c]);
#pragma unroll
      for (int r8 = 0; r8 < RPT; r8 += 8) {
        float kf[8];
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(kt + r0 + r8)), kf);
#pragma unroll
        for (int e = 0; e < 8; ++e) hv[r8 + e] += kf[e] * vt;
      }
      if (zrow) {
        zkc += __bfloat162float(kt[c]);
        zvc += vt;
      }
    }
    float* Hg = p.H + ((int64_t)unit * D + r0) * D + c;
#pragma unroll
    for (int rr = 0; rr < RPT; ++rr) Hg[(int64_t)rr * D] = hv[rr];
    if (zrow) {
      p.zk[(int64_t)unit * D + c] = zkc;
      p.zv[(int64_t)unit * D + c] = zvc;
    }
    if (nown) {
      n_new += (float)(p.fold_end - p.fold_begin);
      p.n[unit] = n_new;
    }
  }
  if (p.q == nullptr) return;

  const int G = p.G;
  float acc[kMaxGroup] = {0.f, 0.f, 0.f, 0.f};
  float zdot[kMaxGroup] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < kMaxGroup; ++i) {
    if (i < G) {
#pragma unroll
      for (int r8 = 0; r8 < RPT; r8 += 8) {
        float qf[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(st.q + i * D + r0 + r8), qf);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i] += qf[e] * hv[r8 + e];
      }
      acc[i] *= p.scale;
      if (zrow) zdot[i] = __bfloat162float(st.q[i * D + c]) * p.scale * zkc;
    }
  }
  __syncthreads();  // every thread has its rows: the stage data becomes the reduction buffer
  float* red = st.data;             // [NH][G][D]
  float* zred = st.data + NH * kMaxGroup * D;  // [G][D]
#pragma unroll
  for (int i = 0; i < kMaxGroup; ++i) {
    if (i < G) {
      red[(h * kMaxGroup + i) * D + c] = acc[i];
      if (zrow) zred[i * D + c] = zdot[i];
    }
  }
  __syncthreads();
  float* lin = p.lin + ((int64_t)unit * p.lin_items + rg) * G * (D + 1);
  if (h == 0) {
    for (int i = 0; i < G; ++i) {
      float s = (rg == 0) ? zvc : 0.f;
#pragma unroll
      for (int hh = 0; hh < NH; ++hh) s += red[(hh * kMaxGroup + i) * D + c];
      lin[i * (D + 1) + c] = s;
    }
  }
  if (rg == 0 && warp == kSelectThreads / 32 - 1) {
    for (int i = 0; i < G; ++i) {
      float s = 0.f;
      for (int cc = lane; cc < D; cc += 32) s += zred[i * D + cc];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
      if (lane == 0) lin[i * (D + 1) + D] = n_new + s;
    }
  }
  // the stage was written through the generic proxy: order that before the
  // next bulk copy into it
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int D>
__global__ void __maxnreg__(kSelectMaxRegs) select_kernel(const SelectParams p) {
  extern __shared__ uint8_t smem_raw[];
  // 128-byte aligned; offsetting the shared array keeps accesses in the shared space
  SelectSmem<D>& sm = *reinterpret_cast<SelectSmem<D>*>(smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u));
  const int tid = threadIdx.x;
  // one thread waits for the predecessor grid (the barrier below holds the rest)
  if (tid == 0) pdl_wait_primary();

  const int it0 = (int)((int64_t)p.total_items * blockIdx.x / gridDim.x);
  const int it1 = (int)((int64_t)p.total_items * (blockIdx.x + 1) / gridDim.x);
  const int n_mine = it1 - it0;
  if (tid == 0) {
    for (int s = 0; s < kSelStages; ++s) mbar_init(&sm.full[s], 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_allow_dependents();  // the attention kernel starts now and streams beside this grid
  int issued = 0;  // thread 0: items whose copies have been started
  if (tid == 0)
    for (; issued < n_mine && issued < kSelStages; ++issued) issue_item<D>(p, sm, it0 + issued, issued);

  for (int i = 0; i < n_mine; ++i) {
    const int it = it0 + i, stage = i % kSelStages;
    const int unit = it / p.items_per_unit, local = it % p.items_per_unit;
    if (tid == 0 && !mbar_wait_bounded(&sm.full[stage], (i / kSelStages) & 1, kWaitLimit)) {
      atomicOr(p.status, HYB_STATUS_TIMEOUT);
      sm.abort = 1;
    }
    __syncthreads();  // the stage's data (or the abort flag) is visible to all
    if (sm.abort) break;
    if (local < p.score_items)
      score_item<D>(p, sm.st[stage], unit, local);
    else
      lin_item<D>(p, sm.st[stage], unit, local - p.score_items);
    __syncthreads();  // the stage is consumed
    if (tid == 0 && issued < n_mine) {
      issue_item<D>(p, sm, it0 + issued, issued % kSelStages);
      ++issued;
    }
  }
  if (sm.abort && tid == 0) {
    // do not leave while copies into this CTA's ring may be in flight
    for (int j = issued - 1; j >= 0 && j >= issued - kSelStages; --j)
      mbar_wait_bounded(&sm.full[j % kSelStages], (j / kSelStages) & 1, kWaitLimit);
  }
}

}  // namespace

size_t select_smem_bytes(int D) {
  return (D == 128 ? sizeof(SelectSmem<128>) : sizeof(SelectSmem<64>)) + 128;
}

cudaError_t prepare_select(int D) {
  const int smem = (int)select_smem_bytes(D);
  const void* f = D == 128 ? (const void*)select_kernel<128> : (const void*)select_kernel<64>;
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // the same carveout as the attention kernels, so that SMs need no
  // reconfiguration between the launches of a decode
  return cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
}

cudaError_t launch_select(const SelectParams& p, int D, int grid, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSelectThreads);
  cfg.dynamicSmemBytes = select_smem_bytes(D);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (D == 128) return cudaLaunchKernelEx(&cfg, select_kernel<128>, p);
  return cudaLaunchKernelEx(&cfg, select_kernel<64>, p);
}

}  // namespace hyb
