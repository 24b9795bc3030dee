// Exact attention over the sinks, the window and the top-k selected blocks,
// the selected blocks' (1 + s) subtraction terms, and the merge under one
// shared normaliser -- the second launch of a decode step.
//
// Work: each unit (batch row, KV head) owns a fixed list of <= 64-token chunks
// of its exact set X: sink pieces, window pieces, then ceil(Bk/64) pieces per
// selected block.  A unit's chunks are dealt to `splits` CTAs, CTA part p taking
// chunks p, p + splits, p + 2*splits, ... (split-K), so every CTA meets its
// window chunks first and its selected chunks last.  The kernel starts beside
// the select kernel (one CTA per SM next to its two) and streams the window
// while the block scores are computed; a CTA waits for the select grid only
// when its next chunk to load is a selected one.  Then warp 0 selects the
// unit's top_k blocks from the scores itself (every CTA of the unit derives the
// same selection; no hand-off between CTAs), while the other warps work on the
// chunks already loaded.  Each CTA writes one partial record; the last CTA of
// a unit to finish (atomic ticket, no spinning) merges the unit's records with
// the global linear term.
//
// Top-k (ties to the lower block index, ascending output, "SPLA: Block Sparse
// Plus Linear Attention for Long Context Modeling", "Principled Block Selection
// via Taylor Expansion"): over order-preserving integer keys of the scores, the
// k-th largest key is the largest value v with count(key >= v) >= k, found bit
// by bit below the common prefix of the smallest and largest key (one warp-wide
// count per bit), then an index-ordered ballot compaction takes every larger
// key and the lowest-index keys equal to it.
//
// CTA: 4 warps.  A 3-stage shared-memory ring is filled with TMA tensor loads
// (cp.async.bulk.tensor, 128-byte swizzle, no multicast): a full 64-token chunk
// as one 64-row box per tensor, a ragged chunk (sinks, the window's tail, a
// partial block) as the 16-row boxes it touches.  After the 4 warps have
// consumed chunk j (CTA barrier) thread 0 refills the stage with chunk j + 3.
// Warp w handles tokens [16w, 16w + 16) of a chunk.
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
// the same pass over each K/V tile ("SPLA", Abstract: residual = global -
// selected; "SLAKE", Abstract: first-order Taylor exp(s) ~ 1 + s).
//
// Merge of a unit (per query head, base-2 exponent m of the exact part):
//   o = (N_ex + 2^{-m} (N_glob - N_sel)) / (D_ex + 2^{-m} (D_glob - D_sel)),
// evaluated as the equal form (N_ex 2^m + ...)/(D_ex 2^m + ...) when m < 0.
// A decode that also appends writes the new token at row T (no kernel of the
// decode reads that row).
//
// Launch chaining (programmatic dependent launch): the select kernel lets this
// grid start at once; it lets the next decode's select kernel launch at its own
// start -- that kernel waits for this grid before touching memory.
#include "hyb_device.cuh"
#include "hyb_internal.h"

namespace hyb {

namespace {

constexpr uint32_t kFull = 0xffffffffu;

struct KVMaps {  // the same KV caches seen with 64-row and 16-row TMA boxes
  CUtensorMap k64, v64, k16, v16;
};

template <int D>
struct AttendSmem {
  static constexpr int kTileBytes = kTile * D * 2;  // one of K or V for 64 tokens
  static constexpr int kBoxBytes = kBoxRows * D * 2;
  uint8_t kv[kStages][2][kTileBytes];               // 1024-byte aligned (base aligned)
  float wpart[2][partial_floats(D)];                // combine slots (contiguous after kv: the
                                                    // merge stages partial records over both)
  float mscr[16];                                   // merge: per-head max, D_ex, D_sel
  float fscr[4 * 64];                               // merge: per-slot, per-head rescale factors
  uint64_t full[kStages];
  uint64_t merge_bar;
  int4 desc[kStages];                               // start, len, is_sel, unit
  int32_t sel_cache[kSelCache];                     // the unit's selection (state 1)
  int sel_state;    // 0 unknown, 1 in sel_cache, 2 in a global row (sel_row), 3 every block
  const int32_t* sel_row;
  int waited;       // thread 0 has waited for the select grid
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

__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// ---------------------------------------------------------------- top-k
constexpr int kKeysPerLane = 16;  // register-resident keys of the fast path (nb <= 512)

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Index-ordered compaction: take every key above tau and the first need_eq
// keys equal to it; dst[0, k) ascending (and the optional copy).
template <class KeyFn>
__device__ __forceinline__ void topk_emit(int nb, uint32_t tau, uint32_t need_eq, KeyFn key, int32_t* dst,
                                          int32_t* copy) {
  const int lane = threadIdx.x & 31;
  uint32_t taken = 0u, eq_seen = 0u;
  for (int base = 0; base < nb; base += 32) {
    const int j = base + lane;
    const uint32_t u = j < nb ? key(j) : 0u;
    const bool gt = j < nb && u > tau;
    const bool eq = j < nb && u == tau;
    const uint32_t beq = __ballot_sync(kFull, eq);
    const uint32_t rank = eq_seen + __popc(beq & lanemask_lt());
    const bool take = gt || (eq && rank < need_eq);
    const uint32_t bt = __ballot_sync(kFull, take);
    if (take) {
      const uint32_t pos = taken + __popc(bt & lanemask_lt());
      dst[pos] = j;
      if (copy) copy[pos] = j;
    }
    taken += __popc(bt);
    eq_seen += __popc(beq);
  }
}

// The k < nb largest of scores[0, nb) by one warp; writes dst[0, k) ascending
// (and copy[0, k) when given).  Keys live in registers when nb <= 32 *
// kKeysPerLane, else in `kbuf` (kbuf_words shared words) when they fit, else
// they are re-read from L2 for every count.  Returns whether a score was NaN.
__device__ bool topk_warp(const float* sc, int nb, int k, int32_t* dst, int32_t* copy, uint32_t* kbuf,
                          int kbuf_words) {
  const int lane = threadIdx.x & 31;
  bool nan = false;
  if (nb <= 32 * kKeysPerLane) {
    uint32_t kr[kKeysPerLane];
    float f[kKeysPerLane];
#pragma unroll
    for (int i = 0; i < kKeysPerLane; ++i) {  // all loads in flight at once
      const int j = lane + 32 * i;
      f[i] = j < nb ? __ldcg(sc + j) : 0.f;
    }
    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int i = 0; i < kKeysPerLane; ++i) {
      const bool v = lane + 32 * i < nb;
      nan |= v && (f[i] != f[i]);
      kr[i] = v ? float_key(f[i]) : 0u;  // 0 is below every key a count can reach
      if (v) {
        kmin = min(kmin, kr[i]);
        kmax = max(kmax, kr[i]);
      }
    }
    kmin = __reduce_min_sync(kFull, kmin);
    kmax = __reduce_max_sync(kFull, kmax);
    const int free_bits = 32 - __clz(kmin ^ kmax);  // bits below the common prefix
    uint32_t tau = free_bits == 32 ? 0u : (kmax & ~((1u << free_bits) - 1u));
    for (int bit = free_bits - 1; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      uint32_t c = 0u;
#pragma unroll
      for (int i = 0; i < kKeysPerLane; ++i) c += (kr[i] >= cand) ? 1u : 0u;
      if (__reduce_add_sync(kFull, c) >= (uint32_t)k) tau = cand;
    }
    uint32_t gt = 0u;
#pragma unroll
    for (int i = 0; i < kKeysPerLane; ++i) gt += (kr[i] > tau) ? 1u : 0u;
    gt = __reduce_add_sync(kFull, gt);
    // the keys of row i are blocks 32i .. 32i+31: index order is row order
    uint32_t taken = 0u, eq_seen = 0u;
    const uint32_t need_eq = (uint32_t)k - gt;
#pragma unroll
    for (int i = 0; i < kKeysPerLane; ++i) {
      if (32 * i < nb) {
        const int j = 32 * i + lane;
        const bool gtb = j < nb && kr[i] > tau;
        const bool eqb = j < nb && kr[i] == tau;
        const uint32_t beq = __ballot_sync(kFull, eqb);
        const uint32_t rank = eq_seen + __popc(beq & lanemask_lt());
        const bool take = gtb || (eqb && rank < need_eq);
        const uint32_t bt = __ballot_sync(kFull, take);
        if (take) {
          const uint32_t pos = taken + __popc(bt & lanemask_lt());
          dst[pos] = j;
          if (copy) copy[pos] = j;
        }
        taken += __popc(bt);
        eq_seen += __popc(beq);
      }
    }
  } else {
    const bool staged = nb <= kbuf_words;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int j0 = 0; j0 < nb; j0 += 32 * kKeysPerLane) {  // batches of loads in flight
      float f[kKeysPerLane];
#pragma unroll
      for (int i = 0; i < kKeysPerLane; ++i) {
        const int j = j0 + lane + 32 * i;
        f[i] = j < nb ? __ldcg(sc + j) : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kKeysPerLane; ++i) {
        const int j = j0 + lane + 32 * i;
        if (j < nb) {
          nan |= (f[i] != f[i]);
          const uint32_t u = float_key(f[i]);
          if (staged) kbuf[j] = u;
          kmin = min(kmin, u);
          kmax = max(kmax, u);
        }
      }
    }
    __syncwarp();
    kmin = __reduce_min_sync(kFull, kmin);
    kmax = __reduce_max_sync(kFull, kmax);
    auto key = [&](int j) -> uint32_t { return staged ? kbuf[j] : float_key(__ldcg(sc + j)); };
    const int free_bits = 32 - __clz(kmin ^ kmax);
    uint32_t tau = free_bits == 32 ? 0u : (kmax & ~((1u << free_bits) - 1u));
    for (int bit = free_bits - 1; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      uint32_t c = 0u;
      for (int j = lane; j < nb; j += 32) c += (key(j) >= cand) ? 1u : 0u;
      if (__reduce_add_sync(kFull, c) >= (uint32_t)k) tau = cand;
    }
    uint32_t gt = 0u;
    for (int j = lane; j < nb; j += 32) gt += (key(j) > tau) ? 1u : 0u;
    gt = __reduce_add_sync(kFull, gt);
    topk_emit(nb, tau, (uint32_t)k - gt, key, dst, copy);
  }
  return __any_sync(kFull, nan);
}

// Make the unit's selection known to this CTA (warp 0, all lanes): the
// caller's row, every block (k >= nb) or none (k == 0), or the top-k of the
// select kernel's scores.  The writer CTA also fills the caller's copy.
template <int D>
__device__ void resolve_selection(const AttendParams& p, AttendSmem<D>& sm, int unit, bool writer) {
  const int lane = threadIdx.x & 31;
  int32_t* copy = (p.sel_out != nullptr && writer) ? p.sel_out + (int64_t)unit * p.top_k : nullptr;
  if (p.sel_given != nullptr) {
    const int32_t* row = p.sel_given + (int64_t)unit * p.top_k;
    if (p.top_k <= kSelCache) {
      for (int j = lane; j < p.top_k; j += 32) sm.sel_cache[j] = __ldg(row + j);
      if (lane == 0) sm.sel_state = 1;
    } else if (lane == 0) {
      sm.sel_row = row;
      sm.sel_state = 2;
    }
  } else if (p.k_eff == 0 || p.k_eff >= p.nb) {  // no block, or every block: no scores needed
    if (copy)
      for (int j = lane; j < p.top_k; j += 32) copy[j] = (p.k_eff > 0 && j < p.nb) ? j : -1;
    if (lane == 0) sm.sel_state = 3;
  } else {
    if (lane == 0 && !sm.waited) {  // the scores come from the select grid
      pdl_wait_primary();
      sm.waited = 1;
    }
    __syncwarp();
    {
      int32_t* dst = p.k_eff <= kSelCache ? sm.sel_cache : p.sel + (int64_t)unit * p.top_k;
      // the combine slots are idle until the main loop ends: they hold the keys
      uint32_t* kbuf = reinterpret_cast<uint32_t*>(&sm.wpart[0][0]);
      const int kbuf_words = (int)(sizeof(sm.wpart) / sizeof(uint32_t));
      const bool nan = topk_warp(p.scores + (int64_t)unit * p.max_blocks, p.nb, p.k_eff, dst, copy, kbuf,
                                 kbuf_words);
      if (copy)
        for (int j = p.k_eff + lane; j < p.top_k; j += 32) copy[j] = -1;
      if (lane == 0) {
        if (nan) atomicOr(p.status, HYB_STATUS_NAN_SCORE);
        sm.sel_row = dst;
        sm.sel_state = p.k_eff <= kSelCache ? 1 : 2;
      }
    }
  }
  __syncwarp();
}

// Merge the `nslot` partial records [slot0, slot0 + nslot) of `unit` with the
// global linear term and write the unit's output.  All threads of the CTA, after
// its own chunks are done (the stage buffers are free).  The unit's records are
// contiguous in the workspace: thread 0 pulls up to kMergeSlots of them into
// shared memory with one bulk copy, then the reductions run from shared memory.
template <int D>
__device__ void merge_unit(const AttendParams& p, int unit, int64_t slot0, int nslot, int tid, AttendSmem<D>& sm) {
  constexpr int PF = partial_floats(D);
  constexpr int CAP = (int)((sizeof(sm.kv) + sizeof(sm.wpart)) / (PF * sizeof(float)));
  static_assert(CAP >= 1 && CAP <= 64, "merge staging capacity");
  constexpr int NV = 2 * D;  // float4 columns of [acc | nsel]
  constexpr int VPT = (NV + kAttendThreads - 1) / kAttendThreads;
  float* rec = reinterpret_cast<float*>(&sm.kv[0][0][0]);  // staged records, then the column sums
  float* s_M = sm.mscr;
  float* s_Dex = sm.mscr + 4;
  float* s_Dsel = sm.mscr + 8;
  const int warp = tid >> 5, lane = tid & 31;
  const float* base = p.partials + slot0 * PF;
  if (tid == 0 && !sm.waited) {  // the linear term comes from the select grid
    pdl_wait_primary();
    sm.waited = 1;
  }
  __syncthreads();
  {                    // warp h: max of head h over all slots
    float mx = -INFINITY;
    for (int k = lane; k < nslot; k += 32) mx = fmaxf(mx, __ldcg(base + (int64_t)k * PF + warp));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    if (lane == 0) s_M[warp] = (mx == -INFINITY) ? 0.f : mx;
  }
  float4 vacc[VPT];
#pragma unroll
  for (int u = 0; u < VPT; ++u) vacc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  float dex = 0.f, dsel = 0.f;
  for (int kb = 0, batch = 0; kb < nslot; kb += CAP, ++batch) {
    const int nb = min(CAP, nslot - kb);
    __syncthreads();  // previous batch consumed; s_M visible
    if (tid == 0) {
      // the records were written by other CTAs' generic-proxy stores (ordered by
      // the ticket); order them before this async-proxy read
      asm volatile("fence.proxy.async.global;" ::: "memory");
      const uint32_t bytes = (uint32_t)(nb * PF * sizeof(float));
      mbar_arrive_expect_tx(&sm.merge_bar, bytes);
      bulk_load(smem_u32(rec), base + (int64_t)kb * PF, bytes, &sm.merge_bar);
    }
    if (!mbar_wait_bounded(&sm.merge_bar, batch & 1, kWaitLimit))
      atomicOr(p.status, HYB_STATUS_TIMEOUT);  // keep the barrier sequence; the output is flagged
    for (int e = tid; e < 4 * nb; e += kAttendThreads) {
      const float m = rec[(e >> 2) * PF + (e & 3)];
      sm.fscr[e] = (m == -INFINITY) ? 0.f : exp2f(m - s_M[e & 3]);
    }
    __syncthreads();
    for (int k = lane; k < nb; k += 32) {  // warp h accumulates head h
      dex += rec[k * PF + 4 + warp] * sm.fscr[4 * k + warp];
      dsel += rec[k * PF + 8 + warp];
    }
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
      const int v = tid + u * kAttendThreads;
      if (v < NV) {
        const int vh = (4 * v) / D;  // head of an acc column (v < D)
        for (int k = 0; k < nb; ++k) {
          const float4 x = *reinterpret_cast<const float4*>(rec + k * PF + 16 + 4 * v);
          const float f = (v < D) ? sm.fscr[4 * k + vh] : 1.f;
          vacc[u].x += x.x * f;
          vacc[u].y += x.y * f;
          vacc[u].z += x.z * f;
          vacc[u].w += x.w * f;
        }
      }
    }
  }
  __syncthreads();  // the staging area is free again
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    dex += __shfl_xor_sync(kFull, dex, o);
    dsel += __shfl_xor_sync(kFull, dsel, o);
  }
  if (lane == 0) {
    s_Dex[warp] = dex;
    s_Dsel[warp] = dsel;
  }
  float* s_vec = rec;  // [8 D] column sums
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int v = tid + u * kAttendThreads;
    if (v < NV) *reinterpret_cast<float4*>(s_vec + 4 * v) = vacc[u];
  }
  __syncthreads();
  const int G = p.G;
  const float* lin = p.lin + (int64_t)unit * p.lin_items * G * (D + 1);  // [lin_items][G][D + 1]
  // every load of the linear term first (independent, in flight together), then
  // the arithmetic and the stores
  constexpr int EPT = kMaxGroup * D / kAttendThreads;  // output elements per thread
  float Ng[EPT], Dg[EPT];
#pragma unroll
  for (int r = 0; r < EPT; ++r) {
    const int e = tid + r * kAttendThreads;
    Ng[r] = 0.f;
    Dg[r] = 0.f;
    if (e < G * D) {
      const int i = e / D, d = e % D;
      for (int g = 0; g < p.lin_items; ++g) Ng[r] += __ldcg(lin + ((int64_t)g * G + i) * (D + 1) + d);
      Dg[r] = __ldcg(lin + (int64_t)i * (D + 1) + D);
    }
  }
  uint32_t flags = 0u;
#pragma unroll
  for (int r = 0; r < EPT; ++r) {
    const int e = tid + r * kAttendThreads;
    if (e < G * D) {
      const int i = e / D, d = e % D;
      const float Ms = s_M[i];
      const float Nex = s_vec[i * D + d], Nsel = s_vec[4 * D + i * D + d];
      const float Dex = s_Dex[i], Dsel = s_Dsel[i];
      float num, den;
      if (Ms >= 0.f) {
        const float f = exp2f(-Ms);
        num = Nex + f * (Ng[r] - Nsel);
        den = Dex + f * (Dg[r] - Dsel);
      } else {
        const float f = exp2f(Ms);
        num = Nex * f + (Ng[r] - Nsel);
        den = Dex * f + (Dg[r] - Dsel);
      }
      const float o = num / den;
      p.out[((int64_t)unit * G + i) * D + d] = o;
      if (!(den > 0.f)) flags |= HYB_STATUS_DENOMINATOR;
      if (!isfinite(o)) flags |= HYB_STATUS_NONFINITE;
    }
  }
  if (flags) atomicOr(p.status, flags);
}

// Hand local chunk j (unit chunk index ci) to stage j % kStages: write its
// descriptor and start the TMA loads of its K and V rows (rows past the chunk
// end inside a box are read too and ignored).  Thread 0.
template <int D>
__device__ void issue_chunk(const KVMaps* tm, const AttendParams& p, AttendSmem<D>& sm, int unit, int ci, int j) {
  using S = AttendSmem<D>;
  const int stage = j % kStages;
  int start = 0, len = 0, is_sel = 0;
  if (ci < p.n_sink_chunks) {
    start = ci * kTile;
    len = min(kTile, p.sink_len - start);
  } else if (ci < p.n_sink_chunks + p.n_win_chunks) {
    start = p.win_start + (ci - p.n_sink_chunks) * kTile;
    len = min(kTile, p.T - start);
  } else {  // the selection is resolved before a selected chunk is issued
    const int s = ci - p.n_sink_chunks - p.n_win_chunks;
    const int slot = s / p.chunks_per_block, piece = s % p.chunks_per_block;
    is_sel = 1;
    int jb = -1;
    if (slot < p.k_eff) {
      const int st = sm.sel_state;
      jb = st == 3 ? slot : st == 1 ? sm.sel_cache[slot] : __ldcg(sm.sel_row + slot);
    }
    if (jb >= 0 && jb < p.nb) {
      const int bs = p.S + jb * p.Bk;
      const int be = min(bs + p.Bk, p.ev_end);
      start = bs + piece * kTile;
      len = max(0, min(kTile, be - start));
    } else if (jb != -1) {
      atomicOr(p.status, HYB_STATUS_BAD_SELECTION);
    }
  }
  sm.desc[stage] = make_int4(start, len, is_sel, unit);
  if (len > 0) {
    const int row = (int)((int64_t)unit * p.cap + start);
    const uint32_t kdst = smem_u32(sm.kv[stage][0]);
    const uint32_t vdst = smem_u32(sm.kv[stage][1]);
    if (len == kTile) {  // full chunk: one 64-row box per tensor
      mbar_arrive_expect_tx(&sm.full[stage], (uint32_t)(2 * S::kTileBytes));
      tma_load_3d(kdst, &tm->k64, 0, 0, row, &sm.full[stage]);
      tma_load_3d(vdst, &tm->v64, 0, 0, row, &sm.full[stage]);
    } else {             // ragged chunk: only the 16-row boxes it touches
      const int nbox = (len + kBoxRows - 1) / kBoxRows;
      mbar_arrive_expect_tx(&sm.full[stage], (uint32_t)(nbox * S::kBoxBytes * 2));
      for (int bx = 0; bx < nbox; ++bx) {
        tma_load_3d(kdst + bx * S::kBoxBytes, &tm->k16, 0, 0, row + bx * kBoxRows, &sm.full[stage]);
        tma_load_3d(vdst + bx * S::kBoxBytes, &tm->v16, 0, 0, row + bx * kBoxRows, &sm.full[stage]);
      }
    }
  } else {
    mbar_arrive(&sm.full[stage]);
  }
}

template <int D>
__global__ void __maxnreg__(kAttendMaxRegs)
    attend_kernel(const __grid_constant__ KVMaps tm, const AttendParams p) {
  constexpr int PF = partial_floats(D);
  constexpr int NT8 = D / 8;   // 8-column tiles of the head dimension
  constexpr int KS = D / 16;   // k-steps of the QK product
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned (the 128-byte swizzle repeats every 1024 bytes); offsetting
  // the shared array keeps every access through `sm` in the shared space
  AttendSmem<D>& sm = *reinterpret_cast<AttendSmem<D>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;

  if (tid == 0) {
    tma_prefetch_desc(&tm.k64);
    tma_prefetch_desc(&tm.v64);
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[s], 1);
    mbar_init(&sm.merge_bar, 1);
    sm.sel_state = 0;
    sm.waited = 0;
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // the next decode's select kernel may be scheduled; it waits for this grid
  pdl_allow_dependents();
  const int unit = cta / p.splits, part = cta % p.splits;
  const int n_local = (p.chunks_per_unit - part + p.splits - 1) / p.splits;  // chunks part + j*splits
  const int n_pre = p.n_sink_chunks + p.n_win_chunks;                       // selection-free chunks
  const int j_sel = part < n_pre ? (n_pre - part + p.splits - 1) / p.splits : 0;  // first selected local chunk
  // the CTA that owns the unit's first selected chunk fills the caller's copy
  // of the selection (part 0 when there is none)
  const bool writer = part == (p.chunks_per_unit > n_pre ? n_pre % p.splits : 0);

  if (warp == 0 && ((j_sel == 0 && n_local > 0) || (writer && p.chunks_per_unit == n_pre)))
    resolve_selection<D>(p, sm, unit, writer);
  int next_issue = 0;  // thread 0: next local chunk to issue
  if (tid == 0)
    for (; next_issue < n_local && next_issue < kStages && (next_issue < j_sel || sm.sel_state != 0); ++next_issue)
      issue_chunk<D>(&tm, p, sm, unit, part + next_issue * p.splits, next_issue);
  if (p.k_new != nullptr && part == 0 && tid < D / 4) {
    // the decode's appended token: row T of the caches (16 bytes per thread)
    const bool is_v = tid >= D / 8;
    const int e = (tid % (D / 8)) * 8;
    const __nv_bfloat16* src = (is_v ? p.v_new : p.k_new) + (int64_t)unit * D + e;
    __nv_bfloat16* dst = (is_v ? p.v_cache : p.k_cache) + ((int64_t)unit * p.cap + p.T) * D + e;
    *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
  }

  const int g = lane >> 2, tig = lane & 3;
  const bool p_lane = g < 4;  // rows 0-3: softmax part; rows 4-7: Taylor part
  const int head = g & 3;
  const bool head_ok = head < p.G;
  const int r0 = warp * 16;
  const int mi = lane >> 3, rr = lane & 7;

  uint32_t qa[KS][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(p.q + ((int64_t)unit * p.G + (head_ok ? head : 0)) * D);
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

  for (int j = 0; j < n_local; ++j) {
    const int stage = j % kStages;
    bool ok = !*(volatile int*)&sm.abort_flag;
    if (ok && !mbar_wait_bounded(&sm.full[stage], (j / kStages) & 1, kWaitLimit)) {
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
    __syncthreads();  // every warp is done with this stage
    if (warp == 0) {
      // the next chunk to load may be the first selected one: warp 0 resolves
      // the selection now, while warps 1-3 go on with the chunks already loaded
      const int ni = __shfl_sync(kFull, next_issue, 0);
      if (ni < n_local && ni >= j_sel && sm.sel_state == 0) resolve_selection<D>(p, sm, unit, writer);
      if (lane == 0)
        for (; next_issue < n_local && next_issue <= j + kStages && !*(volatile int*)&sm.abort_flag; ++next_issue)
          issue_chunk<D>(&tm, p, sm, unit, part + next_issue * p.splits, next_issue);
    }
  }

  // ---- combine the 4 warps' partials in registers (a tree through two shared
  //      slots: warps 2, 3 -> 0, 1, then warp 1 -> 0); warp 0 writes the record
  float l = l_run + __shfl_xor_sync(kFull, l_run, 1);
  l += __shfl_xor_sync(kFull, l, 2);
  float ds = dsel_run + __shfl_xor_sync(kFull, dsel_run, 1);
  ds += __shfl_xor_sync(kFull, ds, 2);
  const int voff = (p_lane ? 0 : 4 * D) + head * D;
  auto emit = [&](float* wp) {  // write this warp's partial (hi + lo rows summed)
    if (tig == 0) {
      if (p_lane) {
        wp[head] = m_run;
        wp[4 + head] = l;
      } else {
        wp[8 + head] = ds;
      }
    }
    float* dst = wp + 16 + voff;
#pragma unroll
    for (int n = 0; n < NT8; ++n)
      *reinterpret_cast<float2*>(dst + n * 8 + 2 * tig) = make_float2(O[n][0] + O[n][2], O[n][1] + O[n][3]);
  };
  auto absorb = [&](const float* wp) {  // fold another warp's partial into this one
    const float mp = wp[head], lp = wp[4 + head], dsp = wp[8 + head];
    float fa = 1.f, fb = 1.f;
    if (p_lane) {
      const float M = fmaxf(m_run, mp);
      fa = (m_run == -INFINITY) ? 0.f : exp2f(m_run - M);
      fb = (mp == -INFINITY) ? 0.f : exp2f(mp - M);
      l = l * fa + lp * fb;
      m_run = M;
    } else {
      ds += dsp;
    }
    const float* src = wp + 16 + voff;
#pragma unroll
    for (int n = 0; n < NT8; ++n) {
      const float2 y = *reinterpret_cast<const float2*>(src + n * 8 + 2 * tig);
      O[n][0] = (O[n][0] + O[n][2]) * fa + y.x * fb;
      O[n][1] = (O[n][1] + O[n][3]) * fa + y.y * fb;
      O[n][2] = O[n][3] = 0.f;
    }
  };
  if (warp >= 2) emit(sm.wpart[warp - 2]);
  __syncthreads();
  if (warp < 2) absorb(sm.wpart[warp]);
  __syncthreads();
  if (warp == 1) emit(sm.wpart[0]);
  __syncthreads();
  if (warp == 0) {
    absorb(sm.wpart[0]);
    emit(p.partials + (int64_t)cta * PF);
    __syncwarp();
    if (lane == 0) {
      __threadfence();  // release the partial record before the ticket
      const uint32_t prev = atomicAdd(&p.tickets[unit], 1u);
      sm.last_flag = (prev == (uint32_t)p.splits - 1u);
      __threadfence();
    }
  }
  __syncthreads();
  if (sm.last_flag) {
    merge_unit<D>(p, unit, (int64_t)unit * p.splits, p.splits, tid, sm);
    if (tid == 0) p.tickets[unit] = 0u;  // ready for the next decode
  }
  if (tid == 0 && *(volatile int*)&sm.abort_flag) {
    // do not leave while copies into this CTA's shared memory may be in flight
    for (int j = next_issue - 1; j >= 0 && j >= next_issue - kStages; --j)
      mbar_wait_bounded(&sm.full[j % kStages], (j / kStages) & 1, kWaitLimit);
  }
  // this grid completes only after the select grid (its scores and linear term
  // are read above; a CTA that needed neither still waits, in one thread)
  if (tid == 0 && !sm.waited) pdl_wait_primary();
}

}  // namespace

size_t attend_smem_bytes(int D) {
  return (D == 128 ? sizeof(AttendSmem<128>) : sizeof(AttendSmem<64>)) + 1024;
}

cudaError_t prepare_attend(int D) {
  const int smem = (int)attend_smem_bytes(D);
  const void* f = D == 128 ? (const void*)attend_kernel<128> : (const void*)attend_kernel<64>;
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
}

cudaError_t launch_attend(const CUtensorMap* maps, const AttendParams& p, int D, cudaStream_t s) {
  KVMaps tm;
  tm.k64 = maps[0];
  tm.v64 = maps[1];
  tm.k16 = maps[2];
  tm.v16 = maps[3];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(kAttendThreads);
  cfg.dynamicSmemBytes = attend_smem_bytes(D);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (D == 128) return cudaLaunchKernelEx(&cfg, attend_kernel<128>, tm, p);
  return cudaLaunchKernelEx(&cfg, attend_kernel<64>, tm, p);
}

}  // namespace hyb
