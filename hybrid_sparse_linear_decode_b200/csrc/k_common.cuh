// Device code shared by the decode kernels (k_fused.cu, k_multi.cu): the warp
// roles' sizes, thread-block-cluster and distributed-shared-memory helpers, the
// 128-byte-swizzle addressing of the K/V tiles, bf16 fragment packing, vector
// loads, and the block-score selections (radix over all statistics threads, one
// warp's bound-and-rank, the streaming top-32 of each statistics warp).  No
// arithmetic of the attention itself lives here.
#pragma once

#include "hyb_device.cuh"
#include "hyb_internal.h"

namespace hyb {
namespace {

constexpr uint32_t kFull = 0xffffffffu;
constexpr int kFThreads = 384;
constexpr int kAttnWarps = 8;       // attention warps: roles 0-7 (4 pairs)
constexpr int kAttnThreads = 32 * kAttnWarps;
constexpr int kAuxWarps = 3;        // statistics warps: roles 8-10
constexpr int kAuxThreads = 32 * kAuxWarps;
constexpr int kConsumerThreads = kAttnThreads + kAuxThreads;  // roles 0-10
static_assert(kConsumerThreads >= 2 * 128, "one thread per channel of the pending K and V rows");
constexpr int kProducerWarp = kAttnWarps + kAuxWarps;         // role 11
// every item's empty-barrier phase takes kEmptyCount arrivals: kEmptyPerAuxWarp
// from each statistics warp, or kEmptyPerAttnWarp from each attention warp
template <int D>
constexpr int kAuxCols = (D + kAuxThreads - 1) / kAuxThreads;  // columns per statistics thread
constexpr int kEmptyCount = 24, kEmptyPerAuxWarp = 8, kEmptyPerAttnWarp = 3;
constexpr int kBarAttn = 1, kBarAux = 2, kBarConsumers = 3, kBarPair0 = 4;   // named barriers

// ---------------------------------------------------------------- cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_rank(uint32_t local_smem, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_smem), "r"(rank));
  return r;
}
__device__ __forceinline__ void remote_arrive(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr) : "memory");
}
__device__ __forceinline__ bool try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait on a barrier that other CTAs of the cluster arrive on (polled
// like mbar_wait_bounded)
__device__ __forceinline__ bool wait_cluster_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (try_wait_cluster(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}
// the two halves of a cluster barrier that orders no memory, for work between them
__device__ __forceinline__ void cluster_arrive_relaxed() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait;" ::: "memory"); }
// Stores into another CTA's shared memory (cluster shared addresses) that
// complete their bytes on the barrier at cluster shared address bar in that CTA.
__device__ __forceinline__ void st_async_v2(uint32_t dst, float x, float y, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(dst), "f"(x),
               "f"(y), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void st_async_v4(uint32_t dst, float x, float y, float z, float w, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(dst),
               "f"(x), "f"(y), "f"(z), "f"(w), "r"(bar)
               : "memory");
}
// 16 bytes to / from a shared-memory address
__device__ __forceinline__ void sts_u4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void lds_u4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Copy `bytes` (a multiple of 16) of this CTA's shared memory at src to the
// cluster shared address dst, completing that many transactions on the barrier
// at cluster shared address bar (in the destination CTA).
__device__ __forceinline__ void bulk_push(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "r"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// This thread's index in role order: role r is hardware warp r.  Warp w runs on
// sub-partition w % 4: each sub-partition runs two attention warps (0-7; the two
// warps of a pair on different sub-partitions) and one statistics warp (8-10)
// or the producer (11); the attention warps idle while the score items stream,
// which is when the statistics warps are busiest.
__device__ __forceinline__ int role_tid() { return (int)threadIdx.x; }
__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

struct KVMaps {  // the same KV caches seen with 64-row and 16-row TMA boxes
  CUtensorMap k64, v64, k16, v16;
};

// Byte offset of (row t, 16-byte chunk C) in a tile written by TMA with the
// 128-byte swizzle: 128-byte line L = t*(D/64) + C/8, chunk slot (C%8) ^ (L%8).
template <int D>
__device__ __forceinline__ uint32_t swz(int t, int C) {
  const int L = t * (D / 64) + (C >> 3);
  return (uint32_t)(L * 128 + (((C & 7) ^ (L & 7)) << 4));
}

// Transpose of an 8x8 matrix of 16-bit elements held in the warp (thread (g,
// tig) holds row g, columns 2tig and 2tig+1).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Blocks [b0, b1) of rank r: equal shares rounded up to 4 blocks, so that every
// share's scores start on a 16-byte boundary (they travel by bulk copy).
__device__ __forceinline__ void block_share(int nb, int C, int r, int& b0, int& b1) {
  const int per = ((nb + C - 1) / C + 3) & ~3;
  b0 = min(nb, r * per);
  b1 = min(nb, b0 + per);
}

template <int CPL>
__device__ __forceinline__ void load_bf16(const __nv_bfloat16* src, float (&f)[CPL]) {
  if constexpr (CPL == 4) {
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(src));
    f[0] = bf16_lo(raw.x); f[1] = bf16_hi(raw.x); f[2] = bf16_lo(raw.y); f[3] = bf16_hi(raw.y);
  } else {
    const uint32_t raw = __ldg(reinterpret_cast<const uint32_t*>(src));
    f[0] = bf16_lo(raw); f[1] = bf16_hi(raw);
  }
}

template <int CPL>
__device__ __forceinline__ void lds_vec(const float* src, float (&f)[CPL]) {
  if constexpr (CPL == 4) {
    const float4 v = *reinterpret_cast<const float4*>(src);
    f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
  } else {
    const float2 v = *reinterpret_cast<const float2*>(src);
    f[0] = v.x; f[1] = v.y;
  }
}

template <int CPL>
__device__ __forceinline__ void sts_vec(float* dst, const float (&f)[CPL]) {
  if constexpr (CPL == 4) {
    *reinterpret_cast<float4*>(dst) = make_float4(f[0], f[1], f[2], f[3]);
  } else {
    *reinterpret_cast<float2*>(dst) = make_float2(f[0], f[1]);
  }
}

// ---------------------------------------------------------------- top-k
// Exclusive prefix sum of v over the statistics threads (named barrier 2);
// returns the sum over threads before this one, and the total in *total.
__device__ __forceinline__ uint32_t aux_scan(uint32_t v, uint32_t* scratch, uint32_t* total) {
  const int a = role_tid() - kAttnThreads, aw = a >> 5, lane = a & 31;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) scratch[aw] = incl;
  named_sync(kBarAux, kAuxThreads);
  uint32_t before = 0;
  for (int w = 0; w < aw; ++w) before += scratch[w];
  uint32_t tot = 0;
  for (int w = 0; w < kAuxWarps; ++w) tot += scratch[w];
  *total = tot;
  named_sync(kBarAux, kAuxThreads);
  return before + incl - v;
}

struct TopkSmem {  // the top-k's shared scratch
  uint32_t* hist;     // [256]
  uint32_t* tk;       // [8]
  uint32_t* tks;      // [2][4]
};

// Order-preserving integer key of score j (from shared memory, or from global
// memory through L2 when the unit's scores do not fit in shared memory).
__device__ __forceinline__ uint32_t score_key(const float* src, bool glob, int j) {
  return float_key(glob ? __ldcg(src + j) : src[j]);
}

// The k < nb largest of the nb scores at src by the statistics threads: an
// 8-bit radix refinement over the keys' value range (at most four histogram
// passes, usually two or three) finds the k-th largest key tau; then every key
// above tau and the lowest-index keys equal to it are taken, in block order,
// through prefix sums over contiguous ranges of blocks.  dst[0, k) ascending
// (and copy[0, k)).  Returns (in every thread) whether a score was NaN.
__device__ __forceinline__ bool aux_topk(const TopkSmem t, const float* src, bool glob, int nb, int k, int32_t* dst,
                                      int32_t* copy) {
  const int a = role_tid() - kAttnThreads, aw = a >> 5, lane = a & 31;
  uint32_t kmin = 0xffffffffu, kmax = 0u, nan = 0u;
#pragma unroll 1
  for (int j = a; j < nb; j += kAuxThreads) {
    const float f = glob ? __ldcg(src + j) : src[j];
    nan |= f != f ? 1u : 0u;
    const uint32_t u = float_key(f);
    kmin = min(kmin, u);
    kmax = max(kmax, u);
  }
  kmin = __reduce_min_sync(kFull, kmin);
  kmax = __reduce_max_sync(kFull, kmax);
  nan = __reduce_or_sync(kFull, nan);
  if (lane == 0) {
    t.tks[aw] = kmin;
    t.tks[4 + aw] = kmax;
    t.tk[4 + aw] = nan;
  }
  named_sync(kBarAux, kAuxThreads);
  uint32_t lo = t.tks[0], hi = t.tks[4];
  bool any_nan = t.tk[4] != 0u;
  for (int w = 1; w < kAuxWarps; ++w) {
    lo = min(lo, t.tks[w]);
    hi = max(hi, t.tks[4 + w]);
    any_nan |= t.tk[4 + w] != 0u;
  }
  uint32_t span = hi - lo;
  uint32_t need = (uint32_t)k;
  uint32_t tau = lo, need_eq = need;  // take u > tau, and the first need_eq keys u == tau
#pragma unroll 1
  for (int pass = 0; pass < 5; ++pass) {
    if (span == 0u) {
      tau = lo;
      need_eq = need;
      break;
    }
    const int bits = 32 - __clz(span);
    const int shift = bits > 8 ? bits - 8 : 0;  // (span >> shift) < 256
    for (int b = a; b < 256; b += kAuxThreads) t.hist[b] = 0u;
    named_sync(kBarAux, kAuxThreads);
#pragma unroll 1
    for (int j = a; j < nb; j += kAuxThreads) {
      const uint32_t d = score_key(src, glob, j) - lo;  // keys below lo wrap past span
      if (d <= span) atomicAdd(&t.hist[d >> shift], 1u);
    }
    named_sync(kBarAux, kAuxThreads);
    if (aw == 0) {  // lane l holds bins 255-8l .. 248-8l, highest first
      uint32_t cnt[8], local = 0u;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        cnt[e] = t.hist[255 - 8 * lane - e];
        local += cnt[e];
      }
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - local;
      if (excl < need && incl >= need) {
        uint32_t c = excl;
        bool found = false;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (!found && c + cnt[e] >= need) {
            t.tk[0] = 255u - 8u * lane - e;  // bin
            t.tk[1] = c;                     // keys above the bin
            t.tk[2] = cnt[e];                // keys in the bin
            found = true;
          }
          c += cnt[e];
        }
      }
    }
    named_sync(kBarAux, kAuxThreads);
    const uint32_t bin = t.tk[0], above = t.tk[1], in_bin = t.tk[2];
    named_sync(kBarAux, kAuxThreads);  // tk is rewritten next pass
    need -= above;
    const uint32_t blo = lo + (bin << shift);
    if (in_bin == need) {  // the whole bin is taken: exactly the keys >= blo
      tau = blo;
      need_eq = 0xffffffffu;
      break;
    }
    lo = blo;
    span = shift == 0 ? 0u : min(span - (bin << shift), (1u << shift) - 1u);
    tau = lo;
    need_eq = need;
  }
  // compaction: thread a owns blocks [a nb / kAuxThreads, (a+1) nb / kAuxThreads)
  const int j0 = (int)((int64_t)a * nb / kAuxThreads), j1 = (int)((int64_t)(a + 1) * nb / kAuxThreads);
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll 1
  for (int j = j0; j < j1; ++j) {
    const uint32_t u = score_key(src, glob, j);
    n_gt += u > tau ? 1u : 0u;
    n_eq += u == tau ? 1u : 0u;
  }
  uint32_t tot;
  const uint32_t eq_before = aux_scan(n_eq, t.tks, &tot);
  const uint32_t eq_take = eq_before >= need_eq ? 0u : min(n_eq, need_eq - eq_before);
  uint32_t pos = aux_scan(n_gt + eq_take, t.tks + 4, &tot);
  uint32_t eq_seen = eq_before;
#pragma unroll 1
  for (int j = j0; j < j1; ++j) {
    const uint32_t u = score_key(src, glob, j);
    bool take = u > tau;
    if (u == tau) {
      take = eq_seen < need_eq;
      ++eq_seen;
    }
    if (take && pos < (uint32_t)k) {
      dst[pos] = j;
      if (copy) copy[pos] = j;
      ++pos;
    }
  }
  return any_nan;
}

// The k-th largest (k <= 32) of the 32 lanes' values v, ties to the lower lane.
__device__ __forceinline__ uint32_t kth_lane_max(uint32_t v, int lane, int k) {
  int r = 0;
#pragma unroll
  for (int l = 0; l < 32; ++l) {
    const uint32_t o = __shfl_sync(kFull, v, l);
    r += (o > v || (o == v && l < lane)) ? 1 : 0;
  }
  return __shfl_sync(kFull, v, __ffs(__ballot_sync(kFull, r == k - 1)) - 1);
}

// The k-th largest (k <= 32) of the 64 values {v0, v1} of the 32 lanes, in the
// strict order by value, then lower lane, then v0 before v1.
__device__ __forceinline__ uint32_t kth_of_lane_pairs(uint32_t v0, uint32_t v1, int lane, int k) {
  int r0 = 0, r1 = 0;  // values ordered before (lane, v0) / before (lane, v1)
#pragma unroll 2
  for (int l = 0; l < 32; ++l) {
    const uint32_t o0 = __shfl_sync(kFull, v0, l), o1 = __shfl_sync(kFull, v1, l);
    r0 += (o0 > v0 || (o0 == v0 && l < lane)) ? 1 : 0;
    r0 += (o1 > v0 || (o1 == v0 && l < lane)) ? 1 : 0;
    r1 += (o0 > v1 || (o0 == v1 && l <= lane)) ? 1 : 0;
    r1 += (o1 > v1 || (o1 == v1 && l < lane)) ? 1 : 0;
  }
  const uint32_t b0 = __ballot_sync(kFull, r0 == k - 1), b1 = __ballot_sync(kFull, r1 == k - 1);
  return b0 ? __shfl_sync(kFull, v0, __ffs(b0) - 1) : __shfl_sync(kFull, v1, __ffs(b1) - 1);
}

// The k <= 32 largest of the nb scores in shared memory (sc) by one warp, ties
// to the lower index.  Lane l's keys are those of blocks l, l + 32, ...; at
// least k lanes hold a key (nb > k), so the k-th largest of the 32 lane maxima,
// tau, is at most the k-th largest key: every key of the top k is >= tau.  The
// keys >= tau (usually a few dozen) are gathered in block order (one ballot per
// row of 32 blocks), packed as key << 32 | ~index so that one comparison
// orders by key and then by lower index, and ranked among themselves; the
// ranks < k are written to dst[0, k) (and copy) in block order.  Returns false,
// writing nothing, when more than cap keys are >= tau.  Above 512 blocks the
// bound is the k-th largest of the lanes' two largest keys (also keys, so still
// at most the k-th largest key, and much closer to it: ~35 candidates of 2016
// instead of ~110, whose exact ranking costs the square of their count).
// Above 512 blocks the selection is written as short loops (its code runs
// once per launch and is fetched cold).
__device__ __forceinline__ bool topk_warp(const float* sc, int nb, int k, int32_t* dst, int32_t* copy,
                                          unsigned long long* cand, int cap, bool& nan_out) {
  constexpr int kRows = 16;  // rows of 32 blocks held in registers up to 512 blocks
  const int lane = role_tid() & 31;
  const uint32_t lt = lanemask_lt();
  uint32_t lmax = 0u;
  bool nan = false;
  int m = 0;  // candidates so far (block order)
  if (nb <= 32 * kRows) {
    // keys in registers, every load issued at once (sc holds at least 32 kRows
    // entries; entries past nb are read but not used): this path runs beside
    // busy attention warps, where independent instructions matter more than
    // the code's size
    uint32_t kr[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const float f = sc[lane + 32 * i];
      const bool v = lane + 32 * i < nb;
      nan |= v && f != f;
      kr[i] = v ? float_key(f) : 0u;
      lmax = max(lmax, kr[i]);
    }
    nan_out = __any_sync(kFull, nan);
    const uint32_t tau = kth_lane_max(lmax, lane, k);
    uint32_t bal[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) bal[i] = __ballot_sync(kFull, lane + 32 * i < nb && kr[i] >= tau);
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const int pos = m + __popc(bal[i] & lt);
      if (((bal[i] >> lane) & 1u) && pos < cap) cand[pos] = ((unsigned long long)kr[i] << 32) | (uint32_t)~(lane + 32 * i);
      m += __popc(bal[i]);
    }
  } else {
    uint32_t lsec = 0u;  // the lane's second largest key (0, below every key, if it has one key)
#pragma unroll 4
    for (int j = lane; j < nb; j += 32) {
      const float f = sc[j];
      nan |= f != f;
      const uint32_t u = float_key(f);
      lsec = max(lsec, min(lmax, u));
      lmax = max(lmax, u);
    }
    nan_out = __any_sync(kFull, nan);
    const uint32_t tau = kth_of_lane_pairs(lmax, lsec, lane, k);
#pragma unroll 1
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t u = j < nb ? float_key(sc[j]) : 0u;
      const uint32_t bal = __ballot_sync(kFull, j < nb && u >= tau);
      const int pos = m + __popc(bal & lt);
      if (((bal >> lane) & 1u) && pos < cap) cand[pos] = ((unsigned long long)u << 32) | (uint32_t)~j;
      m += __popc(bal);
    }
  }
  if (m > cap) return false;
  __syncwarp();
  int base = 0;
#pragma unroll 1
  for (int c0 = 0; c0 < m; c0 += 32) {
    const int c = c0 + lane;
    bool sel = false;
    unsigned long long me = 0ull;
    if (c < m) {
      me = cand[c];
      int rank = 0, o = 0;  // candidates above this one (all packed values differ)
#pragma unroll 2
      for (; o + 4 <= m; o += 4) {
        const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(&cand[o]);
        const ulonglong2 y = *reinterpret_cast<const ulonglong2*>(&cand[o + 2]);
        rank += (x.x > me ? 1 : 0) + (x.y > me ? 1 : 0) + (y.x > me ? 1 : 0) + (y.y > me ? 1 : 0);
      }
      for (; o < m; ++o) rank += cand[o] > me ? 1 : 0;
      sel = rank < k;
    }
    const uint32_t b = __ballot_sync(kFull, sel);
    if (sel) {
      const int q = base + __popc(b & lt);
      const int j = (int)~(uint32_t)me;
      dst[q] = j;
      if (copy) copy[q] = j;
    }
    base += __popc(b);
  }
  return true;
}

// ---------------------------------------------------------------- streaming top-k
// Every statistics warp holds, one per lane, the 32 largest packed keys
// (key << 32 | ~block: one comparison orders by score, then by the lower block
// index) of the items it has scored, sorted descending; an item whose keys all
// fall below the list's last entry is skipped.  Lists are merged with bitonic
// networks across the warp.
__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m) {
  const uint32_t lo = __shfl_xor_sync(kFull, (uint32_t)v, m), hi = __shfl_xor_sync(kFull, (uint32_t)(v >> 32), m);
  return ((unsigned long long)hi << 32) | lo;
}
__device__ __forceinline__ unsigned long long shfl_u64(unsigned long long v, int src) {
  const uint32_t lo = __shfl_sync(kFull, (uint32_t)v, src), hi = __shfl_sync(kFull, (uint32_t)(v >> 32), src);
  return ((unsigned long long)hi << 32) | lo;
}
// One compare-exchange step across the warp: the lane with (lane & j) == 0
// keeps the larger value when `desc`, the smaller otherwise.
__device__ __forceinline__ unsigned long long bitonic_step(unsigned long long v, int lane, int j, bool desc) {
  const unsigned long long o = shfl_xor_u64(v, j);
  const bool keep_max = ((lane & j) == 0) == desc;
  return keep_max ? (o > v ? o : v) : (o < v ? o : v);
}
// Sort the warp's 32 values descending (lane 0 the largest).
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long v, int lane) {
  // straight-line network (15 steps): it runs once per scored item
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) v = bitonic_step(v, lane, j, (lane & k) == 0);
  return v;
}
// The 32 largest of two descending lists (one value per lane), descending: a
// against b reversed, element by element, keeps the larger half as a bitonic
// sequence, which a half-cleaner network sorts.
__device__ __forceinline__ unsigned long long warp_merge_desc(unsigned long long a, unsigned long long b, int lane) {
  const unsigned long long br = shfl_u64(b, 31 - lane);
  unsigned long long v = a > br ? a : br;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) v = bitonic_step(v, lane, j, true);
  return v;
}
// Fold one scored item into the warp's list: lane l offers the packed key of
// block j (valid), 0 (below every key) past the item's blocks.
__device__ __forceinline__ unsigned long long topk_offer(unsigned long long run, float score, int j, bool valid,
                                                         int lane, bool& nan) {
  nan |= valid && score != score;
  const unsigned long long v = valid ? (((unsigned long long)float_key(score) << 32) | (uint32_t)~(uint32_t)j) : 0ull;
  const unsigned long long last = shfl_u64(run, 31);
  if (__ballot_sync(kFull, v > last) == 0u) return run;
  return warp_merge_desc(run, warp_sort_desc(v, lane), lane);
}

}  // namespace
}  // namespace hyb
