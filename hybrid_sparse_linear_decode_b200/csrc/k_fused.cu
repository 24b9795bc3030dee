// One decode step of one layer in one launch: block scores, the global linear
// term, the top-k block selection, exact attention over sinks + window +
// selected blocks with the selected blocks' (1 + s) subtraction, and the merge
// under one shared normaliser; plus the fold of the tokens evicted since the
// previous decode into the state, and the appended token's cache write.
//
// Grid: one thread-block cluster of C CTAs per unit (batch row, KV head), one
// CTA per SM.  Rank r of a unit's cluster owns
//   * its share of the blocks (equal shares rounded up to 4 blocks; score items
//     of 32 blocks each) and rows [r D / C, (r+1) D / C) of H (H items),
//   * window chunks r, r + C, ... and selected chunks r, r + C, ... (64-token
//     pieces of the exact set, split-K).
// Its items stream through a kFStages-deep shared-memory ring in the order score
// items, window chunks, H items, selected chunks: a producer warp issues
// the copies (TMA tensor loads for K/V chunks, untiled bulk copies for the
// statistics and H, no multicast); the other warps consume them.
//
// Warp roles (12 warps; role r runs on hardware warp given by role_tid):
//   0-7  attention, in pairs: chunk c to pair c % 4, all 64 tokens for the scores,
//        one half of the head dimension per warp for PV, on the tensor cores
//        (mma.sync m16n8k16, bf16 in, fp32 accumulate), G <= 4 query heads
//        packed into the 16-row M dimension (rows 0-3 softmax, rows 4-7 the
//        Taylor weights 1 + s of selected-block tokens, rows 8-15 the bf16
//        rounding remainders of rows 0-7);
//   8-10 statistics: block scores (score item i to warp i % 3), the Welford
//        fold, the top-k (one warp), H rows, the linear term;
//   11   producer: lane 0 issues every copy in ring order.
//
// Block score ("SPLA: Block Sparse Plus Linear Attention for Long Context
// Modeling", Abstract; "Principled Block Selection via Taylor Expansion";
// "Grouped Sparsity"): score_j = sum_i ( q'_i . mu_j + 1/2 sum_c q'_ic^2 var_jc ).
// Each rank keeps the scores of its blocks in shared memory and bulk-copies
// them into every other rank's scores array over distributed shared memory
// (completing bytes on that rank's "scores" barrier); every rank then selects
// the same top_k blocks itself (ties to the lower index), while the ring
// streams its window chunks.
//
// Linear term (SLAKE, first-order Taylor exp(s) ~ 1 + s; SPLA residual
// attention): N_glob_i = zv + H^T q'_i, D_glob_i = n + q'_i . zk, each rank
// summing its rows of H.  Merge, each rank a slice of the outputs, over
// distributed shared memory after a cluster barrier (per query head, base-2
// exponent m of the exact part):
//   o = (N_ex + 2^{-m} (N_glob - N_sel)) / (D_ex + 2^{-m} (D_glob - D_sel)),
// as the equal form (N_ex 2^m + ...)/(D_ex 2^m + ...) when m < 0.
//
// Evictions since the previous decode (positions [fold_begin, fold_end), usually
// one token) are folded into the rows an item holds before it is used:
// H += k v^T, zk += k, zv += v, n += 1 (SPLA "Recurrence") and Welford's running
// mean / population variance of the token's block (B. P. Welford,
// Technometrics 4(3), 1962).  With q == null the kernel only folds.
//
// Every wait inside the kernel is bounded (a timeout sets a status bit and the
// CTA skips the rest of its work); all CTAs of a cluster always reach both
// cluster barriers.  The limit of the waits for progress (ring items, the
// scores, the selection, a free stage) comes with the launch; the two waits
// that guard the CTA's exit (copies in flight into its ring, the other ranks'
// merge stores) keep the long default limit.  Launch chaining: programmatic dependent launch -- the CTA
// waits for the predecessor grid before touching memory.
#include "k_common.cuh"

namespace hyb {

namespace {

constexpr int kFStages = 6;
constexpr int kFScoresMax = 2048;   // scores a CTA keeps for its unit (else they go through global memory)
static_assert(kFScoresMax >= 512, "the one-warp top-k reads 512 entries unconditionally");

template <int D>
struct FusedSmem {
  static constexpr int kHalf = kTile * D * 2;        // K (or V) of one 64-token chunk, bytes
  static constexpr int kStageBytes = 2 * kHalf;      // 32 KB at D = 128
  static constexpr int kBoxBytes = kBoxRows * D * 2;
  static constexpr int kPF = partial_floats(D);
  // scores gathered in shared memory (the combine slots hold them); else via L2
  static constexpr int kGather = 2 * kPF < kFScoresMax ? 2 * kPF : kFScoresMax;
  uint8_t ring[kFStages][kStageBytes];               // 1024-byte aligned
  float scores[kFScoresMax];                         // this rank's share of the unit's block scores
  float qs[kMaxGroup][D];                            // q' = q * scale
  float qsT[D][kMaxGroup];                           // q' transposed (H rows: one vector load per row)
  float qsum[2][D];                                  // sum_i q'_i, 1/2 sum_i q'_i^2 (block scores)
  float ktok[D];                                     // K and V rows of the pending token (H fold)
  float vtok[D];
  alignas(16) float wpart[2][kPF];                   // attention combine slots; [0] ends as the record
  float linp[kMaxGroup][D + 1];                      // this rank's linear partial (D_glob in rank 0)
  alignas(16) float mrecv[merge_floats(D)];          // merge: what every rank sends this rank
  float zks[D];                                      // rank 0: zk after the fold
  int32_t sel_cache[kSelCache];
  alignas(16) uint32_t hist[256];                    // top-k: radix histogram, or two warps' candidate lists
  uint32_t tk[8];                                    // top-k: shared scalars
  uint32_t tks[2][4];                                // top-k: per-warp partials / scan scratch
  uint32_t tkw[2];                                   // one-warp top-k: done, NaN seen
  int4 desc[kFStages];                               // chunk items: start, len, is_sel
  float2 xmax[4][2][4];                              // per pair and warp: a chunk's column maxima, then the weight sums
  // A stage's items belong to one of two consumer groups.  Each group has its
  // own "full" barrier per stage and waits only for its own items, in order,
  // so it is never more than one phase ahead of a barrier it waits on (a
  // parity wait cannot tell phase k from phase k - 2).
  uint64_t full_attn[kFStages];                      // window / selected chunks
  uint64_t full_aux[kFStages];                       // score / H items
  uint64_t empty[kFStages];                          // one release per item
  uint64_t scores_bar;                               // C arrivals: every rank's scores are in place
  uint64_t sel_bar;                                  // 1 arrival: the selection is known
  uint64_t merge_bar;                                // 1 arrival + the other ranks' merge bytes
  UnitGeo geo;                                       // this unit's geometry
  int sel_state;                                     // 1 sel_cache, 2 global row (sel_row), 3 every block
  const int32_t* sel_row;
  int abort;
};

}  // namespace
}  // namespace hyb

namespace hyb {
namespace {

// ---------------------------------------------------------------- item sequence
// Items of rank r, in ring order: nS score items, nW window (and sink) chunks,
// nH H items, nX selected chunks.  The scores come first, so that the top-k
// runs while the window chunks and H rows stream in; the statistics warps take
// the H rows after the selection, while the selected chunks stream.  Every
// thread derives the same sequence.
struct Seq {
  int b0, b1, nS;   // blocks [b0, b1), kFBlocks per score item
  int h0, h1, nH;   // rows of H [h0, h1), kFRows per H item
  int nW, nX, n;
};

template <int D>
struct Geo {
  static constexpr int kStageBytes = 2 * kTile * D * 2;
  static constexpr int kBlocks = kStageBytes / (8 * D);  // mean + variance rows per score item
  static constexpr int kRows = kStageBytes / (4 * D);    // rows of H per H item
};

// Does this launch select the top-k from the scores (else: the caller's row,
// every block, or none)?
__device__ __forceinline__ bool runs_topk(const FusedParams& p, const UnitGeo& g) {
  return p.q != nullptr && p.sel_given == nullptr && g.k_eff > 0 && g.k_eff < g.nb;
}

// Above kStreamMin candidate blocks (k <= 32, the unit's scores in shared
// memory) every statistics warp keeps the top 32 of the blocks it scores while
// it scores them; the rank's top-k goes to every other rank instead of its
// scores, and each rank merges the C lists.  The global top-k lies in the union
// of the ranks' top-k, so the result is the same.  (At or below kStreamMin the
// ranks exchange their scores and one warp selects from all of them.)
constexpr int kStreamMin = kStreamBlocks;
template <int D, bool kStream>
__device__ __forceinline__ bool stream_topk(const FusedParams& p, const UnitGeo& g);
// Candidate slot of one rank in the exchange: k packed entries, rounded up to
// an even count (bulk copies move multiples of 16 bytes); the C slots live in
// the attention combine slots, idle until the selection is made.
__device__ __forceinline__ int cand_slot(int k) { return (k + 1) & ~1; }

template <int D>
__device__ __forceinline__ Seq make_seq(const FusedParams& p, const UnitGeo& g, int r) {
  Seq q;
  const int C = p.C;
  block_share(g.nb, C, r, q.b0, q.b1);
  q.nS = (q.b1 - q.b0 + Geo<D>::kBlocks - 1) / Geo<D>::kBlocks;
  q.h0 = r * D / C;
  q.h1 = (r + 1) * D / C;
  q.nH = (q.h1 - q.h0 + Geo<D>::kRows - 1) / Geo<D>::kRows;
  const int n_pre = g.n_sink_chunks + g.n_win_chunks;
  if (p.q != nullptr) {
    q.nW = r < n_pre ? (n_pre - r + C - 1) / C : 0;
    q.nX = r < g.n_sel_chunks ? (g.n_sel_chunks - r + C - 1) / C : 0;
  } else {
    q.nW = q.nX = 0;
  }
  q.n = q.nS + q.nW + q.nH + q.nX;
  return q;
}

// position in the ring order of score item i / H item i / chunk item c (window
// chunks first, then selected chunks)
__device__ __forceinline__ int seq_of_s(const Seq&, int i) { return i; }
__device__ __forceinline__ int seq_of_h(const Seq& s, int i) { return s.nS + s.nW + i; }
__device__ __forceinline__ int seq_of_chunk(const Seq& s, int c) { return c < s.nW ? s.nS + c : s.nS + s.nH + c; }

// (only in the kernel variant built for it: the other variant has no trace of
// it in its scoring loop)
template <int D, bool kStream>
__device__ __forceinline__ bool stream_topk(const FusedParams& p, const UnitGeo& g) {
  return kStream && runs_topk(p, g) && g.nb > kStreamMin && g.k_eff <= 32 && g.nb <= FusedSmem<D>::kGather;
}

// Score items [*i0, *i1) of the rank hold the blocks with pending evictions
// (empty when nothing is pending).  Computed once per launch.
template <int D>
__device__ __forceinline__ void fold_items(const FusedParams& p, const UnitGeo& g, const Seq& s, int* i0, int* i1) {
  *i0 = *i1 = 0;
  if (g.fold_end <= g.fold_begin || s.b1 <= s.b0) return;
  // positions fit in 32 bits (units x capacity < 2^31)
  const int jb0 = (int)(g.fold_begin - p.S) / p.Bk, jb1 = (int)(g.fold_end - 1 - p.S) / p.Bk;
  const int lo = max(jb0, s.b0), hi = min(jb1, s.b1 - 1);
  if (lo > hi) return;
  *i0 = (lo - s.b0) / Geo<D>::kBlocks;
  *i1 = (hi - s.b0) / Geo<D>::kBlocks + 1;
}
// score item idx: does it hold a block with pending evictions?
template <int D>
__device__ __forceinline__ bool score_item_folds(const FusedParams& p, const UnitGeo& g, const Seq& s, int idx) {
  int i0, i1;
  fold_items<D>(p, g, s, &i0, &i1);
  return idx >= i0 && idx < i1;
}

// Producer: the copies of one K/V chunk (rows [start, start + len) of the
// unit's caches) into ring stage `stage`; its descriptor tells the attention
// warps what the stage holds.
template <int D>
__device__ __forceinline__ void issue_chunk(const KVMaps* tm, FusedSmem<D>& sm, int stage, int64_t ubase, int start,
                                            int len, int is_sel, uint64_t pol) {
  using Sm = FusedSmem<D>;
  uint64_t* bar = &sm.full_attn[stage];
  const uint32_t dst = smem_u32(sm.ring[stage]);
  sm.desc[stage] = make_int4(start, len, is_sel, 0);
  if (len <= 0) {
    mbar_arrive(bar);
    return;
  }
  const int row = (int)(ubase + start);
  if (len == kTile) {  // full chunk: one 64-row box per tensor
    mbar_arrive_expect_tx(bar, (uint32_t)(2 * Sm::kHalf));
    tma_load_3d_stream(dst, &tm->k64, 0, 0, row, bar, pol);
    tma_load_3d_stream(dst + Sm::kHalf, &tm->v64, 0, 0, row, bar, pol);
  } else {             // ragged chunk: only the 16-row boxes it touches
    const int nbox = (len + kBoxRows - 1) / kBoxRows;
    mbar_arrive_expect_tx(bar, (uint32_t)(nbox * Sm::kBoxBytes * 2));
    for (int bx = 0; bx < nbox; ++bx) {
      tma_load_3d_stream(dst + bx * Sm::kBoxBytes, &tm->k16, 0, 0, row + bx * kBoxRows, bar, pol);
      tma_load_3d_stream(dst + Sm::kHalf + bx * Sm::kBoxBytes, &tm->v16, 0, 0, row + bx * kBoxRows, bar, pol);
    }
  }
}

}  // namespace
}  // namespace hyb

namespace hyb {
namespace {

// ---------------------------------------------------------------- statistics role
// Fold the pending evictions into the statistics rows of score item `idx` and
// write the rows back: Welford's running mean and population variance, one
// token at a time.  One warp, lane l holding channels [l*CPL, l*CPL + CPL) of
// each block that has pending tokens (usually one).  The ring stage keeps the
// old rows (writing it would need a proxy fence against the copies in flight):
// the block's score is recomputed here from the folded rows and replaces the
// one score_item_warp stored from the old rows.
template <int D>
__device__ __forceinline__ void fold_score_item(const FusedParams& p, const UnitGeo& g, FusedSmem<D>& sm, const Seq& s,
                                                int unit, int idx, int stage) {
  constexpr int CPL = D / 32;
  constexpr int RB = Geo<D>::kBlocks;
  const int lane = role_tid() & 31;
  const int j0 = s.b0 + idx * RB;
  const int nblk = min(RB, s.b1 - j0);
  const float* mrows = reinterpret_cast<const float*>(sm.ring[stage]);
  const float* vrows = mrows + RB * D;
  const int jb0 = (int)(g.fold_begin - p.S) / p.Bk, jb1 = (int)(g.fold_end - 1 - p.S) / p.Bk;
  const int bl0 = max(0, jb0 - j0), bl1 = min(nblk - 1, jb1 - j0);
  float q1[CPL], q2[CPL];
  lds_vec<CPL>(&sm.qsum[0][lane * CPL], q1);
  lds_vec<CPL>(&sm.qsum[1][lane * CPL], q2);
#pragma unroll 1
  for (int bl = bl0; bl <= bl1; ++bl) {
    const int j = j0 + bl;
    const int64_t bs = p.S + (int64_t)j * p.Bk;
    const int64_t t0 = max(bs, (int64_t)g.fold_begin), t1 = min(bs + p.Bk, (int64_t)g.fold_end);
    float m[CPL], v[CPL];
    lds_vec<CPL>(mrows + bl * D + lane * CPL, m);
    lds_vec<CPL>(vrows + bl * D + lane * CPL, v);
#pragma unroll 1
    for (int64_t t = t0; t < t1; ++t) {
      float x[CPL];
      if (g.fold_end - g.fold_begin == 1) {
        lds_vec<CPL>(&sm.ktok[lane * CPL], x);  // staged at the start of the statistics role
      } else {
        load_bf16<CPL>(p.k_cache + ((int64_t)unit * p.cap + t) * D + lane * CPL, x);
      }
      const float cnt = (float)(t - bs + 1);
      const float inv = 1.f / cnt;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        if (t == bs) {  // the block's first token: the stored row is not read
          m[c] = x[c];
          v[c] = 0.f;
        } else {
          const float delta = x[c] - m[c];
          const float m1 = m[c] + delta * inv;
          v[c] = (v[c] * (cnt - 1.f) + delta * (x[c] - m1)) * inv;
          m[c] = m1;
        }
      }
    }
    sts_vec<CPL>(p.mu + ((int64_t)unit * p.max_blocks + j) * D + lane * CPL, m);
    sts_vec<CPL>(p.var + ((int64_t)unit * p.max_blocks + j) * D + lane * CPL, v);
    if (p.q != nullptr) {
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) acc += q1[c] * m[c] + q2[c] * v[c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
      __syncwarp();  // after score_item_warp's stores of the old score
      if (lane == 0) {
        p.scores[(int64_t)unit * p.max_blocks + j] = acc;
        if (g.nb <= FusedSmem<D>::kGather) sm.scores[j] = acc;
      }
    }
  }
  __syncwarp();
}

// Score item `idx` by one warp, score_j = sum_c qsum[0][c] mu_jc +
// qsum[1][c] var_jc (qsum = sum_i q'_i and 1/2 sum_i q'_i^2): lane l forms the
// partial sums of its channels [l*CPL, l*CPL + CPL) for all 32 blocks (each
// row read once, conflict-free, at fixed offsets from one base), then a
// transposing butterfly (31 shuffles in 5 rounds: in the round of width h a
// lane keeps the half of its values whose block index has bit h equal to its
// own) leaves block l's score in lane l.  Rows past the item's last block hold
// stale stage data: their sums stay in their own lanes and are not stored.
template <int D>
__device__ __forceinline__ void score_item_warp(const FusedParams& p, const UnitGeo& g, FusedSmem<D>& sm, const Seq& s,
                                                int unit, int idx, int stage) {
  constexpr int CPL = D / 32;
  constexpr int RB = Geo<D>::kBlocks;
  static_assert(RB == 32, "one block per lane");
  const int lane = role_tid() & 31;
  const int j0 = s.b0 + idx * RB;
  const int nblk = min(RB, s.b1 - j0);
  const float* mrows = reinterpret_cast<const float*>(sm.ring[stage]) + lane * CPL;
  const float* vrows = mrows + RB * D;
  float q1[CPL], q2[CPL];
  lds_vec<CPL>(&sm.qsum[0][lane * CPL], q1);
  lds_vec<CPL>(&sm.qsum[1][lane * CPL], q2);
  float part[RB];
#pragma unroll
  for (int b = 0; b < RB; ++b) {
    float m[CPL], v[CPL];
    lds_vec<CPL>(mrows + b * D, m);
    lds_vec<CPL>(vrows + b * D, v);
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc += q1[c] * m[c] + q2[c] * v[c];
    part[b] = acc;
  }
#pragma unroll
  for (int h = RB / 2; h >= 1; h >>= 1) {
    const bool up = (lane & h) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = up ? part[i] : part[i + h];
      const float keep = up ? part[i + h] : part[i];
      part[i] = keep + __shfl_xor_sync(kFull, send, h);
    }
  }
  if (lane < nblk) {
    p.scores[(int64_t)unit * p.max_blocks + j0 + lane] = part[0];
    if (g.nb <= FusedSmem<D>::kGather) sm.scores[j0 + lane] = part[0];  // this rank's share; pushed to the other ranks
  }
}

// H item `idx`: warp aw takes rows aw, aw + 3, ... of the item; lane l columns
// [l*CPL, l*CPL + CPL).  Folds pending evictions into the rows (written back)
// and accumulates q'_i[r] H[r][c] into hacc (qsT[r] holds q'_0..3[r]).  With
// one pending token (the usual case) its K and V rows come from shared memory.
template <int D, int kFold>  // kFold: 0 none, 1 one token (ktok, vtok), 2 several (global memory)
__device__ __forceinline__ void h_rows(const FusedParams& p, const UnitGeo& g, FusedSmem<D>& sm, int unit, int r0, int nrows,
                                       const float* hrows, float (&hacc)[kMaxGroup][D / 32]) {
  constexpr int CPL = D / 32;
  static_assert(kMaxGroup == 4, "qsT rows are one float4");
  const int a = role_tid() - kAttnThreads, aw = a >> 5, lane = a & 31;
  const int64_t ub = (int64_t)unit * p.cap;
  float v1[CPL];
  if (kFold == 1) lds_vec<CPL>(&sm.vtok[lane * CPL], v1);
  const bool acc = p.q != nullptr;
#pragma unroll 2
  for (int rl = aw; rl < nrows; rl += kAuxWarps) {
    const int row = r0 + rl;
    float h[CPL];
    lds_vec<CPL>(hrows + rl * D + lane * CPL, h);
    if (kFold == 1) {
      const float kr = sm.ktok[row];
#pragma unroll
      for (int c = 0; c < CPL; ++c) h[c] += kr * v1[c];
    } else if (kFold == 2) {
      for (int64_t t = g.fold_begin; t < g.fold_end; ++t) {
        const float kr = __bfloat162float(p.k_cache[(ub + t) * D + row]);
        float vv[CPL];
        load_bf16<CPL>(p.v_cache + (ub + t) * D + lane * CPL, vv);
#pragma unroll
        for (int c = 0; c < CPL; ++c) h[c] += kr * vv[c];
      }
    }
    if (kFold != 0) sts_vec<CPL>(p.H + ((int64_t)unit * D + row) * D + lane * CPL, h);
    if (acc) {
      const float4 qr = *reinterpret_cast<const float4*>(&sm.qsT[row][0]);
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        hacc[0][c] += qr.x * h[c];
        hacc[1][c] += qr.y * h[c];
        hacc[2][c] += qr.z * h[c];
        hacc[3][c] += qr.w * h[c];
      }
    }
  }
}

template <int D>
__device__ __forceinline__ void aux_h_item(const FusedParams& p, const UnitGeo& g, FusedSmem<D>& sm, const Seq& s, int unit,
                                           int idx, int stage,
                                           float (&hacc)[kMaxGroup][D / 32]) {
  constexpr int RH = Geo<D>::kRows;
  const int r0 = s.h0 + idx * RH;
  const int nrows = min(RH, s.h1 - r0);
  const float* hrows = reinterpret_cast<const float*>(sm.ring[stage]);
  const int64_t nf = g.fold_end - g.fold_begin;
  if (nf == 0) h_rows<D, 0>(p, g, sm, unit, r0, nrows, hrows, hacc);
  else if (nf == 1) h_rows<D, 1>(p, g, sm, unit, r0, nrows, hrows, hacc);
  else h_rows<D, 2>(p, g, sm, unit, r0, nrows, hrows, hacc);
}

// After every H item (aux threads): the linear partial of this rank's H rows,
// sum_r q'_i[r] H[r][:], summed over the three warps into linp one warp at a
// time; rank 0 also folds the pending evictions into zk, zv and n (their old
// values were loaded at the start of the role), adds zv (N_glob's count term)
// and forms D_glob = n + q'_i . zk in linp[i][D].
template <int D>
__device__ void aux_finish_linear(const FusedParams& p, const UnitGeo& g, FusedSmem<D>& sm, int unit, int rank,
                                  const float (&hacc)[kMaxGroup][D / 32], const float (&zk0)[kAuxCols<D>],
                                  const float (&zv0)[kAuxCols<D>], float n0) {
  constexpr int CPL = D / 32, NZ = kAuxCols<D>;
  const int a = role_tid() - kAttnThreads, aw = a >> 5, lane = a & 31;
  float zv[NZ];
  float nval = n0;
  if (rank == 0) {
    const int64_t nf = g.fold_end - g.fold_begin;
    const int64_t ub = (int64_t)unit * p.cap;
#pragma unroll
    for (int k = 0; k < NZ; ++k) {
      const int c = a + k * kAuxThreads;
      zv[k] = zv0[k];
      if (c < D) {
        float zk = zk0[k];
        if (nf == 1) {
          zk += sm.ktok[c];
          zv[k] += sm.vtok[c];
        } else if (nf > 1) {
          for (int64_t t = g.fold_begin; t < g.fold_end; ++t) {
            zk += __bfloat162float(p.k_cache[(ub + t) * D + c]);
            zv[k] += __bfloat162float(p.v_cache[(ub + t) * D + c]);
          }
        }
        if (nf > 0) {
          p.zk[(int64_t)unit * D + c] = zk;
          p.zv[(int64_t)unit * D + c] = zv[k];
        }
        sm.zks[c] = zk;
      }
    }
    if (nf > 0) {
      nval += (float)nf;
      if (a == 0) p.n[unit] = nval;
    }
  }
  if (p.q == nullptr) return;
#pragma unroll 1
  for (int w = 0; w < kAuxWarps; ++w) {
    if (aw == w)
#pragma unroll
      for (int i = 0; i < kMaxGroup; ++i)
        if (i < p.G)
#pragma unroll
          for (int c = 0; c < CPL; ++c) {
            float* dst = &sm.linp[i][lane * CPL + c];
            *dst = (w == 0 ? 0.f : *dst) + hacc[i][c];
          }
    named_sync(kBarAux, kAuxThreads);  // also: zks is complete
  }
  if (rank == 0) {
    for (int i = 0; i < p.G; ++i)
#pragma unroll
      for (int k = 0; k < NZ; ++k) {
        const int c = a + k * kAuxThreads;
        if (c < D) sm.linp[i][c] += zv[k];
      }
    if (aw == 0)
      for (int i = 0; i < p.G; ++i) {
        float d = 0.f;
        for (int c = lane; c < D; c += 32) d += sm.qs[i][c] * sm.zks[c];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(kFull, d, o);
        if (lane == 0) sm.linp[i][D] = nval + d;
      }
  }
}

}  // namespace
}  // namespace hyb

namespace hyb {
namespace {

// Statistics threads (all of them): make the unit's selection known to the
// producer (sel_state, then an arrival on sel_bar): the caller's row, every
// block (k >= nb), none (k == 0), or the top-k of the unit's scores once every
// rank's share is in place.  Rank 0 fills the caller's copy.
template <int D, bool kStream>
__device__ void aux_select(const FusedParams& p, const UnitGeo& g, FusedSmem<D>& sm, int unit, int rank) {
  const int a = role_tid() - kAttnThreads;
  int32_t* copy = (p.sel_out != nullptr && rank == 0) ? p.sel_out + (int64_t)unit * p.top_k : nullptr;
  int state = 3;
  const int32_t* row = nullptr;
  if (p.sel_given != nullptr) {
    row = p.sel_given + (int64_t)unit * p.top_k;
    if (p.top_k <= kSelCache) {
      for (int j = a; j < p.top_k; j += kAuxThreads) sm.sel_cache[j] = __ldg(row + j);
      state = 1;
    } else {
      state = 2;
    }
  } else if (!runs_topk(p, g)) {  // no block, or every block
    if (copy)
      for (int j = a; j < p.top_k; j += kAuxThreads) copy[j] = j < g.k_eff ? j : -1;
  } else {
    if (a == 0) {  // one decision for all statistics threads (their barrier counts must match)
      const bool ok = wait_cluster_bounded(&sm.scores_bar, 0, p.wait_ns);
      if (!ok) {
        atomicOr(p.status, HYB_STATUS_TIMEOUT);
        sm.abort = 1;
      }
      sm.tk[7] = ok ? 1u : 0u;
    }
    named_sync(kBarAux, kAuxThreads);
    if (sm.tk[7] != 0u && stream_topk<D, kStream>(p, g)) {  // every rank's candidates are in place: merge them
      int32_t* dst = sm.sel_cache;
      if (a < 32) {
        const int lane = a, k = g.k_eff, kslot = cand_slot(k);
        const unsigned long long* all = reinterpret_cast<const unsigned long long*>(&sm.wpart[0][0]);
        unsigned long long run = lane < k ? all[lane] : 0ull;
#pragma unroll 1
        for (int r = 1; r < p.C; ++r) run = warp_merge_desc(run, lane < k ? all[r * kslot + lane] : 0ull, lane);
        // the k largest in ascending block order: sorted descending by the complement of the index
        const uint32_t j = ~(uint32_t)run;
        const unsigned long long x = lane < k ? (unsigned long long)(0xffffffffu - j) : 0ull;
        const uint32_t js = 0xffffffffu - (uint32_t)warp_sort_desc(x, lane);
        if (lane < k) {
          dst[lane] = (int32_t)js;
          if (copy) copy[lane] = (int32_t)js;
        }
      }
      if (copy)
        for (int j = g.k_eff + a; j < p.top_k; j += kAuxThreads) copy[j] = -1;
      state = 1;
      row = dst;
    } else if (sm.tk[7] != 0u) {
      const bool glob = g.nb > FusedSmem<D>::kGather;
      const float* src = glob ? p.scores + (int64_t)unit * p.max_blocks : sm.scores;
      int32_t* dst = g.k_eff <= kSelCache ? sm.sel_cache : p.sel + (int64_t)unit * p.top_k;
      bool nan = false, done = false;
      if (g.k_eff <= 32 && !glob) {
        if (a < 32) {  // one warp; the candidates go to the attention combine slots, idle until the selection is made
          bool wn;
          const bool ok = topk_warp(sm.scores, g.nb, g.k_eff, dst, copy,
                                    reinterpret_cast<unsigned long long*>(&sm.wpart[0][0]), FusedSmem<D>::kPF, wn);
          if (a == 0) {
            sm.tkw[0] = ok ? 1u : 0u;
            sm.tkw[1] = wn ? 1u : 0u;
          }
        }
        named_sync(kBarAux, kAuxThreads);
        done = sm.tkw[0] != 0u;
        nan = sm.tkw[1] != 0u;
      }
      if (!done) {  // more than 32 blocks, or too many candidates: the radix selection
        const TopkSmem t{sm.hist, sm.tk, &sm.tks[0][0]};
        nan = aux_topk(t, src, glob, g.nb, g.k_eff, dst, copy);
      }
      if (nan && a == 0) atomicOr(p.status, HYB_STATUS_NAN_SCORE);
      if (copy)
        for (int j = g.k_eff + a; j < p.top_k; j += kAuxThreads) copy[j] = -1;
      state = g.k_eff <= kSelCache ? 1 : 2;
      row = dst;
    }
  }
  named_sync(kBarAux, kAuxThreads);
  if (a == 0) {
    sm.sel_row = row;
    sm.sel_state = state;
    mbar_arrive(&sm.sel_bar);  // release: the selection is visible to the producer
  }
}

}  // namespace
}  // namespace hyb

namespace hyb {
namespace {

// ---------------------------------------------------------------- attention role
// Warps 0-3: every window and selected chunk of the rank, in ring order; then
// the 4 warps' partials are combined into sm.wpart[0] (the rank's record:
// m[4], l[4], dsel[4], pad[4], acc[4][D], nsel[4][D]).
template <int D>
__device__ void attn_role(const FusedParams& p, FusedSmem<D>& sm, const Seq& s, int unit) {
  constexpr int NT8 = D / 8;  // 8-column tiles of the head dimension
  constexpr int NH = NT8 / 2;  // the tiles of this warp's half of the columns
  constexpr int KS = D / 16;  // k-steps of the QK product
  const int tid = role_tid(), warp = tid >> 5, lane = tid & 31;
  const int pair = warp >> 1, half = warp & 1;  // chunk c to pair c % 4; PV columns [half D/2, half D/2 + D/2)
  const int g = lane >> 2, tig = lane & 3;
  const bool p_lane = g < 4;  // rows 0-3: softmax part; rows 4-7: Taylor part
  const int head = g & 3;
  const int mi = lane >> 3, rr = lane & 7;

  // B fragments of Q^T for the S^T = K Q^T product: columns n and n + 4 (lane
  // groups g and g + 4) are query head n (zero for n >= G), so that the lanes
  // building the Taylor weights hold their heads' scores themselves
  uint32_t qb[KS][2];
  {
    const bool real = (g & 3) < p.G;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(p.q + ((int64_t)unit * p.G + (real ? (g & 3) : 0)) * D);
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qb[kk][0] = real ? __ldg(qrow + kk * 8 + tig) : 0u;
      qb[kk][1] = real ? __ldg(qrow + kk * 8 + 4 + tig) : 0u;
    }
  }
  float O[NH][4];
#pragma unroll
  for (int n = 0; n < NH; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.f;
  // lanes tig < 2: running max (log2 units) and weight sums of heads 2tig, 2tig+1;
  // lanes tig >= 2: Taylor weight sums of heads 2tig-4, 2tig-3
  const bool soft_lane = tig < 2;
  float mr0 = -INFINITY, mr1 = -INFINITY, acc0 = 0.f, acc1 = 0.f;

  // Chunk items go to the attention warp pairs in turn (chunk c to pair c % 4):
  // each warp of the pair scores and weighs its own 32 of the chunk's tokens,
  // and each computes the PV product of all 64 tokens for half of the head
  // dimension (the weights cross between the two warps through shared
  // memory).  Every attention warp waits for
  // every chunk item in ring order and arrives on its stage's empty barrier
  // (the owner after its work), so that no warp falls two phases behind a
  // stage; a timed-out wait only stops this warp's work.
  bool dead = false;
  uint32_t par = 0u;  // bit s: parity of this group's next item in stage s
#pragma unroll 1
  for (int c = 0; c < s.nW + s.nX; ++c) {
    const int it = seq_of_chunk(s, c);
    const int stage = it % kFStages;
    const uint32_t ph = (par >> stage) & 1u;
    par ^= 1u << stage;
    bool have = false;
    if (!dead) {
      have = __all_sync(kFull, mbar_wait_bounded(&sm.full_attn[stage], ph, p.wait_ns));
      if (!have) {
        dead = true;
        if (lane == 0) {
          sm.abort = 1;
          atomicOr(p.status, HYB_STATUS_TIMEOUT);
        }
      }
    }
    if ((c & 3) != pair) {
      if (lane == 0 && have) mbar_arrive_cnt(&sm.empty[stage], kEmptyPerAttnWarp);
      continue;
    }
    const int4 dsc = sm.desc[stage];
    const int nvalid = have ? dsc.y : 0;
    const uint32_t kb = smem_u32(sm.ring[stage]);
    const uint32_t vb = kb + FusedSmem<D>::kHalf;
    // ---- S^T = K Q^T for this warp's 32 tokens: m-tiles 2 half, 2 half + 1
    // (tokens 32 half .. 32 half + 31), columns = heads.  Both warps of the
    // pair take the same barriers whatever their waits gave (nvalid 0: nothing
    // is computed), so a timed-out wait leaves no warp at a barrier alone.
    float sacc[2][4];
#pragma unroll
    for (int mm = 0; mm < 2; ++mm) sacc[mm][0] = sacc[mm][1] = sacc[mm][2] = sacc[mm][3] = 0.f;
    if (nvalid > 32 * half) {
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {
          const int mt = 2 * half + mm;
          uint32_t a0, a1, a2, a3;
          ldsm_x4(kb + swz<D>(mt * 16 + (mi & 1) * 8 + rr, kk * 2 + (mi >> 1)), a0, a1, a2, a3);
          mma_16816(sacc[mm], a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
        }
      }
    }
    // lane (g, tig): tokens 16mt + g + 8j, columns 2tig, 2tig+1, i.e. heads
    // (2tig, 2tig+1) & 3: softmax weights in lanes tig < 2, Taylor weights
    // 1 + s on selected tokens in lanes tig >= 2.
    const bool sel_tok = dsc.z != 0;
    float w[2][4];
    float t0m = -INFINITY, t1m = -INFINITY;
#pragma unroll
    for (int mm = 0; mm < 2; ++mm)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int t = (2 * half + mm) * 16 + g + 8 * (q >> 1);
        // both kinds of lanes take the same instructions (selects, no
        // divergent branch: half the warp takes each kind)
        const float sv = t < nvalid ? sacc[mm][q] * p.scale : 0.f;
        const float xs = t < nvalid ? sv * kLog2e : -INFINITY;
        const float wt = (t < nvalid && sel_tok) ? 1.f + sv : 0.f;
        w[mm][q] = soft_lane ? xs : wt;
        const float xm = soft_lane ? xs : -INFINITY;
        if (q & 1) t1m = fmaxf(t1m, xm); else t0m = fmaxf(t0m, xm);
      }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      t0m = fmaxf(t0m, __shfl_xor_sync(kFull, t0m, o));
      t1m = fmaxf(t1m, __shfl_xor_sync(kFull, t1m, o));
    }
    // the chunk's column maxima over both warps' tokens
    if (g == 0) sm.xmax[pair][half][tig] = make_float2(t0m, t1m);
    named_sync(kBarPair0 + pair, 64);
    {
      const float2 o = sm.xmax[pair][half ^ 1][tig];
      t0m = fmaxf(t0m, o.x);
      t1m = fmaxf(t1m, o.y);
    }
    const float mn0 = fmaxf(mr0, t0m), mn1 = fmaxf(mr1, t1m);
    const float al0 = (soft_lane && mn0 != -INFINITY) ? exp2f(mr0 - mn0) : 1.f;
    const float al1 = (soft_lane && mn1 != -INFINITY) ? exp2f(mr1 - mn1) : 1.f;
    float ws0 = 0.f, ws1 = 0.f;
#pragma unroll
    for (int mm = 0; mm < 2; ++mm)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float ev = exp2f(w[mm][q] - ((q & 1) ? mn1 : mn0));  // used in the softmax lanes only
        w[mm][q] = soft_lane ? (w[mm][q] == -INFINITY ? 0.f : ev) : w[mm][q];
        if (q & 1) ws1 += w[mm][q]; else ws0 += w[mm][q];
      }
    acc0 = acc0 * al0 + ws0;  // this warp's tokens only: the pair's two sums are added at the end
    acc1 = acc1 * al1 + ws1;
    mr0 = soft_lane ? mn0 : mr0;
    mr1 = soft_lane ? mn1 : mr1;
    // rescale the softmax rows (g < 4) of O by their head's factor
    const float b0 = __shfl_sync(kFull, al0, g >> 1), b1 = __shfl_sync(kFull, al1, g >> 1);
    const float alpha = p_lane ? ((g & 1) ? b1 : b0) : 1.f;
    if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll
      for (int n = 0; n < NH; ++n) {
        O[n][0] *= alpha;
        O[n][1] *= alpha;
        O[n][2] *= alpha;
        O[n][3] *= alpha;
      }
    }
    // A fragments of this warp's two k-tiles (weight columns as rows, transposed
    // 8x8 blocks, hi then lo), handed to the other warp through the first rows
    // of this warp's own K tokens, which nothing reads any more
    uint32_t mf[2][4], of[2][4];  // this warp's k-tiles 2 half + mm, the other warp's
#pragma unroll
    for (int mm = 0; mm < 2; ++mm) {
      uint32_t h0, l0, h1, l1;
      split_bf16(w[mm][0], w[mm][1], h0, l0);
      split_bf16(w[mm][2], w[mm][3], h1, l1);
      mf[mm][0] = movmatrix_t(h0);
      mf[mm][1] = movmatrix_t(l0);
      mf[mm][2] = movmatrix_t(h1);
      mf[mm][3] = movmatrix_t(l1);
    }
    {
      constexpr uint32_t kRows32 = 32u * D * 2u;  // bytes of 32 K rows
      const uint32_t mine_x = kb + (uint32_t)half * kRows32, theirs_x = kb + (uint32_t)(half ^ 1) * kRows32;
#pragma unroll
      for (int mm = 0; mm < 2; ++mm)
        sts_u4(mine_x + (uint32_t)(mm * 512 + lane * 16), mf[mm][0], mf[mm][1], mf[mm][2], mf[mm][3]);
      named_sync(kBarPair0 + pair, 64);
#pragma unroll
      for (int mm = 0; mm < 2; ++mm)
        lds_u4(theirs_x + (uint32_t)(mm * 512 + lane * 16), of[mm][0], of[mm][1], of[mm][2], of[mm][3]);
      // the stage's next copy (async proxy) comes after these generic writes
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    // ---- O += A V over the chunk's 64 tokens.  In a ragged chunk the rows
    // past it have zero weights: k-steps wholly past it are skipped (rows past
    // its 16-row boxes hold stale stage data), and in its last k-step the V
    // fragments of rows past it, which may be unwritten cache rows, are zeroed
    // in registers so that no 0 * NaN arises.
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
      if (kt * 16 >= nvalid) break;
      const bool tail = kt * 16 + 16 > nvalid;  // warp-uniform
      const int tk = kt * 16 + 2 * tig;          // rows of the low halves of b0v / b2v (b1v / b3v: + 8)
      const uint32_t m0 = (tk < nvalid ? 0x0000ffffu : 0u) | (tk + 1 < nvalid ? 0xffff0000u : 0u);
      const uint32_t m1 = (tk + 8 < nvalid ? 0x0000ffffu : 0u) | (tk + 9 < nvalid ? 0xffff0000u : 0u);
      const bool own = (kt >> 1) == half;
      const uint32_t a0 = own ? mf[kt & 1][0] : of[kt & 1][0], a1 = own ? mf[kt & 1][1] : of[kt & 1][1];
      const uint32_t a2 = own ? mf[kt & 1][2] : of[kt & 1][2], a3 = own ? mf[kt & 1][3] : of[kt & 1][3];
#pragma unroll
      for (int np = 0; np < NH / 2; ++np) {
        uint32_t b0v, b1v, b2v, b3v;
        ldsm_x4_t(vb + swz<D>(kt * 16 + (mi & 1) * 8 + rr, (half * NH / 2 + np) * 2 + (mi >> 1)), b0v, b1v, b2v, b3v);
        if (tail) {
          b0v &= m0;
          b1v &= m1;
          b2v &= m0;
          b3v &= m1;
        }
        mma_16816(O[2 * np], a0, a1, a2, a3, b0v, b1v);
        mma_16816(O[2 * np + 1], a0, a1, a2, a3, b2v, b3v);
      }
    }
    __syncwarp();
    if (lane == 0 && have) mbar_arrive_cnt(&sm.empty[stage], kEmptyPerAttnWarp);
  }

  // each warp of a pair summed the weights of its own tokens: add the other's
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    acc0 += __shfl_xor_sync(kFull, acc0, o);
    acc1 += __shfl_xor_sync(kFull, acc1, o);
  }
  if (g == 0) sm.xmax[pair][half][tig] = make_float2(acc0, acc1);
  named_sync(kBarPair0 + pair, 64);
  {
    const float2 o = sm.xmax[pair][half ^ 1][tig];
    acc0 += o.x;
    acc1 += o.y;
  }
  // the combine slots hold the top-k candidates until the selection is made
  // (a rank without selected chunks gets here first)
  if (!dead) mbar_wait_bounded(&sm.sel_bar, 0, p.wait_ns);
  // ---- combine the 4 pairs' partials (a tree through two shared slots: pairs
  //      2, 3 -> 0, 1, then pair 1 -> 0); pair 0 leaves the record in wpart[0].
  //      The two warps of a pair hold the same statistics and disjoint columns.
  // each lane takes the statistics of its O rows' head (rows g < 4 softmax,
  // g >= 4 Taylor); the per-head totals are in every lane of a tig
  float m_run, l, ds;
  {
    const int src = p_lane ? (head >> 1) : 2 + (head >> 1);
    const float v0 = __shfl_sync(kFull, acc0, src), v1 = __shfl_sync(kFull, acc1, src);
    const float m0 = __shfl_sync(kFull, mr0, head >> 1), m1 = __shfl_sync(kFull, mr1, head >> 1);
    const float v = (head & 1) ? v1 : v0;
    m_run = (head & 1) ? m1 : m0;
    l = p_lane ? v : 0.f;
    ds = p_lane ? 0.f : v;
  }
  const int voff = (p_lane ? 0 : 4 * D) + head * D + half * (D / 2);
  auto emit = [&](float* wp) {  // write this warp's partial (hi + lo rows summed)
    if (tig == 0 && half == 0) {
      if (p_lane) {
        wp[head] = m_run;
        wp[4 + head] = l;
      } else {
        wp[8 + head] = ds;
      }
    }
    float* dst = wp + 16 + voff;
#pragma unroll
    for (int n = 0; n < NH; ++n)
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
    for (int n = 0; n < NH; ++n) {
      const float2 y = *reinterpret_cast<const float2*>(src + n * 8 + 2 * tig);
      O[n][0] = (O[n][0] + O[n][2]) * fa + y.x * fb;
      O[n][1] = (O[n][1] + O[n][3]) * fa + y.y * fb;
      O[n][2] = O[n][3] = 0.f;
    }
  };
  if (pair >= 2) emit(sm.wpart[pair - 2]);
  named_sync(kBarAttn, kAttnThreads);
  if (pair < 2) absorb(sm.wpart[pair]);
  named_sync(kBarAttn, kAttnThreads);
  if (pair == 1) emit(sm.wpart[0]);
  named_sync(kBarAttn, kAttnThreads);
  if (pair == 0) {
    absorb(sm.wpart[0]);
    named_sync(kBarPair0, 64);  // both warps have read the statistics before half 0 rewrites them
    emit(sm.wpart[0]);
  }
}

}  // namespace
}  // namespace hyb

namespace hyb {
namespace {

// Statistics warps (roles 8-10): score items, one warp per item (item i to warp
// i % 3); hand the scores to every rank; the selection; H items (rows split
// between the warps); the rank's linear partial.  Every statistics warp waits for every
// statistics item in ring order and arrives once on its stage's empty barrier
// (the owner after its work), so that no warp falls two phases behind a stage.
template <int D, bool kStream>
__device__ void aux_role(const FusedParams& p, const UnitGeo& g, FusedSmem<D>& sm, const Seq& s, int unit, int rank) {
  constexpr int CPL = D / 32;
  const int a = role_tid() - kAttnThreads, aw = a >> 5, lane = a & 31;
  // a timed-out wait only stops this warp's work; it keeps visiting every item
  // and barrier
  bool dead = false;
  uint32_t par = 0u;  // bit s: parity of this group's next item in stage s (items come in order)
  auto wait_item = [&](int it) -> bool {
    const int stage = it % kFStages;
    const uint32_t ph = (par >> stage) & 1u;
    par ^= 1u << stage;
    if (dead) return false;
    const bool have = __all_sync(kFull, mbar_wait_bounded(&sm.full_aux[stage], ph, p.wait_ns));
    if (!have) {
      dead = true;
      if (lane == 0) {
        sm.abort = 1;
        atomicOr(p.status, HYB_STATUS_TIMEOUT);
      }
    }
    return have;
  };
  const int64_t nf = g.fold_end - g.fold_begin;
  // rank 0's zk, zv and n, needed after the last H item: loaded now, so that
  // their round trip is not on the path at the end
  float zk0[kAuxCols<D>], zv0[kAuxCols<D>], n0 = 0.f;
#pragma unroll
  for (int k = 0; k < kAuxCols<D>; ++k) {
    const int c = a + k * kAuxThreads;
    const bool ld = rank == 0 && c < D;
    zk0[k] = ld ? p.zk[(int64_t)unit * D + c] : 0.f;
    zv0[k] = ld ? p.zv[(int64_t)unit * D + c] : 0.f;
  }
  if (rank == 0) n0 = p.n[unit];
  if (p.q != nullptr)
    for (int c = a; c < D; c += kAuxThreads) {
      float q1 = 0.f, q2 = 0.f;
      for (int i = 0; i < p.G; ++i) {
        const float qv = sm.qs[i][c];
        q1 += qv;
        q2 += 0.5f * qv * qv;
      }
      sm.qsum[0][c] = q1;
      sm.qsum[1][c] = q2;
    }
  named_sync(kBarAux, kAuxThreads);
  cluster_wait();  // every rank's barriers are initialised: remote operations are allowed from here on
  int fold_i0, fold_i1;
  fold_items<D>(p, g, s, &fold_i0, &fold_i1);
  const bool stream = stream_topk<D, kStream>(p, g);
  unsigned long long run = 0ull;  // this warp's 32 largest packed keys so far (streaming top-k)
  bool nan = false;
#pragma unroll 1
  for (int idx = 0; idx < s.nS; ++idx) {
    const int it = seq_of_s(s, idx), stage = it % kFStages;
    const bool have = wait_item(it);
    if (have && idx % kAuxWarps == aw) {
      if (p.q != nullptr) score_item_warp<D>(p, g, sm, s, unit, idx, stage);
      if (idx >= fold_i0 && idx < fold_i1) fold_score_item<D>(p, g, sm, s, unit, idx, stage);
      __syncwarp();
      if constexpr (kStream) {
        if (stream) {  // the item's final scores (after any fold) into the warp's list
          const int j = s.b0 + idx * Geo<D>::kBlocks + lane;
          run = topk_offer(run, j < s.b1 ? sm.scores[j] : 0.f, j, j < s.b1, lane, nan);
        }
      }
    }
    if (lane == 0 && have) mbar_arrive_cnt(&sm.empty[stage], kEmptyPerAuxWarp);
  }
  named_sync(kBarAux, kAuxThreads);  // every score of this rank is in place
  // test hook: rank 1 withholds its hand-off, so that the other ranks' bounded
  // wait for it runs out (nothing else ever skips it)
  const bool withhold = (p.test_flags & HYB_TEST_WITHHOLD_SCORES) != 0u && rank == 1;
  if (stream) {
    // this rank's top-k: the three warps' lists merged by warp 0 into the
    // rank's slot of the exchange, then bulk-copied into every other rank's
    // copy of that slot
    unsigned long long* lists = reinterpret_cast<unsigned long long*>(sm.hist);  // 2 x 32 entries
    if (aw > 0) lists[(aw - 1) * 32 + lane] = run;
    nan = __any_sync(kFull, nan);
    if (lane == 0) sm.tk[4 + aw] = nan ? 1u : 0u;
    named_sync(kBarAux, kAuxThreads);
    const int k = g.k_eff, kslot = cand_slot(k);
    unsigned long long* all = reinterpret_cast<unsigned long long*>(&sm.wpart[0][0]);
    if (aw == 0) {
      run = warp_merge_desc(run, lists[lane], lane);
      run = warp_merge_desc(run, lists[32 + lane], lane);
      if (lane < kslot) all[rank * kslot + lane] = lane < k ? run : 0ull;
      if (lane == 0 && (sm.tk[4] | sm.tk[5] | sm.tk[6]) != 0u) atomicOr(p.status, HYB_STATUS_NAN_SCORE);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    named_sync(kBarAux, kAuxThreads);
    if (a == 0 && !withhold) {
      const uint32_t src = smem_u32(all + rank * kslot), bar = smem_u32(&sm.scores_bar);
      for (int rr = 0; rr < p.C; ++rr)
        if (rr != rank) bulk_push(map_rank(src, (uint32_t)rr), src, (uint32_t)(kslot * 8), map_rank(bar, (uint32_t)rr));
    }
  } else if (runs_topk(p, g)) {  // hand this rank's scores to every rank
    if (g.nb <= FusedSmem<D>::kGather) {
      // bulk copies of the share into every other rank's scores array
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      named_sync(kBarAux, kAuxThreads);
      if (a == 0 && s.b1 > s.b0 && !withhold) {
        const uint32_t bytes = (uint32_t)(((s.b1 - s.b0) * 4 + 15) & ~15);
        const uint32_t src = smem_u32(&sm.scores[s.b0]), bar = smem_u32(&sm.scores_bar);
        for (int rr = 0; rr < p.C; ++rr)
          if (rr != rank) bulk_push(map_rank(src, (uint32_t)rr), src, bytes, map_rank(bar, (uint32_t)rr));
      }
    } else {
      // the scores went to global memory: release them at cluster scope
      asm volatile("fence.acq_rel.cluster;" ::: "memory");
      named_sync(kBarAux, kAuxThreads);
      if (a == 0) {
        const uint32_t la = smem_u32(&sm.scores_bar);
        for (int rr = 0; rr < p.C; ++rr) remote_arrive(map_rank(la, (uint32_t)rr));
      }
    }
  }

  if (p.q != nullptr) aux_select<D, kStream>(p, g, sm, unit, rank);
  float hacc[kMaxGroup][CPL];
#pragma unroll
  for (int i = 0; i < kMaxGroup; ++i)
#pragma unroll
    for (int c = 0; c < CPL; ++c) hacc[i][c] = 0.f;
#pragma unroll 1
  for (int idx = 0; idx < s.nH; ++idx) {
    const int it = seq_of_h(s, idx), stage = it % kFStages;
    const bool have = wait_item(it);
    if (have && (p.q != nullptr || nf > 0)) aux_h_item<D>(p, g, sm, s, unit, idx, stage, hacc);
    __syncwarp();
    if (lane == 0 && have) mbar_arrive_cnt(&sm.empty[stage], kEmptyPerAuxWarp);
  }
  aux_finish_linear<D>(p, g, sm, unit, rank, hacc, zk0, zv0, n0);
}

// Producer (role warp 11, lane 0): every copy of the rank, in ring order, one
// short loop per kind of item with running addresses.  Before an item goes into
// a stage that held an earlier item, the stage's empty barrier must have
// completed for that earlier item.
template <int D>
__device__ void producer_role(const KVMaps* tm, const FusedParams& p, const UnitGeo& g, FusedSmem<D>& sm, const Seq& s,
                              int unit, int rank) {
  if ((threadIdx.x & 31) != 0) return;
  constexpr int RB = Geo<D>::kBlocks, RH = Geo<D>::kRows;
  const uint64_t pol = l2_evict_first();  // every copy of the ring streams data read once per launch
  int stage = 0, issued = 0;
  uint32_t epar = 0u;                  // per stage: parity of the next empty-barrier phase to wait for
  uint32_t fpar_aux = 0u, fpar_at = 0u;  // per stage: parity of the next full-barrier phase of each group
  uint32_t last_aux = 0u;              // per stage: the last item issued into it was a statistics item
  bool ok = true;
  auto acquire = [&]() -> bool {
    if (issued >= kFStages) {
      const uint32_t ph = (epar >> stage) & 1u;
      epar ^= 1u << stage;
      if (!mbar_wait_bounded(&sm.empty[stage], ph, p.wait_ns)) {
        atomicOr(p.status, HYB_STATUS_TIMEOUT);
        sm.abort = 1;
        return false;
      }
    }
    return *(volatile int*)&sm.abort == 0;
  };
  auto advance = [&](bool aux) {
    if (aux) {
      fpar_aux ^= 1u << stage;
      last_aux |= 1u << stage;
    } else {
      fpar_at ^= 1u << stage;
      last_aux &= ~(1u << stage);
    }
    ++issued;
    stage = stage + 1 == kFStages ? 0 : stage + 1;
  };
  // score items: the mean and variance rows of RB blocks
  const int64_t brow = (int64_t)unit * p.max_blocks + s.b0;
  for (int i = 0; i < s.nS && ok; ++i) {
    if (!(ok = acquire())) break;
    uint64_t* bar = &sm.full_aux[stage];
    if (p.q != nullptr || score_item_folds<D>(p, g, s, i)) {
      const uint32_t dst = smem_u32(sm.ring[stage]);
      const uint32_t bytes = (uint32_t)(min(RB, s.b1 - s.b0 - i * RB) * D * 4);
      const int64_t off = (brow + (int64_t)i * RB) * D;
      mbar_arrive_expect_tx(bar, 2 * bytes);
      bulk_load_stream(dst, p.mu + off, bytes, bar, pol);
      bulk_load_stream(dst + RB * D * 4, p.var + off, bytes, bar, pol);
    } else {
      mbar_arrive(bar);
    }
    advance(true);
  }
  // window (and sink) chunks: chunk ci = rank + i C of the exact prefix
  const int64_t ubase = (int64_t)unit * p.cap;
  for (int i = 0, ci = rank; i < s.nW && ok; ++i, ci += p.C) {
    if (!(ok = acquire())) break;
    int start, len;
    if (ci < g.n_sink_chunks) {
      start = ci * kTile;
      len = min(kTile, g.sink_len - start);
    } else {
      start = g.win_start + (ci - g.n_sink_chunks) * kTile;
      len = min(kTile, g.T - start);
    }
    issue_chunk<D>(tm, sm, stage, ubase, start, len, 0, pol);
    advance(false);
  }
  // H items: RH rows of H
  const bool h_load = p.q != nullptr || g.fold_end > g.fold_begin;
  for (int i = 0; i < s.nH && ok; ++i) {
    if (!(ok = acquire())) break;
    uint64_t* bar = &sm.full_aux[stage];
    if (h_load) {
      const int r0 = s.h0 + i * RH;
      const uint32_t bytes = (uint32_t)(min(RH, s.h1 - r0) * D * 4);
      mbar_arrive_expect_tx(bar, bytes);
      bulk_load_stream(smem_u32(sm.ring[stage]), p.H + ((int64_t)unit * D + r0) * D, bytes, bar, pol);
    } else {
      mbar_arrive(bar);
    }
    advance(true);
  }
  // selected chunks: chunk sc = rank + i C is piece sc % cpb of selection slot sc / cpb
  if (ok && s.nX > 0 && !mbar_wait_bounded(&sm.sel_bar, 0, p.wait_ns)) {
    atomicOr(p.status, HYB_STATUS_TIMEOUT);
    sm.abort = 1;
    ok = false;
  }
  const int cpb = p.chunks_per_block;
  int slot = rank / cpb, piece = rank - (rank / cpb) * cpb;
  const int st = sm.sel_state;
  for (int i = 0; i < s.nX && ok; ++i) {
    if (!(ok = acquire())) break;
    int jb = -1;
    if (slot < g.k_eff) jb = st == 3 ? slot : st == 1 ? sm.sel_cache[slot] : __ldcg(sm.sel_row + slot);
    int start = 0, len = 0;
    if (jb >= 0 && jb < g.nb) {
      const int bs = p.S + jb * p.Bk;
      start = bs + piece * kTile;
      len = max(0, min(kTile, min(bs + p.Bk, g.ev_end) - start));
    } else if (jb != -1) {
      atomicOr(p.status, HYB_STATUS_BAD_SELECTION);
    }
    issue_chunk<D>(tm, sm, stage, ubase, start, len, 1, pol);
    advance(false);
    if (cpb == 1) {
      slot += p.C;
    } else {
      piece += p.C;
      slot += piece / cpb;
      piece -= (piece / cpb) * cpb;
    }
  }
  if (*(volatile int*)&sm.abort) {
    // do not leave while copies into this CTA's ring may be in flight: wait for
    // the last item issued into each stage (its group's full barrier, its phase);
    // every issued item completes, so this wait keeps the long default limit
    // whatever limit the progress waits have
    for (int j = 0; j < kFStages && j < issued; ++j) {
      const bool aux = (last_aux >> j) & 1u;
      const uint32_t ph = (((aux ? fpar_aux : fpar_at) >> j) & 1u) ^ 1u;  // parity of the last item's phase
      mbar_wait_bounded(aux ? &sm.full_aux[j] : &sm.full_attn[j], ph, kWaitLimit);
    }
  }
}

// Every rank, all threads, once its record (the attention partials of its
// chunks: per head the running max, the weight sums of the exact part and of
// the selected tokens' Taylor terms, and their weighted value sums) and its
// linear partial are final.  Rank r merges outputs [e0(r), e1(r)) of the
// unit's G x D; every rank sends it a header (per head: max, exact weight sum,
// and its share of D_glob - D_sel) and, per output of the slice, its exact
// partial and its share of N_glob - N_sel (the merge needs only those sums).
// Remote parts go by st.async into the receiver's mrecv, completing bytes on
// its merge barrier; the rank's own part is stored locally.
template <int D>
__device__ __forceinline__ void merge_push(const FusedParams& p, FusedSmem<D>& sm, int rank) {
  const int tid = threadIdx.x;
  const int G = p.G, C = p.C, GD = G * D;
  const int stride = p.mstride;
  const float* rec = sm.wpart[0];
  const uint32_t recv0 = smem_u32(sm.mrecv), bar0 = smem_u32(&sm.merge_bar);
  const int hr = tid - (kFThreads - C);  // the last C threads (the fewest outputs): the header for rank hr
  if (hr >= 0) {
    float h[12];
#pragma unroll
    for (int i = 0; i < kMaxGroup; ++i) {
      h[i] = rec[i];
      h[4 + i] = rec[4 + i];
      h[8 + i] = (rank == 0 && i < G ? sm.linp[i][D] : 0.f) - rec[8 + i];
    }
    const int off = rank * stride;
    if (hr == rank) {
#pragma unroll
      for (int k = 0; k < 12; ++k) sm.mrecv[off + k] = h[k];
    } else {
      const uint32_t dst = map_rank(recv0 + 4u * (uint32_t)off, (uint32_t)hr), bar = map_rank(bar0, (uint32_t)hr);
      st_async_v4(dst, h[0], h[1], h[2], h[3], bar);
      st_async_v4(dst + 16u, h[4], h[5], h[6], h[7], bar);
      st_async_v4(dst + 32u, h[8], h[9], h[10], h[11], bar);
    }
  }
  for (int e = tid; e < GD; e += kFThreads) {
    const int r = ((e + 1) * C - 1) / GD;  // the rank that merges output e: mslice[r] <= e < mslice[r + 1]
    const int i = e / D, d = e - i * D;
    const float xa = rec[16 + e], xd = sm.linp[i][d] - rec[16 + 4 * D + e];
    const int off = rank * stride + 16 + 2 * (e - p.mslice[r]);  // this rank's slot in rank r's buffer
    if (r == rank)
      *reinterpret_cast<float2*>(&sm.mrecv[off]) = make_float2(xa, xd);
    else
      st_async_v2(map_rank(recv0 + 4u * (uint32_t)off, (uint32_t)r), xa, xd, map_rank(bar0, (uint32_t)r));
  }
}

// Rank r's merge of its slice from the C slots of mrecv (after its merge
// barrier), one output per thread: per head the global max M over ranks, each
// rank's exact part rescaled by 2^(m_r - M); out = (N_ex + 2^-M (N_glob - N_sel))
// / (D_ex + 2^-M (D_glob - D_sel)), scaled by 2^M or 2^-M, whichever keeps it finite.
template <int D>
__device__ void merge_local(const FusedParams& p, FusedSmem<D>& sm, int unit, int rank) {
  const int tid = threadIdx.x;
  const int G = p.G, C = p.C;
  const int stride = p.mstride;
  // every thread waits; the outcome is made uniform so that all or none merge.
  // Every rank pushes its parts whatever happened before, so this wait keeps
  // the long default limit (no rank leaves with another's stores in flight)
  if (!__syncthreads_and(wait_cluster_bounded(&sm.merge_bar, 0, kWaitLimit))) {
    if (tid == 0) atomicOr(p.status, HYB_STATUS_TIMEOUT);
    return;
  }
  uint32_t flags = 0u;
  const int e0 = p.mslice[rank], e1 = p.mslice[rank + 1];
  for (int e = e0 + tid; e < e1; e += kFThreads) {
    const int i = e / D;
    const float* h = sm.mrecv + i;
    float M = -INFINITY;
#pragma unroll 2
    for (int r = 0; r < C; ++r) M = fmaxf(M, h[r * stride]);
    if (M == -INFINITY) M = 0.f;
    float nex = 0.f, nsub = 0.f, Dex = 0.f, Dsub = 0.f;
#pragma unroll 2
    for (int r = 0; r < C; ++r) {
      const float m = h[r * stride];
      const float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
      const float2 v = *reinterpret_cast<const float2*>(&sm.mrecv[r * stride + 16 + 2 * (e - e0)]);
      nex += v.x * f;
      nsub += v.y;
      Dex += h[r * stride + 4] * f;
      Dsub += h[r * stride + 8];
    }
    float num, den;
    if (M >= 0.f) {
      const float f = exp2f(-M);
      num = nex + f * nsub;
      den = Dex + f * Dsub;
    } else {
      const float f = exp2f(M);
      num = nex * f + nsub;
      den = Dex * f + Dsub;
    }
    const float o = num / den;
    p.out[(int64_t)unit * G * D + e] = o;
    if (!(den > 0.f)) flags |= HYB_STATUS_DENOMINATOR;
    if (!isfinite(o)) flags |= HYB_STATUS_NONFINITE;
  }
  if (flags) atomicOr(p.status, flags);
}

template <int D, bool kTab, bool kStream>
__global__ void __launch_bounds__(kFThreads, 1) fused_kernel(const __grid_constant__ KVMaps tm, const FusedParams p,
                                                             const __grid_constant__ TabArg<kTab> ta) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned (the 128-byte swizzle repeats every 1024 bytes); offsetting
  // the shared array keeps every access through `sm` in the shared space
  FusedSmem<D>& sm = *reinterpret_cast<FusedSmem<D>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = role_tid() >> 5;
  const int rank = (int)cluster_rank();
  const int unit = blockIdx.x / p.C;
  // this unit's row length, budget and fold range (every thread, in registers;
  // the roles read the copy thread 0 leaves in shared memory)
  const UnitTables* tbl = nullptr;
  if constexpr (kTab) tbl = &ta.tb;
  const UnitGeo g0 = unit_geo(tbl, unit, p.Hkv, p.T, p.S, p.W, p.Bk, p.top_k, p.chunks_per_block, p.pending);
  const Seq s = make_seq<D>(p, g0, rank);
  if (warp == kProducerWarp && (tid & 31) == 0) {
    // Before the wait for the previous grid (which may still be running):
    // the rank's block statistics, its first items, are prefetched into L2.
    // L2 is the point of coherence, so a line the previous grid still writes
    // is updated there; nothing enters this CTA before the wait.
    if (s.b1 > s.b0) {
      const int64_t off = ((int64_t)unit * p.max_blocks + s.b0) * D;
      const int64_t bytes = (int64_t)(s.b1 - s.b0) * D * 4;
      for (int64_t o = 0; o < bytes; o += 32768) {
        const uint32_t n = (uint32_t)(bytes - o < 32768 ? bytes - o : 32768);
        bulk_prefetch_l2(reinterpret_cast<const char*>(p.mu + off) + o, n);
        bulk_prefetch_l2(reinterpret_cast<const char*>(p.var + off) + o, n);
      }
    }
  }
  if (tid == 0) {
    tma_prefetch_desc(&tm.k64);
    tma_prefetch_desc(&tm.v64);
    for (int i = 0; i < kFStages; ++i) {
      mbar_init(&sm.full_attn[i], 1);
      mbar_init(&sm.full_aux[i], 1);
      mbar_init(&sm.empty[i], kEmptyCount);
    }
    // scores_bar: the other ranks' shares arriving by bulk copy (one local
    // arrival expecting their bytes), or C arrivals when the scores go
    // through global memory
    sm.geo = g0;
    const bool stream = stream_topk<D, kStream>(p, g0);
    const bool push = runs_topk(p, g0) && g0.nb <= FusedSmem<D>::kGather;
    mbar_init(&sm.scores_bar, push ? 1 : p.C);
    mbar_init(&sm.sel_bar, 1);
    mbar_init(&sm.merge_bar, 1);
    sm.sel_state = 3;
    sm.sel_row = nullptr;
    sm.abort = 0;
    fence_mbar_init();
    if (stream) {  // the other ranks' candidate slots
      mbar_arrive_expect_tx(&sm.scores_bar, (uint32_t)((p.C - 1) * cand_slot(g0.k_eff) * 8));
    } else if (push) {  // the other ranks' shares of the scores
      uint32_t bytes = 0;
      for (int rr = 0; rr < p.C; ++rr) {
        int b0, b1;
        block_share(g0.nb, p.C, rr, b0, b1);
        if (rr != rank) bytes += (uint32_t)(((b1 - b0) * 4 + 15) & ~15);
      }
      mbar_arrive_expect_tx(&sm.scores_bar, bytes);
    }
    if (p.q != nullptr)  // the other ranks' headers and pieces of this rank's slice
      mbar_arrive_expect_tx(&sm.merge_bar, (uint32_t)((p.C - 1) * (48 + 8 * (p.mslice[rank + 1] - p.mslice[rank]))));
    pdl_wait_primary();  // everything below reads what earlier grids wrote
  }
  // This CTA's barriers are initialised and every thread is ordered after the
  // wait for the previous grid.  The cluster barrier is split: the arrival
  // here (the barrier initialisations are released to the cluster by their
  // fence), the wait before a thread's first remote operation (the
  // statistics warps' score push) or after its role, so that the ring's
  // first copies do not wait for the other ranks.
  __syncthreads();
  cluster_arrive_relaxed();
  pdl_allow_dependents();
  const UnitGeo& g = sm.geo;
  if (warp == kProducerWarp) {
    // the producer starts at once: it needs nothing from the lines below
    producer_role<D>(&tm, p, g, sm, s, unit, rank);
    cluster_wait();
  } else {
    const int t = role_tid();  // 0 .. kConsumerThreads - 1
    // The prologue's global loads: one 16-byte load per thread, all issued
    // before any of them is used, so that none waits behind the ring's first
    // copies (a load issued after them waits for most of the start-up burst).
    // Threads [0, QV): q; [QV, QV + D/4): the pending token's K and V rows;
    // [QV + D/4, QV + D/2): the decode's appended token (rank 0).
    constexpr int QV = kMaxGroup * D / 8;
    static_assert(QV + D / 2 <= kConsumerThreads, "one 16-byte piece per thread");
    const int tr = t - QV, ta = t - QV - D / 4;
    const bool ld_q = p.q != nullptr && t < QV && t * 8 < p.G * D;
    const bool ld_row = g.fold_end - g.fold_begin == 1 && tr >= 0 && tr < D / 4;
    const bool ld_new = p.k_new != nullptr && rank == 0 && ta >= 0 && ta < D / 4;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (ld_q) {
      raw = __ldg(reinterpret_cast<const uint4*>(p.q + (int64_t)unit * p.G * D) + t);
    } else if (ld_row) {
      const int e = (tr % (D / 8)) * 8;
      raw = __ldg(reinterpret_cast<const uint4*>((tr >= D / 8 ? p.v_cache : p.k_cache) +
                                                 ((int64_t)unit * p.cap + g.fold_begin) * D + e));
    } else if (ld_new) {
      const int e = (ta % (D / 8)) * 8;
      raw = __ldg(reinterpret_cast<const uint4*>((ta >= D / 8 ? p.v_new : p.k_new) + (int64_t)unit * D + e));
    }
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
    if (p.q != nullptr && t < QV) {  // heads past G stay zero
      const int i = t * 8 / D, d0 = (t * 8) % D;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h2[j]);
        const float q0 = f.x * p.scale, q1 = f.y * p.scale;
        sm.qs[i][d0 + 2 * j] = sm.qsT[d0 + 2 * j][i] = q0;
        sm.qs[i][d0 + 2 * j + 1] = sm.qsT[d0 + 2 * j + 1][i] = q1;
      }
    } else if (ld_row) {  // the pending token's rows, for the folds
      float* dst = (tr >= D / 8 ? sm.vtok : sm.ktok) + (tr % (D / 8)) * 8;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h2[j]);
        dst[2 * j] = f.x;
        dst[2 * j + 1] = f.y;
      }
    } else if (ld_new) {  // the decode's appended token: row T of the caches
      const int e = (ta % (D / 8)) * 8;
      *reinterpret_cast<uint4*>((ta >= D / 8 ? p.v_cache : p.k_cache) + ((int64_t)unit * p.cap + g.T) * D + e) = raw;
    }
    named_sync(kBarConsumers, kConsumerThreads);
    if (warp < kAttnWarps) {
      if (p.q != nullptr) attn_role<D>(p, sm, s, unit);
      cluster_wait();
    } else {
      aux_role<D, kStream>(p, g, sm, s, unit, rank);  // waits on the cluster barrier before its score push
    }
  }
  __syncthreads();  // this rank's record and linear partial are final; its ring is idle
  if (p.q != nullptr) merge_push<D>(p, sm, rank);
  cluster_arrive_relaxed();  // the merge's data is ordered by the merge barriers
  if (p.q != nullptr) merge_local<D>(p, sm, unit, rank);
  cluster_wait();  // no CTA leaves the cluster before every rank has sent its parts
}

}  // namespace

static_assert(sizeof(FusedSmem<128>) + 1024 <= 232448, "shared memory per CTA");
static_assert(sizeof(FusedSmem<64>) + 1024 <= 232448, "shared memory per CTA");

size_t fused_smem_bytes(int D) {
  return (D == 128 ? sizeof(FusedSmem<128>) : sizeof(FusedSmem<64>)) + 1024;
}

template <int D, bool kTab, bool kStream>
cudaError_t set_fused_attributes() {
  const void* f = (const void*)fused_kernel<D, kTab, kStream>;
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fused_smem_bytes(D));
  if (e == cudaSuccess) e = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  return e;
}

template <int D>
cudaError_t set_fused_attributes_all() {
  cudaError_t e = set_fused_attributes<D, false, false>();
  if (e == cudaSuccess) e = set_fused_attributes<D, true, false>();
  if (e == cudaSuccess) e = set_fused_attributes<D, false, true>();
  if (e == cudaSuccess) e = set_fused_attributes<D, true, true>();
  return e;
}

cudaError_t prepare_fused(int D) { return D == 128 ? set_fused_attributes_all<128>() : set_fused_attributes_all<64>(); }

int fused_max_clusters(int D, int c) {
  // both variants have the same shared memory and block size
  const void* f = D == 128 ? (const void*)fused_kernel<128, false, false> : (const void*)fused_kernel<64, false, false>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = fused_smem_bytes(D);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = c;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, f, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

template <int D, bool kTab, bool kStream>
cudaError_t launch_variant(const cudaLaunchConfig_t* cfg, const KVMaps& tm, const FusedParams& p, const TabArg<kTab>& ta) {
  return cudaLaunchKernelEx(cfg, fused_kernel<D, kTab, kStream>, tm, p, ta);
}

template <int D>
cudaError_t launch_d(const cudaLaunchConfig_t* cfg, const KVMaps& tm, const FusedParams& p, const UnitTables& tb,
                     bool stream) {
  if (tb.ragged || tb.per_head) {
    TabArg<true> ta;
    ta.tb = tb;
    return stream ? launch_variant<D, true, true>(cfg, tm, p, ta) : launch_variant<D, true, false>(cfg, tm, p, ta);
  }
  const TabArg<false> none;
  return stream ? launch_variant<D, false, true>(cfg, tm, p, none) : launch_variant<D, false, false>(cfg, tm, p, none);
}

cudaError_t launch_fused(const CUtensorMap* maps, const FusedParams& p, const UnitTables& tb, bool stream, int D,
                         cudaStream_t s) {
  KVMaps tm;
  tm.k64 = maps[0];
  tm.v64 = maps[1];
  tm.k16 = maps[2];
  tm.v16 = maps[3];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.units * p.C));
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = fused_smem_bytes(D);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return D == 128 ? launch_d<128>(&cfg, tm, p, tb, stream) : launch_d<64>(&cfg, tm, p, tb, stream);
}

}  // namespace hyb
