// Multi-query decode: NR consecutive new tokens of every unit in one launch
// (speculative verification of a draft of NR tokens, or a prefill chunk that
// wants every token's output).  Row r is the decode at length T + r -- the
// history and the chunk's tokens 0 .. r-1 -- with its own window, its own
// block statistics, scores and top-k, and its own linear remainder, exactly as
// NR single-token decode + append steps would compute it ("SALSA:
// Training-Consistent Sparse Caching with Sink Preservation for Linearized
// LLMs", abstract: sinks + window + sparse cache + linear state; "SPLA: Block
// Sparse Plus Linear Attention for Long Context Modeling", Abstract: Taylor
// block selection and residual linear attention by subtraction; "SLAKE",
// Abstract: first-order Taylor kernel).  What the rows share is read once:
//
//   the prefix: sinks [0, min(S, T_last)) and the last row's window
//     [pre_win, T_last), T_last = T + NR - 1 (row r's window lies in it, minus
//     the E part below, and row r sees the tokens before T + r);
//   the E part [ev0, pre_win), ev0 = T - W (row 0's eviction edge): at most
//     NR - 1 tokens that later rows have evicted but that are not in the folded
//     state; for row r a token there is exact when it is in row r's window or
//     in a block row r selected, else it takes the Taylor weight 1 + s added to
//     the linear part;
//   the union of the rows' selected blocks, clipped to the state range
//     [S, ev0): for each row that selected a block, exact weights and the
//     block's own (1 + s) terms subtracted from the global state.
//
// The block statistics of the blocks the E tokens fall into differ by row
// (Welford's running mean / variance extended by the row's E tokens, not
// stored); every other block's statistics are shared.  The global state
// (H, zk, zv, n) is folded to ev0 once (the evictions pending from earlier
// calls) and shared by all rows.
//
// Grid and roles as the single-token decode kernel (k_fused.cu): one cluster of
// C CTAs per unit, 8 attention warps in 4 pairs, 3 statistics warps, 1 producer
// lane, a ring of kMStages stages.  The prefix chunks take no Taylor weights, so
// a pair runs two rows on them at once: the 8 mma N columns are rows (a, a + 1)
// x 4 heads, all exact (NR = 2: every pair rows 0, 1, a quarter of the chunks
// each; NR = 4: pairs 0, 1 rows 0, 1 and pairs 2, 3 rows 2, 3, alternate
// chunks).  After the prefix a pair leaves its partial in its combine slot and
// takes one row, with the single-token layout (4 exact + 4 Taylor columns), for
// the E and selected chunks (NR = 2: pairs 0, 1 row 0 and pairs 2, 3 row 1,
// alternate chunks; NR = 4: pair r row r, every chunk that row r selected).
// Selections are made per row by the statistics warps (one warp per row, as
// the single-token kernel does), and the merge covers NR x G x D outputs.
// Every wait is bounded.
#include "k_common.cuh"

namespace hyb {
namespace {

constexpr int kMStages = 4;
constexpr int kMScores = 4096;  // NR rows x stride of block scores in shared memory
// tokens the launch reads from the caches one by one: the pending evictions
// [fold_begin, fold_end) (at most 4: more are folded by the dense fold first)
// and the rows' E tokens after them (at most NR - 1 = 3); staged in shared
// memory by the prologue
constexpr int kMaxPend = 4, kMaxX = 8;
static_assert(kMaxPend >= kFoldKernelMin - 1 && kMaxX >= kMaxPend + 3, "staged token rows");

// merge slot: per row a 16-float header (per head: max, exact weight sum,
// D_glob - D_sel), then (exact part, N_glob - N_sel) pairs of the slice
__host__ __device__ constexpr int mmerge_stride(int NR, int GD, int C) {
  return 16 * NR + ((2 * ((NR * GD + C - 1) / C) + 3) & ~3);
}
__host__ __device__ constexpr int mmerge_floats_for(int NR, int D, int C) { return C * mmerge_stride(NR, kMaxGroup * D, C); }
// at most 8 CTAs per unit (the merge slots of larger clusters would take the
// shared memory of the attention pairs' exchange buffers)
constexpr int kMultiMaxCluster = 8;
__host__ __device__ constexpr int mmerge_floats(int NR, int D, int C = 1) {
  return C > kMultiMaxCluster ? 0
                         : (mmerge_floats_for(NR, D, C) > mmerge_floats(NR, D, C + 1) ? mmerge_floats_for(NR, D, C)
                                                                                       : mmerge_floats(NR, D, C + 1));
}

template <int NR>
struct MultiGeo {   // the rows' shared and per-row geometry (row 0 is the unit's UnitGeo)
  int32_t T_last;                    // T + NR - 1: the last row's length
  int32_t pre_sink, pre_win;         // prefix: [0, pre_sink) and [pre_win, T_last)
  int32_t e0, e1;                    // E part [e0, e1)
  int32_t n_sink_chunks, n_win_chunks, n_e_chunks;
  int32_t nb_max, sstride;           // blocks of the last row; score row stride
  int32_t win_start[NR], ev_end[NR], nb[NR], k_eff[NR];
};

template <int D, int NR>
struct MultiSmem {
  static constexpr int kHalf = kTile * D * 2;
  static constexpr int kStageBytes = 2 * kHalf;
  static constexpr int kBoxBytes = kBoxRows * D * 2;
  static constexpr int kPF = partial_floats(D);
  static constexpr int kRec = 4;  // one slot per attention pair
  static constexpr int kBmWords = kMScores / NR / 32;
  uint8_t ring[kMStages][kStageBytes];               // 1024-byte aligned
  float scores[kMScores];                            // [NR][sstride]
  float qs[NR * kMaxGroup][D];                       // row r head i at r * 4 + i
  float qsT[D][NR * kMaxGroup];
  float qsum[NR][2][D];                              // per row: sum_i q'_i, 1/2 sum_i q'_i^2
  alignas(16) float wpart[kRec][kPF];                // top-k candidates, then the pairs' prefix partials; [r] ends as row r's record
  float linp[NR * kMaxGroup][D + 1];                 // linear partials (D_glob in rank 0)
  alignas(16) float mrecv[mmerge_floats(NR, D)];
  float zks[D];
  alignas(16) float xk[kMaxX][D];                    // keys of [fold_begin, ev_end[NR - 1])
  alignas(16) float xv[kMaxPend][D];                 // values of [fold_begin, fold_end)
  int32_t sel[NR][32];                               // each row's selection (k <= 32), ascending
  uint32_t selbm[NR][kBmWords];                      // each row's selection as a bitmap over blocks
  int32_t uni_j[NR * 32];                            // the union of the selections (state range only)
  uint32_t uni_m[NR * 32];                           // which rows selected it
  alignas(16) uint32_t hist[256];
  uint32_t tk[8];
  uint32_t tks[2][4];
  uint32_t tkw[2 * NR];
  int4 desc[kMStages];                               // chunk items: start, len, kind, row mask
  float2 xmax[4][2][4];                              // per pair and warp: a chunk's column maxima
  float2 xacc[2][4][2][4];                           // per pair and warp: the weight sums at the prefix's end, at the end
  uint4 xfrag[8][2][32];                             // per attention warp: its two k-tiles' PV weight fragments
  uint64_t full_attn[kMStages];
  uint64_t full_aux[kMStages];
  uint64_t empty[kMStages];
  uint64_t scores_bar, sel_bar, merge_bar;
  UnitGeo geo;
  MultiGeo<NR> mg;
  int nuni;
  int abort;
};

enum { kKindPrefix = 0, kKindE = 1, kKindSel = 2 };

template <int NR>
__device__ __forceinline__ MultiGeo<NR> multi_geo(const FusedParams& p, const UnitGeo& g) {
  MultiGeo<NR> m;
  const int S = p.S, W = g.W;
  m.T_last = g.T + NR - 1;
  m.pre_sink = min(S, m.T_last);
  m.pre_win = m.T_last > S ? max(S, m.T_last - W) : m.T_last;
  m.e0 = g.ev_end;
  m.e1 = max(g.ev_end, m.pre_win);
  m.n_sink_chunks = (m.pre_sink + kTile - 1) / kTile;
  m.n_win_chunks = (m.T_last - m.pre_win + kTile - 1) / kTile;
  m.n_e_chunks = (m.e1 - m.e0 + kTile - 1) / kTile;
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    const int Tr = g.T + r;
    m.win_start[r] = Tr > S ? max(S, Tr - W) : Tr;
    m.ev_end[r] = ev_end_at(Tr, S, W);
    m.nb[r] = m.ev_end[r] > S ? (m.ev_end[r] - S + p.Bk - 1) / p.Bk : 0;
    m.k_eff[r] = min(g.top_k, m.nb[r]);
  }
  m.nb_max = m.nb[NR - 1];
  m.sstride = (m.nb_max + 3) & ~3;
  return m;
}

// Items of rank r in ring order: score items (blocks of the last row, shared
// by every row), prefix chunks, H items; then, once the selections are known,
// the post-selection chunks: E chunks and the union's selected chunks.
struct MSeq {
  int b0, b1, nS;
  int h0, h1, nH;
  int nW;
};

template <int D, int NR>
__device__ __forceinline__ MSeq make_mseq(const FusedParams& p, const MultiGeo<NR>& m, int r) {
  MSeq q;
  const int C = p.C;
  block_share(m.nb_max, C, r, q.b0, q.b1);
  constexpr int RB = (2 * kTile * D * 2) / (8 * D), RH = (2 * kTile * D * 2) / (4 * D);
  q.nS = (q.b1 - q.b0 + RB - 1) / RB;
  q.h0 = r * D / C;
  q.h1 = (r + 1) * D / C;
  q.nH = (q.h1 - q.h0 + RH - 1) / RH;
  const int n_pre = m.n_sink_chunks + m.n_win_chunks;
  q.nW = r < n_pre ? (n_pre - r + C - 1) / C : 0;
  return q;
}
// post-selection chunks of rank r out of `total`
__device__ __forceinline__ int post_count(int total, int r, int C) { return r < total ? (total - r + C - 1) / C : 0; }

// ---------------------------------------------------------------- statistics role
// Score item idx for every row: score_rj = sum_c qsum[r][0][c] mu_jc +
// qsum[r][1][c] var_jc, into sm.scores[r][j] (transposing butterfly as in the
// single-token kernel).
template <int D, int NR>
__device__ __forceinline__ void mscore_item(MultiSmem<D, NR>& sm, const MSeq& s, int idx, int stage, int sstride) {
  constexpr int CPL = D / 32;
  constexpr int RB = 32;
  const int lane = role_tid() & 31;
  const int j0 = s.b0 + idx * RB;
  const int nblk = min(RB, s.b1 - j0);
  const float* mrows = reinterpret_cast<const float*>(sm.ring[stage]) + lane * CPL;
  const float* vrows = mrows + RB * D;
#pragma unroll 1
  for (int r = 0; r < NR; ++r) {
    float q1[CPL], q2[CPL];
    lds_vec<CPL>(&sm.qsum[r][0][lane * CPL], q1);
    lds_vec<CPL>(&sm.qsum[r][1][lane * CPL], q2);
    float part[RB];
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      float mm[CPL], vv[CPL];
      lds_vec<CPL>(mrows + b * D, mm);
      lds_vec<CPL>(vrows + b * D, vv);
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) acc += q1[c] * mm[c] + q2[c] * vv[c];
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
    if (lane < nblk) sm.scores[r * sstride + j0 + lane] = part[0];
  }
}

// The blocks of score item idx that the pending evictions [fold_begin, ev0) or
// the rows' E tokens [ev0, ev_end[NR-1]) fall into: Welford's running mean and
// population variance from the stored rows through those tokens in position
// order; at ev_end[r] the row-r statistics give row r's score; the state at ev0
// (row 0's) is written back when a pending token was folded into the block.
// One warp, lane l holding channels [l CPL, l CPL + CPL).
template <int D, int NR>
__device__ __forceinline__ void mfold_item(const FusedParams& p, const UnitGeo& g, const MultiGeo<NR>& m,
                                           MultiSmem<D, NR>& sm, const MSeq& s, int unit, int idx, int stage) {
  constexpr int CPL = D / 32;
  constexpr int RB = 32;
  const int lane = role_tid() & 31;
  const int t_lo = g.fold_begin, t_hi = m.ev_end[NR - 1];
  if (t_hi <= t_lo) return;
  const int j0 = s.b0 + idx * RB;
  const int nblk = min(RB, s.b1 - j0);
  const int jb0 = (t_lo - p.S) / p.Bk, jb1 = (t_hi - 1 - p.S) / p.Bk;
  const int bl0 = max(0, jb0 - j0), bl1 = min(nblk - 1, jb1 - j0);
  const float* mrows = reinterpret_cast<const float*>(sm.ring[stage]);
  const float* vrows = mrows + RB * D;
#pragma unroll 1
  for (int bl = bl0; bl <= bl1; ++bl) {
    const int j = j0 + bl;
    const int bs = p.S + j * p.Bk;
    const int t0 = max(bs, t_lo), t1 = min(bs + p.Bk, t_hi);
    float mm[CPL], vv[CPL];
    lds_vec<CPL>(mrows + bl * D + lane * CPL, mm);
    lds_vec<CPL>(vrows + bl * D + lane * CPL, vv);
    int r = 0;  // next row whose checkpoint (its ev_end) is due
    // rows whose edge lies at or before the block's first new token see the stored statistics
#pragma unroll 1
    for (; r < NR && m.ev_end[r] <= t0; ++r) {
    }
#pragma unroll 1
    for (int t = t0; t < t1; ++t) {
      float x[CPL];
      lds_vec<CPL>(&sm.xk[t - t_lo][lane * CPL], x);
      const float cnt = (float)(t - bs + 1);
      const float inv = 1.f / cnt;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        if (t == bs) {
          mm[c] = x[c];
          vv[c] = 0.f;
        } else {
          const float delta = x[c] - mm[c];
          const float m1 = mm[c] + delta * inv;
          vv[c] = (vv[c] * (cnt - 1.f) + delta * (x[c] - m1)) * inv;
          mm[c] = m1;
        }
      }
      if (t + 1 == g.ev_end && g.fold_end > g.fold_begin && t >= g.fold_begin) {  // row 0's state: stored
        sts_vec<CPL>(p.mu + ((int64_t)unit * p.max_blocks + j) * D + lane * CPL, mm);
        sts_vec<CPL>(p.var + ((int64_t)unit * p.max_blocks + j) * D + lane * CPL, vv);
      }
      // rows whose eviction edge is t + 1: their score of block j
#pragma unroll 1
      for (; r < NR && m.ev_end[r] == t + 1; ++r) {
        float q1[CPL], q2[CPL];
        lds_vec<CPL>(&sm.qsum[r][0][lane * CPL], q1);
        lds_vec<CPL>(&sm.qsum[r][1][lane * CPL], q2);
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc += q1[c] * mm[c] + q2[c] * vv[c];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
        if (lane == 0 && j < m.nb[r]) sm.scores[r * m.sstride + j] = acc;
      }
    }
    // the block ends before the remaining rows' edges: they see its full statistics
    if (t1 == bs + p.Bk) {
      if (t1 > g.fold_begin && t1 <= g.ev_end && g.fold_end > g.fold_begin && t1 != g.ev_end) {
        sts_vec<CPL>(p.mu + ((int64_t)unit * p.max_blocks + j) * D + lane * CPL, mm);
        sts_vec<CPL>(p.var + ((int64_t)unit * p.max_blocks + j) * D + lane * CPL, vv);
      }
#pragma unroll 1
      for (; r < NR; ++r) {
        float q1[CPL], q2[CPL];
        lds_vec<CPL>(&sm.qsum[r][0][lane * CPL], q1);
        lds_vec<CPL>(&sm.qsum[r][1][lane * CPL], q2);
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc += q1[c] * mm[c] + q2[c] * vv[c];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
        if (lane == 0 && j < m.nb[r]) sm.scores[r * m.sstride + j] = acc;
      }
    }
    __syncwarp();
  }
}

// H item: rows of H with the pending evictions folded (written back) and
// q'_{r,i}[row] H[row][:] accumulated for every row r and head i.
template <int D, int NR>
__device__ __forceinline__ void mh_item(const FusedParams& p, const UnitGeo& g, MultiSmem<D, NR>& sm, const MSeq& s,
                                        int unit, int idx, int stage, float (&hacc)[NR][kMaxGroup][D / 32]) {
  constexpr int CPL = D / 32;
  constexpr int RH = (2 * kTile * D * 2) / (4 * D);
  const int a = role_tid() - kAttnThreads, aw = a >> 5, lane = a & 31;
  const int r0 = s.h0 + idx * RH;
  const int nrows = min(RH, s.h1 - r0);
  const float* hrows = reinterpret_cast<const float*>(sm.ring[stage]);
  const bool fold = g.fold_end > g.fold_begin;
#pragma unroll 1
  for (int rl = aw; rl < nrows; rl += kAuxWarps) {
    const int row = r0 + rl;
    float h[CPL];
    lds_vec<CPL>(hrows + rl * D + lane * CPL, h);
    if (fold) {
#pragma unroll 1
      for (int t = 0; t < g.fold_end - g.fold_begin; ++t) {
        const float kr = sm.xk[t][row];
        float vv[CPL];
        lds_vec<CPL>(&sm.xv[t][lane * CPL], vv);
#pragma unroll
        for (int c = 0; c < CPL; ++c) h[c] += kr * vv[c];
      }
      sts_vec<CPL>(p.H + ((int64_t)unit * D + row) * D + lane * CPL, h);
    }
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const float4 qr = *reinterpret_cast<const float4*>(&sm.qsT[row][r * kMaxGroup]);
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        hacc[r][0][c] += qr.x * h[c];
        hacc[r][1][c] += qr.y * h[c];
        hacc[r][2][c] += qr.z * h[c];
        hacc[r][3][c] += qr.w * h[c];
      }
    }
  }
}

// The linear partials of every row into linp (three warps in turn); rank 0
// folds the pending evictions into zk, zv, n and forms D_glob = n + q'.zk.
template <int D, int NR>
__device__ void mfinish_linear(const FusedParams& p, const UnitGeo& g, MultiSmem<D, NR>& sm, int unit, int rank,
                               const float (&hacc)[NR][kMaxGroup][D / 32]) {
  constexpr int CPL = D / 32;
  const int a = role_tid() - kAttnThreads, aw = a >> 5, lane = a & 31;
  float nval = 0.f;
  if (rank == 0) {
    for (int c = a; c < D; c += kAuxThreads) {
      float zk = p.zk[(int64_t)unit * D + c], zv = p.zv[(int64_t)unit * D + c];
      if (g.fold_end > g.fold_begin) {
        for (int t = 0; t < g.fold_end - g.fold_begin; ++t) {
          zk += sm.xk[t][c];
          zv += sm.xv[t][c];
        }
        p.zk[(int64_t)unit * D + c] = zk;
        p.zv[(int64_t)unit * D + c] = zv;
      }
      sm.zks[c] = zk;
      sm.linp[0][c] = zv;  // staged; added to every row's N_glob below
    }
    nval = p.n[unit] + (float)(g.fold_end - g.fold_begin);
    if (a == 0 && g.fold_end > g.fold_begin) p.n[unit] = nval;
  }
  named_sync(kBarAux, kAuxThreads);
  float zvc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) zvc[c] = rank == 0 ? sm.linp[0][lane * CPL + c] : 0.f;
  named_sync(kBarAux, kAuxThreads);
#pragma unroll 1
  for (int w = 0; w < kAuxWarps; ++w) {
    if (aw == w)
#pragma unroll
      for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int i = 0; i < kMaxGroup; ++i)
          if (i < p.G)
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
              float* dst = &sm.linp[r * kMaxGroup + i][lane * CPL + c];
              *dst = (w == 0 ? zvc[c] : *dst) + hacc[r][i][c];
            }
    named_sync(kBarAux, kAuxThreads);
  }
  if (rank == 0 && aw == 0) {
    for (int ri = 0; ri < NR * kMaxGroup; ++ri) {
      if ((ri & 3) >= p.G) continue;
      float d = 0.f;
      for (int c = lane; c < D; c += 32) d += sm.qs[ri][c] * sm.zks[c];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(kFull, d, o);
      if (lane == 0) sm.linp[ri][D] = nval + d;
    }
  }
}

// Every row's selection (statistics threads): the scores of every rank are in
// place; row r's top-k by warp r % 3 (the radix selection over all statistics
// threads for a row whose candidates overflow), then the rows' bitmaps and the
// union of their blocks in the state range with the rows that chose each.
template <int D, int NR>
__device__ void mselect(const FusedParams& p, const MultiGeo<NR>& m, MultiSmem<D, NR>& sm, int unit, int rank,
                        bool ok) {
  const int a = role_tid() - kAttnThreads, aw = a >> 5, lane = a & 31;
  const int nb0 = m.nb[0];
  const int words = (m.nb_max + 31) >> 5;
  for (int i = a; i < NR * MultiSmem<D, NR>::kBmWords; i += kAuxThreads) (&sm.selbm[0][0])[i] = 0u;
  if (ok) {
    // 8-byte entries per warp, an even count: the one-warp ranking reads its
    // candidates 16 bytes at a time, so every warp's buffer starts on 16 bytes
    constexpr int kCap = (MultiSmem<D, NR>::kRec * MultiSmem<D, NR>::kPF / 2 / kAuxWarps) & ~1;
    static_assert(kCap % 2 == 0, "16-byte aligned candidate buffers");
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(&sm.wpart[0][0]) + aw * kCap;
#pragma unroll 1
    for (int r = aw; r < NR; r += kAuxWarps) {
      const int k = m.k_eff[r];
      int32_t* copy = (p.sel_out != nullptr && rank == 0)
                          ? p.sel_out + ((int64_t)r * p.units + unit) * p.top_k : nullptr;
      bool done = true, nan = false;
      if (k > 0 && k < m.nb[r]) {
        done = topk_warp(sm.scores + r * m.sstride, m.nb[r], k, sm.sel[r], copy, cand, kCap, nan);
      } else {
        for (int j = lane; j < k; j += 32) {
          sm.sel[r][j] = j;
          if (copy) copy[j] = j;
        }
      }
      if (lane == 0) {
        sm.tkw[2 * r] = done ? 1u : 0u;
        sm.tkw[2 * r + 1] = nan ? 1u : 0u;
      }
    }
    named_sync(kBarAux, kAuxThreads);
#pragma unroll 1
    for (int r = 0; r < NR; ++r) {
      if (sm.tkw[2 * r] == 0u) {  // too many equal keys for the one-warp ranking
        int32_t* copy = (p.sel_out != nullptr && rank == 0)
                            ? p.sel_out + ((int64_t)r * p.units + unit) * p.top_k : nullptr;
        const TopkSmem t{sm.hist, sm.tk, &sm.tks[0][0]};
        if (aux_topk(t, sm.scores + r * m.sstride, false, m.nb[r], m.k_eff[r], sm.sel[r], copy)) sm.tkw[2 * r + 1] = 1u;
        named_sync(kBarAux, kAuxThreads);
      }
      if (a == 0 && sm.tkw[2 * r + 1] != 0u) atomicOr(p.status, HYB_STATUS_NAN_SCORE);
    }
    if (p.sel_out != nullptr && rank == 0)
      for (int r = 0; r < NR; ++r)
        for (int j = m.k_eff[r] + a; j < p.top_k; j += kAuxThreads)
          p.sel_out[((int64_t)r * p.units + unit) * p.top_k + j] = -1;
    named_sync(kBarAux, kAuxThreads);
    for (int i = a; i < NR * 32; i += kAuxThreads) {
      const int r = i >> 5, e = i & 31;
      if (e < m.k_eff[r]) {
        const int j = sm.sel[r][e];
        atomicOr(&sm.selbm[r][j >> 5], 1u << (j & 31));
      }
    }
  }
  named_sync(kBarAux, kAuxThreads);
  if (aw == 0) {  // union over the state range (blocks < nb0), ascending, with the rows' mask
    int base = 0;
    const uint32_t lt = lanemask_lt();
#pragma unroll 1
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      uint32_t u = 0u;
      if (w < words) {
#pragma unroll
        for (int r = 0; r < NR; ++r) u |= sm.selbm[r][w];
        const int lim = nb0 - (w << 5);  // blocks of this word in the state range
        if (lim <= 0) u = 0u;
        else if (lim < 32) u &= (1u << lim) - 1u;
      }
      const int cnt = __popc(u);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      int pos = base + incl - cnt;
      while (u) {
        const int b = __ffs(u) - 1;
        u &= u - 1u;
        const int j = (w << 5) + b;
        uint32_t mask = 0u;
#pragma unroll
        for (int r = 0; r < NR; ++r) mask |= ((sm.selbm[r][w] >> b) & 1u) << r;
        sm.uni_j[pos] = j;
        sm.uni_m[pos] = mask;
        ++pos;
      }
      base += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) sm.nuni = base;
  }
  // Issue order: by rounds, each round taking the next C blocks of every row in
  // turn, so that the ring's consecutive chunks of a rank (every C-th) belong
  // to different rows and the pairs, one row each, work side by side.  A block
  // chosen by several rows goes at its earliest place: key = min over those
  // rows r of (i / C) (NR C) + r C + i % C, i = the block's place in row r's
  // ascending selection (i < 32, C <= 16: keys < 256, all distinct).
  named_sync(kBarAux, kAuxThreads);
  const int nU = sm.nuni, C = p.C;
  for (int i = a; i < 256; i += kAuxThreads) sm.hist[i] = 0xffffffffu;
  named_sync(kBarAux, kAuxThreads);
  for (int u = a; u < nU; u += kAuxThreads) {
    const int j = sm.uni_j[u];
    const uint32_t msk = sm.uni_m[u];
    int key = 255;
#pragma unroll
    for (int r = 0; r < NR; ++r)
      if ((msk >> r) & 1u) {
        int i = 0;
        for (int e = 0; e < m.k_eff[r]; ++e) i += sm.sel[r][e] < j ? 1 : 0;
        key = min(key, (i / C) * NR * C + r * C + i % C);
      }
    sm.hist[key] = (uint32_t)u;
  }
  named_sync(kBarAux, kAuxThreads);
  if (aw == 0) {  // compaction in key order: lane l takes keys [8 l, 8 l + 8)
    int jj[8];
    uint32_t mm[8], have = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t u = sm.hist[8 * lane + e];
      jj[e] = 0;
      mm[e] = 0u;
      if (u != 0xffffffffu) {
        jj[e] = sm.uni_j[u];
        mm[e] = sm.uni_m[u];
        have |= 1u << e;
      }
    }
    const int cnt = __popc(have);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    __syncwarp();  // every entry is read before any is rewritten
    int pos = incl - cnt;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if ((have >> e) & 1u) {
        sm.uni_j[pos] = jj[e];
        sm.uni_m[pos] = mm[e];
        ++pos;
      }
  }
}

template <int D, int NR>
__device__ void maux_role(const FusedParams& p, const UnitGeo& g, const MultiGeo<NR>& m, MultiSmem<D, NR>& sm,
                          const MSeq& s, int unit, int rank) {
  constexpr int CPL = D / 32;
  const int a = role_tid() - kAttnThreads, aw = a >> 5, lane = a & 31;
  bool dead = false;
  uint32_t par = 0u;
  auto wait_item = [&](int it) -> bool {
    const int stage = it % kMStages;
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
  for (int c = a; c < D; c += kAuxThreads)
#pragma unroll 1
    for (int r = 0; r < NR; ++r) {
      float q1 = 0.f, q2 = 0.f;
      for (int i = 0; i < p.G; ++i) {
        const float qv = sm.qs[r * kMaxGroup + i][c];
        q1 += qv;
        q2 += 0.5f * qv * qv;
      }
      sm.qsum[r][0][c] = q1;
      sm.qsum[r][1][c] = q2;
    }
  named_sync(kBarAux, kAuxThreads);
  cluster_wait();  // every rank's barriers are initialised
  // the blocks the pending evictions or the rows' E tokens fall into
  const int t_lo = g.fold_begin, t_hi = m.ev_end[NR - 1];
  int fi0 = 0, fi1 = 0;
  if (t_hi > t_lo && s.b1 > s.b0) {
    const int jb0 = (t_lo - p.S) / p.Bk, jb1 = (t_hi - 1 - p.S) / p.Bk;
    const int lo = max(jb0, s.b0), hi = min(jb1, s.b1 - 1);
    if (lo <= hi) {
      fi0 = (lo - s.b0) / 32;
      fi1 = (hi - s.b0) / 32 + 1;
    }
  }
#pragma unroll 1
  for (int idx = 0; idx < s.nS; ++idx) {
    const int stage = idx % kMStages;
    const bool have = wait_item(idx);
    if (have && idx % kAuxWarps == aw) {
      mscore_item<D, NR>(sm, s, idx, stage, m.sstride);
      __syncwarp();
      if (idx >= fi0 && idx < fi1) mfold_item<D, NR>(p, g, m, sm, s, unit, idx, stage);
      __syncwarp();
    }
    if (lane == 0 && have) mbar_arrive_cnt(&sm.empty[stage], kEmptyPerAuxWarp);
  }
  named_sync(kBarAux, kAuxThreads);
  // every row's share of the scores to every rank
  const bool topk = m.nb_max > 0;
  if (topk) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    named_sync(kBarAux, kAuxThreads);
    if (a == 0 && s.b1 > s.b0) {
      const uint32_t bytes = (uint32_t)(((s.b1 - s.b0) * 4 + 15) & ~15);
      const uint32_t bar = smem_u32(&sm.scores_bar);
      for (int r = 0; r < NR; ++r) {
        const uint32_t src = smem_u32(&sm.scores[r * m.sstride + s.b0]);
        for (int rr = 0; rr < p.C; ++rr)
          if (rr != rank) bulk_push(map_rank(src, (uint32_t)rr), src, bytes, map_rank(bar, (uint32_t)rr));
      }
    }
  }
  bool ok = true;
  if (topk) {
    if (a == 0) {
      const bool w = wait_cluster_bounded(&sm.scores_bar, 0, p.wait_ns);
      if (!w) {
        atomicOr(p.status, HYB_STATUS_TIMEOUT);
        sm.abort = 1;
      }
      sm.tk[7] = w ? 1u : 0u;
    }
    named_sync(kBarAux, kAuxThreads);
    ok = sm.tk[7] != 0u;
  }
  mselect<D, NR>(p, m, sm, unit, rank, ok);
  named_sync(kBarAux, kAuxThreads);
  if (a == 0) mbar_arrive(&sm.sel_bar);  // release: the union and the bitmaps are visible
  float hacc[NR][kMaxGroup][CPL];
#pragma unroll
  for (int r = 0; r < NR; ++r)
#pragma unroll
    for (int i = 0; i < kMaxGroup; ++i)
#pragma unroll
      for (int c = 0; c < CPL; ++c) hacc[r][i][c] = 0.f;
#pragma unroll 1
  for (int idx = 0; idx < s.nH; ++idx) {
    const int it = s.nS + s.nW + idx, stage = it % kMStages;
    const bool have = wait_item(it);
    if (have) mh_item<D, NR>(p, g, sm, s, unit, idx, stage, hacc);
    __syncwarp();
    if (lane == 0 && have) mbar_arrive_cnt(&sm.empty[stage], kEmptyPerAuxWarp);
  }
  mfinish_linear<D, NR>(p, g, sm, unit, rank, hacc);
}

// ---------------------------------------------------------------- producer
// Chunk copies as the single-token kernel's (TMA tensor loads, 64- or 16-row
// boxes, no multicast); the new tokens a prefix chunk holds are first written
// to the caches by this lane, then made visible to the tensor copy that reads
// them (a proxy fence).
template <int D, int NR>
__device__ __forceinline__ void missue_chunk(const KVMaps* tm, MultiSmem<D, NR>& sm, int stage, int64_t ubase, int start,
                                             int len, int kind, uint32_t mask, uint64_t pol) {
  using Sm = MultiSmem<D, NR>;
  uint64_t* bar = &sm.full_attn[stage];
  const uint32_t dst = smem_u32(sm.ring[stage]);
  sm.desc[stage] = make_int4(start, len, kind, (int)mask);
  if (len <= 0) {
    mbar_arrive(bar);
    return;
  }
  const int row = (int)(ubase + start);
  if (len == kTile) {
    mbar_arrive_expect_tx(bar, (uint32_t)(2 * Sm::kHalf));
    tma_load_3d_stream(dst, &tm->k64, 0, 0, row, bar, pol);
    tma_load_3d_stream(dst + Sm::kHalf, &tm->v64, 0, 0, row, bar, pol);
  } else {
    const int nbox = (len + kBoxRows - 1) / kBoxRows;
    mbar_arrive_expect_tx(bar, (uint32_t)(nbox * Sm::kBoxBytes * 2));
    for (int bx = 0; bx < nbox; ++bx) {
      tma_load_3d_stream(dst + bx * Sm::kBoxBytes, &tm->k16, 0, 0, row + bx * kBoxRows, bar, pol);
      tma_load_3d_stream(dst + Sm::kHalf + bx * Sm::kBoxBytes, &tm->v16, 0, 0, row + bx * kBoxRows, bar, pol);
    }
  }
}

template <int D, int NR>
__device__ void mproducer_role(const KVMaps* tm, const FusedParams& p, const UnitGeo& g, const MultiGeo<NR>& m,
                               MultiSmem<D, NR>& sm, const MSeq& s, int unit, int rank) {
  if ((threadIdx.x & 31) != 0) return;
  constexpr int RB = 32, RH = (2 * kTile * D * 2) / (4 * D);
  const uint64_t pol = l2_evict_first();
  int stage = 0, issued = 0;
  uint32_t epar = 0u, fpar_aux = 0u, fpar_at = 0u, last_aux = 0u;
  bool ok = true;
  auto acquire = [&]() -> bool {
    if (issued >= kMStages) {
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
    stage = stage + 1 == kMStages ? 0 : stage + 1;
  };
  const int64_t brow = (int64_t)unit * p.max_blocks + s.b0;
  for (int i = 0; i < s.nS && ok; ++i) {
    if (!(ok = acquire())) break;
    uint64_t* bar = &sm.full_aux[stage];
    const uint32_t dst = smem_u32(sm.ring[stage]);
    const uint32_t bytes = (uint32_t)(min(RB, s.b1 - s.b0 - i * RB) * D * 4);
    const int64_t off = (brow + (int64_t)i * RB) * D;
    mbar_arrive_expect_tx(bar, 2 * bytes);
    bulk_load_stream(dst, p.mu + off, bytes, bar, pol);
    bulk_load_stream(dst + RB * D * 4, p.var + off, bytes, bar, pol);
    advance(true);
  }
  const int64_t ubase = (int64_t)unit * p.cap;
  for (int i = 0, ci = rank; i < s.nW && ok; ++i, ci += p.C) {
    if (!(ok = acquire())) break;
    int start, len;
    if (ci < m.n_sink_chunks) {
      start = ci * kTile;
      len = min(kTile, m.pre_sink - start);
    } else {
      start = m.pre_win + (ci - m.n_sink_chunks) * kTile;
      len = min(kTile, m.T_last - start);
    }
    // new tokens of the chunk ([T, T_last) of this unit): written before the copy reads them
    const int n0 = max(start, g.T), n1 = min(start + len, m.T_last);
    if (n1 > n0) {
      for (int t = n0; t < n1; ++t) {
        const int r = t - g.T;
        const uint4* ks = reinterpret_cast<const uint4*>(p.k_new + ((int64_t)r * p.units + unit) * D);
        const uint4* vs = reinterpret_cast<const uint4*>(p.v_new + ((int64_t)r * p.units + unit) * D);
        uint4* kd = reinterpret_cast<uint4*>(p.k_cache + (ubase + t) * D);
        uint4* vd = reinterpret_cast<uint4*>(p.v_cache + (ubase + t) * D);
        for (int e = 0; e < D / 8; ++e) {
          kd[e] = __ldg(ks + e);
          vd[e] = __ldg(vs + e);
        }
      }
      asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    missue_chunk<D, NR>(tm, sm, stage, ubase, start, len, kKindPrefix, 0u, pol);
    advance(false);
  }
  for (int i = 0; i < s.nH && ok; ++i) {
    if (!(ok = acquire())) break;
    uint64_t* bar = &sm.full_aux[stage];
    const int r0 = s.h0 + i * RH;
    const uint32_t bytes = (uint32_t)(min(RH, s.h1 - r0) * D * 4);
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load_stream(smem_u32(sm.ring[stage]), p.H + ((int64_t)unit * D + r0) * D, bytes, bar, pol);
    advance(true);
  }
  // after the selections: E chunks, then the union's selected chunks
  if (ok && !mbar_wait_bounded(&sm.sel_bar, 0, p.wait_ns)) {
    atomicOr(p.status, HYB_STATUS_TIMEOUT);
    sm.abort = 1;
    ok = false;
  }
  const int cpb = p.chunks_per_block;
  const int nU = ok ? sm.nuni : 0;
  const int total = m.n_e_chunks + nU * cpb;
  const int nX = post_count(total, rank, p.C);
  for (int i = 0, c = rank; i < nX && ok; ++i, c += p.C) {
    if (!(ok = acquire())) break;
    int start, len, kind;
    uint32_t mask = 0u;
    if (c < m.n_e_chunks) {
      start = m.e0 + c * kTile;
      len = min(kTile, m.e1 - start);
      kind = kKindE;
    } else {
      const int u = (c - m.n_e_chunks) / cpb, piece = (c - m.n_e_chunks) - u * cpb;
      const int j = sm.uni_j[u];
      const int bs = p.S + j * p.Bk;
      start = bs + piece * kTile;
      len = max(0, min(kTile, min(bs + p.Bk, m.e0) - start));
      kind = kKindSel;
      mask = sm.uni_m[u];
    }
    missue_chunk<D, NR>(tm, sm, stage, ubase, start, len, kind, mask, pol);
    advance(false);
  }
  if (*(volatile int*)&sm.abort) {
    for (int j = 0; j < kMStages && j < issued; ++j) {
      const bool aux = (last_aux >> j) & 1u;
      const uint32_t ph = (((aux ? fpar_aux : fpar_at) >> j) & 1u) ^ 1u;
      mbar_wait_bounded(aux ? &sm.full_aux[j] : &sm.full_attn[j], ph, kWaitLimit);
    }
  }
}

// ---------------------------------------------------------------- attention role
// Prefix chunks: pair q handles rows (a, a + 1), a = 2 (q / 2) for NR = 4 (0
// for NR = 2), chunks c with c % (8 / NR) == q % (8 / NR); N column n is row
// a + n / 4, head n % 4.  Post-selection chunks: pair q handles row q * NR / 4,
// and of the chunks that row takes, those whose count (in ring order) is
// q % (4 / NR) modulo 4 / NR; columns 0-3 exact, 4-7 Taylor.
// Token t of a chunk, for row r (T_r = T + r):
//   prefix:   exact when t < T_r;
//   E:        exact when t >= win_start[r] or its block is in row r's
//             selection, else the Taylor weight 1 + s added to the linear part;
//   selected: (row r chose the block) exact, and 1 + s subtracted from the state.
// The Taylor rows of the PV product carry the signed weight (+ subtract,
// - add), so that N_lin = N_glob - sum w v, D_lin = D_glob - sum w.
template <int D, int NR>
__device__ void mattn_role(const FusedParams& p, const UnitGeo& g, const MultiGeo<NR>& m, MultiSmem<D, NR>& sm,
                           const MSeq& s, int unit, int rank) {
  constexpr int NT8 = D / 8, NH = NT8 / 2, KS = D / 16;
  constexpr int kPairsPerRow = 4 / NR, kPrePairs = 8 / NR;
  const int tid = role_tid(), warp = tid >> 5, lane = tid & 31;
  const int pair = warp >> 1, half = warp & 1;
  const int row = pair / kPairsPerRow, sub = pair % kPairsPerRow;
  const int ra = NR == 4 ? (pair >> 1) * 2 : 0, psub = pair % kPrePairs;
  const int g8 = lane >> 2, tig = lane & 3;
  const bool p_lane = g8 < 4;
  const int head = g8 & 3;
  const int mi = lane >> 3, rr = lane & 7;
  const int Tr = g.T + row;
  const int Tpre = g.T + ra + (tig >> 1);  // the row of this lane's prefix columns 2 tig, 2 tig + 1
  const int ws = m.win_start[row];

  uint32_t qb[KS][2];
  auto load_q = [&](int qrow_idx) {  // N column g8: head g8 % 4 of row qrow_idx
    const bool real = (g8 & 3) < p.G;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        p.q + (((int64_t)qrow_idx * p.units + unit) * p.G + (real ? (g8 & 3) : 0)) * D);
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qb[kk][0] = real ? __ldg(qrow + kk * 8 + tig) : 0u;
      qb[kk][1] = real ? __ldg(qrow + kk * 8 + 4 + tig) : 0u;
    }
  };
  load_q(ra + (g8 >> 2));
  float O[NH][4];
#pragma unroll
  for (int n = 0; n < NH; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.f;
  bool pre = true;                    // the prefix chunks: every column exact
  bool soft_lane = true;              // this lane's accumulator columns take softmax weights
  float mr0 = -INFINITY, mr1 = -INFINITY, acc0 = 0.f, acc1 = 0.f;
  // the prefix partial of rows (ra, ra + 1) into this pair's combine slot
  // (free once the selections are made): per column its max and weight sum,
  // then the 8 columns' D outputs
  auto flush_prefix = [&]() {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      acc0 += __shfl_xor_sync(kFull, acc0, o);
      acc1 += __shfl_xor_sync(kFull, acc1, o);
    }
    // each warp of the pair summed its own tokens: add the other's
    if (g8 == 0) sm.xacc[0][pair][half][tig] = make_float2(acc0, acc1);
    named_sync(kBarPair0 + pair, 64);
    {
      const float2 o = sm.xacc[0][pair][half ^ 1][tig];
      acc0 += o.x;
      acc1 += o.y;
    }
    const float v0 = __shfl_sync(kFull, acc0, g8 >> 1), v1 = __shfl_sync(kFull, acc1, g8 >> 1);
    const float m0 = __shfl_sync(kFull, mr0, g8 >> 1), m1 = __shfl_sync(kFull, mr1, g8 >> 1);
    float* wp = sm.wpart[pair];
    if (tig == 0 && half == 0) {
      wp[g8] = (g8 & 1) ? m1 : m0;
      wp[8 + g8] = (g8 & 1) ? v1 : v0;
    }
    float* dst = wp + 16 + g8 * D + half * (D / 2);
#pragma unroll
    for (int n = 0; n < NH; ++n) {
      *reinterpret_cast<float2*>(dst + n * 8 + 2 * tig) = make_float2(O[n][0] + O[n][2], O[n][1] + O[n][3]);
      O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.f;
    }
    mr0 = mr1 = -INFINITY;
    acc0 = acc1 = 0.f;
    pre = false;
    soft_lane = tig < 2;
    load_q(row);
  };

  bool dead = false;
  uint32_t par = 0u;
  int nchunks = s.nW, post_base = s.nS + s.nW + s.nH;
  bool post_known = false;
  int rcount = 0;  // post-selection chunks of this pair's row so far (every pair sees every chunk)
#pragma unroll 1
  for (int c = 0; c < nchunks || !post_known; ++c) {
    if (c == s.nW && !post_known) {  // the selections decide the post-selection chunks
      post_known = true;
      int nU = 0;
      if (!dead && mbar_wait_bounded(&sm.sel_bar, 0, p.wait_ns)) nU = sm.nuni;
      flush_prefix();
      nchunks = s.nW + post_count(m.n_e_chunks + nU * p.chunks_per_block, rank, p.C);
      if (c >= nchunks) break;
    }
    const int it = c < s.nW ? s.nS + c : post_base + (c - s.nW);
    const int stage = it % kMStages;
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
    const int4 dsc = sm.desc[stage];
    bool mine;
    if (pre) {
      mine = (c % kPrePairs) == psub;
    } else {  // the row's chunks go to its pairs in turn
      const bool has = dsc.z != kKindSel || ((dsc.w >> row) & 1);
      mine = has && (rcount % kPairsPerRow) == sub;
      rcount += has ? 1 : 0;
    }
    if (!mine) {
      if (lane == 0 && have) mbar_arrive_cnt(&sm.empty[stage], kEmptyPerAttnWarp);
      continue;
    }
    const int nvalid = have ? dsc.y : 0;
    const uint32_t kb = smem_u32(sm.ring[stage]);
    const uint32_t vb = kb + MultiSmem<D, NR>::kHalf;
    // S^T = K Q^T for this warp's 32 tokens (m-tiles 2 half, 2 half + 1); both
    // warps of the pair take the same barriers whatever their waits gave
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
    const int kind = dsc.z, start = dsc.x;
    float w[2][4];
    float t0m = -INFINITY, t1m = -INFINITY;
#pragma unroll
    for (int mm = 0; mm < 2; ++mm)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int t = (2 * half + mm) * 16 + g8 + 8 * (q >> 1);
        const int pos = start + t;
        const bool valid = t < nvalid;
        bool ex;
        float sg;
        if (kind == kKindSel) {
          ex = true;
          sg = 1.f;
        } else if (kind == kKindPrefix) {
          ex = pos < Tpre;
          sg = 0.f;
        } else {  // E: only the chunk's own positions index the bitmap
          const int blk = valid ? (pos - p.S) / p.Bk : 0;
          const bool in_win = pos >= ws;
          const bool chosen = valid && ((sm.selbm[row][blk >> 5] >> (blk & 31)) & 1u);
          ex = pos < Tr && (in_win || chosen);
          sg = (pos < Tr && !in_win && !chosen) ? -1.f : 0.f;
        }
        const float sv = valid ? sacc[mm][q] * p.scale : 0.f;
        const float xs = (valid && ex) ? sv * kLog2e : -INFINITY;
        const float wt = valid ? sg * (1.f + sv) : 0.f;
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
    if (g8 == 0) sm.xmax[pair][half][tig] = make_float2(t0m, t1m);
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
        const float ev = exp2f(w[mm][q] - ((q & 1) ? mn1 : mn0));
        w[mm][q] = soft_lane ? (w[mm][q] == -INFINITY ? 0.f : ev) : w[mm][q];
        if (q & 1) ws1 += w[mm][q]; else ws0 += w[mm][q];
      }
    acc0 = acc0 * al0 + ws0;  // this warp's tokens only: the pair's two sums are added at the end
    acc1 = acc1 * al1 + ws1;
    mr0 = soft_lane ? mn0 : mr0;
    mr1 = soft_lane ? mn1 : mr1;
    const float b0 = __shfl_sync(kFull, al0, g8 >> 1), b1 = __shfl_sync(kFull, al1, g8 >> 1);
    const float alpha = (p_lane || pre) ? ((g8 & 1) ? b1 : b0) : 1.f;
    if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll
      for (int n = 0; n < NH; ++n) {
        O[n][0] *= alpha;
        O[n][1] *= alpha;
        O[n][2] *= alpha;
        O[n][3] *= alpha;
      }
    }
    // this warp's PV weight fragments to the other warp of the pair
    uint32_t mf[2][4], of[2][4];
#pragma unroll
    for (int mm = 0; mm < 2; ++mm) {
      uint32_t h0, l0, h1, l1;
      split_bf16(w[mm][0], w[mm][1], h0, l0);
      split_bf16(w[mm][2], w[mm][3], h1, l1);
      mf[mm][0] = movmatrix_t(h0);
      mf[mm][1] = movmatrix_t(l0);
      mf[mm][2] = movmatrix_t(h1);
      mf[mm][3] = movmatrix_t(l1);
      sm.xfrag[warp][mm][lane] = make_uint4(mf[mm][0], mf[mm][1], mf[mm][2], mf[mm][3]);
    }
    named_sync(kBarPair0 + pair, 64);
#pragma unroll
    for (int mm = 0; mm < 2; ++mm) {
      const uint4 x = sm.xfrag[warp ^ 1][mm][lane];
      of[mm][0] = x.x;
      of[mm][1] = x.y;
      of[mm][2] = x.z;
      of[mm][3] = x.w;
    }
#pragma unroll
    for (int kt = 0; kt < 4; ++kt) {
      if (kt * 16 >= nvalid) break;
      const bool tail = kt * 16 + 16 > nvalid;
      const int tk = kt * 16 + 2 * tig;
      const uint32_t m0 = (tk < nvalid ? 0x0000ffffu : 0u) | (tk + 1 < nvalid ? 0xffff0000u : 0u);
      const uint32_t m1 = (tk + 8 < nvalid ? 0x0000ffffu : 0u) | (tk + 9 < nvalid ? 0xffff0000u : 0u);
      const bool own = (kt >> 1) == half;
      const uint32_t a0 = own ? mf[kt & 1][0] : of[kt & 1][0], a1 = own ? mf[kt & 1][1] : of[kt & 1][1];
      const uint32_t a2 = own ? mf[kt & 1][2] : of[kt & 1][2], a3 = own ? mf[kt & 1][3] : of[kt & 1][3];
#pragma unroll
      for (int np = 0; np < NH / 2; ++np) {
        uint32_t b0v, b1v, b2v, b3v;
        ldsm_x4_t(vb + swz<D>(kt * 16 + (mi & 1) * 8 + rr, (half * NH / 2 + np) * 2 + (mi >> 1)), b0v, b1v, b2v,
                  b3v);
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

#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    acc0 += __shfl_xor_sync(kFull, acc0, o);
    acc1 += __shfl_xor_sync(kFull, acc1, o);
  }
  if (g8 == 0) sm.xacc[1][pair][half][tig] = make_float2(acc0, acc1);
  named_sync(kBarPair0 + pair, 64);
  {
    const float2 o = sm.xacc[1][pair][half ^ 1][tig];
    acc0 += o.x;
    acc1 += o.y;
  }
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
  auto emit = [&](float* wp) {
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
  auto absorb = [&](const float* wp) {
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
  // the prefix partials of this pair's row: slots 2 X, 2 X + 1 (X = row / 2
  // for NR = 4, the pair's post-selection index for NR = 2), this row's
  // columns; every (slot, row) is taken by exactly one pair
  named_sync(kBarAttn, kAttnThreads);  // every pair's prefix partial is in its slot
  {
    const int X = NR == 4 ? (row >> 1) : sub;
    const int col = (row & 1) * 4 + head;
#pragma unroll 1
    for (int sl = 2 * X; sl < 2 * X + 2; ++sl) {
      const float* wp = sm.wpart[sl];
      if (p_lane) {
        const float mp = wp[col], lp = wp[8 + col];
        const float M = fmaxf(m_run, mp);
        const float fa = (m_run == -INFINITY) ? 0.f : exp2f(m_run - M);
        const float fb = (mp == -INFINITY) ? 0.f : exp2f(mp - M);
        l = l * fa + lp * fb;
        m_run = M;
        const float* src = wp + 16 + col * D + half * (D / 2);
#pragma unroll
        for (int n = 0; n < NH; ++n) {
          const float2 y = *reinterpret_cast<const float2*>(src + n * 8 + 2 * tig);
          O[n][0] = (O[n][0] + O[n][2]) * fa + y.x * fb;
          O[n][1] = (O[n][1] + O[n][3]) * fa + y.y * fb;
          O[n][2] = O[n][3] = 0.f;
        }
      }
    }
  }
  named_sync(kBarAttn, kAttnThreads);  // the slots are read before they are rewritten
  if constexpr (NR == 2) {  // pairs (0, 1) -> row 0 in slot 0, (2, 3) -> row 1 in slot 1
    if (sub == 1) emit(sm.wpart[row]);
    named_sync(kBarAttn, kAttnThreads);
    if (sub == 0) {
      absorb(sm.wpart[row]);
      named_sync(kBarPair0 + row, 64);  // the pair's two warps have read the slot before it is rewritten
      emit(sm.wpart[row]);
    }
  } else {
    emit(sm.wpart[row]);
  }
}

// ---------------------------------------------------------------- merge
template <int D, int NR>
__device__ __forceinline__ void mmerge_push(const FusedParams& p, MultiSmem<D, NR>& sm, int rank) {
  const int tid = threadIdx.x;
  const int G = p.G, C = p.C, GD = G * D, NGD = NR * GD;
  const int stride = p.mstride;
  const uint32_t recv0 = smem_u32(sm.mrecv), bar0 = smem_u32(&sm.merge_bar);
  const int hr = tid - (kFThreads - C);
  if (hr >= 0) {
#pragma unroll 1
    for (int r = 0; r < NR; ++r) {
      const float* rec = sm.wpart[r];
      float h[12];
#pragma unroll
      for (int i = 0; i < kMaxGroup; ++i) {
        h[i] = rec[i];
        h[4 + i] = rec[4 + i];
        h[8 + i] = (rank == 0 && i < G ? sm.linp[r * kMaxGroup + i][D] : 0.f) - rec[8 + i];
      }
      const int off = rank * stride + 16 * r;
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
  }
  for (int e = tid; e < NGD; e += kFThreads) {
    const int r_own = ((e + 1) * C - 1) / NGD;  // the rank that merges output e
    const int row = e / GD, eg = e - row * GD;
    const int i = eg / D, d = eg - i * D;
    const float* rec = sm.wpart[row];
    const float xa = rec[16 + eg], xd = sm.linp[row * kMaxGroup + i][d] - rec[16 + 4 * D + eg];
    const int off = rank * stride + 16 * NR + 2 * (e - p.mslice[r_own]);
    if (r_own == rank)
      *reinterpret_cast<float2*>(&sm.mrecv[off]) = make_float2(xa, xd);
    else
      st_async_v2(map_rank(recv0 + 4u * (uint32_t)off, (uint32_t)r_own), xa, xd, map_rank(bar0, (uint32_t)r_own));
  }
}

template <int D, int NR>
__device__ void mmerge_local(const FusedParams& p, MultiSmem<D, NR>& sm, int unit, int rank) {
  const int tid = threadIdx.x;
  const int G = p.G, C = p.C, GD = G * D;
  const int stride = p.mstride;
  if (!__syncthreads_and(wait_cluster_bounded(&sm.merge_bar, 0, kWaitLimit))) {
    if (tid == 0) atomicOr(p.status, HYB_STATUS_TIMEOUT);
    return;
  }
  uint32_t flags = 0u;
  const int e0 = p.mslice[rank], e1 = p.mslice[rank + 1];
  for (int e = e0 + tid; e < e1; e += kFThreads) {
    const int row = e / GD, eg = e - row * GD, i = eg / D;
    const float* h = sm.mrecv + 16 * row + i;
    float M = -INFINITY;
    for (int r = 0; r < C; ++r) M = fmaxf(M, h[r * stride]);
    if (M == -INFINITY) M = 0.f;
    float nex = 0.f, nsub = 0.f, Dex = 0.f, Dsub = 0.f;
    for (int r = 0; r < C; ++r) {
      const float mm = h[r * stride];
      const float f = (mm == -INFINITY) ? 0.f : exp2f(mm - M);
      const float2 v = *reinterpret_cast<const float2*>(&sm.mrecv[r * stride + 16 * NR + 2 * (e - e0)]);
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
    p.out[((int64_t)row * p.units + unit) * GD + eg] = o;
    if (!(den > 0.f)) flags |= HYB_STATUS_DENOMINATOR;
    if (!isfinite(o)) flags |= HYB_STATUS_NONFINITE;
  }
  if (flags) atomicOr(p.status, flags);
}

template <int D, int NR>
__global__ void __launch_bounds__(kFThreads, 1) multi_kernel(const __grid_constant__ KVMaps tm, const FusedParams p) {
  extern __shared__ uint8_t smem_raw[];
  MultiSmem<D, NR>& sm =
      *reinterpret_cast<MultiSmem<D, NR>*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = role_tid() >> 5;
  const int rank = (int)cluster_rank();
  const int unit = blockIdx.x / p.C;
  const UnitGeo g0 = unit_geo(nullptr, unit, p.Hkv, p.T, p.S, p.W, p.Bk, p.top_k, p.chunks_per_block, p.pending);
  const MultiGeo<NR> m0 = multi_geo<NR>(p, g0);
  const MSeq s = make_mseq<D, NR>(p, m0, rank);
  if (tid == 0) {
    tma_prefetch_desc(&tm.k64);
    tma_prefetch_desc(&tm.v64);
    for (int i = 0; i < kMStages; ++i) {
      mbar_init(&sm.full_attn[i], 1);
      mbar_init(&sm.full_aux[i], 1);
      mbar_init(&sm.empty[i], kEmptyCount);
    }
    sm.geo = g0;
    sm.mg = m0;
    sm.nuni = 0;
    sm.abort = 0;
    mbar_init(&sm.scores_bar, 1);
    mbar_init(&sm.sel_bar, 1);
    mbar_init(&sm.merge_bar, 1);
    fence_mbar_init();
    if (m0.nb_max > 0) {  // every row's share of the scores from every other rank
      uint32_t bytes = 0;
      for (int rr = 0; rr < p.C; ++rr) {
        int b0, b1;
        block_share(m0.nb_max, p.C, rr, b0, b1);
        if (rr != rank) bytes += (uint32_t)(((b1 - b0) * 4 + 15) & ~15);
      }
      mbar_arrive_expect_tx(&sm.scores_bar, (uint32_t)NR * bytes);
    }
    mbar_arrive_expect_tx(&sm.merge_bar,
                          (uint32_t)((p.C - 1) * (48 * NR + 8 * (p.mslice[rank + 1] - p.mslice[rank]))));
    pdl_wait_primary();
  }
  __syncthreads();
  cluster_arrive_relaxed();
  pdl_allow_dependents();
  const UnitGeo& g = sm.geo;
  const MultiGeo<NR>& m = sm.mg;
  if (warp == kProducerWarp) {
    mproducer_role<D, NR>(&tm, p, g, m, sm, s, unit, rank);
    cluster_wait();
  } else {
    const int t = role_tid();
    // q of every row (heads past G stay zero); rank 0 writes the last new
    // token (no row of this launch reads it)
    constexpr int QV = kMaxGroup * D / 8;
    for (int e = t; e < NR * QV; e += kConsumerThreads) {
      const int r = e / QV, et = e - r * QV;
      const int i = et * 8 / D, d0 = (et * 8) % D;
      float qf[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (i < p.G) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p.q + (((int64_t)r * p.units + unit) * p.G + i) * D + d0));
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(h2[j]);
          qf[2 * j] = f.x * p.scale;
          qf[2 * j + 1] = f.y * p.scale;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        sm.qs[r * kMaxGroup + i][d0 + j] = qf[j];
        sm.qsT[d0 + j][r * kMaxGroup + i] = qf[j];
      }
    }
    {  // the pending evictions' keys and values, the E tokens' keys
      const int nk = (m.ev_end[NR - 1] - g.fold_begin) * (D / 8), nv = (g.fold_end - g.fold_begin) * (D / 8);
      for (int e = t; e < nk + nv; e += kConsumerThreads) {
        const bool isk = e < nk;
        const int ee = isk ? e : e - nk, tok = ee / (D / 8), d0 = (ee % (D / 8)) * 8;
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>((isk ? p.k_cache : p.v_cache) +
                                                               ((int64_t)unit * p.cap + g.fold_begin + tok) * D + d0));
        float* dst = isk ? &sm.xk[tok][d0] : &sm.xv[tok][d0];
        *reinterpret_cast<float4*>(dst) = make_float4(bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y));
        *reinterpret_cast<float4*>(dst + 4) = make_float4(bf16_lo(raw.z), bf16_hi(raw.z), bf16_lo(raw.w), bf16_hi(raw.w));
      }
    }
    if (rank == 0 && p.k_new != nullptr)
      for (int e = t; e < D / 4; e += kConsumerThreads) {
        const int ee = (e % (D / 8)) * 8;
        const __nv_bfloat16* src = (e >= D / 8 ? p.v_new : p.k_new) + ((int64_t)(NR - 1) * p.units + unit) * D + ee;
        __nv_bfloat16* dst = (e >= D / 8 ? p.v_cache : p.k_cache) + ((int64_t)unit * p.cap + m.T_last) * D + ee;
        *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
      }
    named_sync(kBarConsumers, kConsumerThreads);
    if (warp < kAttnWarps) {
      mattn_role<D, NR>(p, g, m, sm, s, unit, rank);
      cluster_wait();
    } else {
      maux_role<D, NR>(p, g, m, sm, s, unit, rank);
    }
  }
  __syncthreads();
  mmerge_push<D, NR>(p, sm, rank);
  cluster_arrive_relaxed();
  mmerge_local<D, NR>(p, sm, unit, rank);
  cluster_wait();
}

template <int D, int NR>
constexpr size_t multi_smem_bytes() { return sizeof(MultiSmem<D, NR>) + 1024; }

static_assert(multi_smem_bytes<128, 4>() <= 232448, "shared memory per CTA");
static_assert(multi_smem_bytes<128, 2>() <= 232448, "shared memory per CTA");
static_assert(multi_smem_bytes<64, 4>() <= 232448, "shared memory per CTA");

template <int D, int NR>
cudaError_t set_multi_attributes() {
  const void* f = (const void*)multi_kernel<D, NR>;
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)multi_smem_bytes<D, NR>());
  if (e == cudaSuccess) e = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  return e;
}

template <int D, int NR>
int multi_clusters(int c) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = multi_smem_bytes<D, NR>();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = c;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (const void*)multi_kernel<D, NR>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace

int multi_rows_max() { return 4; }

int multi_score_capacity(int NR) { return kMScores / NR; }

int multi_merge_stride(int NR, int GD, int C) { return mmerge_stride(NR, GD, C); }

cudaError_t prepare_multi(int D) {
  cudaError_t e = D == 128 ? set_multi_attributes<128, 2>() : set_multi_attributes<64, 2>();
  if (e == cudaSuccess) e = D == 128 ? set_multi_attributes<128, 4>() : set_multi_attributes<64, 4>();
  return e;
}

int multi_max_clusters(int D, int NR, int c) {
  if (c > kMultiMaxCluster) return 0;  // the merge slots are sized for at most this many ranks
  if (NR == 2) return D == 128 ? multi_clusters<128, 2>(c) : multi_clusters<64, 2>(c);
  return D == 128 ? multi_clusters<128, 4>(c) : multi_clusters<64, 4>(c);
}

cudaError_t launch_multi(const CUtensorMap* maps, const FusedParams& p, int D, int NR, cudaStream_t s) {
  KVMaps tm;
  tm.k64 = maps[0];
  tm.v64 = maps[1];
  tm.k16 = maps[2];
  tm.v16 = maps[3];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.units * p.C));
  cfg.blockDim = dim3(kFThreads);
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
  if (NR == 2) {
    cfg.dynamicSmemBytes = D == 128 ? multi_smem_bytes<128, 2>() : multi_smem_bytes<64, 2>();
    return D == 128 ? cudaLaunchKernelEx(&cfg, multi_kernel<128, 2>, tm, p) : cudaLaunchKernelEx(&cfg, multi_kernel<64, 2>, tm, p);
  }
  cfg.dynamicSmemBytes = D == 128 ? multi_smem_bytes<128, 4>() : multi_smem_bytes<64, 4>();
  return D == 128 ? cudaLaunchKernelEx(&cfg, multi_kernel<128, 4>, tm, p) : cudaLaunchKernelEx(&cfg, multi_kernel<64, 4>, tm, p);
}

}  // namespace hyb
