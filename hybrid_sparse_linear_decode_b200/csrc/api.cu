// C ABI of the hybrid sparse + linear decode attention: argument checks, the
// workspace layout, TMA descriptors and kernel launches.  Host code only.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <new>

#include <nvtx3/nvToolsExt.h>

#include "../../include/hyb_attn.h"
#include "hyb_internal.h"
#include "k_select.h"

using namespace hyb;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Workspace regions.  The decode uses status, scores and sel; init uses the
// fp64 accumulators H64 and z64; hyb_attn_step_host the staging copies.
struct WsLayout {
  size_t status, scores, sel, H64, z64, stage_q, stage_k, stage_v, stage_out, total;
};

struct Checked {
  int D, G, units;
  int64_t max_blocks;
};

int check_config(const hyb_attn_config* c, Checked* out) {
  if (c == nullptr) return HYB_EINVAL;
  if (c->batch < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1) return HYB_EINVAL;
  if (c->n_q_heads % c->n_kv_heads != 0) return HYB_EINVAL;
  const int G = c->n_q_heads / c->n_kv_heads;
  if (G != 1 && G != 2 && G != 4) return HYB_EINVAL;
  if (c->head_dim != 64 && c->head_dim != 128) return HYB_EINVAL;
  if (c->block_size < 1 || c->n_sink < 0 || c->window < 0 || c->top_k < 0) return HYB_EINVAL;
  if (c->capacity < 1) return HYB_EINVAL;
  if (!(c->scale >= 0.f) || !std::isfinite(c->scale)) return HYB_EINVAL;
  const int64_t units = (int64_t)c->batch * c->n_kv_heads;
  if (units > (1 << 20)) return HYB_EINVAL;
  if (units * c->capacity >= ((int64_t)1 << 31)) return HYB_EINVAL;  // TMA row coordinate is int32
  if ((int64_t)c->n_sink + c->window + c->top_k * (int64_t)c->block_size >= ((int64_t)1 << 30)) return HYB_EINVAL;
  const int64_t ev_cap = c->capacity - c->n_sink - c->window;
  const int64_t mb = ev_cap > 0 ? ceil_div(ev_cap, c->block_size) : 0;
  if (mb >= ((int64_t)1 << 30)) return HYB_EINVAL;
  // per-head budgets refine (window, top_k): windows at least `window`, top-k at most `top_k`
  if ((c->head_window == nullptr) != (c->head_top_k == nullptr)) return HYB_EINVAL;
  if (c->head_window != nullptr) {
    if (c->n_kv_heads > kMaxHeadBudgets) return HYB_EINVAL;
    for (int h = 0; h < c->n_kv_heads; ++h) {
      if (c->head_window[h] < c->window || c->head_top_k[h] < 0 || c->head_top_k[h] > c->top_k) return HYB_EINVAL;
      if ((int64_t)c->n_sink + c->head_window[h] >= ((int64_t)1 << 30)) return HYB_EINVAL;
    }
  }
  if (out) {
    out->D = c->head_dim;
    out->G = G;
    out->units = (int)units;
    out->max_blocks = mb;
  }
  return HYB_OK;
}

WsLayout ws_layout(const hyb_attn_config& c, const Checked& k) {
  WsLayout w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  const size_t U = (size_t)k.units, D = (size_t)k.D, G = (size_t)k.G;
  w.status = take(sizeof(uint32_t));
  w.scores = take(U * (size_t)(k.max_blocks > 0 ? k.max_blocks : 1) * sizeof(float));
  w.sel = take(U * (size_t)(c.top_k > 0 ? c.top_k : 1) * sizeof(int32_t));
  w.H64 = take(U * D * D * sizeof(double));
  w.z64 = take(U * 2 * D * sizeof(double));
  w.stage_q = take(U * G * D * 2);
  w.stage_k = take(U * D * 2);
  w.stage_v = take(U * D * 2);
  w.stage_out = take(U * G * D * sizeof(float));
  w.total = off;
  return w;
}

Geometry geometry(const hyb_attn_config& c, int64_t T) {
  Geometry g{};
  const int64_t S = c.n_sink, W = c.window, Bk = c.block_size;
  g.T = T;
  g.sink_len = T < S ? T : S;
  g.win_start = T > S ? (T - W > S ? T - W : S) : T;
  g.ev_end = T > S + W ? T - W : S;
  g.nb = g.ev_end > S ? ceil_div(g.ev_end - S, Bk) : 0;
  g.k_eff = c.top_k < g.nb ? c.top_k : g.nb;
  g.n_sink_chunks = (int32_t)ceil_div(g.sink_len, kTile);
  g.n_win_chunks = (int32_t)ceil_div(T - g.win_start, kTile);
  g.chunks_per_block = (int32_t)ceil_div(Bk, kTile);
  g.n_sel_chunks = (int32_t)(g.k_eff * g.chunks_per_block);
  g.chunks_per_unit = g.n_sink_chunks + g.n_win_chunks + g.n_sel_chunks;
  return g;
}

// CTAs (one thread-block cluster) per unit: the largest C <= kMaxCluster with
// one CTA per SM for every unit (units * C <= n_sm) and, when the device's
// limits are known (fits[C] = clusters of C CTAs it can hold at once), every
// unit's cluster resident at the same time.
int cluster_ctas(int units, int n_sm, const int* fits) {
  for (int c = kMaxCluster; c > 1; --c)
    if ((int64_t)units * c <= n_sm && (fits == nullptr || fits[c] >= units)) return c;
  return 1;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range around every entry point (visible to Nsight tools; costs a
// call into a stub when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
#define HYB_RANGE NvtxRange hyb_range_(__func__)

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Record a failed CUDA call and map it to HYB_ECUDA.
int cuda_fail(cudaError_t e) {
  g_last_cuda_error = e;
  return HYB_ECUDA;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// KV cache viewed as [rows = B*Hkv*capacity][D/64][64] bf16; a box is
// `box_rows` rows x D columns, swizzled 128 B.
bool make_kv_map(CUtensorMap* m, void* base, int64_t rows, int D, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)(D / 64), (cuuint64_t)rows};
  cuuint64_t strides[2] = {128, (cuuint64_t)D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)(D / 64), (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool is_device_ptr(const void* p, int device) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice && a.device == device;
}

}  // namespace

// Fixed scratch of hyb_attn_decode_noalloc (block scores and the selection of
// one decode): a file-scope device array, one per GPU that loads this library.
// Host code only ever uses its device address, looked up once per device with
// that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[HYB_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

int noalloc_scratch(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return HYB_EINVAL;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[device] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    g_noalloc_addr[device] = p;
  }
  *out = g_noalloc_addr[device];
  return HYB_OK;
}
}  // namespace

struct hyb_attn_ctx {
  hyb_attn_config cfg;
  hyb_attn_buffers buf;
  Checked ck;
  WsLayout ws;
  int64_t T;            // length of the longest row (row b: T - tb.row_lag[b])
  int64_t pending;      // appends whose evictions are not folded into the state yet
  UnitTables tb;        // per-row lengths and per-head budgets (uniform when not given)
  int device, n_sm;
  int fits[kMaxCluster + 1];  // clusters of C CTAs of the decode kernel the device holds at once
  int fits_multi[2][kMaxCluster + 1];  // the same for the multi-query kernel with 2 and 4 rows
  float scale;
  uint64_t wait_ns;     // limit of the kernels' bounded waits for progress
  uint32_t test_flags;  // HYB_TEST_* failure injection (tests only)
  uint32_t* status;     // the device status word (in the context's workspace)
  CUtensorMap maps[4];  // K, V with 64-row boxes; K, V with 16-row boxes
  cudaEvent_t ev_begin, ev_end;
  template <class P>
  P* w(size_t off) const {
    return reinterpret_cast<P*>(static_cast<uint8_t*>(buf.workspace) + off);
  }
};

namespace {

FusedParams fused_params(const hyb_attn_ctx* x) {
  const hyb_attn_config& c = x->cfg;
  const Checked& k = x->ck;
  FusedParams fp{};
  fp.mu = x->buf.mu;
  fp.var = x->buf.var;
  fp.H = x->buf.H;
  fp.zk = x->buf.zk;
  fp.zv = x->buf.zv;
  fp.n = x->buf.n;
  fp.k_cache = static_cast<__nv_bfloat16*>(x->buf.k_cache);
  fp.v_cache = static_cast<__nv_bfloat16*>(x->buf.v_cache);
  fp.scores = x->w<float>(x->ws.scores);
  fp.sel = x->w<int32_t>(x->ws.sel);
  fp.status = x->status;
  fp.cap = c.capacity;
  fp.max_blocks = k.max_blocks > 0 ? k.max_blocks : 1;
  fp.T = (int32_t)x->T;
  fp.S = c.n_sink;
  fp.W = c.window;
  fp.Bk = c.block_size;
  fp.top_k = c.top_k;
  fp.pending = (int32_t)x->pending;
  fp.chunks_per_block = (int32_t)ceil_div(c.block_size, kTile);
  fp.units = k.units;
  fp.Hkv = c.n_kv_heads;
  fp.G = k.G;
  fp.C = cluster_ctas(k.units, x->n_sm, x->fits);
  fp.mstride = merge_stride(k.G * k.D, fp.C);
  for (int r = 0; r <= fp.C; ++r) fp.mslice[r] = merge_slice_begin(k.G * k.D, fp.C, r);
  fp.scale = x->scale;
  fp.wait_ns = x->wait_ns;
  fp.test_flags = x->test_flags;
  return fp;
}

// Does some unit have more than kStreamBlocks candidate blocks?  The most
// blocks are those of the longest row under the smallest window, which is the
// configuration's window (every per-head window is at least that).
bool stream_variant(const hyb_attn_ctx* x) { return geometry(x->cfg, x->T).nb > kStreamBlocks; }

// Several pending appends (a chunked append, or many appends since the last
// fold): one dense pass of fold_kernel over every unit's evictions, so that the
// decode kernel folds at most a few tokens itself.
int fold_pending(hyb_attn_ctx* x, cudaStream_t stream) {
  if (x->pending < kFoldKernelMin) return HYB_OK;
  FoldParams p{};
  p.k_cache = static_cast<const __nv_bfloat16*>(x->buf.k_cache);
  p.v_cache = static_cast<const __nv_bfloat16*>(x->buf.v_cache);
  p.H = x->buf.H;
  p.zk = x->buf.zk;
  p.zv = x->buf.zv;
  p.n = x->buf.n;
  p.mu = x->buf.mu;
  p.var = x->buf.var;
  p.cap = x->cfg.capacity;
  p.max_blocks = x->ck.max_blocks > 0 ? x->ck.max_blocks : 1;
  p.T = (int32_t)x->T;
  p.S = x->cfg.n_sink;
  p.W = x->cfg.window;
  p.Bk = x->cfg.block_size;
  p.pending = (int32_t)x->pending;
  p.units = x->ck.units;
  p.Hkv = x->cfg.n_kv_heads;
  p.tb = x->tb;
  const cudaError_t e = launch_fold(p, x->ck.D, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  x->pending = 0;
  return HYB_OK;
}

// One decode at the current T: one launch of the fused kernel (writes the
// appended token when k_new is given), after fold_kernel when several
// evictions are pending.
int decode_impl(hyb_attn_ctx* x, const void* q, float* out, const int32_t* sel_given, int32_t* sel_out,
                float* scores_out, const void* k_new, const void* v_new, cudaStream_t stream) {
  if (x == nullptr || q == nullptr || out == nullptr) return HYB_EINVAL;
  if (!aligned16(q) || !aligned16(out)) return HYB_EINVAL;
  if (sel_given != nullptr && !aligned16(sel_given)) return HYB_EINVAL;
  if (sel_out != nullptr && (reinterpret_cast<uintptr_t>(sel_out) & 3u)) return HYB_EINVAL;
  if (scores_out != nullptr && (reinterpret_cast<uintptr_t>(scores_out) & 15u)) return HYB_EINVAL;
  if ((k_new == nullptr) != (v_new == nullptr)) return HYB_EINVAL;
  if (k_new != nullptr && (!aligned16(k_new) || !aligned16(v_new))) return HYB_EINVAL;
  if (x->T == 0) return HYB_ESTATE;
  if (k_new != nullptr && x->T >= x->cfg.capacity) return HYB_ECAPACITY;
  const int rf = fold_pending(x, stream);
  if (rf != HYB_OK) return rf;
  FusedParams fp = fused_params(x);
  fp.q = static_cast<const __nv_bfloat16*>(q);
  if (scores_out) fp.scores = scores_out;
  fp.sel_given = sel_given;
  fp.sel_out = sel_given ? nullptr : sel_out;
  fp.out = out;
  fp.k_new = static_cast<const __nv_bfloat16*>(k_new);
  fp.v_new = static_cast<const __nv_bfloat16*>(v_new);
  const bool timed = x->ev_begin != nullptr && x->ev_end != nullptr;
  if (timed && cudaEventRecord(x->ev_begin, stream) != cudaSuccess) return HYB_ECUDA;
  const cudaError_t e = launch_fused(x->maps, fp, x->tb, stream_variant(x), x->ck.D, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  x->pending = 0;
  if (k_new != nullptr) {  // the new token's eviction, if any, is folded by the next decode
    x->T += 1;
    x->pending = 1;
  }
  if (timed && cudaEventRecord(x->ev_end, stream) != cudaSuccess) return HYB_ECUDA;
  return HYB_OK;
}

// Can the multi-query kernel take nr (2 or 4) rows from the current length?
// Uniform lengths and budgets, k <= 32, a window of at least nr - 1 tokens (the
// rows' new tokens then lie in the shared prefix), and the last row's block
// scores for every row fit the kernel's shared memory.
bool multi_fits(const hyb_attn_ctx* x, int nr) {
  const hyb_attn_config& c = x->cfg;
  if (x->tb.ragged || x->tb.per_head) return false;
  if (c.top_k > 32 || c.window < nr - 1) return false;
  if (x->T + nr > c.capacity) return false;
  const Geometry g = geometry(c, x->T + nr - 1);
  if (g.nb > multi_score_capacity(nr)) return false;
  const int C = cluster_ctas(x->ck.units, x->n_sm, x->fits_multi[nr == 2 ? 0 : 1]);
  return C >= 1 && x->ck.G <= kMaxGroup;
}

// nr consecutive decode + append steps in one launch of the multi-query kernel
// (after fold_kernel when many evictions are pending).
int decode_multi(hyb_attn_ctx* x, int nr, const void* q, const void* k_new, const void* v_new, float* out,
                 int32_t* sel_out, cudaStream_t stream) {
  const int rf = fold_pending(x, stream);
  if (rf != HYB_OK) return rf;
  FusedParams fp = fused_params(x);
  const Checked& k = x->ck;
  fp.C = cluster_ctas(k.units, x->n_sm, x->fits_multi[nr == 2 ? 0 : 1]);
  fp.mstride = multi_merge_stride(nr, k.G * k.D, fp.C);
  for (int r = 0; r <= fp.C; ++r) fp.mslice[r] = r * (nr * k.G * k.D) / fp.C;
  fp.q = static_cast<const __nv_bfloat16*>(q);
  fp.out = out;
  fp.sel_out = sel_out;
  fp.k_new = static_cast<const __nv_bfloat16*>(k_new);
  fp.v_new = static_cast<const __nv_bfloat16*>(v_new);
  const bool timed = x->ev_begin != nullptr && x->ev_end != nullptr;
  if (timed && cudaEventRecord(x->ev_begin, stream) != cudaSuccess) return HYB_ECUDA;
  const cudaError_t e = launch_multi(x->maps, fp, k.D, nr, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  x->T += nr;
  x->pending = nr;  // the state is folded to row 0's eviction edge
  if (timed && cudaEventRecord(x->ev_end, stream) != cudaSuccess) return HYB_ECUDA;
  return HYB_OK;
}

}  // namespace

extern "C" {

int hyb_attn_query_sizes(const hyb_attn_config* cfg, hyb_attn_sizes* out) {
  Checked k;
  const int rc = check_config(cfg, &k);
  if (rc != HYB_OK || out == nullptr) return rc != HYB_OK ? rc : HYB_EINVAL;
  const int64_t U = k.units, D = k.D;
  out->kv_cache_elems = U * cfg->capacity * D;
  out->H_elems = U * D * D;
  out->z_elems = U * D;
  out->n_elems = U;
  out->max_blocks = k.max_blocks;
  out->stats_elems = U * k.max_blocks * D;
  out->workspace_bytes = (int64_t)ws_layout(*cfg, k).total;
  return HYB_OK;
}

size_t hyb_attn_workspace_size(const hyb_attn_config* cfg) {
  Checked k;
  if (check_config(cfg, &k) != HYB_OK) return 0;
  return ws_layout(*cfg, k).total;
}

int hyb_attn_plan(const hyb_attn_config* cfg, int64_t T, int32_t n_sm, hyb_attn_plan_info* out) {
  Checked k;
  const int rc = check_config(cfg, &k);
  if (rc != HYB_OK) return rc;
  if (out == nullptr || T < 0 || T > cfg->capacity || n_sm < 1) return HYB_EINVAL;
  const Geometry g = geometry(*cfg, T);
  out->T = T;
  out->n_blocks = g.nb;
  out->k_eff = g.k_eff;
  out->exact_tokens = g.sink_len + (T - g.win_start) + g.k_eff * cfg->block_size;
  out->chunks_per_unit = g.chunks_per_unit;
  out->cluster_ctas = cluster_ctas(k.units, n_sm, nullptr);
  out->grid_ctas = k.units * out->cluster_ctas;
  return HYB_OK;
}

}  // extern "C"

namespace {

// Validate a configuration and its buffers and build the host context of a
// layer at length T (TMA descriptors, kernel attributes); no kernel is launched.
int create_ctx(const hyb_attn_config* cfg, const hyb_attn_buffers* buf, int64_t T, const int64_t* row_T,
               hyb_attn_ctx** out) {
  Checked k;
  if (check_config(cfg, &k) != HYB_OK || buf == nullptr) return HYB_EINVAL;
  UnitTables tb{};
  if (row_T != nullptr) {  // per-row lengths: T is the longest, row b lags it by T - row_T[b]
    if (cfg->batch > kMaxRaggedRows) return HYB_EINVAL;
    T = 0;
    for (int b = 0; b < cfg->batch; ++b) {
      if (row_T[b] < 1 || row_T[b] > cfg->capacity) return HYB_EINVAL;
      T = row_T[b] > T ? row_T[b] : T;
    }
    tb.ragged = 1;
    for (int b = 0; b < cfg->batch; ++b) tb.row_lag[b] = (int32_t)(T - row_T[b]);
  }
  if (T < 0 || T > cfg->capacity) return HYB_EINVAL;
  if (cfg->head_window != nullptr) {
    tb.per_head = 1;
    for (int h = 0; h < cfg->n_kv_heads; ++h) {
      tb.head_W[h] = cfg->head_window[h];
      tb.head_k[h] = cfg->head_top_k[h];
    }
  }
  const void* ptrs[] = {buf->k_cache, buf->v_cache, buf->H, buf->zk, buf->zv, buf->n, buf->workspace};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return HYB_EINVAL;
  if (k.max_blocks > 0 && (buf->mu == nullptr || buf->var == nullptr || !aligned16(buf->mu) || !aligned16(buf->var)))
    return HYB_EINVAL;
  if ((reinterpret_cast<uintptr_t>(buf->workspace) & (kAlign - 1)) != 0) return HYB_EINVAL;
  const WsLayout ws = ws_layout(*cfg, k);
  if (buf->workspace_bytes < ws.total) return HYB_EINVAL;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return HYB_ECUDA;
  if (!is_device_ptr(buf->k_cache, device) || !is_device_ptr(buf->v_cache, device) ||
      !is_device_ptr(buf->workspace, device) || !is_device_ptr(buf->H, device))
    return HYB_EINVAL;
  int n_sm = 0;
  if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return HYB_ECUDA;

  hyb_attn_ctx* x = new (std::nothrow) hyb_attn_ctx();
  if (x == nullptr) return HYB_ENOMEM;
  x->cfg = *cfg;
  x->cfg.head_window = x->cfg.head_top_k = nullptr;  // the caller's arrays are copied into tb
  x->buf = *buf;
  x->ck = k;
  x->ws = ws;
  x->T = T;
  x->pending = 0;
  x->tb = tb;
  x->device = device;
  x->n_sm = n_sm;
  for (int c = 0; c <= kMaxCluster; ++c) x->fits[c] = x->fits_multi[0][c] = x->fits_multi[1][c] = 0;
  x->scale = cfg->scale > 0.f ? cfg->scale : 1.0f / std::sqrt((float)k.D);
  x->wait_ns = kWaitLimit;
  x->test_flags = 0u;
  x->status = x->w<uint32_t>(ws.status);
  x->ev_begin = x->ev_end = nullptr;
  const int64_t rows = (int64_t)k.units * cfg->capacity;
  if (!make_kv_map(&x->maps[0], buf->k_cache, rows, k.D, kTile) ||
      !make_kv_map(&x->maps[1], buf->v_cache, rows, k.D, kTile) ||
      !make_kv_map(&x->maps[2], buf->k_cache, rows, k.D, kBoxRows) ||
      !make_kv_map(&x->maps[3], buf->v_cache, rows, k.D, kBoxRows)) {
    delete x;
    return HYB_ECUDA;
  }
  cudaError_t pe = prepare_fused(k.D);
  if (pe == cudaSuccess) pe = prepare_state(k.D);
  if (pe == cudaSuccess) pe = prepare_multi(k.D);
  if (pe == cudaSuccess) pe = prepare_strided_select(k.D);
  if (pe != cudaSuccess) {
    delete x;
    return cuda_fail(pe);
  }
  for (int c = 2; c <= kMaxCluster; ++c) {
    x->fits[c] = fused_max_clusters(k.D, c);
    x->fits_multi[0][c] = multi_max_clusters(k.D, 2, c);
    x->fits_multi[1][c] = multi_max_clusters(k.D, 4, c);
  }
  *out = x;
  return HYB_OK;
}

}  // namespace

extern "C" {

}  // extern "C"

namespace {

int init_impl(hyb_attn_ctx** out, const hyb_attn_config* cfg, const hyb_attn_buffers* buf, int64_t T0,
              const int64_t* row_T0, cudaStream_t stream) {
  if (out == nullptr) return HYB_EINVAL;
  *out = nullptr;
  hyb_attn_ctx* x = nullptr;
  const int rc = create_ctx(cfg, buf, T0, row_T0, &x);
  if (rc != HYB_OK) return rc;
  const Checked& k = x->ck;
  InitParams ip{};
  ip.k_cache = static_cast<const __nv_bfloat16*>(buf->k_cache);
  ip.v_cache = static_cast<const __nv_bfloat16*>(buf->v_cache);
  ip.H = buf->H;
  ip.zk = buf->zk;
  ip.zv = buf->zv;
  ip.n = buf->n;
  ip.mu = buf->mu;
  ip.var = buf->var;
  ip.H64 = x->w<double>(x->ws.H64);
  ip.z64 = x->w<double>(x->ws.z64);
  ip.status = x->status;
  ip.cap = cfg->capacity;
  ip.max_blocks = k.max_blocks > 0 ? k.max_blocks : 1;
  ip.T = (int32_t)x->T;
  ip.S = cfg->n_sink;
  ip.W = cfg->window;
  ip.Bk = cfg->block_size;
  ip.units = k.units;
  ip.Hkv = cfg->n_kv_heads;
  ip.tb = x->tb;
  // the longest evicted range and the most blocks over the units (the grid's extent)
  int64_t ev_max = 0;
  for (int u = 0; u < k.units; ++u) {
    const UnitGeo g = unit_geo(&x->tb, u, cfg->n_kv_heads, (int32_t)x->T, cfg->n_sink, cfg->window,
                               cfg->block_size, 0, 1, 0);
    ev_max = std::max<int64_t>(ev_max, g.ev_end - cfg->n_sink);
  }
  ip.ev_max = (int32_t)ev_max;
  ip.nb_max = (int32_t)ceil_div(ev_max, cfg->block_size);
  ip.tokens_per_cta = 2048;
  cudaError_t e = cudaMemsetAsync(ip.H64, 0, (size_t)k.units * k.D * k.D * sizeof(double), stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(ip.z64, 0, (size_t)k.units * 2 * k.D * sizeof(double), stream);
  if (e == cudaSuccess) e = launch_init(ip, k.D, stream);
  if (e != cudaSuccess) {
    delete x;
    return cuda_fail(e);
  }
  *out = x;
  return HYB_OK;
}

int attach_impl(hyb_attn_ctx** out, const hyb_attn_config* cfg, const hyb_attn_buffers* buf, int64_t T,
                const int64_t* row_T, cudaStream_t stream) {
  if (out == nullptr) return HYB_EINVAL;
  *out = nullptr;
  hyb_attn_ctx* x = nullptr;
  const int rc = create_ctx(cfg, buf, T, row_T, &x);
  if (rc != HYB_OK) return rc;
  const cudaError_t e = cudaMemsetAsync(x->status, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) {
    delete x;
    return cuda_fail(e);
  }
  *out = x;
  return HYB_OK;
}

}  // namespace

extern "C" {

int hyb_attn_init(hyb_attn_ctx** out, const hyb_attn_config* cfg, const hyb_attn_buffers* buf, int64_t T0,
                  cudaStream_t stream) {
  HYB_RANGE;
  return init_impl(out, cfg, buf, T0, nullptr, stream);
}

int hyb_attn_init_rows(hyb_attn_ctx** out, const hyb_attn_config* cfg, const hyb_attn_buffers* buf,
                       const int64_t* row_T0, cudaStream_t stream) {
  HYB_RANGE;
  if (row_T0 == nullptr) return HYB_EINVAL;
  return init_impl(out, cfg, buf, 0, row_T0, stream);
}

int hyb_attn_attach(hyb_attn_ctx** out, const hyb_attn_config* cfg, const hyb_attn_buffers* buf, int64_t T,
                    cudaStream_t stream) {
  HYB_RANGE;
  return attach_impl(out, cfg, buf, T, nullptr, stream);
}

int hyb_attn_attach_rows(hyb_attn_ctx** out, const hyb_attn_config* cfg, const hyb_attn_buffers* buf,
                         const int64_t* row_T, cudaStream_t stream) {
  HYB_RANGE;
  if (row_T == nullptr) return HYB_EINVAL;
  return attach_impl(out, cfg, buf, 0, row_T, stream);
}

int hyb_attn_append_chunk(hyb_attn_ctx* x, const void* k_new, const void* v_new, int32_t n, cudaStream_t stream) {
  HYB_RANGE;
  if (x == nullptr || k_new == nullptr || v_new == nullptr || n < 1 || n > 65535) return HYB_EINVAL;
  if (!aligned16(k_new) || !aligned16(v_new)) return HYB_EINVAL;
  if (x->T + n > x->cfg.capacity) return HYB_ECAPACITY;
  AppendParams p{};
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.k_cache = static_cast<__nv_bfloat16*>(x->buf.k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(x->buf.v_cache);
  p.cap = x->cfg.capacity;
  p.T = (int32_t)x->T;
  p.units = x->ck.units;
  p.Hkv = x->cfg.n_kv_heads;
  p.n = n;
  p.tb = x->tb;
  const cudaError_t e = launch_append(p, x->ck.D, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  x->T += n;
  x->pending += n;  // their evictions are folded by the next decode or state sync
  return HYB_OK;
}

int hyb_attn_append(hyb_attn_ctx* x, const void* k_new, const void* v_new, cudaStream_t stream) {
  return hyb_attn_append_chunk(x, k_new, v_new, 1, stream);
}

int hyb_attn_sync_state(hyb_attn_ctx* x, cudaStream_t stream) {
  HYB_RANGE;
  if (x == nullptr) return HYB_EINVAL;
  if (x->pending == 0) return HYB_OK;  // nothing appended since the last fold
  if (x->pending >= kFoldKernelMin) return fold_pending(x, stream);
  FusedParams fp = fused_params(x);   // q == null: fold only
  const cudaError_t e = launch_fused(x->maps, fp, x->tb, stream_variant(x), x->ck.D, stream);
  if (e != cudaSuccess) return cuda_fail(e);
  x->pending = 0;
  return HYB_OK;
}

int hyb_attn_decode(hyb_attn_ctx* ctx, const void* q, float* out, int32_t* sel_out, float* scores_out,
                    cudaStream_t stream) {
  HYB_RANGE;
  return decode_impl(ctx, q, out, nullptr, sel_out, scores_out, nullptr, nullptr, stream);
}

int hyb_attn_decode_append(hyb_attn_ctx* ctx, const void* q, const void* k_new, const void* v_new, float* out,
                           int32_t* sel_out, float* scores_out, cudaStream_t stream) {
  HYB_RANGE;
  if (k_new == nullptr || v_new == nullptr) return HYB_EINVAL;
  return decode_impl(ctx, q, out, nullptr, sel_out, scores_out, k_new, v_new, stream);
}

int hyb_attn_decode_chunk(hyb_attn_ctx* x, const void* q, const void* k_new, const void* v_new, int32_t n,
                          float* out, int32_t* sel_out, cudaStream_t stream) {
  HYB_RANGE;
  if (x == nullptr || q == nullptr || k_new == nullptr || v_new == nullptr || out == nullptr || n < 1)
    return HYB_EINVAL;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out)) return HYB_EINVAL;
  if (sel_out != nullptr && (reinterpret_cast<uintptr_t>(sel_out) & 3u)) return HYB_EINVAL;
  if (x->T == 0) return HYB_ESTATE;
  if (x->T + n > x->cfg.capacity) return HYB_ECAPACITY;
  const size_t U = (size_t)x->ck.units, D = (size_t)x->ck.D, G = (size_t)x->ck.G;
  int32_t j = 0;
  while (j < n) {  // rows j, j + 1, ...: decodes at lengths T + j, ..., each then appending its token
    const int want = n - j >= 4 ? 4 : n - j >= 2 ? 2 : 1;
    const bool multi = want > 1 && multi_fits(x, want);
    const int nr = multi ? want : 1;
    const char* qj = static_cast<const char*>(q) + j * U * G * D * 2;
    const char* kj = static_cast<const char*>(k_new) + j * U * D * 2;
    const char* vj = static_cast<const char*>(v_new) + j * U * D * 2;
    int32_t* sj = sel_out == nullptr ? nullptr : sel_out + j * U * (size_t)x->cfg.top_k;
    const int r = multi ? decode_multi(x, nr, qj, kj, vj, out + j * U * G * D, sj, stream)
                        : decode_impl(x, qj, out + j * U * G * D, nullptr, sj, nullptr, kj, vj, stream);
    if (r != HYB_OK) return r;
    j += nr;
  }
  return HYB_OK;
}

int hyb_attn_decode_with_selection(hyb_attn_ctx* ctx, const void* q, const int32_t* sel, float* out,
                                   cudaStream_t stream) {
  HYB_RANGE;
  if (sel == nullptr) return HYB_EINVAL;
  return decode_impl(ctx, q, out, sel, nullptr, nullptr, nullptr, nullptr, stream);
}

int hyb_attn_decode_strided(hyb_attn_ctx* x, const void* q, int32_t k_top, int32_t stride, float* out,
                            int32_t* sel_out, cudaStream_t stream) {
  HYB_RANGE;
  if (x == nullptr || q == nullptr || out == nullptr || stride < 1 || k_top < 0) return HYB_EINVAL;
  if (x->tb.ragged || x->tb.per_head) return HYB_EINVAL;  // one length and one budget for every unit
  if (!aligned16(q) || (sel_out != nullptr && (reinterpret_cast<uintptr_t>(sel_out) & 3u))) return HYB_EINVAL;
  const Geometry g = geometry(x->cfg, x->T);
  const int64_t nb = g.nb, n_fixed = nb / stride;
  const int64_t n_sel = n_fixed + std::min<int64_t>(k_top, nb - n_fixed);
  if (n_sel > x->cfg.top_k) return HYB_EINVAL;  // the selection row holds top_k blocks
  const size_t smem = strided_select_smem(x->ck.D, (int)nb);
  if (nb > 0 && smem == 0) return HYB_EINVAL;
  // Several pending evictions are folded by one dense pass first; a few (the
  // previous step's) are folded by the selection launch for its scores and by
  // the decode into the state, as in a plain decode.
  int rc = fold_pending(x, stream);
  if (rc != HYB_OK) return rc;
  int32_t* sel = x->w<int32_t>(x->ws.sel);
  if (nb > 0) {
    StridedSelParams sp{};
    sp.q = static_cast<const __nv_bfloat16*>(q);
    sp.mu = x->buf.mu;
    sp.var = x->buf.var;
    sp.sel = sel;
    sp.sel_copy = sel_out;
    sp.status = x->status;
    sp.max_blocks = x->ck.max_blocks > 0 ? x->ck.max_blocks : 1;
    sp.units = x->ck.units;
    sp.nb = (int32_t)nb;
    sp.G = x->ck.G;
    sp.k = k_top;
    sp.stride = stride;
    sp.width = x->cfg.top_k;
    sp.scale = x->scale;  // resolved (1/sqrt(d) when the configuration gives 0)
    sp.parts = strided_select_parts((int)nb, x->ck.units, x->n_sm);
    sp.k_cache = static_cast<const __nv_bfloat16*>(x->buf.k_cache);
    sp.cap = x->cfg.capacity;
    sp.S = x->cfg.n_sink;
    sp.Bk = x->cfg.block_size;
    sp.fold_end = ev_end_at((int32_t)x->T, x->cfg.n_sink, x->cfg.window);
    sp.fold_begin = ev_end_at((int32_t)(x->T - x->pending > 0 ? x->T - x->pending : 0), x->cfg.n_sink, x->cfg.window);
    const cudaError_t e = launch_strided_select(sp, x->ck.D, stream);
    if (e != cudaSuccess) return cuda_fail(e);
  } else if (sel_out != nullptr && x->cfg.top_k > 0) {
    if (cudaMemsetAsync(sel_out, 0xff, (size_t)x->ck.units * x->cfg.top_k * sizeof(int32_t), stream) != cudaSuccess)
      return HYB_ECUDA;
  }
  return decode_impl(x, q, out, nb > 0 ? sel : nullptr, nullptr, nullptr, nullptr, nullptr, stream);
}

int hyb_attn_step_host(hyb_attn_ctx* x, const void* q_host, const void* k_host, const void* v_host,
                       float* out_host, cudaStream_t stream) {
  HYB_RANGE;
  if (x == nullptr || q_host == nullptr || out_host == nullptr) return HYB_EINVAL;
  if ((k_host == nullptr) != (v_host == nullptr)) return HYB_EINVAL;
  if (k_host != nullptr && x->T >= x->cfg.capacity) return HYB_ECAPACITY;
  const size_t U = (size_t)x->ck.units, D = (size_t)x->ck.D, G = (size_t)x->ck.G;
  void* dq = x->w<void>(x->ws.stage_q);
  float* dout = x->w<float>(x->ws.stage_out);
  if (cudaMemcpyAsync(dq, q_host, U * G * D * 2, cudaMemcpyHostToDevice, stream) != cudaSuccess) return HYB_ECUDA;
  if (k_host != nullptr) {
    if (cudaMemcpyAsync(x->w<void>(x->ws.stage_k), k_host, U * D * 2, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(x->w<void>(x->ws.stage_v), v_host, U * D * 2, cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return HYB_ECUDA;
  }
  const void* dk = k_host ? x->w<void>(x->ws.stage_k) : nullptr;
  const void* dv = k_host ? x->w<void>(x->ws.stage_v) : nullptr;
  const int rc = decode_impl(x, dq, dout, nullptr, nullptr, nullptr, dk, dv, stream);
  if (rc != HYB_OK) return rc;
  if (cudaMemcpyAsync(out_host, dout, U * G * D * sizeof(float), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return HYB_ECUDA;
  return HYB_OK;
}

size_t hyb_attn_step_layers_staging_bytes(hyb_attn_ctx* const* ctxs, int32_t n_layers) {
  if (ctxs == nullptr || n_layers < 1) return 0;
  size_t in = 0, out = 0;
  for (int32_t l = 0; l < n_layers; ++l) {
    const hyb_attn_ctx* x = ctxs[l];
    if (x == nullptr) return 0;
    const size_t U = (size_t)x->ck.units, D = (size_t)x->ck.D, G = (size_t)x->ck.G;
    in += U * G * D * 2 + 2 * U * D * 2;
    out += U * G * D * 4;
  }
  return align_up(in) + out;
}

int hyb_attn_step_layers_host(hyb_attn_ctx* const* ctxs, int32_t n_layers, const void* in_host, float* out_host,
                              void* staging, size_t staging_bytes, cudaStream_t stream) {
  HYB_RANGE;
  if (ctxs == nullptr || n_layers < 1 || in_host == nullptr || out_host == nullptr || staging == nullptr)
    return HYB_EINVAL;
  if ((reinterpret_cast<uintptr_t>(staging) & (kAlign - 1)) != 0) return HYB_EINVAL;
  const size_t need = hyb_attn_step_layers_staging_bytes(ctxs, n_layers);
  if (need == 0 || staging_bytes < need) return HYB_EINVAL;
  size_t in_bytes = 0, out_bytes = 0;
  for (int32_t l = 0; l < n_layers; ++l) {
    const hyb_attn_ctx* x = ctxs[l];
    if (x->T >= x->cfg.capacity) return HYB_ECAPACITY;  // nothing is enqueued when a layer is full
    const size_t U = (size_t)x->ck.units, D = (size_t)x->ck.D, G = (size_t)x->ck.G;
    in_bytes += U * G * D * 2 + 2 * U * D * 2;
    out_bytes += U * G * D * 4;
  }
  uint8_t* din = static_cast<uint8_t*>(staging);
  float* dout = reinterpret_cast<float*>(din + align_up(in_bytes));
  // one copy in, every layer's decode + append back to back (chained launches), one copy out
  if (cudaMemcpyAsync(din, in_host, in_bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess) return HYB_ECUDA;
  size_t ioff = 0, ooff = 0;
  for (int32_t l = 0; l < n_layers; ++l) {
    hyb_attn_ctx* x = ctxs[l];
    const size_t U = (size_t)x->ck.units, D = (size_t)x->ck.D, G = (size_t)x->ck.G;
    const uint8_t* q = din + ioff;
    const uint8_t* k = q + U * G * D * 2;
    const uint8_t* v = k + U * D * 2;
    const int rc = decode_impl(x, q, dout + ooff, nullptr, nullptr, nullptr, k, v, stream);
    if (rc != HYB_OK) return rc;
    ioff += U * G * D * 2 + 2 * U * D * 2;
    ooff += U * G * D;
  }
  if (cudaMemcpyAsync(out_host, dout, out_bytes, cudaMemcpyDeviceToHost, stream) != cudaSuccess) return HYB_ECUDA;
  return HYB_OK;
}

int hyb_attn_decode_noalloc(hyb_attn_ctx* x, const void* q, float* out, int32_t* sel_out, cudaStream_t stream) {
  HYB_RANGE;
  if (x == nullptr) return HYB_EINVAL;
  int device = -1;
  if (cudaGetDevice(&device) != cudaSuccess) return HYB_ECUDA;
  if (device != x->device) return HYB_EINVAL;
  // the decode's scratch (block scores, the selection) is the workspace regions
  // before the init accumulators; the array takes the same layout
  if (x->ws.H64 > HYB_NOALLOC_SCRATCH_BYTES) return HYB_ESCRATCH;
  void* scratch = nullptr;
  const int rc = noalloc_scratch(device, &scratch);
  if (rc != HYB_OK) return rc;
  // Nothing in the scratch needs to start at zero: every score and selection
  // entry a decode reads it has written first.  The device status word stays
  // the context's own, so that hyb_attn_status reports this call's bits.
  hyb_attn_ctx view = *x;  // the same context with its scratch rebased onto the fixed array
  view.buf.workspace = scratch;
  view.buf.workspace_bytes = HYB_NOALLOC_SCRATCH_BYTES;
  const int drc = decode_impl(&view, q, out, nullptr, sel_out, nullptr, nullptr, nullptr, stream);
  x->pending = view.pending;  // the state buffers are the context's own
  return drc;
}

int64_t hyb_attn_length(const hyb_attn_ctx* x) { return x ? x->T : -1; }

int64_t hyb_attn_row_length(const hyb_attn_ctx* x, int32_t b) {
  if (x == nullptr || b < 0 || b >= x->cfg.batch) return -1;
  return x->T - (x->tb.ragged ? x->tb.row_lag[b] : 0);
}

int hyb_attn_status(hyb_attn_ctx* x, uint32_t* flags, int clear, cudaStream_t stream) {
  HYB_RANGE;
  if (x == nullptr || flags == nullptr) return HYB_EINVAL;
  uint32_t* d = x->w<uint32_t>(x->ws.status);
  if (cudaMemcpyAsync(flags, d, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream) != cudaSuccess) return HYB_ECUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return HYB_ECUDA;
  if (clear && cudaMemsetAsync(d, 0, sizeof(uint32_t), stream) != cudaSuccess) return HYB_ECUDA;
  return HYB_OK;
}

int hyb_attn_set_timing_events(hyb_attn_ctx* x, cudaEvent_t begin, cudaEvent_t end) {
  if (x == nullptr || ((begin == nullptr) != (end == nullptr))) return HYB_EINVAL;
  x->ev_begin = begin;
  x->ev_end = end;
  return HYB_OK;
}

int hyb_attn_set_wait_limit(hyb_attn_ctx* x, uint64_t ns) {
  if (x == nullptr) return HYB_EINVAL;
  if (ns == 0) ns = kWaitLimit;
  if (ns < 100000ull || ns > 60000000000ull) return HYB_EINVAL;
  x->wait_ns = ns;
  return HYB_OK;
}

int hyb_attn_set_test_flags(hyb_attn_ctx* x, uint32_t flags) {
  if (x == nullptr || (flags & ~HYB_TEST_WITHHOLD_SCORES) != 0u) return HYB_EINVAL;
  x->test_flags = flags;
  return HYB_OK;
}

void hyb_attn_destroy(hyb_attn_ctx* x) { delete x; }

const char* hyb_attn_last_cuda_error(void) {
  static thread_local char buf[256];
  snprintf(buf, sizeof(buf), "%s: %s", cudaGetErrorName(g_last_cuda_error), cudaGetErrorString(g_last_cuda_error));
  return buf;
}

const char* hyb_attn_strerror(int code) {
  switch (code) {
    case HYB_OK: return "ok";
    case HYB_EINVAL: return "invalid argument (shape, pointer, alignment or unsupported configuration)";
    case HYB_ECAPACITY: return "KV cache capacity reached";
    case HYB_ECUDA: return "CUDA call or kernel launch failed";
    case HYB_ESTATE: return "call not valid in the current state";
    case HYB_ENOMEM: return "host allocation failed";
    case HYB_ESCRATCH: return "decode scratch exceeds the fixed device area of the no-allocation entry point";
    default: return "unknown error code";
  }
}

}  // extern "C"
