// Device twin of syngen/host.py: fills KV caches of the synthetic workloads in
// HBM with the same bits the numpy generator produces.
//
// Every operation is a correctly rounded fp64 intrinsic (__dadd_rn, __dmul_rn,
// __ddiv_rn, __dsqrt_rn: no fused multiply-add contraction), the series
// coefficients are the same exact hex literals as on the host, and the final
// rounding is fp64 -> fp32 -> bf16, nearest-even at each step.  This library
// holds no arithmetic of the attention method.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__constant__ double kLnCoef[12] = {
    0x1.0000000000000p+0, 0x1.5555555555555p-2, 0x1.999999999999ap-3, 0x1.2492492492492p-3,
    0x1.c71c71c71c71cp-4, 0x1.745d1745d1746p-4, 0x1.3b13b13b13b14p-4, 0x1.1111111111111p-4,
    0x1.e1e1e1e1e1e1ep-5, 0x1.af286bca1af28p-5, 0x1.8618618618618p-5, 0x1.642c8590b2164p-5};
__constant__ double kCosCoef[13] = {
    0x1.0000000000000p+0,  -0x1.0000000000000p-1, 0x1.5555555555555p-5,  -0x1.6c16c16c16c17p-10,
    0x1.a01a01a01a01ap-16, -0x1.27e4fb7789f5cp-22, 0x1.1eed8eff8d898p-29, -0x1.93974a8c07c9dp-37,
    0x1.ae7f3e733b81fp-45, -0x1.6827863b97d97p-53, 0x1.e542ba4020225p-62, -0x1.0ce396db7f853p-70,
    0x1.f2cf01972f578p-80};
__constant__ double kSinCoef[13] = {
    0x1.0000000000000p+0,  -0x1.5555555555555p-3, 0x1.1111111111111p-7,  -0x1.a01a01a01a01ap-13,
    0x1.71de3a556c734p-19, -0x1.ae64567f544e4p-26, 0x1.6124613a86d09p-33, -0x1.ae7f3e733b81fp-41,
    0x1.952c77030ad4ap-49, -0x1.2f49b46814157p-57, 0x1.71b8ef6dcf572p-66, -0x1.761b41316381ap-75,
    0x1.3f3ccdd165fa9p-84};
constexpr double kLn2 = 0x1.62e42fefa39efp-1;
constexpr double kHalfPi = 0x1.921fb54442d18p+0;
constexpr double kSqrtHalf = 0x1.6a09e667f3bcdp-1;

__device__ __forceinline__ uint64_t raw_bits(uint64_t key, uint64_t idx) {
  uint64_t z = key + (idx + 1ull) * kGamma;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ double ln_unit(uint64_t hi) {
  const double n = __dadd_rn((double)hi, 1.0);
  int e;
  double m = frexp(n, &e);  // exact: exponent extraction
  if (m < kSqrtHalf) {
    m = __dmul_rn(m, 2.0);
    e -= 1;
  }
  const double t = __ddiv_rn(__dadd_rn(m, -1.0), __dadd_rn(m, 1.0));
  const double t2 = __dmul_rn(t, t);
  double p = kLnCoef[11];
#pragma unroll
  for (int i = 10; i >= 0; --i) p = __dadd_rn(__dmul_rn(p, t2), kLnCoef[i]);
  const double ln_m = __dmul_rn(__dmul_rn(t, 2.0), p);
  return __dadd_rn(__dmul_rn(__dadd_rn((double)e, -32.0), kLn2), ln_m);
}

__device__ __forceinline__ double cos_turn(uint64_t lo) {
  const int quad = (int)(lo >> 30);
  const double frac = __dmul_rn((double)(lo & 0x3FFFFFFFull), 0x1p-30);
  const double th = __dmul_rn(frac, kHalfPi);
  const double t2 = __dmul_rn(th, th);
  double pc = kCosCoef[12];
#pragma unroll
  for (int i = 11; i >= 0; --i) pc = __dadd_rn(__dmul_rn(pc, t2), kCosCoef[i]);
  double ps = kSinCoef[12];
#pragma unroll
  for (int i = 11; i >= 0; --i) ps = __dadd_rn(__dmul_rn(ps, t2), kSinCoef[i]);
  ps = __dmul_rn(ps, th);
  return quad == 0 ? pc : quad == 1 ? -ps : quad == 2 ? -pc : ps;
}

__device__ __forceinline__ double normal(uint64_t key, uint64_t idx) {
  const uint64_t b = raw_bits(key, idx);
  const double r = __dsqrt_rn(__dmul_rn(ln_unit(b >> 32), -2.0));
  return __dmul_rn(r, cos_turn(b & 0xFFFFFFFFull));
}

__device__ __forceinline__ __nv_bfloat16 to_bf16(double x) { return __float2bfloat16_rn(__double2float_rn(x)); }

struct KVArgs {
  __nv_bfloat16* k;          // [B][Hkv][rows][d], row r holds position t_out0 + r
  __nv_bfloat16* v;
  int64_t rows;              // row stride (cache capacity)
  int64_t t_begin, t_end, t_out0;
  uint64_t key_k, key_v, key_off;
  int32_t layer, batch, n_kv_heads, d;
  int32_t n_sink, block_size;
  int64_t planted_end;       // planted positions lie in [n_sink, planted_end)
  const int32_t* planted;    // [B][Hkv][n_planted] or null
  int32_t n_planted;
  const double* qhat;        // [B][Hkv][d] or null
  double planted_amp, planted_std;
  double offset_std;         // 0: no per-block offset
  const double* head_scale;  // [Hkv]
  int64_t token_stride, block_stride;
};

__global__ void fill_kv_kernel(const KVArgs a) {
  const int64_t ntok = a.t_end - a.t_begin;
  const int64_t total = (int64_t)a.batch * a.n_kv_heads * ntok * a.d;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(e % a.d);
    const int64_t rest = e / a.d;
    const int64_t t = a.t_begin + rest % ntok;
    const int64_t bh = rest / ntok;
    const int h = (int)(bh % a.n_kv_heads);
    const int b = (int)(bh / a.n_kv_heads);
    const uint64_t unit = ((uint64_t)a.layer * a.batch + b) * a.n_kv_heads + h;
    const uint64_t idx = (unit * (uint64_t)a.token_stride + (uint64_t)t) * (uint64_t)a.d + (uint64_t)c;
    const double zk = normal(a.key_k, idx);
    const double zv = normal(a.key_v, idx);
    double base = zk;
    const int64_t rel = t - a.n_sink;
    const int64_t blk = rel >= 0 ? rel / a.block_size : -1;
    if (a.n_planted > 0 && t >= a.n_sink && t < a.planted_end) {
      const int32_t* pl = a.planted + ((int64_t)b * a.n_kv_heads + h) * a.n_planted;
      bool hit = false;
      for (int i = 0; i < a.n_planted; ++i) hit |= (pl[i] == blk);
      if (hit) {
        const double qh = a.qhat[((int64_t)b * a.n_kv_heads + h) * a.d + c];
        base = __dadd_rn(__dmul_rn(qh, a.planted_amp), __dmul_rn(zk, a.planted_std));
      }
    }
    if (a.offset_std > 0.0 && blk >= 0) {
      const uint64_t oidx = (unit * (uint64_t)a.block_stride + (uint64_t)blk) * (uint64_t)a.d + (uint64_t)c;
      base = __dadd_rn(base, __dmul_rn(normal(a.key_off, oidx), a.offset_std));
    }
    const double s = a.head_scale[h];
    const int64_t o = (bh * a.rows + (t - a.t_out0)) * a.d + c;
    a.k[o] = to_bf16(__dmul_rn(base, s));
    a.v[o] = to_bf16(__dmul_rn(zv, s));
  }
}

__global__ void normal_kernel(double* out, uint64_t key, uint64_t idx0, int64_t n) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x)
    out[e] = normal(key, idx0 + (uint64_t)e);
}

}  // namespace

extern "C" {

// Fill positions [t_begin, t_end) of every (b, kv head) of one layer.  All
// pointers are device pointers.  Returns a cudaError_t value (0 = success).
int syngen_fill_kv(void* k, void* v, int64_t rows, int64_t t_begin, int64_t t_end, int64_t t_out0,
                   uint64_t key_k, uint64_t key_v, uint64_t key_off, int32_t layer, int32_t batch,
                   int32_t n_kv_heads, int32_t d, int32_t n_sink, int32_t block_size, int64_t planted_end,
                   const int32_t* planted, int32_t n_planted, const double* qhat, double planted_amp,
                   double planted_std, double offset_std, const double* head_scale, int64_t token_stride,
                   int64_t block_stride, cudaStream_t stream) {
  if (t_end <= t_begin) return 0;
  KVArgs a{static_cast<__nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(v), rows, t_begin, t_end, t_out0, key_k,
           key_v, key_off, layer, batch, n_kv_heads, d, n_sink, block_size, planted_end, planted, n_planted, qhat,
           planted_amp, planted_std, offset_std, head_scale, token_stride, block_stride};
  const int64_t total = (int64_t)batch * n_kv_heads * (t_end - t_begin) * d;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  fill_kv_kernel<<<(unsigned)blocks, 256, 0, stream>>>(a);
  return (int)cudaGetLastError();
}

// n standard normals of stream `key` at indices [idx0, idx0 + n) (for tests).
int syngen_normal(double* out, uint64_t key, uint64_t idx0, int64_t n, cudaStream_t stream) {
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (blocks < 1) return 0;
  normal_kernel<<<(unsigned)blocks, 256, 0, stream>>>(out, key, idx0, n);
  return (int)cudaGetLastError();
}

}  // extern "C"
