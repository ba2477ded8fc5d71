// Float weights -> integer codes and fp16 scales (AlignQuant, App. B.2,
// eq. 5-7), applied to each output row of each bN x bK tile: the granularity
// of the packed format's scales (one fp16 scale per row per tile, App. E.1).
//
// For one row A of one tile (bK = 128 values) and its tile's bit width b:
//   s0 = max(max(0, max A) / q_max, max(0, -min A) / |q_min|, 1e-12)     (eq. 6)
//   search off: s* = s0
//   search on:  s_i = max((1/4 + i/128) s0, 1e-12), i = 0..128, and s* is the
//               s_i with the smallest sum over k of (A_k - s_i Q_k)^2, the
//               earliest i on equal sums                               (eq. 7)
//   codes = clip(rint(A / s*), q_min, q_max)                           (eq. 5)
//   stored scale = fp16(s*), rounded to nearest even from fp64.
// All arithmetic is fp64 with every operation rounded on its own (no fused
// multiply-add) and the error sum taken over k in increasing order, so the
// result is bit-identical to a plain sequential fp64 evaluation.
//
// Mapping: one warp per (row, tile).  The warp stages the row in shared memory
// as fp64; lane l evaluates the grid scales l, l+32, l+64, l+96 over the whole
// row (four independent sequential sums), and the 129th scale (i = 128) is
// evaluated element-parallel with one lane adding the 128 squared errors in
// order.  A warp arg-min with (error, index) ordering picks s*.
//
// The quotient A_k / s feeds only rint, so it is formed as A_k * RN(1/s) and
// replaced by the correctly rounded fp64 division whenever that product lies
// within 1e-12 of a half-integer (|A_k/s| <= 256 there; the product's relative
// error is below 2^-52, i.e. below 6e-14 in that range, so elsewhere both
// quotients round to the same integer; beyond 256 the code clips either way).
#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kQwWarps = 8;
constexpr int kQwThreads = 32 * kQwWarps;
constexpr int kPerLane = 4;          // grid points 0..127 spread over 32 lanes

struct QwArgs {
  const void* w;
  int N, K, ldw, bN, C;
  int wdtype;                        // AQ_F32 or AQ_BF16
  const uint8_t* map;                // [R][C], 1 = INT4
  int search;
  int8_t* codes;                     // [N][K]
  uint16_t* scales;                  // [N][C] fp16 bits
  int* err;                          // bit 0: non-finite weight, bit 1: bad label
};

// IEEE binary64 -> binary16, round to nearest even, from the bit patterns.
// Only finite inputs reach it; values above the fp16 range give infinity.
__device__ __forceinline__ uint16_t f64_to_f16_bits(double v) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(v);
  const uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
  const int e = (int)((u >> 52) & 0x7FF);
  if (e == 0) return sign;                                   // zero or fp64 subnormal: rounds to 0
  const int ex = e - 1023;                                   // v = 1.m * 2^ex
  if (ex > 15) return sign | 0x7C00u;
  const unsigned long long m = (u & 0xFFFFFFFFFFFFFull) | (1ull << 52);
  // fp16 keeps 10 fraction bits at exponent >= -14, fewer below (subnormals)
  const int shift = 42 + (ex < -14 ? (-14 - ex) : 0);
  if (shift > 53) return sign;                               // below half the smallest subnormal
  unsigned long long q = m >> shift;
  const unsigned long long rem = m & ((1ull << shift) - 1), half = 1ull << (shift - 1);
  if (rem > half || (rem == half && (q & 1))) ++q;
  // normal: exponent field (ex + 15) plus fraction; q carries the implicit bit,
  // so adding (ex + 14) << 10 lets a rounding carry move into the exponent
  const unsigned long long h = ex < -14 ? q : ((unsigned long long)(ex + 14) << 10) + q;
  return sign | (uint16_t)(h >= 0x7C00u ? 0x7C00u : h);
}

// rint of the correctly rounded fp64 quotient (the rare near-tie path).
static __device__ __noinline__ double rint_quotient(double a, double s) { return rint(__ddiv_rn(a, s)); }

// clip(rint(a / s), qmin, qmax) given r = RN(1 / s); see the file comment.
__device__ __forceinline__ double weight_code(double a, double s, double r, double qmin, double qmax) {
  const double t = __dmul_rn(a, r);
  double k = rint(t);
  if (fabs(t) <= 256.0 && !(__dsub_rn(0.5, fabs(__dsub_rn(t, k))) > 1e-12)) k = rint_quotient(a, s);
  return fmin(fmax(k, qmin), qmax);
}

__device__ __forceinline__ double sq_err(double a, double s, double q) {
  const double d = __dsub_rn(a, __dmul_rn(s, q));
  return __dmul_rn(d, d);
}

__global__ void __launch_bounds__(kQwThreads) quantize_weights_kernel(QwArgs p) {
  __shared__ double s_row[kQwWarps][kTileK];
  __shared__ double s_sq[kQwWarps][kTileK];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long unit = (long long)blockIdx.x * kQwWarps + warp;  // (row n, tile j) = (unit / C, unit % C)
  if (unit >= (long long)p.N * p.C) return;
  const int n = (int)(unit / p.C), j = (int)(unit % p.C);

  // stage the row's 128 values (4 per lane) as fp64
  double v[4];
  if (p.wdtype == AQ_F32) {
    const float4 f = *reinterpret_cast<const float4*>(static_cast<const float*>(p.w) + (size_t)n * p.ldw +
                                                      (size_t)j * kTileK + 4 * lane);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  } else {
    const uint2 b = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.w) + (size_t)n * p.ldw +
                                                    (size_t)j * kTileK + 4 * lane);
    v[0] = bf16_bits_to_float(b.x & 0xFFFFu); v[1] = bf16_bits_to_float(b.x >> 16);
    v[2] = bf16_bits_to_float(b.y & 0xFFFFu); v[3] = bf16_bits_to_float(b.y >> 16);
  }
  bool finite = true;
  double vmax = v[0], vmin = v[0];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    finite &= isfinite(v[e]);
    vmax = fmax(vmax, v[e]);
    vmin = fmin(vmin, v[e]);
    s_row[warp][4 * lane + e] = v[e];
  }
  const uint8_t label = p.map[(size_t)(n / p.bN) * p.C + j];
  if (lane == 0 && label > 1) atomicOr(p.err, 2);
  if (!__all_sync(0xFFFFFFFFu, finite) && lane == 0) atomicOr(p.err, 1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vmax = fmax(vmax, __shfl_xor_sync(0xFFFFFFFFu, vmax, o));
    vmin = fmin(vmin, __shfl_xor_sync(0xFFFFFFFFu, vmin, o));
  }
  const bool is4 = label == 1;
  const double qmax = is4 ? 7.0 : 127.0, qmin = is4 ? -8.0 : -128.0;
  // eq. 6
  const double s0 = fmax(fmax(__ddiv_rn(fmax(0.0, vmax), qmax), __ddiv_rn(fmax(0.0, -vmin), -qmin)), 1e-12);

  double best = s0;
  if (p.search) {
    __syncwarp();
    double s[kPerLane], r[kPerLane], err[kPerLane];
#pragma unroll
    for (int t = 0; t < kPerLane; ++t) {
      const int i = lane + 32 * t;
      s[t] = fmax(__dmul_rn(0.25 + i / 128.0, s0), 1e-12);
      r[t] = __drcp_rn(s[t]);
      err[t] = 0.0;
    }
#pragma unroll 4
    for (int k = 0; k < kTileK; ++k) {
      const double a = s_row[warp][k];
#pragma unroll
      for (int t = 0; t < kPerLane; ++t)
        err[t] = __dadd_rn(err[t], sq_err(a, s[t], weight_code(a, s[t], r[t], qmin, qmax)));
    }
    // i = 128: squared errors element-parallel, summed in order by lane 0
    const double s128 = fmax(__dmul_rn(1.25, s0), 1e-12), r128 = __drcp_rn(s128);
#pragma unroll
    for (int e = 0; e < 4; ++e) s_sq[warp][4 * lane + e] = sq_err(v[e], s128, weight_code(v[e], s128, r128, qmin, qmax));
    __syncwarp();
    double e_best = err[0];
    int i_best = lane;
#pragma unroll
    for (int t = 1; t < kPerLane; ++t)
      if (err[t] < e_best) { e_best = err[t]; i_best = lane + 32 * t; }
    if (lane == 0) {
      double e128 = 0.0;
      for (int k = 0; k < kTileK; ++k) e128 = __dadd_rn(e128, s_sq[warp][k]);
      if (e128 < e_best) { e_best = e128; i_best = 128; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double eo = __shfl_xor_sync(0xFFFFFFFFu, e_best, o);
      const int io = __shfl_xor_sync(0xFFFFFFFFu, i_best, o);
      if (eo < e_best || (eo == e_best && io < i_best)) { e_best = eo; i_best = io; }
    }
    best = fmax(__dmul_rn(0.25 + i_best / 128.0, s0), 1e-12);
  }

  // eq. 5 with s*, four codes per lane as one 32-bit store
  const double rb = __drcp_rn(best);
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int q = (int)weight_code(v[e], best, rb, qmin, qmax);
    word |= (uint32_t)(q & 0xFF) << (8 * e);
  }
  *reinterpret_cast<uint32_t*>(p.codes + (size_t)n * p.K + (size_t)j * kTileK + 4 * lane) = word;
  if (lane == 0) p.scales[(size_t)n * p.C + j] = f64_to_f16_bits(best);
}

}  // namespace

cudaError_t launch_quantize_weights(const void* w, int wdtype, int N, int K, int ldw, int bN, const uint8_t* map,
                                    int search, int8_t* codes, uint16_t* scales, int* err, cudaStream_t st) {
  const int C = K / kTileK;
  QwArgs p{w, N, K, ldw, bN, C, wdtype, map, search, codes, scales, err};
  const long long units = (long long)N * C;
  const long long blocks = (units + kQwWarps - 1) / kQwWarps;
  quantize_weights_kernel<<<(unsigned)blocks, kQwThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace aq

extern "C" int aq_quantize_weights(const void* w, int wdtype, int N, int K, int ldw, int bN, int bK,
                                   const uint8_t* map, int search, int8_t* codes, uint16_t* scales, void* stream) {
  using namespace aq;
  if (!w || !map || !codes || !scales) return AQ_ERR_ARG;
  if ((uintptr_t)scales & 1) return AQ_ERR_ARG;  // fp16 scales written as 2-byte words
  if (wdtype != AQ_F32 && wdtype != AQ_BF16) return AQ_ERR_ARG;
  if (search != 0 && search != 1) return AQ_ERR_ARG;
  if (!geometry_ok(N, K, bN, bK)) return AQ_ERR_SHAPE;
  if (ldw < K || (ldw % (wdtype == AQ_F32 ? 4 : 8)) || ((uintptr_t)w & 15) || ((uintptr_t)codes & 15))
    return AQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* err_dev = nullptr;
  if (cudaMalloc(&err_dev, sizeof(int)) != cudaSuccess) return AQ_ERR_CUDA;
  int err_h = 0;
  cudaError_t e = cudaMemsetAsync(err_dev, 0, sizeof(int), st);
  if (e == cudaSuccess) e = launch_quantize_weights(w, wdtype, N, K, ldw, bN, map, search, codes, scales, err_dev, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&err_h, err_dev, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaFree(err_dev);
  if (e != cudaSuccess) return AQ_ERR_CUDA;
  if (err_h & 2) return AQ_ERR_ARG;
  return (err_h & 1) ? AQ_ERR_RANGE : AQ_OK;
}
