// Per-token symmetric INT8 activation quantization (AlignQuant, App. B.3 with
// one scale per token; eq. 5 rounding to nearest with ties to even; eq. 6 scale
// floor 1e-12), computed in fp64 as App. B.3 prescribes for the CUDA
// preparation step.
//
// One CTA per token row.  Each thread owns 16-byte vectors (8 bf16) of the row:
// pass 1 reduces max|x| (kept in registers for rows up to 32768 features),
// pass 2 writes the codes as 8-byte stores.  HBM traffic: 2 bytes read and 1
// byte written per element, plus 4 bytes per row.
#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kThreads = 256;
constexpr int kCachedVecs = 16;  // 16 x 256 x 8 = 32768 features held in registers

__device__ __forceinline__ float abs_max8(const uint4& v, float m) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = fmaxf(m, bf16_bits_to_float(w[i] & 0x7FFFu));
    m = fmaxf(m, bf16_bits_to_float((w[i] >> 16) & 0x7FFFu));
  }
  return m;
}

__device__ __forceinline__ int code_of(uint32_t b16, double s) {
  const double q = rint(static_cast<double>(bf16_bits_to_float(b16)) / s);
  return static_cast<int>(fmin(fmax(q, -127.0), 127.0));
}

__device__ __forceinline__ uint2 quantize8(const uint4& v, double s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int c0 = code_of(w[2 * h] & 0xFFFFu, s);
    const int c1 = code_of(w[2 * h] >> 16, s);
    const int c2 = code_of(w[2 * h + 1] & 0xFFFFu, s);
    const int c3 = code_of(w[2 * h + 1] >> 16, s);
    out[h] = (uint32_t)(c0 & 0xFF) | ((uint32_t)(c1 & 0xFF) << 8) | ((uint32_t)(c2 & 0xFF) << 16) |
             ((uint32_t)(c3 & 0xFF) << 24);
  }
  return make_uint2(out[0], out[1]);
}

__global__ void __launch_bounds__(kThreads) quant_act_kernel(const uint16_t* __restrict__ x, int K, int ldx,
                                                             int8_t* __restrict__ xq, float* __restrict__ sx) {
  const int m = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)m * ldx);
  uint2* out = reinterpret_cast<uint2*>(xq + (size_t)m * K);
  const int nvec = K / 8;

  uint4 cache[kCachedVecs];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kCachedVecs; ++i) {
    const int v = threadIdx.x + i * kThreads;
    if (v < nvec) {
      cache[i] = __ldg(row + v);
      amax = abs_max8(cache[i], amax);
    }
  }
  for (int v = threadIdx.x + kCachedVecs * kThreads; v < nvec; v += kThreads) amax = abs_max8(__ldg(row + v), amax);

  __shared__ float red[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);

  double s = static_cast<double>(amax) / 127.0;
  if (s < 1e-12) s = 1e-12;
  if (threadIdx.x == 0) sx[m] = static_cast<float>(s);

#pragma unroll
  for (int i = 0; i < kCachedVecs; ++i) {
    const int v = threadIdx.x + i * kThreads;
    if (v < nvec) out[v] = quantize8(cache[i], s);
  }
  for (int v = threadIdx.x + kCachedVecs * kThreads; v < nvec; v += kThreads) out[v] = quantize8(__ldg(row + v), s);
}

}  // namespace

cudaError_t launch_quant_act(const uint16_t* x, int M, int K, int ldx, int8_t* xq, float* sx, cudaStream_t st) {
  quant_act_kernel<<<M, kThreads, 0, st>>>(x, K, ldx, xq, sx);
  return cudaGetLastError();
}

}  // namespace aq
