// Per-token symmetric INT8 activation quantization (AlignQuant, App. B.3 with
// one scale per token; eq. 5 rounding to nearest with ties to even; eq. 6 scale
// floor 1e-12), with the quotient x / s rounded in fp64 as App. B.3 prescribes
// for the CUDA preparation step (see quant_code for the exact fast path).
//
// One CTA per token row.  Each thread owns 16-byte vectors (8 bf16) of the row:
// pass 1 reduces max|x| (kept in registers for rows up to CV x 2048 features),
// pass 2 writes the codes as 8-byte stores.  HBM traffic: 2 bytes read and 1
// byte written per element, plus 4 bytes per row.  The register cache is sized
// to the row (CV = 1..16 vectors per thread): a fixed 16-vector cache held a
// 2560-feature row's CTA to two per SM, and the latency-bound per-row chain
// then ran at a fraction of HBM bandwidth.
#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxCachedVecs = 16;  // 16 x 256 x 8 = 32768 features held in registers

template <int kCachedVecs>
__global__ void __launch_bounds__(kThreads) quant_act_kernel(const uint16_t* __restrict__ x, int K, int ldx,
                                                             int8_t* __restrict__ xq, float* __restrict__ sx) {
  const int m = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)m * ldx);
  uint2* out = reinterpret_cast<uint2*>(xq + (size_t)m * K);
  const int nvec = K / 8;

  pdl_launch_dependents();
  pdl_wait();  // x may come from the previous kernel; xq / sx may still be read by it

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

  const double s = act_scale(amax);
  const float r32 = act_recip(s);
  if (threadIdx.x == 0) sx[m] = static_cast<float>(s);

#pragma unroll
  for (int i = 0; i < kCachedVecs; ++i) {
    const int v = threadIdx.x + i * kThreads;
    if (v < nvec) out[v] = quantize8(cache[i], s, r32);
  }
  for (int v = threadIdx.x + kCachedVecs * kThreads; v < nvec; v += kThreads)
    out[v] = quantize8(__ldg(row + v), s, r32);
}

}  // namespace

cudaError_t launch_quant_act(const uint16_t* x, int M, int K, int ldx, int8_t* xq, float* sx, cudaStream_t st) {
  const int per_thread = (K / 8 + kThreads - 1) / kThreads;  // 16-byte vectors per thread
  if (per_thread <= 1) return launch_pdl(quant_act_kernel<1>, dim3(M), dim3(kThreads), 0, st, x, K, ldx, xq, sx);
  if (per_thread <= 2) return launch_pdl(quant_act_kernel<2>, dim3(M), dim3(kThreads), 0, st, x, K, ldx, xq, sx);
  if (per_thread <= 4) return launch_pdl(quant_act_kernel<4>, dim3(M), dim3(kThreads), 0, st, x, K, ldx, xq, sx);
  if (per_thread <= 8) return launch_pdl(quant_act_kernel<8>, dim3(M), dim3(kThreads), 0, st, x, K, ldx, xq, sx);
  return launch_pdl(quant_act_kernel<kMaxCachedVecs>, dim3(M), dim3(kThreads), 0, st, x, K, ldx, xq, sx);
}

}  // namespace aq
