// Activation quantization in the paper's own form (AlignQuant, App. B.3 with
// eq. 5 and the 8-bit endpoint scale of eq. 6): one scale per group of 64
// features and b_M rows, b_M = 1 for a single row and 16 otherwise; rows are
// zero-padded to M' = ceil(M / b_M) b_M (padding rows get zero codes).
// For a group A:  s = max(max(0, max A) / 127, max(0, -min A) / 128, 1e-12),
// codes = clip(rint(A / s), -128, 127) with the quotient rounded in fp64 (the
// paper's CUDA preparation computes in FP64), stored scale = fp32(s).
//
// One warp per (row group, 64-feature group).  The group's rows are read as
// 16-byte vectors (8 bf16): lane l takes vectors l, l + 32, ... of the
// b_M x 8 vectors, a warp reduction forms the group's maximum and minimum,
// and every lane writes its codes as 8-byte stores.
#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kGrpWarps = 8;
constexpr int kGrpFeatures = 64;

__global__ void __launch_bounds__(32 * kGrpWarps) quant_act_groups_kernel(const uint16_t* __restrict__ x, int M,
                                                                          int K, int ldx, int bM, int8_t* xq,
                                                                          float* sx) {
  const int lane = threadIdx.x & 31;
  const int G = K / kGrpFeatures;
  const long long unit = (long long)blockIdx.x * kGrpWarps + (threadIdx.x >> 5);
  const int Mp = (M + bM - 1) / bM * bM;
  pdl_launch_dependents();
  pdl_wait();  // x may come from the previous kernel; xq / sx may still be read by it
  if (unit >= (long long)(Mp / bM) * G) return;
  const int g = (int)(unit / G), c = (int)(unit % G);
  const int nvec = bM * (kGrpFeatures / 8);
  uint4 v[4];  // at most 16 rows x 8 vectors / 32 lanes
  float vmax = 0.f, vmin = 0.f;  // padding rows and the max(0, .) terms contribute zeros
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q = lane + 32 * i;
    const int m = g * bM + q / 8;
    v[i] = make_uint4(0u, 0u, 0u, 0u);
    if (q < nvec && m < M) {
      v[i] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)m * ldx + (size_t)c * kGrpFeatures) + (q % 8));
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float f = bf16_bits_to_float((e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu));
        vmax = fmaxf(vmax, f);
        vmin = fminf(vmin, f);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
  }
  // eq. 6 with b = 8 (bf16 values are exact in fp32 and fp64)
  const double s = fmax(fmax((double)vmax / 127.0, -(double)vmin / 128.0), 1e-12);
  if (lane == 0) sx[(size_t)g * G + c] = (float)s;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q = lane + 32 * i;
    if (q >= nvec) break;
    const int m = g * bM + q / 8;
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const double f = bf16_bits_to_float((e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu));
      const int code = (int)fmin(fmax(rint(f / s), -128.0), 127.0);  // eq. 5, fp64 quotient
      out[e >> 2] |= (uint32_t)(code & 0xFF) << (8 * (e & 3));
    }
    *reinterpret_cast<uint2*>(xq + (size_t)m * K + (size_t)c * kGrpFeatures + (q % 8) * 8) = make_uint2(out[0], out[1]);
  }
}

}  // namespace

int act_group_rows(int M) { return M == 1 ? 1 : 16; }

cudaError_t launch_quant_act_groups(const uint16_t* x, int M, int K, int ldx, int8_t* xq, float* sx,
                                    cudaStream_t st) {
  const int bM = act_group_rows(M);
  const long long units = (long long)((M + bM - 1) / bM) * (K / kGrpFeatures);
  const long long blocks = (units + kGrpWarps - 1) / kGrpWarps;
  return launch_pdl(quant_act_groups_kernel, dim3((unsigned)blocks), dim3(32 * kGrpWarps), 0, st, x, M, K, ldx, bM,
                    xq, sx);
}

}  // namespace aq
