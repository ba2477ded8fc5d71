// AlignQuant's own numerics on the GPU (the paper-exact mode):
//  - App. B.1 eq. 4: X~ = X V with V = diag(V_j), one 64 x 64 block per input
//    tile column, and Y = Y~ U with U = diag(U_r), one bN x bN block per
//    output tile row;
//  - App. B.3: activations quantized per group of 64 features x b_M rows
//    (b_M = 1 for one row, 16 otherwise) with the 8-bit endpoint scale of
//    eq. 6 and codes clipped to [-128, 127] (eq. 5), rows zero-padded to M';
//  - App. E.2: one FP32 scale per whole weight tile, 64-wide tiles;
//  - App. E.3 eq. 19: Y~_{m,r} = sum_j s^X_{m,j} s^W_{r,j} P_{m,r,j} with exact
//    integer tile products P.
// It is the reference of the paper's construction on the GPU, computed on the
// CUDA cores for any token count; the per-token layer (aq_linear_decode /
// aq_linear_prefill) is the fast path.
#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kGroup = kPaperTileK;  // 64 features: one activation group = one input tile column

// ------------------------------------------------------------------ activations
// One CTA of 64 threads per (row group g, feature group c): thread k forms
// column k of the group's transformed rows in fp64, the CTA reduces the
// group's maximum and minimum, and every thread writes its codes.
template <int BM>
__global__ void __launch_bounds__(kGroup) paper_act_kernel(const uint16_t* __restrict__ x, int M, int K, int ldx,
                                                           const float* __restrict__ v, int8_t* __restrict__ xq,
                                                           float* __restrict__ sx) {
  __shared__ double xs[BM][kGroup];
  __shared__ __align__(16) float vs[kGroup][kGroup];
  __shared__ double red[2][2];
  const int k = threadIdx.x, lane = k & 31, wid = k >> 5;
  const int G = K / kGroup;
  const int g = blockIdx.x / G, c = blockIdx.x - g * G;
  pdl_launch_dependents();
  if (v != nullptr) {  // the transform block is a parameter: read it before the wait, 16 independent 16-byte loads
    const float4* vb = reinterpret_cast<const float4*>(v + (size_t)c * kGroup * kGroup);
#pragma unroll
    for (int i = 0; i < kGroup * kGroup / 4 / kGroup; ++i)
      reinterpret_cast<float4*>(&vs[0][0])[k + kGroup * i] = __ldg(vb + k + kGroup * i);
  }
  pdl_wait();  // x may come from the previous kernel; xq / sx may still be read by it
#pragma unroll
  for (int r = 0; r < BM; ++r) {
    const int m = g * BM + r;
    xs[r][k] = m < M ? (double)bf16_bits_to_float(x[(size_t)m * ldx + (size_t)c * kGroup + k]) : 0.0;
  }
  __syncthreads();
  double xt[BM];
  double vmax = 0.0, vmin = 0.0;  // padding rows and the max(0, .) terms contribute zeros
#pragma unroll
  for (int r = 0; r < BM; ++r) {
    double acc = xs[r][k];
    if (v != nullptr) {
      acc = 0.0;
#pragma unroll 8
      for (int i = 0; i < kGroup; ++i) acc = fma(xs[r][i], (double)vs[i][k], acc);
    }
    xt[r] = acc;
    vmax = fmax(vmax, acc);
    vmin = fmin(vmin, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    vmax = fmax(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    vmin = fmin(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
  }
  if (lane == 0) {
    red[wid][0] = vmax;
    red[wid][1] = vmin;
  }
  __syncthreads();
  vmax = fmax(red[0][0], red[1][0]);
  vmin = fmin(red[0][1], red[1][1]);
  const double s = fmax(fmax(vmax / 127.0, -vmin / 128.0), 1e-12);  // eq. 6, b = 8
  if (k == 0) sx[(size_t)g * G + c] = (float)s;
#pragma unroll
  for (int r = 0; r < BM; ++r) {
    const int code = (int)fmin(fmax(rint(xt[r] / s), -128.0), 127.0);  // eq. 5, fp64 quotient
    xq[(size_t)(g * BM + r) * K + (size_t)c * kGroup + k] = (int8_t)code;
  }
}

// ------------------------------------------------------------------ linear layer
struct PArgs {
  const uint8_t* bitmap;
  const int32_t* tile_idx;
  const uint8_t* w4;
  const int8_t* w8;
  const float* sw;    // [R][C] fp32 tile scales
  const int8_t* xq;   // [M'][K]
  const float* sx;    // [M'/b_M][C]
  const float* u;     // [R][BN][BN] or null
  const float* bias;  // [N] or null
  float* y;           // [M][ldy]
  int32_t* P;         // debug: [M][N][C]
  int N, K, C, M, bM, ldy;
};

__device__ __forceinline__ int dp4(uint32_t a, uint32_t b, int c) { return __dp4a((int)a, (int)b, c); }

// One CTA per (tile row r, block of MT tokens); 4 threads per output row, thread
// (n, q) covering input columns [16 q, 16 q + 16) of every 64-wide tile.  Per
// tile the four lanes' dp4a sums are combined by shuffles into the exact tile
// product, scaled by s^X s^W and accumulated in fp32 in ascending tile order;
// the block's y~ is then restored by U_r from shared memory.
template <int BN, int MT, bool DEBUG>
__global__ void __launch_bounds__(4 * BN) paper_linear_kernel(const __grid_constant__ PArgs a) {
  static_assert(MT == 1 || MT == 16, "one token, or one 16-row activation group per CTA");
  constexpr int kAcc = MT == 1 ? 1 : MT / 4;
  extern __shared__ __align__(16) float psm[];  // y~ [MT][BN], U_r [BN][BN], tile records [C]
  const int r = blockIdx.x, m0 = blockIdx.y * MT;
  const int n = threadIdx.x >> 2, q = threadIdx.x & 3;
  const int C = a.C, K = a.K;
  const int nrow = r * BN + n;
  float* yt = psm;            // [MT][BN]
  float* us = psm + MT * BN;  // [BN][BN]
  // the tile row's records: physical index with the INT4 label in bit 31, and the
  // tile scale (divided by 16 for INT4 tiles: their products come as 16 q)
  int2* rec = reinterpret_cast<int2*>(psm + MT * BN + (a.u != nullptr ? BN * BN : 0));
  pdl_launch_dependents();
  for (int j = threadIdx.x; j < C; j += 4 * BN) {
    const int t = r * C + j;
    const uint32_t is4 = (__ldg(a.bitmap + (t >> 3)) >> (t & 7)) & 1u;
    const float swt = __ldg(a.sw + t) * (is4 ? 0.0625f : 1.0f);
    rec[j] = make_int2(__ldg(a.tile_idx + t) | (int)(is4 << 31), __float_as_int(swt));
  }
  __syncthreads();
  pdl_wait();
  float acc[kAcc];
#pragma unroll
  for (int i = 0; i < kAcc; ++i) acc[i] = 0.f;
  const int8_t* xbase = a.xq + (size_t)m0 * K + 16 * q;
  const float* sxrow = a.sx + (size_t)(m0 / a.bM) * C;  // one activation scale row per CTA (MT <= b_M)
  constexpr int kUnroll = MT == 1 ? 4 : 1;  // (16 token partials per tile leave no registers for more)
#pragma unroll kUnroll
  for (int j = 0; j < C; ++j) {
    const int2 rj = rec[j];
    const uint32_t is4 = (uint32_t)rj.x >> 31;
    const size_t prow = (size_t)(rj.x & 0x7fffffff) * BN + n;
    int part[MT];
    if (!is4) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(a.w8 + prow * kGroup + 16 * q));
#pragma unroll
      for (int tt = 0; tt < MT; ++tt) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xbase + (size_t)tt * K + (size_t)j * kGroup));
        part[tt] = dp4(w.w, xv.w, dp4(w.z, xv.z, dp4(w.y, xv.y, dp4(w.x, xv.x, 0))));
      }
    } else {
      // nibbles as 16 q: the even-k nibbles moved to the high half of each byte, the odd-k ones kept there
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(a.w4 + prow * (kGroup / 2) + 8 * q));
      const uint32_t e0 = (w.x << 4) & 0xF0F0F0F0u, o0 = w.x & 0xF0F0F0F0u;
      const uint32_t e1 = (w.y << 4) & 0xF0F0F0F0u, o1 = w.y & 0xF0F0F0F0u;
#pragma unroll
      for (int tt = 0; tt < MT; ++tt) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xbase + (size_t)tt * K + (size_t)j * kGroup));
        int p = dp4(e0, __byte_perm(xv.x, xv.y, 0x6420), 0);
        p = dp4(o0, __byte_perm(xv.x, xv.y, 0x7531), p);
        p = dp4(e1, __byte_perm(xv.z, xv.w, 0x6420), p);
        part[tt] = dp4(o1, __byte_perm(xv.z, xv.w, 0x7531), p);
      }
    }
    // exact tile products: lane q ends with the sums over all four lanes of its tokens
    int prod[kAcc];
    if constexpr (MT == 1) {
      int v = part[0];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      prod[0] = v;
    } else {
      // token 4 i + b: first the pair (b, b ^ 2) splits on bit 1 of q, then (b, b ^ 1) on bit 0
      int half[kAcc][2];
#pragma unroll
      for (int i = 0; i < kAcc; ++i)
#pragma unroll
        for (int b0 = 0; b0 < 2; ++b0) {
          const int lo = part[4 * i + b0], hi = part[4 * i + b0 + 2];
          const bool up = (q & 2) != 0;
          half[i][b0] = (up ? hi : lo) + __shfl_xor_sync(0xffffffffu, up ? lo : hi, 2);
        }
#pragma unroll
      for (int i = 0; i < kAcc; ++i) {
        const bool up = (q & 1) != 0;
        prod[i] = (up ? half[i][1] : half[i][0]) + __shfl_xor_sync(0xffffffffu, up ? half[i][0] : half[i][1], 1);
      }
    }
    if constexpr (DEBUG) {
#pragma unroll
      for (int i = 0; i < kAcc; ++i) {
        const int m = MT == 1 ? m0 : m0 + 4 * i + q;
        if ((MT > 1 || q == 0) && m < a.M)
          a.P[((size_t)m * a.N + nrow) * C + j] = is4 ? (prod[i] >> 4) : prod[i];  // 16 q products / 16, exact
      }
    } else {
      const float f = __int_as_float(rj.y) * __ldg(sxrow + j);
#pragma unroll
      for (int i = 0; i < kAcc; ++i) acc[i] = fmaf((float)prod[i], f, acc[i]);  // |prod| < 2^24: exact
    }
  }
  if constexpr (DEBUG) return;

  if constexpr (MT == 1) {
    if (q == 0) yt[n] = acc[0];
  } else {
#pragma unroll
    for (int i = 0; i < kAcc; ++i) yt[(4 * i + q) * BN + n] = acc[i];
  }
  if (a.u != nullptr)
    for (int i = threadIdx.x; i < BN * BN; i += 4 * BN) us[i] = __ldg(a.u + (size_t)r * BN * BN + i);
  __syncthreads();
  for (int o = threadIdx.x; o < MT * BN; o += 4 * BN) {
    const int tt = o / BN, c = o - tt * BN, m = m0 + tt;
    if (m >= a.M) continue;
    float val = yt[tt * BN + c];
    if (a.u != nullptr) {
      val = 0.f;
#pragma unroll 8
      for (int i = 0; i < BN; ++i) val = fmaf(yt[tt * BN + i], us[i * BN + c], val);
    }
    if (a.bias != nullptr) val += __ldg(a.bias + r * BN + c);
    a.y[(size_t)m * a.ldy + r * BN + c] = val;
  }
}

constexpr int kPaperSmemAttr = 200 * 1024;  // >= every launch's request (the tile records take 8 bytes per tile)

template <int BN, int MT, bool DEBUG>
cudaError_t launch_paper_t(const PArgs& a, dim3 grid, cudaStream_t st) {
  const size_t smem = (size_t)(MT * BN + (a.u ? BN * BN : 0)) * sizeof(float) + (size_t)a.C * sizeof(int2);
  if (smem > (size_t)kPaperSmemAttr) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr<paper_linear_kernel<BN, MT, DEBUG>>(kPaperSmemAttr);
  if (e != cudaSuccess) return e;
  return launch_pdl(paper_linear_kernel<BN, MT, DEBUG>, grid, dim3(4 * BN), smem, st, a);
}

template <bool DEBUG>
cudaError_t launch_paper(const PArgs& a, int bN, int R, int Mp, cudaStream_t st) {
  const int MT = a.M == 1 ? 1 : 16;
  const dim3 grid(R, Mp / MT);
  if (bN == 64) return MT == 1 ? launch_paper_t<64, 1, DEBUG>(a, grid, st) : launch_paper_t<64, 16, DEBUG>(a, grid, st);
  return MT == 1 ? launch_paper_t<128, 1, DEBUG>(a, grid, st) : launch_paper_t<128, 16, DEBUG>(a, grid, st);
}

int validate_paper_packed(const aq_packed* w) {
  if (!w) return AQ_ERR_ARG;
  if (w->scale_kind != AQ_SCALES_TILE_FP32) return AQ_ERR_ARG;
  if (!paper_geometry_ok(w->N, w->K, w->bN, w->bK)) return AQ_ERR_SHAPE;
  if (w->R != w->N / w->bN || w->C != w->K / w->bK) return AQ_ERR_SHAPE;
  if (w->T4 < 0 || w->T8 < 0 || (long long)w->T4 + w->T8 != (long long)w->R * w->C) return AQ_ERR_SHAPE;
  if (!w->bitmap || !w->tile_idx || !w->scales) return AQ_ERR_ARG;
  if ((w->T4 > 0 && !w->w4) || (w->T8 > 0 && !w->w8)) return AQ_ERR_ARG;
  if (((uintptr_t)w->w4 & 15) || ((uintptr_t)w->w8 & 15) || ((uintptr_t)w->scales & 3)) return AQ_ERR_ARG;
  if ((uintptr_t)w->tile_idx & 3) return AQ_ERR_ARG;
  return AQ_OK;
}

int paper_call(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* u, const float* bias,
               float* y, int ldy, int32_t* P, void* stream) {
  int rc = validate_paper_packed(w);
  if (rc != AQ_OK) return rc;
  if (!xq || ((uintptr_t)xq & 15) || M < 1 || M > (1 << 20)) return AQ_ERR_ARG;
  if (P == nullptr && (!sx || !y || ldy < w->N)) return AQ_ERR_ARG;
  // fp32 / int32 operands are read and written as 4-byte words
  if (((uintptr_t)sx | (uintptr_t)u | (uintptr_t)bias | (uintptr_t)y | (uintptr_t)P) & 3) return AQ_ERR_ARG;
  const int bM = act_group_rows(M), Mp = (M + bM - 1) / bM * bM;
  if (Mp / bM > 65535) return AQ_ERR_ARG;  // one grid row per activation row group
  PArgs a{w->bitmap, w->tile_idx, w->w4, w->w8, reinterpret_cast<const float*>(w->scales), xq, sx, u, bias, y, P,
          w->N, w->K, w->C, M, bM, ldy};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = P ? launch_paper<true>(a, w->bN, w->R, Mp, st) : launch_paper<false>(a, w->bN, w->R, Mp, st);
  return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
}

}  // namespace
}  // namespace aq

using namespace aq;

extern "C" int aq_paper_quant_act(const uint16_t* x, int M, int K, int ldx, const float* v, int8_t* xq, float* sx,
                                  void* stream) {
  if (!x || !xq || !sx || M < 1 || M > (1 << 20) || K < kGroup || K % kGroup || K > (1 << 20) || ldx < K)
    return AQ_ERR_ARG;
  // V is staged with 16-byte loads; x is read as 2-byte words, sx written as 4-byte words
  if (((uintptr_t)v & 15) || ((uintptr_t)x & 1) || ((uintptr_t)sx & 3)) return AQ_ERR_ARG;
  const int bM = act_group_rows(M), Mp = (M + bM - 1) / bM * bM;
  const long long blocks = (long long)(Mp / bM) * (K / kGroup);
  if (blocks > 0x7fffffffll) return AQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = bM == 1 ? launch_pdl(paper_act_kernel<1>, dim3((unsigned)blocks), dim3(kGroup), 0, st, x, M,
                                             K, ldx, v, xq, sx)
                                : launch_pdl(paper_act_kernel<16>, dim3((unsigned)blocks), dim3(kGroup), 0, st, x, M,
                                             K, ldx, v, xq, sx);
  return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
}

extern "C" int aq_paper_linear(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* u,
                               const float* bias, float* y, int ldy, void* stream) {
  if (!y) return AQ_ERR_ARG;
  return paper_call(w, xq, sx, M, u, bias, y, ldy, nullptr, stream);
}

extern "C" int aq_debug_paper_partials(const aq_packed* w, const int8_t* xq, int M, int32_t* P, void* stream) {
  if (!P) return AQ_ERR_ARG;
  return paper_call(w, xq, nullptr, M, nullptr, nullptr, nullptr, 0, P, stream);
}
