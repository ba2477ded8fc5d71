// Decode-phase linear layer on the CUDA cores for a few tokens (M <= 8).
//
// AlignQuant, Sec. 3.3 "Decode parallelism" and App. E.3: the kernel streams
// the packed tiles straight from HBM, forms INT8 operands on chip, forms
// per-tile INT32 dot products, rescales each tile product by its activation
// and weight scales before FP32 accumulation (eq. 19), and combines split-K
// partial sums in increasing split order.
//
// Work split: grid (S, row blocks).  CTA (s, b) owns tile row b (bN output
// rows) and tile columns [C*s/S, C*(s+1)/S).  A group of 8 adjacent lanes owns
// bN/32 output rows; lane c of the group always owns input columns
// [16c, 16c+16) of every tile, so a warp reads four whole tile rows per
// instruction: 4 x 128 contiguous bytes of an INT8 tile (16-byte loads) or
// 4 x 64 contiguous bytes of an INT4 tile (8-byte loads).
//
// INT4 unpacking stays in registers: (v & 0x0F0F0F0F) ^ 0x08080808 gives the
// even-k codes offset by +8 as unsigned bytes, (v >> 4) likewise the odd-k
// codes; a dp4a of those unsigned bytes with the matching (permuted) signed
// activation bytes, minus 8 x the activation sum of the chunk, is the exact
// signed product.  The 8 lane partials of a row are combined with shuffles.
#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;  // tiles whose loads are in flight together per thread

struct SimtArgs {
  const uint8_t* bitmap;
  const int32_t* tile_idx;
  const uint8_t* w4;
  const int8_t* w8;
  const uint16_t* scales;
  int N, K, bN, R, C;
  const int8_t* xq;
  const float* sx;
  int M;
  const float* bias;
  void* y;
  int ydtype, ldy;
  float* partial;    // [S][M][N] when S > 1
  int* counters;     // [R]
  int S;
  int32_t* P;        // debug: exact tile products [M][N][C], or null
};

__device__ __forceinline__ int dp4a_ss(int a, int b, int c) { return __dp4a(a, b, c); }
__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ void store_out(void* y, int ydtype, size_t idx, float v) {
  if (ydtype == AQ_F32)
    reinterpret_cast<float*>(y)[idx] = v;
  else
    reinterpret_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
}

template <int MT, int RPT>  // MT: tokens (compile-time bound), RPT: rows per lane group = bN / 32
__global__ void __launch_bounds__(kThreads) decode_simt_kernel(SimtArgs a) {
  const int s = blockIdx.x, rb = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = lane & 7;                      // 16-column chunk of the tile this lane owns
  const int row0 = 4 * warp + (lane >> 3);     // first tile row of this lane group
  const int j0 = (int)((long long)a.C * s / a.S), j1 = (int)((long long)a.C * (s + 1) / a.S);
  const int M = a.M;

  float acc[RPT][MT];
#pragma unroll
  for (int i = 0; i < RPT; ++i)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[i][m] = 0.f;

  for (int jb = j0; jb < j1; jb += kUnroll) {
    uint4 raw[kUnroll][RPT];
    uint32_t sw_bits[kUnroll][RPT];
    bool is4[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int j = jb + u;
      is4[u] = false;
      if (j < j1) {
        const int t = rb * a.C + j;
        is4[u] = (__ldg(a.bitmap + (t >> 3)) >> (t & 7)) & 1;
        const size_t p = (size_t)__ldg(a.tile_idx + t);
        if (!is4[u]) {
          const int8_t* base = a.w8 + p * a.bN * kTileK;
#pragma unroll
          for (int i = 0; i < RPT; ++i)
            raw[u][i] = __ldcs(reinterpret_cast<const uint4*>(base + (size_t)(row0 + 32 * i) * kTileK + 16 * c));
        } else {
          const uint8_t* base = a.w4 + p * a.bN * (kTileK / 2);
#pragma unroll
          for (int i = 0; i < RPT; ++i) {
            const uint2 v = __ldcs(reinterpret_cast<const uint2*>(base + (size_t)(row0 + 32 * i) * (kTileK / 2) + 8 * c));
            raw[u][i] = make_uint4(v.x, v.y, 0u, 0u);
          }
        }
#pragma unroll
        for (int i = 0; i < RPT; ++i) sw_bits[u][i] = __ldg(a.scales + (size_t)t * a.bN + row0 + 32 * i);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int j = jb + u;
      if (j >= j1) break;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m >= M) break;
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(a.xq + (size_t)m * a.K + (size_t)j * kTileK + 16 * c));
        int part[RPT];
        if (!is4[u]) {
#pragma unroll
          for (int i = 0; i < RPT; ++i) {
            int d = dp4a_ss((int)raw[u][i].x, (int)xv.x, 0);
            d = dp4a_ss((int)raw[u][i].y, (int)xv.y, d);
            d = dp4a_ss((int)raw[u][i].z, (int)xv.z, d);
            part[i] = dp4a_ss((int)raw[u][i].w, (int)xv.w, d);
          }
        } else {
          // even-k / odd-k activation bytes of the chunk, and 8 x their sum
          const int xe0 = (int)__byte_perm(xv.x, xv.y, 0x6420), xo0 = (int)__byte_perm(xv.x, xv.y, 0x7531);
          const int xe1 = (int)__byte_perm(xv.z, xv.w, 0x6420), xo1 = (int)__byte_perm(xv.z, xv.w, 0x7531);
          int xsum = dp4a_ss((int)xv.x, 0x01010101, 0);
          xsum = dp4a_ss((int)xv.y, 0x01010101, xsum);
          xsum = dp4a_ss((int)xv.z, 0x01010101, xsum);
          xsum = dp4a_ss((int)xv.w, 0x01010101, xsum);
#pragma unroll
          for (int i = 0; i < RPT; ++i) {
            const uint32_t v0 = raw[u][i].x, v1 = raw[u][i].y;
            int d = dp4a_us((v0 & 0x0F0F0F0Fu) ^ 0x08080808u, xe0, -8 * xsum);
            d = dp4a_us(((v0 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u, xo0, d);
            d = dp4a_us((v1 & 0x0F0F0F0Fu) ^ 0x08080808u, xe1, d);
            part[i] = dp4a_us(((v1 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u, xo1, d);
          }
        }
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
          int v = part[i];
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          if (a.P != nullptr && c == 0)
            a.P[((size_t)m * a.N + (size_t)rb * a.bN + row0 + 32 * i) * a.C + j] = v;
          const float sw = __half2float(__ushort_as_half((unsigned short)sw_bits[u][i]));
          acc[i][m] = fmaf((float)v, sw, acc[i][m]);
        }
      }
    }
  }
  if (a.P != nullptr) return;

  // ---- output: direct (S == 1) or fp32 partials + ordered reduction by the last CTA
  if (a.S == 1) {
    if (c == 0) {
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int n = rb * a.bN + row0 + 32 * i;
        const float b = a.bias ? __ldg(a.bias + n) : 0.f;
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < M) store_out(a.y, a.ydtype, (size_t)m * a.ldy + n, fmaf(__ldg(a.sx + m), acc[i][m], b));
      }
    }
    return;
  }
  if (c == 0) {
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const int n = rb * a.bN + row0 + 32 * i;
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < M) __stcg(a.partial + ((size_t)s * M + m) * a.N + n, acc[i][m]);
    }
  }
  __threadfence();
  __syncthreads();
  __shared__ int is_last;
  if (threadIdx.x == 0) is_last = (atomicAdd(a.counters + rb, 1) == a.S - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int e = threadIdx.x; e < M * a.bN; e += kThreads) {
    const int m = e / a.bN, n = rb * a.bN + e % a.bN;
    float sum = 0.f;
    for (int ss = 0; ss < a.S; ++ss) sum += __ldcg(a.partial + ((size_t)ss * M + m) * a.N + n);
    const float b = a.bias ? __ldg(a.bias + n) : 0.f;
    store_out(a.y, a.ydtype, (size_t)m * a.ldy + n, fmaf(__ldg(a.sx + m), sum, b));
  }
  if (threadIdx.x == 0) a.counters[rb] = 0;  // ready for the next call
}

template <int MT>
cudaError_t launch_mt(const SimtArgs& a, dim3 grid, cudaStream_t st) {
  if (a.bN == 128)
    decode_simt_kernel<MT, 4><<<grid, kThreads, 0, st>>>(a);
  else
    decode_simt_kernel<MT, 2><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_simt(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias,
                               void* y, int ydtype, int ldy, void* ws, int32_t* P, cudaStream_t st) {
  const DecodePlan plan = plan_decode(M, w);
  SimtArgs a;
  a.bitmap = w->bitmap; a.tile_idx = w->tile_idx; a.w4 = w->w4; a.w8 = w->w8; a.scales = w->scales;
  a.N = w->N; a.K = w->K; a.bN = w->bN; a.R = w->R; a.C = w->C;
  a.xq = xq; a.sx = sx; a.M = M; a.bias = bias; a.y = y; a.ydtype = ydtype; a.ldy = ldy;
  char* wsb = static_cast<char*>(ws);
  a.counters = reinterpret_cast<int*>(wsb + kWsHeader);
  const size_t cnt_bytes = ((size_t)w->R * sizeof(int) + 255) / 256 * 256;
  a.partial = reinterpret_cast<float*>(wsb + kWsHeader + cnt_bytes);
  a.S = P ? 1 : plan.S;
  a.P = P;
  const dim3 grid(a.S, w->R);
  if (M <= 1) return launch_mt<1>(a, grid, st);
  if (M <= 2) return launch_mt<2>(a, grid, st);
  if (M <= 4) return launch_mt<4>(a, grid, st);
  return launch_mt<8>(a, grid, st);
}

}  // namespace aq
