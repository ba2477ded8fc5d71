// Decode-phase linear layers on the CUDA cores for a few tokens.
//
// AlignQuant, Sec. 3.3 "Decode parallelism" and App. E.3: the kernel streams
// the packed tiles from HBM, forms INT8 operands on chip, takes per-tile INT32
// dot products and rescales each by its activation and weight scales before
// FP32 accumulation (eq. 19).  Sec. 3.3 "Shared activation preparation" and
// App. E.4: projections that read the same input (q/k/v, gate/up) run as one
// launch over their concatenated output rows, and the activation quantization
// can be fused into that launch so each CTA prepares the input from bf16.
//
// Work split: one CTA owns kRows = 16 consecutive output rows of one
// projection and ALL of its input tiles, so there is no cross-CTA reduction.
// The 16-row slice of a tile is contiguous in the packed buffers (2 KB for
// INT8, 1 KB for INT4, plus 32 B of row scales), so thread 0 streams slices
// into a shared-memory ring with one asynchronous bulk copy each
// (cp.async.bulk, completion counted on an mbarrier) and keeps up to
// kMaxStages slices in flight per CTA without spending registers.  The copies
// of the first ring fill are issued before griddepcontrol.wait: weights never
// depend on an earlier kernel, so a launch streams while its predecessor ends.
//
// Thread t owns row t / 8 and, in every tile, the 16 input columns
// [16c, 16c + 16) with c = t % 8; a warp reads 4 whole slice rows per
// shared-memory access (512 contiguous bytes of an INT8 slice, 256 of INT4).
// INT4 nibbles are unpacked in registers: (v & 0x0F0F0F0F) ^ 0x08080808 gives
// the even-k codes plus 8 as unsigned bytes, the shifted word the odd-k codes;
// byte permutes restore k order, an unsigned x signed dp4a against the
// activation bytes gives sum((q + 8) x), and 8 x sum(x) is subtracted.  The 8
// lanes of a row keep separate FP32 sums of (exact lane partial) x (tile
// scale) and are combined with shuffles once, after the last tile.
//
// Every mbarrier wait is bounded; a wait that gives up records AQ_ERR_TIMEOUT
// in the workspace, the CTA stops consuming, and thread 0 waits (bounded) for
// the copies it issued before the CTA exits.
#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kRows = 16;
constexpr int kThreads = kRows * 8;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxC = 256;                       // input tiles per row (K <= 32768)
constexpr int kMaxStages = 24;                   // slices in flight per CTA
constexpr int kSliceW = kRows * kTileK;          // bytes of the largest (INT8) slice
constexpr int kStageBytes = kSliceW + 2 * kRows; // slice + fp16 row scales

struct RowsArgs {
  DecodeProj p[kMaxGroup];
  int G, K, C, M, ydtype, NS;
  const uint16_t* x;   // bf16 activations [M][ldx] (fused quantization), or null
  int ldx;
  const int8_t* xq;    // pre-quantized activations [M][K], or null
  const float* sx;
  int32_t* P;          // debug: exact tile products [M][N][C] of projection 0
  void* ws;            // status word
};

__device__ __forceinline__ int dp4a_ss(int a, int b, int c) { return __dp4a(a, b, c); }
__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Exact int -> float for |v| < 2^22 with an integer add and a float subtract.
__device__ __forceinline__ float small_int_to_float(int v) {
  return __int_as_float(v + 0x4B400000) - 12582912.0f;
}

// Nibble word (8 codes, low nibble = even k) -> two words of (code + 8) bytes in k order.
__device__ __forceinline__ void nibbles_plus8(uint32_t v, uint32_t& a, uint32_t& b) {
  const uint32_t lo = (v & 0x0F0F0F0Fu) ^ 0x08080808u, hi = ((v >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
  a = __byte_perm(lo, hi, 0x5140);
  b = __byte_perm(lo, hi, 0x7362);
}

__device__ __forceinline__ void store_out(void* y, int ydtype, size_t idx, float v) {
  if (ydtype == AQ_F32)
    reinterpret_cast<float*>(y)[idx] = v;
  else
    reinterpret_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
}

template <int MT, bool FUSED>
__global__ void __launch_bounds__(kThreads) decode_rows_kernel(const __grid_constant__ RowsArgs a) {
  // dynamic: ring [NS][kStageBytes], then (FUSED) codes [M][K] int8 and sx [M] fp32
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int32_t desc[kMaxC];  // (physical index << 1) | INT4 label, per tile column
  __shared__ float red[kWarps][MT];
  __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
  __shared__ int flags[2];         // [0] abort, [1] stays 0 (drain waits)

  int b = blockIdx.x, g = 0;
#pragma unroll
  for (int i = 0; i < kMaxGroup - 1; ++i)
    if (g + 1 < a.G && b >= a.p[g].blocks) {
      b -= a.p[g].blocks;
      ++g;
    }
  const DecodeProj& p = a.p[g];
  const int t = threadIdx.x, c = t & 7, lrow = t >> 3, lane = t & 31;
  const int bN = p.bN, C = a.C, K = a.K, M = a.M, NS = a.NS;
  const int row0 = b * kRows;                   // first output row of the CTA (one tile row holds it)
  const int r = row0 / bN, nl0 = row0 - r * bN;
  const int row = row0 + lrow;
  const int tile0 = r * C;
  volatile int* abort_flag = &flags[0];
  volatile int* never_flag = &flags[1];

  if (t == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWarps);
    }
    flags[0] = flags[1] = 0;
    fence_mbar_init();
  }
  for (int j = t; j < C; j += kThreads) {  // tile metadata (independent of earlier kernels)
    const int tt = tile0 + j;
    const int is4 = (__ldg(p.bitmap + (tt >> 3)) >> (tt & 7)) & 1;
    desc[j] = (__ldg(p.tile_idx + tt) << 1) | is4;
  }
  __syncthreads();
  pdl_launch_dependents();

  auto issue = [&](int j) {  // thread 0 only: slice + row scales of tile column j into stage j % NS
    const int s = j % NS;
    const int d = desc[j];
    const size_t pr = (size_t)(d >> 1) * bN + nl0;  // first physical row of the slice
    const uint32_t bytes = (d & 1) ? kRows * (kTileK / 2) : kRows * kTileK;
    const void* src = (d & 1) ? (const void*)(p.w4 + pr * (kTileK / 2)) : (const void*)(p.w8 + pr * kTileK);
    uint8_t* st = smem + (size_t)s * kStageBytes;
    mbar_arrive_expect_tx(&full[s], bytes + 2 * kRows);
    bulk_load(st, src, bytes, &full[s]);
    bulk_load(st + kSliceW, p.scales + (size_t)(tile0 + j) * bN + nl0, 2 * kRows, &full[s]);
  };
  int issued = 0;
  if (t == 0)
    for (; issued < NS && issued < C; ++issued) issue(issued);

  pdl_wait();  // activations (and every global write below) depend on earlier kernels

  const int8_t* xs;
  const float* sxp;
  uint8_t* xbuf = smem + (size_t)NS * kStageBytes;
  if constexpr (FUSED) {
    // per-token absmax over K, then codes into shared memory (same arithmetic as aq_quant_act)
    const int nvec = K / 8;
    float amax[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) amax[m] = 0.f;
    for (int v = t; v < nvec; v += kThreads) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
        if (m < M) amax[m] = abs_max8(__ldg(reinterpret_cast<const uint4*>(a.x + (size_t)m * a.ldx) + v), amax[m]);
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax[m] = fmaxf(amax[m], __shfl_xor_sync(0xffffffffu, amax[m], o));
      if (lane == 0) red[t >> 5][m] = amax[m];
    }
    __syncthreads();
    float* sx_s = reinterpret_cast<float*>(xbuf + (size_t)M * K);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
      float am = red[0][m];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) am = fmaxf(am, red[w][m]);
      const double s = act_scale(am);
      const float r32 = (float)(1.0 / s);
      for (int v = t; v < nvec; v += kThreads) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(a.x + (size_t)m * a.ldx) + v);
        *reinterpret_cast<uint2*>(xbuf + (size_t)m * K + 8 * v) = quantize8(xv, s, r32);
      }
      if (t == 0) sx_s[m] = (float)s;
    }
    __syncthreads();
    xs = reinterpret_cast<const int8_t*>(xbuf);
    sxp = sx_s;
  } else {
    xs = a.xq;
    sxp = a.sx;
  }

  float acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.f;

  bool ok = true;
  for (int j = 0; j < C; ++j) {
    const int s = j % NS;
    const uint32_t ph = (uint32_t)(j / NS) & 1u;
    if (!mbar_wait(&full[s], ph, abort_flag)) {
      *abort_flag = 1;
      record_error(a.ws, AQ_ERR_TIMEOUT, 20);
      ok = false;
      break;
    }
    const uint8_t* st = smem + (size_t)s * kStageBytes;
    const bool is4 = desc[j] & 1;
    const float sw = __half2float(*reinterpret_cast<const __half*>(st + kSliceW + 2 * lrow));
    uint32_t w0, w1, w2, w3;
    if (is4) {
      const uint2 v = *reinterpret_cast<const uint2*>(st + lrow * (kTileK / 2) + 8 * c);
      nibbles_plus8(v.x, w0, w1);
      nibbles_plus8(v.y, w2, w3);
    } else {
      const uint4 v = *reinterpret_cast<const uint4*>(st + lrow * kTileK + 16 * c);
      w0 = v.x; w1 = v.y; w2 = v.z; w3 = v.w;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with stage s
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
      const uint4 xv = *reinterpret_cast<const uint4*>(xs + (size_t)m * K + (size_t)j * kTileK + 16 * c);
      int part;
      if (is4) {
        int xsum = dp4a_ss((int)xv.x, 0x01010101, 0);
        xsum = dp4a_ss((int)xv.y, 0x01010101, xsum);
        xsum = dp4a_ss((int)xv.z, 0x01010101, xsum);
        xsum = dp4a_ss((int)xv.w, 0x01010101, xsum);
        part = dp4a_us(w0, (int)xv.x, -8 * xsum);
        part = dp4a_us(w1, (int)xv.y, part);
        part = dp4a_us(w2, (int)xv.z, part);
        part = dp4a_us(w3, (int)xv.w, part);
      } else {
        part = dp4a_ss((int)w0, (int)xv.x, 0);
        part = dp4a_ss((int)w1, (int)xv.y, part);
        part = dp4a_ss((int)w2, (int)xv.z, part);
        part = dp4a_ss((int)w3, (int)xv.w, part);
      }
      if (a.P != nullptr) {
        int v = part;
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        if (c == 0) a.P[((size_t)m * p.N + row) * C + j] = v;
      }
      acc[m] = fmaf(small_int_to_float(part), sw, acc[m]);
    }
    if (t == 0 && issued < C) {  // refill stage s once every warp has read it
      if (!mbar_wait(&empty[s], ph, abort_flag)) {
        *abort_flag = 1;
        record_error(a.ws, AQ_ERR_TIMEOUT, 21);
        ok = false;
        break;
      }
      issue(issued++);
    }
  }
  if (t == 0 && !ok) {
    // let every issued copy land before the CTA's shared memory is released
    for (int jj = (issued > NS ? issued - NS : 0); jj < issued; ++jj)
      mbar_wait(&full[jj % NS], (uint32_t)(jj / NS) & 1u, never_flag);
  }
  if (!ok || a.P != nullptr) return;

  const float bias = p.bias ? __ldg(p.bias + row) : 0.f;
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if (m >= M) break;
    float v = acc[m];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    if (c == 0) store_out(p.y, a.ydtype, (size_t)m * p.ldy + row, fmaf(sxp[m], v, bias));
  }
}

template <int MT, bool FUSED>
cudaError_t launch_rows_t(const RowsArgs& a, int blocks, size_t smem, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(decode_rows_kernel<MT, FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(kMaxStages * kStageBytes + kFusedMaxBytes));
    if (e != cudaSuccess) return e;
    attr = true;
  }
  return launch_pdl(decode_rows_kernel<MT, FUSED>, dim3(blocks), dim3(kThreads), smem, st, a);
}

template <bool FUSED>
cudaError_t launch_rows_m(const RowsArgs& a, int blocks, size_t smem, cudaStream_t st) {
  if (a.M <= 1) return launch_rows_t<1, FUSED>(a, blocks, smem, st);
  if (a.M <= 2) return launch_rows_t<2, FUSED>(a, blocks, smem, st);
  if (a.M <= 4) return launch_rows_t<4, FUSED>(a, blocks, smem, st);
  return launch_rows_t<8, FUSED>(a, blocks, smem, st);
}

}  // namespace

bool rows_supported(int M, int K) { return M >= 1 && M <= kRowsMaxM && K / kTileK <= kMaxC; }

bool rows_fusable(int M, int K) { return (size_t)M * K + 16 * (size_t)M <= kFusedMaxBytes; }

cudaError_t launch_decode_rows(const DecodeProj* projs, int G, int K, const uint16_t* x, int ldx, const int8_t* xq,
                               const float* sx, int M, int ydtype, int32_t* P, void* ws, cudaStream_t st) {
  RowsArgs a;
  memset(&a, 0, sizeof(a));
  int blocks = 0;
  for (int g = 0; g < G; ++g) {
    a.p[g] = projs[g];
    a.p[g].blocks = projs[g].N / kRows;
    blocks += a.p[g].blocks;
  }
  a.G = G; a.K = K; a.C = K / kTileK; a.M = M; a.ydtype = ydtype;
  a.NS = a.C < kMaxStages ? a.C : kMaxStages;
  a.x = x; a.ldx = ldx; a.xq = xq; a.sx = sx; a.P = P; a.ws = ws;
  const size_t ring = (size_t)a.NS * kStageBytes;
  if (x != nullptr) return launch_rows_m<true>(a, blocks, ring + (size_t)M * K + 16 * (size_t)M, st);
  return launch_rows_m<false>(a, blocks, ring, st);
}

}  // namespace aq
