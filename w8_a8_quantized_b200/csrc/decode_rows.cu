// Decode-phase linear layers on the CUDA cores for a few tokens.
//
// AlignQuant, Sec. 3.3 "Decode parallelism" and App. E.3: the kernel loads the
// packed tiles from HBM, forms INT8 operands on chip, takes per-tile INT32 dot
// products and rescales each by its activation and weight scales before FP32
// accumulation (eq. 19).  Sec. 3.3 "Shared activation preparation" and
// App. E.4: projections that read the same input (q/k/v, gate/up) run as one
// launch over their concatenated output rows, and the activation quantization
// can be fused into that launch so each CTA prepares the input from bf16.
//
// Work split: one CTA owns kRows = 32 consecutive output rows of one
// projection and ALL of its input tiles, so there is no cross-CTA reduction.
// The CTA has KG groups of 64 threads (KG = 1..8, chosen so the launch keeps
// about 16 warps per SM busy; at most 256 threads for short rows so that the
// CTAs of the next launch fit beside it and programmatic dependent launch can
// overlap them); group kg takes tile columns kg, kg + KG, ...
// In a group, thread t owns row t / 2 and half h = t % 2 of every tile row:
// input columns [64h, 64h + 64), i.e. 64 contiguous bytes of an INT8 tile row
// (four 16-byte loads) or 32 bytes of an INT4 tile row (two).  A warp reads 16
// whole tile rows per load step: 2 KB (INT8) or 1 KB (INT4) contiguous.  Big
// per-thread pieces keep the instruction count per weight byte low: at HBM
// rate the SM issue rate, not memory, is what a finer split runs out of.
//
// Memory pipeline: each thread keeps its next kRing tiles in flight in a ring
// of registers (the loop is unrolled kRing times, a load's destination is read
// kRing tiles later, the register scoreboard is the only wait).  Tile
// addresses, INT4 labels and the CTA's fp16 row scales are staged in shared
// memory once, and the first ring of loads is issued before
// griddepcontrol.wait: weights never depend on an earlier kernel, so a launch
// streams while its predecessor finishes.
//
// INT4 nibbles are unpacked in registers without sign extension: a nibble in
// the high half of a byte with a zero low half IS the two's-complement byte
// 16 q, so (v << 4) & 0xF0F0F0F0 holds 16 q of the even k of a word and
// v & 0xF0F0F0F0 of the odd k.  A dp4a against the activation bytes of the
// even / odd k gives 16 x the exact product, and the tile scale is divided by
// 16 (exact).  The fused path stores the activation codes twice in shared
// memory: in k order (for INT8 tiles) and with even and odd k split per
// 8-column group (for INT4 tiles); the pre-quantized path permutes on the fly.
// The 2 lanes of a row keep FP32 sums of (exact lane partial) x (tile scale)
// and are combined once, after the last tile, then the KG groups in order.
#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kRows = kRowsPerCta;
constexpr int kGroupThreads = kRows * 2;  // threads of one tile group
constexpr int kMaxKG = 8;
constexpr int kMaxThreads = kGroupThreads * kMaxKG;
constexpr int kMaxC = 256;  // input tiles per row (K <= 32768)
constexpr int kRing = 4;    // tiles in flight per thread

struct RowsArgs {
  DecodeProj p[kMaxGroup];
  int G, K, C, M, ydtype, KG;
  const uint16_t* x;   // bf16 activations [M][ldx] (fused quantization), or null
  int ldx;
  const int8_t* xq;    // pre-quantized activations [M][K], or null
  const float* sx;
  int32_t* P;          // debug: exact tile products [M][N][C] of projection 0
};

__device__ __forceinline__ int dp4a(uint32_t a, uint32_t b, int c) { return __dp4a((int)a, (int)b, c); }

// Exact int -> float for |v| < 2^22 with an integer add and a float subtract.
__device__ __forceinline__ float small_int_to_float(int v) {
  return __int_as_float(v + 0x4B400000) - 12582912.0f;
}

// even-k / odd-k activation bytes of an 8-column group given in k order
__device__ __forceinline__ uint32_t even_bytes(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x6420); }
__device__ __forceinline__ uint32_t odd_bytes(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x7531); }

__device__ __forceinline__ void store_out(void* y, int ydtype, size_t idx, float v) {
  if (ydtype == AQ_F32)
    reinterpret_cast<float*>(y)[idx] = v;
  else
    reinterpret_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
}

struct Piece {  // one thread's share of one tile row: 64 INT8 bytes or 32 INT4 bytes
  uint4 v[4];
};

template <int MT, bool FUSED, bool DEBUG>
__global__ void __launch_bounds__(kMaxThreads) decode_rows_kernel(const __grid_constant__ RowsArgs a) {
  // dynamic (FUSED only): codes in k order [M][K], codes even/odd split [M][K], sx [M] fp32
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ const uint8_t* tile_ptr[kMaxC];                // slice start (row nl0) of every tile column
  __shared__ __align__(16) uint16_t tile_sw[kMaxC][kRows];  // fp16 row scales of every tile column
  __shared__ uint32_t tile_is4[kMaxC / 32];                  // INT4 labels, one bit per tile column
  __shared__ float red[kMaxKG][kRows][MT];
  __shared__ float redq[kMaxThreads / 32][MT];

  int b = blockIdx.x, g = 0;
#pragma unroll
  for (int i = 0; i < kMaxGroup - 1; ++i)
    if (g + 1 < a.G && b >= a.p[g].blocks) {
      b -= a.p[g].blocks;
      ++g;
    }
  const DecodeProj& p = a.p[g];
  const int nthr = blockDim.x, KG = a.KG;
  const int t = threadIdx.x, kg = t / kGroupThreads, tg = t % kGroupThreads;
  const int h = tg & 1, lrow = tg >> 1, lane = t & 31;
  const int bN = p.bN, C = a.C, K = a.K, M = a.M;
  const int nmine = (C - kg + KG - 1) / KG;  // tile columns of this thread's group
  const int row0 = b * kRows;                // first output row of the CTA (one tile row holds it)
  const int r = row0 / bN, nl0 = row0 - r * bN;
  const int row = row0 + lrow;
  const int tile0 = r * C;

  // ---- per-CTA tile table and scales (independent of earlier kernels): the loads
  // of a pass are all issued before any is used (one round trip for C <= 2 nthr)
  for (int base = 0; base < C; base += 2 * nthr) {
    int idx[2];
    uint32_t lab[2];
    uint4 scv[8];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int j = base + t + q * nthr;
      if (j < C) {
        const int tt = tile0 + j;
        lab[q] = __ldg(p.bitmap + (tt >> 3)) >> (tt & 7);
        idx[q] = __ldg(p.tile_idx + tt);
      }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {  // 32 rows x 2 B = four 16-byte pieces per tile column
      const int e = 4 * base + t + q * nthr;
      if (e < 4 * C)
        scv[q] = __ldg(reinterpret_cast<const uint4*>(p.scales + (size_t)(tile0 + (e >> 2)) * bN + nl0 + 8 * (e & 3)));
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int j0 = base + q * nthr + (t & ~31);  // first tile column of this warp's label word
      if (j0 < C) {
        const int j = base + t + q * nthr;
        const bool is4 = j < C && (lab[q] & 1);
        const unsigned bits = __ballot_sync(0xffffffffu, is4);
        if (lane == 0) tile_is4[j0 >> 5] = bits;
        if (j < C) {
          const size_t pr = (size_t)idx[q] * bN + nl0;
          tile_ptr[j] = is4 ? p.w4 + pr * (kTileK / 2) : reinterpret_cast<const uint8_t*>(p.w8) + pr * kTileK;
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = 4 * base + t + q * nthr;
      if (e < 4 * C) *reinterpret_cast<uint4*>(&tile_sw[e >> 2][8 * (e & 3)]) = scv[q];
    }
  }
  __syncthreads();
  pdl_launch_dependents();
  // the CTA's whole weight slice starts streaming into L2 now, so the DRAM
  // transfer overlaps the activation preparation below and the register ring
  // reads from L2
  for (int j = t; j < C; j += nthr) {
    const bool is4 = (tile_is4[j >> 5] >> (j & 31)) & 1;
    prefetch_l2_bulk(tile_ptr[j], kRows * (is4 ? kTileK / 2 : kTileK));
  }

  // ---- this thread's piece of its i-th tile column (j = kg + KG i)
  auto load = [&](int i, Piece& pc) {
    const int j = kg + KG * i;
    const bool is4 = (tile_is4[j >> 5] >> (j & 31)) & 1;
    if (is4) {
      const uint4* src = reinterpret_cast<const uint4*>(tile_ptr[j] + lrow * (kTileK / 2) + 32 * h);
      pc.v[0] = __ldcs(src);
      pc.v[1] = __ldcs(src + 1);
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(tile_ptr[j] + lrow * kTileK + 64 * h);
      pc.v[0] = __ldcs(src);
      pc.v[1] = __ldcs(src + 1);
      pc.v[2] = __ldcs(src + 2);
      pc.v[3] = __ldcs(src + 3);
    }
  };
  Piece ring[kRing];
#pragma unroll
  for (int q = 0; q < kRing; ++q)
    if (q < nmine) load(q, ring[q]);
  if constexpr (FUSED) {
    // warm L2 with the activations: L2 is coherent, so this is safe even if an
    // earlier kernel is still writing them (the reads below come after the wait)
    const int nlines = (M * a.ldx * 2 + 127) / 128;
    for (int q = t; q < nlines; q += nthr) prefetch_l2(reinterpret_cast<const uint8_t*>(a.x) + 128 * (size_t)q);
  }

  pdl_wait();  // activations (and every global write below) depend on earlier kernels

  const int8_t* xs;    // codes in k order
  const int8_t* xeo;   // codes, even / odd k split per 8 columns (FUSED only)
  const float* sxp;
  if constexpr (FUSED) {
    // per-token absmax over K, then codes into shared memory (same arithmetic as
    // aq_quant_act); each thread keeps up to kXv of its activation vectors in registers
    constexpr int kXv = MT == 1 ? 4 : 2;
    const int nvec = K / 8;
    const int nwarps = nthr / 32;
    float amax[MT];
    uint4 xr[MT][kXv];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      amax[m] = 0.f;
      if (m < M) {
        const uint4* xrow = reinterpret_cast<const uint4*>(a.x + (size_t)m * a.ldx);
#pragma unroll
        for (int q = 0; q < kXv; ++q) {
          const int v = t + q * nthr;
          if (v < nvec) {
            xr[m][q] = __ldg(xrow + v);
            amax[m] = abs_max8(xr[m][q], amax[m]);
          }
        }
        for (int v = t + kXv * nthr; v < nvec; v += nthr) amax[m] = abs_max8(__ldg(xrow + v), amax[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax[m] = fmaxf(amax[m], __shfl_xor_sync(0xffffffffu, amax[m], o));
      if (lane == 0) redq[t >> 5][m] = amax[m];
    }
    __syncthreads();
    uint8_t* cbuf = smem;                       // k order
    uint8_t* ebuf = smem + (size_t)M * K;       // even / odd split
    float* sx_s = reinterpret_cast<float*>(smem + 2 * (size_t)M * K);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
      float am = redq[lane < nwarps ? lane : 0][m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));  // all lanes agree
      const double s = act_scale(am);
      const float r32 = act_recip(s);
      const uint4* xrow = reinterpret_cast<const uint4*>(a.x + (size_t)m * a.ldx);
      auto put = [&](int v, const uint4& xv) {
        const uint2 q = quantize8(xv, s, r32);  // 8 codes of columns 8v .. 8v+7
        *reinterpret_cast<uint2*>(cbuf + (size_t)m * K + 8 * v) = q;
        *reinterpret_cast<uint2*>(ebuf + (size_t)m * K + 8 * v) = make_uint2(even_bytes(q.x, q.y), odd_bytes(q.x, q.y));
      };
#pragma unroll
      for (int q = 0; q < kXv; ++q) {
        const int v = t + q * nthr;
        if (v < nvec) put(v, xr[m][q]);
      }
      for (int v = t + kXv * nthr; v < nvec; v += nthr) put(v, __ldg(xrow + v));
      if (t == 0) sx_s[m] = (float)s;
    }
    __syncthreads();
    xs = reinterpret_cast<const int8_t*>(cbuf);
    xeo = reinterpret_cast<const int8_t*>(ebuf);
    sxp = sx_s;
  } else {
    xs = a.xq;
    xeo = nullptr;
    sxp = a.sx;
  }

  float acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.f;

  auto tile = [&](int i, const Piece& pc) {
    const int j = kg + KG * i;
    const bool is4 = (tile_is4[j >> 5] >> (j & 31)) & 1;
    const float sw = __half2float(__ushort_as_half(tile_sw[j][lrow])) * (is4 ? 0.0625f : 1.0f);
    const size_t xoff = (size_t)j * kTileK + 64 * h;  // this thread's 64 activation columns
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
      int part = 0;
      if (is4) {
        const uint32_t wv[8] = {pc.v[0].x, pc.v[0].y, pc.v[0].z, pc.v[0].w,
                                pc.v[1].x, pc.v[1].y, pc.v[1].z, pc.v[1].w};
        uint4 xe[4];
        if constexpr (FUSED) {
          const uint4* xp = reinterpret_cast<const uint4*>(xeo + (size_t)m * K + xoff);
#pragma unroll
          for (int q = 0; q < 4; ++q) xe[q] = xp[q];  // (even, odd) word pairs of 8-column groups
        } else {
          const uint4* xp = reinterpret_cast<const uint4*>(xs + (size_t)m * K + xoff);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 n = __ldg(xp + q);
            xe[q] = make_uint4(even_bytes(n.x, n.y), odd_bytes(n.x, n.y), even_bytes(n.z, n.w), odd_bytes(n.z, n.w));
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          part = dp4a((wv[2 * q] << 4) & 0xF0F0F0F0u, xe[q].x, part);  // 16 q, even k
          part = dp4a(wv[2 * q] & 0xF0F0F0F0u, xe[q].y, part);         // 16 q, odd k
          part = dp4a((wv[2 * q + 1] << 4) & 0xF0F0F0F0u, xe[q].z, part);
          part = dp4a(wv[2 * q + 1] & 0xF0F0F0F0u, xe[q].w, part);
        }
      } else {
        const uint4* xp = reinterpret_cast<const uint4*>(xs + (size_t)m * K + xoff);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 xv = FUSED ? xp[q] : __ldg(xp + q);
          part = dp4a(pc.v[q].x, xv.x, part);
          part = dp4a(pc.v[q].y, xv.y, part);
          part = dp4a(pc.v[q].z, xv.z, part);
          part = dp4a(pc.v[q].w, xv.w, part);
        }
      }
      if constexpr (DEBUG) {
        int v = part + __shfl_xor_sync(0xffffffffu, part, 1);
        if (h == 0) a.P[((size_t)m * p.N + row) * C + j] = is4 ? (v >> 4) : v;
      }
      acc[m] = fmaf(small_int_to_float(part), sw, acc[m]);
    }
  };

  for (int i0 = 0; i0 < nmine; i0 += kRing) {
#pragma unroll
    for (int q = 0; q < kRing; ++q) {
      const int i = i0 + q;
      if (i < nmine) {
        tile(i, ring[q]);
        if (i + kRing < nmine) load(i + kRing, ring[q]);  // read kRing tiles from now
      }
    }
  }
  if constexpr (DEBUG) return;

  // combine the 2 lanes of a row, then the KG groups, in a fixed order
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    if (m >= M) break;
    const float v = acc[m] + __shfl_xor_sync(0xffffffffu, acc[m], 1);
    if (h == 0) red[kg][lrow][m] = v;
  }
  __syncthreads();
  if (kg == 0 && h == 0) {
    const float bias = p.bias ? __ldg(p.bias + row) : 0.f;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
      float v = red[0][lrow][m];
      for (int q = 1; q < KG; ++q) v += red[q][lrow][m];
      store_out(p.y, a.ydtype, (size_t)m * p.ldy + row, fmaf(sxp[m], v, bias));
    }
  }
}

template <int MT, bool FUSED, bool DEBUG>
cudaError_t launch_rows_t(const RowsArgs& a, int blocks, size_t smem, cudaStream_t st) {
  cudaError_t e = ensure_smem_attr<decode_rows_kernel<MT, FUSED, DEBUG>>((int)kFusedMaxBytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_rows_kernel<MT, FUSED, DEBUG>, dim3(blocks), dim3(kGroupThreads * a.KG), smem, st, a);
}

template <bool FUSED, bool DEBUG>
cudaError_t launch_rows_m(const RowsArgs& a, int blocks, size_t smem, cudaStream_t st) {
  if (a.M <= 1) return launch_rows_t<1, FUSED, DEBUG>(a, blocks, smem, st);
  if (a.M <= 2) return launch_rows_t<2, FUSED, DEBUG>(a, blocks, smem, st);
  if (a.M <= 4) return launch_rows_t<4, FUSED, DEBUG>(a, blocks, smem, st);
  return launch_rows_t<8, FUSED, DEBUG>(a, blocks, smem, st);
}

}  // namespace

bool rows_supported(int M, int K) { return M >= 1 && M <= kRowsMaxM && K / kTileK <= kMaxC; }

cudaError_t launch_decode_rows(const DecodeProj* projs, int G, int K, const uint16_t* x, int ldx, const int8_t* xq,
                               const float* sx, int M, int ydtype, int32_t* P, void* /*ws*/, cudaStream_t st) {
  RowsArgs a;
  memset(&a, 0, sizeof(a));
  int blocks = 0;
  for (int g = 0; g < G; ++g) {
    a.p[g] = projs[g];
    a.p[g].blocks = projs[g].N / kRows;
    blocks += a.p[g].blocks;
  }
  a.G = G; a.K = K; a.C = K / kTileK; a.M = M; a.ydtype = ydtype;
  a.x = x; a.ldx = ldx; a.xq = xq; a.sx = sx; a.P = P;
  // split the tile columns of a CTA over KG thread groups so that ~16 warps per SM stay busy
  const int warps = blocks * (kGroupThreads / 32);
  // at most 256 threads (room for the next launch's CTAs) unless rows are long
  // or the launch has no more CTAs than SMs (then wider CTAs only shorten the
  // per-thread tile loop; with more CTAs 512-thread CTAs would need a second wave)
  const int sms = num_sms();
  const int kg_cap = (a.C >= 32 || blocks <= sms) ? kMaxKG : 4;
  int KG = 1;
  while (KG < kg_cap && warps * KG < 16 * sms && a.C >= 4 * KG) KG *= 2;
  a.KG = KG;
  if (P != nullptr) return launch_rows_m<false, true>(a, blocks, 0, st);
  if (x != nullptr) return launch_rows_m<true, false>(a, blocks, 2 * (size_t)M * K + 16 * (size_t)M, st);
  return launch_rows_m<false, false>(a, blocks, 0, st);
}

}  // namespace aq
