// Decode-phase linear layers on the CUDA cores for 1 or 2 tokens, with every
// warp streaming its own share of the packed weights into shared memory.
//
// AlignQuant, Sec. 3.3 "Decode parallelism" and App. E.3 eq. 19: the packed
// tiles are moved on chip, INT4 tiles are used as INT8 values, every tile
// product is an exact INT32 sum, rescaled by the activation and weight scales
// before FP32 accumulation.  Sec. 3.3 "Shared activation preparation" and
// App. E.4: projections that read the same input (q/k/v, gate/up) run as one
// launch over their concatenated output rows, and for one or two tokens the
// activation quantization is fused into that launch.
//
// Why this shape.  A decode step is a chain of short launches, and each may
// read its activations only once the previous one has finished
// (griddepcontrol.wait); its weights, however, never depend on an earlier
// kernel.  So every warp starts copying its first stages of weights into
// shared memory as soon as its CTA is resident, before the wait, and only the
// activation preparation, the products and the reduction follow the wait.  The
// grid has one CTA per SM.  For launches of up to 100 K weights per SM a CTA
// keeps its shared memory near 104 KB, so the CTAs of two consecutive launches
// fit on every SM side by side: while one launch computes, the next one already
// streams its weights.  Larger launches take the wide shape: one CTA of 16 warps
// with 3-stage rings fills the SM and keeps more bytes in flight through the
// long stream, at the price of the next launch starting its copies only when
// this CTA leaves.  (Measured at 1 token: 8B-class layers 17-20% faster than
// with the narrow shape alone, 14B-class layers 1.6x; a threshold of 200 K made
// the 3B-class model 15% slower, every change of shape between consecutive
// launches costing the next launch its early start.)  (A register-ring
// design that issued its loads from every thread measured a launch-long
// dependent chain: its loads could only start once a CTA had a slot, and a CTA
// only got a slot when the previous launch left.)
//
// Copies.  16-byte cp.async copies, each warp instruction covering 512
// contiguous bytes; measured on B200 they stream at HBM rate (46 GB/s per SM)
// once about 64 KB per SM are in flight, from any number of issuing warps.
// Bulk copies (cp.async.bulk) are not used: an SM completes one about every
// 280 ns whatever the number in flight, which caps pieces of a few KB (rows x
// 64 or 128 bytes of one tile) at 10-30 GB/s per SM.  Each warp owns a ring of
// kRing stages and paces it with cp.async groups (wait_group kRing - 1): no
// stage is handed between warps, so there are no barriers to pair up.  (A
// design with producer and consumer warps paired through mbarriers measured
// far below HBM rate: producers blocked on slots that the consumer of another
// producer's stage held.  A byte-granular ring, packing INT4 stages at half the
// room of INT8 ones so that up to 6 stages per warp were in flight, measured
// 10-25% slower than these fixed slots on every model.)
//
// Work split: the concatenated output rows of the launch are cut into 8-row
// strips and every CTA takes a contiguous range of strips.  The range is
// walked as row blocks of at most kMaxR rows that stay inside one tile row of
// one projection.  A stage is one tile column of one row block: `rows`
// consecutive rows of one packed tile, a single contiguous piece of the INT4
// or INT8 buffer (eq. 16 locates the tile), plus the tile's fp16 scales of
// those rows.  The CTA's stages, block by block, are cut into kWarps
// contiguous runs, one per warp, so a warp changes row block (and reduces its
// lane partials) only once or twice.
//
// Lanes: lane l owns input columns [16 (l % 8), 16 (l % 8) + 16) of a tile and
// the rows 4 i + l / 8, so one warp instruction reads four whole tile rows
// (512 contiguous bytes of INT8, 256 of INT4) from shared memory without bank
// conflicts.  INT4 nibbles are used as 16 q (a nibble in the high half of a
// byte whose low half is zero IS the two's-complement byte 16 q), so one dp4a
// against the even / odd activation bytes gives 16 x the exact product and the
// scale is divided by 16 (exact).  Each lane keeps FP32 sums of (exact lane
// partial) x (tile scale) per row and token; at the end of a row block the 8
// lanes of a row are combined, then the warps in a fixed order.
#include <algorithm>

#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kMaxR = 32;                        // rows of a row block (stage), at most
constexpr int kSlotBytes = kMaxR * kTileK;       // one stage: up to 32 rows of an INT8 tile
constexpr int kSlotScBytes = kMaxR * 2;          // the stage's fp16 row scales
constexpr int kMaxBlocks = 16;
constexpr int kMaxCtaRows = 256;

// The two shapes of the kernel: warps per CTA, stages in flight per warp, CTAs per
// SM the shape is built for, and its shared-memory limit per CTA.
template <int WARPS, int RING, int CTAS_PER_SM, int SMEM_KB>
struct StreamShape {
  static constexpr int kWarps = WARPS, kRing = RING, kCtasPerSm = CTAS_PER_SM;
  static constexpr int kThreads = 32 * WARPS;
  static constexpr size_t kRingBytes = (size_t)WARPS * RING * (kSlotBytes + kSlotScBytes);
  static constexpr size_t kSmemLimit = (size_t)SMEM_KB * 1024;
};
// 12 warps (fewer left the stage loop latency-bound), 2 stages each: two launches' CTAs per SM (228 KB)
using ShapeShared = StreamShape<12, 2, 2, 112>;
// 16 warps, 3 stages each: one CTA per SM (220 KB dynamic + static shared memory < 227 KB)
using ShapeWide = StreamShape<16, 3, 1, 220>;
// launches with more weights than this per SM take the wide shape
constexpr long long kWideWeightsPerSm = 100 * 1024;

struct SProj {
  const uint8_t* bitmap;
  const int32_t* tile_idx;
  const uint8_t* w4;
  const int8_t* w8;
  const uint16_t* scales;
  const float* bias;
  void* y;
  int N, bN, ldy, row0;  // row0: first row of this projection among the launch's rows
};

struct SArgs {
  SProj p[kMaxGroup];
  int G, K, C, M, ydtype;
  int strips;        // 8-row strips over all projections
  int cta_rows;      // rows of the largest CTA range (sizes the reduction buffer)
  const uint16_t* x; // bf16 activations [M][ldx] (fused preparation), or null
  int ldx;
  const int8_t* xq;  // pre-quantized activations [M][K], or null
  const float* sx;
  int32_t* P;        // debug: exact tile products [M][N][C] of projection 0
};

struct Block {
  int g, r, nl0, rows, crow;  // projection, tile row, first row inside the tile row, rows, CTA-local first row
};

// Row blocks of the CTA's row range [lo, hi); -1 if they do not fit kMaxBlocks.
__device__ int cta_blocks(const SArgs& a, int lo, int hi, Block* out) {
  int n = 0, pos = lo;
  while (pos < hi && n < kMaxBlocks) {
    int g = 0;
    while (g + 1 < a.G && pos >= a.p[g + 1].row0) ++g;
    const int local = pos - a.p[g].row0, bN = a.p[g].bN;
    const int r = local / bN, nl0 = local - r * bN;
    int rows = min(hi - pos, a.p[g].N - local);
    rows = min(rows, bN - nl0);
    rows = min(rows, kMaxR);
    out[n].g = g;
    out[n].r = r;
    out[n].nl0 = nl0;
    out[n].rows = rows;
    out[n].crow = pos - lo;
    ++n;
    pos += rows;
  }
  return pos < hi ? -1 : n;
}

__device__ __forceinline__ int dp4a(uint32_t a, uint32_t b, int c) { return __dp4a((int)a, (int)b, c); }

// Exact int -> float for |v| < 2^22 with an integer add and a float subtract.
__device__ __forceinline__ float small_int_to_float(int v) { return __int_as_float(v + 0x4B400000) - 12582912.0f; }

__device__ __forceinline__ uint32_t even_bytes(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x6420); }
__device__ __forceinline__ uint32_t odd_bytes(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x7531); }

// 16-byte global -> shared copy through L2 (no L1 allocation).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Wait until at most N of this thread's most recent cp.async groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Where one stage's bytes come from (computed a batch of 32 stages at a time,
// lane l holding the record of the batch's stage l).
struct StageRec {
  unsigned long long src, scs;
  uint32_t bytes_is4;  // bytes | is4 << 31
};

// (two CTAs per SM: the running launch and the next one, which streams its weights)
template <class Shape, int MT, bool FUSED, bool DEBUG>
__global__ void __launch_bounds__(Shape::kThreads, Shape::kCtasPerSm) decode_stream_kernel(const __grid_constant__ SArgs a) {
  constexpr int kWarps = Shape::kWarps, kRing = Shape::kRing, kStreamThreads = Shape::kThreads;
  constexpr size_t kRingBytes = Shape::kRingBytes;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ Block blocks[kMaxBlocks];
  __shared__ float redq[kWarps][MT];
  __shared__ float sx_s[MT];
  __shared__ int nblocks_s;

  const int C = a.C, K = a.K, M = a.M;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c8 = lane & 7, rq = lane >> 3;
  uint8_t* wring = smem + (size_t)warp * kRing * kSlotBytes;  // this warp's [kRing][kSlotBytes]
  uint8_t* sring = smem + (size_t)kWarps * kRing * kSlotBytes + (size_t)warp * kRing * kSlotScBytes;
  int8_t* act = reinterpret_cast<int8_t*>(smem + kRingBytes);  // [MT][K] codes
  float* red = reinterpret_cast<float*>(act + (size_t)MT * K);  // [kWarps][cta_rows][MT]

  const int lo = (int)((unsigned)a.strips * blockIdx.x / gridDim.x) * 8;  // (strips x grid < 2^32)
  const int hi = (int)((unsigned)a.strips * (blockIdx.x + 1) / gridDim.x) * 8;
  if (threadIdx.x == 0) nblocks_s = cta_blocks(a, lo, hi, blocks);
  __syncthreads();
  const int nb = nblocks_s;
  if (nb < 0) return;  // the host never builds such a launch (rows per CTA are capped)
  const int T = nb * C;  // stages of the CTA: stage g is tile column g % C of row block g / C
  const int g0 = T * warp / kWarps;
  const int Tw = T * (warp + 1) / kWarps - g0;  // this warp's stages g0 .. g0 + Tw - 1

  // record of this warp's stage k (k in [32 q, 32 q + 32) for the batch q held by the lane)
  auto make_rec = [&](int k) {
    StageRec rec;
    rec.src = rec.scs = 0;
    rec.bytes_is4 = 0;
    if (k < Tw) {
      const int g = g0 + k;
      const int b = g / C, j = g - b * C;
      const Block blk = blocks[b];
      const SProj& p = a.p[blk.g];
      const int t = blk.r * C + j;
      const uint32_t is4 = (__ldg(p.bitmap + (t >> 3)) >> (t & 7)) & 1u;
      const size_t prow = (size_t)__ldg(p.tile_idx + t) * p.bN + blk.nl0;
      rec.src = is4 ? reinterpret_cast<unsigned long long>(p.w4 + prow * (kTileK / 2))
                    : reinterpret_cast<unsigned long long>(p.w8 + prow * kTileK);
      rec.scs = reinterpret_cast<unsigned long long>(p.scales + (size_t)t * p.bN + blk.nl0);
      rec.bytes_is4 = (uint32_t)(blk.rows * (is4 ? kTileK / 2 : kTileK)) | (is4 << 31);
    }
    return rec;
  };
  StageRec cur = make_rec(lane), nxt = make_rec(32 + lane);  // batches 0 and 1 (loads in flight together)
  int cur_q = 0;
  uint32_t ring_is4 = 0;  // INT4 label of the stage in each ring slot (bit = slot)
  // copy this warp's stage k into its ring slot k % kRing and commit it as one group
  auto issue = [&](int k) {
    if (k < Tw) {
      if (k >= 32 * (cur_q + 1)) {  // next batch of records; fetch the one after it
        cur = nxt;
        ++cur_q;
        nxt = make_rec(32 * (cur_q + 1) + lane);
      }
      const int src_lane = k - 32 * cur_q;
      const uint8_t* s = reinterpret_cast<const uint8_t*>(__shfl_sync(0xffffffffu, cur.src, src_lane));
      const uint8_t* sc = reinterpret_cast<const uint8_t*>(__shfl_sync(0xffffffffu, cur.scs, src_lane));
      const uint32_t bi = __shfl_sync(0xffffffffu, cur.bytes_is4, src_lane);
      const uint32_t bytes = bi & 0x7FFFFFFFu;
      const uint32_t scb = ((bi >> 31) ? bytes / (kTileK / 2) : bytes / kTileK) * 2;  // rows x 2 bytes
      const int slot = k % kRing;
      ring_is4 = (ring_is4 & ~(1u << slot)) | ((bi >> 31) << slot);
      uint8_t* wd = wring + (size_t)slot * kSlotBytes;
      uint8_t* sd = sring + (size_t)slot * kSlotScBytes;
      for (uint32_t c = 16 * lane; c < bytes; c += 512) cp_async16(wd + c, s + c);
      for (uint32_t c = 16 * lane; c < scb; c += 512) cp_async16(sd + c, sc + c);
    }
    cp_async_commit();  // (an empty group past the warp's last stage keeps the group count uniform)
  };
  // the first kRing stages stream while the previous kernel still runs
#pragma unroll
  for (int k = 0; k < kRing; ++k) issue(k);
  // The next launch may be scheduled as soon as every CTA of this one is resident:
  // its CTAs take the SM's second slot where the shapes allow it and start their
  // own weight copies.  (Measured against triggering after the activation
  // preparation: equal on the 3B- and 8B-class steps, 7% faster on the single
  // 2048 x 2048 layer; without the trigger the 3B-class step takes 20% longer.)
  pdl_launch_dependents();

  for (int i = threadIdx.x; i < kWarps * a.cta_rows * MT; i += kStreamThreads) red[i] = 0.f;
  // warm L2 with the activations: L2 is coherent, so this is safe even while an
  // earlier kernel still writes them (they are read only after the wait)
  {
    const uint8_t* xb = FUSED ? reinterpret_cast<const uint8_t*>(a.x) : reinterpret_cast<const uint8_t*>(a.xq);
    const size_t xbytes = FUSED ? (size_t)M * a.ldx * 2 : (size_t)M * K;
    for (size_t o = 128 * (size_t)threadIdx.x; o < xbytes; o += 128 * (size_t)kStreamThreads) prefetch_l2(xb + o);
  }

  pdl_wait();  // activations (and every global write below) depend on earlier kernels
  if constexpr (FUSED) {
    // per-token absmax over K, then the codes into shared memory (same arithmetic as aq_quant_act)
    constexpr int kXv = 4 / MT;
    const int nvec = K / 8;
    float amax[MT];
    uint4 xr[MT][kXv];
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      amax[m] = 0.f;
      if (m < M) {
        const uint4* xrow = reinterpret_cast<const uint4*>(a.x + (size_t)m * a.ldx);
#pragma unroll
        for (int q = 0; q < kXv; ++q) {
          const int v = threadIdx.x + q * kStreamThreads;
          if (v < nvec) {
            xr[m][q] = __ldg(xrow + v);
            amax[m] = abs_max8(xr[m][q], amax[m]);
          }
        }
        for (int v = threadIdx.x + kXv * kStreamThreads; v < nvec; v += kStreamThreads)
          amax[m] = abs_max8(__ldg(xrow + v), amax[m]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax[m] = fmaxf(amax[m], __shfl_xor_sync(0xffffffffu, amax[m], o));
      if (lane == 0) redq[warp][m] = amax[m];
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
      float am = redq[0][m];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) am = fmaxf(am, redq[w][m]);
      const double s = act_scale(am);
      const float r32 = act_recip(s);
      const uint4* xrow = reinterpret_cast<const uint4*>(a.x + (size_t)m * a.ldx);
      uint2* crow = reinterpret_cast<uint2*>(act + (size_t)m * K);
#pragma unroll
      for (int q = 0; q < kXv; ++q) {
        const int v = threadIdx.x + q * kStreamThreads;
        if (v < nvec) crow[v] = quantize8(xr[m][q], s, r32);
      }
      for (int v = threadIdx.x + kXv * kStreamThreads; v < nvec; v += kStreamThreads)
        crow[v] = quantize8(__ldg(xrow + v), s, r32);
      if (threadIdx.x == 0) sx_s[m] = (float)s;
    }
  } else {
    const int nv = M * K / 16;
    const uint4* src = reinterpret_cast<const uint4*>(a.xq);
    uint4* dst = reinterpret_cast<uint4*>(act);
    for (int v = threadIdx.x; v < nv; v += kStreamThreads) dst[v] = __ldg(src + v);
    if (!DEBUG && threadIdx.x < M) sx_s[threadIdx.x] = __ldg(a.sx + threadIdx.x);
  }
  __syncthreads();

  float acc[kMaxR / 4][MT];
#pragma unroll
  for (int i = 0; i < kMaxR / 4; ++i)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[i][m] = 0.f;

  // the lane partials of a finished row block: 8 lanes per row, then one slot per (warp, row)
  auto flush = [&](int b) {
    const int nins = blocks[b].rows / 4, crow = blocks[b].crow;
#pragma unroll
    for (int i = 0; i < kMaxR / 4; ++i) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float v = acc[i][m];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        if (c8 == 0 && i < nins) red[((size_t)warp * a.cta_rows + crow + 4 * i + rq) * MT + m] = v;
        acc[i][m] = 0.f;
      }
    }
  };

  int cur_b = -1;
  int b = g0 / C, j = g0 - b * C;  // block and tile column of stage g0 + k
  for (int k = 0; k < Tw; ++k) {
    if (k > 0 && ++j == C) {
      j = 0;
      ++b;
    }
    if (b != cur_b) {
      if (cur_b >= 0) flush(cur_b);
      cur_b = b;
    }
    cp_async_wait_group<kRing - 1>();  // this lane's copies of stage k have landed
    __syncwarp();                      // ... and every lane's
    const bool is4 = (ring_is4 >> (k % kRing)) & 1u;
    const int nins = blocks[b].rows / 4;
    const uint8_t* ws = wring + (size_t)(k % kRing) * kSlotBytes;
    const uint16_t* ss = reinterpret_cast<const uint16_t*>(sring + (size_t)(k % kRing) * kSlotScBytes);
    uint4 xk[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m)
      xk[m] = m < M ? *reinterpret_cast<const uint4*>(act + (size_t)m * K + j * kTileK + 16 * c8)
                    : make_uint4(0, 0, 0, 0);
    // Every row group of the slot is loaded (reads past a short block's rows stay
    // inside the slot and are not used), so the loads are issued ahead of the math.
    if (!is4) {
      uint4 w[kMaxR / 4];
      float sw[kMaxR / 4];
#pragma unroll
      for (int i = 0; i < kMaxR / 4; ++i) {
        w[i] = *reinterpret_cast<const uint4*>(ws + (4 * i + rq) * kTileK + 16 * c8);
        sw[i] = i < nins ? __half2float(__ushort_as_half(ss[4 * i + rq])) : 0.f;  // rows past the block add 0
      }
#pragma unroll
      for (int i = 0; i < kMaxR / 4; ++i) {
        if (DEBUG ? i < nins : true) {
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            int p = dp4a(w[i].x, xk[m].x, 0);
            p = dp4a(w[i].y, xk[m].y, p);
            p = dp4a(w[i].z, xk[m].z, p);
            p = dp4a(w[i].w, xk[m].w, p);
            if constexpr (DEBUG) {
              p += __shfl_xor_sync(0xffffffffu, p, 1);
              p += __shfl_xor_sync(0xffffffffu, p, 2);
              p += __shfl_xor_sync(0xffffffffu, p, 4);
              const Block& blk = blocks[b];
              const int n = blk.r * a.p[0].bN + blk.nl0 + 4 * i + rq;
              if (c8 == 0 && m < M) a.P[((size_t)m * a.p[0].N + n) * C + j] = p;
            } else {
              acc[i][m] = fmaf(small_int_to_float(p), sw[i], acc[i][m]);
            }
          }
        }
      }
    } else {
      uint32_t xe0[MT], xo0[MT], xe1[MT], xo1[MT];  // even / odd bytes of columns 0-7 and 8-15
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        xe0[m] = even_bytes(xk[m].x, xk[m].y);
        xo0[m] = odd_bytes(xk[m].x, xk[m].y);
        xe1[m] = even_bytes(xk[m].z, xk[m].w);
        xo1[m] = odd_bytes(xk[m].z, xk[m].w);
      }
      uint2 w[kMaxR / 4];
      float sw[kMaxR / 4];
#pragma unroll
      for (int i = 0; i < kMaxR / 4; ++i) {
        w[i] = *reinterpret_cast<const uint2*>(ws + (4 * i + rq) * (kTileK / 2) + 8 * c8);
        sw[i] = i < nins ? __half2float(__ushort_as_half(ss[4 * i + rq])) * 0.0625f : 0.f;  // rows past the block add 0
      }
#pragma unroll
      for (int i = 0; i < kMaxR / 4; ++i) {
        if (DEBUG ? i < nins : true) {
          const uint32_t e0 = (w[i].x << 4) & 0xF0F0F0F0u, o0 = w[i].x & 0xF0F0F0F0u;
          const uint32_t e1 = (w[i].y << 4) & 0xF0F0F0F0u, o1 = w[i].y & 0xF0F0F0F0u;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            int p = dp4a(e0, xe0[m], 0);  // 16 q, even columns
            p = dp4a(o0, xo0[m], p);      // 16 q, odd columns
            p = dp4a(e1, xe1[m], p);
            p = dp4a(o1, xo1[m], p);
            if constexpr (DEBUG) {
              p += __shfl_xor_sync(0xffffffffu, p, 1);
              p += __shfl_xor_sync(0xffffffffu, p, 2);
              p += __shfl_xor_sync(0xffffffffu, p, 4);
              const Block& blk = blocks[b];
              const int n = blk.r * a.p[0].bN + blk.nl0 + 4 * i + rq;
              if (c8 == 0 && m < M) a.P[((size_t)m * a.p[0].N + n) * C + j] = p >> 4;
            } else {
              acc[i][m] = fmaf(small_int_to_float(p), sw[i], acc[i][m]);
            }
          }
        }
      }
    }
    __syncwarp();       // every lane is done reading the slot before it is refilled
    issue(k + kRing);   // into the slot stage k just left
  }
  cp_async_wait_all();  // (only empty groups remain; no thread leaves with copies in flight)
  if constexpr (DEBUG) return;
  if (cur_b >= 0) flush(cur_b);
  __syncthreads();

  // sum the warps in a fixed order, scale by the token scale, add bias, store
  for (int row = threadIdx.x; row < hi - lo; row += kStreamThreads) {
    const int gpos = lo + row;
    int g = 0;
    while (g + 1 < a.G && gpos >= a.p[g + 1].row0) ++g;
    const SProj& p = a.p[g];
    const int n = gpos - p.row0;
    const float bias = p.bias ? __ldg(p.bias + n) : 0.f;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m >= M) break;
      float v = red[(size_t)row * MT + m];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) v += red[((size_t)w * a.cta_rows + row) * MT + m];
      const float out = fmaf(sx_s[m], v, bias);
      const size_t idx = (size_t)m * p.ldy + n;
      if (a.ydtype == AQ_F32)
        reinterpret_cast<float*>(p.y)[idx] = out;
      else
        reinterpret_cast<__nv_bfloat16*>(p.y)[idx] = __float2bfloat16_rn(out);
    }
  }
}

template <class Shape>
size_t stream_smem(int MT, int K, int cta_rows) {
  return Shape::kRingBytes + (size_t)MT * K + (size_t)Shape::kWarps * cta_rows * MT * 4;
}

template <class Shape, int MT, bool FUSED, bool DEBUG>
cudaError_t launch_stream_t(const SArgs& a, int grid, size_t smem, cudaStream_t st) {
  // all of the SM's unified L1 / shared storage as shared memory (the shared shape:
  // so that the CTAs of two consecutive launches fit side by side)
  cudaError_t e = ensure_smem_attr<decode_stream_kernel<Shape, MT, FUSED, DEBUG>>((int)Shape::kSmemLimit, 100);
  if (e != cudaSuccess) return e;
  return launch_pdl(decode_stream_kernel<Shape, MT, FUSED, DEBUG>, dim3(grid), dim3(Shape::kThreads), smem, st, a);
}

template <class Shape>
cudaError_t launch_stream_s(const SArgs& a, int grid, cudaStream_t st) {
  const size_t smem = stream_smem<Shape>(a.M, a.K, a.cta_rows);
  if (a.M > 2 || smem > Shape::kSmemLimit) return cudaErrorInvalidValue;
  if (a.P != nullptr) return a.M == 1 ? launch_stream_t<Shape, 1, false, true>(a, grid, smem, st)
                                      : launch_stream_t<Shape, 2, false, true>(a, grid, smem, st);
  if (a.x != nullptr) return a.M == 1 ? launch_stream_t<Shape, 1, true, false>(a, grid, smem, st)
                                      : launch_stream_t<Shape, 2, true, false>(a, grid, smem, st);
  return a.M == 1 ? launch_stream_t<Shape, 1, false, false>(a, grid, smem, st)
                  : launch_stream_t<Shape, 2, false, false>(a, grid, smem, st);
}

}  // namespace

// Grid and rows per CTA of a launch over `rows` concatenated output rows.
static void stream_grid(int rows, int* grid, int* cta_rows) {
  // one CTA per SM, unless a CTA would get more rows than its reduction buffer holds
  const int strips = rows / 8;
  const int min_grid = (strips * 8 + kMaxCtaRows - 1) / kMaxCtaRows;
  *grid = std::min(strips, std::max(num_sms(), min_grid));
  *cta_rows = ((strips + *grid - 1) / *grid) * 8;
}

// The wide shape for launches above kWideWeightsPerSm weights per SM, or whose
// activations and reduction buffer do not fit the shared shape.
static bool stream_wide(int M, int K, int rows) {
  int grid, cta_rows;
  stream_grid(rows, &grid, &cta_rows);
  return (long long)rows * K > kWideWeightsPerSm * grid ||
         stream_smem<ShapeShared>(M, K, cta_rows) > ShapeShared::kSmemLimit;
}

bool stream_supported(int M, int K, int rows) {
  if (M < 1 || M > 2 || rows < 8) return false;
  int grid, cta_rows;
  stream_grid(rows, &grid, &cta_rows);
  return stream_wide(M, K, rows) ? stream_smem<ShapeWide>(M, K, cta_rows) <= ShapeWide::kSmemLimit
                                 : stream_smem<ShapeShared>(M, K, cta_rows) <= ShapeShared::kSmemLimit;
}

cudaError_t launch_decode_stream(const DecodeProj* projs, int G, int K, const uint16_t* x, int ldx, const int8_t* xq,
                                 const float* sx, int M, int ydtype, int32_t* P, void* /*ws*/, cudaStream_t st) {
  SArgs a;
  memset(&a, 0, sizeof(a));
  int rows = 0;
  for (int g = 0; g < G; ++g) {
    a.p[g].bitmap = projs[g].bitmap;
    a.p[g].tile_idx = projs[g].tile_idx;
    a.p[g].w4 = projs[g].w4;
    a.p[g].w8 = projs[g].w8;
    a.p[g].scales = projs[g].scales;
    a.p[g].bias = projs[g].bias;
    a.p[g].y = projs[g].y;
    a.p[g].N = projs[g].N;
    a.p[g].bN = projs[g].bN;
    a.p[g].ldy = projs[g].ldy;
    a.p[g].row0 = rows;
    rows += projs[g].N;
  }
  a.G = G; a.K = K; a.C = K / kTileK; a.M = M; a.ydtype = ydtype;
  a.x = x; a.ldx = ldx; a.xq = xq; a.sx = sx; a.P = P;
  a.strips = rows / 8;
  int grid;
  stream_grid(rows, &grid, &a.cta_rows);
  if (M < 1 || M > 2) return cudaErrorInvalidValue;
  return stream_wide(M, K, rows) ? launch_stream_s<ShapeWide>(a, grid, st) : launch_stream_s<ShapeShared>(a, grid, st);
}

}  // namespace aq
