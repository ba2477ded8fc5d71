// Mixed W4/W8 x A8 linear layer on the 5th-generation tensor cores (tcgen05).
//
// AlignQuant, Sec. 3.3 ("Integer operand preparation", "Prefill weight reuse",
// "Output reconstruction") and App. E.3 eq. 19: packed tiles are moved on
// chip, INT4 tiles are sign-extended to INT8 on chip, every tile product is
// an exact INT32 sum, and each is rescaled by its activation and weight
// scales before FP32 accumulation over the input tiles.
//
// Roles in one CTA (persistent over work units; every role walks the same
// sequence of input tiles g = 0, 1, 2, ... of the CTA's units):
//   warp 0      weight producer: INT8 tiles -> swizzled A stage (TMA), INT4
//               tiles -> staging buffer (TMA), the tile's fp16 row scales ->
//               the stage's scale area (bulk copy).  It does not wait for the
//               previous kernel, so the first stages load while it finishes.
//   warp 1      allocates tensor memory; one lane issues tcgen05.mma
//               (kind::i8, M = 128 weight rows, N = NT tokens, K = 32) four
//               times per 128-wide input tile into one of four INT32
//               accumulator buffers in tensor memory.
//   warp 2      tile metadata: all 32 lanes read labels and physical tile
//               indices (AlignQuant, App. E.2 eq. 16) up to 32 tiles ahead and
//               turn them into ready-made copy records in a shared-memory
//               ring, so the producers spend a handful of instructions per tile.
//   warp 3      activation producer: the NT x 128 INT8 activation tile -> B
//               stage (TMA), after the previous kernel (which writes the
//               activations) is done.
//   warps 4-7   transform: one thread per row of the 128-row block.  Tile by
//               tile they put each row's weight scale (fp16 -> fp32, / 16 for
//               INT4) into a shared-memory ring and expand the INT4 staging
//               tiles into the 128-byte-swizzled INT8 A layout
//               (fence.proxy.async before signalling the MMA).  They run ahead
//               of the epilogue, bounded only by the stage ring.
//   warps 8..   epilogue; warp w may read tensor-memory lanes 32 (w % 4) ..
//               32 (w % 4) + 31.  After every input tile it reads the INT32
//               tile product from tensor memory, multiplies by the row's
//               weight scale of that tile and accumulates in FP32 registers;
//               at the end of a work unit it multiplies by the token scale,
//               adds bias and stores.  Tiles are rescaled in pairs (one
//               accumulator wait and one release per two tiles) and the
//               tensor-memory loads are software pipelined: the next 16
//               columns are in flight while the current ones are rescaled.
// A single thread on a busy SM retires roughly one dependent instruction every
// 10-20 cycles, so the per-tile work of each issuing thread is kept to a few
// dozen instructions and spread over three threads, and everything the
// epilogue does per tile besides the rescale runs in other warps.
// Weights are the A operand, so TMEM lane = output row and each epilogue
// thread applies ONE weight scale per input tile.
//
// The FP32 rescale is the co-bottleneck of this design: per input tile and
// output element it costs one add and one fused multiply-add on the CUDA
// cores, as many cycles per SM as the INT8 MMA itself; the float2 forms
// halve the issue slots it takes so tensor-memory work fits beside it.
//
// A launch may cover up to kMaxGroup projections that read the same input
// (q/k/v, gate/up: AlignQuant Sec. 3.3 "Shared activation preparation", App.
// E.4): their 128-row blocks are concatenated, each block belonging to one
// member (every member's rows are a multiple of 128 then), and each role looks
// up the member of the block it works on.
// A work unit is (128-row block of output features, NT-token block, split of
// the input tiles).  Split partial sums go to the workspace; the CTA that
// finishes a unit last sums all splits in increasing split order.
// Every mbarrier wait is bounded (see mbar_wait); a wait that gives up records
// AQ_ERR_TIMEOUT in the workspace and raises a CTA-wide abort flag; every
// role then leaves its loop, the copy issuers give their copies in flight a
// grace period, the MMA lane waits (bounded) for its MMAs, and the CTA frees
// its tensor memory and exits.
#include <algorithm>
#include <cstring>

#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kBufs = 4;        // accumulator buffers in tensor memory
constexpr int kSwRing = 16;     // ring of per-row weight scales, one slot per tile (> stages + kBufs)
constexpr int kMetaSlots = 32;  // metadata ring slots (one per lane of the metadata warp)
constexpr int kDone = 16;       // MMA-completion barriers, one per tile, reused every kDone tiles
constexpr int kMaxTcSplits = 8;  // split-K bound of the decode plan (the reduction unrolls over it)
constexpr int kFirstXfWarp = 4;   // transform warps: INT4 expansion and per-row weight scales
constexpr int kXfWarps = 4;       // 128 threads, one per row of the 128-row block
constexpr int kFirstEpiWarp = kFirstXfWarp + kXfWarps;

template <int NT>
struct TcShape {
  static constexpr int kA = 128 * kTileK;        // swizzled INT8 weight block
  static constexpr int kStg = 128 * kTileK / 2;  // INT4 staging (row-major, 64 B per row)
  static constexpr int kB = NT * kTileK;         // swizzled INT8 activation block
  static constexpr int kStageBytes = kA + kB + kStg;
  static constexpr int kStages = (200 * 1024) / kStageBytes < 8 ? (200 * 1024) / kStageBytes : 8;
  static constexpr int kCols = NT <= 64 ? NT : NT / 2;  // accumulator columns per epilogue thread
  static constexpr int kEpiWarps = 4 * NT / kCols;      // 4 warps (one per lane quadrant) per column group
  static constexpr int kThreads = 32 * kFirstEpiWarp + 32 * kEpiWarps;
  // Tensor-memory columns per load (one 16-column load; two register sets are
  // live while the loads are pipelined).
  static constexpr int kLdCols = 16;
  static_assert(kCols % kLdCols == 0, "load chunks");
  // Registers per thread: the register file over the block's warps, counted in
  // groups of four warps as the hardware allocates them (an explicit cap: the
  // block-size bound makes the compiler trade registers for spills here).
  static constexpr int kMaxRegsRaw = 65536 / (128 * ((kThreads + 127) / 128)) / 8 * 8;
  static constexpr int kMaxRegs = kMaxRegsRaw > 255 ? 255 : kMaxRegsRaw;
  static constexpr int kTmemCols = kBufs * NT <= 32 ? 32 : kBufs * NT <= 64 ? 64 : kBufs * NT <= 128 ? 128
                                   : kBufs * NT <= 256 ? 256 : 512;
  static constexpr int kScBytes = kStages * 256;  // per stage: the tile's 128 row scales (fp16)
  static constexpr int kSwBytes = kSwRing * 128 * 4;  // [kSwRing][row] fp32
  static constexpr int kCtrlBytes = 2048;
  static constexpr int kPreBytes = (32 + kCols) * kEpiWarps * 4;  // per-unit bias and token scales of the epilogue
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kScBytes + kCtrlBytes + kPreBytes + kSwBytes;
  static constexpr uint32_t kIdesc = idesc_i8(128, NT);
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 128, "MMA N");
  static_assert(kBufs * NT <= 512, "tensor memory");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kStages >= 3, "ring depth");
  // the transform warps run at most kStages + kBufs tiles ahead of the epilogue
  // (a stage is refilled only after its MMAs, which wait for an accumulator
  // buffer the epilogue released), so a scale slot is never rewritten early
  static_assert(kStages + kBufs < kSwRing, "scale ring depth");
  // a tile's completion barrier is waited for (by the epilogue, and by the
  // producers refilling its stage) before the MMA can complete tile + kDone
  static_assert(kDone > kStages && kDone > kBufs, "completion ring depth");
  static_assert(kThreads <= 1024, "block size");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

constexpr uint32_t kAccBias = 0x4B400000u;  // fp32 bit pattern of 12582912 = 1.5 * 2^23
constexpr float kAccBiasF = 12582912.0f;
constexpr unsigned long long kAbortGraceNs = 200000;  // copies in flight when a CTA gives up

// One projection of the launch.
struct TcMember {
  const uint8_t* bitmap;
  const int32_t* tile_idx;
  const uint16_t* scales;
  const float* bias;
  void* y;
  int ldy, N, R, T4, T8;
  int rb0;  // first 128-row block of the member among the launch's blocks
};

struct TcArgs {
  TcMember mem[kMaxGroup];
  int G;
  int N, K, bN, C;  // N: rows of all members (the split partial sums span them)
  int tpb;     // tile rows per 128-row block (1 for bN = 128, 2 for bN = 64)
  int nrb;     // number of 128-row blocks
  int M, ntb;  // tokens, token blocks
  int S, units;
  const float* sx;
  int ydtype;
  void* ws;
  float* partial;  // [S][N][Mp], Mp = M rounded up to a multiple of 4
  int* counters;   // [nrb * ntb]
  int ws_clear;    // bytes of split-K counters after the workspace header (0 without splits)
  unsigned long long wait_ns;  // limit of every bounded wait (kWaitTimeoutNs; shorter in the stall test)
  int stop_after;  // >= 0: the weight producer stops after this many tiles (stall test); -1 otherwise
  int32_t* P;      // debug: exact tile products [M][N][C], or null
};

struct Unit {
  int rb, tb, s, j0, j1;
};

// Member owning 128-row block rb (member 0 in a single-projection kernel).
template <bool GROUPED>
__device__ __forceinline__ int member_of(const TcArgs& a, int rb) {
  if constexpr (!GROUPED) return 0;
  int g = 0;
  while (g + 1 < a.G && rb >= a.mem[g + 1].rb0) ++g;
  return g;
}

// Tensor maps of the launch: each member's INT8 and INT4 payloads, and the activations.
struct TcMaps {
  CUtensorMap w8[kMaxGroup];
  CUtensorMap w4[kMaxGroup];
  CUtensorMap x;
};

__device__ __forceinline__ Unit unit_of(const TcArgs& a, int u) {
  Unit x;
  x.s = u % a.S;
  const int rest = u / a.S;
  x.tb = rest % a.ntb;
  x.rb = rest / a.ntb;
  x.j0 = (int)((long long)a.C * x.s / a.S);
  x.j1 = (int)((long long)a.C * (x.s + 1) / a.S);
  return x;
}

// Walks the CTA's input tiles in the order every role processes them.
struct TileIter {
  int u, j;
  Unit x;
  __device__ __forceinline__ explicit TileIter(const TcArgs& a) : u(blockIdx.x), j(0) {
    if (u < a.units) {
      x = unit_of(a, u);
      j = x.j0;
      skip(a);
    }
  }
  __device__ __forceinline__ void skip(const TcArgs& a) {
    while (u < a.units && j >= x.j1) {
      u += gridDim.x;
      if (u < a.units) {
        x = unit_of(a, u);
        j = x.j0;
      }
    }
  }
  __device__ __forceinline__ void next(const TcArgs& a) {
    ++j;
    skip(a);
  }
};

// Per-tile record of the metadata ring: everything the producers need to
// issue the tile's copies.
struct MetaRec {
  uint32_t a_row0, a_row1;  // first row of each sub-tile's weight tile in its precision's buffer
  uint32_t sizes;           // INT8 KiB | INT4 KiB << 8 | member << 16 | kinds << 28 (copy sizes are whole KiB)
  uint32_t sc_off;          // element offset of sub-tile 0's scales in its member (sub-tile 1: + C * bN)
};
// kinds: bits 0-1 INT4 label of sub-tile 0/1, bits 2-3 sub-tile 0/1 exists
// (the last 128-row block of a bN = 64 layer may hold one tile row only).

// Input tiles the CTA processes (identical in every role).
__device__ __forceinline__ uint32_t cta_tiles(const TcArgs& a) {
  uint32_t n = 0;
  for (int u = blockIdx.x; u < a.units; u += gridDim.x) {
    const Unit x = unit_of(a, u);
    n += x.j1 - x.j0;
  }
  return n;
}

// Ring position with its phase parity.
struct RingPos {
  uint32_t i, ph;
  template <int N>
  __device__ __forceinline__ void next() {
    if (++i == N) {
      i = 0;
      ph ^= 1u;
    }
  }
};

// 8 nibbles (low nibble = even k) -> 8 INT8 bytes holding 16 * q in k order.
// A nibble placed in the high half of a byte with a zero low half IS the
// two's-complement byte 16 q, so no sign extension is needed; the MMA then
// yields 16 P for INT4 tiles and the epilogue scales by sw / 16 (exact).
__device__ __forceinline__ uint2 expand8_x16(uint32_t v) {
  const uint32_t lo = (v << 4) & 0xF0F0F0F0u, hi = v & 0xF0F0F0F0u;
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

__device__ __forceinline__ void store_y(void* y, int ydtype, size_t idx, float v) {
  if (ydtype == AQ_F32)
    reinterpret_cast<float*>(y)[idx] = v;
  else
    reinterpret_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
}

// Orders every later use of r after the preceding tcgen05.wait::ld (the
// registers written by tcgen05.ld are valid only after that wait).
__device__ __forceinline__ void tmem_regs_ready(uint32_t (&r)[16]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}

// 4-byte global -> shared copy; with src_bytes = 0 it writes zero and reads nothing.
__device__ __forceinline__ void cp_async4(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Give bulk / tensor copies already issued time to land before the CTA exits
// after an abort (their completion can no longer be awaited on a barrier that
// another role stopped arming).
__device__ __forceinline__ void abort_grace() {
  const unsigned long long t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 < kAbortGraceNs) __nanosleep(1000);
}

// Largest multiple of 4 that divides kCols and is at most lim.
constexpr int chunk_cols(int kCols, int lim) {
  int c = lim;
  while (c > 4 && kCols % c != 0) c -= 4;
  return c;
}

// Sum of the S split partials of a thread's kCols columns (split order
// increasing), scaled by the token scales, plus bias, stored.  CH columns at a
// time with the loads of all (at most SMAX) splits in flight together.
template <int kCols, int CH, int SMAX>
__device__ __forceinline__ void reduce_splits(const TcArgs& a, const TcMember& mb, const float* prow, size_t sstride,
                                              int mcol0, int n, float bias_n) {
  static_assert(kCols % CH == 0 && CH % 4 == 0, "reduction chunks");
  const bool sx_vec = ((uintptr_t)a.sx & 15) == 0;
#pragma unroll 1
  for (int c0 = 0; c0 < kCols; c0 += CH) {
    float4 v[SMAX][CH / 4];
#pragma unroll
    for (int ss = 0; ss < SMAX; ++ss)
#pragma unroll
      for (int i4 = 0; i4 < CH / 4; ++i4)
        v[ss][i4] = (ss < a.S && mcol0 + c0 + 4 * i4 < a.M)
                        ? __ldcg(reinterpret_cast<const float4*>(prow + ss * sstride + c0) + i4)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i4 = 0; i4 < CH / 4; ++i4) {
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int ss = 0; ss < SMAX; ++ss)
        if (ss < a.S) {
          sum.x += v[ss][i4].x;
          sum.y += v[ss][i4].y;
          sum.z += v[ss][i4].z;
          sum.w += v[ss][i4].w;
        }
      const float sv[4] = {sum.x, sum.y, sum.z, sum.w};
      const int m0 = mcol0 + c0 + 4 * i4;
      float xs[4];
      if (sx_vec && m0 + 3 < a.M) {  // four token scales in one load
        const float4 q = __ldg(reinterpret_cast<const float4*>(a.sx + m0));
        xs[0] = q.x; xs[1] = q.y; xs[2] = q.z; xs[3] = q.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) xs[e] = m0 + e < a.M ? __ldg(a.sx + m0 + e) : 0.f;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (m0 + e < a.M) store_y(mb.y, a.ydtype, (size_t)(m0 + e) * mb.ldy + n, fmaf(xs[e], sv[e], bias_n));
    }
  }
}

// MODE: 0 = outputs written directly (one split), 1 = split-K partial sums
// reduced by the last CTA of each unit group, 2 = exact tile products only.
// GROUPED: the launch covers several projections (decode only); single-projection
// kernels compile without the member lookups, which cost the prefill kernels
// registers (3-9% of their rate when always present).
template <int NT, int MODE, bool GROUPED>
__global__ void __maxnreg__(TcShape<NT>::kMaxRegs)
    tc_linear_kernel(const __grid_constant__ TcMaps maps, const __grid_constant__ TcArgs a) {
  using Sh = TcShape<NT>;
  constexpr int S_ = Sh::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  auto stage_a = [&](int st) { return smem + st * Sh::kStageBytes; };
  auto stage_b = [&](int st) { return smem + st * Sh::kStageBytes + Sh::kA; };
  auto stage_g = [&](int st) { return smem + st * Sh::kStageBytes + Sh::kA + Sh::kB; };
  uint8_t* stage_sc = smem + S_ * Sh::kStageBytes;  // [stage][128] fp16 row scales
  uint8_t* ctrl = stage_sc + Sh::kScBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctrl);  // weights (INT8) + activations landed; one arrival per producer
  uint64_t* staged = full + S_;                        // INT4 staging landed (0 bytes when none)
  uint64_t* expanded = staged + S_;                    // transform warps done with the stage (one arrival each)
  // mma_done[g % kDone]: the MMAs of tile g are complete (one commit per tile):
  // its stage may be refilled and its accumulator buffer read
  uint64_t* mma_done = expanded + S_;
  uint64_t* tmem_empty = mma_done + kDone;
  uint64_t* meta_full = tmem_empty + kBufs;
  uint64_t* meta_empty = meta_full + kMetaSlots;
  uint64_t* epi_sync = meta_empty + kMetaSlots;  // epilogue-only rendezvous (bounded, unlike bar.sync)
  uint64_t* drain = epi_sync + 1;                // MMA completion on the way out
  uint64_t* sw_full = drain + 1;                 // [kSwRing] scale slot written (one arrival per transform warp)
  MetaRec* meta = reinterpret_cast<MetaRec*>(sw_full + kSwRing);
  volatile uint32_t* stage_info = reinterpret_cast<volatile uint32_t*>(meta + kMetaSlots);
  uint32_t* tmem_slot = const_cast<uint32_t*>(stage_info + S_);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* never_flag = reinterpret_cast<volatile int*>(tmem_slot + 3);  // stays 0: drain waits
  float* pre_bias = reinterpret_cast<float*>(ctrl + Sh::kCtrlBytes);  // [32 kEpiWarps] bias of each epilogue row
  float* pre_sx = pre_bias + 32 * Sh::kEpiWarps;                       // [kEpiWarps][kCols] token scales
  float* pre_sw = pre_sx + Sh::kEpiWarps * Sh::kCols;                    // [kSwRing][128] weight scale of each row
  static_assert((3 * 8 + kDone + kBufs + 2 * kMetaSlots + 2 + kSwRing) * 8 + kMetaSlots * 16 + (8 + 4) * 4 <=
                    Sh::kCtrlBytes,
                "control area");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < S_; ++st) {
      mbar_init(&full[st], 2);
      mbar_init(&staged[st], 1);
      mbar_init(&expanded[st], kXfWarps);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(&tmem_empty[b], Sh::kEpiWarps);
    }
    for (int i = 0; i < kDone; ++i) mbar_init(&mma_done[i], 1);
    for (int s = 0; s < kMetaSlots; ++s) {
      mbar_init(&meta_full[s], 1);
      mbar_init(&meta_empty[s], 1);
    }
    mbar_init(epi_sync, 32 * Sh::kEpiWarps);
    mbar_init(drain, 1);
    for (int i = 0; i < kSwRing; ++i) mbar_init(&sw_full[i], kXfWarps);
    *abort_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&maps.x);
    for (int g = 0; g < a.G; ++g) {
      if (a.mem[g].T8 > 0) prefetch_tmap(&maps.w8[g]);
      if (a.mem[g].T4 > 0) prefetch_tmap(&maps.w4[g]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Sh::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();

  auto fail = [&](int info) {
    *abort_flag = 1;
    record_error(a.ws, AQ_ERR_TIMEOUT, info, a.ws_clear);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ weight producer
    if (lane == 0) {
      const uint32_t g_total = cta_tiles(a);
      RingPos mr{0, 0}, sr{0, 0};
      bool ok = true;
      for (uint32_t g = 0; g < g_total; ++g) {
        if (a.stop_after >= 0 && g >= (uint32_t)a.stop_after) {  // stall test: later stages never fill
          ok = false;
          break;
        }
        if (!mbar_wait(&meta_full[mr.i], mr.ph, abort_flag, a.wait_ns)) { fail(1); ok = false; break; }
        const MetaRec rec = meta[mr.i];
        mbar_arrive(&meta_empty[mr.i]);
        mr.next<kMetaSlots>();
        if (g >= (uint32_t)S_ && !mbar_wait(&mma_done[(g - S_) % kDone], ((g - S_) / kDone) & 1, abort_flag, a.wait_ns)) {
          fail(2);
          ok = false;
          break;
        }
        const uint32_t kinds = rec.sizes >> 28;
        const uint32_t mg = GROUPED ? (rec.sizes >> 16) & 0xFu : 0u;  // member of the tile's row block
        const uint16_t* scales = a.mem[mg].scales;
        const CUtensorMap* m8 = &maps.w8[mg];
        const CUtensorMap* m4 = &maps.w4[mg];
        const uint32_t sc_bytes = (kinds & 8) ? 4u * a.bN : 2u * a.bN;  // fp16 row scales of the tile's sub-tiles
        stage_info[sr.i] = kinds;  // read by the transform warps after `staged`
        mbar_arrive_expect_tx(&full[sr.i], (rec.sizes & 0xFFu) << 10);
        mbar_arrive_expect_tx(&staged[sr.i], (((rec.sizes >> 8) & 0xFFu) << 10) + sc_bytes);
        uint8_t* scd = stage_sc + sr.i * 256;
        bulk_load(scd, scales + rec.sc_off, a.bN * 2, &staged[sr.i]);
        if (kinds & 8) bulk_load(scd + a.bN * 2, scales + rec.sc_off + (uint32_t)a.C * a.bN, a.bN * 2, &staged[sr.i]);
        if (kinds & 1) tma_load_2d(stage_g(sr.i), m4, 0, rec.a_row0, &staged[sr.i]);
        else tma_load_2d(stage_a(sr.i), m8, 0, rec.a_row0, &full[sr.i]);
        if (kinds & 8) {
          if (kinds & 2) tma_load_2d(stage_g(sr.i) + a.bN * (kTileK / 2), m4, 0, rec.a_row1, &staged[sr.i]);
          else tma_load_2d(stage_a(sr.i) + a.bN * kTileK, m8, 0, rec.a_row1, &full[sr.i]);
        }
        sr.next<S_>();
      }
      if (!ok || *abort_flag) {
        // (stall test: wait for the other roles to give up, then for copies in flight)
        const unsigned long long t0 = globaltimer_ns();
        while (!*abort_flag && globaltimer_ns() - t0 < 2 * a.wait_ns) __nanosleep(1000);
        abort_grace();
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t g_total = cta_tiles(a);
      const uint64_t adesc0 = sw128_desc(smem_u32(stage_a(0)));
      const uint64_t bdesc0 = sw128_desc(smem_u32(stage_b(0)));
      RingPos sr{0, 0}, br{0, 0};
      uint32_t g = 0;
      for (; g < g_total; ++g) {
        if (!mbar_wait(&full[sr.i], sr.ph, abort_flag, a.wait_ns)) { fail(4); break; }
        if (!mbar_wait(&expanded[sr.i], sr.ph, abort_flag, a.wait_ns)) { fail(5); break; }
        // use u of a buffer waits for the epilogue's release number u (release 0 = initial bias)
        if (!mbar_wait(&tmem_empty[br.i], br.ph, abort_flag, a.wait_ns)) { fail(6); break; }
        tc_fence_after();
        const uint64_t soff = (uint64_t)((sr.i * Sh::kStageBytes) >> 4);  // descriptor address field: 16-byte units
        const uint32_t d = tmem_base + br.i * NT;
        // the buffer holds the bias kAccBias in every element; all four MMAs accumulate onto it
#pragma unroll
        for (int k = 0; k < kTileK / 32; ++k)  // K = 32 bytes per instruction: +2 in 16-byte units
          mma_i8(d, adesc0 + soff + 2 * k, bdesc0 + soff + 2 * k, Sh::kIdesc, 1u);
        mma_commit(&mma_done[g % kDone]);
        sr.next<S_>();
        br.next<kBufs>();
      }
      if (g > 0) {  // every MMA issued is complete before tensor memory is freed
        mma_commit(drain);
        mbar_wait(drain, 0, never_flag, a.wait_ns);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ tile metadata
    // Lane l fills the records of tiles g = l, l + 32, ...; the unit and the
    // tile index `base` where that unit starts follow g forward.
    uint32_t g = lane;
    int u = blockIdx.x;
    uint32_t base = 0;
    Unit x = unit_of(a, u < a.units ? u : 0);
    while (u < a.units) {
      while (u < a.units && g >= base + (uint32_t)(x.j1 - x.j0)) {
        base += x.j1 - x.j0;
        u += gridDim.x;
        if (u < a.units) x = unit_of(a, u);
      }
      if (u >= a.units) break;
      const int j = x.j0 + (int)(g - base);
      const int ms = g % kMetaSlots;
      if (!mbar_wait(&meta_empty[ms], ((g / kMetaSlots) & 1) ^ 1, abort_flag, a.wait_ns)) { fail(7); break; }
      uint32_t kinds = 0, bytes8 = 0, bytes4 = 0, row[2] = {0, 0};
      const int mg = member_of<GROUPED>(a, x.rb);
      const TcMember& mb = a.mem[mg];
      const int lrb = GROUPED ? x.rb - mb.rb0 : x.rb;  // row block inside the member
      for (int sub = 0; sub < a.tpb; ++sub) {
        const int r = lrb * a.tpb + sub;
        if (r < mb.R) {
          const int t = r * a.C + j;
          const uint32_t is4 = __ldg(mb.bitmap + (t >> 3)) >> (t & 7) & 1;
          kinds |= (1u << (2 + sub)) | (is4 << sub);
          row[sub] = (uint32_t)__ldg(mb.tile_idx + t) * a.bN;
          if (is4) bytes4 += a.bN * (kTileK / 2);
          else bytes8 += a.bN * kTileK;
        }
      }
      MetaRec rec;
      rec.a_row0 = row[0];
      rec.a_row1 = row[1];
      rec.sizes = (bytes8 >> 10) | ((bytes4 >> 10) << 8) | ((uint32_t)mg << 16) | (kinds << 28);
      rec.sc_off = (uint32_t)((lrb * a.tpb) * a.C + j) * a.bN;
      meta[ms] = rec;
      mbar_arrive(&meta_full[ms]);
      g += kMetaSlots;
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      const uint32_t g_total = cta_tiles(a);
      pdl_wait();  // activations come from an earlier kernel
      TileIter bi(a);
      RingPos sr{0, 0};
      bool ok = true;
      for (uint32_t g = 0; g < g_total; ++g, bi.next(a)) {
        if (g >= (uint32_t)S_ && !mbar_wait(&mma_done[(g - S_) % kDone], ((g - S_) / kDone) & 1, abort_flag, a.wait_ns)) {
          fail(3);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[sr.i], Sh::kB);
        tma_load_2d(stage_b(sr.i), &maps.x, bi.j * kTileK, bi.x.tb * NT, &full[sr.i]);
        sr.next<S_>();
      }
      if (!ok || *abort_flag) abort_grace();
    }
  } else if (warp < kFirstEpiWarp) {
    // ------------------------------------------------------------ transform
    // Tile by tile, in the order of the stage ring: the per-row weight scale
    // (0 for a row past the layer's end; / 16 for INT4, whose codes are
    // expanded as 16 q) into its ring slot, then the INT4 expansion of the
    // staged tile into the swizzled A layout; then signal the MMA (every tile,
    // INT4 or not) and the epilogue.  Weights only: this role does not wait
    // for the previous kernel.
    const int xt = threadIdx.x - 32 * kFirstXfWarp;  // row of the 128-row block
    const int sub = xt / a.bN;
    const uint32_t g_total = cta_tiles(a);
    RingPos sr{0, 0};
    for (uint32_t g = 0; g < g_total; ++g) {
      const int st = sr.i;
      if (!__all_sync(0xffffffffu, mbar_wait(&staged[st], sr.ph, abort_flag, a.wait_ns))) {
        fail(8);
        break;
      }
      const uint32_t info = stage_info[st];
      const uint32_t is4 = info & (info >> 2) & 3u;
      const float swv = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(stage_sc + st * 256)[xt]));
      pre_sw[(g % kSwRing) * 128 + xt] = (info >> (2 + sub) & 1) ? swv * ((is4 >> sub & 1) ? 0.0625f : 1.0f) : 0.f;
      for (int sb = 0; sb < a.tpb; ++sb) {
        if (!(is4 >> sb & 1)) continue;
        const uint8_t* src = stage_g(st) + sb * a.bN * (kTileK / 2);
        uint8_t* dst = stage_a(st) + sb * a.bN * kTileK;
        for (int q = xt; q < a.bN * 4; q += 32 * kXfWarps) {  // 16-byte source chunks
          const int r8 = q >> 2, c4 = q & 3;
          // 32 nibbles -> logical 16-byte chunks 2 c4 and 2 c4 + 1 of the 128-byte row
          const uint4 v = *reinterpret_cast<const uint4*>(src + r8 * 64 + c4 * 16);
          uint8_t* drow = dst + r8 * 128;
          const uint2 e0 = expand8_x16(v.x), e1 = expand8_x16(v.y);
          *reinterpret_cast<uint4*>(drow + (((2 * c4) ^ (r8 & 7)) << 4)) = make_uint4(e0.x, e0.y, e1.x, e1.y);
          const uint2 e2 = expand8_x16(v.z), e3 = expand8_x16(v.w);
          *reinterpret_cast<uint4*>(drow + (((2 * c4 + 1) ^ (r8 & 7)) << 4)) = make_uint4(e2.x, e2.y, e3.x, e3.y);
        }
      }
      if (is4) fence_proxy_async_smem();  // generic-proxy writes -> visible to the MMA's async proxy
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&expanded[st]);
        mbar_arrive(&sw_full[g % kSwRing]);
      }
      sr.next<S_>();
    }
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int kCols = Sh::kCols;
    const int ew = warp - kFirstEpiWarp;
    const int quad = warp & 3;         // tensor-memory lane quadrant this warp may access
    const int cg = ew >> 2;            // column group
    const int row = 32 * quad + lane;  // row inside the 128-row block
    const int sub = row / a.bN;
    // Bias every accumulator buffer: an INT32 sum P accumulated onto 0x4B400000
    // reads, as an fp32 bit pattern, exactly 12582912 + P for |P| < 2^22, so one
    // fp32 subtraction converts it (no int -> float conversion instruction).
    {
      const uint32_t lane_base = tmem_base + ((uint32_t)(32 * quad) << 16) + cg * kCols;
#pragma unroll
      for (int ab = 0; ab < kBufs; ++ab)
#pragma unroll
        for (int c16 = 0; c16 < kCols / 16; ++c16) tmem_st16_const(lane_base + ab * NT + c16 * 16, kAccBias);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0)
        for (int ab = 0; ab < kBufs; ++ab) mbar_arrive(&tmem_empty[ab]);
    }
    const int et = threadIdx.x - 32 * kFirstEpiWarp;  // 0 .. 32 kEpiWarps - 1
    bool ok = true;
    pdl_wait();  // outputs, token scales and workspace may still be in use by an earlier kernel
    const float2 nbias = make_float2(-kAccBiasF, -kAccBiasF);
    uint32_t g = 0, sync_phase = 0;
    for (int u = blockIdx.x; ok && u < a.units; u += gridDim.x) {
      const Unit x = unit_of(a, u);
      const TcMember& mb = a.mem[member_of<GROUPED>(a, x.rb)];
      const int n = x.rb * 128 + row;  // row among all members' rows (split partial sums)
      const int nl = GROUPED ? (x.rb - mb.rb0) * 128 + row : n;  // output feature of this thread in its member
      const bool rvalid = nl < mb.N;
      const int mcol0 = x.tb * NT + cg * kCols;  // first token of this thread's columns
      // bias of this row and the token scales of the warp's columns, copied
      // into shared memory now and read at the end of the unit
      if constexpr (MODE != 2) {
        const bool has_b = rvalid && mb.bias != nullptr;
        cp_async4(pre_bias + et, has_b ? mb.bias + nl : a.sx, has_b ? 4u : 0u);
        for (int c = lane; c < kCols; c += 32) {
          const bool has_s = mcol0 + c < a.M;
          cp_async4(pre_sx + ew * kCols + c, has_s ? a.sx + mcol0 + c : a.sx, has_s ? 4u : 0u);
        }
        cp_async_commit();
      }
      float2 acc[kCols / 2];
#pragma unroll
      for (int i = 0; i < kCols / 2; ++i) acc[i] = make_float2(0.f, 0.f);
      for (int j = x.j0; j < x.j1;) {
        // a pair of tiles (the last one of an odd unit alone): the commit of the
        // second tile's MMAs follows the first's, so one wait covers both
        const int nt = j + 1 < x.j1 ? 2 : 1;
        const uint32_t gl = g + nt - 1;
        // the scale slot of the pair's last tile implies the first one's (the
        // transform warps arrive in tile order)
        if (!__all_sync(0xffffffffu, mbar_wait(&mma_done[gl % kDone], (gl / kDone) & 1, abort_flag, a.wait_ns) &&
                                         mbar_wait(&sw_full[gl % kSwRing], (gl / kSwRing) & 1, abort_flag, a.wait_ns))) {
          fail(9);
          ok = false;
          break;
        }
        tc_fence_after();
        // the pair's accumulators in chunks of kLdCols columns, software
        // pipelined: the load of chunk i + 1 is in flight while chunk i is
        // rescaled (tcgen05.wait::ld waits for every load issued before it, so
        // the next load is issued only after the wait for the current one)
        constexpr int kL = Sh::kLdCols, kCpt = kCols / kL;
        const uint32_t lane_base = tmem_base + ((uint32_t)(32 * quad) << 16) + cg * kCols;
        const uint32_t taddr[2] = {lane_base + (g % kBufs) * NT, lane_base + ((g + 1) % kBufs) * NT};
        float2 sw2[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const float sw = pre_sw[((g + k) % kSwRing) * 128 + row];  // slot g + 1 unused when nt == 1
          sw2[k] = make_float2(sw, sw);
        }
        uint32_t v[2][kL];
        tmem_ld16(taddr[0], v[0]);
        const int nchunks = nt * kCpt;
#pragma unroll
        for (int i = 0; i < 2 * kCpt; ++i) {
          if (i < nchunks) {
            const int k = i / kCpt, c0 = (i % kCpt) * kL;
            tmem_wait_ld();
            tmem_regs_ready(v[i & 1]);
            tmem_st16_const(taddr[k] + c0, kAccBias);  // re-bias for the buffer's next use
            if (i + 1 < nchunks) tmem_ld16(taddr[(i + 1) / kCpt] + ((i + 1) % kCpt) * kL, v[(i + 1) & 1]);
            if constexpr (MODE == 2) {
              // INT4 label read back from the bitmap (debug path only)
              const int tt = (n / a.bN) * a.C + j + k;
              const bool t4 = rvalid && ((__ldg(mb.bitmap + (tt >> 3)) >> (tt & 7)) & 1);
#pragma unroll
              for (int e = 0; e < kL; ++e) {
                const int m = mcol0 + c0 + e;
                if (rvalid && m < a.M) {
                  const int p16 = (int)(v[i & 1][e] - kAccBias);
                  a.P[((size_t)m * a.N + n) * a.C + j + k] = t4 ? (p16 >> 4) : p16;
                }
              }
            } else {
#pragma unroll
              for (int e = 0; e < kL / 2; ++e) {
                const float2 p =
                    __fadd2_rn(make_float2(__uint_as_float(v[i & 1][2 * e]), __uint_as_float(v[i & 1][2 * e + 1])), nbias);
                acc[c0 / 2 + e] = __ffma2_rn(p, sw2[k], acc[c0 / 2 + e]);
              }
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&tmem_empty[g % kBufs]);
          if (nt == 2) mbar_arrive(&tmem_empty[gl % kBufs]);
        }
        g += nt;
        j += nt;
      }
      if (!ok || MODE == 2) continue;
      cp_async_wait_all();
      __syncwarp();  // the token scales were copied by all lanes of the warp
      const float bias_n = pre_bias[et];
      if constexpr (MODE == 0) {
        const float4* sxv = reinterpret_cast<const float4*>(pre_sx + ew * kCols);
        const int mlim = a.M - mcol0;  // columns of this thread that exist
        if (rvalid && a.ydtype == AQ_F32) {
          float* yp = reinterpret_cast<float*>(mb.y) + (size_t)mcol0 * mb.ldy + nl;
#pragma unroll
          for (int i4 = 0; i4 < kCols / 4; ++i4) {
            const float4 s4 = sxv[i4];
            const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int i = 4 * i4 + k;
              if (i < mlim) yp[(size_t)i * mb.ldy] = fmaf(sv[k], i & 1 ? acc[i / 2].y : acc[i / 2].x, bias_n);
            }
          }
        } else if (rvalid) {
          __nv_bfloat16* yp = reinterpret_cast<__nv_bfloat16*>(mb.y) + (size_t)mcol0 * mb.ldy + nl;
#pragma unroll
          for (int i4 = 0; i4 < kCols / 4; ++i4) {
            const float4 s4 = sxv[i4];
            const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int i = 4 * i4 + k;
              if (i < mlim)
                yp[(size_t)i * mb.ldy] = __float2bfloat16_rn(fmaf(sv[k], i & 1 ? acc[i / 2].y : acc[i / 2].x, bias_n));
            }
          }
        }
        __syncwarp();  // the scale slots are rewritten at the next unit's start
        continue;
      }
      // split-K: publish the partial sum, the last CTA of this unit group reduces.
      // Partials are [S][N][Mp] (Mp = M rounded up to 4): a thread's columns
      // are contiguous, written and read as 16-byte vectors.
      const int Mp = (a.M + 3) & ~3;
      float* const prow = a.partial + (size_t)n * Mp + mcol0;  // this thread's split-0 columns
      const size_t sstride = (size_t)a.N * Mp;
      if (rvalid) {
#pragma unroll
        for (int i4 = 0; i4 < kCols / 4; ++i4)
          if (mcol0 + 4 * i4 < a.M)
            __stcg(reinterpret_cast<float4*>(prow + x.s * sstride) + i4,
                   make_float4(acc[2 * i4].x, acc[2 * i4].y, acc[2 * i4 + 1].x, acc[2 * i4 + 1].y));
      }
      __threadfence();
      mbar_arrive(epi_sync);
      if (!__all_sync(0xffffffffu, mbar_wait(epi_sync, sync_phase, abort_flag, a.wait_ns))) { fail(11); ok = false; continue; }
      sync_phase ^= 1;
      if (ew == 0 && lane == 0) *last_flag = (atomicAdd(a.counters + x.rb * a.ntb + x.tb, 1) == a.S - 1);
      mbar_arrive(epi_sync);
      if (!__all_sync(0xffffffffu, mbar_wait(epi_sync, sync_phase, abort_flag, a.wait_ns))) { fail(12); ok = false; continue; }
      sync_phase ^= 1;
      if (*last_flag) {
        __threadfence();
        if (rvalid) {
          // the loads of every split for a chunk of columns are issued before any
          // of them is summed, then the splits are added in increasing order;
          // chunks are as wide as 64 values in flight allow
          if (a.S <= 2) reduce_splits<kCols, chunk_cols(kCols, 32), 2>(a, mb, prow, sstride, mcol0, nl, bias_n);
          else if (a.S <= 4) reduce_splits<kCols, chunk_cols(kCols, 16), 4>(a, mb, prow, sstride, mcol0, nl, bias_n);
          else reduce_splits<kCols, chunk_cols(kCols, 8), kMaxTcSplits>(a, mb, prow, sstride, mcol0, nl, bias_n);
        }
        if (ew == 0 && lane == 0) a.counters[x.rb * a.ntb + x.tb] = 0;
      }
    }
    cp_async_wait_all();  // no copy into shared memory outlives the CTA (abort path)
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Sh::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D uint8 tensor map: `rows` rows of `cols` bytes, box (box_cols x box_rows).
bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
              bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NT, int MODE, bool GROUPED = false>
cudaError_t launch_nt(const aq_packed* const* w, const int8_t* xq, const TcArgs& a, int grid, cudaStream_t st) {
  using Sh = TcShape<NT>;
  cudaError_t e = ensure_smem_attr<tc_linear_kernel<NT, MODE, GROUPED>>(Sh::kSmemBytes);
  if (e != cudaSuccess) return e;
  TcMaps maps;
  memset(&maps, 0, sizeof(maps));
  for (int g = 0; g < a.G; ++g) {
    if (w[g]->T8 > 0 && !make_map(&maps.w8[g], w[g]->w8, kTileK, (uint64_t)w[g]->T8 * w[g]->bN, kTileK, w[g]->bN, true))
      return cudaErrorInvalidValue;
    if (w[g]->T4 > 0 &&
        !make_map(&maps.w4[g], w[g]->w4, kTileK / 2, (uint64_t)w[g]->T4 * w[g]->bN, kTileK / 2, w[g]->bN, false))
      return cudaErrorInvalidValue;
  }
  if (!make_map(&maps.x, xq, w[0]->K, a.M, kTileK, NT, true)) return cudaErrorInvalidValue;
  return launch_pdl(tc_linear_kernel<NT, MODE, GROUPED>, dim3(grid), dim3(Sh::kThreads), (size_t)Sh::kSmemBytes, st,
                    maps, a);
}

}  // namespace

// G members share K and bN; with G > 1 every member's rows are a multiple of 128.
static cudaError_t launch_tc_impl(const aq_packed* const* w, int G, const float* const* bias, void* const* y,
                                  const int* ldy, const int8_t* xq, const float* sx, int M, int ydtype, void* ws,
                                  int32_t* P, int phase, unsigned long long wait_ns, int stop_after, cudaStream_t st) {
  if (G < 1 || G > kMaxGroup || (P != nullptr && G != 1)) return cudaErrorInvalidValue;
  TcArgs a;
  memset(&a, 0, sizeof(a));
  a.wait_ns = wait_ns;
  a.stop_after = stop_after;
  a.G = G;
  a.K = w[0]->K; a.bN = w[0]->bN; a.C = w[0]->C;
  a.tpb = 128 / a.bN;
  int rb = 0;
  for (int g = 0; g < G; ++g) {
    if (w[g]->K != a.K || w[g]->bN != a.bN || (G > 1 && w[g]->N % 128 != 0)) return cudaErrorInvalidValue;
    TcMember& m = a.mem[g];
    m.bitmap = w[g]->bitmap; m.tile_idx = w[g]->tile_idx; m.scales = w[g]->scales;
    m.bias = bias ? bias[g] : nullptr; m.y = y ? y[g] : nullptr; m.ldy = ldy ? ldy[g] : w[g]->N;
    m.N = w[g]->N; m.R = w[g]->R; m.T4 = w[g]->T4; m.T8 = w[g]->T8;
    m.rb0 = rb;
    rb += (w[g]->R + a.tpb - 1) / a.tpb;
  }
  a.nrb = rb;
  a.N = G == 1 ? w[0]->N : rb * 128;
  a.M = M;
  a.sx = sx; a.ydtype = ydtype;
  a.ws = ws;
  a.P = P;
  char* wsb = static_cast<char*>(ws);
  a.counters = reinterpret_cast<int*>(wsb + kWsHeader);

  // token-block width: up to 64 tokens in one block of 16-multiples; beyond,
  // 128 or 96 tokens, whichever leaves the shorter estimated makespan: whole
  // units go to the CTAs in waves, and a 96-token tile costs about
  // (128 + 96) / (128 + 128) of a 128-token one (half of a tile's time is
  // fixed per tile), so 96 wins where it removes a mostly idle last wave
  // (e.g. 2560 output features at 2048 tokens: 440 units in 3 waves instead
  // of 320 in 3)
  const int sms = num_sms();
  int nt = M <= 64 ? (M + 15) / 16 * 16 : 128;
  if (M > 64) {
    auto cost = [&](int t) {
      const long long units = (long long)a.nrb * ((M + t - 1) / t);
      return ((units + sms - 1) / sms) * (128 + t);
    };
    if (cost(96) < cost(128)) nt = 96;
  }
  a.ntb = (M + nt - 1) / nt;
  if (phase == AQ_PHASE_DECODE && P == nullptr) {
    const DecodePlan p = plan_tc_decode(M, a.nrb, a.C);
    a.S = p.S;
    if (a.S > kMaxTcSplits) return cudaErrorInvalidValue;  // the split reduction unrolls over kMaxTcSplits
    const size_t cnt_bytes = ((size_t)p.blocks * sizeof(int) + 255) / 256 * 256;
    a.partial = reinterpret_cast<float*>(wsb + kWsHeader + cnt_bytes);
    a.ws_clear = a.S > 1 ? (int)cnt_bytes : 0;
  } else {
    a.S = 1;
    a.partial = nullptr;
    a.ws_clear = 0;
  }
  a.units = a.nrb * a.ntb * a.S;
  const int grid = std::min(a.units, sms);
  const int mode = P ? 2 : (a.S > 1 ? 1 : 0);
  if (G > 1) {  // grouped launches: decode only (at most 64 tokens)
    if (phase != AQ_PHASE_DECODE || P != nullptr) return cudaErrorInvalidValue;
    switch (nt * 4 + mode) {
#define AQ_TC_CASE_G(NTV)                                                      \
  case NTV * 4 + 0: return launch_nt<NTV, 0, true>(w, xq, a, grid, st);      \
  case NTV * 4 + 1: return launch_nt<NTV, 1, true>(w, xq, a, grid, st);
      AQ_TC_CASE_G(16)
      AQ_TC_CASE_G(32)
      AQ_TC_CASE_G(48)
      AQ_TC_CASE_G(64)
#undef AQ_TC_CASE_G
      default: return cudaErrorInvalidValue;
    }
  }
  switch (nt * 4 + mode) {
#define AQ_TC_CASE(NTV)                                                  \
  case NTV * 4 + 0: return launch_nt<NTV, 0>(w, xq, a, grid, st);      \
  case NTV * 4 + 1: return launch_nt<NTV, 1>(w, xq, a, grid, st);      \
  case NTV * 4 + 2: return launch_nt<NTV, 2>(w, xq, a, grid, st);
    AQ_TC_CASE(16)
    AQ_TC_CASE(32)
    AQ_TC_CASE(48)
    AQ_TC_CASE(64)
#undef AQ_TC_CASE
// more than 64 tokens: prefill only, never split
#define AQ_TC_CASE_WIDE(NTV)                                             \
  case NTV * 4 + 0: return launch_nt<NTV, 0>(w, xq, a, grid, st);      \
  case NTV * 4 + 2: return launch_nt<NTV, 2>(w, xq, a, grid, st);
    AQ_TC_CASE_WIDE(96)
    AQ_TC_CASE_WIDE(128)
#undef AQ_TC_CASE_WIDE
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_tc(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias, void* y,
                      int ydtype, int ldy, void* ws, int32_t* P, int phase, cudaStream_t st) {
  return launch_tc_impl(&w, 1, &bias, &y, &ldy, xq, sx, M, ydtype, ws, P, phase, kWaitTimeoutNs, -1, st);
}

cudaError_t launch_tc_group(const aq_packed* const* w, int G, const float* const* bias, void* const* y,
                            const int* ldy, const int8_t* xq, const float* sx, int M, int ydtype, void* ws, int phase,
                            cudaStream_t st) {
  return launch_tc_impl(w, G, bias, y, ldy, xq, sx, M, ydtype, ws, nullptr, phase, kWaitTimeoutNs, -1, st);
}

cudaError_t launch_tc_stalled(const aq_packed* w, const int8_t* xq, const float* sx, int M, void* y, int ldy,
                              void* ws, int phase, unsigned long long wait_ns, int stop_after, cudaStream_t st) {
  void* yy = y;
  return launch_tc_impl(&w, 1, nullptr, &yy, &ldy, xq, sx, M, AQ_F32, ws, nullptr, phase, wait_ns, stop_after, st);
}

}  // namespace aq
