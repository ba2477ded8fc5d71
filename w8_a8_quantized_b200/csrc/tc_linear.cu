// Mixed W4/W8 x A8 linear layer on the 5th-generation tensor cores (tcgen05).
//
// AlignQuant, Sec. 3.3 ("Integer operand preparation", "Prefill weight reuse",
// "Output reconstruction") and App. E.3 eq. 19: packed tiles are moved on
// chip, INT4 tiles are sign-extended to INT8 on chip, every tile product is
// an exact INT32 sum, and each is rescaled by its activation and weight
// scales before FP32 accumulation over the input tiles.
//
// Roles in one CTA (persistent over work units):
//   warp 0      TMA producer: INT8 tiles -> swizzled A stage, INT4 tiles ->
//               staging buffer, activation tile -> B stage.
//   warp 1      allocates tensor memory; one lane issues tcgen05.mma
//               (kind::i8, M = 128 weight rows, N = NT tokens, K = 32) four
//               times per 128-wide input tile into a double-buffered INT32
//               accumulator in tensor memory.
//   warps 2-3   expand INT4 staging tiles into the 128-byte-swizzled INT8
//               A layout (fence.proxy.async before signalling the MMA).
//   warps 4..   epilogue: after every input tile, read the INT32 tile product
//               from tensor memory, multiply by the row's fp16 weight scale of
//               that tile and accumulate in FP32 registers; at the end of a
//               work unit multiply by the token scale, add bias and store.
// Weights are the A operand, so TMEM lane = output row and each epilogue
// thread applies ONE weight scale per input tile.
//
// A work unit is (128-row block of output features, NT-token block, split of
// the input tiles).  Split partial sums go to the workspace; the CTA that
// finishes a unit last sums all splits in increasing split order.
// Every mbarrier wait is bounded (see mbar_wait); a wait that gives up records
// AQ_ERR_TIMEOUT in the workspace, raises a CTA-wide abort flag, drains the
// copies and MMAs it issued, and the CTA frees its tensor memory and exits.
#include <algorithm>
#include <cstring>

#include "aq_internal.cuh"

namespace aq {
namespace {

template <int NT>
struct TcShape {
  static constexpr int kA = 128 * kTileK;        // swizzled INT8 weight block
  static constexpr int kStg = 128 * kTileK / 2;  // INT4 staging (row-major, 64 B per row)
  static constexpr int kB = NT * kTileK;         // swizzled INT8 activation block
  static constexpr int kStageBytes = kA + kB + kStg;
  static constexpr int kStages = NT >= 256 ? 3 : (NT >= 128 ? 4 : 6);
  static constexpr int kEpiWarps = NT > 64 ? 4 * (NT / 64) : 4;  // 4 warps (one per lane quadrant) per 64 columns
  static constexpr int kCols = NT / (kEpiWarps / 4);             // accumulator columns per epilogue thread (<= 64)
  static constexpr int kThreads = 128 + 32 * kEpiWarps;
  static constexpr int kTmemCols = 2 * NT <= 32 ? 32 : 2 * NT <= 64 ? 64 : 2 * NT <= 128 ? 128 : 2 * NT <= 256 ? 256 : 512;
  static constexpr int kBufStride = kTmemCols / 2;  // column offset of accumulator buffer 1
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kBarBytes;
  static constexpr uint32_t kIdesc = idesc_i8(128, NT);
  static_assert(NT % 16 == 0 && NT >= 16 && NT <= 256, "MMA N");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert((4 * kStages + 5) * 8 + 16 <= kBarBytes, "barrier area");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

constexpr uint32_t kAccBias = 0x4B400000u;  // fp32 bit pattern of 12582912 = 1.5 * 2^23
constexpr float kAccBiasF = 12582912.0f;

struct TcArgs {
  const uint8_t* bitmap;
  const int32_t* tile_idx;
  const uint16_t* scales;
  int N, K, bN, R, C, T4, T8;
  int tpb;     // tile rows per 128-row block (1 for bN = 128, 2 for bN = 64)
  int nrb;     // number of 128-row blocks
  int M, ntb;  // tokens, token blocks
  int S, units;
  const float* sx;
  const float* bias;
  void* y;
  int ydtype, ldy;
  void* ws;
  float* partial;  // [S][M][N]
  int* counters;   // [nrb * ntb]
  int32_t* P;      // debug: exact tile products [M][N][C], or null
};

struct Unit {
  int rb, tb, s, j0, j1;
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

// INT4 label mask (bit sub) and validity mask of the sub-tiles of one input tile.
__device__ __forceinline__ void tile_kinds(const TcArgs& a, int rb, int j, int& valid, int& is4) {
  valid = 0;
  is4 = 0;
  for (int sub = 0; sub < a.tpb; ++sub) {
    const int r = rb * a.tpb + sub;
    if (r < a.R) {
      valid |= 1 << sub;
      const int t = r * a.C + j;
      if ((__ldg(a.bitmap + (t >> 3)) >> (t & 7)) & 1) is4 |= 1 << sub;
    }
  }
}

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

// MODE: 0 = outputs written directly (one split), 1 = split-K partial sums
// reduced by the last CTA of each unit group, 2 = exact tile products only.
template <int NT, int MODE>
__global__ void __launch_bounds__(TcShape<NT>::kThreads, 1)
    tc_linear_kernel(const __grid_constant__ CUtensorMap tm_w8, const __grid_constant__ CUtensorMap tm_w4,
                     const __grid_constant__ CUtensorMap tm_x, const TcArgs a) {
  using Sh = TcShape<NT>;
  constexpr int S_ = Sh::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  auto stage_a = [&](int st) { return smem + st * Sh::kStageBytes; };
  auto stage_b = [&](int st) { return smem + st * Sh::kStageBytes + Sh::kA; };
  auto stage_g = [&](int st) { return smem + st * Sh::kStageBytes + Sh::kA + Sh::kB; };
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S_ * Sh::kStageBytes);
  uint64_t* full = bars;
  uint64_t* staged = bars + S_;
  uint64_t* expanded = bars + 2 * S_;
  uint64_t* empty = bars + 3 * S_;
  uint64_t* tmem_full = bars + 4 * S_;
  uint64_t* tmem_empty = bars + 4 * S_ + 2;
  uint64_t* epi_sync = bars + 4 * S_ + 4;  // epilogue-only rendezvous (bounded, unlike bar.sync)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * S_ + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* never_flag = reinterpret_cast<volatile int*>(tmem_slot + 3);  // stays 0: drain waits

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < S_; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&staged[st], 1);
      mbar_init(&expanded[st], 64);
      mbar_init(&empty[st], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tmem_full[b], 1);
      mbar_init(&tmem_empty[b], 32 * Sh::kEpiWarps);
    }
    mbar_init(epi_sync, 32 * Sh::kEpiWarps);
    *abort_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_x);
    if (a.T8 > 0) prefetch_tmap(&tm_w8);
    if (a.T4 > 0) prefetch_tmap(&tm_w4);
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
    record_error(a.ws, AQ_ERR_TIMEOUT, info);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      pdl_wait();  // activations come from an earlier kernel
      uint32_t g = 0, stg_bits = 0, stg_used = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < a.units; u += gridDim.x) {
        const Unit x = unit_of(a, u);
        for (int j = x.j0; j < x.j1; ++j, ++g) {
          const int st = g % S_;
          const uint32_t use = g / S_;
          if (!mbar_wait(&empty[st], (use & 1) ^ 1, abort_flag)) { fail(1); ok = false; break; }
          int valid, is4;
          tile_kinds(a, x.rb, j, valid, is4);
          uint32_t bytes_full = Sh::kB, bytes_stg = 0;
          for (int sub = 0; sub < a.tpb; ++sub)
            if (valid >> sub & 1) {
              if (is4 >> sub & 1) bytes_stg += a.bN * (kTileK / 2);
              else bytes_full += a.bN * kTileK;
            }
          mbar_arrive_expect_tx(&full[st], bytes_full);
          if (bytes_stg) {
            mbar_arrive_expect_tx(&staged[st], bytes_stg);
            stg_bits ^= 1u << st;
            stg_used |= 1u << st;
          }
          for (int sub = 0; sub < a.tpb; ++sub) {
            if (!(valid >> sub & 1)) continue;
            const int t = (x.rb * a.tpb + sub) * a.C + j;
            const int row = __ldg(a.tile_idx + t) * a.bN;
            if (is4 >> sub & 1)
              tma_load_2d(stage_g(st) + sub * a.bN * (kTileK / 2), &tm_w4, 0, row, &staged[st]);
            else
              tma_load_2d(stage_a(st) + sub * a.bN * kTileK, &tm_w8, 0, row, &full[st]);
          }
          tma_load_2d(stage_b(st), &tm_x, j * kTileK, x.tb * NT, &full[st]);
        }
      }
      if (!ok) {
        // let every copy already issued land before the CTA's memory goes away
        for (int st = 0; st < S_ && (uint32_t)st < g; ++st) {
          const uint32_t last = (g - 1 - st) / S_;  // last use of stage st
          mbar_wait(&full[st], last & 1, never_flag);
          if (stg_used >> st & 1) mbar_wait(&staged[st], ((stg_bits >> st) & 1) ^ 1, never_flag);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t g = 0, kt = 0, exp_bits = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < a.units; u += gridDim.x) {
        const Unit x = unit_of(a, u);
        for (int j = x.j0; j < x.j1; ++j, ++g, ++kt) {
          const int st = g % S_;
          if (!mbar_wait(&full[st], (g / S_) & 1, abort_flag)) { fail(2); ok = false; break; }
          int valid, is4;
          tile_kinds(a, x.rb, j, valid, is4);
          if (is4) {
            if (!mbar_wait(&expanded[st], (exp_bits >> st) & 1, abort_flag)) { fail(3); ok = false; break; }
            exp_bits ^= 1u << st;
          }
          const int ab = kt & 1;  // use kt >> 1 of this buffer waits for the epilogue's release number kt >> 1
          if (!mbar_wait(&tmem_empty[ab], (kt >> 1) & 1, abort_flag)) { fail(4); ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sw128_desc(smem_u32(stage_a(st)));
          const uint64_t bdesc = sw128_desc(smem_u32(stage_b(st)));
          const uint32_t d = tmem_base + ab * Sh::kBufStride;
          // the buffer holds the bias kAccBias in every element; all four MMAs accumulate onto it
#pragma unroll
          for (int k = 0; k < kTileK / 32; ++k)  // K = 32 bytes per instruction: +2 in 16-byte units
            mma_i8(d, adesc + 2 * k, bdesc + 2 * k, Sh::kIdesc, 1u);
          mma_commit(&empty[st]);
          mma_commit(&tmem_full[ab]);
        }
      }
      if (!ok && kt > 0) {  // drain the MMAs issued so far
        const uint32_t last = kt - 1;
        mbar_wait(&tmem_full[last & 1], (last >> 1) & 1, never_flag);
      }
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ INT4 expanders
    const int et = threadIdx.x - 64;  // 0..63
    uint32_t g = 0, stg_bits = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < a.units; u += gridDim.x) {
      const Unit x = unit_of(a, u);
      for (int j = x.j0; j < x.j1; ++j, ++g) {
        int valid, is4;
        tile_kinds(a, x.rb, j, valid, is4);
        if (!is4) continue;
        const int st = g % S_;
        if (!mbar_wait(&staged[st], (stg_bits >> st) & 1, abort_flag)) { fail(5); ok = false; break; }
        stg_bits ^= 1u << st;
        for (int sub = 0; sub < a.tpb; ++sub) {
          if (!(is4 >> sub & 1)) continue;
          const uint8_t* src = stage_g(st) + sub * a.bN * (kTileK / 2);
          uint8_t* dst = stage_a(st) + sub * a.bN * kTileK;
          for (int q = et; q < a.bN * 4; q += 64) {  // 16-byte source chunks
            const int n = q >> 2, c4 = q & 3;
            const uint4 v = *reinterpret_cast<const uint4*>(src + n * 64 + c4 * 16);
            const uint2 e0 = expand8_x16(v.x), e1 = expand8_x16(v.y), e2 = expand8_x16(v.z), e3 = expand8_x16(v.w);
            const int kc0 = 2 * c4, kc1 = 2 * c4 + 1;  // logical 16-byte chunks of the 128-byte row
            *reinterpret_cast<uint4*>(dst + n * 128 + ((kc0 ^ (n & 7)) << 4)) = make_uint4(e0.x, e0.y, e1.x, e1.y);
            *reinterpret_cast<uint4*>(dst + n * 128 + ((kc1 ^ (n & 7)) << 4)) = make_uint4(e2.x, e2.y, e3.x, e3.y);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&expanded[st]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int kCols = Sh::kCols;
    const int ew = warp - 4;
    const int quad = warp & 3;       // tensor-memory lane quadrant this warp may access
    const int cg = ew >> 2;          // column group
    const int row = 32 * quad + lane;  // row inside the 128-row block
    const int sub = row / a.bN, nl = row % a.bN;
    pdl_wait();  // outputs and workspace may still be in use by an earlier kernel
    // Bias both accumulator buffers: an INT32 sum P accumulated onto 0x4B400000
    // reads, as an fp32 bit pattern, exactly 12582912 + P for |P| < 2^22, so one
    // fp32 subtraction converts it (no int -> float conversion instruction).
    {
      const uint32_t lane_base = tmem_base + ((uint32_t)(32 * quad) << 16) + cg * Sh::kCols;
#pragma unroll
      for (int ab = 0; ab < 2; ++ab)
#pragma unroll
        for (int c16 = 0; c16 < Sh::kCols / 16; ++c16) tmem_st16_const(lane_base + ab * Sh::kBufStride + c16 * 16, kAccBias);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&tmem_empty[0]);
      mbar_arrive(&tmem_empty[1]);
    }
    uint32_t kt = 0, sync_phase = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < a.units; u += gridDim.x) {
      const Unit x = unit_of(a, u);
      const int r = x.rb * a.tpb + sub;
      const bool rvalid = r < a.R;
      const int n = r * a.bN + nl;
      const int mcol0 = x.tb * NT + cg * kCols;  // first token of this thread's columns
      float acc[kCols];
#pragma unroll
      for (int i = 0; i < kCols; ++i) acc[i] = 0.f;
      // tile scale and kind of the next input tile are loaded one tile ahead
      auto load_scale = [&](int j, uint32_t& swb, uint32_t& lab) {
        if (rvalid) {
          const int tt = r * a.C + j;
          swb = __ldg(a.scales + (size_t)tt * a.bN + nl);
          lab = __ldg(a.bitmap + (tt >> 3)) >> (tt & 7);
        }
      };
      uint32_t swb_next = 0, lab_next = 0;
      load_scale(x.j0, swb_next, lab_next);
      for (int j = x.j0; j < x.j1; ++j, ++kt) {
        const int ab = kt & 1;
        const uint32_t swb = swb_next, lab = lab_next;
        if (j + 1 < x.j1) load_scale(j + 1, swb_next, lab_next);
        // INT4 tiles were multiplied by 16 during expansion
        const bool t4 = rvalid && (lab & 1);
        const float sw = rvalid ? __half2float(__ushort_as_half((unsigned short)swb)) * (t4 ? 0.0625f : 1.0f) : 0.f;
        // warp-uniform outcome: the tensor-memory loads below are warp-collective
        if (!__all_sync(0xffffffffu, mbar_wait(&tmem_full[ab], (kt >> 1) & 1, abort_flag))) {
          fail(6);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(32 * quad) << 16) + ab * Sh::kBufStride + cg * kCols;
#pragma unroll
        for (int c16 = 0; c16 < kCols / 16; ++c16) {
          uint32_t v[16];
          tmem_ld16(taddr + c16 * 16, v);
          tmem_wait_ld();
          tmem_st16_const(taddr + c16 * 16, kAccBias);  // re-bias for the buffer's next use
          if constexpr (MODE == 2) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int m = mcol0 + c16 * 16 + i;
              if (rvalid && m < a.M) {
                const int p16 = (int)(v[i] - kAccBias);
                a.P[((size_t)m * a.N + n) * a.C + j] = t4 ? (p16 >> 4) : p16;
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              acc[c16 * 16 + i] = fmaf(__uint_as_float(v[i]) - kAccBiasF, sw, acc[c16 * 16 + i]);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&tmem_empty[ab]);
      }
      if (!ok || MODE == 2) continue;
      if constexpr (MODE == 0) {
        if (rvalid) {
          const float b = a.bias ? __ldg(a.bias + n) : 0.f;
#pragma unroll
          for (int i = 0; i < kCols; ++i) {
            const int m = mcol0 + i;
            if (m < a.M) store_y(a.y, a.ydtype, (size_t)m * a.ldy + n, fmaf(__ldg(a.sx + m), acc[i], b));
          }
        }
        continue;
      }
      // split-K: publish the partial sum, the last CTA of this unit group reduces
      if (rvalid) {
#pragma unroll
        for (int i = 0; i < kCols; ++i) {
          const int m = mcol0 + i;
          if (m < a.M) __stcg(a.partial + ((size_t)x.s * a.M + m) * a.N + n, acc[i]);
        }
      }
      __threadfence();
      mbar_arrive(epi_sync);
      if (!__all_sync(0xffffffffu, mbar_wait(epi_sync, sync_phase, abort_flag))) { fail(7); ok = false; continue; }
      sync_phase ^= 1;
      if (ew == 0 && lane == 0) *last_flag = (atomicAdd(a.counters + x.rb * a.ntb + x.tb, 1) == a.S - 1);
      mbar_arrive(epi_sync);
      if (!__all_sync(0xffffffffu, mbar_wait(epi_sync, sync_phase, abort_flag))) { fail(8); ok = false; continue; }
      sync_phase ^= 1;
      if (*last_flag) {
        __threadfence();
        if (rvalid) {
          const float b = a.bias ? __ldg(a.bias + n) : 0.f;
          for (int i = 0; i < kCols; ++i) {
            const int m = mcol0 + i;
            if (m >= a.M) break;
            float sum = 0.f;
            for (int ss = 0; ss < a.S; ++ss) sum += __ldcg(a.partial + ((size_t)ss * a.M + m) * a.N + n);
            store_y(a.y, a.ydtype, (size_t)m * a.ldy + n, fmaf(__ldg(a.sx + m), sum, b));
          }
        }
        if (ew == 0 && lane == 0) a.counters[x.rb * a.ntb + x.tb] = 0;
      }
    }
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

template <int NT, int MODE>
cudaError_t launch_nt(const aq_packed* w, const int8_t* xq, TcArgs a, int grid, cudaStream_t st) {
  using Sh = TcShape<NT>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(tc_linear_kernel<NT, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Sh::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  CUtensorMap m8, m4, mx;
  memset(&m8, 0, sizeof(m8));
  memset(&m4, 0, sizeof(m4));
  if (w->T8 > 0 && !make_map(&m8, w->w8, kTileK, (uint64_t)w->T8 * w->bN, kTileK, w->bN, true))
    return cudaErrorInvalidValue;
  if (w->T4 > 0 && !make_map(&m4, w->w4, kTileK / 2, (uint64_t)w->T4 * w->bN, kTileK / 2, w->bN, false))
    return cudaErrorInvalidValue;
  if (!make_map(&mx, xq, w->K, a.M, kTileK, NT, true)) return cudaErrorInvalidValue;
  return launch_pdl(tc_linear_kernel<NT, MODE>, dim3(grid), dim3(Sh::kThreads), (size_t)Sh::kSmemBytes, st, m8, m4, mx, a);
}

}  // namespace

cudaError_t launch_tc(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias, void* y,
                      int ydtype, int ldy, void* ws, int32_t* P, int phase, cudaStream_t st) {
  TcArgs a;
  a.bitmap = w->bitmap; a.tile_idx = w->tile_idx; a.scales = w->scales;
  a.N = w->N; a.K = w->K; a.bN = w->bN; a.R = w->R; a.C = w->C; a.T4 = w->T4; a.T8 = w->T8;
  a.tpb = 128 / w->bN;
  a.nrb = (w->R + a.tpb - 1) / a.tpb;
  a.M = M;
  a.sx = sx; a.bias = bias; a.y = y; a.ydtype = ydtype; a.ldy = ldy;
  a.ws = ws;
  a.P = P;
  char* wsb = static_cast<char*>(ws);
  a.counters = reinterpret_cast<int*>(wsb + kWsHeader);

  int nt;
  if (phase == AQ_PHASE_DECODE || M <= 64) nt = (M + 15) / 16 * 16;
  else if (M <= 128) nt = 128;
  else nt = 256;
  if (nt > 64 && nt < 128) nt = 128;
  a.ntb = (M + nt - 1) / nt;
  if (phase == AQ_PHASE_DECODE && P == nullptr) {
    const DecodePlan p = plan_decode(M, w);
    a.S = p.S;
    const size_t cnt_bytes = ((size_t)p.blocks * sizeof(int) + 255) / 256 * 256;
    a.partial = reinterpret_cast<float*>(wsb + kWsHeader + cnt_bytes);
  } else {
    a.S = 1;
    a.partial = nullptr;
  }
  a.units = a.nrb * a.ntb * a.S;
  const int grid = std::min(a.units, kNumSMs);
  const int mode = P ? 2 : (a.S > 1 ? 1 : 0);
  switch (nt * 4 + mode) {
#define AQ_TC_CASE(NTV)                                                  \
  case NTV * 4 + 0: return launch_nt<NTV, 0>(w, xq, a, grid, st);      \
  case NTV * 4 + 1: return launch_nt<NTV, 1>(w, xq, a, grid, st);      \
  case NTV * 4 + 2: return launch_nt<NTV, 2>(w, xq, a, grid, st);
    AQ_TC_CASE(16)
    AQ_TC_CASE(32)
    AQ_TC_CASE(48)
    AQ_TC_CASE(64)
    AQ_TC_CASE(128)
    case 256 * 4 + 0: return launch_nt<256, 0>(w, xq, a, grid, st);
    case 256 * 4 + 2: return launch_nt<256, 2>(w, xq, a, grid, st);
#undef AQ_TC_CASE
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace aq
