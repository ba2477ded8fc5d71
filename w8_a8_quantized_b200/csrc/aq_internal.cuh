// Internal declarations shared by the libaq translation units: workspace
// layout, launch helpers and the inline-PTX wrappers (mbarrier, TMA, tcgen05)
// used by the sm_100a kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "../../include/aq.h"

namespace aq {

// ---------------------------------------------------------------- geometry
constexpr int kTileK = 128;          // bK: the only supported input-tile width
constexpr int kMaxDecodeM = 64;
constexpr int kMaxDevices = 64;      // per-device host caches

// Streaming multiprocessors of the current device (cached per device; 148 on a
// B200, also the answer when no device can be queried, e.g. for host-only
// sizing calls on a machine without a GPU).  Sizes grids and split counts.
int num_sms();

// Workspace layout.  The first 256 bytes hold the error word; split-K
// counters and fp32 partial sums follow.
constexpr size_t kWsHeader = 256;
struct WsHeader {
  int err_code;   // 0 or AQ_ERR_TIMEOUT
  int err_info;   // which wait gave up (kernel-specific code)
  int err_clear;  // bytes after the header (split-K counters) to zero again after an error
};

// Bounded waits: any spin on an mbarrier gives up after this long, records
// AQ_ERR_TIMEOUT in the workspace and lets the kernel wind down.
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s

inline bool geometry_ok(int N, int K, int bN, int bK) {
  return N > 0 && K > 0 && (bN == 64 || bN == 128) && bK == kTileK && N % bN == 0 && K % bK == 0 &&
         (long long)N * K < (1ll << 40);
}
// The paper-exact mode's tiles: 64 input columns (the activation group width).
constexpr int kPaperTileK = 64;
// b_M of App. B.3: activation rows per scale group (1 for a single row, else 16).
int act_group_rows(int M);
inline bool paper_geometry_ok(int N, int K, int bN, int bK) {
  return N > 0 && K > 0 && (bN == 64 || bN == 128) && bK == kPaperTileK && N % bN == 0 && K % bK == 0 &&
         (long long)N * K < (1ll << 40);
}

int validate_packed(const aq_packed* w);  // AQ_OK or an error status

// One projection as seen by the CUDA-core decode kernel (a group of up to
// kMaxGroup projections sharing one input runs as a single launch).
constexpr int kMaxGroup = 3;
constexpr int kRowsPerCta = 32;                // output rows per CTA of the CUDA-core decode kernel
constexpr int kRowsMaxM = 8;                   // tokens handled by the CUDA-core decode kernel
constexpr size_t kFusedMaxBytes = 64 * 1024;   // shared memory for fused activation codes
struct DecodeProj {
  const uint8_t* bitmap;
  const int32_t* tile_idx;
  const uint8_t* w4;
  const int8_t* w8;
  const uint16_t* scales;
  const float* bias;
  void* y;
  int N, bN, ldy, blocks;
};
DecodeProj decode_proj(const aq_packed* w, const float* bias, void* y, int ldy);
bool rows_supported(int M, int K);
bool rows_fusable(int M, int K);
cudaError_t launch_decode_rows(const DecodeProj* projs, int G, int K, const uint16_t* x, int ldx, const int8_t* xq,
                               const float* sx, int M, int ydtype, int32_t* P, void* ws,
                               cudaStream_t st);
// The streaming decode kernel (1-2 tokens; same arguments).  stream_supported: whether its shared memory fits a launch over
// `rows` concatenated output rows.
bool stream_supported(int M, int K, int rows);
cudaError_t launch_decode_stream(const DecodeProj* projs, int G, int K, const uint16_t* x, int ldx, const int8_t* xq,
                                 const float* sx, int M, int ydtype, int32_t* P, void* ws,
                                 cudaStream_t st);
// The CUDA-core decode path: the streaming kernel where it applies, else the
// register-ring kernel.  x (fused activation preparation) requires
// cc_fusable(M, K).
bool cc_fusable(int M, int K, int rows);
cudaError_t launch_decode_cc(const DecodeProj* projs, int G, int K, const uint16_t* x, int ldx, const int8_t* xq,
                             const float* sx, int M, int ydtype, int32_t* P, void* ws, cudaStream_t st);

// Split-K plan of the decode kernels (a pure function of the geometry, so
// the workspace size and the launch agree).
struct DecodePlan {
  int kernel;   // 0 = CUDA-core kernel, 1 = tensor-core kernel
  int S;        // splits over tile columns
  int rows;     // output rows per CTA (kRowsPerCta, or 128 for the tensor-core kernel)
  int blocks;   // number of CTA row blocks
};
DecodePlan plan_decode(int M, const aq_packed* w);
// The tensor-core part of the decode plan for `blocks` 128-row blocks of C input tiles.
DecodePlan plan_tc_decode(int M, int blocks, int C);
size_t decode_ws_bytes(int M, const aq_packed* w);
size_t prefill_ws_bytes(int M, const aq_packed* w);

// Launchers (defined next to their kernels).  They assume validated arguments.
cudaError_t launch_quant_act(const uint16_t* x, int M, int K, int ldx, int8_t* xq, float* sx, cudaStream_t st);
cudaError_t launch_pack_payload(const int8_t* codes, const uint16_t* scales, const float* tile_scales,
                                const aq_packed* out, const uint8_t* map_dev, int* err_dev, cudaStream_t st);
// Long-prefill variant: all-INT8 copy of a packed projection in a caller buffer.
size_t expanded_bytes(const aq_packed* w);
cudaError_t launch_expand_int8(const aq_packed* w, void* buf, aq_packed* out, cudaStream_t st);
cudaError_t launch_tc(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias, void* y,
                      int ydtype, int ldy, void* ws, int32_t* P, int phase, cudaStream_t st);
// One tensor-core launch over G projections that share xq (their 128-row blocks
// concatenated; same K and bN; every member's rows a multiple of 128).
cudaError_t launch_tc_group(const aq_packed* const* w, int G, const float* const* bias, void* const* y,
                            const int* ldy, const int8_t* xq, const float* sx, int M, int ydtype, void* ws, int phase,
                            cudaStream_t st);
// Test form of launch_tc: every bounded wait gives up after wait_ns and the
// weight producer stops after `stop_after` tiles (so later stages never fill).
cudaError_t launch_tc_stalled(const aq_packed* w, const int8_t* xq, const float* sx, int M, void* y, int ldy,
                              void* ws, int phase, unsigned long long wait_ns, int stop_after, cudaStream_t st);

// ---------------------------------------------------------------- device helpers
#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Like mbar_try_wait, but a thread whose phase is not complete sleeps in
// hardware until it completes or kWaitSuspendNs pass, instead of spinning
// (spinning waiters take issue slots from the warps doing the work).
constexpr uint32_t kWaitSuspendNs = 20000;
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kWaitSuspendNs)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete.  Returns false when
// `abort` became nonzero or `limit_ns` passed; never waits unbounded.
// Between checks of the abort flag and the clock the thread sleeps (see
// mbar_try_wait_sleep), so the checks cost little.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          unsigned long long limit_ns = kWaitTimeoutNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D tiled TMA load global -> shared, completing on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16), no multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tcgen05 (5th-generation tensor core, accumulators in tensor memory)
__device__ __forceinline__ void tmem_alloc(uint32_t* slot_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, INT8 x INT8 -> INT32, one CTA.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 op this thread issued so far is done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns, every value = v.
__device__ __forceinline__ void tmem_st16_const(uint32_t taddr, uint32_t v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
      "r"(v)
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread t of the warp receives lane
// (warp quadrant * 32 + t), columns col .. col+15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// Shared-memory matrix descriptor, K-major operand in the 128-byte swizzle
// layout: 8-row groups 1024 bytes apart (stride byte offset), version 1,
// layout code 2 (SWIZZLE_128B) in bits 61..63.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
  d |= (uint64_t)(16 >> 4) << 16;      // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;    // stride byte offset
  d |= (uint64_t)1 << 46;              // descriptor version
  d |= (uint64_t)2 << 61;              // SWIZZLE_128B
  return d;
}

// Instruction descriptor for kind::i8: D = S32, A = B = signed 8-bit, both
// K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Records the first error of a launch.  `clear_bytes`: the bytes after the
// header (split-K arrival counters) that a call which gave up may have left
// nonzero; the status call zeroes them so the workspace is ready again.
__device__ __forceinline__ void record_error(void* ws, int code, int info, int clear_bytes) {
  WsHeader* h = reinterpret_cast<WsHeader*>(ws);
  if (atomicCAS(&h->err_code, 0, code) == 0) {
    atomicExch(&h->err_info, info);
    atomicExch(&h->err_clear, clear_bytes);
  }
}

// Programmatic dependent launch controls (no-ops without the launch attribute).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b16) { return __uint_as_float(b16 << 16); }

// ---- per-token INT8 activation quantization (shared by every kernel that prepares activations)
// max(m, |x|) over eight bf16 values.  |x| of a bf16 is its bit pattern with the
// sign cleared, and for non-negative values the float order is the integer order
// of the patterns, so the eight magnitudes reduce with 16-bit-pair integer maxima
// and one conversion at the end.  (A NaN pattern converts to NaN, which fmaxf
// ignores.)
__device__ __forceinline__ float abs_max8(const uint4& v, float m) {
  const uint32_t a = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
  const uint32_t b = __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
  const uint32_t c = __vmaxu2(a, b);
  return fmaxf(m, bf16_bits_to_float(max(c & 0xFFFFu, c >> 16)));
}

// s = max(fl64(amax / 127), 1e-12) (eq. 6 floor).  The quotient is formed from
// the rounded reciprocal R = fl64(1/127) and one exact residual correction
// (the FMA-based quotient correction of P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Develop. 34(1), 1990): q = amax R, r = fma(-q, 127, amax) (exact),
// s = fma(r, R, q).  For every finite bf16 amax this equals the IEEE fp64
// quotient (checked exhaustively against the oracle's division), at a
// fraction of a division's latency.
__device__ __forceinline__ double act_scale(float amax) {
  constexpr double kInv127 = 1.0 / 127.0;
  const double a = static_cast<double>(amax);
  const double q = a * kInv127;
  double s = fma(fma(-q, 127.0, a), kInv127, q);
  return s < 1e-12 ? 1e-12 : s;
}

// r32 for quant_code: fp32 reciprocal of fp32(s), relative error <= 2 * 2^-24.
__device__ __forceinline__ float act_recip(double s) { return __frcp_rn(static_cast<float>(s)); }

// clamp(rint(fl64(x / s)), -127, 127): the oracle's rule, by fp64 division.
static __device__ __forceinline__ int quant_code_exact(float x, double s) {
  const double q = rint(static_cast<double>(x) / s);
  return static_cast<int>(fmin(fmax(q, -127.0), 127.0));
}

// Eight codes of clamp(rint(fl64(x / s)), -127, 127).
// Fast path: t = x * r32 carries at most three roundings of 2^-24 each
// (fp32(s), the reciprocal, the product), so |t - x/s| <= 127 * 3 * 2^-24
// < 2.3e-5 (|x / s| <= 127).  The rounding is done on the FMA pipe: for
// |c| < 2^22, c + 1.5 * 2^23 holds rint(c) (ties to even) in its low mantissa
// bits, so with c = clamp(t, -127, 127) the low byte of that sum's pattern is the
// two's-complement code and subtracting 1.5 * 2^23 again gives k = rint(c)
// exactly (clamping before rounding equals clamping after it for integer
// bounds).  When t is more than 4e-5 away from the nearest half-integer, the
// exact quotient rounds, and clamps, to the same code (for t > 127.49996 the
// test below fails and the element takes the exact path).  Ties and near-ties
// are redone by fp64 division.  They are not rare with bf16 inputs (about 0.3%
// of the elements: ratios of two 8-bit mantissas times 127 land on
// half-integers), so each element position is a branch of its own, taken by
// the warp only when one of its lanes needs that element.
__device__ __forceinline__ uint2 quantize8(const uint4& v, double s, float r32) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float xf[8];
  uint32_t u[8];
  uint32_t slow = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    xf[i] = bf16_bits_to_float((i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu));
    const float t = xf[i] * r32;
    const float r = __fadd_rn(fminf(fmaxf(t, -127.f), 127.f), kRound);
    const float k = __fsub_rn(r, kRound);
    slow |= (0.5f - fabsf(t - k) > 4.0e-5f ? 0u : 1u) << i;
    u[i] = __float_as_uint(r);
  }
  if (__any_sync(__activemask(), slow != 0)) {
    // unrolled: a runtime index would put u[] and xf[] in local memory for the
    // fast path too
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if ((slow >> i) & 1u) u[i] = static_cast<uint32_t>(quant_code_exact(xf[i], s));
  }
  // low bytes of u[0..3] and u[4..7]
  const uint32_t l0 = __byte_perm(u[0], u[1], 0x0040), h0 = __byte_perm(u[2], u[3], 0x0040);
  const uint32_t l1 = __byte_perm(u[4], u[5], 0x0040), h1 = __byte_perm(u[6], u[7], 0x0040);
  return make_uint2(__byte_perm(l0, h0, 0x5410), __byte_perm(l1, h1, 0x5410));
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}

// Start moving `bytes` (a multiple of 16, 16-byte aligned) from HBM into L2;
// no shared memory, no completion to wait for.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
               : "memory");
}

#endif  // __CUDACC__

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel on the stream finishes; it must call pdl_wait() before it
// reads anything an earlier kernel wrote and before its first global write.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Opt a kernel in to `bytes` of dynamic shared memory on the current device.
// The attribute is per device, so it is set once per (kernel, device); the
// flags are atomics, so concurrent host threads at worst set it twice.
// carveout_pct >= 0 also sets the preferred shared-memory carveout (percent).
bool set_smem_attr_once(const void* kernel, int bytes, int carveout_pct, std::atomic<bool>* done_flags);
template <auto Kernel>
cudaError_t ensure_smem_attr(int bytes, int carveout_pct = -1) {
  static std::atomic<bool> done[kMaxDevices];
  return set_smem_attr_once(reinterpret_cast<const void*>(Kernel), bytes, carveout_pct, done)
             ? cudaSuccess
             : cudaErrorInvalidValue;
}

}  // namespace aq
