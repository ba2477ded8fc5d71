// C ABI entry points of libaq: host-side validation, split planning and
// dispatch to the sm_100a kernels.  Every hot-path entry validates its
// arguments, enqueues its kernels on the caller's stream and returns without
// allocating or synchronizing.
#include <algorithm>
#include <atomic>

#include "aq_internal.cuh"

namespace aq {

int num_sms() {
  static std::atomic<int> cached[kMaxDevices];
  constexpr int kFallback = 148;  // B200
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return kFallback;
  }
  int v = cached[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
    cudaGetLastError();
    return kFallback;
  }
  cached[dev].store(v, std::memory_order_relaxed);
  return v;
}

bool set_smem_attr_once(const void* kernel, int bytes, int carveout_pct, std::atomic<bool>* done_flags) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (done_flags[dev].load(std::memory_order_acquire)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  if (carveout_pct >= 0 &&
      cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, carveout_pct) != cudaSuccess)
    return false;
  done_flags[dev].store(true, std::memory_order_release);
  return true;
}

// The streaming kernel takes one token; from two tokens on the register-ring
// kernel measured faster on the benchmark's decode step (1.36 against 1.55 ms
// per Llama-3.2-3B step at 2 tokens), and they tie at 4.
static constexpr int kStreamMaxM = 1;

bool cc_fusable(int M, int K, int rows) {
  return (M <= kStreamMaxM && stream_supported(M, K, rows)) || rows_fusable(M, K);
}

cudaError_t launch_decode_cc(const DecodeProj* projs, int G, int K, const uint16_t* x, int ldx, const int8_t* xq,
                             const float* sx, int M, int ydtype, int32_t* P, void* ws, cudaStream_t st) {
  int rows = 0;
  for (int g = 0; g < G; ++g) rows += projs[g].N;
  if (M <= kStreamMaxM && stream_supported(M, K, rows))
    return launch_decode_stream(projs, G, K, x, ldx, xq, sx, M, ydtype, P, ws, st);
  return launch_decode_rows(projs, G, K, x, ldx, xq, sx, M, ydtype, P, ws, st);
}

int validate_packed(const aq_packed* w) {
  if (!w) return AQ_ERR_ARG;
  if (w->scale_kind != AQ_SCALES_ROW_FP16) return AQ_ERR_ARG;  // the per-token layer's kernels read fp16 row scales
  if (!geometry_ok(w->N, w->K, w->bN, w->bK)) return AQ_ERR_SHAPE;
  if (w->R != w->N / w->bN || w->C != w->K / w->bK) return AQ_ERR_SHAPE;
  if (w->T4 < 0 || w->T8 < 0 || (long long)w->T4 + w->T8 != (long long)w->R * w->C) return AQ_ERR_SHAPE;
  if (!w->bitmap || !w->row_off4 || !w->row_off8 || !w->tile_idx || !w->scales) return AQ_ERR_ARG;
  if ((w->T4 > 0 && !w->w4) || (w->T8 > 0 && !w->w8)) return AQ_ERR_ARG;
  if (((uintptr_t)w->w4 & 15) || ((uintptr_t)w->w8 & 15) || ((uintptr_t)w->scales & 15)) return AQ_ERR_ARG;
  if ((uintptr_t)w->tile_idx & 3) return AQ_ERR_ARG;  // read as 4-byte words
  return AQ_OK;
}

static int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }
static constexpr int kMaxSplits = 8;
// Input tiles per split at least (see plan_decode).
static int min_split_tiles(int M) { return M <= 16 ? 5 : M <= 32 ? 8 : 20; }

// Fusing the activation preparation into every CTA of the CUDA-core decode
// kernel pays off for 1-2 tokens; from 3 tokens on, one preparation kernel plus
// a single grouped launch over pre-quantized codes is faster (the per-CTA
// preparation grows with M).  The fused codes live in shared memory.
bool rows_fusable(int M, int K) { return M <= 2 && 2 * (size_t)M * K + 16 * (size_t)M <= kFusedMaxBytes; }

// Decode: up to 3 tokens on the CUDA cores (bandwidth-bound, one CTA per 32
// output rows, no split); more tokens on the tensor cores with splits over
// tile columns to fill the GPU in one wave.  (Measured on whole steps: at 4
// tokens the tensor cores take 5-24% less time on the 3B- to 14B-class models;
// at 3 tokens the CUDA cores are 10% faster on the 3B-class model.  Groups of
// three or more projections without whole 128-row blocks keep one grouped
// CUDA-core launch up to kRowsMaxM tokens: see group_rows.)
static constexpr int kRowsPreferM = 3;

DecodePlan plan_decode(int M, const aq_packed* w) {
  DecodePlan p;
  if (rows_supported(M, w->K) && M <= kRowsPreferM) {
    p.kernel = 0;
    p.rows = kRowsPerCta;
    p.blocks = w->N / kRowsPerCta;
    p.S = 1;
  } else {
    p = plan_tc_decode(M, ceil_div(w->R, 128 / w->bN), w->C);
  }
  return p;
}

DecodePlan plan_tc_decode(int M, int blocks, int C) {
  DecodePlan p;
  p.kernel = 1;
  p.rows = 128;
  p.blocks = blocks;
  // One wave (blocks x S <= SMs), at most kMaxSplits, and at least
  // min_split_tiles(M) input tiles per split: splitting shortens every CTA's
  // tile chain but costs the unit a round of partial sums that grows with the
  // token count.  From 32 tokens on, a launch whose row blocks alone fill a
  // third of the GPU is not split.  (Measured per projection shape at 16, 32 and
  // 64 tokens for 1-8 splits: this rule is within 4% of the best split count on
  // every shape of the 3B- and 8B-class models.)
  const int sms = num_sms();
  p.S = std::max(1, std::min(std::min(C / min_split_tiles(M), kMaxSplits), sms / p.blocks));
  if (M >= 32 && 3 * p.blocks >= sms) p.S = 1;
  return p;
}

static size_t counters_bytes(int blocks) { return ((size_t)blocks * sizeof(int) + 255) / 256 * 256; }

size_t decode_ws_bytes(int M, const aq_packed* w) {
  const DecodePlan p = plan_decode(M, w);
  if (p.kernel == 0) return kWsHeader;
  size_t b = kWsHeader + counters_bytes(p.blocks);
  if (p.S > 1) b += (size_t)p.S * ((M + 3) & ~3) * w->N * sizeof(float);  // [S][N][M rounded up to 4]
  return b;
}

size_t prefill_ws_bytes(int /*M*/, const aq_packed* w) { return kWsHeader + counters_bytes(w->R); }

DecodeProj decode_proj(const aq_packed* w, const float* bias, void* y, int ldy) {
  DecodeProj d;
  d.bitmap = w->bitmap; d.tile_idx = w->tile_idx; d.w4 = w->w4; d.w8 = w->w8; d.scales = w->scales;
  d.bias = bias; d.y = y; d.N = w->N; d.bN = w->bN; d.ldy = ldy; d.blocks = w->N / kRowsPerCta;
  return d;
}

}  // namespace aq

using namespace aq;

extern "C" const char* aq_status_str(int status) {
  switch (status) {
    case AQ_OK: return "AQ_OK";
    case AQ_ERR_ARG: return "AQ_ERR_ARG: invalid argument";
    case AQ_ERR_SHAPE: return "AQ_ERR_SHAPE: shape violates the tile geometry";
    case AQ_ERR_RANGE: return "AQ_ERR_RANGE: INT4 tile holds a code outside [-8, 7]";
    case AQ_ERR_UNSUPPORTED: return "AQ_ERR_UNSUPPORTED: not implemented by this build";
    case AQ_ERR_WORKSPACE: return "AQ_ERR_WORKSPACE: workspace missing or too small";
    case AQ_ERR_CUDA: return "AQ_ERR_CUDA: CUDA runtime or launch failure";
    case AQ_ERR_TIMEOUT: return "AQ_ERR_TIMEOUT: a kernel gave up on a bounded wait";
    default: return "unknown aq_status";
  }
}

extern "C" int aq_packed_sizes(int N, int K, int bN, int bK, int T4, size_t* out) {
  if (!out) return AQ_ERR_ARG;
  if (!geometry_ok(N, K, bN, bK) && !paper_geometry_ok(N, K, bN, bK)) return AQ_ERR_SHAPE;
  const long long R = N / bN, C = K / bK, T = R * C;
  if (T4 < 0 || T4 > T) return AQ_ERR_ARG;
  const long long B = (long long)bN * bK;
  out[AQ_BUF_BITMAP] = (size_t)((T + 7) / 8);
  out[AQ_BUF_ROW_OFF4] = (size_t)(4 * (R + 1));
  out[AQ_BUF_ROW_OFF8] = (size_t)(4 * (R + 1));
  out[AQ_BUF_TILE_IDX] = (size_t)(4 * T);
  out[AQ_BUF_W4] = (size_t)(B / 2 * T4);
  out[AQ_BUF_W8] = (size_t)(B * (T - T4));
  out[AQ_BUF_SCALES] = (size_t)(2 * T * bN);
  return AQ_OK;
}

extern "C" size_t aq_workspace_bytes(int phase, int M, const aq_packed* w) {
  if (validate_packed(w) != AQ_OK || M < 1) return 0;
  if (phase == AQ_PHASE_DECODE) return M <= kMaxDecodeM ? decode_ws_bytes(M, w) : 0;
  if (phase == AQ_PHASE_PREFILL) return prefill_ws_bytes(M, w);
  return 0;
}

extern "C" int aq_quant_act(const uint16_t* x, int M, int K, int ldx, int8_t* xq, float* sx, void* stream) {
  if (!x || !xq || !sx || M < 1 || K < 16 || K % 16 || K > (1 << 20) || ldx < K || ldx % 8) return AQ_ERR_ARG;
  if (((uintptr_t)x & 15) || ((uintptr_t)xq & 15) || ((uintptr_t)sx & 3)) return AQ_ERR_ARG;
  return launch_quant_act(x, M, K, ldx, xq, sx, static_cast<cudaStream_t>(stream)) == cudaSuccess ? AQ_OK
                                                                                                   : AQ_ERR_CUDA;
}

namespace aq {
// Token scales and bias are fetched as 4-byte words (cp.async of 4 bytes),
// outputs stored as 4- or 2-byte words: a pointer off that grain is an
// argument error, not a misaligned access on the GPU.
bool operands_misaligned(const float* sx, const float* bias, const void* y, int ydtype) {
  return (((uintptr_t)sx | (uintptr_t)bias) & 3) != 0 || ((uintptr_t)y & (ydtype == AQ_F32 ? 3u : 1u)) != 0;
}
}  // namespace aq

static int check_linear(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias,
                        const void* y, int ydtype, int ldy) {
  int rc = validate_packed(w);
  if (rc != AQ_OK) return rc;
  if (!xq || !sx || !y || M < 1 || ldy < w->N) return AQ_ERR_ARG;
  if (ydtype != AQ_F32 && ydtype != AQ_BF16) return AQ_ERR_ARG;
  if (((uintptr_t)xq & 15) || operands_misaligned(sx, bias, y, ydtype)) return AQ_ERR_ARG;
  return AQ_OK;
}

// The workspace holds split-K partial sums written as 16-byte vectors.
static int check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (!ws || ws_bytes < need) return AQ_ERR_WORKSPACE;
  return ((uintptr_t)ws & 15) ? AQ_ERR_ARG : AQ_OK;
}

extern "C" int aq_linear_decode(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias,
                                void* y, int ydtype, int ldy, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_linear(w, xq, sx, M, bias, y, ydtype, ldy);
  if (rc != AQ_OK) return rc;
  if (M > kMaxDecodeM) return AQ_ERR_ARG;
  if ((rc = check_ws(ws, ws_bytes, decode_ws_bytes(M, w))) != AQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (plan_decode(M, w).kernel == 0) {
    const DecodeProj d = decode_proj(w, bias, y, ldy);
    e = launch_decode_cc(&d, 1, w->K, nullptr, 0, xq, sx, M, ydtype, nullptr, ws, st);
  } else {
    e = launch_tc(w, xq, sx, M, bias, y, ydtype, ldy, ws, nullptr, AQ_PHASE_DECODE, st);
  }
  return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
}

extern "C" int aq_linear_prefill(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias,
                                 void* y, int ydtype, int ldy, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_linear(w, xq, sx, M, bias, y, ydtype, ldy);
  if (rc != AQ_OK) return rc;
  if ((rc = check_ws(ws, ws_bytes, prefill_ws_bytes(M, w))) != AQ_OK) return rc;
  cudaError_t e = launch_tc(w, xq, sx, M, bias, y, ydtype, ldy, ws, nullptr, AQ_PHASE_PREFILL,
                            static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
}

namespace aq {
cudaError_t launch_quant_act_groups(const uint16_t* x, int M, int K, int ldx, int8_t* xq, float* sx,
                                    cudaStream_t st);
}  // namespace aq

extern "C" int aq_act_group_rows(int M) { return M < 1 ? 0 : act_group_rows(M); }

extern "C" int aq_quant_act_groups(const uint16_t* x, int M, int K, int ldx, int8_t* xq, float* sx, void* stream) {
  if (!x || !xq || !sx || M < 1 || K < 64 || K % 64 || K > (1 << 20) || ldx < K || ldx % 8) return AQ_ERR_ARG;
  if (((uintptr_t)x & 15) || ((uintptr_t)xq & 7) || ((uintptr_t)sx & 3)) return AQ_ERR_ARG;
  return launch_quant_act_groups(x, M, K, ldx, xq, sx, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? AQ_OK : AQ_ERR_CUDA;
}

extern "C" size_t aq_expanded_bytes(const aq_packed* w) {
  return validate_packed(w) == AQ_OK ? expanded_bytes(w) : 0;
}

extern "C" int aq_expand_int8(const aq_packed* w, void* buf, size_t buf_bytes, aq_packed* out, void* stream) {
  int rc = validate_packed(w);
  if (rc != AQ_OK) return rc;
  if (!buf || !out || ((uintptr_t)buf & 255)) return AQ_ERR_ARG;
  if (buf_bytes < expanded_bytes(w)) return AQ_ERR_WORKSPACE;
  return launch_expand_int8(w, buf, out, static_cast<cudaStream_t>(stream)) == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
}

extern "C" int aq_linear_prefill_expanded(const aq_packed* w, const int8_t* xq, const float* sx, int M,
                                          const float* bias, void* y, int ydtype, int ldy, void* ws, size_t ws_bytes,
                                          void* tmp, size_t tmp_bytes, void* stream) {
  int rc = check_linear(w, xq, sx, M, bias, y, ydtype, ldy);
  if (rc != AQ_OK) return rc;
  if ((rc = check_ws(ws, ws_bytes, prefill_ws_bytes(M, w))) != AQ_OK) return rc;
  if (!tmp || ((uintptr_t)tmp & 255)) return AQ_ERR_ARG;
  if (tmp_bytes < expanded_bytes(w)) return AQ_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  aq_packed e{};
  cudaError_t err = launch_expand_int8(w, tmp, &e, st);
  if (err == cudaSuccess)
    err = launch_tc(&e, xq, sx, M, bias, y, ydtype, ldy, ws, nullptr, AQ_PHASE_PREFILL, st);
  return err == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
}

extern "C" int aq_debug_tile_partials(const aq_packed* w, const int8_t* xq, int M, int phase, int32_t* P, void* ws,
                                      size_t ws_bytes, void* stream) {
  int rc = validate_packed(w);
  if (rc != AQ_OK) return rc;
  if (!xq || !P || M < 1 || ((uintptr_t)xq & 15)) return AQ_ERR_ARG;
  if (phase != AQ_PHASE_DECODE && phase != AQ_PHASE_PREFILL) return AQ_ERR_ARG;
  if (phase == AQ_PHASE_DECODE && M > kMaxDecodeM) return AQ_ERR_ARG;
  if ((uintptr_t)P & 3) return AQ_ERR_ARG;
  if ((rc = check_ws(ws, ws_bytes, kWsHeader)) != AQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (phase == AQ_PHASE_DECODE && plan_decode(M, w).kernel == 0) {
    const DecodeProj d = decode_proj(w, nullptr, nullptr, w->N);
    e = launch_decode_cc(&d, 1, w->K, nullptr, 0, xq, nullptr, M, AQ_F32, P, ws, st);
  } else
    e = launch_tc(w, xq, nullptr, M, nullptr, nullptr, AQ_F32, w->N, ws, P, phase, st);
  return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
}

extern "C" int aq_debug_linear_stalled(const aq_packed* w, const int8_t* xq, const float* sx, int M, int phase,
                                       float* y, int ldy, void* ws, size_t ws_bytes, unsigned long long wait_ns,
                                       int stop_after, void* stream) {
  int rc = check_linear(w, xq, sx, M, nullptr, y, AQ_F32, ldy);
  if (rc != AQ_OK) return rc;
  if (phase != AQ_PHASE_DECODE && phase != AQ_PHASE_PREFILL) return AQ_ERR_ARG;
  if (phase == AQ_PHASE_DECODE && (M > kMaxDecodeM || plan_decode(M, w).kernel != 1)) return AQ_ERR_ARG;
  if (wait_ns < 100000ull || wait_ns > 10000000000ull || stop_after < 0) return AQ_ERR_ARG;
  const size_t need = phase == AQ_PHASE_DECODE ? decode_ws_bytes(M, w) : prefill_ws_bytes(M, w);
  if ((rc = check_ws(ws, ws_bytes, need)) != AQ_OK) return rc;
  return launch_tc_stalled(w, xq, sx, M, y, ldy, ws, phase, wait_ns, stop_after, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? AQ_OK
             : AQ_ERR_CUDA;
}

// ---------------------------------------------------------------- shared-input groups (App. E.4)
static int check_group(int phase, const aq_packed* const* w, int G, const uint16_t* x, int ldx, int M) {
  if (!w || G < 1 || G > kMaxGroup || !x || M < 1) return AQ_ERR_ARG;
  if (phase != AQ_PHASE_DECODE && phase != AQ_PHASE_PREFILL) return AQ_ERR_ARG;
  if (phase == AQ_PHASE_DECODE && M > kMaxDecodeM) return AQ_ERR_ARG;
  for (int g = 0; g < G; ++g) {
    int rc = validate_packed(w[g]);
    if (rc != AQ_OK) return rc;
    if (w[g]->K != w[0]->K) return AQ_ERR_SHAPE;
  }
  const int K = w[0]->K;
  if (ldx < K || ldx % 8 || ((uintptr_t)x & 15)) return AQ_ERR_ARG;
  return AQ_OK;
}

static bool group_fused(int phase, const aq_packed* const* w, int G, int M) {
  if (phase != AQ_PHASE_DECODE || !rows_supported(M, w[0]->K)) return false;
  int rows = 0;
  for (int g = 0; g < G; ++g) rows += w[g]->N;
  return cc_fusable(M, w[0]->K, rows);
}

static size_t align256(size_t b) { return (b + 255) / 256 * 256; }

// Decode: one tensor-core launch over all members' rows when every member would
// run on the tensor cores alone, with the same tile shape and whole 128-row
// blocks per member (q/k/v and gate/up at 32 and 64 tokens: 31-32% less time per
// 3B-class step; prefill gains nothing from it, its launches are long).
static bool group_tc(int phase, const aq_packed* const* w, int G, int M) {
  if (G < 2 || phase != AQ_PHASE_DECODE || M > kMaxDecodeM) return false;
  for (int g = 0; g < G; ++g) {
    if (w[g]->bN != w[0]->bN || w[g]->N % 128 != 0) return false;
    if (phase == AQ_PHASE_DECODE && plan_decode(M, w[g]).kernel != 1) return false;
  }
  return true;
}

// Workspace of the grouped tensor-core launch (header, split counters, split partial sums).
static size_t group_tc_ws_bytes(int phase, int M, const aq_packed* const* w, int G) {
  int blocks = 0, N = 0;
  for (int g = 0; g < G; ++g) {
    blocks += w[g]->N / 128;
    N += w[g]->N;
  }
  if (phase != AQ_PHASE_DECODE) return kWsHeader + counters_bytes(blocks);
  const DecodePlan p = plan_tc_decode(M, blocks, w[0]->C);
  size_t b = kWsHeader + counters_bytes(p.blocks);
  if (p.S > 1) b += (size_t)p.S * ((M + 3) & ~3) * N * sizeof(float);
  return b;
}

static size_t group_ws_bytes(int phase, int M, const aq_packed* const* w, int G) {
  if (group_fused(phase, w, G, M)) return kWsHeader;
  size_t lin = 0;
  for (int g = 0; g < G; ++g)
    lin = std::max(lin, phase == AQ_PHASE_DECODE ? decode_ws_bytes(M, w[g]) : prefill_ws_bytes(M, w[g]));
  if (group_tc(phase, w, G, M)) lin = std::max(lin, group_tc_ws_bytes(phase, M, w, G));
  // the linear workspace (header first), then the prepared activations
  return align256(lin) + align256((size_t)M * w[0]->K) + align256((size_t)M * sizeof(float));
}

// A decode group runs as one CUDA-core launch over all members' rows when every
// member would use the CUDA-core kernel alone, or, up to kRowsMaxM tokens,
// when it has three or more members and cannot take the grouped tensor-core
// launch (one CUDA-core launch beats one tensor-core launch per member: q/k/v
// at 8 tokens, 24.8 against 27.6 us per layer; the grouped tensor-core launch
// beats both: whole 3B- / 8B- / 14B-class steps at 8 tokens 14-16% faster).
static bool group_rows(int phase, const aq_packed* const* w, int G, int M) {
  if (phase != AQ_PHASE_DECODE) return false;
  bool all_rows = true, all_supported = true;
  for (int g = 0; g < G; ++g) {
    all_rows = all_rows && plan_decode(M, w[g]).kernel == 0;
    all_supported = all_supported && rows_supported(M, w[g]->K);
  }
  return all_rows || (G >= 3 && all_supported);
}

extern "C" size_t aq_group_workspace_bytes(int phase, int M, const aq_packed* const* w, int G) {
  if (!w || G < 1 || G > kMaxGroup || M < 1) return 0;
  if (phase != AQ_PHASE_DECODE && phase != AQ_PHASE_PREFILL) return 0;
  if (phase == AQ_PHASE_DECODE && M > kMaxDecodeM) return 0;
  for (int g = 0; g < G; ++g)
    if (validate_packed(w[g]) != AQ_OK || w[g]->K != w[0]->K) return 0;
  return group_ws_bytes(phase, M, w, G);
}

extern "C" int aq_linear_group(int phase, const aq_packed* const* w, int G, const uint16_t* x, int ldx, int M,
                               const float* const* bias, void* const* y, const int* ldy, int ydtype, void* ws,
                               size_t ws_bytes, void* stream) {
  int rc = check_group(phase, w, G, x, ldx, M);
  if (rc != AQ_OK) return rc;
  if (!y || !ldy || (ydtype != AQ_F32 && ydtype != AQ_BF16)) return AQ_ERR_ARG;
  for (int g = 0; g < G; ++g)
    if (!y[g] || ldy[g] < w[g]->N || operands_misaligned(nullptr, bias ? bias[g] : nullptr, y[g], ydtype))
      return AQ_ERR_ARG;
  if ((rc = check_ws(ws, ws_bytes, group_ws_bytes(phase, M, w, G))) != AQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int K = w[0]->K;
  cudaError_t e = cudaSuccess;
  if (group_fused(phase, w, G, M)) {
    DecodeProj d[kMaxGroup];
    for (int g = 0; g < G; ++g) d[g] = decode_proj(w[g], bias ? bias[g] : nullptr, y[g], ldy[g]);
    e = launch_decode_cc(d, G, K, x, ldx, nullptr, nullptr, M, ydtype, nullptr, ws, st);
    return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
  }
  // prepare the shared input once, then run the members on it (one launch
  // over all members' rows when they all use the CUDA-core decode kernel)
  size_t lin = 0;
  for (int g = 0; g < G; ++g)
    lin = std::max(lin, phase == AQ_PHASE_DECODE ? decode_ws_bytes(M, w[g]) : prefill_ws_bytes(M, w[g]));
  if (group_tc(phase, w, G, M)) lin = std::max(lin, group_tc_ws_bytes(phase, M, w, G));
  char* base = static_cast<char*>(ws);
  int8_t* xq = reinterpret_cast<int8_t*>(base + align256(lin));
  float* sx = reinterpret_cast<float*>(base + align256(lin) + align256((size_t)M * K));
  e = launch_quant_act(x, M, K, ldx, xq, sx, st);
  if (e == cudaSuccess && group_rows(phase, w, G, M) && !group_tc(phase, w, G, M)) {  // one CUDA-core launch
    DecodeProj d[kMaxGroup];
    for (int g = 0; g < G; ++g) d[g] = decode_proj(w[g], bias ? bias[g] : nullptr, y[g], ldy[g]);
    e = launch_decode_cc(d, G, K, nullptr, 0, xq, sx, M, ydtype, nullptr, ws, st);
    return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
  }
  if (e == cudaSuccess && group_tc(phase, w, G, M)) {  // one tensor-core launch over all members' rows
    e = launch_tc_group(w, G, bias, y, ldy, xq, sx, M, ydtype, ws, phase, st);
    return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
  }
  for (int g = 0; e == cudaSuccess && g < G; ++g) {
    const float* b = bias ? bias[g] : nullptr;
    if (phase == AQ_PHASE_DECODE && plan_decode(M, w[g]).kernel == 0) {
      const DecodeProj d = decode_proj(w[g], b, y[g], ldy[g]);
      e = launch_decode_cc(&d, 1, K, nullptr, 0, xq, sx, M, ydtype, nullptr, ws, st);
    } else {
      e = launch_tc(w[g], xq, sx, M, b, y[g], ydtype, ldy[g], ws, nullptr, phase, st);
    }
  }
  return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
}

extern "C" int aq_workspace_status(void* ws, void* stream, int* info) {
  if (!ws) return AQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WsHeader h{0, 0, 0};
  if (cudaStreamSynchronize(st) != cudaSuccess) return AQ_ERR_CUDA;
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return AQ_ERR_CUDA;
  if (h.err_code != 0) {
    // a call that gave up may have left split-K arrival counters nonzero: the
    // kernel recorded how many bytes after the header to zero with the error
    const size_t clear = kWsHeader + (size_t)std::max(h.err_clear, 0);
    if (cudaMemset(ws, 0, clear) != cudaSuccess) return AQ_ERR_CUDA;
  }
  if (info) *info = h.err_info;
  return h.err_code == 0 ? AQ_OK : AQ_ERR_TIMEOUT;
}
