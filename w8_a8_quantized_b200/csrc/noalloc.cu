// aq_linear_decode_noalloc: the decode-phase linear layer for callers that
// cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) at the point
// where they run a layer: code that executes inside a custom memory-pool or
// allocator callback, runtimes that forbid allocation after start-up so that
// their memory footprint stays fixed and predictable, and plug-ins that are
// handed only the input and output buffers.  aq_linear_decode needs a
// caller-provided workspace for the split-K partial sums of its tensor-core
// path; this entry point takes its scratch from a fixed array in device memory
// that the library itself holds, so the caller passes only inputs and outputs.
//
// The scratch array is a file-scope __device__ array of kNoAllocScratchBytes
// (4 MiB).  Every GPU that loads the library holds it until the process exits.
// In host code the array's name is only a host-side stand-in, so its device
// address is obtained once per device with cudaGetSymbolAddress (with that
// device current) and cached; the first call on each device does this set-up.
#include <mutex>

#include "aq_internal.cuh"

namespace aq {
bool operands_misaligned(const float* sx, const float* bias, const void* y, int ydtype);  // aq_api.cu

namespace {

constexpr size_t kNoAllocScratchBytes = 4u << 20;  // 4 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return AQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return AQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return AQ_OK;
}

}  // namespace
}  // namespace aq

using namespace aq;

extern "C" int aq_linear_decode_noalloc(const aq_packed* w, const int8_t* xq, const float* sx, int M,
                                        const float* bias, void* y, int ydtype, int ldy, void* stream) {
  int rc = validate_packed(w);
  if (rc != AQ_OK) return rc;
  if (!xq || !sx || !y || M < 1 || M > kMaxDecodeM || ldy < w->N) return AQ_ERR_ARG;
  if (ydtype != AQ_F32 && ydtype != AQ_BF16) return AQ_ERR_ARG;
  if (((uintptr_t)xq & 15) || operands_misaligned(sx, bias, y, ydtype)) return AQ_ERR_ARG;
  const size_t need = decode_ws_bytes(M, w);
  if (need > kNoAllocScratchBytes) return AQ_ERR_WORKSPACE;  // beyond the fixed scratch: use aq_linear_decode
  void* scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc != AQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: clear the status word and the
  // split-K arrival counters, which must start at zero (partial sums need not).
  const DecodePlan plan = plan_decode(M, w);
  const size_t zero_bytes = plan.kernel == 0 ? kWsHeader : kWsHeader + ((size_t)plan.blocks * sizeof(int) + 255) / 256 * 256;
  if (cudaMemsetAsync(scratch, 0, zero_bytes, st) != cudaSuccess) return AQ_ERR_CUDA;
  cudaError_t e;
  if (plan.kernel == 0) {
    const DecodeProj d = decode_proj(w, bias, y, ldy);
    e = launch_decode_cc(&d, 1, w->K, nullptr, 0, xq, sx, M, ydtype, nullptr, scratch, st);
  } else {
    e = launch_tc(w, xq, sx, M, bias, y, ydtype, ldy, scratch, nullptr, AQ_PHASE_DECODE, st);
  }
  return e == cudaSuccess ? AQ_OK : AQ_ERR_CUDA;
}
