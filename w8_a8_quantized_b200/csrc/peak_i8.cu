// Dense INT8 tensor-core throughput of this GPU, measured: the denominator the
// benchmark reports the prefill kernel's INT8 rate against.
//
// One CTA per SM keeps an M = 128 x N = 256 INT32 accumulator in tensor memory
// and issues tcgen05.mma.cta_group::1.kind::i8 (K = 32 per instruction) back to
// back from one thread, on operands that stay in shared memory (a 128 x 128
// weight block and a 256 x 128 activation block in the 128-byte-swizzled K-major
// layout the prefill kernel uses).  Nothing else runs: no loads, no epilogue.
// The result is 2 x 128 x 256 x 32 operations per instruction over the elapsed
// time of the launch (CUDA events around it).
#include <algorithm>

#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kPeakM = 128, kPeakN = 256, kPeakK = 128;  // K of the resident blocks (4 instructions)
constexpr int kPeakThreads = 128;
constexpr size_t kPeakSmem = 1024 + (size_t)(kPeakM + kPeakN) * kPeakK + 64;
constexpr uint32_t kPeakIdesc = idesc_i8(kPeakM, kPeakN);

__global__ void __launch_bounds__(kPeakThreads) i8_peak_kernel(int iters, int* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* a_blk = smem;                      // [128][128] int8
  uint8_t* b_blk = smem + kPeakM * kPeakK;    // [256][128] int8
  uint64_t* done = reinterpret_cast<uint64_t*>(b_blk + kPeakN * kPeakK);
  __shared__ uint32_t tmem_slot;
  __shared__ int never;

  // small nonzero operands (the values do not change the throughput)
  for (int i = threadIdx.x; i < (kPeakM + kPeakN) * kPeakK / 4; i += kPeakThreads)
    reinterpret_cast<uint32_t*>(smem)[i] = 0x01010101u * (uint32_t)((i * 7) & 3);
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    never = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();  // generic-proxy writes -> visible to the MMA's async proxy
  if (threadIdx.x < 32) {
    tmem_alloc(&tmem_slot, kPeakN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 0) {
    const uint64_t adesc = sw128_desc(smem_u32(a_blk)), bdesc = sw128_desc(smem_u32(b_blk));
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int k = 0; k < kPeakK / 32; ++k)  // K = 32 bytes per instruction: +2 in 16-byte units
        mma_i8(tmem, adesc + 2 * k, bdesc + 2 * k, kPeakIdesc, (it | k) != 0);
    }
    mma_commit(done);
    if (!mbar_wait(done, 0, &never)) atomicExch(err, 1);  // bounded: records and goes on
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, kPeakN);
  }
}

}  // namespace
}  // namespace aq

using namespace aq;

extern "C" int aq_measure_i8_peak(int iters, double* tops, void* stream) {
  if (!tops || iters < 1 || iters > (1 << 22)) return AQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (ensure_smem_attr<i8_peak_kernel>((int)kPeakSmem) != cudaSuccess) return AQ_ERR_CUDA;
  int* err = nullptr;
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  int rc = AQ_OK;
  if (cudaMalloc(&err, sizeof(int)) != cudaSuccess || cudaMemsetAsync(err, 0, sizeof(int), st) != cudaSuccess ||
      cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) {
    rc = AQ_ERR_CUDA;
  } else {
    const int grid = num_sms();
    i8_peak_kernel<<<grid, kPeakThreads, kPeakSmem, st>>>(std::max(1, iters / 8), err);  // warm-up
    cudaEventRecord(e0, st);
    i8_peak_kernel<<<grid, kPeakThreads, kPeakSmem, st>>>(iters, err);
    cudaEventRecord(e1, st);
    float ms = 0.f;
    int h_err = 0;
    if (cudaEventSynchronize(e1) != cudaSuccess || cudaEventElapsedTime(&ms, e0, e1) != cudaSuccess ||
        cudaMemcpy(&h_err, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
      rc = AQ_ERR_CUDA;
    } else if (h_err != 0) {
      rc = AQ_ERR_TIMEOUT;
    } else {
      const double ops = 2.0 * kPeakM * kPeakN * 32 * (kPeakK / 32) * (double)iters * grid;
      *tops = ops / (ms * 1e-3) / 1e12;
    }
  }
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  if (err) cudaFree(err);
  return rc;
}
