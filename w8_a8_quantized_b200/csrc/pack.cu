// Packer for the tile-aligned mixed-precision weight format (AlignQuant,
// Sec. 3.2 and App. E.1/E.2).
//
// Host side: precision labels -> bitmap (row-major tiles, eight labels per
// byte, first label in the least significant bit), the two row-offset arrays
// and the physical index of every tile (eq. 16: same-precision tiles in
// earlier tile rows plus same-precision tiles to the left).
// Device side: one CTA per logical tile copies the INT8 tile or nibble-packs
// the INT4 tile (eq. 17: first value in the low nibble) into its precision's
// buffer, checks INT4 codes are in [-8, 7], and copies the tile's fp16 row
// scales into logical tile order (or, for the paper-exact form, the tile's one
// fp32 scale, App. E.2).
#include <vector>

#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kPackThreads = 256;

struct PackArgs {
  const int8_t* codes;
  const uint16_t* scales_in;   // [N][C] fp16 (row scales), or null
  const float* tile_scales_in; // [R][C] fp32 (tile scales), or null
  const uint8_t* map;          // [R][C]
  const int32_t* tile_idx;     // [R*C]
  uint8_t* w4;
  int8_t* w8;
  uint16_t* scales_out;        // [R][C][bN] fp16, or [R][C] fp32 bits
  int N, K, bN, bK, R, C;
  int* err;
};

__global__ void __launch_bounds__(kPackThreads) pack_payload_kernel(PackArgs a) {
  const int t = blockIdx.x;
  const int r = t / a.C, j = t % a.C;
  const bool is4 = a.map[t] != 0;
  const size_t p = (size_t)a.tile_idx[t];
  const int bK = a.bK;
  const int vecs_per_row = bK / 16;  // 16-byte vectors of codes per tile row
  for (int v = threadIdx.x; v < a.bN * vecs_per_row; v += kPackThreads) {
    const int n = v / vecs_per_row, c = v % vecs_per_row;
    const int8_t* src = a.codes + (size_t)(r * a.bN + n) * a.K + (size_t)j * bK + c * 16;
    const int4 q = *reinterpret_cast<const int4*>(src);
    if (!is4) {
      *reinterpret_cast<int4*>(a.w8 + (p * a.bN + n) * bK + c * 16) = q;
    } else {
      const int8_t* b = reinterpret_cast<const int8_t*>(&q);
      uint32_t packed[2] = {0u, 0u};
      bool bad = false;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int q0 = b[2 * i], q1 = b[2 * i + 1];
        bad |= q0 < -8 || q0 > 7 || q1 < -8 || q1 > 7;
        const uint32_t byte = (uint32_t)(q0 & 15) | ((uint32_t)(q1 & 15) << 4);  // eq. 17
        packed[i / 4] |= byte << (8 * (i % 4));
      }
      if (bad) atomicExch(a.err, 1);
      *reinterpret_cast<uint2*>(a.w4 + (p * a.bN + n) * (bK / 2) + c * 8) = make_uint2(packed[0], packed[1]);
    }
  }
  if (a.tile_scales_in != nullptr) {
    if (threadIdx.x == 0) reinterpret_cast<float*>(a.scales_out)[t] = a.tile_scales_in[t];
  } else {
    for (int n = threadIdx.x; n < a.bN; n += kPackThreads)
      a.scales_out[(size_t)t * a.bN + n] = a.scales_in[(size_t)(r * a.bN + n) * a.C + j];
  }
}

}  // namespace

cudaError_t launch_pack_payload(const int8_t* codes, const uint16_t* scales, const float* tile_scales,
                                const aq_packed* out, const uint8_t* map_dev, int* err_dev, cudaStream_t st) {
  PackArgs a{codes, scales, tile_scales, map_dev, out->tile_idx, out->w4, out->w8, out->scales,
             out->N, out->K, out->bN, out->bK, out->R, out->C, err_dev};
  pack_payload_kernel<<<out->R * out->C, kPackThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aq

extern "C" int aq_pack_metadata(const uint8_t* map_host, int R, int C, uint8_t* bitmap, int32_t* row_off4,
                                int32_t* row_off8, int32_t* tile_idx, int32_t* T4_out) {
  if (!map_host || !bitmap || !row_off4 || !row_off8 || !tile_idx || R < 1 || C < 1) return AQ_ERR_ARG;
  const long long T = (long long)R * C;
  for (long long t = 0; t < T; ++t)
    if (map_host[t] > 1) return AQ_ERR_ARG;
  for (long long b = 0; b < (T + 7) / 8; ++b) bitmap[b] = 0;
  row_off4[0] = row_off8[0] = 0;
  for (int r = 0; r < R; ++r) {
    int left4 = 0, left8 = 0;  // same-precision tiles to the left in this row
    for (int j = 0; j < C; ++j) {
      const long long t = (long long)r * C + j;
      if (map_host[t]) {
        bitmap[t >> 3] |= (uint8_t)(1u << (t & 7));
        tile_idx[t] = row_off4[r] + left4++;
      } else {
        tile_idx[t] = row_off8[r] + left8++;
      }
    }
    row_off4[r + 1] = row_off4[r] + left4;
    row_off8[r + 1] = row_off8[r] + left8;
  }
  if (T4_out) *T4_out = row_off4[R];
  return AQ_OK;
}

extern "C" int aq_paper_packed_bytes(int R, int C, int T4, int bN, int bK, size_t* out_bytes) {
  if (!out_bytes || R < 1 || C < 1 || bN < 1 || bK < 1) return AQ_ERR_ARG;
  const unsigned long long B = (unsigned long long)bN * bK, T = (unsigned long long)R * C;
  if ((B & 1) || T4 < 0 || (unsigned long long)T4 > T) return AQ_ERR_ARG;
  const unsigned long long T8 = T - (unsigned long long)T4;
  // eq. 18: payloads, one FP32 scale per tile, labels, two row-offset arrays
  *out_bytes = (size_t)(B * T4 / 2 + B * T8 + 4 * T + (T + 7) / 8 + 8 * ((unsigned long long)R + 1));
  return AQ_OK;
}

// The host part shared by both packers: labels -> metadata (host), then the
// payload kernel.  Exactly one of scales (fp16 row scales) and tile_scales (fp32).
static int pack_common(const int8_t* codes, const uint16_t* scales, const float* tile_scales, const uint8_t* map,
                       int N, int K, int bN, int bK, aq_packed* out, void* stream) {
  using namespace aq;
  const int R = N / bN, C = K / bK;
  const int T = R * C;
  if (((uintptr_t)codes & 15) || ((uintptr_t)out->w8 & 15) || ((uintptr_t)out->w4 & 15)) return AQ_ERR_ARG;
  if (out->T4 < 0 || out->T4 > T) return AQ_ERR_ARG;
  if (!out->bitmap || !out->row_off4 || !out->row_off8 || !out->tile_idx || !out->scales) return AQ_ERR_ARG;
  if ((out->T4 > 0 && !out->w4) || (out->T4 < T && !out->w8)) return AQ_ERR_ARG;
  if (tile_scales != nullptr && ((uintptr_t)out->scales & 3)) return AQ_ERR_ARG;
  // scalar words: tile table (4 B), fp16 row scales (2 B), fp32 tile scales (4 B)
  if (((uintptr_t)out->tile_idx & 3) || ((uintptr_t)out->scales & 1) || ((uintptr_t)scales & 1) ||
      ((uintptr_t)tile_scales & 3))
    return AQ_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  std::vector<uint8_t> map_h(T), bitmap_h((T + 7) / 8);
  std::vector<int32_t> off4_h(R + 1), off8_h(R + 1), idx_h(T);
  if (cudaMemcpyAsync(map_h.data(), map, T, cudaMemcpyDeviceToHost, st) != cudaSuccess) return AQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return AQ_ERR_CUDA;
  int32_t T4 = 0;
  int rc = aq_pack_metadata(map_h.data(), R, C, bitmap_h.data(), off4_h.data(), off8_h.data(), idx_h.data(), &T4);
  if (rc != AQ_OK) return rc;
  if (T4 != out->T4) return AQ_ERR_ARG;

  out->N = N; out->K = K; out->bN = bN; out->bK = bK; out->R = R; out->C = C; out->T8 = T - T4;
  out->scale_kind = tile_scales != nullptr ? AQ_SCALES_TILE_FP32 : AQ_SCALES_ROW_FP16;
  if (cudaMemcpyAsync(out->bitmap, bitmap_h.data(), bitmap_h.size(), cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(out->row_off4, off4_h.data(), 4 * (R + 1), cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(out->row_off8, off8_h.data(), 4 * (R + 1), cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(out->tile_idx, idx_h.data(), 4 * (size_t)T, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return AQ_ERR_CUDA;

  int* err_dev = nullptr;
  if (cudaMalloc(&err_dev, sizeof(int)) != cudaSuccess) return AQ_ERR_CUDA;
  int err_h = 0;
  cudaError_t e = cudaMemsetAsync(err_dev, 0, sizeof(int), st);
  if (e == cudaSuccess) e = launch_pack_payload(codes, scales, tile_scales, out, map, err_dev, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&err_h, err_dev, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaFree(err_dev);
  if (e != cudaSuccess) return AQ_ERR_CUDA;
  return err_h ? AQ_ERR_RANGE : AQ_OK;
}

extern "C" int aq_pack(const int8_t* codes, const uint16_t* scales, const uint8_t* map, int N, int K, int bN,
                       int bK, aq_packed* out, void* stream) {
  if (!codes || !scales || !map || !out) return AQ_ERR_ARG;
  if (!aq::geometry_ok(N, K, bN, bK)) return AQ_ERR_SHAPE;
  return pack_common(codes, scales, nullptr, map, N, K, bN, bK, out, stream);
}

extern "C" int aq_pack_tiles(const int8_t* codes, const float* tile_scales, const uint8_t* map, int N, int K, int bN,
                             int bK, aq_packed* out, void* stream) {
  if (!codes || !tile_scales || !map || !out) return AQ_ERR_ARG;
  if (!aq::paper_geometry_ok(N, K, bN, bK)) return AQ_ERR_SHAPE;
  return pack_common(codes, nullptr, tile_scales, map, N, K, bN, bK, out, stream);
}
