// Long-prefill variant (AlignQuant, App. E.2 and E.3): a mixed projection is
// expanded once into a temporary all-INT8 copy (INT4 codes sign-extended to
// INT8, INT8 tiles copied) and the prefill then runs as a pure INT8 GEMM over
// that copy.  The paper takes this path for long prefills; here it is an
// alternative to expanding INT4 tiles in shared memory inside the prefill
// kernel, over the same packed weights.
//
// The copy is an ordinary packed projection with no INT4 tiles: tile (r, j)
// is INT8 tile r C + j (eq. 16 with every label 0), the bitmap is zero,
// row_off8[r] = r C, row_off4 = 0, and the fp16 scales are the source's own
// buffer (the codes are the same integers, so the scales are unchanged).
//
// One CTA per logical tile; 16-byte loads and stores.  HBM traffic: the source
// payload (bN bK / 2 or bN bK bytes) read and bN bK bytes written per tile.
#include "aq_internal.cuh"

namespace aq {
namespace {

constexpr int kExpThreads = 256;

struct ExpArgs {
  const uint8_t* bitmap;
  const int32_t* tile_idx;
  const uint8_t* w4;
  const int8_t* w8;
  int bN, R, C;
  int8_t* out_w8;         // [R C][bN][128]
  int32_t* out_tile_idx;  // [R C]
  int32_t* out_off8;      // [R + 1]
  int32_t* out_off4;      // [R + 1]
  uint8_t* out_bitmap;    // [ceil(R C / 8)]
};

// 8 nibbles (low nibble = even k, AlignQuant eq. 17) -> 8 sign-extended bytes in k order.
__device__ __forceinline__ uint2 nibbles_to_int8(uint32_t v) {
  const uint32_t lo = __vsub4((v & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);         // even k
  const uint32_t hi = __vsub4(((v >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u, 0x08080808u);  // odd k
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

__global__ void __launch_bounds__(kExpThreads) expand_int8_kernel(ExpArgs a) {
  const int t = blockIdx.x;
  const int r = t / a.C, j = t - r * a.C;
  const bool is4 = (a.bitmap[t >> 3] >> (t & 7)) & 1;
  const size_t p = (size_t)a.tile_idx[t];
  int8_t* dst = a.out_w8 + (size_t)t * a.bN * kTileK;
  if (is4) {
    const uint4* src = reinterpret_cast<const uint4*>(a.w4 + p * a.bN * (kTileK / 2));
    for (int q = threadIdx.x; q < a.bN * (kTileK / 32); q += kExpThreads) {  // 16 source bytes -> 32 codes
      const uint4 v = __ldg(src + q);
      const uint2 e0 = nibbles_to_int8(v.x), e1 = nibbles_to_int8(v.y);
      const uint2 e2 = nibbles_to_int8(v.z), e3 = nibbles_to_int8(v.w);
      uint4* d = reinterpret_cast<uint4*>(dst + (size_t)q * 32);
      d[0] = make_uint4(e0.x, e0.y, e1.x, e1.y);
      d[1] = make_uint4(e2.x, e2.y, e3.x, e3.y);
    }
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(a.w8 + p * a.bN * kTileK);
    uint4* d = reinterpret_cast<uint4*>(dst);
    for (int q = threadIdx.x; q < a.bN * (kTileK / 16); q += kExpThreads) d[q] = __ldg(src + q);
  }
  if (threadIdx.x == 0) {
    a.out_tile_idx[t] = t;
    if ((t & 7) == 0) a.out_bitmap[t >> 3] = 0;
    if (j == 0) {
      a.out_off8[r] = r * a.C;
      a.out_off4[r] = 0;
      if (r == a.R - 1) {
        a.out_off8[a.R] = a.R * a.C;
        a.out_off4[a.R] = 0;
      }
    }
  }
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace

size_t expanded_bytes(const aq_packed* w) {
  const size_t T = (size_t)w->R * w->C;
  return align256(T * w->bN * kTileK) + align256(4 * T) + 2 * align256(4 * ((size_t)w->R + 1)) + align256((T + 7) / 8);
}

cudaError_t launch_expand_int8(const aq_packed* w, void* buf, aq_packed* out, cudaStream_t st) {
  const size_t T = (size_t)w->R * w->C;
  uint8_t* b = static_cast<uint8_t*>(buf);
  int8_t* w8 = reinterpret_cast<int8_t*>(b);
  b += align256(T * w->bN * kTileK);
  int32_t* idx = reinterpret_cast<int32_t*>(b);
  b += align256(4 * T);
  int32_t* off8 = reinterpret_cast<int32_t*>(b);
  b += align256(4 * ((size_t)w->R + 1));
  int32_t* off4 = reinterpret_cast<int32_t*>(b);
  b += align256(4 * ((size_t)w->R + 1));
  uint8_t* bitmap = b;
  *out = *w;
  out->T4 = 0;
  out->T8 = (int32_t)T;
  out->bitmap = bitmap;
  out->row_off4 = off4;
  out->row_off8 = off8;
  out->tile_idx = idx;
  out->w4 = nullptr;
  out->w8 = w8;
  out->scales = w->scales;
  out->scale_kind = AQ_SCALES_ROW_FP16;
  ExpArgs a{w->bitmap, w->tile_idx, w->w4, w->w8, w->bN, w->R, w->C, w8, idx, off8, off4, bitmap};
  expand_int8_kernel<<<(unsigned)T, kExpThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aq
