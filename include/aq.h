/*
 * aq.h -- C ABI of libaq: tile-aligned mixed W4/W8 x A8 linear layers on
 * NVIDIA B200 (sm_100a).
 *
 * The operation is the linear projection Y = X W^T of the AlignQuant paper
 * ("AlignQuant: Tile-Aligned Mixed-Precision Quantization for Efficient LLM
 * Generation", arXiv 2610.07457; Sec. 3.1 defines the projection, Sec. 3.2
 * and App. E.1/E.2 the packed representation, Sec. 3.3 and App. E.3 eq. 19
 * the execution).  W (N x K) is cut into equal bN x bK tiles; every tile holds
 * exactly one integer representation, INT4 or INT8, and one fp16 scale per
 * output row.  X (M x K, bf16) is quantized per token to INT8.  The result is
 *
 *     y[m][n] = sx[m] * sum_j sw[n][j] * P[m][n][j]  (+ bias[n])
 *     P[m][n][j] = sum_{k in tile column j} xq[m][k] * q[n][k]   (exact INT32)
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller unless a
 *    comment says "host".  The library never frees caller memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Hot-path calls (aq_quant_act, aq_linear_decode, aq_linear_prefill) are
 *    asynchronous on `stream`: they enqueue kernels and return; they neither
 *    allocate nor synchronize, so they can be recorded into a CUDA graph.
 *  - Arguments are validated on the host before any launch; a rejected call
 *    launches nothing and returns a negative aq_status.  A launch failure
 *    returns AQ_ERR_CUDA.  Errors found by a kernel while it runs (a bounded
 *    wait that gave up) are recorded in the workspace and reported by
 *    aq_workspace_status().
 *  - Geometry: bN in {64, 128}, bK == 128, N % bN == 0, K % bK == 0.  The
 *    paper-exact mode (aq_pack_tiles, aq_paper_*) takes bK == 64 instead.
 *  - Row-major everywhere; leading dimensions are in elements.
 */
#ifndef AQ_H_
#define AQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  AQ_OK = 0,
  AQ_ERR_ARG = -1,         /* null pointer, bad enum, misaligned pointer, M/K/ld out of range */
  AQ_ERR_SHAPE = -2,       /* N, K, bN, bK violate the tile geometry */
  AQ_ERR_RANGE = -3,       /* an INT4 code outside [-8, 7] (aq_pack); a non-finite weight (aq_quantize_weights) */
  AQ_ERR_UNSUPPORTED = -4, /* a valid request this build does not implement */
  AQ_ERR_WORKSPACE = -5,   /* workspace missing or smaller than aq_workspace_bytes() */
  AQ_ERR_CUDA = -6,        /* a CUDA runtime call or a kernel launch failed */
  AQ_ERR_TIMEOUT = -7      /* a kernel gave up on a bounded wait (see aq_workspace_status) */
} aq_status;

typedef enum { AQ_F32 = 0, AQ_BF16 = 1 } aq_dtype;
typedef enum { AQ_PHASE_DECODE = 0, AQ_PHASE_PREFILL = 1 } aq_phase;

/*
 * One packed projection (App. E.1, E.2).  Every pointer is a device buffer
 * owned by the caller and sized by aq_packed_sizes(); aq_pack() fills them.
 *
 *  bitmap   uint8  [ceil(R*C/8)]   precision label beta_{r,j} of logical tile
 *                                  t = r*C + j is bit (t % 8) of byte t / 8
 *                                  (row-major order, first label in the LSB);
 *                                  beta = 1 marks an INT4 tile.
 *  row_off4 int32  [R+1]           INT4 tiles in tile rows < r (eq. 16, first sum)
 *  row_off8 int32  [R+1]           INT8 tiles in tile rows < r
 *  tile_idx int32  [R*C]           physical index of logical tile t inside its
 *                                  precision's buffer (eq. 16 evaluated once)
 *  w4       uint8  [T4][bN][bK/2]  INT4 tiles in row order; byte i of a tile row
 *                                  holds k = 2i in its low nibble and k = 2i+1 in
 *                                  its high nibble (eq. 17), two's complement
 *  w8       int8   [T8][bN][bK]    INT8 tiles in row order, row-major in the tile
 *  scales   fp16   [R][C][bN]      sw[n][j] at (r*C + j)*bN + (n - r*bN), bits
 *                                  as uint16, logical tile order
 *           (scale_kind == AQ_SCALES_TILE_FP32: fp32 [R][C], one scale per tile
 *                                  at r*C + j, in the first 4*R*C bytes of the
 *                                  same buffer; written by aq_pack_tiles)
 *  scale_kind                      AQ_SCALES_ROW_FP16 (aq_pack; the per-token
 *                                  layer's kernels take only this kind) or
 *                                  AQ_SCALES_TILE_FP32 (aq_pack_tiles; the
 *                                  paper-exact aq_paper_linear takes only this)
 *
 * Inside a tile both precisions use the same element order: output row, then
 * input column.  w4, w8 and scales must start on a 16-byte boundary (the
 * kernels move them with bulk copies; fp32 tile scales need only 4 bytes) and
 * tile_idx on a 4-byte one; a packed layout that breaks this is rejected with
 * AQ_ERR_ARG.
 */
typedef enum { AQ_SCALES_ROW_FP16 = 0, AQ_SCALES_TILE_FP32 = 1 } aq_scale_kind;

typedef struct aq_packed {
  int32_t N, K, bN, bK, R, C, T4, T8;
  uint8_t* bitmap;
  int32_t* row_off4;
  int32_t* row_off8;
  int32_t* tile_idx;
  uint8_t* w4;
  int8_t* w8;
  uint16_t* scales;
  int32_t scale_kind;  /* aq_scale_kind; set by the packers (zero-initialize a struct built by hand) */
} aq_packed;

/* Index of each buffer in the size array of aq_packed_sizes(). */
enum {
  AQ_BUF_BITMAP = 0, AQ_BUF_ROW_OFF4 = 1, AQ_BUF_ROW_OFF8 = 2, AQ_BUF_TILE_IDX = 3,
  AQ_BUF_W4 = 4, AQ_BUF_W8 = 5, AQ_BUF_SCALES = 6, AQ_NUM_BUFS = 7
};

/* Human-readable name of a status code (static string, never NULL). */
const char* aq_status_str(int status);

/*
 * Host only, no CUDA call.  Byte size of each of the seven packed buffers for
 * an N x K projection with bN x bK tiles of which T4 are INT4.
 * out_bytes: host array of AQ_NUM_BUFS entries.
 * Either geometry is accepted (bK == 128, or bK == 64 for aq_pack_tiles).
 * Errors: AQ_ERR_ARG (null out_bytes, T4 outside [0, R*C]), AQ_ERR_SHAPE.
 */
int aq_packed_sizes(int N, int K, int bN, int bK, int T4, size_t* out_bytes);

/*
 * Host only, no CUDA call.  Storage of a packed projection as the paper
 * accounts it (eq. 18, App. E.2): payloads B*T4/2 + B*T8 with B = bN*bK, one
 * 4-byte scale per tile, ceil(R*C/8) label bytes and two (R+1)-entry 4-byte
 * row-offset arrays; T8 = R*C - T4.  Summing it over a model's quantized
 * projections, times 8, over their weight count gives the packed bits per
 * weight of App. G.7 / Table 16.  Any tile shape (bN, bK >= 1, bN*bK even) is
 * accepted; this is accounting only and differs from aq_packed_sizes (fp16
 * scale per row per tile, plus the physical-index table).
 * Errors: AQ_ERR_ARG (null out_bytes, R, C, bN or bK < 1, odd bN*bK, T4 outside
 * [0, R*C]).
 */
int aq_paper_packed_bytes(int R, int C, int T4, int bN, int bK, size_t* out_bytes);

/*
 * Host only, no CUDA call.  Metadata of the packed format from a HOST copy of
 * the precision labels map[R][C] (1 = INT4, 0 = INT8): bitmap, both row-offset
 * arrays and tile_idx, written to HOST buffers of the sizes aq_packed_sizes()
 * gives.  *T4_out (nullable) receives the INT4 tile count.
 * Errors: AQ_ERR_ARG (null pointer, R or C < 1, a label other than 0 or 1).
 * Follows App. E.1 and eq. 16.
 */
int aq_pack_metadata(const uint8_t* map_host, int R, int C, uint8_t* bitmap, int32_t* row_off4,
                     int32_t* row_off8, int32_t* tile_idx, int32_t* T4_out);

/*
 * Pack integer codes into the tile format (App. E.1, E.2; eq. 16, 17).
 *  codes  int8  [N][K] device, row-major, 16-byte aligned: INT8 tiles any value, INT4 tiles in [-8, 7]
 *  scales fp16  [N][C] device (bits as uint16), 2-byte aligned, sw[n][j]
 *  map    uint8 [R][C] device, 1 = INT4 tile, 0 = INT8 tile
 *  out    host struct whose seven pointers the caller set to device buffers of
 *         aq_packed_sizes(N, K, bN, bK, out->T4) bytes; out->T4 must equal the
 *         number of INT4 labels in map; the buffers aligned as the struct's
 *         description states.  The remaining fields are filled in.
 * Offline step: synchronizes `stream` and allocates a few bytes of temporary
 * device memory.  Errors: AQ_ERR_ARG (also when out->T4 disagrees with map, or
 * a pointer is misaligned),
 * AQ_ERR_SHAPE, AQ_ERR_RANGE (an INT4 tile holds a code outside [-8, 7]; the
 * output buffers are then unspecified), AQ_ERR_CUDA.
 */
int aq_pack(const int8_t* codes, const uint16_t* scales, const uint8_t* map, int N, int K, int bN,
            int bK, aq_packed* out, void* stream);

/*
 * Paper-exact packing (App. B.2, E.2): the same format as aq_pack with ONE
 * fp32 scale per whole tile (the paper's FP32 tile scale) and 64-wide tiles.
 *  codes        int8  [N][K] device, as for aq_pack
 *  tile_scales  fp32  [R][C] device, s^W_{r,j}
 *  map          uint8 [R][C] device, 1 = INT4 tile, 0 = INT8 tile
 *  out          as for aq_pack, buffers of aq_packed_sizes(N, K, bN, bK, T4)
 *               bytes; the scales buffer receives the fp32 tile scales and
 *               out->scale_kind = AQ_SCALES_TILE_FP32.
 * Geometry: bN in {64, 128}, bK == 64, N % bN == 0, K % bK == 0.
 * Offline step: synchronizes `stream`.  Errors as for aq_pack.
 */
int aq_pack_tiles(const int8_t* codes, const float* tile_scales, const uint8_t* map, int N, int K, int bN, int bK,
                  aq_packed* out, void* stream);

/*
 * Float weights -> integer codes and scales for aq_pack (App. B.2, eq. 5-7),
 * one scale per output row per tile.  For row n of tile (r, j), A = the bK
 * values w[n][j*bK .. j*bK+bK-1] and b = 4 (INT4 label) or 8 (INT8 label):
 *   s0 = max(max(0, max A) / (2^(b-1) - 1), max(0, -min A) / 2^(b-1), 1e-12)   (eq. 6)
 *   search == 0: s* = s0
 *   search == 1: s* = the s_i = max((1/4 + i/128) s0, 1e-12), i = 0..128, with
 *                the least sum_k (A_k - s_i Q_k)^2, earliest i on ties      (eq. 7)
 *   codes[n][k] = clip(rint(A_k / s*), -2^(b-1), 2^(b-1) - 1)            (eq. 5)
 *   scales[n][j] = fp16(s*), rounded to nearest even from fp64
 * in fp64, each operation rounded separately, error sums in increasing k.
 *  w      fp32 or bf16 (wdtype, aq_dtype) [N][ldw] device, 16-byte aligned,
 *         ldw >= K, ldw % 4 == 0 (fp32) or ldw % 8 == 0 (bf16); read only
 *  map    uint8 [R][C] device, 1 = INT4 tile, 0 = INT8 tile
 *  codes  int8  [N][K] device, 16-byte aligned (written)
 *  scales fp16  [N][C] device, bits as uint16, 2-byte aligned (written)
 * Offline step: synchronizes `stream` and allocates a few bytes of temporary
 * device memory.  Errors: AQ_ERR_ARG (null or misaligned pointer, bad wdtype
 * or search, ldw out of range, a label other than 0 or 1), AQ_ERR_SHAPE,
 * AQ_ERR_RANGE (a weight is NaN or infinite; outputs then unspecified),
 * AQ_ERR_CUDA.
 */
int aq_quantize_weights(const void* w, int wdtype, int N, int K, int ldw, int bN, int bK, const uint8_t* map,
                        int search, int8_t* codes, uint16_t* scales, void* stream);

/*
 * Per-token symmetric INT8 quantization of activations (App. B.3 computed per
 * token; eq. 5 rounding; eq. 6 floor), in fp64:
 *   s = max(max_k |x[m][k]| / 127, 1e-12);  xq[m][k] = clamp(rint(x[m][k] / s), -127, 127)
 *   sx[m] = (float)s          (codes use the fp64 s; rint rounds half to even)
 *  x   bf16 [M][ldx] device (bits as uint16), 16-byte aligned, ldx % 8 == 0, ldx >= K
 *  xq  int8 [M][K] device, 16-byte aligned
 *  sx  fp32 [M] device, 4-byte aligned
 * 1 <= M, 16 <= K <= 1048576 with K % 16 == 0.  Errors: AQ_ERR_ARG, AQ_ERR_CUDA.
 */
int aq_quant_act(const uint16_t* x, int M, int K, int ldx, int8_t* xq, float* sx, void* stream);

/*
 * Long-prefill variant (App. E.2, E.3): the paper expands a mixed projection
 * once per call into a temporary INT8 buffer and then runs a pure INT8 GEMM.
 *
 * aq_expanded_bytes: host only; bytes of the all-INT8 copy of *w (payload
 * R*C*bN*bK, tile table 4*R*C, two offset arrays 4*(R+1) each, bitmap
 * ceil(R*C/8), each rounded up to 256 bytes); 0 when *w is invalid.
 *
 * aq_expand_int8: writes that copy into the caller's device buffer `buf`
 * (256-byte aligned, >= aq_expanded_bytes bytes) and describes it in *out
 * (host struct): T4 = 0, every tile INT8 (INT4 codes sign-extended, INT8
 * tiles copied), tile (r, j) at index r*C + j, and out->scales = w->scales
 * (shared, not copied).  *out is valid while `buf` and w's scales live.
 * Asynchronous on `stream`; no allocation, no synchronization.
 * Errors: AQ_ERR_ARG (null or misaligned pointer), AQ_ERR_SHAPE,
 * AQ_ERR_WORKSPACE (buffer too small), AQ_ERR_CUDA.
 *
 * aq_linear_prefill_expanded: aq_linear_prefill with the expansion done
 * first into `tmp` (as aq_expand_int8, tmp_bytes >= aq_expanded_bytes(w)),
 * both kernels on `stream`.  The results equal aq_linear_prefill's bit for
 * bit.  Errors: as aq_linear_prefill, plus AQ_ERR_ARG / AQ_ERR_WORKSPACE for tmp.
 */
size_t aq_expanded_bytes(const aq_packed* w);
int aq_expand_int8(const aq_packed* w, void* buf, size_t buf_bytes, aq_packed* out, void* stream);
int aq_linear_prefill_expanded(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias,
                               void* y, int ydtype, int ldy, void* ws, size_t ws_bytes, void* tmp, size_t tmp_bytes,
                               void* stream);

/*
 * Activation quantization in the paper's own form (App. B.3; eq. 5, eq. 6 with
 * b = 8), the activation side of its paper-exact numerics: one scale per
 * group of 64 features and b_M rows, b_M = aq_act_group_rows(M) (1 for
 * M = 1, else 16), rows zero-padded to M' = ceil(M / b_M) * b_M:
 *   s = max(max(0, max A) / 127, max(0, -min A) / 128, 1e-12)   over group A
 *   xq = clamp(rint(x / s), -128, 127) (fp64 quotient)            sx = (float)s
 *  x   bf16 [M][ldx] device (bits as uint16), 16-byte aligned, ldx % 8 == 0, ldx >= K
 *  xq  int8 [M'][K] device, 8-byte aligned; padding rows receive zero codes
 *  sx  fp32 [M' / b_M][K / 64] device, row-major, 4-byte aligned
 * 1 <= M, 64 <= K <= 1048576 with K % 64 == 0.  Asynchronous on `stream`.
 * Errors: AQ_ERR_ARG, AQ_ERR_CUDA.  aq_act_group_rows: host only, b_M (0 for M < 1).
 */
int aq_act_group_rows(int M);
int aq_quant_act_groups(const uint16_t* x, int M, int K, int ldx, int8_t* xq, float* sx, void* stream);

/*
 * Paper-exact activation preparation (App. B.1 eq. 4, App. B.3): the
 * transformed activations X~ = X V with V = diag(V_0, V_1, ...), one 64 x 64
 * block per 64 input features, then the groups of aq_quant_act_groups on X~:
 *   x~[m][64c + k] = sum_{i=0..63} x[m][64c + i] * V_c[i][k]      (fp64)
 *   per group A of 64 features x b_M rows of X~ (rows zero-padded to M'):
 *   s = max(max(0, max A) / 127, max(0, -min A) / 128, 1e-12)
 *   xq = clamp(rint(x~ / s), -128, 127) (fp64 quotient)     sx = (float)s
 *  x   bf16 [M][ldx] (bits as uint16), 2-byte aligned
 *  v   fp32 [K/64][64][64], V_c[i][k] at (c*64 + i)*64 + k, 16-byte aligned; NULL = identity
 *      (then the result equals aq_quant_act_groups).  The sums are formed in
 *      fp64; with the paper's transform seeds (entries 0, +-1, +-1/8) and
 *      bf16 inputs they are exact, so the codes do not depend on the order.
 *  xq  int8 [M'][K], sx fp32 [M'/b_M][K/64] (4-byte aligned), M' = ceil(M / b_M) * b_M.
 * Asynchronous.  Errors: AQ_ERR_ARG (null x / xq / sx, misaligned x / v / sx,
 * M < 1, K < 64, K % 64, ldx < K), AQ_ERR_CUDA.
 */
int aq_paper_quant_act(const uint16_t* x, int M, int K, int ldx, const float* v, int8_t* xq, float* sx,
                       void* stream);

/*
 * Paper-exact linear layer (App. E.3 eq. 19, then App. B.1 eq. 4):
 *   y~[m][n] = sum_j sx[m / b_M][j] * sw[n / bN][j] * P[m][n][j]   (fp32, j ascending)
 *   P[m][n][j] = sum_{k in tile column j} xq[m][k] * q[n][k]       (exact INT32)
 *   y[m][r*bN + c] = sum_{i < bN} y~[m][r*bN + i] * U_r[i][c]  (+ bias[r*bN + c])
 *  w     a projection packed by aq_pack_tiles (bK == 64, per-tile fp32 scales)
 *  xq    int8 [M'][K] (16-byte aligned) and sx fp32 [M'/b_M][K/64] as aq_paper_quant_act
 *        writes them; every fp32 pointer here (sx, u, bias, y) 4-byte aligned
 *  u     fp32 [R][bN][bN], U_r[i][c] at (r*bN + i)*bN + c; NULL = identity
 *  bias  fp32 [N] or NULL
 *  y     fp32 [M][ldy]; rows m < M are written, nothing else
 * Any M >= 1 (the CUDA cores compute it; it is the numerics reference of the
 * paper's own construction, not the per-token layer's fast path).
 * Asynchronous, no workspace.  Errors: AQ_ERR_ARG (null or misaligned pointer,
 * M < 1, M > 1,048,560 (65,535 row groups), ldy < N, a packed struct of the
 * other scale kind), AQ_ERR_SHAPE, AQ_ERR_CUDA.
 */
int aq_paper_linear(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* u, const float* bias,
                    float* y, int ldy, void* stream);

/*
 * Test entry: the exact integer tile products P[m][n][j] (int32 [M][N][K/64])
 * of aq_paper_linear, as its kernel forms them (P 4-byte aligned).  Errors as
 * aq_paper_linear.
 */
int aq_debug_paper_partials(const aq_packed* w, const int8_t* xq, int M, int32_t* P, void* stream);

/*
 * Device scratch bytes a linear call needs for `phase` (aq_phase) at M tokens
 * with packed weights *w (host struct; only its geometry is read).  Host only.
 * The workspace must be zero-filled once when allocated; afterwards the library
 * leaves it ready for the next call.  Calls that share a workspace must not run
 * concurrently.  Returns 0 when the arguments are invalid.
 */
size_t aq_workspace_bytes(int phase, int M, const aq_packed* w);

/*
 * Decode-phase linear layer, 1 <= M <= 64 (Sec. 3.3 "Decode parallelism";
 * App. E.3 eq. 19 and the ordered split reduction after it).
 *  w     host struct describing device buffers produced by aq_pack
 *  xq    int8 [M][K] device, 16-byte aligned (from aq_quant_act)
 *  sx    fp32 [M] device, 4-byte aligned
 *  bias  fp32 [N] device, 4-byte aligned, or NULL
 *  y     [M][ldy] device, fp32 or bf16 per ydtype (aq_dtype), aligned to its
 *        element, ldy >= N
 *  ws    device workspace of >= aq_workspace_bytes(AQ_PHASE_DECODE, M, w) bytes,
 *        16-byte aligned
 * Split-K partial sums are reduced in increasing split order, so results are
 * bitwise reproducible for a given (M, w) on a given GPU.
 * Errors: AQ_ERR_ARG (also a misaligned pointer), AQ_ERR_SHAPE,
 * AQ_ERR_WORKSPACE (ws NULL or too small), AQ_ERR_CUDA.
 */
int aq_linear_decode(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias,
                     void* y, int ydtype, int ldy, void* ws, size_t ws_bytes, void* stream);

/*
 * Prefill-phase linear layer, any M >= 1 (Sec. 3.3 "Prefill weight reuse";
 * App. E.3 eq. 19).  Same arguments as aq_linear_decode; the workspace size is
 * aq_workspace_bytes(AQ_PHASE_PREFILL, M, w).  INT4 tiles are expanded to INT8
 * on chip and the INT8 products run on the tensor cores (tcgen05).
 * Errors: AQ_ERR_ARG, AQ_ERR_SHAPE, AQ_ERR_WORKSPACE, AQ_ERR_CUDA.
 */
int aq_linear_prefill(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias,
                      void* y, int ydtype, int ldy, void* ws, size_t ws_bytes, void* stream);

/*
 * Test entry: the exact per-tile INT32 products P[m][n][j] (eq. 19, the
 * parenthesized product) written to P int32 [M][N][C] device (4-byte aligned), computed by the
 * same data path (tile location, INT4 expansion, integer products) as the
 * linear call of `phase`.  Not a hot-path call.
 * Errors: AQ_ERR_ARG, AQ_ERR_SHAPE, AQ_ERR_WORKSPACE, AQ_ERR_CUDA.
 */
int aq_debug_tile_partials(const aq_packed* w, const int8_t* xq, int M, int phase, int32_t* P,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * Test entry for the failure path of the tensor-core linear kernel (the one that
 * runs prefill and decode from 4 tokens): it runs that kernel with a stage that
 * can never fill, without any invalid memory access.  The weight producer stops
 * after `stop_after` input tiles, so the MMA issuer's wait for the next stage,
 * and then every other role's wait, runs out; every bounded wait gives up after
 * `wait_ns` (100 us .. 10 s) instead of the normal 2 s.  The kernel records
 * AQ_ERR_TIMEOUT in `ws` with the code of the first wait that gave up, frees
 * its tensor memory and returns; y (fp32 [M][ldy]) is then unspecified.
 * aq_workspace_status() reports the error and restores the workspace (error
 * word and split-K counters), after which the workspace serves ordinary calls.
 * phase: AQ_PHASE_PREFILL, or AQ_PHASE_DECODE with an M that the tensor-core
 * kernel serves.  Not a hot-path call.
 * Errors: AQ_ERR_ARG, AQ_ERR_SHAPE, AQ_ERR_WORKSPACE, AQ_ERR_CUDA.
 */
int aq_debug_linear_stalled(const aq_packed* w, const int8_t* xq, const float* sx, int M, int phase, float* y,
                            int ldy, void* ws, size_t ws_bytes, unsigned long long wait_ns, int stop_after,
                            void* stream);

/*
 * Shared-input projection group (Sec. 3.3 "Shared activation preparation";
 * App. E.4): G (1..3) projections that read the same activations, e.g. query /
 * key / value or gate / up, prepared once and computed in as few launches as
 * possible.  For every member g:  y[g] = linear(w[g], quant(x)) (+ bias[g]),
 * exactly as aq_quant_act followed by aq_linear_decode / aq_linear_prefill.
 *  phase  AQ_PHASE_DECODE (1 <= M <= 64) or AQ_PHASE_PREFILL (M >= 1)
 *  w      host array of G pointers to packed projections with equal K
 *  x      bf16 [M][ldx] device (bits as uint16), 16-byte aligned, ldx % 8 == 0
 *  bias   host array of G device pointers (each fp32 [N_g], 4-byte aligned, or NULL), or NULL
 *  y      host array of G device outputs [M][ldy[g]], fp32 or bf16 per ydtype, aligned to
 *         their element
 *  ldy    host array of G leading dimensions, ldy[g] >= N_g
 *  ws     device workspace of >= aq_group_workspace_bytes(phase, M, w, G) bytes, 16-byte aligned
 * Decode with one or two tokens runs as ONE launch where the codes fit in
 * shared memory: every CTA quantizes the input it needs itself (same
 * arithmetic as aq_quant_act) and the members' output rows are concatenated.
 * Otherwise x is quantized once into the workspace and the members run on it,
 * in one launch over all their rows where the decode plan allows it (the
 * CUDA-core kernel up to 3 tokens, and for three members up to 8 tokens; the
 * tensor-core kernel from 4 tokens when every member has whole 128-row blocks
 * and all share one tile height), else in one launch per member.
 * Errors: AQ_ERR_ARG (also G outside 1..3, unequal K), AQ_ERR_SHAPE,
 * AQ_ERR_WORKSPACE, AQ_ERR_CUDA.
 */
int aq_linear_group(int phase, const aq_packed* const* w, int G, const uint16_t* x, int ldx, int M,
                    const float* const* bias, void* const* y, const int* ldy, int ydtype, void* ws,
                    size_t ws_bytes, void* stream);

/* Host only.  Workspace bytes of aq_linear_group(phase, ..., M, w, G); 0 when invalid. */
size_t aq_group_workspace_bytes(int phase, int M, const aq_packed* const* w, int G);

/*
 * Decode-phase linear layer for callers that cannot allocate device memory
 * (code running inside an allocator or memory-pool callback, runtimes that
 * forbid allocation after start-up to keep a fixed footprint, plug-ins handed
 * only their input and output buffers).  The paper has no counterpart: this is
 * a deployment convenience of this library.
 *
 * Same arguments and result as aq_linear_decode, without the workspace: the
 * split-K scratch comes from a fixed 4 MiB array in device memory that the
 * library holds on every GPU that loads it, until the process exits.
 *  - Allocates nothing and calls no allocating routine.
 *  - The first call on a device resolves the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture on the device.  The address is kept for the
 *    process: after a cudaDeviceReset of that device it is stale, and this
 *    entry must not be called on that device again.
 *  - Each call clears the parts of the array that must start at zero (status
 *    word, split-K counters) on `stream` before launching.
 *  - All calls share the one array: calls that overlap on the GPU (different
 *    streams, or graphs replayed concurrently) race and produce wrong results.
 *  - A call whose scratch need (aq_workspace_bytes(AQ_PHASE_DECODE, M, w))
 *    exceeds 4 MiB is rejected with AQ_ERR_WORKSPACE; use aq_linear_decode.
 *  - No status query exists for this array; a bounded wait that gives up
 *    inside the kernel leaves y unspecified.
 * Errors: AQ_ERR_ARG, AQ_ERR_SHAPE, AQ_ERR_WORKSPACE, AQ_ERR_CUDA.
 */
int aq_linear_decode_noalloc(const aq_packed* w, const int8_t* xq, const float* sx, int M, const float* bias,
                             void* y, int ydtype, int ldy, void* stream);

/*
 * Measurement helper, not part of the layer: the dense INT8 tensor-core rate of
 * the current GPU.  One CTA per SM issues `iters` x 4 back-to-back
 * tcgen05.mma.kind::i8 instructions (M = 128, N = 256, K = 32, INT32
 * accumulators in tensor memory) on operands resident in shared memory; *tops
 * (host) receives 2 M N K x instructions / elapsed seconds / 1e12 (CUDA events
 * around one launch, after a shorter warm-up launch).  Synchronizes `stream`
 * and allocates 4 bytes of device memory.  1 <= iters <= 2^22; about 20000
 * runs for a few milliseconds on a B200.
 * Errors: AQ_ERR_ARG, AQ_ERR_CUDA, AQ_ERR_TIMEOUT (the completion wait gave up).
 */
int aq_measure_i8_peak(int iters, double* tops, void* stream);

/*
 * Synchronizes `stream`, then reads and clears the error word a kernel left in
 * the workspace `ws`.  Returns AQ_OK, AQ_ERR_TIMEOUT (a bounded wait inside a
 * kernel gave up; *info, nullable, receives where) or AQ_ERR_CUDA.
 */
int aq_workspace_status(void* ws, void* stream, int* info);

#ifdef __cplusplus
}
#endif

#endif /* AQ_H_ */
