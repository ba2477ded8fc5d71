"""CPU oracle for the tile-aligned mixed W4/W8 x A8 linear layer.

TEST INFRASTRUCTURE ONLY.  This module is imported by the tests, by the
``smoke()`` check and by the CPU-baseline leg of the benchmark; the product
path (the CUDA library and its Python binding) never imports or calls it.  It
shares no code with the CUDA path.

It is a plain, slow, directly checkable restatement of what the method
computes, written from the AlignQuant paper ("AlignQuant: Tile-Aligned
Mixed-Precision Quantization for Efficient LLM Generation", arXiv 2610.07457),
with fp64 for every floating-point step:

* the packed representation of App. E.1 / E.2: a one-bit precision label per
  tile (row-major tile order, first label in the least significant bit),
  separate contiguous INT4 and INT8 tile buffers in row order, two INT32
  row-offset arrays of length R+1 (eq. 16 gives the physical index), INT4
  values nibble-packed with the first value in the low nibble (eq. 17);
* per-token symmetric INT8 activation quantization (absmax / 127, round half
  to even, clamp to +-127, scale floored at 1e-12 as in eq. 6), computed in
  fp64 as App. B.3 prescribes for the CUDA preparation;
* per-tile INT32 products of INT8 activations with INT8 (or sign-extended
  INT4) weights, rescaled by the activation and weight scales and summed
  over input tiles (eq. 19, Sec. 3.3 "Output reconstruction").

Readings where the paper is silent or differs from this layer's definition
(each one is listed with its reason in the design notes):
  * weight scales are fp16, one per output row per tile (the paper stores one
    FP32 scale per tile); they are stored in logical tile order
    ``scales[r][j][n_local]``;
  * one activation scale per token over all K (the paper groups 64 features
    x b_M rows) with a symmetric +-127 range (the paper's eq. 6 uses
    asymmetric endpoints);
  * the in-tile element order is row-major (output row, then input column)
    for both precisions; the paper permutes into a CUTLASS layout but keeps
    one order for both precisions, which is kept;
  * the transforms U and V are the identity (the paper's seed Phi_{-1} = I);
  * the float-weight quantizer of App. B.2 (eq. 5-7) is applied to each output
    row of each tile (the scale granularity of this layer) rather than to a
    whole tile; its error sums run over the row's columns in increasing order,
    and the selected fp64 scale is stored rounded to fp16 (the paper stores
    FP32).

Every function here is pinned by the CPU tests to values the paper prints
(the eq. 16 worked example, Table 16's bits per weight through eq. 18), to
hand-derived bytes of eq. 17 and of the label order, and to brute force on
tiny inputs.
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# Packed representation (App. E.1, E.2)
# ---------------------------------------------------------------------------

W4 = 1  # precision label beta = 1 marks a 4-bit tile (App. E.1)
W8 = 0


def labels_to_bitmap(pmap: np.ndarray) -> np.ndarray:
    """Precision labels -> bytes: row-major tile order, eight labels per byte,
    first label in the least significant bit (App. E.1)."""
    flat = [int(v) for v in np.asarray(pmap, dtype=np.uint8).reshape(-1)]
    out = np.zeros((len(flat) + 7) // 8, dtype=np.uint8)
    for t, beta in enumerate(flat):
        if beta:
            out[t // 8] |= np.uint8(1 << (t % 8))
    return out


def label_of(bitmap: np.ndarray, r: int, j: int, C: int) -> int:
    """beta_{r,j} read back from the bitmap (App. E.1)."""
    t = r * C + j
    return (int(bitmap[t // 8]) >> (t % 8)) & 1


def physical_index(pmap: np.ndarray, r: int, j: int, b: int) -> int:
    """eq. 16: tiles of precision b in earlier tile rows (the stored row
    offset) plus tiles of precision b to the left in the same row."""
    want = W4 if b == 4 else W8
    R, C = pmap.shape
    before_rows = sum(1 for rp in range(r) for jp in range(C) if pmap[rp, jp] == want)
    in_row = sum(1 for jp in range(j) if pmap[r, jp] == want)
    return before_rows + in_row


def row_offsets(pmap: np.ndarray, b: int) -> np.ndarray:
    """INT32 row-offset array of length R+1 for precision b (App. E.1, E.2)."""
    want = W4 if b == 4 else W8
    R, C = pmap.shape
    off = np.zeros(R + 1, dtype=np.int32)
    for r in range(R):
        off[r + 1] = off[r] + sum(1 for j in range(C) if pmap[r, j] == want)
    return off


def nibble_byte(q0: int, q1: int) -> int:
    """eq. 17: byte(q0, q1) = (q0 mod 16) + 16 (q1 mod 16)."""
    return (q0 % 16) + 16 * (q1 % 16)


def nibble_value(v: int) -> int:
    """App. E.1: a nibble v expands to v if v < 8, else to v - 16."""
    return v if v < 8 else v - 16


def pack(codes: np.ndarray, scales: np.ndarray, pmap: np.ndarray, bN: int, bK: int) -> dict:
    """Integer codes + per-row-per-tile scales + precision labels -> packed
    projection.  INT4 tiles must hold codes in [-8, 7] (checked)."""
    codes = np.asarray(codes, dtype=np.int8)
    N, K = codes.shape
    R, C = N // bN, K // bK
    assert R * bN == N and C * bK == K and pmap.shape == (R, C) and bK % 2 == 0
    T4 = int((pmap == W4).sum())
    T8 = R * C - T4
    w4 = np.zeros((T4, bN, bK // 2), dtype=np.uint8)
    w8 = np.zeros((T8, bN, bK), dtype=np.int8)
    tile_idx = np.zeros(R * C, dtype=np.int32)
    off4, off8 = row_offsets(pmap, 4), row_offsets(pmap, 8)
    for r in range(R):
        left4 = left8 = 0          # same-precision tiles to the left (eq. 16, 2nd sum)
        for j in range(C):
            tile = codes[r * bN:(r + 1) * bN, j * bK:(j + 1) * bK].astype(np.int64)
            if pmap[r, j] == W4:
                if tile.min() < -8 or tile.max() > 7:
                    raise ValueError(f"INT4 tile ({r},{j}) holds a code outside [-8, 7]")
                p = int(off4[r]) + left4
                left4 += 1
                lo, hi = tile[:, 0::2], tile[:, 1::2]   # consecutive values q0, q1
                w4[p] = ((lo % 16) + 16 * (hi % 16)).astype(np.uint8)
            else:
                p = int(off8[r]) + left8
                left8 += 1
                w8[p] = tile.astype(np.int8)
            tile_idx[r * C + j] = p
    sc = np.asarray(scales, dtype=np.float16).reshape(R, bN, C).transpose(0, 2, 1)
    return dict(N=N, K=K, bN=bN, bK=bK, R=R, C=C, T4=T4, T8=T8,
                bitmap=labels_to_bitmap(pmap), row_off4=off4, row_off8=off8,
                tile_idx=tile_idx, w4=w4, w8=w8,
                scales=np.ascontiguousarray(sc))


def unpack(packed: dict):
    """Packed projection -> (codes int8[N][K], scales float16[N][C], pmap).

    Locates every tile from its logical coordinate the way App. E.1 states:
    label -> buffer, row offset + count of same-precision tiles to the left
    -> physical index, then sign-extends INT4 nibbles (low nibble first)."""
    N, K, bN, bK = packed["N"], packed["K"], packed["bN"], packed["bK"]
    R, C = N // bN, K // bK
    bitmap = packed["bitmap"]
    pmap = np.array([[label_of(bitmap, r, j, C) for j in range(C)] for r in range(R)], dtype=np.uint8)
    codes = np.zeros((N, K), dtype=np.int8)
    for r in range(R):
        seen4 = seen8 = 0
        for j in range(C):
            if pmap[r, j] == W4:
                p = int(packed["row_off4"][r]) + seen4
                seen4 += 1
                b = packed["w4"][p].astype(np.int64)
                lo, hi = b % 16, b // 16
                tile = np.empty((bN, bK), dtype=np.int64)
                tile[:, 0::2] = np.where(lo < 8, lo, lo - 16)
                tile[:, 1::2] = np.where(hi < 8, hi, hi - 16)
            else:
                p = int(packed["row_off8"][r]) + seen8
                seen8 += 1
                tile = packed["w8"][p].astype(np.int64)
            assert int(packed["tile_idx"][r * C + j]) == p
            codes[r * bN:(r + 1) * bN, j * bK:(j + 1) * bK] = tile
    sc = np.asarray(packed["scales"], dtype=np.float16).reshape(R, C, bN).transpose(0, 2, 1).reshape(N, C)
    return codes, np.ascontiguousarray(sc), pmap


def packed_bytes(packed_or_geometry) -> int:
    """Bytes of this layer's packed projection: INT4 and INT8 payloads, fp16
    scales (one per output row per tile), labels, two row-offset arrays and
    the physical-index table."""
    g = packed_or_geometry
    N, bN, bK, R, C, T4, T8 = g["N"], g["bN"], g["bK"], g["R"], g["C"], g["T4"], g["T8"]
    B = bN * bK
    return B * T4 // 2 + B * T8 + 2 * N * C + (R * C + 7) // 8 + 8 * (R + 1) + 4 * R * C


def paper_packed_bytes(R: int, C: int, T4: int, bN: int, bK: int) -> int:
    """eq. 18 (App. E.2): S = B T4/2 + B T8 + 4 (T4 + T8) + ceil(RC/8) + 8 (R+1)
    with B = bN bK and one FP32 scale per tile."""
    B = bN * bK
    T8 = R * C - T4
    return B * T4 // 2 + B * T8 + 4 * (T4 + T8) + math.ceil(R * C / 8) + 8 * (R + 1)


# ---------------------------------------------------------------------------
# Activation quantization (App. B.3 carried out per token; eq. 5/6 rounding)
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact fp64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def quant_act(x_bits: np.ndarray):
    """Per-token symmetric INT8 quantization, fp64 throughout.

    For each token row: amax = max |x|; s = max(amax / 127, 1e-12);
    xq = clamp(round_half_even(x / s), -127, 127); the stored scale is
    fp32(s).  Codes are computed with the fp64 s, not with the rounded fp32
    scale.  Returns (xq int8[M][K], sx float32[M])."""
    x = bf16_bits_to_f64(x_bits)
    M, K = x.shape
    xq = np.zeros((M, K), dtype=np.int8)
    sx = np.zeros(M, dtype=np.float32)
    for m in range(M):
        amax = float(np.max(np.abs(x[m]))) if K else 0.0
        s = amax / 127.0
        if s < 1e-12:
            s = 1e-12
        q = np.rint(x[m] / s)            # np.rint rounds half to even
        xq[m] = np.clip(q, -127, 127).astype(np.int8)
        sx[m] = np.float32(s)
    return xq, sx


# ---------------------------------------------------------------------------
# Products and output reconstruction (Sec. 3.3, App. E.3 eq. 19)
# ---------------------------------------------------------------------------

def tile_partials(codes: np.ndarray, xq: np.ndarray, bK: int) -> np.ndarray:
    """Per-tile integer products P[m][n][j] = sum_{k in tile column j} xq[m,k] q[n,k].

    Computed with an fp64 matrix product: every product is an integer of
    magnitude <= 127*128 < 2^14 and every partial sum over <= bK terms stays
    far below 2^53, so all intermediates are exact integers in any summation
    order.  The result is checked to be integral and to fit INT32."""
    codes = np.asarray(codes)
    xq = np.asarray(xq)
    M, K = xq.shape
    N = codes.shape[0]
    assert codes.shape[1] == K and K % bK == 0 and bK <= 4096
    C = K // bK
    P = np.zeros((M, N, C), dtype=np.int64)
    for j in range(C):
        a = xq[:, j * bK:(j + 1) * bK].astype(np.float64)
        w = codes[:, j * bK:(j + 1) * bK].astype(np.float64)
        pj = a @ w.T
        P[:, :, j] = pj.astype(np.int64)
        assert np.array_equal(P[:, :, j].astype(np.float64), pj)
    assert np.abs(P).max(initial=0) < 2 ** 31
    return P


def reconstruct(P: np.ndarray, sx: np.ndarray, sw: np.ndarray, bias=None) -> np.ndarray:
    """eq. 19 with one activation scale per token: y[m,n] = sum over input
    tiles j (ascending) of sx[m] * sw[n,j] * P[m,n,j], in fp64, plus bias[n]."""
    M, N, C = P.shape
    sxd = np.asarray(sx, dtype=np.float32).astype(np.float64)
    swd = np.asarray(sw, dtype=np.float16).astype(np.float64)
    y = np.zeros((M, N), dtype=np.float64)
    for j in range(C):
        y += sxd[:, None] * swd[None, :, j] * P[:, :, j].astype(np.float64)
    if bias is not None:
        y += np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    return y


def linear_packed(packed: dict, xq: np.ndarray, sx: np.ndarray, bias=None, rows=None, cols=None):
    """Full layer from the packed form: unpack, per-tile products, rescale.

    ``rows`` (token indices) and ``cols`` (output-feature indices) restrict the
    computation to a sample of outputs."""
    codes, sw, _ = unpack(packed)
    return linear_codes(codes, sw, xq, sx, packed["bK"], bias, rows, cols)


def linear_codes(codes, sw, xq, sx, bK, bias=None, rows=None, cols=None):
    """The same as ``linear_packed`` from already unpacked codes and scales."""
    if rows is not None:
        xq, sx = xq[rows], sx[rows]
    if cols is not None:
        codes, sw = codes[cols], sw[cols]
        if bias is not None:
            bias = np.asarray(bias)[cols]
    return reconstruct(tile_partials(codes, xq, bK), sx, sw, bias)


# ---------------------------------------------------------------------------
# Float weights -> codes and scales (App. B.2, eq. 5-7)
# ---------------------------------------------------------------------------

def q_range(b: int):
    """App. B.2: q_min,b = -2^(b-1), q_max,b = 2^(b-1) - 1."""
    return -(2 ** (b - 1)), 2 ** (b - 1) - 1


def quantize_with_scale(a, s: float, b: int) -> np.ndarray:
    """eq. 5: Q_b(A; s) = clip to [q_min, q_max] of round_even(A / s), fp64."""
    qmin, qmax = q_range(b)
    a = np.asarray(a, dtype=np.float64)
    return np.clip(np.rint(a / np.float64(s)), qmin, qmax).astype(np.int64)


def endpoint_scale(a, b: int) -> float:
    """eq. 6: s_0 = max{ max(0, max A) / q_max, max(0, -min A) / |q_min|, 1e-12 }."""
    qmin, qmax = q_range(b)
    a = np.asarray(a, dtype=np.float64)
    return max(max(0.0, float(a.max())) / qmax, max(0.0, -float(a.min())) / abs(qmin), 1e-12)


def squared_error(a, s: float, q) -> float:
    """||A - s Q||_F^2 summed over the elements in increasing index order."""
    e = 0.0
    for av, qv in zip(np.asarray(a, dtype=np.float64).ravel(), np.asarray(q).ravel()):
        d = float(av) - float(s) * float(qv)
        e = e + d * d
    return e


def search_scale(a, b: int) -> float:
    """eq. 7: s_i = max{(1/4 + i/128) s_0, 1e-12} for i = 0..128; the scale with
    the smallest squared reconstruction error, the earliest i on equal errors."""
    s0 = endpoint_scale(a, b)
    best_s, best_e = None, None
    for i in range(129):
        si = max((0.25 + i / 128.0) * s0, 1e-12)
        e = squared_error(a, si, quantize_with_scale(a, si, b))
        if best_e is None or e < best_e:
            best_s, best_e = si, e
    return best_s


def quantize_weights(w, pmap: np.ndarray, bN: int, bK: int, search: bool):
    """Float weights W[N][K] and precision labels -> (codes int8[N][K], fp16
    scales [N][C]).  Each output row of each tile gets its own scale: the
    endpoint scale of eq. 6, or with ``search`` the grid minimum of eq. 7; the
    codes are eq. 5 with that fp64 scale, and the stored scale is its fp16
    rounding.  INT4 tiles (label 1) use b = 4, INT8 tiles b = 8."""
    w = np.asarray(w, dtype=np.float32).astype(np.float64)
    N, K = w.shape
    C = K // bK
    codes = np.zeros((N, K), dtype=np.int8)
    scales = np.zeros((N, C), dtype=np.float16)
    for n in range(N):
        r = n // bN
        for j in range(C):
            a = w[n, j * bK:(j + 1) * bK]
            b = 4 if int(pmap[r, j]) == W4 else 8
            s = search_scale(a, b) if search else endpoint_scale(a, b)
            codes[n, j * bK:(j + 1) * bK] = quantize_with_scale(a, s, b).astype(np.int8)
            scales[n, j] = np.float16(s)
    return codes, scales
