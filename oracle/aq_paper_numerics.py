"""CPU oracle of AlignQuant's own numerics (test infrastructure only; the
product path never imports it).

The product layer quantizes activations per token and keeps one fp16 scale
per output row per tile.  The paper's own construction differs, and this
module states it plainly, in fp64, as the reference for a later paper-exact
mode of the kernels:

  * tile-aligned block-diagonal transforms U = diag(U_r), V = diag(V_j) with
    the transformed tile U_r W_{r,j} V_j and X~ = X V; the output is restored
    by Y = Y~ U, which gives back X W^T before quantization
    (AlignQuant, App. B.1, eq. 4);
  * transform seeds Phi_{-1} = I, Phi_0 = H_64 and Phi_s = D_L P H_64 D_R, with
    H_64 the normalized Hadamard matrix (entries +-1/8); V_j = Phi and
    U_r = Phi^T (App. B.1).  The seeds themselves come from calibration and are
    inputs here;
  * weights: the candidate quantizer of eq. 5-7 applied to each whole
    transformed tile (one FP32 scale per tile, App. B.2, E.2);
  * activations: one scale per group of 64 features and b_M rows, b_M = 1 for
    M = 1 and 16 otherwise, the 8-bit endpoint scale s_{0,8} of eq. 6 (maximum
    over 127, minus the minimum over 128), codes clipped to [-128, 127], rows
    zero-padded to a multiple of b_M and sliced off afterwards (App. B.3);
  * reconstruction: eq. 19, per activation-row group m and output tile row r,
    Y~_{m,r} = sum_j s^X_{m,j} s^W_{r,j} (Q^X_{m,j} Q^W_{r,j}^T), then U_r.

Readings where the pages are silent: the grid search of eq. 7 runs over the
tile's values in row-major order; activation groups are the 64-feature
column blocks, which coincide with the input tiles in the paper's 64 x 64
configuration (eq. 19 indexes both by j); the FP32 scales are the fp64 values
rounded to fp32 after the codes are taken with the fp64 values.
"""
from __future__ import annotations

import numpy as np

from . import aq_oracle as base

GROUP = 64  # activation features per scale group (App. B.3)


def hadamard64() -> np.ndarray:
    """H_64 with +-1/8 entries: the Sylvester +-1 matrix of order 64 scaled by 1/8
    (App. B.1: the normalized Hadamard transform, final butterfly scaling 1/8)."""
    h = np.ones((1, 1))
    while h.shape[0] < 64:
        h = np.block([[h, h], [h, -h]])
    return h / 8.0


def seed_matrix(kind: int, perm=None, d_left=None, d_right=None) -> np.ndarray:
    """Phi_{-1} = I (kind -1), Phi_0 = H_64 (kind 0), and for kind >= 1
    Phi = D_L P H_64 D_R with the permutation ``perm`` (P[i, perm[i]] = 1) and
    the +-1 sign vectors ``d_left``, ``d_right``."""
    if kind == -1:
        return np.eye(64)
    h = hadamard64()
    if kind == 0:
        return h
    p = np.zeros((64, 64))
    p[np.arange(64), np.asarray(perm)] = 1.0
    return np.diag(np.asarray(d_left, float)) @ p @ h @ np.diag(np.asarray(d_right, float))


def block_diag(blocks) -> np.ndarray:
    """diag(B_0, B_1, ...) of square blocks."""
    n = sum(b.shape[0] for b in blocks)
    out = np.zeros((n, n))
    o = 0
    for b in blocks:
        k = b.shape[0]
        out[o:o + k, o:o + k] = b
        o += k
    return out


# ---------------------------------------------------------------------------
# Quantizers (App. B.2 on whole tiles; App. B.3 on activation groups)
# ---------------------------------------------------------------------------

def quantize_weight_tiles(w_tilde, pmap: np.ndarray, bN: int, bK: int, search: bool):
    """Transformed weights W~[N][K] -> (codes int8[N][K], scales fp32[R][C]).
    Each whole bN x bK tile is one quantization group: the endpoint scale of
    eq. 6 over the tile, or the eq. 7 grid minimum (squared errors summed over
    the tile in row-major order); b = 4 for INT4 labels, 8 for INT8.  Codes use
    the fp64 scale, the stored scale is its fp32 rounding."""
    w = np.asarray(w_tilde, dtype=np.float64)
    N, K = w.shape
    R, C = N // bN, K // bK
    codes = np.zeros((N, K), dtype=np.int8)
    scales = np.zeros((R, C), dtype=np.float32)
    for r in range(R):
        for j in range(C):
            tile = w[r * bN:(r + 1) * bN, j * bK:(j + 1) * bK]
            b = 4 if int(pmap[r, j]) == base.W4 else 8
            flat = tile.reshape(-1)
            s = base.search_scale(flat, b) if search else base.endpoint_scale(flat, b)
            codes[r * bN:(r + 1) * bN, j * bK:(j + 1) * bK] = base.quantize_with_scale(tile, s, b).astype(np.int8)
            scales[r, j] = np.float32(s)
    return codes, scales


def row_group(M: int) -> int:
    """b_M of App. B.3: 1 for a single row, 16 otherwise."""
    return 1 if M == 1 else 16


def quantize_activation_groups(x_tilde):
    """Transformed activations X~[M][K] -> (codes int8[M'][K], scales fp32[M'/b_M][K/64], M').
    Rows are zero-padded to M' = ceil(M / b_M) b_M; every block of b_M rows and
    64 features gets s = s_{0,8} (eq. 6 with b = 8) and codes
    clip(rint(A / s), -128, 127) (eq. 5), with the fp64 s."""
    x = np.asarray(x_tilde, dtype=np.float64)
    M, K = x.shape
    assert K % GROUP == 0
    bM = row_group(M)
    Mp = -(-M // bM) * bM
    xp = np.zeros((Mp, K))
    xp[:M] = x
    G = K // GROUP
    codes = np.zeros((Mp, K), dtype=np.int8)
    scales = np.zeros((Mp // bM, G), dtype=np.float32)
    for g in range(Mp // bM):
        for c in range(G):
            blk = xp[g * bM:(g + 1) * bM, c * GROUP:(c + 1) * GROUP]
            s = base.endpoint_scale(blk.reshape(-1), 8)
            codes[g * bM:(g + 1) * bM, c * GROUP:(c + 1) * GROUP] = base.quantize_with_scale(blk, s, 8).astype(np.int8)
            scales[g, c] = np.float32(s)
    return codes, scales, Mp


# ---------------------------------------------------------------------------
# Reconstruction (eq. 19) and the whole layer (eq. 4)
# ---------------------------------------------------------------------------

def reconstruct_groups(xq, sx, qw, sw, bN: int, bK: int, M: int) -> np.ndarray:
    """eq. 19 in fp64: Y~[m, n] = sum over 64-feature groups g (ascending) of
    sx[m // b_M, g] * sw[n // bN, tile of g] * (sum over k in g of xq[m, k] qw[n, k]);
    the integer products are exact.  Returns the first M rows."""
    xq = np.asarray(xq).astype(np.float64)
    qw = np.asarray(qw).astype(np.float64)
    Mp, K = xq.shape
    N = qw.shape[0]
    bM = row_group(M)
    sxd = np.asarray(sx, dtype=np.float32).astype(np.float64)
    swd = np.asarray(sw, dtype=np.float32).astype(np.float64)
    y = np.zeros((Mp, N))
    rows_g = np.arange(Mp) // bM
    cols_r = np.arange(N) // bN
    for g in range(K // GROUP):
        k0 = g * GROUP
        p = xq[:, k0:k0 + GROUP] @ qw[:, k0:k0 + GROUP].T  # exact: |terms| < 2^14, 64 of them
        y += sxd[rows_g, g][:, None] * swd[cols_r, k0 // bK][None, :] * p
    return y[:M]


def paper_linear(x, w, pmap: np.ndarray, bN: int, bK: int, u_blocks=None, v_blocks=None, search: bool = False,
                 bias=None) -> dict:
    """The paper's quantized projection of fp64 inputs X[M][K] and W[N][K].

    ``v_blocks``: one bK x bK matrix per input-tile column (V = diag(V_j));
    ``u_blocks``: one bN x bN matrix per output-tile row (U = diag(U_r));
    None means identity.  X~ = X V, W~ = U W V (App. B.1), weights quantized per
    tile and activations per group (App. B.2, B.3), Y~ by eq. 19, Y = Y~ U
    (eq. 4), plus bias.  Returns the output and every intermediate."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    M, K = x.shape
    N = w.shape[0]
    V = np.eye(K) if v_blocks is None else block_diag(v_blocks)
    U = np.eye(N) if u_blocks is None else block_diag(u_blocks)
    x_t = x @ V
    w_t = U @ w @ V
    qw, sw = quantize_weight_tiles(w_t, pmap, bN, bK, search)
    xq, sx, Mp = quantize_activation_groups(x_t)
    y_t = reconstruct_groups(xq, sx, qw, sw, bN, bK, M)
    y = y_t @ U
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    return {"y": y, "y_tilde": y_t, "x_tilde": x_t, "w_tilde": w_t, "xq": xq, "sx": sx, "qw": qw, "sw": sw,
            "rows_padded": Mp}
