"""The oracle's pins catch plausible mistakes in the oracle.

Each case below plants one mistake in one oracle function, on the CPU, of
the kinds a restatement of the pages can make: a dropped term, a wrong
sign, a wrong index or operand, a wrong rounding or clipping rule, a wrong
constant.  It then runs every pin in tests/test_oracle_pins.py and
tests/test_oracle_paper_numerics.py (all parametrizations) with the mistake
in place, and requires at least one of them to fail.  A mistake that no pin
notices would mean the oracle is only checked against itself there.

The planted versions are wrappers around the oracle's functions, or short
restatements of them with the one change; they live only in this file.
"""
import itertools

import numpy as np
import pytest

import oracle
import test_oracle_paper_numerics as paper_pins
import test_oracle_pins as pins
from oracle import aq_oracle as ao
from oracle import aq_paper_numerics as pn


def _cases(fn):
    """(fn, kwargs) for every parametrization of a pin."""
    axes = []
    for mark in getattr(fn, "pytestmark", []):
        if mark.name != "parametrize":
            continue
        names, values = mark.args[0], mark.args[1]
        names = [s.strip() for s in names.split(",")] if isinstance(names, str) else list(names)
        rows = []
        for v in values:
            v = getattr(v, "values", v)  # pytest.param
            rows.append(dict(zip(names, v if len(names) > 1 else (v,))))
        axes.append(rows)
    return [(fn, {k: v for d in combo for k, v in d.items()}) for combo in itertools.product(*axes)]


PINS = [case for mod in (pins, paper_pins) for name in sorted(dir(mod)) if name.startswith("test_")
        for case in _cases(getattr(mod, name))]


def _first_failing_pin():
    for fn, kw in PINS:
        try:
            with np.errstate(all="ignore"):
                fn(**kw)
        except Exception:  # an assertion, or a crash the mistake causes: either way the pin fails
            return f"{fn.__name__}{kw or ''}"
    return None


def test_every_pin_passes_on_the_oracle_as_written():
    assert len(PINS) > 60
    assert _first_failing_pin() is None


# ----------------------------------------------------------------- planted mistakes

def _nibble_byte_high_first(q0, q1):  # eq. 17 with the nibbles swapped
    return (q1 % 16) + 16 * (q0 % 16)


def _nibble_value_off_by_one(v):  # App. E.1 sign extension with the threshold one too high
    return v if v <= 8 else v - 16


def _pack_high_nibble_first(*args, **kw):  # the packer writes q0 into the high nibble
    p = _REAL["pack"](*args, **kw)
    w4 = p["w4"]
    p["w4"] = ((w4 >> 4) | (w4 << 4)).astype(np.uint8)
    return p


def _unpack_scales_not_transposed(packed):  # stored [R][C][bN] scales read as if [N][C]
    codes, _, pmap = _REAL["unpack"](packed)
    sc = np.asarray(packed["scales"], np.float16).reshape(packed["N"], packed["C"])
    return codes, np.ascontiguousarray(sc), pmap


def _unpack_int4_unsigned(packed):  # INT4 nibbles not sign-extended
    codes, sc, pmap = _REAL["unpack"](packed)
    mask = np.kron(pmap == ao.W4, np.ones((packed["bN"], packed["bK"]), bool))
    out = codes.astype(np.int16)
    out[mask & (out < 0)] += 16
    return out.astype(np.int8), sc, pmap


def _labels_msb_first(pmap):  # App. E.1 label order reversed inside each byte
    flat = np.asarray(pmap, np.uint8).reshape(-1)
    out = np.zeros((len(flat) + 7) // 8, np.uint8)
    for t, beta in enumerate(flat):
        if beta:
            out[t // 8] |= np.uint8(1 << (7 - t % 8))
    return out


def _physical_index_no_in_row_term(pmap, r, j, b):  # eq. 16 without the same-row count
    want = ao.W4 if b == 4 else ao.W8
    return int((np.asarray(pmap)[:r] == want).sum())


def _row_offsets_other_precision(pmap, b):  # offsets counted over the other buffer's tiles
    return _REAL["row_offsets"](pmap, 8 if b == 4 else 4)


def _quant_act_variant(rounding="even", qmax=127.0, floor=1e-12):
    def quant_act(x_bits):
        x = ao.bf16_bits_to_f64(x_bits)
        M, K = x.shape
        xq = np.zeros((M, K), np.int8)
        sx = np.zeros(M, np.float32)
        for m in range(M):
            s = max(float(np.max(np.abs(x[m]))) / qmax, floor)
            t = x[m] / s if s > 0 else np.zeros(K)
            q = np.rint(t) if rounding == "even" else np.sign(t) * np.floor(np.abs(t) + 0.5)
            xq[m] = np.clip(q, -127, 127).astype(np.int8)
            sx[m] = np.float32(s)
        return xq, sx
    return quant_act


def _tile_partials_shifted(codes, xq, bK):  # tile j of the weights paired with tile j + 1 of x
    M, K = xq.shape
    C = K // bK
    P = np.zeros((M, codes.shape[0], C), np.int64)
    for j in range(C):
        jx = (j + 1) % C
        P[:, :, j] = xq[:, jx * bK:(jx + 1) * bK].astype(np.int64) @ codes[:, j * bK:(j + 1) * bK].astype(np.int64).T
    return P


def _tile_partials_transposed_tile(codes, xq, bK):  # the weight tile's columns read in reverse
    M, K = xq.shape
    C = K // bK
    P = np.zeros((M, codes.shape[0], C), np.int64)
    for j in range(C):
        w = codes[:, j * bK:(j + 1) * bK][:, ::-1]
        P[:, :, j] = xq[:, j * bK:(j + 1) * bK].astype(np.int64) @ w.astype(np.int64).T
    return P


def _reconstruct_variant(drop_bias=False, first_scale=False, skip_last=False, bias_sign=1.0):
    def reconstruct(P, sx, sw, bias=None):
        M, N, C = P.shape
        sxd = np.asarray(sx, np.float32).astype(np.float64)
        swd = np.asarray(sw, np.float16).astype(np.float64)
        y = np.zeros((M, N))
        for j in range(C - 1 if skip_last and C > 1 else C):
            y += sxd[:, None] * swd[None, :, 0 if first_scale else j] * P[:, :, j]
        if bias is not None and not drop_bias:
            y += bias_sign * np.asarray(bias, np.float32).astype(np.float64)[None, :]
        return y
    return reconstruct


def _endpoint_scale_symmetric(a, b):  # eq. 6 dividing the negative end by q_max
    qmin, qmax = ao.q_range(b)
    a = np.asarray(a, np.float64)
    return max(max(0.0, float(a.max())) / qmax, max(0.0, -float(a.min())) / qmax, 1e-12)


def _quantize_with_scale_variant(rounding="even", symmetric=False):
    def quantize_with_scale(a, s, b):
        qmin, qmax = ao.q_range(b)
        t = np.asarray(a, np.float64) / np.float64(s)
        q = np.rint(t) if rounding == "even" else np.floor(t + 0.5)
        return np.clip(q, -qmax if symmetric else qmin, qmax).astype(np.int64)
    return quantize_with_scale


def _search_scale_variant(step=128.0, last_on_ties=False, start=0.25, points=129):
    def search_scale(a, b):
        s0 = ao.endpoint_scale(a, b)
        best_s, best_e = None, None
        for i in range(points):
            si = max((start + i / step) * s0, 1e-12)
            e = ao.squared_error(a, si, ao.quantize_with_scale(a, si, b))
            if best_e is None or e < best_e or (last_on_ties and e == best_e):
                best_s, best_e = si, e
        return best_s
    return search_scale


def _squared_error_abs(a, s, q):  # the error without the square
    return float(np.sum(np.abs(np.asarray(a, np.float64) - s * np.asarray(q, np.float64))))


def _paper_bytes_no_offsets(R, C, T4, bN, bK):  # eq. 18 without the 8 (R + 1) offset term
    return _REAL["paper_packed_bytes"](R, C, T4, bN, bK) - 8 * (R + 1)


def _paper_bytes_fp16_scales(R, C, T4, bN, bK):  # eq. 18 with 2-byte tile scales
    return _REAL["paper_packed_bytes"](R, C, T4, bN, bK) - 2 * R * C


def _packed_bytes_no_table(g):  # this layer's bytes without the physical-index table
    return _REAL["packed_bytes"](g) - 4 * g["R"] * g["C"]


def _hadamard_unnormalized():
    return _REAL_PN["hadamard64"]() * 8.0


def _row_group_eight(M):
    return 1 if M == 1 else 8


def _row_group_always_sixteen(M):
    return 16


def _quantize_activation_groups_symmetric(x_tilde):  # groups with the +-127 range of the per-token form
    x = np.asarray(x_tilde, np.float64)
    M, K = x.shape
    bM = pn.row_group(M)
    Mp = -(-M // bM) * bM
    xp = np.zeros((Mp, K))
    xp[:M] = x
    codes = np.zeros((Mp, K), np.int8)
    scales = np.zeros((Mp // bM, K // 64), np.float32)
    for g in range(Mp // bM):
        for c in range(K // 64):
            blk = xp[g * bM:(g + 1) * bM, c * 64:(c + 1) * 64]
            s = max(float(np.abs(blk).max()) / 127.0, 1e-12)
            codes[g * bM:(g + 1) * bM, c * 64:(c + 1) * 64] = np.clip(np.rint(blk / s), -127, 127)
            scales[g, c] = np.float32(s)
    return codes, scales, Mp


def _weight_tiles_scaled_by_first_row(w_tilde, pmap, bN, bK, search):  # the tile scale from its first row only
    w = np.asarray(w_tilde, np.float64)
    N, K = w.shape
    codes = np.zeros((N, K), np.int8)
    scales = np.zeros((N // bN, K // bK), np.float32)
    for r in range(N // bN):
        for j in range(K // bK):
            tile = w[r * bN:(r + 1) * bN, j * bK:(j + 1) * bK]
            b = 4 if int(pmap[r, j]) == ao.W4 else 8
            s = ao.search_scale(tile[0], b) if search else ao.endpoint_scale(tile[0], b)
            codes[r * bN:(r + 1) * bN, j * bK:(j + 1) * bK] = ao.quantize_with_scale(tile, s, b)
            scales[r, j] = np.float32(s)
    return codes, scales


def _reconstruct_groups_first_row_group(xq, sx, qw, sw, bN, bK, M):  # every row scaled by row group 0
    sx0 = np.repeat(np.asarray(sx)[:1], len(sx), axis=0)
    return _REAL_PN["reconstruct_groups"](xq, sx0, qw, sw, bN, bK, M)


def _paper_linear_restored_with_u_transposed(x, w, pmap, bN, bK, u_blocks=None, v_blocks=None, search=False,
                                             bias=None):  # Y = Y~ U^T instead of Y~ U
    out = _REAL_PN["paper_linear"](x, w, pmap, bN, bK, u_blocks, v_blocks, search, bias)
    if u_blocks is None:
        return out
    y = out["y_tilde"] @ pn.block_diag([u.T for u in u_blocks])
    if bias is not None:
        y = y + np.asarray(bias, np.float32).astype(np.float64)[None, :]
    return dict(out, y=y)


_REAL = {k: getattr(ao, k) for k in ("pack", "unpack", "row_offsets", "paper_packed_bytes", "packed_bytes")}
_REAL_PN = {k: getattr(pn, k) for k in ("hadamard64", "reconstruct_groups", "paper_linear")}

MISTAKES = {
    "eq17 nibble order swapped": (ao, "nibble_byte", _nibble_byte_high_first),
    "nibble sign extension off by one": (ao, "nibble_value", _nibble_value_off_by_one),
    "packer writes q0 high": (ao, "pack", _pack_high_nibble_first),
    "unpack reads scales in the wrong order": (ao, "unpack", _unpack_scales_not_transposed),
    "unpack leaves INT4 unsigned": (ao, "unpack", _unpack_int4_unsigned),
    "labels MSB first": (ao, "labels_to_bitmap", _labels_msb_first),
    "eq16 without the in-row term": (ao, "physical_index", _physical_index_no_in_row_term),
    "row offsets of the other buffer": (ao, "row_offsets", _row_offsets_other_precision),
    "activations rounded half away from zero": (ao, "quant_act", _quant_act_variant(rounding="away")),
    "activation scale over 128": (ao, "quant_act", _quant_act_variant(qmax=128.0)),
    "activation scale without the floor": (ao, "quant_act", _quant_act_variant(floor=0.0)),
    "tile products with a shifted x tile": (ao, "tile_partials", _tile_partials_shifted),
    "tile products with a reversed weight tile": (ao, "tile_partials", _tile_partials_transposed_tile),
    "reconstruction drops the bias": (ao, "reconstruct", _reconstruct_variant(drop_bias=True)),
    "reconstruction subtracts the bias": (ao, "reconstruct", _reconstruct_variant(bias_sign=-1.0)),
    "reconstruction uses the first tile's scale": (ao, "reconstruct", _reconstruct_variant(first_scale=True)),
    "reconstruction skips the last tile": (ao, "reconstruct", _reconstruct_variant(skip_last=True)),
    "eq6 symmetric": (ao, "endpoint_scale", _endpoint_scale_symmetric),
    "eq5 rounds half up": (ao, "quantize_with_scale", _quantize_with_scale_variant(rounding="up")),
    "eq5 clips symmetric": (ao, "quantize_with_scale", _quantize_with_scale_variant(symmetric=True)),
    "eq7 grid step 1/64": (ao, "search_scale", _search_scale_variant(step=64.0)),
    "eq7 grid from 1/2": (ao, "search_scale", _search_scale_variant(start=0.5)),
    "eq7 grid without its last point": (ao, "search_scale", _search_scale_variant(points=128)),
    "eq7 keeps the last of equal errors": (ao, "search_scale", _search_scale_variant(last_on_ties=True)),
    "eq7 error without the square": (ao, "squared_error", _squared_error_abs),
    "eq18 without the row offsets": (ao, "paper_packed_bytes", _paper_bytes_no_offsets),
    "eq18 with 2-byte tile scales": (ao, "paper_packed_bytes", _paper_bytes_fp16_scales),
    "packed bytes without the index table": (ao, "packed_bytes", _packed_bytes_no_table),
    "H64 not normalized": (pn, "hadamard64", _hadamard_unnormalized),
    "activation row groups of 8": (pn, "row_group", _row_group_eight),
    "activation groups of 32 features": (pn, "GROUP", 32),
    "weight tile scale from its first row": (pn, "quantize_weight_tiles", _weight_tiles_scaled_by_first_row),
    "one token grouped as 16 rows": (pn, "row_group", _row_group_always_sixteen),
    "activation groups with the symmetric range": (pn, "quantize_activation_groups",
                                                    _quantize_activation_groups_symmetric),
    "eq19 with the first row group's scales for every row": (pn, "reconstruct_groups",
                                                              _reconstruct_groups_first_row_group),
    "eq4 output restored with U transposed": (pn, "paper_linear", _paper_linear_restored_with_u_transposed),
}


# Not planted: eq. 6 without its max(0, .) terms, which changes nothing (max A < 0
# implies -min A > 0, so the two terms are never both negative).
# Not planted either: activation codes taken with the fp32-rounded scale instead of the
# fp64 one.  The two differ only at exact ties of the exact quotient (x = amax / 2
# gives 127 x / amax = 63.5), where the rounding direction of the scale decides
# the side; the pages fix that precision (fp64, App. B.3) but print no value that
# tells the two apart, so a test could only restate the formula.
@pytest.mark.parametrize("mistake", sorted(MISTAKES))
def test_a_planted_mistake_fails_a_pin(mistake, monkeypatch):
    module, name, planted = MISTAKES[mistake]
    monkeypatch.setattr(module, name, planted)
    if module is ao and hasattr(oracle, name):
        monkeypatch.setattr(oracle, name, planted)  # the package re-exports the per-token oracle's names
    assert _first_failing_pin() is not None, f"no pin notices: {mistake}"
