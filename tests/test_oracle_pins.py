"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Sources of truth used here:
  * values the AlignQuant paper prints (the eq. 16 worked example, Table 16's
    packed bits per weight through eq. 18), stored under tests/golden/;
  * bytes worked out by hand from eq. 17 and from the label order of App. E.1;
  * hand-worked activation-quantization cases (ties to even, zero rows);
  * brute force on tiny inputs written as plain loops over unpacked codes;
  * invariants fixed by the mathematics (pack -> unpack identity, an all-INT8
    map is a plain W8A8 product, exact scaling by powers of two, odd
    symmetry, additivity of the integer partials).
"""
import json
import os

import numpy as np
import pytest

import oracle
from w8_a8_quantized_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _random_case(N, K, bN, bK, frac8, seed, M=3):
    p = synth.projection_inputs(N, K, bN, bK, frac8, (seed,))
    x = synth.activations(M, K, (seed, 99))
    return p, x


# ---------------------------------------------------------------- format pins

def test_eq16_worked_example():
    g = _golden("eq16_worked_example.json")
    pmap = np.array([[1 if b == 4 else 0 for b in g["row_precisions"]]], dtype=np.uint8)
    for e in g["expected"]:
        j = e["tile"]
        assert oracle.label_of(oracle.labels_to_bitmap(pmap), 0, j, pmap.shape[1]) == (1 if e["buffer"] == 4 else 0)
        assert oracle.physical_index(pmap, 0, j, e["buffer"]) == e["index"]
    # and through the packer: tile 0 and tile 2 land in W4 slots 0 and 1
    bN, bK = 2, 4
    codes = np.arange(-6, 6, dtype=np.int8).reshape(2, 6) % 7 - 3
    codes = np.tile(codes, (1, 2))[:, :12]
    pk = oracle.pack(codes, np.ones((2, 3), np.float16), pmap, bN, bK)
    assert list(pk["tile_idx"]) == [0, 0, 1]
    assert pk["T4"] == 2 and pk["T8"] == 1
    assert list(pk["row_off4"]) == [0, 2] and list(pk["row_off8"]) == [0, 1]


def test_eq17_bytes_hand_worked():
    for c in _golden("eq17_bytes.json")["cases"]:
        assert oracle.nibble_byte(c["q0"], c["q1"]) == c["byte"]
        assert oracle.nibble_value(c["byte"] & 15) == c["q0"]
        assert oracle.nibble_value(c["byte"] >> 4) == c["q1"]
        # the packer puts q0 (even k) in the low nibble
        codes = np.array([[c["q0"], c["q1"]]], dtype=np.int8)
        pk = oracle.pack(codes, np.ones((1, 1), np.float16), np.ones((1, 1), np.uint8), 1, 2)
        assert int(pk["w4"][0, 0, 0]) == c["byte"]


def test_eq17_exhaustive_roundtrip():
    seen = set()
    for q0 in range(-8, 8):
        for q1 in range(-8, 8):
            b = oracle.nibble_byte(q0, q1)
            assert 0 <= b < 256
            seen.add(b)
            assert (oracle.nibble_value(b % 16), oracle.nibble_value(b // 16)) == (q0, q1)
    assert len(seen) == 256


def test_label_bit_order_hand_worked():
    for c in _golden("label_bit_order.json")["cases"]:
        pmap = np.array(c["labels"], dtype=np.uint8).reshape(c["R"], c["C"])
        assert list(oracle.labels_to_bitmap(pmap)) == c["bytes"]


def test_table16_bits_per_weight():
    g = _golden("table16_packed_bpw.json")
    bN, bK = g["tile"]
    shapes = synth.projections("llama-3.2-3b")
    layers = synth.MODELS["llama-3.2-3b"]["layers"]
    tiles = [(n // bN) * (k // bK) for _, n, k in shapes] * layers
    total = sum(tiles)
    for rho, want in zip(g["w4_fraction"], g["packed_bpw_2dp"]):
        k4 = int(round(rho * total))
        left, S, W = k4, 0, 0
        for (_, n, k), t in zip(shapes * layers, tiles):
            t4 = min(left, t)
            left -= t4
            S += oracle.paper_packed_bytes(n // bN, k // bK, t4, bN, bK)
            W += n * k
        assert round(8 * S / W, 2) == pytest.approx(want, abs=1e-9), rho


def test_scale_and_label_overhead_33_over_B():
    # App. F.2: scales + labels cost about 33/(bN bK) bits per weight
    for bN, bK in [(32, 32), (64, 64), (128, 128)]:
        R, C = 40, 40
        B = bN * bK
        base = oracle.paper_packed_bytes(R, C, 0, bN, bK) - B * R * C - 8 * (R + 1)
        assert 8 * base / (B * R * C) == pytest.approx(33 / B, rel=1e-12)


@pytest.mark.parametrize("frac8", [0.0, 0.25, 0.5, 1.0])
@pytest.mark.parametrize("bN,bK", [(2, 4), (4, 8), (64, 128), (128, 128)])
def test_pack_unpack_identity(frac8, bN, bK):
    N, K = bN * 3, bK * 5
    p = synth.projection_inputs(N, K, bN, bK, frac8, (7, bN, bK))
    pk = oracle.pack(p.codes, p.scales, p.pmap, bN, bK)
    codes, sc, pmap = oracle.unpack(pk)
    assert np.array_equal(codes, p.codes)
    assert np.array_equal(sc.view(np.uint16), p.scales.view(np.uint16))
    assert np.array_equal(pmap, p.pmap)
    # eq. 16 literal double sum agrees with the packer's index table
    for r in range(p.R):
        for j in range(p.C):
            b = 4 if p.pmap[r, j] else 8
            assert oracle.physical_index(p.pmap, r, j, b) == pk["tile_idx"][r * p.C + j]
    assert pk["T4"] + pk["T8"] == p.R * p.C
    assert pk["w4"].nbytes + pk["w8"].nbytes == (pk["T4"] * bN * bK) // 2 + pk["T8"] * bN * bK


def test_int4_codes_stay_in_range():
    p = synth.projection_inputs(256, 512, 128, 128, 0.25, (11,))
    pk = oracle.pack(p.codes, p.scales, p.pmap, 128, 128)
    codes, _, pmap = oracle.unpack(pk)
    is4 = np.repeat(np.repeat(pmap.astype(bool), 128, 0), 128, 1)
    assert codes[is4].min() == -8 and codes[is4].max() == 7
    for bad in (8, -9, 127, -128):
        c = p.codes.copy()
        r, j = map(int, np.argwhere(p.pmap == 1)[0])
        c[r * 128 + 5, j * 128 + 17] = bad
        with pytest.raises(ValueError):
            oracle.pack(c, p.scales, p.pmap, 128, 128)


# -------------------------------------------------------- activation quant pins

def test_act_quant_ties_to_even_unit_scale():
    # amax 127 -> s = 1 exactly, so codes are the half-even rounding of x itself
    x = np.array([[127.0, 2.5, -2.5, 3.5, 0.5, 1.5, -0.5, -127.0, 126.5, -1.5]], np.float32)
    xq, sx = oracle.quant_act(synth.f32_to_bf16_bits(x))
    assert list(xq[0]) == [127, 2, -2, 4, 0, 2, 0, -127, 126, -2]
    assert sx[0] == np.float32(1.0)


def test_act_quant_hand_worked_scale_two():
    # amax 254 -> s = 2: 5/2 = 2.5 -> 2, 7/2 = 3.5 -> 4, 3/2 -> 2, 1/2 -> 0, -254 -> -127
    x = np.array([[5.0, 7.0, 3.0, 1.0, -254.0, 100.0]], np.float32)
    xq, sx = oracle.quant_act(synth.f32_to_bf16_bits(x))
    assert list(xq[0]) == [2, 4, 2, 0, -127, 50]
    assert sx[0] == np.float32(2.0)


def test_act_quant_zero_row_uses_floor():
    xq, sx = oracle.quant_act(np.zeros((2, 64), np.uint16))
    assert not xq.any()
    assert sx[0] == np.float32(1e-12) and sx[1] == np.float32(1e-12)


def test_act_quant_negative_amax_and_properties():
    x = np.array([[-3.0, 1.0, 0.0, 2.0]], np.float32)
    xq, _ = oracle.quant_act(synth.f32_to_bf16_bits(x))
    assert list(xq[0]) == [-127, 42, 0, 85]  # 127/3 = 42.33 -> 42, 254/3 = 84.67 -> 85
    bits = synth.activations(16, 512, (3,), outlier_frac=0.01)
    xq, sx = oracle.quant_act(bits)
    xv = oracle.bf16_bits_to_f64(bits)
    assert np.all(np.abs(xq.astype(int)).max(axis=1) == 127)
    # each code is a nearest integer of x / s (s recovered to fp32 precision)
    err = np.abs(xv / sx.astype(np.float64)[:, None] - xq)
    assert err.max() <= 0.5 + 1e-4


def test_act_quant_power_of_two_and_sign_symmetry():
    bits = synth.activations(8, 256, (5,))
    x = oracle.bf16_bits_to_f64(bits).astype(np.float32)
    xq, sx = oracle.quant_act(bits)
    for e in (-3, 1, 4):
        xq2, sx2 = oracle.quant_act(synth.f32_to_bf16_bits(x * np.float32(2.0 ** e)))
        assert np.array_equal(xq2, xq) and np.array_equal(sx2, sx * np.float32(2.0 ** e))
    xqn, sxn = oracle.quant_act(synth.f32_to_bf16_bits(-x))
    assert np.array_equal(xqn, -xq) and np.array_equal(sxn, sx)


# ------------------------------------------------------------ products + output

def _brute_force(codes, sw, xq, sx, bK, bias=None):
    """y[m][n] = sum_k sx[m] sw[n][k // bK] xq[m][k] q[n][k] (+ bias), plain loops."""
    M, K = xq.shape
    N = codes.shape[0]
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(sx[m]) * float(sw[n, k // bK]) * int(xq[m, k]) * int(codes[n, k])
            y[m, n] = acc + (float(bias[n]) if bias is not None else 0.0)
    return y


@pytest.mark.parametrize("bN,bK,R,C", [(2, 2, 2, 3), (2, 4, 3, 2), (4, 8, 2, 2), (1, 2, 3, 3)])
@pytest.mark.parametrize("frac8", [0.0, 0.5, 1.0])
def test_brute_force_tiny(bN, bK, R, C, frac8):
    N, K = bN * R, bK * C
    p, x = _random_case(N, K, bN, bK, frac8, 100 + bN * 7 + bK + R)
    xq, sx = oracle.quant_act(x)
    pk = oracle.pack(p.codes, p.scales, p.pmap, bN, bK)
    bias = np.linspace(-1, 1, N).astype(np.float32)
    y = oracle.linear_packed(pk, xq, sx, bias=bias)
    yb = _brute_force(p.codes, p.scales, xq, sx, bK, bias)
    np.testing.assert_allclose(y, yb, rtol=1e-12, atol=1e-15)


def test_partials_match_integer_loops():
    p, x = _random_case(8, 16, 4, 8, 0.5, 3)
    xq, _ = oracle.quant_act(x)
    P = oracle.tile_partials(p.codes, xq, 8)
    for m in range(xq.shape[0]):
        for n in range(8):
            for j in range(2):
                want = sum(int(xq[m, k]) * int(p.codes[n, k]) for k in range(8 * j, 8 * j + 8))
                assert P[m, n, j] == want


def test_partials_extreme_magnitude():
    # the largest |P| the format allows: 128 * 127 * (-128) per tile
    codes = np.full((2, 128), -128, np.int8)
    xq = np.full((1, 128), 127, np.int8)
    P = oracle.tile_partials(codes, xq, 128)
    assert P[0, 0, 0] == -128 * 127 * 128


@pytest.mark.parametrize("frac8", [1.0, 0.0])
def test_uniform_map_is_plain_w8a8(frac8):
    p, x = _random_case(256, 384, 128, 128, frac8, 21, M=5)
    xq, sx = oracle.quant_act(x)
    pk = oracle.pack(p.codes, p.scales, p.pmap, 128, 128)
    codes, _, _ = oracle.unpack(pk)
    P = oracle.tile_partials(codes, xq, 128)
    dense = xq.astype(np.int64) @ p.codes.astype(np.int64).T
    assert np.array_equal(P.sum(axis=2), dense)
    # unit scales: the output is the integer GEMM times sx
    ones = np.ones_like(p.scales)
    y = oracle.reconstruct(P, np.ones(5, np.float32), ones)
    assert np.array_equal(y, dense.astype(np.float64))


def test_partials_additive_in_xq():
    p, x = _random_case(128, 256, 128, 128, 0.5, 31, M=4)
    g = np.random.default_rng(0)
    a = g.integers(-63, 64, size=(4, 256)).astype(np.int8)
    b = g.integers(-63, 64, size=(4, 256)).astype(np.int8)
    Pa = oracle.tile_partials(p.codes, a, 128)
    Pb = oracle.tile_partials(p.codes, b, 128)
    Pab = oracle.tile_partials(p.codes, (a + b).astype(np.int8), 128)
    assert np.array_equal(Pa + Pb, Pab)


def test_output_scales_exactly_and_is_odd():
    p, x = _random_case(128, 512, 64, 128, 0.5, 41, M=3)
    pk = oracle.pack(p.codes, p.scales, p.pmap, 64, 128)
    xv = oracle.bf16_bits_to_f64(x).astype(np.float32)
    xq, sx = oracle.quant_act(x)
    y = oracle.linear_packed(pk, xq, sx)
    for e in (2, -5):
        xq2, sx2 = oracle.quant_act(synth.f32_to_bf16_bits(xv * np.float32(2.0 ** e)))
        assert np.array_equal(oracle.linear_packed(pk, xq2, sx2), y * 2.0 ** e)
    xqn, sxn = oracle.quant_act(synth.f32_to_bf16_bits(-xv))
    assert np.array_equal(oracle.linear_packed(pk, xqn, sxn), -y)


def test_sampled_rows_and_cols_match_full():
    p, x = _random_case(256, 256, 128, 128, 0.5, 51, M=6)
    pk = oracle.pack(p.codes, p.scales, p.pmap, 128, 128)
    xq, sx = oracle.quant_act(x)
    y = oracle.linear_packed(pk, xq, sx)
    rows, cols = np.array([5, 0, 3]), np.array([255, 7, 128, 1])
    ys = oracle.linear_packed(pk, xq, sx, rows=rows, cols=cols)
    np.testing.assert_array_equal(ys, y[np.ix_(rows, cols)])


def test_packed_bytes_matches_buffers():
    p = synth.projection_inputs(512, 768, 64, 128, 0.3, (61,))
    pk = oracle.pack(p.codes, p.scales, p.pmap, 64, 128)
    nbytes = sum(pk[k].nbytes for k in ("bitmap", "row_off4", "row_off8", "tile_idx", "w4", "w8", "scales"))
    assert oracle.packed_bytes(pk) == nbytes


def test_synthetic_generators_shape_and_ranges():
    p = synth.projection_inputs(256, 512, 128, 128, 0.25, (1,))
    assert (p.pmap == 0).sum() == round(0.25 * 8)
    s = p.scales.astype(np.float64)
    assert s.min() >= 0.00099 and s.max() <= 0.01001
    x = synth.activations(4, 1000, (2,), outlier_frac=0.01)
    xv = oracle.bf16_bits_to_f64(x)
    big = (np.abs(xv) > 8).any(axis=0)
    assert 1 <= big.sum() <= 10


# ------------------------------------------------- float-weight quantizer pins

def test_weight_quant_hand_worked_endpoint_int4():
    # eq. 6 with b = 4: max(0.5 / 7, 1.0 / 8) = 0.125; eq. 5: 0.5/0.125 = 4,
    # -1/0.125 = -8 (q_min reached, not clipped), 0.25/0.125 = 2
    a = np.array([0.5, -1.0, 0.25, 0.0])
    assert oracle.endpoint_scale(a, 4) == 0.125
    assert list(oracle.quantize_with_scale(a, 0.125, 4)) == [4, -8, 2, 0]


def test_weight_quant_hand_worked_endpoint_int8():
    # b = 8: max(1.27 / 127, 0.5 / 128) = 0.01 -> codes 127, -50, 0.5 -> 0 (tie to even)
    a = np.array([1.27, -0.5, 0.005, 0.015])
    s = oracle.endpoint_scale(a, 8)
    assert abs(s - 0.01) < 1e-17
    assert list(oracle.quantize_with_scale(a, 0.01, 8)) == [127, -50, 0, 2]
    # negative-only row: max(0, max A) = 0, so s = 2.56 / 128 and -2.56 -> -128
    a = np.array([-2.56, -1.0])
    assert oracle.endpoint_scale(a, 8) == 2.56 / 128
    assert list(oracle.quantize_with_scale(a, 2.56 / 128, 8)) == [-128, -50]


def test_weight_quant_clips_and_ties_even():
    # scale 1: 2.5 -> 2, 3.5 -> 4, -2.5 -> -2; 9 -> 7 and -9.4 -> -8 clip at the 4-bit range
    a = np.array([2.5, 3.5, -2.5, 9.0, -9.4])
    assert list(oracle.quantize_with_scale(a, 1.0, 4)) == [2, 4, -2, 7, -8]


def test_weight_quant_zero_row_floor_and_fp16_underflow():
    w = np.zeros((2, 128), np.float32)
    pmap = np.array([[1]], np.uint8)
    for search in (False, True):
        codes, scales = oracle.quantize_weights(w, pmap, 2, 128, search)
        assert not codes.any()
        assert np.all(scales == 0)  # 1e-12 underflows fp16 to +0
    assert oracle.search_scale(np.zeros(4), 8) == 1e-12


def test_weight_search_recovers_grid_row_exactly():
    # A = s q with q reaching both 4-bit ends: every smaller grid scale clips 7,
    # so the first zero-error scale is i = 96, (1/4 + 96/128) s0 = s0 = s.
    q = np.array([7, -8, 1, 0, 3, -5])
    s = 0.0390625
    assert oracle.search_scale(q * s, 4) == s


def test_weight_search_matches_code_brute_force():
    # For each grid scale, minimise the error over ALL code vectors in range
    # (no rounding rule used), then over the grid with earliest-index ties; the
    # oracle's search must reach the same scale and error.
    rng = np.random.default_rng(7)
    for b in (4, 3):
        lo, hi = -(2 ** (b - 1)), 2 ** (b - 1) - 1
        grid = np.arange(lo, hi + 1, dtype=np.float64)
        for trial in range(6):
            a = rng.standard_normal(3) * (0.1 if trial % 2 else 3.0)
            if trial == 5:
                a[0] = 40.0 * abs(a[1])  # one large element: search shrinks the scale
            amax = max(max(0.0, a.max()) / hi, max(0.0, -a.min()) / -lo, 1e-12)
            best = None
            for i in range(129):
                si = max((0.25 + i / 128.0) * amax, 1e-12)
                e = 0.0
                for v in a:  # each element independently: min over the code alphabet
                    e += float(np.min((v - si * grid) ** 2))
                if best is None or e < best[1] - 1e-15 * max(1.0, best[1]):
                    best = (si, e)
            s = oracle.search_scale(a, b)
            e = oracle.squared_error(a, s, oracle.quantize_with_scale(a, s, b))
            assert abs(e - best[1]) <= 1e-12 * max(1.0, best[1])
            assert oracle.squared_error(a, s, oracle.quantize_with_scale(a, s, b)) <= \
                oracle.squared_error(a, amax, oracle.quantize_with_scale(a, amax, b))


def test_weight_search_shrinks_scale_for_an_outlier_row():
    # 0.9 and twenty values of 0.1: with s0 = 0.9/7 the small values round to 1
    # (0.1/0.1286 = 0.78), each off by 0.0286; a smaller scale must win.
    a = np.array([0.9] + [0.1] * 20)
    s0 = oracle.endpoint_scale(a, 4)
    s = oracle.search_scale(a, 4)
    assert s < s0
    e = lambda t: oracle.squared_error(a, t, oracle.quantize_with_scale(a, t, 4))
    assert e(s) < e(s0)


def test_quantize_weights_layout_bits_and_bound():
    N, K, bN, bK = 8, 256, 4, 128
    w = synth.float_weights(N, K, (11,), outlier_frac=0.01)
    pmap = np.array([[1, 0], [0, 1]], np.uint8)
    codes, scales = oracle.quantize_weights(w, pmap, bN, bK, search=False)
    assert codes.shape == (N, K) and scales.shape == (N, 2) and scales.dtype == np.float16
    wv = w.astype(np.float64)
    for n in range(N):
        for j in range(2):
            a = wv[n, j * bK:(j + 1) * bK]
            b = 4 if pmap[n // bN, j] == 1 else 8
            c = codes[n, j * bK:(j + 1) * bK].astype(int)
            assert c.min() >= -(2 ** (b - 1)) and c.max() <= 2 ** (b - 1) - 1
            # the endpoint scale never clips: every element within half a step
            s = max(a.max() / (2 ** (b - 1) - 1), -a.min() / 2 ** (b - 1))
            assert np.abs(a - s * c).max() <= s / 2 * (1 + 1e-12)
            assert scales[n, j] == np.float16(s)
            # the largest magnitude reaches a range end
            assert c.max() == 2 ** (b - 1) - 1 or c.min() == -(2 ** (b - 1))
    # the codes pack: INT4 tiles stay within 4 bits
    oracle.pack(codes, scales, pmap, bN, bK)
    # search never does worse than the endpoint, row by row
    codes_s, scales_s = oracle.quantize_weights(w[:2], pmap[:1], 2, bK, search=True)
    for n in range(2):
        for j in range(2):
            a = wv[n, j * bK:(j + 1) * bK]
            b = 4 if pmap[0, j] == 1 else 8
            s = oracle.search_scale(a, b)
            c = codes_s[n, j * bK:(j + 1) * bK]
            assert np.array_equal(c, oracle.quantize_with_scale(a, s, b))
            assert oracle.squared_error(a, s, c) <= \
                oracle.squared_error(a, oracle.endpoint_scale(a, b), codes[n, j * bK:(j + 1) * bK])
