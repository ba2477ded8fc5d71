"""Pins of the oracle of the paper's own numerics (App. B.1-B.3, eq. 4, 5-7,
19) to facts that do not come from the oracle itself: the closed form of the
Sylvester Hadamard entries, orthogonality, the eq. 4 identity before
quantization, hand-worked activation groups, brute-force loops for eq. 19,
and exact recovery of on-grid inputs."""
import numpy as np
import pytest

import oracle

pn = oracle.aq_paper_numerics


def _popcount(v: int) -> int:
    return bin(v).count("1")


def test_hadamard64_matches_closed_form_and_is_orthogonal():
    h = pn.hadamard64()
    # Sylvester's construction in closed form: H[i, j] = (-1)^popcount(i & j), scaled by 1/8
    want = np.array([[(-1) ** _popcount(i & j) for j in range(64)] for i in range(64)]) / 8.0
    assert np.array_equal(h, want)
    assert np.array_equal(h @ h.T, np.eye(64))  # every entry is a sum of +-1/64 terms: exact
    assert np.array_equal(h, h.T)


def test_seed_matrices_are_orthogonal():
    rng = np.random.default_rng(1)
    for kind in (-1, 0, 1, 6):
        phi = pn.seed_matrix(kind, rng.permutation(64), rng.choice([-1, 1], 64), rng.choice([-1, 1], 64))
        assert np.abs(phi @ phi.T - np.eye(64)).max() < 1e-14
    p = rng.permutation(64)
    phi = pn.seed_matrix(2, p, np.ones(64), np.ones(64))
    assert np.array_equal(phi, pn.hadamard64()[p])  # P H with P[i, p[i]] = 1 picks rows p


def test_eq4_identity_before_quantization():
    # (X V)(U W V)^T U = X W^T for orthogonal block-diagonal U, V
    rng = np.random.default_rng(2)
    M, N, K = 5, 128, 192
    x = rng.standard_normal((M, K))
    w = rng.standard_normal((N, K))
    seeds = lambda n: [pn.seed_matrix(int(k), rng.permutation(64), rng.choice([-1, 1], 64), rng.choice([-1, 1], 64))
                       for k in rng.integers(-1, 7, n)]
    U = pn.block_diag([s.T for s in seeds(N // 64)])
    V = pn.block_diag(seeds(K // 64))
    assert np.abs((x @ V) @ (U @ w @ V).T @ U - x @ w.T).max() < 1e-12 * np.abs(x @ w.T).max() * K


def test_activation_groups_hand_worked():
    # one row (b_M = 1), two 64-feature groups
    x = np.zeros((1, 128))
    x[0, :4] = [2.54, -1.0, 0.0, 0.01]      # s = max(2.54 / 127, 1.0 / 128) = 0.02
    x[0, 64:67] = [-2.56, 1.0, 0.03]        # s = max(1.0 / 127, 2.56 / 128) = 0.02, -2.56 -> -128
    q, s, Mp = pn.quantize_activation_groups(x)
    assert Mp == 1 and s.shape == (1, 2)
    assert s[0, 0] == np.float32(0.02) and s[0, 1] == np.float32(0.02)
    assert list(q[0, :4]) == [127, -50, 0, 0]       # 0.01 / 0.02 = 0.5 -> 0 (ties to even)
    assert list(q[0, 64:67]) == [-128, 50, 2]       # 0.03 / 0.02 = 1.5 -> 2
    # all-zero group: floor 1e-12, codes zero
    q, s, _ = pn.quantize_activation_groups(np.zeros((1, 64)))
    assert s[0, 0] == np.float32(1e-12) and not q.any()


def test_activation_row_groups_and_padding():
    assert pn.row_group(1) == 1 and pn.row_group(2) == 16 and pn.row_group(300) == 16
    rng = np.random.default_rng(3)
    x = rng.standard_normal((17, 64))
    q, s, Mp = pn.quantize_activation_groups(x)
    assert Mp == 32 and q.shape == (32, 64) and s.shape == (2, 1)
    assert not q[17:].any()                          # padded rows quantize to zero
    # group 1 holds only row 16 (plus zero padding): its scale is that row's endpoint scale
    r = x[16]
    assert s[1, 0] == np.float32(max(max(0, r.max()) / 127, max(0, -r.min()) / 128))
    g0 = x[:16]
    assert s[0, 0] == np.float32(max(max(0, g0.max()) / 127, max(0, -g0.min()) / 128))


def test_weight_tiles_use_the_whole_tile():
    # an INT4 tile whose largest magnitude sits in its last row: every row shares that scale
    w = np.full((64, 64), 0.01)
    w[63, 5] = -0.8                                  # endpoint scale 0.8 / 8 = 0.1
    codes, scales = pn.quantize_weight_tiles(w, np.array([[1]], np.uint8), 64, 64, search=False)
    assert scales[0, 0] == np.float32(0.1)
    assert codes[63, 5] == -8 and codes[0, 0] == 0   # 0.01 / 0.1 = 0.1 -> 0


def _brute_force_eq19(xq, sx, qw, sw, bN, bK, M):
    Mp, K = xq.shape
    N = qw.shape[0]
    bM = pn.row_group(M)
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(sx[m // bM, k // 64]) * float(sw[n // bN, k // bK]) * int(xq[m, k]) * int(qw[n, k])
            y[m, n] = acc
    return y


@pytest.mark.parametrize("M,bK", [(1, 64), (3, 128), (18, 64)])
def test_eq19_matches_brute_force(M, bK):
    rng = np.random.default_rng(4 + M)
    N, K, bN = 8, 256, 4
    xq = rng.integers(-128, 128, (-(-M // pn.row_group(M)) * pn.row_group(M), K)).astype(np.int8)
    qw = rng.integers(-128, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-3, 1e-1, (xq.shape[0] // pn.row_group(M), K // 64)).astype(np.float32)
    sw = rng.uniform(1e-3, 1e-1, (N // bN, K // bK)).astype(np.float32)
    y = pn.reconstruct_groups(xq, sx, qw, sw, bN, bK, M)
    assert np.allclose(y, _brute_force_eq19(xq, sx, qw, sw, bN, bK, M), rtol=1e-12, atol=1e-12)


def test_on_grid_inputs_are_recovered_exactly():
    # identity transforms; X and W already on their quantization grids with
    # power-of-two scales, each group / tile reaching its positive endpoint,
    # so every quantizer is exact and the layer returns X W^T exactly
    rng = np.random.default_rng(5)
    M, N, K, bN, bK = 1, 128, 128, 64, 64
    x = rng.integers(-127, 128, (M, K)).astype(np.float64)
    x[0, 0] = x[0, 64] = 127
    x *= 2.0 ** -6
    pmap = np.array([[1, 0], [0, 1]], np.uint8)
    w = np.zeros((N, K))
    for r in range(2):
        for j in range(2):
            hi = 7 if pmap[r, j] else 127
            t = rng.integers(-hi, hi + 1, (bN, bK)).astype(np.float64)
            t[0, 0] = hi
            w[r * bN:(r + 1) * bN, j * bK:(j + 1) * bK] = t * 2.0 ** -(5 + r + j)
    out = pn.paper_linear(x, w, pmap, bN, bK)
    assert np.array_equal(out["y"], x @ w.T)


def test_power_of_two_scaling_is_exact():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((20, 128))
    w = rng.standard_normal((64, 128)) * 0.05
    pmap = np.array([[1, 0]], np.uint8)
    h = pn.hadamard64()
    a = pn.paper_linear(x, w, pmap, 64, 64, u_blocks=[h], v_blocks=[h, h])
    b = pn.paper_linear(x * 8.0, w, pmap, 64, 64, u_blocks=[h], v_blocks=[h, h])
    assert np.array_equal(b["xq"], a["xq"])
    assert np.array_equal(b["y"], a["y"] * 8.0)


def test_transforms_restore_output_coordinates():
    # all-INT8 tiles with non-symmetric seeds: the quantized layer stays within the
    # INT8 quantization error of X W^T; a transform applied on the wrong side or
    # transposed would scramble the outputs (errors of the order of the outputs)
    rng = np.random.default_rng(7)
    M, N, K = 20, 128, 128
    x = rng.standard_normal((M, K))
    w = rng.standard_normal((N, K)) * 0.05
    mk = lambda: pn.seed_matrix(int(rng.integers(1, 7)), rng.permutation(64), rng.choice([-1, 1], 64),
                                rng.choice([-1, 1], 64))
    u = [mk().T for _ in range(2)]
    v = [mk() for _ in range(2)]
    assert not np.allclose(u[0], u[0].T)
    out = pn.paper_linear(x, w, np.zeros((2, 2), np.uint8), 64, 64, u_blocks=u, v_blocks=v)
    ref = x @ w.T
    assert np.abs(out["y"] - ref).max() < 0.02 * np.abs(ref).max()
