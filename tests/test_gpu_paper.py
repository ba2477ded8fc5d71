"""The paper-exact mode on the GPU against the oracle of the paper's own
numerics (AlignQuant App. B.1 eq. 4, App. B.3, App. E.2, App. E.3 eq. 19):
transformed and group-quantized activations bit-exact, integer tile products
bit-exact, outputs within the layer's tolerance of the oracle's fp64 result,
with non-identity transform seeds on both sides."""
import numpy as np
import pytest
import torch

import oracle
from aq_testutil import assert_output_close, dev_bf16
from w8_a8_quantized_b200 import aq, synth

pytestmark = pytest.mark.gpu
pn = oracle.aq_paper_numerics


def _bf16_values(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _seeds(n_blocks: int, rng, kinds=(0, 1, 3, -1)):
    """One 64 x 64 seed per block, cycling through I, H_64 and D_L P H_64 D_R."""
    out = []
    for b in range(n_blocks):
        kind = kinds[b % len(kinds)]
        out.append(pn.seed_matrix(kind, rng.permutation(64), rng.choice([-1, 1], 64), rng.choice([-1, 1], 64)))
    return out


def _u_blocks(R: int, bN: int, rng):
    """bN x bN orthogonal output blocks: one seed (bN = 64) or two seeds on the diagonal (bN = 128)."""
    per = bN // 64
    seeds = _seeds(R * per, rng, kinds=(3, 0, 1))
    return [pn.block_diag(seeds[r * per:(r + 1) * per]) for r in range(R)]


def _dev_f32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float32))).cuda()


@pytest.mark.parametrize("M,K", [(1, 64), (1, 576), (7, 256), (16, 128), (40, 320)])
def test_identity_transform_equals_group_quantizer(M, K):
    x = synth.activations(M, K, (2100 + M, K), outlier_frac=0.02)
    xq, sx = aq.aq_paper_quant_act(dev_bf16(x))
    xq_g, sx_g = aq.aq_quant_act_groups(dev_bf16(x))
    assert torch.equal(xq, xq_g) and torch.equal(sx, sx_g)
    xq_ref, sx_ref, _ = pn.quantize_activation_groups(_bf16_values(x))
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(sx.cpu().numpy(), sx_ref)


@pytest.mark.parametrize("M,K", [(1, 64), (1, 1024), (3, 192), (16, 256), (33, 576)])
def test_transformed_activations_bit_exact(M, K):
    """X~ = X V with Hadamard-type seeds (entries 0, +-1, +-1/8): codes and fp32
    scales equal the oracle's quantization of its fp64 X V."""
    rng = np.random.default_rng(M * 1000 + K)
    v_blocks = _seeds(K // 64, rng)
    x = synth.activations(M, K, (2200 + M, K), outlier_frac=0.02)
    xq, sx = aq.aq_paper_quant_act(dev_bf16(x), _dev_f32(np.stack(v_blocks)))
    x_t = _bf16_values(x) @ pn.block_diag(v_blocks)
    xq_ref, sx_ref, Mp = pn.quantize_activation_groups(x_t)
    assert xq.shape == (Mp, K)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(sx.cpu().numpy(), sx_ref)


def _paper_case(M, N, K, bN, frac8, seed, search=False, with_bias=True):
    rng = np.random.default_rng(seed)
    R, C = N // bN, K // 64
    pmap = synth.precision_map(R, C, frac8, (seed, 1))
    w = synth.float_weights(N, K, (seed, 2), outlier_frac=0.005)
    x_bits = synth.activations(M, K, (seed, 3), outlier_frac=0.01)
    v_blocks = _seeds(C, rng)
    u_blocks = _u_blocks(R, bN, rng)
    bias = rng.standard_normal(N).astype(np.float32) if with_bias else None
    ref = pn.paper_linear(_bf16_values(x_bits), w, pmap, bN, 64, u_blocks, v_blocks, search=search, bias=bias)
    packed = aq.aq_pack_tiles(torch.from_numpy(ref["qw"]).cuda(), torch.from_numpy(ref["sw"]).cuda(),
                              torch.from_numpy(pmap).cuda(), bN, 64)
    return ref, packed, x_bits, v_blocks, u_blocks, bias


@pytest.mark.parametrize("M", [1, 5, 16, 33])
@pytest.mark.parametrize("N,K,bN,frac8", [(256, 576, 64, 0.4), (384, 320, 128, 0.25), (128, 1024, 64, 1.0),
                                          (128, 256, 128, 0.0)])
def test_paper_linear_matches_oracle(M, N, K, bN, frac8):
    ref, packed, x_bits, v_blocks, u_blocks, bias = _paper_case(M, N, K, bN, frac8, 2300 + M + N + K)
    assert packed.struct.scale_kind == aq.AQ_SCALES_TILE_FP32
    xq, sx = aq.aq_paper_quant_act(dev_bf16(x_bits), _dev_f32(np.stack(v_blocks)))
    assert np.array_equal(xq.cpu().numpy(), ref["xq"]) and np.array_equal(sx.cpu().numpy(), ref["sx"])
    # exact integer tile products (eq. 19's P) against plain integer sums of the oracle's codes
    P = aq.aq_debug_paper_partials(packed, xq, M).cpu().numpy()
    xq64, qw64 = ref["xq"][:M].astype(np.int64), ref["qw"].astype(np.int64)
    want = np.stack([xq64[:, j * 64:(j + 1) * 64] @ qw64[:, j * 64:(j + 1) * 64].T for j in range(K // 64)], axis=-1)
    assert np.array_equal(P, want)
    y = aq.aq_paper_linear(packed, xq, sx, M, u=_dev_f32(np.stack(u_blocks)), bias=_dev_f32(bias))
    assert_output_close(y, ref["y"])


def test_paper_linear_without_transforms_and_with_search():
    """U = V = I (the paper's seed Phi_-1) and weights from the eq. 7 scale search."""
    M, N, K, bN = 2, 128, 128, 64
    pmap = synth.precision_map(N // bN, K // 64, 0.5, (2400, 1))
    w = synth.float_weights(N, K, (2400, 2), outlier_frac=0.01)
    x_bits = synth.activations(M, K, (2400, 3))
    ref = pn.paper_linear(_bf16_values(x_bits), w, pmap, bN, 64, search=True)
    packed = aq.aq_pack_tiles(torch.from_numpy(ref["qw"]).cuda(), torch.from_numpy(ref["sw"]).cuda(),
                              torch.from_numpy(pmap).cuda(), bN, 64)
    xq, sx = aq.aq_paper_quant_act(dev_bf16(x_bits))
    y = aq.aq_paper_linear(packed, xq, sx, M)
    assert_output_close(y, ref["y"])


def test_paper_operands_are_checked_before_any_launch():
    """Codes, scales and token counts that do not match the packed weights raise
    on the host: the kernels read xq as [M'][K] and sx as [M'/b_M][K/64]."""
    _, packed, x_bits, v_blocks, _, _ = _paper_case(5, 256, 576, 64, 0.4, 2500)
    xq, sx = aq.aq_paper_quant_act(dev_bf16(x_bits), _dev_f32(np.stack(v_blocks)))
    assert xq.shape == (16, 576) and sx.shape == (1, 9)
    with pytest.raises(ValueError):
        aq.aq_paper_linear(packed, xq[:, :512].contiguous(), sx, 5)   # K does not match the weights
    with pytest.raises(ValueError):
        aq.aq_paper_linear(packed, xq, sx, 17)                        # 17 tokens pad to 32 code rows
    with pytest.raises(ValueError):
        aq.aq_paper_linear(packed, xq, sx[:, :4].contiguous(), 5)     # fewer group scales than tiles
    with pytest.raises(ValueError):
        aq.aq_paper_linear(packed, xq, sx, 0)
    with pytest.raises(ValueError):
        aq.aq_debug_paper_partials(packed, xq, 17)
