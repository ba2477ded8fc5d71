"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer and byte results (packed buffers, activation codes and scales, per-tile
INT32 products) must be bit-exact.  Floating-point outputs must meet the
tolerance in aq_testutil.assert_output_close.  Sizes span several tiles with
ragged token counts and, for 64-row tiles, an odd number of tile rows."""
import functools

import numpy as np
import pytest
import torch

import oracle
from aq_testutil import assert_output_close, dev_bf16, dev_projection, oracle_linear, packed_case
from w8_a8_quantized_b200 import aq, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _no_kernel_errors():
    yield
    aq.check_all_workspaces()


# ------------------------------------------------------------------ packer

@pytest.mark.parametrize("N,K,bN,frac8,seed", [
    (256, 384, 128, 0.5, 1), (192, 256, 64, 0.25, 2), (128, 128, 128, 1.0, 3), (128, 256, 128, 0.0, 4),
    (640, 1280, 64, 0.5, 5), (1024, 3072, 128, 0.25, 6)])
def test_pack_matches_oracle(N, K, bN, frac8, seed):
    p = synth.projection_inputs(N, K, bN, 128, frac8, (seed,))
    w = aq.aq_pack(*dev_projection(p), bN, 128)
    ref = oracle.pack(p.codes, p.scales, p.pmap, bN, 128)
    got = w.host_buffers()
    assert (w.T4, w.T8, w.R, w.C) == (ref["T4"], ref["T8"], ref["R"], ref["C"])
    for name in aq.BUF_NAMES:
        want = np.ascontiguousarray(ref[name]).view(np.uint8).reshape(-1)
        assert np.array_equal(got[name], want), name


def test_pack_rejects_int4_code_out_of_range():
    p = synth.projection_inputs(256, 256, 128, 128, 0.5, (9,))
    r, j = map(int, np.argwhere(p.pmap == 1)[0])
    for bad in (8, -9):
        codes = p.codes.copy()
        codes[r * 128 + 3, j * 128 + 77] = bad
        with pytest.raises(aq.AqError) as e:
            aq.aq_pack(*dev_projection(synth.SingleProjection(p.N, p.K, 128, 128, p.pmap, codes, p.scales)), 128, 128)
        assert e.value.status == -3


# ------------------------------------------------------------------ activation quantization

@pytest.mark.parametrize("M,K,pad,outlier", [(1, 128, 0, 0.0), (3, 2048, 8, 0.0), (17, 3072, 0, 0.01),
                                             (2, 17408, 0, 0.01), (2, 40960, 16, 0.0), (64, 640, 0, 0.01)])
def test_quant_act_bit_exact(M, K, pad, outlier):
    x = synth.activations(M, K + pad, (M, K, pad), outlier_frac=outlier)
    x[0, : K // 2] = 0                       # partial zero row
    if M > 2:
        x[2, :K] = 0                         # all-zero row: scale floor
    xd = dev_bf16(x)
    xq, sx = aq.aq_quant_act(xd, K=K)
    xq_ref, sx_ref = oracle.quant_act(x[:, :K])
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), sx_ref.view(np.uint32))


def test_quant_act_ties_round_half_even():
    x = np.array([[127.0, 2.5, -2.5, 3.5, 0.5, 1.5, -0.5, -127.0] * 2], np.float32)
    xq, sx = aq.aq_quant_act(dev_bf16(synth.f32_to_bf16_bits(x)))
    assert list(xq.cpu().numpy()[0][:8]) == [127, 2, -2, 4, 0, 2, 0, -127]
    assert sx.item() == 1.0


# ------------------------------------------------------------------ exact per-tile products

@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 16, 17, 33, 64])
@pytest.mark.parametrize("bN", [128, 64])
def test_decode_tile_products_bit_exact(M, bN):
    p, x, w, xq, sx = packed_case(bN * 5, 128 * 6, bN, 0.5, 100 + M, M)
    P = aq.aq_debug_tile_partials(w, xq, aq.AQ_PHASE_DECODE)
    assert np.array_equal(xq.cpu().numpy(), oracle.quant_act(x)[0])
    ref = oracle.tile_partials(p.codes, oracle.quant_act(x)[0], 128)
    assert np.array_equal(P.cpu().numpy(), ref)


@pytest.mark.parametrize("M", [1, 64, 100, 257, 300])
@pytest.mark.parametrize("bN,frac8", [(128, 0.5), (64, 0.25), (128, 0.0), (128, 1.0)])
def test_prefill_tile_products_bit_exact(M, bN, frac8):
    p, x, w, xq, sx = packed_case(bN * 5, 128 * 7, bN, frac8, 200 + M, M)
    P = aq.aq_debug_tile_partials(w, xq, aq.AQ_PHASE_PREFILL)
    ref = oracle.tile_partials(p.codes, oracle.quant_act(x)[0], 128)
    assert np.array_equal(P.cpu().numpy(), ref)


# ------------------------------------------------------------------ outputs

@pytest.mark.parametrize("M", [1, 2, 4, 7, 8, 12, 16, 32, 40, 64])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_matches_oracle(M, out_dtype):
    N, K = 640, 1536
    p, x, w, xq, sx = packed_case(N, K, 128, 0.25, 300 + M, M, outlier=0.01)
    bias = np.linspace(-2, 2, N).astype(np.float32)
    y = aq.aq_linear_decode(w, xq, sx, bias=torch.from_numpy(bias).cuda(), out_dtype=out_dtype)
    assert_output_close(y, oracle_linear(p, x, bias=bias))


@pytest.mark.parametrize("M", [1, 3, 8, 33])
def test_decode_64_row_tiles_and_strided_output(M):
    N, K = 64 * 7, 128 * 9
    p, x, w, xq, sx = packed_case(N, K, 64, 0.5, 400 + M, M)
    out = torch.full((M, N + 32), 7.0, device="cuda")
    aq.aq_linear_decode(w, xq, sx, out=out[:, :N])
    assert_output_close(out[:, :N], oracle_linear(p, x))
    assert (out[:, N:] == 7.0).all()


@pytest.mark.parametrize("M", [1, 50, 128, 300, 700])
@pytest.mark.parametrize("bN,frac8", [(128, 0.4), (64, 0.3)])
def test_prefill_matches_oracle(M, bN, frac8):
    N, K = bN * 9, 128 * 10
    p, x, w, xq, sx = packed_case(N, K, bN, frac8, 500 + M, M, outlier=0.01)
    bias = np.linspace(-1, 1, N).astype(np.float32)
    y = aq.aq_linear_prefill(w, xq, sx, bias=torch.from_numpy(bias).cuda())
    assert_output_close(y, oracle_linear(p, x, bias=bias))
    yb = aq.aq_linear_prefill(w, xq, sx, out_dtype=torch.bfloat16)
    assert_output_close(yb, oracle_linear(p, x))


@pytest.mark.parametrize("N,K,M", [(1024, 3072, 8), (1024, 3072, 16), (1024, 8192, 40), (512, 8192, 64)])
def test_split_reduction_is_deterministic(N, K, M):
    """Tensor-core decode with split-K partial sums (the workspace holds them):
    repeated calls agree bit for bit and match the oracle."""
    p, x, w, xq, sx = packed_case(N, K, 128, 0.25, 600 + M, M)
    assert aq.aq_workspace_bytes(aq.AQ_PHASE_DECODE, M, w) >= 2 * M * N * 4  # at least two splits
    ys = [aq.aq_linear_decode(w, xq, sx).cpu().numpy() for _ in range(3)]
    assert all(np.array_equal(ys[0].view(np.uint32), y.view(np.uint32)) for y in ys[1:])
    assert_output_close(torch.from_numpy(ys[0]), oracle_linear(p, x))


@pytest.mark.parametrize("phase,M", [(0, 1), (0, 8), (0, 32), (1, 300)])
def test_exact_sign_and_power_of_two_symmetry(phase, M):
    """y(-X) = -y(X) and y(2^e X) = 2^e y(X) hold exactly for the GPU path too."""
    p = synth.projection_inputs(512, 1024, 128, 128, 0.5, (700 + M,))
    w = aq.aq_pack(*dev_projection(p), 128, 128)
    x = synth.activations(M, 1024, (701 + M,))
    xf = oracle.bf16_bits_to_f64(x).astype(np.float32)
    run = aq.aq_linear_decode if phase == 0 else aq.aq_linear_prefill

    def y_of(xbits):
        xq, sx = aq.aq_quant_act(dev_bf16(xbits))
        return run(w, xq, sx).cpu().numpy()

    y = y_of(x)
    assert np.array_equal(y_of(synth.f32_to_bf16_bits(-xf)), -y)
    assert np.array_equal(y_of(synth.f32_to_bf16_bits(xf * np.float32(8.0))), y * 8)


def test_decode_and_prefill_agree_on_products():
    p, x, w, xq, sx = packed_case(384, 1024, 128, 0.5, 800, 24)
    Pd = aq.aq_debug_tile_partials(w, xq, aq.AQ_PHASE_DECODE)
    Pp = aq.aq_debug_tile_partials(w, xq, aq.AQ_PHASE_PREFILL)
    assert torch.equal(Pd, Pp)


def test_device_errors_are_reported():
    p, x, w, xq, sx = packed_case(256, 256, 128, 0.5, 900, 4)
    with pytest.raises(aq.AqError) as e:
        aq.aq_linear_decode(w, xq, sx, ws=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == -5
    big = torch.zeros((65, 256), dtype=torch.int8, device="cuda")
    with pytest.raises(aq.AqError) as e:
        aq.aq_linear_decode(w, big, torch.ones(65, device="cuda"), ws=aq.workspace(0, 4, w))
    assert e.value.status == -1


# ------------------------------------------------------------------ fast quantization path: ties and near-ties

def test_quant_act_exact_ties_everywhere():
    """amax = 127 * 2^e makes s = 2^e exact, and every (k + 0.5) 2^e is a tie."""
    rows = []
    for e in (-6, 0, 3):
        ks = np.arange(0, 127)
        vals = np.concatenate([(ks + 0.5), -(ks + 0.5), [127.0]]) * 2.0 ** e
        vals = np.concatenate([vals, np.zeros(256 - vals.size)])
        rows.append(vals)
    x = synth.f32_to_bf16_bits(np.array(rows, np.float32))
    xq, sx = aq.aq_quant_act(dev_bf16(x))
    xq_ref, sx_ref = oracle.quant_act(x)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(sx.cpu().numpy(), sx_ref)


def test_quant_act_million_random_elements():
    x = synth.activations(256, 4096, (31337,), outlier_frac=0.01)
    xq, sx = aq.aq_quant_act(dev_bf16(x))
    xq_ref, sx_ref = oracle.quant_act(x)
    assert np.array_equal(xq.cpu().numpy(), xq_ref)
    assert np.array_equal(sx.cpu().numpy(), sx_ref)


# ------------------------------------------------------------------ shared-input groups

def _group_case(shapes, M, seed, phase, bN=128, frac8=0.25):
    ps = [synth.projection_inputs(N, K, bN, 128, frac8, (seed, g)) for g, (N, K) in enumerate(shapes)]
    ws = [aq.aq_pack(*dev_projection(p), bN, 128) for p in ps]
    x = synth.activations(M, shapes[0][1], (seed, 9), outlier_frac=0.01)
    return ps, ws, x


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K,bN", [(256, 6144, 128), (384, 5120, 64), (1536, 4096, 128)])
def test_decode_long_rows_reuse_every_ring_slot(M, N, K, bN):
    """Few rows per CTA and long rows: every CTA of the streaming decode kernel
    walks many more stages than its ring has slots (each slot is refilled several
    times, across row blocks), so the ring's phase bookkeeping is exercised.
    Outputs against the oracle, per-tile products bit-exact."""
    p, x, w, xq, sx = packed_case(N, K, bN, 0.3, 1400 + M + N, M, outlier=0.01)
    assert_output_close(aq.aq_linear_decode(w, xq, sx), oracle_linear(p, x))
    P = aq.aq_debug_tile_partials(w, xq, aq.AQ_PHASE_DECODE)
    assert np.array_equal(P.cpu().numpy(), oracle.tile_partials(p.codes, oracle.quant_act(x)[0], 128))


@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("N,K,bN", [(4096, 8192, 128), (2560, 14336, 64)])
def test_decode_wide_launch(M, N, K, bN):
    """Launches above 200 K weights per SM: at 1 token the streaming kernel takes
    its wide shape (16 warps, 3-stage rings, one CTA per SM).  Outputs against
    the oracle, per-tile products bit-exact."""
    p, x, w, xq, sx = packed_case(N, K, bN, 0.4, 1600 + M + N, M, outlier=0.01)
    assert_output_close(aq.aq_linear_decode(w, xq, sx), oracle_linear(p, x))
    P = aq.aq_debug_tile_partials(w, xq, aq.AQ_PHASE_DECODE)
    assert np.array_equal(P.cpu().numpy(), oracle.tile_partials(p.codes, oracle.quant_act(x)[0], 128))


def test_group_fused_wide_launch():
    """A gate/up-style group of 2 x 8192 rows over K = 4096 at 1 token: one fused
    launch (activation preparation inside) in the wide shape."""
    shapes = [(8192, 4096), (8192, 4096)]
    ps, ws, x = _group_case(shapes, 1, 1700, aq.AQ_PHASE_DECODE)
    grp = aq.Group(ws, aq.AQ_PHASE_DECODE, 1)
    outs = [torch.empty((1, N), device="cuda") for N, _ in shapes]
    for _ in range(2):
        grp(dev_bf16(x), outs)
    for p, o in zip(ps, outs):
        assert_output_close(o, oracle_linear(p, x))
    rc, _ = aq.aq_workspace_status(grp.ws)
    assert rc == 0


@pytest.mark.parametrize("M", [1, 2])
def test_group_fused_long_rows(M):
    """A fused q/k/v-style group whose CTAs each stream several row blocks of 40
    tile columns (ring slots refilled many times)."""
    shapes = [(1024, 5120), (256, 5120), (256, 5120)]
    ps, ws, x = _group_case(shapes, M, 1500 + M, aq.AQ_PHASE_DECODE)
    grp = aq.Group(ws, aq.AQ_PHASE_DECODE, M)
    outs = [torch.empty((M, N), device="cuda") for N, _ in shapes]
    for _ in range(3):  # repeated calls reuse the same graph of barriers from a clean start
        grp(dev_bf16(x), outs)
    for p, o in zip(ps, outs):
        assert_output_close(o, oracle_linear(p, x))
    rc, _ = aq.aq_workspace_status(grp.ws)
    assert rc == 0


@pytest.mark.parametrize("M", [1, 3, 8])
def test_decode_wide_layer_matches_oracle(M):
    """A layer wider than one 32-row CUDA-core block per SM (so blocks queue
    behind each other); bf16 output, with bias."""
    N, K = 4864, 1024
    p, x, w, xq, sx = packed_case(N, K, 128, 0.25, 1200 + M, M, outlier=0.01)
    bias = np.linspace(-1, 1, N).astype(np.float32)
    y = aq.aq_linear_decode(w, xq, sx, bias=torch.from_numpy(bias).cuda(), out_dtype=torch.bfloat16)
    assert_output_close(y, oracle_linear(p, x, bias=bias))
    aq.check_all_workspaces()


@pytest.mark.parametrize("M", [1, 2, 5, 8, 9, 24, 64])
@pytest.mark.parametrize("members", [3, 2])
def test_group_decode_matches_separate_calls_and_oracle(M, members):
    shapes = [(768, 1024), (256, 1024), (256, 1024)][:members]
    ps, ws, x = _group_case(shapes, M, 1000 + M, aq.AQ_PHASE_DECODE)
    xd = dev_bf16(x)
    grp = aq.Group(ws, aq.AQ_PHASE_DECODE, M)
    outs = [torch.empty((M, N), device="cuda") for N, _ in shapes]
    biases = [torch.linspace(-1, 1, N, device="cuda") for N, _ in shapes]
    grp(xd, outs, bias=biases)
    xq, sx = aq.aq_quant_act(xd)
    for g, (p, w) in enumerate(zip(ps, ws)):
        sep = aq.aq_linear_decode(w, xq, sx, bias=biases[g])
        # same kernel family and split plan as the separate call (whole 128-row blocks per member)
        assert torch.equal(outs[g], sep), g
        assert_output_close(outs[g], oracle_linear(p, x, bias=biases[g].cpu().numpy()))
        assert_output_close(sep, oracle_linear(p, x, bias=biases[g].cpu().numpy()))
    aq.check_all_workspaces()
    rc, _ = aq.aq_workspace_status(grp.ws)
    assert rc == 0


@pytest.mark.parametrize("M", [5, 8])
def test_group_rows_launch_for_ragged_members(M):
    """Three members whose rows are not whole 128-row blocks (64-row tiles, odd
    tile-row counts) cannot share a tensor-core launch; up to 8 tokens they run as
    one CUDA-core launch over the codes."""
    shapes = [(320, 1024), (192, 1024), (64, 1024)]
    ps, ws, x = _group_case(shapes, M, 1200 + M, aq.AQ_PHASE_DECODE, bN=64, frac8=0.3)
    grp = aq.Group(ws, aq.AQ_PHASE_DECODE, M)
    outs = [torch.empty((M, N), device="cuda") for N, _ in shapes]
    grp(dev_bf16(x), outs)
    for p, o in zip(ps, outs):
        assert_output_close(o, oracle_linear(p, x))
    rc, _ = aq.aq_workspace_status(grp.ws)
    assert rc == 0


@pytest.mark.parametrize("M,K,bN", [(16, 4096, 128), (40, 8192, 128), (24, 4096, 64), (64, 2048, 64)])
def test_group_tensor_core_launch(M, K, bN):
    """A decode group on the tensor cores runs as one launch over the members'
    concatenated 128-row blocks (split-K partial sums included where the plan
    splits): bf16 outputs into strided buffers with bias, identical to separate
    calls (same split plan per member here) and within tolerance of the oracle."""
    shapes = [(384, K), (256, K), (128, K)]
    ps, ws, x = _group_case(shapes, M, 1300 + M + K, aq.AQ_PHASE_DECODE, bN=bN, frac8=0.3)
    xd = dev_bf16(x)
    grp = aq.Group(ws, aq.AQ_PHASE_DECODE, M)
    outs_full = [torch.full((M, N + 16), 3.0, device="cuda", dtype=torch.bfloat16) for N, _ in shapes]
    outs = [o[:, :N] for o, (N, _) in zip(outs_full, shapes)]
    biases = [torch.linspace(-1, 1, N, device="cuda") for N, _ in shapes]
    grp(xd, outs, bias=biases)
    xq, sx = aq.aq_quant_act(xd)
    for g, (p, w) in enumerate(zip(ps, ws)):
        sep = aq.aq_linear_decode(w, xq, sx, bias=biases[g], out_dtype=torch.bfloat16)
        assert torch.equal(outs[g], sep), g
        assert_output_close(outs[g], oracle_linear(p, x, bias=biases[g].cpu().numpy()))
        assert (outs_full[g][:, shapes[g][0]:] == 3.0).all()
    aq.check_all_workspaces()
    rc, _ = aq.aq_workspace_status(grp.ws)
    assert rc == 0


@pytest.mark.parametrize("M", [1, 300])
def test_group_prefill_matches_oracle(M):
    shapes = [(512, 768), (384, 768)]
    ps, ws, x = _group_case(shapes, M, 1100 + M, aq.AQ_PHASE_PREFILL, bN=64, frac8=0.4)
    grp = aq.Group(ws, aq.AQ_PHASE_PREFILL, M)
    outs = [torch.empty((M, N), device="cuda", dtype=torch.bfloat16) for N, _ in shapes]
    grp(dev_bf16(x), outs)
    for p, o in zip(ps, outs):
        assert_output_close(o, oracle_linear(p, x))
    rc, _ = aq.aq_workspace_status(grp.ws)
    assert rc == 0


def test_group_rejects_mismatched_inputs():
    ps, ws, x = _group_case([(256, 512), (256, 512)], 4, 1200, aq.AQ_PHASE_DECODE)
    p2 = synth.projection_inputs(256, 384, 128, 128, 0.5, (1201,))
    w2 = aq.aq_pack(*dev_projection(p2), 128, 128)
    with pytest.raises(ValueError):
        aq.Group([ws[0], w2], aq.AQ_PHASE_DECODE, 4)
    with pytest.raises(ValueError):
        aq.Group(ws, aq.AQ_PHASE_DECODE, 65)


def test_quant_act_every_bf16_absmax():
    """Every positive finite bf16 value as a row's absmax: the scale (and the codes)
    must match the oracle's fp64 division bit for bit."""
    amax_bits = np.arange(1, 0x7F80, dtype=np.uint32).astype(np.uint16)
    x = np.zeros((amax_bits.size, 16), np.uint16)
    x[:, 0] = amax_bits
    x[:, 1] = amax_bits | 0x8000                                   # -amax
    x[:, 2:] = synth.activations(amax_bits.size, 14, (77,))         # small values
    xv = oracle.bf16_bits_to_f64(x).astype(np.float32)
    xv[:, 2:] = np.minimum(np.abs(xv[:, 2:]), oracle.bf16_bits_to_f64(amax_bits)[:, None].astype(np.float32)) * np.sign(xv[:, 2:])
    x = synth.f32_to_bf16_bits(xv)
    xq, sx = aq.aq_quant_act(dev_bf16(x))
    xq_ref, sx_ref = oracle.quant_act(x)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), sx_ref.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), xq_ref)


# ------------------------------------------------------------------ float-weight quantizer

def _crafted_weights(N, K, seed):
    """Random weights with rows that reach the method's special cases."""
    w = synth.float_weights(N, K, (seed,), outlier_frac=0.002)
    rng = np.random.default_rng(seed)
    w[0, 0:128] = 0.0                                                    # zero row: scale floor, fp16 0
    w[1, 0:128] = -np.abs(w[1, 0:128])                                   # negative-only row
    # quarter steps of s0 = 0.125 (INT4 tile): A / s_i hits exact half-integers at i = 32 and 96
    w[2, 0:128] = (rng.integers(-32, 29, 128) / 4.0 * 0.125).astype(np.float32)
    w[2, 0], w[2, 1] = 7 * 0.125, -8 * 0.125
    w[3, 0:128] = (rng.standard_normal(128) * 1e-6).astype(np.float32)  # fp16 subnormal scales
    w[4, 0:128] = 0.01
    w[4, 5] = 7.0 * (1 + 2.0 ** -11)                                     # s0 = 1 + 2^-11: fp16 tie -> 1.0
    w[5, 0:128] = 0.02
    w[5, 9] = 7.0 * (1 + 3 * 2.0 ** -11)                                 # fp16 tie -> 1 + 2^-9
    w[6, 0:128] = 0.1
    w[6, 0] = 0.9                                                        # the search shrinks the scale
    w[7, 128:256] = 3.0e6                                                # scale beyond fp16: infinity
    return w


def _oracle_quantize(w, pmap, bN, search):
    with np.errstate(over="ignore"):
        return oracle.quantize_weights(w, pmap, bN, 128, search)


@pytest.mark.parametrize("search", [False, True])
@pytest.mark.parametrize("bN,wdtype", [(64, torch.float32), (128, torch.bfloat16)])
def test_quantize_weights_bit_exact(search, bN, wdtype):
    N, K = 128, 384
    w = _crafted_weights(N, K, 21)
    pmap = synth.precision_map(N // bN, K // 128, 0.5, (22,))
    pmap[0, 0] = 1
    pmap[0, 1] = 1
    if wdtype == torch.bfloat16:
        bits = synth.f32_to_bf16_bits(w)
        w = oracle.bf16_bits_to_f64(bits).astype(np.float32)
        wd = dev_bf16(bits)
    else:
        wd = torch.from_numpy(w).cuda()
    codes, scales = aq.aq_quantize_weights(wd, torch.from_numpy(pmap).cuda(), bN, 128, search)
    rc, rs = _oracle_quantize(w, pmap, bN, search)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), rs.view(np.uint16))


def test_quantize_weights_strided_input_and_all_int8():
    N, K, ldw = 64, 256, 384
    big = synth.float_weights(N, ldw, (31,), outlier_frac=0.01)
    pmap = np.zeros((1, 2), np.uint8)
    wd = torch.from_numpy(big).cuda()[:, :K]
    codes, scales = aq.aq_quantize_weights(wd, torch.from_numpy(pmap).cuda(), 64, 128, True)
    rc, rs = _oracle_quantize(np.ascontiguousarray(big[:, :K]), pmap, 64, True)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), rs.view(np.uint16))


@pytest.mark.parametrize("search", [False, True])
def test_quantize_weights_full_size_sampled(search):
    # a 4096 x 4096 projection with 128-row tiles; the oracle checks 40 sampled
    # (row, tile) pairs one by one, every code is checked against its range
    N = K = 4096
    w = synth.float_weights(N, K, (41,), outlier_frac=0.001)
    pmap = synth.precision_map(N // 128, K // 128, 0.25, (42,))
    codes, scales = aq.aq_quantize_weights(torch.from_numpy(w).cuda(), torch.from_numpy(pmap).cuda(), 128, 128,
                                           search)
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    is4 = np.repeat(np.repeat(pmap.astype(bool), 128, 0), 128, 1)
    assert codes[is4].min() >= -8 and codes[is4].max() <= 7
    rng = np.random.default_rng(43)
    for n, j in zip(rng.integers(0, N, 40), rng.integers(0, K // 128, 40)):
        seg = w[n:n + 1, j * 128:(j + 1) * 128]
        rc, rs = _oracle_quantize(seg, pmap[n // 128:n // 128 + 1, j:j + 1], 1, search)
        assert np.array_equal(codes[n, j * 128:(j + 1) * 128], rc[0])
        assert scales[n, j].view(np.uint16) == rs[0, 0].view(np.uint16)


def test_quantize_weights_reports_non_finite():
    w = synth.float_weights(64, 128, (51,))
    w[10, 17] = np.nan
    pmap = torch.ones((1, 1), dtype=torch.uint8, device="cuda")
    with pytest.raises(aq.AqError) as e:
        aq.aq_quantize_weights(torch.from_numpy(w).cuda(), pmap, 64, 128, True)
    assert e.value.status == -3
    w[10, 17] = np.inf
    with pytest.raises(aq.AqError) as e:
        aq.aq_quantize_weights(torch.from_numpy(w).cuda(), pmap, 64, 128, False)
    assert e.value.status == -3
    with pytest.raises(aq.AqError) as e:  # a label other than 0 / 1
        aq.aq_quantize_weights(torch.zeros((64, 128), device="cuda"), pmap * 2, 64, 128, False)
    assert e.value.status == -1


_QP = dict(N=256, K=512, bN=128)


@functools.lru_cache(maxsize=1)
def _quantize_and_pack_case():
    N, K, bN = _QP["N"], _QP["K"], _QP["bN"]
    w = synth.float_weights(N, K, (61,), outlier_frac=0.005)
    pmap = synth.precision_map(N // bN, K // 128, 0.5, (62,))
    return w, pmap, _oracle_quantize(w, pmap, bN, True)


@pytest.mark.parametrize("M", [1, 8, 300])
def test_quantize_and_pack_feeds_the_linear_layer(M):
    N, K, bN = _QP["N"], _QP["K"], _QP["bN"]
    w, pmap, (rc, rs) = _quantize_and_pack_case()
    pw = aq.aq_quantize_and_pack(torch.from_numpy(w).cuda(), torch.from_numpy(pmap).cuda(), bN, 128, True)
    ref = oracle.pack(rc, rs, pmap, bN, 128)
    got = pw.host_buffers()
    for name in aq.BUF_NAMES:
        assert np.array_equal(got[name], np.ascontiguousarray(ref[name]).view(np.uint8).reshape(-1)), name
    x = synth.activations(M, K, (63, M))
    xq, sx = aq.aq_quant_act(dev_bf16(x))
    y = (aq.aq_linear_decode if M <= 64 else aq.aq_linear_prefill)(pw, xq, sx)
    ref_p = synth.SingleProjection(N, K, bN, 128, pmap, rc, rs)
    assert_output_close(y, oracle_linear(ref_p, x))


# ------------------------------------------------------------------ long-prefill variant

@pytest.mark.parametrize("N,K,bN,frac8", [(256, 384, 128, 0.5), (192, 512, 64, 0.3), (128, 256, 128, 0.0),
                                          (384, 256, 64, 1.0)])
def test_expand_int8_matches_oracle_codes(N, K, bN, frac8):
    p = synth.projection_inputs(N, K, bN, 128, frac8, (71, N))
    w = aq.aq_pack(*dev_projection(p), bN, 128)
    e = aq.ExpandedWeights(w)
    torch.cuda.synchronize()
    R, C = N // bN, K // 128
    assert (e.T4, e.T8) == (0, R * C)
    got = e.host_buffers()
    codes, _, _ = oracle.unpack(oracle.pack(p.codes, p.scales, p.pmap, bN, 128))
    want = codes.reshape(R, bN, C, 128).transpose(0, 2, 1, 3).reshape(R * C, bN, 128).astype(np.int8)
    assert np.array_equal(got["w8"], want)
    assert not got["bitmap"].any() and not got["row_off4"].any()
    assert np.array_equal(got["row_off8"], np.arange(R + 1) * C)
    assert np.array_equal(got["tile_idx"], np.arange(R * C))


@pytest.mark.parametrize("M,bN,frac8,out_dtype", [(300, 128, 0.4, torch.float32), (1, 64, 0.3, torch.float32),
                                                  (700, 64, 0.25, torch.bfloat16), (129, 128, 0.0, torch.float32)])
def test_prefill_expanded_equals_prefill_bit_for_bit(M, bN, frac8, out_dtype):
    p, x, w, xq, sx = packed_case(512, 768, bN, frac8, 73, M, outlier=0.01)
    bias = torch.from_numpy(np.random.default_rng(74).standard_normal(512).astype(np.float32)).cuda()
    y1 = aq.aq_linear_prefill(w, xq, sx, bias=bias, out_dtype=out_dtype)
    y2 = aq.aq_linear_prefill_expanded(w, xq, sx, bias=bias, out_dtype=out_dtype)
    assert torch.equal(y1, y2)
    assert_output_close(y2, oracle_linear(p, x, bias=bias.cpu().numpy()))


# ------------------------------------------------------------------ paper-form activation quantization

@pytest.mark.parametrize("M,K,pad,outlier", [(1, 64, 0, 0.0), (1, 3072, 8, 0.01), (2, 128, 0, 0.0),
                                             (17, 2560, 0, 0.01), (300, 640, 16, 0.0), (2048, 2560, 0, 0.01)])
def test_quant_act_groups_bit_exact(M, K, pad, outlier):
    pn = oracle.aq_paper_numerics
    x = synth.activations(M, K + pad, (M, K, pad, 7), outlier_frac=outlier)
    if M > 2:
        x[1, :64] = 0                                  # a zero row inside a group
    if M >= 17:
        x[16:, 64:128] = synth.f32_to_bf16_bits(-np.abs(oracle.bf16_bits_to_f64(x[16:, 64:128])).astype(np.float32))
    xd = dev_bf16(x)
    xq, sx = aq.aq_quant_act_groups(xd, K)
    ref_q, ref_s, Mp = pn.quantize_activation_groups(oracle.bf16_bits_to_f64(x[:, :K]))
    assert xq.shape == (Mp, K)
    assert np.array_equal(xq.cpu().numpy(), ref_q)
    assert np.array_equal(sx.cpu().numpy(), ref_s)


def test_quant_act_groups_ties_and_endpoints():
    # group scale 1 (max 127, min > -128): codes are rint of the values themselves;
    # group scale 2 through the negative endpoint: -256 -> -128
    pn = oracle.aq_paper_numerics
    x = np.zeros((1, 128), np.float32)
    x[0, :8] = [127.0, 2.5, -2.5, 3.5, 0.5, 1.5, -0.5, -127.0]
    x[0, 64:70] = [-256.0, 5.0, 3.0, 1.0, -7.0, 100.0]
    bits = synth.f32_to_bf16_bits(x)
    xq, sx = aq.aq_quant_act_groups(dev_bf16(bits))
    q = xq.cpu().numpy()
    assert list(q[0, :8]) == [127, 2, -2, 4, 0, 2, 0, -127]
    assert list(q[0, 64:70]) == [-128, 2, 2, 0, -4, 50]
    assert list(sx.cpu().numpy()[0]) == [1.0, 2.0]
    ref_q, ref_s, _ = pn.quantize_activation_groups(oracle.bf16_bits_to_f64(bits))
    assert np.array_equal(q, ref_q) and np.array_equal(sx.cpu().numpy(), ref_s)
