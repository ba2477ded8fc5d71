"""Helpers shared by the GPU tests: move seeded synthetic inputs to the
device, and compare CUDA results with the CPU oracle under the stated
tolerance."""
import numpy as np
import torch

import oracle
from w8_a8_quantized_b200 import aq, synth


def dev_projection(p: synth.SingleProjection, device="cuda"):
    codes = torch.from_numpy(np.ascontiguousarray(p.codes)).to(device)
    scales = torch.from_numpy(np.ascontiguousarray(p.scales)).to(device)
    pmap = torch.from_numpy(np.ascontiguousarray(p.pmap)).to(device)
    return codes, scales, pmap


def dev_bf16(bits: np.ndarray, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def packed_case(N, K, bN, frac8, seed, M, outlier=0.0):
    """Seeded projection + activations, packed on the GPU and quantized on the GPU."""
    p = synth.projection_inputs(N, K, bN, 128, frac8, (seed,))
    x = synth.activations(M, K, (seed, 1), outlier_frac=outlier)
    w = aq.aq_pack(*dev_projection(p), bN, 128)
    xq, sx = aq.aq_quant_act(dev_bf16(x))
    return p, x, w, xq, sx


def bf16_round(y64: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 (via fp32, round to nearest even) -> fp64."""
    bits = synth.f32_to_bf16_bits(y64.astype(np.float32)).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def assert_output_close(y_dev: torch.Tensor, y_ref: np.ndarray):
    """Tolerance of the linear outputs against the oracle's fp64 result.

    fp32 outputs: relative error <= 1e-3 where |y| >= 1, absolute <= 1e-2 where
    |y| < 1.  bf16 outputs: rounding to bf16 alone costs up to 2^-9 relative,
    so they must lie within one bf16 ulp of the bf16-rounded oracle value
    where |y| >= 1 (and within 1e-2 absolute where |y| < 1)."""
    y = y_dev.float().cpu().numpy().astype(np.float64)
    assert y.shape == y_ref.shape
    assert np.isfinite(y).all()
    small = np.abs(y_ref) < 1.0
    if y_dev.dtype == torch.float32:
        rel = np.abs(y - y_ref) / np.maximum(np.abs(y_ref), 1e-300)
        bad = (~small & (rel > 1e-3)) | (small & (np.abs(y - y_ref) > 1e-2))
    else:
        r = bf16_round(y_ref)
        _, e = np.frexp(np.abs(r))
        ulp = np.ldexp(1.0, e - 8)  # bf16 keeps 8 significant bits: spacing above |r| is 2^(floor(log2|r|) - 7)
        bad = (~small & (np.abs(y - r) > ulp)) | (small & (np.abs(y - y_ref) > 1e-2))
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{bad.sum()} outputs out of tolerance; first at {tuple(i)}: "
                             f"gpu {y[tuple(i)]!r} oracle {y_ref[tuple(i)]!r}")


def oracle_linear(p: synth.SingleProjection, x_bits: np.ndarray, bias=None, rows=None, cols=None):
    xq, sx = oracle.quant_act(x_bits if rows is None else x_bits[rows])
    return oracle.linear_codes(p.codes, p.scales, xq, sx, p.bK, bias=bias, cols=cols)
