"""Seeded synthetic inputs for the mixed W4/W8 x A8 linear layer.

This module only draws random numbers and shapes them; it holds none of the
method's arithmetic (no quantization, no packing, no products).  Both the CUDA
path and the CPU oracle are fed from it.

What it produces, per projection (N output features x K input features):
  * a precision map ``pmap[R][C]`` (uint8, 1 = INT4 tile, 0 = INT8 tile) with
    exactly ``round_half_even(f_int8 * R * C)`` INT8 tiles chosen by a seeded
    permutation;
  * integer weight codes ``codes[N][K]`` (int8): uniform over [-128, 127] in
    INT8 tiles and over [-8, 7] in INT4 tiles;
  * per-row-per-tile weight scales ``scales[N][C]`` drawn uniform in
    [1e-3, 1e-2] and rounded to fp16;
  * float weights ``W[N][K]`` (fp32) drawn N(0, 0.02^2), optionally with a
    seeded fraction of entries multiplied by 10 (outlier weights), for the
    weight quantizer;
  * activations ``X[M][K]`` drawn N(0, 1) in fp32, optionally with a seeded
    set of outlier input channels multiplied by 20, rounded to bf16 and
    returned as raw bf16 bit patterns (uint16).

The model shapes mirror the models the AlignQuant paper evaluates
(Llama-3.2-3B, Qwen3-4B, an 8B-class dense model, Qwen3-14B); no checkpoint is
read: all weights are random.
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = [
    "MODELS", "projections", "precision_map", "weight_codes", "weight_scales",
    "activations", "f32_to_bf16_bits", "projection_inputs", "SingleProjection",
    "float_weights", "device_projection_inputs", "device_activations",
]

# (hidden, q-proj out, k/v-proj out, MLP intermediate, layers)
MODELS = {
    "llama-3.2-3b": dict(hidden=3072, q_out=3072, kv_out=1024, inter=8192, layers=28),
    "qwen3-4b": dict(hidden=2560, q_out=4096, kv_out=1024, inter=9728, layers=36),
    "dense-8b": dict(hidden=4096, q_out=4096, kv_out=1024, inter=14336, layers=32),
    "qwen3-14b": dict(hidden=5120, q_out=5120, kv_out=1024, inter=17408, layers=40),
    "single-2048": dict(hidden=2048, q_out=2048, kv_out=2048, inter=2048, layers=1),
}

PROJ_IDS = {"q": 0, "k": 1, "v": 2, "o": 3, "gate": 4, "up": 5, "down": 6}


def projections(model: str):
    """The seven linear projections of one decoder layer as (name, N, K)."""
    if model == "single-2048":
        return [("q", 2048, 2048)]
    m = MODELS[model]
    h, q, kv, i = m["hidden"], m["q_out"], m["kv_out"], m["inter"]
    return [("q", q, h), ("k", kv, h), ("v", kv, h), ("o", h, q),
            ("gate", i, h), ("up", i, h), ("down", h, i)]


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def precision_map(R: int, C: int, frac_int8: float, seed) -> np.ndarray:
    """uint8[R][C], 1 marks an INT4 tile; exactly round_half_even(f*R*C) INT8 tiles."""
    T = R * C
    t8 = int(round(frac_int8 * T))  # Python round() is round-half-even
    perm = _rng(*_key(seed), 1).permutation(T)
    pmap = np.ones(T, dtype=np.uint8)
    pmap[perm[:t8]] = 0
    return pmap.reshape(R, C)


def weight_codes(N: int, K: int, pmap: np.ndarray, bN: int, bK: int, seed) -> np.ndarray:
    """int8[N][K]: uniform over the full INT8 range, or over [-8, 7] in INT4 tiles."""
    R, C = pmap.shape
    assert R * bN == N and C * bK == K
    words = np.random.PCG64(np.random.SeedSequence(list(_key(seed)) + [2])).random_raw((N * K + 7) // 8)
    raw = words.view(np.uint8)[: N * K].reshape(R, bN, C, bK)
    # INT4 tiles: (b & 15) - 8, computed modulo 256 as (b & 15) + 248
    np.copyto(raw, (raw & np.uint8(15)) + np.uint8(248), where=pmap.astype(bool)[:, None, :, None])
    return raw.view(np.int8).reshape(N, K)


def weight_scales(N: int, C: int, seed) -> np.ndarray:
    """float16[N][C] uniform in [1e-3, 1e-2] (drawn in fp64, rounded to fp16)."""
    return _rng(*_key(seed), 3).uniform(1e-3, 1e-2, size=(N, C)).astype(np.float16)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> 16) & 1
    return ((b + np.uint32(0x7FFF) + lsb) >> 16).astype(np.uint16)


def activations(M: int, K: int, seed, outlier_frac: float = 0.0, outlier_mult: float = 20.0) -> np.ndarray:
    """uint16[M][K] bf16 bits of N(0,1) activations; round(outlier_frac*K) seeded
    input channels (the same for every token) are multiplied by outlier_mult."""
    g = _rng(*_key(seed), 4)
    x = g.standard_normal((M, K), dtype=np.float32)
    n_out = int(round(outlier_frac * K))
    if n_out:
        cols = g.choice(K, size=n_out, replace=False)
        x[:, cols] *= np.float32(outlier_mult)
    return f32_to_bf16_bits(x)


def float_weights(N: int, K: int, seed, outlier_frac: float = 0.0, outlier_mult: float = 10.0) -> np.ndarray:
    """float32[N][K] drawn N(0, 0.02^2); round(outlier_frac*N*K) seeded entries
    are multiplied by outlier_mult."""
    g = _rng(*_key(seed), 5)
    w = (g.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    n_out = int(round(outlier_frac * N * K))
    if n_out:
        idx = g.choice(N * K, size=n_out, replace=False)
        w.reshape(-1)[idx] *= np.float32(outlier_mult)
    return w


def _key(seed):
    return tuple(seed) if isinstance(seed, (tuple, list)) else (int(seed),)


@dataclasses.dataclass
class SingleProjection:
    """Host-side synthetic inputs of one projection."""
    N: int
    K: int
    bN: int
    bK: int
    pmap: np.ndarray      # uint8[R][C], 1 = INT4
    codes: np.ndarray     # int8[N][K]
    scales: np.ndarray    # float16[N][C]

    @property
    def R(self):
        return self.N // self.bN

    @property
    def C(self):
        return self.K // self.bK


def projection_inputs(N: int, K: int, bN: int, bK: int, frac_int8: float, seed) -> SingleProjection:
    """Map, codes and scales of one projection from one seed tuple."""
    R, C = N // bN, K // bK
    pmap = precision_map(R, C, frac_int8, seed)
    return SingleProjection(N, K, bN, bK, pmap,
                            weight_codes(N, K, pmap, bN, bK, seed),
                            weight_scales(N, C, seed))


def device_projection_inputs(N: int, K: int, bN: int, bK: int, frac_int8: float, seed, device):
    """The recipe of projection_inputs drawn with torch's generator on a CUDA
    device (for models too large to draw on the host in reasonable time): map
    with exactly round_half_even(f*R*C) INT8 tiles chosen by a seeded
    permutation, codes uniform over [-128, 127] in INT8 tiles and [-8, 7] in INT4
    tiles, scales uniform in [1e-3, 1e-2] rounded to fp16.  The same seed gives
    the same values on any device of the same kind; they differ from
    projection_inputs' values (another generator).  Returns (codes int8 [N][K],
    scales float16 [N][C], pmap uint8 [R][C]) on `device`."""
    import torch
    R, C = N // bN, K // bK
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence(list(_key(seed))).generate_state(1, np.uint64)[0] >> 1))
    T = R * C
    t8 = int(round(frac_int8 * T))
    pmap = torch.ones(T, dtype=torch.uint8, device=device)
    pmap[torch.randperm(T, generator=g, device=device)[:t8]] = 0
    pmap = pmap.view(R, C)
    raw = torch.randint(-128, 128, (N, K), dtype=torch.int16, generator=g, device=device)
    int4 = pmap.bool().repeat_interleave(bN, 0).repeat_interleave(bK, 1)
    codes = torch.where(int4, (raw & 15) - 8, raw).to(torch.int8)
    scales = (torch.rand((N, C), dtype=torch.float32, generator=g, device=device) * 9e-3 + 1e-3).to(torch.float16)
    return codes, scales, pmap


def device_activations(M: int, K: int, seed, device, outlier_frac: float = 0.0, outlier_mult: float = 20.0):
    """The recipe of activations drawn with torch's generator on a CUDA device:
    bf16 [M][K] N(0,1) values, round(outlier_frac*K) seeded input channels
    multiplied by outlier_mult.  Other values than activations' (another
    generator)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence(list(_key(seed)) + [4]).generate_state(1, np.uint64)[0] >> 1))
    x = torch.randn((M, K), dtype=torch.float32, generator=g, device=device)
    n_out = int(round(outlier_frac * K))
    if n_out:
        cols = torch.randperm(K, generator=g, device=device)[:n_out]
        x[:, cols] *= outlier_mult
    return x.to(torch.bfloat16)
