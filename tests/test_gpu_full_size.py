"""Parity at the full benchmark sizes, in the launch configuration the
benchmark times (one layer of each model, run through the same grouped calls
as ``bench.py``'s step), checked against the CPU oracle on sampled outputs:
a few whole token rows (every output feature) and a few whole output columns
(every token).  Per-tile products at these sizes would take gigabytes, so
they are checked bit-exactly at the smaller sizes of test_gpu_parity.py."""
import numpy as np
import pytest
import torch

import bench
from aq_testutil import assert_output_close, oracle_linear
from w8_a8_quantized_b200 import synth

pytestmark = pytest.mark.gpu


def _layer_outputs(workload: str, M: int, bN=None, frac8=None):
    """One layer of the workload, stepped once as the benchmark does."""
    wl = dict(bench.WORKLOADS[workload], gen="host")  # the oracle regenerates the host-drawn values
    if bN is not None:
        wl["bN"] = bN
    if frac8 is not None:
        wl["frac8"] = frac8
    m = bench.Model(wl, M, torch.device("cuda"), 0, layers=1)
    m.step("group")
    torch.cuda.synchronize()
    return wl, m


def _check_sampled(wl, m, n_rows: int, n_cols: int, seed: int):
    cfg = bench.CFG_ID[wl["model"]]
    rng = np.random.default_rng(seed)
    for pid, (name, N, K) in enumerate(m.projs):
        p = synth.projection_inputs(N, K, wl["bN"], 128, wl["frac8"], (cfg, 0, pid))
        kind = bench.INPUT_OF[name]
        x_bits = m.x_host_sets[0][kind].view(torch.int16).numpy().view(np.uint16)
        y = m.y[name]
        rows = sorted(set(rng.choice(m.M, size=min(n_rows, m.M), replace=False).tolist()) | {m.M - 1})
        cols = sorted(set(rng.choice(N, size=n_cols, replace=False).tolist()) | {0, N - 1})
        assert_output_close(y[rows], oracle_linear(p, x_bits, rows=rows))
        assert_output_close(y[:, cols], oracle_linear(p, x_bits, cols=cols))


@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_llama3b_decode_layer_full_size(M):
    wl, m = _layer_outputs("decode-llama-3.2-3b", M)
    _check_sampled(wl, m, n_rows=M, n_cols=64, seed=M)


def test_qwen3_4b_prefill_layer_full_size():
    wl, m = _layer_outputs("prefill-qwen3-4b", 2048)
    _check_sampled(wl, m, n_rows=12, n_cols=48, seed=2048)


@pytest.mark.parametrize("bN", [128, 64])
def test_dense8b_prefill_layer_full_size(bN):
    wl, m = _layer_outputs("prefill-dense-8b", 4096, bN=bN)
    _check_sampled(wl, m, n_rows=8, n_cols=24, seed=bN)


def test_qwen3_14b_prefill_chunk_full_size():
    wl, m = _layer_outputs("prefill-qwen3-14b", 8192)
    _check_sampled(wl, m, n_rows=6, n_cols=12, seed=8192)


@pytest.mark.parametrize("M", [1, 16])
def test_single_2048_layer_as_specified(M):
    """The single 2048 x 2048 layer: 128 x 128 tiles, 50% INT8, M = 1 and 16."""
    wl, m = _layer_outputs("decode-single-2048", M)
    assert (wl["bN"], wl["frac8"]) == (128, 0.5)
    _check_sampled(wl, m, n_rows=M, n_cols=256, seed=20 + M)


# 8B-class decode: 64- and 128-row tiles across the INT8 fractions and token
# counts (1: streaming CUDA-core kernel; 5: tensor cores, two 64-row tile rows
# per 128-row accumulator block; 16 and 64: tensor cores with split reduction)
@pytest.mark.parametrize("bN,frac8,M", [(64, 0.0, 1), (64, 0.25, 5), (64, 0.5, 16), (64, 1.0, 64),
                                        (64, 0.5, 1), (64, 0.25, 64), (128, 0.5, 1), (128, 1.0, 16)])
def test_dense8b_decode_layer_full_size(bN, frac8, M):
    wl, m = _layer_outputs("decode-dense-8b", M, bN=bN, frac8=frac8)
    _check_sampled(wl, m, n_rows=M, n_cols=48, seed=30 + M)


@pytest.mark.parametrize("M", [1, 2, 16, 64])
def test_qwen3_14b_decode_layer_full_size(M):
    """K = 17408 in the MLP down projection: at 2 tokens its activations do not
    fit the fused preparation, so it runs as activation quantization plus the
    CUDA-core kernel on the codes."""
    wl, m = _layer_outputs("decode-qwen3-14b", M)
    _check_sampled(wl, m, n_rows=M, n_cols=32, seed=40 + M)
