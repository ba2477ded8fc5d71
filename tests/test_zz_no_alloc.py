"""aq_linear_decode_noalloc: the decode layer for callers that cannot allocate
device memory (allocator callbacks, fixed-footprint runtimes, plug-ins handed
only their buffers).  It must give the same results as aq_linear_decode with a
caller workspace, on consecutive calls that share the library's fixed scratch,
whether this file runs alone in a fresh process or after every other test."""
import numpy as np
import pytest
import torch

from aq_testutil import dev_bf16, dev_projection
from w8_a8_quantized_b200 import aq, synth

pytestmark = pytest.mark.gpu


def _case(N, K, M, seed):
    p = synth.projection_inputs(N, K, 128, 128, 0.25, (seed,))
    w = aq.aq_pack(*dev_projection(p), 128, 128)
    xq, sx = aq.aq_quant_act(dev_bf16(synth.activations(M, K, (seed, 1))))
    return w, xq, sx


def _assert_same_within_tolerance(y_new, y_ref):
    a = y_new.float().cpu().numpy().astype(np.float64)
    b = y_ref.float().cpu().numpy().astype(np.float64)
    small = np.abs(b) < 1.0
    assert np.all(np.abs(a - b)[small] <= 1e-2)
    assert np.all((np.abs(a - b) / np.maximum(np.abs(b), 1e-300))[~small] <= 1e-3)


@pytest.mark.parametrize("N,K,M", [(1024, 3072, 24), (512, 2048, 48), (1024, 1024, 4)])
def test_noalloc_matches_workspace_entry_on_two_calls(N, K, M):
    w, xq, sx = _case(N, K, M, 4000 + M)
    assert aq.aq_workspace_bytes(aq.AQ_PHASE_DECODE, M, w) <= 4 << 20
    ref = aq.aq_linear_decode(w, xq, sx, ws=torch.zeros(aq.aq_workspace_bytes(aq.AQ_PHASE_DECODE, M, w),
                                                         dtype=torch.uint8, device="cuda"))
    out1 = torch.full_like(ref, float("nan"))
    out2 = torch.full_like(ref, float("nan"))
    aq.aq_linear_decode_noalloc(w, xq, sx, out=out1)
    aq.aq_linear_decode_noalloc(w, xq, sx, out=out2)  # second call reuses the shared scratch
    torch.cuda.synchronize()
    _assert_same_within_tolerance(out1, ref)
    _assert_same_within_tolerance(out2, ref)


def test_noalloc_back_to_back_different_shapes():
    wa, xqa, sxa = _case(1024, 3072, 32, 4100)
    wb, xqb, sxb = _case(2048, 2048, 16, 4101)
    ref_a = aq.aq_linear_decode(wa, xqa, sxa)
    ref_b = aq.aq_linear_decode(wb, xqb, sxb)
    out_a = aq.aq_linear_decode_noalloc(wa, xqa, sxa)
    out_b = aq.aq_linear_decode_noalloc(wb, xqb, sxb)
    torch.cuda.synchronize()
    _assert_same_within_tolerance(out_a, ref_a)
    _assert_same_within_tolerance(out_b, ref_b)


def test_noalloc_rejects_scratch_beyond_limit():
    w, xq, sx = _case(3072, 3072, 64, 4200)
    assert aq.aq_workspace_bytes(aq.AQ_PHASE_DECODE, 64, w) > 4 << 20
    with pytest.raises(aq.AqError) as e:
        aq.aq_linear_decode_noalloc(w, xq, sx)
    assert e.value.status == -5
