"""aq_linear_decode_noalloc: the decode layer for callers that cannot allocate
device memory (allocator callbacks, fixed-footprint runtimes, plug-ins handed
only their buffers).  It must give the same results as aq_linear_decode with a
caller workspace, on consecutive calls that share the library's fixed scratch,
whether this file runs alone in a fresh process or after every other test."""
import pytest
import torch

from aq_testutil import assert_output_close, dev_bf16, dev_projection, oracle_linear
from w8_a8_quantized_b200 import aq, synth

pytestmark = pytest.mark.gpu


def _case(N, K, M, seed):
    p = synth.projection_inputs(N, K, 128, 128, 0.25, (seed,))
    x = synth.activations(M, K, (seed, 1))
    w = aq.aq_pack(*dev_projection(p), 128, 128)
    xq, sx = aq.aq_quant_act(dev_bf16(x))
    return p, x, w, xq, sx


def _device_free_bytes():
    free, _ = torch.cuda.mem_get_info()
    return free


@pytest.mark.parametrize("N,K,M", [(1024, 3072, 24), (512, 2048, 48), (1024, 1024, 4), (768, 3072, 1)])
def test_noalloc_matches_workspace_entry_on_two_calls(N, K, M):
    """Same kernels as aq_linear_decode, so the same bits; both within tolerance of
    the oracle; and a call neither allocates device memory through torch nor
    changes the device's free memory (the first call on the device resolves the
    scratch array's address, so it is made before the measurement)."""
    p, x, w, xq, sx = _case(N, K, M, 4000 + M)
    assert aq.aq_workspace_bytes(aq.AQ_PHASE_DECODE, M, w) <= 4 << 20
    ref = aq.aq_linear_decode(w, xq, sx, ws=torch.zeros(aq.aq_workspace_bytes(aq.AQ_PHASE_DECODE, M, w),
                                                         dtype=torch.uint8, device="cuda"))
    out1 = torch.full_like(ref, float("nan"))
    out2 = torch.full_like(ref, float("nan"))
    aq.aq_linear_decode_noalloc(w, xq, sx, out=out1)  # set-up call (also the first of two compared)
    torch.cuda.synchronize()
    torch_before, free_before = torch.cuda.memory_allocated(), _device_free_bytes()
    aq.aq_linear_decode_noalloc(w, xq, sx, out=out2)  # second call reuses the shared scratch
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == torch_before
    assert _device_free_bytes() == free_before
    assert torch.equal(out1, ref)
    assert torch.equal(out2, ref)
    assert_output_close(out2, oracle_linear(p, x))


def test_noalloc_back_to_back_different_shapes():
    pa, xa, wa, xqa, sxa = _case(1024, 3072, 32, 4100)
    pb, xb, wb, xqb, sxb = _case(2048, 2048, 16, 4101)
    ref_a = aq.aq_linear_decode(wa, xqa, sxa)
    ref_b = aq.aq_linear_decode(wb, xqb, sxb)
    out_a = aq.aq_linear_decode_noalloc(wa, xqa, sxa)
    out_b = aq.aq_linear_decode_noalloc(wb, xqb, sxb)
    torch.cuda.synchronize()
    assert torch.equal(out_a, ref_a)
    assert torch.equal(out_b, ref_b)
    assert_output_close(out_a, oracle_linear(pa, xa))


def test_noalloc_rejects_scratch_beyond_limit():
    # a long-K projection at 64 tokens keeps split-K partial sums beyond the 4 MiB scratch
    _, _, w, xq, sx = _case(6144, 16384, 64, 4200)
    assert aq.aq_workspace_bytes(aq.AQ_PHASE_DECODE, 64, w) > 4 << 20
    with pytest.raises(aq.AqError) as e:
        aq.aq_linear_decode_noalloc(w, xq, sx)
    assert e.value.status == -5
