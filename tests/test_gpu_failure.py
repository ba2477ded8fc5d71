"""Failure detection of the tensor-core linear kernel, without any GPU fault.

Every wait inside the kernel on an mbarrier is bounded; when one gives up the
kernel records AQ_ERR_TIMEOUT with the code of that wait in the workspace,
every role leaves its loop, copies in flight are given time to land, tensor
memory is freed and the kernel returns.  aq_debug_linear_stalled makes this
happen on purpose: the weight producer stops after one input tile, so the next
stage never fills (a barrier nothing completes), and every wait is limited to
20 ms.  The host then reads the error through aq_workspace_status, which also
restores the workspace, and the same workspace serves ordinary calls again."""
import time

import pytest
import torch

from aq_testutil import assert_output_close, oracle_linear, packed_case
from w8_a8_quantized_b200 import aq

pytestmark = pytest.mark.gpu

# codes of the waits that can give up first when the weight stream stops:
# 3 activation producer (stage reuse), 4 MMA issuer (stage full), 7 metadata
# warp (record slot), 8 transform warps (staged weights), 9 epilogue (MMA done)
STALL_CODES = {3, 4, 7, 8, 9}
WAIT_NS = 20_000_000


def test_prefill_stall_times_out_and_workspace_serves_next_call():
    p, x, w, xq, sx = packed_case(256, 128 * 6, 128, 0.5, 1600, 130)
    ws = torch.zeros(aq.aq_workspace_bytes(aq.AQ_PHASE_PREFILL, 130, w), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.monotonic()
    aq.aq_debug_linear_stalled(w, xq, sx, aq.AQ_PHASE_PREFILL, ws, wait_ns=WAIT_NS, stop_after=1)
    rc, info = aq.aq_workspace_status(ws)  # synchronizes
    elapsed = time.monotonic() - t0
    assert rc == -7, rc
    assert info in STALL_CODES, info
    assert elapsed < 5.0, elapsed  # bounded: about a few wait limits, not the normal 2 s ones stacked up
    assert int(ws.count_nonzero()) == 0  # error word cleared
    y = aq.aq_linear_prefill(w, xq, sx, ws=ws)
    assert_output_close(y, oracle_linear(p, x))
    assert aq.aq_workspace_status(ws) == (0, 0)


def test_decode_split_stall_clears_counters_and_recovers():
    """Decode from 5 tokens splits the input tiles over CTAs and counts finished
    splits in the workspace; a call that gave up may leave those counters
    nonzero.  Here they are poisoned before the stalled call: the status call must
    zero them with the error word, or the next ordinary call would reduce too early."""
    M = 16
    p, x, w, xq, sx = packed_case(256, 128 * 16, 128, 0.5, 1610, M)
    need = aq.aq_workspace_bytes(aq.AQ_PHASE_DECODE, M, w)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    counters = ws[256:512]  # the counter area follows the 256-byte header (256 bytes for 2 row blocks)
    counters.fill_(7)
    aq.aq_debug_linear_stalled(w, xq, sx, aq.AQ_PHASE_DECODE, ws, wait_ns=WAIT_NS, stop_after=1)
    rc, info = aq.aq_workspace_status(ws)
    assert rc == -7 and info in STALL_CODES, (rc, info)
    assert int(ws[:512].count_nonzero()) == 0
    for _ in range(2):
        y = aq.aq_linear_decode(w, xq, sx, ws=ws)
        assert_output_close(y, oracle_linear(p, x))
    assert aq.aq_workspace_status(ws) == (0, 0)


def test_stall_entry_rejects_bad_arguments():
    p, x, w, xq, sx = packed_case(256, 128 * 4, 128, 0.5, 1620, 8)
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    for kw in (dict(wait_ns=10), dict(wait_ns=20_000_000_000), dict(stop_after=-1)):
        with pytest.raises(aq.AqError):
            aq.aq_debug_linear_stalled(w, xq, sx, aq.AQ_PHASE_PREFILL, ws, **kw)
    with pytest.raises(aq.AqError):  # 2 tokens decode on the CUDA cores: no tensor-core kernel to stall
        aq.aq_debug_linear_stalled(w, xq[:2].contiguous(), sx[:2].contiguous(), aq.AQ_PHASE_DECODE, ws)
