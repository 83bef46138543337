"""Failure detection on the GPU without a GPU fault.

Every pipeline wait of the decode kernel is bounded: when it runs out, the
block raises ARCHEAD_STATUS_WAIT_TIMEOUT in the workspace status word, skips
its remaining work and exits, so the call returns and the context stays
usable.  The test hook archead_test_decode_waits makes one wait run out on
purpose (a barrier that nothing completes, with a 1 ms limit); the host reads
the status back, and the next call on the cleared workspace is correct.
"""
import ctypes

import numpy as np
import pytest
import torch

import archead_inputs as gen
import oracle
from parity import check_argmax, check_lse_ce

pytestmark = pytest.mark.gpu


def _status(qoh, ws, clear):
    v = ctypes.c_uint32(0)
    rc = qoh._lib.archead_workspace_status(ws.data_ptr(), 1 if clear else 0,
                                           torch.cuda.current_stream().cuda_stream, ctypes.byref(v))
    return rc, int(v.value)


@pytest.mark.parametrize("T", [3, 11])   # one decode launch, two (g_B = 32 keeps every T on the decode kernel)
def test_decode_wait_expiry_reports_timeout_and_recovers(T):
    import quantized_output_head_b200 as qoh
    lib = qoh._lib
    shape = (2000, 256, 32, 8, 64, 32)
    comps = gen.random_components(gen.HeadShape(*shape), seed=909)
    h_bits, targets = gen.random_hidden(256, T, seed=910, V=shape[0])
    head = qoh.PackedHead(*shape, comps)
    assert head.forward_kernel(T) == "decode"
    hd = torch.from_numpy(h_bits.view(np.int16)).cuda()
    td = torch.from_numpy(targets).cuda()
    ws = head.workspace(T)
    assert _status(qoh, ws, clear=True)[0] == qoh.ARCHEAD_OK
    assert lib.archead_test_decode_waits(head.handle, 1_000_000, 1) == qoh.ARCHEAD_OK
    try:
        head.lse_argmax(hd, td)                       # the call returns; its outputs are invalid
        torch.cuda.synchronize()
        rc, v = _status(qoh, ws, clear=True)
        assert rc == qoh.ARCHEAD_ETIMEOUT and v & qoh.STATUS_WAIT_TIMEOUT
    finally:
        assert lib.archead_test_decode_waits(head.handle, 2_000_000_000, 0) == qoh.ARCHEAD_OK
    assert lib.archead_test_decode_waits(head.handle, 0, 0) == qoh.ARCHEAD_EINVAL
    # the context and the workspace are usable again
    lse, am, ce = head.lse_argmax(hd, td)
    y, rowmax = oracle.logits(comps, 64, 32, h_bits)
    tol = oracle.tolerance(h_bits, rowmax)
    check_lse_ce(lse.cpu().numpy(), ce.cpu().numpy(), y, tol, targets)
    check_argmax(am.cpu().numpy(), y, tol)
    assert _status(qoh, ws, clear=True) == (qoh.ARCHEAD_OK, 0)
