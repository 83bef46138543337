"""The allocation-free entry point gives the same results as the workspace one.

archead_logits_lse_argmax_static exists for callers that cannot allocate
device memory when they run the head (graph capture under an allocator that
forbids it, host frameworks that own all device memory).  It takes no
workspace; its scratch is a fixed device array inside the library, whose
status word archead_static_workspace_status reads back.  This file is
collected last so that a failure here stops a -x run only after every other
test has run; it must also pass on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import archead_inputs as gen
import oracle
from parity import check_argmax, check_lse_ce

pytestmark = pytest.mark.gpu


def _static_status(lib, stream, clear=True):
    v = ctypes.c_uint32(0)
    rc = lib.archead_static_workspace_status(1 if clear else 0, stream, ctypes.byref(v))
    return rc, int(v.value)


@pytest.mark.parametrize("T", [5, 24])   # the decode kernel, then the tensor-core kernel
def test_static_entry_matches_workspace_entry_twice(T):
    """Two calls in a row on a non-blocking stream (possibly the first static
    call of the process, whose set-up clears the status word on that stream),
    each equal to the workspace entry point and within the oracle's tolerance,
    with the status word clean after each."""
    import quantized_output_head_b200 as qoh
    lib = qoh._lib
    shape = (1000, 256, 32, 8, 64, 64)
    comps = gen.random_components(gen.HeadShape(*shape), seed=2024)
    h_bits, targets = gen.random_hidden(256, T, seed=2025, V=shape[0])
    head = qoh.PackedHead(*shape, comps)
    assert head.forward_kernel(T) == ("decode" if T <= 8 else "tensor_core")
    hd = torch.from_numpy(h_bits.view(np.int16)).cuda()
    td = torch.from_numpy(targets).cuda()
    ref_lse, ref_am, ref_ce = head.lse_argmax(hd, td)
    y, rowmax = oracle.logits(comps, 64, 64, h_bits)
    tol = oracle.tolerance(h_bits, rowmax)
    side = torch.cuda.Stream()                       # torch streams do not sync with the legacy stream
    side.wait_stream(torch.cuda.current_stream())
    stream = side.cuda_stream
    for _ in range(2):
        with torch.cuda.stream(side):
            lse = torch.full((T,), float("nan"), device="cuda")
            am = torch.full((T,), -1, dtype=torch.int32, device="cuda")
            ce = torch.full((T,), float("nan"), device="cuda")
        rc = lib.archead_logits_lse_argmax_static(head.handle, hd.data_ptr(), T, td.data_ptr(), lse.data_ptr(),
                                                   am.data_ptr(), ce.data_ptr(), stream)
        assert rc == qoh.ARCHEAD_OK, lib.archead_status_string(rc)
        side.synchronize()
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=0, atol=float(tol.max()))
        np.testing.assert_allclose(ce.cpu().numpy(), ref_ce.cpu().numpy(), rtol=0, atol=2 * float(tol.max()))
        assert np.array_equal(am.cpu().numpy(), ref_am.cpu().numpy())
        check_lse_ce(lse.cpu().numpy(), ce.cpu().numpy(), y, tol, targets)
        check_argmax(am.cpu().numpy(), y, tol)
        assert _static_status(lib, stream) == (qoh.ARCHEAD_OK, 0)


def test_static_entry_reports_a_bad_target_and_clears_it():
    """A target outside [0, V) gives CE = NaN for that token and raises
    ARCHEAD_STATUS_BAD_TARGET in the fixed array's status word; clearing it
    leaves the word at zero for the next call."""
    import quantized_output_head_b200 as qoh
    lib = qoh._lib
    shape = (1000, 256, 32, 8, 64, 64)
    comps = gen.random_components(gen.HeadShape(*shape), seed=77)
    h_bits, targets = gen.random_hidden(256, 3, seed=78, V=shape[0])
    head = qoh.PackedHead(*shape, comps)
    hd = torch.from_numpy(h_bits.view(np.int16)).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    _static_status(lib, stream)                      # start from a clean word
    bad = targets.copy()
    bad[1] = shape[0]
    out = [torch.empty(3, device="cuda"), torch.empty(3, dtype=torch.int32, device="cuda"),
           torch.empty(3, device="cuda")]
    bad_d, good_d = torch.from_numpy(bad).cuda(), torch.from_numpy(targets).cuda()
    rc = lib.archead_logits_lse_argmax_static(head.handle, hd.data_ptr(), 3, bad_d.data_ptr(),
                                               *[t.data_ptr() for t in out], stream)
    assert rc == qoh.ARCHEAD_OK
    ce = out[2].cpu().numpy()
    assert np.isfinite(ce[0]) and np.isnan(ce[1]) and np.isfinite(ce[2])
    assert _static_status(lib, stream, clear=False) == (qoh.ARCHEAD_OK, qoh.STATUS_BAD_TARGET)
    assert _static_status(lib, stream, clear=True) == (qoh.ARCHEAD_OK, qoh.STATUS_BAD_TARGET)
    rc = lib.archead_logits_lse_argmax_static(head.handle, hd.data_ptr(), 3, good_d.data_ptr(),
                                               *[t.data_ptr() for t in out], stream)
    assert rc == qoh.ARCHEAD_OK
    assert np.all(np.isfinite(out[2].cpu().numpy()))
    assert _static_status(lib, stream) == (qoh.ARCHEAD_OK, 0)


def test_static_entry_rejects_too_many_tokens():
    import quantized_output_head_b200 as qoh
    lib = qoh._lib
    shape = (64, 64, 16, 8, 16, 16)
    head = qoh.PackedHead(*shape, gen.random_components(gen.HeadShape(*shape), seed=7))
    cap = lib.archead_static_workspace_capacity()
    T = 1
    while lib.archead_workspace_bytes(head.handle, T) <= cap:
        T *= 2
    rc = lib.archead_logits_lse_argmax_static(head.handle, 4096, T, None, 4096, 4096, None, None)
    assert rc == qoh.ARCHEAD_ENOMEM
