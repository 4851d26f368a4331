"""Failure detection on the GPU without a fault.

Every mbarrier wait in the tensor-core kernels is bounded: on expiry it sets
MXMOE_ETIMEOUT in the device error word, lets its kernel return and leaves the context
usable. mxmoe_selftest_wait_timeout runs that same bounded wait on an mbarrier that
nothing completes; the test checks the status the host reads and that the device keeps
computing afterwards. Nothing traps, faults or hangs.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_reports_timeout_and_context_survives():
    from mxfp4_block_scaled_moe_b200 import binding as B
    B.mxmoe_check()                      # start from a clear error word
    B.mxmoe_selftest_wait_timeout()
    with pytest.raises(B.MxmoeError) as err:
        B.mxmoe_check()
    assert err.value.rc == B.ETIMEOUT
    B.mxmoe_check()                      # the word was cleared by the read
    # the context still computes: quantize a small tensor and decode it back exactly
    w = torch.zeros(4, 64, device="cuda")
    w[0, 0], w[1, 5], w[3, 40] = 1.5, -6.0, 0.25
    blocks = torch.empty(4, 32, dtype=torch.uint8, device="cuda")
    scales = torch.empty(4, 2, dtype=torch.uint8, device="cuda")
    B.mxfp4_quantize(w, blocks, scales)
    back = B.mxfp4_dequantize(blocks, scales, torch.float32)
    B.mxmoe_check()
    assert torch.equal(back, w)
