"""The tensor-pipe rate probe (mxmoe_tc_rate_probe) that gives the benchmark its FP8
roofline denominator: it runs to completion without a device error, reports the FLOPs
of its MMAs, and measures a rate within the physically possible range for a B200 (the
tensor pipe of 148 SMs between ~1 and ~2 GHz)."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _rate(B, n, copy, iters=4000, random_operands=True):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    f = B.mxmoe_tc_rate_probe(n, copy, iters, random_operands=random_operands)
    e1.record()
    torch.cuda.synchronize()
    B.mxmoe_check()
    return f, f / (e0.elapsed_time(e1) / 1e3) / 1e12


def test_rate_probe_runs_and_reports_its_flops():
    from mxfp4_block_scaled_moe_b200 import binding as B
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B.mxmoe_tc_rate_probe(256, False, 10)          # load
    runs = [_rate(B, 256, False) for _ in range(3)]
    f, tf = runs[0][0], max(r[1] for r in runs)
    assert f == 2.0 * 128 * 256 * 32 * 4 * 4000 * sms
    # a block-scaled M=128 N=256 K=32 MMA moves at most 2*128*256*32 / 128 = 16384 FLOP per
    # SM cycle; 148 SMs at 1.0-2.1 GHz bound the measured rate
    assert 0.2 * 16384 * sms * 1.0e9 / 1e12 < tf < 16384 * sms * 2.1e9 / 1e12 * 1.05
    tf_copy = max(_rate(B, 240, True)[1] for _ in range(3))
    # the scale copy only takes pipe time (and N = 240 does 15/16 of the work per MMA); the
    # margin is the SM clock's drift between timed runs under the power cap
    assert 0.0 < tf_copy < tf * 1.15
    # zero operands: the same FLOPs, a rate in the same physical range
    fz, tz = max((_rate(B, 256, False, random_operands=False) for _ in range(3)), key=lambda r: r[1])
    assert fz == f and 0.2 * 16384 * sms * 1.0e9 / 1e12 < tz < 16384 * sms * 2.1e9 / 1e12 * 1.05
