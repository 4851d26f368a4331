"""GPU parity of the dense all-experts path (moe_mxfp4_forward_dense).

"quantization_mxfp4" (KerasFormers), As GPT-OSS's native format: long prefills may run
every expert on every token instead of dispatching the routed ones, with identical output.
The router gates are zero off each token's top-k, so the dense weighted sum over all E
experts equals the routed sum term for term. Checks: against the oracle (its dense mode,
which equals its routed mode bit for bit) within the layer bar; and bit for bit against the
GPU's routed path where both run the same expert kernels (T > 64), since every output row
of the grouped GEMMs depends only on its own activation row.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from helpers import output_tolerance_ok, pack, to_device
from mxfp4_block_scaled_moe_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from mxfp4_block_scaled_moe_b200 import binding
    return binding


def _run(B, fn, d, k, act_scale=None):
    out = fn(d["x"], d["router_w"], d["router_b"], d["gu_blocks"], d["gu_scales"], d["gu_bias"],
             d["d_blocks"], d["d_scales"], d["d_bias"], k, act_scale=act_scale)
    B.mxmoe_check()
    return out


@pytest.mark.parametrize("E,k,T,H,I,fp8", [(4, 2, 16, 256, 256, False), (4, 2, 16, 256, 256, True),
                                          (8, 3, 77, 320, 192, False), (8, 3, 77, 320, 192, True),
                                          (16, 4, 200, 512, 384, True)])
def test_dense_matches_the_oracle(B, E, k, T, H, I, fp8):
    lay = inputs.small_layer(E=E, k=k, T=T, H=H, I=I, seed=31, router_bias=True,
                             router_std=1.0 / np.sqrt(H))
    p = pack(lay)
    d = to_device(p)
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, k) if fp8 else None
    got = inputs.bits(_run(B, B.moe_mxfp4_forward_dense, d, k, s))
    ob, oacc, oidx, _ = p.oracle_forward(act_scale=s, dense=True)
    gi, _ = B.moe_route_topk(d["x"], d["router_w"], d["router_b"], k)
    ol = oracle.router_logits(p.x, p.router_w, p.router_b)
    srt = -np.sort(-ol, axis=1)
    clear = srt[:, k - 1] - srt[:, k] > 1e-5 * np.abs(ol).max()
    assert np.array_equal(gi.cpu().numpy()[clear], oidx[clear])
    ok, rel, excess = output_tolerance_ok(got[clear], oacc[clear])
    assert ok, f"max|d|/max|ref| = {rel:.3e}, worst excess {excess:.3e}"


@pytest.mark.parametrize("fp8", [True, False])
def test_dense_equals_routed_bit_for_bit(B, fp8):
    """T = 300 > 64: both paths run the tcgen05 grouped GEMMs (FP8, or bf16 as two e4m3
    parts); the dense one on all 8 experts for every token, the routed one on the top 4."""
    lay = inputs.small_layer(E=8, k=4, T=300, H=512, I=512, seed=33, router_bias=True,
                             router_std=1.0 / np.sqrt(512))
    p = pack(lay)
    d = to_device(p)
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, 4) if fp8 else None
    routed = _run(B, B.moe_mxfp4_forward, d, 4, s)
    dense = _run(B, B.moe_mxfp4_forward_dense, d, 4, s)
    assert torch.equal(routed.view(torch.int16), dense.view(torch.int16))


def test_dense_rejects_shapes_its_kernels_do_not_take(B):
    p = pack(inputs.small_layer(E=4, k=2, T=8, H=352, I=224, seed=1))
    d = to_device(p)
    with pytest.raises(B.MxmoeError) as ei:
        _run(B, B.moe_mxfp4_forward_dense, d, 2)
    assert ei.value.rc == B.EUNSUPPORTED


@pytest.mark.parametrize("fp8", [True, False])
def test_every_expert_selected_runs_dense_and_matches_the_oracle(B, fp8):
    """k == E above the decode sizes: moe_mxfp4_forward takes the dense path (the measured
    crossover); the result still matches the oracle's routed (= dense) layer."""
    lay = inputs.small_layer(E=8, k=8, T=150, H=256, I=256, seed=35, router_bias=True,
                             router_std=1.0 / np.sqrt(256))
    p = pack(lay)
    d = to_device(p)
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, 8) if fp8 else None
    got = _run(B, B.moe_mxfp4_forward, d, 8, s)
    dense_launches = B.mxmoe_last_launch_count()
    dense = _run(B, B.moe_mxfp4_forward_dense, d, 8, s)
    assert dense_launches == B.mxmoe_last_launch_count()
    assert torch.equal(got.view(torch.int16), dense.view(torch.int16))
    _, oacc, _, _ = p.oracle_forward(act_scale=s)
    ok, rel, excess = output_tolerance_ok(inputs.bits(got), oacc)
    assert ok, f"max|d|/max|ref| = {rel:.3e}, worst excess {excess:.3e}"
