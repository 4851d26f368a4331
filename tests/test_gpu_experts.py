"""The layer's expert half on pre-grouped rows (moe_mxfp4_experts) and its weighted combine
(moe_combine): the two pieces a partition of the experts over several GPUs uses around
its exchange of rows. Together, on the rows the layer's own routing and permutation give,
they reproduce moe_mxfp4_forward bit for bit (same expert kernels above the decode sizes).

"quantization_mxfp4" (KerasFormers), As GPT-OSS's native format (routed experts, outputs
summed with their router gates).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import pack, to_device
from mxfp4_block_scaled_moe_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from mxfp4_block_scaled_moe_b200 import binding
    return binding


@pytest.mark.parametrize("fp8", [True, False])
def test_grouped_experts_and_combine_reproduce_the_layer(B, fp8):
    lay = inputs.small_layer(E=8, k=2, T=300, H=512, I=384, seed=41, router_bias=True,
                             router_std=1.0 / np.sqrt(512))
    p = pack(lay)
    d = to_device(p)
    k = lay.k
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, k) if fp8 else None
    ref = B.moe_mxfp4_forward(d["x"], d["router_w"], d["router_b"], d["gu_blocks"], d["gu_scales"],
                              d["gu_bias"], d["d_blocks"], d["d_scales"], d["d_bias"], k, act_scale=s)
    idx, w = B.moe_route_topk(d["x"], d["router_w"], d["router_b"], k)
    offsets, perm_token, perm_slot = B.moe_permute(idx, lay.E)
    rows = d["x"][perm_token.long()].contiguous()          # test-side gather of the grouped rows
    y = B.moe_mxfp4_experts(rows, offsets, d["gu_blocks"], d["gu_scales"], d["gu_bias"], d["d_blocks"],
                            d["d_scales"], d["d_bias"], act_scale=s)
    inv = torch.empty(lay.T * k, dtype=torch.int32, device="cuda")
    inv[(perm_token * k + perm_slot).long()] = torch.arange(lay.T * k, dtype=torch.int32, device="cuda")
    out = B.moe_combine(y, idx, w, inv)
    B.mxmoe_check()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    # and each expert row against the oracle's per-pair FFN
    yo = oracle.expert_rows(inputs.bits(rows), np.repeat(np.arange(lay.E, dtype=np.int32),
                                                          np.diff(offsets.cpu().numpy())), *p.weights,
                            act_scale=s)
    yg = y.cpu().numpy()
    assert np.max(np.abs(yg - yo)) <= 2e-3 * np.max(np.abs(yo))
