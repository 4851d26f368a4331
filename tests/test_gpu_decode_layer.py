"""GPU parity of the one-launch decode layer (T <= 8 tokens: router logits, top-k softmax,
token parts, gate_up + SwiGLU, down and the combine in one persistent grid) against the
oracle, element by element over every output.

Page "quantization_mxfp4" (KerasFormers), As GPT-OSS's native format (routed experts,
(E, 2I, H) / (E, H, I) packed layout, full-precision biases); W-MXFP4/A-FP8 option from
"amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8", Quantization schemes.

Bar: |out - ref| <= 2e-3 * max|ref| + half a bf16 ulp of the reference element (the layer
tolerance of the other layer tests), on every token whose k-th and (k+1)-th router logits
are not a near tie. Every case also checks that the forward was one kernel launch.
"""
import dataclasses

import numpy as np
import pytest
import oracle
from helpers import output_tolerance_ok, pack, to_device
from mxfp4_block_scaled_moe_b200 import inputs

pytestmark = pytest.mark.gpu

_CACHE = {}


@pytest.fixture(scope="module")
def B():
    from mxfp4_block_scaled_moe_b200 import binding
    return binding


def case(E, k, T, H, I, seed, router_std=0.02, router_bias=True, cache=True):
    key = (E, k, T, H, I, seed, router_std, router_bias)
    if cache and key in _CACHE:
        return _CACHE[key]
    lay = inputs.small_layer(E=E, k=k, T=T, H=H, I=I, seed=seed, router_bias=router_bias, router_std=router_std)
    p = pack(lay)
    d = to_device(p)
    if cache:
        _CACHE[key] = (p, d)
    return p, d


def forward(B, p, d, act_scale=None, x=None):
    out = B.moe_mxfp4_forward(d["x"] if x is None else x, d["router_w"], d["router_b"], d["gu_blocks"],
                              d["gu_scales"], d["gu_bias"], d["d_blocks"], d["d_scales"], d["d_bias"], p.lay.k,
                              act_scale=act_scale)
    launches = B.mxmoe_last_launch_count()
    B.mxmoe_check()
    return out, launches


def check(p, out, act_scale=None, x_bits=None):
    k, E = p.lay.k, p.lay.E
    x = p.x if x_bits is None else x_bits
    ob, oacc, oidx, _ = oracle.moe_forward(x, p.router_w, p.router_b, *p.weights, k, act_scale=act_scale)
    ol = oracle.router_logits(x, p.router_w, p.router_b)
    if E > k:
        srt = -np.sort(-ol, axis=1)
        clear = srt[:, k - 1] - srt[:, k] > 1e-5 * np.abs(ol).max()
    else:
        clear = np.ones(x.shape[0], bool)
    assert clear.any()
    got = inputs.bits(out)
    ok, rel, excess = output_tolerance_ok(got[clear], oacc[clear])
    assert ok, f"max|d|/max|ref| = {rel:.3e}, worst excess over the bound {excess:.3e}"
    return rel


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 6, 7, 8])
def test_every_batch_size(B, T, fp8):
    """N = 16 (T <= 4) and N = 32 (T = 5 .. 8) token operands, H = I = 512: two 256-deep
    stages, four gate_up tiles, two down tile pairs per expert."""
    p, d = case(32, 4, T, 512, 512, seed=31)
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, 4) if fp8 else None
    out, n = forward(B, p, d, act_scale=s)
    assert n == 1
    check(p, out, act_scale=s)


@pytest.mark.parametrize("fp8", [False, True])
def test_ragged_tiles_and_stages_every_expert(B, fp8):
    """k = E = 4: every token in every expert. H = 384 (a 128-deep last gate_up stage),
    I = 320 (a 64-row last gate_up tile, a 64-deep last down stage), H != I."""
    p, d = case(4, 4, 8, 384, 320, seed=32)
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, 4) if fp8 else None
    out, n = forward(B, p, d, act_scale=s)
    assert n == 1
    check(p, out, act_scale=s)


def test_largest_expert_count_and_k(B):
    """E = 256, k = 8, T = 8: up to 64 routed experts, the most the layer handles."""
    p, d = case(256, 8, 8, 256, 256, seed=33, router_std=1.0 / 16)
    out, n = forward(B, p, d)
    assert n == 1
    check(p, out)


def test_single_expert(B):
    """E = k = 1: every token through the one expert with weight 1."""
    p, d = case(1, 1, 3, 128, 128, seed=34)
    out, n = forward(B, p, d)
    assert n == 1
    check(p, out)


@pytest.mark.parametrize("T", [1, 4])
def test_120b_shape(B, T):
    """The 120B expert set (E = 128, H = I = 2880) at decode batch sizes."""
    if "120b" not in _CACHE:
        p = pack(inputs.decode_layer(T=8, E=128, seed=35))
        _CACHE["120b"] = (p, to_device(p))
    p8, d8 = _CACHE["120b"]
    p = dataclasses.replace(p8, x=p8.x[:T], lay=dataclasses.replace(p8.lay, T=T, x=p8.lay.x[:T]))
    d = dict(d8, x=d8["x"][:T].contiguous())
    out, n = forward(B, p, d)
    assert n == 1
    check(p, out)


def test_repeated_calls_and_other_paths_between(B):
    """Counters return to zero: three different one-token inputs in a row, then a 64-token
    and a 300-token call on the same workspace, then the one-token inputs again."""
    p, d = case(32, 4, 8, 512, 512, seed=36)
    xs = [d["x"][i:i + 1].contiguous() for i in range(3)]
    outs = []
    for x in xs:
        out, n = forward(B, p, d, x=x)
        assert n == 1
        outs.append(inputs.bits(out).copy())
    for T in (64, 300):
        big = inputs.small_layer(E=32, k=4, T=T, H=512, I=512, seed=36, router_bias=True)
        B.moe_mxfp4_forward(big.x.cuda(), d["router_w"], d["router_b"], d["gu_blocks"], d["gu_scales"],
                            d["gu_bias"], d["d_blocks"], d["d_scales"], d["d_bias"], 4)
        B.mxmoe_check()
    for i, x in enumerate(xs):
        out, _ = forward(B, p, d, x=x)
        assert np.array_equal(inputs.bits(out), outs[i])   # bit-identical on a rerun
        check(p, out, x_bits=p.x[i:i + 1])
