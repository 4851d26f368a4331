"""GPU parity of the MXFP4 codec along an arbitrary axis, the MXFP4 weight-only linear
(optionally with FP8 activations) and the FP8 E4M3 static per-tensor linear, against the
oracle.

Pages: "quantization_mxfp4" (KerasFormers), Primitives (MXFP4Quantizer along one axis,
moved to the end; bit-exact decode) and As a quantize_model scheme (a Dense kernel stored
MXFP4, dequantized on the fly); "amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8",
Quantization schemes (FP8 per-tensor activations); "gpt-oss-120b-mxfp4-fp8attn-v2",
Model Details / Quantization Recipe (attention projections with FP8 E4M3 weights and
static per-tensor weight and input scales).

Bars: the codec is bit-exact. A linear's output is within 2e-3 * max|ref| plus half a
bf16 ulp of the oracle's fp32 result (the layer's bar: fp32 accumulation in another
order, then one bf16 rounding).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import output_tolerance_ok
from mxfp4_block_scaled_moe_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from mxfp4_block_scaled_moe_b200 import binding
    return binding


def _codec_tensor(shape, seed):
    n = int(np.prod(shape))
    w = inputs.codec_tensor(1, n, seed=seed, tag="axis", device="cuda").reshape(shape)
    return w.contiguous()


@pytest.mark.parametrize("shape,axis", [((64, 7, 5), 0), ((3, 96, 40), 1), ((2, 5, 64), 2), ((2880, 96), 0),
                                        ((32, 1), 0), ((6, 32, 33), 1)])
def test_axis_codec_bit_exact(B, shape, axis):
    w = _codec_tensor(shape, seed=sum(shape) + axis)
    gb, gs = B.mxfp4_quantize_axis(w, axis)
    ob, os_ = oracle.quantize_axis(w.cpu().numpy(), axis)
    assert np.array_equal(gb.cpu().numpy(), ob) and np.array_equal(gs.cpu().numpy(), os_)
    for dt, name in ((torch.float32, "f32"), (torch.bfloat16, "bf16")):
        g = B.mxfp4_dequantize_axis(gb, gs, axis, dt)
        o = oracle.dequantize_axis(ob, os_, axis, out=name)
        gv = g.cpu().view(torch.int32 if dt == torch.float32 else torch.int16).numpy()
        assert np.array_equal(gv.view(np.uint32 if dt == torch.float32 else np.uint16),
                              o.view(np.uint32) if dt == torch.float32 else o)


def _bf16(shape, seed, std=1.0):
    return inputs.normal(shape, std, seed, "lin_x", 0, "cuda", torch.bfloat16)


@pytest.mark.parametrize("T,K,N,fp8,bias", [(1, 2880, 512, False, True), (8, 2880, 512, True, True),
                                            (64, 640, 256, False, False), (65, 2880, 640, True, True),
                                            (300, 640, 256, False, True), (300, 640, 256, True, False),
                                            (77, 352, 224, False, True), (130, 352, 224, True, True)])
def test_mxfp4_linear(B, T, K, N, fp8, bias):
    """T <= 64 and odd multiples of 32 run the register-dequant kernel; more tokens with K,
    N multiples of 64 the tcgen05 grouped GEMM (FP8, or bf16 as two e4m3 parts)."""
    x = _bf16((T, K), seed=T + K)
    w = inputs.normal((N, K), 0.02, 3, "lin_w", 0, "cuda")
    blocks, scales = B.mxfp4_quantize(w)
    b = inputs.normal((N,), 0.01, 4, "lin_b", 0, "cuda") if bias else None
    s = float(x.float().abs().max()) / 448.0 if fp8 else None
    got = B.mxfp4_linear(x, blocks, scales, b, act_scale=s)
    B.mxmoe_check()
    _, ref = oracle.linear(inputs.bits(x), blocks.cpu().numpy(), scales.cpu().numpy(),
                           None if b is None else b.cpu().numpy(), act_scale=s)
    ok, rel, excess = output_tolerance_ok(inputs.bits(got), ref)
    assert ok, f"max|d|/max|ref| = {rel:.3e}, worst excess {excess:.3e}"


@pytest.mark.parametrize("T,K,N,bias", [(1, 2880, 512, True), (7, 640, 1024, True), (64, 2880, 512, False),
                                        (130, 640, 512, True), (300, 352, 264, True), (600, 512, 256, False)])
def test_fp8_linear(B, T, K, N, bias):
    """Few tokens split K over the SMs (fp32 partials added in split order); more run one
    unit per (128-token, 256-row) tile; ragged T, N and K tails (K = 352 = 2.75 x 128)."""
    x = _bf16((T, K), seed=2 * T + K)
    w = inputs.normal((N, K), 0.03, 5, "fp8_w", 0, "cuda")
    s_w = float(w.abs().max()) / 448.0
    wq = B.moe_fp8_quantize(w.to(torch.bfloat16), s_w)
    s_x = float(x.float().abs().max()) / 448.0
    b = inputs.normal((N,), 0.01, 6, "fp8_b", 0, "cuda") if bias else None
    got = B.fp8_linear(x, wq, s_x, s_w, b)
    B.mxmoe_check()
    _, ref = oracle.fp8_linear(inputs.bits(x), wq.cpu().numpy(), np.float32(s_x), np.float32(s_w),
                               None if b is None else b.cpu().numpy())
    ok, rel, excess = output_tolerance_ok(inputs.bits(got), ref)
    assert ok, f"max|d|/max|ref| = {rel:.3e}, worst excess {excess:.3e}"


def test_fp8_linear_attention_shapes_sampled(B):
    """The 120B model's attention projections at a prefill batch: fused Q/K/V (2880 ->
    5120) and O (4096 -> 2880), T = 1024, compared on sampled rows."""
    for K, N in ((2880, 5120), (4096, 2880)):
        T = 1024
        x = _bf16((T, K), seed=K)
        w = inputs.normal((N, K), 0.02, 7, "attn_w", K, "cuda")
        s_w = float(w.abs().max()) / 448.0
        wq = B.moe_fp8_quantize(w.to(torch.bfloat16), s_w)
        s_x = float(x.float().abs().max()) / 448.0
        b = inputs.normal((N,), 0.01, 8, "attn_b", K, "cuda")
        got = B.fp8_linear(x, wq, s_x, s_w, b)
        B.mxmoe_check()
        rows = np.array([0, 1, 127, 128, 500, 1023])
        _, ref = oracle.fp8_linear(inputs.bits(x)[rows], wq.cpu().numpy(), np.float32(s_x), np.float32(s_w),
                                   b.cpu().numpy())
        ok, rel, excess = output_tolerance_ok(inputs.bits(got)[rows], ref)
        assert ok, f"K={K} N={N}: max|d|/max|ref| = {rel:.3e}, worst excess {excess:.3e}"


def test_linear_argument_errors(B):
    x = _bf16((4, 96), seed=1)
    blocks = torch.zeros(48, 48, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(48, 3, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.MxmoeError) as ei:
        B.mxfp4_linear(x[:, :80].contiguous(), blocks[:, :40].contiguous(), scales[:, :2].contiguous())
    assert ei.value.rc == B.EALIGN
    with pytest.raises(B.MxmoeError) as ei:
        B.fp8_linear(x, torch.zeros(12, 96, dtype=torch.uint8, device="cuda"), 1.0, 1.0)
    assert ei.value.rc == B.EALIGN
    with pytest.raises(B.MxmoeError) as ei:
        B.fp8_linear(x, torch.zeros(16, 96, dtype=torch.uint8, device="cuda"), 0.0, 1.0)
    assert ei.value.rc == B.EINVAL
