"""Pins for the oracle's MXFP4 quantizer along an arbitrary axis, its MXFP4 weight-only
linear (optionally with FP8 activations) and its FP8 E4M3 static per-tensor linear.

Pages: "quantization_mxfp4" (KerasFormers), Primitives (MXFP4Quantizer.quantize(w, axis):
one contracting axis, moved to the end; a value-exact inverse on the lattice) and "As a
quantize_model scheme" (any Dense kernel stored MXFP4 and dequantized on the fly; the
contracting dim a multiple of 32, else a clear error); "gpt-oss-120b-mxfp4-fp8attn-v2",
Model Details / Quantization Recipe (attention Q/K/V/O projections in FP8 E4M3 with a
static per-tensor weight scale and input scale from a min-max observer).

The independent side: numpy matmul over values decoded from the e2m1 bit fields
(numpy_ref) and torch's own float8_e4m3fn casts.
"""
import numpy as np
import pytest
import torch

import numpy_ref
import oracle

_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _lattice_along(shape, axis, seed):
    """Values on the scaled e2m1 grid: every 32-value block along `axis` holds grid points
    times 2^e_b with one of them in {4, 6} (so the block's exponent is exactly e_b)."""
    rng = np.random.default_rng(seed)
    moved = np.moveaxis(np.empty(shape), axis, -1).shape
    K = moved[-1]
    g = rng.choice(_GRID, size=moved) * rng.choice([-1.0, 1.0], size=moved)
    nb = K // 32
    e = rng.integers(-60, 60, size=moved[:-1] + (nb,))
    g = g.reshape(moved[:-1] + (nb, 32))
    g[..., 0] = rng.choice([4.0, 6.0, -4.0, -6.0], size=moved[:-1] + (nb,))
    vals = np.ldexp(g, e[..., None]).reshape(moved)
    return np.moveaxis(vals, -1, axis).astype(np.float32), (e + 127).astype(np.uint8)


@pytest.mark.parametrize("shape,axis", [((64, 6, 5), 0), ((3, 96, 4), 1), ((2, 5, 32), 2),
                                        ((32, 7), 0), ((5, 64), -1)])
def test_axis_quantizer_is_value_exact_on_the_lattice_along_its_axis(shape, axis):
    w, scale_bytes = _lattice_along(shape, axis, seed=sum(shape))
    blocks, scales = oracle.quantize_axis(w, axis)
    K = shape[axis]
    moved = np.moveaxis(w, axis, -1).shape
    assert blocks.shape == moved[:-1] + (K // 2,) and scales.shape == moved[:-1] + (K // 32,)
    assert np.array_equal(scales, scale_bytes)          # blocks run along the axis
    back = oracle.dequantize_axis(blocks, scales, axis)
    assert back.shape == w.shape
    assert np.array_equal(back.view(np.uint32), w.view(np.uint32))


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_axis_quantizer_moves_the_axis_last(axis):
    rng = np.random.default_rng(axis)
    w = (rng.standard_normal((64, 96, 32)) * 0.05).astype(np.float32)
    b, s = oracle.quantize_axis(w, axis)
    rb, rs = oracle.quantize(np.ascontiguousarray(np.moveaxis(w, axis, -1)))
    assert np.array_equal(b, rb) and np.array_equal(s, rs)
    deq = numpy_ref.dequant(rb, rs)                        # bit-field decode, then the axis back
    assert np.array_equal(oracle.dequantize_axis(b, s, axis).astype(np.float64), np.moveaxis(deq, -1, axis))


def test_axis_quantizer_rejects_a_contracting_dim_off_the_block_size():
    with pytest.raises(oracle.OracleError) as ei:
        oracle.quantize_axis(np.zeros((33, 4), np.float32), 0)
    assert ei.value.rc == oracle.EALIGN


def _bf16_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("fp8", [False, True])
def test_mxfp4_linear_matches_numpy(fp8):
    rng = np.random.default_rng(7 + fp8)
    T, K, N = 9, 320, 48
    x = _bf16_bits(rng.standard_normal((T, K)))
    blocks, scales = oracle.quantize((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    bias = (rng.standard_normal(N) * 0.01).astype(np.float32)
    s = np.float32(np.abs(numpy_ref.bf16_to_f64(x)).max() / 448.0) if fp8 else None
    out, acc = oracle.linear(x, blocks, scales, bias, act_scale=s)
    xv = numpy_ref.bf16_to_f64(x)
    if fp8:
        xv = numpy_ref.fp8_e4m3((xv.astype(np.float32) / s).astype(np.float32))
    dot = xv @ numpy_ref.dequant(blocks, scales).T
    ref = (np.float64(s if fp8 else 1.0) * dot).astype(np.float32) + bias
    assert np.array_equal(acc.view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(out, _bf16_bits(ref))
    # no bias means a zero bias
    _, acc0 = oracle.linear(x, blocks, scales, None, act_scale=s)
    assert np.array_equal(acc0, (np.float64(s if fp8 else 1.0) * dot).astype(np.float32) + np.float32(0.0))


def test_mxfp4_linear_rejects_a_contracting_dim_off_the_block_size():
    with pytest.raises(oracle.OracleError) as ei:
        oracle.linear(np.zeros((2, 48), np.uint16), np.zeros((4, 24), np.uint8), np.zeros((4, 1), np.uint8))
    assert ei.value.rc == oracle.EALIGN


def test_fp8_linear_matches_numpy_and_torch_casts():
    rng = np.random.default_rng(11)
    T, K, N = 7, 200, 40
    xf = rng.standard_normal((T, K)).astype(np.float32)
    xf[:, 3] *= 50.0                                      # an outlier channel: saturates at 448
    x = _bf16_bits(xf)
    w = (rng.standard_normal((N, K)) * 0.03).astype(np.float32)
    s_w = np.float32(np.abs(w).max() / 448.0)             # static per-tensor, min-max observer
    wq = oracle.fp8_quantize(w, s_w)
    assert (wq & 0x7F).max() == 0x7E                    # the largest magnitude maps to 448
    s_x = np.float32(4.0 / 448.0)
    bias = (rng.standard_normal(N) * 0.01).astype(np.float32)
    out, acc = oracle.fp8_linear(x, wq, s_x, s_w, bias)
    xv = numpy_ref.fp8_e4m3((numpy_ref.bf16_to_f64(x).astype(np.float32) / s_x).astype(np.float32))
    wv = torch.from_numpy(wq).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    dot = xv @ wv.T
    ref = (np.float64(s_x) * np.float64(s_w) * dot).astype(np.float32) + bias
    assert np.array_equal(acc.view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(out, _bf16_bits(ref))
