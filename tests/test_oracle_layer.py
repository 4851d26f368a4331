"""Pins for the oracle's MoE expert layer.

Page "quantization_mxfp4" (KerasFormers), "As GPT-OSS's native format": experts are
(E, 2I, H) gate_up and (E, H, I) down packed blocks + scales with full-precision biases;
decode dequantizes only the top-k routed experts "at identical output" to the dense
all-experts path (about 8x less dequant per layer); "Footprint": GPT-OSS-120B experts
are ~57 GB packed vs ~230 GB in bf16. Activation path W-MXFP4/A-FP8:
"amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8", Quantization schemes.
"""
import json
import os

import numpy as np
import pytest

import oracle
from helpers import bf16_bits_to_f32, pack
from mxfp4_block_scaled_moe_b200 import inputs
import numpy_ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


@pytest.fixture(scope="module")
def tiny():
    return pack(inputs.tiny_layer(seed=0))


@pytest.fixture(scope="module")
def small():
    return pack(inputs.small_layer(E=8, k=3, T=24, H=192, I=128, seed=5, router_bias=True))


def _fp8_scales(p):
    return oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, p.lay.k)


@pytest.mark.parametrize("case", ["tiny", "small"])
@pytest.mark.parametrize("fp8", [False, True])
def test_layer_matches_numpy_restatement(case, fp8, request):
    p = request.getfixturevalue(case)
    acts = _fp8_scales(p) if fp8 else None
    out, acc, idx, w = p.oracle_forward(act_scale=acts)
    ref_acc, ref_idx, ref_w = numpy_ref.moe_forward(p.x, p.router_w, p.router_b, *p.weights,
                                                    p.lay.k, act_scale=acts)
    assert np.array_equal(idx, ref_idx)
    assert np.allclose(w, ref_w, rtol=1e-6, atol=0)
    scale = np.abs(ref_acc).max()
    # both sides differ only in the order of exact-product double sums
    assert np.max(np.abs(acc - ref_acc)) <= 1e-5 * scale
    # out is the bf16 rounding of acc
    assert np.array_equal(out, oracle.bf16_round(acc))


@pytest.mark.parametrize("fp8", [False, True])
def test_routed_equals_dense_bit_exact(tiny, small, fp8):
    for p in (tiny, small):
        acts = _fp8_scales(p) if fp8 else None
        r = p.oracle_forward(act_scale=acts, dense=False)
        d = p.oracle_forward(act_scale=acts, dense=True)
        assert np.array_equal(r[0], d[0]) or np.array_equal(
            bf16_bits_to_f32(r[0]), bf16_bits_to_f32(d[0]))
        assert np.array_equal(r[1], d[1])


def test_single_expert_ffn_against_triple_loop():
    """k = E = 1 makes the layer one expert FFN with gate 1; check it element by element
    with plain Python loops on a very small shape."""
    lay = inputs.small_layer(E=1, k=1, T=2, H=64, I=32, seed=9)
    p = pack(lay)
    out, acc, idx, w = p.oracle_forward()
    assert (idx == 0).all() and (w == 1.0).all()
    wgu = numpy_ref.dequant(p.gu_blocks, p.gu_scales)[0]
    wd = numpy_ref.dequant(p.d_blocks, p.d_scales)[0]
    x = numpy_ref.bf16_to_f64(p.x)
    H, I = 64, 32
    for t in range(2):
        g = []
        for r in range(2 * I):
            s = 0.0
            for h in range(H):
                s += x[t, h] * wgu[r, h]
            g.append(np.float32(np.float32(s) + p.gu_bias[0, r]))
        a = []
        for i in range(I):
            gate, up = float(g[i]), float(g[I + i])
            a.append(numpy_ref.round_bf16(np.array([gate / (1 + np.exp(-gate)) * up],
                                                   np.float32))[0])
        for r in range(H):
            s = 0.0
            for i in range(I):
                s += a[i] * wd[r, i]
            y = np.float32(np.float32(s) + p.d_bias[0, r])
            assert abs(float(acc[t, r]) - float(y)) <= 1e-6 * max(1.0, abs(float(y)))


def test_fp8_path_uses_the_static_scales(tiny):
    """A-FP8 output stays close to the bf16-activation output (two e4m3 roundings of
    the activations, relative error a few percent of the output scale) and is not equal
    to it."""
    acts = _fp8_scales(tiny)
    _, acc16, _, _ = tiny.oracle_forward()
    _, acc8, _, _ = tiny.oracle_forward(act_scale=acts)
    rel = np.abs(acc8 - acc16).max() / np.abs(acc16).max()
    assert 1e-4 < rel < 0.1


def test_calibration_is_minmax_over_448(tiny):
    s = _fp8_scales(tiny)
    x = bf16_bits_to_f32(tiny.x)
    assert s[0] == np.float32(np.abs(x).max()) / np.float32(448.0)
    # s1 from the numpy restatement's gated activations on the routed pairs
    ref = numpy_ref
    xf = ref.bf16_to_f64(tiny.x)
    logits = (xf @ ref.bf16_to_f64(tiny.router_w).T + ref.bf16_to_f64(tiny.router_b)).astype(np.float32)
    idx, _ = ref.topk_softmax(logits, tiny.lay.k)
    wgu = ref.dequant(tiny.gu_blocks, tiny.gu_scales)
    I = tiny.lay.I
    amax = 0.0
    for t in range(xf.shape[0]):
        for e in idx[t]:
            g = (wgu[e] @ xf[t]).astype(np.float32) + tiny.gu_bias[e]
            gate, up = g[:I].astype(np.float64), g[I:].astype(np.float64)
            a = (gate / (1 + np.exp(-gate)) * up).astype(np.float32)
            amax = max(amax, float(np.abs(a).max()))
    assert abs(s[1] - np.float32(amax) / np.float32(448)) <= 1e-5 * s[1]


# ------------------------------------------------------------- page figures ----


def test_footprint_matches_page_figures():
    g = json.load(open(GOLDEN))
    H = I = g["hidden_size"]["value"]
    E = g["experts_120b"]["value"]
    L = g["layers_120b"]["value"]
    gu = np.zeros((2 * I, H), np.float32)
    dn = np.zeros((H, I), np.float32)
    b1, s1 = oracle.quantize(gu)
    b2, s2 = oracle.quantize(dn)
    per_expert = b1.nbytes + s1.nbytes + b2.nbytes + s2.nbytes
    assert per_expert == 13_219_200
    assert per_expert * 8 / (gu.size + dn.size) == 4.25        # bits per weight
    packed = per_expert * E * L
    assert round(packed / 2 ** 30) == g["experts_packed_gb_120b"]["value"]     # ~57
    bf16 = (gu.size + dn.size) * 2 * E * L
    assert round(bf16 / 1e9, -1) == g["experts_bf16_gb_120b"]["value"]         # ~230
    assert abs(bf16 / packed - g["ratio_vs_bf16"]["value"]) < 0.3              # ~4x


def test_routed_decode_dequantizes_k_of_E_experts():
    g = json.load(open(GOLDEN))
    lay = inputs.small_layer(E=g["experts_20b"]["value"], k=g["top_k"]["value"], T=1,
                             H=64, I=64, seed=11)
    p = pack(lay)
    _, _, idx, _ = p.oracle_forward()
    touched = len(set(idx[0].tolist()))
    assert touched == lay.k
    assert lay.E / touched == g["decode_dequant_saving"]["value"]   # ~8x
