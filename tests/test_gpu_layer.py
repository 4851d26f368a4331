"""GPU parity of the whole MoE expert layer (moe_mxfp4_forward) against the oracle.

Page "quantization_mxfp4" (KerasFormers), As GPT-OSS's native format (routed experts,
(E, 2I, H) / (E, H, I) packed layout, full-precision biases); W-MXFP4/A-FP8 option from
"amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8", Quantization schemes.

Bar (stated for the layer output): |out - ref| <= 2e-3 * max|ref| + half a bf16 ulp of
the reference element, where ref is the oracle's fp32 accumulator (the bf16 output
carries one extra rounding the fp32 arithmetic does not). Routing indices are compared
bit-exactly wherever the k-th and (k+1)-th router logits are not a near tie.

Weights are MXFP4-packed by the oracle's quantizer; the GPU consumes the same bytes.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from helpers import Packed, covering_rows, output_tolerance_ok, pack, to_device
from mxfp4_block_scaled_moe_b200 import inputs

pytestmark = pytest.mark.gpu

_CACHE = {}


def packed_weights(E, H, I, seed=0):
    """Oracle-packed expert weights of a synthetic layer (cached per shape)."""
    key = (E, H, I, seed)
    if key not in _CACHE:
        lay = inputs.small_layer(E=E, k=1, T=1, H=H, I=I, seed=seed, device="cuda")
        p = pack(lay)
        _CACHE[key] = (p, to_device(p))
    return _CACHE[key]


def layer_case(lay: inputs.Layer):
    """Pair a layer's activations/router with the cached packed weights of its shape."""
    wp, wd = packed_weights(lay.E, lay.H, lay.I, lay.seed)
    rb = None if lay.router_b is None else inputs.bits(lay.router_b)
    p = Packed(lay, inputs.bits(lay.x), inputs.bits(lay.router_w), rb, wp.gu_blocks,
               wp.gu_scales, wp.gu_bias, wp.d_blocks, wp.d_scales, wp.d_bias)
    d = dict(wd)
    d.update(x=lay.x.contiguous(), router_w=lay.router_w.contiguous(),
             router_b=None if lay.router_b is None else lay.router_b.contiguous())
    return p, d


@pytest.fixture(scope="module")
def B():
    from mxfp4_block_scaled_moe_b200 import binding
    return binding


def run_gpu(B, d, k, act_scale=None):
    out = B.moe_mxfp4_forward(d["x"], d["router_w"], d["router_b"], d["gu_blocks"],
                              d["gu_scales"], d["gu_bias"], d["d_blocks"], d["d_scales"],
                              d["d_bias"], k, act_scale=act_scale)
    B.mxmoe_check()
    return out


def check_rows(B, p: Packed, d, rows, act_scale=None, out=None):
    """Compare the GPU output rows `rows` with the oracle, routing gaps respected."""
    k = p.lay.k
    if out is None:
        out = run_gpu(B, d, k, act_scale)
    got = inputs.bits(out)[rows]
    ob, oacc, oidx, _ = p.oracle_forward(act_scale=act_scale, rows=rows)
    # routing: the GPU's indices must equal the oracle's wherever the selection is clear
    gi, _, gl = B.moe_route_topk(d["x"], d["router_w"], d["router_b"], k, with_logits=True)
    gi = gi.cpu().numpy()[rows]
    ol = oracle.router_logits(p.x[rows], p.router_w, p.router_b)
    srt = -np.sort(-ol, axis=1)
    clear = (srt[:, k - 1] - srt[:, k] > 1e-5 * np.abs(ol).max()) if p.lay.E > k else np.ones(len(rows), bool)
    assert np.array_equal(gi[clear], oidx[clear])
    ok, rel, excess = output_tolerance_ok(got[clear], oacc[clear])
    assert ok, f"max|d|/max|ref| = {rel:.3e}, worst excess over the bound {excess:.3e}"
    return rel


def test_tiny_bf16_all_outputs(B):
    p = pack(inputs.tiny_layer(seed=0))
    d = to_device(p)
    check_rows(B, p, d, np.arange(p.lay.T))


def test_tiny_fp8_all_outputs(B):
    p = pack(inputs.tiny_layer(seed=0))
    d = to_device(p)
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, p.lay.k)
    check_rows(B, p, d, np.arange(p.lay.T), act_scale=s)


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("H,I", [(320, 192), (352, 224)])
def test_small_ragged_layer(B, fp8, H, I):
    # T = 77 > 64 with a handful of rows per expert. H = 320 (10 blocks), I = 192 (6): the
    # tcgen05 grouped GEMMs with H != I and K tails (2.5 and 1.5 k-tiles of 128). H = 352,
    # I = 224 (odd multiples of 32, which neither tensor-core path takes): the register-
    # dequant kernels with H != I.
    p = pack(inputs.small_layer(E=8, k=3, T=77, H=H, I=I, seed=5, router_bias=True))
    d = to_device(p)
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, p.lay.k) if fp8 else None
    check_rows(B, p, d, np.arange(p.lay.T), act_scale=s)


@pytest.mark.parametrize("T", [1, 8, 64])
def test_decode_20b_shape_all_outputs(B, T):
    p, d = layer_case(inputs.decode_layer(T=T, E=32, device="cuda"))
    check_rows(B, p, d, np.arange(T))


@pytest.mark.parametrize("T", [1, 8])
def test_decode_20b_shape_fp8(B, T):
    """FP8 activations on a decode batch (static scales from the calibration batch): the
    e4m3 values are what the tensor-core decode path splits into e2m1 parts; T = 1 also
    takes the split-K reduction."""
    p, d = layer_case(inputs.decode_layer(T=T, E=32, device="cuda"))
    xc = inputs.calibration_x(device="cuda")
    s = oracle.calibrate(inputs.bits(xc), p.router_w, p.router_b, *p.weights, p.lay.k)
    check_rows(B, p, d, np.arange(T), act_scale=s)


@pytest.mark.parametrize("T,fp8", [(64, False), (57, True), (56, False), (29, False)])
def test_decode_row_groups(B, T, fp8):
    """Top-4 of 4 experts: every expert takes all T tokens. Above 56 routed rows an
    expert splits into row groups (56 + the rest), and groups wider than 28 rows take
    both accumulator slots of the decode GEMM."""
    p, d = layer_case(inputs.small_layer(E=4, k=4, T=T, H=512, I=512, seed=3, device="cuda"))
    s = None
    if fp8:
        xc = inputs.calibration_x(H=512, device="cuda")
        s = oracle.calibrate(inputs.bits(xc), p.router_w, p.router_b, *p.weights, p.lay.k)
    check_rows(B, p, d, np.arange(T), act_scale=s)


def test_decode_after_other_workspace_users(B):
    """The decode path's split-K and combine tickets share workspace bytes with other
    calls' buffers (here the router's logits): a call that overwrites them between two
    decode calls must not disturb the second."""
    p, d = layer_case(inputs.decode_layer(T=8, E=32, device="cuda"))
    check_rows(B, p, d, np.arange(8))
    big = inputs.small_layer(E=64, k=4, T=2000, H=320, I=192, seed=9, device="cuda")
    B.moe_route_topk(big.x, big.router_w, None, 4)   # logits land in the workspace
    torch.cuda.synchronize()
    check_rows(B, p, d, np.arange(8))


def test_decode_23_experts(B):
    p, d = layer_case(inputs.decode_layer(T=8, E=23, device="cuda"))
    check_rows(B, p, d, np.arange(8))


@pytest.mark.parametrize("H,I,E,k,T", [(512, 512, 8, 2, 600), (320, 320, 8, 3, 600),
                                       (2880, 2880, 6, 4, 300)])
def test_fp8_prefill_tcgen05_path(B, H, I, E, k, T):
    """T*k >= 1024 routed pairs with FP8 activations run the tcgen05 grouped GEMMs:
    K a multiple of 128, K with a 64-value tail (320 = 2.5 x 128), partial N tiles
    (I = 320 is 2 x 120 + 80 gate/up rows, H = 320 is 240 + 80 down rows), ragged
    expert loads."""
    lay = inputs.small_layer(E=E, k=k, T=T, H=H, I=I, seed=7, router_bias=True,
                             router_std=1.0 / np.sqrt(H))
    p = pack(lay)
    d = to_device(p)
    s = oracle.calibrate(p.x[:256], p.router_w, p.router_b, *p.weights, p.lay.k)
    out = run_gpu(B, d, k, act_scale=s)
    rows = np.arange(T) if H <= 512 else _sample_rows(T, 24, 3)
    check_rows(B, p, d, rows, act_scale=s, out=out)


@pytest.mark.parametrize("E,k,H,I,T,fp8", [
    (1, 1, 64, 32, 5, False),        # one expert: every token routes to it with weight 1
    (8, 8, 128, 96, 40, False),      # k = E: every expert selected, the routed path is the dense one
    (8, 8, 128, 96, 40, True),
    (256, 8, 256, 256, 200, False),  # the largest E and k the library takes
    (256, 8, 256, 256, 200, True),   # 1600 routed pairs: the tcgen05 FP8 path, ~6 rows per expert
    (16, 4, 32, 32, 70, False),      # the smallest contracting dims: one 32-value block
])
def test_degenerate_and_maximum_shapes(B, E, k, H, I, T, fp8):
    lay = inputs.small_layer(E=E, k=k, T=T, H=H, I=I, seed=11, router_bias=True,
                             router_std=1.0 / np.sqrt(H))
    p = pack(lay)
    d = to_device(p)
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, k) if fp8 else None
    check_rows(B, p, d, np.arange(T), act_scale=s)


@pytest.mark.parametrize("H,I,E,k,T", [(512, 512, 8, 2, 600), (320, 320, 8, 3, 600),
                                       (2880, 2880, 6, 4, 300)])
def test_bf16_prefill_two_part_tcgen05_path(B, H, I, E, k, T):
    """T*k >= 1024 routed pairs with bf16 activations run the tcgen05 grouped GEMMs with each
    activation split into two e4m3 parts: K a multiple of 128, K with a 64-value tail,
    partial N tiles, ragged expert loads."""
    lay = inputs.small_layer(E=E, k=k, T=T, H=H, I=I, seed=7, router_bias=True,
                             router_std=1.0 / np.sqrt(H))
    p = pack(lay)
    d = to_device(p)
    out = run_gpu(B, d, k)
    rows = np.arange(T) if H <= 512 else _sample_rows(T, 24, 3)
    check_rows(B, p, d, rows, out=out)


def _gpu_idx(B, d, k):
    idx, _ = B.moe_route_topk(d["x"], d["router_w"], d["router_b"], k)
    return idx.cpu().numpy()


def test_prefill_120b_shape_bf16_every_expert_tile(B):
    lay = inputs.prefill_layer(T=4096, E=128, device="cuda")
    p, d = layer_case(lay)
    out1 = run_gpu(B, d, lay.k)
    out2 = run_gpu(B, d, lay.k)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))   # run-to-run identical
    rows = covering_rows(_gpu_idx(B, d, lay.k), lay.E, extra=(0, 4095))
    check_rows(B, p, d, rows, out=out1)


@pytest.mark.parametrize("T,fp8", [(400, True), (400, False), (8, False), (8, True), (24, False), (24, True)])
def test_tensor_core_paths_with_H_ne_I(B, T, fp8):
    """H = 320 (2.5 k-tiles of 128), I = 192 (1.5): 1600 routed pairs take the tcgen05
    prefill GEMMs (FP8, or bf16 as two e4m3 parts), T = 8 the one-launch decode layer,
    T = 24 the tensor-core decode GEMMs (down's second 256-row unit holds 64 live rows in
    its first tile and none in its second)."""
    lay = inputs.small_layer(E=8, k=4, T=T, H=320, I=192, seed=13, router_bias=True,
                             router_std=1.0 / np.sqrt(320))
    p = pack(lay)
    d = to_device(p)
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, p.lay.k) if fp8 else None
    check_rows(B, p, d, np.arange(T), act_scale=s)


def _sample_rows(T, n, seed):
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(T, size=n, replace=False))
    rows[0], rows[-1] = 0, T - 1
    return rows


def test_prefill_120b_shape_fp8_every_expert_tile(B):
    lay = inputs.prefill_layer(T=4096, E=128, device="cuda")
    p, d = layer_case(lay)
    xc = inputs.calibration_x(device="cuda")
    s = oracle.calibrate(inputs.bits(xc), p.router_w, p.router_b, *p.weights, lay.k)
    out1 = run_gpu(B, d, lay.k, act_scale=s)
    out2 = run_gpu(B, d, lay.k, act_scale=s)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))   # run-to-run identical
    rows = covering_rows(_gpu_idx(B, d, lay.k), lay.E, extra=(0, 4095))
    check_rows(B, p, d, rows, act_scale=s, out=out1)


def test_prefill_zipf_skew_every_expert_tile(B):
    lay = inputs.zipf_layer(T=16384, E=128, device="cuda")
    p, d = layer_case(lay)
    idx = _gpu_idx(B, d, lay.k)
    load = np.bincount(idx.reshape(-1), minlength=lay.E)
    assert (load == 0).sum() >= 3 and load.max() > 10 * load.mean()
    xc = inputs.calibration_x(device="cuda")
    s = oracle.calibrate(inputs.bits(xc), p.router_w, p.router_b, *p.weights, lay.k)
    rows = covering_rows(idx, lay.E, extra=(0, 16383))
    check_rows(B, p, d, rows, act_scale=s)


def test_calibration_matches_oracle(B):
    lay = inputs.decode_layer(T=1, E=32, device="cuda")
    p, d = layer_case(lay)
    xc = inputs.calibration_x(device="cuda")
    g = B.moe_mxfp4_calibrate(xc, d["router_w"], d["router_b"], d["gu_blocks"], d["gu_scales"],
                              d["gu_bias"], d["d_blocks"], d["d_scales"], d["d_bias"], lay.k).cpu().numpy()
    o = oracle.calibrate(inputs.bits(xc), p.router_w, p.router_b, *p.weights, lay.k)
    assert g[0] == o[0]
    assert abs(g[1] - o[1]) <= 1e-5 * o[1]


def test_empty_batch_and_bad_arguments(B):
    p = pack(inputs.tiny_layer(seed=0))
    d = to_device(p)
    empty = dict(d, x=d["x"][:0])
    out = B.moe_mxfp4_forward(empty["x"], d["router_w"], d["router_b"], d["gu_blocks"],
                              d["gu_scales"], d["gu_bias"], d["d_blocks"], d["d_scales"],
                              d["d_bias"], 2)
    assert out.shape == (0, 256)
    L = B.lib()
    vp = lambda t: torch.cuda.current_stream().cuda_stream if t is None else t.data_ptr()
    args = [d[n].data_ptr() for n in ("x", "router_w", "router_b", "gu_blocks", "gu_scales",
                                       "gu_bias", "d_blocks", "d_scales", "d_bias")]
    o = torch.empty(16, 256, dtype=torch.bfloat16, device="cuda")
    import ctypes
    c = [ctypes.c_void_p(a) for a in args]
    assert L.moe_mxfp4_forward(*c, 4, 5, 16, 256, 256, None, ctypes.c_void_p(o.data_ptr()), None) == B.EUNSUPPORTED
    assert L.moe_mxfp4_forward(*c, 4, 2, 16, 250, 256, None, ctypes.c_void_p(o.data_ptr()), None) == B.EALIGN
    assert L.moe_mxfp4_forward(*c, 4, 2, 16, 256, 200, None, ctypes.c_void_p(o.data_ptr()), None) == B.EALIGN
    assert L.moe_mxfp4_forward(*c, 300, 2, 16, 256, 256, None, ctypes.c_void_p(o.data_ptr()), None) == B.EUNSUPPORTED
    c_bad = list(c)
    c_bad[0] = ctypes.c_void_p(args[0] + 2)
    assert L.moe_mxfp4_forward(*c_bad, 4, 2, 16, 256, 256, None, ctypes.c_void_p(o.data_ptr()), None) == B.EINVAL
    assert L.moe_mxfp4_forward(*c, 4, 2, 16, 256, 256, None, None, None) == B.EINVAL


# ------------------------------------------------ activation outliers, wide scale ranges --

_OUTLIER_CHANNELS = ((17, 1000.0), (1000, 300.0))


def _with_outliers(x: torch.Tensor) -> torch.Tensor:
    """x with two channels scaled up (one 10^3 x, one 300 x the rest), as bf16."""
    y = x.float().clone()
    for c, m in _OUTLIER_CHANNELS:
        y[:, c % x.shape[1]] *= m
    return y.to(torch.bfloat16)


@pytest.mark.parametrize("path,T,fp8", [("decode", 1, False), ("decode", 8, False), ("decode", 64, False),
                                        ("decode", 1, True), ("decode", 8, True),
                                        ("parts", 300, False), ("fp8", 300, True)])
def test_activation_outlier_channels(B, path, T, fp8):
    """Tokens whose row holds one channel 1000x and one 300x the others. On the decode
    path (T <= 64) each activation becomes four e2m1 parts under per-32-value block scales
    (a row-wide scale would leave the other values only the bits below the outlier's); on
    the bf16 prefill path two e4m3 parts under block scales; FP8 activations saturate at
    +-448 s0 with the scales of a calibration batch that has the same outlier channels."""
    if path == "decode":
        lay = inputs.decode_layer(T=T, E=32, device="cuda")
        rows = np.arange(T)
    else:
        lay = inputs.small_layer(E=6, k=4, T=T, H=2880, I=2880, seed=7, router_bias=True,
                                 router_std=1.0 / np.sqrt(2880), device="cuda")
        rows = _sample_rows(T, 24, 5)
    lay = dataclasses.replace(lay, x=_with_outliers(lay.x))
    p, d = layer_case(lay)
    s = None
    if fp8:
        xc = _with_outliers(inputs.calibration_x(device="cuda"))
        s = oracle.calibrate(inputs.bits(xc), p.router_w, p.router_b, *p.weights, p.lay.k)
    check_rows(B, p, d, rows, act_scale=s)


def _wide_scale_pack(lay: inputs.Layer, mode: str) -> Packed:
    """The layer's weights with C2's outliers (1% of values x 8) before the oracle's
    quantizer, then scale bytes rewritten: mode "tiny" sets 2% of the blocks to bytes 0-3
    (2^-127 .. 2^-124: subnormal products), mode "huge" sets 0.3% of them to bytes 136-140
    (2^9 .. 2^13 times the others' range) while outputs stay finite. Oracle and GPU consume
    the same bytes."""
    E, H, I = lay.E, lay.H, lay.I
    rng = np.random.default_rng(1234 + (mode == "huge"))
    gu_b = np.empty((E, 2 * I, H // 2), np.uint8)
    gu_s = np.empty((E, 2 * I, H // 32), np.uint8)
    d_b = np.empty((E, H, I // 2), np.uint8)
    d_s = np.empty((E, H, I // 32), np.uint8)

    def one(w):
        w = w.cpu().numpy().copy()
        w[rng.random(w.shape) < 0.01] *= 8.0
        b, sc = oracle.quantize(w)
        if mode == "tiny":
            m = rng.random(sc.shape) < 0.02
            sc[m] = rng.integers(0, 4, size=int(m.sum()))
        else:
            m = rng.random(sc.shape) < 0.003
            sc[m] = rng.integers(136, 141, size=int(m.sum()))
        return b, sc

    for e in range(E):
        gu_b[e], gu_s[e] = one(lay.gate_up(e))
        d_b[e], d_s[e] = one(lay.down(e))
    rb = None if lay.router_b is None else inputs.bits(lay.router_b)
    return Packed(lay, inputs.bits(lay.x), inputs.bits(lay.router_w), rb, gu_b, gu_s,
                  lay.gu_bias.cpu().numpy(), d_b, d_s, lay.d_bias.cpu().numpy())


@pytest.mark.parametrize("mode", ["tiny", "huge"])
@pytest.mark.parametrize("T,k,H,fp8", [(600, 2, 512, True), (600, 2, 512, False), (8, 4, 512, False),
                                       (8, 4, 512, True), (24, 4, 512, False), (100, 2, 480, False)])
def test_wide_e8m0_weight_scales(B, mode, T, k, H, fp8):
    """Weights whose e8m0 scale bytes span the format: blocks at bytes 0-3 beside ordinary
    ones near 120, or a few blocks at 136-140, on every path: the tcgen05 prefill GEMMs
    (T = 600, FP8 and bf16 as two parts), the one-launch decode layer (T = 8), the
    tensor-core decode GEMMs (T = 24) and the
    register-dequant kernels (H = I = 480, not a multiple of 64, which neither tensor-core
    path takes)."""
    lay = inputs.small_layer(E=8, k=k, T=T, H=H, I=H, seed=21, router_bias=True,
                             router_std=1.0 / np.sqrt(H), device="cuda")
    p = _wide_scale_pack(lay, mode)
    d = to_device(p)
    s = None
    if fp8:
        s = oracle.calibrate(p.x[: min(T, 256)], p.router_w, p.router_b, *p.weights, k)
    out = run_gpu(B, d, k, act_scale=s)
    assert torch.isfinite(out.float()).all()
    check_rows(B, p, d, np.arange(T), act_scale=s, out=out)
