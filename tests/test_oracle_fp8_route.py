"""Pins for the oracle's FP8 E4M3 cast, router, top-k softmax and permutation.

FP8: "amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8", Quantization schemes (FP8
symmetric per-tensor activations); "gpt-oss-120b-mxfp4-fp8attn-v2", Model Details
(E4M3, static per-tensor scales). Router: GPT-OSS top-4 routing ("gpt-oss-120b-mxfp4-
fp8attn-v2", Model Details: 128 experts, top-4) kept unquantized (same page,
config.json). Permutation: the routed dispatch of "quantization_mxfp4", As GPT-OSS's
native format.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_moe_b200 import inputs

# ------------------------------------------------------------------------- FP8 ----


def test_fp8_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.fp8_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok].view(np.uint32), ref[ok].view(np.uint32))
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF]) and got[0x7E] == 448.0


def test_fp8_encode_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    vals = oracle.fp8_decode(codes)
    assert np.array_equal(oracle.fp8_quantize(vals, 1.0), codes)


def _torch_e4m3(x32):
    return (torch.from_numpy(x32).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
            .view(torch.uint8).numpy())


def test_fp8_encode_matches_torch_cast_including_ties():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000) * 30,
        rng.standard_normal(5000) * 2.0 ** -7,        # subnormal range
        rng.standard_normal(2000) * 2.0 ** -12,       # underflow to +-0
        np.array([0.0, -0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11]),
    ]).astype(np.float32)
    # exact midpoints between adjacent finite codes (ties-to-even must decide)
    v = oracle.fp8_decode(np.arange(0x7E, dtype=np.uint8)).astype(np.float64)
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (v[:-1] + v[1:]) / 2)
    x = np.concatenate([x, mids, -mids])
    assert np.array_equal(oracle.fp8_quantize(x, 1.0), _torch_e4m3(x))


def test_fp8_saturates_beyond_448_and_keeps_nan():
    x = np.array([449.0, 464.0, 480.0, 1e30, np.inf, -500.0, -np.inf, np.nan], np.float32)
    q = oracle.fp8_quantize(x, 1.0)
    assert q[:5].tolist() == [0x7E] * 5 and q[5:7].tolist() == [0xFE] * 2
    assert (q[7] & 0x7F) == 0x7F


def test_fp8_static_scale_is_one_fp32_division():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(50000) * 3).astype(np.float32)
    for s in [np.float32(0.0123), np.float32(3.7), np.float32(1 / 448)]:
        with np.errstate(over="ignore"):
            quot = (x / s).astype(np.float32)
        assert np.array_equal(oracle.fp8_quantize(x, float(s)), _torch_e4m3(quot))


# ---------------------------------------------------------------------- router ----


def _bf16_bits_to_f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_router_logits_match_exactly_rounded_sum():
    lay = inputs.small_layer(E=8, T=12, H=96, router_bias=True, seed=3)
    x, rw, rb = inputs.bits(lay.x), inputs.bits(lay.router_w), inputs.bits(lay.router_b)
    got = oracle.router_logits(x, rw, rb)
    xf, wf, bf = _bf16_bits_to_f64(x), _bf16_bits_to_f64(rw), _bf16_bits_to_f64(rb)
    for t in range(x.shape[0]):
        for e in range(rw.shape[0]):
            exact = math.fsum(list(xf[t] * wf[e]) + [bf[e]])   # bf16 products exact in f64
            ref = np.float32(exact)
            assert abs(np.float64(got[t, e]) - np.float64(ref)) <= np.spacing(np.abs(ref))


def test_router_logits_match_numpy_matmul_and_null_bias():
    lay = inputs.small_layer(E=16, T=33, H=256, seed=4)
    x, rw = inputs.bits(lay.x), inputs.bits(lay.router_w)
    got = oracle.router_logits(x, rw, None)
    ref = (_bf16_bits_to_f64(x) @ _bf16_bits_to_f64(rw).T).astype(np.float32)
    assert np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-3)) < 1e-6


# ----------------------------------------------------------------------- top-k ----


@pytest.mark.parametrize("E,k", [(4, 2), (32, 4), (128, 4), (23, 4), (8, 8), (256, 8)])
def test_topk_matches_full_stable_sort_with_ties(E, k):
    logits = inputs.random_logits(64, E, seed=E + k, tie_frac=0.3)
    logits[0, :] = 1.5            # all equal: ids 0..k-1
    logits[1, ::2] = np.nan       # NaN ranks last
    idx, w = oracle.topk_softmax(logits, k)
    for t in range(logits.shape[0]):
        key = np.where(np.isnan(logits[t]), -np.inf, logits[t].astype(np.float64))
        nan_rank = np.isnan(logits[t]).astype(np.int64)
        order = np.lexsort((np.arange(E), -key, nan_rank))
        assert idx[t].tolist() == order[:k].tolist()
    assert idx[0].tolist() == list(range(k))
    sel = np.take_along_axis(logits.astype(np.float64), idx.astype(np.int64), 1)
    ok = ~np.isnan(sel).any(1)
    p = np.exp(sel[ok] - sel[ok, :1])
    ref = (p / p.sum(1, keepdims=True))
    assert np.allclose(w[ok], ref, rtol=1e-6, atol=0)
    assert np.allclose(w[ok].astype(np.float64).sum(1), 1.0, atol=1e-6)
    assert np.all(np.diff(w[ok], axis=1) <= 0)   # descending logits -> descending gates


# --------------------------------------------------------------------- permute ----


@pytest.mark.parametrize("T,E,k,skew", [(16, 4, 2, 0.0), (1, 32, 4, 0.0), (64, 32, 4, 0.0),
                                        (700, 128, 4, 1.1), (3, 256, 8, 0.0)])
def test_permute_matches_stable_argsort(T, E, k, skew):
    idx = inputs.random_topk_idx(T, E, k, seed=T + E, skew=skew)
    offsets, pt, ps, inv = oracle.permute(idx, E)
    flat = idx.reshape(-1)
    order = np.argsort(flat, kind="stable")
    assert np.array_equal(pt, order // k) and np.array_equal(ps, order % k)
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    assert np.array_equal(inv[order], np.arange(T * k))
    for e in range(E):  # every segment holds only expert e, tokens ascending
        seg = slice(offsets[e], offsets[e + 1])
        assert (idx[pt[seg], ps[seg]] == e).all()
        assert np.all(np.diff(pt[seg]) > 0)
