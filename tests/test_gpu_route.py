"""GPU parity of routing: top-k (bit-exact on identical logits), router logits (fp32
tolerance), the permutation (bit-exact) and the FP8 activation cast (bit-exact).

GPT-OSS routing: 128/32/23 experts, top-4 ("gpt-oss-120b-mxfp4-fp8attn-v2", Model
Details; "amd/gpt-oss-20b-BF16-w8a8-llmcompressor", Quantization; "xpuenabler/gpt-oss-
15.5b-23E-nf4-GPU", Notes); router kept in bf16; FP8 E4M3 per-tensor activations
("amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8", Quantization schemes).
"""
import numpy as np
import pytest
import torch

import oracle
from mxfp4_block_scaled_moe_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from mxfp4_block_scaled_moe_b200 import binding
    return binding


@pytest.mark.parametrize("T,E,k", [(1, 32, 4), (64, 32, 4), (333, 128, 4), (50, 23, 4),
                                   (17, 4, 2), (40, 256, 8), (9, 8, 8), (5, 1, 1)])
def test_topk_from_identical_logits_bit_exact(B, T, E, k):
    logits = inputs.random_logits(T, E, seed=T * 7 + E, tie_frac=0.3)
    logits[0, :] = 0.5
    if T > 3:
        logits[3, ::3] = np.nan
    gi, gw = B.moe_topk_from_logits(torch.from_numpy(logits).cuda(), k)
    oi, ow = oracle.topk_softmax(logits, k)
    assert np.array_equal(gi.cpu().numpy(), oi)
    ok = ~np.isnan(np.take_along_axis(logits, oi.astype(np.int64), 1)).any(1)
    gw = gw.cpu().numpy()
    assert np.allclose(gw[ok], ow[ok], rtol=2e-6, atol=1e-7)


# T <= 32: the GEMV router; T > 32 with H % 64 == 0, E % 8 == 0, E <= 256: the tensor-core
# router, split over K ranges (T = 129 ragged second tile, E = 256 the widest MMA, H = 64 a
# single K range, T = 4096 the prefill shape); otherwise the mma.sync router (E = 23,
# H = 2912 not a multiple of 64).
@pytest.mark.parametrize("T,E,H,bias", [(1, 32, 2880, False), (8, 32, 2880, False),
                                        (64, 32, 2880, False), (200, 128, 2880, False),
                                        (37, 23, 2880, True), (5, 4, 256, True),
                                        (129, 256, 2880, True), (300, 64, 64, True),
                                        (150, 128, 2912, False), (4096, 128, 2880, True)])
def test_router_logits_and_indices(B, T, E, H, bias):
    lay = inputs.small_layer(E=E, k=4 if E >= 4 else E, T=T, H=H, I=32, seed=T + E,
                             router_std=1.0 / np.sqrt(H), router_bias=bias, device="cuda")
    k = lay.k
    gi, gw, gl = B.moe_route_topk(lay.x, lay.router_w, lay.router_b, k, with_logits=True)
    xb, wb = inputs.bits(lay.x), inputs.bits(lay.router_w)
    bb = None if lay.router_b is None else inputs.bits(lay.router_b)
    ol = oracle.router_logits(xb, wb, bb)
    gl = gl.cpu().numpy()
    # fp32 accumulation vs a double sum: bounded by sum |x w| * 2^-14 (a few hundred fp32 adds)
    xf = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    wf = (wb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    mag = np.abs(xf) @ np.abs(wf).T
    assert np.all(np.abs(gl - ol) <= mag * 2.0 ** -14 + 1e-30)
    # indices: identical where the k-th / (k+1)-th gap is not a near-tie
    oi, ow = oracle.topk_softmax(ol, k)
    srt = -np.sort(-ol, axis=1)
    gap = srt[:, k - 1] - srt[:, k] if E > k else np.full(T, np.inf)
    clear = gap > 1e-5 * np.abs(ol).max()
    gi = gi.cpu().numpy()
    assert clear.mean() > 0.9
    assert np.array_equal(gi[clear], oi[clear])
    # and the GPU top-k is exactly the top-k of its own logits
    si, _ = oracle.topk_softmax(gl, k)
    assert np.array_equal(gi, si)


@pytest.mark.parametrize("T,E,k,skew", [(1, 32, 4, 0.0), (8, 32, 4, 0.0), (64, 32, 4, 0.0),
                                        (1000, 128, 4, 0.0), (1025, 128, 4, 0.0),
                                        (4096, 128, 4, 0.0), (16384, 128, 4, 1.1),
                                        (3, 256, 8, 0.0), (513, 23, 4, 2.0), (129, 32, 4, 0.0),
                                        (40000, 128, 4, 0.0), (65536, 256, 4, 0.5)])
def test_permute_bit_exact(B, T, E, k, skew):
    idx = inputs.random_topk_idx(T, E, k, seed=T + E, skew=skew) if T <= 4096 else None
    if idx is None:   # large case: draw on the host with numpy, vectorised
        rng = np.random.default_rng(T)
        p = np.arange(1, E + 1) ** -skew
        p /= p.sum()
        keys = rng.random((T, E)) ** (1.0 / p)[None, :]
        idx = np.argsort(-keys, axis=1)[:, :k].astype(np.int32)
    go, gt, gs = B.moe_permute(torch.from_numpy(idx).cuda(), E)
    oo, ot, os_, _ = oracle.permute(idx, E)
    assert np.array_equal(go.cpu().numpy(), oo)
    assert np.array_equal(gt.cpu().numpy(), ot)
    assert np.array_equal(gs.cpu().numpy(), os_)


def test_permute_flags_bad_expert_id(B):
    idx = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device="cuda")
    B.moe_permute(idx, 4)
    with pytest.raises(B.MxmoeError) as e:
        B.mxmoe_check()
    assert e.value.rc == B.EDEVICE
    B.mxmoe_check()   # cleared


def test_permute_flags_bad_expert_id_in_a_late_chunk(B):
    # 3000 tokens x 4 = 12000 pairs span many chunks; only the last pair is bad
    idx = torch.from_numpy(inputs.random_topk_idx(3000, 64, 4, seed=5)).cuda()
    idx[-1, -1] = 64
    B.moe_permute(idx, 64)
    with pytest.raises(B.MxmoeError) as e:
        B.mxmoe_check()
    assert e.value.rc == B.EDEVICE
    B.mxmoe_check()   # cleared


def test_permute_empty(B):
    go, gt, gs = B.moe_permute(torch.empty(0, 4, dtype=torch.int32, device="cuda"), 8)
    assert go.cpu().tolist() == [0] * 9


@pytest.mark.parametrize("s", [0.0123, 1.0 / 448, 3.75])
def test_fp8_activation_cast_bit_exact(B, s):
    x = inputs.normal((4097, 96), 2.0, seed=5, tag="fp8x", device="cuda", dtype=torch.bfloat16)
    x[0, :8] = torch.tensor([0.0, -0.0, 1e-30, -1e-30, 3e4, -3e4, float("inf"), 448.0 * s])
    q = B.moe_fp8_quantize(x, s).cpu().numpy()
    xf = x.float().cpu().numpy()
    assert np.array_equal(q, oracle.fp8_quantize(xf, np.float32(s)))
