"""GPU parity of the standalone MXFP4 codec kernels against the oracle: bit-exact.

Page "quantization_mxfp4" (KerasFormers), Primitives: dequantize is a bit-exact decode
(max |delta| 0.0), quantize_to_mxfp4 its inverse on the lattice. Workload of the codec
sweep: one 120B-shaped expert set, gate_up (128, 5760, 2880) and down (128, 2880, 2880),
fp32 N(0, 0.02) with 1% outliers x8, unpacked to bf16 and fp32.
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


def test_dequant_exhaustive_matches_oracle(B):
    nib = np.tile(np.arange(16, dtype=np.uint8), 2)
    row = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
    blocks = np.tile(row, (256, 1))
    scales = np.arange(256, dtype=np.uint8)[:, None]
    gb, gs = torch.from_numpy(blocks).cuda(), torch.from_numpy(scales).cuda()
    f32 = B.mxfp4_dequantize(gb, gs, torch.float32).cpu().numpy()
    b16 = inputs.bits(B.mxfp4_dequantize(gb, gs, torch.bfloat16))
    assert np.array_equal(f32.view(np.uint32), oracle.dequantize(blocks, scales, out="f32").view(np.uint32))
    assert np.array_equal(b16, oracle.dequantize(blocks, scales, out="bf16"))


def test_dequant_random_bytes_matches_oracle(B):
    rng = np.random.default_rng(0)
    rows, K = 777, 2880
    blocks = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    scales = rng.integers(0, 256, size=(rows, K // 32), dtype=np.uint8)
    gb, gs = torch.from_numpy(blocks).cuda(), torch.from_numpy(scales).cuda()
    f32 = B.mxfp4_dequantize(gb, gs, torch.float32).cpu().numpy()
    b16 = inputs.bits(B.mxfp4_dequantize(gb, gs, torch.bfloat16))
    assert np.array_equal(f32.view(np.uint32), oracle.dequantize(blocks, scales, out="f32").view(np.uint32))
    assert np.array_equal(b16, oracle.dequantize(blocks, scales, out="bf16"))


def _quant_cases():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((517, 352)) * 0.02
    x *= np.where(rng.random(x.shape) < 0.01, 8.0, 1.0)
    x[3] *= 1e-39                   # subnormal inputs, clamped scale
    x[5] *= 2.0 ** 120              # large block
    x[7, :64] = 0.0                 # zero blocks
    x[8, :32] = -0.0
    x[9, :] = np.float32(np.finfo(np.float32).max) * np.sign(x[9])
    # every grid midpoint with the block exponent pinned to 0 by a 4
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 7.99])
    x[10, :] = 0
    x[10, 0] = 4.0
    x[10, 1:1 + 2 * len(mids)] = np.concatenate([mids, -mids])
    return x.astype(np.float32)


def test_quantize_matches_oracle_edge_cases(B):
    x = _quant_cases()
    gblk, gsc = B.mxfp4_quantize(torch.from_numpy(x).cuda())
    oblk, osc = oracle.quantize(x)
    assert np.array_equal(gsc.cpu().numpy(), osc)
    assert np.array_equal(gblk.cpu().numpy(), oblk)


def test_quantize_roundtrip_on_lattice(B):
    rng = np.random.default_rng(2)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    g = grid[rng.integers(0, 8, size=(2000, 64))] * rng.choice([-1.0, 1.0], size=(2000, 64))
    g[:, 0] = 6.0
    g[:, 32] = -4.0
    e = rng.integers(-127, 126, size=(2000, 1))
    x = np.ldexp(g, e).astype(np.float32)
    xt = torch.from_numpy(x).cuda()
    back = B.mxfp4_dequantize(*B.mxfp4_quantize(xt), torch.float32)
    assert torch.equal(back.view(torch.int32), xt.view(torch.int32))


@pytest.mark.parametrize("K", [31, 48, 2880 + 16])
def test_codec_rejects_K_not_multiple_of_32(B, K):
    w = torch.zeros(4, K, device="cuda")
    with pytest.raises(B.MxmoeError) as e:
        B.mxfp4_quantize(w, blocks=torch.empty(4, K, dtype=torch.uint8, device="cuda"),
                         scales=torch.empty(4, K, dtype=torch.uint8, device="cuda"))
    assert e.value.rc == B.EALIGN


def test_codec_empty_and_bad_dtype(B):
    b = torch.empty(0, 16, dtype=torch.uint8, device="cuda")
    s = torch.empty(0, 1, dtype=torch.uint8, device="cuda")
    assert B.mxfp4_dequantize(b, s).shape == (0, 32)
    L = B.lib()
    rc = L.mxfp4_dequantize(None, None, 1, 32, None, 7, None)
    assert rc == B.EUNSUPPORTED


def test_codec_sweep_full_size_sampled(B):
    """The full 120B-shaped expert set: quantize on the GPU, compare sampled rows with
    the oracle bit for bit; dequantize random packed bytes of the same shape to bf16 and
    fp32 and compare sampled rows."""
    torch.cuda.empty_cache()
    rng = np.random.default_rng(3)
    for tag, rows, K in (("gate_up", 128 * 5760, 2880), ("down", 128 * 2880, 2880)):
        w = inputs.codec_tensor(rows, K, seed=0, tag=tag, device="cuda")
        blk, sc = B.mxfp4_quantize(w)
        sample = np.sort(rng.choice(rows, size=96, replace=False))
        sample[-1] = rows - 1
        ws = w[torch.from_numpy(sample).cuda()].cpu().numpy()
        oblk, osc = oracle.quantize(ws)
        idx = torch.from_numpy(sample).cuda()
        assert np.array_equal(sc[idx].cpu().numpy(), osc)
        assert np.array_equal(blk[idx].cpu().numpy(), oblk)
        del w
        # dequantize: random packed bytes (scales in a realistic band plus extremes)
        rb = torch.randint(0, 256, (rows, K // 2), dtype=torch.uint8, device="cuda")
        rs = torch.randint(100, 140, (rows, K // 32), dtype=torch.uint8, device="cuda")
        rs[:7] = torch.randint(0, 256, (7, K // 32), dtype=torch.uint8, device="cuda")
        sample[:7] = np.arange(7)
        idx = torch.from_numpy(sample).cuda()
        for dt in (torch.bfloat16, torch.float32):
            out = B.mxfp4_dequantize(rb, rs, dt)
            got = out[idx]
            ob, os_ = rb[idx].cpu().numpy(), rs[idx].cpu().numpy()
            if dt == torch.float32:
                exp = oracle.dequantize(ob, os_, out="f32")
                assert np.array_equal(got.cpu().numpy().view(np.uint32), exp.view(np.uint32))
            else:
                assert np.array_equal(inputs.bits(got), oracle.dequantize(ob, os_, out="bf16"))
            del out
        del rb, rs, blk, sc
        torch.cuda.empty_cache()


def test_quantize_round_to_grid_exhaustive_fp32(B):
    """Every fp32 value in (-8, 8), both signs, through the GPU quantizer at scale 2^0
    (blocks anchored by 4.0): nibbles bit-identical to the oracle's. The oracle's own
    rounding is pinned against brute force in tests/test_oracle_codec.py."""
    import helpers
    top = int(np.float32(8.0).view(np.uint32))
    step = 1 << 26
    buf = helpers.AnchoredBlocks(step)
    for negative in (False, True):
        for lo in range(0, top, step):
            blocks = buf.fill(lo, min(top, lo + step), negative)
            oblk, osc = oracle.quantize(blocks)
            gblk, gsc = B.mxfp4_quantize(torch.from_numpy(blocks).cuda())
            assert np.array_equal(gsc.cpu().numpy(), osc), (negative, lo)
            assert np.array_equal(gblk.cpu().numpy(), oblk), (negative, lo)
