"""Pins for the oracle's MXFP4 codec against closed forms, invariants and brute force.

Page: "quantization_mxfp4" (KerasFormers), sections "Primitives" (dequantize is
codebook[nibble] * 2^(e8m0 - 127), max |delta| 0.0 against the reference decoder;
quantize picks floor(log2(amax)) - 2 and rounds to the nearest FP4 grid point, a
value-exact inverse on the lattice) and "As a quantize_model scheme" (contracting
dimension a multiple of 32, else a clear error).
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

# ---------------------------------------------------------------- closed forms ----


def e2m1_closed_form(n: int):
    """E2M1 from its bit fields: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.

    Returns (sign, exact magnitude)."""
    sign = -1.0 if n & 8 else 1.0
    ex, man = (n >> 1) & 3, n & 1
    if ex == 0:
        mag = Fraction(man, 2)
    else:
        mag = Fraction(2) ** (ex - 1) * (1 + Fraction(man, 2))
    return sign, mag


def test_dequant_exhaustive_16_nibbles_x_256_scales():
    # one row per scale byte; 32 elements = nibbles 0..15 twice
    nib = np.tile(np.arange(16, dtype=np.uint8), 2)
    row = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
    blocks = np.tile(row, (256, 1))
    scales = np.arange(256, dtype=np.uint8)[:, None]
    got32 = oracle.dequantize(blocks, scales, out="f32")
    got16 = oracle.dequantize(blocks, scales, out="bf16")
    exp64 = np.empty((256, 32), np.float64)
    for s in range(256):
        for i in range(32):
            sign, mag = e2m1_closed_form(int(nib[i]))
            exp64[s, i] = math.copysign(float(mag * Fraction(2) ** (s - 127)), sign)
    with np.errstate(over="ignore"):
        exp32 = exp64.astype(np.float32)
    exp16 = torch.from_numpy(exp64).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got32.view(np.uint32), exp32.view(np.uint32))
    assert np.array_equal(got16, exp16)
    # spot checks that the table covers what it should: subnormals and overflow
    assert got32[0, 1] == np.float32(2.0 ** -128)          # 0.5 * 2^-127, fp32 subnormal
    assert np.isinf(got32[255, 2]) and got32[255, 1] == np.float32(2.0 ** 127)


def test_dequant_rejects_K_not_multiple_of_32():
    with pytest.raises(oracle.OracleError) as e:
        oracle.dequantize(np.zeros((2, 8), np.uint8), np.zeros((2, 1), np.uint8), K=16)
    assert e.value.rc == oracle.EALIGN


@pytest.mark.parametrize("K", [31, 33, 2880 + 16])
def test_quantize_rejects_K_not_multiple_of_32(K):
    with pytest.raises(oracle.OracleError) as e:
        oracle.quantize(np.ones((3, K), np.float32))
    assert e.value.rc == oracle.EALIGN


# ------------------------------------------------------------------ invariants ----

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def test_roundtrip_on_the_lattice():
    """dequantize(quantize(x)) == x for every block g_i * 2^e with g_i on the grid."""
    rng = np.random.default_rng(0)
    rows = 4000
    e = rng.integers(-127, 126, size=rows)
    g = GRID[rng.integers(0, 8, size=(rows, 32))] * rng.choice([-1.0, 1.0], size=(rows, 32))
    # half the rows carry a value of magnitude 4 or 6 (block exponent == e); the other
    # half keep whatever the draw gave, restricted to exponents that cannot clamp
    big = rng.random(rows) < 0.5
    g[big, rng.integers(0, 32, size=big.sum())] = rng.choice([4.0, 6.0, -4.0, -6.0], size=big.sum())
    e = np.where(big, e, np.maximum(e, -120))
    x = np.ldexp(g, e[:, None]).astype(np.float32)
    assert np.array_equal(x.astype(np.float64), np.ldexp(g, e[:, None]))  # exact inputs
    blocks, scales = oracle.quantize(x)
    back = oracle.dequantize(blocks, scales, out="f32")
    assert np.array_equal(back.view(np.uint32), x.view(np.uint32))


def test_negative_zero_and_zero_block():
    x = np.zeros((2, 32), np.float32)
    x[1, :] = -0.0
    blocks, scales = oracle.quantize(x)
    assert scales.tolist() == [[0], [0]]
    assert (blocks[0] == 0).all() and (blocks[1] == 0x88).all()
    back = oracle.dequantize(blocks, scales, out="f32")
    assert np.array_equal(back.view(np.uint32), x.view(np.uint32))


def test_packing_even_element_in_low_nibble():
    x = np.zeros((1, 32), np.float32)
    x[0, 0], x[0, 1] = 4.0, 1.0      # block exponent 0 -> codes 6 and 2
    blocks, scales = oracle.quantize(x)
    assert scales[0, 0] == 127 and blocks[0, 0] == 0x26


# ------------------------------------------------------------------ brute force ----


def floor_log2(a: float) -> int:
    m, ex = math.frexp(a)   # a = m * 2^ex, m in [0.5, 1)
    return ex - 1


def brute_code(r: Fraction) -> int:
    """Nearest E2M1 magnitude code to r >= 0; ties to the even code; saturate at 6."""
    if r >= 6:
        return 7
    best, bestd = None, None
    for c in range(8):
        d = abs(r - Fraction(GRID[c]))
        if best is None or d < bestd or (d == bestd and c % 2 == 0):
            best, bestd = c, d
    return best


def brute_quantize(x: np.ndarray):
    rows, K = x.shape
    blocks = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 32), np.uint8)
    for r in range(rows):
        for b in range(K // 32):
            blk = [float(v) for v in x[r, 32 * b:32 * b + 32]]
            amax = max(abs(v) for v in blk)
            e = -127 if amax == 0 else min(127, max(-127, floor_log2(amax) - 2))
            scales[r, b] = e + 127
            for i, v in enumerate(blk):
                code = brute_code(Fraction(abs(v)) / Fraction(2) ** e)
                nib = code | (8 if math.copysign(1.0, v) < 0 else 0)
                k = 32 * b + i
                blocks[r, k // 2] |= nib << (4 * (k % 2))
    return blocks, scales


def test_quantize_matches_brute_force_random():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((48, 64)) * 0.02
    x *= np.where(rng.random(x.shape) < 0.05, 8.0, 1.0)
    x[3] *= 1e-39        # fp32 subnormal inputs -> clamped scale
    x[5] *= 2.0 ** 120   # huge block
    x[7, :32] = 0.0
    x = x.astype(np.float32)
    got = oracle.quantize(x)
    exp = brute_quantize(x)
    assert np.array_equal(got[1], exp[1])
    assert np.array_equal(got[0], exp[0])


def test_quantize_ties_and_saturation():
    """Every midpoint between grid points, with block exponent fixed to 0 by a 4."""
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    near = [v + d for v in mids for d in (-2.0 ** -20, 2.0 ** -20)]
    sat = [6.0, 6.5, 7.0, 7.99, 4.0, 0.0]
    vals = mids + near + sat
    vals = vals + [-v for v in vals]
    n = len(vals)
    nblk = (n + 30) // 31
    x = np.zeros((nblk, 32), np.float32)
    for i, v in enumerate(vals):
        x[i // 31, 1 + i % 31] = v
    x[:, 0] = 4.0
    got = oracle.quantize(x)
    exp = brute_quantize(x)
    assert (got[1] == 127).all()
    assert np.array_equal(got[0], exp[0])
    # the decoded values of the exact midpoints go to the even neighbour
    back = oracle.dequantize(*got, out="f32")
    flat = {vals[i]: back[i // 31, 1 + i % 31] for i in range(n)}
    assert [flat[m] for m in mids] == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    assert flat[6.5] == 6.0 and flat[7.99] == 6.0 and flat[-7.0] == -6.0


@pytest.mark.parametrize("amax", [4.0, float(np.nextafter(np.float32(4.0), np.float32(0))), 8.0,
                                  2.0 ** -130, 2.0 ** -149, 3 * 2.0 ** 100,
                                  float(np.finfo(np.float32).max), 1.0, 0.02])
def test_scale_byte_selection(amax):
    x = np.zeros((1, 32), np.float32)
    x[0, 7] = amax
    x[0, 3] = amax / 3
    blocks, scales = oracle.quantize(x)
    a = float(np.float32(amax))
    exp = min(127, max(-127, floor_log2(a) - 2)) + 127
    assert scales[0, 0] == exp


def test_quantize_then_dequantize_error_bound():
    """Away from saturation, each element's FP4 rounding error is at most half the grid
    spacing at its magnitude: 0.25, 0.5 or 1 (times 2^e) below 2, 4 and 6."""
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((256, 128)) * 0.02).astype(np.float32)
    blocks, scales = oracle.quantize(x)
    back = oracle.dequantize(blocks, scales, out="f32").astype(np.float64)
    e = np.repeat(scales.astype(np.int64) - 127, 32, axis=1)
    r = np.abs(x.astype(np.float64)) / np.ldexp(1.0, e)
    step = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0))
    err = np.abs(back - x) / np.ldexp(1.0, e)
    unsat = r <= 6
    assert (err[unsat] <= step[unsat]).all()


# ------------------------------------------- round-to-grid against brute force ------

_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _brute_force_codes(vals: np.ndarray) -> np.ndarray:
    """E2M1 code of each fp32 value at scale 2^0 by exhaustive search: the grid point at
    the least distance (ties to the point with the even code), sign bit from the value's
    own sign bit (so -0 and tiny negatives keep it)."""
    r = np.abs(vals.astype(np.float64))
    d = np.abs(r[:, None] - _GRID[None, :])
    cand = d == d.min(axis=1, keepdims=True)
    even = cand & (np.arange(8) % 2 == 0)
    mag = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1)).astype(np.uint8)
    return mag | ((vals.view(np.uint32) >> 31).astype(np.uint8) << 3)


def _pattern_ranges():
    """fp32 bit-pattern ranges below 8.0 that hold every decision of the rounding: 2^18
    patterns on each side of each midpoint between grid points and of each grid point,
    every 251st pattern of the whole range, and the subnormals' first 2^16."""
    f = lambda x: int(np.float32(x).view(np.uint32))
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    ranges = [(f(m) - (1 << 18), f(m) + (1 << 18)) for m in mids]
    ranges += [(max(f(g) - (1 << 18), 0), f(g) + (1 << 18)) for g in _GRID[1:]]
    ranges += [(0, 1 << 16), (f(8.0) - (1 << 18), f(8.0))]
    return ranges


@pytest.mark.parametrize("negative", [False, True])
def test_round_to_grid_matches_brute_force(negative):
    import helpers
    stride = np.arange(0, int(np.float32(8.0).view(np.uint32)), 251, dtype=np.uint32)
    chunks = [helpers.anchored_blocks(lo, hi, negative) for lo, hi in _pattern_ranges()]
    s = stride | np.uint32(0x80000000) if negative else stride
    body = np.zeros(-(-s.size // 31) * 31, np.float32)
    body[: s.size] = s.view(np.float32)
    sb = np.empty((body.size // 31, 32), np.float32)
    sb[:, 0], sb[:, 1:] = helpers.GRID_ANCHOR, body.reshape(-1, 31)
    chunks.append(sb)
    for blocks in chunks:
        packed, scales = oracle.quantize(blocks)
        assert (scales == 127).all()                       # amax in [4, 8): exponent 0
        codes = helpers.nibble_codes(packed)
        assert (codes[:, 0] == 6).all()                    # the anchor 4.0
        assert np.array_equal(codes[:, 1:], _brute_force_codes(blocks[:, 1:].reshape(-1)).reshape(-1, 31))
