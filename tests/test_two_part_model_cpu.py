"""The two-part e4m3 representation of bf16 activations that the bf16 prefill GEMMs use,
checked as a model on the CPU (no GPU, no library code).

Per 32-value block of a row: s1 = floor(log2 amax) - 7, part 1 = e4m3(x / 2^s1) rounded to
nearest even; the residual r = x - part1 * 2^s1; s2 = floor(log2 max|r|) - 7, part 2 =
e4m3(r / 2^s2). Claims checked here: nothing saturates; x = part1 * 2^s1 + part2 * 2^s2
exactly wherever both parts are rounded at normal e4m3 binades; every element is within
max(2^(s2 - 10), 2^(s1 - 14)) of x (about 2^-21 of its block's maximum at most); on N(0, 1)
activations all but a tiny fraction of elements are exact. The e4m3 rounding is torch's
float8_e4m3fn cast."""
import numpy as np
import torch


def _exponent(amax: np.ndarray) -> np.ndarray:
    """floor(log2 amax) - 7 clamped to [-127, 127]; 0 for an all-zero block."""
    m, e = np.frexp(amax)                 # amax = m * 2^e, m in [0.5, 1)
    s = np.clip(e - 1 - 7, -127, 127)
    return np.where(amax > 0, s, 0).astype(np.int64)


def _e4m3(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def _split(x: np.ndarray):
    """x: (blocks, 32) float64 holding bf16 values. Returns parts and exponents."""
    s1 = _exponent(np.abs(x).max(axis=1))[:, None]
    q1 = x * np.ldexp(1.0, -s1)
    assert np.abs(q1).max() < 256.0                       # never near e4m3's 448
    p1 = _e4m3(q1)
    r = x - p1 * np.ldexp(1.0, s1)                       # exact in float64
    s2 = _exponent(np.abs(r).max(axis=1))[:, None]
    q2 = r * np.ldexp(1.0, -s2)
    assert np.abs(q2).max() < 256.0
    p2 = _e4m3(q2)
    return p1, s1, p2, s2, r


def _bf16_blocks(vals: np.ndarray) -> np.ndarray:
    return torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy().reshape(-1, 32)


def _check(x):
    p1, s1, p2, s2, r = _split(x)
    recon = p1 * np.ldexp(1.0, s1) + p2 * np.ldexp(1.0, s2)
    err = np.abs(x - recon)
    # part 2 rounds the residual: half of its smallest step, or (where part 1 was subnormal
    # and the residual keeps more than 4 bits) half an ulp of a residual below 2^(s1 - 10)
    assert (err <= np.maximum(np.ldexp(1.0, s2 - 10), np.ldexp(1.0, s1 - 14))).all()
    # exact where both parts were rounded at a normal e4m3 binade (|x / 2^s| >= 2^-6)
    q1, q2 = x * np.ldexp(1.0, -s1), r * np.ldexp(1.0, -s2)
    normal = (np.abs(q1) >= 2.0 ** -6) & ((np.abs(q2) >= 2.0 ** -6) | (r == 0))
    assert (err[normal] == 0).all()
    return err


def test_two_parts_reproduce_normal_activations_exactly():
    rng = np.random.default_rng(5)
    x = _bf16_blocks(rng.standard_normal(32 * 20000))
    err = _check(x)
    assert (err == 0).mean() > 0.999


def test_two_parts_on_wide_dynamic_range_and_outliers():
    rng = np.random.default_rng(6)
    wide = rng.standard_normal(32 * 4000) * np.ldexp(1.0, rng.integers(-30, 30, 32 * 4000))
    _check(_bf16_blocks(wide))
    out = rng.standard_normal(32 * 4000)
    out[::32] *= 1e4                                      # one outlier per block
    _check(_bf16_blocks(out))
    tiny = rng.standard_normal(32 * 100) * 1e-38           # bf16 subnormals and near them
    _check(_bf16_blocks(tiny))


def test_two_parts_of_zero_blocks_and_signed_zeros():
    x = np.zeros((3, 32))
    x[1] = -0.0
    p1, s1, p2, s2, _ = _split(x)
    assert (s1 == 0).all() and (s2 == 0).all() and (p1 == 0).all() and (p2 == 0).all()
