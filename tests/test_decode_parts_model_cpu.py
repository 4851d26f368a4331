"""The decode path's four-part e2m1 expansion of the activations, checked as a model on the
CPU (no GPU, no library code).

Part p of a value is the residual left by parts 0..p-1, rounded to the nearest e2m1 grid
point (ties to the even code) under a power-of-two scale 2^s, s the smallest exponent with
max|residual| / 2^s <= 6 over the scale's group. The decode GEMMs give every 32-value block
its own scale per part (gate_up's input x and down's input a alike). The claims checked:
over 2880-long dot products with N(0, 0.02) weights the four-part expansion changes the
result by about 1.5e-4 of the largest output, an order of magnitude inside the layer's 2e-3
bar; each part removes about three bits of the residual; and with an outlier channel (one
value 1000x the rest of its row) block scales keep the error near that bound while one
scale for the whole row would not (the other values would keep only the bits left below
the outlier's, 4e-3 of the output)."""
import numpy as np

_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _e2m1_rne(q: np.ndarray) -> np.ndarray:
    """Nearest e2m1 value of each |q| <= 6 (ties to the even code), sign kept."""
    d = np.abs(np.abs(q)[..., None] - _GRID)
    cand = d == d.min(axis=-1, keepdims=True)
    even = cand & (np.arange(8) % 2 == 0)
    code = np.where(even.any(axis=-1), even.argmax(axis=-1), cand.argmax(axis=-1))
    return np.copysign(_GRID[code], q)


def _part_exponent(m: np.ndarray) -> np.ndarray:
    """The smallest s with m / 2^s <= 6 (0 where m == 0)."""
    _, e = np.frexp(m)                    # m = f * 2^e, f in [0.5, 1)
    s = e - 3                             # m / 2^s in [4, 8)
    s = np.where(m > 6.0 * np.ldexp(1.0, s), s + 1, s)
    return np.where(m > 0, s, 0)


def _expand(v: np.ndarray, group: int, parts: int = 4) -> np.ndarray:
    """Sum of the first `parts` parts of each row of v, scales per `group` values."""
    rows, K = v.shape
    r = v.copy().reshape(rows, K // group, group)
    total = np.zeros_like(r)
    for _ in range(parts):
        s = _part_exponent(np.abs(r).max(axis=-1, keepdims=True))
        q = r * np.ldexp(1.0, -s)
        assert np.abs(q).max() <= 6.0
        c = _e2m1_rne(q) * np.ldexp(1.0, s)
        total += c
        r -= c                            # exact: c has two significant bits
    return total.reshape(rows, K)


def _rel_err(x, w, group):
    g = x @ w.T
    gp = _expand(x, group) @ w.T
    return np.abs(g - gp).max() / np.abs(g).max()


def test_four_e2m1_parts_keep_dot_products_within_3e4_of_their_size():
    rng = np.random.default_rng(9)
    K = 2880
    x = rng.standard_normal((8, K)).astype(np.float32).astype(np.float64)
    w = rng.normal(0.0, 0.02, (512, K))
    row = _rel_err(x, w, K)               # one scale per part for the whole row
    blk = _rel_err(x, w, 32)              # one scale per part per 32 values (the kernels')
    assert row < 3e-4 and blk < 2e-4 and blk < row
    assert blk < 2e-3 / 10                # well inside the layer bar


def test_block_scales_absorb_outlier_channels():
    rng = np.random.default_rng(9)
    K = 2880
    x = rng.standard_normal((8, K))
    x[:, 17] *= 1000.0                    # one channel 10^3 x the rest
    x[:, 1000] *= 300.0
    w = rng.normal(0.0, 0.02, (512, K))
    assert _rel_err(x, w, 32) < 1e-3      # block scales: inside the bar with room
    assert _rel_err(x, w, K) > 2e-3       # a row-wide scale would break it


def test_parts_converge_and_keep_small_values():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((4, 2880))
    errs = [np.abs(_expand(x, 32, p) - x).max() for p in (1, 2, 3, 4)]
    assert all(b < a / 6 for a, b in zip(errs, errs[1:]))  # every part removes ~3 bits
    assert errs[-1] < 1e-3 * np.abs(x).max()
