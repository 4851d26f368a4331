"""The test helpers that choose which outputs the full-size parity tests compare."""
import numpy as np

from helpers import covering_rows
from mxfp4_block_scaled_moe_b200 import inputs


def test_covering_rows_reach_every_tile():
    """The row picker itself: on a skewed routing every expert's first and last tile is
    reached by some chosen token."""
    idx = inputs.random_topk_idx(3000, 64, 4, seed=3, skew=1.1)
    rows = covering_rows(idx, 64)
    E = 64
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E)
    for e in np.nonzero(counts)[0]:
        toks = np.nonzero((idx == e).any(1))[0]        # ascending: the expert's rows in order
        last = (counts[e] - 1) // 128
        pos = {int(t): i for i, t in enumerate(toks)}
        tiles = {pos[int(t)] // 128 for t in rows if int(t) in pos}
        assert 0 in tiles and last in tiles
    assert len(rows) < 2 * E
