"""Test helpers: MXFP4-pack a synthetic layer with the oracle's quantizer and call the
oracle on it. Packed bytes made here are what both the oracle and the CUDA library
consume in parity tests, so no oracle input comes from the CUDA path."""
from __future__ import annotations

import dataclasses

import numpy as np

import oracle
from mxfp4_block_scaled_moe_b200 import inputs


@dataclasses.dataclass
class Packed:
    lay: inputs.Layer
    x: np.ndarray          # (T, H) bf16 bits
    router_w: np.ndarray   # (E, H) bf16 bits
    router_b: np.ndarray | None
    gu_blocks: np.ndarray  # (E, 2I, H/2)
    gu_scales: np.ndarray  # (E, 2I, H/32)
    gu_bias: np.ndarray    # (E, 2I) fp32
    d_blocks: np.ndarray   # (E, H, I/2)
    d_scales: np.ndarray   # (E, H, I/32)
    d_bias: np.ndarray     # (E, H) fp32

    @property
    def weights(self):
        return (self.gu_blocks, self.gu_scales, self.gu_bias, self.d_blocks, self.d_scales,
                self.d_bias)

    def oracle_forward(self, act_scale=None, dense=False, rows=None):
        x = self.x if rows is None else self.x[rows]
        return oracle.moe_forward(x, self.router_w, self.router_b, *self.weights, self.lay.k,
                                  act_scale=act_scale, dense=dense)

    def oracle_calibrate(self, x_bits):
        return oracle.calibrate(x_bits, self.router_w, self.router_b, *self.weights, self.lay.k)


def pack(lay: inputs.Layer) -> Packed:
    E, H, I = lay.E, lay.H, lay.I
    gu_b = np.empty((E, 2 * I, H // 2), np.uint8)
    gu_s = np.empty((E, 2 * I, H // 32), np.uint8)
    d_b = np.empty((E, H, I // 2), np.uint8)
    d_s = np.empty((E, H, I // 32), np.uint8)
    for e in range(E):
        gu_b[e], gu_s[e] = oracle.quantize(lay.gate_up(e).cpu().numpy())
        d_b[e], d_s[e] = oracle.quantize(lay.down(e).cpu().numpy())
    rb = None if lay.router_b is None else inputs.bits(lay.router_b)
    return Packed(lay, inputs.bits(lay.x), inputs.bits(lay.router_w), rb, gu_b, gu_s,
                  lay.gu_bias.cpu().numpy(), d_b, d_s, lay.d_bias.cpu().numpy())


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def output_tolerance_ok(out_bits: np.ndarray, ref_acc: np.ndarray, rel: float = 2e-3):
    """The layer-output bar: a bf16 output may differ from the oracle's fp32 accumulator
    by rel * max|ref| (fp32 arithmetic, accumulation order) plus half a bf16 ulp of the
    reference element (the single bf16 rounding of the output).

    Returns (ok, max|delta|/max|ref|, worst excess)."""
    got = bf16_bits_to_f32(out_bits).astype(np.float64)
    ref = ref_acc.astype(np.float64)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64) * 2.0 ** 16
    bound = rel * scale + 0.5 * ulp
    err = np.abs(got - ref)
    excess = float(np.max(err - bound)) if ref.size else 0.0
    return bool(np.all(err <= bound)), float(np.max(err) / scale) if scale else 0.0, excess


# ------------------------------------------------------------- row selection ----

def covering_rows(idx: np.ndarray, E: int, tile: int = 128, extra=()):
    """Tokens whose outputs, compared with the oracle, reach every expert's first and last
    row tile of the grouped GEMMs (an expert's routed rows are its tokens in ascending
    order, cut into tiles of `tile` rows; an expert with 1-3 rows is one partial tile).
    Greedy: for each target tile not yet reached, the token of that tile that reaches the
    most targets still open. Returns the sorted token ids (plus `extra`)."""
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")             # pairs grouped by expert, ascending t
    counts = np.bincount(flat, minlength=E)
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]])
    rank = np.empty_like(flat)
    rank[order] = np.arange(flat.size) - starts[flat[order]]
    tile_of = (rank // tile).reshape(T, k)              # tile of each (token, slot) in its expert
    open_ = set()
    for e in np.nonzero(counts)[0]:
        open_.add((int(e), 0))
        open_.add((int(e), int((counts[e] - 1) // tile)))
    members = {}                                        # target tile -> its tokens
    for t in range(T):
        for j in range(k):
            key = (int(idx[t, j]), int(tile_of[t, j]))
            if key in open_:
                members.setdefault(key, []).append(t)
    chosen = set(int(r) for r in extra)
    for t in chosen:
        for j in range(k):
            open_.discard((int(idx[t, j]), int(tile_of[t, j])))
    for key in sorted(open_):
        if key not in open_:
            continue
        best = max(members[key], key=lambda t: sum((int(idx[t, j]), int(tile_of[t, j])) in open_
                                                   for j in range(k)))
        chosen.add(best)
        for j in range(k):
            open_.discard((int(idx[best, j]), int(tile_of[best, j])))
    assert not open_
    return np.array(sorted(chosen), dtype=np.int64)


# ------------------------------------------------------------------ GPU helpers ----

def to_device(p: Packed, device="cuda"):
    """The packed layer as torch tensors on the GPU (bf16 bits become torch.bfloat16)."""
    import torch
    u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    bf = lambda a: None if a is None else inputs.from_bits(a, device)
    return dict(x=bf(p.x), router_w=bf(p.router_w), router_b=bf(p.router_b),
                gu_blocks=u8(p.gu_blocks), gu_scales=u8(p.gu_scales), gu_bias=f32(p.gu_bias),
                d_blocks=u8(p.d_blocks), d_scales=u8(p.d_scales), d_bias=f32(p.d_bias))


def gpu_bits(t) -> np.ndarray:
    """bf16 CUDA tensor -> numpy uint16 bits."""
    return inputs.bits(t)


# ------------------------------------------------- exhaustive round-to-grid blocks ----

GRID_ANCHOR = 4.0   # a block holding 4.0 and values below 8 has amax in [4, 8): scale 2^0


class AnchoredBlocks:
    """fp32 bit patterns [lo, hi) (with the sign bit when ``negative``) as (nb, 32) blocks:
    column 0 is the anchor 4.0, columns 1..31 the values in pattern order (the last block
    padded with zeros). With patterns below 8.0 every block's scale exponent is 0, so each
    value's nibble is the round-to-grid of the value itself. The storage for chunks of up
    to ``step`` patterns is allocated once and refilled by ``fill``."""

    def __init__(self, step: int):
        self.idx = np.arange(step, dtype=np.uint32)
        nb = -(-step // 31)
        self.body = np.zeros(nb * 31, np.uint32)
        self.buf = np.empty((nb, 32), np.uint32)
        self.buf[:, 0] = np.float32(GRID_ANCHOR).view(np.uint32)

    def fill(self, lo: int, hi: int, negative: bool) -> np.ndarray:
        n = hi - lo
        nb = -(-n // 31)
        body = self.body[: nb * 31]
        np.add(self.idx[:n], np.uint32(lo), out=body[:n])
        if negative:
            np.bitwise_or(body[:n], np.uint32(0x80000000), out=body[:n])
        body[n:] = 0
        self.buf[:nb, 1:] = body.reshape(nb, 31)
        return self.buf[:nb].view(np.float32)


def anchored_blocks(lo: int, hi: int, negative: bool) -> np.ndarray:
    """AnchoredBlocks for one range, as a fresh array."""
    return AnchoredBlocks(hi - lo).fill(lo, hi, negative).copy()


def nibble_codes(blocks_packed: np.ndarray) -> np.ndarray:
    """(nb, 16) packed bytes -> (nb, 32) nibbles, element 2j in the low nibble of byte j."""
    return np.stack([blocks_packed & 15, blocks_packed >> 4], axis=-1).reshape(blocks_packed.shape[0], 32)
