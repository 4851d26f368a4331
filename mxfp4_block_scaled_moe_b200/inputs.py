"""Seeded synthetic inputs for the MXFP4 MoE layer (shared by tests, smoke and bench).

This module only draws random numbers in the shapes and distributions of the
workloads; it holds none of the layer's arithmetic (no quantization, routing, GEMM or
activation). Weights come out as fp32; turning them into MXFP4 is the caller's job
(the oracle in tests, the library's own quantizer in the benchmark).

Every tensor has its own generator seeded from (seed, tensor tag[, expert]), so a tensor
does not depend on which other tensors were drawn before it, and one expert can be
regenerated alone. Draws happen on ``device`` (torch's Philox generator on CUDA, its
CPU generator on CPU); the two devices give different streams, so a test draws every
input of one case on one device.

Workloads (hidden H and intermediate I are 2880 in the GPT-OSS shapes):
  tiny     E=4  k=2 H=256  I=256  T=16   x~N(0,1), Wr~N(0,0.02), br=0
  decode   E=32 k=4 H=I=2880 T in {1,8,64}; Wr~N(0,0.02)
  prefill  E=128 k=4 H=I=2880 T=4096; Wr~N(0,1/sqrt(H)) so logits ~ N(0,1)
  zipf     E=128 k=4 H=I=2880 T=16384; Wr~N(0,0.02), br[e] = ln p_pi(e), p_r ~ r^-1.1
Expert weights ~N(0,0.02) fp32, expert biases ~N(0,0.01) fp32. The standalone codec
sweep uses N(0,0.02) with a Bernoulli(0.01) mask of outliers scaled by 8.
"""
from __future__ import annotations

import dataclasses
import math
import zlib

import numpy as np
import torch


def _seed(seed: int, tag: str, sub: int = 0) -> int:
    h = zlib.crc32(tag.encode()) & 0xFFFF
    return (int(seed) * 1_000_003 + h * 8191 + int(sub) * 131) & 0x7FFF_FFFF_FFFF


def _gen(device, seed, tag, sub=0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(seed, tag, sub))
    return g


def normal(shape, std, seed, tag, sub=0, device="cpu", dtype=torch.float32) -> torch.Tensor:
    """N(0, std^2) samples, drawn in fp32 and cast once to ``dtype``."""
    g = _gen(device, seed, tag, sub)
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray, device="cpu") -> torch.Tensor:
    """numpy uint16 bit patterns -> bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


@dataclasses.dataclass
class Layer:
    """One synthetic MoE layer. Weights are fp32 (E, 2I, H) / (E, H, I)."""
    name: str
    E: int
    k: int
    T: int
    H: int
    I: int
    seed: int
    device: str
    x: torch.Tensor          # (T, H) bf16
    router_w: torch.Tensor   # (E, H) bf16
    router_b: torch.Tensor | None  # (E,) bf16
    gu_bias: torch.Tensor    # (E, 2I) fp32
    d_bias: torch.Tensor     # (E, H) fp32
    w_std: float = 0.02

    def gate_up(self, e: int) -> torch.Tensor:
        """fp32 gate_up_proj of expert e, (2I, H): rows [0,I) gate, [I,2I) up."""
        return normal((2 * self.I, self.H), self.w_std, self.seed, "gate_up", e, self.device)

    def down(self, e: int) -> torch.Tensor:
        """fp32 down_proj of expert e, (H, I)."""
        return normal((self.H, self.I), self.w_std, self.seed, "down", e, self.device)


def _layer(name, E, k, T, H, I, seed, device, router_std, router_bias=None) -> Layer:
    x = normal((T, H), 1.0, seed, "x", 0, device, torch.bfloat16)
    rw = normal((E, H), router_std, seed, "router_w", 0, device, torch.bfloat16)
    gb = normal((E, 2 * I), 0.01, seed, "gu_bias", 0, device)
    db = normal((E, H), 0.01, seed, "d_bias", 0, device)
    return Layer(name, E, k, T, H, I, seed, device, x, rw, router_bias, gb, db)


def tiny_layer(seed: int = 0, device="cpu", T: int = 16) -> Layer:
    """E=4, top-2, H=I=256, T=16; router bias present and zero."""
    rb = torch.zeros(4, dtype=torch.bfloat16, device=device)
    return _layer("tiny", 4, 2, T, 256, 256, seed, device, 0.02, rb)


def small_layer(E=8, k=2, T=40, H=320, I=192, seed=0, device="cpu", router_std=0.02,
                router_bias=False) -> Layer:
    """Generic small layer for parity cases that span several tiles and ragged tails."""
    rb = normal((E,), 0.5, seed, "router_b", 0, device, torch.bfloat16) if router_bias else None
    return _layer(f"small_E{E}_k{k}_T{T}_H{H}_I{I}", E, k, T, H, I, seed, device, router_std, rb)


def decode_layer(T: int, E: int = 32, seed: int = 0, device="cpu") -> Layer:
    """20B-shaped decode layer: E=32 (or 23), top-4, H=I=2880, router ~N(0,0.02)."""
    return _layer(f"decode_E{E}_T{T}", E, 4, T, 2880, 2880, seed, device, 0.02, None)


def prefill_layer(T: int = 4096, E: int = 128, seed: int = 0, device="cpu") -> Layer:
    """120B-shaped prefill layer: router ~N(0,1/sqrt(H)) gives N(0,1)-ish logits."""
    return _layer(f"prefill_E{E}_T{T}", E, 4, T, 2880, 2880, seed, device,
                  1.0 / math.sqrt(2880), None)


def zipf_router_bias(E: int, s: float = 1.1, seed: int = 0) -> np.ndarray:
    """br[e] = ln p_{pi(e)} with p_r proportional to r^-s, pi a seeded permutation (fp32)."""
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    p /= p.sum()
    perm = np.random.default_rng(_seed(seed, "zipf_perm")).permutation(E)
    return np.log(p[perm]).astype(np.float32)


def zipf_layer(T: int = 16384, E: int = 128, seed: int = 0, device="cpu") -> Layer:
    """120B-shaped prefill with Zipf(1.1)-skewed expert loads."""
    rb = torch.from_numpy(zipf_router_bias(E, 1.1, seed)).to(torch.bfloat16).to(device)
    return _layer(f"zipf_E{E}_T{T}", E, 4, T, 2880, 2880, seed, device, 0.02, rb)


def calibration_x(H: int = 2880, T: int = 256, seed: int = 1, device="cpu") -> torch.Tensor:
    """Calibration batch for the static FP8 scales: 256 tokens, x~N(0,1) bf16, seed 1."""
    return normal((T, H), 1.0, seed, "x_calib", 0, device, torch.bfloat16)


def codec_tensor(rows: int, K: int, seed: int, tag: str, sub: int = 0, device="cpu",
                 std: float = 0.02, outlier_p: float = 0.01, outlier_mult: float = 8.0):
    """fp32 (rows, K) ~N(0,std^2) with a Bernoulli(outlier_p) mask of values times 8."""
    w = normal((rows, K), std, seed, tag, sub, device)
    g = _gen(device, seed, tag + "_mask", sub)
    mask = torch.rand((rows, K), generator=g, device=device) < outlier_p
    w[mask] *= outlier_mult
    return w


def random_logits(T: int, E: int, seed: int, tie_frac: float = 0.2) -> np.ndarray:
    """fp32 logits with exact ties planted (a fraction of entries copy a neighbour)."""
    rng = np.random.default_rng(_seed(seed, "logits"))
    l = rng.standard_normal((T, E)).astype(np.float32)
    m = rng.random((T, E)) < tie_frac
    src = rng.integers(0, E, size=(T, E))
    rows = np.arange(T)[:, None].repeat(E, 1)
    l[m] = l[rows[m], src[m]]
    return l


def random_topk_idx(T: int, E: int, k: int, seed: int, skew: float = 0.0) -> np.ndarray:
    """(T, k) int32 distinct expert ids per token; skew > 0 concentrates the load."""
    rng = np.random.default_rng(_seed(seed, "topk_idx"))
    w = np.arange(1, E + 1, dtype=np.float64) ** (-skew)
    w /= w.sum()
    out = np.empty((T, k), np.int32)
    for t in range(T):
        out[t] = rng.choice(E, size=k, replace=False, p=w)
    return out
