"""A second, independent restatement of the MoE layer in numpy (tiny shapes only).

Test infrastructure used to pin the C++ oracle. It is written from the definitions
rather than from the oracle: the E2M1 value comes from the bit fields (sign, 2-bit
exponent with bias 1, 1-bit mantissa, subnormal at exponent 0) instead of a table, dot
products use numpy matmul, FP8 and bf16 roundings use torch's own casts, top-k uses a
full stable sort.
"""
from __future__ import annotations

import numpy as np
import torch


def e2m1_from_bits(nib: np.ndarray) -> np.ndarray:
    nib = nib.astype(np.int64)
    sign = np.where(nib & 8, -1.0, 1.0)
    ex = (nib >> 1) & 3
    man = nib & 1
    mag = np.where(ex == 0, 0.5 * man, np.ldexp(1.0 + 0.5 * man, ex - 1))
    return sign * mag


def dequant(blocks: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """(..., K/2) u8 + (..., K/32) u8 -> float64 (..., K), exact."""
    lo = blocks & 0x0F
    hi = blocks >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(blocks.shape[:-1] + (blocks.shape[-1] * 2,))
    sc = np.repeat(scales.astype(np.int64) - 127, 32, axis=-1)
    return np.ldexp(e2m1_from_bits(nib), sc)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(x32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (torch's RNE cast) -> float64."""
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.to(torch.float64).numpy()


def fp8_e4m3(x32: np.ndarray) -> np.ndarray:
    """fp32 -> e4m3fn via torch's cast after clamping to +/-448 -> float64 value."""
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).clamp(-448.0, 448.0)
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def topk_softmax(logits: np.ndarray, k: int):
    T, E = logits.shape
    idx = np.empty((T, k), np.int64)
    for t in range(T):
        order = np.lexsort((np.arange(E), -logits[t].astype(np.float64)))
        idx[t] = order[:k]
    sel = np.take_along_axis(logits.astype(np.float64), idx, 1)
    p = np.exp(sel - sel[:, :1])
    w = (p / p.sum(1, keepdims=True)).astype(np.float32)
    return idx, w


def moe_forward(x_bits, rw_bits, rb_bits, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales,
                d_bias, k, act_scale=None):
    """Returns (acc fp32 (T,H), idx, w). Routed-only, ascending-expert fp32 combine."""
    x = bf16_to_f64(x_bits)
    logits = x @ bf16_to_f64(rw_bits).T
    if rb_bits is not None:
        logits = logits + bf16_to_f64(rb_bits)[None, :]
    logits = logits.astype(np.float32)
    idx, w = topk_softmax(logits, k)
    T, H = x.shape
    I = d_blocks.shape[-1] * 2
    wgu = dequant(gu_blocks, gu_scales)   # (E, 2I, H)
    wd = dequant(d_blocks, d_scales)      # (E, H, I)
    acc = np.zeros((T, H), np.float32)
    for t in range(T):
        for j in np.argsort(idx[t], kind="stable"):
            e = idx[t, j]
            if act_scale is not None:
                s0, s1 = np.float32(act_scale[0]), np.float32(act_scale[1])
                xin = fp8_e4m3(x[t].astype(np.float32) / s0)
            else:
                s0 = s1 = np.float32(1.0)
                xin = x[t]
            g = (np.float64(s0) * (wgu[e] @ xin)).astype(np.float32) + gu_bias[e]
            gate, up = g[:I].astype(np.float64), g[I:].astype(np.float64)
            a = (gate / (1.0 + np.exp(-gate)) * up).astype(np.float32)
            ain = fp8_e4m3(a / s1) if act_scale is not None else round_bf16(a)
            y = (np.float64(s1) * (wd[e] @ ain)).astype(np.float32) + d_bias[e]
            acc[t] = acc[t] + (np.float32(w[t, j]) * y).astype(np.float32)
    return acc, idx, w
