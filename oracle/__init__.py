"""CPU oracle for the MXFP4 routed-MoE expert layer -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package. It shares no code with the CUDA library: the arithmetic lives
in ``oracle.cpp`` (plain scalar C++, double accumulation, no fast-math, no FP
contraction), reached here through ctypes on numpy arrays.

Every function cites the web page and section it follows (see ``oracle.cpp`` header).
bf16 tensors cross this interface as ``uint16`` bit patterns.

Parity status: every function below is pinned by ``tests/test_oracle_*.py`` against
closed forms, invariants, brute force or library routines. Nothing is unpinned except
the two layout readings that need a real checkpoint (nibble order inside a byte, gate/up
row order), which no test here can check.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

OK, EINVAL, EALIGN, EUNSUPPORTED = 0, -1, -2, -3


class OracleError(RuntimeError):
    def __init__(self, rc: int, what: str):
        super().__init__(f"oracle {what} failed with code {rc}")
        self.rc = rc


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        _LIB = ctypes.CDLL(path)
    return _LIB


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def _check(rc, what):
    if rc != OK:
        raise OracleError(rc, what)


def _i64(v):
    return ctypes.c_int64(int(v))


def dequantize(blocks, scales, K=None, out="f32"):
    """MXFP4 -> float. ("quantization_mxfp4", Primitives: codebook[nibble] * 2^(s-127).)

    blocks: (..., K/2) uint8, scales: (..., K/32) uint8. Returns float32 or bf16 bits
    (uint16) with shape (..., K).
    """
    blocks = _c(blocks, np.uint8)
    scales = _c(scales, np.uint8)
    if K is None:
        K = blocks.shape[-1] * 2
    lead = blocks.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    f32 = np.empty(lead + (K,), np.float32) if out == "f32" else None
    b16 = np.empty(lead + (K,), np.uint16) if out == "bf16" else None
    _check(lib().orc_dequantize(_p(blocks), _p(scales), _i64(rows), _i64(K), _p(f32), _p(b16)),
           "dequantize")
    return f32 if out == "f32" else b16


def quantize(w):
    """float32 (..., K) -> (blocks (..., K/2) uint8, scales (..., K/32) uint8).

    ("quantization_mxfp4", Primitives: scale exponent floor(log2(amax)) - 2, nearest
    FP4 grid point; "As a quantize_model scheme": K must be a multiple of 32.)
    """
    w = _c(w, np.float32)
    K = w.shape[-1]
    lead = w.shape[:-1]
    rows = int(np.prod(lead)) if lead else 1
    if K % 32:
        _check(lib().orc_quantize(None, _i64(rows), _i64(K), None, None), "quantize")
    blocks = np.empty(lead + (K // 2,), np.uint8)
    scales = np.empty(lead + (K // 32,), np.uint8)
    _check(lib().orc_quantize(_p(w), _i64(rows), _i64(K), _p(blocks), _p(scales)), "quantize")
    return blocks, scales


def fp8_quantize(x, s):
    """FP8 E4M3 static per-tensor: q = e4m3_rne_satfinite(fp32(x / s)).

    ("amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8", Quantization schemes.)
    """
    x = _c(x, np.float32)
    q = np.empty(x.shape, np.uint8)
    _check(lib().orc_fp8_quantize(_p(x), _i64(x.size), ctypes.c_float(s), _p(q)), "fp8_quantize")
    return q


def fp8_decode(q):
    q = _c(q, np.uint8)
    out = np.empty(q.shape, np.float32)
    _check(lib().orc_fp8_decode(_p(q), _i64(q.size), _p(out)), "fp8_decode")
    return out


def bf16_round(x):
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    _check(lib().orc_bf16_round(_p(x), _i64(x.size), _p(out)), "bf16_round")
    return out


def router_logits(x, router_w, router_b=None):
    """logits (T, E) fp32 = sum_h x*Wr (double) + br; router kept in bf16.

    ("gpt-oss-120b-mxfp4-fp8attn-v2", config.json: router not converted.)
    """
    x = _c(x, np.uint16)
    router_w = _c(router_w, np.uint16)
    T, H = x.shape
    E = router_w.shape[0]
    rb = None if router_b is None else _c(router_b, np.uint16)
    logits = np.empty((T, E), np.float32)
    _check(lib().orc_router_logits(_p(x), _p(router_w), _p(rb), T, H, E, _p(logits)),
           "router_logits")
    return logits


def topk_softmax(logits, k):
    """Top-k (descending, ties to the lower expert id) + softmax over the k selected."""
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    _check(lib().orc_topk_softmax(_p(logits), T, E, k, _p(idx), _p(w)), "topk_softmax")
    return idx, w


def permute(idx, E):
    """Stable counting sort of (token, slot) pairs by expert.

    Returns offsets (E+1), perm_token (T*k), perm_slot (T*k), inv (T*k).
    """
    idx = _c(idx, np.int32)
    T, k = idx.shape
    offsets = np.empty(E + 1, np.int32)
    pt = np.empty(T * k, np.int32)
    ps = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    _check(lib().orc_permute(_p(idx), T, E, k, _p(offsets), _p(pt), _p(ps), _p(inv)), "permute")
    return offsets, pt, ps, inv


def moe_forward(x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales,
                d_bias, k, act_scale=None, dense=False):
    """The MoE expert layer ("quantization_mxfp4", As GPT-OSS's native format).

    Returns (out bf16 bits (T,H), acc fp32 (T,H), idx (T,k), w (T,k)).
    """
    x = _c(x, np.uint16)
    router_w = _c(router_w, np.uint16)
    rb = None if router_b is None else _c(router_b, np.uint16)
    gu_blocks = _c(gu_blocks, np.uint8)
    gu_scales = _c(gu_scales, np.uint8)
    gu_bias = _c(gu_bias, np.float32)
    d_blocks = _c(d_blocks, np.uint8)
    d_scales = _c(d_scales, np.uint8)
    d_bias = _c(d_bias, np.float32)
    T, H = x.shape
    E = router_w.shape[0]
    I = d_blocks.shape[-1] * 2
    acts = None if act_scale is None else np.ascontiguousarray(np.asarray(act_scale, np.float32))
    out = np.empty((T, H), np.uint16)
    acc = np.empty((T, H), np.float32)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    _check(lib().orc_moe_forward(_p(x), _p(router_w), _p(rb), _p(gu_blocks), _p(gu_scales),
                                 _p(gu_bias), _p(d_blocks), _p(d_scales), _p(d_bias), E, k, T, H,
                                 I, _p(acts), int(bool(dense)), _p(out), _p(acc), _p(idx), _p(w)),
           "moe_forward")
    return out, acc, idx, w


def expert_rows(x, expert, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias, act_scale=None):
    """y (P, H) fp32 = the expert FFN of each (row, expert) pair, with the layer's arithmetic
    ("quantization_mxfp4", As GPT-OSS's native format)."""
    x = _c(x, np.uint16)
    expert = _c(expert, np.int32)
    P, H = x.shape
    E = np.asarray(gu_blocks).shape[0]
    I = np.asarray(d_blocks).shape[-1] * 2
    acts = None if act_scale is None else np.ascontiguousarray(np.asarray(act_scale, np.float32))
    y = np.empty((P, H), np.float32)
    _check(lib().orc_expert_rows(_p(x), _p(expert), P, _p(_c(gu_blocks, np.uint8)), _p(_c(gu_scales, np.uint8)),
                                 _p(_c(gu_bias, np.float32)), _p(_c(d_blocks, np.uint8)),
                                 _p(_c(d_scales, np.uint8)), _p(_c(d_bias, np.float32)), E, H, I, _p(acts), _p(y)),
           "expert_rows")
    return y


def calibrate(x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias,
              k):
    """Static per-tensor FP8 scales {s0, s1} = {amax|x|, amax|a|} / 448 (min-max observer).

    ("gpt-oss-120b-mxfp4-fp8attn-v2", Quantization Recipe: static per-tensor scales.)
    """
    x = _c(x, np.uint16)
    router_w = _c(router_w, np.uint16)
    rb = None if router_b is None else _c(router_b, np.uint16)
    T, H = x.shape
    E = router_w.shape[0]
    I = np.asarray(d_blocks).shape[-1] * 2
    s = np.empty(2, np.float32)
    _check(lib().orc_calibrate(_p(x), _p(router_w), _p(rb), _p(_c(gu_blocks, np.uint8)),
                               _p(_c(gu_scales, np.uint8)), _p(_c(gu_bias, np.float32)),
                               _p(_c(d_blocks, np.uint8)), _p(_c(d_scales, np.uint8)),
                               _p(_c(d_bias, np.float32)), E, k, T, H, I, _p(s)), "calibrate")
    return s


def quantize_axis(w, axis):
    """MXFP4 along one contracting axis, moved to the end ("quantization_mxfp4",
    Primitives: MXFP4Quantizer.quantize(w, axis)). Returns blocks (shape with `axis` moved
    last, K/2 there) and scales (K/32 there)."""
    w = _c(w, np.float32)
    axis = axis % w.ndim
    K = w.shape[axis]
    outer = int(np.prod(w.shape[:axis])) if axis else 1
    inner = int(np.prod(w.shape[axis + 1:])) if axis + 1 < w.ndim else 1
    moved = w.shape[:axis] + w.shape[axis + 1:]
    if K % 32:
        _check(lib().orc_quantize_axis(None, _i64(outer), _i64(K), _i64(inner), None, None), "quantize_axis")
    blocks = np.empty(moved + (K // 2,), np.uint8)
    scales = np.empty(moved + (K // 32,), np.uint8)
    _check(lib().orc_quantize_axis(_p(w), _i64(outer), _i64(K), _i64(inner), _p(blocks), _p(scales)),
           "quantize_axis")
    return blocks, scales


def dequantize_axis(blocks, scales, axis, out="f32"):
    """Inverse of quantize_axis: the packed axis (last) goes back to position `axis`."""
    blocks = _c(blocks, np.uint8)
    scales = _c(scales, np.uint8)
    K = blocks.shape[-1] * 2
    moved = blocks.shape[:-1]
    nd = len(moved) + 1
    axis = axis % nd
    shape = moved[:axis] + (K,) + moved[axis:]
    outer = int(np.prod(shape[:axis])) if axis else 1
    inner = int(np.prod(shape[axis + 1:])) if axis + 1 < nd else 1
    f32 = np.empty(shape, np.float32) if out == "f32" else None
    b16 = np.empty(shape, np.uint16) if out == "bf16" else None
    _check(lib().orc_dequantize_axis(_p(blocks), _p(scales), _i64(outer), _i64(K), _i64(inner), _p(f32),
                                     _p(b16)), "dequantize_axis")
    return f32 if out == "f32" else b16


def linear(x, blocks, scales, bias=None, act_scale=None):
    """MXFP4 weight-only linear, optional FP8 activations: out = bf16(fp32(s * x.W^T) + b).

    ("quantization_mxfp4", As a quantize_model scheme.) Returns (out bf16 bits (T, N),
    acc fp32 (T, N))."""
    x = _c(x, np.uint16)
    blocks = _c(blocks, np.uint8)
    scales = _c(scales, np.uint8)
    T, K = x.shape
    N = blocks.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    s = None if act_scale is None else np.array([act_scale], np.float32)
    out = np.empty((T, N), np.uint16)
    acc = np.empty((T, N), np.float32)
    _check(lib().orc_linear(_p(x), T, K, _p(blocks), _p(scales), N, _p(b), _p(s), _p(out), _p(acc)), "linear")
    return out, acc


def fp8_linear(x, wq, s_x, s_w, bias=None):
    """FP8 E4M3 static per-tensor linear: out = bf16(fp32(s_x s_w dec(xq).dec(wq)^T) + b).

    ("gpt-oss-120b-mxfp4-fp8attn-v2", Model Details / Quantization Recipe.) Returns
    (out bf16 bits (T, N), acc fp32 (T, N))."""
    x = _c(x, np.uint16)
    wq = _c(wq, np.uint8)
    T, K = x.shape
    N = wq.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((T, N), np.uint16)
    acc = np.empty((T, N), np.float32)
    _check(lib().orc_fp8_linear(_p(x), T, K, _p(wq), N, ctypes.c_float(s_x), ctypes.c_float(s_w), _p(b),
                                _p(out), _p(acc)), "fp8_linear")
    return out, acc


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS, else all cores)."""
    v = os.environ.get("OMP_NUM_THREADS")
    return int(v) if v else (os.cpu_count() or 1)
