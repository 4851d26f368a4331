"""Thin Python binding of libmxfp4moe (include/mxfp4_moe.h), same names as the C ABI.

Argument marshalling only: torch tensors give their device pointers and the current
CUDA stream; every step of the computation runs in the library's kernels. There is no
CPU path: without a CUDA device, or without the built library, every call raises.
bf16 tensors are passed as their bit patterns (torch.bfloat16 storage).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmxfp4moe.so")

OK, EINVAL, EALIGN, EUNSUPPORTED, ECUDA, ETIMEOUT, ENOMEM, EDEVICE = 0, -1, -2, -3, -4, -5, -6, -7
OUT_F32, OUT_BF16 = 0, 1

_lib = None
_lock = threading.Lock()

_vp, _i64, _i32, _f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
_SIGS = {
    "mxfp4_quantize": [_vp, _i64, _i64, _vp, _vp, _vp],
    "mxfp4_dequantize": [_vp, _vp, _i64, _i64, _vp, _i32, _vp],
    "mxfp4_quantize_axis": [_vp, _i64, _i64, _i64, _vp, _vp, _vp],
    "mxfp4_dequantize_axis": [_vp, _vp, _i64, _i64, _i64, _vp, _i32, _vp],
    "mxfp4_linear": [_vp, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _vp],
    "fp8_linear": [_vp, _i32, _i32, _vp, _i32, _f32, _f32, _vp, _vp, _vp],
    "moe_route_topk": [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp],
    "moe_topk_from_logits": [_vp, _i32, _i32, _i32, _vp, _vp, _vp],
    "moe_permute": [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp],
    "moe_permute_noalloc": [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp],
    "moe_fp8_quantize": [_vp, _i64, _f32, _vp, _vp],
    "moe_mxfp4_forward": [_vp] * 9 + [_i32] * 5 + [_vp, _vp, _vp],
    "moe_mxfp4_forward_dense": [_vp] * 9 + [_i32] * 5 + [_vp, _vp, _vp],
    "moe_mxfp4_calibrate": [_vp] * 9 + [_i32] * 5 + [_vp, _vp],
    "moe_mxfp4_experts": [_vp, _vp, _i32, _i32, _i32, _i32] + [_vp] * 9,
    "moe_combine": [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp],
    "mxmoe_check": [_vp],
    "mxmoe_last_error": [],
    "mxmoe_last_launch_count": [],
    "mxmoe_release": [],
    "mxmoe_selftest_wait_timeout": [_vp],
    "mxmoe_tc_rate_probe": [_i32, _i32, _i32, _i32, _i32, _vp, _vp],
    "mxmoe_profile_enable": [_i32],
    "mxmoe_profile_read": [_vp, _vp, _vp, _i32],
}


class MxmoeError(RuntimeError):
    def __init__(self, rc: int, fn: str, msg: str):
        super().__init__(f"{fn} failed ({rc}): {msg}")
        self.rc = rc


def lib() -> ctypes.CDLL:
    """Load the library (once). Raises if it is missing or no CUDA device is visible."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not torch.cuda.is_available():
                    raise RuntimeError("libmxfp4moe needs a CUDA device; there is no CPU path")
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(f"{LIB_PATH} is missing: run mxfp4_block_scaled_moe_b200/build.py")
                L = ctypes.CDLL(LIB_PATH)
                for name, args in _SIGS.items():
                    fn = getattr(L, name)
                    fn.argtypes = args
                    fn.restype = ctypes.c_char_p if name == "mxmoe_last_error" else ctypes.c_int
                _lib = L
    return _lib


def _call(name, *args):
    L = lib()
    rc = getattr(L, name)(*args)
    if rc != OK:
        msg = L.mxmoe_last_error().decode(errors="replace")
        raise MxmoeError(rc, name, msg)
    return rc


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, dtype, name):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


# ----------------------------------------------------------------------- codec -----

def mxfp4_quantize(w: torch.Tensor, blocks=None, scales=None, stream=None):
    """fp32 (..., K) -> (blocks (..., K/2) uint8, scales (..., K/32) uint8)."""
    _dev(w, torch.float32, "w")
    K = w.shape[-1]
    rows = w.numel() // K if K else 0
    if blocks is None:
        blocks = torch.empty(*w.shape[:-1], K // 2, dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(*w.shape[:-1], max(K // 32, 0), dtype=torch.uint8, device=w.device)
    _call("mxfp4_quantize", _ptr(w), rows, K, _ptr(blocks), _ptr(scales), _stream(stream))
    return blocks, scales


def mxfp4_dequantize(blocks: torch.Tensor, scales: torch.Tensor, out_dtype=torch.float32,
                     out=None, stream=None):
    """(..., K/2) uint8 + (..., K/32) uint8 -> (..., K) fp32 or bf16."""
    _dev(blocks, torch.uint8, "blocks")
    _dev(scales, torch.uint8, "scales")
    K = blocks.shape[-1] * 2
    rows = blocks.numel() // blocks.shape[-1] if blocks.shape[-1] else 0
    code = OUT_F32 if out_dtype == torch.float32 else OUT_BF16
    if out is None:
        out = torch.empty(*blocks.shape[:-1], K, dtype=out_dtype, device=blocks.device)
    _call("mxfp4_dequantize", _ptr(blocks), _ptr(scales), rows, K, _ptr(out), code, _stream(stream))
    return out


# --------------------------------------------------------------------- routing -----

def moe_route_topk(x, router_w, router_b, k, with_logits=False, stream=None):
    """Returns (topk_idx int32 (T,k), topk_w fp32 (T,k)[, logits fp32 (T,E)])."""
    _dev(x, torch.bfloat16, "x")
    _dev(router_w, torch.bfloat16, "router_w")
    _dev(router_b, torch.bfloat16, "router_b")
    T, H = x.shape
    E = router_w.shape[0]
    idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    logits = torch.empty(T, E, dtype=torch.float32, device=x.device) if with_logits else None
    _call("moe_route_topk", _ptr(x), _ptr(router_w), _ptr(router_b), T, H, E, k, _ptr(logits),
          _ptr(idx), _ptr(w), _stream(stream))
    return (idx, w, logits) if with_logits else (idx, w)


def moe_topk_from_logits(logits, k, stream=None):
    _dev(logits, torch.float32, "logits")
    T, E = logits.shape
    idx = torch.empty(T, k, dtype=torch.int32, device=logits.device)
    w = torch.empty(T, k, dtype=torch.float32, device=logits.device)
    _call("moe_topk_from_logits", _ptr(logits), T, E, k, _ptr(idx), _ptr(w), _stream(stream))
    return idx, w


def moe_permute(topk_idx, E, stream=None):
    """Returns (offsets (E+1), perm_token (T*k), perm_slot (T*k)), all int32."""
    _dev(topk_idx, torch.int32, "topk_idx")
    T, k = topk_idx.shape
    dev = topk_idx.device
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    pt = torch.empty(T * k, dtype=torch.int32, device=dev)
    ps = torch.empty(T * k, dtype=torch.int32, device=dev)
    _call("moe_permute", _ptr(topk_idx), T, E, k, _ptr(offsets), _ptr(pt), _ptr(ps), _stream(stream))
    return offsets, pt, ps


def moe_permute_noalloc(topk_idx, E, offsets, perm_token, perm_slot, stream=None):
    """moe_permute into caller-provided outputs without any device allocation by the
    library (its scratch is a fixed array; T*k <= 262144, E <= 256)."""
    _dev(topk_idx, torch.int32, "topk_idx")
    T, k = topk_idx.shape
    _call("moe_permute_noalloc", _ptr(topk_idx), T, E, k, _ptr(offsets), _ptr(perm_token),
          _ptr(perm_slot), _stream(stream))
    return offsets, perm_token, perm_slot


def moe_fp8_quantize(x, s, stream=None):
    """bf16 tensor -> uint8 E4M3 codes of x / s."""
    _dev(x, torch.bfloat16, "x")
    q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _call("moe_fp8_quantize", _ptr(x), x.numel(), float(s), _ptr(q), _stream(stream))
    return q


def _axis_view(shape, axis):
    axis = axis % len(shape)
    K = int(shape[axis])
    outer = 1
    for d in shape[:axis]:
        outer *= int(d)
    inner = 1
    for d in shape[axis + 1:]:
        inner *= int(d)
    return axis, outer, K, inner


def mxfp4_quantize_axis(w: torch.Tensor, axis: int, stream=None):
    """fp32 tensor -> (blocks, scales) along `axis`, moved to the end: blocks have the
    shape of w with that axis last and K/2 long, scales K/32 long."""
    _dev(w, torch.float32, "w")
    axis, outer, K, inner = _axis_view(w.shape, axis)
    moved = tuple(w.shape[:axis]) + tuple(w.shape[axis + 1:])
    blocks = torch.empty(*moved, K // 2, dtype=torch.uint8, device=w.device)
    scales = torch.empty(*moved, max(K // 32, 0), dtype=torch.uint8, device=w.device)
    _call("mxfp4_quantize_axis", _ptr(w), outer, K, inner, _ptr(blocks), _ptr(scales), _stream(stream))
    return blocks, scales


def mxfp4_dequantize_axis(blocks: torch.Tensor, scales: torch.Tensor, axis: int, out_dtype=torch.float32,
                          out=None, stream=None):
    """Inverse of mxfp4_quantize_axis: the packed (last) axis goes back to position `axis`."""
    _dev(blocks, torch.uint8, "blocks")
    _dev(scales, torch.uint8, "scales")
    K = blocks.shape[-1] * 2
    moved = tuple(blocks.shape[:-1])
    nd = len(moved) + 1
    axis = axis % nd
    shape = moved[:axis] + (K,) + moved[axis:]
    _, outer, _, inner = _axis_view(shape, axis)
    if out is None:
        out = torch.empty(shape, dtype=out_dtype, device=blocks.device)
    code = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    _call("mxfp4_dequantize_axis", _ptr(blocks), _ptr(scales), outer, K, inner, _ptr(out), code, _stream(stream))
    return out


def mxfp4_linear(x, blocks, scales, bias=None, act_scale=None, out=None, stream=None):
    """out (T, N) bf16 = x (T, K) bf16 . W^T + bias with W MXFP4 (blocks (N, K/2), scales
    (N, K/32)); act_scale (one float) casts the input to FP8 E4M3 first."""
    _dev(x, torch.bfloat16, "x")
    _dev(blocks, torch.uint8, "blocks")
    _dev(scales, torch.uint8, "scales")
    _dev(bias, torch.float32, "bias")
    T, K = x.shape
    N = blocks.shape[0]
    if out is None:
        out = torch.empty(T, N, dtype=torch.bfloat16, device=x.device)
    s = None if act_scale is None else ctypes.byref(ctypes.c_float(float(act_scale)))
    _call("mxfp4_linear", _ptr(x), T, K, _ptr(blocks), _ptr(scales), N, _ptr(bias), s, _ptr(out), _stream(stream))
    return out


def fp8_linear(x, wq, s_x, s_w, bias=None, out=None, stream=None):
    """out (T, N) bf16 = bf16(s_x s_w e4m3(x / s_x) . wq^T + bias); wq: (N, K) uint8 E4M3 codes."""
    _dev(x, torch.bfloat16, "x")
    _dev(wq, torch.uint8, "wq")
    _dev(bias, torch.float32, "bias")
    T, K = x.shape
    N = wq.shape[0]
    if out is None:
        out = torch.empty(T, N, dtype=torch.bfloat16, device=x.device)
    _call("fp8_linear", _ptr(x), T, K, _ptr(wq), N, float(s_x), float(s_w), _ptr(bias), _ptr(out), _stream(stream))
    return out


# ----------------------------------------------------------------------- layer -----

def _layer_ptrs(x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias):
    _dev(x, torch.bfloat16, "x")
    _dev(router_w, torch.bfloat16, "router_w")
    _dev(router_b, torch.bfloat16, "router_b")
    for n, t in (("gu_blocks", gu_blocks), ("gu_scales", gu_scales), ("d_blocks", d_blocks),
                 ("d_scales", d_scales)):
        _dev(t, torch.uint8, n)
    _dev(gu_bias, torch.float32, "gu_bias")
    _dev(d_bias, torch.float32, "d_bias")
    T, H = x.shape
    E = router_w.shape[0]
    I = d_blocks.shape[-1] * 2
    ptrs = [_ptr(t) for t in (x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks,
                              d_scales, d_bias)]
    return ptrs, E, T, H, I


def _forward(name, x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales,
             d_bias, k, act_scale, out, stream):
    ptrs, E, T, H, I = _layer_ptrs(x, router_w, router_b, gu_blocks, gu_scales, gu_bias,
                                   d_blocks, d_scales, d_bias)
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=x.device)
    _dev(out, torch.bfloat16, "out")
    acts = None
    if act_scale is not None:
        s = [float(v) for v in act_scale]
        acts = (ctypes.c_float * 2)(s[0], s[1])
    _call(name, *ptrs, E, k, T, H, I,
          ctypes.cast(acts, ctypes.c_void_p) if acts is not None else None, _ptr(out),
          _stream(stream))
    return out


def moe_mxfp4_forward(x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales,
                      d_bias, k, act_scale=None, out=None, stream=None):
    """The MoE expert layer; act_scale = None (bf16 activations) or two floats {s0, s1}."""
    return _forward("moe_mxfp4_forward", x, router_w, router_b, gu_blocks, gu_scales, gu_bias,
                    d_blocks, d_scales, d_bias, k, act_scale, out, stream)


def moe_mxfp4_forward_dense(x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks,
                            d_scales, d_bias, k, act_scale=None, out=None, stream=None):
    """The same layer by the dense all-experts path (every token through all E experts,
    zero gates off the top-k)."""
    return _forward("moe_mxfp4_forward_dense", x, router_w, router_b, gu_blocks, gu_scales,
                    gu_bias, d_blocks, d_scales, d_bias, k, act_scale, out, stream)


def moe_mxfp4_calibrate(x, router_w, router_b, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales,
                        d_bias, k, stream=None):
    """Static FP8 scales {s0, s1} (device fp32 (2,)) from a calibration batch x."""
    ptrs, E, T, H, I = _layer_ptrs(x, router_w, router_b, gu_blocks, gu_scales, gu_bias,
                                   d_blocks, d_scales, d_bias)
    out = torch.empty(2, dtype=torch.float32, device=x.device)
    _call("moe_mxfp4_calibrate", *ptrs, E, k, T, H, I, _ptr(out), _stream(stream))
    return out


def moe_mxfp4_experts(x_rows, offsets, gu_blocks, gu_scales, gu_bias, d_blocks, d_scales, d_bias,
                      act_scale=None, y=None, stream=None):
    """fp32 (P, H) expert outputs of rows grouped by expert (offsets: int32 (E+1))."""
    _dev(x_rows, torch.bfloat16, "x_rows")
    _dev(offsets, torch.int32, "offsets")
    P, H = x_rows.shape
    E = gu_blocks.shape[0]
    I = d_blocks.shape[-1] * 2
    if y is None:
        y = torch.empty(P, H, dtype=torch.float32, device=x_rows.device)
    acts = None
    if act_scale is not None:
        s = [float(v) for v in act_scale]
        acts = (ctypes.c_float * 2)(s[0], s[1])
    _call("moe_mxfp4_experts", _ptr(x_rows), _ptr(offsets), E, P, H, I, _ptr(gu_blocks), _ptr(gu_scales),
          _ptr(gu_bias), _ptr(d_blocks), _ptr(d_scales), _ptr(d_bias),
          ctypes.cast(acts, ctypes.c_void_p) if acts is not None else None, _ptr(y), _stream(stream))
    return y


def moe_combine(y, topk_idx, topk_w, inv, out=None, stream=None):
    """bf16 (T, H): each token's k expert outputs y[inv] weighted and summed in ascending expert id."""
    _dev(y, torch.float32, "y")
    T, k = topk_idx.shape
    H = y.shape[1]
    if out is None:
        out = torch.empty(T, H, dtype=torch.bfloat16, device=y.device)
    _call("moe_combine", _ptr(y), _ptr(topk_idx), _ptr(topk_w), _ptr(inv), T, H, k, _ptr(out), _stream(stream))
    return out


def mxmoe_check(stream=None):
    _call("mxmoe_check", _stream(stream))


def mxmoe_last_launch_count() -> int:
    return lib().mxmoe_last_launch_count()


def mxmoe_release():
    _call("mxmoe_release")


def mxmoe_tc_rate_probe(n=256, with_scale_copy=False, iters=20000, ctas=None, stream=None,
                        random_operands=True) -> float:
    """Launch the tensor-pipe rate probe (kind::mxf8f6f4 MMAs, M = 128, N = n) on `ctas`
    CTAs (default: one per SM), on pseudo-random operands (or zeros); returns the FLOPs the
    launch performs. Time it with CUDA events on `stream`."""
    if ctas is None:
        ctas = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    f = ctypes.c_double(0.0)
    _call("mxmoe_tc_rate_probe", int(n), 1 if with_scale_copy else 0, 1 if random_operands else 0, int(iters),
          int(ctas), ctypes.byref(f), _stream(stream))
    return f.value


def mxmoe_selftest_wait_timeout(stream=None):
    """Launch a bounded device wait that expires (about a second); the next
    mxmoe_check raises MxmoeError with MXMOE_ETIMEOUT."""
    _call("mxmoe_selftest_wait_timeout", _stream(stream))


def mxmoe_profile_enable(on: bool = True):
    _call("mxmoe_profile_enable", 1 if on else 0)


def mxmoe_profile_read(max_entries: int = 32):
    """{stage: (total_ms, calls)} recorded since profiling was enabled or last read."""
    L = lib()
    names = ctypes.create_string_buffer(32 * max_entries)
    ms = (ctypes.c_float * max_entries)()
    calls = (ctypes.c_int * max_entries)()
    n = L.mxmoe_profile_read(names, ms, calls, max_entries)
    if n < 0:
        raise MxmoeError(n, "mxmoe_profile_read", L.mxmoe_last_error().decode(errors="replace"))
    out = {}
    for i in range(min(n, max_entries)):
        nm = names.raw[32 * i:32 * (i + 1)].split(b"\0", 1)[0].decode()
        out[nm] = (float(ms[i]), int(calls[i]))
    return out
