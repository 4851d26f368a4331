"""The C ABI's argument checks and error codes, exercised without a GPU.

Every call below is invalid (or has no work) and returns from the library's argument
checks before any CUDA call, so the fake device pointers are never dereferenced. The
module is skipped where a GPU is visible: there a call that passed its checks would launch
kernels on those pointers, and the GPU suite covers the same checks with real buffers.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="argument checks with fake pointers: CPU only")

OK, EINVAL, EALIGN, EUNSUPPORTED = 0, -1, -2, -3
A = ctypes.c_void_p(1 << 20)          # a 16-byte aligned fake device address (never read)
MIS = ctypes.c_void_p((1 << 20) + 4)  # a misaligned one


@pytest.fixture(scope="module")
def L():
    from mxfp4_block_scaled_moe_b200 import binding, build
    lib = ctypes.CDLL(build.build())
    for name, args in binding._SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "mxmoe_last_error" else ctypes.c_int
    return lib


def err(L):
    return L.mxmoe_last_error().decode()


def test_codec_argument_checks(L):
    assert L.mxfp4_quantize(A, 4, 31, A, A, None) == EALIGN and "multiple of 32" in err(L)
    assert L.mxfp4_quantize(A, -1, 32, A, A, None) == EINVAL
    assert L.mxfp4_quantize(None, 4, 32, A, A, None) == EINVAL
    assert L.mxfp4_quantize(MIS, 4, 32, A, A, None) == EINVAL and "aligned" in err(L)
    assert L.mxfp4_quantize(None, 0, 32, None, None, None) == OK      # no work
    assert L.mxfp4_dequantize(A, A, 4, 33, A, 0, None) == EALIGN
    assert L.mxfp4_dequantize(A, A, 4, 32, A, 7, None) == EUNSUPPORTED
    assert L.mxfp4_dequantize(A, A, 4, 32, MIS, 1, None) == EINVAL
    assert L.mxfp4_dequantize(A, A, 4, 32, None, 0, None) == EINVAL


@pytest.mark.parametrize("T,E,k,code", [(-1, 8, 2, EINVAL), (1 << 24, 8, 2, EUNSUPPORTED), (4, 0, 1, EINVAL),
                                        (4, 257, 4, EUNSUPPORTED), (4, 8, 0, EUNSUPPORTED),
                                        (4, 16, 9, EUNSUPPORTED), (4, 3, 4, EUNSUPPORTED)])
def test_routing_argument_checks(L, T, E, k, code):
    assert L.moe_route_topk(A, A, None, T, 64, E, k, None, A, A, None) == code
    assert L.moe_topk_from_logits(A, T, E, k, A, A, None) == code
    assert L.moe_permute(A, T, E, k, A, A, A, None) == code
    assert err(L)


def test_router_and_permute_pointer_checks(L):
    assert L.moe_route_topk(A, A, None, 4, 31, 8, 2, None, A, A, None) == EALIGN
    assert L.moe_route_topk(A, A, None, 4, 0, 8, 2, None, A, A, None) == EINVAL
    assert L.moe_route_topk(None, A, None, 4, 64, 8, 2, None, A, A, None) == EINVAL
    assert L.moe_route_topk(MIS, A, None, 4, 64, 8, 2, None, A, A, None) == EINVAL
    assert L.moe_route_topk(None, None, None, 0, 64, 8, 2, None, None, None, None) == OK   # T = 0
    assert L.moe_topk_from_logits(None, 4, 8, 2, A, A, None) == EINVAL
    assert L.moe_topk_from_logits(None, 0, 8, 2, None, None, None) == OK
    assert L.moe_permute(A, 4, 8, 2, None, A, A, None) == EINVAL
    assert L.moe_permute(None, 4, 8, 2, A, A, A, None) == EINVAL


def test_fp8_cast_checks(L):
    assert L.moe_fp8_quantize(A, -1, 1.0, A, None) == EINVAL
    assert L.moe_fp8_quantize(A, 16, 0.0, A, None) == EINVAL and "scale" in err(L)
    assert L.moe_fp8_quantize(None, 16, 1.0, A, None) == EINVAL
    assert L.moe_fp8_quantize(None, 0, 1.0, None, None) == OK


def _layer(L, fn, E=4, k=2, T=16, H=256, I=256, tail=(A, None), **over):
    p = dict(x=A, rw=A, rb=None, gub=A, gus=A, gubias=A, db=A, ds=A, dbias=A)
    p.update(over)
    return getattr(L, fn)(p["x"], p["rw"], p["rb"], p["gub"], p["gus"], p["gubias"], p["db"], p["ds"],
                          p["dbias"], E, k, T, H, I, *tail)


def test_layer_argument_checks(L):
    fwd = lambda **kw: _layer(L, "moe_mxfp4_forward", tail=kw.pop("tail", (None, A, None)), **kw)
    assert fwd(T=0) == OK                                     # empty batch: no work
    assert fwd(T=0, k=5) == EUNSUPPORTED                      # still checks the routing shape
    assert fwd(H=250) == EALIGN and fwd(I=200) == EALIGN
    assert fwd(H=0) == EINVAL
    assert fwd(k=5) == EUNSUPPORTED and fwd(E=300) == EUNSUPPORTED
    assert fwd(x=None) == EINVAL and "x is NULL" in err(L)
    assert fwd(gub=MIS) == EINVAL and "gu_blocks" in err(L)
    assert fwd(rb=MIS) == EINVAL and "router_b" in err(L)
    assert fwd(tail=(None, None, None)) == EINVAL              # out
    assert fwd(tail=(None, MIS, None)) == EINVAL
    bad = (ctypes.c_float * 2)(0.0, 1.0)
    assert fwd(tail=(ctypes.cast(bad, ctypes.c_void_p), A, None)) == EINVAL and "act_scale" in err(L)
    cal = lambda **kw: _layer(L, "moe_mxfp4_calibrate", tail=kw.pop("tail", (A, None)), **kw)
    assert cal(T=0) == EINVAL
    assert cal(tail=(None, None)) == EINVAL
    assert cal(dbias=None) == EINVAL and "d_bias" in err(L)


def test_rate_probe_argument_checks(L):
    f = ctypes.c_double(0.0)
    assert L.mxmoe_tc_rate_probe(8, 0, 1, 10, 1, ctypes.byref(f), None) == EINVAL and "multiple of 16" in err(L)
    assert L.mxmoe_tc_rate_probe(264, 0, 1, 10, 1, ctypes.byref(f), None) == EINVAL
    assert L.mxmoe_tc_rate_probe(256, 0, 2, 10, 1, ctypes.byref(f), None) == EINVAL and "random_operands" in err(L)
    assert L.mxmoe_tc_rate_probe(256, 0, 1, 0, 1, ctypes.byref(f), None) == EINVAL and "iters" in err(L)
    assert L.mxmoe_tc_rate_probe(256, 0, 1, 10, 0, ctypes.byref(f), None) == EINVAL and "ctas" in err(L)
