"""The C ABI library loads without a GPU and exports every entry point the header
declares (no compute calls: this file runs on CPU-only machines)."""
import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mxfp4_moe.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["mxfp4_quantize", "mxfp4_dequantize", "moe_route_topk", "moe_mxfp4_forward",
              "moe_topk_from_logits", "moe_permute", "mxmoe_last_error", "mxmoe_check"]:
        assert n in names


def test_library_builds_loads_and_exports_every_declared_symbol():
    from mxfp4_block_scaled_moe_b200 import build
    path = build.build()
    lib = ctypes.CDLL(path)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_names_match_the_header():
    from mxfp4_block_scaled_moe_b200 import binding
    assert set(binding._SIGS) == set(declared_functions())


def test_binding_refuses_to_run_without_a_gpu():
    import torch
    from mxfp4_block_scaled_moe_b200 import binding
    if torch.cuda.is_available():
        return
    try:
        binding.lib()
    except RuntimeError as e:
        assert "no CPU path" in str(e)
    else:
        raise AssertionError("binding loaded without a GPU")
