"""The C ABI on a machine without a GPU: the library loads, exports every
function include/moe.h declares, and rejects bad arguments before any CUDA
call (so these run on the CPU)."""
import ctypes as C
import os
import re

import pytest

from mixed_precision_moe_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(moe_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for n in ("moe_route_topk", "moe_permute", "moe_grouped_ffn_mixed", "moe_combine",
              "moe_set_expert_precision", "moe_layer_create", "moe_layer_destroy",
              "moe_quantize_weights", "moe_get_device_status", "moe_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"libmoe.so does not export {n}"
    assert set(names) == set(binding.SIGNATURES), "binding and header disagree"


def test_abi_version(lib):
    assert lib.moe_abi_version() == 1


def _err(lib):
    return lib.moe_last_error().decode()


def test_host_validation_before_any_cuda_call(lib):
    h = C.c_void_p()
    assert lib.moe_layer_create(100, 512, 8, 2, C.byref(h)) == -2      # H % 128
    assert "128" in _err(lib)
    assert lib.moe_layer_create(256, 512, 0, 1, C.byref(h)) == -2      # E < 1
    assert lib.moe_layer_create(256, 512, 513, 1, C.byref(h)) == -2    # E > 512
    assert lib.moe_layer_create(256, 512, 8, 9, C.byref(h)) == -1      # k > E
    assert lib.moe_layer_create(256, 512, 32, 17, C.byref(h)) == -1    # k > 16
    assert lib.moe_layer_create(256, 512, 8, 2, None) == -1
    assert lib.moe_layer_destroy(None) == -1
    assert lib.moe_route_topk(None, 4, 8, 9, 1, None, None, None) == -1
    assert lib.moe_route_topk(None, -1, 8, 2, 1, None, None, None) == -1
    assert lib.moe_route_topk(None, 4, 600, 2, 1, None, None, None) == -2
    assert lib.moe_route_topk(None, 4, 8, 2, 1, None, None, None) == -1   # null pointers
    assert lib.moe_route_topk(None, 0, 8, 2, 1, None, None, None) == 0    # T = 0: nothing to do
    # router projection + top-k: H a multiple of 64, E <= 512, k <= min(E, 16)
    assert lib.moe_router_topk(None, None, 4, 100, 8, 2, 1, None, None, None, None) == -2
    assert lib.moe_router_topk(None, None, 4, 256, 513, 2, 1, None, None, None, None) == -2
    assert lib.moe_router_topk(None, None, 4, 256, 8, 9, 1, None, None, None, None) == -1
    assert lib.moe_router_topk(None, None, -1, 256, 8, 2, 1, None, None, None, None) == -1
    assert lib.moe_router_topk(None, None, 4, 256, 8, 2, 1, None, None, None, None) == -1
    assert lib.moe_router_topk(None, None, 0, 256, 8, 2, 1, None, None, None, None) == 0
    assert lib.moe_layer_forward_hidden(None, None, None, 4, 1, None, None, None, None, None,
                                        None, None, None, None, 0, None, None) == -1
    assert lib.moe_permute(None, None, 4, 0, 2, 256, None, None, None, None, None) == -2
    assert lib.moe_permute(None, None, 4, 8, 2, 100, None, None, None, None, None) == -2
    assert lib.moe_combine(None, None, None, 4, 0, 256, None, None) == -1
    assert lib.moe_combine(None, None, None, 4, 2, 100, None, None) == -2
    assert lib.moe_combine(None, None, None, 0, 2, 256, None, None) == 0
    assert lib.moe_quantize_weights(None, 4, 100, 2, None, None, None) == -2
    assert lib.moe_quantize_weights(None, 4, 128, 0, None, None, None) == -1  # BF16 is not a code
    assert lib.moe_ffn_workspace_bytes(None, 4, None) == -1
    assert lib.moe_grouped_ffn_mixed(None, None, None, 4, None, None, 0, None) == -1
    assert lib.moe_get_device_status(None) == -1


def test_last_error_is_cleared_by_success(lib):
    assert lib.moe_combine(None, None, None, 4, 0, 256, None, None) == -1
    assert _err(lib)
    assert lib.moe_combine(None, None, None, 0, 2, 256, None, None) == 0
    assert _err(lib) == ""


def test_binding_refuses_host_tensors_instead_of_falling_back(lib):
    """No CPU path exists: every entry point of the binding rejects tensors that
    are not contiguous CUDA tensors of the expected dtype, before any library call."""
    import torch
    logits = torch.zeros((4, 8), dtype=torch.float32)
    x = torch.zeros((4, 256), dtype=torch.bfloat16)
    idx = torch.zeros((4, 2), dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        binding.moe_route_topk(logits, 2)
    with pytest.raises(ValueError, match="CUDA"):
        binding.moe_permute(idx, x, 8)
    with pytest.raises(ValueError, match="CUDA"):
        binding.moe_combine(x, idx, torch.zeros((4, 2)))
    with pytest.raises(ValueError, match="CUDA"):
        binding.moe_quantize_weights(x, binding.INT4)
    with pytest.raises(ValueError):
        binding.moe_route_topk(logits.double(), 2)
