"""The allocation-free grouped FFN entry point (moe_grouped_ffn_mixed_noalloc).

Some callers cannot pass the library a workspace -- for example an operator
inside another framework with no handle on that framework's allocator, or a
latency-critical loop that must not call cudaMalloc.  For them the library keeps
a fixed scratch array in device memory.  This test calls that entry point
through the C ABI twice in a row, with different inputs, and checks each result
against the workspace entry point (moe_grouped_ffn_mixed) on the same inputs,
within the tolerance the parity tests use (and, the kernel being deterministic,
bit for bit).  It also checks that a call too large for the scratch is refused.

It lives in a file of its own that pytest collects last, and builds everything
it needs itself, so it passes alone in a fresh process and after the others.
"""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_moe_b200 import binding as B
from mixed_precision_moe_b200 import build, synth
from helpers import check_close, gpu_layer, oracle_experts, to_gpu_bf16

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    assert torch.cuda.is_available(), "GPU test"
    build.build()
    H, I = 512, 384
    precs = [oracle.BF16, oracle.INT8, oracle.INT4, oracle.INT4, oracle.BF16, oracle.INT8]
    exps = oracle_experts(H, I, precs, 314)
    layer = gpu_layer(H, I, len(precs), len(precs), exps)
    B.moe_get_device_status()
    try:
        for call, (groups, seed) in enumerate([([3, 40, 0, 17, 128, 9], 11),
                                               ([64, 1, 77, 30, 0, 5], 12),
                                               ([5, 5, 5, 5, 5, 5], 13)]):
            if call == 2:   # a fresh look-up of the scratch address gives the same results
                B.moe_ffn_noalloc_reset()
            offsets = np.concatenate([[0], np.cumsum(groups)]).astype(np.int32)
            off = torch.from_numpy(offsets).cuda()
            xp = to_gpu_bf16(synth.gen_x(int(offsets[-1]), H, seed))
            ref = B.moe_grouped_ffn_mixed(layer, xp, off)
            got = B.moe_grouped_ffn_mixed_noalloc(layer, xp, off)
            torch.cuda.synchronize()
            check_close(got.float().double().cpu().numpy(), ref.float().double().cpu().numpy(),
                        f"no-alloc call {call + 1}")
            assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), f"call {call + 1}"
        assert B.moe_get_device_status() == 0
    finally:
        layer.close()


def test_noalloc_refuses_calls_larger_than_its_scratch():
    build.build()
    limit = B.moe_ffn_noalloc_max_bytes()
    assert limit == 8 << 20
    H, I = 256, 512
    layer = B.MoELayer(H, I, 2, 2)
    try:
        rows = (limit - 8192) // (2 * I) + 1          # one row past the limit
        xp = torch.zeros((rows, H), dtype=torch.bfloat16, device="cuda")
        off = torch.tensor([0, rows, rows], dtype=torch.int32, device="cuda")
        with pytest.raises(B.MoeError) as ei:
            B.moe_grouped_ffn_mixed_noalloc(layer, xp, off)
        assert ei.value.code == -2 and "scratch" in str(ei.value)
    finally:
        layer.close()
