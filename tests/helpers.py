"""Shared test helpers: the same seeded experts for the oracle and the GPU.

The oracle quantises the bf16 masters itself (CPU); the GPU path receives
those codes and scales, so a GPU/oracle mismatch in the FFN tests points at
the FFN kernels and not at the quantiser (which has its own parity test).
"""
import numpy as np
import torch

import oracle
from mixed_precision_moe_b200 import synth

# Tolerances for the bf16 layer output against the binary64 oracle.
MEAN_REL_TOL = 5e-3     # sum|gpu - oracle| / sum|oracle|
MAX_ABS_TOL = 1e-2      # max|gpu - oracle| <= MAX_ABS_TOL * max|oracle|


def oracle_experts(H, I, precs, seed, masters=None):
    return oracle.seeded_experts(H, I, precs, seed, masters)


def to_gpu_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_gpu_f16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).cuda()


def gpu_expert_tensors(ex):
    """Oracle-side expert (numpy, storage format) -> device tensors."""
    if ex.prec == oracle.BF16:
        return to_gpu_bf16(ex.w13), None, to_gpu_bf16(ex.w2), None
    return (torch.from_numpy(np.ascontiguousarray(ex.w13)).cuda(), to_gpu_f16(ex.s13),
            torch.from_numpy(np.ascontiguousarray(ex.w2)).cuda(), to_gpu_f16(ex.s2))


def gpu_layer(H, I, E, k, experts):
    from mixed_precision_moe_b200.binding import MoELayer
    layer = MoELayer(H, I, E, k)
    for e, ex in enumerate(experts):
        layer.set_expert(e, ex.prec, *gpu_expert_tensors(ex))
    return layer


def bf16_to_f64(t):
    return t.float().double().cpu().numpy()


def check_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    mean_rel = err.sum() / max(np.abs(ref).sum(), 1e-300)
    max_abs = err.max() if err.size else 0.0
    bound = MAX_ABS_TOL * (np.abs(ref).max() if ref.size else 0.0)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    assert mean_rel <= MEAN_REL_TOL, f"{what}: mean-relative error {mean_rel:.3e} > {MEAN_REL_TOL}"
    assert max_abs <= bound, f"{what}: max-abs error {max_abs:.3e} > {bound:.3e}"
    return mean_rel, max_abs
