"""The whole-layer entry point (moe_layer_forward, the call the benchmark times)
against the CPU oracle, buffer by buffer.

For T <= 128 moe_layer_forward runs routing, grouping and the row gather as one
fused kernel; for larger T the separate kernels.  Every intermediate it writes
is compared with the oracle: topk_idx, expert_offsets, perm_token, dest_row and
x_perm bit for bit (routing and permutation are exact by definition: ExactMoE
Section 3.1 routing equation with ties to the lower expert id, grouping of
Figure 1), topk_w within 1e-6, and the bf16 output within the layer tolerance.
The same buffers from the separate entry points (moe_route_topk, moe_permute)
must be identical too.
"""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_moe_b200 import binding as B
from mixed_precision_moe_b200 import build, synth
from helpers import bf16_to_f64, check_close, gpu_layer, oracle_experts, to_gpu_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    B.lib()
    B.moe_get_device_status()  # clear
    yield
    torch.cuda.synchronize()


def _bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _check_forward_buffers(layer, logits, x, k, renorm, exps=None, H=None, I=None, tokens=None):
    """Run layer.forward and compare every buffer it wrote with the oracle and
    with the separate entry points; returns the output (binary64)."""
    T, E = logits.shape
    lg, xg = torch.from_numpy(logits).cuda(), to_gpu_bf16(x)
    bufs = layer.alloc_buffers(T)
    for t in (bufs["route"][0], bufs["permute"][0], bufs["permute"][1], bufs["permute"][2]):
        t.fill_(-7)          # every element the call must write is overwritten
    out = layer.forward(lg, xg, renormalize=renorm, bufs=bufs)
    torch.cuda.synchronize()

    idx_o, w_o = oracle.route_topk(logits, k, renorm)
    off_o, perm_o, dest_o, inv = oracle.permute(idx_o, E)
    R = T * k
    assert inv == 0 and int(off_o[-1]) == R
    idx, w = bufs["route"]
    off, perm, dest, xp = bufs["permute"]
    assert np.array_equal(idx.cpu().numpy(), idx_o), "topk_idx"
    assert np.max(np.abs(w.cpu().numpy().astype(np.float64) - w_o)) <= 1e-6, "topk_w"
    assert np.array_equal(off.cpu().numpy(), off_o), "expert_offsets"
    assert np.array_equal(perm.cpu().numpy()[:R], perm_o[:R]), "perm_token"
    assert np.array_equal(dest.cpu().numpy(), dest_o), "dest_row"
    assert np.array_equal(_bits(xp), x[perm_o[:R]]), "x_perm"

    # the separate entry points give the same buffers, bit for bit
    idx2, w2 = B.moe_route_topk(lg, k, renorm)
    off2, perm2, dest2, xp2 = B.moe_permute(idx2, xg, E)
    assert torch.equal(idx2, idx) and torch.equal(w2, w)
    assert torch.equal(off2, off) and torch.equal(perm2[:R], perm[:R])
    assert torch.equal(dest2, dest) and torch.equal(xp2.view(torch.int16), xp.view(torch.int16))

    got = bf16_to_f64(out)
    if exps is not None:
        _, _, ref = oracle.moe_layer(logits, x, exps, k, H, I, renormalize=renorm, tokens=tokens)
        sel = np.arange(T) if tokens is None else tokens
        check_close(got[sel], ref, f"T={T} E={E} k={k} renorm={renorm}")
    assert B.moe_get_device_status() == 0
    return got


@pytest.mark.parametrize("renorm", [True, False])
def test_forward_qwen3_30b_decode_buffers(renorm):
    """The benchmark's headline workload exactly (H2048 I768 E128 top-8 T32,
    Zipf 1.1, 32 hottest BF16 + 96 INT4), through the fused front kernel."""
    cfg = synth.CONFIGS["qwen3_30b_decode"]
    ranks = synth.zipf_ranks(cfg.E, cfg.seed)
    precs = synth.precision_map(ranks, cfg.tiers)
    exps = oracle_experts(cfg.H, cfg.I, precs, cfg.seed)
    layer = gpu_layer(cfg.H, cfg.I, cfg.E, cfg.k, exps)
    for b in range(2):   # two of the benchmark's batches
        x = synth.gen_x(cfg.T, cfg.H, cfg.seed * 1000 + b)
        logits = synth.gen_logits(cfg.T, cfg.E, cfg.seed * 1000 + b, cfg.zipf_s, ranks)
        _check_forward_buffers(layer, logits, x, cfg.k, renorm, exps, cfg.H, cfg.I)
    layer.close()


def test_forward_tiny_buffers():
    cfg = synth.CONFIGS["tiny"]
    exps = oracle_experts(cfg.H, cfg.I, [oracle.INT4] * cfg.E, cfg.seed)
    layer = gpu_layer(cfg.H, cfg.I, cfg.E, cfg.k, exps)
    x = synth.gen_x(cfg.T, cfg.H, cfg.seed)
    logits = synth.gen_logits(cfg.T, cfg.E, cfg.seed)
    for renorm in (True, False):
        _check_forward_buffers(layer, logits, x, cfg.k, renorm, exps, cfg.H, cfg.I)
    layer.close()


# T at and around the fused kernel's limit (128) and the separate path above it;
# E up to 512, k up to 16.
SHAPES = [(1, 8, 2), (16, 128, 8), (32, 512, 10), (127, 64, 16), (128, 128, 8),
          (128, 512, 16), (129, 128, 8), (33, 300, 5), (96, 17, 16)]


@pytest.mark.parametrize("T,E,k", SHAPES)
def test_forward_buffers_shapes(T, E, k):
    H, I = 256, 256
    precs = [(oracle.INT4, oracle.BF16, oracle.INT8)[e % 3] for e in range(E)]
    exps = oracle_experts(H, I, precs, 600 + E)
    layer = gpu_layer(H, I, E, k, exps)
    x = synth.gen_x(T, H, 601 + T)
    logits = synth.gen_logits(T, E, 602 + T, 1.1)
    tokens = None if T <= 32 else np.unique(np.concatenate(
        [[0, T - 1], np.random.default_rng(T).choice(T, 12, replace=False)])).astype(np.int32)
    _check_forward_buffers(layer, logits, x, k, True, exps, H, I, tokens)
    layer.close()


@pytest.mark.parametrize("T,E,k", [(32, 64, 8), (128, 512, 16), (7, 16, 16)])
def test_forward_buffers_tied_logits(T, E, k):
    """Many equal logits (small integers) and signed zeros: the tie rule (lower
    id first) decides the top-k and the group order."""
    H, I = 256, 256
    exps = oracle_experts(H, I, [oracle.INT4] * E, 700 + E)
    layer = gpu_layer(H, I, E, k, exps)
    rng = np.random.default_rng(T + E)
    logits = rng.integers(-2, 3, (T, E)).astype(np.float32)
    logits[rng.random(logits.shape) < 0.3] = -0.0
    logits[0] = 0.0
    x = synth.gen_x(T, H, 703)
    for renorm in (True, False):
        _check_forward_buffers(layer, logits, x, k, renorm, exps, H, I)
    layer.close()


# ----------------------------------------------------------- row bounds --

def test_ffn_leaves_out_experts_whose_rows_exceed_the_buffers():
    """expert_offsets that reach past `rows`: the expert is skipped and flagged,
    nothing is written past y_perm's rows, the other experts are unchanged."""
    H, I, E = 256, 256, 3
    exps = oracle_experts(H, I, [oracle.INT4, oracle.BF16, oracle.INT8], 31)
    layer = gpu_layer(H, I, E, 1, exps)
    rows = 12
    x_perm = synth.gen_x(rows, H, 32)
    good = np.array([0, 4, 8, 12], np.int32)
    y_ref = B.moe_grouped_ffn_mixed(layer, to_gpu_bf16(x_perm), torch.from_numpy(good).cuda())
    B.moe_get_device_status()
    for bad in ([0, 4, 8, 20], [0, 4, -3, 12], [0, 9, 8, 12]):
        y_big = torch.full((rows + 8, H), 3.0, dtype=torch.bfloat16, device="cuda")
        B.moe_grouped_ffn_mixed(layer, to_gpu_bf16(x_perm), torch.tensor(bad, dtype=torch.int32,
                                                                         device="cuda"),
                                y_perm=y_big[:rows])
        st = B.moe_get_device_status()
        assert st & B.STATUS_BAD_ROW_INDEX, bad
        assert torch.all(y_big[rows:] == 3.0), "write past the rows"
        valid = [(bad[e], bad[e + 1]) for e in range(E) if 0 <= bad[e] <= bad[e + 1] <= rows]
        for e in range(E):
            # an expert with its good range that no other kept expert overlaps
            # matches the good run (overlapping kept ranges write the same rows)
            a, b = bad[e], bad[e + 1]
            alone = sum(1 for (c, d) in valid if c < b and a < d) == 1
            if (a, b) == (good[e], good[e + 1]) and alone:
                assert torch.equal(y_big[a:b].view(torch.int16), y_ref[a:b].view(torch.int16))
    layer.close()


def test_combine_skips_rows_past_the_buffer():
    T, k, H = 4, 2, 256
    y = to_gpu_bf16(synth.gen_x(T * k, H, 41))
    w = torch.full((T, k), 0.5, dtype=torch.float32, device="cuda")
    dest = torch.arange(T * k, dtype=torch.int32, device="cuda").view(T, k).contiguous()
    ref = B.moe_combine(y, dest, w)
    dest_bad = dest.clone()
    dest_bad[1, 1] = T * k + 100
    out = B.moe_combine(y, dest_bad, w)
    assert B.moe_get_device_status() & B.STATUS_BAD_ROW_INDEX
    mask = torch.ones(T, dtype=torch.bool)
    mask[1] = False
    assert torch.equal(out[mask.cuda()].view(torch.int16), ref[mask.cuda()].view(torch.int16))
    # token 1 keeps only its first pair: 0.5 * y[2] (exact in fp32), one rounding
    only = (0.5 * y[2].float()).to(torch.bfloat16)
    assert torch.equal(out[1].view(torch.int16), only.view(torch.int16))


# ------------------------------------------------------------ wave split --

@pytest.mark.parametrize("renorm", [False, True])
@pytest.mark.parametrize("cfg_name,waves", [("tiny", 2), ("tiny", 4), ("qwen3_30b_decode", 4)])
def test_wave_split_execution_matches_oracle(cfg_name, waves, renorm):
    """ExactMoE Section 3.4: with fewer resident slots than experts, the experts
    run in waves; each wave's grouped FFN covers only its experts, the router
    weights are kept (not renormalised within a wave) and the wave outputs are
    summed.  Here each wave is one FFN launch whose expert_offsets give rows
    only to the wave's experts (a contiguous id range), followed by a combine
    over the wave's pairs; the sum over waves is compared with the whole layer
    of the oracle."""
    cfg = synth.CONFIGS[cfg_name]
    ranks = synth.zipf_ranks(cfg.E, cfg.seed)
    precs = synth.precision_map(ranks, cfg.tiers)
    exps = oracle_experts(cfg.H, cfg.I, precs, cfg.seed)
    layer = gpu_layer(cfg.H, cfg.I, cfg.E, cfg.k, exps)
    x = synth.gen_x(cfg.T, cfg.H, cfg.seed + 5)
    logits = synth.gen_logits(cfg.T, cfg.E, cfg.seed + 5, cfg.zipf_s, ranks)
    idx, w = B.moe_route_topk(torch.from_numpy(logits).cuda(), cfg.k, renorm)
    off, perm, dest, xp = B.moe_permute(idx, to_gpu_bf16(x), cfg.E)
    bounds = np.linspace(0, cfg.E, waves + 1).astype(int)
    total = np.zeros((cfg.T, cfg.H), np.float64)
    neg = torch.full_like(dest, -1)
    for a, b in zip(bounds[:-1], bounds[1:]):
        off_w = torch.clamp(off, min=int(off[a]), max=int(off[b])).contiguous()
        y_w = B.moe_grouped_ffn_mixed(layer, xp, off_w)
        in_wave = (idx >= int(a)) & (idx < int(b))
        total += bf16_to_f64(B.moe_combine(y_w, torch.where(in_wave, dest, neg), w))
    _, _, ref = oracle.moe_layer(logits, x, exps, cfg.k, cfg.H, cfg.I, renormalize=renorm)
    check_close(total, ref, f"{cfg_name} in {waves} waves")
    assert B.moe_get_device_status() == 0
    layer.close()
