"""GPU path (through the C ABI) against the CPU oracle.

Standards: routing indices and the permutation bit-exact; the quantiser's codes
and scales bit-exact; gating weights within 1e-6; the bf16 layer output within
mean-relative 5e-3 and max-abs 1e-2 * max|oracle| of the binary64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_moe_b200 import binding as B
from mixed_precision_moe_b200 import build, synth
from helpers import bf16_to_f64, check_close, gpu_expert_tensors, gpu_layer, oracle_experts, \
    to_gpu_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    B.lib()
    B.moe_get_device_status()  # clear
    yield
    torch.cuda.synchronize()


def _status():
    return B.moe_get_device_status()


# ------------------------------------------------------------------ routing --

ROUTE_CASES = [(64, 8, 2, 0.0), (32, 128, 8, 1.1), (4096, 128, 8, 1.1), (32, 512, 10, 1.2),
               (7, 33, 16, 0.0), (1, 1, 1, 0.0), (300, 64, 8, 0.0), (5, 512, 16, 0.0)]


@pytest.mark.parametrize("T,E,k,zipf", ROUTE_CASES)
@pytest.mark.parametrize("renorm", [True, False])
def test_route_matches_oracle(T, E, k, zipf, renorm):
    logits = synth.gen_logits(T, E, 100 + T + E, zipf)
    idx_o, w_o = oracle.route_topk(logits, k, renorm)
    idx_g, w_g = B.moe_route_topk(torch.from_numpy(logits).cuda(), k, renorm)
    assert np.array_equal(idx_g.cpu().numpy(), idx_o)
    assert np.max(np.abs(w_g.cpu().numpy().astype(np.float64) - w_o)) <= 1e-6
    assert _status() == 0


def test_route_ties_and_signed_zero():
    rng = np.random.default_rng(9)
    for E, k in [(8, 3), (64, 8), (128, 16), (512, 10)]:
        z = rng.integers(-2, 3, (257, E)).astype(np.float32)
        z[rng.random(z.shape) < 0.3] = -0.0
        z[0] = 0.0
        z[1] = -0.0
        idx_o, w_o = oracle.route_topk(z, k)
        idx_g, w_g = B.moe_route_topk(torch.from_numpy(z).cuda(), k)
        assert np.array_equal(idx_g.cpu().numpy(), idx_o)
        assert list(idx_o[0]) == list(range(k)) and list(idx_o[1]) == list(range(k))
        assert np.max(np.abs(w_g.cpu().numpy() - w_o)) <= 1e-6


def test_route_k_equals_e_and_infinities():
    z = np.array([[1.0, -np.inf, 3.0, 2.0], [-np.inf, -np.inf, 0.0, -np.inf]], np.float32)
    idx, w = B.moe_route_topk(torch.from_numpy(z).cuda(), 4)
    assert idx.cpu().tolist() == [[2, 3, 0, 1], [2, 0, 1, 3]]
    w = w.cpu().numpy()
    assert w[1, 0] == 1.0 and np.all(w[1, 1:] == 0.0) and w[0, 3] == 0.0
    assert _status() == 0


def test_route_nan_is_ordered_last_and_flagged():
    z = np.array([[0.5, np.nan, -1.0, 2.0]], np.float32)
    idx, w = B.moe_route_topk(torch.from_numpy(z).cuda(), 3)
    assert idx.cpu().tolist() == [[3, 0, 2]]
    assert _status() & B.STATUS_NONFINITE_LOGIT


# -------------------------------------------------------------- permutation --

# T > 512 takes the grouping split over CTAs of 256 tokens (ragged last chunk included)
@pytest.mark.parametrize("T,E,k", [(64, 8, 2), (32, 128, 8), (4096, 128, 8), (32, 512, 10),
                                   (1, 1, 1), (1000, 16, 16), (33, 300, 5), (2049, 300, 5),
                                   (513, 512, 1)])
def test_permute_bit_exact(T, E, k):
    H = 256
    logits = synth.gen_logits(T, E, 200 + T, 1.1)
    idx, _ = oracle.route_topk(logits, k)
    off_o, perm_o, dest_o, inv = oracle.permute(idx, E)
    x = synth.gen_x(T, H, 201)
    off, perm, dest, xp = B.moe_permute(torch.from_numpy(idx).cuda(), to_gpu_bf16(x), E)
    R = int(off_o[-1])
    assert inv == 0 and R == T * k
    assert np.array_equal(off.cpu().numpy(), off_o)
    assert np.array_equal(perm.cpu().numpy()[:R], perm_o[:R])
    assert np.array_equal(dest.cpu().numpy(), dest_o)
    xp_bits = xp.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(xp_bits, x[perm_o])
    assert _status() == 0


@pytest.mark.parametrize("T", [40, 1300])   # one CTA, split over CTAs
def test_permute_invalid_and_repeated_ids(T):
    E, k, H = 6, 3, 128
    rng = np.random.default_rng(3)
    idx = rng.integers(-2, E + 2, (T, k)).astype(np.int32)
    idx[5] = [1, 1, 2]
    off_o, perm_o, dest_o, inv = oracle.permute(idx, E)
    assert inv > 0
    x = synth.gen_x(T, H, 5)
    off, perm, dest, xp = B.moe_permute(torch.from_numpy(idx).cuda(), to_gpu_bf16(x), E)
    R = int(off_o[-1])
    assert np.array_equal(off.cpu().numpy(), off_o)
    assert np.array_equal(perm.cpu().numpy()[:R], perm_o[:R])
    assert np.array_equal(dest.cpu().numpy(), dest_o)
    assert _status() & B.STATUS_BAD_EXPERT_ID


def test_permute_no_tokens():
    off = torch.full((9,), 7, dtype=torch.int32, device="cuda")
    idx = torch.empty((0, 2), dtype=torch.int32, device="cuda")
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    B.moe_permute(idx, x, 8, (off, torch.empty(1, dtype=torch.int32, device="cuda"),
                             torch.empty((0, 2), dtype=torch.int32, device="cuda"),
                             torch.empty((1, 128), dtype=torch.bfloat16, device="cuda")))
    assert off.cpu().tolist() == [0] * 9


# ---------------------------------------------------------------- quantiser --

@pytest.mark.parametrize("prec", [oracle.INT8, oracle.INT4])
def test_quantiser_bit_exact(prec):
    rows, K = 384, 1024
    rng = np.random.default_rng(40 + prec)
    W = rng.standard_normal((rows, K)).astype(np.float32) * np.float32(0.02)
    W[0] = 0.0                                   # all-zero groups
    W[1, :128] = -0.3                            # a group of only -amax
    W[2, 128:256] = 1e-9                         # scale underflows fp16
    W[3] *= 1e4                                  # large values
    W[4, ::7] = 0.5 * 2.0 ** -20                 # subnormal-range scales
    bits = synth.to_bf16_bits(W)
    q_o, s_o = oracle.quantize(bits, prec)
    q_g, s_g = B.moe_quantize_weights(to_gpu_bf16(bits), prec)
    assert np.array_equal(q_g.cpu().numpy().view(np.uint8), q_o.view(np.uint8))
    assert np.array_equal(s_g.cpu().view(torch.int16).numpy().view(np.uint16), s_o)


# ------------------------------------------------------------------ combine --

def test_combine_matches_oracle_and_skips_missing_pairs():
    T, k, H = 50, 8, 512
    R = T * k
    rng = np.random.default_rng(11)
    y = synth.gen_x(R, H, 12)
    dest = rng.permutation(R).astype(np.int32).reshape(T, k)
    dest[3, 2] = -1
    w = rng.random((T, k)).astype(np.float32)
    ref = oracle.combine(synth.bf16_bits_to_f32(y).astype(np.float64), dest, w.astype(np.float64))
    out = B.moe_combine(to_gpu_bf16(y), torch.from_numpy(dest).cuda(), torch.from_numpy(w).cuda())
    got = bf16_to_f64(out)
    # fp32 accumulation of k terms, one bf16 rounding
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)


# ---------------------------------------------------------- grouped FFN ----

FFN_GROUPS = [1, 3, 16, 17, 64, 127, 128, 129, 200, 256, 0, 300]


def _mode_k(mode, groups):
    """The library picks the MMA orientation from T = ceil(rows / k): weights-as-M
    ("swap") when T <= 128, tokens-as-M ("tile") otherwise."""
    R, E = sum(groups), len(groups)
    if mode == "swap":
        assert -(-R // E) <= 128
        return E
    assert R > 128
    return 1


def _ffn_case(H, I, precs, groups, seed, random_codes=False):
    E = len(groups)
    exps = oracle_experts(H, I, precs, seed)
    if random_codes:   # arbitrary codes, including INT4 q = -8 and INT8 q = -128
        for e, ex in enumerate(exps):
            if ex.prec != oracle.BF16:
                ex.w13, ex.s13 = synth.gen_random_codes(2 * I, H, ex.prec, seed, 2 * e)
                ex.w2, ex.s2 = synth.gen_random_codes(H, I, ex.prec, seed, 2 * e + 1)
    offsets = np.concatenate([[0], np.cumsum(groups)]).astype(np.int32)
    R = int(offsets[-1])
    x_perm = synth.gen_x(R, H, seed + 1)
    y_o = oracle.grouped_ffn(x_perm, offsets, exps, H, I)
    return exps, offsets, x_perm, y_o


@pytest.mark.parametrize("mode", ["swap", "tile"])
@pytest.mark.parametrize("H,I", [(512, 384), (384, 256)])
def test_grouped_ffn_mixed_precisions_ragged_groups(mode, H, I):
    precs = [oracle.BF16, oracle.INT8, oracle.INT4] * 4
    exps, offsets, x_perm, y_o = _ffn_case(H, I, precs, FFN_GROUPS, 50 + H)
    E = len(FFN_GROUPS)
    layer = gpu_layer(H, I, E, _mode_k(mode, FFN_GROUPS), exps)
    y = B.moe_grouped_ffn_mixed(layer, to_gpu_bf16(x_perm), torch.from_numpy(offsets).cuda())
    y = bf16_to_f64(y)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            check_close(y[a:b], y_o[a:b], f"expert {e} prec {precs[e]} rows {b - a}")
    check_close(y, y_o, "all rows")
    assert _status() == 0
    layer.close()


@pytest.mark.parametrize("mode", ["swap", "tile"])
def test_grouped_ffn_arbitrary_codes(mode):
    H, I = 256, 256
    groups = [5, 128, 33, 0, 77, 1]
    precs = [oracle.INT4, oracle.INT8, oracle.INT4, oracle.INT8, oracle.INT8, oracle.INT4]
    exps, offsets, x_perm, y_o = _ffn_case(H, I, precs, groups, 77, random_codes=True)
    layer = gpu_layer(H, I, len(groups), _mode_k(mode, groups), exps)
    y = B.moe_grouped_ffn_mixed(layer, to_gpu_bf16(x_perm), torch.from_numpy(offsets).cuda())
    check_close(bf16_to_f64(y), y_o, "arbitrary codes")
    layer.close()


@pytest.mark.parametrize("mode", ["swap", "tile"])
def test_grouped_equals_per_expert_launch_bit_for_bit(mode):
    H, I = 256, 256
    groups = [40, 0, 129, 7, 64]
    precs = [oracle.INT4, oracle.BF16, oracle.INT8, oracle.BF16, oracle.INT4]
    exps, offsets, x_perm, _ = _ffn_case(H, I, precs, groups, 91)
    E = len(groups)
    layer = gpu_layer(H, I, E, _mode_k(mode, groups), exps)
    xg = to_gpu_bf16(x_perm)
    y1 = B.moe_grouped_ffn_mixed(layer, xg, torch.from_numpy(offsets).cuda())
    y2 = B.moe_grouped_ffn_mixed(layer, xg, torch.from_numpy(offsets).cuda())
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), "not deterministic"
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b == a:
            continue
        solo = np.where(np.arange(E + 1) <= e, a, b).astype(np.int32)   # only expert e has rows
        ys = B.moe_grouped_ffn_mixed(layer, xg, torch.from_numpy(solo).cuda())
        assert torch.equal(ys[a:b].view(torch.int16), y1[a:b].view(torch.int16)), f"expert {e}"
    layer.close()


def test_unset_expert_is_rejected():
    layer = B.MoELayer(256, 256, 4, 2)
    ex = oracle_experts(256, 256, [oracle.INT4] * 3, 5)
    for e in range(3):
        layer.set_expert(e, ex[e].prec, *gpu_expert_tensors(ex[e]))
    xp = torch.zeros((8, 256), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 2, 4, 6, 8], dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError) as ei:
        B.moe_grouped_ffn_mixed(layer, xp, off)
    assert ei.value.code == -3
    assert layer.precision(3) == -1 and layer.precision(0) == oracle.INT4
    layer.close()


# -------------------------------------------------------------- whole layer --

def _run_layer(layer, logits, x, k, renorm=True):
    idx, w = B.moe_route_topk(torch.from_numpy(logits).cuda(), k, renorm)
    off, perm, dest, xp = B.moe_permute(idx, to_gpu_bf16(x), layer.E)
    y = B.moe_grouped_ffn_mixed(layer, xp, off)
    out = B.moe_combine(y, dest, w)
    return idx.cpu().numpy(), off.cpu().numpy(), bf16_to_f64(out)


def _layer_parity(cfg, tokens=None, masters=None):
    ranks = synth.zipf_ranks(cfg.E, cfg.seed)
    precs = synth.precision_map(ranks, cfg.tiers)
    exps = oracle_experts(cfg.H, cfg.I, precs, cfg.seed, masters)
    x = synth.gen_x(cfg.T, cfg.H, cfg.seed)
    logits = synth.gen_logits(cfg.T, cfg.E, cfg.seed, cfg.zipf_s, ranks)
    layer = gpu_layer(cfg.H, cfg.I, cfg.E, cfg.k, exps)
    idx_g, off_g, out_g = _run_layer(layer, logits, x, cfg.k)
    idx_o, w_o, out_o = oracle.moe_layer(logits, x, exps, cfg.k, cfg.H, cfg.I, tokens=tokens)
    assert np.array_equal(idx_g, idx_o)
    assert np.array_equal(off_g, oracle.permute(idx_o, cfg.E)[0])
    sel = np.arange(cfg.T) if tokens is None else tokens
    check_close(out_g[sel], out_o, cfg.name)
    assert _status() == 0
    layer.close()


def test_layer_tiny():
    _layer_parity(synth.CONFIGS["tiny"])


def test_layer_qwen3_30b_decode():
    _layer_parity(synth.CONFIGS["qwen3_30b_decode"])


def test_layer_qwen3_30b_prefill_sampled_tokens():
    cfg = synth.CONFIGS["qwen3_30b_prefill"]
    rng = np.random.default_rng(0)
    tokens = np.unique(np.concatenate([np.arange(8), cfg.T - 8 + np.arange(8),
                                       rng.choice(cfg.T, 32, replace=False)])).astype(np.int32)
    _layer_parity(cfg, tokens)


@pytest.fixture(scope="module")
def mixtral_experts():
    cfg = synth.mixtral_config(1)
    masters = [synth.gen_expert_master(cfg.H, cfg.I, 40, e) for e in range(cfg.E)]
    exps = oracle_experts(cfg.H, cfg.I, [oracle.INT4] * cfg.E, 40, masters)
    del masters
    layer = gpu_layer(cfg.H, cfg.I, cfg.E, cfg.k, exps)
    yield exps, layer
    layer.close()


@pytest.mark.parametrize("T", synth.MIXTRAL_BATCHES)
def test_layer_mixtral_batch_sweep(mixtral_experts, T):
    exps, layer = mixtral_experts
    cfg = synth.mixtral_config(T)
    x = synth.gen_x(T, cfg.H, cfg.seed)
    logits = synth.gen_logits(T, cfg.E, cfg.seed)
    tokens = None if T <= 8 else np.unique(np.concatenate(
        [[0, T - 1], np.random.default_rng(T).choice(T, 10, replace=False)])).astype(np.int32)
    idx_g, off_g, out_g = _run_layer(layer, logits, x, cfg.k)
    idx_o, w_o, out_o = oracle.moe_layer(logits, x, exps, cfg.k, cfg.H, cfg.I, tokens=tokens)
    assert np.array_equal(idx_g, idx_o)
    sel = np.arange(T) if tokens is None else tokens
    check_close(out_g[sel], out_o, cfg.name)
    assert _status() == 0


def test_wave_split_sums_to_whole_layer():
    cfg = synth.CONFIGS["tiny"]
    exps = oracle_experts(cfg.H, cfg.I, [oracle.INT4] * cfg.E, 7)
    layer = gpu_layer(cfg.H, cfg.I, cfg.E, cfg.k, exps)
    x = to_gpu_bf16(synth.gen_x(cfg.T, cfg.H, 7))
    idx, w = B.moe_route_topk(torch.from_numpy(synth.gen_logits(cfg.T, cfg.E, 7)).cuda(), cfg.k)
    off, perm, dest, xp = B.moe_permute(idx, x, cfg.E)
    y = B.moe_grouped_ffn_mixed(layer, xp, off)
    wave = idx < cfg.E // 2          # experts 0..3 in wave A, 4..7 in wave B
    neg = torch.full_like(dest, -1)
    whole = bf16_to_f64(B.moe_combine(y, dest, w))
    a = bf16_to_f64(B.moe_combine(y, torch.where(wave, dest, neg), w))
    b = bf16_to_f64(B.moe_combine(y, torch.where(wave, neg, dest), w))
    # each of a, b, whole carries one bf16 rounding (<= 2^-9 relative to itself)
    # on top of an fp32 sum; the partial sums may be larger than their total
    assert np.all(np.abs(a + b - whole) <= 2.0 ** -8 * (np.abs(a) + np.abs(b) + np.abs(whole)) + 1e-6)
    layer.close()


def test_handle_swap_is_stream_ordered():
    H, I, E, k, T = 256, 256, 4, 2, 16
    masters = [synth.gen_expert_master(H, I, 8, e) for e in range(E)]
    low = oracle_experts(H, I, [oracle.INT4] * E, 8, masters)
    high = oracle_experts(H, I, [oracle.BF16] * E, 8, masters)
    layer = gpu_layer(H, I, E, k, low)
    x = synth.gen_x(T, H, 8)
    logits = synth.gen_logits(T, E, 8)
    lg, xg = torch.from_numpy(logits).cuda(), to_gpu_bf16(x)
    bufs1, bufs2 = layer.alloc_buffers(T), layer.alloc_buffers(T)
    out1 = layer.forward(lg, xg, bufs=bufs1)                 # enqueued before the swap
    for e in (0, 2):
        layer.set_expert(e, oracle.BF16, *gpu_expert_tensors(high[e]))
    out2 = layer.forward(lg, xg, bufs=bufs2)                 # enqueued after the swap
    torch.cuda.synchronize()
    mixed = [high[0], low[1], high[2], low[3]]
    _, _, ref1 = oracle.moe_layer(logits, x, low, k, H, I)
    _, _, ref2 = oracle.moe_layer(logits, x, mixed, k, H, I)
    check_close(bf16_to_f64(out1), ref1, "before swap")
    check_close(bf16_to_f64(out2), ref2, "after swap")
    assert layer.precision(0) == oracle.BF16 and layer.precision(1) == oracle.INT4
    layer.close()


def test_grouped_ffn_cuda_core_units_against_oracle():
    """INT8/INT4 experts of one or two rows whose projections span at least 16
    CUDA-core stages (K = 4224: INT4 stages of 256 K-elements, the last one half
    past K, read as zeros) are computed on CUDA cores from the codes; an INT4
    expert of three rows (tensor core) and a BF16 expert share the launch.
    Arbitrary codes (INT4 -8, INT8 -128) and quantiser codes; every expert's
    rows equal its own launch bit for bit."""
    H = I = 4224
    groups = [1, 2, 2, 1, 2, 3, 1]
    precs = [oracle.INT4, oracle.INT8, oracle.INT4, oracle.INT8, oracle.BF16, oracle.INT4,
             oracle.INT4]
    exps, offsets, x_perm, y_o = _ffn_case(H, I, precs, groups, 4224)
    for e in (2, 3):   # arbitrary codes for two of the CUDA-core experts
        ex = exps[e]
        ex.w13, ex.s13 = synth.gen_random_codes(2 * I, H, ex.prec, 4224, 2 * e)
        ex.w2, ex.s2 = synth.gen_random_codes(H, I, ex.prec, 4224, 2 * e + 1)
    y_o = oracle.grouped_ffn(x_perm, offsets, exps, H, I)
    E = len(groups)
    layer = gpu_layer(H, I, E, E, exps)   # k = E: T = 2 tokens, swap orientation
    xg = to_gpu_bf16(x_perm)
    off = torch.from_numpy(offsets).cuda()
    y = B.moe_grouped_ffn_mixed(layer, xg, off)
    y64 = bf16_to_f64(y)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        check_close(y64[a:b], y_o[a:b], f"expert {e} prec {precs[e]} rows {b - a}")
        solo = np.where(np.arange(E + 1) <= e, a, b).astype(np.int32)
        ys = B.moe_grouped_ffn_mixed(layer, xg, torch.from_numpy(solo).cuda())
        assert torch.equal(ys[a:b].view(torch.int16), y[a:b].view(torch.int16)), f"expert {e}"
    assert _status() == 0
    layer.close()
