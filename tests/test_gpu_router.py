"""The router projection fused with top-k (moe_router_topk) and the layer from
hidden states (moe_layer_forward_hidden) against the CPU oracle.

What the path computes: z_t = W_r h_t with bf16 operands (ExactMoE Section 3.1
routing equation; the router stays in BF16, Abstract), then the top-k of
Section 3.1 with ties to the lower expert id and the gating weights.  The
oracle computes z in binary64 from the same bf16 bits.

Tolerance of the logits, from the arithmetic: every bf16 x bf16 product is
exact in fp32, and the kernel sums them in fp32 on the tensor cores (four K=16
MMAs per 64-element k-block, then at most 16 partial sums of the cluster's K
split).  Counting two units of 2^-23 (relative to the sum of the products'
magnitudes) per MMA and one per partial sum gives
    |z_gpu - z| <= delta = (8 * H/64 + 16 + 2) * 2^-23 * sum_h |h_h W_eh|.
The top-k is an integer decision made in fp32 on the kernel's logits, so the
exact ids are compared where the oracle's logits decide them by more than the
tolerance, and elsewhere the selection must be a valid top-k of some logits
within delta of the oracle's: no selected expert may be beaten by an
unselected one, and no pick by a later pick, by more than the two deltas.
With small integer inputs every partial sum is exact, so there the logits, the
ids (ties included) and the weights are compared with the oracle directly.
"""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_moe_b200 import binding as B
from mixed_precision_moe_b200 import build, synth
from helpers import gpu_layer, oracle_experts, to_gpu_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    B.lib()
    B.moe_get_device_status()  # clear
    yield
    torch.cuda.synchronize()


def _delta(h_bits, w_bits):
    H = h_bits.shape[1]
    a = np.abs(synth.bf16_bits_to_f32(h_bits).astype(np.float64))
    b = np.abs(synth.bf16_bits_to_f32(w_bits).astype(np.float64))
    return (8 * (H // 64) + 18) * 2.0 ** -23 * (a @ b.T)


def _check_topk_valid(idx, w, zo, delta, k, renorm):
    """idx/w: the GPU's picks and weights; zo: oracle logits (binary64);
    delta: per-logit tolerance.  Returns the number of tokens whose top-k the
    oracle's logits decide unambiguously (there the ids must be equal)."""
    T, E = zo.shape
    decided = 0
    for t in range(T):
        p = idx[t]
        assert len(set(p.tolist())) == k and p.min() >= 0 and p.max() < E, f"token {t}: ids {p}"
        z, d = zo[t], delta[t]
        # order among the picks
        for j in range(k - 1):
            assert z[p[j]] - z[p[j + 1]] >= -(d[p[j]] + d[p[j + 1]]), f"token {t}: order {p}"
        # no unselected expert beats a pick by more than the tolerance
        rest = np.setdiff1d(np.arange(E), p)
        if rest.size:
            worst = p[np.argmin(z[p] + d[p])]
            assert np.all(z[rest] - d[rest] <= z[worst] + d[worst]), f"token {t}: set {p}"
        # the oracle's own top-k, and whether its margins exceed the tolerance
        order = sorted(range(E), key=lambda e: (-z[e], e))
        lo, hi = z - d, z + d
        sure = all(lo[order[j]] > hi[order[j + 1]] for j in range(k - 1))
        if k < E:
            sure = sure and lo[order[k - 1]] > np.max(hi[order[k:]])
        if sure:
            assert p.tolist() == order[:k], f"token {t}: {p} vs oracle {order[:k]}"
            decided += 1
        # weights: the oracle's softmax at the GPU's picks; a logit error of
        # delta moves each exp by at most e^(2 delta) and the sum likewise
        m = z[p[0]]
        ex = np.exp(z - m)
        den = ex[p].sum() if renorm else ex.sum()
        ref = ex[p] / den
        dmax = d.max()
        tol = ref * (np.expm1(4 * dmax) + (E + 8) * 2.0 ** -23) + 1e-7
        assert np.all(np.abs(w[t] - ref) <= tol), f"token {t}: weights {w[t]} vs {ref}"
    return decided


CASES = [
    # name, T, H, E, k, zipf_s, renormalize
    ("tiny", 64, 256, 8, 2, 0.0, True),
    ("qwen3_30b_decode", 32, 2048, 128, 8, 1.1, True),
    ("qwen3_30b_decode_full_softmax", 32, 2048, 128, 8, 1.1, False),
    ("qwen3_30b_prefill", 4096, 2048, 128, 8, 1.1, True),
    ("mixtral_t1", 1, 4096, 8, 2, 0.0, True),
    ("mixtral_t512", 512, 4096, 8, 2, 0.0, True),
    ("qwen3_80b_stack", 32, 2048, 512, 10, 1.2, True),
    ("ragged_e300_k16", 200, 384, 300, 16, 0.0, True),
    ("ragged_t129", 129, 2048, 128, 8, 1.1, True),
    ("single_expert", 3, 64, 1, 1, 0.0, True),
]


@pytest.mark.parametrize("name,T,H,E,k,zipf_s,renorm", CASES, ids=[c[0] for c in CASES])
def test_router_topk_against_oracle(name, T, H, E, k, zipf_s, renorm):
    hb, wb = synth.gen_router(T, H, E, 700 + T + E, zipf_s)
    h, wr = to_gpu_bf16(hb), to_gpu_bf16(wb)
    logits = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    idx, w = B.moe_router_topk(h, wr, k, renorm, logits=logits)
    torch.cuda.synchronize()
    assert B.moe_get_device_status() == 0

    zo = oracle.router_logits(hb, wb)
    delta = _delta(hb, wb)
    zg = logits.cpu().numpy().astype(np.float64)
    err = np.abs(zg - zo)
    assert np.all(err <= delta), f"{name}: logit error {err.max():.3e} (ratio {np.max(err / delta):.3f})"
    decided = _check_topk_valid(idx.cpu().numpy(), w.cpu().numpy().astype(np.float64), zo, delta,
                                k, renorm)
    # not vacuous: most tokens are decided by the oracle alone (>= 0.906 on every case here)
    assert decided >= 0.85 * T, f"{name}: only {decided} of {T} tokens decided by the oracle"

    # the fused top-k equals the separate routing kernel on the kernel's own logits
    idx2, w2 = B.moe_route_topk(logits, k, renorm)
    assert torch.equal(idx, idx2) and torch.equal(w, w2)
    # deterministic: the K split is summed in a fixed order
    logits3 = torch.empty_like(logits)
    idx3, w3 = B.moe_router_topk(h, wr, k, renorm, logits=logits3)
    assert torch.equal(logits3.view(torch.int32), logits.view(torch.int32))
    assert torch.equal(idx3, idx) and torch.equal(w3, w)


@pytest.mark.parametrize("T,H,E,k", [(64, 2048, 128, 8), (300, 512, 512, 10), (5, 4096, 8, 2),
                                     (130, 256, 16, 16)])
def test_router_integer_inputs_exact(T, H, E, k):
    """Small integers: every partial sum is exact, so the GPU logits equal the
    oracle's bit for bit, and the ids (with many exact ties, broken to the
    lower id) equal the oracle's top-k of those logits."""
    rng = np.random.default_rng(T + H + E)
    hb = synth.to_bf16_bits(rng.integers(-2, 3, (T, H)).astype(np.float32))
    wb = synth.to_bf16_bits(rng.integers(-1, 2, (E, H)).astype(np.float32))
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    idx, w = B.moe_router_topk(to_gpu_bf16(hb), to_gpu_bf16(wb), k, True, logits=logits)
    torch.cuda.synchronize()
    zo = oracle.router_logits(hb, wb)
    assert np.array_equal(logits.cpu().numpy().astype(np.float64), zo)
    idx_o, w_o = oracle.route_topk(zo.astype(np.float32), k)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert np.max(np.abs(w.cpu().numpy().astype(np.float64) - w_o)) <= 1e-6
    ties = sum(len(set(zo[t].tolist())) < E for t in range(T))
    assert ties > 0   # the case exercises the tie rule


def test_router_without_logits_output_and_empty_batch():
    hb, wb = synth.gen_router(40, 1024, 64, 9)
    h, wr = to_gpu_bf16(hb), to_gpu_bf16(wb)
    logits = torch.empty((40, 64), dtype=torch.float32, device="cuda")
    idx, w = B.moe_router_topk(h, wr, 6, logits=logits)
    idx2, w2 = B.moe_router_topk(h, wr, 6)
    assert torch.equal(idx, idx2) and torch.equal(w, w2)
    e_idx, e_w = B.moe_router_topk(h[:0], wr, 6)
    assert e_idx.shape == (0, 6)
    torch.cuda.synchronize()
    assert B.moe_get_device_status() == 0


@pytest.mark.parametrize("T", [32, 300])
def test_layer_forward_hidden_equals_forward_on_its_logits(T):
    """moe_layer_forward_hidden (router kernel, then the fused small-batch
    front for T <= 128 or the router's own top-k above) gives the buffers and
    output of moe_layer_forward on the logits it wrote, bit for bit; its logits
    are moe_router_topk's."""
    H, I, E, k = 2048, 768, 128, 8
    ranks = synth.zipf_ranks(E, 2)
    precs = synth.precision_map(ranks, synth.CONFIGS["qwen3_30b_decode"].tiers)
    exps = oracle_experts(H, I, precs, 2)
    layer = gpu_layer(H, I, E, k, exps)
    hb, wb = synth.gen_router(T, H, E, 800 + T, 1.1, ranks)
    x, wr = to_gpu_bf16(hb), to_gpu_bf16(wb)
    b1 = layer.alloc_buffers(T)
    out1 = layer.forward_hidden(x, wr, bufs=b1).clone()
    b2 = layer.alloc_buffers(T)
    out2 = layer.forward(b1["logits"], x, bufs=b2)
    torch.cuda.synchronize()
    lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
    B.moe_router_topk(x, wr, k, logits=lg)
    torch.cuda.synchronize()
    assert torch.equal(lg.view(torch.int32), b1["logits"].view(torch.int32))
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    for a, b in zip(b1["route"] + b1["permute"][:3], b2["route"] + b2["permute"][:3]):
        assert torch.equal(a, b)
    assert B.moe_get_device_status() == 0
    layer.close()
