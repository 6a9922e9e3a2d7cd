"""Pins for the CPU oracle against things other than itself.

Each test checks an oracle function against brute force, a closed form, an
invariant or an independent library routine (numpy / torch / scipy), so that a
plausible mistake in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a wrong tie-break or nibble order) fails one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from mixed_precision_moe_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- formats --

def test_fp16_to_double_matches_numpy_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.fp16_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_fp16_from_float_matches_numpy_rne():
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * np.float32(1e-3),
        (rng.standard_normal(4000) * 2.0 ** rng.integers(-30, 17, 4000)).astype(np.float32),
        # exact ties between fp16 neighbours (normal and subnormal ranges)
        (np.arange(1, 600, dtype=np.float64) * 2.0 ** -25).astype(np.float32),
        (1.0 + (2 * np.arange(0, 300) + 1) * 2.0 ** -11).astype(np.float32),
        np.array([65504, 65519.99, 65520, 7e4, 0.0, -0.0, 2 ** -24, 2 ** -25, 3 * 2 ** -26],
                 dtype=np.float32),
    ])
    ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.fp16_from_float(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_to_double_matches_torch():
    rng = np.random.default_rng(8)
    bits = rng.integers(0, 65536, 5000).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]  # finite only
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([oracle.bf16_to_double(int(b)) for b in bits])
    assert np.array_equal(got, ref)


# ------------------------------------------------------- router projection --

def _bf16_bits(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def _bf16_values(bits):
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16) \
        .double().numpy()


@pytest.mark.parametrize("T,H,E", [(5, 256, 8), (33, 384, 128), (3, 2048, 17), (0, 128, 4)])
def test_router_logits_match_numpy_fp64_matmul(T, H, E):
    # z = W_r h (routing equation): numpy's fp64 product of the bf16 values;
    # the products are exact, only the summation order differs
    rng = np.random.default_rng(T * 1000 + E)
    h = _bf16_bits(rng.standard_normal((T, H)))
    wr = _bf16_bits(rng.standard_normal((E, H)) * 0.02)
    z = oracle.router_logits(h, wr)
    ref = _bf16_values(h) @ _bf16_values(wr).T
    assert z.shape == (T, E)
    bound = H * 2.0 ** -52 * (np.abs(_bf16_values(h)) @ np.abs(_bf16_values(wr)).T)
    assert np.all(np.abs(z - ref) <= bound)


def test_router_one_hot_rows_select_hidden_entries():
    # row e of W_r = unit vector at column j_e  =>  z[t][e] = h[t][j_e] exactly
    rng = np.random.default_rng(3)
    T, H, E = 7, 256, 16
    h = _bf16_bits(rng.standard_normal((T, H)))
    cols = rng.permutation(H)[:E]
    w = np.zeros((E, H), np.float32)
    w[np.arange(E), cols] = 1.0
    z = oracle.router_logits(h, _bf16_bits(w))
    assert np.array_equal(z, _bf16_values(h)[:, cols])


def test_router_integer_inputs_are_exact_and_tie():
    # small integers: every partial sum is an exact integer, checked against
    # Python's own integer arithmetic; the ties this produces are then broken
    # to the lower id by the top-k
    rng = np.random.default_rng(4)
    T, H, E = 6, 128, 12
    hi = rng.integers(-2, 3, (T, H))
    wi = rng.integers(-1, 2, (E, H))
    wi[5] = wi[2]                      # experts 2 and 5 tie on every token
    z = oracle.router_logits(_bf16_bits(hi), _bf16_bits(wi))
    exact = np.array([[sum(int(a) * int(b) for a, b in zip(hi[t], wi[e])) for e in range(E)]
                      for t in range(T)])
    assert np.array_equal(z, exact.astype(np.float64))
    idx, _ = oracle.route_topk(z.astype(np.float32), E)
    for t in range(T):
        order = idx[t].tolist()
        assert order.index(2) < order.index(5)


# ---------------------------------------------------------------- routing --

def _brute_topk(z, k):
    # full sort of (-z, id): IEEE equality makes -0.0 == +0.0
    return [e for _, e in sorted((-float(v), e) for e, v in enumerate(z))][:k]


@pytest.mark.parametrize("E,k", [(1, 1), (2, 1), (3, 3), (8, 2), (16, 5), (16, 16), (64, 8)])
def test_topk_matches_bruteforce_sort(E, k):
    rng = np.random.default_rng(E * 100 + k)
    # many ties: small integer logits, plus signed zeros
    z = rng.integers(-3, 4, (200, E)).astype(np.float32)
    z[rng.random((200, E)) < 0.2] = -0.0
    z[:50] = rng.standard_normal((50, E)).astype(np.float32)
    idx, _ = oracle.route_topk(z, k)
    for t in range(z.shape[0]):
        assert list(idx[t]) == _brute_topk(z[t], k)


def test_topk_special_rows():
    E, k = 8, 3
    z = np.zeros((3, E), np.float32)
    z[1] = -0.0
    z[2, [5, 6]] = 2.0
    idx, w = oracle.route_topk(z, k)
    assert list(idx[0]) == [0, 1, 2]          # all equal -> lowest ids
    assert list(idx[1]) == [0, 1, 2]          # -0.0 == +0.0
    assert list(idx[2]) == [5, 6, 0]
    assert np.allclose(w[0], 1.0 / 3, rtol=0, atol=1e-15)
    full, _ = oracle.route_topk(np.random.default_rng(1).standard_normal((4, E)).astype(np.float32), E)
    for row in full:
        assert sorted(row) == list(range(E))  # k = E -> a permutation


def test_topk_rejects_nonfinite():
    z = np.zeros((2, 4), np.float32)
    z[1, 2] = np.nan
    with pytest.raises(RuntimeError):
        oracle.route_topk(z, 2)


def test_gating_weights_invariants_and_closed_forms():
    rng = np.random.default_rng(3)
    z = (rng.standard_normal((300, 32)) * 3).astype(np.float32)
    for k in (1, 2, 4, 8):
        idx, w = oracle.route_topk(z, k)
        assert np.all(np.abs(w.sum(1) - 1.0) <= k * 2.0 ** -52 * 4)
        assert np.all(np.diff(w, axis=1) <= 0)               # descending with the logits
        if k == 1:
            assert np.all(w == 1.0)
        if k == 2:                                          # w0 = sigmoid(z0 - z1)
            zs = np.take_along_axis(z, idx, 1).astype(np.float64)
            ref = torch.sigmoid(torch.from_numpy(zs[:, 0] - zs[:, 1])).numpy()
            assert np.allclose(w[:, 0], ref, rtol=1e-14, atol=0)


def test_unrenormalised_weights_are_full_softmax():
    from scipy.special import softmax
    rng = np.random.default_rng(4)
    z = rng.standard_normal((100, 16)).astype(np.float32)
    idx, w = oracle.route_topk(z, 4, renormalize=False)
    full = softmax(z.astype(np.float64), axis=1)
    assert np.allclose(w, np.take_along_axis(full, idx, 1), rtol=1e-13, atol=0)
    _, wr = oracle.route_topk(z, 4, renormalize=True)
    assert np.allclose(w / w.sum(1, keepdims=True), wr, rtol=1e-13, atol=0)


# ------------------------------------------------------------ permutation --

def test_permute_invariants_and_bruteforce():
    rng = np.random.default_rng(5)
    for T, E, k in [(1, 1, 1), (7, 4, 2), (64, 8, 2), (33, 16, 5), (50, 64, 8)]:
        z = rng.standard_normal((T, E)).astype(np.float32)
        idx, _ = oracle.route_topk(z, k)
        off, perm_token, dest, inv = oracle.permute(idx, E)
        assert inv == 0 and off[0] == 0 and off[E] == T * k
        assert np.all(np.diff(off) >= 0)
        # brute force: rows of expert e are the tokens choosing e, ascending
        expect = []
        for e in range(E):
            toks = [t for t in range(T) for j in range(k) if idx[t, j] == e]
            assert off[e + 1] - off[e] == len(toks)
            expect += toks
        assert list(perm_token) == expect
        for t in range(T):
            for j in range(k):
                r = dest[t, j]
                assert perm_token[r] == t and off[idx[t, j]] <= r < off[idx[t, j] + 1]
        assert sorted(dest.ravel()) == list(range(T * k))   # bijection


def test_permute_marks_invalid_ids():
    idx = np.array([[0, 5], [-1, 1], [1, 1]], np.int32)
    off, perm_token, dest, inv = oracle.permute(idx, 2)
    assert inv == 3 and list(off) == [0, 1, 3]
    assert dest[0, 1] == -1 and dest[1, 0] == -1 and dest[2, 1] == -1
    assert list(perm_token[:3]) == [0, 1, 2] and list(dest[:, 0]) == [0, -1, 2]


# ------------------------------------------------------------- quantiser --

def _exact_groups(rows, K, prec, rng):
    """W = s * q exactly representable in bf16, each group holding |q| = Q."""
    Q = 7 if prec == oracle.INT4 else 127
    q = rng.integers(-Q, Q + 1, (rows, K))
    q[:, ::128] = Q * rng.choice([-1, 1], (rows, K // 128))
    if prec == oracle.INT4:   # s with <= 5 significant bits: 7 s fits bf16's 8
        s = (rng.integers(16, 32, (rows, K // 128)) * 2.0 ** rng.integers(-14, -8, (rows, K // 128)))
    else:                     # power of two: 127 s fits bf16's 8 bits
        s = 2.0 ** rng.integers(-14, -6, (rows, K // 128)).astype(np.float64)
    W = q * np.repeat(s, 128, axis=1)
    bits = synth.to_bf16_bits(W.astype(np.float32))
    assert np.array_equal(synth.bf16_bits_to_f32(bits).astype(np.float64), W)
    return bits, q, s


@pytest.mark.parametrize("prec", [oracle.INT4, oracle.INT8])
def test_quantiser_exact_round_trip(prec):
    rng = np.random.default_rng(11 + prec)
    rows, K = 40, 512
    bits, q, s = _exact_groups(rows, K, prec, rng)
    codes, scales = oracle.quantize(bits, prec)
    got_s = scales.view(np.float16).astype(np.float64).T          # [rows, K/128]
    assert np.array_equal(got_s, s)
    W = oracle.dequantize(prec, codes, scales, rows, K)
    assert np.array_equal(W, synth.bf16_bits_to_f32(bits).astype(np.float64))
    if prec == oracle.INT8:
        assert np.array_equal(codes.astype(np.int64), q)
    else:
        lo = (codes & 15).astype(np.int64) - 8
        hi = (codes >> 4).astype(np.int64) - 8
        assert np.array_equal(lo, q[:, 0::2]) and np.array_equal(hi, q[:, 1::2])


def test_quantiser_special_groups():
    K = 256
    W = np.zeros((3, K), np.float32)
    W[1, :128] = -0.375            # group of only -amax: q = -7, s = 0.375 / 7
    W[2, 128:] = 1e-9              # amax / 7 underflows fp16 -> s = 0, q = 0
    codes, scales = oracle.quantize(synth.to_bf16_bits(W), oracle.INT4)
    assert np.all(codes[0] == 0x88) and np.all(scales[:, 0] == 0)
    assert np.all(codes[1, :64] == 0x11)                    # u = 1 -> q = -7
    assert scales[0, 1] == np.float16(np.float32(0.375) / np.float32(7)).view(np.uint16)
    assert scales[1, 2] == 0 and np.all(codes[2, 64:] == 0x88)


def test_quantiser_error_bound_and_range():
    rng = np.random.default_rng(12)
    rows, K = 64, 1024
    bits = synth.to_bf16_bits(rng.standard_normal((rows, K)).astype(np.float32) * 0.02)
    Wf = synth.bf16_bits_to_f32(bits).astype(np.float64)
    for prec, Q in ((oracle.INT4, 7), (oracle.INT8, 127)):
        codes, scales = oracle.quantize(bits, prec)
        s = scales.view(np.float16).astype(np.float64).T
        amax = np.abs(Wf.reshape(rows, K // 128, 128)).max(-1)
        # s is amax/Q (binary32 quotient) rounded to fp16: within half an fp16 ulp
        assert np.all(np.abs(s - amax / Q) <= np.abs(amax / Q) * 2.0 ** -11 * 1.0001)
        Wd = oracle.dequantize(prec, codes, scales, rows, K)
        err = np.abs(Wd - Wf).reshape(rows, K // 128, 128)
        assert np.all(err <= s[..., None] * 0.5 * (1 + 1e-6))  # round-to-nearest bound


def test_int4_storage_size_matches_memory_formula():
    # ExactMoE Section 3.2 memory formula: P (4/8 + 16/(128*8)) bytes
    rows, K = 2 * 768, 2048
    codes, scales = oracle.quantize(np.zeros((rows, K), np.uint16), oracle.INT4)
    P = rows * K
    assert codes.nbytes + scales.nbytes == P * (4 / 8 + 16 / (128 * 8))


def test_int4_nibble_golden_fixture():
    lines = [l.split() for l in open(os.path.join(GOLDEN, "int4_nibble_decode.txt"))
             if l.strip() and not l.startswith("#")]
    d = {l[0]: l[1:] for l in lines}
    scale = int(d["scale_fp16"][0], 16)
    head = [int(b, 16) for b in d["bytes"]]
    q_expect = [int(v) for v in d["q"]]
    row = np.full((1, 64), 0x88, np.uint8)
    row[0, :len(head)] = head
    s = np.full((1, 1), scale, np.uint16)
    W = oracle.dequantize(oracle.INT4, row, s, 1, 128)
    assert list(W[0, :len(q_expect)]) == [q * 0.5 for q in q_expect]
    assert np.all(W[0, len(q_expect):] == 0.0)


def test_int8_decode_of_all_codes():
    codes = np.arange(-128, 128, dtype=np.int8).reshape(2, 128)
    s = np.array([[0x3C00, 0x4000]], np.uint16)      # scales 1.0 (row 0), 2.0 (row 1)
    W = oracle.dequantize(oracle.INT8, codes, s, 2, 128)
    assert np.array_equal(W[0], np.arange(-128, 0)) and np.array_equal(W[1], 2.0 * np.arange(0, 128))


def test_scale_layout_is_group_major():
    # row r, group g scale at s[g, r]: make every (r, g) scale distinct
    rows, K = 3, 256
    codes = np.full((rows, K), 1, np.int8)
    s = np.array([[0x3C00, 0x4000, 0x4200], [0x4400, 0x4500, 0x4600]], np.uint16)
    W = oracle.dequantize(oracle.INT8, codes, s, rows, K)
    expect = s.view(np.float16).astype(np.float64).T     # [rows, groups]
    assert np.array_equal(W[:, ::128], expect)


# ------------------------------------------------------------------- FFN --

def _dense_swiglu(x, wg, wu, wd):
    """Dense SwiGLU MLP with torch's fp64 silu and matmul."""
    xt, g, u = torch.from_numpy(x), torch.from_numpy(wg), torch.from_numpy(wu)
    h = torch.nn.functional.silu(xt @ g.T) * (xt @ u.T)
    return (h @ torch.from_numpy(wd).T).numpy()


def _experts_from_master(H, I, E, seed, precs):
    out = []
    for e in range(E):
        w13, w2 = synth.gen_expert_master(H, I, seed, e)
        p = int(precs[e])
        if p == oracle.BF16:
            out.append(oracle.Expert(p, w13, None, w2, None))
        else:
            q13, s13 = oracle.quantize(w13, p)
            q2, s2 = oracle.quantize(w2, p)
            out.append(oracle.Expert(p, q13, s13, q2, s2))
    return out


def _dequant_expert(ex, H, I):
    if ex.prec == oracle.BF16:
        return (synth.bf16_bits_to_f32(ex.w13).astype(np.float64),
                synth.bf16_bits_to_f32(ex.w2).astype(np.float64))
    return (oracle.dequantize(ex.prec, ex.w13, ex.s13, 2 * I, H),
            oracle.dequantize(ex.prec, ex.w2, ex.s2, H, I))


@pytest.mark.parametrize("prec", [oracle.BF16, oracle.INT8, oracle.INT4])
def test_single_expert_top1_is_dense_swiglu(prec):
    H, I, T = 256, 384, 9
    ex = _experts_from_master(H, I, 1, 21, [prec])
    x = synth.gen_x(T, H, 21)
    logits = np.zeros((T, 1), np.float32)
    idx, w, out = oracle.moe_layer(logits, x, ex, 1, H, I)
    assert np.all(idx == 0) and np.all(w == 1.0)
    w13, w2 = _dequant_expert(ex[0], H, I)
    ref = _dense_swiglu(synth.bf16_bits_to_f32(x).astype(np.float64), w13[:I], w13[I:], w2)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-14)


def test_gate_and_up_are_not_interchangeable():
    # silu(g) * u != silu(u) * g: catches swapped gate/up halves of W13
    H, I = 128, 128
    ex = _experts_from_master(H, I, 1, 22, [oracle.BF16])
    x = synth.gen_x(4, H, 22)
    _, _, out = oracle.moe_layer(np.zeros((4, 1), np.float32), x, ex, 1, H, I)
    w13, w2 = _dequant_expert(ex[0], H, I)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    swapped = _dense_swiglu(xf, w13[I:], w13[:I], w2)
    assert not np.allclose(out, swapped, rtol=1e-3)


def test_closed_form_single_path():
    # x = a e_0, one nonzero weight per matrix: y_m = d_m * silu(a g) * (a u)
    H, I = 128, 128
    a, g, u = 1.5, 0.75, -2.0
    d = np.zeros(H); d[3], d[70] = 0.5, -1.25
    w13 = np.zeros((2 * I, H), np.float32); w13[5, 0] = g; w13[I + 5, 0] = u
    w2 = np.zeros((H, I), np.float32); w2[:, 5] = d
    ex = [oracle.Expert(oracle.BF16, synth.to_bf16_bits(w13), None, synth.to_bf16_bits(w2), None)]
    x = np.zeros((1, H), np.float32); x[0, 0] = a
    _, _, out = oracle.moe_layer(np.zeros((1, 1), np.float32), synth.to_bf16_bits(x), ex, 1, H, I)
    hg = a * g
    expect = d * (hg / (1.0 + math.exp(-hg))) * (a * u)
    assert np.allclose(out[0], expect, rtol=1e-15, atol=0)


def test_integer_weights_give_exact_projections():
    # INT4 with all scales 1: integer weights; integer x -> g, u exact integers
    H, I = 128, 128
    rng = np.random.default_rng(23)
    codes, _ = synth.gen_random_codes(2 * I, H, oracle.INT4, 23)
    q2, _ = synth.gen_random_codes(H, I, oracle.INT4, 23, key=1)
    one = np.full((1, 2 * I), 0x3C00, np.uint16)
    ex = [oracle.Expert(oracle.INT4, codes, one, q2, np.full((1, H), 0x3C00, np.uint16))]
    xi = rng.integers(-3, 4, (2, H)).astype(np.float32)
    _, _, out = oracle.moe_layer(np.zeros((2, 1), np.float32), synth.to_bf16_bits(xi), ex, 1, H, I)
    lo = (codes & 15).astype(np.int64) - 8; hi = (codes >> 4).astype(np.int64) - 8
    Wq = np.empty((2 * I, H), np.int64); Wq[:, 0::2] = lo; Wq[:, 1::2] = hi
    l2 = (q2 & 15).astype(np.int64) - 8; h2 = (q2 >> 4).astype(np.int64) - 8
    W2 = np.empty((H, I), np.int64); W2[:, 0::2] = l2; W2[:, 1::2] = h2
    gi = xi.astype(np.int64) @ Wq[:I].T; ui = xi.astype(np.int64) @ Wq[I:].T
    h = torch.nn.functional.silu(torch.from_numpy(gi.astype(np.float64))).numpy() * ui
    assert np.allclose(out, h @ W2.T, rtol=1e-12, atol=1e-9)


def test_layer_equals_route_permute_ffn_combine_and_numpy():
    cfg = synth.CONFIGS["tiny"]
    H, I, E, k, T = cfg.H, cfg.I, cfg.E, cfg.k, cfg.T
    ex = _experts_from_master(H, I, E, cfg.seed, [oracle.INT4] * E)
    x = synth.gen_x(T, H, cfg.seed)
    logits = synth.gen_logits(T, E, cfg.seed)
    idx, w, out = oracle.moe_layer(logits, x, ex, k, H, I)
    off, perm_token, dest, _ = oracle.permute(idx, E)
    y = oracle.grouped_ffn(x[perm_token], off, ex, H, I)
    assert np.allclose(oracle.combine(y, dest, w), out, rtol=1e-13, atol=1e-16)
    # independent fp64 recomputation with torch matmuls over dequantised experts
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = np.zeros((T, H))
    for e in range(E):
        w13, w2 = _dequant_expert(ex[e], H, I)
        ye = _dense_swiglu(xf, w13[:I], w13[I:], w2)
        for j in range(k):
            sel = idx[:, j] == e
            ref[sel] += w[sel, j, None] * ye[sel]
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-14)


def test_layer_result_does_not_depend_on_thread_count():
    """The work is split over (expert, row) and tokens only: one thread and all
    threads give the same bits (the timed CPU baseline reports both)."""
    cfg = synth.CONFIGS["tiny"]
    H, I, E, k, T = cfg.H, cfg.I, cfg.E, cfg.k, cfg.T
    ex = _experts_from_master(H, I, E, cfg.seed, [oracle.INT4, oracle.INT8, oracle.BF16, oracle.INT4,
                                                  oracle.INT8, oracle.BF16, oracle.INT4, oracle.INT4])
    x = synth.gen_x(T, H, cfg.seed)
    logits = synth.gen_logits(T, E, cfg.seed)
    n = oracle.num_threads()
    try:
        oracle.set_num_threads(1)
        one = oracle.moe_layer(logits, x, ex, k, H, I)
    finally:
        oracle.set_num_threads(n)
    many = oracle.moe_layer(logits, x, ex, k, H, I)
    for a, b in zip(one, many):
        assert np.array_equal(a, b)


# --------------------------------------------------------------- combine --

def test_combine_one_hot_linearity_and_wave_split():
    rng = np.random.default_rng(31)
    T, k, H, R = 6, 3, 128, 18
    y = rng.standard_normal((R, H))
    dest = rng.permutation(R).astype(np.int32).reshape(T, k)
    w1 = np.zeros((T, k)); w1[:, 1] = 1.0
    assert np.array_equal(oracle.combine(y, dest, w1), y[dest[:, 1]])
    w = rng.random((T, k))
    assert np.allclose(oracle.combine(y, dest, 2.5 * w), 2.5 * oracle.combine(y, dest, w),
                       rtol=1e-14)
    # disjoint waves (expert subsets), weights not renormalised per wave, sum to the whole
    wave = rng.random((T, k)) < 0.5
    d1 = np.where(wave, dest, -1).astype(np.int32)
    d2 = np.where(~wave, dest, -1).astype(np.int32)
    whole = oracle.combine(y, dest, w)
    assert np.allclose(oracle.combine(y, d1, w) + oracle.combine(y, d2, w), whole, rtol=1e-14)
