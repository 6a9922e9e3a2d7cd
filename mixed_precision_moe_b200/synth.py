"""Seeded synthetic inputs for the mixed-precision MoE layer.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It draws random numbers and lays them out; it holds none of the layer's own
arithmetic (no routing, grouping, quantisation or matmul).

Value distributions follow the workloads named for this layer: activations
~N(0, 1) and expert weights ~N(0, 0.02^2), both rounded to bfloat16 by torch's
fp32->bf16 conversion; router logits fp32 ~N(0, 1) plus a Zipf popularity bias
b_e = -s * ln(rank_e), where rank_e = pi(e) + 1 for a seeded permutation pi of
the experts.  ln(rank^-s) is the log of the Zipf(s) mass up to a constant, and
a constant shift changes neither the top-k nor the softmax.  "Hottest" expert =
lowest rank.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

BF16, INT8, INT4 = 0, 1, 2
PREC_NAMES = {BF16: "bf16", INT8: "int8", INT4: "int4"}


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), rounded by torch."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def gen_x(T: int, H: int, seed: int) -> np.ndarray:
    """Activations bf16 bits [T, H], ~N(0, 1)."""
    return to_bf16_bits(_rng(seed, 1).standard_normal((T, H), dtype=np.float32))


def zipf_ranks(E: int, seed: int) -> np.ndarray:
    """rank_e in 1..E (1 = hottest) from a seeded permutation of the experts."""
    return _rng(seed, 2).permutation(E).astype(np.int64) + 1


def gen_logits(T: int, E: int, seed: int, zipf_s: float = 0.0,
               ranks: np.ndarray | None = None) -> np.ndarray:
    """Router logits fp32 [T, E] ~N(0, 1) + Zipf bias -s*ln(rank)."""
    z = _rng(seed, 3).standard_normal((T, E), dtype=np.float32)
    if zipf_s:
        if ranks is None:
            ranks = zipf_ranks(E, seed)
        z = z + (-zipf_s * np.log(ranks.astype(np.float64))).astype(np.float32)[None, :]
    return np.ascontiguousarray(z, dtype=np.float32)


def gen_router(T: int, H: int, E: int, seed: int, zipf_s: float = 0.0,
               ranks: np.ndarray | None = None):
    """Hidden states h bf16 bits [T, H] and router weights W_r bf16 bits
    [E, H] for z = W_r h.  h ~N(0, 1) and W_r ~N(0, 1/H), so that z is about
    N(0, 1) like gen_logits.  With zipf_s, the last hidden coordinate is the
    constant 1 and W_r[e, H-1] = -zipf_s * ln(rank_e) (bf16-rounded): the
    Zipf popularity bias of gen_logits carried by the weights, since a
    router has no bias term of its own."""
    h = _rng(seed, 5).standard_normal((T, H), dtype=np.float32)
    w = _rng(seed, 6).standard_normal((E, H), dtype=np.float32) * np.float32(1.0 / np.sqrt(H))
    if zipf_s:
        if ranks is None:
            ranks = zipf_ranks(E, seed)
        h[:, H - 1] = 1.0
        w[:, H - 1] = (-zipf_s * np.log(ranks.astype(np.float64))).astype(np.float32)
    return to_bf16_bits(h), to_bf16_bits(w)


def gen_expert_master(H: int, I: int, seed: int, e: int, std: float = 0.02):
    """bf16 master weights of expert e: (w13 [2I, H], w2 [H, I]) as bf16 bits.

    Rows 0..I-1 of w13 are the gate projection, rows I..2I-1 the up projection.
    """
    r = _rng(seed, 4, e)
    w13 = r.standard_normal((2 * I, H), dtype=np.float32) * np.float32(std)
    w2 = r.standard_normal((H, I), dtype=np.float32) * np.float32(std)
    return to_bf16_bits(w13), to_bf16_bits(w2)


def precision_map(ranks: np.ndarray, tiers) -> np.ndarray:
    """tiers: [(count, prec), ...] assigned from the hottest rank down."""
    prec = np.empty(len(ranks), np.int32)
    order = np.argsort(ranks, kind="stable")   # hottest first
    start = 0
    for count, p in tiers:
        prec[order[start:start + count]] = p
        start += count
    assert start == len(ranks), "tiers must cover every expert"
    return prec


def gen_random_codes(rows: int, K: int, prec: int, seed: int, key: int = 0):
    """Arbitrary stored codes and fp16 scales (any nibble / byte value).

    Used to exercise the decoder on codes the quantiser never emits (e.g. the
    INT4 code -8).  Scales are positive fp16 values in [2^-10, 2^-5).
    """
    r = _rng(seed, 5, key)
    if prec == INT4:
        w = r.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    else:
        w = r.integers(-128, 128, (rows, K), dtype=np.int8)
    mant = r.integers(0, 1024, (K // 128, rows), dtype=np.uint16)
    expo = r.integers(5, 10, (K // 128, rows), dtype=np.uint16)   # 2^-10 .. 2^-6
    s = ((expo << 10) | mant).astype(np.uint16)
    return w, s


@dataclass
class LayerConfig:
    """One routed-expert layer workload (sizes, routing skew, precision tiers)."""
    name: str
    H: int
    I: int
    E: int
    k: int
    T: int
    seed: int
    zipf_s: float = 0.0
    tiers: list = field(default_factory=list)   # [(count, prec)], hottest first

    @property
    def rows(self) -> int:
        return self.T * self.k


CONFIGS = {
    # hidden 256, intermediate 512, 8 experts, top-2, 64 tokens, all INT4
    "tiny": LayerConfig("tiny", H=256, I=512, E=8, k=2, T=64, seed=1, tiers=[(8, INT4)]),
    # Qwen3-30B-A3B-shaped decode, batch 32, 32 hottest BF16 + 96 INT4, Zipf 1.1
    "qwen3_30b_decode": LayerConfig("qwen3_30b_decode", H=2048, I=768, E=128, k=8, T=32,
                                    seed=2, zipf_s=1.1, tiers=[(32, BF16), (96, INT4)]),
    # same layer, prefill 4096 tokens, 24 BF16 / 40 INT8 / 64 INT4, Zipf 1.1
    "qwen3_30b_prefill": LayerConfig("qwen3_30b_prefill", H=2048, I=768, E=128, k=8, T=4096,
                                     seed=3, zipf_s=1.1,
                                     tiers=[(24, BF16), (40, INT8), (64, INT4)]),
}

# Mixtral-8x7B-shaped layer: all INT4, uniform logits, token batch sweep.
MIXTRAL_BATCHES = (1, 8, 32, 128, 512, 4096)


def mixtral_config(T: int) -> LayerConfig:
    i = MIXTRAL_BATCHES.index(T) if T in MIXTRAL_BATCHES else 0
    return LayerConfig(f"mixtral_8x7b_T{T}", H=4096, I=14336, E=8, k=2, T=T,
                       seed=40 + i, tiers=[(8, INT4)])


# Qwen3-80B-scale stack: 4 layers, hidden 2048, intermediate 512, 512 experts,
# top-10, decode batch 32, 256 steps, Zipf 1.2 with the hot set redrawn every
# 64 steps; top-64 BF16, rest INT4.
STACK = dict(layers=4, H=2048, I=512, E=512, k=10, T=32, steps=256, epoch=64,
             zipf_s=1.2, n_hot=64, seed=5)


def stack_ranks(layer: int, epoch: int) -> np.ndarray:
    return zipf_ranks(STACK["E"], STACK["seed"] * 1000 + 10 * layer + epoch)


def stack_logits(layer: int, step: int) -> np.ndarray:
    ranks = stack_ranks(layer, step // STACK["epoch"])
    return gen_logits(STACK["T"], STACK["E"], STACK["seed"] * 100000 + 1000 * layer + step,
                      STACK["zipf_s"], ranks)


def stack_x(layer: int, step: int) -> np.ndarray:
    return gen_x(STACK["T"], STACK["H"], STACK["seed"] * 100000 + 1000 * layer + step)


def stack_master(layer: int, e: int):
    """bf16 master weights of expert e of stack layer `layer`."""
    return gen_expert_master(STACK["H"], STACK["I"], STACK["seed"] * 10 + layer, e)
