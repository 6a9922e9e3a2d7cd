"""ctypes marshalling for ``moe_oracle.c`` (test infrastructure only).

Every function takes and returns numpy arrays; no arithmetic of the method is
done here.  Page citations for each step are in ``moe_oracle.c``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from dataclasses import dataclass

import numpy as np

BF16, INT8, INT4 = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so with gcc (-O2, OpenMP, IEEE)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _L():
    global _lib
    if _lib is None:
        # MOE_ORACLE_LIB lets the mutation tests load a deliberately broken copy.
        _lib = C.CDLL(os.environ.get("MOE_ORACLE_LIB") or build())
        _lib.oracle_bf16_to_double.restype = C.c_double
        _lib.oracle_bf16_to_double.argtypes = [C.c_uint16]
        _lib.oracle_fp16_to_double.restype = C.c_double
        _lib.oracle_fp16_to_double.argtypes = [C.c_uint16]
        _lib.oracle_fp16_from_float.restype = C.c_uint16
        _lib.oracle_fp16_from_float.argtypes = [C.c_float]
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p)


def _check(rc, what):
    if rc < 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")
    return rc


def num_threads() -> int:
    return int(_L().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """OpenMP threads of later calls; results do not depend on the count."""
    _L().oracle_set_num_threads(int(n))


def bf16_to_double(b: int) -> float:
    return float(_L().oracle_bf16_to_double(int(b)))


def fp16_to_double(h: int) -> float:
    return float(_L().oracle_fp16_to_double(int(h)))


def fp16_from_float(f: float) -> int:
    return int(_L().oracle_fp16_from_float(C.c_float(f)))


@dataclass
class Expert:
    """One expert in the storage format of include/moe.h (numpy, host)."""
    prec: int
    w13: np.ndarray          # [2I, H] bf16 bits (uint16) | int8 | uint8 [2I, H/2]
    s13: np.ndarray | None   # fp16 bits uint16 [H/128, 2I]
    w2: np.ndarray           # [H, I] (same encodings, K = I)
    s2: np.ndarray | None    # fp16 bits uint16 [I/128, H]


def quantize(w_bf16: np.ndarray, prec: int):
    """bf16 bits [rows, K] -> (codes in storage format, fp16 scale bits [K/128, rows])."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    rows, K = w.shape
    q = np.zeros((rows, K // 2), np.uint8) if prec == INT4 else np.zeros((rows, K), np.int8)
    s = np.zeros((K // 128, rows), np.uint16)
    _check(_L().oracle_quantize(_p(w), rows, K, prec, _p(q), _p(s)), "quantize")
    return q, s


def dequantize(prec: int, w: np.ndarray, s: np.ndarray | None, rows: int, K: int) -> np.ndarray:
    out = np.zeros((rows, K), np.float64)
    w = np.ascontiguousarray(w)
    sp = _p(np.ascontiguousarray(s)) if s is not None else None
    _check(_L().oracle_dequantize(prec, _p(w), sp, rows, K, _p(out)), "dequantize")
    return out


def router_logits(h: np.ndarray, wr: np.ndarray) -> np.ndarray:
    """z = W_r h per token in binary64 (ExactMoE Section 3.1 routing equation).
    h: bf16 bit patterns uint16 [T][H]; wr: uint16 [E][H]."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    wr = np.ascontiguousarray(wr, dtype=np.uint16)
    T, H = h.shape
    E, H2 = wr.shape
    if H2 != H:
        raise ValueError("router rows must have the hidden size")
    z = np.zeros((T, E), np.float64)
    _check(_L().oracle_router_logits(_p(h), _p(wr), T, H, E, _p(z)), "router")
    return z


def route_topk(logits: np.ndarray, k: int, renormalize: bool = True):
    z = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = z.shape
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    _check(_L().oracle_route_topk(_p(z), T, E, k, int(bool(renormalize)), _p(idx), _p(w)), "route")
    return idx, w


def permute(idx: np.ndarray, E: int):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    offsets = np.zeros(E + 1, np.int32)
    perm_token = np.full(T * k, -1, np.int32)
    dest_row = np.zeros(T * k, np.int32)
    invalid = _check(_L().oracle_permute(_p(idx), T, E, k, _p(offsets), _p(perm_token),
                                         _p(dest_row)), "permute")
    return offsets, perm_token, dest_row.reshape(T, k), invalid


def _expert_arrays(experts):
    E = len(experts)
    keep = []

    def ptrs(attr):
        arr = (C.c_void_p * E)()
        for e, ex in enumerate(experts):
            a = getattr(ex, attr)
            if a is None:
                arr[e] = None
            else:
                a = np.ascontiguousarray(a)
                keep.append(a)
                arr[e] = a.ctypes.data
        return arr

    prec = np.array([ex.prec for ex in experts], np.int32)
    return prec, ptrs("w13"), ptrs("s13"), ptrs("w2"), ptrs("s2"), keep


def grouped_ffn(x_perm: np.ndarray, offsets: np.ndarray, experts, H: int, I: int,
                rows: np.ndarray | None = None) -> np.ndarray:
    """y_perm (binary64) for all permuted rows, or only for `rows`."""
    x_perm = np.ascontiguousarray(x_perm, dtype=np.uint16)
    offsets = np.ascontiguousarray(offsets, dtype=np.int32)
    prec, w13, s13, w2, s2, keep = _expert_arrays(experts)
    if rows is None:
        n, rp = int(offsets[-1]), None
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int32)
        n, rp = len(rows), _p(rows)
    y = np.zeros((n, H), np.float64)
    _check(_L().oracle_grouped_ffn(_p(x_perm), _p(offsets), H, I, len(experts), _p(prec),
                                   w13, s13, w2, s2, rp, n, _p(y)), "grouped_ffn")
    del keep
    return y


def combine(y_perm: np.ndarray, dest_row: np.ndarray, w: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y_perm, dtype=np.float64)
    d = np.ascontiguousarray(dest_row, dtype=np.int32)
    wt = np.ascontiguousarray(w, dtype=np.float64)
    T, k = d.shape
    H = y.shape[1]
    out = np.zeros((T, H), np.float64)
    _check(_L().oracle_combine(_p(y), _p(d), _p(wt), T, k, H, _p(out)), "combine")
    return out


def moe_layer(logits: np.ndarray, x: np.ndarray, experts, k: int, H: int, I: int,
              renormalize: bool = True, tokens: np.ndarray | None = None):
    """Whole layer: returns (idx [T,k], w [T,k] binary64, out [n_tok, H] binary64)."""
    z = np.ascontiguousarray(logits, dtype=np.float32)
    x = np.ascontiguousarray(x, dtype=np.uint16)
    T, E = z.shape
    prec, w13, s13, w2, s2, keep = _expert_arrays(experts)
    if tokens is None:
        n, tp = T, None
    else:
        tokens = np.ascontiguousarray(tokens, dtype=np.int32)
        n, tp = len(tokens), _p(tokens)
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    out = np.zeros((n, H), np.float64)
    _check(_L().oracle_moe_layer(_p(z), _p(x), T, H, I, E, k, int(bool(renormalize)), _p(prec),
                                 w13, s13, w2, s2, tp, n, _p(idx), _p(w), _p(out)), "moe_layer")
    del keep
    return idx, w, out


def seeded_experts(H: int, I: int, precs, seed: int, masters=None):
    """The oracle-side experts of a seeded workload: each expert's bf16 master
    (from the shared seeded input generators, or `masters[e]` if given) kept as
    is for BF16, or quantised by this oracle's own group-128 quantiser for
    INT8/INT4.  The GPU side receives exactly these codes and scales."""
    from mixed_precision_moe_b200 import synth   # seeded generators only, no method arithmetic
    out = []
    for e, p in enumerate(precs):
        w13, w2 = masters[e] if masters is not None else synth.gen_expert_master(H, I, seed, e)
        p = int(p)
        if p == BF16:
            out.append(Expert(p, w13, None, w2, None))
        else:
            q13, s13 = quantize(w13, p)
            q2, s2 = quantize(w2, p)
            out.append(Expert(p, q13, s13, q2, s2))
    return out
