"""Qwen3-80B-scale sparse layer stack with per-layer precision swaps.

Four layers (hidden 2048, expert intermediate 512, 512 experts, top-10), decode
batch 32 for 256 steps, Zipf(1.2) routing whose hot set is redrawn every 64
steps.  Every expert of every layer stays resident as INT4 (quantised on the
GPU from its bf16 master); from step 0 the 64 hottest experts of the first
epoch are BF16.  At each step 64 m the 64 experts selected most often in the
previous 64 steps (ties to the lower id) become BF16 and the rest INT4: the
bf16 masters of the newly promoted experts are copied to the device on a side
stream, the compute stream waits on that copy's event, and each change goes
through moe_set_expert_precision (DynaExq abstract: promotion and demotion by
swapping stable expert handles to fully materialised versions).  The forward
always runs on fully materialised handles.

Parity: routing of every step equals the oracle's bit for bit (it also drives
the swap decisions); the layer output is compared with the oracle, under the
same precision map, on every 16th step and on the step right after each swap's
first step.  The four layers take independent inputs, so they are run one
after another (each with its own 256 steps and swaps).
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
from mixed_precision_moe_b200 import binding as B
from mixed_precision_moe_b200 import synth
from helpers import check_close, to_gpu_bf16

pytestmark = pytest.mark.gpu

S = synth.STACK


def _hot_set(counts, n):
    """The n most selected experts, ties to the lower id (sorted ids)."""
    order = np.lexsort((np.arange(len(counts)), -counts))
    return np.sort(order[:n])


def _bf16_f64(t):
    u = t.view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def test_layer_stack_with_precision_swaps():
    H, I, E, k, T = S["H"], S["I"], S["E"], S["k"], S["T"]
    steps, epoch, n_hot = S["steps"], S["epoch"], S["n_hot"]
    sampled = set(range(0, steps, 16)) | {epoch * m + 1 for m in range(1, steps // epoch)}
    dev = torch.device("cuda", 0)
    compute = torch.cuda.Stream(dev)
    copy = torch.cuda.Stream(dev)
    B.moe_get_device_status()
    workers = max(1, min(16, os.cpu_count() or 1))
    for layer in range(S["layers"]):
        with ThreadPoolExecutor(workers) as pool:
            masters = list(pool.map(lambda e: synth.stack_master(layer, e), range(E)))
        L = B.MoELayer(H, I, E, k)
        int4 = []
        for e in range(E):   # resident INT4 of every expert, quantised on the GPU
            w13, w2 = to_gpu_bf16(masters[e][0]), to_gpu_bf16(masters[e][1])
            q13, s13 = B.moe_quantize_weights(w13, B.INT4)
            q2, s2 = B.moe_quantize_weights(w2, B.INT4)
            int4.append((q13, s13, q2, s2))
        torch.cuda.synchronize()

        def materialise(ids):
            """bf16 masters of `ids` copied on the side stream; returns them and the event."""
            out = {}
            with torch.cuda.stream(copy):
                for e in ids:
                    h13 = torch.from_numpy(masters[e][0].view(np.int16)).pin_memory()
                    h2 = torch.from_numpy(masters[e][1].view(np.int16)).pin_memory()
                    out[e] = (h13.to(dev, non_blocking=True).view(torch.bfloat16),
                              h2.to(dev, non_blocking=True).view(torch.bfloat16))
                ev = torch.cuda.Event()
                ev.record(copy)
            return out, ev

        hot = np.sort(np.argsort(synth.stack_ranks(layer, 0), kind="stable")[:n_hot])
        bf16, ev = materialise(hot)
        compute.wait_event(ev)
        for e in range(E):
            if e in bf16:
                L.set_expert(e, B.BF16, bf16[e][0], None, bf16[e][1], None, stream=compute)
            else:
                q13, s13, q2, s2 = int4[e]
                L.set_expert(e, B.INT4, q13, s13, q2, s2, stream=compute)

        bufs = L.alloc_buffers(T, dev)
        counts = np.zeros(E, np.int64)
        oracle_int4 = {}
        n_swapped = 0
        for step in range(steps):
            if step > 0 and step % epoch == 0:          # precision update before this step
                new_hot = _hot_set(counts, n_hot)
                counts[:] = 0
                promote = [e for e in new_hot if e not in bf16]
                demote = [e for e in hot if e not in set(new_hot.tolist())]
                fresh, ev = materialise(promote)
                compute.wait_event(ev)
                for e in demote:
                    q13, s13, q2, s2 = int4[e]
                    L.set_expert(e, B.INT4, q13, s13, q2, s2, stream=compute)
                    del bf16[e]
                for e in promote:
                    bf16[e] = fresh[e]
                    L.set_expert(e, B.BF16, bf16[e][0], None, bf16[e][1], None, stream=compute)
                n_swapped += len(promote) + len(demote)
                hot = new_hot
            logits = synth.stack_logits(layer, step)
            x = synth.stack_x(layer, step)
            with torch.cuda.stream(compute):
                out = L.forward(torch.from_numpy(logits).to(dev), to_gpu_bf16(x), bufs=bufs,
                                stream=compute)
            compute.synchronize()
            status = B.moe_get_device_status()
            assert status == 0, f"layer {layer} step {step}: device status {status:#x}"
            idx = bufs["route"][0].cpu().numpy()
            counts += np.bincount(idx.ravel(), minlength=E)
            if step not in sampled:
                continue
            exps = {}
            for e in np.unique(idx).tolist():
                if e in bf16:
                    exps[e] = oracle.Expert(oracle.BF16, masters[e][0], None, masters[e][1], None)
                else:
                    if e not in oracle_int4:
                        q13, s13 = oracle.quantize(masters[e][0], oracle.INT4)
                        q2, s2 = oracle.quantize(masters[e][1], oracle.INT4)
                        oracle_int4[e] = oracle.Expert(oracle.INT4, q13, s13, q2, s2)
                    exps[e] = oracle_int4[e]
            filler = next(iter(exps.values()))        # never read: selected by no token
            idx_o, _, out_o = oracle.moe_layer(logits, x, [exps.get(e, filler) for e in range(E)],
                                               k, H, I)
            assert np.array_equal(idx, idx_o), f"layer {layer} step {step}: routing"
            check_close(_bf16_f64(out), out_o, f"stack layer {layer} step {step}")
        assert n_swapped > 0, "the hot set never changed"
        assert sorted(e for e in range(E) if L.precision(e) == B.BF16) == hot.tolist()
        torch.cuda.synchronize()
        L.close()
        del masters, int4, bf16, oracle_int4
    assert B.moe_get_device_status() == 0
