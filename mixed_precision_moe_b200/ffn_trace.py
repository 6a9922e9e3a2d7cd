"""Per-unit timeline of the grouped FFN kernel (profiling build).

Builds libmoe_trace.so (-DMOE_FFN_TRACE: every role of the persistent kernel
stamps each work unit with %globaltimer and sums the SM cycles it spent waiting
on its barriers), runs one workload's grouped FFN after warm-up with the L2
flushed before each launch, and prints, per kind of unit (precision x
projection), the mean time each role spends on a unit and its waits, plus the
kernel's and the CTAs' spans.

    python -m mixed_precision_moe_b200.ffn_trace [--workload decode] [--reps 5]
        [--out timeline.json]

Workloads: decode (Qwen3-30B-A3B-shaped, batch 32, 32 BF16 + 96 INT4, Zipf 1.1),
decode-int4 / decode-bf16 (same routing, every expert INT4 / BF16),
mixtral-T1 / mixtral-T32 (Mixtral-8x7B-shaped, all INT4, uniform logits).
"""
from __future__ import annotations

import argparse
import ctypes as C
import json
import os
import sys

import numpy as np

FIELDS = ["unit", "kind", "sched", "prod_beg", "prod_end", "prod_wait", "code_wait", "mma_beg",
          "mma_end", "mma_wait", "dq_beg", "dq_end", "dq_wait_q", "dq_wait_w", "epi_beg",
          "epi_end", "mma_issue", "dq_conv", "dq_store", "publish"]
F = {n: i for i, n in enumerate(FIELDS)}
CTAS, UNITS = 160, 96


def classify(kind: int) -> str:
    flags, prec = kind & 0xFF, (kind >> 8) & 0xFF
    return {0: "bf16", 1: "int8", 2: "int4"}.get(prec, "?") + (" gate/up" if flags & 2 else " down")


def summarise(rec: np.ndarray, sm_ghz: float) -> dict:
    """rec [CTAS][UNITS][fields] of one launch -> per-class means (us) and spans."""
    valid = rec[:, :, F["sched"]] != 0
    rows = rec[valid]
    t0 = rows[:, F["sched"]].min()
    last = max(rows[:, F["epi_end"]].max(), rows[:, F["dq_end"]].max())
    out = {"units": int(len(rows)), "kernel_span_us": float((last - t0) / 1e3),
           "sm_ghz_assumed": sm_ghz}
    cyc = 1e-3 / sm_ghz   # cycles -> us
    groups: dict = {}
    for r in rows:
        g = groups.setdefault(classify(int(r[F["kind"]])), [])
        g.append(r)
    for key, g in sorted(groups.items()):
        g = np.array(g)
        o = {"n": int(len(g)), "mean_rows": float(np.mean((g[:, F["kind"]] >> 16) & 0xFF))}
        def span(a, b):   # mean over the units the role stamped (CUDA-core units skip some)
            m = g[:, F[a]] != 0
            return float(np.mean(g[m, F[b]] - g[m, F[a]]) / 1e3) if m.any() else None
        o["prod_us"] = span("prod_beg", "prod_end")
        o["mma_us"] = span("mma_beg", "mma_end")
        o["epi_us"] = span("epi_beg", "epi_end")
        o["dq_span_us"] = span("dq_beg", "dq_end")
        for w in ("prod_wait", "code_wait", "mma_wait", "mma_issue", "dq_wait_q", "dq_wait_w",
                  "dq_conv", "dq_store", "publish"):
            o[w + "_us"] = float(np.mean(g[:, F[w]]) * cyc)
        out[key] = o
    spans, busy = [], []
    for c in range(rec.shape[0]):
        r = rec[c][rec[c][:, F["sched"]] != 0]
        if len(r):
            end = max(r[:, F["epi_end"]].max(), r[:, F["dq_end"]].max())
            spans.append((end - r[:, F["prod_beg"]].min()) / 1e3)
            busy.append((r[:, F["prod_beg"]].min() - t0) / 1e3)
    out["cta_span_us"] = {"min": float(np.min(spans)), "mean": float(np.mean(spans)),
                          "max": float(np.max(spans))}
    out["cta_first_copy_us"] = {"min": float(np.min(busy)), "mean": float(np.mean(busy)),
                                "max": float(np.max(busy))}
    return out


def cta_timeline(rec: np.ndarray, cta: int, t0: int) -> list:
    r = rec[cta][rec[cta][:, F["sched"]] != 0]
    return [{"unit": int(u[F["unit"]]), "kind": classify(int(u[F["kind"]])),
             "rows": int((u[F["kind"]] >> 16) & 0xFF),
             "prod": [round((u[F["prod_beg"]] - t0) / 1e3, 2), round((u[F["prod_end"]] - t0) / 1e3, 2)],
             "mma": [round((u[F["mma_beg"]] - t0) / 1e3, 2), round((u[F["mma_end"]] - t0) / 1e3, 2)],
             "epi": [round((u[F["epi_beg"]] - t0) / 1e3, 2), round((u[F["epi_end"]] - t0) / 1e3, 2)]}
            for u in r]


def build_workload(name, device):
    """(layer, x_perm, offsets, rows buffers) for one launch of the grouped FFN."""
    import torch
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from mixed_precision_moe_b200 import binding as B
    from mixed_precision_moe_b200 import synth
    if name == "stack":   # layer 0 of the Qwen3-80B-scale stack, step 0 (experts drawn on the device)
        S = synth.STACK
        T, E = S["T"], S["E"]
        gen = torch.Generator(device=device)
        gen.manual_seed(S["seed"])
        layer = B.MoELayer(S["H"], S["I"], E, S["k"])
        hot = set(np.argsort(synth.stack_ranks(0, 0), kind="stable")[:S["n_hot"]].tolist())
        for e in range(E):
            w13 = bench.device_master(2 * S["I"], S["H"], gen, device)
            w2 = bench.device_master(S["H"], S["I"], gen, device)
            if e in hot:
                layer.set_expert(e, B.BF16, w13, None, w2, None)
            else:
                q13, s13 = B.moe_quantize_weights(w13, B.INT4)
                q2, s2 = B.moe_quantize_weights(w2, B.INT4)
                layer.set_expert(e, B.INT4, q13, s13, q2, s2)
        lg, x = synth.stack_logits(0, 0), synth.stack_x(0, 0)
        dev_batches = [(torch.from_numpy(lg).to(device),
                        torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device))]
    elif name.startswith("decode"):
        base = synth.CONFIGS["qwen3_30b_decode"]
        tiers = {"decode": base.tiers, "decode-int4": [(base.E, synth.INT4)],
                 "decode-bf16": [(base.E, synth.BF16)]}[name]
        cfg = synth.LayerConfig(base.name, base.H, base.I, base.E, base.k, base.T, base.seed,
                                base.zipf_s, tiers)
        layer, ranks, _ = bench.build_layer(cfg, device)
        _, dev_batches = bench.make_inputs(cfg, ranks, 1, device)
        T = cfg.T
    else:
        T = int(name.split("-T")[1])
        cfg = synth.mixtral_config(T)
        gen = torch.Generator(device=device)
        gen.manual_seed(cfg.seed)
        layer = B.MoELayer(cfg.H, cfg.I, cfg.E, cfg.k)
        for e in range(cfg.E):
            w13 = bench.device_master(2 * cfg.I, cfg.H, gen, device)
            w2 = bench.device_master(cfg.H, cfg.I, gen, device)
            q13, s13 = B.moe_quantize_weights(w13, B.INT4)
            q2, s2 = B.moe_quantize_weights(w2, B.INT4)
            layer.set_expert(e, B.INT4, q13, s13, q2, s2)
            del w13, w2
        lg = synth.gen_logits(T, cfg.E, cfg.seed * 1000)
        x = synth.gen_x(T, cfg.H, cfg.seed * 1000)
        dev_batches = [(torch.from_numpy(lg).to(device),
                        torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device))]
    bufs = layer.alloc_buffers(T, device)
    for _ in range(3):
        layer.forward(*dev_batches[0], bufs=bufs)
        torch.cuda.synchronize()
        st = B.moe_get_device_status()
        print(f"warm-up forward: status {st:#x}", flush=True)
    return layer, bufs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "decode-int4", "decode-bf16", "mixtral-T1", "mixtral-T32",
                             "stack"])
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--sm-ghz", type=float, default=1.965, help="SM clock for cycle sums")
    ap.add_argument("--ctas", type=int, default=2, help="CTAs whose unit timeline is printed")
    ap.add_argument("--out", default=None)
    args = ap.parse_args()
    from mixed_precision_moe_b200 import build
    if not os.environ.get("MOE_LIB_PATH"):   # else: a profiling build given by the caller
        os.environ["MOE_LIB_PATH"] = build.build(trace=True)
    import torch
    from mixed_precision_moe_b200 import binding as B

    dev = torch.device("cuda", 0)
    layer, bufs = build_workload(args.workload, dev)
    L = B.lib()
    L.moe_ffn_trace_bytes.restype = C.c_size_t
    L.moe_ffn_trace_read.argtypes = [C.c_void_p, C.c_size_t]
    L.moe_ffn_giveup_read.argtypes = [C.c_void_p, C.c_size_t]
    giveup = np.zeros((CTAS, 4), np.int32)
    assert L.moe_ffn_giveup_read(giveup.ctypes.data, giveup.nbytes) == 0   # clears it
    nbytes = int(L.moe_ffn_trace_bytes())
    assert nbytes == CTAS * UNITS * len(FIELDS) * 8, (nbytes, "trace layout changed")
    off, _, _, xp = bufs["permute"]
    y, ws = bufs["ffn"]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)
    graph = torch.cuda.CUDAGraph()   # timed as the benchmark times it: a graph replay
    with torch.cuda.graph(graph, stream=stream):
        B.moe_grouped_ffn_mixed(layer, xp, off, y, ws, stream=stream)
    torch.cuda.synchronize()
    launches, times, kstamps = [], [], []
    L.moe_ffn_kstamp_read.argtypes = [C.c_void_p, C.c_size_t]
    for _ in range(args.reps):
        torch.cuda.synchronize()
        assert L.moe_ffn_trace_reset() == 0
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            flush.zero_()
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e3)
        buf = np.zeros(nbytes // 8, np.int64)
        assert L.moe_ffn_trace_read(buf.ctypes.data, nbytes) == 0
        launches.append(buf.reshape(CTAS, UNITS, len(FIELDS)))
        ks = np.zeros((CTAS, 5), np.int64)
        assert L.moe_ffn_kstamp_read(ks.ctypes.data, ks.nbytes) == 0
        ks = ks[:148] if ks[148:].max() == 0 else ks
        t0 = ks[:, 0].min()
        rel = (ks - t0) / 1e3
        kstamps.append({"entry_max": float(rel[:, 0].max()), "setup_done_mean": float(rel[:, 1].mean()),
                        "table_done_mean": float(rel[:, 2].mean()), "table_done_max": float(rel[:, 2].max()),
                        "final_barrier_min": float(rel[:, 3].min()),
                        "final_barrier_mean": float(rel[:, 3].mean()),
                        "exit_max": float(rel[:, 4].max())})
        status = B.moe_get_device_status()
        assert L.moe_ffn_giveup_read(giveup.ctypes.data, giveup.nbytes) == 0
        gave = [(c, *giveup[c][:3].tolist()) for c in range(CTAS) if giveup[c][0]]
        print(f"launch {len(times)}: {times[-1]:.1f} us, status {status:#x}, "
              f"{len(gave)} CTAs gave up (cta, role, unit seq, thread): {gave[:12]}", flush=True)
        if status:
            raise RuntimeError(f"device status {status:#x}")
    res = {"workload": args.workload, "event_us": times, "kernel_stamps_us": kstamps,
           "summary": summarise(launches[-1], args.sm_ghz)}
    rec = launches[-1]
    t0 = int(rec[rec[:, :, F["sched"]] != 0][:, F["sched"]].min())
    res["timelines"] = {c: cta_timeline(rec, c, t0) for c in range(min(args.ctas, CTAS))}
    print(json.dumps(res, indent=1))
    if args.out:
        rows = rec[rec[:, :, F["sched"]] != 0]
        json.dump({"fields": FIELDS, "result": res, "rows": rows.tolist(),
                   "cta_of_row": np.nonzero(rec[:, :, F["sched"]] != 0)[0].tolist()},
                  open(args.out, "w"))
    layer.close()


if __name__ == "__main__":
    main()
