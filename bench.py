"""Benchmark of the mixed-precision routed-expert layer on B200.

Headline workload: one Qwen3-30B-A3B-shaped MoE layer at decode batch 32
(H=2048, I=768, E=128, top-8, Zipf(1.1) routing skew, the 32 hottest experts
BF16 and the other 96 INT4 group-128).  A step is one whole layer forward
(route -> permute -> grouped FFN -> combine) on one batch of 32 tokens; the
same layer at prefill 4096 tokens (24 BF16 / 40 INT8 / 64 INT4 experts) is
reported in the "prefill" object.  Inputs are seeded synthetic data with the
shapes and value distributions of those workloads.

Timing: each step is a CUDA-graph replay timed by CUDA events on the launching
stream, with a 256 MiB write between steps to flush the 126 MB L2.  Multi-GPU
runs are independent replicas (the layer does not shard): every rank runs the
same workload and value = all ranks' tokens / the slowest rank's time.

`--impl reference` times the CPU oracle on the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixed_precision_moe_b200 import synth  # noqa: E402

METRIC = "MoE-layer tokens/s at decode B=32 and prefill 4096; % HBM / BF16-tensor roofline"
FLUSH_BYTES = 256 << 20


def expert_bytes(prec, H, I):
    """Stored bytes of one expert (weights + fp16 group-128 scales)."""
    P = 3 * H * I
    return {synth.BF16: 2 * P, synth.INT8: P + P // 64, synth.INT4: P // 2 + P // 64}[int(prec)]


FFN_SOURCES = ("grouped_ffn.cuh", "ptx.cuh", "common.cuh")
FFN_PROFILE = os.path.join(ROOT, "profiles", "grouped_ffn_decode_qwen3_30b_b32.md")


def ffn_kernel_hash():
    h = hashlib.sha256()
    for f in FFN_SOURCES:
        with open(os.path.join(ROOT, "mixed_precision_moe_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ffn_traffic(bytes_per_launch):
    """DRAM read + write bytes of one decode FFN launch from the committed ncu
    capture, scaled to `bytes_per_launch` algorithmic bytes by the captured
    launch's own algorithmic bytes; None if the kernel sources changed since."""
    try:
        text = open(FFN_PROFILE).read()
    except OSError:
        return None
    m = re.search(r"traffic-record: kernel_sha256=(\w+) dram_bytes=(\d+) algorithmic_bytes=(\d+)",
                  text)
    if not m or m.group(1) != ffn_kernel_hash():
        return None
    return int(m.group(2)) * bytes_per_launch / int(m.group(3))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def workload_name(cfg):
    tiers = " + ".join(f"{n} {synth.PREC_NAMES[p].upper()}" for n, p in cfg.tiers)
    return (f"{cfg.name}: H={cfg.H} I={cfg.I} E={cfg.E} top-{cfg.k} T={cfg.T}, "
            f"Zipf({cfg.zipf_s}) routing, experts {tiers}")


# --------------------------------------------------------------- clocks --

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(", ") for r in out.strip().splitlines() if r.count(",") >= 6]
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[3:7]) if v.strip() == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(rows[0][1]) if rows[0][1].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------- our arm (GPU) --

def build_layer(cfg, device):
    """Experts from seeded bf16 masters; INT8/INT4 ones quantised on the GPU."""
    from mixed_precision_moe_b200 import binding as B
    ranks = synth.zipf_ranks(cfg.E, cfg.seed)
    precs = synth.precision_map(ranks, cfg.tiers)
    layer = B.MoELayer(cfg.H, cfg.I, cfg.E, cfg.k)
    for e in range(cfg.E):
        w13, w2 = synth.gen_expert_master(cfg.H, cfg.I, cfg.seed, e)
        m13 = torch.from_numpy(w13.view(np.int16)).view(torch.bfloat16).to(device)
        m2 = torch.from_numpy(w2.view(np.int16)).view(torch.bfloat16).to(device)
        p = int(precs[e])
        if p == synth.BF16:
            layer.set_expert(e, p, m13, None, m2, None)
        else:
            q13, s13 = B.moe_quantize_weights(m13, p)
            q2, s2 = B.moe_quantize_weights(m2, p)
            layer.set_expert(e, p, q13, s13, q2, s2)
    torch.cuda.synchronize()
    return layer, ranks, precs


def make_inputs(cfg, ranks, n_batches, device):
    batches = []
    for b in range(n_batches):
        x = synth.gen_x(cfg.T, cfg.H, cfg.seed * 1000 + b)
        lg = synth.gen_logits(cfg.T, cfg.E, cfg.seed * 1000 + b, cfg.zipf_s, ranks)
        batches.append((torch.from_numpy(lg), torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)))
    dev = [(lg.to(device), x.to(device)) for lg, x in batches]
    return batches, dev


def time_graphs(graphs, steps, warmup, flush, stream):
    """Replay graphs[i % len] `steps` times after `warmup`; per-step event times (ms).
    The flush, the replays and the events all go to `stream`."""
    with torch.cuda.stream(stream):
        for i in range(warmup):
            flush.zero_()
            graphs[i % len(graphs)].replay()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(steps):
            flush.zero_()
            ev[i][0].record(stream)
            graphs[i % len(graphs)].replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def make_twin(layer, precs, cfg):
    """A second instance of the layer: the same expert weights in separate memory."""
    from mixed_precision_moe_b200 import binding as B
    twin = B.MoELayer(cfg.H, cfg.I, cfg.E, cfg.k)
    for e in range(cfg.E):
        w13, s13, w2, s2 = layer._weights[e]
        twin.set_expert(e, int(precs[e]), w13.clone(), None if s13 is None else s13.clone(),
                        w2.clone(), None if s2 is None else s2.clone())
    torch.cuda.synchronize()
    return twin


def time_steady(graphs_a, graphs_b, steps, warmup, stream):
    """Steps replayed back to back, alternating the two instances' graphs (step i:
    instance i % 2, batch i % len): each step's experts evict the other
    instance's from the L2, so no flush is needed.  Returns (ms per step over the
    run, per-step intervals in ms)."""
    n = len(graphs_a)
    pick = lambda i: (graphs_a if i % 2 == 0 else graphs_b)[i % n]
    with torch.cuda.stream(stream):
        for i in range(warmup):
            pick(i).replay()
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
        for i in range(steps):
            ev[i].record(stream)
            pick(i).replay()
        ev[steps].record(stream)
        torch.cuda.synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    return ev[0].elapsed_time(ev[steps]) / steps, per


def capture_layer_graphs(layer, dev_batches, bufs, stream):
    """One graph per batch for the whole forward, and one for the grouped FFN alone."""
    from mixed_precision_moe_b200 import binding as B
    step_graphs, ffn_graphs = [], []
    for b in range(len(dev_batches)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            layer.forward(*dev_batches[b], bufs=bufs[b], stream=stream)
        step_graphs.append(g)
        off, perm, dest, xp = bufs[b]["permute"]
        y, ws = bufs[b]["ffn"]
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream):
            B.moe_grouped_ffn_mixed(layer, xp, off, y, ws, stream=stream)
        ffn_graphs.append(g2)
    torch.cuda.synchronize()
    return step_graphs, ffn_graphs


def run_workload(cfg, steps, warmup, device, with_e2e, dist_barrier):
    """Returns a dict of timings and accounting for one layer config."""
    from mixed_precision_moe_b200 import binding as B
    layer, ranks, precs = build_layer(cfg, device)
    n_batches = 4
    host_batches, dev_batches = make_inputs(cfg, ranks, n_batches, device)
    stream = torch.cuda.Stream(device)
    bufs = [layer.alloc_buffers(cfg.T, device) for _ in range(n_batches)]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    # warm the library (attributes, tensor-map encoder) before capture
    with torch.cuda.stream(stream):
        for b in range(n_batches):
            layer.forward(*dev_batches[b], bufs=bufs[b])
    torch.cuda.synchronize()

    step_graphs, ffn_graphs = capture_layer_graphs(layer, dev_batches, bufs, stream)
    twin = make_twin(layer, precs, cfg)
    twin_bufs = [twin.alloc_buffers(cfg.T, device) for _ in range(n_batches)]
    with torch.cuda.stream(stream):
        for b in range(n_batches):
            twin.forward(*dev_batches[b], bufs=twin_bufs[b], stream=stream)
    torch.cuda.synchronize()
    twin_graphs, twin_ffn = capture_layer_graphs(twin, dev_batches, twin_bufs, stream)
    del twin_ffn

    # algorithmic accounting from this run's routing (read back after the fact)
    touched_bytes, pairs, n_touched = [], [], []
    selections = np.zeros(cfg.E, np.int64)
    for b in range(n_batches):
        idx = bufs[b]["route"][0].cpu().numpy()
        selections += np.bincount(idx.ravel(), minlength=cfg.E)
        te = np.unique(idx)
        n_touched.append(len(te))
        touched_bytes.append(sum(expert_bytes(precs[e], cfg.H, cfg.I) for e in te))
        pairs.append(idx.size)
    io_bytes = cfg.T * (2 * cfg.H + 4 * cfg.E + 2 * cfg.H)

    dist_barrier()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    steady_ms, t_step = time_steady(step_graphs, twin_graphs, steps, warmup, stream)
    clk = clocks.stop()
    t_iso = time_graphs(step_graphs, steps, warmup, flush, stream)
    t_ffn = time_graphs(ffn_graphs, steps, warmup, flush, stream)
    dist_barrier()

    res = {"step_ms": steady_ms, "ffn_ms": float(np.mean(t_ffn)),
           "isolated_step_ms": float(np.mean(t_iso)),
           "step_ms_all": t_step, "clocks": clk,
           "touched_bytes": float(np.mean([touched_bytes[i % n_batches] for i in range(steps)])),
           "io_bytes": io_bytes, "n_touched": float(np.mean(n_touched)),
           "pairs": float(np.mean(pairs)), "n_batches": n_batches,
           "selections": selections.tolist(),
           # this library's kernels per step: fused routing/grouping (T <= 128) or
           # routing + grouping + gather, then the grouped FFN and the combine
           "launches_per_step": 3 if cfg.T <= 128 else 5}

    if with_e2e:   # public API with host buffers: H2D inputs, forward, D2H output, every step
        # Each step's inputs (logits, then x at a 256-byte boundary) sit in one pinned
        # host buffer and travel in one host->device copy; the layer reads device views.
        lg_bytes = cfg.T * cfg.E * 4
        x_off = (lg_bytes + 255) // 256 * 256
        stage_bytes = x_off + cfg.T * cfg.H * 2
        pin, dstage, dl, dx = [], [], [], []
        for lg, x in host_batches:
            h = torch.empty(stage_bytes, dtype=torch.uint8).pin_memory()
            h[:lg_bytes].copy_(lg.contiguous().view(torch.uint8).reshape(-1))
            h[x_off:].copy_(x.contiguous().view(torch.uint8).reshape(-1))
            d = torch.empty(stage_bytes, dtype=torch.uint8, device=device)
            pin.append(h)
            dstage.append(d)
            dl.append(d[:lg_bytes].view(torch.float32).view(cfg.T, cfg.E))
            dx.append(d[x_off:].view(torch.bfloat16).view(cfg.T, cfg.H))
        outs = [torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory()
                for _ in range(n_batches)]
        torch.cuda.synchronize()
        ref_out = [bufs[b]["out"].clone() for b in range(n_batches)]   # from the graph replays

        # A serving loop through the public call: step i's inputs travel host->device
        # on one copy stream and step i-1's output device->host on another while the
        # compute stream runs step i's layer (buffers are reused every n_batches
        # steps, each reuse ordered by events).  Every step's copies lie inside the
        # timed region, which spans the whole run: e2e = steps / (last D2H done -
        # first H2D issued).  Steps alternate between two instances of the layer
        # (the same weights, in separate memory), as consecutive layers of a model
        # would: between two steps of one instance the other streams its ~300 MB of
        # experts through the 126 MB L2, so no step finds its weights there (the
        # device-timed steps flush the L2 instead).
        h2d_s, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
        new_ev = torch.cuda.Event
        in_ready = [new_ev() for _ in range(n_batches)]   # H2D of the slot done
        in_free = [None] * n_batches                       # its last reader (the layer) done
        out_ready = [new_ev() for _ in range(n_batches)]  # layer output written
        out_free = [None] * n_batches                      # its D2H done

        def e2e_step(i):
            b = i % n_batches
            with torch.cuda.stream(h2d_s):
                if in_free[b] is not None:
                    h2d_s.wait_event(in_free[b])
                dstage[b].copy_(pin[b], non_blocking=True)
                in_ready[b].record(h2d_s)
            stream.wait_event(in_ready[b])
            if out_free[b] is not None:
                stream.wait_event(out_free[b])
            lay, lb = (layer, bufs[b]) if i % 2 == 0 else (twin, twin_bufs[b])
            out = lay.forward(dl[b], dx[b], bufs=lb, stream=stream)
            out_ready[b].record(stream)
            in_free[b] = out_ready[b]
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(out_ready[b])
                outs[b].copy_(out, non_blocking=True)
                ev = new_ev()
                ev.record(d2h_s)
                out_free[b] = ev

        for i in range(warmup):
            e2e_step(i)
        torch.cuda.synchronize()
        t0, t1 = new_ev(enable_timing=True), new_ev(enable_timing=True)
        t0.record(h2d_s)
        for i in range(steps):
            e2e_step(i)
        d2h_s.wait_stream(stream)
        t1.record(d2h_s)
        torch.cuda.synchronize()
        res["e2e_ms"] = t0.elapsed_time(t1) / steps
        for b in range(min(n_batches, max(warmup, steps))):   # the batches the loops ran
            if not torch.equal(outs[b].to(device), ref_out[b]):
                raise RuntimeError(f"end-to-end output of batch {b} differs from the graph's")
        res["h2d_bytes"] = lg_bytes + cfg.T * cfg.H * 2   # the logits and x bytes of a step
        res["d2h_bytes"] = cfg.T * cfg.H * 2
    status = B.moe_get_device_status()
    if status:
        raise RuntimeError(f"device status {status:#x} after the benchmark")
    del step_graphs, ffn_graphs, twin_graphs
    twin.close()
    layer.close()
    return res


class OracleRunner:
    """The CPU oracle on the same workload (experts the batch selects only)."""

    def __init__(self, cfg):
        import oracle
        self.oracle, self.cfg = oracle, cfg
        ranks = synth.zipf_ranks(cfg.E, cfg.seed)
        precs = synth.precision_map(ranks, cfg.tiers)
        self.logits = synth.gen_logits(cfg.T, cfg.E, cfg.seed * 1000, cfg.zipf_s, ranks)
        self.x = synth.gen_x(cfg.T, cfg.H, cfg.seed * 1000)
        idx = np.argsort(-self.logits, axis=1, kind="stable")[:, :cfg.k]
        needed = set(np.unique(idx).tolist())
        # unselected experts are never read; they stay in their bf16 master form
        self.experts = oracle.seeded_experts(cfg.H, cfg.I, [precs[e] if e in needed else synth.BF16
                                                     for e in range(cfg.E)], cfg.seed)
        self.cores = oracle.num_threads()

    def run(self, n_tok):
        c = self.cfg
        tokens = np.arange(min(n_tok, c.T), dtype=np.int32)
        t0 = time.perf_counter()
        self.oracle.moe_layer(self.logits, self.x, self.experts, c.k, c.H, c.I, tokens=tokens)
        return len(tokens), time.perf_counter() - t0


def oracle_baseline(cfg, budget_s=10.0, single_s=3.0):
    """Time the CPU oracle on whole decode batches for about budget_s seconds on
    all host threads, then on 8-token slices for about single_s seconds on one."""
    r = OracleRunner(cfg)
    done, total = 0, 0.0
    while total < budget_s:
        n, dt = r.run(cfg.T)
        done, total = done + n, total + dt
    one, t1, sl = 0, 0.0, 8
    r.oracle.set_num_threads(1)
    try:
        while t1 < single_s:
            n, dt = r.run(sl)
            one, t1 = one + n, t1 + dt
    finally:
        r.oracle.set_num_threads(r.cores)
    return {"value": done / total, "unit": "tokens/s", "cores": r.cores, "kind": "oracle",
            "sample": f"{done // cfg.T} whole batches of {cfg.T} tokens of the {cfg.name} "
                      f"workload ({total:.1f} s), binary64 C oracle",
            "single_thread": {"value": one / t1, "unit": "tokens/s",
                              "sample": f"{one // sl} slices of {sl} tokens ({t1:.1f} s)"}}


# ---------------------------------------------- secondary workloads --
# Timing-only: their experts are drawn on the device (weights ~N(0, 0.02^2),
# rounded to bf16) because the work does not depend on the values and the host
# draw of several GB would dominate the run.  Parity on these shapes is covered
# by the GPU tests with the host-drawn masters.

def device_master(rows, K, gen, device, std=0.02):
    return (torch.randn((rows, K), generator=gen, device=device) * std).to(torch.bfloat16)


def mixtral_sweep(args, device, hbm_gbs, tf_burst, peak_src, batches=None):
    """Mixtral-8x7B-shaped layer, all experts INT4, uniform logits, over the
    token batch sweep: per batch the layer step, the grouped FFN alone and the
    FFN against its bound, max(expert bytes / HBM, flops / bf16 peak)."""
    from mixed_precision_moe_b200 import binding as B
    c0 = synth.mixtral_config(synth.MIXTRAL_BATCHES[0])
    H, I, E, k = c0.H, c0.I, c0.E, c0.k
    gen = torch.Generator(device=device)
    gen.manual_seed(c0.seed)
    layer = B.MoELayer(H, I, E, k)
    for e in range(E):
        w13 = device_master(2 * I, H, gen, device)
        w2 = device_master(H, I, gen, device)
        q13, s13 = B.moe_quantize_weights(w13, B.INT4)
        q2, s2 = B.moe_quantize_weights(w2, B.INT4)
        layer.set_expert(e, B.INT4, q13, s13, q2, s2)
        del w13, w2
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    steps, warmup = max(10, args.steps // 4), args.warmup
    eb = expert_bytes(synth.INT4, H, I)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    points = []
    batches = list(batches or synth.MIXTRAL_BATCHES)
    for T in batches:
        cfg = synth.mixtral_config(T)
        n_b = 2
        dev_b = []
        for b in range(n_b):
            lg = synth.gen_logits(T, E, cfg.seed * 1000 + b)
            x = synth.gen_x(T, H, cfg.seed * 1000 + b)
            dev_b.append((torch.from_numpy(lg).to(device),
                          torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)))
        bufs = [layer.alloc_buffers(T, device) for _ in range(n_b)]
        with torch.cuda.stream(stream):
            for b in range(n_b):
                layer.forward(*dev_b[b], bufs=bufs[b], stream=stream)
        torch.cuda.synchronize()
        step_g, ffn_g = capture_layer_graphs(layer, dev_b, bufs, stream)
        t_step = time_graphs(step_g, steps, warmup, flush, stream)
        t_ffn = time_graphs(ffn_g, steps, warmup, flush, stream)
        d = [len(np.unique(bufs[b]["route"][0].cpu().numpy())) for b in range(n_b)]
        d_mean = float(np.mean([d[i % n_b] for i in range(steps)]))
        step_ms, ffn_ms = float(np.mean(t_step)), float(np.mean(t_ffn))
        wbytes = d_mean * eb
        flops = 6.0 * H * I * T * k
        t_bytes = wbytes / (hbm_gbs * 1e9) * 1e3
        t_flops = flops / (tf_burst * 1e12) * 1e3
        if t_bytes >= t_flops:
            bound, achieved, peak, unit = "hbm", wbytes / (ffn_ms * 1e-3) / 1e9, hbm_gbs, "GB/s"
        else:
            bound, achieved, peak, unit = ("tensor", flops / (ffn_ms * 1e-3) / 1e12, tf_burst,
                                           "TFLOP/s")
        points.append({"T": T, "tokens_per_s": T / (step_ms * 1e-3), "ms_per_step": step_ms,
                       "ffn_ms": ffn_ms, "distinct_experts": d_mean, "expert_bytes": wbytes,
                       "flops": flops, "bound": bound, "bound_ms": max(t_bytes, t_flops),
                       "achieved": achieved, "peak": peak, "unit": unit,
                       "frac": achieved / peak})
        del step_g, ffn_g, bufs, dev_b
    clk = clocks.stop()
    status = B.moe_get_device_status()
    if status:
        raise RuntimeError(f"device status {status:#x} after the sweep")
    layer.close()
    return {"workload": f"mixtral_8x7b sweep: H={H} I={I} E={E} top-{k}, all experts INT4 "
                        f"group-128, uniform N(0,1) logits, T in {batches}",
            "data": "synthetic (logits and x host-seeded; experts drawn on the device)",
            "timing": f"CUDA graphs, {steps} timed replays after {warmup}, L2 flushed between",
            "peaks": {"hbm_gbs": hbm_gbs, "bf16_tflops": tf_burst, "source": peak_src},
            "points": points, "clocks": clk}


ROUTER_CASES = [  # name, T, H, E, k, zipf_s
    ("qwen3_30b_decode", 32, 2048, 128, 8, 1.1),
    ("qwen3_30b_prefill", 4096, 2048, 128, 8, 1.1),
    ("qwen3_80b_stack_layer", 32, 2048, 512, 10, 1.2),
    ("mixtral_8x7b_t1", 1, 4096, 8, 2, 0.0),
    ("mixtral_8x7b_t4096", 4096, 4096, 8, 2, 0.0),
]


def router_run(args, device, hbm_gbs, peak_src):
    """The router projection fused with top-k (moe_router_topk, one launch) on
    the layers' shapes: time per launch and its bytes (h, W_r, the top-k
    outputs) against HBM, from CUDA-graph replays with L2 flushed between."""
    from mixed_precision_moe_b200 import binding as B
    stream = torch.cuda.Stream(device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    steps, warmup = max(20, args.steps // 4), args.warmup
    points = []
    for name, T, H, E, k, zs in ROUTER_CASES:
        hb, wb = synth.gen_router(T, H, E, 900 + T + E, zs)
        h = torch.from_numpy(hb.view(np.int16)).view(torch.bfloat16).to(device)
        wr = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16).to(device)
        idx = torch.empty((T, k), dtype=torch.int32, device=device)
        w = torch.empty((T, k), dtype=torch.float32, device=device)
        with torch.cuda.stream(stream):
            B.moe_router_topk(h, wr, k, topk_idx=idx, topk_w=w, stream=stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            B.moe_router_topk(h, wr, k, topk_idx=idx, topk_w=w, stream=stream)
        ms = float(np.mean(time_graphs([g], steps, warmup, flush, stream)))
        nbytes = 2 * T * H + 2 * E * H + 8 * T * k
        gbs = nbytes / (ms * 1e-3) / 1e9
        points.append({"workload": name, "T": T, "H": H, "E": E, "k": k, "us": ms * 1e3,
                       "tokens_per_s": T / (ms * 1e-3), "bytes": nbytes, "achieved_gbs": gbs,
                       "frac_hbm": gbs / hbm_gbs, "tflops": 2.0 * T * E * H / (ms * 1e-3) / 1e12})
        del g
    status = B.moe_get_device_status()
    if status:
        raise RuntimeError(f"device status {status:#x} after the router runs")
    return {"kernel": "router_topk_kernel (z = W_r h on tcgen05, K split over a cluster, "
                      "top-k in the epilogue)",
            "timing": f"CUDA graph of one launch, {steps} timed replays after {warmup}, "
                      "L2 flushed between",
            "peaks": {"hbm_gbs": hbm_gbs, "source": peak_src}, "points": points}


def stack_run(args, device, hbm_gbs, peak_src, n_layers=None, n_steps=None):
    """Qwen3-80B-scale stack: layers of H 2048, I 512, 512 experts, top-10 at
    decode batch 32, Zipf(1.2) routing whose popularity order is redrawn every
    64 steps (4 layers x 256 steps by default).  Every expert stays resident as
    INT4; the 64 hottest are BF16, managed on the device per layer
    (mixed_precision_moe_b200.precision_manager): the routing kernels count the
    selections, the hot set of the last 64-step window is selected on the device
    at each step 64 m, the promoted experts' BF16 weights are copied into the
    idle slot set on a side stream once the selection is known (a non-blocking
    event query; experts already BF16 are copied device to device), and the
    handle swap runs on the device once the copies are done.  The compute stream
    never waits on a copy in flight; the gap between consecutive steps is the
    stall an update costs.  The host runs at most 8 steps ahead of the GPU.  A step is every layer's forward (one CUDA graph per
    layer and step)."""
    from mixed_precision_moe_b200 import binding as B
    from mixed_precision_moe_b200.precision_manager import PrecisionManager
    S = synth.STACK
    nl = n_layers or S["layers"]
    steps = n_steps or S["steps"]
    H, I, E, k, T = S["H"], S["I"], S["E"], S["k"], S["T"]
    epoch, n_hot = S["epoch"], S["n_hot"]
    compute = torch.cuda.Stream(device)
    copy = torch.cuda.Stream(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(S["seed"])
    layers, mgrs, keep = [], [], []
    chunk = 64
    for l in range(nl):
        L = B.MoELayer(H, I, E, k)
        h13 = torch.empty((E, 2 * I, H), dtype=torch.bfloat16, pin_memory=True)
        h2 = torch.empty((E, H, I), dtype=torch.bfloat16, pin_memory=True)
        q = []
        for e0 in range(0, E, chunk):
            w13 = device_master(chunk * 2 * I, H, gen, device).view(chunk, 2 * I, H)
            w2 = device_master(chunk * H, I, gen, device).view(chunk, H, I)
            h13[e0:e0 + chunk].copy_(w13)
            h2[e0:e0 + chunk].copy_(w2)
            for j in range(chunk):
                q.append(B.moe_quantize_weights(w13[j], B.INT4) +
                         B.moe_quantize_weights(w2[j], B.INT4))
            del w13, w2
        for e in range(E):
            q13, s13, q2, s2 = q[e]
            L.set_expert(e, B.INT4, q13, s13, q2, s2, stream=compute)
        assert L.hot_set_size(n_hot * (expert_bytes(synth.BF16, H, I) -
                                       expert_bytes(synth.INT4, H, I))) == n_hot
        mgr = PrecisionManager(L, [(h13[e], h2[e]) for e in range(E)], n_hot, device, copy)
        mgr.bootstrap(np.argsort(synth.stack_ranks(l, 0), kind="stable")[:n_hot], compute)
        layers.append(L)
        mgrs.append(mgr)
        keep.append((q, h13, h2))
    torch.cuda.synchronize()

    lg_all = torch.empty((steps, nl, T, E), dtype=torch.float32, device=device)
    x_all = torch.empty((steps, nl, T, H), dtype=torch.bfloat16, device=device)
    for st in range(steps):
        for l in range(nl):
            lg_all[st, l].copy_(torch.from_numpy(synth.stack_logits(l, st)))
            x_all[st, l].copy_(torch.from_numpy(synth.stack_x(l, st).view(np.int16))
                               .view(torch.bfloat16))
    hist = torch.zeros((steps, nl, T, k), dtype=torch.int32, device=device)
    bufs = [layers[l].alloc_buffers(T, device) for l in range(nl)]
    with torch.cuda.stream(compute):
        for l in range(nl):
            layers[l].forward(lg_all[0, l], x_all[0, l], bufs=bufs[l], stream=compute)
    torch.cuda.synchronize()
    for m in mgrs:   # the warm-up forwards counted: start the first window clean
        m.counts.zero_()
    pool = torch.cuda.graph_pool_handle()
    graphs = []
    with torch.cuda.stream(compute):
        for st in range(steps):
            row = []
            for l in range(nl):
                b = dict(bufs[l])
                b["route"] = (hist[st, l], bufs[l]["route"][1])
                g = torch.cuda.CUDAGraph()
                g.capture_begin(pool=pool)
                layers[l].forward(lg_all[st, l], x_all[st, l], bufs=b, stream=compute)
                g.capture_end()
                row.append(g)
            graphs.append(row)
    torch.cuda.synchronize()
    for m in mgrs:   # capture ran no kernels, but zero again to be certain
        m.counts.zero_()
    torch.cuda.synchronize()

    def new_event():
        return torch.cuda.Event(enable_timing=True)

    ev_s = [new_event() for _ in range(steps)]
    ev_e = [new_event() for _ in range(steps)]
    swap_steps = set()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    lag = 8   # the host stays at most this many steps ahead of the GPU, as a
    #          serving loop that consumes each step's output does
    with torch.cuda.stream(compute):
        for st in range(steps):
            if st >= lag:
                ev_e[st - lag].synchronize()
            ev_s[st].record(compute)
            for l in range(nl):
                if mgrs[l].poll(st, compute):
                    swap_steps.add(st)
                if st > 0 and st % epoch == 0:
                    mgrs[l].end_window(st, compute)
                graphs[st][l].replay()
            ev_e[st].record(compute)
    torch.cuda.synchronize()
    clk = clocks.stop()
    status = B.moe_get_device_status()
    if status:
        raise RuntimeError(f"device status {status:#x} after the stack run")

    step_ms = np.array([a.elapsed_time(b) for a, b in zip(ev_s, ev_e)])
    gaps = np.array([ev_e[i - 1].elapsed_time(ev_s[i]) for i in range(1, steps)])
    total_ms = ev_s[0].elapsed_time(ev_e[-1])
    sel = hist.cpu().numpy()
    # touched expert bytes of every step under the precision map in effect then
    # (a swap enqueued at step s precedes that step's forwards on the stream)
    touched = np.zeros(steps)
    for l in range(nl):
        sets = [(s_, set(d.tolist())) for s_, e_, d in mgrs[l].log if e_ in ("bootstrap", "swap")]
        for st in range(steps):
            hot = [h for s_, h in sets if s_ <= st][-1]
            for e in np.unique(sel[st, l]).tolist():
                touched[st] += expert_bytes(synth.BF16 if e in hot else synth.INT4, H, I)
    updates = [{"layer": l, "step": s_, "event": e_} for l in range(nl)
               for s_, e_, d in mgrs[l].log if e_ != "bootstrap"]
    gbs = float(np.mean(touched / (step_ms * 1e-3) / 1e9))
    mean_step = float(step_ms.mean())
    res = {"workload": f"qwen3_80b_stack: {nl} layers x {steps} steps, H={H} I={I} E={E} "
                       f"top-{k} T={T}, Zipf({S['zipf_s']}) popularity redrawn every {epoch} "
                       f"steps, {n_hot} hottest BF16 per layer (device-side hot sets), every "
                       f"expert resident as INT4",
           "data": "synthetic (logits and x host-seeded; experts drawn on the device)",
           "timing": "CUDA events on the compute stream; a step is one CUDA graph per layer; "
                     "no L2 flush (a step streams hundreds of MB of experts through the L2)",
           "tokens_per_s": T / (mean_step * 1e-3), "ms_per_step": mean_step,
           "ms_per_layer": mean_step / nl,
           "ms_per_step_p50": float(np.median(step_ms)),
           "ms_per_step_max": float(step_ms.max()),
           "tokens_per_s_with_updates": T * steps / (total_ms * 1e-3), "total_ms": total_ms,
           "touched_bytes_per_step": float(touched.mean()),
           "achieved_gbs": gbs, "frac_of_hbm": gbs / hbm_gbs, "peak_source": peak_src,
           "stall_ms": {"max_gap_between_steps": float(gaps.max()),
                        "mean_gap": float(gaps.mean()),
                        "max_gap_at_swap_steps": float(max([gaps[s_ - 1] for s_ in swap_steps
                                                            if s_ > 0] or [0.0]))},
           "h2d_bytes": int(sum(m.h2d_bytes for m in mgrs)),
           "swap_steps": sorted(swap_steps),
           "updates": updates, "clocks": clk}
    del graphs
    for m in mgrs:
        m.close()
    for L in layers:
        L.close()
    return res


# ----------------------------------------------------------------- main --

def prefill_result(args, world, device, barrier, tf_burst, peak_src):
    """The prefill workload (tile orientation, tensor-bound) as a JSON object."""
    pcfg = synth.CONFIGS["qwen3_30b_prefill"]
    pre = run_workload(pcfg, max(10, args.steps // 10), args.warmup, device, False, barrier)
    p_step = max_over_ranks(pre["step_ms"], world, device)
    p_ffn = max_over_ranks(pre["ffn_ms"], world, device)
    flops = 6.0 * pcfg.H * pcfg.I * pre["pairs"]
    tflops = flops / (p_ffn * 1e-3) / 1e12
    return {"workload": workload_name(pcfg), "value": world * pcfg.T / (p_step * 1e-3),
            "unit": "tokens/s", "ms_per_step": p_step, "ffn_ms": p_ffn,
            "isolated_ms_per_step": max_over_ranks(pre["isolated_step_ms"], world, device),
            "timing": "steps back to back alternating two instances of the layer (no flush; "
                      "a step streams ~570 MB of experts); FFN alone: one graph after a "
                      "256 MiB L2 flush",
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": tf_burst,
                         "unit": "TFLOP/s", "frac": tflops / tf_burst,
                         "frac_of_spec_2250": tflops / 2250.0,
                         "flops_per_launch": flops, "peak_source": peak_src + " burst",
                         "traffic": None},
            "touched_experts": pre["n_touched"], "clocks": pre["clocks"]}


def max_over_ranks(v, world, device):
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the shortened Mixtral and stack workloads of the default line")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the prefill workload and print its object (for profiling)")
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "mixtral-sweep", "stack", "router"],
                    help="decode: the headline line; mixtral-sweep / stack / router: one JSON object "
                         "for that workload instead (one GPU)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    cfg = synth.CONFIGS["qwen3_30b_decode"]

    if args.impl == "reference":
        if rank != 0:
            return
        import oracle
        oracle.build()
        r = OracleRunner(cfg)
        sample = 8   # tokens per step: a bounded slice of the 32-token batch
        per = []
        for i in range(args.warmup + args.steps):
            n, dt = r.run(sample)
            if i >= args.warmup:
                per.append(dt / n)
        v = 1.0 / float(np.mean(per))
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * sample * float(np.mean(per)), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": workload_name(cfg), "parallelism": "none (CPU)"},
                "cpu_baseline": {"value": v, "unit": "tokens/s", "kind": "oracle", "cores": r.cores,
                                 "sample": f"{args.steps} steps of {sample} tokens of the "
                                           f"{cfg.T}-token decode batch"},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    from mixed_precision_moe_b200 import build as mbuild
    if rank == 0:
        mbuild.build()
    barrier()

    hbm_gbs, tf_burst, tf_sust, peak_src = load_peaks()
    if args.workload != "decode":
        if world > 1:
            raise SystemExit(f"--workload {args.workload} runs on one GPU")
        if args.workload == "mixtral-sweep":
            print(json.dumps(mixtral_sweep(args, device, hbm_gbs, tf_burst, peak_src)))
        elif args.workload == "router":
            print(json.dumps(router_run(args, device, hbm_gbs, peak_src)))
        else:
            print(json.dumps(stack_run(args, device, hbm_gbs, peak_src)))
        return
    if args.prefill_only:
        pre = prefill_result(args, world, device, barrier, tf_burst, peak_src)
        if rank == 0:
            print(json.dumps(pre))
        return
    dec = run_workload(cfg, args.steps, args.warmup, device, True, barrier)

    step_ms = max_over_ranks(dec["step_ms"], world, device)
    step_p50 = max_over_ranks(float(np.median(dec["step_ms_all"])), world, device)
    step_p90 = max_over_ranks(float(np.percentile(dec["step_ms_all"], 90)), world, device)
    ffn_ms = max_over_ranks(dec["ffn_ms"], world, device)
    e2e_ms = max_over_ranks(dec["e2e_ms"], world, device)
    iso_ms = max_over_ranks(dec["isolated_step_ms"], world, device)
    value = world * cfg.T / (step_ms * 1e-3)
    ffn_gbs = dec["touched_bytes"] / (ffn_ms * 1e-3) / 1e9

    prefill = None
    if not args.no_prefill:
        prefill = prefill_result(args, world, device, barrier, tf_burst, peak_src)

    secondary = None
    if not args.no_secondary:
        # the other workloads of the layer, shortened so the default run stays
        # within minutes: three points of the Mixtral sweep and one stack layer
        # over two 64-step windows (one device-side hot-set update)
        secondary = {"mixtral": mixtral_sweep(args, device, hbm_gbs, tf_burst, peak_src,
                                              batches=(1, 32, 4096)),
                     "stack": stack_run(args, device, hbm_gbs, peak_src, n_layers=1,
                                        n_steps=128),
                     "router": router_run(args, device, hbm_gbs, peak_src)}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        cpu = oracle_baseline(cfg, budget_s=10.0)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "ms_per_step_p50": step_p50, "ms_per_step_p90": step_p90,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; Qwen3-30B-A3B-shaped layer, random-init experts)",
            "config": {"workload": workload_name(cfg), "global_batch": world * cfg.T,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "steps back to back alternating two instances of the layer (same "
                             "weights, separate memory): each step's ~300 MB of touched experts "
                             "evicts the other instance's from the 126 MB L2, no flush",
                       "graph": "CUDA graph per step"},
            "isolated_step": {"ms_per_step": iso_ms, "tokens_per_s": world * cfg.T / (iso_ms * 1e-3),
                              "timing": "one step per measurement: a 256 MiB L2 flush, then "
                                        "the step's graph, CUDA events around the graph alone"},
            "roofline": {"bound": "hbm",
                         "kernel": "grouped_ffn_kernel (gate/up + SwiGLU + down, one launch)",
                         "achieved": ffn_gbs, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": ffn_gbs / hbm_gbs, "frac_of_8000": ffn_gbs / 8000.0,
                         "bytes_per_launch": dec["touched_bytes"],
                         "touched_experts": dec["n_touched"],
                         "peak_source": peak_src,
                         "traffic": ffn_traffic(dec["touched_bytes"])},
            "e2e": {"value": world * cfg.T / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": dec["h2d_bytes"], "d2h_bytes_per_step": dec["d2h_bytes"],
                    "timing": "MoELayer.forward per step from pinned host buffers, the H2D of "
                              "step i and the D2H of step i-1 on side streams beside the layer "
                              "of step i; whole run timed; steps alternate between two "
                              "instances of the layer (same weights, separate memory), so "
                              "each step finds its experts out of L2"},
            "gpu_launches": dec["launches_per_step"] * args.steps,
            "routing": {"distinct_experts": dec["n_touched"], "batches": dec["n_batches"],
                        "selections_per_expert": dec["selections"]},
            "clocks": dec["clocks"],
            "cpu_baseline": cpu,
            "prefill": prefill,
            "secondary": secondary,
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
