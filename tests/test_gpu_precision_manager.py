"""Device-side precision management (DynaExq, arXiv 2511.15015, abstract) on the
Qwen3-80B-scale stack shape: 512 experts (H 2048, I 512, top-10), decode batch
32, Zipf(1.2) routing whose popularity order is redrawn every 64 steps; every
expert resident as INT4, the 64 hottest as BF16.

The hotness counts are accumulated by the routing kernels, the hot set is
selected on the device at the end of every 64-step window, and the handle swap
runs on the device; the host only issues the BF16 copies into the idle slot set
once the selection's event has completed, and the swap follows once the copies'
event has (mixed_precision_moe_b200.precision_manager).  Checked here against
the oracle:
  - every selection equals the oracle's top-64 of the oracle's routing counts
    over the same window (ties to the lower id), bit for bit;
  - routing is bit-exact on every step;
  - the layer output matches the oracle, under the precision map in effect at
    that step (known from the order of the swaps on the stream), on every 16th
    step and on the step of every swap;
  - moe_select_hot_experts alone against brute force on tied counts.
"""
import numpy as np
import pytest
import torch

import oracle
from mixed_precision_moe_b200 import binding as B
from mixed_precision_moe_b200 import build, synth
from mixed_precision_moe_b200.precision_manager import PrecisionManager
from helpers import check_close, to_gpu_bf16

pytestmark = pytest.mark.gpu
S = synth.STACK


def _hot_set(counts, n):
    order = np.lexsort((np.arange(len(counts)), -counts))
    return np.sort(order[:n])


def _bf16_f64(t):
    u = t.view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available()
    build.build()
    B.moe_get_device_status()
    yield


@pytest.mark.parametrize("E,n", [(512, 64), (8, 3), (130, 130), (64, 0)])
def test_select_hot_experts_matches_brute_force(E, n):
    rng = np.random.default_rng(E + n)
    counts = rng.integers(0, 6, E).astype(np.int32)   # many ties
    c = torch.from_numpy(counts).cuda()
    hot = B.moe_select_hot_experts(c, n, zero_counts=True) if n else None
    torch.cuda.synchronize()
    if n:
        assert np.array_equal(hot.cpu().numpy(), _hot_set(counts, n))
    assert torch.count_nonzero(c).item() == 0 or n == 0


def test_stack_layer_with_device_hot_sets():
    H, I, E, k, T = S["H"], S["I"], S["E"], S["k"], S["T"]
    epoch, n_hot = S["epoch"], S["n_hot"]
    steps = 256
    layer_id = 0
    dev = torch.device("cuda", 0)
    compute = torch.cuda.Stream(dev)
    masters = [synth.stack_master(layer_id, e) for e in range(E)]
    L = B.MoELayer(H, I, E, k)
    assert L.hot_set_size(n_hot * (2 * 3 * H * I - (3 * H * I // 2 + 3 * H * I // 64))) == n_hot
    q = []
    for e in range(E):   # base versions: every expert INT4, quantised on the GPU
        w13, w2 = to_gpu_bf16(masters[e][0]), to_gpu_bf16(masters[e][1])
        q13, s13 = B.moe_quantize_weights(w13, B.INT4)
        q2, s2 = B.moe_quantize_weights(w2, B.INT4)
        q.append((q13, s13, q2, s2))
        L.set_expert(e, B.INT4, q13, s13, q2, s2, stream=compute)
    pinned = [(torch.from_numpy(m13.view(np.int16)).view(torch.bfloat16).pin_memory(),
               torch.from_numpy(m2.view(np.int16)).view(torch.bfloat16).pin_memory())
              for m13, m2 in masters]
    mgr = PrecisionManager(L, pinned, n_hot, dev)
    mgr.bootstrap(np.argsort(synth.stack_ranks(layer_id, 0), kind="stable")[:n_hot], compute)
    torch.cuda.synchronize()

    oracle_int4 = {}

    def oracle_expert(e, bf16):
        if bf16:
            return oracle.Expert(oracle.BF16, masters[e][0], None, masters[e][1], None)
        if e not in oracle_int4:
            q13, s13 = oracle.quantize(masters[e][0], oracle.INT4)
            q2, s2 = oracle.quantize(masters[e][1], oracle.INT4)
            oracle_int4[e] = oracle.Expert(oracle.INT4, q13, s13, q2, s2)
        return oracle_int4[e]

    bufs = L.alloc_buffers(T, dev)
    window = np.zeros(E, np.int64)    # oracle counts since the last selection
    n_sel = n_swap = 0
    for step in range(steps):
        swapped = mgr.poll(step, compute)
        n_swap += swapped
        if step > 0 and step % epoch == 0:
            if mgr.end_window(step, compute):
                torch.cuda.synchronize()      # test only: read the selection back now
                got = np.sort(mgr.hot_host[mgr.target][:n_hot].numpy())
                assert np.array_equal(got, _hot_set(window, n_hot)), f"selection at step {step}"
                window[:] = 0
                n_sel += 1
        hot = set(mgr.hot_experts().tolist())
        logits = synth.stack_logits(layer_id, step)
        x = synth.stack_x(layer_id, step)
        with torch.cuda.stream(compute):
            out = L.forward(torch.from_numpy(logits).to(dev), to_gpu_bf16(x), bufs=bufs,
                            stream=compute)
        compute.synchronize()
        st = B.moe_get_device_status()
        assert st == 0, f"step {step}: device status {st:#x}"
        idx = bufs["route"][0].cpu().numpy()
        idx_o, _ = oracle.route_topk(logits, k)
        assert np.array_equal(idx, idx_o), f"step {step}: routing"
        window += np.bincount(idx_o.ravel(), minlength=E)
        if step % 16 == 0 or swapped:
            used = np.unique(idx_o)
            filler = oracle_expert(int(used[0]), int(used[0]) in hot)
            exps = [filler] * E
            for e in used.tolist():
                exps[e] = oracle_expert(e, e in hot)
            _, _, out_o = oracle.moe_layer(logits, x, exps, k, H, I)
            check_close(_bf16_f64(out), out_o, f"step {step} ({len(hot)} BF16)")
    assert n_sel == 3 and n_swap >= 2, (n_sel, n_swap, mgr.log)
    mgr.close()
    torch.cuda.synchronize()
    L.close()
